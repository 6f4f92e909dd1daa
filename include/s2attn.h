/*
 * s2attn.h -- C ABI of the B200 (sm_100a) shifted-short-attention library.
 *
 * The operation (LongLoRA's S^2-Attn, as described on the LongLoRA pages):
 *   - "LongLoRA paper notes" (smallflyingpig blog), section 3.3: a sequence of
 *     length N is cut into groups of G tokens and attention runs only inside each
 *     group, lowering the cost from O(N^2) to O(N^2 / (N/G)); a shifted pattern moves
 *     the groups by half a group so that information crosses group borders
 *     (drawing: groups 1-4, 5-8, 9-12 become 3-6, 7-10, 11-14).
 *   - "LLaMA2 context to 100k" (nearauto.com), section on shift short attention:
 *     two steps, (1) shift the tokens in half of the attention heads, (2) move the
 *     features from the token dimension into the batch dimension.
 *   - python88.com article, mechanism paragraph: the heads are split into two halves
 *     and shifting one half lets neighbouring groups exchange information.
 *   - "LongLoRA paper notes", section 3.1, and the model page (model.aibase.cn),
 *     features list: inference uses ordinary full attention.
 * Precisely, with scale = 1/sqrt(D) and shift s_h = G/2 for heads
 * h >= H - shift_heads (0 otherwise): rolled row r of head h holds original token
 * (r + s_h) mod N; group j owns rolled rows [jG, (j+1)G); query row r attends to the
 * rolled rows r' of its own group with r' <= r (causal, in rolled order); the result
 * of rolled row r is stored back at its original token.  G = N with shift_heads = 0
 * is full causal attention (the inference case).
 *
 * Conventions for every entry point:
 *   - Tensors are dense row-major [B, N, H, D] ("token-major"); lse and delta are
 *     [B, H, N] fp32, indexed by ORIGINAL token.
 *   - Every pointer is a device pointer owned by the caller, 16-byte aligned; the
 *     library never frees or keeps caller memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work and return; nothing synchronizes.
 *   - Return value: S2ATTN_OK or a negative s2attn_status.  Argument errors are
 *     detected on the host before anything is enqueued.  A failure inside a kernel
 *     (a bounded wait that timed out) is recorded in a per-device error word that
 *     s2attn_get_device_error() reads after the caller synchronizes.
 *   - The calls are thread-safe with respect to each other.
 */
#ifndef S2ATTN_H_
#define S2ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  S2ATTN_OK = 0,
  S2ATTN_ERR_INVALID_ARG = -1,    /* bad shape, null or misaligned pointer */
  S2ATTN_ERR_UNSUPPORTED = -2,    /* valid, but not a shape this path handles */
  S2ATTN_ERR_WORKSPACE = -3,      /* workspace missing or too small */
  S2ATTN_ERR_CUDA = -4,           /* a CUDA runtime/driver call failed */
  S2ATTN_ERR_DEVICE_TIMEOUT = -5  /* a kernel gave up on a bounded wait */
} s2attn_status;

/* Version of this ABI (major * 100 + minor). */
int s2attn_version(void);

/* Human-readable name of a status code (static string). */
const char* s2attn_status_string(int status);

/*
 * Forward pass, bf16 in / bf16 out, fp32 accumulation (tcgen05 tensor cores).
 *   q, k, v : [B,N,H,D] bf16 inputs
 *   o       : [B,N,H,D] bf16 output (attention output at each original token)
 *   lse     : [B,H,N] fp32 output, natural log of sum over visible keys of exp(scale*q.k)
 * Requirements: D == 128; G >= 1 divides N; 0 <= shift_heads <= H; G % 128 == 0;
 * if shift_heads > 0 then (G/2) % 128 == 0.  Other valid shapes return
 * S2ATTN_ERR_UNSUPPORTED (the fp32 entry points take any valid shape).
 */
int s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int D, int G,
               int shift_heads, void* stream);

/* Bytes of device workspace s2attn_bwd needs: an fp32 dQ accumulator [B,N,H,D]
 * followed by delta [B,H,N] fp32 (each start 256-byte aligned).  0 on bad sizes. */
size_t s2attn_bwd_workspace_bytes(int B, int N, int H, int D);

/*
 * Backward pass, bf16, same shape rules as s2attn_fwd.  Inputs: q, k, v, the
 * forward output o and lse, and the output gradient dout.  Outputs dq, dk, dv
 * ([B,N,H,D] bf16).  `workspace` (device, caller-owned, >= the size above,
 * 256-byte aligned) is overwritten.  Runs s2attn_bwd_preprocess, s2attn_bwd_main
 * and s2attn_bwd_dq_convert in that order on `stream`.
 */
int s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, int B, int N, int H, int D, int G, int shift_heads, void* workspace,
               size_t workspace_bytes, void* stream);

/* Backward stage 1: delta[b,h,t] = sum_d dout[b,t,h,d] * o[b,t,h,d] (fp32, delta is
 * [B,H,N]) and dq_acc ([B,N,H,D] fp32) := 0.  D must be 128. */
int s2attn_bwd_preprocess(const void* o, const void* dout, float* delta, float* dq_acc, int B, int N, int H, int D,
                          void* stream);

/* Backward stage 2 (tensor cores): writes dk, dv (bf16) and adds the unscaled
 * dQ = dS K into dq_acc (fp32, zeroed by stage 1).  Same shape rules as s2attn_fwd. */
int s2attn_bwd_main(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                    const float* delta, float* dq_acc, void* dk, void* dv, int B, int N, int H, int D, int G,
                    int shift_heads, void* stream);

/* Backward stage 3: dq = bf16(dq_acc / sqrt(D)), round to nearest even. */
int s2attn_bwd_dq_convert(const float* dq_acc, void* dq, int B, int N, int H, int D, void* stream);

/*
 * Decoding step of full causal attention (inference).  Inference runs ordinary
 * full attention, not S^2-Attn ("LongLoRA paper notes", section 3.1; model.aibase.cn,
 * features list: the shifted attention is only needed in training).  A step appends
 * M new tokens to a sequence of N positions:
 *   q    : [B,M,H,D] bf16, the new queries; query m sits at position N-M+m
 *   k, v : [B,N,H,D] bf16, all N positions (the M new ones included)
 *   o    : [B,M,H,D] bf16 output; query m attends to the keys at positions
 *          0 .. N-M+m with scale 1/sqrt(D)
 *   lse  : [B,H,M] fp32 output, natural log of sum over those keys of exp(scale*q.k)
 * Requirements: 1 <= M <= N; M <= 128 and D == 128 (else S2ATTN_ERR_UNSUPPORTED).
 * One query runs on CUDA cores (HBM-bound matrix-vector work); 2..128 queries run one
 * 128-row query tile on the tensor cores (speculative decoding, chunked prefill).
 * `workspace` (device, caller-owned, 256-byte aligned, at least
 * s2attn_decode_workspace_bytes bytes) receives per-split partial results and is
 * overwritten; its size holds fp32 partials (D outputs, max, sum per query) of at most
 * min(64, ceil(N/64)) splits per (b, h), independent of the device; 0 means invalid sizes.
 * V rows past a query's causal limit are multiplied by a zero weight, so k and v must hold
 * finite values at every position.  Runs two kernels on `stream`; the second (the split
 * combine) is a programmatic dependent launch that waits on the device for the first.
 */
size_t s2attn_decode_workspace_bytes(int B, int M, int N, int H, int D);
int s2attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int M, int N, int H,
                  int D, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Halo rows of sequence-sharded S^2-Attn.  The groups are independent, so a sequence
 * split across ranks in whole groups needs one exchange ("LongLoRA paper notes",
 * section 3.3; nearauto.com article, "shift short attention" steps (1) and (2)).  A
 * rank holding tokens [t0, t0+N) of every head (N a multiple of G) runs the forward and
 * backward above on its own tensors with the shift; their last rolled group of a
 * shifted head reads the rank's tail and then its rows [0, G/2).  Those rows of the
 * shifted heads belong to the previous rank's last group, so the sharded path swaps the
 * next rank's first G/2 rows (the halo) into them for the duration of the calls and
 * swaps them back afterwards; the results written to them belong to the halo's tokens
 * and are returned to their owner.  These two calls are the copies that swap needs:
 *   s2attn_halo_rows: for each of n_tensors bf16 [B,N,H,D] tensors x[i] and contiguous
 *     buffers buf[i] [B, G/2, shift_heads, D]:  to_buf != 0: buf[i][b,r,s,:] =
 *     x[i][b, r, H-shift_heads+s, :] for r < G/2;  to_buf == 0: the reverse copy.
 *   s2attn_halo_lse: the same rows of fp32 [B,H,N] tensors (lse, softmax statistics),
 *     buffers [B, shift_heads, G/2].
 * x and buf are host arrays of n_tensors device pointers (1 <= n_tensors <= 8), bf16
 * pointers 16-byte aligned (lse pointers 4-byte aligned), owned by the caller.
 * Requirements: G divides N, G even, 1 <= shift_heads <= H, D*2 a multiple of 16.
 * One kernel launch per call on `stream`; buffers and tensors must not overlap.
 */
int s2attn_halo_rows(void* const* x, void* const* buf, int n_tensors, int to_buf, int B, int N, int H, int D,
                     int G, int shift_heads, void* stream);
int s2attn_halo_lse(float* const* lse, float* const* buf, int n_tensors, int to_buf, int B, int N, int H, int G,
                    int shift_heads, void* stream);

/*
 * fp32 forward/backward on CUDA cores, any valid shape with 1 <= D <= 128
 * (G >= 1 divides N; G even when shift_heads > 0).  Same tensor layouts, all fp32.
 * s2attn_bwd_f32 uses the delta part of the workspace only
 * (size from s2attn_bwd_workspace_bytes).
 */
int s2attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int N, int H, int D,
                   int G, int shift_heads, void* stream);
int s2attn_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* dout,
                   const float* lse, float* dq, float* dk, float* dv, int B, int N, int H, int D, int G,
                   int shift_heads, void* workspace, size_t workspace_bytes, void* stream);

/*
 * RoPE with position interpolation ("LongLoRA paper notes", section 3.4: positions
 * [0, L) are squeezed into [0, L0)), applied in place to bf16 q and k ([B,N,H,D]).
 * Token t is rotated as if at position t * pos_scale (pos_scale = L0 / N).  Element
 * i < D/2 pairs with element i + D/2; the pair turns by angle a = (t*pos_scale) *
 * theta_i with theta_i = base^(-2i/D).  Evaluation order (bit-for-bit contract):
 *   theta_i = (float) pow(base, -2i/D) in double;  a = ((float)t * pos_scale) * theta_i
 *   in float;  c, s = (float) cos/sin((double) a);  y1 = x1*c - x2*s;  y2 = x2*c + x1*s,
 *   every product and sum rounded to fp32, then rounded to bf16 (nearest even).
 * The cos/sin table is computed on the host on first use of each (device, N, D,
 * pos_scale, base) and cached in device memory owned by the library until exit.
 * Either q or k may be NULL.  Requires D % 16 == 0, D <= 256.
 * Backward: with -pos_scale every angle is negated exactly (the products above round
 * symmetrically, cos is even and sin odd), which applies the transposed rotation -- the
 * gradient through RoPE-PI -- to dq and dk in the same operation order.
 */
int rope_pi_apply(void* q, void* k, int B, int N, int H, int D, float pos_scale, float base, void* stream);

/*
 * RoPE-PI as above for tensors whose row t is the token at position pos0 + t: the new
 * tokens of a decoding step (q and the k rows appended to the cache sit at positions
 * N_cache - M .. N_cache - 1).  Identical, bit for bit, to rows pos0 .. pos0+N-1 of
 * rope_pi_apply over the whole sequence (same operation order and table entries).
 * Requires pos0 >= 0 and pos0 + N <= 2^24.  The table is built on the host and cached in
 * device memory for the next power of two >= pos0 + N positions (at least 1024): D*4 bytes
 * per position, 64 MB for 128k positions at D = 128.
 */
int rope_pi_apply_offset(void* q, void* k, int B, int N, int H, int D, int pos0, float pos_scale, float base,
                         void* stream);

/*
 * LoRA-adapted linear projections, the steps on either side of S^2-Attn in a LongLoRA
 * layer ("LongLoRA paper notes", section 3.2: low-rank adapters on the Q, K, V and O
 * projections; nearauto.com article, "long-context LoRA improvement").  For `parts`
 * projections stacked along the output (3 for q, k, v; 1 for o), part p computes
 *   y[p] = x W_p^T + scaling * (x A_p^T) B_p^T
 * and the first `rope_parts` parts are then rotated by RoPE-PI, so q and k come out ready
 * for s2attn_fwd.  All bf16, accumulated in fp32 on the tensor cores:
 *   x      : [T, K], T = B*seq_len tokens (row t is position t mod seq_len)
 *   w      : [parts*n_out, K], the frozen weights (the layout of a linear layer's weight)
 *   lora_a : [parts*r, K], the adapters' down projections (NULL when r == 0)
 *   lora_b : [parts*n_out, r], the adapters' up projections (NULL when r == 0)
 *   y      : [parts, T, n_out] output; y[p] is a contiguous [B, seq_len, H, D] tensor when
 *            n_out = H*D, so q, k and v need no copy before attention
 * Rounding: the rank-r intermediate is held in bf16 after scaling, bf16(scaling * x A_p^T),
 * and y is rounded once (nearest even) from the fp32 accumulator.  With rope_parts > 0,
 * the rotated parts are bit-identical to this call with rope_parts = 0 followed by
 * rope_pi_apply(y[p], ..., B, seq_len, n_out/head_dim, head_dim, pos_scale, base) on
 * each: the same table (cached per device, seq_len, head_dim, pos_scale, base) and the
 * same fp32 operation order, applied to the bf16-rounded projection.  As for rope_pi_apply,
 * the first call with a new table builds it on the host and copies it synchronously; make
 * that call before any stream capture.
 * Requirements: K >= 8 and K % 8 == 0; 0 <= r <= 64; 0 <= rope_parts <= parts;
 * n_out % 256 == 0 and K >= 64 (else S2ATTN_ERR_UNSUPPORTED); x, w, y, lora_a 16-byte aligned; with
 * rope_parts > 0: head_dim in {32, 64, 128, 256}, T % seq_len == 0, base > 0.
 * `workspace` (device, caller-owned, 256-byte aligned, at least
 * lora_proj_workspace_bytes(T, K, n_out, parts, r) bytes; may be NULL when r == 0) holds the
 * zero-padded adapters and the intermediate and is overwritten.  Runs up to three kernels
 * on `stream` (adapter padding, the rank-r down projection, the projection); invalid
 * arguments return before any launch.
 */
size_t lora_proj_workspace_bytes(int T, int K, int n_out, int parts, int r);
int lora_proj_fwd(const void* x, const void* w, const void* lora_a, const void* lora_b, void* y, int T, int K,
                  int n_out, int parts, int r, float scaling, int rope_parts, int head_dim, int seq_len,
                  float pos_scale, float base, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of lora_proj_fwd for training (the frozen W gets no gradient; notes section 3.2):
 *   dx       = sum_p dy_p W_p + s (dy_p B_p) A_p           [T, K]
 *   d_lora_a = per part, s (dy_p B_p)^T x                  [parts*r, K]
 *   d_lora_b = per part, s dy_p^T (x A_p^T)                [parts*n_out, r]
 * dy [parts, T, n_out] is the gradient of y before RoPE: take dq and dk back through the
 * rotation first with rope_pi_apply(dq, dk, ..., -pos_scale, ...).  Same layouts and
 * requirements as lora_proj_fwd (K >= 64, n_out % 256 == 0, r <= 64); d_lora_a / d_lora_b may be
 * NULL when r == 0.  `workspace` (device, caller-owned, 256-byte aligned, at least
 * lora_proj_bwd_workspace_bytes bytes) holds the padded adapters, the recomputed intermediate
 * s x A^T, s dy B, and fp32 accumulators for the adapter gradients.  The adapter gradients add
 * fp32 partial sums over token ranges, so they are not bitwise reproducible run to run.
 */
size_t lora_proj_bwd_workspace_bytes(int T, int K, int n_out, int parts, int r);
int lora_proj_bwd(const void* x, const void* w, const void* lora_a, const void* lora_b, const void* dy, void* dx,
                  void* d_lora_a, void* d_lora_b, int T, int K, int n_out, int parts, int r, float scaling,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass that allocates nothing.  The LongLoRA pages have no counterpart of
 * this entry point; it exists for callers that cannot allocate device memory on
 * the call path (a runtime whose allocator already holds the device's memory, a
 * plugin whose enqueue step must not allocate, or a latency-critical loop that
 * cannot afford cudaMalloc's implicit device synchronisation) and so cannot hand
 * s2attn_bwd a workspace.
 * Same arguments, shape rules and results as s2attn_bwd, minus the workspace: the
 * fp32 dQ accumulator and delta live in a fixed array of
 * S2ATTN_NOALLOC_SCRATCH_BYTES in the library's device memory, held until the
 * process exits.  The array is reserved when the module holding it is loaded on a
 * device; with CUDA's lazy module loading (the default) that happens inside the
 * first call on each device, which looks up the array's device address (with that
 * device current) and caches it.  So the first call on a device does take
 * S2ATTN_NOALLOC_SCRATCH_BYTES of device memory: make it before the caller's own
 * allocator reserves the device (else it fails with S2ATTN_ERR_CUDA) and before any
 * stream capture.  Later calls take no device memory.
 * Problems needing more (B*N*H*D*4 + B*H*N*4 bytes, each part rounded up to 256)
 * return S2ATTN_ERR_WORKSPACE; at D = 128 that is about 130k (token, head) rows.
 * Every call uses the same array and leaves its last contents there (the
 * accumulator is zeroed at the start of each call): calls whose work overlaps on
 * the GPU -- on different streams, or on different host threads -- race on it.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define S2ATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int s2attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int D, int G,
                       int shift_heads, void* stream);

/*
 * Reads the current device's error word: S2ATTN_OK if no kernel has failed since
 * the last clear, else S2ATTN_ERR_DEVICE_TIMEOUT with *detail (if non-NULL) set to
 * (kernel << 8) | site (kernel 1 = forward, 2 = backward, 4 = decoding step,
 * 5 = LoRA projection).  In the
 * bounds-checked build (libs2attn_debug.so, compiled with S2ATTN_DEBUG) a site with bit
 * 0x80 set is a global store or reduction whose computed index fell outside its tensor;
 * the access was skipped.  Synchronize the streams
 * that ran library kernels first.
 */
int s2attn_get_device_error(int* detail);

/* Resets the current device's error word to 0 (synchronous). */
int s2attn_clear_device_error(void);

/*
 * Self-test of the device-side failure path used by every kernel above: launches one
 * thread that waits on a barrier nothing ever arrives at, with a wait limit of
 * `timeout_us` microseconds (1 .. 1000000).  After the caller synchronizes `stream`,
 * s2attn_get_device_error() returns S2ATTN_ERR_DEVICE_TIMEOUT with detail
 * (3 << 8) | 1, and the context stays usable (clear the word to continue).  The
 * kernels' own waits give up after 2 s the same way instead of hanging the GPU.
 */
int s2attn_selftest_bounded_wait(unsigned timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H_ */
