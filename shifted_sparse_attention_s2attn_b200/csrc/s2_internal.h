// s2_internal.h -- launch functions shared between the library's translation units.
// Host-only declarations; kernels live in the .cu files that define these.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace s2 {

// Device error codes (first failure wins; read with s2attn_get_device_error).
// code = (kernel << 8) | site
enum Kernel : int { K_FWD = 1, K_BWD = 2, K_SELFTEST = 3, K_DEC = 4, K_LORA = 5 };

// Argument rules of the bf16 tensor-core entry points (shape, D == 128, tile alignment of G and
// G/2, and the index-overflow guards): S2ATTN_OK or the status those entry points return.
int check_tensor_core_args(int B, int N, int H, int D, int G, int shift_heads);

// Problem description after validation.  Rows of a [B,N,H,D] tensor for head h
// are addressed through 3-D tensor maps with dims {D, H, B*N}.
struct Shape {
  int B, N, H, D, G, shift_heads;
};

// Forward, bf16, D == 128: one launch of the tcgen05 kernel, a persistent grid of at most
// n_sm CTAs (one per SM).
cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             void* o, float* lse, const Shape& s, int n_sm, int* err, cudaStream_t st);

// Backward main kernel, bf16, D == 128: dK, dV written, dQ accumulated (fp32) into dq_acc.
// Tensor maps: 128-row boxes of 64 columns, 128-byte swizzle, for q, k, v and dout.
// n_sm: the device's SM count (short folds run on a persistent grid of one CTA per SM).
cudaError_t launch_bwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const float* lse, const float* delta, float* dq_acc, void* dk,
                             void* dv, const Shape& s, int n_sm, int* err, cudaStream_t st);

// delta[b,h,t] = sum_d dO*O (fp32) and dq_acc := 0.
cudaError_t launch_bwd_preprocess(const void* o, const void* dout, float* delta, float* dq_acc, const Shape& s,
                                  cudaStream_t st);
// dq = bf16(scale * dq_acc)
cudaError_t launch_dq_convert(const float* dq_acc, void* dq, const Shape& s, cudaStream_t st);

// fp32 CUDA-core path (any valid shape).
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, const Shape& s,
                           cudaStream_t st);
cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* dout,
                           const float* lse, float* dq, float* dk, float* dv, float* delta, const Shape& s,
                           cudaStream_t st);

// Decoding step (full causal attention of the last M <= 128 positions), D == 128; the
// CUDA-core kernel below takes M <= kDecodeSimtMaxM.
// The K/V of each (b, h) is cut into `S` splits of `tiles_per_split` key tiles
// (decode_splits picks them for `n_sm` SMs, at most kDecodeMaxSplits); the split kernel
// writes fp32 partials (part_o [B*H][S][M][128], part_ml [B*H][S][M][2]) and a second
// kernel combines them into o and lse.  Tensor maps: 64-row boxes of 64 columns,
// 128-byte swizzle, over k and v ([B,N,H,D]).
constexpr int kDecodeMaxSplits = 64;
constexpr int kDecodeTileKeys = 64;       // key tile of the CUDA-core kernel (its tensor maps' box height)
// Up to this many queries the CUDA-core kernel runs, above it the tensor-core one (measured at
// 32k: M = 1 0.096 vs 0.125 ms, M = 2 0.127 vs 0.126, M = 4 0.202 vs 0.126, M = 16 0.352 vs 0.128).
constexpr int kDecodeSimtMaxM = 1;
constexpr int kDecodeMaxM = 128;          // one 128-row query tile on the tensor-core path
// Tensor-core variant (M up to 128): 64-key tiles, two CTAs per SM; tensor maps with 128-row
// boxes over q ([B,M,H,D]) and kDecodeTileKeys-row boxes over k and v.
int decode_splits_tc(int B, int N, int H, int n_sm, int* tiles_per_split);
cudaError_t launch_decode_tc_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                                   float* lse, float* part_o, float* part_ml, int B, int M, int N, int H, int S,
                                   int tiles_per_split, int* err, cudaStream_t st);
int decode_splits(int B, int N, int H, int n_sm, int* tiles_per_split);
cudaError_t launch_decode_sm100(const CUtensorMap& tk, const CUtensorMap& tv, const void* q, void* o, float* lse,
                                float* part_o, float* part_ml, int B, int M, int N, int H, int S,
                                int tiles_per_split, int* err, cudaStream_t st);

// LoRA-adapted projections y = x W^T + s (x A^T) B^T (lora_proj_sm100.cu).  The rank
// dimension is zero-padded to kLoraRankPad (one 64-wide K block); the projection's output
// tile is kLoraProjTileN columns, so n_out must be a multiple of it.
constexpr int kLoraRankPad = 64;
constexpr int kLoraMaxRank = kLoraRankPad;
constexpr int kLoraProjTileN = 256;
// a [parts*r, K], b [parts*n_out, r] -> a_pad [parts*64, K], b_pad [parts*n_out, 64] (zeros beyond r).
cudaError_t launch_lora_pad(const void* a, const void* b, void* a_pad, void* b_pad, int parts, int r, int K,
                            int n_out, cudaStream_t st);
// u [parts, T, 64] = bf16(scaling * x a_pad^T).  Tensor maps (128-byte swizzle, 64-column
// boxes): tx over x [T, K] with 128-row boxes, ta_pad over a_pad with 64-row boxes.
cudaError_t launch_lora_down(const CUtensorMap& tx, const CUtensorMap& ta_pad, void* u, int T, int K, int parts,
                             float scaling, int n_sm, int* err, cudaStream_t st);
// y [parts, T, n_out] = bf16(x W^T + u_part b_pad^T), RoPE-PI on parts [0, rope_parts).
// Tensor maps: tx as above; tw over W [parts*n_out, K] with 256-row boxes; tu over u as
// {64, T, parts} with {64, 128, 1} boxes; tb over b_pad with 256-row boxes (r == 0: tu, tb unused).
cudaError_t launch_lora_proj(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& tu,
                             const CUtensorMap& tb, void* y, int T, int K, int n_out, int parts, int r,
                             int rope_parts, int head_dim, int seq_len, const float* cos_tab, const float* sin_tab,
                             int n_sm, int* err, cudaStream_t st);

// Backward of the projections (lora_bwd_sm100.cu): g = bf16(s dy_p b_pad_p) [parts, T, 64], then
// dx = sum_p dy_p W_p + g_p a_pad_p, dA_acc += g^T x and dB_acc += dy_p^T u_p (fp32, zeroed here),
// then dA, dB in bf16.  Tensor maps (3-D, 128-byte swizzle, 64-column boxes):
//   dy_k {n_out, T, parts} 128-row boxes; dy_mn, bpad {64, n_out, parts}, w_mn {K, n_out, parts},
//   apad {K, 64, parts}, g_mn / u_mn {64, T, parts}, x_mn {K, T, 1}: 64-row boxes; g_k {64, T, parts} 128-row.
cudaError_t launch_lora_bwd(const CUtensorMap& dy_k, const CUtensorMap& dy_mn, const CUtensorMap& bpad,
                            const CUtensorMap& w_mn, const CUtensorMap& g_k, const CUtensorMap& apad,
                            const CUtensorMap& g_mn, const CUtensorMap& x_mn, const CUtensorMap& u_mn, void* g,
                            void* dx, float* da_acc, float* db_acc, void* da, void* db, int T, int K, int n_out,
                            int parts, int r, float scaling, int n_sm, int* err, cudaStream_t st);

// Halo rows of the sequence-sharded path (s2attn_halo.cu): rows [0, G/2) of heads
// [H - shift_heads, H) of up to kHaloMaxTensors tensors, to (to_buf = 1) or from (0)
// contiguous buffers [B, G/2, shift_heads, D] (bf16 rows) or [B, shift_heads, G/2] (fp32 lse).
constexpr int kHaloMaxTensors = 8;
cudaError_t launch_halo_rows(void* const* x, void* const* buf, int n, int to_buf, int B, int N, int H, int D,
                             int G, int shift_heads, int n_sm, cudaStream_t st);
cudaError_t launch_halo_lse(float* const* x, float* const* buf, int n, int to_buf, int B, int N, int H, int G,
                            int shift_heads, int n_sm, cudaStream_t st);

// RoPE-PI in place on bf16 q and k, with a cos/sin table [N, D/2] (fp32 each).
cudaError_t launch_rope_pi(void* q, void* k, const float* cos_tab, const float* sin_tab, int B, int N, int H,
                           int D, cudaStream_t st);

}  // namespace s2
