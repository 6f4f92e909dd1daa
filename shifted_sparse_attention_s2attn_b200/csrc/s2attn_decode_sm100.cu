// s2attn_decode_sm100.cu -- a decoding step of full causal attention on B200 (sm_100a).
//
// Inference runs ordinary full attention; S^2-Attn is a training-time device only
// ("LongLoRA paper notes", section 3.1; model.aibase.cn, features list).  A decoding
// step appends M (<= 128) tokens to a sequence of N positions: k, v [B,N,H,D] hold all
// N positions (the new ones included), q [B,M,H,D] the M new queries; query m sits at
// position N-M+m and sees keys 0 .. N-M+m.
//
// Two kernels, chosen by M (kDecodeSimtMaxM).  With one query the step is a matrix-vector
// product over the whole K/V of every head: 2*N*D*2 bytes per head and 4*D FLOPs per key,
// bound by HBM, not by arithmetic -- the first kernel runs on the CUDA cores, and its job
// is to stream K and V at full bandwidth (it is written for up to 16 queries, but from two
// queries on the tensor-core kernel further down is faster):
//   * split-KV: CTA (b, h, split) takes a run of 64-key tiles of one head, so that the
//     grid fills every SM even for one sequence (B*H*splits CTAs, sized to whole waves);
//   * a producer thread streams the tiles with TMA (four 64-row x 64-column boxes per
//     tile: K and V, two column halves each, 128-byte swizzle) through a 3-stage ring,
//     starting before the queries are staged; two CTAs fit on an SM, so one CTA's
//     start-up and merge overlap the other's streaming;
//   * consumer warps take 32 keys of each tile (and, for more than 8 queries, half of
//     the queries): lane = key for Q.K (16-byte swizzled row reads, conflict-free), an
//     online base-2 softmax per warp, then lane = 4 head dims for P.V (the
//     probabilities broadcast from shared memory);
//   * the warps' partial (max, sum, unnormalised output) merge in shared memory and the
//     CTA writes one fp32 partial per (b, h, split, m); a second kernel combines the
//     splits into o (bf16) and lse.
#include <atomic>

#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace dec {

constexpr int HD = 128;
constexpr int TK = kDecodeTileKeys;          // keys per tile (64; the tensor maps' box height)
constexpr uint32_t BOX = TK * 128;            // 64 rows x 128 B (64 bf16 columns)
constexpr uint32_t TILE_BYTES = 4 * BOX;      // K box 0, K box 1, V box 0, V box 1
constexpr int NST = 3;                        // ring stages
constexpr int MAXM = 16;
constexpr int KW = TK / 32;                   // key warps: 32 keys of each tile per warp
constexpr int MAXW = 2 * KW;                  // consumer warps with the queries split in two
constexpr uint32_t OFF_Q = NST * TILE_BYTES;              // float [MAXM][HD], scaled to the log2 domain
constexpr uint32_t OFF_P = OFF_Q + MAXM * HD * 4;         // float [warp][32 keys][queries of the warp]
constexpr uint32_t OFF_BAR = OFF_P + MAXW * 32 * 8 * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + 2 * NST * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;     // + slack to align the base to 1024 B
static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs must fit on an SM");
// Queries per consumer warp and consumer warps, for a query count padded to MT.
template <int MT> struct Cfg {
  static constexpr int QW = MT > 8 ? 8 : MT;
  static constexpr int NCW = KW * (MT / QW);
  static constexpr int NTHREADS = (NCW + 1) * 32;  // + producer warp
};

struct Params {
  const __nv_bfloat16* q;
  float* part_o;   // [B*H][S][M][HD] unnormalised
  float* part_ml;  // [B*H][S][M][2]  (running max in the log2 domain, sum)
  int B, M, N, H, S, tiles_per_split;
  float qscale;    // log2(e) / sqrt(D)
  int* err;
};

enum Site : int { SITE_LOAD = 1, SITE_CONSUME = 2, SITE_DRAIN = 3 };

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int MT>
__global__ void __launch_bounds__(Cfg<MT>::NTHREADS, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                        const Params p) {
  constexpr int QW = Cfg<MT>::QW, NCW = Cfg<MT>::NCW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + NST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC);
  float* qs = reinterpret_cast<float*>(smem + OFF_Q);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // consecutive CTAs take the same split of consecutive heads: the CTAs resident at one
  // time then read whole [H, D] token rows (8 KB at H = 32) rather than one head's 256 B
  // of each, so every DRAM page they open is read in full
  const int units = p.B * p.H;
  const int bh = (int)(blockIdx.x % units);
  const int split = (int)(blockIdx.x / units);
  const int h = bh % p.H, b = bh / p.H;
  const int t_begin = split * p.tiles_per_split * TK;
  const int t_end = min(p.N, t_begin + p.tiles_per_split * TK);
  const int n_tiles = t_end > t_begin ? (t_end - t_begin + TK - 1) / TK : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = (*(volatile int*)p.err != 0) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool skip = *abort_flag != 0;
  // the combine kernel may be scheduled now; it waits for this whole grid to finish
  // (griddepcontrol.wait) before it reads anything this grid writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == NCW) {
    // ---------------- TMA producer ----------------
    if (!skip && lane == 0) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int slot = i % NST;
        if (i >= NST) ok = wait_bounded(&empty[slot], ((i / NST) - 1) & 1, abort_flag, p.err);
        if (!ok) break;
        uint8_t* dst = smem + slot * TILE_BYTES;
        const int row = b * p.N + t_begin + i * TK;
        mbar_arrive_expect_tx(&full[slot], TILE_BYTES);
        tma_load_3d(dst, &tk, 0, h, row, &full[slot]);
        tma_load_3d(dst + BOX, &tk, 64, h, row, &full[slot]);
        tma_load_3d(dst + 2 * BOX, &tv, 0, h, row, &full[slot]);
        tma_load_3d(dst + 3 * BOX, &tv, 64, h, row, &full[slot]);
        issued = i + 1;
      }
      if (!ok) {
        report_error(p.err, (K_DEC << 8) | SITE_LOAD);
        *abort_flag = 1;
      }
      bool dok = true;
      for (int i = (issued > NST ? issued - NST : 0); i < issued; ++i)
        dok &= wait_drain(&full[i % NST], (i / NST) & 1);
      if (!dok) report_error(p.err, (K_DEC << 8) | SITE_DRAIN);
    }
    return;  // the producer warp takes no part in the merge below
  }

  // ---------------- consumers: 32 keys of each tile and QW queries per warp ----------------
  // queries of this head, scaled into the log2 domain; rows m >= M are zero (the
  // producer's first copies are already in flight)
  for (int i = threadIdx.x; i < MT * HD; i += NCW * 32) {
    const int m = i / HD, d = i % HD;
    float x = 0.0f;
    if (m < p.M) x = __bfloat162float(p.q[((size_t)(b * p.M + m) * p.H + h) * HD + d]) * p.qscale;
    qs[i] = x;
  }
  named_bar_sync(1, NCW * 32);
  const int kw = warp % KW;          // which 32 keys of each tile
  const int q0 = (warp / KW) * QW;   // first query of this warp
  float m_run[QW], l_lane[QW], o_acc[QW][4];
#pragma unroll
  for (int m = 0; m < QW; ++m) {
    m_run[m] = -INFINITY;
    l_lane[m] = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) o_acc[m][e] = 0.0f;
  }
  const float4* q4 = reinterpret_cast<const float4*>(qs + q0 * HD);
  float* pbuf = reinterpret_cast<float*>(smem + OFF_P) + warp * 32 * QW;
  const int lim0 = p.N - p.M + q0;  // query q0 + m sees keys t <= lim0 + m
  bool ok = !skip;
  for (int i = 0; i < n_tiles && ok; ++i) {
    const int slot = i % NST;
    ok = wait_bounded(&full[slot], (i / NST) & 1, abort_flag, p.err);
    if (!ok) break;
    const uint8_t* kb = smem + slot * TILE_BYTES;
    const uint8_t* vb = kb + 2 * BOX;
    const int t0 = t_begin + i * TK + 32 * kw;  // first key of this warp's 32
    // ---- scores, lane = key: s_m = (q_m * log2e / sqrt(D)) . k_t
    const int r = 32 * kw + lane;
    const int t = t0 + lane;
    float s[QW];
#pragma unroll
    for (int m = 0; m < QW; ++m) s[m] = 0.0f;
#pragma unroll 4
    for (int c = 0; c < HD / 8; ++c) {
      const uint4 kw = *reinterpret_cast<const uint4*>(kb + (c >> 3) * BOX + r * 128 + (((c & 7) ^ (r & 7)) << 4));
      float kf[8];
      bf16x8_to_f32(kw, kf);
#pragma unroll
      for (int m = 0; m < QW; ++m) {
        const float4 qa = q4[(m * HD + 8 * c) / 4], qb = q4[(m * HD + 8 * c) / 4 + 1];
        float a = s[m];
        a = fmaf(qa.x, kf[0], a);
        a = fmaf(qa.y, kf[1], a);
        a = fmaf(qa.z, kf[2], a);
        a = fmaf(qa.w, kf[3], a);
        a = fmaf(qb.x, kf[4], a);
        a = fmaf(qb.y, kf[5], a);
        a = fmaf(qb.z, kf[6], a);
        a = fmaf(qb.w, kf[7], a);
        s[m] = a;
      }
    }
    // ---- online softmax over this warp's 32 keys (keys past the split or the causal
    // limit of query m count as -inf)
#pragma unroll
    for (int m = 0; m < QW; ++m) {
      const bool vis = t < t_end && t <= lim0 + m;
      const float sm = vis ? s[m] : -INFINITY;
      const float m_new = fmaxf(m_run[m], warp_max(sm));
      float pr = 0.0f;
      if (m_new != -INFINITY) {  // warp-uniform
        if (m_new != m_run[m]) {
          const float alpha = ex2_approx(m_run[m] - m_new);  // 0 while m_run is -inf
          l_lane[m] *= alpha;
#pragma unroll
          for (int e = 0; e < 4; ++e) o_acc[m][e] *= alpha;
          m_run[m] = m_new;
        }
        pr = vis ? ex2_approx(sm - m_new) : 0.0f;
      }
      l_lane[m] += pr;
      pbuf[lane * QW + m] = pr;
    }
    __syncwarp();
    // ---- o += p . v, lane = head dims [4*lane, 4*lane + 4)
    const int nv = min(32, t_end - t0);  // keys of this warp that exist (warp-uniform)
    const uint32_t vcol = (lane >> 4) * BOX + (lane & 1) * 8;
    const int vchunk = (lane & 15) >> 1;
    for (int j = 0; j < nv; ++j) {
      const int rr = 32 * kw + j;
      const uint2 vw = *reinterpret_cast<const uint2*>(vb + vcol + rr * 128 + ((vchunk ^ (rr & 7)) << 4));
      const float v0 = __uint_as_float(vw.x << 16), v1 = __uint_as_float(vw.x & 0xffff0000u);
      const float v2 = __uint_as_float(vw.y << 16), v3 = __uint_as_float(vw.y & 0xffff0000u);
      const float* pj = pbuf + j * QW;
      if constexpr (QW >= 4) {
#pragma unroll
        for (int m = 0; m < QW; m += 4) {
          const float4 p4 = *reinterpret_cast<const float4*>(pj + m);
          const float pm[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            o_acc[m + u][0] = fmaf(pm[u], v0, o_acc[m + u][0]);
            o_acc[m + u][1] = fmaf(pm[u], v1, o_acc[m + u][1]);
            o_acc[m + u][2] = fmaf(pm[u], v2, o_acc[m + u][2]);
            o_acc[m + u][3] = fmaf(pm[u], v3, o_acc[m + u][3]);
          }
        }
      } else {
#pragma unroll
        for (int m = 0; m < QW; ++m) {
          const float pm = pj[m];
          o_acc[m][0] = fmaf(pm, v0, o_acc[m][0]);
          o_acc[m][1] = fmaf(pm, v1, o_acc[m][1]);
          o_acc[m][2] = fmaf(pm, v2, o_acc[m][2]);
          o_acc[m][3] = fmaf(pm, v3, o_acc[m][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  if (!ok && !skip) {
    report_error(p.err, (K_DEC << 8) | SITE_CONSUME);
    *abort_flag = 1;
  }

  // ---------------- merge the key warps' partials (consumer threads only) ----------------
  // Every tile has been consumed, so no copy is in flight and the ring's memory is free.
  // Query q0 + m of warp w goes to slot (kw, q0 + m).
  named_bar_sync(1, NCW * 32);
  float* wo = reinterpret_cast<float*>(smem);                 // [KW][MT][HD]
  float* wml = wo + KW * MT * HD;                             // [KW][MT][2]
#pragma unroll
  for (int m = 0; m < QW; ++m) {
    const float l = warp_sum(l_lane[m]);
    *reinterpret_cast<float4*>(wo + (kw * MT + q0 + m) * HD + 4 * lane) =
        make_float4(o_acc[m][0], o_acc[m][1], o_acc[m][2], o_acc[m][3]);
    if (lane == 0) {
      wml[(kw * MT + q0 + m) * 2] = m_run[m];
      wml[(kw * MT + q0 + m) * 2 + 1] = l;
    }
  }
  named_bar_sync(1, NCW * 32);
  if (skip || *abort_flag) return;
  const size_t part = (size_t)bh * p.S + split;
  for (int i = threadIdx.x; i < p.M * HD; i += NCW * 32) {
    const int m = i / HD, d = i % HD;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < KW; ++w) mx = fmaxf(mx, wml[(w * MT + m) * 2]);
    float l = 0.0f, o = 0.0f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < KW; ++w) {
        const float wm = wml[(w * MT + m) * 2];
        const float wgt = ex2_approx(wm - mx);  // 0 for a warp that saw no visible key
        l += wgt * wml[(w * MT + m) * 2 + 1];
        o += wgt * wo[(w * MT + m) * HD + d];
      }
    }
    const size_t n_parts = (size_t)p.B * p.H * p.S * p.M;
    if (in_bounds((part * p.M + m) * HD + d, 1, n_parts * HD, p.err, (K_DEC << 8) | SITE_CONSUME))
      p.part_o[(part * p.M + m) * HD + d] = o;
    if (d == 0 && in_bounds((part * p.M + m) * 2, 2, n_parts * 2, p.err, (K_DEC << 8) | SITE_CONSUME)) {
      p.part_ml[(part * p.M + m) * 2] = mx;
      p.part_ml[(part * p.M + m) * 2 + 1] = l;
    }
  }
}

// o[b, m, h, :] = sum_s 2^(m_s - mx) o_s / sum_s 2^(m_s - mx) l_s ;  lse = ln2 * (mx + log2 L).
// One CTA per (b, h, m) with CG groups of HD threads: the splits' (max, sum) pairs and the
// partial outputs (group g: splits g, g+CG, ... of its column d) are loaded in one parallel
// round, so the step costs about one memory latency.  Split 0 holds key 0,
// visible to every query, so mx is finite.
constexpr int CG = 4;
__global__ void __launch_bounds__(CG * HD) decode_combine_kernel(const float* part_o, const float* part_ml,
                                                                 __nv_bfloat16* o, float* lse, int M, int H,
                                                                 int S) {
  static_assert(kDecodeMaxSplits <= HD, "the first HD threads hold one split each");
  __shared__ float wgt[kDecodeMaxSplits];
  __shared__ float red[HD / 32][2];
  __shared__ float part[CG][HD];
  const int m = (int)(blockIdx.x % M);
  const int bh = (int)(blockIdx.x / M);
  const int h = bh % H, b = bh / H;
  const int tid = threadIdx.x, grp = tid / HD, d = tid % HD, warp = tid / 32, lane = tid % 32;
  // launched as a programmatic dependent of the split kernel: wait until that grid has
  // completed and its writes are visible (a no-op under ordinary stream order)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // group grp: splits grp, grp + CG, ... (at most kDecodeMaxSplits / CG = 16) of column d.  These
  // loads do not depend on the weights, so they go out together with the (max, sum) loads below:
  // the two rounds of memory latency overlap.
  const float* po = part_o + ((size_t)bh * S * M + m) * HD + d;  // split s at po[s * M * HD]
  constexpr int PER = kDecodeMaxSplits / CG;
  float v[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int sidx = grp + u * CG;
    v[u] = sidx < S ? po[(size_t)sidx * M * HD] : 0.0f;
  }
  const float* ml = part_ml + (size_t)bh * S * M * 2;
  // group 0: thread d holds split d; mx = max over splits, L = sum of weighted sums
  float ms = -INFINITY, ls = 0.0f;
  if (grp == 0 && d < S) {
    ms = ml[(d * M + m) * 2];
    ls = ml[(d * M + m) * 2 + 1];
  }
  float x = ms;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  if (grp == 0 && lane == 0) red[warp][0] = x;
  __syncthreads();
  float mx = red[0][0];
#pragma unroll
  for (int w = 1; w < HD / 32; ++w) mx = fmaxf(mx, red[w][0]);
  const float w_s = (grp == 0 && d < S && ms != -INFINITY) ? exp2f(ms - mx) : 0.0f;
  if (grp == 0 && d < S) wgt[d] = w_s;
  float y = w_s * ls;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
  if (grp == 0 && lane == 0) red[warp][1] = y;
  __syncthreads();
  float acc = 0.0f;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int sidx = grp + u * CG;
    if (sidx < S) acc = fmaf(wgt[sidx], v[u], acc);
  }
  part[grp][d] = acc;
  __syncthreads();
  if (grp == 0) {
    float L = 0.0f;
#pragma unroll
    for (int w = 0; w < HD / 32; ++w) L += red[w][1];
    float tot = 0.0f;
#pragma unroll
    for (int g = 0; g < CG; ++g) tot += part[g][d];
    o[((size_t)(b * M + m) * H + h) * HD + d] = __float2bfloat16_rn(tot / L);
    if (d == 0) lse[(size_t)bh * M + m] = (mx + log2f(L)) * 0.69314718055994531f;
  }
}

template <int MT>
cudaError_t launch_split(const CUtensorMap& tk, const CUtensorMap& tv, const Params& p, cudaStream_t st) {
  // the shared-memory limit is a per-device function attribute: set it once per device
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (!bit || !(done_mask.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(decode_split_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    done_mask.fetch_or(bit, std::memory_order_acq_rel);
  }
  const long long grid = (long long)p.B * p.H * p.S;
  decode_split_kernel<MT><<<(unsigned)grid, Cfg<MT>::NTHREADS, SMEM_BYTES, st>>>(tk, tv, p);
  return cudaGetLastError();
}

}  // namespace dec

// ---------------------------------------------------------------------------------------
// Tensor-core decoding step for more queries (M up to 128: speculative decoding, chunked
// prefill).  With M > 8 the CUDA-core kernel runs out of arithmetic (4*M*D FLOPs per key),
// so here the step is the forward's tcgen05 machinery on one query tile of 128 rows (rows
// >= M are padding and discarded) against the split's 64-key tiles:
//   S(i) = Q K(i)^T (SS, N = 64, fp32 in TMEM, two buffers), P(i) = exp2(S*scale*log2e - m)
//   written back over S(i) as bf16, O += P(i) V(i) (TS), online softmax with the lazy rescale.
// The issue order S(i) | PV(i-1) lets the softmax of tile i-1 run while S(i) computes.
// 64-key tiles keep a CTA at 256 TMEM columns and ~97 KB of shared memory, so two CTAs share
// an SM and one's start-up (TMEM allocation, the Q tile, the first K/V latency) overlaps the
// other's streaming.  Warps 0-3: softmax (thread = query row = TMEM lane); warp 4: TMA
// producer and TMEM owner; warp 5: MMA issuer.  The partials go to the same workspace
// layout as above.
namespace dtc {

// Wait of the MMA-issuing thread: polls the barrier with test_wait instead of suspending in
// try_wait, checking the abort flags and the time limit every 1024 polls.  Here it is 1.5-2.5 %
// faster at every M (the softmax warps' arrival is seen sooner); in the attention forward and
// backward, whose MMA thread shares its SM sub-partition with busy warps, polling was slower.
__device__ __forceinline__ bool wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort, const int* gerr) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_test_wait(bar, parity)) return true;
    if ((n & 1023u) == 0) {
      if (*abort || *(const volatile int*)gerr) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) return false;
    }
  }
}


constexpr int HD = 128, BM = 128, BN = kDecodeTileKeys;  // 64 keys per tile
constexpr uint32_t QBOX = BM * 128;           // 128 rows x 128 B (64 bf16 columns)
constexpr uint32_t KBOX = BN * 128;           // 64 rows x 128 B
constexpr uint32_t QTILE = 2 * QBOX;          // 128 query rows x 128 bf16
constexpr uint32_t KTILE = 2 * KBOX;          // 64 key rows x 128 bf16
// K and V stream through rings of their own: a K slot is free once S(i) has read it, a V slot
// only once PV(i) has, so the load of K(i+1) no longer waits for PV(i-1) (measured at 32k,
// H = 32: M = 16 0.126 -> 0.108 ms, M = 128 0.171 -> 0.148 ms; a third K stage or longer
// splits changed nothing).
constexpr int KST = 2;                        // K ring stages
constexpr int VST = 2;                        // V ring stages
constexpr int NTHREADS = 192;
constexpr int WARP_LOAD = 4, WARP_MMA = 5;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + QTILE;             // [KST]
constexpr uint32_t OFF_V = OFF_K + KST * KTILE;       // [VST]
constexpr uint32_t OFF_BAR = OFF_V + VST * KTILE;
// barriers: q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], p_ready[2],
// pv_done, o_final, drain.
// p_ready is double-buffered by tile parity: S(i) is issued before the wait for P(i-1), so
// the softmax may finish tile i before that wait looks; with a single barrier it would then
// be two phases ahead and the parity wait would miss the completed phase.
constexpr int NBARS = 1 + 2 * KST + 2 * VST + 2 + 2 + 3;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16;  // the dynamic smem base is 1024-byte aligned
static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs must fit on an SM");
constexpr uint32_t TM_COLS = 256;                       // two CTAs per SM
constexpr uint32_t TM_O = 128;                          // S buffers at columns 0 and 64

struct Params {
  float* part_o;
  float* part_ml;
  int B, M, N, H, S, tiles_per_split;
  float sl2;  // log2(e) / sqrt(D)
  int* err;
};

enum Site : int { SITE_LOAD = 5, SITE_MMA = 6, SITE_SOFTMAX = 7, SITE_DRAIN = 8, SITE_ALIGN = 9 };

// S[128 x 64] = Q K^T: both K-major; the 64-column halves of the head dim are QBOX / KBOX apart.
__device__ __forceinline__ void issue_s(uint32_t d, uint32_t sq, uint32_t sk, uint32_t idesc) {
  const uint64_t dq = sdesc_sw128(sq, 16, 1024), dk = sdesc_sw128(sk, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    mma_ss(d, sdesc_add(dq, (kk / 4) * QBOX + (kk % 4) * 32), sdesc_add(dk, (kk / 4) * KBOX + (kk % 4) * 32), idesc,
           kk > 0 ? 1u : 0u);
  }
}

// O[128 x 128] += P V: P (bf16 pairs) from TMEM, V^T viewed MN-major (64-dim blocks KBOX apart,
// 16 key rows = 2 KB per k-step).
__device__ __forceinline__ void issue_pv(uint32_t d, uint32_t tp, uint32_t sv, uint32_t idesc, bool first) {
  const uint64_t dv = sdesc_sw128(sv, KBOX, 1024);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) mma_ts(d, tp + kk * 8, sdesc_add(dv, kk * 2048), idesc, (first && kk == 0) ? 0u : 1u);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// P row = exp2(s * sl2 - m) with columns c > lim masked (MASK; without it every column is
// visible), written as bf16 pairs over the first 32 TMEM columns of the row's S buffer; returns
// the fp32 row sum.
template <bool MASK>
__device__ __forceinline__ float p_row(const uint32_t (&sr)[64], int lim, float sl2, float neg_m, uint32_t t_s) {
  const float2 scale2 = make_float2(sl2, sl2), shift2 = make_float2(neg_m, neg_m);
  float2 sp[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) sp[e] = make_float2(0.f, 0.f);
  uint32_t pk[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), scale2, shift2);
    float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
    if (MASK) {
      p0 = 2 * c <= lim ? p0 : 0.f;
      p1 = 2 * c + 1 <= lim ? p1 : 0.f;
    }
    sp[c % 4].x += p0;
    sp[c % 4].y += p1;
    pk[c] = pack_bf16x2(p0, p1);
  }
  tmem_st_x32(t_s, pk);
  return ((sp[0].x + sp[1].x) + (sp[2].x + sp[3].x)) + ((sp[0].y + sp[1].y) + (sp[2].y + sp[3].y));
}

__global__ void __launch_bounds__(NTHREADS, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;       // [2]
  uint64_t* p_ready = s_full + 2;         // [2]
  uint64_t* pv_done = s_full + 4;
  uint64_t* o_final = s_full + 5;
  uint64_t* drain = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int units = p.B * p.H;
  const int bh = (int)(blockIdx.x % units);  // consecutive CTAs: the same split of consecutive heads
  const int split = (int)(blockIdx.x / units);
  const int h = bh % p.H, b = bh / p.H;
  const int t_begin = split * p.tiles_per_split * BN;
  const int t_end = min(p.N, t_begin + p.tiles_per_split * BN);
  const int n_tiles = t_end > t_begin ? (t_end - t_begin + BN - 1) / BN : 0;

  // 128-byte-swizzled TMA boxes and MMA descriptors assume 1024-byte aligned tiles.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_error(p.err, (K_DEC << 8) | SITE_ALIGN);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_ready[0], 4);
    mbar_init(&p_ready[1], 4);
    mbar_init(pv_done, 1);
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    *abort_flag = (*(volatile int*)p.err != 0) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == WARP_LOAD) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort_flag != 0 || n_tiles == 0;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (!skip && warp == WARP_LOAD && lane == 0) {
    // ---------------- TMA producer ----------------
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    bool ok = true;
    int k_issued = 0, v_issued = 0;
    mbar_arrive_expect_tx(q_full, QTILE);
    for (int x = 0; x < 2; ++x) tma_load_3d(smem + OFF_Q + x * QBOX, &tq, x * 64, h, b * p.M, q_full);
    // issue order K(0), then K(j+1), V(j): S(i) (reads K(i)) is issued before PV(i-1) (reads V(i-1))
    auto load_k = [&](int i) -> bool {
      const int slot = i % KST;
      if (i >= KST && !wait_bounded(&k_empty[slot], ((i / KST) - 1) & 1, abort_flag, p.err)) return false;
      const int row = b * p.N + t_begin + i * BN;
      mbar_arrive_expect_tx(&k_full[slot], KTILE);
      for (int x = 0; x < 2; ++x) tma_load_3d(smem + OFF_K + slot * KTILE + x * KBOX, &tk, x * 64, h, row, &k_full[slot]);
      k_issued = i + 1;
      return true;
    };
    auto load_v = [&](int i) -> bool {
      const int slot = i % VST;
      if (i >= VST && !wait_bounded(&v_empty[slot], ((i / VST) - 1) & 1, abort_flag, p.err)) return false;
      const int row = b * p.N + t_begin + i * BN;
      mbar_arrive_expect_tx(&v_full[slot], KTILE);
      for (int x = 0; x < 2; ++x) tma_load_3d(smem + OFF_V + slot * KTILE + x * KBOX, &tv, x * 64, h, row, &v_full[slot]);
      v_issued = i + 1;
      return true;
    };
    ok = load_k(0);
    for (int i = 0; i < n_tiles && ok; ++i) {
      if (i + 1 < n_tiles) ok = load_k(i + 1);
      if (ok) ok = load_v(i);
    }
    if (!ok) {
      report_error(p.err, (K_DEC << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
    bool dok = wait_drain(q_full, 0);
    for (int i = (k_issued > KST ? k_issued - KST : 0); i < k_issued; ++i) dok &= wait_drain(&k_full[i % KST], (i / KST) & 1);
    for (int i = (v_issued > VST ? v_issued - VST : 0); i < v_issued; ++i) dok &= wait_drain(&v_full[i % VST], (i / VST) & 1);
    if (!dok) report_error(p.err, (K_DEC << 8) | SITE_DRAIN);
  } else if (!skip && warp == WARP_MMA && lane == 0) {
    // ---------------- MMA issuer: S(i) | PV(i-1) ----------------
    const uint32_t id_s = idesc_bf16_f32(BM, BN, false, false);
    const uint32_t id_pv = idesc_bf16_f32(BM, HD, false, true);
    const uint32_t sq = smem_u32(smem + OFF_Q), sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
    bool ok = wait_spin(q_full, 0, abort_flag, p.err);
    for (int i = 0; i <= n_tiles && ok; ++i) {
      if (i < n_tiles) {
        ok = wait_spin(&k_full[i % KST], (i / KST) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        issue_s(tmem + (uint32_t)BN * (i & 1), sq, sk + (i % KST) * KTILE, id_s);
        mma_commit(&s_full[i & 1]);
        mma_commit(&k_empty[i % KST]);  // K(i) read once S(i) completes
      }
      if (i > 0) {
        ok = wait_spin(&p_ready[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, p.err);
        if (ok) ok = wait_spin(&v_full[(i - 1) % VST], ((i - 1) / VST) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        issue_pv(tmem + TM_O, tmem + (uint32_t)BN * ((i - 1) & 1), sv + ((i - 1) % VST) * KTILE, id_pv, i == 1);
        mma_commit(pv_done);
        mma_commit(&v_empty[(i - 1) % VST]);
      }
    }
    if (ok) mma_commit(o_final);
    if (!ok) {
      report_error(p.err, (K_DEC << 8) | SITE_MMA);
      *abort_flag = 1;
    }
    mma_commit(drain);
    if (!wait_drain(drain, 0)) report_error(p.err, (K_DEC << 8) | SITE_DRAIN);
  } else if (!skip && warp < 4) {
    // ---------------- softmax: thread = query row r ----------------
    const int r = warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = p.sl2;
    const int last_vis = min(p.N - p.M + r, t_end - 1);  // last key row r sees in this split
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int buf = i & 1;
      ok = wait_bounded(&s_full[buf], (i >> 1) & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_s = lane_addr + (uint32_t)BN * buf;
      uint32_t s0[64];
      tmem_ld_x64(t_s, s0);
      const int lim = last_vis - (t_begin + i * BN);  // columns c <= lim are visible (may be < 0)
      // every column of the tile visible to all rows of the warp (all but the last tiles of
      // the sequence): no mask compares
      const bool full = __all_sync(0xffffffffu, lim >= BN - 1);
      float mxp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mxp[e] = -INFINITY;
      if (full) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          mxp[c % 8] = max3f(mxp[c % 8], __uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1]));
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          mxp[c % 8] = max3f(mxp[c % 8], 2 * c <= lim ? __uint_as_float(s0[2 * c]) : -INFINITY,
                             2 * c + 1 <= lim ? __uint_as_float(s0[2 * c + 1]) : -INFINITY);
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                             fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
      // lazy rescale: move the running max only when it grows by more than 2^8 (a row that has
      // seen no visible key yet keeps -inf, and its P stays 0)
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool need = (m_new - m_run) > 8.0f;
      const bool rescale = __any_sync(0xffffffffu, need);
      const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
      if (need) m_run = m_new;
      l_run *= alpha;
      l_run += full ? p_row<false>(s0, lim, sl2, -m_run, t_s) : p_row<true>(s0, lim, sl2, -m_run, t_s);
      if (rescale && i > 0) {
        // O was last written by PV(i-1): wait for it, then scale this row of O
        ok = wait_bounded(pv_done, (i - 1) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD; c += 32) {
          uint32_t rr[32];
          tmem_ld_x32(lane_addr + TM_O + c, rr);
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
          tmem_st_x32(lane_addr + TM_O + c, rr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[buf]);
    }
    if (ok) ok = wait_bounded(o_final, 0, abort_flag, p.err);
    if (ok) {
      // partial of this split: unnormalised O row, running max (log2 domain) and sum
      tc_fence_after();
      const size_t part = (size_t)bh * p.S + split;
      const size_t n_parts = (size_t)p.B * p.H * p.S * p.M;
      const bool row_ok = r < p.M && in_bounds((part * p.M + r) * HD, HD, n_parts * HD, p.err,
                                                 (K_DEC << 8) | SITE_SOFTMAX);
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t rr[32];
        tmem_ld_x32(lane_addr + TM_O + c, rr);
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + (part * p.M + r) * HD + c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(rr[4 * e]), __uint_as_float(rr[4 * e + 1]),
                                 __uint_as_float(rr[4 * e + 2]), __uint_as_float(rr[4 * e + 3]));
        }
      }
      if (row_ok) {
        p.part_ml[(part * p.M + r) * 2] = m_run;
        p.part_ml[(part * p.M + r) * 2 + 1] = l_run;
      }
    } else {
      report_error(p.err, (K_DEC << 8) | SITE_SOFTMAX);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_LOAD) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace dtc

int decode_splits(int B, int N, int H, int n_sm, int* tiles_per_split) {
  const int n_tiles = (N + dec::TK - 1) / dec::TK;
  const long long units = (long long)B * H;
  const long long slots = 2LL * n_sm;                          // two CTAs per SM
  const long long base_ctas = units * ((n_tiles + 15) / 16);  // about 16 tiles (1024 keys) per CTA
  const long long waves = (base_ctas + slots - 1) / slots;
  long long s = (waves * slots) / units;
  if (s < 1) s = 1;
  if (s > n_tiles) s = n_tiles;
  if (s > kDecodeMaxSplits) s = kDecodeMaxSplits;
  const int tps = (int)((n_tiles + s - 1) / s);
  *tiles_per_split = tps;
  return (n_tiles + tps - 1) / tps;
}

// The combine kernel is a programmatic dependent launch: it is scheduled while the split
// kernel drains, which hides its launch latency.
static cudaError_t launch_combine(const float* part_o, const float* part_ml, void* o, float* lse, int B, int M,
                                  int H, int S, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)B * H * M));
  cfg.blockDim = dim3(dec::CG * dec::HD);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dec::decode_combine_kernel, part_o, part_ml, static_cast<__nv_bfloat16*>(o), lse,
                            M, H, S);
}

int decode_splits_tc(int B, int N, int H, int n_sm, int* tiles_per_split) {
  const int n_tiles = (N + dtc::BN - 1) / dtc::BN;
  const long long units = (long long)B * H;
  const long long slots = 2LL * n_sm;                          // two CTAs per SM
  // about 32 tiles (2048 keys) per CTA: the fp32 partials grow with M times the number of splits
  // (at 32k and M = 128, 16-tile splits write and read back 138 MB of partials against 537 MB of
  // K/V; 32-tile splits: M = 128 0.149 -> 0.137 ms, M = 64 0.122 -> 0.118 ms, M <= 16 unchanged)
  const long long base_ctas = units * ((n_tiles + 31) / 32);
  const long long waves = (base_ctas + slots - 1) / slots;
  long long s = (waves * slots) / units;
  if (s < 1) s = 1;
  if (s > n_tiles) s = n_tiles;
  if (s > kDecodeMaxSplits) s = kDecodeMaxSplits;
  const int tps = (int)((n_tiles + s - 1) / s);
  *tiles_per_split = tps;
  return (n_tiles + tps - 1) / tps;
}

cudaError_t launch_decode_tc_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                                   float* lse, float* part_o, float* part_ml, int B, int M, int N, int H, int S,
                                   int tiles_per_split, int* err, cudaStream_t st) {
  dtc::Params p;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.B = B;
  p.M = M;
  p.N = N;
  p.H = H;
  p.S = S;
  p.tiles_per_split = tiles_per_split;
  p.sl2 = (float)(1.4426950408889634 / sqrt((double)dtc::HD));
  p.err = err;
  const long long grid = (long long)B * H * S;
  if (grid <= 0 || grid > 0x7fffffffLL || M < 1 || M > dtc::BM) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (!bit || !(done_mask.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(dtc::decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dtc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    done_mask.fetch_or(bit, std::memory_order_acq_rel);
  }
  dtc::decode_tc_kernel<<<(unsigned)grid, dtc::NTHREADS, dtc::SMEM_BYTES, st>>>(tq, tk, tv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_combine(part_o, part_ml, o, lse, B, M, H, S, st);
}

cudaError_t launch_decode_sm100(const CUtensorMap& tk, const CUtensorMap& tv, const void* q, void* o, float* lse,
                                float* part_o, float* part_ml, int B, int M, int N, int H, int S,
                                int tiles_per_split, int* err, cudaStream_t st) {
  dec::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.B = B;
  p.M = M;
  p.N = N;
  p.H = H;
  p.S = S;
  p.tiles_per_split = tiles_per_split;
  p.qscale = (float)(1.4426950408889634 / sqrt((double)dec::HD));
  p.err = err;
  const long long grid = (long long)B * H * S;
  if (grid <= 0 || grid > 0x7fffffffLL || M < 1 || M > dec::MAXM) return cudaErrorInvalidValue;
  static_assert(kDecodeSimtMaxM == 1, "instantiate decode_split_kernel for the query counts dispatched here");
  if (M != 1) return cudaErrorInvalidValue;
  cudaError_t e = dec::launch_split<1>(tk, tv, p, st);
  if (e != cudaSuccess) return e;
  return launch_combine(part_o, part_ml, o, lse, B, M, H, S, st);
}

}  // namespace s2
