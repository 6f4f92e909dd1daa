// s2attn_decode_sm100.cu -- a decoding step of full causal attention on B200 (sm_100a).
//
// Inference runs ordinary full attention; S^2-Attn is a training-time device only
// ("LongLoRA paper notes", section 3.1; model.aibase.cn, features list).  A decoding
// step appends M (<= 16) tokens to a sequence of N positions: k, v [B,N,H,D] hold all
// N positions (the new ones included), q [B,M,H,D] the M new queries; query m sits at
// position N-M+m and sees keys 0 .. N-M+m.
//
// With a handful of queries the step is a matrix-vector product over the whole K/V of
// every head: 2*N*D*2 bytes per head and 4*M*D FLOPs per key, so it is bound by HBM, not
// by arithmetic -- it runs on the CUDA cores, and its job is to stream K and V at full
// bandwidth:
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
    p.part_o[(part * p.M + m) * HD + d] = o;
    if (d == 0) {
      p.part_ml[(part * p.M + m) * 2] = mx;
      p.part_ml[(part * p.M + m) * 2 + 1] = l;
    }
  }
}

// o[b, m, h, :] = sum_s 2^(m_s - mx) o_s / sum_s 2^(m_s - mx) l_s ;  lse = ln2 * (mx + log2 L).
// One CTA per (b, h, m) with CG groups of HD threads: the splits' (max, sum) pairs are loaded
// in one parallel round, and group g sums splits g, g+CG, ... of its column d with
// independent loads, so the step costs about two memory latencies.  Split 0 holds key 0,
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
  // group grp: splits grp, grp + CG, ... (at most kDecodeMaxSplits / CG = 16), loads first
  const float* po = part_o + ((size_t)bh * S * M + m) * HD + d;  // split s at po[s * M * HD]
  constexpr int PER = kDecodeMaxSplits / CG;
  float v[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int sidx = grp + u * CG;
    v[u] = sidx < S ? po[(size_t)sidx * M * HD] : 0.0f;
  }
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
  cudaError_t e;
  if (M == 1) e = dec::launch_split<1>(tk, tv, p, st);
  else if (M == 2) e = dec::launch_split<2>(tk, tv, p, st);
  else if (M <= 4) e = dec::launch_split<4>(tk, tv, p, st);
  else if (M <= 8) e = dec::launch_split<8>(tk, tv, p, st);
  else e = dec::launch_split<16>(tk, tv, p, st);
  if (e != cudaSuccess) return e;
  // the combine kernel is a programmatic dependent launch: it is scheduled while the
  // split kernel drains, which hides its launch latency
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
  return cudaLaunchKernelEx(&cfg, dec::decode_combine_kernel, static_cast<const float*>(part_o),
                            static_cast<const float*>(part_ml), static_cast<__nv_bfloat16*>(o), lse, M, H, S);
}

}  // namespace s2
