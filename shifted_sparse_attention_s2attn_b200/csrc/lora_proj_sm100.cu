// lora_proj_sm100.cu -- LoRA-adapted linear projections on B200 (sm_100a), the steps on
// either side of S^2-Attn: y = x W^T + s (x A^T) B^T for one or several projections
// stacked along the output (q, k and v in one launch, or o alone), with RoPE-PI applied
// in the epilogue to the first parts (q and k) when asked.
//
// Method (LongLoRA pages: "LongLoRA paper notes" section 3.2 -- low-rank adapters on the
// Q, K, V and O projections; nearauto.com article, "long-context LoRA improvement"):
// the frozen weight W gets a trainable low-rank update B A of rank r, scaled by s
// (alpha / r).  Position interpolation ("LongLoRA paper notes" section 3.4) rotates the
// q and k rows before attention; doing it here, on the tile the projection has just
// computed, removes the separate RoPE pass over q and k in HBM.
//
// Three launches:
//   1. pad:  A and B copied into zero-padded operands of rank 64 (a_pad [parts*64, K],
//            b_pad [parts*n_out, 64]), so the rank dimension is one 64-wide K block.
//   2. down: u = bf16(s * x a_pad^T), written [parts, T, 64] (columns >= r are zero).
//   3. proj: y = x W^T + u_part b_pad^T: the K loop over x and W, then one more K block
//            whose operands are u (this part's 64 columns) and b_pad, accumulated into
//            the same TMEM tile.  The epilogue rounds to bf16 and, for the rotated parts,
//            applies RoPE-PI to the rounded values with the same fp32 operations and table
//            as rope_pi_apply, so the fused result equals projection-then-rope_pi_apply.
// down and proj are one kernel template: persistent CTAs walk 128 x BN output tiles in
// groups of 16 row blocks (so the x rows and W columns in flight stay in L2), with
//   warp 0      TMA producer (x and W boxes of 64 columns through a 4-stage ring)
//   warp 1      MMA issuer (tcgen05, M = 128, N = BN, K = 16 per instruction); TMEM owner
//   warps 2-5   epilogue (thread = output row; TMEM lane quarter = warp % 4)
// and two TMEM accumulators, so the epilogue of one tile overlaps the K loop of the next.
#include <algorithm>

#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace lora {

constexpr int BM = 128;          // output rows per tile
constexpr int BK = 64;           // K columns per stage (one 128-byte swizzle row of bf16)
constexpr int NTHREADS = 192;
constexpr int WARP_LOAD = 0, WARP_MMA = 1;
constexpr int STAGES = 4;
constexpr int GROUP_M = 16;      // row blocks walked together (tile raster)

template <int BN>
struct Cfg {
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t OFF_BAR = STAGES * STAGE_BYTES;
  // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
  static constexpr int NBARS = 2 * STAGES + 5;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024 B
  static constexpr uint32_t TMEM_COLS = 2 * BN;                 // two fp32 accumulators
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "tcgen05 N for M = 128");
  static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS >= 32 && TMEM_COLS <= 512, "TMEM allocation");
};

struct Params {
  __nv_bfloat16* y;        // [parts, T, n_out]
  int T, n_out;            // rows; output columns per part (a multiple of BN)
  int n_kb;                // 64-column K blocks of x / W
  int n_mblk, n_nblk, n_tiles;
  int lora_k16;            // K=16 MMA steps of the rank block (LORA kernels only)
  float out_scale;         // multiplies the accumulator before rounding
  int rope_cols;           // output columns [0, rope_cols) (whole parts) get RoPE-PI; 0: none
  int head_dim, seq_len;   // RoPE pairing (i, i + head_dim/2); row t is position t mod seq_len
  const float* cos_tab;    // [seq_len, head_dim/2]
  const float* sin_tab;
  int* err;
};

enum Site : int { SITE_LOAD = 1, SITE_MMA = 2, SITE_EPILOGUE = 3, SITE_DRAIN = 4 };

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Tile i -> (row block, column block): groups of GROUP_M row blocks, row block fastest.
__device__ __forceinline__ void tile_coords(int i, int n_mblk, int n_nblk, int& mb, int& nb) {
  const int per_group = GROUP_M * n_nblk;
  const int g = i / per_group;
  const int first = g * GROUP_M;
  const int gsize = min(GROUP_M, n_mblk - first);
  const int local = i - g * per_group;
  mb = first + local % gsize;
  nb = local / gsize;
}

__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// LORA: the K loop ends with the rank block (operands tu / tb).  Without it tu / tb are unused.
template <int BN, bool LORA>
__global__ void __launch_bounds__(NTHREADS, BN <= 64 ? 2 : 1)
    lora_gemm_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
                     const __grid_constant__ CUtensorMap tu, const __grid_constant__ CUtensorMap tb,
                     const Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_kb_total = p.n_kb + (LORA ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = (*(volatile int*)p.err != 0) ? 1 : 0;  // an earlier launch failed: skip the work
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort_flag != 0;

  if (!skip && warp == WARP_LOAD && lane == 0) {
    // ---------------- TMA producer ----------------
    prefetch_tmap(&tx);
    prefetch_tmap(&tw);
    if (LORA) {
      prefetch_tmap(&tu);
      prefetch_tmap(&tb);
    }
    bool ok = true;
    int g = 0;  // loads armed (ring position)
    for (int i = blockIdx.x; i < p.n_tiles && ok; i += gridDim.x) {
      int mb, nb;
      tile_coords(i, p.n_mblk, p.n_nblk, mb, nb);
      const int m0 = mb * BM, n0 = nb * BN;
      for (int kb = 0; kb < n_kb_total; ++kb) {
        const int s = g % STAGES;
        ok = wait_bounded(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag, p.err);
        if (!ok) break;
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        if (!LORA || kb < p.n_kb) {
          tma_load_2d(sa, &tx, kb * BK, m0, &full[s]);
          tma_load_2d(sb, &tw, kb * BK, n0, &full[s]);
        } else {
          tma_load_3d(sa, &tu, 0, m0, n0 / p.n_out, &full[s]);  // u of this tile's part
          tma_load_2d(sb, &tb, 0, n0, &full[s]);
        }
        ++g;
      }
    }
    if (!ok) {
      report_error(p.err, (K_LORA << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
    // Drain: every copy this thread started must land before the CTA can exit.
    bool dok = true;
    for (int t = (g > STAGES ? g - STAGES : 0); t < g; ++t) dok &= wait_drain(&full[t % STAGES], (t / STAGES) & 1);
    if (!dok) report_error(p.err, (K_LORA << 8) | SITE_DRAIN);
  } else if (!skip && warp == WARP_MMA && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
    const uint32_t s_base = smem_u32(smem);
    bool ok = true;
    int g = 0, lt = 0;
    for (int i = blockIdx.x; i < p.n_tiles && ok; i += gridDim.x, ++lt) {
      const int buf = lt & 1;
      const uint32_t d = tmem + (uint32_t)(buf * BN);
      // the epilogue has read this accumulator's previous tile out
      ok = wait_bounded(&acc_empty[buf], ((lt >> 1) & 1) ^ 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      // the K loop: four K=16 MMAs per stage, a compile-time count (unrolled) ...
      for (int kb = 0; kb < p.n_kb; ++kb) {
        const int s = g % STAGES;
        ok = wait_bounded(&full[s], (g / STAGES) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = s_base + s * C::STAGE_BYTES, sb = sa + C::A_BYTES;
        // K-major operands: 128-byte rows, 8-row groups 1024 B apart; K=16 steps are 32 B
        const uint64_t da = sdesc_sw128(sa, 16, 1024), db = sdesc_sw128(sb, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_ss(d, sdesc_add(da, kk * 32), sdesc_add(db, kk * 32), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        ++g;
      }
      // ... then the rank block, ceil(r/16) MMAs
      if (LORA && ok) {
        const int s = g % STAGES;
        ok = wait_bounded(&full[s], (g / STAGES) & 1, abort_flag, p.err);
        if (ok) {
          tc_fence_after();
          const uint32_t sa = s_base + s * C::STAGE_BYTES, sb = sa + C::A_BYTES;
          const uint64_t da = sdesc_sw128(sa, 16, 1024), db = sdesc_sw128(sb, 16, 1024);
          for (int kk = 0; kk < p.lora_k16; ++kk) mma_ss(d, sdesc_add(da, kk * 32), sdesc_add(db, kk * 32), idesc, 1u);
          mma_commit(&empty[s]);
          ++g;
        }
      }
      if (!ok) break;
      mma_commit(&acc_full[buf]);
    }
    if (!ok) {
      report_error(p.err, (K_LORA << 8) | SITE_MMA);
      *abort_flag = 1;
    }
    // Drain: all issued MMAs complete before TMEM is released.
    mma_commit(drain);
    if (!wait_drain(drain, 0)) report_error(p.err, (K_LORA << 8) | SITE_DRAIN);
  } else if (!skip && warp >= 2) {
    // ---------------- epilogue ----------------
    const int wq = warp % 4;  // TMEM lanes [32 wq, 32 wq + 32) are this warp's
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
    const float osc = p.out_scale;
    bool ok = true;
    int lt = 0;
    for (int i = blockIdx.x; i < p.n_tiles; i += gridDim.x, ++lt) {
      int mb, nb;
      tile_coords(i, p.n_mblk, p.n_nblk, mb, nb);
      const int buf = lt & 1;
      ok = wait_bounded(&acc_full[buf], (lt >> 1) & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const int grow = mb * BM + row;
      const int n0 = nb * BN;
      const int part = n0 / p.n_out;
      const bool row_ok =
          grow < p.T && in_bounds(((size_t)part * p.T + grow) * p.n_out + (n0 - part * p.n_out), BN,
                                  (size_t)p.T * p.n_out * (p.n_nblk * BN / p.n_out), p.err,
                                  (K_LORA << 8) | SITE_EPILOGUE);
      __nv_bfloat16* yrow = p.y + ((size_t)part * p.T + grow) * p.n_out + (n0 - part * p.n_out);
      const uint32_t ta = lane_addr + (uint32_t)(buf * BN);
      if (n0 < p.rope_cols) {
        // RoPE-PI on the bf16-rounded outputs: pair (i, i + D/2) of each head of the tile
        const int D = p.head_dim, half = D / 2;
        const int t = grow % p.seq_len;
        const float* ct = p.cos_tab + (size_t)t * half;
        const float* st = p.sin_tab + (size_t)t * half;
        for (int h0 = 0; h0 < BN; h0 += D) {
          for (int c = 0; c < half; c += 16) {
            uint32_t a[16], b[16];
            tmem_ld_x16(ta + h0 + c, a);
            tmem_ld_x16(ta + h0 + half + c, b);
            float cs[16], sn[16];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float4 cv = __ldg(reinterpret_cast<const float4*>(ct + c) + e);
              const float4 sv = __ldg(reinterpret_cast<const float4*>(st + c) + e);
              cs[4 * e] = cv.x; cs[4 * e + 1] = cv.y; cs[4 * e + 2] = cv.z; cs[4 * e + 3] = cv.w;
              sn[4 * e] = sv.x; sn[4 * e + 1] = sv.y; sn[4 * e + 2] = sv.z; sn[4 * e + 3] = sv.w;
            }
            uint32_t lo[8], hi[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float y1[2], y2[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int k = 2 * e + u;
                const float x1 = bf16_round(__uint_as_float(a[k]) * osc);
                const float x2 = bf16_round(__uint_as_float(b[k]) * osc);
                y1[u] = __fsub_rn(__fmul_rn(x1, cs[k]), __fmul_rn(x2, sn[k]));
                y2[u] = __fadd_rn(__fmul_rn(x2, cs[k]), __fmul_rn(x1, sn[k]));
              }
              lo[e] = pack_bf16x2(y1[0], y1[1]);
              hi[e] = pack_bf16x2(y2[0], y2[1]);
            }
            if (row_ok) {
              uint4* d1 = reinterpret_cast<uint4*>(yrow + h0 + c);
              uint4* d2 = reinterpret_cast<uint4*>(yrow + h0 + half + c);
              d1[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
              d1[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
              d2[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
              d2[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_x32(ta + c, r);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * osc, __uint_as_float(r[2 * e + 1]) * osc);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(yrow + c);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (!ok) {
      report_error(p.err, (K_LORA << 8) | SITE_EPILOGUE);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// a_pad[p*64 + j, :] = a[p*r + j, :] for j < r, else 0;  b_pad[c, j] = b[c, j] for j < r, else 0.
__global__ void lora_pad_kernel(const uint16_t* __restrict__ a, const uint16_t* __restrict__ b,
                                uint16_t* __restrict__ a_pad, uint16_t* __restrict__ b_pad, int parts, int r, int K,
                                long long b_rows) {
  const long long a_chunks = (long long)parts * kLoraRankPad * (K / 8);  // 8 elements each
  const long long total = a_chunks + b_rows * kLoraRankPad;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    if (w < a_chunks) {
      const long long row = w / (K / 8);
      const int c = (int)(w % (K / 8)) * 8;
      const int part = (int)(row / kLoraRankPad), j = (int)(row % kLoraRankPad);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (j < r) v = *reinterpret_cast<const uint4*>(a + ((size_t)part * r + j) * K + c);
      *reinterpret_cast<uint4*>(a_pad + (size_t)row * K + c) = v;
    } else {
      const long long e = w - a_chunks;
      const long long row = e / kLoraRankPad;
      const int j = (int)(e % kLoraRankPad);
      b_pad[e] = j < r ? b[row * r + j] : (uint16_t)0;
    }
  }
}

template <int BN, bool LORA>
cudaError_t launch_gemm(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& tu, const CUtensorMap& tb,
                        const Params& p, int ctas, cudaStream_t st) {
  using C = Cfg<BN>;
  cudaError_t e = cudaFuncSetAttribute(lora_gemm_kernel<BN, LORA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  lora_gemm_kernel<BN, LORA><<<ctas, NTHREADS, C::SMEM_BYTES, st>>>(tx, tw, tu, tb, p);
  return cudaGetLastError();
}

Params base_params(void* y, int T, int K, int n_out, int n_total, int bn, float out_scale, int* err) {
  Params p{};
  p.y = static_cast<__nv_bfloat16*>(y);
  p.T = T;
  p.n_out = n_out;
  p.n_kb = (K + BK - 1) / BK;
  p.n_mblk = (T + BM - 1) / BM;
  p.n_nblk = n_total / bn;
  p.n_tiles = p.n_mblk * p.n_nblk;
  p.out_scale = out_scale;
  p.head_dim = 128;
  p.seq_len = 1;
  p.err = err;
  return p;
}

}  // namespace lora

cudaError_t launch_lora_pad(const void* a, const void* b, void* a_pad, void* b_pad, int parts, int r, int K,
                            int n_out, cudaStream_t st) {
  const long long b_rows = (long long)parts * n_out;
  const long long total = (long long)parts * kLoraRankPad * (K / 8) + b_rows * kLoraRankPad;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 4096);
  lora::lora_pad_kernel<<<(unsigned)blocks, threads, 0, st>>>(
      static_cast<const uint16_t*>(a), static_cast<const uint16_t*>(b), static_cast<uint16_t*>(a_pad),
      static_cast<uint16_t*>(b_pad), parts, r, K, b_rows);
  return cudaGetLastError();
}

cudaError_t launch_lora_down(const CUtensorMap& tx, const CUtensorMap& ta_pad, void* u, int T, int K, int parts,
                             float scaling, int n_sm, int* err, cudaStream_t st) {
  constexpr int BN = kLoraRankPad;
  lora::Params p = lora::base_params(u, T, K, BN, parts * BN, BN, scaling, err);
  const int ctas = std::max(1, std::min(p.n_tiles, 2 * n_sm));  // two CTAs fit on an SM
  return lora::launch_gemm<BN, false>(tx, ta_pad, tx, ta_pad, p, ctas, st);
}

cudaError_t launch_lora_proj(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& tu,
                             const CUtensorMap& tb, void* y, int T, int K, int n_out, int parts, int r,
                             int rope_parts, int head_dim, int seq_len, const float* cos_tab, const float* sin_tab,
                             int n_sm, int* err, cudaStream_t st) {
  constexpr int BN = kLoraProjTileN;
  lora::Params p = lora::base_params(y, T, K, n_out, parts * n_out, BN, 1.0f, err);
  p.lora_k16 = (r + 15) / 16;
  p.rope_cols = rope_parts * n_out;
  if (rope_parts > 0) {
    p.head_dim = head_dim;
    p.seq_len = seq_len;
    p.cos_tab = cos_tab;
    p.sin_tab = sin_tab;
  }
  const int ctas = std::max(1, std::min(p.n_tiles, n_sm));
  if (r > 0) return lora::launch_gemm<BN, true>(tx, tw, tu, tb, p, ctas, st);
  return lora::launch_gemm<BN, false>(tx, tw, tx, tw, p, ctas, st);
}

}  // namespace s2
