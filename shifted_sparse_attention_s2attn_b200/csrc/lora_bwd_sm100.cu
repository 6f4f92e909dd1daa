// lora_bwd_sm100.cu -- backward of the LoRA-adapted projections on B200 (sm_100a).
//
// Method (LongLoRA pages: "LongLoRA paper notes" section 3.2 -- the low-rank adapters on the
// Q, K, V and O projections are what trains; the frozen weight W gets no gradient).  For
// y_p = x W_p^T + s (x A_p^T) B_p^T and the gradient dy [parts, T, n_out] of y (before RoPE:
// rope_pi_apply with -pos_scale takes dq and dk back through the rotation):
//   g_p  = s dy_p B_p                      [T, r]      held in bf16, [parts, T, 64] zero-padded
//   dx   = sum_p dy_p W_p + g_p A_p        [T, K]
//   dA_p = g_p^T x                         [r, K]
//   dB_p = dy_p^T u_p,  u_p = s x A_p^T    [n_out, r]  (u recomputed by the forward's down kernel)
//
// Four GEMMs share one persistent warp-specialised kernel (the forward's layout: warp 0 TMA
// producer, warp 1 single-thread tcgen05 issuer, warps 2-5 epilogue, two TMEM accumulators),
// instantiated per GEMM.  Every operand arrives through 3-D tensor maps in 64-column,
// 128-byte-swizzled boxes, either K-major (contraction along the 128-byte rows) or MN-major
// (contraction along the rows, M or N along the 128-byte rows), the two forms the attention
// kernels already use:
//   G   M = T rows,        N = 64 per part,  contract n_out    A = dy (K-major)   B = b_pad (MN)
//   DX  M = T rows,        N = K,            contract parts*n_out, then one rank block per part
//                                              A = dy, then g (K-major)        B = W, then a_pad (MN)
//   DA  M = (part, j) 128, N = K,            contract T (split)  A = g (MN)      B = x (MN)
//   DB  M = (part, n) 128, N = 64,           contract T (split)  A = dy (MN)     B = u (MN)
// DA and DB split the token contraction across CTAs and add their fp32 partial tiles into a
// zeroed accumulator with red.global.add; a last kernel rounds dA, dB to bf16 and drops the
// rank padding.
#include <algorithm>

#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace lorab {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NTHREADS = 192;
constexpr int WARP_LOAD = 0, WARP_MMA = 1;
constexpr int STAGES = 4;
constexpr int GROUP_M = 16;
constexpr uint32_t BOX64 = 64 * 128;   // a {64 elements, 64 rows} bf16 box: 8 KB
constexpr int RANK_PAD = 64;

enum Kind : int { KIND_G = 0, KIND_DX = 1, KIND_DA = 2, KIND_DB = 3 };

template <int KIND>
struct KCfg {
  static constexpr int BN = (KIND == KIND_G || KIND == KIND_DB) ? 64 : 256;
  static constexpr bool A_MN = (KIND == KIND_DA || KIND == KIND_DB);
  static constexpr bool B_MN = true;
  static constexpr bool RED = (KIND == KIND_DA || KIND == KIND_DB);
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int NBARS = 2 * STAGES + 5;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
};

struct Params {
  void* out;           // G: bf16 [parts, T, 64]; DX: bf16 [T, K]; DA: fp32 [n_mblk*128, K]; DB: fp32 [parts*n_out, 64]
  int T, K, n_out, parts;
  int m_rows;          // output rows that exist (G, DX: T; DA: parts*64; DB: parts*n_out)
  int ld;              // output row length in elements (G: 64; DX, DA: K; DB: 64)
  int n_cols;          // output columns that exist (G: 64; DX, DA: K; DB: 64)
  int n_mblk, n_nblk, n_tiles, n_splits, n_items;
  int kb_main;         // contraction blocks of a whole tile (DX: the main part, before the rank blocks)
  int kb_per_split;
  int rank_blocks;     // DX: one per part; else 0
  int rank_k16;        // DX: K=16 MMA steps of each rank block
  float out_scale;
  int* err;
};

enum Site : int { SITE_LOAD = 1, SITE_MMA = 2, SITE_EPILOGUE = 3, SITE_DRAIN = 4 };

__device__ __forceinline__ void tile_coords(int tile, int n_mblk, int n_nblk, int& mb, int& nb) {
  const int per_group = GROUP_M * n_nblk;
  const int g = tile / per_group;
  const int first = g * GROUP_M;
  const int gsize = min(GROUP_M, n_mblk - first);
  const int local = tile - g * per_group;
  mb = first + local % gsize;
  nb = local / gsize;
}

// Work item -> tile and contraction-block range [kb0, kb1).  Items of one split are
// consecutive, so the CTAs in flight share the split's token rows in L2.
__device__ __forceinline__ void item_range(const Params& p, int item, int& mb, int& nb, int& kb0, int& kb1) {
  const int split = item / p.n_tiles;
  tile_coords(item - split * p.n_tiles, p.n_mblk, p.n_nblk, mb, nb);
  kb0 = split * p.kb_per_split;
  kb1 = min(p.kb_main, kb0 + p.kb_per_split);
}

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

template <int KIND>
__device__ __forceinline__ void load_stage(uint8_t* sa, uint8_t* sb, const CUtensorMap* tA, const CUtensorMap* tB,
                                           const CUtensorMap* tA2, const CUtensorMap* tB2, const Params& p, int mb,
                                           int nb, int kb, bool rank, uint64_t* bar) {
  const int m0 = mb * BM, n0 = nb * KCfg<KIND>::BN;
  if (KIND == KIND_G) {
    tma_load_3d(sa, tA, kb * BK, m0, nb, bar);                 // dy_p rows m0.., n columns kb*64..
    tma_load_3d(sb, tB, 0, kb * BK, nb, bar);                  // b_pad_p rows (n) kb*64.., 64 rank columns
  } else if (KIND == KIND_DX) {
    if (!rank) {
      const int part = (kb * BK) / p.n_out, n = kb * BK - part * p.n_out;
      tma_load_3d(sa, tA, n, m0, part, bar);                   // dy_part rows m0.., n columns n..
#pragma unroll
      for (int i = 0; i < 4; ++i) tma_load_3d(sb + i * BOX64, tB, n0 + 64 * i, n, part, bar);   // W rows n.., K cols
    } else {
      const int part = kb;
      tma_load_3d(sa, tA2, 0, m0, part, bar);                  // g_part rows m0.., 64 rank columns
#pragma unroll
      for (int i = 0; i < 4; ++i) tma_load_3d(sb + i * BOX64, tB2, n0 + 64 * i, 0, part, bar);  // a_pad rows j
    }
  } else if (KIND == KIND_DA) {
    const int t = kb * BK;
#pragma unroll
    for (int i = 0; i < 2; ++i) tma_load_3d(sa + i * BOX64, tA, 0, t, 2 * mb + i, bar);      // g of parts 2mb, 2mb+1
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_load_3d(sb + i * BOX64, tB, n0 + 64 * i, t, 0, bar);     // x rows t.., K cols
  } else {  // KIND_DB
    const int t = kb * BK;
    const int part = m0 / p.n_out, n = m0 - part * p.n_out;
#pragma unroll
    for (int i = 0; i < 2; ++i) tma_load_3d(sa + i * BOX64, tA, n + 64 * i, t, part, bar);   // dy_part rows t.., n cols
    tma_load_3d(sb, tB, 0, t, part, bar);                                                     // u_part rows t..
  }
}

template <int KIND>
__device__ __forceinline__ void issue_stage(uint32_t d, uint32_t sa, uint32_t sb, uint32_t idesc, int nk,
                                            bool first) {
  using C = KCfg<KIND>;
  const uint64_t da = C::A_MN ? sdesc_sw128(sa, BOX64, 1024) : sdesc_sw128(sa, 16, 1024);
  const uint64_t db = sdesc_sw128(sb, BOX64, 1024);   // B is MN-major in every kind
  for (int kk = 0; kk < nk; ++kk)
    mma_ss(d, sdesc_add(da, C::A_MN ? kk * 2048 : kk * 32), sdesc_add(db, kk * 2048), idesc,
           (first && kk == 0) ? 0u : 1u);
}

template <int KIND>
__global__ void __launch_bounds__(NTHREADS, KCfg<KIND>::BN <= 64 ? 2 : 1)
    lora_bwd_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                    const __grid_constant__ CUtensorMap tA2, const __grid_constant__ CUtensorMap tB2,
                    const Params p) {
  using C = KCfg<KIND>;
  constexpr int BN = C::BN;
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
    *abort_flag = (*(volatile int*)p.err != 0) ? 1 : 0;
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
    prefetch_tmap(&tA);
    prefetch_tmap(&tB);
    if (KIND == KIND_DX) {
      prefetch_tmap(&tA2);
      prefetch_tmap(&tB2);
    }
    bool ok = true;
    int g = 0;
    for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
      int mb, nb, kb0, kb1;
      item_range(p, it, mb, nb, kb0, kb1);
      const int n_blocks = (kb1 - kb0) + p.rank_blocks;
      for (int b = 0; b < n_blocks; ++b) {
        const int s = g % STAGES;
        ok = wait_bounded(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag, p.err);
        if (!ok) break;
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        const bool rank = b >= kb1 - kb0;
        load_stage<KIND>(sa, sa + C::A_BYTES, &tA, &tB, &tA2, &tB2, p, mb, nb, rank ? b - (kb1 - kb0) : kb0 + b,
                         rank, &full[s]);
        ++g;
      }
    }
    if (!ok) {
      report_error(p.err, (K_LORA << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
    bool dok = true;
    for (int t = (g > STAGES ? g - STAGES : 0); t < g; ++t) dok &= wait_drain(&full[t % STAGES], (t / STAGES) & 1);
    if (!dok) report_error(p.err, (K_LORA << 8) | SITE_DRAIN);
  } else if (!skip && warp == WARP_MMA && lane == 0) {
    const uint32_t idesc = idesc_bf16_f32(BM, BN, C::A_MN, C::B_MN);
    const uint32_t s_base = smem_u32(smem);
    bool ok = true;
    int g = 0, lt = 0;
    for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x, ++lt) {
      int mb, nb, kb0, kb1;
      item_range(p, it, mb, nb, kb0, kb1);
      const int buf = lt & 1;
      const uint32_t d = tmem + (uint32_t)(buf * BN);
      ok = wait_bounded(&acc_empty[buf], ((lt >> 1) & 1) ^ 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      // the K loop: four K=16 MMAs per stage (a compile-time count) ...
      for (int b = 0; b < kb1 - kb0; ++b, ++g) {
        const int s = g % STAGES;
        ok = wait_bounded(&full[s], (g / STAGES) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = s_base + s * C::STAGE_BYTES;
        issue_stage<KIND>(d, sa, sa + C::A_BYTES, idesc, BK / 16, b == 0);
        mma_commit(&empty[s]);
      }
      // ... then the rank blocks (DX), ceil(r/16) MMAs each
      for (int b = 0; b < p.rank_blocks && ok; ++b, ++g) {
        const int s = g % STAGES;
        ok = wait_bounded(&full[s], (g / STAGES) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = s_base + s * C::STAGE_BYTES;
        issue_stage<KIND>(d, sa, sa + C::A_BYTES, idesc, p.rank_k16, false);
        mma_commit(&empty[s]);
      }
      if (!ok) break;
      mma_commit(&acc_full[buf]);
    }
    if (!ok) {
      report_error(p.err, (K_LORA << 8) | SITE_MMA);
      *abort_flag = 1;
    }
    mma_commit(drain);
    if (!wait_drain(drain, 0)) report_error(p.err, (K_LORA << 8) | SITE_DRAIN);
  } else if (!skip && warp >= 2) {
    const int wq = warp % 4;
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
    bool ok = true;
    int lt = 0;
    for (int it = blockIdx.x; it < p.n_items; it += gridDim.x, ++lt) {
      int mb, nb, kb0, kb1;
      item_range(p, it, mb, nb, kb0, kb1);
      const int buf = lt & 1;
      ok = wait_bounded(&acc_full[buf], (lt >> 1) & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const int grow = mb * BM + row;
      const int n0 = nb * BN;
      const bool row_ok = grow < p.m_rows;
      const uint32_t ta = lane_addr + (uint32_t)(buf * BN);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld_x32(ta + c, r);
        if (C::RED) {
          float* dst = static_cast<float*>(p.out) + (size_t)grow * p.ld + n0 + c;
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (n0 + c + e < p.n_cols) red_add_f32(dst + e, __uint_as_float(r[e]));
          }
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * p.out_scale, __uint_as_float(r[2 * e + 1]) * p.out_scale);
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                               (KIND == KIND_G ? ((size_t)nb * p.T + grow) * RANK_PAD + c
                                               : (size_t)grow * p.ld + n0 + c);
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 4; ++e)   // 8 columns per store; n_cols is a multiple of 8
              if (KIND == KIND_G || n0 + c + 8 * e < p.n_cols)
                reinterpret_cast<uint4*>(dst)[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
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

// dA [parts*r, K] = bf16(dA_acc rows p*64 + j, j < r);  dB [parts*n_out, r] = bf16(dB_acc[:, :r]).
__global__ void lora_bwd_convert_kernel(const float* __restrict__ da_acc, const float* __restrict__ db_acc,
                                        __nv_bfloat16* __restrict__ da, __nv_bfloat16* __restrict__ db, int parts,
                                        int r, int K, long long db_rows) {
  const long long na = (long long)parts * r * K;
  const long long total = na + db_rows * r;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    if (w < na) {
      const long long row = w / K;
      const int k = (int)(w - row * K);
      const int part = (int)(row / r), j = (int)(row - (long long)part * r);
      da[w] = __float2bfloat16_rn(da_acc[((size_t)part * RANK_PAD + j) * K + k]);
    } else {
      const long long e = w - na;
      const long long row = e / r;
      const int j = (int)(e - row * r);
      db[e] = __float2bfloat16_rn(db_acc[(size_t)row * RANK_PAD + j]);
    }
  }
}

template <int KIND>
cudaError_t launch(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tA2, const CUtensorMap& tB2,
                   const Params& p, int ctas, cudaStream_t st) {
  using C = KCfg<KIND>;
  cudaError_t e = cudaFuncSetAttribute(lora_bwd_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  lora_bwd_kernel<KIND><<<ctas, NTHREADS, C::SMEM_BYTES, st>>>(tA, tB, tA2, tB2, p);
  return cudaGetLastError();
}

// Splits of a token contraction so that tiles x splits fill about two waves of `slots`.
void choose_splits(Params& p, int slots) {
  int want = std::max(1, std::min(p.kb_main, (2 * slots + p.n_tiles - 1) / p.n_tiles));
  p.kb_per_split = (p.kb_main + want - 1) / want;
  p.n_splits = (p.kb_main + p.kb_per_split - 1) / p.kb_per_split;   // every split gets >= 1 block
  p.n_items = p.n_tiles * p.n_splits;
}

}  // namespace lorab

// Maps (all 3-D, 128-byte swizzle, 64-column boxes; see the table at the top of the file):
//   dy_k  {n_out, T, parts} box {64,128,1}   dy_mn {n_out, T, parts} box {64,64,1}
//   bpad  {64, n_out, parts} box {64,64,1}   w_mn  {K, n_out, parts} box {64,64,1}
//   g_k   {64, T, parts} box {64,128,1}      apad  {K, 64, parts} box {64,64,1}
//   g_mn  {64, T, parts} box {64,64,1}       x_mn  {K, T, 1} box {64,64,1}
//   u_mn  {64, T, parts} box {64,64,1}
cudaError_t launch_lora_bwd(const CUtensorMap& dy_k, const CUtensorMap& dy_mn, const CUtensorMap& bpad,
                            const CUtensorMap& w_mn, const CUtensorMap& g_k, const CUtensorMap& apad,
                            const CUtensorMap& g_mn, const CUtensorMap& x_mn, const CUtensorMap& u_mn, void* g,
                            void* dx, float* da_acc, float* db_acc, void* da, void* db, int T, int K, int n_out,
                            int parts, int r, float scaling, int n_sm, int* err, cudaStream_t st) {
  using namespace lorab;
  const int n_mblk_T = (T + BM - 1) / BM;
  const int kb_T = (T + BK - 1) / BK;
  cudaError_t e = cudaSuccess;
  if (r > 0) {  // g = bf16(s dy_p b_pad_p), [parts, T, 64]
    Params p{};
    p.out = g; p.T = T; p.K = K; p.n_out = n_out; p.parts = parts;
    p.m_rows = T; p.ld = RANK_PAD; p.n_cols = RANK_PAD;
    p.n_mblk = n_mblk_T; p.n_nblk = parts; p.n_tiles = p.n_mblk * p.n_nblk;
    p.kb_main = n_out / BK; p.kb_per_split = p.kb_main; p.n_splits = 1; p.n_items = p.n_tiles;
    p.out_scale = scaling; p.err = err;
    e = launch<KIND_G>(dy_k, bpad, dy_k, bpad, p, std::max(1, std::min(p.n_items, 2 * n_sm)), st);
    if (e != cudaSuccess) return e;
  }
  {  // dx = sum_p dy_p W_p + g_p a_pad_p, [T, K]
    Params p{};
    p.out = dx; p.T = T; p.K = K; p.n_out = n_out; p.parts = parts;
    p.m_rows = T; p.ld = K; p.n_cols = K;
    p.n_mblk = n_mblk_T; p.n_nblk = (K + 255) / 256; p.n_tiles = p.n_mblk * p.n_nblk;
    p.kb_main = parts * n_out / BK; p.kb_per_split = p.kb_main; p.n_splits = 1; p.n_items = p.n_tiles;
    p.rank_blocks = r > 0 ? parts : 0; p.rank_k16 = (r + 15) / 16;
    p.out_scale = 1.0f; p.err = err;
    e = launch<KIND_DX>(dy_k, w_mn, g_k, apad, p, std::max(1, std::min(p.n_items, n_sm)), st);
    if (e != cudaSuccess) return e;
  }
  if (r == 0) return cudaSuccess;
  const int m_da = (parts * RANK_PAD + BM - 1) / BM;
  e = cudaMemsetAsync(da_acc, 0, sizeof(float) * (size_t)m_da * BM * K, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(db_acc, 0, sizeof(float) * (size_t)parts * n_out * RANK_PAD, st);
  if (e != cudaSuccess) return e;
  {  // dA_acc += g^T x (split over tokens)
    Params p{};
    p.out = da_acc; p.T = T; p.K = K; p.n_out = n_out; p.parts = parts;
    p.m_rows = parts * RANK_PAD; p.ld = K; p.n_cols = K;
    p.n_mblk = m_da; p.n_nblk = (K + 255) / 256; p.n_tiles = p.n_mblk * p.n_nblk;
    p.kb_main = kb_T; p.err = err;
    choose_splits(p, n_sm);
    e = launch<KIND_DA>(g_mn, x_mn, g_mn, x_mn, p, std::max(1, std::min(p.n_items, n_sm)), st);
    if (e != cudaSuccess) return e;
  }
  {  // dB_acc += dy_p^T u_p (split over tokens)
    Params p{};
    p.out = db_acc; p.T = T; p.K = K; p.n_out = n_out; p.parts = parts;
    p.m_rows = parts * n_out; p.ld = RANK_PAD; p.n_cols = RANK_PAD;
    p.n_mblk = parts * n_out / BM; p.n_nblk = 1; p.n_tiles = p.n_mblk;
    p.kb_main = kb_T; p.err = err;
    choose_splits(p, 2 * n_sm);
    e = launch<KIND_DB>(dy_mn, u_mn, dy_mn, u_mn, p, std::max(1, std::min(p.n_items, 2 * n_sm)), st);
    if (e != cudaSuccess) return e;
  }
  const long long total = (long long)parts * r * K + (long long)parts * n_out * r;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 4096);
  lora_bwd_convert_kernel<<<(unsigned)blocks, threads, 0, st>>>(da_acc, db_acc, static_cast<__nv_bfloat16*>(da),
                                                                 static_cast<__nv_bfloat16*>(db), parts, r, K,
                                                                 (long long)parts * n_out);
  return cudaGetLastError();
}

}  // namespace s2
