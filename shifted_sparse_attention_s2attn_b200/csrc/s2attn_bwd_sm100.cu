// s2attn_bwd_sm100.cu -- S^2-Attn backward on B200 (sm_100a): tcgen05 MMAs with TMEM
// accumulators on 128x128 tiles, TMA loads, dQ accumulated with coalesced fp32
// reductions into L2.
//
// Gradient of grouped causal softmax attention (the pages only say the method keeps
// FlashAttention compatibility; the gradient itself follows from the forward):
//   P = exp(scale*S - lse), dV = P^T dO, dP = dO V^T, dS = P o (dP - delta),
//   dK = scale * dS^T Q, dQ = scale * dS K, with delta_t = sum_d dO[t,d] O[t,d].
// Group/shift addressing is the forward's: rolled row r of a shifted head is original
// token (r + G/2) mod N, and every 128-row tile of rolled rows is a contiguous run of
// original rows, so TMA boxes and stores address the original tensors directly.
//
// Shared memory: K, V; a 3-stage Q (+ lse) ring and a 2-stage dO (+ delta) ring; once
// dP(g) is complete dO(g) is dead, and its slot receives dS^T(g) for dK(g) and dQ(g).
//
// Work item: (b, h, group j, key tile kt of 128 keys).  The CTA keeps K and V in
// shared memory and walks the query tiles of the group that can see these keys
// (tiles kt .. G/128-1), computing per tile
//   S^T = K Q^T, dP^T = V dO^T           (M = 128 keys,  N = 128 queries)
//   dV += P^T dO (P^T from TMEM), dK += dS^T Q   (M = 128 keys, N = 128 dims)
//   dQ^T = K^T dS^T                      (M = 128 dims,  N = 128 queries)
// Every MMA has N = 128: a tcgen05 MMA with N = 64 takes as long as one with N = 128.
// Work is folded: fold (group, f) holds key tiles f and n_kt-1-f of one group, so every fold
// walks the same number of query tiles, and consecutive folds share a group: its Q, dO and
// dQ accumulator rows stay in L2.  One CTA per fold, or, when folds are short (G <= 4096:
// the CTA's fixed start-up and drain then weigh most), a persistent grid of one CTA per SM
// that takes folds blockIdx.x, blockIdx.x + gridDim.x, ... in turn.
//
// TMEM (512 columns): S^T [0,128), with P^T for queries [64w, 64w+64) written as bf16
// pairs over columns [64w, 64w+32); dP^T [128,256), which dQ^T reuses once the dS warps have read dP^T;
// dK [256,384); dV [384,512).
// MMA issue order per query tile g (one thread; tcgen05 MMAs execute in issue order):
//   dP(g) [after dQ(g-1) was drained] | dV(g) [after P(g)] | S(g+1) | dQ(g), dK(g)
// dP(g) needs only dO(g) and the drained dP/dQ columns, so it runs while the P/dS warps
// are still computing P(g), and dS(g) can start as soon as P(g) is done: the warps' P and
// dS passes follow each other with no wait for a dV + dP round trip in between.  dK(g-1)
// overlaps the dQ(g-1) drain, and S(g+1) the dS(g) work.  dS^T(g) goes into the slot of
// dO(g), which dV(g) reads: the dS warps store it only after dV(g) has completed.
//
// Warp roles (512 threads; registers rebalanced with setmaxnreg, see REGS_*):
//   warps 0-3, 4-7  P / dS, thread = key row (TMEM lane); warpgroup w takes query
//                   columns [64w, 64w+64) of each tile: P^T to TMEM (bf16), dS^T to
//                   a 128-byte-swizzled smem tile; at the end of an item warpgroup 0
//                   stores dK and warpgroup 1 stores dV
//   warps 8-11      dQ drain: thread = head dim d; dQ^T from TMEM, one coalesced
//                   fp32 reduction per (query, warp) into the global accumulator
//   warp  12        TMA producer (K, V per item; Q + lse and dO + delta through rings)
//   warp  13        MMA issuer
//   warp  14        lse converter (-lse * log2(e) in place, once per tile)
#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace bwd {

constexpr int BK = 128;  // keys per item
constexpr int BQ = 128;  // queries per tile
constexpr int HD = 128;
constexpr uint32_t BOX = 128 * 128;        // 128 rows x 128 B (64 bf16 columns)
constexpr uint32_t TILE = 2 * BOX;         // 128 rows x 128 bf16 = 32 KB
// Q (+ lse) ring of 3 tiles, dO (+ delta) ring of 2.  Once dP(g) has completed, dO(g) is
// dead and its slot receives dS^T(g) (2 boxes: queries 0-63, 64-127), read by dK(g), dQ(g).
constexpr int QSTAGES = 3, DSTAGES = 2;
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = TILE;
constexpr uint32_t OFF_Q = 2 * TILE;                   // [QSTAGES] tiles
constexpr uint32_t OFF_DO = OFF_Q + QSTAGES * TILE;    // [DSTAGES] tiles (dO, then dS^T)
constexpr uint32_t OFF_LSE = OFF_DO + DSTAGES * TILE;  // [QSTAGES] x lse[128] fp32
constexpr uint32_t OFF_DELTA = OFF_LSE + QSTAGES * BQ * 4;  // [DSTAGES] x delta[128] fp32
constexpr uint32_t OFF_BAR = OFF_DELTA + DSTAGES * BQ * 4;
constexpr int NBARS = 25;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16;  // the dynamic smem base must be 1024-byte aligned
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
constexpr int NTHREADS = 512;  // warpgroups: P/dS, P/dS, dQ drain, producer + MMA (+2 idle warps)
constexpr int WARP_DQ0 = 8, WARP_LOAD = 12, WARP_MMA = 13, WARP_CVT = 14;
// Launch: 512 threads x 128 registers = 65536.  After setmaxnreg: P/dS warpgroups keep 128,
// the dQ drain gets 168 (it holds a whole 128-column dQ^T row), producer/MMA drop to 88:
// 2 x 128 x 128 + 128 x 168 + 128 x 88 = 65536.
constexpr int REGS_DRAIN = 168, REGS_CONTROL = 88;
constexpr uint32_t PDS_WARPS = 8;

constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DK = 256, TM_DV = 384;
constexpr float LOG2E = 1.4426950408889634f;

struct Params {
  const float* lse;
  const float* delta;
  float* dq_acc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int B, N, H, G, shift_heads;
  int n_groups, n_kt;
  int persistent, n_folds;
  float scale, sl2;
  int* err;
};

enum Site : int { SITE_LOAD = 1, SITE_MMA = 2, SITE_PDS = 3, SITE_DQ = 4, SITE_DRAIN = 5, SITE_ALIGN = 6 };

// D[M=128, N=128] = A[128 x 128 dims] * B[128 x 128 dims]^T, both K-major (S^T and dP^T).
__device__ __forceinline__ void issue_kq(uint32_t d, uint32_t sa, uint32_t sb, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk / 4) * BOX + (kk % 4) * 32;
    mma_ss(d, sdesc_sw128(sa + off, 16, 1024), sdesc_sw128(sb + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// Stores one 128-column fp32 accumulator row (TMEM) as bf16, times `mul`, to global memory
// (the TMEM loads are warp-collective and always run; `store` gates the global writes).
__device__ __forceinline__ void store_row_bf16(uint32_t taddr, __nv_bfloat16* dst_row, float mul, bool store) {
#pragma unroll
  for (int c = 0; c < HD; c += 32) {
    uint32_t r[32], pk[16];
    tmem_ld_x32(taddr + c, r);
#pragma unroll
    for (int e = 0; e < 16; ++e)
      pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
    uint4* dst = reinterpret_cast<uint4*>(dst_row + c);
    if (store) {
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
    }
  }
}

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

__global__ void __launch_bounds__(NTHREADS, 1)
    s2attn_bwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                      const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;     // [3]
  uint64_t* q_empty = bars + 5;    // [3]
  uint64_t* do_full = bars + 8;    // [2]
  uint64_t* do_empty = bars + 10;  // [2]
  uint64_t* s_full = bars + 12;
  uint64_t* p_ready = bars + 13;
  uint64_t* dp_full = bars + 14;
  uint64_t* ds_ready = bars + 15;
  uint64_t* dq_full = bars + 16;
  uint64_t* dq_free = bars + 17;
  uint64_t* mma_done = bars + 18;
  uint64_t* dkv_empty = bars + 19;
  uint64_t* drain = bars + 20;
  uint64_t* lse_ready = bars + 21;  // [3] lse(g) of Q slot g%3 rewritten as -lse*log2(e)
  uint64_t* dv_done = bars + 24;    // dV(g) complete: dO(g) no longer read, its slot may take dS^T(g)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // 128-byte-swizzled TMA boxes and MMA descriptors assume 1024-byte aligned tiles.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_error(p.err, (K_BWD << 8) | SITE_ALIGN);
    return;
  }

  // ---- work items: fold (group, f) = key tiles f (heavy) and n_kt-1-f (light) ----
  const int n_fold = (p.n_kt + 1) / 2;
  struct Item {
    int kt, b, h, shift, row0;  // key tile, batch, head, roll, first rolled row of the group
  };
  // this CTA's item `it`, or kt = -1 past its last item (the persistent grid is used only
  // when every fold holds two key tiles)
  auto item_of = [&](int it) {
    Item w;
    w.kt = -1;
    int f, sub;
    if (p.persistent) {
      f = (int)blockIdx.x + (it >> 1) * (int)gridDim.x;
      sub = it & 1;
      if (f >= p.n_folds) return w;
    } else {
      f = (int)blockIdx.x;
      sub = it;
      if (sub > 1) return w;
    }
    const int fi = f % n_fold, unit = f / n_fold;
    if (sub == 1 && fi == p.n_kt - 1 - fi) return w;
    w.kt = sub ? p.n_kt - 1 - fi : fi;
    const int j = unit % p.n_groups;
    w.h = (unit / p.n_groups) % p.H;
    w.b = unit / (p.n_groups * p.H);
    w.shift = (w.h >= p.H - p.shift_heads) ? p.G / 2 : 0;
    w.row0 = j * p.G;
    return w;
  };
  // original token of a local (rolled) row of the item's group; tiles never wrap
  auto token_of = [&](const Item& w, int local_row) {
    int t = w.row0 + local_row + w.shift;
    return t >= p.N ? t - p.N : t;
  };
  auto steps_of = [&](int kt) { return p.n_kt - kt; };  // query tiles kt .. n_kt-1

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < QSTAGES; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < DSTAGES; ++s) {
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_ready, PDS_WARPS);
    mbar_init(dp_full, 1);
    mbar_init(ds_ready, PDS_WARPS);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(mma_done, 1);
    mbar_init(dkv_empty, PDS_WARPS);
    mbar_init(drain, 1);
    for (int s = 0; s < QSTAGES; ++s) mbar_init(&lse_ready[s], 1);
    mbar_init(dv_done, 1);
    *abort_flag = (*(volatile int*)p.err != 0) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == WARP_LOAD) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort_flag != 0;
  const int wg = __shfl_sync(0xffffffffu, (int)threadIdx.x / 128, 0);  // warp-uniform warpgroup index

  // setmaxnreg must dominate the code that relies on the new register budget
  if (wg == 3) {
   regs_dec<REGS_CONTROL>();
   if (!skip && warp == WARP_LOAD && lane == 0) {
    // ---------------- TMA producer ----------------
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    prefetch_tmap(&tdo);
    bool ok = true;
    int kv_loads = 0, q_armed = 0, do_armed = 0;
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.kt < 0) break;
      const int kt = w.kt, h = w.h;
      const int row_base = w.b * p.N;
      const size_t stat_base = ((size_t)w.b * p.H + w.h) * p.N;
      if (it > 0) {
        ok = wait_bounded(kv_empty, (it - 1) & 1, abort_flag, p.err);
        if (!ok) break;
      }
      const int key_tok0 = token_of(w, kt * BK);
      mbar_arrive_expect_tx(kv_full, 2 * TILE);
      for (int x = 0; x < 2; ++x) {
        tma_load_3d(smem + OFF_K + x * BOX, &tk, x * 64, h, row_base + key_tok0, kv_full);
        tma_load_3d(smem + OFF_V + x * BOX, &tv, x * 64, h, row_base + key_tok0, kv_full);
      }
      ++kv_loads;
      const int nsteps = steps_of(kt);
      for (int s = 0; s < nsteps; ++s) {
        const int g = q_armed;
        const int tok = token_of(w, (kt + s) * BQ);
        const int qs = g % QSTAGES, ds = g % DSTAGES;
        ok = wait_bounded(&q_empty[qs], ((g / QSTAGES) & 1) ^ 1, abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(&q_full[qs], TILE + BQ * 4);
        for (int x = 0; x < 2; ++x)
          tma_load_3d(smem + OFF_Q + qs * TILE + x * BOX, &tq, x * 64, h, row_base + tok, &q_full[qs]);
        bulk_load(smem + OFF_LSE + qs * BQ * 4, p.lse + stat_base + tok, BQ * 4, &q_full[qs]);
        q_armed = g + 1;
        ok = wait_bounded(&do_empty[ds], ((g / DSTAGES) & 1) ^ 1, abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(&do_full[ds], TILE + BQ * 4);
        for (int x = 0; x < 2; ++x)
          tma_load_3d(smem + OFF_DO + ds * TILE + x * BOX, &tdo, x * 64, h, row_base + tok, &do_full[ds]);
        bulk_load(smem + OFF_DELTA + ds * BQ * 4, p.delta + stat_base + tok, BQ * 4, &do_full[ds]);
        do_armed = g + 1;
      }
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
    bool dok = kv_loads == 0 || wait_drain(kv_full, (kv_loads - 1) & 1);
    for (int g = (q_armed > QSTAGES ? q_armed - QSTAGES : 0); g < q_armed; ++g)
      dok &= wait_drain(&q_full[g % QSTAGES], (g / QSTAGES) & 1);
    for (int g = (do_armed > DSTAGES ? do_armed - DSTAGES : 0); g < do_armed; ++g)
      dok &= wait_drain(&do_full[g % DSTAGES], (g / DSTAGES) & 1);
    if (!dok) report_error(p.err, (K_BWD << 8) | SITE_DRAIN);
   } else if (!skip && warp == WARP_MMA && lane == 0) {
    // ---------------- MMA issuer ----------------
    // Each group of 8 MMAs blocks this thread until it is nearly all dispatched, so a
    // barrier check that resolves only after the previous group leaves a bubble in the
    // tensor pipe.  The barriers of the next sync point are therefore probed (non-blocking)
    // before the group ahead of it is issued; a blocking wait follows only if the probe
    // found them incomplete.  Sync points per query tile g:
    //   B: dO(g) loaded, dQ^T(g-1) drained from the shared columns        -> dP(g)
    //   A: P^T(g) in TMEM (item start: previous dK/dV read out)            -> dV(g)
    //   C: Q(g+1) loaded                                                   -> S(g+1)
    //   D: dS^T(g) in smem                                                 -> dQ(g), dK(g)
    const uint32_t id_kq = idesc_bf16_f32(BK, BQ, false, false);   // S^T, dP^T
    const uint32_t id_dkv = idesc_bf16_f32(BK, HD, false, true);   // dV (A = P^T in TMEM), dK (A = dS^T)
    const uint32_t id_dq = idesc_bf16_f32(HD, BQ, true, true);     // dQ^T = K^T dS^T
    const uint32_t sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
    const uint32_t sq0 = smem_u32(smem + OFF_Q), sdo0 = smem_u32(smem + OFF_DO);
    auto ready_a = [&](int g, int it, int s, bool block) -> bool {
      const bool need_empty = s == 0 && it > 0;
      if (!block)
        return mbar_test_wait(p_ready, g & 1) && (!need_empty || mbar_test_wait(dkv_empty, (it - 1) & 1));
      return wait_bounded(p_ready, g & 1, abort_flag, p.err) &&
             (!need_empty || wait_bounded(dkv_empty, (it - 1) & 1, abort_flag, p.err));
    };
    bool ok = true;
    int g0 = 0;  // global index of the current item's first query tile
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.kt < 0) break;
      const int nsteps = steps_of(w.kt);
      // prologue: S(g0)
      ok = wait_bounded(kv_full, it & 1, abort_flag, p.err);
      if (ok) ok = wait_bounded(&q_full[g0 % QSTAGES], (g0 / QSTAGES) & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      issue_kq(tmem + TM_S, sk, sq0 + (g0 % QSTAGES) * TILE, id_kq);
      mma_commit(s_full);
      for (int s = 0; s < nsteps && ok; ++s) {
        const int g = g0 + s;
        const bool next = s + 1 < nsteps;
        const uint32_t sq = sq0 + (g % QSTAGES) * TILE;
        const uint32_t sdo = sdo0 + (g % DSTAGES) * TILE;  // dO(g), later dS^T(g)
        // ---- B: dP^T = V dO^T, into the columns dQ^T(g-1) has left
        ok = wait_bounded(&do_full[g % DSTAGES], (g / DSTAGES) & 1, abort_flag, p.err);
        if (ok && g > 0) ok = wait_bounded(dq_free, (g - 1) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        const bool pre_a = ready_a(g, it, s, false);
        issue_kq(tmem + TM_DP, sv, sdo, id_kq);
        mma_commit(dp_full);
        // ---- A: dV += P^T dO
        if (!pre_a) ok = ready_a(g, it, s, true);
        if (!ok) break;
        tc_fence_after();
        const bool pre_c = !next || mbar_test_wait(&q_full[(g + 1) % QSTAGES], ((g + 1) / QSTAGES) & 1);
        {
          const uint64_t db = sdesc_sw128(sdo, BOX, 1024);
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ts(tmem + TM_DV, tmem + TM_S + (kk / 4) * 64 + (kk % 4) * 8, sdesc_add(db, kk * 2048), id_dkv,
                   (s > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(dv_done);  // dO(g) read: the dS warps may overwrite its slot with dS^T(g)
        // ---- C: S(g+1): its columns held P^T(g), read by the dV MMAs above (issued first)
        bool pre_d;
        if (next) {
          if (!pre_c) ok = wait_bounded(&q_full[(g + 1) % QSTAGES], ((g + 1) / QSTAGES) & 1, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          pre_d = mbar_test_wait(ds_ready, g & 1);
          issue_kq(tmem + TM_S, sk, sq0 + ((g + 1) % QSTAGES) * TILE, id_kq);
          mma_commit(s_full);
        } else {
          pre_d = mbar_test_wait(ds_ready, g & 1);
        }
        // ---- D: dQ^T = K^T dS^T (into dP^T's columns, which the dS warps have read), issued
        // first so that the drain can start early; dK += dS^T Q
        if (!pre_d) ok = wait_bounded(ds_ready, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        {
          const uint64_t dds_mn = sdesc_sw128(sdo, BOX, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(tmem + TM_DP, sdesc_sw128(sk + kk * 2048, BOX, 1024), sdesc_add(dds_mn, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
          mma_commit(dq_full);
          const uint64_t dds_k = sdesc_sw128(sdo, 16, 1024), dq_mn = sdesc_sw128(sq, BOX, 1024);
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ss(tmem + TM_DK, sdesc_add(dds_k, (kk / 4) * BOX + (kk % 4) * 32), sdesc_add(dq_mn, kk * 2048), id_dkv,
                   (s > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&q_empty[g % QSTAGES]);   // Q(g) and dS^T(g) (in the dO slot) no longer read
        mma_commit(&do_empty[g % DSTAGES]);
      }
      if (!ok) break;
      mma_commit(mma_done);  // dK, dV of this item complete
      mma_commit(kv_empty);  // K, V no longer read
      g0 += nsteps;
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_MMA);
      *abort_flag = 1;
    }
    mma_commit(drain);
    if (!wait_drain(drain, 0)) report_error(p.err, (K_BWD << 8) | SITE_DRAIN);
   } else if (!skip && warp == WARP_CVT) {
    // ---------------- lse converter ----------------
    // Rewrites each tile's lse (natural log, as loaded) in place as -lse * log2(e), so that
    // the P warps form exp2(s * scale * log2(e) - lse * log2(e)) with one FFMA per element
    // instead of recomputing the 128 products in each of 256 threads.
    bool ok = true;
    int g = 0;
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.kt < 0) break;
      const int nsteps = steps_of(w.kt);
      for (int s = 0; s < nsteps; ++s, ++g) {
        ok = wait_bounded(&q_full[g % QSTAGES], (g / QSTAGES) & 1, abort_flag, p.err);
        if (!ok) break;
        float4* l4 = reinterpret_cast<float4*>(smem + OFF_LSE + (g % QSTAGES) * BQ * 4) + lane;
        float4 v = *l4;
        v.x *= -LOG2E;
        v.y *= -LOG2E;
        v.z *= -LOG2E;
        v.w *= -LOG2E;
        *l4 = v;
        fence_proxy_async_smem();  // the slot is refilled by TMA once the tile is done
        __syncwarp();
        if (lane == 0) mbar_arrive(&lse_ready[g % QSTAGES]);
      }
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
   }
  } else if (wg < 2) {
   if (!skip) {
    // ---------------- P / dS warps: thread = key row, 64 query columns per warpgroup ----------------
    const int hf = warp / 4;
    const int kr = (warp % 4) * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const float sl2 = p.sl2;
    bool ok = true;
    int g = 0;
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.kt < 0) break;
      const int kt = w.kt;
      const int nsteps = steps_of(kt);
      for (int s = 0; s < nsteps; ++s, ++g) {
        const float* lse_s = reinterpret_cast<const float*>(smem + OFF_LSE + (g % QSTAGES) * BQ * 4) + 64 * hf;
        const float* delta_s = reinterpret_cast<const float*>(smem + OFF_DELTA + (g % DSTAGES) * BQ * 4) + 64 * hf;
        ok = wait_bounded(&lse_ready[g % QSTAGES], (g / QSTAGES) & 1, abort_flag, p.err);
        if (ok) ok = wait_bounded(s_full, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        // P^T row (this warpgroup's 64 queries), kept as bf16 pairs for dS
        uint32_t pp[32];
        {
          uint32_t sr[64];
          tmem_ld_x64(lane_addr + TM_S + 64 * hf, sr);
          // on the diagonal tile (s == 0) query column c of the tile is visible iff c >= key row
          const int lim = (s == 0) ? kr - 64 * hf : -1;
          const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 l4 = reinterpret_cast<const float4*>(lse_s)[c4];  // -lse * log2(e)
            // s * scale * log2(e) - lse * log2(e), two elements per packed fp32x2 FMA
            const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1])),
                                          sl2x2, make_float2(l4.x, l4.y));
            const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                          sl2x2, make_float2(l4.z, l4.w));
            float pv[4] = {ex2_approx(x01.x), ex2_approx(x01.y), ex2_approx(x23.x), ex2_approx(x23.y)};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (4 * c4 + e < lim) pv[e] = 0.0f;
            pp[2 * c4] = pack_bf16x2(pv[0], pv[1]);
            pp[2 * c4 + 1] = pack_bf16x2(pv[2], pv[3]);
          }
        }
        // P^T goes over the first half of this warpgroup's own S^T columns (the other
        // warpgroup may still be reading its S^T columns)
        tmem_st_x32(lane_addr + TM_S + 64 * hf, pp);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);

        // dP(g) complete: dP^T(g) in TMEM (delta(g) arrived with dO(g)).  dS^T(g) goes into the
        // slot of dO(g) once dV(g) has read it (dv_done, below)
        ok = wait_bounded(&do_full[g % DSTAGES], (g / DSTAGES) & 1, abort_flag, p.err);
        if (ok) ok = wait_bounded(dp_full, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        // dS^T row kr: this warpgroup's 64 queries = box hf, one 128-byte row of 8 chunks;
        // chunk c is stored at chunk slot c ^ (kr % 8) (128-byte swizzle)
        uint8_t* dsrow = smem + OFF_DO + (g % DSTAGES) * TILE + hf * BOX + kr * 128;
        uint32_t dr0[32], dr1[32];
        tmem_ld_x32_nowait(lane_addr + TM_DP + 64 * hf, dr0);
        tmem_ld_x32_nowait(lane_addr + TM_DP + 64 * hf + 32, dr1);
        tmem_wait_ld_x32(dr0);
        tmem_mark_loaded_x32(dr1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t* dr = half == 0 ? dr0 : dr1;
          uint32_t pk[16];
          // dS = P o (dP - delta): the difference in fp32, the product in bf16x2 (keeps
          // the fp32 pipe, which slows concurrent MMAs when busy, at a low duty)
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 d4 = reinterpret_cast<const float4*>(delta_s)[8 * half + c4];
            // dP - delta, two elements per packed fp32x2 add
            const float2 g01 = __fadd2_rn(make_float2(__uint_as_float(dr[4 * c4]), __uint_as_float(dr[4 * c4 + 1])),
                                          make_float2(-d4.x, -d4.y));
            const float2 g23 = __fadd2_rn(make_float2(__uint_as_float(dr[4 * c4 + 2]), __uint_as_float(dr[4 * c4 + 3])),
                                          make_float2(-d4.z, -d4.w));
            pk[2 * c4] = mul_bf16x2(pp[16 * half + 2 * c4], pack_bf16x2(g01.x, g01.y));
            pk[2 * c4 + 1] = mul_bf16x2(pp[16 * half + 2 * c4 + 1], pack_bf16x2(g23.x, g23.y));
          }
          if (half == 0) ok = wait_bounded(dv_done, g & 1, abort_flag, p.err);  // dO(g) read by dV(g)
          if (ok) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(dsrow + (((4 * half + c) ^ (kr & 7)) * 16)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
        if (!ok) break;
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_ready);
      }
      if (ok) ok = wait_bounded(mma_done, it & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const int tok = token_of(w, kt * BK) + kr;
      const size_t row_first = ((size_t)(w.b * p.N + tok) * p.H + w.h) * HD;
      const bool row_ok = in_bounds(row_first, HD, (size_t)p.B * p.N * p.H * HD, p.err, (K_BWD << 8) | SITE_PDS);
      if (hf == 0)
        store_row_bf16(lane_addr + TM_DK, p.dk + row_first, p.scale, row_ok);
      else
        store_row_bf16(lane_addr + TM_DV, p.dv + row_first, 1.0f, row_ok);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkv_empty);
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_PDS);
      *abort_flag = 1;
    }
   }
  } else {
   regs_inc<REGS_DRAIN>();
   if (!skip) {
    // ---------------- dQ drain: thread = head dim d ----------------
    const int d = (warp - WARP_DQ0) * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    bool ok = true;
    int g = 0;
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.kt < 0) break;
      const int kt = w.kt;
      const int nsteps = steps_of(kt);
      for (int s = 0; s < nsteps; ++s, ++g) {
        ok = wait_bounded(dq_full, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        // query q of this tile -> dq_acc[b, tok0 + q, h, d]; a warp covers 32 consecutive d (128 B)
        float* dst = p.dq_acc + ((size_t)(w.b * p.N + token_of(w, (kt + s) * BQ)) * p.H + w.h) * HD + d;
        const size_t row_stride = (size_t)p.H * HD;
#ifdef S2ATTN_DEBUG
        // the 128 queries of the tile: dst + q * row_stride for q < 128 (the release build keeps
        // this path free of the check: the drain's registers are at their limit)
        const bool dq_ok = in_bounds((size_t)(dst - p.dq_acc), (BQ - 1) * row_stride + 1,
                                     (size_t)p.B * p.N * p.H * HD, p.err, (K_BWD << 8) | SITE_DQ);
#else
        constexpr bool dq_ok = true;
#endif
        uint32_t r0[64], r1[64];
        tmem_ld_x64(lane_addr + TM_DP, r0);
        tmem_ld_x64(lane_addr + TM_DP + 64, r1);
        // all of dQ^T(g) is in registers: release the columns before the reductions
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);
        // one running address (consecutive queries are row_stride floats apart)
        if (dq_ok) {
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            red_add_f32(dst, __uint_as_float(r0[e]));
            dst += row_stride;
          }
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            red_add_f32(dst, __uint_as_float(r1[e]));
            dst += row_stride;
          }
        }
      }
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_DQ);
      *abort_flag = 1;
    }
   }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_LOAD) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd

cudaError_t launch_bwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const float* lse, const float* delta, float* dq_acc, void* dk,
                             void* dv, const Shape& s, int n_sm, int* err, cudaStream_t st) {
  bwd::Params p;
  p.lse = lse;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = s.B;
  p.N = s.N;
  p.H = s.H;
  p.G = s.G;
  p.shift_heads = s.shift_heads;
  p.n_groups = s.N / s.G;
  p.n_kt = s.G / bwd::BK;
  p.scale = (float)(1.0 / sqrt((double)s.D));
  p.sl2 = (float)(1.4426950408889634 / sqrt((double)s.D));
  p.err = err;
  const long long folds = (long long)((p.n_kt + 1) / 2) * s.B * s.H * p.n_groups;
  if (folds <= 0 || folds > 0x7fffffffLL || n_sm <= 0) return cudaErrorInvalidValue;
  // Persistent only for short folds: measured (same-run A/B) +7 % at G = 2048, N = 8k, +4.5 % at
  // G = 2048, N = 64k, +1.4-1.8 % at G = 4096 (N = 16k, 32k); neutral at G = 8192 and 2 % slower at
  // G = 25600, where the block scheduler's dynamic assignment of equal CTAs balances better than a
  // fixed stride.
  p.n_folds = (int)folds;
  p.persistent = (p.n_kt % 2 == 0 && p.n_kt <= 32) ? 1 : 0;
  const long long grid = p.persistent ? (folds < n_sm ? folds : n_sm) : folds;
  cudaError_t e = cudaFuncSetAttribute(bwd::s2attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bwd::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  bwd::s2attn_bwd_kernel<<<(unsigned)grid, bwd::NTHREADS, bwd::SMEM_BYTES, st>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

}  // namespace s2
