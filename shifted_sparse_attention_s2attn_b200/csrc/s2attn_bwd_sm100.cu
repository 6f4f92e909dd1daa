// s2attn_bwd_sm100.cu -- S^2-Attn backward on B200 (sm_100a): tcgen05 MMAs with TMEM
// accumulators, TMA loads, dQ accumulated with TMA bulk reduce-add.
//
// Gradient of grouped causal softmax attention (the pages only say the method keeps
// FlashAttention compatibility; the gradient itself follows from the forward):
//   P = exp(scale*S - lse), dV = P^T dO, dP = dO V^T, dS = P o (dP - delta),
//   dK = scale * dS^T Q, dQ = scale * dS K, with delta_t = sum_d dO[t,d] O[t,d].
// Group/shift addressing is the forward's: rolled row r of a shifted head is original
// token (r + G/2) mod N, and every tile of rolled rows is a contiguous run of
// original rows, so TMA boxes and epilogue stores address the original tensors.
//
// CTA work item: (b, h, group j, key tile kt of 128 keys).  The CTA keeps K and V in
// shared memory and walks the query rows of the group that can see these keys
// (local rows >= 128*kt) in steps of 64, computing per step
//   S^T = K Q^T, dP^T = V dO^T                    (M=128 keys, N=64 queries)
//   dV += P^T dO  (P^T from TMEM), dK += dS^T Q   (M=128 keys, N=128 dims)
//   dQ^T = K^T dS^T                               (M=128 dims, N=64 queries)
// dQ^T leaves TMEM through shared memory and is added into an fp32 accumulator in
// global memory by one TMA reduce-add per step.  Each CTA runs two key tiles of one
// group, kt and n_kt-1-kt, so every CTA walks the same number of query steps, and
// consecutive CTAs share a group: its Q, dO and dQ accumulator rows stay in L2.
//
// Warp roles (320 threads):
//   warps 0-3  P / dS: thread = key row (TMEM lanes); writes P^T into TMEM and dS^T
//              (bf16, 128-byte swizzled) into shared memory; final dK, dV stores
//   warps 4-7  dQ drain: thread = head dim d; TMEM -> smem fp32 -> TMA reduce-add
//   warp  8    TMA producer (K, V once; Q, dO, lse, delta through a 2-stage ring)
//   warp  9    MMA issuer
// TMEM: S^T/P^T [0,64), dP^T [64,128), dQ^T [128,192), dK [256,384), dV [384,512).
#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace bwd {

constexpr int BK = 128;  // keys per CTA
constexpr int BQ = 64;   // queries per step
constexpr int HD = 128;
constexpr uint32_t KBOX = 128 * 128;        // 128 rows x 128 B
constexpr uint32_t KTILE = 2 * KBOX;        // 32 KB
constexpr uint32_t QBOX = 64 * 128;         // 64 rows x 128 B
constexpr uint32_t QTILE = 2 * QBOX;        // 16 KB
constexpr int QSTAGES = 2;
constexpr uint32_t ST_Q = 0, ST_DO = QTILE, ST_LSE = 2 * QTILE, ST_DELTA = 2 * QTILE + 256;
constexpr uint32_t STAGE_BYTES = 2 * QTILE + 1024;
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = KTILE;
constexpr uint32_t OFF_STAGE = 2 * KTILE;
constexpr uint32_t OFF_DS = OFF_STAGE + QSTAGES * STAGE_BYTES;
constexpr uint32_t DS_BYTES = BK * 128;     // 128 key rows x 64 bf16
constexpr uint32_t OFF_DQ = OFF_DS + 2 * DS_BYTES;
constexpr uint32_t DQ_BYTES = BQ * HD * 4;  // fp32 staging tile
constexpr uint32_t OFF_BAR = OFF_DQ + DQ_BYTES;
// kv_full, q_full[2], q_empty[2], s_full, dp_full, p_ready, ds_ready, ds_free[2], dq_full, dq_free,
// mma_done, drain, kv_empty, dkv_empty
constexpr int NBARS = 17;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int NTHREADS = 320;
constexpr int WARP_LOAD = 8, WARP_MMA = 9;

constexpr uint32_t TM_S = 0, TM_DP = 64, TM_DQ = 128, TM_DK = 256, TM_DV = 384;
constexpr float LOG2E = 1.4426950408889634f;

struct Params {
  const float* lse;
  const float* delta;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int B, N, H, G, shift_heads;
  int n_groups, n_kt;
  float scale, sl2;
  int* err;
};

enum Site : int { SITE_LOAD = 1, SITE_MMA = 2, SITE_PDS = 3, SITE_DQ = 4, SITE_DRAIN = 5 };

// D[M=128, N=64] = A[128 x 128 dims] * B[64 x 128 dims]^T, both K-major (S^T and dP^T).
__device__ __forceinline__ void issue_kq(uint32_t d, uint32_t sa, uint32_t sb, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t oa = (kk / 4) * KBOX + (kk % 4) * 32;
    const uint32_t ob = (kk / 4) * QBOX + (kk % 4) * 32;
    mma_ss(d, sdesc_sw128(sa + oa, 16, 1024), sdesc_sw128(sb + ob, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    s2attn_bwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                      const __grid_constant__ CUtensorMap tdq, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = bars + 3;
  uint64_t* s_full = bars + 5;
  uint64_t* dp_full = bars + 6;
  uint64_t* p_ready = bars + 7;
  uint64_t* ds_ready = bars + 8;
  uint64_t* ds_free = bars + 9;
  uint64_t* dq_full = bars + 11;
  uint64_t* dq_free = bars + 12;
  uint64_t* mma_done = bars + 13;
  uint64_t* drain = bars + 14;
  uint64_t* kv_empty = bars + 15;
  uint64_t* dkv_empty = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work items: one group (b, h, j); key tiles kt0 (heavy) and n_kt-1-kt0 (light) ----
  const int n_fold = (p.n_kt + 1) / 2;
  const int unit = (int)(blockIdx.x / n_fold);
  const int fi = (int)(blockIdx.x % n_fold);
  const int j = unit % p.n_groups;
  const int h = (unit / p.n_groups) % p.H;
  const int b = unit / (p.n_groups * p.H);
  int kts[2];
  int n_items = 0;
  kts[n_items++] = fi;
  if (fi != p.n_kt - 1 - fi) kts[n_items++] = p.n_kt - 1 - fi;
  const int shift = (h >= p.H - p.shift_heads) ? p.G / 2 : 0;
  const int group_row0 = j * p.G;
  auto token_of = [&](int local_row) {  // original token of a local (rolled) row; tiles never wrap
    int t = group_row0 + local_row + shift;
    return t >= p.N ? t - p.N : t;
  };
  auto steps_of = [&](int kt) { return p.G / BQ - 2 * kt; };  // query steps of 64 rows: rows 128*kt .. G-1

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < QSTAGES; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&ds_free[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 4);
    mbar_init(ds_ready, 4);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(mma_done, 1);
    mbar_init(dkv_empty, 4);
    mbar_init(drain, 1);
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

  if (!skip && warp == WARP_LOAD && lane == 0) {
    // ---------------- TMA producer ----------------
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    prefetch_tmap(&tdo);
    bool ok = true;
    const int row_base = b * p.N;
    const size_t stat_base = ((size_t)b * p.H + h) * p.N;
    int kv_loads = 0, q_armed = 0;
    for (int it = 0; it < n_items && ok; ++it) {
      const int kt = kts[it];
      if (it > 0) {
        ok = wait_bounded(kv_empty, (it - 1) & 1, abort_flag, p.err);
        if (!ok) break;
      }
      const int key_tok0 = token_of(kt * BK);
      mbar_arrive_expect_tx(kv_full, 2 * KTILE);
      for (int x = 0; x < 2; ++x) {
        tma_load_3d(smem + OFF_K + x * KBOX, &tk, x * 64, h, row_base + key_tok0, kv_full);
        tma_load_3d(smem + OFF_V + x * KBOX, &tv, x * 64, h, row_base + key_tok0, kv_full);
      }
      ++kv_loads;
      const int nsteps = steps_of(kt);
      for (int s = 0; s < nsteps; ++s) {
        const int g = q_armed;
        const int st = g % QSTAGES;
        ok = wait_bounded(&q_empty[st], ((g / QSTAGES) & 1) ^ 1, abort_flag, p.err);
        if (!ok) break;
        uint8_t* stage = smem + OFF_STAGE + st * STAGE_BYTES;
        const int tok = token_of((2 * kt + s) * BQ);
        mbar_arrive_expect_tx(&q_full[st], 2 * QTILE + 512);
        for (int x = 0; x < 2; ++x) {
          tma_load_3d(stage + ST_Q + x * QBOX, &tq, x * 64, h, row_base + tok, &q_full[st]);
          tma_load_3d(stage + ST_DO + x * QBOX, &tdo, x * 64, h, row_base + tok, &q_full[st]);
        }
        bulk_load(stage + ST_LSE, p.lse + stat_base + tok, 256, &q_full[st]);
        bulk_load(stage + ST_DELTA, p.delta + stat_base + tok, 256, &q_full[st]);
        q_armed = g + 1;
      }
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
    bool dok = kv_loads == 0 || wait_drain(kv_full, (kv_loads - 1) & 1);
    for (int g = (q_armed > QSTAGES ? q_armed - QSTAGES : 0); g < q_armed; ++g)
      dok &= wait_drain(&q_full[g % QSTAGES], (g / QSTAGES) & 1);
    if (!dok) report_error(p.err, (K_BWD << 8) | SITE_DRAIN);
  } else if (!skip && warp == WARP_MMA && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t id_kq = idesc_bf16_f32(BK, BQ, false, false);   // S^T, dP^T
    const uint32_t id_dkv = idesc_bf16_f32(BK, HD, false, true);   // dV (A in TMEM), dK (A = dS^T smem)
    const uint32_t id_dq = idesc_bf16_f32(HD, BQ, true, true);     // dQ^T = K^T dS^T
    const uint32_t sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
    const uint32_t sstage = smem_u32(smem + OFF_STAGE), sds = smem_u32(smem + OFF_DS);
    bool ok = true;
    int g0 = 0;  // global index of the current item's first query step
    for (int it = 0; it < n_items && ok; ++it) {
      const int nsteps = steps_of(kts[it]);
      ok = wait_bounded(kv_full, it & 1, abort_flag, p.err);
      if (ok) ok = wait_bounded(&q_full[g0 % QSTAGES], (g0 / QSTAGES) & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      issue_kq(tmem + TM_S, sk, sstage + (g0 % QSTAGES) * STAGE_BYTES + ST_Q, id_kq);
      mma_commit(s_full);
      issue_kq(tmem + TM_DP, sv, sstage + (g0 % QSTAGES) * STAGE_BYTES + ST_DO, id_kq);
      mma_commit(dp_full);
      for (int s = 0; s < nsteps && ok; ++s) {
        const int g = g0 + s;
        const int st = g % QSTAGES;
        const uint32_t sq = sstage + st * STAGE_BYTES + ST_Q, sdo = sstage + st * STAGE_BYTES + ST_DO;
        const uint32_t sdst = sds + st * DS_BYTES;
        // dV += P^T dO
        ok = wait_bounded(p_ready, g & 1, abort_flag, p.err);
        if (ok && s == 0 && it > 0) ok = wait_bounded(dkv_empty, (it - 1) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_ts(tmem + TM_DV, tmem + TM_S + kk * 8, sdesc_sw128(sdo + kk * 2048, QBOX, 1024), id_dkv,
                 (s > 0 || kk > 0) ? 1u : 0u);
        // next S^T (its columns held P^T, which the dV MMAs above read first: in-order issue)
        if (s + 1 < nsteps) {
          const int st1 = (g + 1) % QSTAGES;
          ok = wait_bounded(&q_full[st1], ((g + 1) / QSTAGES) & 1, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          issue_kq(tmem + TM_S, sk, sstage + st1 * STAGE_BYTES + ST_Q, id_kq);
          mma_commit(s_full);
        }
        // dK += dS^T Q ; dQ^T = K^T dS^T
        ok = wait_bounded(ds_ready, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_ss(tmem + TM_DK, sdesc_sw128(sdst + kk * 32, 16, 1024), sdesc_sw128(sq + kk * 2048, QBOX, 1024),
                 id_dkv, (s > 0 || kk > 0) ? 1u : 0u);
        if (g > 0) {
          ok = wait_bounded(dq_free, (g - 1) & 1, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_ss(tmem + TM_DQ, sdesc_sw128(sk + kk * 2048, KBOX, 1024), sdesc_sw128(sdst + kk * 2048, QBOX, 1024),
                 id_dq, kk > 0 ? 1u : 0u);
        mma_commit(dq_full);
        mma_commit(&ds_free[st]);
        mma_commit(&q_empty[st]);
        // next dP^T (the P/dS warps finished reading dP^T before signalling ds_ready)
        if (s + 1 < nsteps) {
          const int st1 = (g + 1) % QSTAGES;
          issue_kq(tmem + TM_DP, sv, sstage + st1 * STAGE_BYTES + ST_DO, id_kq);
          mma_commit(dp_full);
        }
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
  } else if (!skip && warp < 4) {
    // ---------------- P / dS warps: thread = key row ----------------
    const int kr = warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = p.sl2;
    bool ok = true;
    int g = 0;
    for (int it = 0; it < n_items && ok; ++it) {
      const int kt = kts[it];
      const int nsteps = steps_of(kt);
      const int key_local = kt * BK + kr;
      for (int s = 0; s < nsteps; ++s, ++g) {
        const int st = g % QSTAGES;
        const int q_local0 = (2 * kt + s) * BQ;
        const float* lse_s = reinterpret_cast<const float*>(smem + OFF_STAGE + st * STAGE_BYTES + ST_LSE);
        const float* delta_s = reinterpret_cast<const float*>(smem + OFF_STAGE + st * STAGE_BYTES + ST_DELTA);
        ok = wait_bounded(&q_full[st], (g / QSTAGES) & 1, abort_flag, p.err);
        if (ok) ok = wait_bounded(s_full, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        float pr[64];
        {
          uint32_t sr[64];
          tmem_ld_x64(lane_addr + TM_S, sr);
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float e = ex2_approx(__uint_as_float(sr[c]) * sl2 - lse_s[c] * LOG2E);
            pr[c] = (key_local > q_local0 + c) ? 0.0f : e;  // causal: key after query -> masked
          }
        }
        {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
          tmem_st_x32(lane_addr + TM_S, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);

        ok = wait_bounded(dp_full, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        uint32_t pk[32];
        {
          uint32_t dr[64];
          tmem_ld_x64(lane_addr + TM_DP, dr);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float d0 = pr[2 * c] * (__uint_as_float(dr[2 * c]) - delta_s[2 * c]);
            const float d1 = pr[2 * c + 1] * (__uint_as_float(dr[2 * c + 1]) - delta_s[2 * c + 1]);
            pk[c] = pack_bf16x2(d0, d1);
          }
        }
        tc_fence_before();
        if (g >= QSTAGES) {
          ok = wait_bounded(&ds_free[st], ((g - QSTAGES) / QSTAGES) & 1, abort_flag, p.err);
          if (!ok) break;
        }
        // dS^T row kr: 64 bf16 = 8 chunks of 16 B, chunk c stored at chunk slot c ^ (kr % 8)
        uint8_t* dsrow = smem + OFF_DS + st * DS_BYTES + kr * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(dsrow + ((c ^ (kr & 7)) * 16)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_ready);
      }
      if (ok) ok = wait_bounded(mma_done, it & 1, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const int tok = token_of(kt * BK) + kr;
      __nv_bfloat16* dkrow = p.dk + ((size_t)(b * p.N + tok) * p.H + h) * HD;
      __nv_bfloat16* dvrow = p.dv + ((size_t)(b * p.N + tok) * p.H + h) * HD;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t r[32], pk[16];
        tmem_ld_x32(lane_addr + TM_DK + c, r);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * p.scale, __uint_as_float(r[2 * e + 1]) * p.scale);
        uint4* dst = reinterpret_cast<uint4*>(dkrow + c);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        tmem_ld_x32(lane_addr + TM_DV + c, r);
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
        dst = reinterpret_cast<uint4*>(dvrow + c);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkv_empty);
    }
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_PDS);
      *abort_flag = 1;
    }
  } else if (!skip && warp >= 4 && warp < 8) {
    // ---------------- dQ drain: thread = head dim ----------------
    const int d = (warp - 4) * 32 + lane;
    const bool leader = (warp == 4 && lane == 0);
    const uint32_t lane_addr = tmem + ((uint32_t)((warp - 4) * 32) << 16);
    float* stage = reinterpret_cast<float*>(smem + OFF_DQ);
    bool ok = true;
    int g = 0;
    for (int it = 0; it < n_items && ok; ++it) {
      const int kt = kts[it];
      const int nsteps = steps_of(kt);
      for (int s = 0; s < nsteps; ++s, ++g) {
        ok = wait_bounded(dq_full, g & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        uint32_t r[64];
        tmem_ld_x64(lane_addr + TM_DQ, r);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);
        if (leader && g > 0) bulk_wait_group_read0();  // previous reduce finished reading the staging tile
        named_bar_sync(1, 128);
#pragma unroll
        for (int c = 0; c < BQ; ++c) stage[c * HD + d] = __uint_as_float(r[c]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader) {
          tma_reduce_add_3d(&tdq, stage, 0, h, b * p.N + token_of((2 * kt + s) * BQ));
          bulk_commit_group();
        }
      }
    }
    if (leader) bulk_wait_group0();
    if (!ok) {
      report_error(p.err, (K_BWD << 8) | SITE_DQ);
      *abort_flag = 1;
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

cudaError_t launch_bwd_sm100(const CUtensorMap& tq64, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo64, const CUtensorMap& tdq_acc, const float* lse,
                             const float* delta, void* dk, void* dv, const Shape& s, int* err, cudaStream_t st) {
  bwd::Params p;
  p.lse = lse;
  p.delta = delta;
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
  const long long grid = (long long)((p.n_kt + 1) / 2) * s.B * s.H * p.n_groups;
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd::s2attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bwd::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  bwd::s2attn_bwd_kernel<<<(unsigned)grid, bwd::NTHREADS, bwd::SMEM_BYTES, st>>>(tq64, tk, tv, tdo64, tdq_acc, p);
  return cudaGetLastError();
}

}  // namespace s2
