// s2attn_fwd_sm100.cu -- S^2-Attn forward on B200 (sm_100a): tcgen05 MMAs with
// TMEM accumulators, TMA tile loads, warp-specialised CTA.
//
// Method (LongLoRA pages: "LongLoRA paper notes" section 3.3; nearauto.com article,
// "shift short attention" steps (1) and (2)): for every head, cut the sequence into
// groups of G tokens and run causal softmax attention inside each group; heads
// h >= H - shift_heads first see the sequence rolled by G/2.  Here the roll and the
// token->batch regrouping are pure address arithmetic: rolled row r of a shifted
// head is original token (r + G/2) mod N, and because G/2 and N are multiples of the
// 128-row tile, every 128-row tile of rolled rows is a contiguous run of original
// rows.  Each TMA box therefore loads straight from the original [B,N,H,D] tensor
// and each output row is stored straight back to its original token: no rolled copy
// of Q/K/V/O ever exists.
//
// Work item: (batch b, head h, group j, pair m) -> the two query tiles 2m and 2m+1 of
// the group (128 rows each), which share every K/V tile they load.  Only the causal
// lower triangle is visited: query tile qt needs key tiles 0..qt, and only tile qt
// (the diagonal) is masked.  Pair m costs 2m+2 K/V steps.  Two schedules:
//   fold:  one CTA per (group, f) runs pair n_pairs-1-f and then pair f, so every CTA
//          does the same work; consecutive CTAs share a group, which keeps that
//          group's K/V resident in L2;
//   snake: a persistent grid of P CTAs (one per SM) over the list of all pairs,
//          heaviest first; in round r CTA c takes item r*P + c (r even) or
//          r*P + P-1-c (r odd).  This evens out unequal pairs when the fold leaves a
//          large partial last wave, but concurrent CTAs work on different groups, so
//          it is chosen only when all of K and V fits in L2.
//
// Warp roles (320 threads):
//   warps 0-3  softmax for query tile 0 (thread = row; TMEM lanes 0..127)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer (Q once; K and V through 2-stage rings); TMEM owner
//   warp  9    MMA issuer: S_i = Q_i K^T (SS), O_i += P_i V (TS: P read from TMEM)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P_i is
// written as bf16 pairs over the first 64 columns of S_i.  tcgen05 MMAs issued by
// one thread execute in issue order, so S_i(t+1) may be issued right after the
// PV_i(t) that still reads P_i(t) from the same columns.
//
// Softmax: online, base 2, with a lazy rescale -- the running max is only moved (and
// O rescaled) when a row's max grows by more than 2^8, so P <= 256 and most tiles
// skip the O round trip through registers.
#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace fwd {

constexpr int BM = 128;                      // query rows per tile
constexpr int BN = 128;                      // keys per tile
constexpr int HD = 128;                      // head dim
constexpr int NBOX = HD / 64;                // 64-column (128-byte) swizzle boxes per row
constexpr uint32_t BOX_BYTES = 128 * 128;    // 128 rows x 128 B
constexpr uint32_t TILE_BYTES = NBOX * BOX_BYTES;
constexpr int STAGES = 2;
constexpr int NTHREADS = 320;
constexpr int WARP_LOAD = 8, WARP_MMA = 9;

constexpr uint32_t OFF_Q0 = 0;
constexpr uint32_t OFF_Q1 = OFF_Q0 + TILE_BYTES;
constexpr uint32_t OFF_K = OFF_Q1 + TILE_BYTES;
constexpr uint32_t OFF_V = OFF_K + STAGES * TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_V + STAGES * TILE_BYTES;
// barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_ready[2], o_final[2], drain,
// q_empty, o_empty[2]
constexpr int NBARS = 19;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024 B

// TMEM column of S_i / O_i for query tile i
__device__ __forceinline__ uint32_t tm_s(int i) { return i == 0 ? 0u : 128u; }
__device__ __forceinline__ uint32_t tm_o(int i) { return i == 0 ? 256u : 384u; }
constexpr float LN2 = 0.69314718055994530942f;

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int B, N, H, G, shift_heads;
  int n_qt, n_pairs, n_groups;
  int snake;  // 1: persistent snake schedule, 0: folded pairs (one CTA per fold)
  float sl2;  // softmax scale * log2(e)
  int* err;
};

enum Site : int { SITE_LOAD = 1, SITE_MMA = 2, SITE_SOFTMAX = 3, SITE_EPILOGUE = 4, SITE_DRAIN = 5 };

// Descriptors are built once per GEMM and stepped by constant offsets, so each MMA
// costs the issuing thread (which shares its SM sub-partition with softmax warps) only
// a few instructions.
__device__ __forceinline__ void issue_s(uint32_t d, uint32_t sq, uint32_t sk, uint32_t idesc) {
  const uint64_t dq = sdesc_sw128(sq, 16, 1024), dk = sdesc_sw128(sk, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk / 4) * BOX_BYTES + (kk % 4) * 32;
    mma_ss(d, sdesc_add(dq, off), sdesc_add(dk, off), idesc, kk > 0 ? 1u : 0u);
  }
}

__device__ __forceinline__ void issue_pv(uint32_t d, uint32_t tp, uint32_t sv, uint32_t idesc, bool first) {
  // B = V^T viewed MN-major: 16 key rows (2 KB) per k-step, 64-column boxes BOX_BYTES apart.
  const uint64_t dv = sdesc_sw128(sv, BOX_BYTES, 1024);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) mma_ts(d, tp + kk * 8, sdesc_add(dv, kk * 2048), idesc, (first && kk == 0) ? 0u : 1u);
}

// P = exp2(s * sl2 - m) for one 128-column row of S, packed to bf16 pairs and written
// over the first 64 TMEM columns of S.  Columns c > lim are masked (diagonal tile).
// Returns the row sum of the fp32 P values (eight independent partial sums).  The
// scale-and-shift uses the packed fp32x2 FMA (two elements per instruction): one softmax
// warp per SM sub-partition is active at a time, so the row is issue-bound around its
// 128 MUFU exponentials.
template <bool MASK>
__device__ __forceinline__ float softmax_p_row(const uint32_t (&s0)[64], const uint32_t (&s1)[64], int lim,
                                               float sl2, float neg_m, uint32_t t_s) {
  const float2 scale2 = make_float2(sl2, sl2), shift2 = make_float2(neg_m, neg_m);
  float2 sp[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) sp[e] = make_float2(0.f, 0.f);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t(&sr)[64] = h == 0 ? s0 : s1;
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), scale2, shift2);
      float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
      if (MASK) {
        p0 = 64 * h + 2 * c <= lim ? p0 : 0.f;
        p1 = 64 * h + 2 * c + 1 <= lim ? p1 : 0.f;
      }
      sp[c % 4].x += p0; sp[c % 4].y += p1;
      pk[c] = pack_bf16x2(p0, p1);
    }
    tmem_st_x32(t_s + 32 * h, pk);
  }
  return ((sp[0].x + sp[1].x) + (sp[2].x + sp[3].x)) + ((sp[0].y + sp[1].y) + (sp[2].y + sp[3].y));
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__global__ void __launch_bounds__(NTHREADS, 1)
    s2attn_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 3;
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 7;
  uint64_t* s_full = bars + 9;
  uint64_t* p_ready = bars + 11;
  uint64_t* o_final = bars + 13;
  uint64_t* drain = bars + 15;
  uint64_t* q_empty = bars + 16;
  uint64_t* o_empty = bars + 17;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work items ----
  const int n_units = p.B * p.H * p.n_groups;
  const int n_total = p.n_pairs * n_units;
  const int n_fold = (p.n_pairs + 1) / 2;
  struct Item {
    int m, b, h, shift, row0;  // pair, batch, head, roll, first rolled row of the group
  };
  // this CTA's item r, or m = -1 past its last item
  const int cta = (int)blockIdx.x;
  auto item_of = [&](int r) {
    Item w;
    w.m = -1;
    int unit;
    if (p.snake) {
      const int P = (int)gridDim.x;
      const long long i = (long long)r * P + ((r & 1) ? P - 1 - cta : cta);
      if (i >= n_total) return w;
      unit = (int)(i % n_units);
      w.m = p.n_pairs - 1 - (int)(i / n_units);
    } else {
      const int fi = cta % n_fold;
      unit = cta / n_fold;
      if (r > 1 || (r == 1 && fi == p.n_pairs - 1 - fi)) return w;
      w.m = r == 0 ? p.n_pairs - 1 - fi : fi;
    }
    const int j = unit % p.n_groups;
    w.h = (unit / p.n_groups) % p.H;
    w.b = unit / (p.n_groups * p.H);
    w.shift = (w.h >= p.H - p.shift_heads) ? p.G / 2 : 0;
    w.row0 = j * p.G;
    return w;
  };
  // first original token of the 128-row tile `tile` of the item's group (tiles never wrap)
  auto tile_token0 = [&](const Item& w, int tile) {
    int t = w.row0 + tile * BM + w.shift;
    return t >= p.N ? t - p.N : t;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 4);
      mbar_init(&o_final[i], 1);
      mbar_init(&o_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = (*(volatile int*)p.err != 0) ? 1 : 0;  // an earlier CTA failed: skip the work
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
    bool ok = true;
    int q_loads = 0, kv = 0, k_armed = 0, v_armed = 0;  // loads issued
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.m < 0) break;
      const int row_base = w.b * p.N, h = w.h;
      const int qa = 2 * w.m, qb = qa + 1;
      const bool has_b = qb < p.n_qt;
      const int nkv = (has_b ? qb : qa) + 1;
      if (it > 0) {
        ok = wait_bounded(q_empty, (it - 1) & 1, abort_flag, p.err);
        if (!ok) break;
      }
      mbar_arrive_expect_tx(q_full, (has_b ? 2u : 1u) * TILE_BYTES);
      for (int x = 0; x < NBOX; ++x) {
        tma_load_3d(smem + OFF_Q0 + x * BOX_BYTES, &tq, x * 64, h, row_base + tile_token0(w, qa), q_full);
        if (has_b) tma_load_3d(smem + OFF_Q1 + x * BOX_BYTES, &tq, x * 64, h, row_base + tile_token0(w, qb), q_full);
      }
      ++q_loads;
      for (int t = 0; t < nkv; ++t, ++kv) {
        const int st = kv % STAGES;
        const uint32_t ph = (kv / STAGES) & 1;
        const int row = row_base + tile_token0(w, t);
        ok = wait_bounded(&k_empty[st], ph ^ 1, abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        for (int x = 0; x < NBOX; ++x)
          tma_load_3d(smem + OFF_K + st * TILE_BYTES + x * BOX_BYTES, &tk, x * 64, h, row, &k_full[st]);
        k_armed = kv + 1;
        ok = wait_bounded(&v_empty[st], ph ^ 1, abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        for (int x = 0; x < NBOX; ++x)
          tma_load_3d(smem + OFF_V + st * TILE_BYTES + x * BOX_BYTES, &tv, x * 64, h, row, &v_full[st]);
        v_armed = kv + 1;
      }
    }
    if (!ok) {
      report_error(p.err, (K_FWD << 8) | SITE_LOAD);
      *abort_flag = 1;
    }
    // Drain: every copy this thread started must land before the CTA can exit.
    bool dok = q_loads == 0 || wait_drain(q_full, (q_loads - 1) & 1);
    for (int t = (k_armed > STAGES ? k_armed - STAGES : 0); t < k_armed; ++t)
      dok &= wait_drain(&k_full[t % STAGES], (t / STAGES) & 1);
    for (int t = (v_armed > STAGES ? v_armed - STAGES : 0); t < v_armed; ++t)
      dok &= wait_drain(&v_full[t % STAGES], (t / STAGES) & 1);
    if (!dok) report_error(p.err, (K_FWD << 8) | SITE_DRAIN);
  } else if (!skip && warp == WARP_MMA && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t id_s = idesc_bf16_f32(BM, BN, false, false);
    const uint32_t id_pv = idesc_bf16_f32(BM, HD, false, true);
    const uint32_t sq[2] = {smem_u32(smem + OFF_Q0), smem_u32(smem + OFF_Q1)};
    const uint32_t sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
    uint32_t p_phase[2] = {0, 0};
    int o_items[2] = {0, 0};  // items whose O_i has been produced
    int kv0 = 0;              // K/V ring position of tile 0 of the current item
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.m < 0) break;
      const int qa = 2 * w.m, qb = qa + 1;
      const bool has_b = qb < p.n_qt;
      const int nkv = (has_b ? qb : qa) + 1;
      const int qts[2] = {qa, qb};
      ok = wait_bounded(q_full, it & 1, abort_flag, p.err);
      for (int t = 0; t <= nkv && ok; ++t) {
        const bool has_prev = t > 0, has_cur = t < nkv;
        const int g = kv0 + t;  // ring position of K/V tile t
        if (has_cur) ok = wait_bounded(&k_full[g % STAGES], (g / STAGES) & 1, abort_flag, p.err);
        if (ok && has_prev) ok = wait_bounded(&v_full[(g - 1) % STAGES], ((g - 1) / STAGES) & 1, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        for (int i = 0; i < 2 && ok; ++i) {
          if (i == 1 && !has_b) break;
          const int qt = qts[i];
          if (has_prev && t - 1 <= qt) {
            ok = wait_bounded(&p_ready[i], p_phase[i], abort_flag, p.err);
            p_phase[i] ^= 1;
            if (ok && t == 1 && o_items[i] > 0)  // O_i of the previous item read out by its epilogue
              ok = wait_bounded(&o_empty[i], (o_items[i] - 1) & 1, abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            issue_pv(tmem + tm_o(i), tmem + tm_s(i), sv + ((g - 1) % STAGES) * TILE_BYTES, id_pv, t == 1);
            if (t - 1 == qt) {
              mma_commit(&o_final[i]);
              ++o_items[i];
            }
          }
          if (has_cur && t <= qt) {
            issue_s(tmem + tm_s(i), sq[i], sk + (g % STAGES) * TILE_BYTES, id_s);
            mma_commit(&s_full[i]);
          }
        }
        if (!ok) break;
        if (has_prev) mma_commit(&v_empty[(g - 1) % STAGES]);
        if (has_cur) mma_commit(&k_empty[g % STAGES]);
        if (t == nkv - 1) mma_commit(q_empty);  // the item's last S MMAs read Q for the last time
      }
      kv0 += nkv;
    }
    if (!ok) {
      report_error(p.err, (K_FWD << 8) | SITE_MMA);
      *abort_flag = 1;
    }
    // Drain: all issued MMAs complete before TMEM is released.
    mma_commit(drain);
    if (!wait_drain(drain, 0)) report_error(p.err, (K_FWD << 8) | SITE_DRAIN);
  } else if (!skip && warp < 8) {
    // ---------------- softmax warpgroups ----------------
    const int i = warp / 4;
    const int row = (warp % 4) * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t t_s = lane_addr + tm_s(i), t_o = lane_addr + tm_o(i);
    const float sl2 = p.sl2;
    uint32_t s_phase = 0;
    int o_items = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const Item w = item_of(it);
      if (w.m < 0) break;
      const int qa = 2 * w.m, qb = qa + 1;
      const bool has_b = qb < p.n_qt;
      if (i == 1 && !has_b) continue;
      const int qt = i == 0 ? qa : qb;
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = 0; t <= qt; ++t) {
        ok = wait_bounded(&s_full[i], s_phase, abort_flag, p.err);
        s_phase ^= 1;
        if (!ok) break;
        tc_fence_after();
        uint32_t s0[64], s1[64];
        tmem_ld_x64(t_s, s0);
        tmem_ld_x64(t_s + 64, s1);
        // diagonal tile: key column c is visible to row `row` iff c <= row
        const int lim = (t == qt) ? row : 127;
        // row max: 8 independent partial maxima of three-input maxima (a single chain would
        // serialise the compares)
        float mxp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mxp[e] = -INFINITY;
        if (t == qt) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            mxp[c % 8] = fmax3(mxp[c % 8], c <= lim ? __uint_as_float(s0[c]) : -INFINITY,
                               c + 64 <= lim ? __uint_as_float(s1[c]) : -INFINITY);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) mxp[c % 8] = fmax3(mxp[c % 8], __uint_as_float(s0[c]), __uint_as_float(s1[c]));
        }
        const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                               fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool need = (m_new - m_run) > 8.0f;
        const bool rescale = __any_sync(0xffffffffu, need);
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
        if (need) m_run = m_new;
        l_run *= alpha;
        const float neg_m = -m_run;
        const float sum = (t == qt) ? softmax_p_row<true>(s0, s1, lim, sl2, neg_m, t_s)
                                    : softmax_p_row<false>(s0, s1, 127, sl2, neg_m, t_s);
        l_run += sum;
        if (rescale && t > 0) {
          // O_i was last written by PV_i(t-1), which completed before S_i(t) did.
#pragma unroll
          for (int c = 0; c < HD; c += 32) {
            uint32_t r[32];
            tmem_ld_x32(t_o + c, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st_x32(t_o + c, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready[i]);
      }
      if (ok) ok = wait_bounded(&o_final[i], o_items & 1, abort_flag, p.err);
      if (!ok) break;
      // ---- epilogue: O row / l, stored at its original token; lse in natural log ----
      tc_fence_after();
      const int tok = tile_token0(w, qt) + row;
      const int b = w.b, h = w.h;
      const float inv_l = 1.0f / l_run;
      const size_t o_first = ((size_t)(b * p.N + tok) * p.H + h) * HD;
      const size_t lse_idx = ((size_t)b * p.H + h) * p.N + tok;
      const bool o_ok = in_bounds(o_first, HD, (size_t)p.B * p.N * p.H * HD, p.err, (K_FWD << 8) | SITE_EPILOGUE);
      const bool lse_ok = in_bounds(lse_idx, 1, (size_t)p.B * p.H * p.N, p.err, (K_FWD << 8) | SITE_EPILOGUE);
      __nv_bfloat16* orow = p.o + o_first;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t r[32];
        tmem_ld_x32(t_o + c, r);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + c);
        if (o_ok) {
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (lse_ok) p.lse[lse_idx] = (m_run + log2f(l_run)) * LN2;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[i]);
      ++o_items;
    }
    if (!ok) {
      report_error(p.err, (K_FWD << 8) | SITE_SOFTMAX);
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

}  // namespace fwd

cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                             float* lse, const Shape& s, int n_sm, int* err, cudaStream_t st) {
  fwd::Params p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = s.B;
  p.N = s.N;
  p.H = s.H;
  p.G = s.G;
  p.shift_heads = s.shift_heads;
  p.n_qt = s.G / fwd::BM;
  p.n_pairs = (p.n_qt + 1) / 2;
  p.n_groups = s.N / s.G;
  p.sl2 = (float)(1.4426950408889634 / sqrt((double)s.D));
  p.err = err;
  const long long n_units = (long long)s.B * s.H * p.n_groups;
  const long long n_items = (long long)p.n_pairs * n_units;
  if (n_items <= 0 || n_items > 0x7fffffffLL || n_sm <= 0) return cudaErrorInvalidValue;
  // The fold's equal CTAs run in ceil(folds / n_sm) waves; when the last wave is much
  // less than full and K and V together fit in L2 (the snake's concurrent CTAs read
  // different groups), the snake schedule balances the pairs instead.
  const long long folds = (long long)((p.n_pairs + 1) / 2) * n_units;
  const long long waves = (folds + n_sm - 1) / n_sm;
  const double kv_bytes = 2.0 * s.B * s.N * s.H * s.D * 2;
  p.snake = (folds * 10 < waves * n_sm * 9 && kv_bytes <= 160e6) ? 1 : 0;
  const long long grid = p.snake ? (n_items < n_sm ? n_items : n_sm) : folds;
  cudaError_t e = cudaFuncSetAttribute(fwd::s2attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwd::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  fwd::s2attn_fwd_kernel<<<(unsigned)grid, fwd::NTHREADS, fwd::SMEM_BYTES, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace s2
