// s2attn_simt.cu -- the memory-bound and CUDA-core kernels of the library:
//   * RoPE with position interpolation (in place, bf16), from a cos/sin table
//   * backward preprocess: delta = rowsum(dO * O) and zeroing of the dQ accumulator
//   * dQ conversion: fp32 accumulator -> bf16, times the softmax scale
//   * an fp32 S^2-Attn forward/backward on CUDA cores (any valid shape; used for
//     fp32 inputs, where bf16 tensor-core inputs would not meet an fp32 tolerance)
#include "s2_internal.h"
#include "s2_ptx.cuh"

namespace s2 {
namespace {

__host__ __device__ inline int grid_for(long long work, int block) {
  long long g = (work + block - 1) / block;
  const long long cap = 148LL * 32;  // grid-stride beyond 32 blocks per SM
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

// ---- RoPE-PI -------------------------------------------------------------------
// "LongLoRA paper notes", section 3.4: position interpolation squeezes positions
// [0, L) into [0, L0).  Token t is rotated as if it sat at t * pos_scale.  Element i
// pairs with element i + D/2 and turns by angle pos * base^(-2i/D); the cos/sin of
// that angle come from the table.  The rotation is evaluated exactly as
//   y1 = x1*c - x2*s,  y2 = x2*c + x1*s   (each product rounded to fp32 first),
// then rounded to bf16, nearest even.
__device__ __forceinline__ void rope8(uint4& lo, uint4& hi, const float4 c0, const float4 c1, const float4 s0,
                                      const float4 s1) {
  const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  __nv_bfloat162* a = reinterpret_cast<__nv_bfloat162*>(&lo);
  __nv_bfloat162* b = reinterpret_cast<__nv_bfloat162*>(&hi);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x1 = __bfloat1622float2(a[e]);
    const float2 x2 = __bfloat1622float2(b[e]);
    const float c_0 = cs[2 * e], c_1 = cs[2 * e + 1], s_0 = sn[2 * e], s_1 = sn[2 * e + 1];
    const float y1a = __fsub_rn(__fmul_rn(x1.x, c_0), __fmul_rn(x2.x, s_0));
    const float y1b = __fsub_rn(__fmul_rn(x1.y, c_1), __fmul_rn(x2.y, s_1));
    const float y2a = __fadd_rn(__fmul_rn(x2.x, c_0), __fmul_rn(x1.x, s_0));
    const float y2b = __fadd_rn(__fmul_rn(x2.y, c_1), __fmul_rn(x1.y, s_1));
    a[e] = __floats2bfloat162_rn(y1a, y1b);
    b[e] = __floats2bfloat162_rn(y2a, y2b);
  }
}

__global__ void rope_pi_kernel(__nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k,
                               const float* __restrict__ cos_tab, const float* __restrict__ sin_tab, int N, int H,
                               int D, long long rows) {
  const int half = D / 2;
  const int chunks = half / 8;  // 8 pairs per thread
  const long long total = rows * chunks;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const long long row = w / chunks;
    const int i0 = (int)(w % chunks) * 8;
    const int t = (int)((row / H) % N);
    const float4* ct = reinterpret_cast<const float4*>(cos_tab + (size_t)t * half + i0);
    const float4* st = reinterpret_cast<const float4*>(sin_tab + (size_t)t * half + i0);
    const float4 c0 = __ldg(ct), c1 = __ldg(ct + 1), s0 = __ldg(st), s1 = __ldg(st + 1);
    if (q) {
      uint4* p1 = reinterpret_cast<uint4*>(q + row * D + i0);
      uint4* p2 = reinterpret_cast<uint4*>(q + row * D + half + i0);
      uint4 lo = *p1, hi = *p2;
      rope8(lo, hi, c0, c1, s0, s1);
      *p1 = lo;
      *p2 = hi;
    }
    if (k) {
      uint4* p1 = reinterpret_cast<uint4*>(k + row * D + i0);
      uint4* p2 = reinterpret_cast<uint4*>(k + row * D + half + i0);
      uint4 lo = *p1, hi = *p2;
      rope8(lo, hi, c0, c1, s0, s1);
      *p1 = lo;
      *p2 = hi;
    }
  }
}

// ---- backward preprocess / dQ convert ------------------------------------------
// One thread per 8 elements of a [B,N,H,D] row; D/8 consecutive threads share a row.
__global__ void bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                      float* __restrict__ delta, float* __restrict__ dq_acc, int N, int H, int D,
                                      long long rows) {
  const int per_row = D / 8;  // power of two <= 32 (D in {64, 128, 256})
  const long long total = rows * per_row;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long w0 = blockIdx.x * (long long)blockDim.x; w0 < total; w0 += stride) {
    const long long w = w0 + threadIdx.x;
    float acc = 0.f;
    long long row = 0;
    if (w < total) {
      row = w / per_row;
      const int c = (int)(w % per_row) * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + c);
      const uint4 g = *reinterpret_cast<const uint4*>(dout + row * D + c);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(g2[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + row * D + c);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int off = per_row / 2; off > 0; off /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (w < total && (w % per_row) == 0) {
      const long long bt = row / H;  // b*N + t
      const int h = (int)(row % H);
      const long long b = bt / N, t = bt % N;
      delta[(b * H + h) * N + t] = acc;
    }
  }
}

__global__ void dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, float scale,
                                  long long n8) {
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < n8; w += (long long)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * w];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * w + 1];
    uint4 out;
    out.x = pack_bf16x2(a.x * scale, a.y * scale);
    out.y = pack_bf16x2(a.z * scale, a.w * scale);
    out.z = pack_bf16x2(b.x * scale, b.y * scale);
    out.w = pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[w] = out;
  }
}

// ---- fp32 S^2-Attn on CUDA cores --------------------------------------------------
constexpr int F32_MAX_D = 128;

struct F32Shape {
  int B, N, H, D, G, shift_heads;
  float scale;
};

__device__ __forceinline__ int f32_shift(const F32Shape& s, int h) {
  return (h >= s.H - s.shift_heads) ? s.G / 2 : 0;
}
__device__ __forceinline__ size_t f32_row(const F32Shape& s, int b, int t, int h) {
  return ((size_t)(b * s.N + t) * s.H + h) * s.D;
}

// One thread per (b, h, rolled row r): causal softmax over the keys r0..r of its group.
__global__ void fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                               float* __restrict__ o, float* __restrict__ lse, F32Shape s) {
  const long long total = (long long)s.B * s.H * s.N;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total; w += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(w % s.N);
    const int h = (int)((w / s.N) % s.H);
    const int b = (int)(w / ((long long)s.N * s.H));
    const int sh = f32_shift(s, h);
    const int t = (r + sh) % s.N;
    const int r0 = (r / s.G) * s.G;
    const float* qr = q + f32_row(s, b, t, h);
    float acc[F32_MAX_D];
    for (int d = 0; d < s.D; ++d) acc[d] = 0.f;
    float m = -INFINITY, l = 0.f;
    for (int kk = r0; kk <= r; ++kk) {
      const int tk = (kk + sh) % s.N;
      const float* kr = k + f32_row(s, b, tk, h);
      const float* vr = v + f32_row(s, b, tk, h);
      float dot = 0.f;
      for (int d = 0; d < s.D; ++d) dot = fmaf(qr[d], kr[d], dot);
      const float x = dot * s.scale;
      const float m_new = fmaxf(m, x);
      const float corr = expf(m - m_new);
      const float pw = expf(x - m_new);
      l = l * corr + pw;
      for (int d = 0; d < s.D; ++d) acc[d] = fmaf(pw, vr[d], acc[d] * corr);
      m = m_new;
    }
    float* orow = o + f32_row(s, b, t, h);
    const float inv = 1.f / l;
    for (int d = 0; d < s.D; ++d) orow[d] = acc[d] * inv;
    lse[((size_t)b * s.H + h) * s.N + t] = m + logf(l);
  }
}

// Query side: delta_t = dO_t . O_t, and dQ_t = scale * sum_k dS[t,k] K_k.
__global__ void bwd_f32_query_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                     const float* __restrict__ v, const float* __restrict__ o,
                                     const float* __restrict__ dout, const float* __restrict__ lse,
                                     float* __restrict__ dq, float* __restrict__ delta, F32Shape s) {
  const long long total = (long long)s.B * s.H * s.N;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total; w += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(w % s.N);
    const int h = (int)((w / s.N) % s.H);
    const int b = (int)(w / ((long long)s.N * s.H));
    const int sh = f32_shift(s, h);
    const int t = (r + sh) % s.N;
    const int r0 = (r / s.G) * s.G;
    const float* qr = q + f32_row(s, b, t, h);
    const float* gr = dout + f32_row(s, b, t, h);
    const float* orow = o + f32_row(s, b, t, h);
    float dl = 0.f;
    for (int d = 0; d < s.D; ++d) dl = fmaf(gr[d], orow[d], dl);
    const float ls = lse[((size_t)b * s.H + h) * s.N + t];
    float acc[F32_MAX_D];
    for (int d = 0; d < s.D; ++d) acc[d] = 0.f;
    for (int kk = r0; kk <= r; ++kk) {
      const int tk = (kk + sh) % s.N;
      const float* kr = k + f32_row(s, b, tk, h);
      const float* vr = v + f32_row(s, b, tk, h);
      float qk = 0.f, dp = 0.f;
      for (int d = 0; d < s.D; ++d) {
        qk = fmaf(qr[d], kr[d], qk);
        dp = fmaf(gr[d], vr[d], dp);
      }
      const float pw = expf(qk * s.scale - ls);
      const float ds = pw * (dp - dl);
      for (int d = 0; d < s.D; ++d) acc[d] = fmaf(ds, kr[d], acc[d]);
    }
    float* dqr = dq + f32_row(s, b, t, h);
    for (int d = 0; d < s.D; ++d) dqr[d] = acc[d] * s.scale;
    delta[((size_t)b * s.H + h) * s.N + t] = dl;
  }
}

// Key side: dV_k = sum_t P[t,k] dO_t ; dK_k = scale * sum_t dS[t,k] Q_t over the
// queries t at or after k in the same group.
__global__ void bwd_f32_key_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                   const float* __restrict__ v, const float* __restrict__ dout,
                                   const float* __restrict__ lse, const float* __restrict__ delta,
                                   float* __restrict__ dk, float* __restrict__ dv, F32Shape s) {
  const long long total = (long long)s.B * s.H * s.N;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total; w += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(w % s.N);
    const int h = (int)((w / s.N) % s.H);
    const int b = (int)(w / ((long long)s.N * s.H));
    const int sh = f32_shift(s, h);
    const int tk = (r + sh) % s.N;
    const int r_end = (r / s.G + 1) * s.G;
    const float* kr = k + f32_row(s, b, tk, h);
    const float* vr = v + f32_row(s, b, tk, h);
    float ak[F32_MAX_D], av[F32_MAX_D];
    for (int d = 0; d < s.D; ++d) ak[d] = av[d] = 0.f;
    for (int qq = r; qq < r_end; ++qq) {
      const int t = (qq + sh) % s.N;
      const float* qr = q + f32_row(s, b, t, h);
      const float* gr = dout + f32_row(s, b, t, h);
      float qk = 0.f, dp = 0.f;
      for (int d = 0; d < s.D; ++d) {
        qk = fmaf(qr[d], kr[d], qk);
        dp = fmaf(gr[d], vr[d], dp);
      }
      const size_t st = ((size_t)b * s.H + h) * s.N + t;
      const float pw = expf(qk * s.scale - lse[st]);
      const float ds = pw * (dp - delta[st]);
      for (int d = 0; d < s.D; ++d) {
        av[d] = fmaf(pw, gr[d], av[d]);
        ak[d] = fmaf(ds, qr[d], ak[d]);
      }
    }
    float* dkr = dk + f32_row(s, b, tk, h);
    float* dvr = dv + f32_row(s, b, tk, h);
    for (int d = 0; d < s.D; ++d) {
      dkr[d] = ak[d] * s.scale;
      dvr[d] = av[d];
    }
  }
}

F32Shape f32_shape(const Shape& s) {
  return F32Shape{s.B, s.N, s.H, s.D, s.G, s.shift_heads, (float)(1.0 / sqrt((double)s.D))};
}

}  // namespace

cudaError_t launch_rope_pi(void* q, void* k, const float* cos_tab, const float* sin_tab, int B, int N, int H, int D,
                           cudaStream_t st) {
  const long long rows = (long long)B * N * H;
  const int block = 256;
  rope_pi_kernel<<<grid_for(rows * (D / 16), block), block, 0, st>>>(
      static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), cos_tab, sin_tab, N, H, D, rows);
  return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(const void* o, const void* dout, float* delta, float* dq_acc, const Shape& s,
                                  cudaStream_t st) {
  const long long rows = (long long)s.B * s.N * s.H;
  const int block = 256;
  bwd_preprocess_kernel<<<grid_for(rows * (s.D / 8), block), block, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), delta, dq_acc, s.N, s.H, s.D,
      rows);
  return cudaGetLastError();
}

cudaError_t launch_dq_convert(const float* dq_acc, void* dq, const Shape& s, cudaStream_t st) {
  const long long n8 = (long long)s.B * s.N * s.H * s.D / 8;
  const int block = 256;
  dq_convert_kernel<<<grid_for(n8, block), block, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dq),
                                                           (float)(1.0 / sqrt((double)s.D)), n8);
  return cudaGetLastError();
}

cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, const Shape& s,
                           cudaStream_t st) {
  const long long total = (long long)s.B * s.H * s.N;
  fwd_f32_kernel<<<grid_for(total, 128), 128, 0, st>>>(q, k, v, o, lse, f32_shape(s));
  return cudaGetLastError();
}

cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* dout,
                           const float* lse, float* dq, float* dk, float* dv, float* delta, const Shape& s,
                           cudaStream_t st) {
  const long long total = (long long)s.B * s.H * s.N;
  bwd_f32_query_kernel<<<grid_for(total, 128), 128, 0, st>>>(q, k, v, o, dout, lse, dq, delta, f32_shape(s));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_f32_key_kernel<<<grid_for(total, 128), 128, 0, st>>>(q, k, v, dout, lse, delta, dk, dv, f32_shape(s));
  return cudaGetLastError();
}

}  // namespace s2
