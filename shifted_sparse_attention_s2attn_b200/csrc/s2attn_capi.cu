// s2attn_capi.cu -- the extern "C" boundary: argument validation, tensor-map
// construction, the RoPE table cache, the device error word, and kernel launches.
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "s2_internal.h"
#include "s2_ptx.cuh"
#include "s2attn.h"

namespace {

__device__ int g_error_word;

constexpr int kMaxDevices = 64;

// ---- error word -----------------------------------------------------------------
int* error_word_ptr() {
  static std::mutex mu;
  static int* cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

// ---- tensor maps ----------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// A [B,N,H,D] tensor viewed as 3-D {D, H, B*N}; a box is box_rows tokens x box_cols
// elements of one head.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, size_t esize, int B, int N, int H, int D,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)B * (cuuint64_t)N};
  cuuint64_t strides[2] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize};
  cuuint32_t box[3] = {box_cols, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool map_bf16_sw128(CUtensorMap* m, const void* base, const s2::Shape& s, uint32_t rows) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.B, s.N, s.H, s.D, 64, rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// A row-major bf16 matrix [outer, inner] (rank 2), or a stack [d2, outer, inner] (rank 3,
// boxes one matrix deep), with 128-byte swizzled boxes of box_inner x box_outer elements;
// out-of-range elements read as zero.  The rank must match the kernel's load instruction.
bool map_rows_bf16(CUtensorMap* m, const void* base, int rank, uint64_t inner, uint64_t outer, uint64_t d2,
                   uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, outer, d2};
  cuuint64_t strides[2] = {inner * 2, inner * outer * 2};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (rank != 2 && rank != 3) return false;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---- validation -----------------------------------------------------------------
bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int N, int H, int D, int G, int shift_heads) {
  if (B < 1 || N < 1 || H < 1 || D < 1 || G < 1) return S2ATTN_ERR_INVALID_ARG;
  if (N % G != 0) return S2ATTN_ERR_INVALID_ARG;
  if (shift_heads < 0 || shift_heads > H) return S2ATTN_ERR_INVALID_ARG;
  if (shift_heads > 0 && (G % 2) != 0) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)B * N > INT_MAX / 2) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)B * N * H > (LLONG_MAX / 8) / D) return S2ATTN_ERR_INVALID_ARG;
  return S2ATTN_OK;
}

int check_tensor_core_shape(int B, int N, int H, int D, int G, int shift_heads) {
  int rc = check_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (D != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (G % 128 != 0) return S2ATTN_ERR_UNSUPPORTED;
  if (shift_heads > 0 && (G / 2) % 128 != 0) return S2ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H * (N / G) * (G / 128) > INT_MAX) return S2ATTN_ERR_UNSUPPORTED;
  return S2ATTN_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? S2ATTN_OK : S2ATTN_ERR_CUDA; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---- RoPE tables ------------------------------------------------------------------
struct RopeTable {
  float* cos_d = nullptr;
  float* sin_d = nullptr;
};

// theta_i = (float) base^(-2i/D) (pow in double); a = ((float)t * pos_scale) * theta_i in
// float; table entries (float) cos((double)a), (float) sin((double)a).
int rope_table(int dev, int N, int D, float pos_scale, float base, RopeTable* out) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, uint32_t, uint32_t>, RopeTable> cache;
  uint32_t ps, bs;
  std::memcpy(&ps, &pos_scale, 4);
  std::memcpy(&bs, &base, 4);
  auto key = std::make_tuple(dev, N, D, ps, bs);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return S2ATTN_OK;
  }
  const int half = D / 2;
  std::vector<float> c((size_t)N * half), s((size_t)N * half);
  std::vector<float> theta(half);
  for (int i = 0; i < half; ++i) theta[i] = (float)std::pow((double)base, -2.0 * (double)i / (double)D);
  for (int t = 0; t < N; ++t) {
    volatile float pos = (float)t * pos_scale;
    for (int i = 0; i < half; ++i) {
      volatile float a = pos * theta[i];
      c[(size_t)t * half + i] = (float)std::cos((double)a);
      s[(size_t)t * half + i] = (float)std::sin((double)a);
    }
  }
  RopeTable tab;
  const size_t bytes = sizeof(float) * c.size();
  if (cudaMalloc(&tab.cos_d, bytes) != cudaSuccess) return S2ATTN_ERR_CUDA;
  if (cudaMalloc(&tab.sin_d, bytes) != cudaSuccess) {
    cudaFree(tab.cos_d);
    return S2ATTN_ERR_CUDA;
  }
  if (cudaMemcpy(tab.cos_d, c.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(tab.sin_d, s.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(tab.cos_d);
    cudaFree(tab.sin_d);
    return S2ATTN_ERR_CUDA;
  }
  cache[key] = tab;
  *out = tab;
  return S2ATTN_OK;
}

// One thread waits on an mbarrier that nothing ever arrives at; the bounded wait must
// give up after timeout_ns and record (K_SELFTEST << 8) | 1 in the error word.
__global__ void selftest_wait_kernel(int* err, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    s2::mbar_init(&bar, 1);
    abort_flag = 0;
    s2::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !s2::wait_bounded_ns(&bar, 0, &abort_flag, err, timeout_ns))
    s2::report_error(err, (s2::K_SELFTEST << 8) | 1);
}

int sm_count();

int bwd_main_impl(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                  const float* delta, float* dq_acc, void* dk, void* dv, const s2::Shape& s, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  if (!map_bf16_sw128(&tq, q, s, 128) || !map_bf16_sw128(&tk, k, s, 128) || !map_bf16_sw128(&tv, v, s, 128) ||
      !map_bf16_sw128(&tdo, dout, s, 128))
    return S2ATTN_ERR_CUDA;
  int* err = error_word_ptr();
  if (!err) return S2ATTN_ERR_CUDA;
  return cuda_status(s2::launch_bwd_sm100(tq, tk, tv, tdo, lse, delta, dq_acc, dk, dv, s, sm_count(), err, st));
}

// SM count of the current device, looked up once per device.
int sm_count() {
  static std::mutex mu;
  static int cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev] && cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    cache[dev] = 0;
  return cache[dev];
}

int check_decode_shape(int B, int M, int N, int H, int D) {
  if (B < 1 || M < 1 || N < 1 || H < 1 || D < 1 || M > N) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)B * N > INT_MAX / 2) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)B * N * H > (LLONG_MAX / 8) / D) return S2ATTN_ERR_INVALID_ARG;
  if (D != 128 || M > s2::kDecodeMaxM) return S2ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H * M > INT_MAX || (long long)B * H * s2::kDecodeMaxSplits > INT_MAX)
    return S2ATTN_ERR_UNSUPPORTED;
  return S2ATTN_OK;
}

// Splits the workspace is sized for: the most any device can get (1 per key tile,
// at most kDecodeMaxSplits), so that the size does not depend on the device.
int decode_max_splits(int N) {
  const int tiles = (N + s2::kDecodeTileKeys - 1) / s2::kDecodeTileKeys;
  return tiles < s2::kDecodeMaxSplits ? tiles : s2::kDecodeMaxSplits;
}

// LoRA workspace: u [parts, T, 64] bf16, then a_pad, then b_pad (each 256-byte aligned).
size_t lora_u_bytes(int T, int parts) { return align256((size_t)parts * T * s2::kLoraRankPad * 2); }

size_t decode_part_o_bytes(int B, int M, int N, int H, int D) {
  return align256((size_t)B * H * decode_max_splits(N) * M * D * sizeof(float));
}

}  // namespace

namespace s2 {
int check_tensor_core_args(int B, int N, int H, int D, int G, int shift_heads) {
  return check_tensor_core_shape(B, N, H, D, G, shift_heads);
}
}  // namespace s2

extern "C" {

int s2attn_version(void) { return 100; }

const char* s2attn_status_string(int status) {
  switch (status) {
    case S2ATTN_OK: return "ok";
    case S2ATTN_ERR_INVALID_ARG: return "invalid argument";
    case S2ATTN_ERR_UNSUPPORTED: return "unsupported shape for this path";
    case S2ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case S2ATTN_ERR_CUDA: return "CUDA call failed";
    case S2ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int D, int G,
               int shift_heads, void* stream) {
  int rc = check_tensor_core_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2ATTN_ERR_INVALID_ARG;
  const s2::Shape s{B, N, H, D, G, shift_heads};
  CUtensorMap tq, tk, tv;
  if (!map_bf16_sw128(&tq, q, s, 128) || !map_bf16_sw128(&tk, k, s, 128) || !map_bf16_sw128(&tv, v, s, 128))
    return S2ATTN_ERR_CUDA;
  int* err = error_word_ptr();
  if (!err) return S2ATTN_ERR_CUDA;
  return cuda_status(s2::launch_fwd_sm100(tq, tk, tv, o, lse, s, sm_count(), err, static_cast<cudaStream_t>(stream)));
}

size_t s2attn_bwd_workspace_bytes(int B, int N, int H, int D) {
  if (B < 1 || N < 1 || H < 1 || D < 1) return 0;
  return align256((size_t)B * N * H * D * sizeof(float)) + align256((size_t)B * H * N * sizeof(float));
}

int s2attn_bwd_preprocess(const void* o, const void* dout, float* delta, float* dq_acc, int B, int N, int H, int D,
                          void* stream) {
  int rc = check_shape(B, N, H, D, N, 0);
  if (rc) return rc;
  if (D != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(o) || !aligned16(dout) || !aligned16(delta) || !aligned16(dq_acc)) return S2ATTN_ERR_INVALID_ARG;
  const s2::Shape s{B, N, H, D, N, 0};
  return cuda_status(s2::launch_bwd_preprocess(o, dout, delta, dq_acc, s, static_cast<cudaStream_t>(stream)));
}

int s2attn_bwd_main(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                    const float* delta, float* dq_acc, void* dk, void* dv, int B, int N, int H, int D, int G,
                    int shift_heads, void* stream) {
  int rc = check_tensor_core_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(delta) || !aligned16(dq_acc) || !aligned16(dk) || !aligned16(dv))
    return S2ATTN_ERR_INVALID_ARG;
  const s2::Shape s{B, N, H, D, G, shift_heads};
  return bwd_main_impl(q, k, v, dout, lse, delta, dq_acc, dk, dv, s, static_cast<cudaStream_t>(stream));
}

int s2attn_bwd_dq_convert(const float* dq_acc, void* dq, int B, int N, int H, int D, void* stream) {
  int rc = check_shape(B, N, H, D, N, 0);
  if (rc) return rc;
  if (D % 8 != 0) return S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(dq_acc) || !aligned16(dq)) return S2ATTN_ERR_INVALID_ARG;
  const s2::Shape s{B, N, H, D, N, 0};
  return cuda_status(s2::launch_dq_convert(dq_acc, dq, s, static_cast<cudaStream_t>(stream)));
}

int s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, int B, int N, int H, int D, int G, int shift_heads, void* workspace,
               size_t workspace_bytes, void* stream) {
  int rc = check_tensor_core_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return S2ATTN_ERR_INVALID_ARG;
  const size_t need = s2attn_bwd_workspace_bytes(B, N, H, D);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2ATTN_ERR_WORKSPACE;
  float* dq_acc = static_cast<float*>(workspace);
  float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256((size_t)B * N * H * D * 4));
  const s2::Shape s{B, N, H, D, G, shift_heads};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = cuda_status(s2::launch_bwd_preprocess(o, dout, delta, dq_acc, s, st)))) return rc;
  if ((rc = bwd_main_impl(q, k, v, dout, lse, delta, dq_acc, dk, dv, s, st))) return rc;
  return cuda_status(s2::launch_dq_convert(dq_acc, dq, s, st));
}

int s2attn_halo_rows(void* const* x, void* const* buf, int n_tensors, int to_buf, int B, int N, int H, int D,
                     int G, int shift_heads, void* stream) {
  int rc = check_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (shift_heads < 1 || n_tensors < 1 || n_tensors > s2::kHaloMaxTensors || !x || !buf) return S2ATTN_ERR_INVALID_ARG;
  if ((D * 2) % 16 != 0) return S2ATTN_ERR_UNSUPPORTED;
  for (int i = 0; i < n_tensors; ++i)
    if (!aligned16(x[i]) || !aligned16(buf[i])) return S2ATTN_ERR_INVALID_ARG;
  const int n_sm = sm_count();
  if (n_sm <= 0) return S2ATTN_ERR_CUDA;
  return cuda_status(s2::launch_halo_rows(x, buf, n_tensors, to_buf ? 1 : 0, B, N, H, D, G, shift_heads, n_sm,
                                          static_cast<cudaStream_t>(stream)));
}

int s2attn_halo_lse(float* const* lse, float* const* buf, int n_tensors, int to_buf, int B, int N, int H, int G,
                    int shift_heads, void* stream) {
  int rc = check_shape(B, N, H, 1, G, shift_heads);
  if (rc) return rc;
  if (shift_heads < 1 || n_tensors < 1 || n_tensors > s2::kHaloMaxTensors || !lse || !buf)
    return S2ATTN_ERR_INVALID_ARG;
  for (int i = 0; i < n_tensors; ++i)
    if (!lse[i] || !buf[i] || (reinterpret_cast<uintptr_t>(lse[i]) & 3u) || (reinterpret_cast<uintptr_t>(buf[i]) & 3u))
      return S2ATTN_ERR_INVALID_ARG;
  const int n_sm = sm_count();
  if (n_sm <= 0) return S2ATTN_ERR_CUDA;
  return cuda_status(s2::launch_halo_lse(lse, buf, n_tensors, to_buf ? 1 : 0, B, N, H, G, shift_heads, n_sm,
                                         static_cast<cudaStream_t>(stream)));
}

size_t s2attn_decode_workspace_bytes(int B, int M, int N, int H, int D) {
  if (check_decode_shape(B, M, N, H, D)) return 0;
  return decode_part_o_bytes(B, M, N, H, D) +
         align256((size_t)B * H * decode_max_splits(N) * M * 2 * sizeof(float));
}

int s2attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int M, int N, int H,
                  int D, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_decode_shape(B, M, N, H, D);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2ATTN_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < s2attn_decode_workspace_bytes(B, M, N, H, D) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2ATTN_ERR_WORKSPACE;
  const int n_sm = sm_count();
  if (n_sm <= 0) return S2ATTN_ERR_CUDA;
  float* part_o = static_cast<float*>(workspace);
  float* part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + decode_part_o_bytes(B, M, N, H, D));
  const s2::Shape s{B, N, H, D, N, 0};
  int* err = error_word_ptr();
  if (!err) return S2ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int tps = 0;
  if (M <= s2::kDecodeSimtMaxM) {
    const int S = s2::decode_splits(B, N, H, n_sm, &tps);
    CUtensorMap tk, tv;
    if (!map_bf16_sw128(&tk, k, s, s2::kDecodeTileKeys) || !map_bf16_sw128(&tv, v, s, s2::kDecodeTileKeys))
      return S2ATTN_ERR_CUDA;
    return cuda_status(s2::launch_decode_sm100(tk, tv, q, o, lse, part_o, part_ml, B, M, N, H, S, tps, err, st));
  }
  const int S = s2::decode_splits_tc(B, N, H, n_sm, &tps);
  const s2::Shape sq{B, M, H, D, M, 0};
  CUtensorMap tq, tk, tv;
  if (!map_bf16_sw128(&tq, q, sq, 128) || !map_bf16_sw128(&tk, k, s, s2::kDecodeTileKeys) ||
      !map_bf16_sw128(&tv, v, s, s2::kDecodeTileKeys))
    return S2ATTN_ERR_CUDA;
  return cuda_status(s2::launch_decode_tc_sm100(tq, tk, tv, o, lse, part_o, part_ml, B, M, N, H, S, tps, err, st));
}

int s2attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int N, int H, int D,
                   int G, int shift_heads, void* stream) {
  int rc = check_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (D > 128) return S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2ATTN_ERR_INVALID_ARG;
  const s2::Shape s{B, N, H, D, G, shift_heads};
  return cuda_status(s2::launch_fwd_f32(q, k, v, o, lse, s, static_cast<cudaStream_t>(stream)));
}

int s2attn_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* dout,
                   const float* lse, float* dq, float* dk, float* dv, int B, int N, int H, int D, int G,
                   int shift_heads, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_shape(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  if (D > 128) return S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return S2ATTN_ERR_INVALID_ARG;
  const size_t need = s2attn_bwd_workspace_bytes(B, N, H, D);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2ATTN_ERR_WORKSPACE;
  float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256((size_t)B * N * H * D * 4));
  const s2::Shape s{B, N, H, D, G, shift_heads};
  return cuda_status(
      s2::launch_bwd_f32(q, k, v, o, dout, lse, dq, dk, dv, delta, s, static_cast<cudaStream_t>(stream)));
}

int rope_pi_apply(void* q, void* k, int B, int N, int H, int D, float pos_scale, float base, void* stream) {
  if (B < 1 || N < 1 || H < 1 || D < 16 || D % 16 != 0 || D > 256) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)B * N * H > (LLONG_MAX / 8) / D) return S2ATTN_ERR_INVALID_ARG;
  if (!q && !k) return S2ATTN_ERR_INVALID_ARG;
  if ((q && !aligned16(q)) || (k && !aligned16(k))) return S2ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(pos_scale) || !std::isfinite(base) || !(base > 0.f)) return S2ATTN_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return S2ATTN_ERR_CUDA;
  RopeTable tab;
  int rc = rope_table(dev, N, D, pos_scale, base, &tab);
  if (rc) return rc;
  return cuda_status(
      s2::launch_rope_pi(q, k, tab.cos_d, tab.sin_d, B, N, H, D, static_cast<cudaStream_t>(stream)));
}

int rope_pi_apply_offset(void* q, void* k, int B, int N, int H, int D, int pos0, float pos_scale, float base,
                         void* stream) {
  if (B < 1 || N < 1 || H < 1 || D < 16 || D % 16 != 0 || D > 256 || pos0 < 0) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)pos0 + N > (1LL << 24)) return S2ATTN_ERR_INVALID_ARG;
  if ((long long)B * N * H > (LLONG_MAX / 8) / D) return S2ATTN_ERR_INVALID_ARG;
  if (!q && !k) return S2ATTN_ERR_INVALID_ARG;
  if ((q && !aligned16(q)) || (k && !aligned16(k))) return S2ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(pos_scale) || !std::isfinite(base) || !(base > 0.f)) return S2ATTN_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return S2ATTN_ERR_CUDA;
  // Row p of a table holds position p whatever the table's length, so the table of the
  // next power of two >= pos0 + N (cached like any other) serves every offset below it,
  // and a decoding loop that grows its sequence builds only a few tables.
  int rows = 1024;
  while (rows < pos0 + N) rows *= 2;
  RopeTable tab;
  int rc = rope_table(dev, rows, D, pos_scale, base, &tab);
  if (rc) return rc;
  const size_t off = (size_t)pos0 * (D / 2);
  return cuda_status(s2::launch_rope_pi(q, k, tab.cos_d + off, tab.sin_d + off, B, N, H, D,
                                        static_cast<cudaStream_t>(stream)));
}

size_t lora_proj_workspace_bytes(int T, int K, int n_out, int parts, int r) {
  if (T < 1 || K < 1 || n_out < 1 || parts < 1 || r < 0 || r > s2::kLoraMaxRank) return 0;
  if (r == 0) return 0;
  return lora_u_bytes(T, parts) + align256((size_t)parts * s2::kLoraRankPad * K * 2) +
         align256((size_t)parts * n_out * s2::kLoraRankPad * 2);
}

int lora_proj_fwd(const void* x, const void* w, const void* lora_a, const void* lora_b, void* y, int T, int K,
                  int n_out, int parts, int r, float scaling, int rope_parts, int head_dim, int seq_len,
                  float pos_scale, float base, void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 1 || K < 8 || K % 8 != 0 || n_out < 1 || parts < 1 || r < 0 || r > s2::kLoraMaxRank)
    return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return S2ATTN_ERR_INVALID_ARG;
  if (r > 0 && (!aligned16(lora_a) || !lora_b || !std::isfinite(scaling))) return S2ATTN_ERR_INVALID_ARG;
  if (rope_parts < 0 || rope_parts > parts) return S2ATTN_ERR_INVALID_ARG;
  if (rope_parts > 0) {
    if (head_dim != 32 && head_dim != 64 && head_dim != 128 && head_dim != 256) return S2ATTN_ERR_INVALID_ARG;
    if (seq_len < 1 || T % seq_len != 0) return S2ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(pos_scale) || !std::isfinite(base) || !(base > 0.f)) return S2ATTN_ERR_INVALID_ARG;
  }
  if (n_out % s2::kLoraProjTileN != 0) return S2ATTN_ERR_UNSUPPORTED;
  if (K < 64) return S2ATTN_ERR_UNSUPPORTED;   // the tensor maps' 64-column boxes must fit in a row of x and W
  if ((long long)parts * n_out > INT_MAX || (long long)T + 128 > INT_MAX) return S2ATTN_ERR_UNSUPPORTED;
  if (((long long)T + 127) / 128 * ((long long)parts * n_out / s2::kLoraProjTileN) > INT_MAX)
    return S2ATTN_ERR_UNSUPPORTED;
  if (r > 0) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return S2ATTN_ERR_WORKSPACE;
    if (workspace_bytes < lora_proj_workspace_bytes(T, K, n_out, parts, r)) return S2ATTN_ERR_WORKSPACE;
  }
  int* err = error_word_ptr();
  if (!err) return S2ATTN_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return S2ATTN_ERR_CUDA;
  RopeTable tab;
  if (rope_parts > 0) {
    int rc = rope_table(dev, seq_len, head_dim, pos_scale, base, &tab);
    if (rc) return rc;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap tx, tw, tu, tb, ta;
  if (!map_rows_bf16(&tx, x, 2, K, T, 1, 64, 128) ||
      !map_rows_bf16(&tw, w, 2, K, (uint64_t)parts * n_out, 1, 64, s2::kLoraProjTileN))
    return S2ATTN_ERR_CUDA;
  tu = tx;
  tb = tw;
  if (r > 0) {
    char* ws = static_cast<char*>(workspace);
    void* u = ws;
    void* a_pad = ws + lora_u_bytes(T, parts);
    void* b_pad = ws + lora_u_bytes(T, parts) + align256((size_t)parts * s2::kLoraRankPad * K * 2);
    if (!map_rows_bf16(&ta, a_pad, 2, K, (uint64_t)parts * s2::kLoraRankPad, 1, 64, s2::kLoraRankPad) ||
        !map_rows_bf16(&tu, u, 3, s2::kLoraRankPad, T, parts, 64, 128) ||
        !map_rows_bf16(&tb, b_pad, 2, s2::kLoraRankPad, (uint64_t)parts * n_out, 1, 64, s2::kLoraProjTileN))
      return S2ATTN_ERR_CUDA;
    cudaError_t e = s2::launch_lora_pad(lora_a, lora_b, a_pad, b_pad, parts, r, K, n_out, st);
    if (e == cudaSuccess) e = s2::launch_lora_down(tx, ta, u, T, K, parts, scaling, sm_count(), err, st);
    if (e != cudaSuccess) return S2ATTN_ERR_CUDA;
  }
  return cuda_status(s2::launch_lora_proj(tx, tw, tu, tb, y, T, K, n_out, parts, r, rope_parts, head_dim, seq_len,
                                          tab.cos_d, tab.sin_d, sm_count(), err, st));
}

size_t lora_proj_bwd_workspace_bytes(int T, int K, int n_out, int parts, int r) {
  if (T < 1 || K < 1 || n_out < 1 || parts < 1 || r < 0 || r > s2::kLoraMaxRank) return 0;
  const size_t apad = align256((size_t)parts * s2::kLoraRankPad * K * 2);
  const size_t bpad = align256((size_t)parts * n_out * s2::kLoraRankPad * 2);
  const size_t da_acc = align256((size_t)((parts * s2::kLoraRankPad + 127) / 128) * 128 * K * 4);
  const size_t db_acc = align256((size_t)parts * n_out * s2::kLoraRankPad * 4);
  return 2 * lora_u_bytes(T, parts) + apad + bpad + da_acc + db_acc;   // u, g, a_pad, b_pad, accumulators
}

int lora_proj_bwd(const void* x, const void* w, const void* lora_a, const void* lora_b, const void* dy, void* dx,
                  void* d_lora_a, void* d_lora_b, int T, int K, int n_out, int parts, int r, float scaling,
                  void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 1 || K < 8 || K % 8 != 0 || n_out < 1 || parts < 1 || r < 0 || r > s2::kLoraMaxRank)
    return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(dy) || !aligned16(dx)) return S2ATTN_ERR_INVALID_ARG;
  if (r > 0 && (!aligned16(lora_a) || !lora_b || !d_lora_a || !d_lora_b || !std::isfinite(scaling)))
    return S2ATTN_ERR_INVALID_ARG;
  if (n_out % s2::kLoraProjTileN != 0) return S2ATTN_ERR_UNSUPPORTED;
  if (K < 64) return S2ATTN_ERR_UNSUPPORTED;   // the tensor maps' 64-column boxes must fit in a row of x and W
  if ((long long)parts * n_out > INT_MAX || (long long)T + 128 > INT_MAX) return S2ATTN_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return S2ATTN_ERR_WORKSPACE;
  if (workspace_bytes < lora_proj_bwd_workspace_bytes(T, K, n_out, parts, r)) return S2ATTN_ERR_WORKSPACE;
  int* err = error_word_ptr();
  if (!err) return S2ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const size_t ub = lora_u_bytes(T, parts);
  void* u = ws;
  void* g = ws + ub;
  void* a_pad = ws + 2 * ub;
  void* b_pad = static_cast<char*>(a_pad) + align256((size_t)parts * s2::kLoraRankPad * K * 2);
  float* da_acc = reinterpret_cast<float*>(static_cast<char*>(b_pad) +
                                           align256((size_t)parts * n_out * s2::kLoraRankPad * 2));
  float* db_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(da_acc) +
                                           align256((size_t)((parts * s2::kLoraRankPad + 127) / 128) * 128 * K * 4));
  const int RP = s2::kLoraRankPad;
  CUtensorMap dy_k, dy_mn, bpad, w_mn, g_k, apad, g_mn, x_mn, u_mn, tx, ta;
  bool ok = map_rows_bf16(&dy_k, dy, 3, n_out, T, parts, 64, 128) && map_rows_bf16(&dy_mn, dy, 3, n_out, T, parts, 64, 64) &&
            map_rows_bf16(&w_mn, w, 3, K, n_out, parts, 64, 64) && map_rows_bf16(&x_mn, x, 3, K, T, 1, 64, 64);
  if (r > 0)
    ok = ok && map_rows_bf16(&bpad, b_pad, 3, RP, n_out, parts, 64, 64) && map_rows_bf16(&g_k, g, 3, RP, T, parts, 64, 128) &&
         map_rows_bf16(&apad, a_pad, 3, K, RP, parts, 64, 64) && map_rows_bf16(&g_mn, g, 3, RP, T, parts, 64, 64) &&
         map_rows_bf16(&u_mn, u, 3, RP, T, parts, 64, 64) && map_rows_bf16(&tx, x, 2, K, T, 1, 64, 128) &&
         map_rows_bf16(&ta, a_pad, 2, K, (uint64_t)parts * RP, 1, 64, RP);
  else
    bpad = g_k = apad = g_mn = u_mn = dy_k;   // unused without an adapter
  if (!ok) return S2ATTN_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  if (r > 0) {
    e = s2::launch_lora_pad(lora_a, lora_b, a_pad, b_pad, parts, r, K, n_out, st);
    if (e == cudaSuccess) e = s2::launch_lora_down(tx, ta, u, T, K, parts, scaling, sm_count(), err, st);
    if (e != cudaSuccess) return S2ATTN_ERR_CUDA;
  }
  return cuda_status(s2::launch_lora_bwd(dy_k, dy_mn, bpad, w_mn, g_k, apad, g_mn, x_mn, u_mn, g, dx, da_acc, db_acc,
                                         d_lora_a, d_lora_b, T, K, n_out, parts, r, scaling, sm_count(), err, st));
}

int s2attn_selftest_bounded_wait(unsigned timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return S2ATTN_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (!err) return S2ATTN_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, 1000ull * timeout_us);
  return cuda_status(cudaGetLastError());
}

int s2attn_get_device_error(int* detail) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return S2ATTN_ERR_CUDA;
  if (detail) *detail = v;
  return v == 0 ? S2ATTN_OK : S2ATTN_ERR_DEVICE_TIMEOUT;
}

int s2attn_clear_device_error(void) {
  const int zero = 0;
  return cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) == cudaSuccess ? S2ATTN_OK : S2ATTN_ERR_CUDA;
}

}  // extern "C"
