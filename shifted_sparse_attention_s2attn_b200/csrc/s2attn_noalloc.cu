// s2attn_noalloc.cu -- the backward pass for callers that cannot allocate device memory.
//
// s2attn_bwd needs a caller-provided workspace (an fp32 dQ accumulator and the
// per-row delta).  Some callers cannot produce one on the call path: a runtime whose
// allocator has already reserved the device's memory for itself, a plugin interface
// whose enqueue step must not allocate, or a latency-critical loop where cudaMalloc's
// implicit device-wide synchronisation is not acceptable.  s2attn_bwd_noalloc runs the
// same three kernels with the workspace taken from a fixed-size array that lives in
// this file's device module instead, and allocates nothing.
#include <cstdint>
#include <mutex>

#include "s2_internal.h"
#include "s2attn.h"

namespace {

// The scratch: S2ATTN_NOALLOC_SCRATCH_BYTES per device, reserved when this file's module is
// loaded on a device and held until the process exits.  Every call shares it.  Under CUDA's
// lazy module loading (the default) the module is loaded by the first address lookup below,
// i.e. inside the first call on each device: that call is where the memory is taken.
static __device__ __align__(256) unsigned char g_bwd_scratch[S2ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of g_bwd_scratch on the current device.  In host code the array's
// name only stands for the symbol, so the address is looked up once per device with
// that device current, and cached.
void* scratch_ptr() {
  static std::mutex mu;
  static void* cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess) return nullptr;
    cache[dev] = p;
  }
  return cache[dev];
}

}  // namespace

extern "C" int s2attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                  const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int D, int G,
                                  int shift_heads, void* stream) {
  // The argument rules of s2attn_bwd (the same check, overflow guards included), applied
  // here so that nothing is enqueued on error.
  int rc = s2::check_tensor_core_args(B, N, H, D, G, shift_heads);
  if (rc) return rc;
  const void* ptrs[] = {q, k, v, o, dout, lse, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!ptr || (reinterpret_cast<uintptr_t>(ptr) & 15u)) return S2ATTN_ERR_INVALID_ARG;
  const size_t elems = (size_t)B * N * H * D;
  const size_t acc_bytes = align256(elems * sizeof(float));
  if (acc_bytes + align256((size_t)B * H * N * sizeof(float)) > (size_t)S2ATTN_NOALLOC_SCRATCH_BYTES)
    return S2ATTN_ERR_WORKSPACE;  // the problem does not fit the fixed scratch
  char* base = static_cast<char*>(scratch_ptr());
  if (!base) return S2ATTN_ERR_CUDA;
  float* dq_acc = reinterpret_cast<float*>(base);
  float* delta = reinterpret_cast<float*>(base + acc_bytes);
  // The accumulator is zeroed by the preprocess stage on every call, so nothing left
  // in the scratch by an earlier call leaks into this one.
  if ((rc = s2attn_bwd_preprocess(o, dout, delta, dq_acc, B, N, H, D, stream))) return rc;
  if ((rc = s2attn_bwd_main(q, k, v, dout, lse, delta, dq_acc, dk, dv, B, N, H, D, G, shift_heads, stream)))
    return rc;
  return s2attn_bwd_dq_convert(dq_acc, dq, B, N, H, D, stream);
}
