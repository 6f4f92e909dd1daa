// s2attn_halo.cu -- the halo rows of sequence-sharded S^2-Attn.
//
// Method ("LongLoRA paper notes", section 3.3; nearauto.com article, "shift short
// attention" steps (1) and (2)): groups of G tokens are independent, so a sequence split
// across ranks in whole groups needs one exchange.  A rank holds tokens [t0, t0 + Np) of
// every head.  The rolled groups of a shifted head start G/2 tokens into the rank's run,
// so its last one ends G/2 tokens into the next rank's run (cyclically), and the rank's
// own first G/2 rows of the shifted heads belong to the previous rank's last group.
//
// The attention kernels roll a shifted head cyclically inside the tensors they are given:
// rolled row r is local token (r + G/2) mod Np.  Their last rolled group therefore reads
// the rank's own tail followed by its own rows [0, G/2) -- exactly the rows that the
// previous rank needs and this rank does not.  So the sharded path puts the next rank's
// first G/2 rows (the halo) in place of those rows for the duration of a call, runs the
// unmodified kernels with the shift, and restores the rows afterwards; the results that
// land in rows [0, G/2) belong to the halo's tokens and travel back to their owner.
// Only G/2 rows of the shifted heads per tensor move; no local copy of a whole tensor is
// made.  These kernels are the two copies that step needs:
//   rows  [B, N, H, D] bf16 <-> buf [B, G/2, S, D]   rows [0, G/2) of heads [H-S, H)
//   lse   [B, H, N]    fp32 <-> buf [B, S, G/2]      the same rows of the softmax statistics
// with S = shift_heads.  One launch moves up to kHaloMaxTensors tensors.
#include <cstdint>

#include "s2_internal.h"

namespace s2 {
namespace halo {

struct RowsArgs {
  uint4* x[kHaloMaxTensors];
  uint4* buf[kHaloMaxTensors];
};
struct LseArgs {
  float* x[kHaloMaxTensors];
  float* buf[kHaloMaxTensors];
};

// One thread moves 16 bytes (8 bf16 elements of a row of D).  blockIdx.y selects the tensor.
__global__ void __launch_bounds__(256) rows_kernel(const RowsArgs a, int to_buf, int B, int N, int H, int cpr,
                                                   int half, int hs) {
  const int S = H - hs;
  const long long total = (long long)B * half * S * cpr;
  uint4* x = a.x[blockIdx.y];
  uint4* buf = a.buf[blockIdx.y];
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(w % cpr);
    long long rest = w / cpr;
    const int s = (int)(rest % S);
    rest /= S;
    const int i = (int)(rest % half);
    const int b = (int)(rest / half);
    const long long xi = (((long long)b * N + i) * H + hs + s) * cpr + c;
    if (to_buf)
      buf[w] = x[xi];
    else
      x[xi] = buf[w];
  }
}

__global__ void __launch_bounds__(256) lse_kernel(const LseArgs a, int to_buf, int B, int N, int H, int half,
                                                  int hs) {
  const int S = H - hs;
  const long long total = (long long)B * S * half;
  float* x = a.x[blockIdx.y];
  float* buf = a.buf[blockIdx.y];
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(w % half);
    long long rest = w / half;
    const int s = (int)(rest % S);
    const int b = (int)(rest / S);
    const long long xi = ((long long)b * H + hs + s) * N + i;
    if (to_buf)
      buf[w] = x[xi];
    else
      x[xi] = buf[w];
  }
}

int grid_x(long long total, int n_sm) {
  const long long blocks = (total + 255) / 256;
  const long long cap = 8LL * (n_sm > 0 ? n_sm : 148);
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace halo

cudaError_t launch_halo_rows(void* const* x, void* const* buf, int n, int to_buf, int B, int N, int H, int D,
                             int G, int shift_heads, int n_sm, cudaStream_t st) {
  halo::RowsArgs a{};
  for (int i = 0; i < n; ++i) {
    a.x[i] = static_cast<uint4*>(x[i]);
    a.buf[i] = static_cast<uint4*>(buf[i]);
  }
  const int cpr = D * 2 / 16;
  const long long total = (long long)B * (G / 2) * shift_heads * cpr;
  dim3 grid(halo::grid_x(total, n_sm), n);
  halo::rows_kernel<<<grid, 256, 0, st>>>(a, to_buf, B, N, H, cpr, G / 2, H - shift_heads);
  return cudaGetLastError();
}

cudaError_t launch_halo_lse(float* const* x, float* const* buf, int n, int to_buf, int B, int N, int H, int G,
                            int shift_heads, int n_sm, cudaStream_t st) {
  halo::LseArgs a{};
  for (int i = 0; i < n; ++i) {
    a.x[i] = x[i];
    a.buf[i] = buf[i];
  }
  const long long total = (long long)B * shift_heads * (G / 2);
  dim3 grid(halo::grid_x(total, n_sm), n);
  halo::lse_kernel<<<grid, 256, 0, st>>>(a, to_buf, B, N, H, G / 2, H - shift_heads);
  return cudaGetLastError();
}

}  // namespace s2
