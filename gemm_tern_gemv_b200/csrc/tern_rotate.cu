// Activation-side block Hadamard rotation y = R x, R = H_1024 S / 32, per 1024-element block of each
// row ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "블록 단위 하다마드 회전": the weights
// live in the basis R = H_n S / sqrt(n), n = 1024, and each layer computes W (R x); section "처리량":
// every projection is preceded by the sign flip and a block fast Walsh-Hadamard transform, which the
// CUDA backend spreads over a whole thread block).
//
// One CTA of 128 threads per block: thread t holds elements t + 128 r (r = 0..7) in fp32, applies
// the sign as it loads, and runs the ten butterfly stages of the Sylvester-order transform: the
// three on index bits 7-9 inside its registers, the five on bits 0-4 with warp shuffles, the two on
// bits 5-6 through shared memory. The result is scaled by 1/32 and rounded once to fp16. Every
// element of a block is read before any is written, so y may alias x.
#include <cuda_fp16.h>

#include "tern_fwht.cuh"
#include "tern_internal.cuh"

namespace tern {
namespace {

__global__ void __launch_bounds__(kRotThreads) rotate_kernel(const uint16_t* x, const int8_t* __restrict__ signs,
                                                             uint16_t* y, int64_t k, int nblk) {
  __shared__ float sh[kRotBlock];
  const int blk = blockIdx.x % nblk;
  const int64_t row = blockIdx.x / nblk;
  const int t = threadIdx.x;
  const int64_t base = row * k + (int64_t)blk * kRotBlock;
  float v[8];
#pragma unroll
  for (int r = 0; r < 8; r++) {
    const int i = t + kRotThreads * r;
    const float xv = __half2float(__ushort_as_half(x[base + i]));
    v[r] = signs[i] < 0 ? -xv : xv;
  }
  fwht1024(v, sh, t, SyncCta{});
#pragma unroll
  for (int r = 0; r < 8; r++)
    y[base + t + kRotThreads * r] = __half_as_ushort(__float2half_rn(v[r] * 0.03125f));
}

}  // namespace

cudaError_t launch_rotate(const uint16_t* x, int64_t batch, int64_t k, const int8_t* signs, uint16_t* y,
                          cudaStream_t st) {
  const int nblk = (int)(k / kRotBlock);
  const int64_t ctas = batch * nblk;
  rotate_kernel<<<(unsigned)ctas, kRotThreads, 0, st>>>(x, signs, y, k, nblk);
  return cudaGetLastError();
}

}  // namespace tern
