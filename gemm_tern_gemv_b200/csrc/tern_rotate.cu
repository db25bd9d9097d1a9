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

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kRotBlock = 1024;
constexpr int kRotThreads = 128;

__global__ void __launch_bounds__(kRotThreads) rotate_kernel(const uint16_t* x, const int8_t* __restrict__ signs,
                                                             uint16_t* y, int64_t k, int nblk) {
  __shared__ float sh[kRotBlock];
  const int blk = blockIdx.x % nblk;
  const int64_t row = blockIdx.x / nblk;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t base = row * k + (int64_t)blk * kRotBlock;
  float v[8];
#pragma unroll
  for (int r = 0; r < 8; r++) {
    const int i = t + kRotThreads * r;
    const float xv = __half2float(__ushort_as_half(x[base + i]));
    v[r] = signs[i] < 0 ? -xv : xv;
  }
  // butterflies (a, b) -> (a + b, a - b), a the element whose index bit is clear
#pragma unroll
  for (int m = 1; m < 8; m <<= 1)  // index bits 7..9: register index r
#pragma unroll
    for (int r = 0; r < 8; r++)
      if (!(r & m)) {
        const float a = v[r], b = v[r | m];
        v[r] = a + b;
        v[r | m] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1)  // index bits 0..4: lane
#pragma unroll
    for (int r = 0; r < 8; r++) {
      const float p = __shfl_xor_sync(0xFFFFFFFFu, v[r], m);
      v[r] = (lane & m) ? p - v[r] : v[r] + p;
    }
#pragma unroll
  for (int m = 1; m < 4; m <<= 1) {  // index bits 5..6: warp
#pragma unroll
    for (int r = 0; r < 8; r++) sh[t + kRotThreads * r] = v[r];
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; r++) {
      const float p = sh[(t ^ (m << 5)) + kRotThreads * r];
      v[r] = (warp & m) ? p - v[r] : v[r] + p;
    }
    __syncthreads();
  }
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
