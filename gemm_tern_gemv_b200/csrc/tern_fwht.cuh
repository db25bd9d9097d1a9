// Sign flip + Sylvester-order fast Walsh-Hadamard transform of one 1024-element block by 128 threads
// ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "블록 단위 하다마드 회전": R = H_n S / sqrt(n),
// n = 1024, applied to x before each projection). Shared by the rotation kernel and the GEMV that
// rotates x while it builds its activation fragments, so that both produce the same fp32 values.
#pragma once

#include <cstdint>

namespace tern {

constexpr int kRotBlock = 1024;
constexpr int kRotThreads = 128;

// v[r] holds element t + 128 r of the block (t = thread index within the 128, sign already applied).
// The ten butterfly stages (a, b) -> (a + b, a - b), a the element whose index bit is clear: the three
// on index bits 7-9 inside the registers, the five on bits 0-4 with warp shuffles, the two on bits 5-6
// through sh (1024 floats of shared memory). sync() must synchronize exactly these 128 threads.
template <class Sync>
__device__ __forceinline__ void fwht1024(float (&v)[8], float* sh, int t, Sync sync) {
  const int lane = t & 31, warp = t >> 5;
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
    sync();
#pragma unroll
    for (int r = 0; r < 8; r++) {
      const float p = sh[(t ^ (m << 5)) + kRotThreads * r];
      v[r] = (warp & m) ? p - v[r] : v[r] + p;
    }
    sync();
  }
}

// The two synchronizations fwht1024 is used with: the whole CTA of 128 threads, or one group of
// 128 threads (4 whole warps) of a larger CTA on its own named barrier (ids 1..15; 0 is __syncthreads).
struct SyncCta {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct SyncGroup128 {
  int id;
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
};

}  // namespace tern
