// Transposed ternary product dx[b][k] = sum_n s[n][k/128] t[n][k] dy[b][n], the input gradient of the
// straight-through-estimator backward of a ternary layer ("Metal 환경에서 ... Bonsai 8B를
// 파인튜닝", molayo1419.me, paragraph "그것을 파인튜닝하는 방법": gradients flow through the
// ternarized forward to the latent weights and the layer input).
//
// The contraction runs over the rows of W, so a warp reads whole rows: CTA (column block, row slice)
// covers 64 code bytes of every row of its slice (256 columns of Q2_0_g128, 320 of base-3, 512 of
// the binary Q1_0_g128); thread t owns byte t % 64 of rows t / 64, t / 64 + 4, ... and accumulates its
// 4, 5 or 8 columns for every batch row in fp32 with s * dy formed once per row. The four row phases
// of a CTA are summed through shared memory in two halving steps; row slices write fp32 partials that a second kernel sums in slice order
// (deterministic), or the single slice stores dx directly.
#include <cuda_fp16.h>

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kTThreads = 256;
constexpr int kTBytes = 64;  // code bytes of a row per column block

template <int LAYOUT> constexpr int cols_per_byte() {
  return LAYOUT == TERN_Q2_0_G128 ? 4 : LAYOUT == TERN_Q1_0_G128 ? 8 : 5;
}
constexpr int kPhases = kTThreads / kTBytes;

template <int LAYOUT, int BATCH>
__global__ void __launch_bounds__(kTThreads) gemv_t_kernel(const uint8_t* __restrict__ codes, int64_t cstride,
                                                           const uint16_t* __restrict__ scales, int64_t sstride,
                                                           const uint16_t* __restrict__ dy, int batch, int64_t n,
                                                           int64_t k, int64_t rows_per_slice, float* part,
                                                           uint16_t* dx) {
  constexpr int C = cols_per_byte<LAYOUT>();
  __shared__ float red[kPhases / 2][kTBytes * C][BATCH];
  const int t = threadIdx.x, phase = t / kTBytes, byte = t % kTBytes;
  const int64_t col0 = (int64_t)blockIdx.x * kTBytes * C + (int64_t)byte * C;  // first column of this byte
  const int64_t n0 = (int64_t)blockIdx.y * rows_per_slice;
  const int64_t n1 = n0 + rows_per_slice < n ? n0 + rows_per_slice : n;
  const int64_t byte_off = (int64_t)blockIdx.x * kTBytes + byte;
  const int64_t data_bytes = LAYOUT == TERN_Q2_0_G128 ? k / 4 : LAYOUT == TERN_Q1_0_G128 ? k / 8 : (k + 4) / 5;
  // groups of this byte's columns (a base-3 byte can straddle two 128-column groups)
  const int64_t g_first = col0 / kGroup, g_last = (col0 + C - 1) / kGroup;
  float acc[C][BATCH];
#pragma unroll
  for (int i = 0; i < C; i++)
#pragma unroll
    for (int b = 0; b < BATCH; b++) acc[i][b] = 0.f;
  if (byte_off < data_bytes) {
    for (int64_t r = n0 + phase; r < n1; r += kTThreads / kTBytes) {
      uint32_t v = __ldg(codes + r * cstride + byte_off);
      const float s0 = __half2float(__ushort_as_half(__ldg(scales + r * sstride + g_first)));
      const float s1 = (g_last != g_first && g_last < k / kGroup)
                           ? __half2float(__ushort_as_half(__ldg(scales + r * sstride + g_last))) : s0;
      float d[BATCH];
#pragma unroll
      for (int b = 0; b < BATCH; b++) d[b] = b < batch ? __half2float(__ushort_as_half(__ldg(dy + (int64_t)b * n + r))) : 0.f;
#pragma unroll
      for (int i = 0; i < C; i++) {
        float tv;
        if (LAYOUT == TERN_Q2_0_G128) {
          const uint32_t f = (v >> (2 * i)) & 3u;  // two's complement field; 0b10 (invalid) reads as 0
          tv = f == 1u ? 1.f : (f == 3u ? -1.f : 0.f);
        } else if (LAYOUT == TERN_Q1_0_G128) {
          tv = (v >> i) & 1u ? 1.f : -1.f;  // sign bit, 1 = +1
        } else {
          const uint32_t c = v % 3u;  // digit i, c = t + 1 (an invalid byte gives unspecified t)
          v /= 3u;
          tv = (float)((int)c - 1);
        }
        const float sc = (col0 + i) / kGroup == g_first ? s0 : s1;
#pragma unroll
        for (int b = 0; b < BATCH; b++) acc[i][b] = fmaf(tv, sc * d[b], acc[i][b]);
      }
    }
  }
  // sum the four row phases: phases 2, 3 hand their sums to phases 0, 1, which store theirs added
  if (phase >= kPhases / 2) {
#pragma unroll
    for (int i = 0; i < C; i++)
#pragma unroll
      for (int b = 0; b < BATCH; b++) red[phase - kPhases / 2][byte * C + i][b] = acc[i][b];
  }
  __syncthreads();
  if (phase < kPhases / 2) {
#pragma unroll
    for (int i = 0; i < C; i++)
#pragma unroll
      for (int b = 0; b < BATCH; b++) red[phase][byte * C + i][b] += acc[i][b];
  }
  __syncthreads();
  for (int e = t; e < kTBytes * C * BATCH; e += kTThreads) {
    const int c = e / BATCH, b = e % BATCH;
    const int64_t col = (int64_t)blockIdx.x * kTBytes * C + c;
    if (b >= batch || col >= k) continue;
    float v = 0.f;
#pragma unroll
    for (int p = 0; p < kPhases / 2; p++) v += red[p][c][b];
    if (part) part[((int64_t)blockIdx.y * batch + b) * k + col] = v;
    else dx[(int64_t)b * k + col] = __half_as_ushort(__float2half_rn(v));
  }
}

__global__ void __launch_bounds__(256) gemv_t_reduce(const float* __restrict__ part, int slices, int64_t total,
                                                     uint16_t* dx) {
  for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < total; e += (int64_t)gridDim.x * 256) {
    float v = 0.f;
    for (int s = 0; s < slices; s++) v += part[(int64_t)s * total + e];
    dx[e] = __half_as_ushort(__float2half_rn(v));
  }
}

template <int LAYOUT, int BATCH>
cudaError_t launch_t(const tern_matrix& W, const uint16_t* dy, int batch, uint16_t* dx, float* part,
                     const GemvTPlan& p, cudaStream_t st) {
  dim3 grid(p.col_blocks, p.slices);
  gemv_t_kernel<LAYOUT, BATCH><<<grid, kTThreads, 0, st>>>(static_cast<const uint8_t*>(W.codes), W.code_row_stride,
                                                          W.scales, W.scale_row_stride, dy, batch, W.n, W.k,
                                                          p.rows_per_slice, p.slices > 1 ? part : nullptr, dx);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.slices == 1) return e;
  const int64_t total = (int64_t)batch * W.k;
  const int64_t blocks = (total + 255) / 256;
  gemv_t_reduce<<<(unsigned)(blocks < 4 * sm_count() ? blocks : 4 * sm_count()), 256, 0, st>>>(part, p.slices,
                                                                                              total, dx);
  return cudaGetLastError();
}

template <int LAYOUT>
cudaError_t dispatch_t(const tern_matrix& W, const uint16_t* dy, int batch, uint16_t* dx, float* part,
                       const GemvTPlan& p, cudaStream_t st) {
  if (batch <= 1) return launch_t<LAYOUT, 1>(W, dy, batch, dx, part, p, st);
  if (batch <= 2) return launch_t<LAYOUT, 2>(W, dy, batch, dx, part, p, st);
  if (batch <= 4) return launch_t<LAYOUT, 4>(W, dy, batch, dx, part, p, st);
  return launch_t<LAYOUT, 8>(W, dy, batch, dx, part, p, st);
}

}  // namespace

GemvTPlan gemv_t_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  GemvTPlan p{};
  const int64_t cols = (int64_t)kTBytes * (layout == TERN_Q2_0_G128 ? 4 : layout == TERN_Q1_0_G128 ? 8 : 5);
  p.col_blocks = (int)((k + cols - 1) / cols);
  // about two CTAs per SM; every slice keeps at least 64 rows
  int64_t slices = (2 * (int64_t)sms + p.col_blocks - 1) / p.col_blocks;
  slices = std::max<int64_t>(1, std::min<int64_t>(slices, (n + 63) / 64));
  p.rows_per_slice = (n + slices - 1) / slices;
  p.slices = (int)((n + p.rows_per_slice - 1) / p.rows_per_slice);
  p.ws_bytes = p.slices > 1 ? (size_t)p.slices * batch * k * sizeof(float) : 0;
  return p;
}

cudaError_t launch_gemv_t(const tern_matrix& W, const uint16_t* dy, int batch, uint16_t* dx, void* workspace,
                          const GemvTPlan& plan, cudaStream_t st) {
  float* part = static_cast<float*>(workspace);
  if (W.layout == TERN_Q2_0_G128) return dispatch_t<TERN_Q2_0_G128>(W, dy, batch, dx, part, plan, st);
  if (W.layout == TERN_Q1_0_G128) return dispatch_t<TERN_Q1_0_G128>(W, dy, batch, dx, part, plan, st);
  return dispatch_t<TERN_T3_5PB_G128>(W, dy, batch, dx, part, plan, st);
}

}  // namespace tern
