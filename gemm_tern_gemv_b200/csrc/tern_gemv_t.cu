// Transposed ternary product dx[b][k] = sum_n s[n][k/128] t[n][k] dy[b][n], the input gradient of the
// straight-through-estimator backward of a ternary layer ("Metal 환경에서 ... Bonsai 8B를
// 파인튜닝", molayo1419.me, paragraph "그것을 파인튜닝하는 방법": gradients flow through the
// ternarized forward to the latent weights and the layer input).
//
// The contraction runs over the rows of W, so the kernel streams whole rows with vector loads:
//   * A warp covers a column block of 32 x LB bytes of every row it reads (LB = 16 / B bytes per lane,
//     8 / B for the binary layout, B = the batch rounded up to 1, 2, 4 or 8), one LB-byte load per lane
//     and row. Each lane keeps fp32 accumulators for its 64 (Q2_0_g128, binary) or 80 (base-3) / B
//     columns and all B batch rows.
//   * Decode straight to fp32: a two's-complement field moved to bits 30..31 of a float is +-2.0 or 0
//     (sign and exponent MSB), so a multiply (the shift) and a mask give 2t exactly; a binary sign bit
//     moved to bit 31 and XOR-ed with 0xC0000000 gives +-2.0. The FFMA multiplies by s * dy / 2, which
//     is exact in fp32, so every product is exact and only the fp32 sums round.
//   * The 8 warps of a CTA read interleaved rows of the same column block and are summed through
//     shared memory in warp order; row slices write fp32 partials that a second kernel sums in slice
//     order (deterministic), or the single slice stores dx directly.
#include <cuda_fp16.h>

#include "tern_internal.cuh"
#include "tern_t3.cuh"

namespace tern {
namespace {

constexpr int kTWarps = 8;
constexpr int kTThreads = kTWarps * 32;

template <int LAYOUT> constexpr int cols_per_byte() {
  return LAYOUT == TERN_Q2_0_G128 ? 4 : LAYOUT == TERN_Q1_0_G128 ? 8 : 5;
}
template <int LAYOUT, int B> constexpr int lane_bytes() { return (LAYOUT == TERN_Q1_0_G128 ? 8 : 16) / B; }
template <int LAYOUT, int B> constexpr size_t red_bytes() {
  return (size_t)kTWarps * 32 * lane_bytes<LAYOUT, B>() * cols_per_byte<LAYOUT>() * B * sizeof(float);
}

// The LB code bytes of a lane as little-endian 32-bit words (bytes past LB read as zero).
template <int LB>
__device__ __forceinline__ void load_codes(const uint8_t* p, uint32_t (&w)[(LB + 3) / 4]) {
  if constexpr (LB == 16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (LB == 8) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (LB == 4) {
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
  } else if constexpr (LB == 2) {
    w[0] = __ldg(reinterpret_cast<const unsigned short*>(p));
  } else {
    w[0] = __ldg(p);
  }
}

template <int LAYOUT, int B>
__global__ void __launch_bounds__(kTThreads) gemv_t_kernel(const uint8_t* __restrict__ codes, int64_t cstride,
                                                           const uint16_t* __restrict__ scales, int64_t sstride,
                                                           const uint16_t* __restrict__ dy, int batch, int64_t n,
                                                           int64_t k, int64_t row_bytes, int64_t rows_per_slice,
                                                           float* part, uint16_t* dx) {
  constexpr int LB = lane_bytes<LAYOUT, B>();
  constexpr int CPB = cols_per_byte<LAYOUT>();
  constexpr int CL = LB * CPB;  // columns of one lane
  constexpr int NWD = (LB + 3) / 4;
  extern __shared__ float red[];  // [warp][lane * CL + column][B]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t byte0 = ((int64_t)blockIdx.x * 32 + lane) * LB;  // this lane's first byte of a row
  const int64_t col0 = byte0 * CPB;
  const int64_t n0 = (int64_t)blockIdx.y * rows_per_slice;
  const int64_t n1 = n0 + rows_per_slice < n ? n0 + rows_per_slice : n;
  const int64_t groups = k / kGroup;
  // a base-3 lane's 80 columns can straddle two groups: columns before `split` use the first scale
  const int64_t g_first = col0 / kGroup;
  const int64_t g_last = (col0 + CL - 1) / kGroup < groups ? (col0 + CL - 1) / kGroup : g_first;
  const int split = (int)((g_first + 1) * kGroup - col0);

  float acc[CL][B];
#pragma unroll
  for (int c = 0; c < CL; c++)
#pragma unroll
    for (int b = 0; b < B; b++) acc[c][b] = 0.f;

  // byte0 and row_bytes are multiples of LB, so a lane with byte0 < row_bytes reads inside the row
  if (byte0 < row_bytes && g_first < groups) {
    const uint32_t k0 = (130u | (130u << 16)) + 0xC000C000u;
    for (int64_t r = n0 + warp; r < n1; r += kTWarps) {
      uint32_t w[NWD];
      load_codes<LB>(codes + r * cstride + byte0, w);
      const float s0 = __half2float(__ushort_as_half(__ldg(scales + r * sstride + g_first)));
      const float s1 = g_last != g_first ? __half2float(__ushort_as_half(__ldg(scales + r * sstride + g_last))) : s0;
      float sd0[B], sd1[B];
#pragma unroll
      for (int b = 0; b < B; b++) {
        const float d = b < batch ? __half2float(__ushort_as_half(__ldg(dy + (int64_t)b * n + r))) : 0.f;
        sd0[b] = 0.5f * s0 * d;  // exact: products of fp16 values fit fp32
        sd1[b] = 0.5f * s1 * d;
      }
      if constexpr (LAYOUT == TERN_Q2_0_G128) {
#pragma unroll
        for (int c = 0; c < CL; c++) {  // field c % 16 of word c / 16 is column c
          const float tv = __uint_as_float((w[c / 16] * (1u << (30 - 2 * (c % 16)))) & 0xC0000000u);
#pragma unroll
          for (int b = 0; b < B; b++) acc[c][b] = fmaf(tv, sd0[b], acc[c][b]);
        }
      } else if constexpr (LAYOUT == TERN_Q1_0_G128) {
#pragma unroll
        for (int c = 0; c < CL; c++) {  // bit c % 32 of word c / 32 is column c
          const float tv = __uint_as_float(((w[c / 32] * (1u << (31 - (c % 32)))) & 0x80000000u) ^ 0xC0000000u);
#pragma unroll
          for (int b = 0; b < B; b++) acc[c][b] = fmaf(tv, sd0[b], acc[c][b]);
        }
      } else {
#pragma unroll
        for (int wd = 0; wd < NWD; wd++) {
          uint32_t o[10];
          dec_t3_word(w[wd], k0, o);
#pragma unroll
          for (int h = 0; h < 2; h++)
#pragma unroll
            for (int i = 0; i < 5; i++)
#pragma unroll
              for (int hi = 0; hi < 2; hi++) {
                // byte h (low half) or 2 + h (high half) of the word, digit 4 - i
                const int c = 5 * (4 * wd + h + 2 * hi) + (4 - i);
                if (c < CL) {
                  const float tv = __uint_as_float(hi ? (o[5 * h + i] & 0xC0000000u) : (o[5 * h + i] << 16));
#pragma unroll
                  for (int b = 0; b < B; b++) acc[c][b] = fmaf(tv, c < split ? sd0[b] : sd1[b], acc[c][b]);
                }
              }
        }
      }
    }
  }
  // sum the warps' row phases in warp order
  float* mine = red + (size_t)warp * 32 * CL * B + (size_t)lane * CL * B;
#pragma unroll
  for (int c = 0; c < CL; c++)
#pragma unroll
    for (int b = 0; b < B; b++) mine[c * B + b] = acc[c][b];
  __syncthreads();
  for (int e = threadIdx.x; e < 32 * CL * B; e += kTThreads) {
    const int cl = e / B, b = e % B;
    const int64_t col = (int64_t)blockIdx.x * 32 * CL + cl;
    if (b >= batch || col >= k) continue;
    float v = 0.f;
#pragma unroll
    for (int p = 0; p < kTWarps; p++) v += red[(size_t)p * 32 * CL * B + e];
    if (part) part[((int64_t)blockIdx.y * batch + b) * k + col] = v;
    else dx[(int64_t)b * k + col] = __half_as_ushort(__float2half_rn(v));
  }
}

// Sums the slices' fp32 partials of 32 consecutive outputs per CTA: the 8 warps take every eighth
// slice (loads of one warp are 128 contiguous bytes, four in flight per lane), then one warp adds the
// 8 warp sums. The order is fixed (slices sg, sg + 8, ... within warp sg, then warps 0..7), so the
// result depends only on the inputs.
__global__ void __launch_bounds__(256) gemv_t_reduce(const float* __restrict__ part, int slices, int64_t total,
                                                     uint16_t* dx) {
  __shared__ float red[8][33];
  const int c = threadIdx.x & 31, sg = threadIdx.x >> 5;
  for (int64_t e0 = (int64_t)blockIdx.x * 32; e0 < total; e0 += (int64_t)gridDim.x * 32) {
    const int64_t e = e0 + c;
    float v = 0.f;
    if (e < total) {
#pragma unroll 4
      for (int s = sg; s < slices; s += 8) v += part[(int64_t)s * total + e];
    }
    red[sg][c] = v;
    __syncthreads();
    if (sg == 0 && e < total) {
      float t = red[0][c];
#pragma unroll
      for (int j = 1; j < 8; j++) t += red[j][c];
      dx[e] = __half_as_ushort(__float2half_rn(t));
    }
    __syncthreads();
  }
}

int batch_slots(int64_t batch) { return batch <= 1 ? 1 : batch <= 2 ? 2 : batch <= 4 ? 4 : 8; }

template <int LAYOUT, int B>
cudaError_t launch_t(const tern_matrix& W, const uint16_t* dy, int batch, uint16_t* dx, float* part,
                     const GemvTPlan& p, cudaStream_t st) {
  constexpr size_t smem = red_bytes<LAYOUT, B>();
  auto kern = gemv_t_kernel<LAYOUT, B>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.col_blocks, p.slices);
  kern<<<grid, kTThreads, smem, st>>>(static_cast<const uint8_t*>(W.codes), W.code_row_stride, W.scales,
                                      W.scale_row_stride, dy, batch, W.n, W.k, row_bytes(W.layout, W.k),
                                      p.rows_per_slice, p.slices > 1 ? part : nullptr, dx);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.slices == 1) return e;
  const int64_t total = (int64_t)batch * W.k;
  const int64_t blocks = (total + 31) / 32;
  gemv_t_reduce<<<(unsigned)(blocks < 8 * sm_count() ? blocks : 8 * sm_count()), 256, 0, st>>>(part, p.slices,
                                                                                              total, dx);
  return cudaGetLastError();
}

template <int LAYOUT>
cudaError_t dispatch_t(const tern_matrix& W, const uint16_t* dy, int batch, uint16_t* dx, float* part,
                       const GemvTPlan& p, cudaStream_t st) {
  switch (batch_slots(batch)) {
    case 1: return launch_t<LAYOUT, 1>(W, dy, batch, dx, part, p, st);
    case 2: return launch_t<LAYOUT, 2>(W, dy, batch, dx, part, p, st);
    case 4: return launch_t<LAYOUT, 4>(W, dy, batch, dx, part, p, st);
    default: return launch_t<LAYOUT, 8>(W, dy, batch, dx, part, p, st);
  }
}

}  // namespace

// Column blocks of 32 lanes x LB bytes; row slices so that about two CTAs run per SM, each warp
// reading at least 8 rows of its slice.
GemvTPlan gemv_t_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  GemvTPlan p{};
  const int64_t lb = (layout == TERN_Q1_0_G128 ? 8 : 16) / batch_slots(batch);
  const int64_t block_bytes = 32 * lb;
  p.col_blocks = (int)((row_bytes(layout, k) + block_bytes - 1) / block_bytes);
  int64_t slices = (2 * (int64_t)sms + p.col_blocks - 1) / p.col_blocks;
  slices = std::max<int64_t>(1, std::min<int64_t>(slices, (n + 8 * kTWarps - 1) / (8 * kTWarps)));
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
