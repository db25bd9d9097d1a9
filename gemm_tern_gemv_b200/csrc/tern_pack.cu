// Ternarize-and-pack and unpack kernels for the packed layouts.
//
// All are HBM-streaming kernels: one thread owns one 16-byte chunk of a packed row (64 weights
// for Q2_0_g128, 80 for base-3, 128 for the binary Q1_0_g128), reads or writes the matching fp16 weights with 16-byte vectors,
// and the grid is sized in whole waves of the SM count with a grid-stride loop.
//
// Ternarize rule (QAT re-ternarize step of "Metal 환경에서 ... Bonsai 8B를 파인튜닝", molayo1419.me,
// paragraph "그것을 파인튜닝하는 방법"): t = round(clamp(w/s, -1, 1)), ties to even. For fp16 w
// and s the quotient test |w/s| > 1/2 is exactly 2|w| > |s| in fp32 (both sides are exact), so the
// kernel never divides: t = sign(w)*sign(s) when 2|w| > |s| and s != 0, else 0. NaN compares false
// and gives 0; an infinite w with finite non-zero s gives +-1; an infinite s gives 0.
#include <cuda_fp16.h>

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kThreads = 256;

// t in {-1, 0, +1} of one weight (as int)
__device__ __forceinline__ int ternary_value(uint16_t wbits, float s_abs, bool s_neg) {
  float w = __half2float(__ushort_as_half(wbits));
  bool big = (2.0f * fabsf(w) > s_abs) && (s_abs != 0.0f);
  return big ? (((w > 0.0f) != s_neg) ? 1 : -1) : 0;
}

// The base-3 and binary kernels decide two weights at a time, one per 16-bit lane of a 32-bit word of fp16 pairs.
// 0xFFFF in each lane where 2|w| > |s| (s2 = |s| in both lanes): doubling an fp16 value is exact
// unless it overflows, and then it is infinite, which is also the fp32 answer (2|w| > 65504 >= |s|);
// NaN compares false. The caller handles s = 0 (every t is 0).
__device__ __forceinline__ uint32_t big2(uint32_t pair, __half2 s2) {
  __half2 a;
  const uint32_t abs_bits = pair & 0x7FFF7FFFu;
  a = *reinterpret_cast<const __half2*>(&abs_bits);
  return __hgt2_mask(__hadd2(a, a), s2);
}
// 0xFFFF in each lane whose weight is neither +-0 nor NaN (the binary sign rule)
__device__ __forceinline__ uint32_t nonzero2(uint32_t pair) {
  const uint32_t abs_bits = pair & 0x7FFF7FFFu;
  return __hgt2_mask(*reinterpret_cast<const __half2*>(&abs_bits), __float2half2_rn(0.0f));
}
__device__ __forceinline__ uint32_t comp(const uint4& q, int e) { return e == 0 ? q.x : e == 1 ? q.y : e == 2 ? q.z : q.w; }

// ---- Q2_0_g128: chunk = 16 bytes = 64 weights, all inside one 128-weight group -------------
__global__ void __launch_bounds__(kThreads) pack_q2_kernel(const uint16_t* __restrict__ w, int64_t w_stride,
                                                           const uint16_t* __restrict__ s, int64_t s_stride,
                                                           uint8_t* __restrict__ codes, int64_t c_stride,
                                                           const uint8_t* __restrict__ prev, int64_t p_stride,
                                                           unsigned long long* __restrict__ flips,
                                                           int64_t n, int chunks_per_row) {
  const int64_t total = n * chunks_per_row;
  int flipped = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / chunks_per_row;
    const int ch = (int)(i - row * chunks_per_row);
    const int k0 = ch * 64;
    const float sv = __half2float(__ushort_as_half(s[row * s_stride + k0 / kGroup]));
    const float s_abs = fabsf(sv);
    const bool s_neg = sv < 0.0f;
    const uint4* src = reinterpret_cast<const uint4*>(w + row * w_stride + k0);
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; j++) v[j] = __ldg(src + j);
    uint32_t out[4];
#pragma unroll
    for (int word = 0; word < 4; word++) {
      uint32_t acc = 0;
#pragma unroll
      for (int h = 0; h < 16; h++) {  // weight 16*word + h
        const uint4& q = v[(16 * word + h) / 8];
        const int e = (16 * word + h) % 8;
        const uint32_t pair = (e / 2 == 0) ? q.x : (e / 2 == 1) ? q.y : (e / 2 == 2) ? q.z : q.w;
        const uint16_t bits = (e & 1) ? (uint16_t)(pair >> 16) : (uint16_t)(pair & 0xFFFFu);
        acc |= ((uint32_t)ternary_value(bits, s_abs, s_neg) & 3u) << (2 * h);  // 2-bit two's complement
      }
      out[word] = acc;
    }
    *reinterpret_cast<uint4*>(codes + row * c_stride + (int64_t)ch * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    if (prev) {  // a weight flips when its 2-bit field differs from the previous packing
      const uint4 pv = __ldg(reinterpret_cast<const uint4*>(prev + row * p_stride + (int64_t)ch * 16));
      const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int word = 0; word < 4; word++) {
        const uint32_t d = out[word] ^ pw[word];
        flipped += __popc((d | (d >> 1)) & 0x55555555u);
      }
    }
  }
  if (flips) {
    flipped = __reduce_add_sync(0xFFFFFFFFu, flipped);
    if ((threadIdx.x & 31) == 0 && flipped) atomicAdd(flips, (unsigned long long)flipped);
  }
}

// ---- Q1_0_g128 (binary): chunk = 16 bytes = 128 weights = one group; t = -1 iff w * s < 0 ----
__global__ void __launch_bounds__(kThreads) pack_q1_kernel(const uint16_t* __restrict__ w, int64_t w_stride,
                                                           const uint16_t* __restrict__ s, int64_t s_stride,
                                                           uint8_t* __restrict__ codes, int64_t c_stride,
                                                           const uint8_t* __restrict__ prev, int64_t p_stride,
                                                           unsigned long long* __restrict__ flips,
                                                           int64_t n, int chunks_per_row) {
  const int64_t total = n * chunks_per_row;
  int flipped = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / chunks_per_row;
    const int ch = (int)(i - row * chunks_per_row);
    const uint16_t sb = s[row * s_stride + ch];
    const bool s_ok = (sb & 0x7FFFu) != 0 && (sb & 0x7FFFu) <= 0x7C00u;  // s = 0 or NaN: every t is +1
    const uint32_t sneg = (sb & 0x8000u) ? 0x80008000u : 0u;
    const uint4* src = reinterpret_cast<const uint4*>(w + row * w_stride + (int64_t)ch * kGroup);
    uint4 v[16];
#pragma unroll
    for (int j = 0; j < 16; j++) v[j] = __ldg(src + j);
    uint32_t out[4];
#pragma unroll
    for (int word = 0; word < 4; word++) {
      uint32_t negs = 0;  // bit i set: weight 32 word + i has t = -1 (w * s < 0)
#pragma unroll
      for (int j = 0; j < 16; j++) {  // weights 32 word + 2j (low lane) and + 1 (high lane)
        const uint32_t pair = comp(v[4 * word + j / 4], j % 4);
        const uint32_t x = (pair ^ sneg) & nonzero2(pair);
        negs |= (((x >> 15) & 1u) | ((x >> 30) & 2u)) << (2 * j);
      }
      out[word] = s_ok ? ~negs : 0xFFFFFFFFu;
    }
    *reinterpret_cast<uint4*>(codes + row * c_stride + (int64_t)ch * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    if (prev) {  // a weight flips when its sign bit differs from the previous packing
      const uint4 pv = __ldg(reinterpret_cast<const uint4*>(prev + row * p_stride + (int64_t)ch * 16));
      flipped += __popc(out[0] ^ pv.x) + __popc(out[1] ^ pv.y) + __popc(out[2] ^ pv.z) + __popc(out[3] ^ pv.w);
    }
  }
  if (flips) {
    flipped = __reduce_add_sync(0xFFFFFFFFu, flipped);
    if ((threadIdx.x & 31) == 0 && flipped) atomicAdd(flips, (unsigned long long)flipped);
  }
}

// ---- base-3: chunk = 16 bytes = 80 trits; trits at k >= K are c = 1 --------------------------
__global__ void __launch_bounds__(kThreads) pack_t3_kernel(const uint16_t* __restrict__ w, int64_t w_stride,
                                                           const uint16_t* __restrict__ s, int64_t s_stride,
                                                           uint8_t* __restrict__ codes, int64_t c_stride,
                                                           const uint8_t* __restrict__ prev, int64_t p_stride,
                                                           unsigned long long* __restrict__ flips,
                                                           int64_t n, int k, int chunks_per_row) {
  const int64_t total = n * chunks_per_row;
  int flipped = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / chunks_per_row;
    const int ch = (int)(i - row * chunks_per_row);
    const int k0 = ch * 80;
    const uint16_t* wr = w + row * w_stride;
    const uint16_t* sr = s + row * s_stride;
    // C[p]: the digits c = t + 1 of weights 2p (low lane) and 2p + 1 (high lane) of the chunk
    uint32_t C[40];
#pragma unroll
    for (int j = 0; j < 10; j++) {  // 10 vectors of 8 weights; K % 8 == 0 so a vector is all in or all out
      const int kv = k0 + 8 * j;
      if (kv < k) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(wr + kv));
        const uint16_t sb = sr[kv / kGroup];  // 8 | 128: one scale per vector
        const uint32_t sneg = (sb & 0x8000u) ? 0x80008000u : 0u;
        const uint32_t sabs = sb & 0x7FFFu;
        const uint32_t s2b = sabs | (sabs << 16);
        const __half2 s2 = *reinterpret_cast<const __half2*>(&s2b);
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const uint32_t pair = comp(q, e);
          const uint32_t m = sabs ? big2(pair, s2) : 0u;
          const uint32_t nb = ((pair ^ sneg) >> 15) & 0x00010001u;  // t = -1 where set (and m)
          // c = 2 - 2 neg where |t| = 1, else 1
          C[4 * j + e] = (m & (0x00020002u - (nb << 1))) | (~m & 0x00010001u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; e++) C[4 * j + e] = 0x00010001u;  // trits past K: c = 1
      }
    }
    // byte b = sum_i c(5b + i) 3^i; a pair's lo + 3 hi is bits 16..31 of pair * 0x00010003
    auto pair3 = [](uint32_t p) { return (p * 0x00010003u) >> 16; };
    uint32_t out[4];
#pragma unroll
    for (int word = 0; word < 4; word++) {
      uint32_t acc = 0;
#pragma unroll
      for (int b4 = 0; b4 < 4; b4++) {
        const int b = 4 * word + b4, w0 = 5 * b;
        uint32_t byte;
        if ((w0 & 1) == 0)  // c0 c1 | c2 c3 | c4 (low lane)
          byte = pair3(C[w0 / 2]) + 9u * pair3(C[w0 / 2 + 1]) + 81u * (C[w0 / 2 + 2] & 0xFFFFu);
        else  // c0 (high lane) | c1 c2 | c3 c4
          byte = (C[w0 / 2] >> 16) + 3u * pair3(C[w0 / 2 + 1]) + 27u * pair3(C[w0 / 2 + 2]);
        acc |= byte << (8 * b4);
      }
      out[word] = acc;
    }
    *reinterpret_cast<uint4*>(codes + row * c_stride + (int64_t)ch * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    if (prev) {  // a weight (k < K) flips when its base-3 digit differs from the previous packing
      const uint4 pv = __ldg(reinterpret_cast<const uint4*>(prev + row * p_stride + (int64_t)ch * 16));
      const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int b = 0; b < 16; b++) {
        uint32_t old = (pw[b / 4] >> (8 * (b % 4))) & 0xFFu;
        const uint32_t neu = (out[b / 4] >> (8 * (b % 4))) & 0xFFu;
        if (old == neu) continue;
#pragma unroll
        for (int f = 0; f < 5; f++) {
          const int wi = 5 * b + f;
          const uint32_t cw = (C[wi / 2] >> (16 * (wi & 1))) & 0xFFFFu;
          flipped += (old % 3u != cw) && (k0 + wi < k);
          old /= 3u;
        }
      }
    }
  }
  if (flips) {
    flipped = __reduce_add_sync(0xFFFFFFFFu, flipped);
    if ((threadIdx.x & 31) == 0 && flipped) atomicAdd(flips, (unsigned long long)flipped);
  }
}

// ---- unpack --------------------------------------------------------------------------------
template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) unpack_kernel(const uint8_t* __restrict__ codes, int64_t c_stride,
                                                          const uint16_t* __restrict__ s, int64_t s_stride,
                                                          uint16_t* __restrict__ w_out, int64_t w_stride,
                                                          int8_t* __restrict__ t_out, int64_t t_stride,
                                                          int32_t* __restrict__ invalid_count,
                                                          int64_t n, int k, int chunks_per_row) {
  constexpr int W = (LAYOUT == TERN_Q2_0_G128) ? 64 : (LAYOUT == TERN_Q1_0_G128) ? 128 : 80;  // weights per chunk
  const int64_t total = n * chunks_per_row;
  int bad = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / chunks_per_row;
    const int ch = (int)(i - row * chunks_per_row);
    const int k0 = ch * W;
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(codes + row * c_stride + (int64_t)ch * 16));
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
    int8_t t[W];
#pragma unroll
    for (int b = 0; b < 16; b++) {
      const uint32_t byte = (qw[b / 4] >> (8 * (b % 4))) & 0xFFu;
      if (LAYOUT == TERN_Q1_0_G128) {
#pragma unroll
        for (int f = 0; f < 8; f++) t[8 * b + f] = ((byte >> f) & 1u) ? (int8_t)1 : (int8_t)-1;
      } else if (LAYOUT == TERN_Q2_0_G128) {
#pragma unroll
        for (int f = 0; f < 4; f++) {
          const uint32_t c = (byte >> (2 * f)) & 3u;  // 2-bit two's complement; 0b10 is invalid
          const bool inv = (c == 2u);
          bad += inv;
          t[4 * b + f] = inv ? 0 : (c == 3u ? (int8_t)-1 : (int8_t)c);
        }
      } else {
        const bool inv = byte > 242u;
        uint32_t v = byte;
#pragma unroll
        for (int f = 0; f < 5; f++) {
          const uint32_t c = v % 3u;
          v /= 3u;
          const int kk = k0 + 5 * b + f;
          bad += (inv && kk < k);
          t[5 * b + f] = inv ? 0 : (int8_t)((int)c - 1);
        }
      }
    }
    // outputs: vectors of 8 (fp16) / 16 (int8) weights; K % 16 == 0 so each vector is all in or out
#pragma unroll
    for (int j = 0; j < W / 8; j++) {
      const int kv = k0 + 8 * j;
      if (w_out && kv < k) {
        const float sv = __half2float(__ushort_as_half(s[row * s_stride + kv / kGroup]));
        uint32_t pr[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          // s * t is exact in fp16: +-s or 0
          const __half lo = __float2half_rn(sv * (float)t[8 * j + 2 * e]);
          const __half hi = __float2half_rn(sv * (float)t[8 * j + 2 * e + 1]);
          pr[e] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
        }
        *reinterpret_cast<uint4*>(w_out + row * w_stride + kv) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      }
    }
#pragma unroll
    for (int j = 0; j < W / 16; j++) {
      const int kv = k0 + 16 * j;
      if (t_out && kv < k) {
        uint32_t pr[4];
#pragma unroll
        for (int e = 0; e < 4; e++)
          pr[e] = (uint32_t)(uint8_t)t[16 * j + 4 * e] | ((uint32_t)(uint8_t)t[16 * j + 4 * e + 1] << 8) |
                  ((uint32_t)(uint8_t)t[16 * j + 4 * e + 2] << 16) | ((uint32_t)(uint8_t)t[16 * j + 4 * e + 3] << 24);
        *reinterpret_cast<uint4*>(t_out + row * t_stride + kv) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      }
    }
  }
  if (invalid_count) {
    bad = __reduce_add_sync(0xFFFFFFFFu, bad);
    if ((threadIdx.x & 31) == 0 && bad) atomicAdd(invalid_count, bad);
  }
}

int grid_for(int64_t work) {
  const int64_t waves = (int64_t)sm_count() * 8;  // 8 resident 256-thread blocks per SM
  const int64_t blocks = (work + kThreads - 1) / kThreads;
  return (int)(blocks < waves ? (blocks > 0 ? blocks : 1) : waves);
}

}  // namespace

cudaError_t launch_pack(int32_t layout, int64_t n, int64_t k, const uint16_t* w, int64_t w_stride,
                        const uint16_t* s, int64_t s_stride, uint8_t* codes, int64_t c_stride,
                        const uint8_t* prev, int64_t p_stride, unsigned long long* flips, cudaStream_t st) {
  const int chunks = (int)(row_bytes(layout, k) / 16);
  const int grid = grid_for(n * chunks);
  if (layout == TERN_Q2_0_G128)
    pack_q2_kernel<<<grid, kThreads, 0, st>>>(w, w_stride, s, s_stride, codes, c_stride, prev, p_stride, flips, n,
                                              chunks);
  else if (layout == TERN_Q1_0_G128)
    pack_q1_kernel<<<grid, kThreads, 0, st>>>(w, w_stride, s, s_stride, codes, c_stride, prev, p_stride, flips, n,
                                              chunks);
  else
    pack_t3_kernel<<<grid, kThreads, 0, st>>>(w, w_stride, s, s_stride, codes, c_stride, prev, p_stride, flips, n,
                                              (int)k, chunks);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const tern_matrix& W, uint16_t* w_out, int64_t w_stride, int8_t* t_out,
                          int64_t t_stride, int32_t* invalid_count, cudaStream_t st) {
  const int chunks = (int)(row_bytes(W.layout, W.k) / 16);
  const int grid = grid_for(W.n * chunks);
  const uint8_t* c = static_cast<const uint8_t*>(W.codes);
  if (W.layout == TERN_Q2_0_G128)
    unpack_kernel<TERN_Q2_0_G128><<<grid, kThreads, 0, st>>>(c, W.code_row_stride, W.scales, W.scale_row_stride,
                                                             w_out, w_stride, t_out, t_stride, invalid_count,
                                                             W.n, (int)W.k, chunks);
  else if (W.layout == TERN_Q1_0_G128)
    unpack_kernel<TERN_Q1_0_G128><<<grid, kThreads, 0, st>>>(c, W.code_row_stride, W.scales, W.scale_row_stride,
                                                             w_out, w_stride, t_out, t_stride, invalid_count,
                                                             W.n, (int)W.k, chunks);
  else
    unpack_kernel<TERN_T3_5PB_G128><<<grid, kThreads, 0, st>>>(c, W.code_row_stride, W.scales, W.scale_row_stride,
                                                               w_out, w_stride, t_out, t_stride, invalid_count,
                                                               W.n, (int)W.k, chunks);
  return cudaGetLastError();
}

}  // namespace tern
