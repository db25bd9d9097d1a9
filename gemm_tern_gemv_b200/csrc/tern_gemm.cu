// Prefill GEMM  Y[m][n] = sum_k X[m][k] * s[n][k/128] * t[n][k]  on tcgen05 tensor cores.
//
// The prior-art CUDA backend fuses ternary unpack and the group scale into the matrix product
// ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "하이브리드 어텐션을 위한 저비트 커널");
// prefill is compute bound (same page, section "처리량", pp512 column). Here:
//
//   * One persistent CTA per SM walks 128 (weight rows) x 256 (tokens) output tiles.
//   * TMA streams, per 64-wide K block, the fp16 X tile (256 x 64, 128-byte swizzle) and the packed
//     codes of the W tile (128 rows x 16 bytes for Q2_0_g128 and the binary Q1_0_g128, 32 for
//     base-3) into a 4-stage ring.
//   * Four decoder warps expand the codes to fp16 2*s*t (exact) straight into the K-major
//     128-byte-swizzled shared-memory layout a tcgen05 descriptor reads; a K block lies inside one
//     128-weight group, so one scale per row and block.
//   * One thread issues tcgen05.mma kind::f16 (M = 128, N = 256, K = 16) with D in tensor memory,
//     two accumulators so the epilogue of one tile overlaps the MMAs of the next.
//   * Four epilogue warps read D with tcgen05.ld, scale by 1/2 and store fp16 Y.
//   * Every pipeline wait is bounded in wall time; on expiry the CTA raises an abort flag, ORs
//     TERN_DEVICE_TIMEOUT into the caller's status word, drains its in-flight copies and MMAs,
//     frees tensor memory and exits.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>

#include "sm100.cuh"
#include "tern_internal.cuh"

namespace tern {
namespace {

using namespace sm100;

constexpr int BM = 128;        // weight rows per tile (MMA M)
constexpr int BN = 256;        // tokens per tile (MMA N)
constexpr int BK = 64;         // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int STAGES = 4;      // TMA ring depth
constexpr int DSTAGES = 3;     // decoded-W ring depth
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue, warps 6-9 decode
constexpr uint32_t kTmemCols = 2 * BN;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

constexpr int X_STAGE_BYTES = BN * BK * 2;      // 32 KB
constexpr int A_STAGE_BYTES = BM * BK * 2;      // 16 KB
// Packed codes of a K block, per row: Q2_0_g128 16 bytes; base-3 a 32-byte box at the 16-byte
// boundary below the block's first byte (the block's 64 trits span at most 14 bytes); binary the
// 16-byte box holding the block's 8 bytes (TMA boxes start on 16-byte boundaries).
template <int LAYOUT> constexpr int p_row_bytes() { return LAYOUT == TERN_T3_5PB_G128 ? 32 : 16; }
constexpr int P_STAGE_BYTES = BM * 32;          // room for any layout
constexpr int OFF_X = 0;
constexpr int OFF_A = OFF_X + STAGES * X_STAGE_BYTES;
constexpr int OFF_P = OFF_A + DSTAGES * A_STAGE_BYTES;
constexpr int OFF_LUT = OFF_P + STAGES * P_STAGE_BYTES;  // base-3 byte -> five 2-bit fields
constexpr int OFF_BAR = OFF_LUT + 256 * 4;
constexpr int NUM_BARS = 2 * STAGES + 2 * DSTAGES + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024

struct Params {
  int m, n, k;
  int n_tiles, m_tiles;
  const uint16_t* scales;
  int64_t sstride;
  uint16_t* y;
  uint32_t* status;
};

// t code fields of one 32-bit word (16 codes, code i at bits 2i) -> fp16 pair (2 t_{2j}, 2 t_{2j+1}).
// The pre-mask keeps the two fields; one multiply places them at bits 14..15 and 30..31, where a
// two's-complement field is the fp16 sign + exponent MSB of +-2.0 (or 0).
__device__ __forceinline__ uint32_t pair_2t(uint32_t w, int j) {
  const uint32_t lo = (j < 4) ? w : (w >> 16);
  const int jj = j & 3;
  const uint32_t x = lo & (0xFu << (4 * jj));
  const uint32_t a = 14 - 4 * jj;  // field 2j (bits 4jj..) -> bit 14; field 2j+1 -> bit 30
  return (x * ((1u << a) + (1u << (a + 14)))) & 0xC000C000u;
}

// Binary sign bits (bit i of w = weight i, 1 = +1) -> fp16 pair (2 t_p, 2 t_{p+1}) for an even
// p <= 14: one multiply moves bit p to bit 15 and bit p + 1 to bit 31, and flipping the sign and the
// exponent MSB turns a set sign bit into +2.0 (0x4000) and a clear one into -2.0 (0xC000).
__device__ __forceinline__ uint32_t pair_2t_bin(uint32_t w, int p) {
  const uint32_t x = w & (3u << p);
  return ((x * ((1u << (15 - p)) + (1u << (30 - p)))) & 0x80008000u) ^ 0xC000C000u;
}

// Base-3 K block whose first trit is digit R0 of its first byte: the 64 weights -> fp16 2 s t in the
// 128-byte-swizzled K-major row `arow`. F[j] holds the five 2-bit two's-complement fields of byte j
// (table lookup); a pair of weights in one byte is one masked multiply as in pair_2t, a pair across
// a byte boundary (digit 4, digit 0) is assembled from both bytes. All offsets are compile-time.
template <int R0>
__device__ __forceinline__ void t3_block(const uint8_t* prow, const uint32_t* lut, __half2 s2, uint8_t* arow, int rsw) {
  constexpr int NB = (R0 + 63) / 5 + 1;
  uint32_t F[NB];
#pragma unroll
  for (int j = 0; j < NB; j++) F[j] = lut[prow[j]];
#pragma unroll
  for (int c = 0; c < 8; c++) {  // 16-byte chunk c holds k = 8c .. 8c + 7 of the block
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int i1 = R0 + 8 * c + 2 * e, i2 = i1 + 1;
      const int b1 = i1 / 5, d1 = i1 % 5, b2 = i2 / 5;
      uint32_t two_t;
      if (b1 == b2) {
        const uint32_t x = F[b1] & (0xFu << (2 * d1));
        const uint32_t a = 14 - 2 * d1;
        two_t = (x * ((1u << a) + (1u << (a + 14)))) & 0xC000C000u;
      } else {  // digit 4 of byte b1, digit 0 of byte b2
        two_t = ((F[b1] << 6) & 0x0000C000u) | (F[b2] << 30);
      }
      const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&two_t), s2);  // 2 s t, exact
      o[e] = *reinterpret_cast<const uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(arow + ((c ^ rsw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;                       // TMA -> decoders + MMA
  uint64_t* empty = full + STAGES;             // MMA commit -> TMA
  uint64_t* dfull = empty + STAGES;            // decoders -> MMA
  uint64_t* dempty = dfull + DSTAGES;          // MMA commit -> decoders
  uint64_t* tfull = dempty + DSTAGES;          // MMA commit -> epilogue (2)
  uint64_t* tempty = tfull + 2;                // epilogue -> MMA (2)
  uint64_t* drain = tempty + 2;                // MMA completion on abort
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles = p.n_tiles * p.m_tiles;
  const int kblocks = p.k / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; i++) { mbar_init(full + i, 1); mbar_init(empty + i, 1); }
    for (int i = 0; i < DSTAGES; i++) { mbar_init(dfull + i, 4); mbar_init(dempty + i, 1); }
    for (int i = 0; i < 2; i++) { mbar_init(tfull + i, 1); mbar_init(tempty + i, 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) { prefetch_tmap(&tmap_x); prefetch_tmap(&tmap_w); }
  if (LAYOUT == TERN_T3_5PB_G128) {
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + OFF_LUT);
    for (int v = threadIdx.x; v < 256; v += kThreads) {
      uint32_t f = 0, r = (uint32_t)v;
      if (v < 243) {
#pragma unroll
        for (int d = 0; d < 5; d++) { f |= (((r % 3u) + 3u) & 3u) << (2 * d); r /= 3u; }  // c - 1 as 2 bits
      }
      lut[v] = f;  // an invalid byte reads as five t = 0
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool pending[STAGES] = {};
      uint32_t pend_par[STAGES] = {};
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int n0 = (tile / p.m_tiles) * BM, m0 = (tile % p.m_tiles) * BN;
        for (int kb = 0; kb < kblocks; kb++, it++) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(empty + s, ph ^ 1u, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + s, X_STAGE_BYTES + BM * p_row_bytes<LAYOUT>());
          tma_load_2d(smem + OFF_X + s * X_STAGE_BYTES, &tmap_x, full + s, kb * BK, m0);
          const int px = LAYOUT == TERN_Q2_0_G128 ? kb * (BK / 4)
                         : LAYOUT == TERN_Q1_0_G128 ? (kb * (BK / 8)) & ~15
                                                    : ((kb * BK) / 5) & ~15;
          tma_load_2d(smem + OFF_P + s * P_STAGE_BYTES, &tmap_w, full + s, px, n0);
          pending[s] = true;
          pend_par[s] = ph;
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int s = 0; s < STAGES; s++)
          if (pending[s]) mbar_wait_bounded(full + s, pend_par[s], abort_flag, nullptr, 0, kWaitLimitNs / 4 + 1) ||
                          mbar_try_wait(full + s, pend_par[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN);
      uint32_t it = 0, lt = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, lt++) {
        const uint32_t acc = lt & 1u, aph = (lt >> 1) & 1u;
        if (!mbar_wait_bounded(tempty + acc, aph ^ 1u, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; kb++, it++) {
          const int s = it % STAGES, d = it % DSTAGES;
          const uint32_t ph = (it / STAGES) & 1u, dph = (it / DSTAGES) & 1u;
          if (!mbar_wait_bounded(full + s, ph, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs) ||
              !mbar_wait_bounded(dfull + d, dph, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(smem + OFF_A + d * A_STAGE_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + OFF_X + s * X_STAGE_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++)
            mma_f16_ss(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
          issued = true;
          mma_commit(empty + s);
          mma_commit(dempty + d);
        }
        if (!ok) break;
        mma_commit(tfull + acc);
      }
      if (!ok && issued) {  // wait for the MMAs already issued before tensor memory is freed
        mma_commit(drain);
        mbar_wait_bounded(drain, 0, abort_flag, nullptr, 0, kWaitLimitNs / 4 + 1) || mbar_try_wait(drain, 0);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // tcgen05.ld lane quadrant of this warp
    const int row = quad * 32 + lane;
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, lt++) {
      const int n0 = (tile / p.m_tiles) * BM, m0 = (tile % p.m_tiles) * BN;
      const uint32_t acc = lt & 1u, aph = (lt >> 1) & 1u;
      if (!mbar_wait_bounded(tfull + acc, aph, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs)) break;
      tc_fence_after();
      const int n = n0 + row;
      const uint32_t taddr = tmem_base + acc * BN + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c0, r);
        tmem_ld_wait();
        if (n < p.n) {
#pragma unroll
          for (int j = 0; j < 32; j++) {
            const int m = m0 + c0 + j;
            if (m < p.m)
              p.y[(int64_t)m * p.n + n] = __half_as_ushort(__float2half_rn(0.5f * __uint_as_float(r[j])));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
    }
  } else {
    // ------------------------------------------------------------------ decoders: one W row each
    const int r = (warp - 6) * 32 + lane;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      const int n0 = (tile / p.m_tiles) * BM;
      const int n = n0 + r;
      const uint16_t* srow = p.scales + (int64_t)(n < p.n ? n : 0) * p.sstride;
      for (int kb = 0; kb < kblocks; kb++, it++) {
        const int s = it % STAGES, d = it % DSTAGES;
        const uint32_t ph = (it / STAGES) & 1u, dph = (it / DSTAGES) & 1u;
        const uint16_t sbits = (n < p.n) ? __ldg(srow + (kb * BK) / kGroup) : (uint16_t)0;
        if (!mbar_wait_bounded(full + s, ph, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs) ||
            !mbar_wait_bounded(dempty + d, dph ^ 1u, abort_flag, p.status, TERN_DEVICE_TIMEOUT, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const __half2 s2 = __halves2half2(__ushort_as_half(sbits), __ushort_as_half(sbits));
        uint8_t* arow = smem + OFF_A + d * A_STAGE_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
        if (LAYOUT == TERN_Q2_0_G128) {
          const uint4 pk = *reinterpret_cast<const uint4*>(smem + OFF_P + s * P_STAGE_BYTES + r * 16);
          const uint32_t wv[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int c = 0; c < 8; c++) {  // 16-byte chunk c holds k = 8c .. 8c + 7
            const uint32_t w = wv[c >> 1];
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
              const uint32_t two_t = pair_2t(w, (c & 1) * 4 + e);
              const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&two_t), s2);  // 2 s t, exact
              o[e] = *reinterpret_cast<const uint32_t*>(&v);
            }
            *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else if (LAYOUT == TERN_Q1_0_G128) {
          // the block's 8 bytes are the low or high half of the 16-byte box
          const uint2 pk = *reinterpret_cast<const uint2*>(smem + OFF_P + s * P_STAGE_BYTES + r * 16 + 8 * (kb & 1));
#pragma unroll
          for (int c = 0; c < 8; c++) {  // byte c holds k = 8c .. 8c + 7
            const uint32_t w = (c < 4 ? pk.x : pk.y) >> (c & 2 ? 16 : 0);
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
              const uint32_t two_t = pair_2t_bin(w, 8 * (c & 1) + 2 * e);
              const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&two_t), s2);  // 2 s t, exact
              o[e] = *reinterpret_cast<const uint32_t*>(&v);
            }
            *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
          // the block's trits start at digit r0 of byte b0; the box starts at the 16-byte boundary below b0
          const int b0 = (kb * BK) / 5, r0 = (kb * BK) % 5;
          const uint8_t* prow = smem + OFF_P + s * P_STAGE_BYTES + r * 32 + (b0 & 15);
          const uint32_t* lut = reinterpret_cast<const uint32_t*>(smem + OFF_LUT);
          switch (r0) {
            case 0: t3_block<0>(prow, lut, s2, arow, r & 7); break;
            case 1: t3_block<1>(prow, lut, s2, arow, r & 7); break;
            case 2: t3_block<2>(prow, lut, s2, arow, r & 7); break;
            case 3: t3_block<3>(prow, lut, s2, arow, r & 7); break;
            default: t3_block<4>(prow, lut, s2, arow, r & 7); break;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(dfull + d);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm(const tern_matrix& W, const uint16_t* X, int64_t m, uint16_t* Y, uint32_t* device_status,
                        cudaStream_t st) {
  CUtensorMap mx, mw;
  const uint64_t k = (uint64_t)W.k, n = (uint64_t)W.n;
  const bool t3 = W.layout == TERN_T3_5PB_G128;
  if (!tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, k, (uint64_t)m, k * 2, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // codes [n][row data bytes]: Q2 and binary boxes of 16 bytes, base-3 boxes of 32 bytes (zero-filled
  // past the data)
  const uint64_t data_bytes = W.layout == TERN_Q2_0_G128 ? k / 4 : W.layout == TERN_Q1_0_G128 ? k / 8 : (k + 4) / 5;
  if (!tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.codes, data_bytes, n, (uint64_t)W.code_row_stride,
               t3 ? 32 : 16, BM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  Params p;
  p.m = (int)m;
  p.n = (int)W.n;
  p.k = (int)W.k;
  p.n_tiles = (int)((W.n + BM - 1) / BM);
  p.m_tiles = (int)((m + BN - 1) / BN);
  p.scales = W.scales;
  p.sstride = W.scale_row_stride;
  p.y = Y;
  p.status = device_status;
  auto kern = W.layout == TERN_Q2_0_G128   ? gemm_kernel<TERN_Q2_0_G128>
              : W.layout == TERN_Q1_0_G128 ? gemm_kernel<TERN_Q1_0_G128>
                                           : gemm_kernel<TERN_T3_5PB_G128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = p.n_tiles * p.m_tiles;
  const int grid = tiles < sm_count() ? tiles : sm_count();
  kern<<<grid, kThreads, SMEM_BYTES, st>>>(mx, mw, p);
  return cudaGetLastError();
}

}  // namespace tern
