// Decode GEMV y = W x for packed ternary (and binary) W, batch 1..64, on mma.sync tensor cores.
//
// What is computed ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "그룹 단위 스케일을
// 공유하는 삼진 형식", eq. w_i = s_g t_i; section "하이브리드 어텐션을 위한 저비트 커널": the
// product reads packed codes and fuses unpack + group scale):
//     y[b][n] = sum_g s[n][g] * sum_{k in g} t[n][k] * x[b][k]
//
// How (B200, sm_100a). The weights are streamed once and every code has to be turned into a tensor-
// core operand, so the integer decode sets the pace (IMAD and LOP3 each issue at half rate, on two
// different pipes, and an HMMA with freshly decoded operands barely overlaps them):
//   * Decode = one IMAD + one LOP3 per two weights. A Q2_0_g128 code is t as a 2-bit two's-
//     complement field; shifted to bits 14..15 of an fp16 half, the field IS the half's sign bit
//     and exponent MSB: 0b01 -> +2.0, 0b11 -> -2.0, 0b00 -> 0. So (word << (14 - 2i)) & 0xC000C000
//     is the tensor-core A fragment (2 t_i, 2 t_{i+8}) exactly. B is the fp16 activation itself;
//     the MMA accumulates D = 2 sum t x in fp32 and the epilogue applies s/2 per group: no offset,
//     no cancellation, exact products. The base-3 layout reaches the same fragments with three
//     integer operations per pair (see dec_t3_word).
//   * The 8 MMA columns carry (batch, group-within-window) pairs, so each group's partial sum gets
//     its own scale in the fp32 epilogue. Activations are laid out once per CTA in fragment order.
// Two kernels:
//   * gemv_reg_kernel (Q2_0_g128 batch <= 4, base-3 batch <= 2, binary Q1_0_g128 in pairs of batch
//     rows): one window = 64 code bytes of each row of a 32-row warp tile; every warp streams its
//     windows through its own ring of TMA boxes (codes and scales, out-of-range reads zero-filled) and
//     decodes them in registers. Work split: when K is one slice, each CTA owns whole row tiles and its
//     warps split them into equal runs, shared tiles being summed in shared memory (CTA-local);
//     otherwise the (tile, window) units of a K slice are split into equal runs dealt over all warps
//     (stream-K) and tiles shared by several runs are summed through the workspace by the last run to
//     arrive. Both orders are deterministic. 16 warps x 1 CTA or 8 warps x 2 CTAs per SM, by the
//     number of row tiles. As a programmatic dependent launch it can request its first weight boxes
//     before the preceding kernel on the stream completes (see tern_gemv_ex).
//   * gemv_kernel (larger batches): per-warp cp.async rings over 32- or 16-row tiles, base-3
//     windows expanded to 2-bit fields in shared memory first; K is split across CTAs for narrow
//     matrices, with the last-arriver reduction.
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "sm100.cuh"
#include "tern_internal.cuh"
#include "tern_t3.cuh"

namespace tern {
namespace {

using sm100::smem_u32;

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;        // per-warp ring depth, Q2_0_g128 (one pair-window per stage)
constexpr int kT3Stages = 3;      // per-warp ring depth, base-3 (one 5-group window per stage)
constexpr int kT3Window = 5;      // base-3 window: 5 groups = 640 trits = 128 bytes per row
constexpr int kQ2RowStride = 192; // bytes per row of the expanded base-3 buffer (160 used)

struct Args {
  const uint8_t* codes;
  int64_t cstride;
  const uint16_t* scales;
  int64_t sstride;
  const uint16_t* x;
  uint16_t* y;
  float* ws;        // [splits][batch][n] fp32 partials
  int* counters;    // one per row tile
  int n, k, batch, groups, gps, splits, tiles;
  int run;          // register kernel: (tile, window) units per warp run (stream-K)
  int kmax;         // register kernel: partial-sum slots per tile and slice
  uint32_t unit;    // always 1 (see `mul` in the kernel)
  int early;        // register kernel: W may be read before earlier work on the stream completes
  int local;        // register kernel: CTA-local reduction of whole tiles (no workspace)
  uint32_t* status;  // register kernel: optional device status word (TERN_DEVICE_TIMEOUT on a wait that ran out)
  uint64_t wait_ns;  // register kernel: bound on each pipeline wait
};

// ---- small device helpers --------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared-memory loads by 32-bit shared-window address (keeps address arithmetic 32-bit).
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// Loads 8 bytes into v only when pred is set (otherwise v keeps its value).
__device__ __forceinline__ void lds64_if(uint2& v, uint32_t addr, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p ld.shared.v2.u32 {%0,%1}, [%3];\n\t}"
      : "+r"(v.x), "+r"(v.y)
      : "r"((uint32_t)pred), "r"(addr));
}
__device__ __forceinline__ void cp_async16_u32(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void mma_f16(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The first MMA of an accumulation chain: D = A * B (zero accumulator, no register zeroing).
__device__ __forceinline__ void mma_f16_first(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// A fragment of slot S (0..7) of a 16-code word: codes (S, S+8) as the fp16 pair (2 t_S, 2 t_S+8).
// `mul` is 2^(14 - 2S) held in a register, so the shift issues as an IMAD on the FMA pipe.
__device__ __forceinline__ uint32_t slot(uint32_t w, uint32_t mul) { return (w * mul) & 0xC000C000u; }

// Binary A fragment of slot S (0..15) of a 32-bit word of sign bits: bits (S, S+16) as the fp16 pair
// (2 t_S, 2 t_S+16). `mul` = 2^(15 - S) moves the bits to the two sign positions; flipping sign and
// exponent MSB then gives +2.0 (0x4000) for a set bit and -2.0 (0xC000) for a clear one.
__device__ __forceinline__ uint32_t slot_bin(uint32_t w, uint32_t mul) {
  return ((w * mul) & 0x80008000u) ^ 0xC000C000u;
}

// ---- shared-memory plan (host and device agree on it) -------------------------------------------
__host__ __device__ inline int pair_windows(int layout, int gps) {
  return layout == TERN_T3_5PB_G128 ? 3 * ((gps + kT3Window - 1) / kT3Window) : (gps + 1) / 2;
}
// `bs` = batch slots of the fragment layout (a compile-time stride >= batch, see bs_for()).
__host__ __device__ inline size_t frag_bytes(int layout, int gps, int bs) {
  return (size_t)pair_windows(layout, gps) * 16 * bs * 4 * 8;  // uint2 per (window, mma, batch slot, q)
}
__host__ __device__ inline size_t warp_ring_bytes(int layout, int rt) {
  if (layout == TERN_Q2_0_G128) return (size_t)kStages * (rt * 16 * 64 + rt * 16 * 16);  // codes + scale chunk
  // raw 5-group windows + two 16-byte scale chunks per row, then the expanded 2-bit buffer
  return (size_t)kT3Stages * (rt * 16 * 128 + rt * 16 * 32) + (size_t)rt * 16 * kQ2RowStride;
}
__host__ __device__ inline size_t smem_bytes(int layout, int rt, int gps, int bs) {
  size_t s = frag_bytes(layout, gps, bs);
  s = (s + 127) / 128 * 128;
  s += (layout == TERN_T3_5PB_G128 ? 256 * 4 : 0);
  s += (size_t)kWarps * warp_ring_bytes(layout, rt);
  return s;
}

// ---- prologue: activations into B-fragment order --------------------------------------------------
// frag (uint2): [pair-window][j 0..15][batch][q 0..3]; halves (b0.lo, b0.hi, b1.lo, b1.hi).
// In a pair-window lane q owns bytes [16q, 16q + 16) of the 64 code bytes: codes o = 64q + 16*word + i
// (i = code in word), i.e. group g' = q / 2. Word `word` feeds MMAs j = 4*word .. 4*word + 3; MMA j
// uses slots s0 = 2*(j % 4) (-> b0) and s0 + 1 (-> b1); slot s holds codes (s, s + 8) (lo, hi).
template <int BS>
__device__ void build_fragments(const Args& a, int g0, int ngroups, uint2* frag) {
  uint16_t* fh = reinterpret_cast<uint16_t*>(frag);
  const int B = a.batch;
  const int items = ngroups * B * 16;  // item = 8 consecutive codes of one (group, batch row)
  for (int e = threadIdx.x; e < items; e += kThreads) {
    const int v = e & 15;
    const int gb = e >> 4;
    const int bb = gb % B, gl = gb / B;
    const uint4 xv = *reinterpret_cast<const uint4*>(a.x + (int64_t)bb * a.k + (int64_t)(g0 + gl) * kGroup + 8 * v);
    const int win = gl >> 1, gp = gl & 1;
    const int o = 128 * gp + 8 * v;  // first code of the vector within the pair-window
    const int q = o >> 6, word = (o & 63) >> 4, h = v & 1;
    uint16_t* base = fh + ((((size_t)win * 16 + 4 * word) * BS + bb) * 4 + q) * 4 + h;
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int el = 0; el < 8; el++)  // code i = 8h + el sits in slot el, MMA j = 4*word + el/2
      base[(size_t)(el >> 1) * BS * 16 + (el & 1) * 2] = (uint16_t)(xw[el >> 1] >> (16 * (el & 1)));
  }
}

// ---- one pair-window: 16 MMAs per row tile, then the fp32 epilogue of the two groups' scales ------
// `bpre` holds the window's B fragments for small batches; it lives across windows so lanes whose
// column never carries data keep zeros without re-zeroing.
template <int NT, int RT, int BS>
struct BFrag {
  static constexpr bool kPre = NT <= 2;
  uint2 v[kPre ? 16 : 1][kPre ? NT : 1];
};

// `fr` = shared address of this lane's fragment entry in the window: frag + ((pw*16*BS + g/2)*4 + q)*8.
template <int NT, int RT, int BS>
__device__ __forceinline__ void mma_pair(const uint4 (&cw)[RT][2], const uint32_t (&sc)[RT][2], uint32_t fr,
                                         const uint32_t (&mul)[8], int gh, const bool (&bload)[NT],
                                         BFrag<NT, RT, BS>& bf, float (&acc)[RT][NT][2]) {
  constexpr bool kPre = BFrag<NT, RT, BS>::kPre;
  if (kPre) {
#pragma unroll
    for (int j = 0; j < 16; j++)
#pragma unroll
      for (int jt = 0; jt < NT; jt++) lds64_if(bf.v[kPre ? j : 0][kPre ? jt : 0], fr + (j * BS + 4 * jt) * 32, bload[jt]);
  }
  // two independent accumulator chains (even / odd MMA) per row tile for small batches; larger
  // batches already have NT independent chains
  constexpr int CH = NT <= 2 ? 2 : 1;
  float d[RT][NT][CH][4];
#pragma unroll
  for (int word = 0; word < 4; word++) {
    uint32_t wl[RT], wh[RT];
#pragma unroll
    for (int rt = 0; rt < RT; rt++) {
      wl[rt] = word == 0 ? cw[rt][0].x : word == 1 ? cw[rt][0].y : word == 2 ? cw[rt][0].z : cw[rt][0].w;
      wh[rt] = word == 0 ? cw[rt][1].x : word == 1 ? cw[rt][1].y : word == 2 ? cw[rt][1].z : cw[rt][1].w;
    }
#pragma unroll
    for (int sp = 0; sp < 4; sp++) {
      const int j = 4 * word + sp;
      uint32_t a0[RT], a1[RT], a2[RT], a3[RT];
#pragma unroll
      for (int rt = 0; rt < RT; rt++) {
        a0[rt] = slot(wl[rt], mul[2 * sp]);
        a2[rt] = slot(wl[rt], mul[2 * sp + 1]);
        a1[rt] = slot(wh[rt], mul[2 * sp]);
        a3[rt] = slot(wh[rt], mul[2 * sp + 1]);
      }
#pragma unroll
      for (int jt = 0; jt < NT; jt++) {
        uint2 b;
        if (kPre) {
          b = bf.v[kPre ? j : 0][kPre ? jt : 0];
        } else {
          b = make_uint2(0u, 0u);
          lds64_if(b, fr + (j * BS + 4 * jt) * 32, bload[jt]);
        }
#pragma unroll
        for (int rt = 0; rt < RT; rt++) {
          if (j < CH) mma_f16_first(d[rt][jt][j % CH], a0[rt], a1[rt], a2[rt], a3[rt], b.x, b.y);
          else mma_f16(d[rt][jt][j % CH], a0[rt], a1[rt], a2[rt], a3[rt], b.x, b.y);
        }
      }
    }
  }
  // lane (g, q) holds columns 2q, 2q+1 = (b' = q, g' = 0 / 1) of rows g and g + 8; D = 2 sum t x
  // (the factor 1/2 is applied once per tile in finish_tile)
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int hr = 0; hr < 2; hr++) {
      const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sc[rt][hr]));
#pragma unroll
      for (int jt = 0; jt < NT; jt++) {
        float d0 = d[rt][jt][0][2 * hr], d1 = d[rt][jt][0][2 * hr + 1];
        if (CH == 2) {
          d0 += d[rt][jt][CH - 1][2 * hr];
          d1 += d[rt][jt][CH - 1][2 * hr + 1];
        }
        float v = fmaf(sf.x, d0, acc[rt][jt][hr]);
        if (gh > 1) v = fmaf(sf.y, d1, v);
        acc[rt][jt][hr] = v;
      }
    }
}

// ---- end of a row tile: store y, or publish a K-slice partial and let the last slice reduce -----
template <int NT, int RT>
__device__ __forceinline__ void finish_tile(const Args& a, int tile, int split, int lane, float (&acc)[RT][NT][2]) {
  const int g = lane >> 2, q = lane & 3;
  const int row_base = tile * 16 * RT;
  if (a.splits == 1) {
#pragma unroll
    for (int rt = 0; rt < RT; rt++)
#pragma unroll
      for (int jt = 0; jt < NT; jt++)
#pragma unroll
        for (int hr = 0; hr < 2; hr++) {
          const int row = row_base + rt * 16 + g + 8 * hr;
          const int b = 4 * jt + q;
          if (row < a.n && b < a.batch)
            a.y[(int64_t)b * a.n + row] = __half_as_ushort(__float2half_rn(0.5f * acc[rt][jt][hr]));
        }
    return;
  }
  float* part = a.ws + (size_t)split * a.batch * a.n;
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int jt = 0; jt < NT; jt++)
#pragma unroll
      for (int hr = 0; hr < 2; hr++) {
        const int row = row_base + rt * 16 + g + 8 * hr;
        const int b = 4 * jt + q;
        if (row < a.n && b < a.batch) part[(size_t)b * a.n + row] = 0.5f * acc[rt][jt][hr];
      }
  __threadfence();
  __syncwarp();
  int prev = 0;
  if (lane == 0) prev = atomicAdd(a.counters + tile, 1);
  prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
  if (prev != a.splits - 1) return;
  __threadfence();
  const int rows = min(16 * RT, a.n - row_base);
  for (int e = lane; e < rows * a.batch; e += 32) {
    const int b = e / rows, row = row_base + e % rows;
    float v = 0.f;
    for (int sp = 0; sp < a.splits; sp++) v += __ldcg(a.ws + ((size_t)sp * a.batch + b) * a.n + row);
    a.y[(int64_t)b * a.n + row] = __half_as_ushort(__float2half_rn(v));
  }
  __syncwarp();
  if (lane == 0) a.counters[tile] = 0;  // ready for the next call
}

// ---- base-3 stream ------------------------------------------------------------------------------
// Ring stage = one 5-group window: raw bytes [row][128 B] plus two 16-byte scale chunks per row
// covering groups [8*c0, 8*c0 + 16) with c0 = floor(first group / 8).
template <int RT>
__device__ __forceinline__ void issue_t3(const Args& a, uint8_t* ring, int slot, int tile, int grp0, int lane) {
  constexpr int ROWS = RT * 16;
  uint8_t* raw = ring + (size_t)slot * (ROWS * 128);
  uint8_t* scs = ring + (size_t)kT3Stages * ROWS * 128 + (size_t)slot * (ROWS * 32);
  const int t3_row_bytes = (a.k + 4) / 5;
  const int byte0 = (grp0 / kT3Window) * 128;
#pragma unroll
  for (int u = 0; u < ROWS * 8 / 32; u++) {
    const int idx = lane + 32 * u;
    const int r = idx >> 3, ch = idx & 7;
    const int row = tile * ROWS + r;
    const bool ok = row < a.n && byte0 + 16 * ch < t3_row_bytes;
    cp_async16(raw + r * 128 + 16 * ch, a.codes + (int64_t)(ok ? row : 0) * a.cstride + (ok ? byte0 + 16 * ch : 0), ok);
  }
  const int c0 = grp0 >> 3;
#pragma unroll
  for (int u = 0; u < ROWS * 2 / 32; u++) {
    const int idx = lane + 32 * u;
    const int r = idx >> 1, c = c0 + (idx & 1);
    const int row = tile * ROWS + r;
    const bool ok = row < a.n && 8 * c < a.sstride;
    cp_async16(scs + r * 32 + 16 * (idx & 1), a.scales + (int64_t)(ok ? row : 0) * a.sstride + (ok ? 8 * c : 0), ok);
  }
}

// Expand one raw 5-group window of 16*RT rows into 2-bit two's-complement fields (16 codes per
// word, code k at bits 2*(k % 16)), 160 bytes per row at stride kQ2RowStride.
template <int RT>
__device__ __forceinline__ void expand_t3(const uint8_t* raw, const uint32_t* lut, uint8_t* out, int lane) {
  constexpr int ROWS = RT * 16;
  for (int idx = lane; idx < ROWS * 8; idx += 32) {
    const int r = idx >> 3, ch = idx & 7;
    const uint4 qv = *reinterpret_cast<const uint4*>(raw + r * 128 + 16 * ch);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    uint32_t o[5] = {0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const uint32_t f = lut[(qw[j >> 2] >> (8 * (j & 3))) & 0xFFu];  // five 2-bit fields
      const int off = 10 * j;
      o[off >> 5] |= f << (off & 31);
      if ((off & 31) > 22) o[(off >> 5) + 1] |= f >> (32 - (off & 31));
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(out + r * kQ2RowStride + ch * 20);
#pragma unroll
    for (int w = 0; w < 5; w++) dst[w] = o[w];
  }
}

template <int LAYOUT, int NT, int RT, int BS>
__global__ void __launch_bounds__(kThreads) gemv_kernel(Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane / 4, q = lane % 4;
  const int split = blockIdx.y;
  const int g0 = split * a.gps;
  const int ngroups = min(a.gps, a.groups - g0);

  uint2* frag = reinterpret_cast<uint2*>(smem);
  uint8_t* p = smem + (frag_bytes(LAYOUT, a.gps, BS) + 127) / 128 * 128;
  uint32_t* lut = reinterpret_cast<uint32_t*>(p);
  if (LAYOUT == TERN_T3_5PB_G128) p += 256 * 4;
  uint8_t* ring = p + (size_t)warp * warp_ring_bytes(LAYOUT, RT);

  // tiles of this warp: t = first + i * stride
  const int first = blockIdx.x * kWarps + warp;
  const int stride = gridDim.x * kWarps;
  const int my_tiles = first < a.tiles ? (a.tiles - 1 - first) / stride + 1 : 0;

  // ---- once per CTA: activation fragments of this K slice (and the base-3 table) ----
  if (LAYOUT == TERN_T3_5PB_G128) {
    for (int v = threadIdx.x; v < 256; v += kThreads) {
      uint32_t f = 0, r = v < 243 ? v : 121;  // an invalid byte decodes as five t = 0 trits
#pragma unroll
      for (int i = 0; i < 5; i++) { f |= (((r % 3u) + 3u) & 3u) << (2 * i); r /= 3u; }  // c - 1, 2-bit two's complement
      lut[v] = f;
    }
    for (int w5 = 0; w5 * kT3Window < ngroups; w5++)  // groups of 5-window w5 -> pair-windows 3*w5 + (0,0,1,1,2)
      build_fragments<BS>(a, g0 + w5 * kT3Window, min(kT3Window, ngroups - w5 * kT3Window),
                          frag + (size_t)w5 * 3 * 16 * BS * 4);
  } else {
    build_fragments<BS>(a, g0, ngroups, frag);
  }

  // shift multipliers 2^(14 - 2S), built from a runtime 1 so they stay IMAD operands
  uint32_t mul[8];
#pragma unroll
  for (int S = 0; S < 8; S++) mul[S] = a.unit << (14 - 2 * S);
  // B column of this lane: (b' = g/2, g' = g&1); it carries data when g' is the lane's group
  const bool bcol = ((g & 1) == (q >> 1));
  bool bload[NT];
#pragma unroll
  for (int jt = 0; jt < NT; jt++) bload[jt] = bcol && (4 * jt + (g >> 1) < a.batch);
  BFrag<NT, RT, BS> bf;
  if (BFrag<NT, RT, BS>::kPre) {
#pragma unroll
    for (int j = 0; j < (BFrag<NT, RT, BS>::kPre ? 16 : 1); j++)
#pragma unroll
      for (int jt = 0; jt < (BFrag<NT, RT, BS>::kPre ? NT : 1); jt++) bf.v[j][jt] = make_uint2(0u, 0u);
  }

  float acc[RT][NT][2];
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int jt = 0; jt < NT; jt++) acc[rt][jt][0] = acc[rt][jt][1] = 0.f;

  if (LAYOUT == TERN_Q2_0_G128) {
    // Ring stage = one pair-window of the warp's 16*RT rows: codes [row][64 B] (each lane copies
    // and later reads its own 16 bytes of rows g, g+8 of each row tile) and the 16-byte scale chunk
    // [8c, 8c + 8) holding the window's two groups for every row (lane L copies row L).
    // All shared-memory addresses are 32-bit offsets fixed per lane, plus a per-stage base.
    constexpr int ROWS = RT * 16;
    constexpr uint32_t kCodeStage = ROWS * 64, kScStage = ROWS * 16;
    const uint32_t cring_u = smem_u32(ring);
    const uint32_t sring_u = cring_u + kStages * kCodeStage;
    const uint32_t frag_lane_u = smem_u32(frag) + (((g >> 1) * 4 + q) * 8);
    constexpr uint32_t kFragWindow = 16 * BS * 4 * 8;
    uint32_t coff[RT][2], soff[RT][2];
#pragma unroll
    for (int rt = 0; rt < RT; rt++)
#pragma unroll
      for (int hr = 0; hr < 2; hr++) {
        coff[rt][hr] = (rt * 16 + g + 8 * hr) * 64 + 16 * q;
        soff[rt][hr] = (rt * 16 + g + 8 * hr) * 16;
      }
    const int npair = (ngroups + 1) / 2;
    const int total = my_tiles * npair;
    // issue cursor
    int is_tile = 0, is_pw = 0;
    uint32_t is_cdst = cring_u, is_sdst = sring_u + lane * 16;
    const uint8_t* rp[RT][2];
    uint32_t rsz[RT][2];
    const uint16_t* srow = a.scales;
    uint32_t ssz = 0;
    auto set_issue_tile = [&](int ti) {
      const int row0 = (first + ti * stride) * ROWS;
#pragma unroll
      for (int rt = 0; rt < RT; rt++)
#pragma unroll
        for (int hr = 0; hr < 2; hr++) {
          const int row = row0 + rt * 16 + g + 8 * hr;
          rsz[rt][hr] = row < a.n ? 16u : 0u;
          rp[rt][hr] = a.codes + (int64_t)(row < a.n ? row : 0) * a.cstride + (int64_t)g0 * 32 + 16 * q;
        }
      const int srow_i = row0 + lane;
      ssz = (lane < ROWS && srow_i < a.n) ? 16u : 0u;
      srow = a.scales + (int64_t)(ssz ? srow_i : 0) * a.sstride;
    };
    auto issue_next = [&]() {
      const int gl0 = 2 * is_pw;
      const uint32_t mine = ((q >> 1) < ngroups - gl0) ? 0xFFFFFFFFu : 0u;  // the last window may be half
#pragma unroll
      for (int rt = 0; rt < RT; rt++)
#pragma unroll
        for (int hr = 0; hr < 2; hr++) cp_async16_u32(is_cdst + coff[rt][hr], rp[rt][hr] + gl0 * 32, rsz[rt][hr] & mine);
      // one scale row per lane; with 16-row tiles lanes 16..31 issue nothing (a zero-size copy
      // would still zero-fill its 16 destination bytes, outside this stage)
      if (ROWS == 32 || lane < ROWS) cp_async16_u32(is_sdst, srow + ((g0 + gl0) & ~7), ssz);
      is_cdst += kCodeStage;
      is_sdst += kScStage;
      if (is_cdst == cring_u + kStages * kCodeStage) {
        is_cdst = cring_u;
        is_sdst = sring_u + lane * 16;
      }
      if (++is_pw == npair) {
        is_pw = 0;
        if (++is_tile < my_tiles) set_issue_tile(is_tile);
      }
    };
    if (total > 0) set_issue_tile(0);
    for (int st = 0; st < kStages - 1; st++) {
      if (st < total) issue_next();
      cp_async_commit();
    }
    __syncthreads();  // fragments visible to every warp
    int c_tile = 0, c_pw = 0;
    uint32_t c_cbase = cring_u, c_sbase = sring_u;
    for (int st = 0; st < total; st++) {
      if (st + kStages - 1 < total) issue_next();
      cp_async_commit();
      cp_async_wait<kStages - 1>();
      __syncwarp();
      const int gl0 = 2 * c_pw;
      const uint32_t sb = c_sbase + 2 * ((g0 + gl0) & 7);
      uint4 cw[RT][2];
      uint32_t sc[RT][2];
#pragma unroll
      for (int rt = 0; rt < RT; rt++)
#pragma unroll
        for (int hr = 0; hr < 2; hr++) {
          cw[rt][hr] = lds128(c_cbase + coff[rt][hr]);
          sc[rt][hr] = lds32(sb + soff[rt][hr]);
        }
      mma_pair<NT, RT, BS>(cw, sc, frag_lane_u + c_pw * kFragWindow, mul, min(2, ngroups - gl0), bload, bf, acc);
      __syncwarp();
      c_cbase += kCodeStage;
      c_sbase += kScStage;
      if (c_cbase == cring_u + kStages * kCodeStage) {
        c_cbase = cring_u;
        c_sbase = sring_u;
      }
      if (++c_pw == npair) {
        finish_tile<NT, RT>(a, first + c_tile * stride, split, lane, acc);
#pragma unroll
        for (int rt = 0; rt < RT; rt++)
#pragma unroll
          for (int jt = 0; jt < NT; jt++) acc[rt][jt][0] = acc[rt][jt][1] = 0.f;
        c_pw = 0;
        c_tile++;
      }
    }
  } else {
    constexpr int ROWS = RT * 16;
    const int n5 = (ngroups + kT3Window - 1) / kT3Window;
    const int total = my_tiles * n5;
    uint8_t* q2buf = ring + (size_t)kT3Stages * (ROWS * 128 + ROWS * 32);
    auto issue = [&](int st) {
      const int i = st / n5, w5 = st - i * n5;
      issue_t3<RT>(a, ring, st % kT3Stages, first + i * stride, g0 + w5 * kT3Window, lane);
    };
    for (int st = 0; st < kT3Stages - 1; st++) {
      if (st < total) issue(st);
      cp_async_commit();
    }
    __syncthreads();  // fragments and table visible to every warp
    for (int st = 0; st < total; st++) {
      if (st + kT3Stages - 1 < total) issue(st + kT3Stages - 1);
      cp_async_commit();
      cp_async_wait<kT3Stages - 1>();
      __syncwarp();
      const int slot = st % kT3Stages;
      const int i = st / n5, w5 = st - i * n5;
      const int grp0 = g0 + w5 * kT3Window;
      const int gn = min(kT3Window, ngroups - w5 * kT3Window);
      expand_t3<RT>(ring + (size_t)slot * ROWS * 128, lut, q2buf, lane);
      __syncwarp();
      const uint16_t* scs = reinterpret_cast<const uint16_t*>(ring + (size_t)kT3Stages * ROWS * 128 + (size_t)slot * ROWS * 32);
      const int sbase = grp0 - 8 * (grp0 >> 3);  // first group of the window inside the 16-scale chunk pair
      for (int iw = 0; iw < (gn + 1) / 2; iw++) {
        const int gh = min(2, gn - 2 * iw);
        const bool mine = (q >> 1) < gh;
        uint4 cw[RT][2];
        uint32_t sc[RT][2];
#pragma unroll
        for (int rt = 0; rt < RT; rt++)
#pragma unroll
          for (int hr = 0; hr < 2; hr++) {
            const int r = rt * 16 + g + 8 * hr;
            cw[rt][hr] = mine ? *reinterpret_cast<const uint4*>(q2buf + r * kQ2RowStride + (2 * iw) * 32 + 16 * q)
                              : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t s_lo = scs[r * 16 + sbase + 2 * iw];
            const uint32_t s_hi = scs[r * 16 + sbase + 2 * iw + 1];
            sc[rt][hr] = s_lo | (s_hi << 16);
          }
        mma_pair<NT, RT, BS>(cw, sc, smem_u32(frag) + ((((3 * w5 + iw) * 16 * BS + (g >> 1)) * 4 + q) * 8), mul, gh,
                             bload, bf, acc);
      }
      __syncwarp();
      if (w5 == n5 - 1) {
        finish_tile<NT, RT>(a, first + i * stride, split, lane, acc);
#pragma unroll
        for (int rt = 0; rt < RT; rt++)
#pragma unroll
          for (int jt = 0; jt < NT; jt++) acc[rt][jt][0] = acc[rt][jt][1] = 0.f;
      }
    }
  }
  cp_async_wait<0>();
}

// ---- small batches: every layout decoded in registers -----------------------------------------------
// One window = 64 code bytes of every row of a warp tile: 256 weights (two groups) of Q2_0_g128,
// 320 weights of the base-3 layout or 512 weights (four groups) of the binary Q1_0_g128. Lane (g, q) owns bytes [16q, 16q + 16) of rows g and g + 8 of
// each 16-row tile, decodes them straight into mma.sync A fragments and never writes codes back to
// shared memory:
//   * Q2_0_g128: slot S of a 16-code word is (word * 2^(14 - 2S)) & 0xC000C000 (see slot()).
//   * Q1_0_g128: slot S of a 32-bit word is bits (S, S + 16) placed as two signs (see slot_bin());
//     a lane's 16 bytes are exactly one group.
//   * base-3: bytes (0, 2) and (1, 3) of a word sit in 16-bit lanes V; with c = t + 1 the five digits
//     come out most significant first from one multiply-add and a chain of "times three" steps:
//     R = V * 202 + 130 maps each byte v to r = floor(R / 64) in [256 v / 81, 256 (v + 1) / 81), so
//     bits 14..15 of R hold the leading digit and bits 6..13 the scaled remainder p; R' = 3 p * 64
//     then yields the next digit the same way. Adding 0xC000 per lane turns the digit c into the
//     two's-complement field of t = c - 1, i.e. the fp16 +-2 / 0 pattern of slot(). Exhaustively
//     checked over all byte pairs (the carry one lane passes to the other only touches bits that are
//     masked or already garbage); an invalid byte (> 242) gives unspecified trits.
// The MMA columns are (batch, group-within-window) pairs: a base-3 window touches three groups, so a
// lane's four k-slots may belong to two groups and the activation fragments are stored per column.
// A binary window holds four groups, so its eight columns carry two batch rows.
// Two CTA shapes, NW warps x CPS CTAs per SM: 16 x 1 puts all of an SM's warps on the few row tiles
// of a small matrix; 8 x 2 (two independent CTAs per SM, each with its own fragment build and
// reduction) is faster once there are several row tiles per CTA.
constexpr int kWinBytes = 64;

template <int LAYOUT> struct Lay;
template <> struct Lay<TERN_Q2_0_G128> {
  static constexpr int J = 16;   // MMAs per 16-row tile and window
  static constexpr int C = 1;    // stored fragment columns per batch row (the lane's group is q / 2)
  static constexpr int SC = 1;   // 16-byte scale chunks per row and window
  static constexpr int W = 256;  // weights per row and window
};
template <> struct Lay<TERN_T3_5PB_G128> {
  static constexpr int J = 20;
  static constexpr int C = 3;
  static constexpr int SC = 2;
  static constexpr int W = 320;
};
template <> struct Lay<TERN_Q1_0_G128> {
  static constexpr int J = 32;
  static constexpr int C = 1;    // the lane's group is q
  static constexpr int SC = 1;
  static constexpr int W = 512;
};

__host__ __device__ inline int s_windows(int layout, int ngroups) {
  return layout == TERN_Q2_0_G128   ? (ngroups + 1) / 2
         : layout == TERN_Q1_0_G128 ? (ngroups + 3) / 4
                                    : (ngroups * kGroup + 319) / 320;
}
__host__ __device__ constexpr uint32_t s_frag_window_bytes(int layout, int bs) {
  return layout == TERN_Q2_0_G128   ? 8u * bs * 1 * 4 * 16
         : layout == TERN_Q1_0_G128 ? 16u * bs * 1 * 4 * 16
                                    : 10u * bs * 3 * 4 * 16;
}
__host__ __device__ constexpr uint32_t s_stage_bytes(int layout, int rt) {
  return (uint32_t)rt * 16 * (kWinBytes + 16 * (layout == TERN_T3_5PB_G128 ? 2 : 1));
}
__host__ __device__ inline size_t s_smem_bytes(int layout, int rt, int stages, int gps, int bs, int nw) {
  return (size_t)s_frag_window_bytes(layout, bs) * (s_windows(layout, gps) + 1) +
         (size_t)nw * stages * (s_stage_bytes(layout, rt) + 8) + 16;  // + full barriers, abort flag
}

__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}


// Activation fragments of one K slice, one entry (uint2 = the lane's b0, b1) per
// [window][mma j / 2][batch slot][column c < C][q][j % 2], so a lane reads two MMAs' worth with one
// 16-byte load. Column c is the group within the window (base-3) or implied by q (Q2). One extra
// window of zeros follows: lanes whose MMA column carries no data read it.
// Built from (window, lane chunk q, batch row, half) units whose code positions are compile-time.
template <int LAYOUT, int BS, int HF>
__device__ __forceinline__ void s_frag_half(const Args& a, int g0, int kslice, int w, int q, int b, uint16_t* fh) {
  using L = Lay<LAYOUT>;
  constexpr int HW = L::W / 8;  // weights of a lane chunk half: 32 (Q2), 40 (base-3) or 64 (binary)
  const int k0 = w * L::W + (L::W / 4) * q + HF * HW;  // first weight within the slice
  const uint16_t* xs = a.x + (int64_t)b * a.k + (int64_t)g0 * kGroup + k0;
  uint32_t xw[HW / 2];
#pragma unroll
  for (int v = 0; v < HW / 8; v++) {
    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
    if (k0 + 8 * v < kslice) xv = *reinterpret_cast<const uint4*>(xs + 8 * v);
    xw[4 * v] = xv.x; xw[4 * v + 1] = xv.y; xw[4 * v + 2] = xv.z; xw[4 * v + 3] = xv.w;
  }
  const int colbase = LAYOUT == TERN_Q2_0_G128 ? 0 : 320 * (w & 1) + 80 * q + HF * HW;
#pragma unroll
  for (int cc = 0; cc < HW; cc++) {
    const int c = HF * HW + cc;  // position within the lane's chunk
    int j, e4, col = 0;
    if (LAYOUT == TERN_Q2_0_G128) {
      const int word = c >> 4, i = c & 15, S = i & 7;
      j = 4 * word + (S >> 1);
      e4 = 2 * (S & 1) + (i >> 3);
    } else if (LAYOUT == TERN_Q1_0_G128) {
      const int word = c >> 5, i = c & 31, S = i & 15;
      j = 8 * word + (S >> 1);
      e4 = 2 * (S & 1) + (i >> 4);
    } else {
      const int bl = c / 5, d = c - 5 * bl, word = bl >> 2, bb = bl & 3;
      const int r = 5 * (bb & 1) + (4 - d);
      j = 5 * word + (r >> 1);
      e4 = 2 * (r & 1) + (bb >> 1);
      col = ((colbase + cc) >> 7) - 2 * (w & 1);
    }
    const int entry = (((((w * (L::J / 2) + (j >> 1)) * BS + b) * L::C + col) * 4 + q) * 2 + (j & 1));
    fh[entry * 4 + e4] = (uint16_t)(xw[cc >> 1] >> (16 * (cc & 1)));
  }
}

template <int LAYOUT, int BS, int NT>
__device__ void s_build_frag(const Args& a, int g0, int ngroups, int nwin_alloc, uint8_t* frag) {
  constexpr uint32_t FW = s_frag_window_bytes(LAYOUT, BS);
  uint4* f4 = reinterpret_cast<uint4*>(frag);
  if (LAYOUT != TERN_T3_5PB_G128) {
    // every entry a data lane reads is written below (zero past the slice); only the zero block
    for (int i = threadIdx.x; i < (int)(FW / 16); i += NT)
      f4[(size_t)nwin_alloc * FW / 16 + i] = make_uint4(0u, 0u, 0u, 0u);
  } else {
    // base-3 entries hold one group column each: the other columns must read as zero
    for (int i = threadIdx.x; i < (int)((nwin_alloc + 1) * FW / 16); i += NT) f4[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
  }
  uint16_t* fh = reinterpret_cast<uint16_t*>(frag);
  const int kslice = ngroups * kGroup;
  const int nwin = s_windows(LAYOUT, ngroups);
  const int items = nwin * 4 * a.batch * 2;
  for (int e = threadIdx.x; e < items; e += NT) {
    const int hf = e & 1, q = (e >> 1) & 3, rest = e >> 3;
    const int b = rest % a.batch, w = rest / a.batch;
    if (hf == 0) s_frag_half<LAYOUT, BS, 0>(a, g0, kslice, w, q, b, fh);
    else s_frag_half<LAYOUT, BS, 1>(a, g0, kslice, w, q, b, fh);
  }
}

// Stream-K bookkeeping of the small-batch kernel. In every K slice the units (tile, window), tile-
// major, are cut into runs of a.run consecutive units, run i going to warp i / gridDim.x of CTA
// i % gridDim.x (the last run may be shorter; warps past the last run idle). The runs that touch a
// tile are consecutive and each writes one partial-sum slot.
template <int LAYOUT>
__device__ __forceinline__ int s_nseg(const Args& a, int split, int tile) {  // runs touching a tile in a slice
  const int ng = min(a.gps, a.groups - split * a.gps);
  const int nwin = s_windows(LAYOUT, ng);
  const uint32_t f = (uint32_t)tile * nwin;
  return (int)((f + nwin - 1) / (uint32_t)a.run - f / (uint32_t)a.run) + 1;
}

template <int LAYOUT>
__device__ __forceinline__ int s_contributors(const Args& a, int tile) {  // runs touching a tile, all slices
  int c = 0;
  for (int sp = 0; sp < a.splits; sp++) c += s_nseg<LAYOUT>(a, sp, tile);
  return c;
}

// Lane (g, q) accumulates rows g, g + 8 of each 16-row tile. Q2: lane q holds batch q. Base-3 and
// binary: lanes q and q ^ 1 hold batch q / 2 (base-3: groups 0-1 and 2 of each window; binary: groups
// 0-1 and 2-3) and are summed here; the even lane of the pair stores.
template <int LAYOUT, int RT>
__device__ __forceinline__ void s_combine(float (&acc)[RT][2], int& b, bool& owner, int q) {
  b = q;
  owner = true;
  if (LAYOUT != TERN_Q2_0_G128) {
#pragma unroll
    for (int rt = 0; rt < RT; rt++)
#pragma unroll
      for (int hr = 0; hr < 2; hr++) acc[rt][hr] += __shfl_xor_sync(0xFFFFFFFFu, acc[rt][hr], 1);
    b = q >> 1;
    owner = (q & 1) == 0;
  }
}

// y for a tile this run covers alone, or the run's fp32 partial in its (slice, rank) slot.
template <int LAYOUT, int RT>
__device__ __forceinline__ void s_store(const Args& a, int tile, int slot, int lane, float (&acc)[RT][2]) {
  const int g = lane >> 2, q = lane & 3;
  int b;
  bool owner;
  s_combine<LAYOUT, RT>(acc, b, owner, q);
  const int row_base = tile * 16 * RT;
  float* part = slot >= 0 ? a.ws + (size_t)slot * a.batch * a.n : nullptr;
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int hr = 0; hr < 2; hr++) {
      const int row = row_base + rt * 16 + g + 8 * hr;
      if (owner && row < a.n && b < a.batch) {
        if (slot < 0) a.y[(int64_t)b * a.n + row] = __half_as_ushort(__float2half_rn(0.5f * acc[rt][hr]));
        else part[(size_t)b * a.n + row] = 0.5f * acc[rt][hr];
      }
    }
}

// The last run to arrive at a tile sums every slot in (slice, rank) order (so the result does not
// depend on timing), stores y and re-arms the tile's counter for the next call.
template <int LAYOUT, int RT>
__device__ __forceinline__ void s_reduce_tile(const Args& a, int tile, int lane) {
  const int row_base = tile * 16 * RT;
  const int rows = min(16 * RT, a.n - row_base);
  for (int e = lane; e < rows * a.batch; e += 32) {
    const int bb = e / rows, row = row_base + e % rows;
    float v = 0.f;
    for (int sp = 0; sp < a.splits; sp++) {
      const int ns = s_nseg<LAYOUT>(a, sp, tile);
      const float* src = a.ws + ((size_t)(sp * a.kmax) * a.batch + bb) * a.n + row;
      const size_t slot_stride = (size_t)a.batch * a.n;
      float pv[4];
      int k = 0;
      for (; k + 4 <= ns; k += 4) {
#pragma unroll
        for (int u = 0; u < 4; u++) pv[u] = __ldcg(src + (k + u) * slot_stride);
#pragma unroll
        for (int u = 0; u < 4; u++) v += pv[u];
      }
      for (; k < ns; k++) v += __ldcg(src + k * slot_stride);
    }
    a.y[(int64_t)bb * a.n + row] = __half_as_ushort(__float2half_rn(v));
  }
  __syncwarp();
  if (lane == 0) a.counters[tile] = 0;
}

// Publishes the partial slots a run wrote (at most two tiles: the one it started inside and the one
// it ended inside) with one fence, then takes part in the arrival count of each; the partial stores
// and the fence are issued by every lane before lane 0's atomics, and the last arriver fences again
// before reading the other runs' slots.
template <int LAYOUT, int RT>
__device__ __forceinline__ void s_publish(const Args& a, const int (&tile)[2], const int (&contrib)[2], int n, int lane) {
  __threadfence();
  __syncwarp();
  int prev[2] = {0, 0};
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < 2; i++)
      if (i < n) prev[i] = atomicAdd(a.counters + tile[i], 1);
  }
#pragma unroll
  for (int i = 0; i < 2; i++) {
    if (i >= n) break;
    const int p = __shfl_sync(0xFFFFFFFFu, prev[i], 0);
    if (p == contrib[i] - 1) {
      __threadfence();
      s_reduce_tile<LAYOUT, RT>(a, tile[i], lane);
    }
  }
}

constexpr uint64_t kRegWaitLimitNs = 1000000000ull;  // 1 s: far beyond any healthy TMA latency

template <int LAYOUT, int RT, int BS, int STAGES, int NW, int CPS>
__global__ void __launch_bounds__(NW * 32, CPS)
    gemv_reg_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales, Args a) {
  using L = Lay<LAYOUT>;
  constexpr int ROWS = RT * 16;
  constexpr uint32_t FW = s_frag_window_bytes(LAYOUT, BS);
  constexpr uint32_t STAGE = s_stage_bytes(LAYOUT, RT);
  constexpr uint32_t kCodeBytes = ROWS * kWinBytes;
  constexpr uint32_t kJP = BS * L::C * 64;  // bytes between fragment pairs (j / 2) of one window
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int split = blockIdx.y;
  const int g0 = split * a.gps;
  const int ngroups = min(a.gps, a.groups - g0);
  const int nwin = s_windows(LAYOUT, ngroups);
  const int nwin_alloc = s_windows(LAYOUT, a.gps);
  uint8_t* frag = smem;
  uint8_t* rings = smem + (size_t)(nwin_alloc + 1) * FW;
  uint8_t* ring = rings + (size_t)warp * STAGES * STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(rings + (size_t)NW * STAGES * STAGE) + warp * STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(
      reinterpret_cast<uint64_t*>(rings + (size_t)NW * STAGES * STAGE) + NW * STAGES);

  if (lane == 0) {
    for (int s = 0; s < STAGES; s++) sm100::mbar_init(full + s, 1);
    sm100::fence_mbar_init();
    sm100::prefetch_tmap(&tm_codes);
    sm100::prefetch_tmap(&tm_scales);
  }
  if (threadIdx.x == 0) *abort_flag = 0;
  __syncwarp();
  // The next kernel on the stream may be scheduled as soon as this grid's CTAs leave their SMs
  // (programmatic dependent launch; a no-op for plain launches).
  sm100::griddep_launch_dependents();

  // this warp's run of (tile, window) units in the slice (empty past the last run).
  //   stream-K: runs of a.run units are dealt to CTAs round-robin, so both CTAs on an SM, and all SMs,
  //     get the same number of runs (+-1); tiles shared by runs are summed through the workspace.
  //   a.local: CTA c owns the whole tiles [t_lo, t_hi) (counts differ by at most one) and its warps
  //     split their units into equal runs; shared tiles are summed in shared memory.
  int wi, u_begin, u_end, t_lo = 0, t_hi = 0, lrun = 1, lbase = 0;
  if (a.local) {
    t_lo = (int)(((long long)blockIdx.x * a.tiles) / gridDim.x);
    t_hi = (int)(((long long)(blockIdx.x + 1) * a.tiles) / gridDim.x);
    const int ucta = (t_hi - t_lo) * nwin;
    lrun = max(1, (ucta + NW - 1) / NW);
    lbase = t_lo * nwin;
    wi = warp;
    u_begin = lbase + min(warp * lrun, ucta);
    u_end = lbase + min(warp * lrun + lrun, ucta);
  } else {
    wi = blockIdx.x + warp * gridDim.x;
    const int units = a.tiles * nwin;
    u_begin = min(wi * a.run, units);
    u_end = min(u_begin + a.run, units);
  }
  const int total = u_end - u_begin;
  const int tile0 = u_begin / nwin, w0 = u_begin - tile0 * nwin;

  // ---- issue side (lane 0): one TMA box of codes [ROWS][64 B] and one of scales per window; reads
  // past the row data, the scale columns or the last row are zero-filled by the tensor maps
  const int slice_x0 = LAYOUT == TERN_Q2_0_G128   ? g0 * (kGroup / 4)
                       : LAYOUT == TERN_Q1_0_G128 ? g0 * (kGroup / 8)
                                                  : (g0 / 5) * 128;
  int is_tile = tile0, is_w = w0, is_slot = 0;
  auto issue_next = [&]() {
    uint64_t* bar = full + is_slot;
    uint8_t* dst = ring + is_slot * STAGE;
    const int gfirst = LAYOUT == TERN_Q2_0_G128   ? g0 + 2 * is_w
                       : LAYOUT == TERN_Q1_0_G128 ? g0 + 4 * is_w
                                                  : g0 + (5 * is_w) / 2;
    sm100::mbar_arrive_expect_tx(bar, STAGE);
    sm100::tma_load_2d(dst, &tm_codes, bar, slice_x0 + kWinBytes * is_w, is_tile * ROWS);
    sm100::tma_load_2d(dst + kCodeBytes, &tm_scales, bar, 8 * (gfirst >> 3), is_tile * ROWS);
    if (++is_slot == STAGES) is_slot = 0;
    if (++is_w == nwin) {
      is_w = 0;
      ++is_tile;
    }
  };
  // With a.early the first code / scale boxes are requested before waiting for the preceding grid: the
  // caller guarantees that no work still in flight writes W. x, y and the workspace are only touched
  // after the wait, which returns at once for plain launches.
  if (a.early && lane == 0)
    for (int st = 0; st < STAGES && st < total; st++) issue_next();
  sm100::griddep_wait();
  if (!a.early && lane == 0)
    for (int st = 0; st < STAGES && st < total; st++) issue_next();

  s_build_frag<LAYOUT, BS, NW * 32>(a, g0, ngroups, nwin_alloc, frag);

  // B column of this lane and the fragment address it reads (zero block when it carries no data)
  int fb, fcol;
  bool fdata;
  if (LAYOUT == TERN_Q2_0_G128) {
    fb = g >> 1; fcol = 0; fdata = ((g & 1) == (q >> 1)) && fb < a.batch;
  } else if (LAYOUT == TERN_Q1_0_G128) {
    fb = g >> 2; fcol = 0; fdata = ((g & 3) == q) && fb < a.batch;
  } else {
    fb = g >> 2; fcol = g & 3; fdata = fcol < 3 && fb < a.batch;
  }
  const uint32_t fbase = fdata ? smem_u32(frag) + ((fb * L::C + fcol) * 4 + q) * 16
                               : smem_u32(frag) + (uint32_t)nwin_alloc * FW;
  const uint32_t fstep = fdata ? FW : 0u;

  uint32_t mul[8], mulb[16];
#pragma unroll
  for (int S = 0; S < 8; S++) mul[S] = a.unit << (14 - 2 * S);
#pragma unroll
  for (int S = 0; S < 16; S++) mulb[S] = a.unit << (15 - S);
  const uint32_t k0 = a.unit * (130u | (130u << 16)) + 0xC000C000u;

  float acc[RT][2];
#pragma unroll
  for (int rt = 0; rt < RT; rt++) acc[rt][0] = acc[rt][1] = 0.f;

  __syncthreads();  // fragments and barrier initialisation visible to every warp
  const uint32_t ring_u = smem_u32(ring);
  const uint32_t lane_code = (g * kWinBytes) + 16 * q;       // + (rt * 16 + 8 hr) * 64
  const uint32_t lane_scale = kCodeBytes + g * (16 * L::SC);  // + (rt * 16 + 8 hr) * 16 * SC
  int c_tile = tile0, c_w = w0, c_slot = 0;
  int pend_tile[2] = {0, 0}, pend_contrib[2] = {0, 0}, npend = 0;  // partial tiles awaiting their count
  float first_part[RT][2];  // a.local: partial of the run's first tile when that tile is shared
  bool has_first = false;
  int st = 0;
  for (; st < total; st++) {
    if (!sm100::mbar_wait_bounded(full + c_slot, (st / STAGES) & 1, abort_flag, a.status, TERN_DEVICE_TIMEOUT,
                                  a.wait_ns))
      break;
    const uint32_t stage_u = ring_u + c_slot * STAGE;
    // codes of the window; activation fragments follow one code word ahead of the MMAs that use them
    // (fewer live registers than a whole window's worth, latency still covered)
    const uint32_t fa = fbase + (uint32_t)c_w * fstep;
    uint4 cw[RT][2];
#pragma unroll
    for (int rt = 0; rt < RT; rt++)
#pragma unroll
      for (int hr = 0; hr < 2; hr++) cw[rt][hr] = lds128(stage_u + lane_code + (rt * 16 + 8 * hr) * kWinBytes);
    // fragment pairs a word needs: Q2 word w uses pairs 2w, 2w + 1; binary word w pairs 4w .. 4w + 3;
    // base-3 word w pairs floor(5w / 2) .. floor((5w + 4) / 2)
    constexpr int NB = LAYOUT == TERN_Q2_0_G128 ? 2 : LAYOUT == TERN_Q1_0_G128 ? 4 : 3;
    auto pair0 = [](int word) {
      return LAYOUT == TERN_Q2_0_G128 ? 2 * word : LAYOUT == TERN_Q1_0_G128 ? 4 * word : (5 * word) >> 1;
    };
    uint4 bcur[NB], bnext[NB];
#pragma unroll
    for (int i = 0; i < NB; i++) bcur[i] = lds128(fa + (pair0(0) + i) * kJP);
    float d[RT][4];
#pragma unroll
    for (int word = 0; word < 4; word++) {
      if (word < 3) {
#pragma unroll
        for (int i = 0; i < NB; i++) bnext[i] = lds128(fa + (pair0(word + 1) + i) * kJP);
      }
      if (LAYOUT == TERN_Q1_0_G128) {
        uint32_t wl[RT], wh[RT];
#pragma unroll
        for (int rt = 0; rt < RT; rt++) {
          wl[rt] = word == 0 ? cw[rt][0].x : word == 1 ? cw[rt][0].y : word == 2 ? cw[rt][0].z : cw[rt][0].w;
          wh[rt] = word == 0 ? cw[rt][1].x : word == 1 ? cw[rt][1].y : word == 2 ? cw[rt][1].z : cw[rt][1].w;
        }
#pragma unroll
        for (int sp = 0; sp < 8; sp++) {
          const int j = 8 * word + sp;
          const uint4 bq = bcur[(j >> 1) - pair0(word)];
          const uint32_t b0 = (j & 1) ? bq.z : bq.x, b1 = (j & 1) ? bq.w : bq.y;
#pragma unroll
          for (int rt = 0; rt < RT; rt++) {
            const uint32_t a0 = slot_bin(wl[rt], mulb[2 * sp]), a2 = slot_bin(wl[rt], mulb[2 * sp + 1]);
            const uint32_t a1 = slot_bin(wh[rt], mulb[2 * sp]), a3 = slot_bin(wh[rt], mulb[2 * sp + 1]);
            if (j == 0) mma_f16_first(d[rt], a0, a1, a2, a3, b0, b1);
            else mma_f16(d[rt], a0, a1, a2, a3, b0, b1);
          }
        }
      } else if (LAYOUT == TERN_Q2_0_G128) {
        uint32_t wl[RT], wh[RT];
#pragma unroll
        for (int rt = 0; rt < RT; rt++) {
          wl[rt] = word == 0 ? cw[rt][0].x : word == 1 ? cw[rt][0].y : word == 2 ? cw[rt][0].z : cw[rt][0].w;
          wh[rt] = word == 0 ? cw[rt][1].x : word == 1 ? cw[rt][1].y : word == 2 ? cw[rt][1].z : cw[rt][1].w;
        }
#pragma unroll
        for (int sp = 0; sp < 4; sp++) {
          const int j = 4 * word + sp;
          const uint4 bq = bcur[(j >> 1) - pair0(word)];
          const uint32_t b0 = (j & 1) ? bq.z : bq.x, b1 = (j & 1) ? bq.w : bq.y;
#pragma unroll
          for (int rt = 0; rt < RT; rt++) {
            const uint32_t a0 = slot(wl[rt], mul[2 * sp]), a2 = slot(wl[rt], mul[2 * sp + 1]);
            const uint32_t a1 = slot(wh[rt], mul[2 * sp]), a3 = slot(wh[rt], mul[2 * sp + 1]);
            if (j == 0) mma_f16_first(d[rt], a0, a1, a2, a3, b0, b1);
            else mma_f16(d[rt], a0, a1, a2, a3, b0, b1);
          }
        }
      } else {
        uint32_t o[RT][2][10];
#pragma unroll
        for (int rt = 0; rt < RT; rt++)
#pragma unroll
          for (int hr = 0; hr < 2; hr++) {
            const uint32_t wv = word == 0 ? cw[rt][hr].x : word == 1 ? cw[rt][hr].y : word == 2 ? cw[rt][hr].z : cw[rt][hr].w;
            dec_t3_word(wv, k0, o[rt][hr]);
          }
#pragma unroll
        for (int m = 0; m < 5; m++) {
          const int j = 5 * word + m;
          const uint4 bq = bcur[(j >> 1) - pair0(word)];
          const uint32_t b0 = (j & 1) ? bq.z : bq.x, b1 = (j & 1) ? bq.w : bq.y;
#pragma unroll
          for (int rt = 0; rt < RT; rt++) {
            if (j == 0) mma_f16_first(d[rt], o[rt][0][2 * m], o[rt][1][2 * m], o[rt][0][2 * m + 1], o[rt][1][2 * m + 1], b0, b1);
            else mma_f16(d[rt], o[rt][0][2 * m], o[rt][1][2 * m], o[rt][0][2 * m + 1], o[rt][1][2 * m + 1], b0, b1);
          }
        }
      }
      if (word < 3) {
#pragma unroll
        for (int i = 0; i < NB; i++) bcur[i] = bnext[i];
      }
    }
    // the two scales this lane's columns use, per row (columns without data have D = 0)
    float sa[RT][2], sb[RT][2];
    {
      const int gfirst = LAYOUT == TERN_Q2_0_G128   ? g0 + 2 * c_w
                         : LAYOUT == TERN_Q1_0_G128 ? g0 + 4 * c_w
                                                    : g0 + (5 * c_w) / 2;
      const int ja = LAYOUT == TERN_Q2_0_G128 ? 0 : 2 * (q & 1);
      const uint32_t so = stage_u + lane_scale + 2 * ((gfirst & 7) + ja);
#pragma unroll
      for (int rt = 0; rt < RT; rt++)
#pragma unroll
        for (int hr = 0; hr < 2; hr++) {
          const uint32_t ra = so + (rt * 16 + 8 * hr) * (16 * L::SC);
          if (LAYOUT != TERN_T3_5PB_G128) {
            const uint32_t pr = lds32(ra);  // groups gfirst + ja, gfirst + ja + 1 (an even first group)
            const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&pr));
            sa[rt][hr] = sf.x;
            sb[rt][hr] = sf.y;
          } else {
            sa[rt][hr] = __half2float(__ushort_as_half((unsigned short)lds16(ra)));
            sb[rt][hr] = __half2float(__ushort_as_half((unsigned short)lds16(ra + 2)));
          }
        }
    }
    // lane (g, q) holds columns 2q, 2q + 1 of rows g (d[0..1]) and g + 8 (d[2..3]); D = 2 sum t x
#pragma unroll
    for (int rt = 0; rt < RT; rt++)
#pragma unroll
      for (int hr = 0; hr < 2; hr++)
        acc[rt][hr] = fmaf(sb[rt][hr], d[rt][2 * hr + 1], fmaf(sa[rt][hr], d[rt][2 * hr], acc[rt][hr]));
    // every lane has read this stage: refill it with the window STAGES ahead
    __syncwarp();
    if (lane == 0 && st + STAGES < total) issue_next();
    if (++c_slot == STAGES) c_slot = 0;
    if (++c_w == nwin || st == total - 1) {
      // end of this warp's run inside the tile: a tile covered by this run alone gets y now; a shared
      // one gets this run's partial in the slot of its rank among the tile's runs (workspace), or in
      // this warp's first- or last-tile slot in shared memory (a.local)
      int contributors;
      if (a.local) {
        const int rel0 = c_tile * nwin - lbase;
        contributors = (rel0 + nwin - 1) / lrun - rel0 / lrun + 1;
      } else {
        contributors = s_contributors<LAYOUT>(a, c_tile);
      }
      if (contributors == 1) {
        s_store<LAYOUT, RT>(a, c_tile, -1, lane, acc);
      } else if (a.local) {
        // the partial of the run's first tile waits in registers; the last tile's is only reached at
        // the run's last window, when every box of this warp's ring has been consumed, so it goes
        // straight to the ring (partials: [first / last tile][lane][rt, hr] floats at the ring base)
        if (c_tile == tile0) {
#pragma unroll
          for (int rt = 0; rt < RT; rt++) {
            first_part[rt][0] = acc[rt][0];
            first_part[rt][1] = acc[rt][1];
          }
          has_first = true;
        } else {
          float* dst = reinterpret_cast<float*>(ring) + (32 + lane) * (2 * RT);
#pragma unroll
          for (int rt = 0; rt < RT; rt++) {
            dst[2 * rt] = acc[rt][0];
            dst[2 * rt + 1] = acc[rt][1];
          }
        }
      } else {
        const int seg = wi - (c_tile * nwin) / a.run;
        s_store<LAYOUT, RT>(a, c_tile, split * a.kmax + seg, lane, acc);
        if (npend == 2) {  // only with several K slices and a run over three or more tiles
          s_publish<LAYOUT, RT>(a, pend_tile, pend_contrib, npend, lane);
          npend = 0;
        }
        pend_tile[npend] = c_tile;
        pend_contrib[npend] = contributors;
        npend++;
      }
#pragma unroll
      for (int rt = 0; rt < RT; rt++) acc[rt][0] = acc[rt][1] = 0.f;
      if (c_w == nwin) {
        c_w = 0;
        c_tile++;
      }
    }
  }
  if (npend) s_publish<LAYOUT, RT>(a, pend_tile, pend_contrib, npend, lane);
  if (a.local) {
    if (has_first) {
      float* dst = reinterpret_cast<float*>(ring) + lane * (2 * RT);
#pragma unroll
      for (int rt = 0; rt < RT; rt++) {
        dst[2 * rt] = first_part[rt][0];
        dst[2 * rt + 1] = first_part[rt][1];
      }
    }
    // every run of the CTA has parked its shared-tile partials; each shared tile is summed by its first
    // contributor, over the contributors in warp order (deterministic), and stored
    __syncthreads();
    for (int t = t_lo; t < t_hi; t++) {
      const int rel0 = t * nwin - lbase;
      if (rel0 / lrun != warp) continue;
      const int wl = (rel0 + nwin - 1) / lrun;
      if (wl == warp) continue;
      float sum[RT][2];
#pragma unroll
      for (int rt = 0; rt < RT; rt++) sum[rt][0] = sum[rt][1] = 0.f;
      for (int w = warp; w <= wl; w++) {
        const int first = (lbase + w * lrun) / nwin;  // the first tile of warp w's run
        const float* src = reinterpret_cast<const float*>(rings + (size_t)w * STAGES * STAGE) +
                           ((t == first ? 0 : 32) + lane) * (2 * RT);
#pragma unroll
        for (int rt = 0; rt < RT; rt++) {
          sum[rt][0] += src[2 * rt];
          sum[rt][1] += src[2 * rt + 1];
        }
      }
      s_store<LAYOUT, RT>(a, t, -1, lane, sum);
    }
  }
  // After a timeout, let the boxes still in flight land (again bounded in time) before the CTA's
  // shared memory is released.
  if (st < total) {
    const int issued = min(total, st + STAGES);
    const uint64_t t0 = sm100::globaltimer_ns();
    for (int k = st; k < issued; k++)
      while (!sm100::mbar_try_wait(full + (k % STAGES), (k / STAGES) & 1) &&
             sm100::globaltimer_ns() - t0 < kRegWaitLimitNs) {
      }
  }
}

// ---- host side ------------------------------------------------------------------------------------
int nt_for(int64_t batch) {
  const int nt = (int)((batch + 3) / 4);
  return nt <= 2 ? nt : nt <= 4 ? 4 : nt <= 8 ? 8 : 16;
}
int rt_for(int nt) { return nt == 1 ? 2 : 1; }
// batch slots of the activation-fragment layout: a compile-time stride >= batch
int bs_for(int64_t batch) { return batch <= 1 ? 1 : batch <= 2 ? 2 : batch <= 4 ? 4 : 4 * nt_for(batch); }

template <int LAYOUT, int NT, int RT, int BS>
cudaError_t launch_t(const Args& a, int gx_hint, cudaStream_t st) {
  const size_t smem = smem_bytes(LAYOUT, RT, a.gps, BS);
  auto kern = gemv_kernel<LAYOUT, NT, RT, BS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // persistent CTAs: at most one full wave, each warp walking row tiles of its CTA's K slice
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int wave = sm_count() * per_sm;
  int gx = (wave + a.splits - 1) / a.splits;
  gx = std::min(gx, std::max(1, gx_hint));
  dim3 grid(gx, a.splits);
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int LAYOUT>
cudaError_t dispatch(const Args& a, int gx_hint, cudaStream_t st) {
  // the register-decode kernel takes Q2_0_g128 batches 1-4 and base-3 batches 1-2
  switch (bs_for(a.batch)) {
    case 4:
      if (LAYOUT == TERN_T3_5PB_G128) return launch_t<LAYOUT, 1, 2, 4>(a, gx_hint, st);
      break;
    case 8: return launch_t<LAYOUT, 2, 1, 8>(a, gx_hint, st);
    case 16: return launch_t<LAYOUT, 4, 1, 16>(a, gx_hint, st);
    case 32: return launch_t<LAYOUT, 8, 1, 32>(a, gx_hint, st);
    case 64: return launch_t<LAYOUT, 16, 1, 64>(a, gx_hint, st);
    default: break;
  }
  return cudaErrorInvalidValue;
}

template <int LAYOUT, int RT, int BS, int STAGES, int NW, int CPS>
cudaError_t launch_reg(const CUtensorMap& tc, const CUtensorMap& ts, const Args& a, int grid_x, cudaStream_t st) {
  const size_t smem = s_smem_bytes(LAYOUT, RT, STAGES, a.gps, BS, NW);
  auto kern = gemv_reg_kernel<LAYOUT, RT, BS, STAGES, NW, CPS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (!a.early) {
    kern<<<dim3(grid_x, a.splits), NW * 32, smem, st>>>(tc, ts, a);
    return cudaGetLastError();
  }
  // programmatic dependent launch: the grid may start while the preceding kernel finishes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_x, a.splits);
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tc, ts, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

#ifndef TERN_REG_RT
#define TERN_REG_RT 2
#endif
#ifndef TERN_REG_STAGES_Q2
#define TERN_REG_STAGES_Q2 4
#endif
#ifndef TERN_REG_STAGES_T3
#define TERN_REG_STAGES_T3 3
#endif
constexpr int kRegRT = TERN_REG_RT;
constexpr int kRegStagesQ2 = TERN_REG_STAGES_Q2;
constexpr int kRegStagesT3 = TERN_REG_STAGES_T3;

bool use_reg_kernel(int32_t layout, int64_t n, int64_t k, int64_t batch) {
  // (tile, window) unit indices are 32-bit
  const int64_t units = (n + 16 * kRegRT - 1) / (16 * kRegRT) * s_windows(layout, (int)(k / kGroup));
  if (units >= ((int64_t)1 << 30)) return false;
  // the binary layout has no other small-batch kernel: larger batches run in pairs of rows
  return layout == TERN_Q2_0_G128 ? batch <= 4 : layout == TERN_Q1_0_G128 ? true : batch <= 2;
}

template <int LAYOUT, int BS, int STAGES>
cudaError_t launch_shape(const CUtensorMap& tc, const CUtensorMap& ts, const Args& a, int grid_x, int warps,
                         cudaStream_t st) {
  if (warps == 8) return launch_reg<LAYOUT, kRegRT, BS, STAGES, 8, 2>(tc, ts, a, grid_x, st);
  return launch_reg<LAYOUT, kRegRT, BS, STAGES, 16, 1>(tc, ts, a, grid_x, st);
}

cudaError_t dispatch_reg(const tern_matrix& W, const Args& a, int grid_x, int warps, cudaStream_t st) {
  // tensor maps: codes [n][row data bytes] in boxes of 64 B x tile rows; scales [n][groups] in boxes
  // of 8 (Q2, binary) or 16 (base-3) groups x tile rows
  const bool q2 = W.layout == TERN_Q2_0_G128, q1 = W.layout == TERN_Q1_0_G128;
  const uint64_t data_bytes = q2 ? (uint64_t)W.k / 4 : q1 ? (uint64_t)W.k / 8 : (uint64_t)(W.k + 4) / 5;
  CUtensorMap tc, ts;
  if (!tmap_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.codes, data_bytes, (uint64_t)W.n, (uint64_t)W.code_row_stride,
               kWinBytes, 16 * kRegRT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!tmap_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT16, W.scales, (uint64_t)(W.k / kGroup), (uint64_t)W.n,
               (uint64_t)W.scale_row_stride * 2, q2 || q1 ? 8 : 16, 16 * kRegRT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (q1) {
    if (a.batch == 1) return launch_shape<TERN_Q1_0_G128, 1, kRegStagesQ2>(tc, ts, a, grid_x, warps, st);
    return launch_shape<TERN_Q1_0_G128, 2, kRegStagesQ2>(tc, ts, a, grid_x, warps, st);
  }
  if (q2) {
    switch (bs_for(a.batch)) {
      case 1: return launch_shape<TERN_Q2_0_G128, 1, kRegStagesQ2>(tc, ts, a, grid_x, warps, st);
      case 2: return launch_shape<TERN_Q2_0_G128, 2, kRegStagesQ2>(tc, ts, a, grid_x, warps, st);
      default: return launch_shape<TERN_Q2_0_G128, 4, kRegStagesQ2>(tc, ts, a, grid_x, warps, st);
    }
  }
  if (a.batch == 1) return launch_shape<TERN_T3_5PB_G128, 1, kRegStagesT3>(tc, ts, a, grid_x, warps, st);
  return launch_shape<TERN_T3_5PB_G128, 2, kRegStagesT3>(tc, ts, a, grid_x, warps, st);
}

}  // namespace

// Register kernel with NW warps x CPS CTAs per SM: the fewest K slices whose activation fragments
// leave room for CPS CTAs per SM, one full wave of CTAs, and the slice's (tile, window) units spread
// evenly over the warps.
static GemvPlan reg_plan_shape(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms, int nw, int cps) {
  GemvPlan p{};
  p.reg = true;
  p.warps = nw;
  if (layout == TERN_Q1_0_G128) batch = std::min<int64_t>(batch, kBinChunk);  // one launch per pair of rows
  const int groups = (int)(k / kGroup);
  // K-slice granularity in groups: one window
  const int unit = layout == TERN_T3_5PB_G128 ? kT3Window : layout == TERN_Q1_0_G128 ? 4 : 2;
  const int units = (groups + unit - 1) / unit;
  const int stages = layout == TERN_T3_5PB_G128 ? kRegStagesT3 : kRegStagesQ2;
  const int bs = bs_for(batch);
  // shared memory of one CTA when cps of them share an SM (228 KB, 1 KB reserved each)
  const size_t cap = (size_t)(228 / cps - 1) * 1024;
  int upc = units;
  while (upc > 1 && s_smem_bytes(layout, kRegRT, stages, upc * unit, bs, nw) > cap) upc = (upc + 1) / 2;
  const int splits = (units + upc - 1) / upc;
  const int gps = std::min(groups, upc * unit);
  const size_t smem = s_smem_bytes(layout, kRegRT, stages, gps, bs, nw);
  const int per_sm = std::max(1, std::min(cps, (int)(227 * 1024 / (smem + 1024))));
  p.rows_per_cta = 16 * kRegRT;
  p.row_blocks = (int)((n + p.rows_per_cta - 1) / p.rows_per_cta);
  p.splits = splits;
  p.groups_per_split = gps;
  const int nwin_full = s_windows(layout, gps);
  const int64_t u_full = (int64_t)p.row_blocks * nwin_full;
  // runs of `run` units, at most one per warp of a full wave; the longest run sets the time
  const int64_t warps = (int64_t)std::max(1, (sms * per_sm) / splits) * nw;
  p.run = (int)std::max<int64_t>(1, (u_full + warps - 1) / warps);
  const int64_t runs = (u_full + p.run - 1) / p.run;
  // a full wave of CTAs whenever there are runs for it (runs are dealt round-robin over CTAs)
  p.grid_x = (int)std::min<int64_t>(std::max(1, (sms * per_sm) / splits), runs);
  p.kmax = (nwin_full - 1 + p.run - 1) / p.run + 1;  // runs that can touch one tile
  // CTA-local reduction when K is one slice and it costs each warp at most one window more than
  // stream-K: no workspace, and the global partial-sum round trips (store, fence, counter, reload)
  // leave the end of the kernel.
  if (splits == 1) {
    const int64_t grid_l = std::min<int64_t>(p.row_blocks, (int64_t)sms * per_sm);
    const int64_t tmax = (p.row_blocks + grid_l - 1) / grid_l;
    const int64_t lwin = (tmax * nwin_full + nw - 1) / nw;
    if (lwin <= p.run + 1) {
      p.local = true;
      p.grid_x = (int)grid_l;
      return p;
    }
  }
  const bool whole_tiles = splits == 1 && p.run % nwin_full == 0;
  if (!whole_tiles) {
    p.ws_partial_bytes = (size_t)splits * p.kmax * batch * n * sizeof(float);
    p.ws_bytes = (p.ws_partial_bytes + (size_t)p.row_blocks * sizeof(int) + 15) / 16 * 16;
  }
  return p;
}

// The CTA shape for a register-kernel launch: 8 warps x 2 CTAs per SM once there are at least four row
// tiles per SM and K still fits one slice in the smaller CTA; 16 warps x 1 CTA otherwise.
static GemvPlan reg_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  const int64_t tiles = (n + 16 * kRegRT - 1) / (16 * kRegRT);
  if (tiles >= 4 * (int64_t)sms) {
    const GemvPlan p = reg_plan_shape(layout, n, k, batch, sms, 8, 2);
    if (p.splits == 1) return p;
  }
  return reg_plan_shape(layout, n, k, batch, sms, 16, 1);
}

// Batches from this size on run on the tcgen05 prefill GEMM kernel: its tensor core takes the decoded
// weights at a fixed rate whatever the number of tokens sharing them, which beats the mma.sync
// kernels once a weight serves this many rows of x.
constexpr int kGemmMinBatch = 17;
// The binary register kernel takes two rows of x per launch, so from this batch on the GEMM kernel
// (one pass over W) is the faster of the two.
constexpr int kGemmMinBatchBinary = 5;
static bool use_gemm(int32_t layout, int64_t n, int64_t batch) {
  return n % 8 == 0 && batch >= (layout == TERN_Q1_0_G128 ? kGemmMinBatchBinary : kGemmMinBatch);
}

bool gemv_supported(int32_t layout, int64_t n, int64_t k, int64_t batch) {
  if (layout != TERN_Q1_0_G128) return true;
  return use_gemm(layout, n, batch) || use_reg_kernel(layout, n, k, batch);
}

GemvPlan gemv_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  // batches 1-2 on the int8-plane kernel; binary batches the GEMM does not take as pairs of rows on it
  const bool bin_pairs = layout == TERN_Q1_0_G128 && !use_gemm(layout, n, batch);
  if (batch <= 2 || bin_pairs) {
    const I8Plan ip = i8_plan(layout, n, k, std::min<int64_t>(batch, 2), sms);
    if (ip.ok) {
      GemvPlan p{};
      p.i8 = true;
      p.i8p = ip;
      p.splits = 1;
      return p;
    }
  }
  if (use_gemm(layout, n, batch)) {
    GemvPlan p{};
    p.gemm = true;
    p.splits = 1;
    return p;
  }
  if (use_reg_kernel(layout, n, k, batch)) return reg_plan(layout, n, k, batch, sms);
  GemvPlan p{};
  const int nt = nt_for(batch);
  const int rt = rt_for(nt);
  p.rows_per_cta = 16 * rt;  // rows per warp tile
  p.row_blocks = (int)((n + p.rows_per_cta - 1) / p.rows_per_cta);
  const int groups = (int)(k / kGroup);
  const int unit = (layout == TERN_T3_5PB_G128) ? kT3Window : 2;  // K-slice granularity in groups
  const int units = (groups + unit - 1) / unit;
  // Enough streaming warps to keep ~10 MB in flight (about 1000 warps); split K only when the row
  // tiles alone cannot supply them.
  const int want_warps = std::min(1024, 7 * sms);
  int splits = std::max(1, std::min(units, (want_warps + p.row_blocks - 1) / p.row_blocks));
  int upc = (units + splits - 1) / splits;
  const size_t smem_cap = 200 * 1024;
  while (upc > 1 && smem_bytes(layout, rt, upc * unit, bs_for(batch)) > smem_cap) upc = (upc + 1) / 2;
  splits = (units + upc - 1) / upc;
  p.splits = splits;
  p.groups_per_split = std::min(groups, upc * unit);
  if (p.splits > 1) {
    p.ws_partial_bytes = (size_t)p.splits * batch * n * sizeof(float);
    p.ws_bytes = (p.ws_partial_bytes + (size_t)p.row_blocks * sizeof(int) + 15) / 16 * 16;
  }
  return p;
}

cudaError_t launch_gemv(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, void* workspace,
                        const GemvPlan& plan, cudaStream_t st, uint32_t flags, uint32_t* status, uint64_t wait_ns,
                        const int8_t* signs) {
  if (plan.i8) {
    // one launch per pair of rows of x, in order on the stream (binary batches 3-4)
    for (int b0 = 0; b0 < batch; b0 += 2) {
      const cudaError_t e = launch_gemv_i8(W, x + (int64_t)b0 * W.k, std::min(2, batch - b0), y + (int64_t)b0 * W.n,
                                           plan.i8p, st, flags, status, wait_ns, signs);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (signs) return cudaErrorInvalidValue;  // only the int8-plane kernel rotates x itself
  if (plan.gemm) return launch_gemm(W, x, batch, y, status, st);
  Args a;
  a.codes = static_cast<const uint8_t*>(W.codes);
  a.cstride = W.code_row_stride;
  a.scales = W.scales;
  a.sstride = W.scale_row_stride;
  a.x = x;
  a.y = y;
  a.n = (int)W.n;
  a.k = (int)W.k;
  a.batch = batch;
  a.groups = (int)(W.k / kGroup);
  a.gps = plan.groups_per_split;
  a.splits = plan.splits;
  a.tiles = plan.row_blocks;
  a.unit = 1u;
  a.run = plan.run;
  a.kmax = plan.kmax;
  a.early = (flags & TERN_GEMV_STATIC_WEIGHTS) ? 1 : 0;
  a.local = plan.local ? 1 : 0;
  a.status = status;
  a.wait_ns = wait_ns ? wait_ns : kRegWaitLimitNs;
  a.ws = plan.ws_bytes ? static_cast<float*>(workspace) : nullptr;
  a.counters = plan.ws_bytes ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + plan.ws_partial_bytes) : nullptr;
  if (plan.reg && W.layout == TERN_Q1_0_G128) {
    // the binary kernel's MMA columns hold two batch rows: one launch per pair, in order on the stream
    // (the split-K partials and counters of one launch are consumed before the next starts)
    for (int b0 = 0; b0 < batch; b0 += kBinChunk) {
      a.batch = std::min(kBinChunk, batch - b0);
      a.x = x + (int64_t)b0 * W.k;
      a.y = y + (int64_t)b0 * W.n;
      const cudaError_t e = dispatch_reg(W, a, plan.grid_x, plan.warps, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (plan.reg) return dispatch_reg(W, a, plan.grid_x, plan.warps, st);
  const int gx_hint = (plan.row_blocks + kWarps - 1) / kWarps;
  if (W.layout == TERN_Q2_0_G128) return dispatch<TERN_Q2_0_G128>(a, gx_hint, st);
  return dispatch<TERN_T3_5PB_G128>(a, gx_hint, st);
}

// ---- allocation-free variant ---------------------------------------------------------------------
// Split-K scratch in a file-scope device array, for callers that cannot hand the library device
// memory. Every GPU that loads the library holds these bytes until the process exits.
static __device__ __align__(256) unsigned char tern_noalloc_scratch[TERN_GEMV_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of tern_noalloc_scratch on the current device, looked up once per device. In
// host code the array's name is only a host-side stand-in, so it must never be passed to a kernel.
cudaError_t noalloc_scratch(void** out) {
  static std::mutex mu;
  static std::vector<void*> addr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= (int)addr.size()) addr.resize(dev + 1, nullptr);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, tern_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

tern_status gemv_noalloc(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, cudaStream_t st) {
  const GemvPlan plan = gemv_plan(W.layout, W.n, W.k, batch, sm_count());
  if (plan.ws_bytes > (size_t)TERN_GEMV_NOALLOC_SCRATCH_BYTES) return TERN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (plan.ws_bytes) {
    if (noalloc_scratch(&scratch) != cudaSuccess) return TERN_ERR_CUDA;
    // the arrival counters must start at zero; the array keeps whatever the previous call left
    const size_t counters = plan.ws_bytes - plan.ws_partial_bytes;
    if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + plan.ws_partial_bytes, 0, counters, st) != cudaSuccess)
      return TERN_ERR_CUDA;
  }
  return launch_gemv(W, x, batch, y, scratch, plan, st) == cudaSuccess ? TERN_OK : TERN_ERR_CUDA;
}

}  // namespace tern
