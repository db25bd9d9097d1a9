// Decode GEMV y = W x for packed ternary W (batch 1..64) on mma.sync tensor cores.
//
// What is computed ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "그룹 단위 스케일을
// 공유하는 삼진 형식", eq. w_i = s_g t_i; section "하이브리드 어텐션을 위한 저비트 커널": the
// product reads packed codes and fuses unpack + group scale):
//     y[b][n] = sum_g s[n][g] * sum_{k in g} t[n][k] * x[b][k]
//
// How (B200, sm_100a). Batch-1 decode at HBM rate leaves about 0.7 ALU-pipe instructions per
// weight (LOP3/SHF/PRMT issue at half rate on this SM, on a different pipe than IMAD), and the
// weights are streamed once, so the kernel is built around two things:
//   * Decode = one IMAD + one LOP3 per two weights. A Q2_0_g128 code is t as a 2-bit two's-
//     complement field; shifted to bits 14..15 of an fp16 half, the field IS the half's sign bit
//     and exponent MSB: 0b01 -> +2.0, 0b11 -> -2.0, 0b00 -> 0. So (word << (14 - 2i)) & 0xC000C000
//     is the tensor-core A fragment (2 t_i, 2 t_{i+8}) exactly. B is the fp16 activation itself;
//     the MMA accumulates D = 2 sum t x in fp32 and the epilogue applies s/2 per group: no offset,
//     no cancellation, exact products.
//   * Memory-level parallelism: every warp owns a ring of cp.async stages (16-byte copies straight
//     to shared memory, no registers) several windows deep and streams its row tiles through it
//     continuously, so each SM keeps ~100 KB of codes in flight.
// Layout of the work:
//   * The 8 MMA columns carry (batch, group-of-window) pairs: a window is two consecutive 128-
//     weight groups of a row (64 bytes); each lane owns 16 contiguous bytes of it, and the two
//     groups' partial sums land in different columns, so each gets its own scale in the fp32
//     epilogue. Up to 4 batch rows share one m16n8k16 tile; larger batches use more n-tiles.
//   * Activations are written once per CTA into shared memory in B-fragment order.
//   * Warps walk 32-row tiles of their CTA's K slice. Narrow matrices split K across CTAs; the last
//     warp to finish a tile (atomic counter) sums the fp32 partials in slice order (deterministic),
//     stores fp16 y and resets the counter.
//   * The base-3 layout streams 5-group windows (128 bytes per row) through the ring and expands
//     them per warp into the same 2-bit fields through a 256-entry table before the same MMA loop.
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "sm100.cuh"
#include "tern_internal.cuh"

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
  uint32_t unit;    // always 1 (see `mul` in the kernel)
};

// ---- small device helpers --------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0)
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
  switch (bs_for(a.batch)) {
    case 1: return launch_t<LAYOUT, 1, 2, 1>(a, gx_hint, st);
    case 2: return launch_t<LAYOUT, 1, 2, 2>(a, gx_hint, st);
    case 4: return launch_t<LAYOUT, 1, 2, 4>(a, gx_hint, st);
    case 8: return launch_t<LAYOUT, 2, 1, 8>(a, gx_hint, st);
    case 16: return launch_t<LAYOUT, 4, 1, 16>(a, gx_hint, st);
    case 32: return launch_t<LAYOUT, 8, 1, 32>(a, gx_hint, st);
    default: return launch_t<LAYOUT, 16, 1, 64>(a, gx_hint, st);
  }
}

}  // namespace

GemvPlan gemv_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
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
                        const GemvPlan& plan, cudaStream_t st) {
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
  a.ws = plan.splits > 1 ? static_cast<float*>(workspace) : nullptr;
  a.counters = plan.splits > 1 ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + plan.ws_partial_bytes) : nullptr;
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
