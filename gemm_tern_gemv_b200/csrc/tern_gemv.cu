// Decode GEMV y = W x for packed ternary W (batch 1..64) on mma.sync tensor cores.
//
// What is computed ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "그룹 단위 스케일을
// 공유하는 삼진 형식", eq. w_i = s_g t_i; section "하이브리드 어텐션을 위한 저비트 커널": the
// product reads packed codes and fuses unpack + group scale):
//     y[b][n] = sum_g s[n][g] * sum_{k in g} t[n][k] * x[b][k]
//
// How (B200, sm_100a). Batch-1 decode at HBM rate leaves about 0.7 ALU-pipe instructions per
// weight (LOP3/SHF/PRMT issue at half rate on this SM, on a different pipe than IMAD), so:
//   * A Q2_0_g128 code is t as a 2-bit two's-complement field. Shifted to bits 14..15 of an fp16
//     half, the field IS the half's sign bit and exponent MSB: 0b01 -> +2.0, 0b11 -> -2.0,
//     0b00 -> 0. So A = (word << (14 - 2i)) & 0xC000C000 is the tensor-core A fragment
//     (2 t_i, 2 t_{i+8}) exactly: one IMAD (the shift, FMA pipe) and one LOP3 per two weights.
//   * B is the fp16 activation itself (no rescaling), the MMA accumulates D = 2 sum t x in fp32,
//     and the epilogue applies s/2 per group: no offset, no cancellation, exact products.
//   * The 8 MMA columns carry (batch, group-of-window) pairs: a window is two consecutive 128-
//     weight groups of a row (64 bytes), each lane loads 16 contiguous bytes of it, and the two
//     groups' partial sums land in different columns, so each gets its own scale in the fp32
//     epilogue. Up to 4 batch rows share one m16n8k16 tile; larger batches use more n-tiles.
//   * The base-3 layout is first expanded, per warp, into the same 2-bit fields in shared memory
//     through a 256-entry table, then runs the same MMA loop.
//   * Narrow matrices split K across CTAs; the last CTA of a row block sums the fp32 partials in
//     slice order (deterministic) and stores fp16 y. The arrival counters reset themselves.
#include <cuda_fp16.h>

#include <algorithm>

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kQ2RowStride = 192;   // bytes per row of the per-warp expanded base-3 buffer (160 used)
constexpr int kT3Window = 5;        // base-3 windows: 5 groups = 640 trits = 128 bytes per row

struct Args {
  const uint8_t* codes;
  int64_t cstride;
  const uint16_t* scales;
  int64_t sstride;
  const uint16_t* x;
  uint16_t* y;
  float* ws;        // [splits][batch][n] fp32 partials
  int* counters;    // [row_blocks]
  int n, k, batch, groups, gps, splits;
  uint32_t unit;    // always 1 (see `mul` in the kernel)
};

__device__ __forceinline__ void mma_f16(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// A fragment of slot S (0..7) of a 16-code word: codes (S, S+8) as the fp16 pair (2 t_S, 2 t_S+8).
// `mul` is 2^(14 - 2S) held in a register, so the shift issues as an IMAD on the FMA pipe.
__device__ __forceinline__ uint32_t slot(uint32_t w, uint32_t mul) { return (w * mul) & 0xC000C000u; }

// Number of dynamic shared-memory bytes the kernel needs.
__host__ __device__ inline size_t smem_bytes(int layout, int nt, int rt, int gps) {
  const int wins = (gps + 1) / 2 + (layout == TERN_T3_5PB_G128 ? gps / kT3Window + 1 : 0);
  size_t frag = (size_t)wins * 16 * nt * 16 * 8;  // uint2 per (window, mma, n-tile, b', q)
  size_t extra = 0;
  if (layout == TERN_T3_5PB_G128) extra = 256 * 4 + (size_t)kWarps * 16 * rt * kQ2RowStride;
  return frag + extra;
}

// ---- prologue: activations into B-fragment order ----------------------------------------------
// frag layout (uint2): [window][j 0..15][n-tile][b' 0..3][q 0..3]; halves (b0.lo, b0.hi, b1.lo, b1.hi).
// In window w, lane q owns bytes [16q, 16q + 16) of the 64 code bytes: codes o = 64q + 16*word + i
// (i = code in word), i.e. group g' = q / 2. Word `word` feeds MMAs j = 4*word .. 4*word + 3; MMA j
// uses slots s0 = 2*(j % 4) (-> b0) and s0 + 1 (-> b1); slot s holds codes (s, s + 8) (lo, hi).
template <int NT>
__device__ void build_fragments(const Args& a, int g0, int ngroups, uint2* frag) {
  // work item = 8 consecutive codes (one 16-byte vector of x) of one (group, batch row)
  uint16_t* fh = reinterpret_cast<uint16_t*>(frag);
  const int items = ngroups * a.batch * 16;
  for (int e = threadIdx.x; e < items; e += kThreads) {
    const int v = e & 15;
    const int gb = e >> 4;
    const int bb = gb % a.batch, gl = gb / a.batch;
    const uint4 xv = *reinterpret_cast<const uint4*>(a.x + (int64_t)bb * a.k + (int64_t)(g0 + gl) * kGroup + 8 * v);
    const int win = gl >> 1, gp = gl & 1;
    const int jt = bb >> 2, bp = bb & 3;
    const int o = 128 * gp + 8 * v;       // first code of the vector within the window
    const int q = o >> 6, word = (o & 63) >> 4, h = v & 1;
    uint16_t* base = fh + (((size_t)win * 16 + 4 * word) * NT + jt) * 64 + (bp * 4 + q) * 4 + h;
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int el = 0; el < 8; el++) {      // code i = 8h + el: slot el, MMA j = 4*word + el/2
      const uint16_t val = (uint16_t)(xw[el >> 1] >> (16 * (el & 1)));
      base[(size_t)(el >> 1) * NT * 64 + (el & 1) * 2] = val;
    }
  }
}

// Expand one base-3 window (5 groups) of `rows` rows into 2-bit fields (16 codes per 32-bit word,
// code k at bits 2*(k%16)) in the warp's buffer: row r at buf + r*kQ2RowStride, 160 bytes.
__device__ __forceinline__ void expand_t3_window(const Args& a, int row0, int rows, int win5, int lane,
                                                 const uint32_t* lut, uint8_t* buf) {
  // 8 chunks of 16 bytes per row; lane -> (row, chunk)
  const int t3_row_bytes = (int)((a.k + 4) / 5);
  for (int u = lane; u < rows * 8; u += 32) {
    const int r = u / 8, ch = u % 8;
    const int row = row0 + r;
    const int byte0 = win5 * 128 + ch * 16;
    uint4 q = make_uint4(0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u);  // 121: five t = 0 trits
    if (row < a.n && byte0 < t3_row_bytes) q = __ldg(reinterpret_cast<const uint4*>(a.codes + (int64_t)row * a.cstride + byte0));
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
    uint32_t out[5] = {0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const uint32_t byte = (qw[j / 4] >> (8 * (j % 4))) & 0xFFu;
      const uint32_t f = lut[byte];  // 10-bit: five 2-bit fields
      const int off = 10 * j;
      out[off / 32] |= f << (off % 32);
      if ((off % 32) > 22) out[off / 32 + 1] |= f >> (32 - off % 32);
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(buf + r * kQ2RowStride + ch * 20);
#pragma unroll
    for (int w = 0; w < 5; w++) dst[w] = out[w];
  }
}

// Codes and scales of one pair-window for the lane's rows: rows row_base + 16*rt + g (+8).
template <int RT>
struct PairCodesT {
  uint4 cw[RT][2];
  uint32_t sc[RT][2];  // two fp16 scales (group g' = 0 in the low half, g' = 1 in the high half)
};

template <int RT>
__device__ __forceinline__ void load_scales(const Args& a, int row_base, int grp, int gh, int g, PairCodesT<RT>& p) {
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int hr = 0; hr < 2; hr++) {
      const int row = row_base + rt * 16 + g + 8 * hr;
      uint32_t s2 = 0;
      if (row < a.n) {
        const uint16_t* sp = a.scales + (int64_t)row * a.sstride + grp;
        s2 = (uint32_t)__ldg(sp) | ((gh > 1) ? ((uint32_t)__ldg(sp + 1) << 16) : 0u);
      }
      p.sc[rt][hr] = s2;
    }
}

// Q2_0_g128: the pair-window of groups (g0 + gl0, g0 + gl0 + 1) is 64 contiguous bytes of a row.
template <int RT>
__device__ __forceinline__ void load_pair_q2(const Args& a, int row_base, int g0, int gl0, int gh, int g, int q,
                                             PairCodesT<RT>& p) {
  const bool mine = (q >> 1) < gh;
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int hr = 0; hr < 2; hr++) {
      const int row = row_base + rt * 16 + g + 8 * hr;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);  // t = 0
      if (row < a.n && mine)
        v = __ldg(reinterpret_cast<const uint4*>(a.codes + (int64_t)row * a.cstride + (int64_t)(g0 + gl0) * 32 + 16 * q));
      p.cw[rt][hr] = v;
    }
  load_scales<RT>(a, row_base, g0 + gl0, gh, g, p);
}

// base-3: the pair-window comes from the warp's expanded 2-bit buffer (groups lw0, lw0 + 1 of the
// 5-group window at byte offset 32 * lw0 of each 160-byte row).
template <int RT>
__device__ __forceinline__ void load_pair_t3(const Args& a, int row_base, int g0, int gl0, int gh, int g, int q,
                                             const uint8_t* t3buf, int lw0, PairCodesT<RT>& p) {
  const bool mine = (q >> 1) < gh;
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int hr = 0; hr < 2; hr++) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);  // t = 0
      if (mine) v = *reinterpret_cast<const uint4*>(t3buf + (rt * 16 + g + 8 * hr) * kQ2RowStride + lw0 * 32 + 16 * q);
      p.cw[rt][hr] = v;
    }
  load_scales<RT>(a, row_base, g0 + gl0, gh, g, p);
}

// 16 MMAs over one pair-window, then the fp32 epilogue that applies the two groups' scales.
template <int NT, int RT>
__device__ __forceinline__ void mma_pair(const PairCodesT<RT>& p, const uint2* frag, const uint32_t (&mul)[8], int pw,
                                         int gh, int g, int q, const bool (&bload)[NT], float (&acc)[RT][NT][2]) {
  float d[RT][NT][4];
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int jt = 0; jt < NT; jt++) d[rt][jt][0] = d[rt][jt][1] = d[rt][jt][2] = d[rt][jt][3] = 0.f;
  const uint2* fr = frag + (size_t)pw * 16 * NT * 16 + (g >> 1) * 4 + q;
#pragma unroll
  for (int word = 0; word < 4; word++) {
    uint32_t wl[RT], wh[RT];
#pragma unroll
    for (int rt = 0; rt < RT; rt++) {
      const uint4& lo = p.cw[rt][0];
      const uint4& hi = p.cw[rt][1];
      wl[rt] = word == 0 ? lo.x : word == 1 ? lo.y : word == 2 ? lo.z : lo.w;
      wh[rt] = word == 0 ? hi.x : word == 1 ? hi.y : word == 2 ? hi.z : hi.w;
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
        uint2 b = make_uint2(0u, 0u);
        if (bload[jt]) b = fr[((size_t)j * NT + jt) * 16];
#pragma unroll
        for (int rt = 0; rt < RT; rt++) mma_f16(d[rt][jt], a0[rt], a1[rt], a2[rt], a3[rt], b.x, b.y);
      }
    }
  }
  // lane (g, q) holds columns 2q, 2q+1 = (b' = q, g' = 0 / 1) of rows g and g + 8; D = 2 sum t x
#pragma unroll
  for (int rt = 0; rt < RT; rt++)
#pragma unroll
    for (int hr = 0; hr < 2; hr++) {
      const float s_a = 0.5f * __half2float(__ushort_as_half((uint16_t)(p.sc[rt][hr] & 0xFFFFu)));
      const float s_b = 0.5f * __half2float(__ushort_as_half((uint16_t)(p.sc[rt][hr] >> 16)));
#pragma unroll
      for (int jt = 0; jt < NT; jt++) {
        float v = fmaf(s_a, d[rt][jt][2 * hr], acc[rt][jt][hr]);
        if (gh > 1) v = fmaf(s_b, d[rt][jt][2 * hr + 1], v);
        acc[rt][jt][hr] = v;
      }
    }
}

template <int LAYOUT, int NT, int RT>
__global__ void __launch_bounds__(kThreads) gemv_kernel(Args a) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int last;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane / 4, q = lane % 4;
  constexpr int ROWS = kWarps * 16 * RT;
  const int split = blockIdx.y;
  const int g0 = split * a.gps;
  const int ngroups = min(a.gps, a.groups - g0);
  const int row_blocks = (a.n + ROWS - 1) / ROWS;
  // shared-memory carve-up must match smem_bytes(), which the host computes from a.gps
  const int wins = (a.gps + 1) / 2 + (LAYOUT == TERN_T3_5PB_G128 ? a.gps / kT3Window + 1 : 0);

  uint2* frag = reinterpret_cast<uint2*>(smem);
  uint8_t* extra = smem + (size_t)wins * 16 * NT * 16 * 8;
  uint32_t* lut = reinterpret_cast<uint32_t*>(extra);
  uint8_t* t3buf = extra + 256 * 4 + (size_t)warp * 16 * RT * kQ2RowStride;

  // ---- once per CTA: the activation fragments of this K slice (and the base-3 table) ----
  if (LAYOUT == TERN_T3_5PB_G128) {
    for (int v = threadIdx.x; v < 256; v += kThreads) {
      uint32_t f = 0, r = v < 243 ? v : 121;  // an invalid byte decodes as five t = 0 trits
#pragma unroll
      for (int i = 0; i < 5; i++) { f |= (((r % 3u) + 3u) & 3u) << (2 * i); r /= 3u; }  // c-1 as 2-bit two's complement
      lut[v] = f;
    }
    // groups of 5-window w5 go to pair-windows 3*w5 + (0,0,1,1,2)
    for (int w5 = 0; w5 * kT3Window < ngroups; w5++) {
      const int gn = min(kT3Window, ngroups - w5 * kT3Window);
      build_fragments<NT>(a, g0 + w5 * kT3Window, gn, frag + (size_t)w5 * 3 * 16 * NT * 16);
    }
  } else {
    build_fragments<NT>(a, g0, ngroups, frag);
  }
  __syncthreads();

  // shift multipliers 2^(14 - 2S), built from a runtime 1 so they stay IMAD operands
  uint32_t mul[8];
#pragma unroll
  for (int S = 0; S < 8; S++) mul[S] = a.unit << (14 - 2 * S);
  // B column of this lane: (b' = g/2, g' = g&1); it carries data when g' is the lane's group
  const bool bcol = ((g & 1) == (q >> 1));
  bool bload[NT];
#pragma unroll
  for (int jt = 0; jt < NT; jt++) bload[jt] = bcol && (4 * jt + (g >> 1) < a.batch);

  for (int rb = blockIdx.x; rb < row_blocks; rb += gridDim.x) {
    const int row_base = rb * ROWS + warp * 16 * RT;
    float acc[RT][NT][2];
#pragma unroll
    for (int rt = 0; rt < RT; rt++)
#pragma unroll
      for (int jt = 0; jt < NT; jt++) acc[rt][jt][0] = acc[rt][jt][1] = 0.f;

    PairCodesT<RT> cur;
    if (LAYOUT == TERN_Q2_0_G128) {
      const int npair = (ngroups + 1) / 2;
      load_pair_q2<RT>(a, row_base, g0, 0, min(2, ngroups), g, q, cur);
      for (int pw = 0; pw < npair; pw++) {
        const int gh = min(2, ngroups - 2 * pw);
        PairCodesT<RT> nxt;
        if (pw + 1 < npair) load_pair_q2<RT>(a, row_base, g0, 2 * (pw + 1), min(2, ngroups - 2 * (pw + 1)), g, q, nxt);
        mma_pair<NT, RT>(cur, frag, mul, pw, gh, g, q, bload, acc);
        if (pw + 1 < npair) cur = nxt;
      }
    } else {
      const int n5 = (ngroups + kT3Window - 1) / kT3Window;
      for (int ow = 0; ow < n5; ow++) {
        const int gn = min(kT3Window, ngroups - ow * kT3Window);
        __syncwarp();
        expand_t3_window(a, row_base, 16 * RT, (g0 + ow * kT3Window) / kT3Window, lane, lut, t3buf);
        __syncwarp();
        for (int iw = 0; iw < (gn + 1) / 2; iw++) {
          const int gh = min(2, gn - 2 * iw);
          load_pair_t3<RT>(a, row_base, g0, ow * kT3Window + 2 * iw, gh, g, q, t3buf, 2 * iw, cur);
          mma_pair<NT, RT>(cur, frag, mul, 3 * ow + iw, gh, g, q, bload, acc);
        }
      }
    }

    // ---- output: lane (g, q) owns y[4*jt + q][row_base + rt*16 + g + 8*hr] ----
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
              a.y[(int64_t)b * a.n + row] = __half_as_ushort(__float2half_rn(acc[rt][jt][hr]));
          }
      continue;
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
          if (row < a.n && b < a.batch) part[(size_t)b * a.n + row] = acc[rt][jt][hr];
        }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int prev = atomicAdd(a.counters + rb, 1);
      last = (prev == a.splits - 1);
      if (last) a.counters[rb] = 0;  // ready for the next call
    }
    __syncthreads();
    if (last) {
      __threadfence();
      const int r0 = rb * ROWS;
      const int nrows = min(ROWS, a.n - r0);
      for (int e = threadIdx.x; e < nrows * a.batch; e += kThreads) {
        const int b = e / nrows, row = r0 + e % nrows;
        float v = 0.f;
        for (int sp = 0; sp < a.splits; sp++) v += __ldcg(a.ws + ((size_t)sp * a.batch + b) * a.n + row);
        a.y[(int64_t)b * a.n + row] = __half_as_ushort(__float2half_rn(v));
      }
    }
    __syncthreads();
  }
}

template <int LAYOUT, int NT, int RT>
cudaError_t launch_t(const Args& a, int row_blocks, cudaStream_t st) {
  const size_t smem = smem_bytes(LAYOUT, NT, RT, a.gps);
  auto kern = gemv_kernel<LAYOUT, NT, RT>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  // persistent CTAs: one full wave, each walking row blocks of its K slice
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int wave = sm_count() * per_sm;
  int gx = (wave + a.splits - 1) / a.splits;
  if (gx > row_blocks) gx = row_blocks;
  if (gx < 1) gx = 1;
  dim3 grid(gx, a.splits);
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int LAYOUT>
cudaError_t dispatch_nt(const Args& a, int nt, int row_blocks, cudaStream_t st) {
  switch (nt) {
    case 1: return launch_t<LAYOUT, 1, 2>(a, row_blocks, st);
    case 2: return launch_t<LAYOUT, 2, 1>(a, row_blocks, st);
    case 3: case 4: return launch_t<LAYOUT, 4, 1>(a, row_blocks, st);
    case 5: case 6: case 7: case 8: return launch_t<LAYOUT, 8, 1>(a, row_blocks, st);
    default: return launch_t<LAYOUT, 16, 1>(a, row_blocks, st);
  }
}

int nt_for(int64_t batch) {
  const int nt = (int)((batch + 3) / 4);
  return nt <= 2 ? nt : nt <= 4 ? 4 : nt <= 8 ? 8 : 16;
}

}  // namespace

GemvPlan gemv_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  GemvPlan p{};
  const int nt = nt_for(batch);
  const int rt = nt == 1 ? 2 : 1;
  p.rows_per_cta = kWarps * 16 * rt;
  p.row_blocks = (int)((n + p.rows_per_cta - 1) / p.rows_per_cta);
  const int groups = (int)(k / kGroup);
  const int unit = (layout == TERN_T3_5PB_G128) ? kT3Window : 2;  // slice granularity in groups
  const int units = (groups + unit - 1) / unit;
  // Aim for about 4 CTAs per SM; cap the shared-memory footprint of the activation fragments.
  const int target = 4 * sms;
  int splits = (int)std::min<int64_t>(units, std::max<int64_t>(1, (target + p.row_blocks - 1) / p.row_blocks));
  int upc = (units + splits - 1) / splits;  // units per CTA
  const size_t smem_cap = 160 * 1024;
  while (upc > 1 && smem_bytes(layout, nt, rt, upc * unit) > smem_cap) upc = (upc + 1) / 2;
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
  a.unit = 1u;
  a.ws = plan.splits > 1 ? static_cast<float*>(workspace) : nullptr;
  a.counters = plan.splits > 1 ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + plan.ws_partial_bytes) : nullptr;
  const int nt = nt_for(batch);
  if (W.layout == TERN_Q2_0_G128) return dispatch_nt<TERN_Q2_0_G128>(a, nt, plan.row_blocks, st);
  return dispatch_nt<TERN_T3_5PB_G128>(a, nt, plan.row_blocks, st);
}

}  // namespace tern
