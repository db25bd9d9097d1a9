// Decode GEMV y = W x for batch 1-2 on int8 mma.sync tensor cores, weights streamed by TMA.
//
// What is computed ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "그룹 단위 스케일을
// 공유하는 삼진 형식", eq. w_i = s_g t_i; section "하이브리드 어텐션을 위한 저비트 커널": the product
// reads the packed codes and fuses unpack and group scale):
//     y[b][n] = sum_g s[n][g] * sum_{k in g} t[n][k] * x[b][k]
//
// How (B200, sm_100a). At batch 1 every weight is used once, so the kernel has to turn codes into
// tensor-core operands at HBM speed; LOP3 / SHF / PRMT issue at half rate, which makes the number of
// integer operations per weight the budget. int8 operands need half as many as fp16 ones:
//   * Activations become exact int8 planes. Per batch row, X = round(x * 2^S) with S chosen from
//     max|x| so that |X| < 2^28 (S <= 24 keeps every fp16 value exact); X is written as four balanced
//     base-256 digits d_p in [-128, 127], X = sum_p d_p 2^(8p). The MMA's 8 columns are
//     (group slot 0/1) x (plane 0..3); the epilogue recombines planes in int32 / fp32 and applies the
//     group scale in fp32.
//   * Q2_0_g128: (word << (6 - 2j)) & 0xC0C0C0C0 puts field j of each byte at bits 6..7, i.e. the
//     int8 value 64 t: one IMAD + one LOP3 per four weights (the shift is an IMAD on the FMA pipe).
//   * Q1_0_g128: (word << (7 - j)) & 0x80808080 is the u8 value 128 b (t = 2b - 1); the -sum x of each
//     group is added in the epilogue.
//   * base-3: byte v holds digits c_j = floor(v / 3^j) mod 3. The A operands are the quotients
//     q_j = floor(v / 3^j) (u8; q_0 = v is the byte itself) and a constant 1; since
//     c_j = q_j - 3 q_{j+1}, sum_j (c_j - 1) x_j = sum_j q_j (x_j - 3 x_{j-1}) - sum_j x_j, so the
//     B operand carries the transformed activations and the quotients need no digit extraction.
//     q_{j+1} = (85 q_j + 80) >> 8 for every q_j <= 242: one IMAD per two bytes (16-bit lanes) and
//     one PRMT to bring the quotient back to the low byte. A unit is 32 bytes (160 trits) of a row:
//     aligned at 160 c, it starts at most 96 trits into a group, so it never touches more than two.
//   * Weight tiles (16 rows x one K slice) are streamed into a shared-memory ring by one producer
//     thread with 2-D TMA boxes up to 1 KB wide (wide rows keep DRAM pages open); the consumer warps
//     of the CTA split the slice along K, so each tile is read as whole row segments.
//   * Narrow matrices split K over a thread-block cluster of 2 or 4 CTAs; the partial sums are
//     added through distributed shared memory in a fixed order (no workspace, deterministic).
//   * Every pipeline wait is bounded; a wait that runs out makes the CTA give up, write NaN to the
//     outputs it owns and OR TERN_DEVICE_TIMEOUT into the caller's status word.
#include <cuda_fp16.h>

#include <algorithm>

#include "sm100.cuh"
#include "tern_fwht.cuh"
#include "tern_internal.cuh"

namespace tern {
namespace {

using sm100::smem_u32;

// CTA shapes: one CTA of up to 17 consumer warps per SM, or two CTAs of up to 8 (each with its own
// producer warp, ring and activation fragments). Two per SM overlap one CTA's prologue and drain with
// the other's streaming, which pays on matrices with many tiles per SM; one per SM has the deeper ring.
constexpr int kI8MaxNW1 = 17, kI8MaxNW2 = 8;
__host__ __device__ constexpr int i8_max_nw(int cps) { return cps == 2 ? kI8MaxNW2 : kI8MaxNW1; }
constexpr uint64_t kI8DefaultWaitNs = 1000000000ull;
constexpr uint64_t kI8DrainNs = 200000000ull;  // bound on waiting for copies in flight at exit
constexpr int kXV = 4;  // vectors of 8 activations a thread converts per row of x (slice <= 32 x threads)

template <int L> struct I8L;
// units: 16 rows x kUnitB bytes of codes; a thread holds kUnitB / 4 bytes of rows g and g + 8
template <> struct I8L<TERN_Q2_0_G128> { static constexpr int kUnitK = 256, kUnitB = 64, kWords = 4, kMP = 4, kEnt = 16; };
template <> struct I8L<TERN_Q1_0_G128> { static constexpr int kUnitK = 256, kUnitB = 32, kWords = 2, kMP = 4, kEnt = 16; };
template <> struct I8L<TERN_T3_5PB_G128> { static constexpr int kUnitK = 160, kUnitB = 32, kWords = 2, kMP = 3, kEnt = 32; };

struct I8Params {
  const uint16_t* x;  // [batch][k]
  uint16_t* y;        // [batch][n]
  uint32_t* status;   // optional device status word
  uint64_t wait_ns;   // bound on each pipeline wait
  int n, k, batch, groups;
  int tiles;          // ceil(n / 16)
  int units;          // units per row
  int L;              // units per K slice (the last slice may be shorter)
  int nw;             // consumer warps
  uint32_t nw_rcp;    // floor(2^20 / nw) + 1: x / nw = (x * nw_rcp) >> 20 for 0 <= x < 2^20 / nw
  int early;          // weight tiles may be requested before the preceding grid completes
  int box_b, nfull, rem_b;  // code boxes of one stage: nfull x box_b bytes, then rem_b bytes (0 = none)
  int sc_w;           // scale box width (halves, multiple of 8)
  int stage_bytes, code_bytes, stages;
  int tmax;           // largest number of tiles a cluster owns
  int xk;             // activations held per CTA (halves, multiple of 8)
  const int8_t* signs;  // non-null: multiply by R x (block Hadamard rotation of x, done in the prologue)
  int rot_off;        // rotated x: byte offset within the partial-sum space (past X and the FWHT scratch)
  int rot_bytes;      // bytes of that space the rotation needs
};

// ---- small device helpers --------------------------------------------------------------------------
__device__ __forceinline__ void imma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void imma_u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The same products with a zero accumulator (the first IMMA of a chain: no register has to be cleared).
__device__ __forceinline__ void imma_s8_z(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}
__device__ __forceinline__ void imma_u8_z(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint16_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
// 16 bytes into v when pred is set; otherwise v keeps its (zero) value.
__device__ __forceinline__ void lds128_if(uint4& v, uint32_t a, bool pred) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t@p ld.shared.v4.u32 {%0,%1,%2,%3}, [%5];\n\t}"
               : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
               : "r"((uint32_t)pred), "r"(a));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `bar` with this parity. Gives up when *abort is raised by another thread or
// after limit_ns of wall time, raising *abort itself and OR-ing TERN_DEVICE_TIMEOUT into *status.
// Limits under a millisecond poll without suspending (try_wait may itself sleep for longer than that).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t* status,
                                          uint64_t limit_ns) {
  const bool poll = limit_ns < 1000000ull;
  if (poll ? mbar_test(bar, parity) : mbar_try(bar, parity)) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (poll ? mbar_test(bar, parity) : mbar_try(bar, parity)) return true;
    if (poll || (it & 15u) == 0) {
      if (*abort) return false;
      if (sm100::globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        if (status) atomicOr(status, TERN_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// Balanced base-256 digits of X (|X| < 2^31): byte p of the result is d_p as an int8.
__device__ __forceinline__ uint32_t digits(int X) { return ((uint32_t)X + 0x00808080u) ^ 0x00808080u; }

// k of the weight in byte i of the A register (m, half) of lane q in unit u (u counted from the row start).
template <int LAYOUT>
__device__ __forceinline__ int a_k(int u, int m, int half, int q, int i) {
  if (LAYOUT == TERN_Q2_0_G128) return 256 * u + 64 * q + 16 * (m >> 1) + 4 * i + 2 * (m & 1) + half;
  if (LAYOUT == TERN_Q1_0_G128) return 256 * u + 64 * q + 32 * (m >> 2) + 8 * i + 2 * (m & 3) + half;
  return 160 * u + 5 * (8 * q + 4 * half + i) + m;  // base-3: trit m of byte i of word `half` (m = 5: constant)
}

// ---- the kernel ---------------------------------------------------------------------------------------
// NPR: 1 = every consumer warp owns exactly one unit of each tile slice (activation fragments kept in
// registers); 0 = any split (fragments read from shared memory per unit).
template <int LAYOUT, int BATCH, int NPR, int CPS>
__global__ void __launch_bounds__((i8_max_nw(CPS) + 1) * 32, CPS)
    gemv_i8_kernel(const __grid_constant__ CUtensorMap mcf, const __grid_constant__ CUtensorMap mcr,
                   const __grid_constant__ CUtensorMap msc, const I8Params p) {
  using T = I8L<LAYOUT>;
  constexpr int kMP = T::kMP, kEnt = T::kEnt;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int NW = p.nw;

  // shared-memory plan (host mirror: i8_smem_bytes)
  const uint32_t ring = smem_u32(smem);
  const uint32_t full0 = ring + (uint32_t)p.stages * (uint32_t)p.stage_bytes;
  const uint32_t empty0 = full0 + 8u * (uint32_t)p.stages;
  int* ctl = reinterpret_cast<int*>(smem + (size_t)p.stages * p.stage_bytes + 16 * p.stages);  // [0] abort, [1..] S_b
  volatile int* abort_flag = ctl;
  uint4* frag = reinterpret_cast<uint4*>(ctl + 8);
  float* red = reinterpret_cast<float*>(frag + (size_t)p.L * kMP * BATCH * kEnt);  // [32][BATCH]; Q1: + corr
  float* corr = red + 32 * BATCH;                                                      // Q1: [L][2][BATCH]
  // the partial sums of the main loop share their space with X, which only the prologue uses
  float* part = corr + (LAYOUT == TERN_Q1_0_G128 ? (p.L * 2 * BATCH + 3) / 4 * 4 : 0);  // [tmax][NW][BATCH][16], 16-B aligned
  int* Xs = reinterpret_cast<int*>(part);  // [BATCH][xk]: X = round(x * 2^S) of the CTA's activations, zero past K

  // work: cluster c owns tiles [t0, t1); CTA rank r of the cluster owns K slice r (units [u0, u1))
  const int KS = (int)cluster_size();
  const int rank = (int)cluster_rank();
  const int ncl = (int)cluster_count(), cid = (int)cluster_id();
  const int t0 = (int)((int64_t)cid * p.tiles / ncl), t1 = (int)((int64_t)(cid + 1) * p.tiles / ncl);
  const int nt = t1 - t0;
  const int u0 = rank * p.L, u1 = min(p.units, u0 + p.L);
  const int kx0 = u0 * T::kUnitK;  // first activation this CTA needs

  if (tid == 0) {
    for (int s = 0; s < p.stages; s++) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, (uint32_t)NW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    ctl[0] = 0;
  }
  __syncthreads();
  sm100::griddep_launch_dependents();

  const bool producer = (warp == NW && lane == 0);
  const int code_x0 = u0 * T::kUnitB / 4;  // first code column of the slice, in 32-bit words
  int sx0;                                 // first scale column of the box (multiple of 8)
  {
    const int g0 = (u0 * T::kUnitK) / kGroup;
    sx0 = g0 & ~7;
  }
  auto issue = [&](int i) {
    const int s = i % p.stages;
    const uint32_t st = ring + (uint32_t)s * (uint32_t)p.stage_bytes;
    const uint32_t fb = full0 + 8u * s;
    mbar_expect_tx(fb, (uint32_t)p.code_bytes + 16u * 2u * (uint32_t)p.sc_w);
    const int row = (t0 + i) * 16;
    for (int b = 0; b < p.nfull; b++)
      tma2d(st + (uint32_t)b * 16u * (uint32_t)p.box_b, &mcf, code_x0 + b * (p.box_b / 4), row, fb);
    if (p.rem_b) tma2d(st + (uint32_t)p.nfull * 16u * (uint32_t)p.box_b, &mcr, code_x0 + p.nfull * (p.box_b / 4), row, fb);
    tma2d(st + (uint32_t)p.code_bytes, &msc, sx0, row, fb);
  };
  int issued = 0;
  const int first = min(p.stages, nt);
  if (producer) {
    sm100::prefetch_tmap(&mcf);
    if (p.rem_b) sm100::prefetch_tmap(&mcr);
    sm100::prefetch_tmap(&msc);
    if (!p.early) sm100::griddep_wait();
    for (; issued < first; issued++) issue(issued);
  }
  sm100::griddep_wait();  // x, y and the outputs of earlier work are touched only from here on

  // ---- activations: x -> int8 planes in B-fragment order -----------------------------------------
  const int xend = min(p.k, u1 * T::kUnitK);  // activations past K (base-3 padding) read as zero
  // the activations the fragments are built from: x itself, or R x for the 1024-blocks that cover this
  // CTA's slice, rotated here into shared memory by groups of 128 threads (the same transform and fp16
  // rounding as tern_hadamard_rotate, so the product equals W applied to that kernel's output)
  const uint16_t* xsrc = p.x;
  int64_t xsrc_stride = p.k;
  int xsrc_off = 0;
  if (p.signs) {
    const int blk0 = kx0 / kRotBlock, nb = (xend + kRotBlock - 1) / kRotBlock - blk0;
    uint16_t* xr = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(part) + p.rot_off);  // [BATCH][nb * 1024]
    float* fsh = part;  // [groups][1024] floats: the FWHT exchange buffer (X is written only afterwards)
    const int groups = min((int)blockDim.x / kRotThreads, 4), grp = tid / kRotThreads, t = tid % kRotThreads;
    if (grp < groups) {
      for (int it = grp; it < BATCH * nb; it += groups) {
        const int b = it / nb, j = it % nb;
        const uint16_t* src = p.x + (int64_t)b * p.k + (int64_t)(blk0 + j) * kRotBlock;
        float v[8];
#pragma unroll
        for (int r = 0; r < 8; r++) {
          const int i = t + kRotThreads * r;
          const float xv = __half2float(__ushort_as_half(src[i]));
          v[r] = p.signs[i] < 0 ? -xv : xv;
        }
        fwht1024(v, fsh + grp * kRotBlock, t, SyncGroup128{grp + 1});
#pragma unroll
        for (int r = 0; r < 8; r++)
          xr[b * nb * kRotBlock + j * kRotBlock + t + kRotThreads * r] = __half_as_ushort(__float2half_rn(v[r] * 0.03125f));
      }
    }
    __syncthreads();
    xsrc = xr;
    xsrc_stride = (int64_t)nb * kRotBlock;
    xsrc_off = blk0 * kRotBlock;
  }
  // pass 1: each thread loads up to kXV vectors of 8 activations per row of x, the CTA takes max|x|,
  // and every activation is converted once to X = round(x * 2^S) (exact for S = 24)
  uint4 xv[BATCH][kXV];
  for (int b = 0; b < BATCH; b++) {
    float mx = 0.f;
#pragma unroll
    for (int j = 0; j < kXV; j++) {
      uint4 v = make_uint4(0, 0, 0, 0);
      const int e = (tid + j * (int)blockDim.x) * 8;
      const int kk = kx0 + e;
      if (e < p.xk) {
        if (kk + 8 <= xend) {
          v = *reinterpret_cast<const uint4*>(xsrc + (int64_t)b * xsrc_stride + (kk - xsrc_off));
        } else if (kk < xend) {
          uint16_t h[8];
          for (int jj = 0; jj < 8; jj++)
            h[jj] = (kk + jj < xend) ? xsrc[(int64_t)b * xsrc_stride + (kk + jj - xsrc_off)] : (uint16_t)0;
          v = make_uint4(h[0] | (uint32_t)h[1] << 16, h[2] | (uint32_t)h[3] << 16, h[4] | (uint32_t)h[5] << 16,
                         h[6] | (uint32_t)h[7] << 16);
        }
      }
      xv[b][j] = v;
      const __half2* hv = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int jj = 0; jj < 4; jj++) {
        const float2 f = __half22float2(hv[jj]);
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));  // NaN inputs are ignored here
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp * BATCH + b] = mx;
  }
  __syncthreads();
  int S[BATCH];
#pragma unroll
  for (int b = 0; b < BATCH; b++) {
    float mx = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) mx = fmaxf(mx, red[w * BATCH + b]);
    // mx < 2^E with E = biased exponent - 126 (mx is a finite fp16 value, so normal in fp32)
    const int E = (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 126;
    // |X| < 2^28 (Q2, binary); base-3 B values sum up to ten activations: |X| < 2^27
    const int top = LAYOUT == TERN_T3_5PB_G128 ? 27 : 28;
    S[b] = (mx > 0.f && mx <= 65504.f) ? min(24, top - E) : 24;
    const float xscale = __uint_as_float((uint32_t)(127 + S[b]) << 23);  // 2^S
#pragma unroll
    for (int j = 0; j < kXV; j++) {
      const int e = (tid + j * (int)blockDim.x) * 8;
      if (e < p.xk) {
        const __half2* hv = reinterpret_cast<const __half2*>(&xv[b][j]);
        int o[8];
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
          const float2 f = __half22float2(hv[jj]);
          o[2 * jj] = __float2int_rn(f.x * xscale);
          o[2 * jj + 1] = __float2int_rn(f.y * xscale);
        }
        int4* d = reinterpret_cast<int4*>(Xs + b * p.xk + e);
        d[0] = make_int4(o[0], o[1], o[2], o[3]);
        d[1] = make_int4(o[4], o[5], o[6], o[7]);
      }
    }
  }
  __syncthreads();
  // four consecutive X of row b starting at activation kk (a multiple of 4)
  auto X4 = [&](int b, int kk) -> int4 { return *reinterpret_cast<const int4*>(Xs + b * p.xk + (kk - kx0)); };
  {
    const int nu = u1 - u0;
    if constexpr (kEnt == 16) {
      // Q2 / Q1: lane q's k values all lie in group 2u + q/2, read by the lanes of that slot
      const int per_unit = kMP * 4;
      for (int it = tid; it < nu * per_unit * BATCH; it += blockDim.x) {
        const int b = it % BATCH;
        const int r0 = it / BATCH;
        const int ul = r0 / per_unit, rem = r0 % per_unit;
        const int u = u0 + ul;
        const int mp = rem >> 2, qq = rem & 3;
        // the lane's 16 activations: k = base + stride i + r (r = 2 (m & 1) + half of IMMA m = 2 mp + (r >> 1))
        const int base = a_k<LAYOUT>(u, 2 * mp, 0, qq, 0), stride = a_k<LAYOUT>(u, 2 * mp, 0, qq, 1) - base;
        uint32_t D[4][4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int4 v = X4(b, base + stride * i);
          D[0][i] = digits(v.x);
          D[1][i] = digits(v.y);
          D[2][i] = digits(v.z);
          D[3][i] = digits(v.w);
        }
        // this code runs once per launch, fetched cold: the plane loop stays rolled to keep it short
#pragma unroll 1
        for (int pl = 0; pl < 4; pl++) {
          const uint32_t sel = (uint32_t)pl | ((uint32_t)(pl + 4) << 4);
          uint32_t w[4];
#pragma unroll
          for (int r = 0; r < 4; r++)
            w[r] = __byte_perm(__byte_perm(D[r][0], D[r][1], sel), __byte_perm(D[r][2], D[r][3], sel), 0x5410);
          frag[(((size_t)ul * kMP + mp) * BATCH + b) * kEnt + qq * 4 + pl] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    } else {
      // base-3: one item per (unit, lane chunk qq, group slot sl): the lane's 40 trits are converted
      // once; feature m of byte i of word h gets x_m - 3 x_{m-1} (trits of slot sl only), and the
      // constant feature (m = 5, word 0) minus the sum of both words' byte-i trits of that slot
      for (int it = tid; it < nu * 8 * BATCH; it += blockDim.x) {
        const int b = it % BATCH;
        const int r0 = it / BATCH;
        const int ul = r0 >> 3, qq = (r0 >> 1) & 3, sl = r0 & 1;
        const int u = u0 + ul;
        const int k0 = 160 * u + 40 * qq;       // first trit of the lane's 8 bytes
        const int g0 = (160 * u) >> 7;          // first group of the unit (kGroup = 128)
        int Xl[40];
#pragma unroll
        for (int e = 0; e < 40; e += 4) {
          const int4 v = X4(b, k0 + e);
          Xl[e] = v.x;
          Xl[e + 1] = v.y;
          Xl[e + 2] = v.z;
          Xl[e + 3] = v.w;
        }
#pragma unroll
        for (int e = 0; e < 40; e++)
          if (((k0 + e) >> 7) - g0 != sl) Xl[e] = 0;
        // V[m][h][i]: m = 0..4 features, m = 5 (h = 0) the constant
        uint32_t D[6][2][4];
#pragma unroll
        for (int h = 0; h < 2; h++)
#pragma unroll
          for (int i = 0; i < 4; i++) {
            const int e0 = 5 * (4 * h + i);
#pragma unroll
            for (int m = 0; m < 5; m++) D[m][h][i] = digits(Xl[e0 + m] - (m ? 3 * Xl[e0 + m - 1] : 0));
          }
#pragma unroll
        for (int i = 0; i < 4; i++) {
          int sum = 0;
#pragma unroll
          for (int j = 0; j < 5; j++) sum += Xl[5 * i + j] + Xl[5 * (4 + i) + j];
          D[5][0][i] = digits(-sum);
          D[5][1][i] = 0;
        }
        // entry (unit, pair mp, lane (g = 4 sl + pl, qq)) word r = IMMA m = 2 mp + (r >> 1), half r & 1
#pragma unroll 1
        for (int pl = 0; pl < 4; pl++) {
          const uint32_t sel = (uint32_t)pl | ((uint32_t)(pl + 4) << 4);
#pragma unroll
          for (int mp = 0; mp < 3; mp++) {
            uint32_t w[4];
#pragma unroll
            for (int r = 0; r < 4; r++) {
              const int m = 2 * mp + (r >> 1), h = r & 1;
              w[r] = __byte_perm(__byte_perm(D[m][h][0], D[m][h][1], sel), __byte_perm(D[m][h][2], D[m][h][3], sel), 0x5410);
            }
            frag[(((size_t)ul * kMP + mp) * BATCH + b) * kEnt + (4 * sl + pl) * 4 + qq] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    if constexpr (LAYOUT == TERN_Q1_0_G128) {
      // -64 sum_{k in g} X_k per (unit, slot, row of x): the t = 2b - 1 offset, added by the plane-0
      // lanes; one warp per group, four activations per lane
      for (int it = warp; it < nu * 2 * BATCH; it += (int)(blockDim.x >> 5)) {
        const int b = it % BATCH, sl = (it / BATCH) & 1, ul = it / (2 * BATCH);
        const int4 v = X4(b, 256 * (u0 + ul) + 128 * sl + 4 * lane);
        long long sx = (long long)v.x + v.y + v.z + v.w;
#pragma unroll
        for (int o = 16; o; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
        if (lane == 0) corr[(ul * 2 + sl) * BATCH + b] = -64.f * (float)sx;
      }
    }
  }
  __syncthreads();
  if (warp == NW) {
    // producer: the rest of the tiles, each into a slot the consumers have released
    if (lane == 0) {
      for (; issued < nt; issued++) {
        const int s = issued % p.stages;
        if (!mbar_wait(empty0 + 8u * s, ((issued / p.stages) - 1) & 1, abort_flag, p.status, p.wait_ns)) break;
        issue(issued);
      }
      // copies still in flight must land before the CTA's shared memory goes away (also after a
      // timeout, so this wait ignores the abort flag; it is bounded on its own)
      const uint64_t t0 = sm100::globaltimer_ns();
      for (int i = max(0, issued - p.stages); i < issued; i++)
        while (!mbar_try(full0 + 8u * (i % p.stages), (i / p.stages) & 1) &&
               sm100::globaltimer_ns() - t0 < kI8DrainNs) {
        }
    }
  } else {
    // ---- consumers ------------------------------------------------------------------------------
    // Chunk c of a stage is local units [c nu / NW, (c + 1) nu / NW). With NPR every warp keeps its
    // own chunk (one unit); otherwise warp w takes chunk (w + i) mod NW in stage i, so a warp with a
    // larger chunk in one stage has a smaller one in the next and no warp runs ahead of the others by
    // more than one chunk (the chunks differ by one unit when NW does not divide nu).
    const int nu = u1 - u0;
    int ck = warp;
    auto chunk_lo = [&](int c) { return (int)(((uint32_t)(c * nu) * p.nw_rcp) >> 20); };
    int ub = chunk_lo(ck), ue = chunk_lo(ck + 1);
    const bool bval = kEnt == 32 || ((g >> 2) == (q >> 1));
    const uint32_t fbase = smem_u32(frag) + (uint32_t)(kEnt == 32 ? lane : (q * 4 + (g & 3))) * 16u;
    uint32_t mul[4];
#pragma unroll
    for (int j = 0; j < 4; j++) mul[j] = LAYOUT == TERN_Q1_0_G128 ? (1u << (7 - 2 * j)) : (1u << (6 - 2 * j));
    uint32_t mul_b[4];  // binary: shifts 7 - (2j + 1)
#pragma unroll
    for (int j = 0; j < 4; j++) mul_b[j] = 1u << (6 - 2 * j);
    // opaque to the compiler, so that shifts stay on the FMA pipe as IMADs
    asm volatile("" : "+r"(mul[0]), "+r"(mul[1]), "+r"(mul[2]), "+r"(mul[3]));
    asm volatile("" : "+r"(mul_b[0]), "+r"(mul_b[1]), "+r"(mul_b[2]), "+r"(mul_b[3]));
    uint32_t k85 = 85u, kc80 = 0x00500050u;
    asm volatile("" : "+r"(k85), "+r"(kc80));
    const float plane_w = (q & 1) ? 65536.f : 1.f;
    float outscale[BATCH];
    for (int b = 0; b < BATCH; b++)  // 2^-S (base-3) or 2^(-S-6) (the A values of Q2 / binary are 64 t / 128 b)
      outscale[b] = plane_w * __uint_as_float((uint32_t)(127 - S[b] - (LAYOUT == TERN_T3_5PB_G128 ? 0 : 6)) << 23);
    // Shared-memory addresses of a local unit within a stage; every tile has the same layout, so
    // they depend on the unit and the lane only: a slice is one box (box_b = slice bytes <= 1 KB) or
    // 1 KB boxes plus a narrower last one.
    const bool box1k = p.box_b == 1024;
    const uint32_t box_stride = 16u * (uint32_t)p.box_b;
    const uint32_t frag_unit = (uint32_t)(kMP * BATCH * kEnt) * 16u;
    const int lane_off = q * (T::kUnitB / 4);
    const uint32_t cR_one = (uint32_t)(g * p.box_b + lane_off);             // one-box slices
    const uint32_t c8_one = 8u * (uint32_t)p.box_b;
    const uint32_t sR_lane = (uint32_t)(p.code_bytes + (g * p.sc_w - sx0) * 2);
    struct UA {
      uint32_t cR, c8, sR, fr;  // codes of row g, row-8 distance, scale of row g, fragments
      bool sval;
    };
    auto unit_addr = [&](int ul) -> UA {
      UA a;
      if (box1k) {
        const int off = ul * T::kUnitB + lane_off;
        const int bo = off >> 10;
        const uint32_t width = (uint32_t)(bo < p.nfull ? p.box_b : p.rem_b);
        a.cR = (uint32_t)bo * box_stride + (uint32_t)g * width + (uint32_t)(off & 1023);
        a.c8 = 8u * width;
      } else {
        a.cR = cR_one + (uint32_t)(ul * T::kUnitB);
        a.c8 = c8_one;
      }
      const int u = u0 + ul;
      int grp;
      a.sval = true;
      if (LAYOUT == TERN_T3_5PB_G128) {
        // a unit starts 0, 32, 64 or 96 trits into group (160 u) / 128 and always reaches the next
        // group; slot 1 carries no data when that group is past K
        const int g0 = (5 * u) >> 2;  // (160 u) / 128
        grp = g0 + (q >> 1);
        a.sval = grp < p.groups;
        if (!a.sval) grp = g0;
      } else {
        grp = 2 * u + (q >> 1);
      }
      a.sR = sR_lane + (uint32_t)grp * 2u;
      a.fr = fbase + (uint32_t)ul * frag_unit;
      return a;
    };
    const uint32_t s8 = 16u * (uint32_t)p.sc_w;  // scale rows g -> g + 8

    // activation fragments of the warp's unit, kept in registers when it owns exactly one
    uint4 breg[NPR ? kMP : 1][NPR ? BATCH : 1];
    float creg[BATCH];
    UA a1 = unit_addr(ub);
    if (NPR) {
#pragma unroll
      for (int mp = 0; mp < kMP; mp++)
#pragma unroll
        for (int b = 0; b < BATCH; b++) {
          breg[mp][b] = make_uint4(0, 0, 0, 0);
          lds128_if(breg[mp][b], a1.fr + (uint32_t)((mp * BATCH + b) * kEnt) * 16u, bval && ub < ue);
        }
    }
#pragma unroll
    for (int b = 0; b < BATCH; b++) {
      creg[b] = 0.f;
      if (LAYOUT == TERN_Q1_0_G128 && NPR && ub < ue && (q & 1) == 0) creg[b] = corr[(ub * 2 + (q >> 1)) * BATCH + b];
    }
    const uint32_t ones = 0x01010101u;
    const uint32_t part_w = smem_u32(part) + (uint32_t)(warp * BATCH * 16 + g) * 4u;  // + tile * NW * BATCH * 64
    const uint32_t part_tile = (uint32_t)(NW * BATCH * 16) * 4u;

    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nt; i++) {
      const uint32_t st = ring + (uint32_t)s * (uint32_t)p.stage_bytes;
      if (!NPR && i > 0) {
        if (++ck == NW) ck = 0;
        ub = ck ? ue : 0;
        ue = chunk_lo(ck + 1);
      }
      // every lane waits (each must observe the copy's completion); the verdict is made warp-uniform,
      // so that a lane whose wait ran out cannot leave the others stuck in the shuffles below
      if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8u * s, ph, abort_flag, p.status, p.wait_ns))) break;
      float acc[BATCH][2];
#pragma unroll
      for (int b = 0; b < BATCH; b++) acc[b][0] = acc[b][1] = 0.f;
      for (int ul = ub; ul < ue; ul++) {
        const UA ua = NPR ? a1 : unit_addr(ul);
        // this lane's codes of rows g and g + 8, and its two group scales
        uint32_t wR[T::kWords], wR8[T::kWords];
        const uint32_t ca = st + ua.cR;
        if constexpr (T::kWords == 4) {
          const uint4 a = lds128(ca), c = lds128(ca + ua.c8);
          wR[0] = a.x; wR[1] = a.y; wR[2] = a.z; wR[3] = a.w;
          wR8[0] = c.x; wR8[1] = c.y; wR8[2] = c.z; wR8[3] = c.w;
        } else if constexpr (T::kWords == 2) {
          const uint2 a = lds64(ca), c = lds64(ca + ua.c8);
          wR[0] = a.x; wR[1] = a.y;
          wR8[0] = c.x; wR8[1] = c.y;
        } else {
          wR[0] = lds32(ca);
          wR8[0] = lds32(ca + ua.c8);
        }
        const uint32_t sa = st + ua.sR;
        float sR = __half2float(__ushort_as_half(lds16(sa)));
        float sR8 = __half2float(__ushort_as_half(lds16(sa + s8)));
        if (LAYOUT == TERN_T3_5PB_G128 && !ua.sval) sR = sR8 = 0.f;
        uint4 bf[kMP][BATCH];
#pragma unroll
        for (int mp = 0; mp < kMP; mp++)
#pragma unroll
          for (int b = 0; b < BATCH; b++) {
            if (NPR) {
              bf[mp][b] = breg[mp][b];
            } else if (kEnt == 32) {
              bf[mp][b] = lds128(ua.fr + (uint32_t)((mp * BATCH + b) * kEnt) * 16u);
            } else {
              bf[mp][b] = make_uint4(0, 0, 0, 0);
              lds128_if(bf[mp][b], ua.fr + (uint32_t)((mp * BATCH + b) * kEnt) * 16u, bval);
            }
          }
        // two independent accumulator chains (even / odd IMMA) halve the dependent MMA latency
        int c[BATCH][4], cx[BATCH][4];
        if constexpr (LAYOUT == TERN_Q2_0_G128) {
#pragma unroll
          for (int m = 0; m < 8; m++) {
            const int w = m >> 1, j0 = 2 * (m & 1);
            const uint32_t a0 = (wR[w] * mul[j0]) & 0xC0C0C0C0u, a1 = (wR8[w] * mul[j0]) & 0xC0C0C0C0u;
            const uint32_t a2 = (wR[w] * mul[j0 + 1]) & 0xC0C0C0C0u, a3 = (wR8[w] * mul[j0 + 1]) & 0xC0C0C0C0u;
#pragma unroll
            for (int b = 0; b < BATCH; b++) {
              const uint4& bb = bf[m >> 1][b];
              if (m == 0) imma_s8_z(c[b], a0, a1, a2, a3, bb.x, bb.y);
              else if (m == 1) imma_s8_z(cx[b], a0, a1, a2, a3, bb.z, bb.w);
              else if (m & 1) imma_s8(cx[b], a0, a1, a2, a3, bb.z, bb.w);
              else imma_s8(c[b], a0, a1, a2, a3, bb.x, bb.y);
            }
          }
        } else if constexpr (LAYOUT == TERN_Q1_0_G128) {
#pragma unroll
          for (int m = 0; m < 8; m++) {
            const int w = m >> 2, jj = m & 3;  // bits j = 2 jj and 2 jj + 1 of each byte
            const uint32_t a0 = (wR[w] * mul[jj]) & 0x80808080u, a1 = (wR8[w] * mul[jj]) & 0x80808080u;
            const uint32_t a2 = (wR[w] * mul_b[jj]) & 0x80808080u, a3 = (wR8[w] * mul_b[jj]) & 0x80808080u;
#pragma unroll
            for (int b = 0; b < BATCH; b++) {
              const uint4& bb = bf[m >> 1][b];
              if (m == 0) imma_u8_z(c[b], a0, a1, a2, a3, bb.x, bb.y);
              else if (m == 1) imma_u8_z(cx[b], a0, a1, a2, a3, bb.z, bb.w);
              else if (m & 1) imma_u8(cx[b], a0, a1, a2, a3, bb.z, bb.w);
              else imma_u8(c[b], a0, a1, a2, a3, bb.x, bb.y);
            }
          }
        } else {
          // base-3 quotient features of the lane's two words, rows g and g + 8: IMMA m < 5 takes feature
          // m of word 0 (a0 / a1) and of word 1 (a2 / a3); IMMA 5 the constant (a0 / a1)
          uint32_t F[2][2][5];  // [row g / g + 8][word][feature]
#pragma unroll
          for (int rr = 0; rr < 2; rr++)
#pragma unroll
            for (int h = 0; h < 2; h++) {
              const uint32_t Wd = rr ? wR8[h] : wR[h];
              uint32_t E = Wd & 0x00FF00FFu, O = __byte_perm(Wd, 0u, 0x4341);
              F[rr][h][0] = Wd;
#pragma unroll
              for (int j = 1; j <= 4; j++) {
                E = E * k85 + kc80;
                O = O * k85 + kc80;
                F[rr][h][j] = __byte_perm(E, O, 0x7351);
                if (j < 4) {
                  E = __byte_perm(E, 0u, 0x4341);
                  O = __byte_perm(O, 0u, 0x4341);
                }
              }
            }
#pragma unroll
          for (int m = 0; m < 6; m++) {
            const uint32_t a0 = m < 5 ? F[0][0][m] : ones, a1 = m < 5 ? F[1][0][m] : ones;
            const uint32_t a2 = m < 5 ? F[0][1][m] : 0u, a3 = m < 5 ? F[1][1][m] : 0u;
#pragma unroll
            for (int b = 0; b < BATCH; b++) {
              const uint4& bb = bf[m >> 1][b];
              if (m == 0) imma_u8_z(c[b], a0, a1, a2, a3, bb.x, bb.y);
              else if (m == 1) imma_u8_z(cx[b], a0, a1, a2, a3, bb.z, bb.w);
              else if (m & 1) imma_u8(cx[b], a0, a1, a2, a3, bb.z, bb.w);
              else imma_u8(c[b], a0, a1, a2, a3, bb.x, bb.y);
            }
          }
        }
        // epilogue: planes (2 (q & 1), 2 (q & 1) + 1) of this lane's group slot, scaled in fp32
        float cr[BATCH];
#pragma unroll
        for (int b = 0; b < BATCH; b++) {
          cr[b] = 0.f;
          if (LAYOUT == TERN_Q1_0_G128 && (q & 1) == 0)
            cr[b] = NPR ? creg[b] : corr[(ul * 2 + (q >> 1)) * BATCH + b];
          const int vR = (c[b][0] + cx[b][0]) + 256 * (c[b][1] + cx[b][1]);
          const int vR8 = (c[b][2] + cx[b][2]) + 256 * (c[b][3] + cx[b][3]);
          acc[b][0] = fmaf(sR, (float)vR + cr[b], acc[b][0]);
          acc[b][1] = fmaf(sR8, (float)vR8 + cr[b], acc[b][1]);
        }
      }
      // every lane has read this stage: one arrival per warp hands the slot back to the producer
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8u * s);
      // quad sum (planes 0-1 + 2^16 x planes 2-3, both group slots), one partial per row and warp
#pragma unroll
      for (int b = 0; b < BATCH; b++) {
        float a = acc[b][0] * outscale[b], c8 = acc[b][1] * outscale[b];
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        c8 += __shfl_xor_sync(0xffffffffu, c8, 1);
        c8 += __shfl_xor_sync(0xffffffffu, c8, 2);
        if (q == 0) {
          const uint32_t pa = part_w + (uint32_t)i * part_tile + (uint32_t)b * 64u;
          asm volatile("st.shared.f32 [%0], %1;\n\tst.shared.f32 [%0+32], %2;" ::"r"(pa), "f"(a), "f"(c8) : "memory");
        }
      }
      if (++s == p.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  __syncthreads();
  // ---- reduction over warps (and the cluster's K slices, in rank order) -------------------------------
  if (KS > 1) cluster_sync();
  const int ab = *abort_flag;
  int any_abort = ab;
  if (KS > 1) {
    // a slice that gave up poisons the whole tile
    for (int r = 0; r < KS; r++) any_abort |= ld_cluster_s32(smem_u32(ctl), (uint32_t)r) != 0 ? 1 : 0;
  }
  const uint32_t part_a = smem_u32(part);
  for (int e = tid; e < nt * 16 * BATCH; e += blockDim.x) {
    const int tl = e / (16 * BATCH), rr = e % (16 * BATCH), b = rr / 16, row = rr % 16;
    if (tl % KS != rank) continue;
    const int n = (t0 + tl) * 16 + row;
    if (n >= p.n) continue;
    float sum = 0.f;
    for (int r = 0; r < KS; r++)
      for (int w = 0; w < NW; w++) {
        const uint32_t a = part_a + (uint32_t)(((((size_t)tl * NW + w) * BATCH + b) * 16 + row) * 4);
        sum += KS > 1 ? ld_cluster_f32(a, (uint32_t)r) : *reinterpret_cast<const float*>(part + (a - part_a) / 4);
      }
    if (any_abort) sum = __int_as_float(0x7fc00000);
    p.y[(int64_t)b * p.n + n] = __half_as_ushort(__float2half_rn(sum));
  }
  if (KS > 1) cluster_sync();  // no CTA leaves while another may still read its shared memory
}

// ---- host side ------------------------------------------------------------------------------------------
template <int LAYOUT>
size_t i8_smem_bytes(const I8Params& p, int batch) {
  using T = I8L<LAYOUT>;
  size_t s = 1024;  // alignment slack
  s += (size_t)p.stages * p.stage_bytes + 16 * (size_t)p.stages + 32;
  s += (size_t)p.L * T::kMP * batch * T::kEnt * 16;
  s += 4 * 32 * (size_t)batch;
  if (LAYOUT == TERN_Q1_0_G128) s += 4 * (((size_t)p.L * 2 * batch + 3) / 4 * 4);
  // partials / X / the rotated x (disjoint in time)
  s += std::max({4 * (size_t)p.tmax * p.nw * batch * 16, 4 * (size_t)batch * p.xk, (size_t)p.rot_bytes});
  return s;
}

template <int LAYOUT, int BATCH, int NPR, int CPS>
const void* i8_kernel() {
  return reinterpret_cast<const void*>(&gemv_i8_kernel<LAYOUT, BATCH, NPR, CPS>);
}

}  // namespace

// Plan for `cps` CTAs per SM; ok = false when nothing fits.
// Plan for exactly `cps` CTAs per SM, a K split over `ks` CTAs of a cluster and `nw` consumer warps
// (fewer when a slice has fewer units); ok = false when it does not fit.
static I8Plan i8_plan_cfg(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms, int cps, int ks, int nw,
                          bool rotate = false) {
  if (batch < 1 || batch > 2) return I8Plan{};
  const int unit_k = layout == TERN_T3_5PB_G128 ? 160 : 256;
  const int unit_b = layout == TERN_Q2_0_G128 ? 64 : 32;
  const int ent_bytes = (layout == TERN_T3_5PB_G128 ? 3 * 32 : 4 * 16) * 16;  // fragment bytes per unit and row of x
  const int64_t rb = row_bytes(layout, k);
  // whole units only (Q2_0_g128 and Q1_0_g128: K a multiple of 256); other shapes use the older kernels
  if (rb <= 0 || rb % unit_b || n > (int64_t)INT32_MAX) return I8Plan{};
  const int units = (int)(rb / unit_b);
  const int L = (units + ks - 1) / ks;
  if (ks > 1 && L < 8) return I8Plan{};
  nw = std::min(nw, L);
  if (nw < 1 || nw > i8_max_nw(cps)) return I8Plan{};
  I8Plan pl{};
  pl.ks = ks;
  pl.L = L;
  pl.units = units;
  pl.tiles = (int)((n + 15) / 16);
  pl.groups = (int)(k / kGroup);
  const int slice_b = L * unit_b;
  pl.box_b = std::min(1024, slice_b);
  pl.nfull = slice_b / pl.box_b;
  pl.rem_b = slice_b - pl.nfull * pl.box_b;
  // scale box: from the first slice group rounded down to 8, wide enough for every slice
  int scw = 8;
  for (int r = 0; r < ks; r++) {
    const int ua = r * L, ue = std::min(units, ua + L);
    if (ua >= ue) continue;
    const int g0 = ua * unit_k / kGroup, g1 = std::min(pl.groups, (ue * unit_k + kGroup - 1) / kGroup);
    scw = std::max(scw, g1 - (g0 & ~7));
  }
  pl.sc_w = (scw + 7) / 8 * 8;
  if (pl.sc_w > 256) return I8Plan{};
  pl.code_bytes = 16 * slice_b;
  pl.stage_bytes = (pl.code_bytes + 16 * pl.sc_w * 2 + 1023) / 1024 * 1024;
  pl.xk = (L * unit_k + 7) / 8 * 8;
  if (pl.xk > kXV * 8 * (nw + 1) * 32) return I8Plan{};  // every activation of the slice converted in one pass
  const int clusters = std::max(1, cps * sms / ks);
  pl.tmax = (pl.tiles + clusters - 1) / clusters;
  if (rotate) {
    // groups of 128 threads rotate the 1024-blocks covering the slice: exchange buffers of 4 KB per
    // group (sharing space with X), then the rotated fp16 activations of every covering block
    const int groups = std::min((nw + 1) * 32 / kRotThreads, 4);
    if (k % kRotBlock || groups < 1) return I8Plan{};
    int64_t cover = 0;
    for (int r = 0; r < ks; r++) {
      const int64_t a = (int64_t)r * L * unit_k, e = std::min<int64_t>(k, (int64_t)(r + 1) * L * unit_k);
      if (a < e) cover = std::max(cover, ((e + kRotBlock - 1) / kRotBlock - a / kRotBlock) * kRotBlock);
    }
    pl.rot_off = (int)((std::max<size_t>(4 * (size_t)batch * pl.xk, (size_t)groups * kRotBlock * 4) + 15) / 16 * 16);
    pl.rot_bytes = pl.rot_off + (int)(2 * batch * cover);
  }
  const size_t cap = (size_t)(228 / cps - 1) * 1024;
  const size_t fixed = 1024 + 48 + (size_t)L * ent_bytes * batch + 128 * (size_t)batch +
                       (layout == TERN_Q1_0_G128 ? 4 * (((size_t)L * 2 * batch + 3) / 4 * 4) : 0) +
                       std::max({64 * (size_t)pl.tmax * nw * batch, 4 * (size_t)batch * pl.xk, (size_t)pl.rot_bytes});
  if (fixed + 2 * (size_t)(pl.stage_bytes + 16) > cap) return I8Plan{};
  pl.nw = nw;
  pl.npr = (L % nw == 0 && L / nw == 1) ? 1 : 0;
  pl.stages = (int)std::min<size_t>(8, (cap - fixed) / (pl.stage_bytes + 16));
  pl.cps = cps;
  pl.ok = true;
  return pl;
}

// Plan of the int8 kernel for (layout, n, k, batch) on `sms` SMs; ok = false when it does not apply.
// The rule comes from a sweep of every (CTAs per SM, K split, warps) on B200 at batch 1 with weights
// streamed from HBM: one K slice whenever the slice fits; then two CTAs of 8 consumer warps per SM
// once one CTA per SM would own at least 14 row tiles (LM head, 27B-class layers: 2-10 % faster),
// otherwise one CTA of 16 warps, or of 8 when it owns at most two tiles (4096 x 4096: 7-9 %); a slice
// that does not fit is split over a pair of CTAs at one CTA of 12 warps per SM (K = 12288 / 17408:
// 30-35 % faster than four CTAs at two per SM). A split over four is never faster; it stays as the
// last resort before the older kernels.
// The same CTA shape and work split as `base` (so the same sums in the same order) with room for the
// block Hadamard rotation of x in the prologue; ok = false when it does not fit.
I8Plan i8_plan_rotate(const I8Plan& base, int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  if (!base.ok) return I8Plan{};
  const I8Plan r = i8_plan_cfg(layout, n, k, batch, sms, base.cps, base.ks, base.nw, true);
  return (r.ok && r.nw == base.nw && r.L == base.L && r.tmax == base.tmax) ? r : I8Plan{};
}

I8Plan i8_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms) {
  const I8Plan one = i8_plan_cfg(layout, n, k, batch, sms, 1, 1, 16);
  if (one.ok) {
    if (one.tmax >= 14) {
      const I8Plan two = i8_plan_cfg(layout, n, k, batch, sms, 2, 1, 8);
      if (two.ok) return two;
    }
    if (one.tmax <= 2) {
      const I8Plan few = i8_plan_cfg(layout, n, k, batch, sms, 1, 1, 8);
      if (few.ok) return few;
    }
    return one;
  }
  // one slice with the most warps the pass over x allows (a slice too long for 16 warps' threads)
  const I8Plan wide = i8_plan_cfg(layout, n, k, batch, sms, 1, 1, kI8MaxNW1);
  if (wide.ok) return wide;
  // two rows of x with a K split and >= 32 tiles per cluster keep a partial sum per tile, which leaves
  // room for two ring stages only: the older kernels are faster there (LM head, batch 2: 84 vs 95 us)
  if (batch == 2) {
    const int tiles = (int)((n + 15) / 16), tmax2 = (tiles + sms / 2 - 1) / (sms / 2);
    if (tmax2 >= 32) return I8Plan{};
  }
  for (int nw : {12, 16, 8, kI8MaxNW1, 10, 6, 4}) {
    const I8Plan pair = i8_plan_cfg(layout, n, k, batch, sms, 1, 2, nw);
    if (pair.ok) return pair;
  }
  for (int cps : {2, 1})
    for (int nw : {8, 16, kI8MaxNW1, 12, 6, 4}) {
      const I8Plan four = i8_plan_cfg(layout, n, k, batch, sms, cps, 4, nw);
      if (four.ok) return four;
    }
  return I8Plan{};
}

namespace {

template <int LAYOUT, int BATCH, int NPR, int CPS>
cudaError_t launch_i8_t(const tern_matrix& W, const uint16_t* x, uint16_t* y, const I8Plan& pl, cudaStream_t st,
                        uint32_t flags, uint32_t* status, uint64_t wait_ns, const int8_t* signs) {
  using T = I8L<LAYOUT>;
  I8Params p{};
  p.x = x;
  p.y = y;
  p.status = status;
  p.wait_ns = wait_ns ? wait_ns : kI8DefaultWaitNs;
  p.n = (int)W.n;
  p.k = (int)W.k;
  p.batch = BATCH;
  p.groups = pl.groups;
  p.tiles = pl.tiles;
  p.units = pl.units;
  p.L = pl.L;
  p.nw = pl.nw;
  // chunk bounds c nu / nw by a reciprocal: exact while nw^2 L < 2^20 (then (c nu) e < 2^20 with
  // e = nw_rcp nw - 2^20 <= nw), far above any slice a plan holds
  p.nw_rcp = (1u << 20) / (uint32_t)pl.nw + 1u;
  if ((int64_t)pl.nw * pl.nw * pl.L >= (1 << 20)) return cudaErrorInvalidValue;
  p.early = (flags & TERN_GEMV_STATIC_WEIGHTS) ? 1 : 0;
  p.box_b = pl.box_b;
  p.nfull = pl.nfull;
  p.rem_b = pl.rem_b;
  p.sc_w = pl.sc_w;
  p.stage_bytes = pl.stage_bytes;
  p.code_bytes = pl.code_bytes;
  p.stages = pl.stages;
  p.tmax = pl.tmax;
  p.xk = pl.xk;
  p.signs = signs;
  p.rot_off = signs ? pl.rot_off : 0;
  p.rot_bytes = signs ? pl.rot_bytes : 0;
  if (signs && !pl.rot_bytes) return cudaErrorInvalidValue;  // the plan has no room for the rotation
  const size_t smem = i8_smem_bytes<LAYOUT>(p, BATCH);
  const void* kern = i8_kernel<LAYOUT, BATCH, NPR, CPS>();
  // the planned grid: clusters own disjoint tiles and never wait on one another, so clusters that
  // do not fit at once simply run in a later wave
  const int clusters = std::max(1, CPS * sm_count() / pl.ks);
  if ((pl.tiles + clusters - 1) / clusters > pl.tmax) return cudaErrorInvalidValue;  // plan and device disagree
  const size_t smem2 = smem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
  if (e != cudaSuccess) return e;
  // tensor maps: codes as 32-bit words [n][row bytes / 4] (boxes box_b / 4 and rem_b / 4 wide, 16 rows);
  // scales [n][groups] halves (box sc_w x 16); reads past the matrix are zero-filled
  const uint64_t rwords = (uint64_t)row_bytes(W.layout, W.k) / 4;
  CUtensorMap mcf, mcr, msc;
  if (!tmap_2d(&mcf, CU_TENSOR_MAP_DATA_TYPE_UINT32, W.codes, rwords, (uint64_t)W.n, (uint64_t)W.code_row_stride,
               (uint32_t)pl.box_b / 4, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  mcr = mcf;
  if (pl.rem_b && !tmap_2d(&mcr, CU_TENSOR_MAP_DATA_TYPE_UINT32, W.codes, rwords, (uint64_t)W.n,
                           (uint64_t)W.code_row_stride, (uint32_t)pl.rem_b / 4, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!tmap_2d(&msc, CU_TENSOR_MAP_DATA_TYPE_UINT16, W.scales, (uint64_t)pl.groups, (uint64_t)W.n,
               (uint64_t)W.scale_row_stride * 2, (uint32_t)pl.sc_w, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(clusters * pl.ks);
  cfg.blockDim = dim3((pl.nw + 1) * 32);
  cfg.dynamicSmemBytes = smem2;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int na = 0;
  at[na].id = cudaLaunchAttributeClusterDimension;
  at[na].val.clusterDim.x = pl.ks;
  at[na].val.clusterDim.y = 1;
  at[na].val.clusterDim.z = 1;
  na++;
  // always a programmatic dependent: x, y and the status word are touched only after the preceding
  // grid completes; with TERN_GEMV_STATIC_WEIGHTS the weight tiles are requested before that
  at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[na].val.programmaticStreamSerializationAllowed = 1;
  na++;
  cfg.attrs = at;
  cfg.numAttrs = na;
  (void)T::kUnitK;
  e = cudaLaunchKernelEx(&cfg, gemv_i8_kernel<LAYOUT, BATCH, NPR, CPS>, mcf, mcr, msc, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int LAYOUT, int CPS>
cudaError_t launch_i8_c(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, const I8Plan& pl,
                        cudaStream_t st, uint32_t flags, uint32_t* status, uint64_t wait_ns, const int8_t* signs) {
  if (batch == 1)
    return pl.npr ? launch_i8_t<LAYOUT, 1, 1, CPS>(W, x, y, pl, st, flags, status, wait_ns, signs)
                  : launch_i8_t<LAYOUT, 1, 0, CPS>(W, x, y, pl, st, flags, status, wait_ns, signs);
  return pl.npr ? launch_i8_t<LAYOUT, 2, 1, CPS>(W, x, y, pl, st, flags, status, wait_ns, signs)
                : launch_i8_t<LAYOUT, 2, 0, CPS>(W, x, y, pl, st, flags, status, wait_ns, signs);
}
template <int LAYOUT>
cudaError_t launch_i8_l(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, const I8Plan& pl,
                        cudaStream_t st, uint32_t flags, uint32_t* status, uint64_t wait_ns, const int8_t* signs) {
  return pl.cps == 2 ? launch_i8_c<LAYOUT, 2>(W, x, batch, y, pl, st, flags, status, wait_ns, signs)
                     : launch_i8_c<LAYOUT, 1>(W, x, batch, y, pl, st, flags, status, wait_ns, signs);
}

}  // namespace

cudaError_t launch_gemv_i8(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, const I8Plan& pl,
                           cudaStream_t st, uint32_t flags, uint32_t* status, uint64_t wait_ns, const int8_t* signs) {
  if (W.layout == TERN_Q2_0_G128) return launch_i8_l<TERN_Q2_0_G128>(W, x, batch, y, pl, st, flags, status, wait_ns, signs);
  if (W.layout == TERN_Q1_0_G128) return launch_i8_l<TERN_Q1_0_G128>(W, x, batch, y, pl, st, flags, status, wait_ns, signs);
  return launch_i8_l<TERN_T3_5PB_G128>(W, x, batch, y, pl, st, flags, status, wait_ns, signs);
}

}  // namespace tern
