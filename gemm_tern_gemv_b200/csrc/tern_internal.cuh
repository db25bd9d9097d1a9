// Internal declarations shared by the library's translation units (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstdint>

#include "tern.h"

namespace tern {

constexpr int kGroup = TERN_GROUP;
constexpr int kBinChunk = 2;  // batch rows per launch of the binary register kernel

// Minimum packed row stride in bytes (see tern_row_bytes); -1 on invalid arguments.
int64_t row_bytes(int32_t layout, int64_t k);

// Number of streaming multiprocessors of the current device (cached per device).
int sm_count();

// 2-D TMA tensor map over [outer][inner] elements with rows row_stride_bytes apart, boxes of
// box_outer x box_inner, out-of-range elements read as zero; encoded once per distinct argument set.
bool tmap_2d(CUtensorMap* out, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);

// ---- launchers (arguments already validated by the C ABI layer) ----------------------------
// prev / flips: optional previous packing of the same matrix and the flip counter it feeds
cudaError_t launch_pack(int32_t layout, int64_t n, int64_t k, const uint16_t* w, int64_t w_stride,
                        const uint16_t* s, int64_t s_stride, uint8_t* codes, int64_t c_stride,
                        const uint8_t* prev, int64_t p_stride, unsigned long long* flips, cudaStream_t st);

cudaError_t launch_unpack(const tern_matrix& W, uint16_t* w_out, int64_t w_stride, int8_t* t_out,
                          int64_t t_stride, int32_t* invalid_count, cudaStream_t st);

// Plan of the int8-plane GEMV (batch 1-2): K slices per cluster, consumer warps, TMA stage geometry.
struct I8Plan {
  bool ok;
  int ks;          // K slices = CTAs per cluster (1, 2 or 4)
  int L;           // units per slice
  int nw;          // consumer warps per CTA
  int npr;         // 1: each consumer warp owns exactly one unit of a slice
  int units, tiles, groups;
  int box_b, nfull, rem_b, sc_w;  // TMA boxes of one stage
  int code_bytes, stage_bytes, stages;
  int xk;          // activations per CTA (halves)
  int tmax;        // tiles per cluster (upper bound)
  int cps;         // CTAs per SM (1 or 2)
  int rot_off, rot_bytes;  // block Hadamard rotation of x in the prologue (0 = no room planned)
};
I8Plan i8_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms);
// `base` with room for rotating x in the prologue, same work split; ok = false when it does not fit
I8Plan i8_plan_rotate(const I8Plan& base, int32_t layout, int64_t n, int64_t k, int64_t batch, int sms);
// status / wait_ns: optional device status word and bound on each pipeline wait (0 = 1 s);
// signs: non-null to multiply by R x (the plan must come from i8_plan_rotate)
cudaError_t launch_gemv_i8(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, const I8Plan& pl,
                           cudaStream_t st, uint32_t flags, uint32_t* status, uint64_t wait_ns,
                           const int8_t* signs = nullptr);

// Split-K plan of the decode GEMV for one (layout, n, k, batch) on a device with `sms` SMs.
struct GemvPlan {
  bool gemm;            // Q2_0_g128 with many rows of x: the tcgen05 GEMM kernel (no workspace)
  bool reg;             // small-batch kernel with in-register decode (else the shared-memory one)
  int rows_per_cta;     // output rows of one warp tile
  int row_blocks;       // ceil(n / rows_per_cta)
  int splits;           // K slices (1 = no workspace)
  int groups_per_split; // 128-weight groups per slice (a multiple of 5 for base-3 when splits > 1)
  int grid_x;           // register kernel: CTAs per K slice
  int run;              // register kernel: (tile, window) units per warp run
  int kmax;             // register kernel: partial-sum slots per tile and K slice
  bool local;           // register kernel: each CTA owns whole row tiles, summed in shared memory
  int warps;            // register kernel: warps per CTA (16, one CTA per SM; or 8, two per SM)
  size_t ws_partial_bytes;  // fp32 partial sums [splits * slots][batch][n]
  size_t ws_bytes;          // partials + one int32 counter per row block, rounded to 16
  bool i8;                  // batch 1-2: the int8-plane kernel (no workspace)
  I8Plan i8p;
};
GemvPlan gemv_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms);
// False only for a binary matrix too large for the register kernel's 32-bit unit indices at a batch
// the GEMM kernel does not take.
bool gemv_supported(int32_t layout, int64_t n, int64_t k, int64_t batch);

// flags: TERN_GEMV_* bits of tern_gemv_ex (0 for tern_gemv).
// status / wait_ns: optional device status word and wait bound of the kernels that wait on a pipeline.
// signs: non-null only with an int8-plane plan from i8_plan_rotate (x is rotated in the prologue).
cudaError_t launch_gemv(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y,
                        void* workspace, const GemvPlan& plan, cudaStream_t st, uint32_t flags = 0,
                        uint32_t* status = nullptr, uint64_t wait_ns = 0, const int8_t* signs = nullptr);

// tern_gemv_noalloc's work after argument checks (scratch in a static device array).
tern_status gemv_noalloc(const tern_matrix& W, const uint16_t* x, int batch, uint16_t* y, cudaStream_t st);

cudaError_t launch_gemm(const tern_matrix& W, const uint16_t* X, int64_t m, uint16_t* Y,
                        uint32_t* device_status, cudaStream_t st);

// Transposed product dx = W^T dy: column blocks x row slices; fp32 partials per slice when sliced.
struct GemvTPlan {
  int col_blocks;
  int slices;
  int64_t rows_per_slice;
  size_t ws_bytes;
};
GemvTPlan gemv_t_plan(int32_t layout, int64_t n, int64_t k, int64_t batch, int sms);
cudaError_t launch_gemv_t(const tern_matrix& W, const uint16_t* dy, int batch, uint16_t* dx, void* workspace,
                          const GemvTPlan& plan, cudaStream_t st);

cudaError_t launch_rotate(const uint16_t* x, int64_t batch, int64_t k, const int8_t* signs, uint16_t* y,
                          cudaStream_t st);

}  // namespace tern
