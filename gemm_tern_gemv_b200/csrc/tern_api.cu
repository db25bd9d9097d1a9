// C ABI entry points: argument validation, size arithmetic and dispatch to the kernels.
// Every argument check runs on the host before any CUDA call, so a rejected call touches no
// device state (and works on a machine without a GPU).
#include <cmath>
#include <mutex>
#include <vector>

#include "tern_fwht.cuh"
#include "tern_internal.cuh"

namespace tern {

int64_t row_bytes(int32_t layout, int64_t k) {
  if (k <= 0 || k % kGroup) return -1;
  int64_t b;
  if (layout == TERN_Q2_0_G128) b = k / 4;           // 4 two-bit codes per byte
  else if (layout == TERN_T3_5PB_G128) b = (k + 4) / 5;  // 5 trits per byte
  else if (layout == TERN_Q1_0_G128) b = k / 8;      // 8 sign bits per byte
  else return -1;
  return (b + 15) / 16 * 16;
}

int sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= (int)cache.size()) cache.resize(dev + 1, 0);
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

}  // namespace tern

using namespace tern;

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline bool valid_layout(int32_t l) {
  return l == TERN_Q2_0_G128 || l == TERN_T3_5PB_G128 || l == TERN_Q1_0_G128;
}

// Checks shared by every call that takes a packed matrix.
static tern_status check_matrix(const tern_matrix* W) {
  if (!W) return TERN_ERR_INVALID_ARG;
  if (!valid_layout(W->layout)) return TERN_ERR_UNSUPPORTED;
  if (W->n <= 0 || W->k <= 0 || W->k % kGroup) return TERN_ERR_INVALID_ARG;
  if (W->n > (int64_t)INT32_MAX || W->k > (int64_t)INT32_MAX / 2) return TERN_ERR_INVALID_ARG;
  if (!W->codes || !W->scales) return TERN_ERR_INVALID_ARG;
  if (W->code_row_stride < row_bytes(W->layout, W->k)) return TERN_ERR_INVALID_ARG;
  if (W->scale_row_stride < W->k / kGroup) return TERN_ERR_INVALID_ARG;
  if (!aligned16(W->codes) || !aligned16(W->scales)) return TERN_ERR_ALIGNMENT;
  if (W->code_row_stride % 16 || W->scale_row_stride % 8) return TERN_ERR_ALIGNMENT;
  return TERN_OK;
}

static tern_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TERN_OK : TERN_ERR_CUDA; }

extern "C" {

int64_t tern_row_bytes(int32_t layout, int64_t k) { return row_bytes(layout, k); }

int64_t tern_packed_bytes(int32_t layout, int64_t n, int64_t k) {
  int64_t rb = row_bytes(layout, k);
  if (rb < 0 || n <= 0) return -1;
  return n * rb;
}

double tern_bits_per_weight(int32_t layout, int64_t k) {
  int64_t rb = row_bytes(layout, k);
  if (rb < 0) return -1.0;
  return (double)(rb * 8 + (k / kGroup) * 16) / (double)k;
}

static tern_status pack_common(int32_t layout, int64_t n, int64_t k, const uint16_t* w, int64_t w_row_stride,
                               const uint16_t* scales, int64_t scale_row_stride, void* codes,
                               int64_t code_row_stride, const void* prev, int64_t prev_row_stride,
                               uint64_t* flips, void* stream) {
  if (!valid_layout(layout)) return TERN_ERR_UNSUPPORTED;
  if (n <= 0 || k <= 0 || k % kGroup || n > (int64_t)INT32_MAX || k > (int64_t)INT32_MAX / 2)
    return TERN_ERR_INVALID_ARG;
  if (!w || !scales || !codes) return TERN_ERR_INVALID_ARG;
  if (w_row_stride < k || scale_row_stride < k / kGroup || code_row_stride < row_bytes(layout, k))
    return TERN_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(scales) || !aligned16(codes)) return TERN_ERR_ALIGNMENT;
  if (w_row_stride % 8 || scale_row_stride % 8 || code_row_stride % 16) return TERN_ERR_ALIGNMENT;
  if (prev) {
    if (!flips || prev_row_stride < row_bytes(layout, k)) return TERN_ERR_INVALID_ARG;
    if (!aligned16(prev) || prev_row_stride % 16 || (reinterpret_cast<uintptr_t>(flips) & 7u)) return TERN_ERR_ALIGNMENT;
  }
  return from_cuda(launch_pack(layout, n, k, w, w_row_stride, scales, scale_row_stride,
                               static_cast<uint8_t*>(codes), code_row_stride,
                               static_cast<const uint8_t*>(prev), prev_row_stride,
                               reinterpret_cast<unsigned long long*>(flips), static_cast<cudaStream_t>(stream)));
}

tern_status tern_pack(int32_t layout, int64_t n, int64_t k, const uint16_t* w, int64_t w_row_stride,
                      const uint16_t* scales, int64_t scale_row_stride, void* codes,
                      int64_t code_row_stride, void* stream) {
  return pack_common(layout, n, k, w, w_row_stride, scales, scale_row_stride, codes, code_row_stride, nullptr, 0,
                     nullptr, stream);
}

tern_status tern_pack_flips(int32_t layout, int64_t n, int64_t k, const uint16_t* w, int64_t w_row_stride,
                            const uint16_t* scales, int64_t scale_row_stride, void* codes, int64_t code_row_stride,
                            const void* prev_codes, int64_t prev_row_stride, uint64_t* flips, void* stream) {
  if (!prev_codes || !flips) return TERN_ERR_INVALID_ARG;
  if (prev_codes == codes) return TERN_ERR_INVALID_ARG;  // the previous codes must survive the pack
  return pack_common(layout, n, k, w, w_row_stride, scales, scale_row_stride, codes, code_row_stride, prev_codes,
                     prev_row_stride, flips, stream);
}

tern_status tern_unpack(const tern_matrix* W, uint16_t* w_out, int64_t w_row_stride, int8_t* t_out,
                        int64_t t_row_stride, int32_t* invalid_count, void* stream) {
  tern_status s = check_matrix(W);
  if (s != TERN_OK) return s;
  if (!w_out && !t_out) return TERN_ERR_INVALID_ARG;
  if (w_out && w_row_stride < W->k) return TERN_ERR_INVALID_ARG;
  if (t_out && t_row_stride < W->k) return TERN_ERR_INVALID_ARG;
  if ((w_out && (!aligned16(w_out) || w_row_stride % 8)) || (t_out && (!aligned16(t_out) || t_row_stride % 16)))
    return TERN_ERR_ALIGNMENT;
  if (invalid_count && (reinterpret_cast<uintptr_t>(invalid_count) & 3u)) return TERN_ERR_ALIGNMENT;
  return from_cuda(launch_unpack(*W, w_out, w_row_stride, t_out, t_row_stride, invalid_count,
                                 static_cast<cudaStream_t>(stream)));
}

size_t tern_gemv_workspace_bytes(const tern_matrix* W, int64_t batch) {
  if (!W || W->n <= 0 || W->k <= 0 || W->k % kGroup) return 0;
  if (!valid_layout(W->layout)) return 0;
  if (batch < 1 || batch > TERN_GEMV_MAX_BATCH) return 0;
  return gemv_plan(W->layout, W->n, W->k, batch, sm_count()).ws_bytes;
}

tern_status tern_gemv(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return tern_gemv_ex(W, x, batch, y, workspace, workspace_bytes, 0u, stream);
}

tern_status tern_gemv_ex(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y, void* workspace,
                         size_t workspace_bytes, uint32_t flags, void* stream) {
  tern_gemv_opts o{};
  o.flags = flags;
  return tern_gemv_opt(W, x, batch, y, workspace, workspace_bytes, &o, stream);
}

// The plan of tern_gemv_opt: the GEMV plan, and whether x is rotated inside the int8-plane kernel (same
// work split as without the rotation) or first into the workspace at rot_off.
struct OptPlan {
  GemvPlan plan;
  bool fused;
  size_t rot_off, ws;
};
static OptPlan opt_plan(const tern_matrix& W, int64_t batch, bool rotate) {
  OptPlan o{};
  o.plan = gemv_plan(W.layout, W.n, W.k, batch, sm_count());
  o.ws = o.plan.ws_bytes;
  if (rotate) {
    if (o.plan.i8) {
      const I8Plan r = i8_plan_rotate(o.plan.i8p, W.layout, W.n, W.k, std::min<int64_t>(batch, 2), sm_count());
      if (r.ok) {
        o.plan.i8p = r;
        o.fused = true;
        return o;
      }
    }
    o.rot_off = (o.ws + 255) / 256 * 256;
    o.ws = o.rot_off + (size_t)batch * (size_t)W.k * 2;
  }
  return o;
}

size_t tern_gemv_opt_workspace_bytes(const tern_matrix* W, int64_t batch, const tern_gemv_opts* opts) {
  const bool rotate = opts && opts->rotate_signs;
  if (!rotate) return tern_gemv_workspace_bytes(W, batch);
  if (!W || W->n <= 0 || W->k <= 0 || W->k % kRotBlock) return 0;
  if (!valid_layout(W->layout)) return 0;
  if (batch < 1 || batch > TERN_GEMV_MAX_BATCH) return 0;
  return opt_plan(*W, batch, true).ws;
}

tern_status tern_gemv_opt(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y, void* workspace,
                          size_t workspace_bytes, const tern_gemv_opts* opts, void* stream) {
  const uint32_t flags = opts ? opts->flags : 0u;
  uint32_t* status = opts ? opts->device_status : nullptr;
  const uint64_t wait_ns = opts ? opts->wait_limit_ns : 0u;
  const int8_t* signs = opts ? opts->rotate_signs : nullptr;
  if (flags & ~(uint32_t)TERN_GEMV_STATIC_WEIGHTS) return TERN_ERR_INVALID_ARG;
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return TERN_ERR_ALIGNMENT;
  tern_status s = check_matrix(W);
  if (s != TERN_OK) return s;
  if (batch < 1 || batch > TERN_GEMV_MAX_BATCH || !x || !y) return TERN_ERR_INVALID_ARG;
  if (signs && W->k % kRotBlock) return TERN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TERN_ERR_ALIGNMENT;
  if (!gemv_supported(W->layout, W->n, W->k, batch)) return TERN_ERR_UNSUPPORTED;
  const OptPlan op = opt_plan(*W, batch, signs != nullptr);
  if (op.ws) {
    if (!workspace || workspace_bytes < op.ws) return TERN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return TERN_ERR_ALIGNMENT;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (signs && !op.fused) {
    uint16_t* xr = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + op.rot_off);
    const cudaError_t e = launch_rotate(x, batch, W->k, signs, xr, st);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(launch_gemv(*W, xr, (int)batch, y, workspace, op.plan, st, flags, status, wait_ns));
  }
  return from_cuda(launch_gemv(*W, x, (int)batch, y, workspace, op.plan, st, flags, status, wait_ns, signs));
}

tern_status tern_gemv_plan_describe(const tern_matrix* W, int64_t batch, const tern_gemv_opts* opts,
                                    tern_gemv_plan_info* out) {
  if (!out) return TERN_ERR_INVALID_ARG;
  const uint32_t flags = opts ? opts->flags : 0u;
  const int8_t* signs = opts ? opts->rotate_signs : nullptr;
  if (flags & ~(uint32_t)TERN_GEMV_STATIC_WEIGHTS) return TERN_ERR_INVALID_ARG;
  tern_status s = check_matrix(W);
  if (s != TERN_OK) return s;
  if (batch < 1 || batch > TERN_GEMV_MAX_BATCH) return TERN_ERR_INVALID_ARG;
  if (signs && W->k % kRotBlock) return TERN_ERR_INVALID_ARG;
  if (!gemv_supported(W->layout, W->n, W->k, batch)) return TERN_ERR_UNSUPPORTED;
  const OptPlan op = opt_plan(*W, batch, signs != nullptr);
  const GemvPlan& p = op.plan;
  tern_gemv_plan_info info{};
  if (p.i8) {
    info.kernel = TERN_GEMV_KERNEL_INT8_PLANES;
    info.launches = (int32_t)((batch + 1) / 2);  // one launch per pair of rows
    info.k_slices = p.i8p.ks;
    info.ctas_per_sm = p.i8p.cps;
    info.warps = p.i8p.nw;
    info.stages = p.i8p.stages;
  } else if (p.gemm) {
    info.kernel = TERN_GEMV_KERNEL_TCGEN05;
    info.launches = 1;
    info.k_slices = 1;
  } else if (p.reg) {
    info.kernel = TERN_GEMV_KERNEL_REGISTER;
    info.launches = W->layout == TERN_Q1_0_G128 ? (int32_t)((batch + kBinChunk - 1) / kBinChunk) : 1;
    info.k_slices = p.splits;
    info.ctas_per_sm = p.warps == 8 ? 2 : 1;
    info.warps = p.warps;
  } else {
    info.kernel = TERN_GEMV_KERNEL_SHARED;
    info.launches = 1;
    info.k_slices = p.splits;
  }
  info.rotation_fused = op.fused ? 1 : 0;
  if (signs && !op.fused) info.launches += 1;  // tern_hadamard_rotate's kernel into the workspace
  info.workspace_bytes = op.ws;
  *out = info;
  return TERN_OK;
}

tern_status tern_gemv_noalloc(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y, void* stream) {
  tern_status s = check_matrix(W);
  if (s != TERN_OK) return s;
  if (batch < 1 || batch > TERN_GEMV_MAX_BATCH || !x || !y) return TERN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TERN_ERR_ALIGNMENT;
  if (!gemv_supported(W->layout, W->n, W->k, batch)) return TERN_ERR_UNSUPPORTED;
  return gemv_noalloc(*W, x, (int)batch, y, static_cast<cudaStream_t>(stream));
}

tern_status tern_gemm(const tern_matrix* W, const uint16_t* X, int64_t m, uint16_t* Y,
                      uint32_t* device_status, void* stream) {
  tern_status s = check_matrix(W);
  if (s != TERN_OK) return s;
  if (m <= 0 || m > (int64_t)INT32_MAX || !X || !Y) return TERN_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return TERN_ERR_ALIGNMENT;
  if (W->n % 8) return TERN_ERR_ALIGNMENT;  // Y rows are stored as 16-byte vectors
  if (device_status && (reinterpret_cast<uintptr_t>(device_status) & 3u)) return TERN_ERR_ALIGNMENT;
  return from_cuda(launch_gemm(*W, X, m, Y, device_status, static_cast<cudaStream_t>(stream)));
}

size_t tern_gemv_t_workspace_bytes(const tern_matrix* W, int64_t batch) {
  if (!W || W->n <= 0 || W->k <= 0 || W->k % kGroup) return 0;
  if (!valid_layout(W->layout)) return 0;
  if (batch < 1 || batch > TERN_GEMV_T_MAX_BATCH) return 0;
  return gemv_t_plan(W->layout, W->n, W->k, batch, sm_count()).ws_bytes;
}

tern_status tern_gemv_t(const tern_matrix* W, const uint16_t* dy, int64_t batch, uint16_t* dx, void* workspace,
                        size_t workspace_bytes, void* stream) {
  tern_status s = check_matrix(W);
  if (s != TERN_OK) return s;
  if (batch < 1 || batch > TERN_GEMV_T_MAX_BATCH || !dy || !dx) return TERN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(dx)) & 1u) return TERN_ERR_ALIGNMENT;
  const GemvTPlan plan = gemv_t_plan(W->layout, W->n, W->k, batch, sm_count());
  if (plan.ws_bytes) {
    if (!workspace || workspace_bytes < plan.ws_bytes) return TERN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return TERN_ERR_ALIGNMENT;
  }
  return from_cuda(launch_gemv_t(*W, dy, (int)batch, dx, workspace, plan, static_cast<cudaStream_t>(stream)));
}

tern_status tern_hadamard_rotate(const uint16_t* x, int64_t batch, int64_t k, const int8_t* signs, uint16_t* y,
                                 void* stream) {
  if (!x || !y || !signs || batch < 1 || k <= 0 || k % 1024) return TERN_ERR_INVALID_ARG;
  if (batch > (int64_t)INT32_MAX / (k / 1024) || batch * k > (int64_t)1 << 40) return TERN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 1u) return TERN_ERR_ALIGNMENT;
  return from_cuda(launch_rotate(x, batch, k, signs, y, static_cast<cudaStream_t>(stream)));
}

tern_status tern_device_result(uint32_t device_status, int64_t invalid_count) {
  if (device_status & TERN_DEVICE_TIMEOUT) return TERN_ERR_TIMEOUT;
  if (invalid_count > 0) return TERN_ERR_INVALID_CODE;
  return TERN_OK;
}

const char* tern_status_string(tern_status status) {
  switch (status) {
    case TERN_OK: return "ok";
    case TERN_ERR_INVALID_ARG: return "invalid argument";
    case TERN_ERR_UNSUPPORTED: return "unsupported layout or size";
    case TERN_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case TERN_ERR_WORKSPACE: return "split-K workspace missing or too small";
    case TERN_ERR_INVALID_CODE: return "invalid packed code";
    case TERN_ERR_TIMEOUT: return "device pipeline wait timed out";
    case TERN_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

int32_t tern_version(void) { return 100; }

}  // extern "C"
