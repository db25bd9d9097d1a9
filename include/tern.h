/*
 * tern.h — C ABI of the ternary group-scaled matrix-product library for NVIDIA B200 (sm_100a).
 *
 * Weights are ternary codes t in {-1, 0, +1} with one IEEE fp16 scale s per 128 consecutive
 * weights along K, so w = s * t ("Bonsai 27B와 1비트가 살아남는 법", velog.io, section "포맷의
 * 정체", eq. w_i = s_g * t_i; "Ternary Bonsai 2 27B, 5.93GB로 줄이고도 FP16 성능의 98.2%를 지킨
 * 삼진 모델", discuss.pytorch.kr, section "그룹 단위 스케일을 공유하는 삼진 형식"). The product
 * kernels read the packed codes directly and never materialise fp16 weights in device memory
 * (same page, section "하이브리드 어텐션을 위한 저비트 커널").
 *
 * Packed layouts (the pages name the containers but print no bit layout; these are this
 * library's definitions):
 *   TERN_Q2_0_G128   t as a 2-bit two's-complement field (0b00 = 0, 0b01 = +1, 0b11 = -1;
 *                    0b10 is an invalid code); weight k of a row is in byte k/4 at bits
 *                    2*(k%4)..2*(k%4)+1. A row is K/4 bytes. 2 + 16/128 = 2.125 bits per weight,
 *                    the 34-bytes-per-128-weights container of the page above, section "두 가지
 *                    패킹: PTQ1_0과 PQ2_0". A zero-filled row is an all-zero row.
 *   TERN_T3_5PB_G128 dense base-3: byte j of a row is sum_{i<5} c_{5j+i} * 3^i, c = t + 1; trits
 *                    past K are c = 1; the row is padded to a multiple of 16 bytes with bytes of
 *                    value 121 (five c = 1 trits). About 1.725 bits per weight at K = 5120, a
 *                    stand-in for the denser PTQ1_0 packing of the same section. A byte > 242
 *                    is invalid.
 *   TERN_Q1_0_G128   binary sibling, t in {-1, +1} ("Bonsai 27B와 1비트가 살아남는 법", section
 *                    "ternary와 binary가 뭔가": binary with the group scale is 1.125 bits per
 *                    weight; the 1-bit GGUF Q1_0_g128 of that page's model card): weight k of a
 *                    row is bit k%8 of byte k/8, 1 = +1 and 0 = -1. A row is K/8 bytes; every bit
 *                    pattern is valid. tern_pack binarizes: t = -1 exactly when w * s < 0.
 * Scales are a separate fp16 array s[n][g], g = k / 128, with a row stride in halves.
 *
 * Conventions for every call:
 *   - Memory: every pointer argument named as device memory must be device memory (or managed)
 *     on the current device; the caller owns all buffers. The library allocates no device memory
 *     per call. tern_gemm keeps a small host-side cache of TMA descriptors.
 *   - fp16 values are passed as uint16_t bit patterns (IEEE binary16).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). All device work is enqueued
 *     on it asynchronously; the call returns before the GPU finishes.
 *   - Argument errors are detected on the host before any launch and returned synchronously; no
 *     CUDA call is made in that case. A launch failure returns TERN_ERR_CUDA.
 *   - Alignment: device pointers must be 16-byte aligned and row strides in bytes multiples of 16
 *     (code_row_stride, 2*scale_row_stride, 2*w_row_stride); otherwise TERN_ERR_ALIGNMENT.
 *   - Dense activations and outputs are contiguous row-major: x[batch][K], y[batch][N],
 *     X[M][K], Y[M][N]; products accumulate in fp32 and round the result to fp16 once.
 *   - No call validates codes except tern_unpack; products on invalid codes give unspecified
 *     (finite) values.
 */
#ifndef TERN_H
#define TERN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TERN_API __attribute__((visibility("default")))
#else
#define TERN_API
#endif

#define TERN_GROUP 128           /* weights per fp16 scale */
#define TERN_GEMV_MAX_BATCH 64   /* largest batch tern_gemv accepts */

typedef enum tern_status {
  TERN_OK = 0,
  TERN_ERR_INVALID_ARG = 1,   /* NULL pointer, non-positive size, K % 128 != 0, stride too small */
  TERN_ERR_UNSUPPORTED = 2,   /* unknown layout id, or a layout/size this entry point lacks */
  TERN_ERR_ALIGNMENT = 3,     /* pointer or stride not 16-byte aligned */
  TERN_ERR_WORKSPACE = 4,     /* split-K workspace missing or smaller than required */
  TERN_ERR_INVALID_CODE = 5,  /* tern_device_result: tern_unpack counted invalid codes */
  TERN_ERR_TIMEOUT = 6,       /* tern_device_result: a pipeline wait of a product ran out */
  TERN_ERR_CUDA = 7           /* a CUDA runtime call or kernel launch failed */
} tern_status;

typedef enum tern_layout {
  TERN_Q2_0_G128 = 1,
  TERN_T3_5PB_G128 = 2,
  TERN_Q1_0_G128 = 3
} tern_layout;

/* Bits of the device status word that tern_gemm and tern_gemv_opt write (atomic OR) when given one. */
#define TERN_DEVICE_TIMEOUT 1u   /* a pipeline wait exceeded its bound; the tile was abandoned */

/* A packed ternary matrix W[n][k] (n output features, k reduction length). Host struct holding
 * device pointers; the library reads it during the call only. */
typedef struct tern_matrix {
  int32_t layout;                 /* tern_layout */
  int64_t n;                      /* rows (output features), >= 1 */
  int64_t k;                      /* reduction length, a positive multiple of 128 */
  const void* codes;              /* device, uint8 [n][code_row_stride] */
  int64_t code_row_stride;        /* bytes, >= tern_row_bytes(layout, k), multiple of 16 */
  const uint16_t* scales;         /* device, fp16 [n][scale_row_stride] */
  int64_t scale_row_stride;       /* halves, >= k / 128, multiple of 8 */
} tern_matrix;

/* ---- size arithmetic (host only, no CUDA) ------------------------------------------------ */

/* Minimum packed row stride in bytes: K/4 for Q2_0_g128, ceil(K/5) rounded up to 16 for base-3,
 * K/8 for Q1_0_g128 (the containers of "Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "두
 * 가지 패킹: PTQ1_0과 PQ2_0": 2-bit slots, dense trits; "Bonsai 27B와 1비트가 살아남는 법" velog.io,
 * section "ternary와 binary가 뭔가": one bit per binary weight; codes only, scales are separate).
 * Returns -1 for an unknown layout or K not a positive multiple of 128. */
TERN_API int64_t tern_row_bytes(int32_t layout, int64_t k);

/* n * tern_row_bytes(layout, k): bytes of packed codes at the minimum stride (scales excluded); with
 * n * (k/128) * 2 bytes of scales this is what a product streams per call (section "두 가지 패킹" of
 * the page above gives the per-128-weight container sizes it is checked against).
 * Returns -1 on invalid arguments. */
TERN_API int64_t tern_packed_bytes(int32_t layout, int64_t n, int64_t k);

/* Stored bits per weight at the minimum stride, counting the fp16 scale per 128 weights:
 * exactly 2.125 for Q2_0_g128 and 1.125 for Q1_0_g128; 1.725 for base-3 at K = 5120 ("두 가지 패킹" section's
 * containers and the information bound log2(3) + 16/128 of section "그룹 단위 스케일을 공유하는
 * 삼진 형식", eq. b_eff, bound it from below). Returns -1 on invalid arguments. */
TERN_API double tern_bits_per_weight(int32_t layout, int64_t k);

/* ---- ternarize + pack --------------------------------------------------------------------- */

/* The QAT re-ternarize-and-repack step ("Metal 환경에서 ... Bonsai 8B를 파인튜닝", molayo1419.me,
 * paragraph "그것을 파인튜닝하는 방법": ternarize each 128-weight group on every forward pass,
 * then re-pack to 2 bits): t = round(clamp(w / s, -1, 1)) per weight with its group's scale,
 * ties |w/s| = 1/2 rounding to even (t = 0); s == 0 or NaN, or w NaN, give t = 0. The result is
 * bit-identical to that rule evaluated with exact division. For TERN_Q1_0_G128 the rule is the
 * binary one: t = -1 exactly when w * s < 0, else +1 (zero, NaN and s == 0 give +1).
 *   w       device fp16 [n][w_row_stride] latent weights (first k of each row used)
 *   scales  device fp16 [n][scale_row_stride]
 *   codes   device uint8 [n][code_row_stride] output; exactly tern_row_bytes(layout, k) bytes of
 *           each row are written (padding included), the rest of the stride is left untouched.
 * Errors: TERN_ERR_INVALID_ARG, TERN_ERR_UNSUPPORTED, TERN_ERR_ALIGNMENT, TERN_ERR_CUDA. */
TERN_API tern_status tern_pack(int32_t layout, int64_t n, int64_t k,
                      const uint16_t* w, int64_t w_row_stride,
                      const uint16_t* scales, int64_t scale_row_stride,
                      void* codes, int64_t code_row_stride, void* stream);

/* tern_pack that also counts code flips against the previous packing of the same matrix: the QAT
 * loop watches how many weights change their code from one step to the next ("Metal 환경에서 ...
 * Bonsai 8B를 파인튜닝", molayo1419.me, paragraph "그것을 파인튜닝하는 방법" and its lr study: flips,
 * not the loss, show whether training moves the model).
 *   prev_codes       device uint8 [n][prev_row_stride]: the previous packed codes, same layout and
 *                    k; must not overlap `codes`
 *   flips            device uint64: the number of weights (k < K) whose code field (Q2 2-bit field,
 *                    base-3 digit, binary sign bit) differs from prev_codes is ADDED (the caller zeroes it); for
 *                    valid codes that is the number of weights whose t changed
 * Errors: those of tern_pack; TERN_ERR_INVALID_ARG for NULL prev_codes / flips, prev_codes ==
 *         codes or a short prev_row_stride; TERN_ERR_ALIGNMENT for a misaligned prev_codes,
 *         prev_row_stride or flips. */
TERN_API tern_status tern_pack_flips(int32_t layout, int64_t n, int64_t k, const uint16_t* w, int64_t w_row_stride,
                                     const uint16_t* scales, int64_t scale_row_stride, void* codes,
                                     int64_t code_row_stride, const void* prev_codes, int64_t prev_row_stride,
                                     uint64_t* flips, void* stream);

/* ---- unpack (test / debug path; the products never call it) ------------------------------ */

/* Expands W to dense form: w = s * t per weight ("Bonsai 27B와 1비트가 살아남는 법", section "포맷의
 * 정체", eq. w_i = s_g * t_i), the exact inverse of tern_pack on its codes ("Metal 환경에서 ... Bonsai
 * 8B를 파인튜닝", paragraph "그것을 파인튜닝하는 방법": lossless re-encode). Either output may be NULL,
 * not both.
 *   w_out          device fp16 [n][w_row_stride]: s * t (exact in fp16), 0 for invalid codes
 *   t_out          device int8 [n][t_row_stride]: t, 0 for invalid codes (t_row_stride bytes)
 *   invalid_count  device int32 or NULL: the number of weights with an invalid code is ADDED to
 *                  *invalid_count (caller zeroes it). An invalid base-3 byte counts once per
 *                  weight it holds. No trap, no abort. */
TERN_API tern_status tern_unpack(const tern_matrix* W, uint16_t* w_out, int64_t w_row_stride,
                        int8_t* t_out, int64_t t_row_stride, int32_t* invalid_count, void* stream);

/* ---- decode GEMV (batch 1..64) -------------------------------------------------------------- */

/* Bytes of split-K workspace tern_gemv needs for this matrix and batch (0 when it needs none; batches
 * 1-2 of matrices whose rows are whole 32- or 64-byte units split K over thread-block clusters
 * instead). The product is the decode GEMV of "Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section
 * "처리량" (batch-1 token generation).
 * Depends only on (W->layout, W->n, W->k, batch) and the current device's SM count.
 * Returns 0 also for invalid arguments (tern_gemv then reports the error). */
TERN_API size_t tern_gemv_workspace_bytes(const tern_matrix* W, int64_t batch);

/* y[b][n] = sum_g s[n][g] * sum_{k in group g} t[n][k] * x[b][k] for b < batch ("Ternary Bonsai 2
 * 27B ..." discuss.pytorch.kr, section "그룹 단위 스케일을 공유하는 삼진 형식", eq. w_i = s_g t_i; the
 * packed codes are read directly and unpack and group scale are fused, section "하이브리드 어텐션을
 * 위한 저비트 커널"); the activations' own precision is kept (x exact as int8 planes or fp16), fp32
 * accumulation, fp16 result. Batches 1-2 run on int8 mma.sync kernels fed by TMA (K split over a
 * cluster for narrow matrices; rows that are not whole 64-byte (Q2) / 32-byte units, and batch-2 K
 * splits of tall matrices, use the fp16 kernels); batches 3-16 on fp16 mma.sync kernels; batches of 17 or more with
 * n % 8 == 0 on the tcgen05 kernel of tern_gemm (no workspace), as do Q1_0_g128 batches of 5 or
 * more with n % 8 == 0. Other Q1_0_g128 batches run as one launch per two rows of x.
 * The result of a call depends only on (W, x, batch) and the device.
 *   x          device fp16 [batch][k], contiguous
 *   y          device fp16 [batch][n], contiguous
 *   workspace  device, >= tern_gemv_workspace_bytes(W, batch) bytes, 16-byte aligned; may be
 *              NULL when that size is 0. Its trailing counter words must be zero before the first
 *              call that uses this workspace (e.g. cudaMemset once); every call leaves them zero
 *              again. Calls that share a workspace must not overlap on the GPU.
 * Errors: TERN_ERR_INVALID_ARG (batch outside 1..64, ...), TERN_ERR_UNSUPPORTED (also a Q1_0_g128
 *         matrix of 2^30 or more (32-row tile, 512-weight window) units at a batch the GEMM kernel
 *         does not take), TERN_ERR_ALIGNMENT, TERN_ERR_WORKSPACE, TERN_ERR_CUDA. */
TERN_API tern_status tern_gemv(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Flag of tern_gemv_ex: nothing that may still be running on the GPU when the call is made writes
 * W's codes or scales (the usual case in a decode loop over fixed weights). With it, the int8-plane
 * GEMV (batches 1-2, and Q1_0_g128 pairs of rows; always launched as a programmatic dependent of the
 * preceding kernel on the stream) and the register-decode GEMV (batches 3-4 of Q2_0_g128 and the
 * shapes the int8-plane kernel does not take; then launched as one) request W's first tiles as soon
 * as their CTAs start, while the preceding grid finishes; x, y and the workspace are only touched
 * after the preceding grid has completed. Other paths ignore the flag. */
#define TERN_GEMV_STATIC_WEIGHTS 1u

/* tern_gemv with flags (0 or TERN_GEMV_STATIC_WEIGHTS); same arguments, result and errors, plus
 * TERN_ERR_INVALID_ARG for an unknown flag bit. This entry point is an engineering addition; the
 * pages have no counterpart to it. */
TERN_API tern_status tern_gemv_ex(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y,
                                  void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);

/* Options of tern_gemv_opt. Zero-initialise and set what you need. */
typedef struct tern_gemv_opts {
  uint32_t flags;            /* 0 or TERN_GEMV_STATIC_WEIGHTS (see tern_gemv_ex) */
  uint32_t* device_status;   /* device uint32 or NULL: TERN_DEVICE_TIMEOUT is OR-ed in when a pipeline
                                wait of the call runs out; the caller zeroes it and reads it back */
  uint64_t wait_limit_ns;    /* bound on each internal pipeline wait; 0 = the default of one second */
  const int8_t* rotate_signs; /* device int8 [1024] or NULL: multiply by R x instead of x, R the block
                                Hadamard rotation of tern_hadamard_rotate with these signs (k a
                                multiple of 1024); see tern_gemv_opt */
} tern_gemv_opts;

/* tern_gemv_ex with a device status word and a wait bound. The pages ask a runtime to refuse loudly
 * what it cannot carry out rather than emit garbage ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr,
 * the runtime notes after section "블록 단위 하다마드 회전"); a GEMV whose pipeline wait runs out
 * (a producer that never delivers, a limit set too short) abandons its tiles, writes NaN to the
 * outputs of the rows it owns (batches 1-2), and reports TERN_DEVICE_TIMEOUT through device_status.
 * It never traps or hangs. Same arguments, result and errors as tern_gemv_ex otherwise, plus
 * TERN_ERR_ALIGNMENT for a device_status that is not 4-byte aligned. opts may be NULL (= all zero).
 *
 * With opts->rotate_signs the call computes y = W (R x), R = H S / 32 on every 1024-element block of
 * each row of x ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "블록 단위 하다마드 회전": the
 * weights live in the rotated basis and each layer multiplies by R x; section "처리량": the sign flip
 * and block transform precede every projection). The result equals tern_hadamard_rotate followed by
 * tern_gemv_opt on its output. Where the int8-plane kernel runs (batches 1-2 of most shapes) it
 * rotates x itself while it builds its activation fragments: one launch, no extra memory; elsewhere
 * the call rotates x into the workspace first (two launches). The workspace must then hold
 * tern_gemv_opt_workspace_bytes(W, batch, opts) bytes. Errors as above, plus TERN_ERR_INVALID_ARG
 * for k not a multiple of 1024 with rotate_signs. */
TERN_API tern_status tern_gemv_opt(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y,
                                   void* workspace, size_t workspace_bytes, const tern_gemv_opts* opts,
                                   void* stream);

/* Workspace bytes tern_gemv_opt needs for these options (tern_gemv_workspace_bytes plus room for the
 * rotated x when the rotation cannot be done inside the GEMV kernel); 0 on invalid arguments or when
 * none is needed. Host only. */
TERN_API size_t tern_gemv_opt_workspace_bytes(const tern_matrix* W, int64_t batch, const tern_gemv_opts* opts);

/* Bytes of device memory tern_gemv_noalloc keeps for its split-K scratch (per GPU, for the
 * lifetime of the process). */
#define TERN_GEMV_NOALLOC_SCRATCH_BYTES (8u << 20)

/* tern_gemv without a caller-provided workspace, for callers that cannot allocate device memory
 * or hand it to a library: e.g. plugins running inside a host runtime that owns every device
 * allocation and exposes no allocator to them, or loops where cudaMalloc / cudaFree (which can
 * synchronize the device) are not allowed. This entry point is an engineering addition; the pages
 * have no counterpart to it.
 * Same arguments and result as tern_gemv minus the workspace. The split-K scratch it needs lives in
 * a static device array of TERN_GEMV_NOALLOC_SCRATCH_BYTES that every GPU loading the library
 * holds until exit; the call allocates nothing and calls no cudaMalloc / cudaFree.
 *   - The first call on a device looks up that array's device address (cudaGetSymbolAddress) for
 *     the current device; make that first call before any stream capture.
 *   - Each call clears the scratch's arrival counters with a stream-ordered memset.
 *   - Every call on a device shares the one array: calls that overlap on the GPU (different
 *     streams without ordering between them) race and give wrong results. Order them.
 *   - A matrix / batch whose split-K workspace (tern_gemv_workspace_bytes) exceeds
 *     TERN_GEMV_NOALLOC_SCRATCH_BYTES returns TERN_ERR_WORKSPACE before any launch. Checked on the
 *     host for a 148-SM B200 (the plan depends on the SM count): batch <= 8 fits for N <= 151936 at
 *     K = 4096 and for N <= 34816 up to K = 17408, and batches of 17 or more with N % 8 == 0 need
 *     no scratch.
 * Errors: those of tern_gemv, TERN_ERR_WORKSPACE as above, TERN_ERR_CUDA if the address lookup
 * or the memset fails. */
TERN_API tern_status tern_gemv_noalloc(const tern_matrix* W, const uint16_t* x, int64_t batch, uint16_t* y,
                                       void* stream);

/* ---- prefill GEMM on tcgen05 tensor cores --------------------------------------------------- */

/* Y[m][n] = sum_k X[m][k] * s[n][k/128] * t[n][k], the prefill (prompt-processing) product of
 * "Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section "처리량" (pp512, compute-bound); packed tiles
 * are decoded to fp16 s*t (exact) in shared memory and multiplied on the 5th-generation tensor
 * cores with fp32 accumulation in tensor memory.
 *   X              device fp16 [m][k], contiguous;  Y device fp16 [m][n], contiguous
 *   device_status  device uint32 or NULL: TERN_DEVICE_TIMEOUT is OR-ed in if an internal pipeline
 *                  wait exceeds its bound (the kernel then abandons its work and exits; Y is
 *                  incomplete). The caller zeroes it.
 * Every layout: a base-3 K block of 64 weights spans at most 14 bytes and is decoded through a
 * byte -> five-field table; Q2_0_g128 and Q1_0_g128 through one masked multiply per pair of
 * weights.
 * Errors: TERN_ERR_INVALID_ARG, TERN_ERR_UNSUPPORTED (unknown layout), TERN_ERR_ALIGNMENT,
 * TERN_ERR_CUDA. */
TERN_API tern_status tern_gemm(const tern_matrix* W, const uint16_t* X, int64_t m, uint16_t* Y,
                      uint32_t* device_status, void* stream);

/* ---- transposed product (STE backward) ------------------------------------------------------ */

#define TERN_GEMV_T_MAX_BATCH 8

/* Bytes of fp32 workspace tern_gemv_t needs (0 when it needs none); a function of (layout, n, k,
 * batch) and the device's SM count. Returns 0 also for invalid arguments. */
TERN_API size_t tern_gemv_t_workspace_bytes(const tern_matrix* W, int64_t batch);

/* dx[b][k] = sum_n s[n][k/128] * t[n][k] * dy[b][n] for b < batch: the input gradient W^T dy of the
 * straight-through-estimator backward through a ternary layer ("Metal 환경에서 ... Bonsai 8B를
 * 파인튜닝", molayo1419.me, paragraph "그것을 파인튜닝하는 방법": the latents are trained through
 * the ternarized forward). fp32 accumulation, fp16 result; deterministic (row slices are summed
 * in order).
 *   dy         device fp16 [batch][n], contiguous;  dx device fp16 [batch][k], contiguous
 *   workspace  device, >= tern_gemv_t_workspace_bytes(W, batch) bytes, 16-byte aligned; may be NULL
 *              when that size is 0. Calls that share a workspace must not overlap on the GPU.
 * Errors: TERN_ERR_INVALID_ARG (batch outside 1..8, NULL pointer, bad matrix), TERN_ERR_UNSUPPORTED,
 *         TERN_ERR_ALIGNMENT (dy / dx not 2-byte aligned, workspace not 16-byte aligned, matrix
 *         alignment), TERN_ERR_WORKSPACE, TERN_ERR_CUDA. */
TERN_API tern_status tern_gemv_t(const tern_matrix* W, const uint16_t* dy, int64_t batch, uint16_t* dx,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ---- activation-side block Hadamard rotation ------------------------------------------------ */

/* y = R x for every 1024-element block of every row, R = H S / 32 ("Ternary Bonsai 2 27B ..."
 * discuss.pytorch.kr, section "블록 단위 하다마드 회전": stored weights live in the basis
 * R = H_n S / sqrt(n), n = 1024, and a layer computes W (R x); section "처리량": the sign flip and
 * the block fast Walsh-Hadamard transform precede every projection):
 *   y[b][1024 j + i] = (1/32) sum_m H[i][m] * sgn(signs[m]) * x[b][1024 j + m],
 * H the Sylvester-order Walsh-Hadamard matrix, H[i][m] = (-1)^popcount(i & m).
 *   x, y   device fp16 [batch][k], contiguous, k a positive multiple of 1024; y may equal x
 *   signs  device int8 [1024], the diagonal of S: negative entries are -1, all others +1
 * fp32 butterflies, fp16 result rounded once; stream-ordered, no allocation.
 * Errors: TERN_ERR_INVALID_ARG (NULL pointer, batch < 1, k not a positive multiple of 1024,
 *         batch * k too large), TERN_ERR_ALIGNMENT (x or y not 2-byte aligned), TERN_ERR_CUDA. */
TERN_API tern_status tern_hadamard_rotate(const uint16_t* x, int64_t batch, int64_t k, const int8_t* signs,
                                          uint16_t* y, void* stream);

/* Turns the device-side results a caller has read back into a status, so that a failure is refused
 * loudly ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, the runtime notes after section "블록 단위
 * 하다마드 회전": a runtime must reject what it cannot carry out, not emit garbage):
 *   device_status  the value of the status word given to tern_gemm / tern_gemv_opt
 *   invalid_count  the value of the counter given to tern_unpack (0 if none)
 * Returns TERN_ERR_TIMEOUT if TERN_DEVICE_TIMEOUT is set, else TERN_ERR_INVALID_CODE if
 * invalid_count > 0, else TERN_OK. Host only; makes no CUDA call. */
TERN_API tern_status tern_device_result(uint32_t device_status, int64_t invalid_count);

/* What a tern_gemv_opt call with these arguments would launch: the kernel, its work split and the
 * workspace it needs. Host only (no CUDA call beyond reading the device's SM count once); for tests,
 * logs and tuning. This entry point is an engineering addition; the pages have no counterpart to it. */
typedef struct tern_gemv_plan_info {
  int32_t kernel;          /* TERN_GEMV_KERNEL_*: the kernel that computes the product */
  int32_t launches;        /* kernel launches of the call, a rotation into the workspace included */
  int32_t k_slices;        /* K split: CTAs of a cluster (int8-plane kernel) or slices (others); 1 = none */
  int32_t ctas_per_sm;     /* CTAs per SM (int8-plane and register kernels; 0 = not fixed) */
  int32_t warps;           /* consumer warps per CTA (int8-plane and register kernels; else 0) */
  int32_t stages;          /* TMA ring stages (int8-plane kernel; else 0) */
  int32_t rotation_fused;  /* 1: opts->rotate_signs is applied inside the GEMV kernel's prologue */
  int32_t reserved;
  uint64_t workspace_bytes; /* = tern_gemv_opt_workspace_bytes */
} tern_gemv_plan_info;
#define TERN_GEMV_KERNEL_INT8_PLANES 1  /* batch 1-2: int8 mma.sync on TMA-streamed tiles */
#define TERN_GEMV_KERNEL_REGISTER 2     /* fp16 mma.sync, decode in registers from TMA windows */
#define TERN_GEMV_KERNEL_SHARED 3       /* fp16 mma.sync, decode through shared memory */
#define TERN_GEMV_KERNEL_TCGEN05 4      /* the tcgen05 GEMM kernel (batches >= 17, N % 8 == 0) */

/* Fills *out for tern_gemv_opt(W, x, batch, y, ..., opts, ...). Errors: those of tern_gemv_opt's
 * argument checks on W, batch and opts (x, y and the workspace are not looked at); out != NULL. */
TERN_API tern_status tern_gemv_plan_describe(const tern_matrix* W, int64_t batch, const tern_gemv_opts* opts,
                                             tern_gemv_plan_info* out);

/* Static description of a status code (never NULL). */
TERN_API const char* tern_status_string(tern_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
TERN_API int32_t tern_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TERN_H */
