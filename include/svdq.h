/*
 * svdq.h -- C ABI of libsvdq, the SVDQuant W4A4 linear layer (svdq_w4a4) for one
 * NVIDIA B200 (sm_100a).
 *
 * The layer replaces nn.Linear (y = x W^T + b) in a diffusion transformer and
 * computes
 *
 *     Y = X^ L1 L2 + dequant( Q4(X^) Q4(R) ) + b,      X^ = X diag(lambda)^-1
 *
 * "Hugging Face встроила Nunchaku в Diffusers ..." (iitog.ru), paragraph
 * "Суть метода": weights AND activations in 4 bits, activation outliers moved
 * into the weights (lambda), the hardest part of each weight matrix kept in a
 * 16-bit low-rank branch (L1 L2), the residual R quantized to 4 bits.  Next
 * paragraph: the runtime layer svdq_w4a4 comes in INT4 and NVFP4 variants and
 * replaces nn.Linear in attention and MLP projections.  Paragraph on hardware:
 * an unsupported GPU gets a clear error, never a wrong result.
 *
 * Conventions
 *   - Row-major everywhere.  X [M,K] bf16, W [N,K] bf16 (nn.Linear layout),
 *     Y [M,N] bf16.  bf16/fp16 values travel as uint16_t bit patterns.
 *   - Shapes: K % 256 == 0, N % 16 == 0, N >= 16, 0 <= rank <= min(K,N),
 *     rank % 16 == 0 and rank <= 128 (the GPU path).  M >= 0 (M == 0 is a
 *     no-op).  Anything else returns SVDQ_ERR_INVALID_ARG.
 *   - Formats: SVDQ_INT4_G64  -- signed 4-bit integers, groups of 64 along K,
 *                                fp16 group scales.
 *              SVDQ_NVFP4_G16 -- E2M1 codes, blocks of 16 along K, E4M3 block
 *                                scales, plus one binary32 per-tensor scale for
 *                                the weight (g_w) and one for the activation
 *                                (g_x, static, from calibration).
 *   - Packed 4-bit codes: two per byte, element 2i in bits 0..3, element 2i+1 in
 *     bits 4..7.  INT4 nibbles are two's complement.
 *   - Ownership: every pointer argument is owned by the caller.  Host functions
 *     take host pointers; svdq_forward and friends take device pointers and a
 *     stream and only enqueue work.  The library allocates no device memory
 *     (svdq_forward_noalloc's fixed scratch array, below, is static device data
 *     of the library module, not a run-time allocation).
 *   - Errors: every call returns an svdq_status; nothing aborts, throws or exits.
 *     Device-side failures (an in-kernel wait that ran past its limit) are
 *     recorded in a status word inside the caller's workspace and read with
 *     svdq_read_status.  A failed call leaves its outputs unspecified.
 *   - Devices: a layer belongs to the device that was current when it was
 *     created, and its blob must be memory of that device.  Every call that
 *     enqueues work must be made with that device current (it is a per-thread
 *     setting); otherwise the call returns SVDQ_ERR_INVALID_ARG and enqueues
 *     nothing, instead of launching kernels that would read another GPU's memory.
 *   - Thread safety: functions are re-entrant; a layer handle may be used from
 *     several threads at once; calls that share a workspace must not overlap.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* bad shape, format, pointer alignment or size */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 2, /* device is not compute capability 10.0 */
  SVDQ_ERR_OOM = 3,                /* a host allocation failed (svdq_prepare/pack) */
  SVDQ_ERR_CUDA = 4,               /* a CUDA runtime/driver call failed */
  SVDQ_ERR_NUMERIC = 5,            /* non-finite input to svdq_prepare */
  SVDQ_ERR_TIMEOUT = 6,            /* an in-kernel wait ran past its limit */
  SVDQ_ERR_BOUNDS = 7              /* debug build only: a kernel computed a global address outside its
                                      buffer; the access was skipped (see svdq_debug_build) */
} svdq_status;

typedef enum svdq_format { SVDQ_INT4_G64 = 1, SVDQ_NVFP4_G16 = 2 } svdq_format;

/* Human-readable name of a status code (static string, never NULL). */
const char* svdq_status_string(int status);

/* 1 in the library's bounds-checked debug variant (libsvdq_debug.so, built with
 * -DSVDQ_DEBUG_BOUNDS), 0 in the release library.  In the debug variant every
 * global access that a kernel addresses itself is checked against its buffer;
 * one that would leave it records SVDQ_ERR_BOUNDS in the status word and is
 * skipped (nothing traps).  Same entry points and results otherwise, slower. */
int svdq_debug_build(void);

/* ABI version of this header (increments on incompatible change).
 * 2: the svdq workspace control block holds the per-call g_x and the first
 *    pass's maxima; the awq blob's scale rows are padded to 8 entries, its codes
 *    are offset binary and it ends in a status word; the W8A8 layer. */
#define SVDQ_ABI_VERSION 2
int svdq_abi_version(void);

/* ------------------------------------------------------------------------ */
/* Prepared weights in canonical (format-defined) layout, host memory.       */
/* ------------------------------------------------------------------------ */
typedef struct svdq_canonical {
  int64_t N, K;      /* output / input features */
  int32_t rank;      /* low-rank branch width r */
  int32_t fmt;       /* svdq_format */
  float alpha;       /* smoothing migration strength used */
  float g_x;         /* NVFP4 activation per-tensor scale (1 for INT4); 0 selects the
                        dynamic scale: computed per call from the input's largest |x^| */
  float g_w;         /* NVFP4 weight per-tensor scale (1 for INT4) */
  float reserved;
  float* lambda;     /* [K]  smoothing factors, binary32 */
  float* inv_lambda; /* [K]  1/lambda rounded to binary32 */
  uint16_t* L1;      /* [K, rank] bf16 */
  uint16_t* L2;      /* [rank, N] bf16 */
  uint8_t* wcodes;   /* [N, K/2] packed 4-bit residual codes */
  void* wscales;     /* INT4: uint16_t fp16 [N, K/64]; NVFP4: uint8_t E4M3 [N, K/16] */
  uint16_t* bias;    /* [N] bf16 (zeros when the layer has no bias) */
} svdq_canonical;

/* Byte sizes of the seven canonical arrays, in the struct's order:
 * sizes[0] lambda, [1] inv_lambda, [2] L1, [3] L2, [4] wcodes, [5] wscales, [6] bias. */
svdq_status svdq_canonical_sizes(int64_t N, int64_t K, int rank, int fmt, size_t sizes[7]);

/* Offline preparation of one layer, on the host ("Суть метода" paragraph):
 *   lambda_j = amax_x[j]^alpha / amax_w[j]^(1-alpha)  (1 if either is 0),
 *   W^ = W diag(lambda),  rank-r truncated SVD W^ ~ U S V^T,
 *   L1 = V_r S_r^(1/2) and L2 = S_r^(1/2) U_r^T rounded to bf16,
 *   R = W^ - (L1 L2)^T, group-quantized to 4 bits in `fmt`.
 * act_absmax[K] is the per-input-channel max |x| seen on calibration inputs
 * (the layer's own input: no calibration dataset is needed).  W is [N,K] bf16,
 * bias [N] bf16 or NULL.  `out` must have N, K, rank, fmt set and every array
 * pointer pointing at caller memory of svdq_canonical_sizes bytes; the call
 * fills the arrays and alpha/g_x/g_w.  Synchronous; uses all host cores.  The
 * truncated SVD is a randomized subspace iteration in binary64.
 * Errors: INVALID_ARG (shape/pointers), NUMERIC (non-finite W or act_absmax),
 * OOM (host scratch). */
svdq_status svdq_prepare(const uint16_t* W, const uint16_t* bias, const float* act_absmax, float alpha,
                         svdq_canonical* out);

/* ------------------------------------------------------------------------ */
/* Device layout of a prepared layer ("packed blob").                        */
/* ------------------------------------------------------------------------ */
/* Size in bytes of the packed blob for a layer shape. */
svdq_status svdq_packed_size(int64_t N, int64_t K, int rank, int fmt, size_t* bytes);

/* Re-lay canonical weights into the blob the kernels read (a pure permutation
 * plus exact re-encodings; no rounding).  `blob` is host memory of
 * svdq_packed_size bytes; copy it to the device (256-byte aligned) and pass the
 * device pointer to svdq_layer_create.  Layout, each region 1024-byte aligned:
 *   inv_lambda f32 [K] | L1^T bf16 [rank, K] | L2^T bf16 [N, rank] (NVFP4: times
 *   1/(g_x g_w), an exact power of two) | bias f32 [N] |
 *   wcodes: NVFP4 -> the packed E2M1 codes u8 [N, K/2]; INT4 -> one byte per
 *   code, u8 [N, K], holding the FP8 E4M3 encoding of the code's integer value
 *   (exact for every integer in [-8, 7]; the tensor cores of CC 10.0 have no
 *   4-bit integer kind, so INT4 weights are held at one byte per code) |
 *   wscales: NVFP4 -> E4M3 in 192-row tiles of the tensor-core scale-factor
 *   layout, INT4 -> the fp16 group scales widened exactly to f32, [K/64, N]. */
svdq_status svdq_pack(const svdq_canonical* c, void* blob, size_t blob_bytes);

/* ------------------------------------------------------------------------ */
/* Device side.                                                              */
/* ------------------------------------------------------------------------ */
/* SVDQ_OK iff `device` is compute capability 10.0 (sm_100a build target).
 * Setting the environment variable SVDQ_FAULT=bad_arch makes it fail, to
 * exercise the capability error path without such a device. */
svdq_status svdq_device_check(int device);

typedef struct svdq_layer svdq_layer; /* opaque host-side handle */

/* Bind a device-resident packed blob (from svdq_pack) to a host handle.  No
 * device memory is allocated; the blob must outlive the handle.  Fails with
 * UNSUPPORTED_DEVICE on a device other than CC 10.0 (current device), and with
 * INVALID_ARG when the CUDA runtime reports the blob as host memory or as memory
 * of another device.
 * NVFP4: g_w and g_x must be powers of two, or g_x = 0 for the dynamic
 * activation scale (the blob must then have been packed with g_x = 0 too: its
 * L2 carries 1/g_w only).  A dynamic layer's svdq_quantize_act runs a first pass
 * over X for its largest |x^| = |fl32(x * inv_lambda)| (per-CTA maxima in the
 * workspace), takes g_x = the smallest power of two >= that / (6 * 448) (1 for
 * an all-zero X), quantizes with it, stores t / g_x (exact) as the workspace's
 * t, and leaves g_x in word 1 of the control block for svdq_gemm. */
svdq_status svdq_layer_create(const void* dev_blob, size_t blob_bytes, int64_t N, int64_t K, int rank, int fmt,
                              float g_x, float g_w, svdq_layer** out);
/* Frees the host handle only (never the blob); NULL is a no-op. */
void svdq_layer_destroy(svdq_layer* layer);

/* Workspace for M tokens: quantized activations, low-rank t and a status word.
 * layout: offsets/sizes[0] act codes (NVFP4: packed E2M1 u8 [M, K/2]; INT4: one
 * FP8 E4M3 byte per code holding its integer value, u8 [M, K]); [1] act scales
 * (NVFP4: E4M3 in the tensor-core scale-factor layout of 128-row tiles; INT4:
 * fp16 [K/64, M'], M' = M rounded up to a multiple of 128, columns >= M unused);
 * [2] t bf16 [M, rank] (t / g_x for a dynamic-scale layer); [3] status word
 * int32, the first word of a control block that also holds the per-call g_x of a
 * dynamic-scale layer (word 1, float), the quantizer's split-K counters and the
 * first pass's per-CTA maxima.  The total size also covers the quantizer's fp32
 * partial sums of t.  Both calls are host-only; INVALID_ARG for a NULL argument
 * or M < 0.
 * Every call below that takes (ws, ws_bytes) checks first that ws (device
 * memory) is non-NULL, 256-byte aligned, ws_bytes >= svdq_workspace_size(M) and
 * 0 <= M <= 2^30, and returns SVDQ_ERR_INVALID_ARG with nothing enqueued
 * otherwise.  The workspace is caller-owned.  Region offsets depend on M, so a
 * buffer sized for M serves a call with M' < M only after svdq_workspace_init
 * for M' (the control block then sits at M''s offset). */
svdq_status svdq_workspace_size(const svdq_layer* layer, int64_t M, size_t* bytes);
svdq_status svdq_workspace_layout(const svdq_layer* layer, int64_t M, size_t offsets[4], size_t sizes[4]);

/* Zero the workspace control block: the status word and the quantizer's split-K
 * counters (enqueued on `stream`, a cudaStream_t).  Required once before the
 * first svdq_forward on a fresh workspace; the kernels keep the counters at zero
 * between calls, and the status is sticky until the next init. */
svdq_status svdq_workspace_init(const svdq_layer* layer, int64_t M, void* ws, size_t ws_bytes, void* stream);

/* Y[M,N] = layer(X[M,K]).  X, Y, ws are device pointers (16-byte aligned),
 * `stream` a cudaStream_t.  Enqueues the activation-quantize kernel, then the
 * W4A4 GEMM with its dequantize / low-rank / bias epilogue.  Asynchronous:
 * returns launch errors only; device-side errors land in the status word. */
svdq_status svdq_forward(const svdq_layer* layer, const void* X, int64_t M, void* Y, void* ws, size_t ws_bytes,
                         void* stream);

/* The two halves of svdq_forward, for parity checks of the intermediate
 * results: svdq_quantize_act fills workspace regions 0..2 from X;
 * svdq_gemm reads them and writes Y. */
svdq_status svdq_quantize_act(const svdq_layer* layer, const void* X, int64_t M, void* ws, size_t ws_bytes,
                              void* stream);
svdq_status svdq_gemm(const svdq_layer* layer, int64_t M, void* Y, void* ws, size_t ws_bytes, void* stream);

/* INT4 only, for parity of the integer path: after svdq_quantize_act, write the
 * per-group int32 accumulators acc[g, m, n] = sum_{k in group g} qx[m,k] qw[n,k]
 * (device int32 [K/64, M, N]) using the same GEMM main loop. */
svdq_status svdq_int4_group_acc(const svdq_layer* layer, int64_t M, void* ws, size_t ws_bytes, int32_t* acc,
                                void* stream);

/* ------------------------------------------------------------------------ */
/* Cross-layer fusion of a transformer block's MLP pair: up -> GELU -> down. */
/* ------------------------------------------------------------------------ */
/* "Hugging Face встроила Nunchaku в Diffusers ..." (paragraph on Nunchaku
 * Lite): the engine's speed comes from fused, model-specific kernels.  Here the
 * up-projection's GEMM epilogue computes, per output element,
 *     h = bf16(y_up),   x' = bf16(GELU(h)),   GELU(h) = h/2 (1 + erf(h/sqrt 2)),
 * evaluated in binary32 as h/2 erfc(-h/sqrt 2) (no cancellation for h < 0),
 * and quantizes x' as the down-projection's input exactly as svdq_quantize_act
 * would (x^' = f32(x') inv_lambda', E4M3 block scales and E2M1 codes under the
 * down layer's static g_x', t' = bf16(bf16(x^') L1')), writing codes, scales and
 * t' into the down layer's workspace; y_up itself is never written.
 * Requirements (else SVDQ_ERR_INVALID_ARG): both layers NVFP4, up.N == down.K,
 * up.N a multiple of 192, the down layer's activation scale static (g_x != 0)
 * and its rank <= 32, both layers on the current device. */
svdq_status svdq_mlp_fusable(const svdq_layer* up, const svdq_layer* down);

/* After svdq_quantize_act(up, X, M, ws_up, ...): the fused up-projection GEMM.
 * ws_up / ws_dn are the two layers' workspaces for M tokens (device, 256-byte
 * aligned; ws_dn initialised once with svdq_workspace_init; M <= 32768, else
 * SVDQ_ERR_INVALID_ARG); H, if not NULL, is
 * a device bf16 [M, up.N] array (16-byte aligned) that receives x' (a parity
 * export; costs one extra write).  Then svdq_gemm(down, M, Y, ws_dn, ...) gives
 * the block's MLP output.  Asynchronous on `stream`; device-side errors land in
 * ws_up's status word. */
svdq_status svdq_gemm_gelu_quantize(const svdq_layer* up, const svdq_layer* down, int64_t M, void* ws_up,
                                    size_t ws_up_bytes, void* ws_dn, size_t ws_dn_bytes, void* H, void* stream);

/* Y[M, down.N] = down(GELU(up(X))): svdq_quantize_act(up), svdq_gemm_gelu_quantize,
 * svdq_gemm(down), all on `stream`.  The pair and M <= 32768 are checked before
 * anything is enqueued (SVDQ_ERR_INVALID_ARG). */
svdq_status svdq_mlp_forward(const svdq_layer* up, const svdq_layer* down, const void* X, int64_t M, void* Y,
                             void* ws_up, size_t ws_up_bytes, void* ws_dn, size_t ws_dn_bytes, void* stream);

/* Synchronously read the workspace status word (0 = fine, else an svdq_status
 * recorded by a kernel).  With ws == NULL and ws_bytes == 0 it reads instead the
 * status word of the last svdq_forward_noalloc call for M tokens on the current
 * device (which must be the layer's); that word is zeroed by the next such
 * call, so read it after the call's work has finished and before the next one. */
svdq_status svdq_read_status(const svdq_layer* layer, int64_t M, const void* ws, size_t ws_bytes,
                             int* device_status);

/* svdq_forward for callers that cannot allocate device memory: for example an
 * extension running inside a host framework that owns every device allocation
 * and forbids cudaMalloc, or a service that must not allocate after start-up.
 * (No counterpart in the method's description; it is a deployment variant.)
 * X, Y are device pointers (16-byte aligned), `stream` a cudaStream_t, and the
 * current device must be the layer's.  Instead of a caller workspace, the
 * quantized activations, t and the status word live in one library-owned
 * device array of 32 MiB, which exists once per GPU that loads the library and
 * stays allocated until the process exits.  Problems whose workspace
 * (svdq_workspace_size) exceeds 32 MiB return SVDQ_ERR_INVALID_ARG (e.g. at
 * K = 12288, rank 32: up to 4480 tokens in NVFP4, 2458 in INT4).  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress), so make that
 * first call before any stream capture.  Each call zeroes the control block;
 * the array keeps the last call's contents otherwise.  All calls share the
 * array: calls whose GPU work can overlap (other streams, other threads) race
 * and must be serialized by the caller.  Allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine); asynchronous like svdq_forward.
 * Device-side failures (an in-kernel wait past its limit) are read with
 * svdq_read_status(layer, M, NULL, 0, &status).  A failed address lookup is
 * not cached: the next call tries again.  M > 2^30 returns INVALID_ARG. */
svdq_status svdq_forward_noalloc(const svdq_layer* layer, const void* X, int64_t M, void* Y, void* stream);

/* Upper bound, in SM clock cycles, on every in-kernel wait of later launches
 * (default 2^31, about a second).  A wait that runs past it makes the kernel
 * record SVDQ_ERR_TIMEOUT, drain its own in-flight copies, free its tensor
 * memory and return.  0 restores the default. */
svdq_status svdq_set_wait_limit(uint64_t cycles);

/* ------------------------------------------------------------------------ */
/* awq_w4a16: 4-bit weights, 16-bit activations.                            */
/* ------------------------------------------------------------------------ */
/* The second runtime layer of "Hugging Face встроила Nunchaku в Diffusers ..."
 * (paragraph on Nunchaku Lite): precision-sensitive normalization and
 * modulation layers (adaLN in FLUX) keep bf16 activations and store only the
 * weights in 4 bits, prepared activation-aware (AWQ).  The pages name it and
 * give no arithmetic; this library computes
 *
 *     y = (f32(x) * inv_s) . dequant( Q4(W diag(s)) )^T + b
 *
 * with s_j = mean|x_j|^alpha (1 where the mean is 0), alpha the first point of
 * the grid 0, 0.05, ..., 1 with the smallest squared output error on the
 * calibration input, and Q4 the INT4 group-64 quantizer of the svdq_w4a4
 * residual (symmetric, fp16 scale amax/7, round-half-even codes clamped to
 * [-8, 7]).  Shapes: K % 64 == 0, 64 <= K <= 12288, N >= 1; M >= 0. */
typedef struct svdq_awq_canonical {
  int64_t N, K;
  float alpha;       /* the grid point chosen */
  float reserved;
  float* s;          /* [K] per-input-channel scale, binary32 */
  float* inv_s;      /* [K] 1/s rounded to binary32 */
  uint8_t* wcodes;   /* [N, K/2] packed INT4 codes of W diag(s) */
  uint16_t* wscales; /* [N, K/64] fp16 group scales */
  uint16_t* bias;    /* [N] bf16 (zeros when the layer has no bias) */
} svdq_awq_canonical;

/* Byte sizes of the five arrays in struct order: s, inv_s, wcodes, wscales, bias. */
svdq_status svdq_awq_canonical_sizes(int64_t N, int64_t K, size_t sizes[5]);

/* Host, synchronous, all cores.  W [N,K] bf16, bias [N] bf16 or NULL, X_calib
 * [M_calib, K] bf16 (the layer's own inputs; M_calib >= 1).  `out` must have N
 * and K set and its arrays point at caller memory of svdq_awq_canonical_sizes
 * bytes.  Errors: INVALID_ARG (shape, pointers), NUMERIC (non-finite W or X). */
svdq_status svdq_awq_prepare(const uint16_t* W, const uint16_t* bias, const uint16_t* X_calib, int64_t M_calib,
                             svdq_awq_canonical* out);

/* Device layout ("awq blob"), each region 1024-byte aligned: inv_s f32 [K] |
 * bias f32 [N] | wscales fp16 [N, G'] with G' = K/64 rounded up to a multiple of
 * 8 (padding entries zero; a run of rows is then a whole number of 16-byte
 * units) | wcodes u8 [N, K/2] (the canonical packing with every nibble in
 * offset binary, n + 8 = n ^ 8, kept at 4 bits per weight: the layer is a
 * weight-streaming GEMV at the batch sizes of modulation layers) | status int32 (zero in a packed blob; the kernel writes a nonzero
 * code there when one of its bounded waits expires). */
svdq_status svdq_awq_packed_size(int64_t N, int64_t K, size_t* bytes);
svdq_status svdq_awq_pack(const svdq_awq_canonical* c, void* blob, size_t blob_bytes);

typedef struct svdq_awq_layer svdq_awq_layer; /* opaque host-side handle */

/* Bind a device-resident awq blob (256-byte aligned) to a handle; allocates no
 * device memory; UNSUPPORTED_DEVICE on a device other than CC 10.0, INVALID_ARG
 * for a blob in host memory or on another device. */
svdq_status svdq_awq_layer_create(const void* dev_blob, size_t blob_bytes, int64_t N, int64_t K,
                                  svdq_awq_layer** out);
/* Frees the host handle only (never the blob); NULL is a no-op. */
void svdq_awq_layer_destroy(svdq_awq_layer* layer);

/* Synchronous read of the blob's status word: 0, or SVDQ_ERR_TIMEOUT after a
 * kernel gave up waiting for its weight copies (the outputs of that call are
 * then incomplete).  The word is sticky until the blob is re-uploaded. */
svdq_status svdq_awq_read_status(const svdq_awq_layer* layer, int* device_status);

/* Y[M,N] = layer(X[M,K]), X and Y device pointers (16-byte aligned), `stream`
 * a cudaStream_t; asynchronous, returns launch errors only.  Token rows are
 * processed two at a time: the weights are streamed once per pair of rows, so
 * the kernel is meant for the small M of modulation layers (the batch size);
 * it is correct for any M. */
svdq_status svdq_awq_forward(const svdq_awq_layer* layer, const void* X, int64_t M, void* Y, void* stream);

/* ------------------------------------------------------------------------ */
/* INT8 tensorwise W8A8 layer: the 8-bit variant that "SVDQuant ускоряет      */
/* Krea 2 вдвое ..." (section "Решение: INT8 и W4A4") compares with W4A4.     */
/*   s = fl32(max|v| / 127) per tensor, q = clamp(rne(v * fl32(1/s)), +-127); */
/*   the weight's s_w is fixed at preparation, the activation's s_x is taken   */
/*   from each input (a first pass for max|x|);                              */
/*   Y = bf16(s_x s_w (qx . qw^T) + b).  No smoothing, no low-rank branch.     */
/* Shapes: N >= 8 and N % 8 == 0, K >= 128 and K % 128 == 0.                  */
/* ------------------------------------------------------------------------ */
typedef struct svdq_w8a8_layer svdq_w8a8_layer; /* opaque host-side handle */

/* Host, synchronous.  W [N,K] bf16 -> wcodes int8 [N,K] (row-major) and *s_w.
 * Errors: INVALID_ARG (shape, pointers), NUMERIC (non-finite W). */
svdq_status svdq_w8a8_prepare(const uint16_t* W, int64_t N, int64_t K, int8_t* wcodes, float* s_w);

/* Device layout ("w8a8 blob"), regions 1024-byte aligned: bias f32 [N] | wcodes
 * int8 [N, K] row-major.  bias bf16 [N] or NULL (zeros). */
svdq_status svdq_w8a8_packed_size(int64_t N, int64_t K, size_t* bytes);
svdq_status svdq_w8a8_pack(int64_t N, int64_t K, const int8_t* wcodes, const uint16_t* bias, void* blob,
                           size_t blob_bytes);

/* Bind a device-resident w8a8 blob (256-byte aligned) to a handle with the
 * weight scale s_w (finite, >= 0); allocates no device memory.
 * UNSUPPORTED_DEVICE on a device other than CC 10.0, INVALID_ARG for a blob in
 * host memory or on another device. */
svdq_status svdq_w8a8_layer_create(const void* dev_blob, size_t blob_bytes, int64_t N, int64_t K, float s_w,
                                   svdq_w8a8_layer** out);
/* Frees the host handle only (never the blob); NULL is a no-op. */
void svdq_w8a8_layer_destroy(svdq_w8a8_layer* layer);

/* Workspace for M tokens (caller device memory, 256-byte aligned): activation
 * codes int8 [M, K] at offset 0 | at the next 1024-byte boundary a control
 * block: int32 status, float s_x of the last quantized input, 8 bytes unused,
 * then the first pass's per-CTA maxima (1024 floats).  Needs no initialisation. */
svdq_status svdq_w8a8_workspace_size(const svdq_w8a8_layer* layer, int64_t M, size_t* bytes);

/* Asynchronous on `stream`; launch errors only.  X [M,K] bf16 and Y [M,N] bf16
 * are device pointers (16-byte aligned).  quantize_act runs the max|x| pass and
 * the quantizer; gemm the int8 tensor-core product with the scale and bias. */
svdq_status svdq_w8a8_quantize_act(const svdq_w8a8_layer* layer, const void* X, int64_t M, void* ws,
                                   size_t ws_bytes, void* stream);
svdq_status svdq_w8a8_gemm(const svdq_w8a8_layer* layer, int64_t M, void* Y, void* ws, size_t ws_bytes,
                           void* stream);
svdq_status svdq_w8a8_forward(const svdq_w8a8_layer* layer, const void* X, int64_t M, void* Y, void* ws,
                              size_t ws_bytes, void* stream);
/* Synchronous read of the workspace status word (SVDQ_ERR_TIMEOUT after a wait
 * ran past its limit). */
svdq_status svdq_w8a8_read_status(const svdq_w8a8_layer* layer, int64_t M, const void* ws, size_t ws_bytes,
                                  int* device_status);

#ifdef __cplusplus
}
#endif
#endif /* SVDQ_H_ */
