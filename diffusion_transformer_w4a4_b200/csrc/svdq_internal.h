// Internal declarations shared by the host half and the kernels of libsvdq.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstddef>
#include <cstdint>

#include "svdq.h"

namespace svdq {

// Tile geometry of the kernels (compile-time contract between pack, the
// activation quantizer and the GEMMs).
constexpr int kKStage = 256;       // K elements per pipeline stage / per quantizer chunk
constexpr int kGemmBM = 128;       // GEMM tile rows (tokens), = tcgen05 M
constexpr int kNvfp4BN = 192;      // NVFP4 GEMM tile columns (output features)
constexpr int kInt4BN = 128;       // INT4 GEMM tile columns
constexpr int kSfAtomRows = 128;   // rows per tensor-core scale-factor atom
constexpr int kSfAtomBytes = 512;  // 128 rows x 4 blocks of 16
constexpr int kMaxRank = 128;
constexpr int kQRows = 128;   // activation quantizer: token rows per CTA (= tcgen05 M)
constexpr int kQChunk = 256;  // activation quantizer: K columns per chunk
constexpr int kQSmCount = 148;  // SM count the quantizer's K-split is sized for (fixed, so sizes are device-free)
constexpr size_t kAlign = 1024;
constexpr int kAmaxSlots = 1024;  // per-CTA maxima of the dynamic activation-scale pass
// The fused MLP kernel keeps one counter per 32-row group in the down layer's
// first-pass slots (4 per 128-row tile), which bounds its token count.
constexpr int64_t kFusedMlpMaxM = 32 * (int64_t)kAmaxSlots;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with programmatic dependent launch allowed: the kernel lets the next
// one on the stream be scheduled early (griddepcontrol.launch_dependents) and
// waits (griddepcontrol.wait) before it touches what earlier work on the stream
// produced or still reads, so its prologue (barriers, tensor memory, tensor-map
// fetches) overlaps the tail of the kernel before it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// NVTX range around the host-side enqueue of a kernel group ("svdq/quantize",
// "svdq/gemm", ...), so a timeline tool can attribute the launches; without a
// tool attached the calls do nothing.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Byte offset of the E4M3 scale of (row, block) in a scale-factor atom tiling
// whose row tiles are `tile_rows` rows (128 for activations, 192 for weights)
// and each tile is padded to a multiple of 128 rows:
//   tile t = row / tile_rows, atom a = (row % tile_rows) / 128 inside the tile,
//   k-atom = block / 4, within the atom: (row%32)*16 + ((row/32)%4)*4 + block%4.
inline __host__ __device__ size_t sf_offset(int64_t row, int64_t block, int64_t katoms, int tile_rows) {
  const int64_t tile = row / tile_rows;
  const int64_t rin = row % tile_rows;
  const int atoms_per_tile = (tile_rows + kSfAtomRows - 1) / kSfAtomRows;
  const int64_t a = rin / kSfAtomRows;
  const int64_t ra = rin % kSfAtomRows;
  return (size_t)(((tile * katoms + block / 4) * atoms_per_tile + a) * kSfAtomBytes + (ra % 32) * 16 +
                  ((ra / 32) % 4) * 4 + (block % 4));
}

struct Blob {  // offsets (bytes) of the packed-weight regions
  size_t inv_lambda, L1t, L2t, bias, wcodes, wscales, total;
};
Blob blob_layout(int64_t N, int64_t K, int rank, int fmt);

// INT4 activation scales are fp16 [K/64, int4_scale_ld(M)]: each group's row is
// padded to whole 128-token tiles so the GEMM can stage it with TMA.
inline int64_t int4_scale_ld(int64_t M) { return (M + kQRows - 1) / kQRows * kQRows; }

// Number of K slices the activation quantizer splits each 128-row block into,
// so that about one CTA per SM is in flight; partial low-rank sums of the
// slices are reduced in a fixed order.
inline int quant_slices(int64_t M, int64_t K) {
  const int64_t rb = (M + kQRows - 1) / kQRows;
  const int64_t nch = K / kQChunk;
  int64_t ns = kQSmCount / (rb > 0 ? rb : 1);
  if (ns < 1) ns = 1;
  if (ns > nch) ns = nch;
  return (int)ns;
}

struct Workspace {
  // status: control block = [0] status word, [4] the per-call activation scale
  // g_x (dynamic layers), [16, ...) split-K counters, then at `amax` the
  // kAmaxSlots per-CTA maxima of the dynamic-scale pass
  size_t codes, scales, t, status, amax, tpart, total;
  size_t codes_bytes, scales_bytes, t_bytes, ctrl_bytes, tpart_bytes;
  int nslices;
};
Workspace workspace_layout(int64_t N, int64_t K, int rank, int fmt, int64_t M);

struct LowRankChunks {
  int n;
  int off[4];
  int width[4];  // 64, 32 or 16 bf16 columns
};
LowRankChunks lowrank_chunks(int rank);

}  // namespace svdq

// The opaque layer handle.
struct svdq_layer {
  int64_t N, K;
  int rank, fmt;
  float g_x, g_w;  // g_x == 0: NVFP4 activation scale computed per call (dynamic)
  bool dyn_gx;
  int device;
  const uint8_t* blob;
  svdq::Blob off;
  const float* inv_lambda;
  const uint16_t* L1t;  // [rank, K]
  const uint16_t* L2t;  // [N, rank]
  const float* bias;    // [N]
  const uint8_t* wcodes;
  const uint8_t* wscales;
  CUtensorMap map_w;         // weight codes
  CUtensorMap map_l1;        // L1^T, box {64, rank}, 128B swizzle (quantizer)
  CUtensorMap map_l2[3];     // L2^T chunks of width 64/32/16
};

namespace svdq {

namespace host {
int prepare(const uint16_t* W, const uint16_t* bias, const float* act_absmax, float alpha, svdq_canonical* c);
int awq_prepare(const uint16_t* W, const uint16_t* bias, const uint16_t* X, int64_t Mc, svdq_awq_canonical* c);
uint16_t f32_to_bf16(float f);
float bf16_to_f32(uint16_t h);
float f16_to_f32(uint16_t h);
uint8_t f32_to_e4m3_sat(float f);
uint8_t int_to_e4m3(int v);
}  // namespace host

// Tensor-map encoding through the driver entry point (no link-time libcuda).
int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

unsigned long long wait_limit_cycles();
int device_sm_count(int dev);  // multiprocessor count, cached per device (148 if the query fails)
// SVDQ_OK iff `dev` (a layer's device) is the calling thread's current device,
// INVALID_ARG otherwise (kernels launched there would read another GPU's memory),
// SVDQ_ERR_CUDA if the query fails.
int require_current_device(int dev);
// INVALID_ARG when the runtime reports `p` as host memory or as memory of a
// device other than `dev`; SVDQ_OK otherwise (managed memory, or a pointer the
// runtime cannot classify, is left to the caller).
int check_blob_pointer(const void* p, int dev);

// Kernel launchers (return svdq_status).
// dynamic activation scale: grid of the amax pass (its CTA count is the number
// of valid slots) and its launch
void act_amax_grid(int64_t M, int64_t K, int* gx, int* gy);
int launch_act_amax(const svdq_layer* L, const void* X, int64_t M, uint8_t* ws, const Workspace& w,
                    cudaStream_t stream);
// the same pass for any bf16 [M, K] tensor, with (inv_lambda) or without smoothing
int launch_act_amax_raw(const void* X, int64_t M, int64_t K, const float* inv_lambda, float* slots,
                        cudaStream_t stream);
int launch_quantize(const svdq_layer* L, const void* X, int64_t M, uint8_t* ws, const Workspace& w,
                    cudaStream_t stream);
int launch_gemm_nvfp4(const svdq_layer* L, int64_t M, void* Y, uint8_t* ws, const Workspace& w,
                      cudaStream_t stream);
int launch_gemm_int4(const svdq_layer* L, int64_t M, void* Y, uint8_t* ws, const Workspace& w, int32_t* acc_dbg,
                     cudaStream_t stream);
// MLP pair fusion: the up layer's GEMM whose epilogue writes the down layer's
// quantized input (GELU between them) into the down layer's workspace
int fused_mlp_supported(const svdq_layer* up, const svdq_layer* down);
int launch_gemm_gelu_quant(const svdq_layer* up, const svdq_layer* down, int64_t M, uint8_t* ws_up,
                           const Workspace& w_up, uint8_t* ws_dn, const Workspace& w_dn, void* H, cudaStream_t stream);
// status word of the last svdq_forward_noalloc on the current device (M tokens)
int read_status_noalloc(const svdq_layer* L, int64_t M, int* device_status);

}  // namespace svdq
