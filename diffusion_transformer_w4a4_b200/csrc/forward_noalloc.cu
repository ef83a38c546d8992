// svdq_forward_noalloc: the layer forward for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand the library a workspace: code running
// inside a framework or plugin that owns every device allocation and forbids
// cudaMalloc from extensions, or a host that must not allocate once set up.
// This entry point runs the same two kernels as svdq_forward, but their scratch
// (quantized activation codes, scales, the low-rank t and the status word) lives
// in one fixed-size array in device global memory that this file declares.  The
// array exists once per GPU that loads the library and stays allocated until the
// process exits.  Every call shares it, so calls whose GPU work overlaps (on
// different streams, or from different threads) race on it and must be
// serialized by the caller.
#include <mutex>

#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Host code may not use g_noalloc_scratch as a pointer: in host code the name
// stands for a host-side shadow, not a device address.  The device address is
// looked up once per device, with that device current.
struct ScratchSlot {
  std::once_flag once;
  uint8_t* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
ScratchSlot g_slots[64];

uint8_t* scratch_on(int dev, cudaError_t* err) {
  ScratchSlot& s = g_slots[dev];
  std::call_once(s.once, [&s] {
    void* p = nullptr;
    s.err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    s.ptr = (s.err == cudaSuccess) ? (uint8_t*)p : nullptr;
  });
  *err = s.err;
  return s.ptr;
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" svdq_status svdq_forward_noalloc(const svdq_layer* L, const void* X, int64_t M, void* Y, void* stream) {
  if (!L || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || ((uintptr_t)X & 15) || ((uintptr_t)Y & 15)) return SVDQ_ERR_INVALID_ARG;
  const Workspace w = workspace_layout(L->N, L->K, L->rank, L->fmt, M);
  if (w.total > kNoAllocScratchBytes) return SVDQ_ERR_INVALID_ARG;  // problem too large for the fixed scratch
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SVDQ_ERR_CUDA;
  if (dev != L->device) return SVDQ_ERR_INVALID_ARG;
  cudaError_t e;
  uint8_t* ws = scratch_on(dev, &e);
  if (e != cudaSuccess || !ws) return SVDQ_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // the control block (status word, split-K counters) must start at zero; the
  // rest is fully rewritten by the kernels
  if (cudaMemsetAsync(ws + w.status, 0, w.ctrl_bytes, s) != cudaSuccess) return SVDQ_ERR_CUDA;
  int st = L->dyn_gx ? launch_act_amax(L, X, M, ws, w, s) : SVDQ_OK;
  if (st != SVDQ_OK) return (svdq_status)st;
  st = launch_quantize(L, X, M, ws, w, s);
  if (st != SVDQ_OK) return (svdq_status)st;
  if (L->fmt == SVDQ_NVFP4_G16) return (svdq_status)launch_gemm_nvfp4(L, M, Y, ws, w, s);
  return (svdq_status)launch_gemm_int4(L, M, Y, ws, w, nullptr, s);
}
