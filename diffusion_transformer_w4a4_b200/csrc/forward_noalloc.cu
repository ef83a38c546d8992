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
#include <atomic>
#include <mutex>

#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Host code may not use g_noalloc_scratch as a pointer: in host code the name
// stands for a host-side shadow, not a device address.  The device address is
// looked up per device, with that device current, and cached only once the
// lookup has succeeded: a failed lookup (for example one attempted during a
// stream capture) is retried by the next call instead of disabling the device.
struct ScratchSlot {
  std::mutex mu;
  std::atomic<uint8_t*> ptr{nullptr};
};
ScratchSlot g_slots[64];

uint8_t* scratch_on(int dev, cudaError_t* err) {
  ScratchSlot& s = g_slots[dev];
  *err = cudaSuccess;
  if (uint8_t* p = s.ptr.load(std::memory_order_acquire)) return p;
  std::lock_guard<std::mutex> lock(s.mu);
  if (uint8_t* p = s.ptr.load(std::memory_order_acquire)) return p;
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (*err != cudaSuccess || !p) {
    cudaGetLastError();  // leave no sticky launch error behind
    if (*err == cudaSuccess) *err = cudaErrorInvalidSymbol;
    return nullptr;
  }
  s.ptr.store((uint8_t*)p, std::memory_order_release);
  return (uint8_t*)p;
}

// The workspace layout of a call, or INVALID_ARG when the problem does not fit
// the fixed scratch (the same M bound as every workspace entry point first, so
// the layout's size arithmetic cannot wrap).
int noalloc_layout(const svdq_layer* L, int64_t M, Workspace* w) {
  if (!L || M < 0 || M > ((int64_t)1 << 30)) return SVDQ_ERR_INVALID_ARG;
  *w = workspace_layout(L->N, L->K, L->rank, L->fmt, M);
  if (w->total > kNoAllocScratchBytes) return SVDQ_ERR_INVALID_ARG;  // too large for the fixed scratch
  return SVDQ_OK;
}

int current_layer_device(const svdq_layer* L, int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= 64) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return *dev == L->device ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
}

}  // namespace

// Status word of the last svdq_forward_noalloc call on the current device for a
// problem of M tokens (svdq_read_status with a null workspace lands here).
int read_status_noalloc(const svdq_layer* L, int64_t M, int* device_status) {
  Workspace w;
  int st = noalloc_layout(L, M, &w);
  if (st != SVDQ_OK) return st;
  int dev = -1;
  st = current_layer_device(L, &dev);
  if (st != SVDQ_OK) return st;
  cudaError_t e;
  uint8_t* ws = scratch_on(dev, &e);
  if (e != cudaSuccess || !ws) return SVDQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws + w.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  *device_status = v;
  return SVDQ_OK;
}

}  // namespace svdq

using namespace svdq;

extern "C" svdq_status svdq_forward_noalloc(const svdq_layer* L, const void* X, int64_t M, void* Y, void* stream) {
  Workspace w;
  int st = noalloc_layout(L, M, &w);
  if (st != SVDQ_OK) return (svdq_status)st;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || ((uintptr_t)X & 15) || ((uintptr_t)Y & 15)) return SVDQ_ERR_INVALID_ARG;
  int dev = -1;
  st = current_layer_device(L, &dev);
  if (st != SVDQ_OK) return (svdq_status)st;
  cudaError_t e;
  uint8_t* ws = scratch_on(dev, &e);
  if (e != cudaSuccess || !ws) return SVDQ_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  NvtxRange range("svdq/forward_noalloc");
  // the control block (status word, split-K counters) must start at zero; the
  // rest is fully rewritten by the kernels
  if (cudaMemsetAsync(ws + w.status, 0, w.ctrl_bytes, s) != cudaSuccess) return SVDQ_ERR_CUDA;
  st = L->dyn_gx ? launch_act_amax(L, X, M, ws, w, s) : SVDQ_OK;
  if (st != SVDQ_OK) return (svdq_status)st;
  st = launch_quantize(L, X, M, ws, w, s);
  if (st != SVDQ_OK) return (svdq_status)st;
  if (L->fmt == SVDQ_NVFP4_G16) return (svdq_status)launch_gemm_nvfp4(L, M, Y, ws, w, s);
  return (svdq_status)launch_gemm_int4(L, M, Y, ws, w, nullptr, s);
}
