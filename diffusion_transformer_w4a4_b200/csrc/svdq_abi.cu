// libsvdq C ABI: argument checks, layouts, packing, layer handles, tensor-map
// encoding, and the forward entry points.  See include/svdq.h for the contract.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "svdq_internal.h"

namespace svdq {

static std::atomic<unsigned long long> g_wait_limit{0};
unsigned long long wait_limit_cycles() {
  unsigned long long v = g_wait_limit.load();
  return v ? v : (1ull << 31);
}

int device_sm_count(int dev) {
  static std::atomic<int> cache[64];
  if (dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load();
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n);
  }
  return n;
}

int require_current_device(int dev) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return cur == dev ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
}

int check_blob_pointer(const void* p, int dev) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_OK;
  }
  if (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeUnregistered) return SVDQ_ERR_INVALID_ARG;
  if (a.type == cudaMemoryTypeDevice && a.device != dev) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

LowRankChunks lowrank_chunks(int rank) {
  LowRankChunks c{};
  int off = 0;
  while (off < rank && c.n < 4) {
    const int left = rank - off;
    const int w = left >= 64 ? 64 : (left >= 32 ? 32 : 16);
    c.off[c.n] = off;
    c.width[c.n] = w;
    ++c.n;
    off += w;
  }
  return c;
}

static bool shape_ok(int64_t N, int64_t K, int rank, int fmt) {
  if (fmt != SVDQ_INT4_G64 && fmt != SVDQ_NVFP4_G16) return false;
  if (K <= 0 || N < 16 || K % kKStage != 0 || N % 16 != 0) return false;
  if (rank < 0 || rank % 16 != 0 || rank > kMaxRank || rank > K || rank > N) return false;
  if (K > (1 << 30) || N > (1 << 30)) return false;
  return true;
}

Blob blob_layout(int64_t N, int64_t K, int rank, int fmt) {
  Blob b{};
  size_t o = 0;
  b.inv_lambda = o;
  o = align_up(o + (size_t)K * 4, kAlign);
  b.L1t = o;
  o = align_up(o + (size_t)rank * K * 2, kAlign);
  b.L2t = o;
  o = align_up(o + (size_t)N * rank * 2, kAlign);
  b.bias = o;
  o = align_up(o + (size_t)N * 4, kAlign);
  b.wcodes = o;  // NVFP4: packed E2M1 pairs; INT4: one E4M3 byte per code
  o = align_up(o + (fmt == SVDQ_NVFP4_G16 ? (size_t)N * K / 2 : (size_t)N * K), kAlign);
  b.wscales = o;
  if (fmt == SVDQ_NVFP4_G16) {
    const size_t tiles = (size_t)((N + kNvfp4BN - 1) / kNvfp4BN);
    o = align_up(o + tiles * (size_t)(K / 64) * 2 * kSfAtomBytes, kAlign);
  } else {
    o = align_up(o + (size_t)(K / 64) * N * 4, kAlign);
  }
  b.total = o;
  return b;
}

Workspace workspace_layout(int64_t N, int64_t K, int rank, int fmt, int64_t M) {
  (void)N;
  Workspace w{};
  size_t o = 0;
  w.codes = o;
  w.codes_bytes = fmt == SVDQ_NVFP4_G16 ? (size_t)M * K / 2 : (size_t)M * K;
  o = align_up(o + w.codes_bytes, kAlign);
  w.scales = o;
  if (fmt == SVDQ_NVFP4_G16)  // whole 128-row atoms
    w.scales_bytes = (size_t)((M + kSfAtomRows - 1) / kSfAtomRows) * (size_t)(K / 64) * kSfAtomBytes;
  else
    w.scales_bytes = (size_t)(K / 64) * (size_t)int4_scale_ld(M) * 2;
  o = align_up(o + w.scales_bytes, kAlign);
  w.t = o;
  w.t_bytes = (size_t)M * rank * 2;
  o = align_up(o + w.t_bytes, kAlign);
  // control block: status word and per-call g_x, one arrival counter per
  // 128-row block, then the slots of the dynamic activation-scale pass
  w.status = o;
  w.amax = o + align_up(16 + 4 * (size_t)((M + kQRows - 1) / kQRows), 16);
  w.ctrl_bytes = (w.amax - o) + 4 * (size_t)kAmaxSlots;
  o = align_up(o + w.ctrl_bytes, kAlign);
  // fp32 partial low-rank sums of the quantizer's K slices
  w.nslices = quant_slices(M, K);
  w.tpart = o;
  w.tpart_bytes = (w.nslices > 1 && rank > 0) ? (size_t)w.nslices * M * rank * 4 : 0;
  o = align_up(o + w.tpart_bytes, kAlign);
  w.total = o;
  return w;
}

// ------------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  });
  return fn;
}

int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = get_encode();
  if (!fn) return SVDQ_ERR_CUDA;
  if (((uintptr_t)base & 15) || (row_bytes & 15)) return SVDQ_ERR_INVALID_ARG;
  if (outer == 0) outer = 1;  // an empty tensor is never read; keep the descriptor valid
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace svdq

using namespace svdq;

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG: invalid shape, format, pointer alignment or size";
    case SVDQ_ERR_UNSUPPORTED_DEVICE:
      return "SVDQ_ERR_UNSUPPORTED_DEVICE: svdq_w4a4 kernels need an sm_100a (compute capability 10.0) GPU";
    case SVDQ_ERR_OOM: return "SVDQ_ERR_OOM: host allocation failed";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA: a CUDA call failed";
    case SVDQ_ERR_NUMERIC: return "SVDQ_ERR_NUMERIC: non-finite input";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT: an in-kernel wait ran past its limit";
    case SVDQ_ERR_BOUNDS: return "SVDQ_ERR_BOUNDS: a kernel addressed memory outside its buffer (debug build)";
    default: return "SVDQ_ERR_UNKNOWN";
  }
}

int svdq_abi_version(void) { return SVDQ_ABI_VERSION; }

int svdq_debug_build(void) {
#ifdef SVDQ_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

svdq_status svdq_canonical_sizes(int64_t N, int64_t K, int rank, int fmt, size_t sizes[7]) {
  if (!sizes || !shape_ok(N, K, rank, fmt)) return SVDQ_ERR_INVALID_ARG;
  sizes[0] = (size_t)K * 4;
  sizes[1] = (size_t)K * 4;
  sizes[2] = (size_t)K * rank * 2;
  sizes[3] = (size_t)rank * N * 2;
  sizes[4] = (size_t)N * K / 2;
  sizes[5] = fmt == SVDQ_INT4_G64 ? (size_t)N * (K / 64) * 2 : (size_t)N * (K / 16);
  sizes[6] = (size_t)N * 2;
  return SVDQ_OK;
}

svdq_status svdq_prepare(const uint16_t* W, const uint16_t* bias, const float* act_absmax, float alpha,
                         svdq_canonical* out) {
  if (!W || !act_absmax || !out) return SVDQ_ERR_INVALID_ARG;
  if (!shape_ok(out->N, out->K, out->rank, out->fmt)) return SVDQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return SVDQ_ERR_INVALID_ARG;
  if (!out->lambda || !out->inv_lambda || !out->wcodes || !out->wscales || !out->bias) return SVDQ_ERR_INVALID_ARG;
  if (out->rank > 0 && (!out->L1 || !out->L2)) return SVDQ_ERR_INVALID_ARG;
  const char* f = std::getenv("SVDQ_FAULT");
  if (f && std::strcmp(f, "alloc") == 0) return SVDQ_ERR_OOM;
  if (f && std::strcmp(f, "nan_input") == 0) return SVDQ_ERR_NUMERIC;
  try {
    return (svdq_status)host::prepare(W, bias, act_absmax, alpha, out);
  } catch (const std::bad_alloc&) {
    return SVDQ_ERR_OOM;
  } catch (...) {
    return SVDQ_ERR_INVALID_ARG;
  }
}

svdq_status svdq_packed_size(int64_t N, int64_t K, int rank, int fmt, size_t* bytes) {
  if (!bytes || !shape_ok(N, K, rank, fmt)) return SVDQ_ERR_INVALID_ARG;
  *bytes = blob_layout(N, K, rank, fmt).total;
  return SVDQ_OK;
}

svdq_status svdq_pack(const svdq_canonical* c, void* blob_v, size_t blob_bytes) {
  if (!c || !blob_v || !shape_ok(c->N, c->K, c->rank, c->fmt)) return SVDQ_ERR_INVALID_ARG;
  const int64_t N = c->N, K = c->K;
  const int r = c->rank, fmt = c->fmt;
  const Blob b = blob_layout(N, K, r, fmt);
  if (blob_bytes < b.total) return SVDQ_ERR_INVALID_ARG;
  if (!c->inv_lambda || !c->wcodes || !c->wscales || (r > 0 && (!c->L1 || !c->L2))) return SVDQ_ERR_INVALID_ARG;
  uint8_t* blob = (uint8_t*)blob_v;
  std::memset(blob, 0, b.total);
  std::memcpy(blob + b.inv_lambda, c->inv_lambda, (size_t)K * 4);
  uint16_t* L1t = (uint16_t*)(blob + b.L1t);
  for (int64_t k = 0; k < K; ++k)
    for (int j = 0; j < r; ++j) L1t[(int64_t)j * K + k] = c->L1[k * r + j];
  // NVFP4: L2 / (g_x g_w), a power of two, so the low-rank product accumulates in
  // the units of the 4-bit block-scaled product.  With the dynamic activation
  // scale (g_x = 0) only 1/g_w is folded here; the quantizer stores t / g_x.
  float l2_scale = 1.0f;
  if (fmt == SVDQ_NVFP4_G16) {
    const float gg = (c->g_x == 0.f ? 1.0f : c->g_x) * c->g_w;
    int e;
    if (!(gg > 0.f) || std::frexp(gg, &e) != 0.5f) return SVDQ_ERR_INVALID_ARG;  // must be a power of two
    l2_scale = 1.0f / gg;
  }
  uint16_t* L2t = (uint16_t*)(blob + b.L2t);
  for (int j = 0; j < r; ++j)
    for (int64_t n = 0; n < N; ++n) {
      const float v = host::bf16_to_f32(c->L2[(int64_t)j * N + n]) * l2_scale;  // exact
      L2t[n * r + j] = host::f32_to_bf16(v);
    }
  float* bias = (float*)(blob + b.bias);
  for (int64_t n = 0; n < N; ++n) bias[n] = c->bias ? host::bf16_to_f32(c->bias[n]) : 0.f;
  if (fmt == SVDQ_NVFP4_G16) {
    std::memcpy(blob + b.wcodes, c->wcodes, (size_t)N * K / 2);
  } else {
    // each two's-complement nibble becomes the E4M3 byte of the same integer,
    // which the tensor core reads directly (every integer in [-8, 7] is exact)
    uint8_t lut[16];
    for (int v = 0; v < 16; ++v) lut[v] = host::int_to_e4m3(v < 8 ? v : v - 16);
    const size_t nb = (size_t)N * K / 2;
    uint8_t* d = blob + b.wcodes;
    for (size_t i = 0; i < nb; ++i) {
      d[2 * i] = lut[c->wcodes[i] & 15];
      d[2 * i + 1] = lut[c->wcodes[i] >> 4];
    }
  }
  if (fmt == SVDQ_NVFP4_G16) {
    const uint8_t* s = (const uint8_t*)c->wscales;
    const int64_t B = K / 16;
    for (int64_t n = 0; n < N; ++n)
      for (int64_t blk = 0; blk < B; ++blk) blob[b.wscales + sf_offset(n, blk, K / 64, kNvfp4BN)] = s[n * B + blk];
  } else {
    const uint16_t* s = (const uint16_t*)c->wscales;
    float* d = (float*)(blob + b.wscales);
    const int64_t G = K / 64;
    for (int64_t n = 0; n < N; ++n)
      for (int64_t g = 0; g < G; ++g) d[g * N + n] = host::f16_to_f32(s[n * G + g]);  // exact
  }
  return SVDQ_OK;
}

svdq_status svdq_device_check(int device) {
  const char* f = std::getenv("SVDQ_FAULT");
  if (f && std::strcmp(f, "bad_arch") == 0) return SVDQ_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  return (major == 10 && minor == 0) ? SVDQ_OK : SVDQ_ERR_UNSUPPORTED_DEVICE;
}

svdq_status svdq_layer_create(const void* dev_blob, size_t blob_bytes, int64_t N, int64_t K, int rank, int fmt,
                              float g_x, float g_w, svdq_layer** out) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!dev_blob || !shape_ok(N, K, rank, fmt) || ((uintptr_t)dev_blob & 255)) return SVDQ_ERR_INVALID_ARG;
  const Blob b = blob_layout(N, K, rank, fmt);
  if (blob_bytes < b.total) return SVDQ_ERR_INVALID_ARG;
  if (fmt == SVDQ_NVFP4_G16) {  // g_x == 0 selects the dynamic activation scale
    int e;
    if (!(g_x >= 0.f) || !(g_w > 0.f) || std::frexp((g_x == 0.f ? 1.0f : g_x) * g_w, &e) != 0.5f)
      return SVDQ_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  svdq_status st = svdq_device_check(dev);
  if (st != SVDQ_OK) return st;
  st = (svdq_status)check_blob_pointer(dev_blob, dev);
  if (st != SVDQ_OK) return st;
  svdq_layer* L = new (std::nothrow) svdq_layer();
  if (!L) return SVDQ_ERR_OOM;
  L->N = N;
  L->K = K;
  L->rank = rank;
  L->fmt = fmt;
  L->g_x = fmt == SVDQ_NVFP4_G16 ? g_x : 1.0f;
  L->g_w = fmt == SVDQ_NVFP4_G16 ? g_w : 1.0f;
  L->dyn_gx = fmt == SVDQ_NVFP4_G16 && g_x == 0.f;
  L->device = dev;
  L->blob = (const uint8_t*)dev_blob;
  L->off = b;
  L->inv_lambda = (const float*)(L->blob + b.inv_lambda);
  L->L1t = (const uint16_t*)(L->blob + b.L1t);
  L->L2t = (const uint16_t*)(L->blob + b.L2t);
  L->bias = (const float*)(L->blob + b.bias);
  L->wcodes = L->blob + b.wcodes;
  L->wscales = L->blob + b.wscales;
  int e = SVDQ_OK;
  if (fmt == SVDQ_NVFP4_G16) {  // 256 codes (128 B) per row per stage, swizzled for the MMA
    e = encode_tmap_2d(&L->map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->wcodes, (uint64_t)K / 2, (uint64_t)N,
                       (uint64_t)K / 2, 128, kNvfp4BN, CU_TENSOR_MAP_SWIZZLE_128B);
  } else  // 128 E4M3 codes (128 B) per row per stage, swizzled for the MMA
    e = encode_tmap_2d(&L->map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->wcodes, (uint64_t)K, (uint64_t)N, (uint64_t)K,
                       128, kInt4BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == SVDQ_OK && rank > 0) {
    e = encode_tmap_2d(&L->map_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->L1t, (uint64_t)K, (uint64_t)rank,
                       (uint64_t)K * 2, 64, (uint32_t)rank, CU_TENSOR_MAP_SWIZZLE_128B);
    const int widths[3] = {64, 32, 16};
    const CUtensorMapSwizzle swz[3] = {CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_SWIZZLE_64B,
                                       CU_TENSOR_MAP_SWIZZLE_32B};
    const uint32_t bn = fmt == SVDQ_NVFP4_G16 ? kNvfp4BN : kInt4BN;
    for (int i = 0; i < 3 && e == SVDQ_OK; ++i) {
      if (widths[i] > rank) continue;
      e = encode_tmap_2d(&L->map_l2[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->L2t, (uint64_t)rank, (uint64_t)N,
                         (uint64_t)rank * 2, widths[i], bn, swz[i]);
    }
  }
  if (e != SVDQ_OK) {
    delete L;
    return (svdq_status)e;
  }
  *out = L;
  return SVDQ_OK;
}

void svdq_layer_destroy(svdq_layer* layer) { delete layer; }

svdq_status svdq_workspace_size(const svdq_layer* L, int64_t M, size_t* bytes) {
  if (!L || !bytes || M < 0) return SVDQ_ERR_INVALID_ARG;
  *bytes = workspace_layout(L->N, L->K, L->rank, L->fmt, M).total;
  return SVDQ_OK;
}

svdq_status svdq_workspace_layout(const svdq_layer* L, int64_t M, size_t offsets[4], size_t sizes[4]) {
  if (!L || !offsets || !sizes || M < 0) return SVDQ_ERR_INVALID_ARG;
  const Workspace w = workspace_layout(L->N, L->K, L->rank, L->fmt, M);
  offsets[0] = w.codes;
  offsets[1] = w.scales;
  offsets[2] = w.t;
  offsets[3] = w.status;
  sizes[0] = w.codes_bytes;
  sizes[1] = w.scales_bytes;
  sizes[2] = w.t_bytes;
  sizes[3] = 4;
  return SVDQ_OK;
}

static svdq_status check_ws(const svdq_layer* L, int64_t M, const void* ws, size_t ws_bytes, Workspace* w) {
  if (!L || M < 0 || M > (int64_t)1 << 30 || !ws || ((uintptr_t)ws & 255)) return SVDQ_ERR_INVALID_ARG;
  *w = workspace_layout(L->N, L->K, L->rank, L->fmt, M);
  if (ws_bytes < w->total) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

svdq_status svdq_workspace_init(const svdq_layer* L, int64_t M, void* ws, size_t ws_bytes, void* stream) {
  Workspace w;
  svdq_status st = check_ws(L, M, ws, ws_bytes, &w);
  if (st != SVDQ_OK) return st;
  st = (svdq_status)require_current_device(L->device);
  if (st != SVDQ_OK) return st;
  if (cudaMemsetAsync((uint8_t*)ws + w.status, 0, w.ctrl_bytes, (cudaStream_t)stream) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

svdq_status svdq_quantize_act(const svdq_layer* L, const void* X, int64_t M, void* ws, size_t ws_bytes,
                              void* stream) {
  Workspace w;
  svdq_status st = check_ws(L, M, ws, ws_bytes, &w);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;
  if (!X || ((uintptr_t)X & 15)) return SVDQ_ERR_INVALID_ARG;
  st = (svdq_status)require_current_device(L->device);
  if (st != SVDQ_OK) return st;
  NvtxRange range("svdq/quantize");
  if (L->dyn_gx) {  // first pass: the tensor's largest |x^|
    const int e = launch_act_amax(L, X, M, (uint8_t*)ws, w, (cudaStream_t)stream);
    if (e != SVDQ_OK) return (svdq_status)e;
  }
  return (svdq_status)launch_quantize(L, X, M, (uint8_t*)ws, w, (cudaStream_t)stream);
}

svdq_status svdq_gemm(const svdq_layer* L, int64_t M, void* Y, void* ws, size_t ws_bytes, void* stream) {
  Workspace w;
  svdq_status st = check_ws(L, M, ws, ws_bytes, &w);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;
  if (!Y || ((uintptr_t)Y & 15)) return SVDQ_ERR_INVALID_ARG;
  st = (svdq_status)require_current_device(L->device);
  if (st != SVDQ_OK) return st;
  NvtxRange range("svdq/gemm");
  if (L->fmt == SVDQ_NVFP4_G16) return (svdq_status)launch_gemm_nvfp4(L, M, Y, (uint8_t*)ws, w, (cudaStream_t)stream);
  return (svdq_status)launch_gemm_int4(L, M, Y, (uint8_t*)ws, w, nullptr, (cudaStream_t)stream);
}

svdq_status svdq_forward(const svdq_layer* L, const void* X, int64_t M, void* Y, void* ws, size_t ws_bytes,
                         void* stream) {
  svdq_status st = svdq_quantize_act(L, X, M, ws, ws_bytes, stream);
  if (st != SVDQ_OK) return st;
  return svdq_gemm(L, M, Y, ws, ws_bytes, stream);
}

svdq_status svdq_mlp_fusable(const svdq_layer* up, const svdq_layer* down) {
  return (svdq_status)fused_mlp_supported(up, down);
}

svdq_status svdq_gemm_gelu_quantize(const svdq_layer* up, const svdq_layer* down, int64_t M, void* ws_up,
                                    size_t ws_up_bytes, void* ws_dn, size_t ws_dn_bytes, void* H, void* stream) {
  Workspace wu, wd;
  svdq_status st = check_ws(up, M, ws_up, ws_up_bytes, &wu);
  if (st != SVDQ_OK) return st;
  st = check_ws(down, M, ws_dn, ws_dn_bytes, &wd);
  if (st != SVDQ_OK) return st;
  st = (svdq_status)fused_mlp_supported(up, down);
  if (st != SVDQ_OK) return st;
  if (M > kFusedMlpMaxM) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (H && ((uintptr_t)H & 15)) return SVDQ_ERR_INVALID_ARG;
  st = (svdq_status)require_current_device(up->device);  // the pair shares one device
  if (st != SVDQ_OK) return st;
  NvtxRange range("svdq/gemm_gelu_quantize");
  return (svdq_status)launch_gemm_gelu_quant(up, down, M, (uint8_t*)ws_up, wu, (uint8_t*)ws_dn, wd, H,
                                             (cudaStream_t)stream);
}

svdq_status svdq_mlp_forward(const svdq_layer* up, const svdq_layer* down, const void* X, int64_t M, void* Y,
                             void* ws_up, size_t ws_up_bytes, void* ws_dn, size_t ws_dn_bytes, void* stream) {
  svdq_status st = (svdq_status)fused_mlp_supported(up, down);
  if (st != SVDQ_OK) return st;
  if (M > kFusedMlpMaxM) return SVDQ_ERR_INVALID_ARG;  // before anything is enqueued
  st = svdq_quantize_act(up, X, M, ws_up, ws_up_bytes, stream);
  if (st != SVDQ_OK) return st;
  st = svdq_gemm_gelu_quantize(up, down, M, ws_up, ws_up_bytes, ws_dn, ws_dn_bytes, nullptr, stream);
  if (st != SVDQ_OK) return st;
  return svdq_gemm(down, M, Y, ws_dn, ws_dn_bytes, stream);
}

svdq_status svdq_int4_group_acc(const svdq_layer* L, int64_t M, void* ws, size_t ws_bytes, int32_t* acc,
                                void* stream) {
  Workspace w;
  svdq_status st = check_ws(L, M, ws, ws_bytes, &w);
  if (st != SVDQ_OK) return st;
  if (L->fmt != SVDQ_INT4_G64 || !acc || ((uintptr_t)acc & 15)) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  st = (svdq_status)require_current_device(L->device);
  if (st != SVDQ_OK) return st;
  return (svdq_status)launch_gemm_int4(L, M, nullptr, (uint8_t*)ws, w, acc, (cudaStream_t)stream);
}

svdq_status svdq_read_status(const svdq_layer* L, int64_t M, const void* ws, size_t ws_bytes, int* device_status) {
  if (!ws && ws_bytes == 0) {  // the fixed scratch of svdq_forward_noalloc
    if (!device_status) return SVDQ_ERR_INVALID_ARG;
    return (svdq_status)read_status_noalloc(L, M, device_status);
  }
  Workspace w;
  svdq_status st = check_ws(L, M, ws, ws_bytes, &w);
  if (st != SVDQ_OK) return st;
  if (!device_status) return SVDQ_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpy(&v, (const uint8_t*)ws + w.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  *device_status = v;
  return SVDQ_OK;
}

svdq_status svdq_set_wait_limit(uint64_t cycles) {
  g_wait_limit.store((unsigned long long)cycles);
  return SVDQ_OK;
}

}  // extern "C"
