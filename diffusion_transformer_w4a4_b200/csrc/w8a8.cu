// INT8 tensorwise W8A8 linear layer: the 8-bit variant that "SVDQuant ускоряет
// Krea 2 вдвое ..." (section "Решение: INT8 и W4A4") compares with W4A4.
//
//   s_w = fl32(max|W| / 127) (prepared once),  s_x = fl32(max|X| / 127) (per call),
//   q = clamp(rne(v * fl32(1/s)), -127, 127),
//   Y = bf16( (s_x s_w) * (qx . qw^T) + b ),
//
// No smoothing and no low-rank branch.  Three kernels per forward:
//   k_act_amax (shared with the dynamic NVFP4 scale, no 1/lambda here): per-CTA
//     maxima of |x| into the workspace's control block;
//   k_w8_quantize (HBM-bound): reduces the maxima, derives s_x, writes the int8
//     codes [M, K] and leaves s_x in the control block;
//   k_gemm_w8a8: tcgen05.mma kind::i8 (s8 x s8 -> s32 in tensor memory), tile
//     128 x 256, 128 K per stage through a 4-stage TMA ring (128-byte swizzle);
//     warp 0 TMA, warp 1 MMA (4 instructions of K = 32 per stage), warps 2-9 the
//     epilogue: two per tensor-memory lane quarter, 128 columns each, 32x32b
//     loads (one row per thread), y = fmaf(float(acc), s_x s_w, b), bf16
//     stores.  The two 256-column accumulators alternate between tiles, so the
//     epilogue of one tile overlaps the next tile's MMAs.  Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "sm100.cuh"
#include "svdq_internal.h"

struct svdq_w8a8_layer {
  int64_t N, K;
  int device;
  float s_w;
  const float* bias;   // [N]
  const int8_t* wcodes;  // [N, K]
  CUtensorMap map_w;
};

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;  // BK bytes = codes per stage
constexpr int STAGES = 4;
constexpr int STAGE_A = BM * BK, STAGE_B = BN * BK;
constexpr int STAGE_BYTES = STAGE_A + STAGE_B;  // 48 KiB
constexpr int EPI_WARP0 = 2, EPI_WARPS = 8;
constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;  // two accumulators of BN columns
constexpr uint32_t IDESC = idesc_s8_s32(BM, BN);
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
constexpr int kQuantThreads = 256;

// ------------------------------------------------------------------ blob / workspace
struct W8Blob {
  size_t bias, wcodes, total;
};
W8Blob w8_blob_layout(int64_t N, int64_t K) {
  auto up = [](size_t x) { return (x + kAlign - 1) / kAlign * kAlign; };
  W8Blob b{};
  b.bias = 0;
  b.wcodes = up((size_t)N * 4);
  b.total = up(b.wcodes + (size_t)N * K);
  return b;
}
struct W8Ws {
  size_t codes, ctrl, slots, total;  // ctrl: [0] status, [4] s_x; slots: kAmaxSlots floats
};
W8Ws w8_ws_layout(int64_t M, int64_t K) {
  W8Ws w{};
  w.codes = 0;
  w.ctrl = ((size_t)M * K + kAlign - 1) / kAlign * kAlign;
  w.slots = w.ctrl + 16;
  w.total = w.slots + 4 * (size_t)kAmaxSlots;
  return w;
}
bool w8_shape_ok(int64_t N, int64_t K) {
  return N >= 8 && N % 8 == 0 && N <= (1 << 24) && K >= BK && K % BK == 0 && K <= (1 << 20);
}

// ------------------------------------------------------------------ quantizer
__global__ void __launch_bounds__(kQuantThreads) k_w8_quantize(const uint4* __restrict__ x, int64_t nvec16,
                                                             const float* __restrict__ slots, int nslots,
                                                             uint4* __restrict__ codes, float* __restrict__ s_out,
                                                             int* __restrict__ status) {
  __shared__ float red[kQuantThreads / 32];
  float m = 0.f;
  for (int i = threadIdx.x; i < nslots; i += kQuantThreads) m = fmaxf(m, slots[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, red[i]);
  const float s = __fdiv_rn(m, 127.f);               // binary32, as prepared for the weight
  const float inv = s > 0.f ? __fdiv_rn(1.f, s) : 0.f;  // s == 0: every code 0
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *s_out = s;
    *status = 0;  // the GEMM that follows records errors here
  }
  for (int64_t i = (int64_t)blockIdx.x * kQuantThreads + threadIdx.x; i < nvec16;
       i += (int64_t)gridDim.x * kQuantThreads) {
    const uint4 a = __ldcs(x + 2 * i), b = __ldcs(x + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t packed = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t v = w[2 * j + h];
        int q0 = __float2int_rn(__uint_as_float(v << 16) * inv);  // round half to even
        int q1 = __float2int_rn(__uint_as_float(v & 0xFFFF0000u) * inv);
        q0 = max(-127, min(127, q0));
        q1 = max(-127, min(127, q1));
        packed |= ((uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8)) << (16 * h);
      }
      out[j] = packed;
    }
    codes[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// ------------------------------------------------------------------ GEMM
struct W8Params {
  int M, N, K, m_tiles, n_tiles, num_tiles, k_stages;
  float s_w;
  const float* s_x;  // left by the quantizer
  const float* bias;
  uint16_t* Y;
  int* status;
  unsigned long long limit;
};
struct W8Maps {
  CUtensorMap a, b;
};

__global__ void __launch_bounds__(THREADS, 1) k_gemm_w8a8(const __grid_constant__ W8Maps maps,
                                                         const __grid_constant__ W8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;  // [STAGES][A | B]
  uint64_t* full = (uint64_t*)(stages + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.status, p.limit};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);  // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&maps.a);
      prefetch_tmap(&maps.b);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int ks = 0; ks < p.k_stages; ++ks, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(&maps.a, &full[s], st, ks * BK, mt * BM);
          tma_load_2d(&maps.b, &full[s], st + STAGE_A, ks * BK, nt * BN);
        }
      }
      if (!ok) {  // drain copies still in flight
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, p.limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++local) {
        const int b = local & 1;
        if (!mbar_wait(&acc_empty[b], ((local >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        for (int ks = 0; ks < p.k_stages; ++ks, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + s * STAGE_BYTES), b_addr = a_addr + STAGE_A;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)  // K = 32 codes (bytes) per instruction
            mma_s8(tmem + b * BN, make_sdesc(a_addr + 32 * kk, 16, 1024, LAYOUT_SW128),
                   make_sdesc(b_addr + 32 * kk, 16, 1024, LAYOUT_SW128), IDESC, (ks | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[b]);
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, p.limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                     // tensor-memory lane quarter
    const int h = (warp - EPI_WARP0) >> 2;      // column half: 128 columns
    const float scale = *p.s_x * p.s_w;         // binary32, as the product of the two scales
    int local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int b = local & 1;
      if (!mbar_wait(&acc_full[b], (local >> 1) & 1, wc)) break;
      tc_fence_after();
      const int m = mt * BM + 32 * q + lane;
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN + h * 128);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + 32 * c, r);
        tmem_ld_wait_regs(r);
        if (c == 3) {  // every column of this accumulator is in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        const int n0 = nt * BN + h * 128 + 32 * c;
        if (m < p.M) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {  // 8 columns per 16-byte store
            const int n = n0 + 8 * v;
            if (n >= p.N) break;
            const float4 b0 = __ldg((const float4*)(p.bias + n)), b1 = __ldg((const float4*)(p.bias + n) + 1);
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float y0 = fmaf((float)(int)r[8 * v + 2 * e], scale, bb[2 * e]);
              const float y1 = fmaf((float)(int)r[8 * v + 2 * e + 1], scale, bb[2 * e + 1]);
              __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
              o[e] = *(uint32_t*)&hv;
            }
            *(uint4*)(p.Y + (size_t)m * p.N + n) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

int launch_w8_quantize(const svdq_w8a8_layer* L, const void* X, int64_t M, uint8_t* ws, cudaStream_t stream) {
  const W8Ws w = w8_ws_layout(M, L->K);
  int st = launch_act_amax_raw(X, M, L->K, nullptr, (float*)(ws + w.slots), stream);
  if (st != SVDQ_OK) return st;
  int gx = 0, gy = 0;
  act_amax_grid(M, L->K, &gx, &gy);
  const int64_t nvec16 = M * L->K / 16;
  int64_t grid = (nvec16 + kQuantThreads - 1) / kQuantThreads;
  const int64_t cap = 8 * (int64_t)device_sm_count(L->device);
  if (grid > cap) grid = cap;
  k_w8_quantize<<<(unsigned)grid, kQuantThreads, 0, stream>>>((const uint4*)X, nvec16, (const float*)(ws + w.slots),
                                                              gx * gy, (uint4*)(ws + w.codes),
                                                              (float*)(ws + w.ctrl + 4), (int*)(ws + w.ctrl));
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

int launch_w8_gemm(const svdq_w8a8_layer* L, int64_t M, void* Y, uint8_t* ws, cudaStream_t stream) {
  const W8Ws w = w8_ws_layout(M, L->K);
  W8Maps maps;
  std::memset(&maps, 0, sizeof(maps));
  int st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.codes, (uint64_t)L->K, (uint64_t)M,
                          (uint64_t)L->K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  maps.b = L->map_w;
  W8Params p{};
  p.M = (int)M;
  p.N = (int)L->N;
  p.K = (int)L->K;
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = (int)((L->N + BN - 1) / BN);
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.k_stages = (int)(L->K / BK);
  p.s_w = L->s_w;
  p.s_x = (const float*)(ws + w.ctrl + 4);
  p.bias = L->bias;
  p.Y = (uint16_t*)Y;
  p.status = (int*)(ws + w.ctrl);
  p.limit = wait_limit_cycles();
  {  // the shared-memory attribute belongs to the kernel on each device: set it once per device
    static std::mutex mu;
    static bool attr_set[64] = {};
    if (L->device < 0 || L->device >= 64) return SVDQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[L->device]) {
      if (cudaFuncSetAttribute(k_gemm_w8a8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
          cudaSuccess)
        return SVDQ_ERR_CUDA;
      attr_set[L->device] = true;
    }
  }
  const int sms = device_sm_count(L->device);
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  k_gemm_w8a8<<<grid, THREADS, SMEM_BYTES, stream>>>(maps, p);
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

svdq_status svdq_w8a8_prepare(const uint16_t* W, int64_t N, int64_t K, int8_t* wcodes, float* s_w) {
  if (!W || !wcodes || !s_w || !w8_shape_ok(N, K)) return SVDQ_ERR_INVALID_ARG;
  float amax = 0.f;
  for (int64_t i = 0; i < N * K; ++i) {
    const float v = host::bf16_to_f32(W[i]);
    if (!std::isfinite(v)) return SVDQ_ERR_NUMERIC;
    amax = std::max(amax, std::fabs(v));
  }
  const float s = amax / 127.f;  // binary32 division
  const float inv = s > 0.f ? 1.f / s : 0.f;
  for (int64_t i = 0; i < N * K; ++i) {
    const float prod = host::bf16_to_f32(W[i]) * inv;  // binary32 product
    const float q = std::nearbyint(prod);            // round half to even (default rounding mode)
    wcodes[i] = (int8_t)std::max(-127.f, std::min(127.f, q));
  }
  *s_w = s;
  return SVDQ_OK;
}

svdq_status svdq_w8a8_packed_size(int64_t N, int64_t K, size_t* bytes) {
  if (!bytes || !w8_shape_ok(N, K)) return SVDQ_ERR_INVALID_ARG;
  *bytes = w8_blob_layout(N, K).total;
  return SVDQ_OK;
}

svdq_status svdq_w8a8_pack(int64_t N, int64_t K, const int8_t* wcodes, const uint16_t* bias, void* blob_v,
                           size_t blob_bytes) {
  if (!wcodes || !blob_v || !w8_shape_ok(N, K)) return SVDQ_ERR_INVALID_ARG;
  const W8Blob b = w8_blob_layout(N, K);
  if (blob_bytes < b.total) return SVDQ_ERR_INVALID_ARG;
  uint8_t* blob = (uint8_t*)blob_v;
  std::memset(blob, 0, b.total);
  float* bf = (float*)(blob + b.bias);
  for (int64_t n = 0; n < N; ++n) bf[n] = bias ? host::bf16_to_f32(bias[n]) : 0.f;
  std::memcpy(blob + b.wcodes, wcodes, (size_t)N * K);
  return SVDQ_OK;
}

svdq_status svdq_w8a8_layer_create(const void* dev_blob, size_t blob_bytes, int64_t N, int64_t K, float s_w,
                                   svdq_w8a8_layer** out) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!dev_blob || !w8_shape_ok(N, K) || ((uintptr_t)dev_blob & 255) || !(s_w >= 0.f) || !std::isfinite(s_w))
    return SVDQ_ERR_INVALID_ARG;
  const W8Blob b = w8_blob_layout(N, K);
  if (blob_bytes < b.total) return SVDQ_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  svdq_status st = svdq_device_check(dev);
  if (st != SVDQ_OK) return st;
  st = (svdq_status)check_blob_pointer(dev_blob, dev);
  if (st != SVDQ_OK) return st;
  svdq_w8a8_layer* L = new (std::nothrow) svdq_w8a8_layer();
  if (!L) return SVDQ_ERR_OOM;
  const uint8_t* base = (const uint8_t*)dev_blob;
  L->N = N;
  L->K = K;
  L->device = dev;
  L->s_w = s_w;
  L->bias = (const float*)(base + b.bias);
  L->wcodes = (const int8_t*)(base + b.wcodes);
  if (encode_tmap_2d(&L->map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->wcodes, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK,
                     BN, CU_TENSOR_MAP_SWIZZLE_128B) != SVDQ_OK) {
    delete L;
    return SVDQ_ERR_CUDA;
  }
  *out = L;
  return SVDQ_OK;
}

void svdq_w8a8_layer_destroy(svdq_w8a8_layer* layer) { delete layer; }

svdq_status svdq_w8a8_workspace_size(const svdq_w8a8_layer* L, int64_t M, size_t* bytes) {
  if (!L || !bytes || M < 0 || M > (1 << 30)) return SVDQ_ERR_INVALID_ARG;
  *bytes = w8_ws_layout(M, L->K).total;
  return SVDQ_OK;
}

static svdq_status w8_check(const svdq_w8a8_layer* L, int64_t M, const void* ws, size_t ws_bytes) {
  if (!L || M < 0 || M > (1 << 30) || !ws || ((uintptr_t)ws & 255)) return SVDQ_ERR_INVALID_ARG;
  if (ws_bytes < w8_ws_layout(M, L->K).total) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

svdq_status svdq_w8a8_quantize_act(const svdq_w8a8_layer* L, const void* X, int64_t M, void* ws, size_t ws_bytes,
                                   void* stream) {
  svdq_status st = w8_check(L, M, ws, ws_bytes);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;
  if (!X || ((uintptr_t)X & 15)) return SVDQ_ERR_INVALID_ARG;
  st = (svdq_status)require_current_device(L->device);
  if (st != SVDQ_OK) return st;
  NvtxRange range("svdq/w8a8_quantize");
  return (svdq_status)launch_w8_quantize(L, X, M, (uint8_t*)ws, (cudaStream_t)stream);
}

svdq_status svdq_w8a8_gemm(const svdq_w8a8_layer* L, int64_t M, void* Y, void* ws, size_t ws_bytes, void* stream) {
  svdq_status st = w8_check(L, M, ws, ws_bytes);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;
  if (!Y || ((uintptr_t)Y & 15)) return SVDQ_ERR_INVALID_ARG;
  st = (svdq_status)require_current_device(L->device);
  if (st != SVDQ_OK) return st;
  NvtxRange range("svdq/w8a8_gemm");
  return (svdq_status)launch_w8_gemm(L, M, Y, (uint8_t*)ws, (cudaStream_t)stream);
}

svdq_status svdq_w8a8_forward(const svdq_w8a8_layer* L, const void* X, int64_t M, void* Y, void* ws,
                              size_t ws_bytes, void* stream) {
  svdq_status st = svdq_w8a8_quantize_act(L, X, M, ws, ws_bytes, stream);
  if (st != SVDQ_OK) return st;
  return svdq_w8a8_gemm(L, M, Y, ws, ws_bytes, stream);
}

svdq_status svdq_w8a8_read_status(const svdq_w8a8_layer* L, int64_t M, const void* ws, size_t ws_bytes,
                                  int* device_status) {
  svdq_status st = w8_check(L, M, ws, ws_bytes);
  if (st != SVDQ_OK) return st;
  if (!device_status) return SVDQ_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpy(&v, (const uint8_t*)ws + w8_ws_layout(M, L->K).ctrl, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  *device_status = v;
  return SVDQ_OK;
}

}  // extern "C"
