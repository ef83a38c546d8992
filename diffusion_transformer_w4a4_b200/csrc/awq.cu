// awq_w4a16: the 4-bit-weight / 16-bit-activation runtime layer
// ("Hugging Face встроила Nunchaku в Diffusers ...", paragraph on Nunchaku
// Lite: normalization and modulation layers such as adaLN in FLUX).
//
//   y[m,n] = sum_k (f32(x[m,k]) * inv_s[k]) * q[n,k] * S[n, k/64] + b[n]
//
// At the batch sizes of modulation layers (M = 1 or 2 conditioning vectors) the
// layer is a weight-streaming matrix-vector product, bound by reading the
// 4-bit weights from HBM, so it runs on CUDA cores and keeps the weights packed.
//
// k_awq_gemv: one thread per 32-code (16-byte) chunk of K.  A thread keeps
// its chunk of x^ = f32(x) * inv_s for up to two token rows in registers and
// streams the matching 16 bytes of every weight row, eight rows per batch (one
// load each, all in flight together).  A code u (two's complement nibble n,
// u = n ^ 8 in [0, 15], value u - 8) is turned into the binary32 1 + u/16 by
// placing u in the mantissa (byte arithmetic and one byte permute per code), so
// a chunk's sum is
//   sum_e (u_e - 8) x^_e = 16 sum_e (1 + u_e/16) x^_e - 24 sum_e x^_e,
// with the last sum computed once per thread.  The chunk's partial times its
// group scale is reduced over the CTA (warp shuffles, then shared memory).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>
#include <mutex>
#include <new>

#include "sm100.cuh"
#include "svdq_internal.h"

struct svdq_awq_layer {
  int64_t N, K;
  int device;
  const float* inv_s;
  const float* bias;
  const uint16_t* wscales;
  const uint8_t* wcodes;
};

namespace svdq {
namespace {

constexpr int kAwqRows = 8;  // weight rows per batch
constexpr int kAwqMaxMB = 2;  // token rows per launch (their x^ chunks live in registers)
constexpr int kAwqStagesMax = 4;  // weight batches in flight per CTA (2 for the widest K)

struct AwqBlob {
  size_t inv_s, bias, wscales, wcodes, total;
};

// fp16 group scales per blob row: K/64 rounded up to even, so every row starts
// 4-byte aligned and a thread's 4-byte scale pair stays inside its row
__host__ __device__ inline int64_t awq_scale_ld(int64_t K) { return (K / 64 + 1) / 2 * 2; }

AwqBlob awq_blob_layout(int64_t N, int64_t K) {
  auto up = [](size_t x) { return (x + kAlign - 1) / kAlign * kAlign; };
  AwqBlob b{};
  size_t o = 0;
  b.inv_s = o;
  o = up(o + (size_t)K * 4);
  b.bias = o;
  o = up(o + (size_t)N * 4);
  b.wscales = o;
  o = up(o + (size_t)N * awq_scale_ld(K) * 2);
  b.wcodes = o;
  o = up(o + (size_t)N * (K / 2));
  b.total = o;
  return b;
}

bool awq_shape_ok(int64_t N, int64_t K) { return N >= 1 && K >= 64 && K % 64 == 0 && K <= 12288 && N <= (1 << 30); }

struct AwqParams {
  int M, N, K, m0;
  const uint16_t* x;
  const float* inv_s;
  const uint8_t* codes;
  const uint16_t* scales;
  const float* bias;
  uint16_t* y;
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Persistent: a CTA walks batches of kAwqRows weight rows.  Each thread copies
// its own 16-byte chunk of the batches ahead, and the 4-byte pair of fp16
// group scales that holds its chunk's scale, into a STG-deep ring in
// shared memory (cp.async) and reads back only what it copied, so the group
// wait alone orders the pipeline.
template <int MB, int STG>
__global__ void __launch_bounds__(384) k_awq_gemv(const __grid_constant__ AwqParams p) {
  // [STG][kAwqRows][threads] 16-byte weight chunks, then the same
  // index space of 4-byte scale pairs
  extern __shared__ __align__(16) uint8_t awq_smem[];
  __shared__ float red[12][kAwqRows * MB];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x, nwarps = nthr >> 5;
  const int nchunk = p.K >> 5;
  const bool active = tid < nchunk;
  const int k0 = tid * 32;

  const size_t row_bytes = (size_t)p.K / 2, row_groups = (size_t)awq_scale_ld(p.K);
  const int stride = gridDim.x * kAwqRows;
  const size_t nslots = (size_t)STG * kAwqRows * nthr;
  auto slot = [&](int st, int r) -> size_t { return ((size_t)st * kAwqRows + r) * nthr + tid; };
  auto wslot = [&](int st, int r) -> uint8_t* { return awq_smem + slot(st, r) * 16; };
  auto sslot = [&](int st, int r) -> uint8_t* { return awq_smem + nslots * 16 + slot(st, r) * 4; };
  auto issue = [&](int nb, int st) {
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r) {
      const int n = nb + r;
      if (active && n < p.N) {
        cp_async16(wslot(st, r), p.codes + (size_t)n * row_bytes + 16 * (size_t)tid);
        // groups 2(tid/4) and 2(tid/4)+1: a 4-byte-aligned pair holding this chunk's group tid/2
        cp_async4(sslot(st, r), p.scales + (size_t)n * row_groups + 2 * (tid >> 2));
      }
    }
  };

  const int nb0 = blockIdx.x * kAwqRows;
#pragma unroll
  for (int j = 0; j < STG - 1; ++j) {  // prologue: the first batches in flight
    issue(nb0 + j * stride, j);
    cp_async_commit();
  }

  // this thread's 32 activations of each token row, times 1/s (while the
  // first weight batches are on their way)
  float xh[MB][32];
  float xsum[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    xsum[m] = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) xh[m][e] = 0.f;
  }
  if (active) {
    float is[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v = __ldg((const float4*)(p.inv_s + k0) + q);
      is[4 * q] = v.x;
      is[4 * q + 1] = v.y;
      is[4 * q + 2] = v.z;
      is[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      if (p.m0 + m >= p.M) continue;
      const uint4* xr = (const uint4*)(p.x + (size_t)(p.m0 + m) * p.K + k0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = __ldg(xr + q);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int e = 8 * q + 2 * h;
          xh[m][e] = __uint_as_float(w[h] << 16) * is[e];  // binary32 product, as in the smoothing step
          xh[m][e + 1] = __uint_as_float(w[h] & 0xFFFF0000u) * is[e + 1];
        }
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) xsum[m] += xh[m][e];
    }
  }

  int it = 0;
  for (int nb = nb0; nb < p.N; nb += stride, ++it) {
    issue(nb + (STG - 1) * stride, (it + STG - 1) % STG);
    cp_async_commit();
    cp_async_wait<STG - 1>();  // this batch's own copies have landed
    const int st = it % STG;
    float part[kAwqRows][MB];
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r) {
      uint4 wv = make_uint4(0u, 0u, 0u, 0u);
      float sc = 0.f;
      if (active && nb + r < p.N) {
        wv = *(const uint4*)wslot(st, r);
        const uint32_t pair = *(const uint32_t*)sslot(st, r);
        sc = __half2float(__ushort_as_half((unsigned short)(((tid >> 1) & 1) ? (pair >> 16) : (pair & 0xFFFFu))));
      }
      const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
      float acc[MB];
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[m] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // offset-binary codes u = n ^ 8; each byte of te / to becomes the third
        // byte 0x80 | u << 3 of the binary32 1 + u/16 for the even / odd code of
        // that byte, and one byte permute per code adds the top byte 0x3F
        const uint32_t v = wr[j] ^ 0x88888888u;
        const uint32_t te = ((v << 3) & 0x78787878u) | 0x80808080u;
        const uint32_t to = ((v >> 1) & 0x78787878u) | 0x80808080u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float fe = __uint_as_float(__byte_perm(te, 0x3F000000u, 0x7054u | (i << 8)));
          const float fo = __uint_as_float(__byte_perm(to, 0x3F000000u, 0x7054u | (i << 8)));
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            acc[m] = fmaf(fe, xh[m][8 * j + 2 * i], acc[m]);
            acc[m] = fmaf(fo, xh[m][8 * j + 2 * i + 1], acc[m]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) part[r][m] = sc * fmaf(16.f, acc[m], -24.f * xsum[m]);
    }
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        float v = part[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][r * MB + m] = v;
      }
    __syncthreads();
    if (tid < kAwqRows * MB) {
      const int r = tid / MB, m = tid % MB, n = nb + r;
      float v = 0.f;
      for (int wi = 0; wi < nwarps; ++wi) v += red[wi][tid];
      if (n < p.N && p.m0 + m < p.M)
        p.y[(size_t)(p.m0 + m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v + p.bias[n]));
    }
    __syncthreads();
  }
  cp_async_wait<0>();  // no copy may still target shared memory when the CTA exits
}

int awq_sm_count(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Shared memory of one CTA: STG stages of kAwqRows 16-byte chunks and 4-byte
// scale pairs per thread.
constexpr size_t awq_smem_bytes(int stg, int threads) { return (size_t)stg * kAwqRows * threads * 20; }

// CTAs per SM for one kernel variant and block size, found once per device and
// cached (the attribute call and the occupancy query cost microseconds of host
// time that would otherwise precede every launch)
// The largest block a variant is launched with: four stages up to 256 threads
// (K <= 8192), two stages up to 384.  The dynamic shared-memory attribute belongs
// to the kernel, not to a block size, so it is set once to this largest need.
constexpr int awq_max_threads(int stg) { return stg == kAwqStagesMax ? 256 : 384; }

template <int MB, int STG>
int awq_blocks_per_sm(int dev, int threads) {
  static std::mutex mu;
  static int cache[64][13] = {};  // [device][threads / 32]
  static bool attr_set[64] = {};
  if (dev < 0 || dev >= 64 || threads < 32 || threads > awq_max_threads(STG)) return -1;
  std::lock_guard<std::mutex> lock(mu);
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(k_awq_gemv<MB, STG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)awq_smem_bytes(STG, awq_max_threads(STG))) != cudaSuccess)
      return -1;
    attr_set[dev] = true;
  }
  int& c = cache[dev][threads / 32];
  if (c == 0) {
    const size_t smem = awq_smem_bytes(STG, threads);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_awq_gemv<MB, STG>, threads, smem) != cudaSuccess ||
        per_sm < 1)
      return -1;
    c = per_sm;
  }
  return c;
}

template <int MB, int STG>
int launch_awq_stg(const AwqParams& p, int dev, int threads, cudaStream_t stream) {
  const int per_sm = awq_blocks_per_sm<MB, STG>(dev, threads);
  if (per_sm < 1) return SVDQ_ERR_CUDA;
  // enough CTAs to fill the SMs, but each walking several batches so that its
  // ring reaches steady state (a CTA's setup and first round trip are not hidden)
  const int batches = (p.N + kAwqRows - 1) / kAwqRows;
  const int sms = awq_sm_count(dev);
  int grid = sms * per_sm;
  const int by_work = batches / STG;
  if (grid > by_work) grid = by_work > sms ? by_work : sms;
  if (grid > batches) grid = batches;
  k_awq_gemv<MB, STG><<<grid, threads, awq_smem_bytes(STG, threads), stream>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

template <int MB>
int launch_awq(const AwqParams& p, int dev, cudaStream_t stream) {
  const int threads = ((p.K / 32) + 31) / 32 * 32;
  if (threads <= awq_max_threads(kAwqStagesMax)) return launch_awq_stg<MB, kAwqStagesMax>(p, dev, threads, stream);
  return launch_awq_stg<MB, 2>(p, dev, threads, stream);
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

svdq_status svdq_awq_canonical_sizes(int64_t N, int64_t K, size_t sizes[5]) {
  if (!sizes || !awq_shape_ok(N, K)) return SVDQ_ERR_INVALID_ARG;
  sizes[0] = (size_t)K * 4;
  sizes[1] = (size_t)K * 4;
  sizes[2] = (size_t)N * (K / 2);
  sizes[3] = (size_t)N * (K / 64) * 2;
  sizes[4] = (size_t)N * 2;
  return SVDQ_OK;
}

svdq_status svdq_awq_prepare(const uint16_t* W, const uint16_t* bias, const uint16_t* X_calib, int64_t M_calib,
                             svdq_awq_canonical* out) {
  if (!W || !X_calib || !out || M_calib < 1 || !awq_shape_ok(out->N, out->K)) return SVDQ_ERR_INVALID_ARG;
  if (!out->s || !out->inv_s || !out->wcodes || !out->wscales || !out->bias) return SVDQ_ERR_INVALID_ARG;
  try {
    return (svdq_status)host::awq_prepare(W, bias, X_calib, M_calib, out);
  } catch (const std::bad_alloc&) {
    return SVDQ_ERR_OOM;
  }
}

svdq_status svdq_awq_packed_size(int64_t N, int64_t K, size_t* bytes) {
  if (!bytes || !awq_shape_ok(N, K)) return SVDQ_ERR_INVALID_ARG;
  *bytes = awq_blob_layout(N, K).total;
  return SVDQ_OK;
}

svdq_status svdq_awq_pack(const svdq_awq_canonical* c, void* blob_v, size_t blob_bytes) {
  if (!c || !blob_v || !awq_shape_ok(c->N, c->K)) return SVDQ_ERR_INVALID_ARG;
  if (!c->inv_s || !c->wcodes || !c->wscales) return SVDQ_ERR_INVALID_ARG;
  const int64_t N = c->N, K = c->K;
  const AwqBlob b = awq_blob_layout(N, K);
  if (blob_bytes < b.total) return SVDQ_ERR_INVALID_ARG;
  uint8_t* blob = (uint8_t*)blob_v;
  std::memset(blob, 0, b.total);
  std::memcpy(blob + b.inv_s, c->inv_s, (size_t)K * 4);
  float* bias = (float*)(blob + b.bias);
  for (int64_t n = 0; n < N; ++n) bias[n] = c->bias ? host::bf16_to_f32(c->bias[n]) : 0.f;
  const int64_t G = K / 64, ld = awq_scale_ld(K);
  for (int64_t n = 0; n < N; ++n) std::memcpy(blob + b.wscales + (size_t)n * ld * 2, c->wscales + n * G, (size_t)G * 2);
  std::memcpy(blob + b.wcodes, c->wcodes, (size_t)N * (K / 2));
  return SVDQ_OK;
}

svdq_status svdq_awq_layer_create(const void* dev_blob, size_t blob_bytes, int64_t N, int64_t K,
                                  svdq_awq_layer** out) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!dev_blob || !awq_shape_ok(N, K) || ((uintptr_t)dev_blob & 255)) return SVDQ_ERR_INVALID_ARG;
  const AwqBlob b = awq_blob_layout(N, K);
  if (blob_bytes < b.total) return SVDQ_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  const svdq_status st = svdq_device_check(dev);
  if (st != SVDQ_OK) return st;
  svdq_awq_layer* L = new (std::nothrow) svdq_awq_layer();
  if (!L) return SVDQ_ERR_OOM;
  const uint8_t* base = (const uint8_t*)dev_blob;
  L->N = N;
  L->K = K;
  L->device = dev;
  L->inv_s = (const float*)(base + b.inv_s);
  L->bias = (const float*)(base + b.bias);
  L->wscales = (const uint16_t*)(base + b.wscales);
  L->wcodes = base + b.wcodes;
  *out = L;
  return SVDQ_OK;
}

void svdq_awq_layer_destroy(svdq_awq_layer* layer) { delete layer; }

svdq_status svdq_awq_forward(const svdq_awq_layer* L, const void* X, int64_t M, void* Y, void* stream) {
  if (!L || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || ((uintptr_t)X & 15) || ((uintptr_t)Y & 15) || M > (1 << 30)) return SVDQ_ERR_INVALID_ARG;
  AwqParams p{};
  p.M = (int)M;
  p.N = (int)L->N;
  p.K = (int)L->K;
  p.x = (const uint16_t*)X;
  p.inv_s = L->inv_s;
  p.codes = L->wcodes;
  p.scales = L->wscales;
  p.bias = L->bias;
  p.y = (uint16_t*)Y;
  cudaStream_t s = (cudaStream_t)stream;
  for (int64_t m0 = 0; m0 < M; m0 += kAwqMaxMB) {
    p.m0 = (int)m0;
    const int64_t mb = (M - m0) < kAwqMaxMB ? (M - m0) : kAwqMaxMB;
    int st;
    st = (mb == 1) ? launch_awq<1>(p, L->device, s) : launch_awq<2>(p, L->device, s);
    if (st != SVDQ_OK) return (svdq_status)st;
  }
  return SVDQ_OK;
}

}  // extern "C"
