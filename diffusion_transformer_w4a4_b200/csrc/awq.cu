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
// k_awq_gemv: a thread owns one 32-code (16-byte) chunk of K and keeps that
// chunk of x^ = f32(x) * inv_s for up to two token rows in registers; it reads
// the matching 16 bytes of several weight rows from a shared-memory ring that a
// producer warp fills with bulk copies of consecutive rows.  The device copy of
// the codes is offset binary (u = n + 8 in [0, 15] for the two's complement
// nibble n).  A code becomes a binary32 with one logic operation, u masked into
// the mantissa of 1.0 at bit p, and an exact packed subtraction of 1 leaves
// u 2^(p-23); the x^ chunk is pre-scaled by 2^(23-p) once, so the packed FMAs
// accumulate sum_e u_e x^_e directly (no cancelling offset), and a chunk's sum
// is that minus 8 sum_e x^_e.  The partial times its group scale is reduced over
// the thread's row group (warp shuffles, then shared memory).  The pre-scaling
// by at most 2^15 needs |x^| < 2^113.  The decode's integer work (10 logic and
// shift operations per 8 codes on the half-rate ALU pipe) rather than HBM is
// the first limit at these shapes.
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
  int* status;
};

namespace svdq {
namespace {

constexpr int kAwqRpt = 4;           // weight rows per row group and batch
constexpr int kAwqMaxMB = 2;         // token rows per launch (their x^ chunks live in registers)
constexpr int kAwqMaxStages = 6;     // ring depth bound
constexpr int kAwqConsumers = 384;   // consumer threads per CTA, at most
constexpr int kAwqMaxThreads = kAwqConsumers + 32;  // plus the producer warp
constexpr size_t kAwqRingBudget = 110 * 1024;  // ring bytes per CTA: two CTAs per SM
// 2^(23 - p) for the mantissa position p at which code k of a 32-bit word is decoded
__constant__ float kAwqPrescale[8] = {32768.f, 2048.f, 32768.f, 2048.f, 128.f, 32768.f, 2048.f, 128.f};

struct AwqBlob {
  size_t inv_s, bias, wscales, wcodes, status, total;
};

// fp16 group scales per blob row: K/64 rounded up to a multiple of 8, so a run
// of rows is a whole number of 16-byte units for the bulk copies
__host__ __device__ inline int64_t awq_scale_ld(int64_t K) { return (K / 64 + 7) / 8 * 8; }

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
  b.status = o;  // int32 written by the kernel on a device-side error
  o = up(o + 16);
  b.total = o;
  return b;
}

bool awq_shape_ok(int64_t N, int64_t K) { return N >= 1 && K >= 64 && K % 64 == 0 && K <= 12288 && N <= (1 << 30); }

struct AwqParams {
  int M, N, K, m0;
  int T;       // threads per row group: K/32 rounded up to whole warps
  int G;       // row groups per CTA (a power of two, at most 8)
  int stages;  // ring depth
  int xs_off;  // byte offset of the x^ staging area (the ring's tail, reused once set up)
  int* status;
  unsigned long long limit;
  const uint16_t* x;
  const float* inv_s;
  const uint8_t* codes;
  const uint16_t* scales;
  const float* bias;
  uint16_t* y;
};

template <int S>
__device__ __forceinline__ uint32_t shl_b32(uint32_t v) {
  uint32_t r;
  asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "n"(S));
  return r;
}
template <int S>
__device__ __forceinline__ uint32_t shr_b32(uint32_t v) {
  uint32_t r;
  asm("shr.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "n"(S));
  return r;
}
// binary32 with bits (w & mask) over the encoding of 1.0: one lop3, (a & b) | c
__device__ __forceinline__ float mant_one(uint32_t w, uint32_t mask) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(mask), "r"(0x3F800000u));
  return __uint_as_float(r);
}

// Persistent and warp-specialized.  The CTA's last warp is the producer: its
// lane 0 fills a ring of `stages` batches, each R = G * kAwqRpt consecutive
// weight rows (the rows' packed codes and their scale rows, two bulk copies,
// both contiguous), completing on per-stage "full" mbarriers.  The other warps
// form G row groups of T threads: thread t of a group owns the 32-code chunk t
// of K, with that chunk of x^ = f32(x) * inv_s for each token row in registers,
// and group g computes rows g*kAwqRpt .. g*kAwqRpt + kAwqRpt - 1 of every batch.
// A group reduces its partial sums over its warps (shuffles, then shared memory
// and a named barrier of its own), releases the stage on the stage's "empty"
// mbarrier (one arrival per group) and its first threads add the bias and store
// y.  Groups never wait for one another.  Waits are bounded; a group whose
// wait fails leaves as a whole (the named barrier reduces the outcome), the
// producer drains its copies, and the status word records the error.
template <int MB>
__global__ void __launch_bounds__(kAwqMaxThreads) k_awq_gemv(const __grid_constant__ AwqParams p) {
  extern __shared__ __align__(128) uint8_t awq_smem[];  // [stages][R scale rows] then [stages][R rows of codes]
  __shared__ float red[2][kAwqConsumers / 32][kAwqRpt * MB];  // per-warp partials, by batch parity
  __shared__ uint64_t full[kAwqMaxStages], empty[kAwqMaxStages];
  __shared__ uint64_t xs_free;  // every consumer warp has its x^ chunk in registers
  __shared__ int abort_flag;
  const int tid = threadIdx.x, lane = tid & 31;
  const int T = p.T, G = p.G, S = p.stages;
  const int R = G * kAwqRpt;
  const int nbatch = (p.N + R - 1) / R;
  const size_t row_bytes = (size_t)p.K / 2, ld = (size_t)awq_scale_ld(p.K);
  const size_t wstage = (size_t)R * row_bytes, sstage = (size_t)R * ld * 2;
  uint8_t* sring = awq_smem;
  uint8_t* wring = awq_smem + (size_t)S * sstage;
  WaitCtl wc{&abort_flag, p.status, p.limit};

  if (tid == 0) {
    for (int j = 0; j < S; ++j) {
      mbar_init(&full[j], 1);
      mbar_init(&empty[j], G);
    }
    mbar_init(&xs_free, (G * T) >> 5);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (tid == 0) pdl_launch_dependents();  // the next layer's CTAs may start as SMs free up

  if (tid >= G * T) {  // ---------------------------------------- producer
    if (lane != 0) return;
    // This kernel may start before the previous one on the stream has finished
    // (programmatic dependent launch): warm L2 with the first batches' weights,
    // which is only a hint, then wait for the previous kernel before copying.
    for (int b = blockIdx.x, jj = 0; b < nbatch && jj < S; b += gridDim.x, ++jj) {
      const int rows = (p.N - b * R) < R ? (p.N - b * R) : R;
      prefetch_l2_bulk(p.codes + (size_t)b * R * row_bytes, (uint32_t)(rows * row_bytes));
      prefetch_l2_bulk(p.scales + (size_t)b * R * ld, (uint32_t)(rows * ld * 2));
    }
    pdl_wait();
    int s = 0, j = 0;
    uint32_t ph = 0;  // parity of the current fill of stage s
    const size_t xs_lo = (size_t)p.xs_off;
    for (int b = blockIdx.x; b < nbatch; b += gridDim.x, ++j) {
      if (j >= S && !mbar_wait(&empty[s], ph ^ 1, wc)) break;  // the previous fill's batch is released
      if (j < S && S * sstage + (s + 1) * wstage > xs_lo &&
          !mbar_wait(&xs_free, 0, wc))
        break;  // a first fill that overwrites the x^ staging area waits until it is read
      const int rows = (p.N - b * R) < R ? (p.N - b * R) : R;
      mbar_arrive_expect_tx(&full[s], (uint32_t)(rows * (row_bytes + ld * 2)));
      bulk_load(wring + s * wstage, p.codes + (size_t)b * R * row_bytes, (uint32_t)(rows * row_bytes), &full[s]);
      bulk_load(sring + s * sstage, p.scales + (size_t)b * R * ld, (uint32_t)(rows * ld * 2), &full[s]);
      if (++s == S) {
        s = 0;
        ph ^= 1;
      }
    }
    if (abort_flag) {  // the ring must not be left with copies in flight
      for (int st = 0; st < S && st < j; ++st) mbar_wait_drain(&full[st], ((j - 1 - st) / S) & 1, p.limit);
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  const int g = tid / T, t = tid - g * T;
  const int warp = tid >> 5, wbase = g * (T >> 5);
  const int nchunk = p.K >> 5;
  const bool active = t < nchunk;

  pdl_wait();  // x and y belong to the stream's order
  // x^ = f32(x) * inv_s for the CTA's token rows, computed once with coalesced
  // loads into the ring's tail; float4 q of chunk c of token m sits at unit
  // m*K/4 + c*8 + (q ^ (c & 7)), so that each thread's reads of its own chunk
  // are free of bank conflicts
  {
    float4* xs = (float4*)(awq_smem + p.xs_off);
    const int kq = p.K >> 2;
    for (int i = tid; i < MB * kq; i += G * T) {
      const int m = i / kq, w = i - m * kq;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p.m0 + m < p.M) {
        const float4 is = __ldg((const float4*)p.inv_s + w);
        const uint2 xv = __ldg((const uint2*)(p.x + (size_t)(p.m0 + m) * p.K) + w);
        o.x = __uint_as_float(xv.x << 16) * is.x;  // binary32 products, as in the smoothing step
        o.y = __uint_as_float(xv.x & 0xFFFF0000u) * is.y;
        o.z = __uint_as_float(xv.y << 16) * is.z;
        o.w = __uint_as_float(xv.y & 0xFFFF0000u) * is.w;
      }
      const int c = w >> 3, q = w & 7;
      xs[m * kq + c * 8 + (q ^ (c & 7))] = o;
    }
  }
  named_bar_sync(9, G * T);  // the consumers only (barriers 1..8 belong to the row groups)
  float2 xh[MB][16];  // pairs (x^_2j, x^_2j+1) of the chunk, pre-scaled for the decode
  float xsum[MB];
  {
    const float4* xs = (const float4*)(awq_smem + p.xs_off);
    const int kq = p.K >> 2;
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      xsum[m] = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = active ? xs[m * kq + t * 8 + (q ^ (t & 7))] : make_float4(0.f, 0.f, 0.f, 0.f);
        xsum[m] += v.x;
        xsum[m] += v.y;
        xsum[m] += v.z;
        xsum[m] += v.w;
        // pre-scale by 2^(23 - p) for the mantissa position p of each code's
        // nibble in the decode below (exact: powers of two)
        xh[m][2 * q] = make_float2(v.x * kAwqPrescale[(4 * q) & 7], v.y * kAwqPrescale[(4 * q + 1) & 7]);
        xh[m][2 * q + 1] = make_float2(v.z * kAwqPrescale[(4 * q + 2) & 7], v.w * kAwqPrescale[(4 * q + 3) & 7]);
      }
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&xs_free);

  const int fr = t / MB, fm = t - (t / MB) * MB;  // finishing thread t: group row fr, token fm
  int s = 0, j = 0;
  uint32_t ph = 0;
  for (int b = blockIdx.x; b < nbatch; b += gridDim.x, ++j) {
    const int n0 = b * R + g * kAwqRpt;  // this group's first row
    float bias_v = 0.f;
    if (t < kAwqRpt * MB && n0 + fr < p.N) bias_v = __ldg(p.bias + n0 + fr);
    const bool ok = mbar_wait(&full[s], ph, wc);
    float part[kAwqRpt][MB];
#pragma unroll
    for (int r = 0; r < kAwqRpt; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) part[r][m] = 0.f;
    if (ok) {
      const uint8_t* ws = wring + s * wstage + (size_t)g * kAwqRpt * row_bytes;
      const uint16_t* ss = (const uint16_t*)(sring + s * sstage) + (size_t)g * kAwqRpt * ld;
#pragma unroll
      for (int r = 0; r < kAwqRpt; ++r) {
        if (!active || n0 + r >= p.N) continue;
        const uint4 wv = *(const uint4*)(ws + r * row_bytes + 16 * t);
        const float sc = __half2float(__ushort_as_half(ss[r * ld + (t >> 1)]));
        const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
        float2 acc[MB];  // even- and odd-position codes, one packed FMA per pair
#pragma unroll
        for (int m = 0; m < MB; ++m) acc[m] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          // code k of word q (bits 4k..4k+3, offset binary u) is masked into the
          // mantissa of 1.0 at bit p = 8, 12, 8, 12, 16, 8, 12, 16 (from the word
          // shifted left by 8 for k < 2, as is for k = 2..4, shifted right by 12
          // for k > 4): one logic operation makes 1 + u 2^(p-23), and subtracting
          // 1 leaves u 2^(p-23) exactly, which meets the pre-scaled x^
          // (written as explicit shifts and 3-input logic operations, so that the
          // shifted words are computed once rather than re-derived per code)
          const uint32_t v = wr[q], a = shl_b32<8>(v), c = shr_b32<12>(v);
          const float2 m1 = make_float2(-1.f, -1.f);
          const float2 g01 = __fadd2_rn(make_float2(mant_one(a, 0x00F00u), mant_one(a, 0x0F000u)), m1);
          const float2 g23 = __fadd2_rn(make_float2(mant_one(v, 0x00F00u), mant_one(v, 0x0F000u)), m1);
          const float2 g45 = __fadd2_rn(make_float2(mant_one(v, 0xF0000u), mant_one(c, 0x00F00u)), m1);
          const float2 g67 = __fadd2_rn(make_float2(mant_one(c, 0x0F000u), mant_one(c, 0xF0000u)), m1);
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            acc[m] = __ffma2_rn(g01, xh[m][4 * q], acc[m]);
            acc[m] = __ffma2_rn(g23, xh[m][4 * q + 1], acc[m]);
            acc[m] = __ffma2_rn(g45, xh[m][4 * q + 2], acc[m]);
            acc[m] = __ffma2_rn(g67, xh[m][4 * q + 3], acc[m]);
          }
        }
        // sum_e (u_e - 8) x^_e = sum_e u_e x^_e - 8 sum_e x^_e
#pragma unroll
        for (int m = 0; m < MB; ++m) part[r][m] = sc * fmaf(-8.f, xsum[m], acc[m].x + acc[m].y);
      }
    }
#pragma unroll
    for (int r = 0; r < kAwqRpt; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        float v = part[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[j & 1][warp][r * MB + m] = v;
      }
    if (!named_bar_and(1 + g, T, ok)) break;  // the group's reads of stage s and its partials are done
    if (t == 0) mbar_arrive(&empty[s]);
    if (t < kAwqRpt * MB) {
      float v = 0.f;
      for (int w = 0; w < (T >> 5); ++w) v += red[j & 1][wbase + w][t];
      const int n = n0 + fr;
      if (n < p.N && p.m0 + fm < p.M)
        p.y[(size_t)(p.m0 + fm) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v + bias_v));
    }
    if (++s == S) {
      s = 0;
      ph ^= 1;
    }
  }
}

// Launch shape for a K: row groups, ring depth and dynamic shared memory.
struct AwqShape {
  int T, G, stages, xs_off;
  size_t smem;
};
AwqShape awq_shape(int K, int MB) {
  AwqShape a{};
  a.T = ((K / 32) + 31) / 32 * 32;
  a.G = 1;
  while (a.G < 8 && 2 * a.G * a.T <= kAwqConsumers) a.G *= 2;
  const size_t stage = (size_t)a.G * kAwqRpt * ((size_t)K / 2 + (size_t)awq_scale_ld(K) * 2);
  size_t st = kAwqRingBudget / stage;
  a.stages = (int)(st < 2 ? 2 : (st > (size_t)kAwqMaxStages ? (size_t)kAwqMaxStages : st));
  const size_t ring = (size_t)a.stages * stage, xs = (size_t)MB * K * 4;
  a.xs_off = ring >= xs ? (int)((ring - xs) / 128 * 128) : 0;
  a.smem = ring > (size_t)a.xs_off + xs ? ring : (size_t)a.xs_off + xs;
  return a;
}

// CTAs per SM for one kernel variant and K, found once per device and cached:
// the attribute call and the occupancy query cost microseconds of host time
// that would otherwise precede every launch.  The dynamic shared-memory
// attribute belongs to the kernel, not to a launch, so it is set once to the
// ring budget, which bounds every K's ring.
template <int MB>
int awq_blocks_per_sm(int dev, const AwqShape& a, int K) {
  static std::mutex mu;
  static int cache[64][12288 / 64 + 1] = {};  // [device][K / 64]
  static bool attr_set[64] = {};
  if (dev < 0 || dev >= 64 || K < 64 || K > 12288 || a.smem > kAwqRingBudget) return -1;
  std::lock_guard<std::mutex> lock(mu);
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(k_awq_gemv<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAwqRingBudget) !=
        cudaSuccess)
      return -1;
    attr_set[dev] = true;
  }
  int& c = cache[dev][K / 64];
  if (c == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_awq_gemv<MB>, a.G * a.T + 32, a.smem) !=
            cudaSuccess ||
        per_sm < 1)
      return -1;
    c = per_sm;
  }
  return c;
}

template <int MB>
int launch_awq(AwqParams p, int dev, cudaStream_t stream) {
  const AwqShape a = awq_shape(p.K, MB);
  p.T = a.T;
  p.xs_off = a.xs_off;
  p.G = a.G;
  p.stages = a.stages;
  const int per_sm = awq_blocks_per_sm<MB>(dev, a, p.K);
  if (per_sm < 1) return SVDQ_ERR_CUDA;
  const int R = a.G * kAwqRpt;
  const int nbatch = (p.N + R - 1) / R;
  int grid = device_sm_count(dev) * per_sm;
  if (grid > nbatch) grid = nbatch;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(a.G * a.T + 32);
  cfg.dynamicSmemBytes = a.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait in the kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_awq_gemv<MB>, p) != cudaSuccess) return SVDQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
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
  // offset binary on the device: nibble n -> n ^ 8 = n + 8 (mod 16), per nibble
  const uint8_t* src = c->wcodes;
  uint8_t* dst = blob + b.wcodes;
  for (size_t i = 0, e = (size_t)N * (K / 2); i < e; ++i) dst[i] = src[i] ^ 0x88u;
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
  svdq_status st = svdq_device_check(dev);
  if (st != SVDQ_OK) return st;
  st = (svdq_status)check_blob_pointer(dev_blob, dev);
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
  L->status = (int*)(base + b.status);
  *out = L;
  return SVDQ_OK;
}

void svdq_awq_layer_destroy(svdq_awq_layer* layer) { delete layer; }

svdq_status svdq_awq_read_status(const svdq_awq_layer* L, int* device_status) {
  if (!L || !device_status) return SVDQ_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpy(&v, L->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  *device_status = v;
  return SVDQ_OK;
}

svdq_status svdq_awq_forward(const svdq_awq_layer* L, const void* X, int64_t M, void* Y, void* stream) {
  if (!L || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || ((uintptr_t)X & 15) || ((uintptr_t)Y & 15) || M > (1 << 30)) return SVDQ_ERR_INVALID_ARG;
  if (const int e = require_current_device(L->device); e != SVDQ_OK) return (svdq_status)e;
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
  p.status = L->status;
  p.limit = wait_limit_cycles();
  cudaStream_t s = (cudaStream_t)stream;
  NvtxRange range("svdq/awq_gemv");
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
