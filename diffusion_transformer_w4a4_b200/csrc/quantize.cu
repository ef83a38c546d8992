// K1: fused activation quantizer of the svdq_w4a4 layer.
//
// One pass over X [M,K] bf16 computes, per "Суть метода" ("Hugging Face встроила
// Nunchaku в Diffusers ..."): the smoothed activation x^ = x * (1/lambda)
// (outliers moved into the weights), its 4-bit group codes and scales (INT4:
// groups of 64, fp16 scale; NVFP4: blocks of 16, E4M3 scale under a static
// per-tensor scale g_x), and the 16-bit low-rank down-projection
// t = bf16( bf16(x^) L1 ) with fp32 accumulation.
//
// Work split: a CTA owns 128 token rows and one slice of K (the K range is cut
// into enough slices that about one CTA per SM is in flight).  Per 128-column
// chunk, with C quantizing warps (16, or 8 for ranks above 80):
//   warp C      TMA: the X tile [128 x 128], and a bulk copy of the chunk's
//               128 entries of 1/lambda, into a ring that the quantizing warps
//               release as soon as they have read it;
//   warp C+2    TMA: the matching L1^T slice [rank x 128] (two 64-column boxes,
//               128-byte swizzle) into a small ring released by the MMAs;
//   warps 0..C-1 quantize 128/C rows each (a lane holds 16 consecutive
//               elements: one NVFP4 block, or a quarter of a 64-element INT4
//               group whose maximum takes two warp shuffles; products in packed
//               f32x2), store codes and scales, and write bf16(x^) into a
//               128-byte-swizzled K-major tile;
//   warp C+1    issues tcgen05.mma kind::f16 (M = 128 tokens, N = rank, K = 16)
//               on that tile and the L1^T slice, accumulating the slice's part of
//               t in tensor memory.
// At the end the slice's fp32 partial of t leaves tensor memory; the last CTA of
// a row block to finish (arrival counter) adds the slices in a fixed order and
// writes bf16 t, so the result does not depend on scheduling.  HBM traffic is
// one read of X plus the codes, scales and t.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kRows = kQRows;    // 128
constexpr int kChunk = kQChunk;  // 128
// Quantizing warps per CTA: 16 (8 rows each) where the registers allow it, 8
// (16 rows each) for ranks above 80, whose fp32 partial of t takes a register per
// rank column; the three role warps follow them.
template <int RANK>
struct Roles {
  static constexpr int kConsumerWarps = RANK <= 80 ? 16 : 8;
  static constexpr int kRowsPerWarp = 128 / kConsumerWarps;
  static constexpr int kTmaWarp = kConsumerWarps;
  static constexpr int kMmaWarp = kConsumerWarps + 1;
  static constexpr int kL1Warp = kConsumerWarps + 2;
  static constexpr int kThreads = (kConsumerWarps + 3) * 32;
};
constexpr int kXTileBytes = kRows * kChunk * 2;  // 32 KiB
constexpr int kIlBytes = kChunk * 4;              // the chunk's 1/lambda slice
constexpr int kXStageBytes = kXTileBytes + kIlBytes;
// the X ring, padded so the 128-byte-swizzled tiles after it stay 1024-aligned
__host__ __device__ constexpr int xring_bytes(int xs) { return (xs * kXStageBytes + 1023) & ~1023; }
constexpr int kAHalfBytes = kRows * 128;         // 64 bf16 columns, 128B-swizzled
constexpr int kATileBytes = 2 * kAHalfBytes;     // 32 KiB
constexpr int kSmemBudget = 220 * 1024;

struct QParams {
  int M, K, xstages, lstages, nslices, nch, katoms;
  int64_t sld;  // INT4: row stride of the fp16 [K/64, sld] scales
  const float* inv_lambda;
  float g, inv_g, den;  // NVFP4 per-tensor scale, its exact inverse, 6*g
  // dynamic per-tensor scale: the first pass's per-CTA maxima of |x^| (else null),
  // and where this kernel leaves the resulting g_x for the GEMM
  const float* amax_slots;
  int nslots;
  float* g_out;
  uint8_t* codes;
  uint8_t* scales;
  uint16_t* t;
  float* tpart;  // [nslices, M, rank] when nslices > 1
  int* counters;
  int* status;
  unsigned long long limit;
};

__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

__device__ __forceinline__ uint32_t cvt_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// two floats -> two E4M3 bytes, `lo` in bits 0..7
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {  // c in [0, 0x7E]
  const uint32_t e = (c >> 3) & 0xF, m = c & 7;
  if (e == 0) return (float)m * (1.0f / 512.0f);
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <int RANK>
__host__ __device__ constexpr uint32_t tmem_cols() {
  return RANK <= 32 ? 32u : (RANK <= 64 ? 64u : 128u);
}

// bf16 t times a power of two (1 for the static scale): exact in binary32, and
// the product has the bf16 value's significand, so the rounding back is exact
__device__ __forceinline__ __nv_bfloat162 scale_t(__nv_bfloat162 h, float s) {
  return __floats2bfloat162_rn(__low2float(h) * s, __high2float(h) * s);
}

// The per-tensor NVFP4 scale for a tensor maximum: the smallest power of two g
// with 6 * 448 * g >= amax (1 for an all-zero tensor); every comparison is exact.
__device__ __forceinline__ float nvfp4_tensor_scale_dev(float amax) {
  if (!(amax > 0.f)) return 1.f;
  int e;
  frexpf(amax, &e);
  int k = e - 12;  // 2688 = 0.65625 * 2^12
  while (ldexpf(2688.f, k) < amax) ++k;
  while (ldexpf(2688.f, k - 1) >= amax) --k;
  return ldexpf(1.f, k);
}

template <int FMT, int RANK>
__global__ void __launch_bounds__(Roles<RANK>::kThreads, 1)
    k_quantize(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_l1, QParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int kConsumerWarps = Roles<RANK>::kConsumerWarps, kTmaWarp = Roles<RANK>::kTmaWarp;
  constexpr int kMmaWarp = Roles<RANK>::kMmaWarp, kL1Warp = Roles<RANK>::kL1Warp, kThreads = Roles<RANK>::kThreads;
  constexpr int kRowsPerWarp = Roles<RANK>::kRowsPerWarp;
  const int XS = p.xstages, LS = p.lstages;
  constexpr int kL1Bytes = RANK * kChunk * 2;  // two boxes of RANK rows x 128 B
  uint8_t* xring = smem;                          // [XS][X tile | 1/lambda slice]
  uint8_t* atile = xring + xring_bytes(XS);       // [2][kATileBytes] when RANK > 0 (1024-aligned)
  uint8_t* lring = atile + (RANK > 0 ? 2 * kATileBytes : 0);  // [LS][kL1Bytes]
  float* rtab = (float*)(lring + LS * kL1Bytes);  // [128] 1/e4m3
  uint64_t* full_x = (uint64_t*)(rtab + 128);
  uint64_t* empty_x = full_x + XS;
  uint64_t* full_l = empty_x + XS;
  uint64_t* empty_l = full_l + LS;
  uint64_t* xready = empty_l + LS;  // [2]
  uint64_t* xfree = xready + 2;     // [2]
  uint64_t* tdone = xfree + 2;
  uint32_t* tmem_slot = (uint32_t*)(tdone + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* ticket = abort_flag + 1;
  volatile int* decision = abort_flag + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rowblock = blockIdx.x, slice = blockIdx.y;
  const int m0 = rowblock * kRows;
  const int c_begin = (int)((int64_t)slice * p.nch / p.nslices);
  const int c_end = (int)((int64_t)(slice + 1) * p.nch / p.nslices);
  const int nchunks = c_end - c_begin;
  WaitCtl wc{abort_flag, p.status, p.limit};

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(&full_x[s], 1);
      mbar_init(&empty_x[s], kConsumerWarps);
    }
    for (int s = 0; s < LS; ++s) {
      mbar_init(&full_l[s], 1);
      mbar_init(&empty_l[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&xready[b], kConsumerWarps);
      mbar_init(&xfree[b], 1);
    }
    mbar_init(tdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (FMT == SVDQ_NVFP4_G16 && threadIdx.x < 128)  // exact reciprocals of the E4M3 values
    rtab[threadIdx.x] = (threadIdx.x == 0 || threadIdx.x == 0x7F) ? 0.f : __frcp_rn(e4m3_value(threadIdx.x));
  if constexpr (RANK > 0) {
    if (warp == kMmaWarp) {
      tmem_alloc(tmem_slot, tmem_cols<RANK>());
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // NVFP4 per-tensor scale: the prepared static one, or the dynamic one from the
  // first pass's maxima (then t is stored as t / g_x, an exact power-of-two
  // scaling, because the packed L2 carries only 1/g_w)
  float gs = p.g, inv_gs = p.inv_g, dens = p.den, tsc = 1.f;
  if (FMT == SVDQ_NVFP4_G16 && p.amax_slots != nullptr) {
    __shared__ float dred[kThreads / 32];
    float m = 0.f;
    for (int i = threadIdx.x; i < p.nslots; i += kThreads) m = fmaxf(m, p.amax_slots[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) dred[warp] = m;
    __syncthreads();
    m = dred[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) m = fmaxf(m, dred[i]);
    gs = nvfp4_tensor_scale_dev(m);
    inv_gs = 1.0f / gs;  // exact: a power of two
    dens = 6.0f * gs;
    tsc = inv_gs;
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.g_out = gs;
  }

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ X producer
    if (lane == 0) {
      prefetch_tmap(&map_x);
      int issued = 0;
      for (int i = 0; i < nchunks; ++i) {
        const int s = i % XS;
        if (!mbar_wait(&empty_x[s], ((i / XS) & 1) ^ 1, wc)) break;
        uint8_t* dst = xring + s * kXStageBytes;
        mbar_arrive_expect_tx(&full_x[s], kXStageBytes);
        tma_load_2d(&map_x, &full_x[s], dst, (c_begin + i) * kChunk, m0);
        bulk_load(dst + kXTileBytes, p.inv_lambda + (size_t)(c_begin + i) * kChunk, kIlBytes, &full_x[s]);
        issued = i + 1;
      }
      if (*abort_flag) {  // drain copies that are still in flight before leaving
        for (int i = (issued > XS ? issued - XS : 0); i < issued; ++i)
          mbar_wait_drain(&full_x[i % XS], (i / XS) & 1, p.limit);
      }
    }
  } else if (warp == kL1Warp) {
    // ------------------------------------------------------------ L1^T producer
    if constexpr (RANK > 0) {
      if (lane == 0) {
        prefetch_tmap(&map_l1);
        int issued = 0;
        for (int i = 0; i < nchunks; ++i) {
          const int s = i % LS;
          if (!mbar_wait(&empty_l[s], ((i / LS) & 1) ^ 1, wc)) break;
          const int k0 = (c_begin + i) * kChunk;
          uint8_t* dst = lring + s * kL1Bytes;
          mbar_arrive_expect_tx(&full_l[s], kL1Bytes);
          tma_load_2d(&map_l1, &full_l[s], dst, k0, 0);
          tma_load_2d(&map_l1, &full_l[s], dst + RANK * 128, k0 + 64, 0);
          issued = i + 1;
        }
        if (*abort_flag) {
          for (int i = (issued > LS ? issued - LS : 0); i < issued; ++i)
            mbar_wait_drain(&full_l[i % LS], (i / LS) & 1, p.limit);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if constexpr (RANK > 0) {
      if (lane == 0) {
        const uint32_t tmem = *tmem_slot;
        constexpr uint32_t idesc = idesc_bf16_f32(kRows, RANK);
        for (int i = 0; i < nchunks; ++i) {
          const int s = i % LS, buf = i & 1;
          if (!mbar_wait(&xready[buf], (i >> 1) & 1, wc)) break;
          if (!mbar_wait(&full_l[s], (i / LS) & 1, wc)) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(atile + buf * kATileBytes);
          const uint32_t b_addr = smem_u32(lring + s * kL1Bytes);
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            const uint32_t h = kk >> 2, koff = (kk & 3) * 32;
            mma_bf16(tmem, make_sdesc(a_addr + h * kAHalfBytes + koff, 16, 1024, LAYOUT_SW128),
                     make_sdesc(b_addr + h * RANK * 128 + koff, 16, 1024, LAYOUT_SW128), idesc,
                     (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&xfree[buf]);
          umma_commit(&empty_l[s]);
        }
        umma_commit(tdone);  // fires when every MMA above has completed
        if (*abort_flag) mbar_wait_drain(tdone, 0, p.limit);
      }
    }
  } else {
    // ------------------------------------------------------------ quantizing warps
    const int rsub = lane >> 3;  // row within the warp's 4-row step
    const int j = lane & 7;      // 16-column group within the chunk
    const int K2 = p.K / 2;
    for (int i = 0; i < nchunks; ++i) {
      const int s = i % XS, buf = i & 1;
      bool ok = mbar_wait(&full_x[s], (i / XS) & 1, wc);
      if constexpr (RANK > 0) ok = ok && mbar_wait(&xfree[buf], ((i >> 1) & 1) ^ 1, wc);
      if (ok) {
        const uint8_t* st = xring + s * kXStageBytes;
        const int k0 = (c_begin + i) * kChunk;
        const int kk0 = k0 + 16 * j;
        float il[16];
        const float4* ils = (const float4*)(st + kXTileBytes) + 4 * j;  // staged with the X tile
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 t4 = ils[q];
          il[4 * q] = t4.x;
          il[4 * q + 1] = t4.y;
          il[4 * q + 2] = t4.z;
          il[4 * q + 3] = t4.w;
        }
        uint8_t* at = atile + buf * kATileBytes + (j >> 2) * kAHalfBytes;
#pragma unroll 2
        for (int it = 0; it < kRowsPerWarp / 4; ++it) {
          const int row = warp * kRowsPerWarp + 4 * it + rsub;
          const int m = m0 + row;
          const uint4 r0 = *(const uint4*)(st + row * (kChunk * 2) + 32 * j);
          const uint4 r1 = *(const uint4*)(st + row * (kChunk * 2) + 32 * j + 16);
          const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
          float v[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            mul2(v[2 * e], v[2 * e + 1], il[2 * e], il[2 * e + 1]);
          }
          float amax = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
          uint2 packed = make_uint2(0u, 0u);
          if (FMT == SVDQ_NVFP4_G16) {
            const uint32_t sb = cvt_e4m3(__fdiv_rn(amax, dens));
            if (sb != 0) {
              // 1 / (e4m3(sb) * g) exactly: g is a power of two
              const float inv = rtab[sb] * inv_gs;
              float q0[8], q1[8];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                q0[2 * e] = v[2 * e];
                q0[2 * e + 1] = v[2 * e + 1];
                q1[2 * e] = v[8 + 2 * e];
                q1[2 * e + 1] = v[9 + 2 * e];
                mul2(q0[2 * e], q0[2 * e + 1], inv, inv);
                mul2(q1[2 * e], q1[2 * e + 1], inv, inv);
              }
              packed = make_uint2(cvt_e2m1x8(q0), cvt_e2m1x8(q1));
            }
            const int base = lane & ~3;  // 4 lanes = 64 columns = one scale-factor atom word
            const uint32_t s1 = __shfl_sync(0xffffffffu, sb, base + 1);
            const uint32_t s2 = __shfl_sync(0xffffffffu, sb, base + 2);
            const uint32_t s3 = __shfl_sync(0xffffffffu, sb, base + 3);
            if ((lane & 3) == 0 && m < p.M)
              *(uint32_t*)(p.scales + sf_offset(m, kk0 / 16, p.katoms, kSfAtomRows)) =
                  sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
          } else {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
            const float S16 = __half2float(s16);
            uint32_t qb[4] = {0u, 0u, 0u, 0u};
            if (S16 != 0.f) {
              const float inv = __frcp_rn(S16);
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                float y0 = v[e], y1 = v[e + 1];
                mul2(y0, y1, inv, inv);
                // clamp, then round half to even: (y + 1.5 * 2^23) - 1.5 * 2^23
                // is the nearest integer (a +0 for codes of zero), and E4M3
                // holds every integer of [-8, 7] exactly
                y0 = fminf(fmaxf(y0, -8.0f), 7.0f);
                y1 = fminf(fmaxf(y1, -8.0f), 7.0f);
                y0 = __fsub_rn(__fadd_rn(y0, 12582912.0f), 12582912.0f);
                y1 = __fsub_rn(__fadd_rn(y1, 12582912.0f), 12582912.0f);
                qb[e >> 2] |= cvt_e4m3x2(y0, y1) << (8 * (e & 2));
              }
            }
            if ((lane & 3) == 0 && m < p.M) ((__half*)p.scales)[(size_t)(kk0 / 64) * p.sld + m] = s16;
            if (m < p.M) *(uint4*)(p.codes + (size_t)m * p.K + kk0) = make_uint4(qb[0], qb[1], qb[2], qb[3]);
          }
          if (FMT == SVDQ_NVFP4_G16 && m < p.M) *(uint2*)(p.codes + (size_t)m * K2 + kk0 / 2) = packed;
          if constexpr (RANK > 0) {
            uint32_t b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
              b[e] = *(uint32_t*)&h;
            }
            const int c0 = 2 * (j & 3);
            *(uint4*)(at + row * 128 + ((c0 ^ (row & 7)) << 4)) = make_uint4(b[0], b[1], b[2], b[3]);
            *(uint4*)(at + row * 128 + (((c0 + 1) ^ (row & 7)) << 4)) = make_uint4(b[4], b[5], b[6], b[7]);
          }
        }
      }
      if constexpr (RANK > 0) fence_proxy_async_smem();  // x^ tile -> tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty_x[s]);  // the X tile has been read
        if constexpr (RANK > 0) mbar_arrive(&xready[buf]);
      }
    }

    if constexpr (RANK > 0) {
      if (warp < 4) {
        // the slice's partial t leaves tensor memory (warp w owns lanes 32w..32w+31)
        mbar_wait(tdone, 0, wc);
        tc_fence_after();
        const int row = 32 * warp + lane;
        const int m = m0 + row;
        const uint32_t tl = *tmem_slot + ((uint32_t)(32 * warp) << 16);
        float acc[RANK];
#pragma unroll
        for (int c = 0; c < RANK / 16; ++c) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(tl + 16 * c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[16 * c + j] = __uint_as_float(r[j]);
        }
        // one go/no-go decision for all 128 threads, so every barrier below is uniform
        named_bar_sync(2, 128);
        if (threadIdx.x == 0) *decision = *abort_flag ? 0 : 1;
        named_bar_sync(2, 128);
        if (*decision) {
          if (p.nslices == 1) {
            if (m < p.M) {
#pragma unroll
              for (int j = 0; j < RANK; j += 2) {
                __nv_bfloat162 h = scale_t(__floats2bfloat162_rn(acc[j], acc[j + 1]), tsc);
                *(uint32_t*)(p.t + (size_t)m * RANK + j) = *(uint32_t*)&h;
              }
            }
          } else {
            if (m < p.M) {
              float* dst = p.tpart + ((size_t)slice * p.M + m) * RANK;
#pragma unroll
              for (int j = 0; j < RANK; j += 4)
                *(float4*)(dst + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
            }
            __threadfence();
            named_bar_sync(2, 128);
            if (threadIdx.x == 0) *ticket = atomicAdd(p.counters + rowblock, 1);
            named_bar_sync(2, 128);
            if (*ticket == p.nslices - 1) {  // last slice of this row block: fixed-order sum
              __threadfence();
              if (m < p.M) {
#pragma unroll
                for (int j = 0; j < RANK; j += 4) {
                  float4 sum = __ldcg((const float4*)(p.tpart + (size_t)m * RANK + j));
                  for (int sl = 1; sl < p.nslices; ++sl) {
                    const float4 v = __ldcg((const float4*)(p.tpart + ((size_t)sl * p.M + m) * RANK + j));
                    sum.x += v.x;
                    sum.y += v.y;
                    sum.z += v.z;
                    sum.w += v.w;
                  }
                  __nv_bfloat162 h0 = scale_t(__floats2bfloat162_rn(sum.x, sum.y), tsc);
                  __nv_bfloat162 h1 = scale_t(__floats2bfloat162_rn(sum.z, sum.w), tsc);
                  *(uint2*)(p.t + (size_t)m * RANK + j) = make_uint2(*(uint32_t*)&h0, *(uint32_t*)&h1);
                }
              }
              if (threadIdx.x == 0) p.counters[rowblock] = 0;  // ready for the next call
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (RANK > 0) {
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(*tmem_slot, tmem_cols<RANK>());
    }
  }
}

template <int FMT, int RANK>
int launch_rank(const CUtensorMap& mx, const CUtensorMap& ml1, const QParams& p, int64_t M, cudaStream_t stream) {
  constexpr int kL1Bytes = RANK * kChunk * 2;
  constexpr int kFixed = (RANK > 0 ? 2 * kATileBytes : 0) + 512 + 512;
  QParams q = p;
  q.lstages = RANK > 0 ? (RANK <= 64 ? 3 : 2) : 0;
  int XS = 5;
  while (XS > 2 && xring_bytes(XS) + kFixed + q.lstages * kL1Bytes > kSmemBudget) --XS;
  q.xstages = XS;
  const size_t smem = 1024 + (size_t)xring_bytes(XS) + (size_t)q.lstages * kL1Bytes + kFixed;
  auto kern = k_quantize<FMT, RANK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  const dim3 grid((unsigned)((M + kRows - 1) / kRows), (unsigned)p.nslices);
  kern<<<grid, Roles<RANK>::kThreads, smem, stream>>>(mx, ml1, q);
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

template <int FMT>
int launch_fmt(const CUtensorMap& mx, const CUtensorMap& ml1, const QParams& p, int64_t M, int rank,
               cudaStream_t stream) {
  switch (rank) {
    case 0: return launch_rank<FMT, 0>(mx, ml1, p, M, stream);
    case 16: return launch_rank<FMT, 16>(mx, ml1, p, M, stream);
    case 32: return launch_rank<FMT, 32>(mx, ml1, p, M, stream);
    case 48: return launch_rank<FMT, 48>(mx, ml1, p, M, stream);
    case 64: return launch_rank<FMT, 64>(mx, ml1, p, M, stream);
    case 80: return launch_rank<FMT, 80>(mx, ml1, p, M, stream);
    case 96: return launch_rank<FMT, 96>(mx, ml1, p, M, stream);
    case 112: return launch_rank<FMT, 112>(mx, ml1, p, M, stream);
    case 128: return launch_rank<FMT, 128>(mx, ml1, p, M, stream);
    default: return SVDQ_ERR_INVALID_ARG;
  }
}

}  // namespace

int launch_quantize(const svdq_layer* L, const void* X, int64_t M, uint8_t* ws, const Workspace& w,
                    cudaStream_t stream) {
  CUtensorMap mx;
  int st = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)L->K, (uint64_t)M,
                          (uint64_t)L->K * 2, kChunk, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != SVDQ_OK) return st;
  QParams p{};
  p.M = (int)M;
  p.K = (int)L->K;
  p.nch = (int)(L->K / kChunk);
  p.nslices = w.nslices;
  p.katoms = (int)(L->K / 64);
  p.sld = int4_scale_ld(M);
  p.inv_lambda = L->inv_lambda;
  p.g = L->g_x;
  p.inv_g = 1.0f / L->g_x;  // exact: g_x is a power of two
  p.den = 6.0f * L->g_x;
  if (L->dyn_gx) {  // the first pass (k_act_amax) ran just before on this stream
    int gx = 0, gy = 0;
    act_amax_grid(M, L->K, &gx, &gy);
    p.amax_slots = (const float*)(ws + w.amax);
    p.nslots = gx * gy;
    p.g_out = (float*)(ws + w.status + 4);
    p.g = p.inv_g = p.den = 0.f;  // set in the kernel
  }
  p.codes = ws + w.codes;
  p.scales = ws + w.scales;
  p.t = (uint16_t*)(ws + w.t);
  p.tpart = (float*)(ws + w.tpart);
  p.status = (int*)(ws + w.status);
  p.counters = (int*)(ws + w.status + 16);
  p.limit = wait_limit_cycles();
  if (L->fmt == SVDQ_NVFP4_G16) return launch_fmt<SVDQ_NVFP4_G16>(mx, L->map_l1, p, M, L->rank, stream);
  return launch_fmt<SVDQ_INT4_G64>(mx, L->map_l1, p, M, L->rank, stream);
}

}  // namespace svdq
