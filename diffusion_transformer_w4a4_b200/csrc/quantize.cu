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
// into enough slices that about one CTA per SM is in flight).  Per 256-column
// chunk, with C quantizing warps (16, or 8 for ranks above 80):
//   warps 0..C-1 load their rows of the chunk straight from global memory into
//               registers (16 lanes cover a row's 512-byte run, so a load
//               instruction reads two whole runs; the 1/lambda entries come from
//               the L2-resident weight blob), then quantize them: a lane holds
//               16 consecutive elements (one NVFP4 block, or a quarter of a
//               64-element INT4 group whose maximum takes two warp shuffles;
//               products in packed f32x2), stores codes and scales, and writes
//               bf16(x^) into a 128-byte-swizzled K-major tile;
//   warp C+1    TMA: the matching L1^T slice [rank x 256] (four 64-column
//               boxes, 128-byte swizzle) into a small ring released by the MMAs;
//   warp C      issues tcgen05.mma kind::f16 (M = 128 tokens, N = rank, K = 16)
//               on that tile and the L1^T slice, accumulating the slice's part of
//               t in tensor memory.
// Loading through registers rather than a TMA ring keeps one independent stream
// per warp in flight (measured on the FLUX MLP shapes: 16 warp streams of
// 512-byte runs read X at about 4.1 TB/s, one TMA ring per SM at about 3.6 TB/s).
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
constexpr int kChunk = kQChunk;  // 256
// Quantizing warps per CTA: 16 (8 rows each) where the registers allow it, 8
// (16 rows each) for ranks above 80, whose fp32 partial of t takes a register per
// rank column; the two role warps follow them.
template <int RANK>
struct Roles {
  static constexpr int kConsumerWarps = RANK <= 80 ? 16 : 8;
  static constexpr int kRowsPerWarp = 128 / kConsumerWarps;
  static constexpr int kMmaWarp = kConsumerWarps;
  static constexpr int kL1Warp = kConsumerWarps + 1;
  static constexpr int kThreads = (kConsumerWarps + 2) * 32;
};
constexpr int kABlockBytes = kRows * 128;       // 64 bf16 columns, 128B-swizzled
constexpr int kATileBytes = (kChunk / 64) * kABlockBytes;  // 64 KiB
constexpr int kSmemBudget = 220 * 1024;

struct QParams {
  int M, K, lstages, nslices, nch, katoms;
  int64_t sld;  // INT4: row stride of the fp16 [K/64, sld] scales
  const uint16_t* x;  // [M, K] bf16
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
  // buffer extents in bytes, for the debug variant's bounds checks
  size_t x_bytes, il_bytes, codes_bytes, scales_bytes, t_bytes, tpart_bytes, cnt_bytes;
};

// eight floats (as four pairs, element order a.x a.y b.x b.y ...) -> eight E2M1
// codes, element 2i in the low nibble of byte i
__device__ __forceinline__ uint32_t cvt_e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
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
    k_quantize(const __grid_constant__ CUtensorMap map_l1, QParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int kConsumerWarps = Roles<RANK>::kConsumerWarps;
  constexpr int kMmaWarp = Roles<RANK>::kMmaWarp, kL1Warp = Roles<RANK>::kL1Warp, kThreads = Roles<RANK>::kThreads;
  constexpr int kRowsPerWarp = Roles<RANK>::kRowsPerWarp;
  const int LS = p.lstages;
  constexpr int kL1Bytes = RANK * kChunk * 2;  // kChunk/64 boxes of RANK rows x 128 B
  uint8_t* atile = smem;                                      // [2][kATileBytes] when RANK > 0
  uint8_t* lring = atile + (RANK > 0 ? 2 * kATileBytes : 0);  // [LS][kL1Bytes]
  float* rtab = (float*)(lring + LS * kL1Bytes);              // [128] 1/e4m3
  uint64_t* full_l = (uint64_t*)(rtab + 128);
  uint64_t* empty_l = full_l + 2;
  uint64_t* xready = empty_l + 2;  // [2]
  uint64_t* xfree = xready + 2;    // [2]
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
  if (threadIdx.x == 0) pdl_launch_dependents();  // the GEMM's prologue may start as SMs free up

  // NVFP4 per-tensor scale: the prepared static one, or the dynamic one from the
  // first pass's maxima (then t is stored as t / g_x, an exact power-of-two
  // scaling, because the packed L2 carries only 1/g_w)
  float inv_gs = p.inv_g, dens = p.den, tsc = 1.f;
  if (FMT == SVDQ_NVFP4_G16 && p.amax_slots != nullptr) {
    pdl_wait();  // the first pass's maxima
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
    const float gs = nvfp4_tensor_scale_dev(m);
    inv_gs = 1.0f / gs;  // exact: a power of two
    dens = 6.0f * gs;
    tsc = inv_gs;
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.g_out = gs;
  }

  if (warp == kL1Warp) {
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
#pragma unroll
          for (int h = 0; h < kChunk / 64; ++h) tma_load_2d(&map_l1, &full_l[s], dst + h * RANK * 128, k0 + 64 * h, 0);
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
            mma_bf16(tmem, make_sdesc(a_addr + h * kABlockBytes + koff, 16, 1024, LAYOUT_SW128),
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
    // A lane owns 16 consecutive columns (one NVFP4 block, a quarter of an INT4
    // group) of two rows... of the warp's rows: 16 lanes cover a row's 256-column
    // chunk, so a warp reads two rows (two 512-byte runs) per load instruction.
    // Each warp loads its rows of a chunk straight from global memory into
    // registers (no staging), then quantizes them.
    pdl_wait();  // X and the workspace belong to the stream's order
    const int rsub = lane >> 4;  // row within the warp's 2-row step
    const int j = lane & 15;     // 16-column block within the chunk
    constexpr int ITS = kRowsPerWarp / 2;
    // Row step `it` handles row rbase + 2 it.  Its code, scale and x^-tile
    // offsets are affine in `it` (a warp's rows stay inside one 32-row group of
    // the scale-factor atom), so only the step-0 values are kept.
    const int rbase = warp * kRowsPerWarp + rsub;
    const int64_t mbase = m0 + rbase;
    const int kk0 = c_begin * kChunk + 16 * j;
    const size_t code_row = FMT == SVDQ_NVFP4_G16 ? (size_t)p.K / 2 : (size_t)p.K;
    const size_t coff0 = (size_t)mbase * code_row + (FMT == SVDQ_NVFP4_G16 ? kk0 / 2 : kk0);
    const size_t soff0 = FMT == SVDQ_NVFP4_G16 ? sf_offset(mbase, kk0 / 16, p.katoms, kSfAtomRows)
                                               : ((size_t)(kk0 / 64) * p.sld + mbase) * 2;
    constexpr int kScaleRowStep = FMT == SVDQ_NVFP4_G16 ? 2 * 16 : 2 * 2;  // bytes per 2 rows
    const int c0 = 2 * (j & 3);
    const int ablk = (j >> 2) * kABlockBytes;
    const float* ilp = p.inv_lambda + kk0;
    constexpr size_t kCodeStep = FMT == SVDQ_NVFP4_G16 ? kChunk / 2 : kChunk;
    const size_t scale_step = FMT == SVDQ_NVFP4_G16 ? (kChunk / 64) * kSfAtomBytes : (kChunk / 32) * (size_t)p.sld;
    for (int i = 0; i < nchunks; ++i) {
      const int buf = i & 1;
      // this chunk's rows and 1/lambda, straight into registers (rows past M read row 0)
      uint4 xr[ITS][2];
#pragma unroll
      for (int it = 0; it < ITS; ++it) {
        const int64_t m = mbase + 2 * it;
        const int64_t mr = m < p.M ? m : 0;  // rows past M read row 0 (never stored)
        const size_t xe = (size_t)mr * p.K + kk0 + (size_t)i * kChunk;
        const uint4* src = (const uint4*)(p.x + xe);
        if (SVDQ_INB(p.status, 2 * xe, 32, p.x_bytes)) {
          xr[it][0] = __ldcs(src);
          xr[it][1] = __ldcs(src + 1);
        } else {
          xr[it][0] = xr[it][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      float2 il[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const size_t ioff = ((size_t)(kk0 + i * kChunk) + 4 * q) * 4;
        const float4 t4 = SVDQ_INB(p.status, ioff, 16, p.il_bytes) ? __ldg((const float4*)(ilp + (size_t)i * kChunk) + q)
                                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        il[2 * q] = make_float2(t4.x, t4.y);
        il[2 * q + 1] = make_float2(t4.z, t4.w);
      }
      bool ok = true;
      if constexpr (RANK > 0) ok = mbar_wait(&xfree[buf], ((i >> 1) & 1) ^ 1, wc);
      if (ok) {
        uint8_t* at = atile + buf * kATileBytes;
#pragma unroll
        for (int it = 0; it < ITS; ++it) {
          const uint32_t w[8] = {xr[it][0].x, xr[it][0].y, xr[it][0].z, xr[it][0].w,
                                 xr[it][1].x, xr[it][1].y, xr[it][1].z, xr[it][1].w};
          float2 v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            v[e] = __fmul2_rn(make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)), il[e]);
          float mx[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) mx[e] = fmaxf(fabsf(v[e].x), fabsf(v[e].y));
#pragma unroll
          for (int e = 0; e < 4; ++e) mx[e] = fmaxf(mx[e], mx[e + 4]);
          float amax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
          const bool live = mbase + 2 * it < p.M;
          const size_t cbyte = coff0 + 2 * it * code_row + (size_t)i * kCodeStep;
          const size_t sbyte = soff0 + it * kScaleRowStep + (size_t)i * scale_step;
          if (FMT == SVDQ_NVFP4_G16) {
            const uint32_t sb = cvt_e4m3(__fdiv_rn(amax, dens));
            // 1 / (e4m3(sb) * g) exactly (g is a power of two); 0 for sb = 0
            const float inv = rtab[sb] * inv_gs;
            const float2 inv2 = make_float2(inv, inv);
            float2 q[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] = __fmul2_rn(v[e], inv2);
            uint2 packed = make_uint2(cvt_e2m1x8(q[0], q[1], q[2], q[3]), cvt_e2m1x8(q[4], q[5], q[6], q[7]));
            if (sb == 0) packed = make_uint2(0u, 0u);  // a zero block scale: all codes +0
            const int base = lane & ~3;  // 4 lanes = 64 columns = one scale-factor atom word
            const uint32_t s1 = __shfl_sync(0xffffffffu, sb, base + 1);
            const uint32_t s2 = __shfl_sync(0xffffffffu, sb, base + 2);
            const uint32_t s3 = __shfl_sync(0xffffffffu, sb, base + 3);
            if ((lane & 3) == 0 && live && SVDQ_INB(p.status, sbyte, 4, p.scales_bytes))
              *(uint32_t*)(p.scales + sbyte) = sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
            if (live && SVDQ_INB(p.status, cbyte, 8, p.codes_bytes)) *(uint2*)(p.codes + cbyte) = packed;
          } else {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
            const float S16 = __half2float(s16);
            // a zero scale gives inv = 0: every product is +-0 and rounds to the code +0
            const float inv = S16 != 0.f ? __frcp_rn(S16) : 0.f;
            const float2 inv2 = make_float2(inv, inv);
            const float2 magic = make_float2(12582912.0f, 12582912.0f), nmagic = make_float2(-12582912.0f, -12582912.0f);
            uint32_t qb[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float2 y0 = __fmul2_rn(v[e], inv2), y1 = __fmul2_rn(v[e + 1], inv2);
              // clamp, then round half to even: (y + 1.5 * 2^23) - 1.5 * 2^23
              // is the nearest integer (a +0 for codes of zero), and E4M3
              // holds every integer of [-8, 7] exactly
              y0 = make_float2(fminf(fmaxf(y0.x, -8.0f), 7.0f), fminf(fmaxf(y0.y, -8.0f), 7.0f));
              y1 = make_float2(fminf(fmaxf(y1.x, -8.0f), 7.0f), fminf(fmaxf(y1.y, -8.0f), 7.0f));
              y0 = __fadd2_rn(__fadd2_rn(y0, magic), nmagic);
              y1 = __fadd2_rn(__fadd2_rn(y1, magic), nmagic);
              qb[e >> 1] = cvt_e4m3x2(y0.x, y0.y) | (cvt_e4m3x2(y1.x, y1.y) << 16);
            }
            if ((lane & 3) == 0 && live && SVDQ_INB(p.status, sbyte, 2, p.scales_bytes))
              *(__half*)(p.scales + sbyte) = s16;
            if (live && SVDQ_INB(p.status, cbyte, 16, p.codes_bytes))
              *(uint4*)(p.codes + cbyte) = make_uint4(qb[0], qb[1], qb[2], qb[3]);
          }
          if constexpr (RANK > 0) {
            uint32_t b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              __nv_bfloat162 h = __float22bfloat162_rn(v[e]);
              b[e] = *(uint32_t*)&h;
            }
            const int row = rbase + 2 * it;
            uint8_t* arow = at + ablk + row * 128;
            *(uint4*)(arow + ((c0 ^ (row & 7)) << 4)) = make_uint4(b[0], b[1], b[2], b[3]);
            *(uint4*)(arow + (((c0 + 1) ^ (row & 7)) << 4)) = make_uint4(b[4], b[5], b[6], b[7]);
          }
        }
      }
      if constexpr (RANK > 0) {
        fence_proxy_async_smem();  // x^ tile -> tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&xready[buf]);
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
                if (SVDQ_INB(p.status, ((size_t)m * RANK + j) * 2, 4, p.t_bytes))
                  *(uint32_t*)(p.t + (size_t)m * RANK + j) = *(uint32_t*)&h;
              }
            }
          } else {
            if (m < p.M) {
              float* dst = p.tpart + ((size_t)slice * p.M + m) * RANK;
#pragma unroll
              for (int j = 0; j < RANK; j += 4)
                if (SVDQ_INB(p.status, (((size_t)slice * p.M + m) * RANK + j) * 4, 16, p.tpart_bytes))
                  *(float4*)(dst + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
            }
            __threadfence();
            named_bar_sync(2, 128);
            if (threadIdx.x == 0)
              *ticket = SVDQ_INB(p.status, (size_t)rowblock * 4, 4, p.cnt_bytes) ? atomicAdd(p.counters + rowblock, 1) : -1;
            named_bar_sync(2, 128);
            if (*ticket == p.nslices - 1) {  // last slice of this row block: fixed-order sum
              __threadfence();
              if (m < p.M) {
                // the slices' partials in slice order; the loads of a batch of slices (and of
                // two column quads) are issued together, the sums keep their order
                constexpr int SB = RANK > 80 ? 2 : 4;
#pragma unroll 1
                for (int j = 0; j < RANK; j += 8) {
                  float4 sum[2];
#pragma unroll 1
                  for (int s0 = 0; s0 < p.nslices; s0 += SB) {
                    float4 v[2][SB];
#pragma unroll
                    for (int i = 0; i < SB; ++i)
#pragma unroll
                      for (int h = 0; h < 2; ++h) {
                        const size_t e = ((size_t)(s0 + i) * p.M + m) * RANK + j + 4 * h;
                        v[h][i] = (s0 + i < p.nslices && j + 4 * h < RANK && SVDQ_INB(p.status, e * 4, 16, p.tpart_bytes))
                                      ? __ldcg((const float4*)(p.tpart + e))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                      }
#pragma unroll
                    for (int i = 0; i < SB; ++i)
#pragma unroll
                      for (int h = 0; h < 2; ++h) {
                        if (s0 + i >= p.nslices) continue;
                        if (s0 + i == 0) {
                          sum[h] = v[h][0];
                        } else {
                          sum[h].x += v[h][i].x;
                          sum[h].y += v[h][i].y;
                          sum[h].z += v[h][i].z;
                          sum[h].w += v[h][i].w;
                        }
                      }
                  }
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const int jj = j + 4 * h;
                    if (jj >= RANK) break;
                    __nv_bfloat162 h0 = scale_t(__floats2bfloat162_rn(sum[h].x, sum[h].y), tsc);
                    __nv_bfloat162 h1 = scale_t(__floats2bfloat162_rn(sum[h].z, sum[h].w), tsc);
                    if (SVDQ_INB(p.status, ((size_t)m * RANK + jj) * 2, 8, p.t_bytes))
                      *(uint2*)(p.t + (size_t)m * RANK + jj) = make_uint2(*(uint32_t*)&h0, *(uint32_t*)&h1);
                  }
                }
              }
              if (threadIdx.x == 0 && SVDQ_INB(p.status, (size_t)rowblock * 4, 4, p.cnt_bytes))
                p.counters[rowblock] = 0;  // ready for the next call
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
int launch_rank(const CUtensorMap& ml1, const QParams& p, int64_t M, cudaStream_t stream) {
  constexpr int kL1Bytes = RANK * kChunk * 2;
  QParams q = p;
  q.lstages = RANK == 0 ? 0 : (2 * kATileBytes + 2 * kL1Bytes + 2048 <= kSmemBudget ? 2 : 1);
  const size_t smem = 1024 + (RANK > 0 ? 2 * (size_t)kATileBytes : 0) + (size_t)q.lstages * kL1Bytes + 512 + 256;
  auto kern = k_quantize<FMT, RANK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  const dim3 grid((unsigned)((M + kRows - 1) / kRows), (unsigned)p.nslices);
  if (launch_pdl(kern, grid, dim3(Roles<RANK>::kThreads), smem, stream, ml1, q) != cudaSuccess) return SVDQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

template <int FMT>
int launch_fmt(const CUtensorMap& ml1, const QParams& p, int64_t M, int rank, cudaStream_t stream) {
  switch (rank) {
    case 0: return launch_rank<FMT, 0>(ml1, p, M, stream);
    case 16: return launch_rank<FMT, 16>(ml1, p, M, stream);
    case 32: return launch_rank<FMT, 32>(ml1, p, M, stream);
    case 48: return launch_rank<FMT, 48>(ml1, p, M, stream);
    case 64: return launch_rank<FMT, 64>(ml1, p, M, stream);
    case 80: return launch_rank<FMT, 80>(ml1, p, M, stream);
    case 96: return launch_rank<FMT, 96>(ml1, p, M, stream);
    case 112: return launch_rank<FMT, 112>(ml1, p, M, stream);
    case 128: return launch_rank<FMT, 128>(ml1, p, M, stream);
    default: return SVDQ_ERR_INVALID_ARG;
  }
}

}  // namespace

int launch_quantize(const svdq_layer* L, const void* X, int64_t M, uint8_t* ws, const Workspace& w,
                    cudaStream_t stream) {
  QParams p{};
  p.M = (int)M;
  p.K = (int)L->K;
  p.nch = (int)(L->K / kChunk);
  p.nslices = w.nslices;
  p.katoms = (int)(L->K / 64);
  p.sld = int4_scale_ld(M);
  p.x = (const uint16_t*)X;
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
  p.x_bytes = (size_t)M * L->K * 2;
  p.il_bytes = (size_t)L->K * 4;
  p.codes_bytes = w.codes_bytes;
  p.scales_bytes = w.scales_bytes;
  p.t_bytes = w.t_bytes;
  p.tpart_bytes = w.tpart_bytes;
  p.cnt_bytes = w.amax - (w.status + 16);
  if (L->fmt == SVDQ_NVFP4_G16) return launch_fmt<SVDQ_NVFP4_G16>(L->map_l1, p, M, L->rank, stream);
  return launch_fmt<SVDQ_INT4_G64>(L->map_l1, p, M, L->rank, stream);
}

}  // namespace svdq
