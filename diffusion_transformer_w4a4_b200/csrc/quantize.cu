// K1: fused activation quantizer of the svdq_w4a4 layer.
//
// One pass over X [M,K] bf16 computes, per "Суть метода" ("Hugging Face встроила
// Nunchaku в Diffusers ..."): the smoothed activation x^ = x * (1/lambda)
// (outliers moved into the weights), its 4-bit group codes and scales (INT4:
// groups of 64, fp16 scale; NVFP4: blocks of 16, E4M3 scale under a static
// per-tensor scale g_x), and the 16-bit low-rank down-projection
// t = bf16( bf16(x^) L1 ) with fp32 accumulation.
//
// Layout of the work: a CTA owns 32 token rows and walks K in 256-column
// chunks.  A producer warp streams X chunks [32 x 256] and the matching L1^T
// slices [rank x 256] (four 64-column boxes, 128-byte swizzle) into a
// multi-stage shared-memory ring with TMA.  Eight consumer warps quantize four
// rows each (a lane holds 8 consecutive elements, so a 16-element NVFP4 block
// is a lane pair and a 64-element INT4 group is 8 lanes; group maxima use
// warp shuffles), write codes/scales with coalesced stores, stage bf16(x^) in
// shared memory, then run the down-projection on tensor cores with
// mma.sync m16n8k16 (fp32 accumulation) from ldmatrix fragments.  HBM traffic
// is one read of X plus the 4-bit codes, scales and t.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kRows = 32;          // token rows per CTA
constexpr int kConsumerWarps = 8;  // 4 rows each
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kXTileBytes = kRows * kKStage * 2;  // 16 KiB
constexpr int kAPitch = kKStage * 2 + 16;         // padded bf16 row pitch (conflict-free ldmatrix)
constexpr int kATileBytes = kRows * kAPitch;

struct QParams {
  int M, K, rank, stages, nchunks, katoms;
  const float* inv_lambda;
  float g, den;  // NVFP4 per-tensor scale and 6*g
  uint8_t* codes;
  uint8_t* scales;
  uint16_t* t;
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

__device__ __forceinline__ float e4m3_value(uint32_t c) {  // c in [0, 0x7E]
  const uint32_t e = (c >> 3) & 0xF, m = c & 7;
  if (e == 0) return (float)m * (1.0f / 512.0f);
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Accumulator layout per warp: WN warps split the rank's n8 tiles, WK warps
// split the 16 k-steps of a chunk; 2 m16 tiles (32 rows) x NT n8 tiles.
constexpr int gcd_c(int a, int b) { return b == 0 ? a : gcd_c(b, a % b); }
template <int RANK>
struct RankCfg {
  static constexpr int NT8 = RANK / 8;
  static constexpr int WN = NT8 > 0 ? gcd_c(NT8, kConsumerWarps) : 1;  // divides both
  static constexpr int WK = kConsumerWarps / WN;
  static constexpr int NT = NT8 > 0 ? NT8 / WN : 0;
};

template <int FMT, int RANK>
__global__ void __launch_bounds__(kThreads, 1)
    k_quantize(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_l1, QParams p) {
  using C = RankCfg<RANK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int S = p.stages;
  const int l1_bytes = RANK * kKStage * 2;  // 4 boxes of RANK rows x 128 B
  const int stage_bytes = kXTileBytes + l1_bytes;
  uint8_t* atile = smem + S * stage_bytes;                      // 2 x [32][kAPitch]
  uint64_t* full = (uint64_t*)(atile + 2 * kATileBytes);        // [S]
  uint64_t* empty = full + S;                                   // [S]
  volatile int* abort_flag = (volatile int*)(empty + S);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kRows;
  WaitCtl wc{abort_flag, p.status, p.limit};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&map_x);
      if constexpr (RANK > 0) prefetch_tmap(&map_l1);
      int issued = 0;
      for (int c = 0; c < p.nchunks; ++c) {
        const int s = c % S;
        if (!mbar_wait(&empty[s], ((c / S) & 1) ^ 1, wc)) break;
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        tma_load_2d(&map_x, &full[s], st, c * kKStage, m0);
        if constexpr (RANK > 0) {
#pragma unroll
          for (int b = 0; b < 4; ++b) tma_load_2d(&map_l1, &full[s], st + kXTileBytes + b * RANK * 128, c * kKStage + 64 * b, 0);
        }
        issued = c + 1;
      }
      if (*abort_flag) {  // drain copies that are still in flight before leaving
        for (int c = (issued > S ? issued - S : 0); c < issued; ++c)
          mbar_wait_drain(&full[c % S], (c / S) & 1, p.limit);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    float acc[2][C::NT > 0 ? C::NT : 1][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < (C::NT > 0 ? C::NT : 1); ++b)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][b][q] = 0.f;
    const int wn = warp % C::WN, wk = warp / C::WN;
    const int K2 = p.K / 2;

    for (int c = 0; c < p.nchunks; ++c) {
      const int s = c % S;
      const bool ok = mbar_wait(&full[s], (c / S) & 1, wc);
      uint8_t* st = smem + s * stage_bytes;
      uint8_t* at = atile + (c & 1) * kATileBytes;
      if (ok) {
        const int k0 = c * kKStage + lane * 8;
        const float4 il0 = __ldg((const float4*)(p.inv_lambda + k0));
        const float4 il1 = __ldg((const float4*)(p.inv_lambda + k0 + 4));
        const float il[8] = {il0.x, il0.y, il0.z, il0.w, il1.x, il1.y, il1.z, il1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = warp * 4 + i;
          const int m = m0 + row;
          const uint4 raw = *(const uint4*)(st + row * (kKStage * 2) + lane * 16);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          float v[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[2 * j] = __fmul_rn(__uint_as_float(w[j] << 16), il[2 * j]);
            v[2 * j + 1] = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), il[2 * j + 1]);
          }
          float amax = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
          uint32_t packed = 0;
          if (FMT == SVDQ_NVFP4_G16) {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            const uint32_t sb = cvt_e4m3(__fdiv_rn(amax, p.den));
            if (sb != 0) {
              const float inv = __fdiv_rn(1.0f, __fmul_rn(e4m3_value(sb), p.g));
              float q[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) q[j] = __fmul_rn(v[j], inv);
              packed = cvt_e2m1x8(q);
            }
            // gather the four block scales of each 64-column atom into one word
            const int base = lane & ~7;
            const uint32_t s0 = __shfl_sync(0xffffffffu, sb, base + 0);
            const uint32_t s1 = __shfl_sync(0xffffffffu, sb, base + 2);
            const uint32_t s2 = __shfl_sync(0xffffffffu, sb, base + 4);
            const uint32_t s3 = __shfl_sync(0xffffffffu, sb, base + 6);
            if ((lane & 7) == 0 && m < p.M) {
              const int blk = c * (kKStage / 16) + (lane >> 3) * 4;
              *(uint32_t*)(p.scales + sf_offset(m, blk, p.katoms, kSfAtomRows)) =
                  s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
            }
          } else {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
            const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
            const float S16 = __half2float(s16);
            if (S16 != 0.f) {
              const float inv = __fdiv_rn(1.0f, S16);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                int q = __float2int_rn(__fmul_rn(v[j], inv));
                q = max(-8, min(7, q));
                packed |= (uint32_t)(q & 0xF) << (4 * j);
              }
            }
            if ((lane & 7) == 0 && m < p.M) {
              const int grp = c * (kKStage / 64) + (lane >> 3);
              ((__half*)p.scales)[(size_t)grp * p.M + m] = s16;
            }
          }
          if (m < p.M) *(uint32_t*)(p.codes + (size_t)m * K2 + c * (kKStage / 2) + lane * 4) = packed;
          if constexpr (RANK > 0) {
            uint4 xb;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
            xb.x = *(uint32_t*)&h0;
            xb.y = *(uint32_t*)&h1;
            xb.z = *(uint32_t*)&h2;
            xb.w = *(uint32_t*)&h3;
            *(uint4*)(at + row * kAPitch + lane * 16) = xb;
          }
        }
      }
      if constexpr (RANK > 0) {
        named_bar_sync(1, kConsumerWarps * 32);  // bf16(x^) tile complete
        if (ok) {
          const uint8_t* l1t = st + kXTileBytes;
          const uint32_t a_base = smem_u32(at);
          const uint32_t l_base = smem_u32(l1t);
#pragma unroll 4
          for (int ks = wk; ks < kKStage / 16; ks += C::WK) {
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              const int row = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
              const int col = ks * 16 + 8 * (lane >> 4);
              ldmatrix_x4(a_base + row * kAPitch + col * 2, af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
            }
#pragma unroll
            for (int nt = 0; nt < (C::NT > 0 ? C::NT : 1); ++nt) {
              const int n = 8 * (wn + C::WN * nt) + (lane & 7);
              const int kl = ks * 16 + 8 * ((lane >> 3) & 1);
              const int box = kl >> 6, chunk = (kl & 63) >> 3;
              const uint32_t addr = l_base + box * (RANK * 128) + n * 128 + ((chunk ^ (n & 7)) << 4);
              uint32_t b0, b1;
              ldmatrix_x2(addr, b0, b1);
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) mma_16816(acc[mt][nt], af[mt], b0, b1);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    if constexpr (RANK > 0) {
      // cross-warp reduction of the k-split partial sums in a fixed order
      // (k-split 0, then 1, ...), in place in one [32][RANK] fp32 buffer
      named_bar_sync(1, kConsumerWarps * 32);  // all MMAs done: the A tiles are free
      float* red = (float*)atile;
      const int g = lane >> 2, q = lane & 3;
      for (int k = 0; k < C::WK; ++k) {
        if (wk == k) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < (C::NT > 0 ? C::NT : 1); ++nt) {
              const int col = 8 * (wn + C::WN * nt) + 2 * q;
              float* r0 = red + (size_t)(mt * 16 + g) * RANK + col;
              float* r1 = red + (size_t)(mt * 16 + g + 8) * RANK + col;
              if (k == 0) {
                r0[0] = acc[mt][nt][0]; r0[1] = acc[mt][nt][1];
                r1[0] = acc[mt][nt][2]; r1[1] = acc[mt][nt][3];
              } else {
                r0[0] += acc[mt][nt][0]; r0[1] += acc[mt][nt][1];
                r1[0] += acc[mt][nt][2]; r1[1] += acc[mt][nt][3];
              }
            }
        }
        named_bar_sync(1, kConsumerWarps * 32);
      }
      if (!*abort_flag) {
        for (int idx = threadIdx.x; idx < kRows * RANK / 2; idx += kConsumerWarps * 32) {
          const int row = idx / (RANK / 2), col = 2 * (idx % (RANK / 2));
          const float s0 = red[(size_t)row * RANK + col], s1 = red[(size_t)row * RANK + col + 1];
          const int m = m0 + row;
          if (m < p.M) {
            __nv_bfloat162 h = __floats2bfloat162_rn(s0, s1);
            *(uint32_t*)(p.t + (size_t)m * RANK + col) = *(uint32_t*)&h;
          }
        }
      }
    }
  }
  __syncthreads();
}

template <int FMT, int RANK>
int launch_rank(const CUtensorMap& mx, const CUtensorMap& ml1, const QParams& p, int64_t M, cudaStream_t stream) {
  const int l1_bytes = RANK * kKStage * 2;
  const int stage_bytes = kXTileBytes + l1_bytes;
  QParams q = p;
  int S = (200 * 1024 - 2 * kATileBytes) / stage_bytes;
  if (S > 4) S = 4;
  if (S < 1) S = 1;
  q.stages = S;
  const size_t smem = 1024 + (size_t)S * stage_bytes + 2 * kATileBytes + 2 * S * sizeof(uint64_t) + 16;
  auto kern = k_quantize<FMT, RANK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  const unsigned grid = (unsigned)((M + kRows - 1) / kRows);
  kern<<<grid, kThreads, smem, stream>>>(mx, ml1, q);
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
                          (uint64_t)L->K * 2, kKStage, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != SVDQ_OK) return st;
  QParams p{};
  p.M = (int)M;
  p.K = (int)L->K;
  p.rank = L->rank;
  p.nchunks = (int)(L->K / kKStage);
  p.katoms = (int)(L->K / 64);
  p.inv_lambda = L->inv_lambda;
  p.g = L->g_x;
  p.den = 6.0f * L->g_x;
  p.codes = ws + w.codes;
  p.scales = ws + w.scales;
  p.t = (uint16_t*)(ws + w.t);
  p.status = (int*)(ws + w.status);
  p.limit = wait_limit_cycles();
  if (L->fmt == SVDQ_NVFP4_G16) return launch_fmt<SVDQ_NVFP4_G16>(mx, L->map_l1, p, M, L->rank, stream);
  return launch_fmt<SVDQ_INT4_G64>(mx, L->map_l1, p, M, L->rank, stream);
}

}  // namespace svdq
