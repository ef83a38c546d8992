// K3: INT4 W4A4 GEMM of the svdq_w4a4 layer on 5th-generation tensor cores.
//
//   Y = t . L2  +  sum_g  s_x[m,g] s_w[n,g] acc_g[m,n]  +  b,
//   acc_g[m,n] = sum_{k in group g} qx[m,k] qw[n,k]   (exact int32)
//
// "Суть метода" ("Hugging Face встроила Nunchaku в Diffusers ...") with the INT4
// variant of the next paragraph: signed 4-bit codes in groups of 64 along K with
// fp16 group scales.  Tensor cores have no 4-bit integer kind, so the packed
// codes are widened to int8 in shared memory and multiplied with
// tcgen05.mma kind::i8 (int32 accumulation).  Because both scales change every
// 64 columns of K, each group's int32 accumulator is drained and rescaled by
// the epilogue warps into an fp32 running sum held in registers, while the
// tensor core fills the next of four accumulators.  Every accumulator starts
// at the integer 0x4B400000, the bit pattern of 1.5 * 2^23: after adding a
// group sum (|sum| <= 64 * 8 * 8 = 4096) the int32 result read as binary32 is
// exactly 1.5 * 2^23 + sum, so one packed subtraction recovers the sum as a
// float without an integer-to-float conversion.
//
// Persistent, warp-specialized CTA (one per SM), tile 128 x 128:
//   warp 0      TMA producer: packed codes [128 x 128 B] (128-byte swizzle)
//               for A and B per 256-column K stage (raw ring), and the bf16
//               t / L2^T chunks of the low-rank branch (own buffer).
//   warp 1      owns tensor memory (4 x 128 columns) and issues the MMAs:
//               kind::f16 for t . L2 (its own accumulator unit, which seeds the
//               running sum), then 2 x kind::i8 (K=32) per 64-group, four
//               groups per stage.
//   warps 2-3   converters: raw int4 -> int8, sign-extended, written in the
//               128-byte-swizzled K-major layout the MMA reads (conv ring).
//   warps 4-11  epilogue (two per lane quarter, 64 columns each): tcgen05.ld
//               each unit; y += s_x s_w float(acc);
//               bias, bf16 round-to-nearest-even, 16-byte stores.  With a
//               debug output pointer it instead writes the raw int32 group
//               accumulators (integer-path parity).
// Every wait is bounded (sm100.cuh); no load uses cluster multicast.
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include <cstring>

#include "sm100.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = kGemmBM;  // 128
constexpr int BN = kInt4BN;  // 128
constexpr int BK = 256;      // K elements per stage (4 groups of 64)
constexpr int GPS = BK / 64;  // groups per stage
constexpr int RAW_STAGES = 2;
constexpr int CONV_STAGES = 2;
constexpr int RAW_A = BM * BK / 2;  // 16 KiB packed, one 128-byte swizzled row per token
constexpr int RAW_B = BN * BK / 2;
constexpr int RAW_BYTES = RAW_A + RAW_B;
constexpr int CONV_HALF = BM * 128;  // int8 sub-tile of 128 K columns, 128-byte swizzled
constexpr int CONV_A = 2 * CONV_HALF;
constexpr int CONV_B = 2 * CONV_HALF;
constexpr int CONV_BYTES = CONV_A + CONV_B;
constexpr int LR_A = BM * 128;  // one low-rank chunk: up to 64 bf16 per row
constexpr int LR_B = BN * 128;
constexpr int EPI_WARPS = 8;  // two per tensor-memory lane quarter, 64 columns each
constexpr int EPI_COLS = BN / 2;
constexpr int CONV_WARPS = 2;
constexpr int EPI_WARP0 = 2 + CONV_WARPS;
constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;  // 12 warps: 3 per scheduler, up to 168 registers each
constexpr uint32_t TMEM_COLS = 512;
constexpr int NACC = 4;  // accumulator buffers
constexpr uint32_t MAGIC_BITS = 0x4B400000u;  // 1.5 * 2^23 as binary32
constexpr float MAGIC = 12582912.0f;
constexpr uint32_t IDESC_S8 = idesc_s8_s32(BM, BN);
constexpr uint32_t IDESC_BF16 = idesc_bf16_f32(BM, BN);

struct I4Maps {
  CUtensorMap a, b, t[3], l2[3];
};

struct I4Params {
  int M, N, K, m_tiles, n_tiles, num_tiles, k_stages, groups;
  int n_lr;
  int lr_off[4], lr_w[4];
  const __half* sx;  // [K/64, M]
  const float* sw;   // [K/64, N], fp16 group scales widened to f32
  const float* bias;
  uint16_t* Y;
  int32_t* acc_dbg;  // [K/64, M, N] or null
  int* status;
  unsigned long long limit;
};

__device__ __forceinline__ int lr_map_index(int w) { return w == 64 ? 0 : (w == 32 ? 1 : 2); }

// 32 lanes x 32 columns of tensor memory <- the magic integer
__device__ __forceinline__ void tmem_fill_magic(uint32_t taddr) {
  const uint32_t v = MAGIC_BITS;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

__device__ __forceinline__ void sub2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "sub.rn.f32x2 z, x, y;\n\tmov.b64 {%0, %1}, z;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mul.rn.f32x2 z, x, y;\n\tmov.b64 {%0, %1}, z;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
// (y0, y1) += (a0, a1) * (b0, b1), one rounding each
__device__ __forceinline__ void fma2(float& y0, float& y1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %5};\n\tmov.b64 z, {%0, %1};\n\t"
      "fma.rn.f32x2 z, x, y, z;\n\tmov.b64 {%0, %1}, z;\n\t}"
      : "+f"(y0), "+f"(y1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 8 packed nibbles (two's complement, element 2i in the low nibble of byte i)
// -> 8 sign-extended int8, in element order, as two words.
__device__ __forceinline__ uint2 widen8(uint32_t w) {
  const uint32_t lo = __vsub4((w & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);         // elements 0,2,4,6
  const uint32_t hi = __vsub4(((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);  // elements 1,3,5,7
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

template <bool DBG>
__global__ void __launch_bounds__(THREADS, 1) k_gemm_int4(const __grid_constant__ I4Maps maps, const I4Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* conv = smem;                                // [CONV_STAGES][CONV_BYTES]  (1024-aligned)
  uint8_t* lrbuf = conv + CONV_STAGES * CONV_BYTES;    // [LR_A + LR_B]
  uint8_t* raw = lrbuf + LR_A + LR_B;                  // [RAW_STAGES][RAW_BYTES]
  uint64_t* raw_full = (uint64_t*)(raw + RAW_STAGES * RAW_BYTES);
  uint64_t* raw_empty = raw_full + RAW_STAGES;
  uint64_t* conv_full = raw_empty + RAW_STAGES;
  uint64_t* conv_empty = conv_full + CONV_STAGES;
  uint64_t* lr_full = conv_empty + CONV_STAGES;
  uint64_t* lr_empty = lr_full + 1;
  uint64_t* acc_full = lr_empty + 1;      // [NACC]
  uint64_t* acc_empty = acc_full + NACC;  // [NACC]
  uint64_t* mma_done = acc_empty + NACC;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.status, p.limit};

  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_STAGES; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], CONV_WARPS);
    }
    for (int s = 0; s < CONV_STAGES; ++s) {
      mbar_init(&conv_full[s], CONV_WARPS);
      mbar_init(&conv_empty[s], 1);
    }
    mbar_init(lr_full, 1);
    mbar_init(lr_empty, 1);
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS * 32);
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
  if (warp >= EPI_WARP0) {  // every accumulator starts at the magic integer
    const uint32_t tq = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(((warp - EPI_WARP0) >> 2) * EPI_COLS);
    for (int b = 0; b < NACC; ++b) {
      tmem_fill_magic(tq + b * BN);
      tmem_fill_magic(tq + b * BN + 32);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&maps.a);
      prefetch_tmap(&maps.b);
      int rit = 0, lit = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int u = 0; u < p.n_lr && ok; ++u, ++lit) {
          if (!mbar_wait(lr_empty, (lit & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          const int w = p.lr_w[u], mi = lr_map_index(w);
          mbar_arrive_expect_tx(lr_full, (uint32_t)(BM + BN) * 2 * w);
          tma_load_2d(&maps.t[mi], lr_full, lrbuf, p.lr_off[u], mt * BM);
          tma_load_2d(&maps.l2[mi], lr_full, lrbuf + LR_A, p.lr_off[u], nt * BN);
        }
        for (int ks = 0; ks < p.k_stages && ok; ++ks, ++rit) {
          const int s = rit % RAW_STAGES;
          if (!mbar_wait(&raw_empty[s], ((rit / RAW_STAGES) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = raw + s * RAW_BYTES;
          mbar_arrive_expect_tx(&raw_full[s], RAW_BYTES);
          tma_load_2d(&maps.a, &raw_full[s], st, ks * (BK / 2), mt * BM);
          tma_load_2d(&maps.b, &raw_full[s], st + RAW_A, ks * (BK / 2), nt * BN);
        }
      }
      if (!ok) {  // drain copies still in flight
        for (int j = (rit > RAW_STAGES ? rit - RAW_STAGES : 0); j < rit; ++j)
          mbar_wait_drain(&raw_full[j % RAW_STAGES], (j / RAW_STAGES) & 1, p.limit);
        if (lit > 0) mbar_wait_drain(lr_full, (lit - 1) & 1, p.limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int cit = 0, lit = 0, unit = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        if (p.n_lr > 0) {
          const int b = unit % NACC;
          if (!mbar_wait(&acc_empty[b], ((unit / NACC) & 1) ^ 1, wc)) break;
          tc_fence_after();
          uint32_t accum = 0;
          for (int u = 0; u < p.n_lr; ++u, ++lit) {
            if (!mbar_wait(lr_full, lit & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int w = p.lr_w[u];
            const uint32_t layout = w == 64 ? LAYOUT_SW128 : (w == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
            const uint32_t sbo = 16u * (uint32_t)w;
            const uint32_t a_addr = smem_u32(lrbuf), b_addr = a_addr + LR_A;
            for (int kk = 0; kk < w / 16; ++kk) {
              mma_bf16(tmem + b * BN, make_sdesc(a_addr + 32 * kk, 16, sbo, layout),
                       make_sdesc(b_addr + 32 * kk, 16, sbo, layout), IDESC_BF16, accum);
              accum = 1;
            }
            umma_commit(lr_empty);
          }
          if (!ok) break;
          umma_commit(&acc_full[b]);
          ++unit;
        }
        for (int ks = 0; ks < p.k_stages && ok; ++ks, ++cit) {
          const int s = cit % CONV_STAGES;
          if (!mbar_wait(&conv_full[s], (cit / CONV_STAGES) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(conv + s * CONV_BYTES), b_addr = a_addr + CONV_A;
          for (int g = 0; g < GPS; ++g, ++unit) {
            const int b = unit % NACC;
            if (!mbar_wait(&acc_empty[b], ((unit / NACC) & 1) ^ 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const uint32_t off = (g >> 1) * CONV_HALF + 64 * (g & 1) + 32 * kk;
              mma_s8(tmem + b * BN, make_sdesc(a_addr + off, 16, 1024, LAYOUT_SW128),
                     make_sdesc(b_addr + off, 16, 1024, LAYOUT_SW128), IDESC_S8, 1u);
            }
            umma_commit(&acc_full[b]);
          }
          umma_commit(&conv_empty[s]);
        }
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, p.limit);
    }
  } else if (warp < EPI_WARP0) {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - 64;  // 0..CONV_WARPS*32-1
    int rit = 0, cit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      for (int ks = 0; ks < p.k_stages; ++ks, ++rit, ++cit) {
        const int rs = rit % RAW_STAGES, cs = cit % CONV_STAGES;
        ok = mbar_wait(&raw_full[rs], (rit / RAW_STAGES) & 1, wc) &&
             mbar_wait(&conv_empty[cs], ((cit / CONV_STAGES) & 1) ^ 1, wc);
        if (!ok) break;
        const uint8_t* src = raw + rs * RAW_BYTES;
        uint8_t* dst = conv + cs * CONV_BYTES;
#pragma unroll
        for (int op = 0; op < 2; ++op) {  // A then B
          const uint8_t* sh = src + op * RAW_A;
          uint8_t* dh = dst + op * CONV_A;
#pragma unroll 4
          for (int i = 0; i < (BM * 16) / (CONV_WARPS * 32); ++i) {
            const int id = i * (CONV_WARPS * 32) + ct;
            const int row = id >> 4, c8 = id & 15;  // 8 packed bytes = 16 codes
            const uint2 pk = *(const uint2*)(sh + row * 128 + ((((c8 >> 1) ^ (row & 7)) << 4) | ((c8 & 1) << 3)));
            const uint2 w0 = widen8(pk.x), w1 = widen8(pk.y);
            *(uint4*)(dh + (c8 >> 3) * CONV_HALF + row * 128 + (((c8 & 7) ^ (row & 7)) << 4)) =
                make_uint4(w0.x, w0.y, w1.x, w1.y);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&conv_full[cs]);
          mbar_arrive(&raw_empty[rs]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int half = (warp - EPI_WARP0) >> 2;
    const int row = 32 * q + lane;
    int unit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int m = mt * BM + row;
      const int n0 = nt * BN + half * EPI_COLS;
      const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * EPI_COLS);
      float y[EPI_COLS];
#pragma unroll
      for (int j = 0; j < EPI_COLS; ++j) y[j] = 0.f;
      if (p.n_lr > 0) {
        const int b = unit % NACC;
        if (!mbar_wait(&acc_full[b], (unit / NACC) & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < EPI_COLS / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tl + b * BN + 32 * c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) y[32 * c + j] = __uint_as_float(r[j]);
        }
        tmem_fill_magic(tl + b * BN);  // re-arm for an integer unit
        tmem_fill_magic(tl + b * BN + 32);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
        ++unit;
      }
      for (int g = 0; g < p.groups; ++g, ++unit) {
        const int b = unit % NACC;
        if (!mbar_wait(&acc_full[b], (unit / NACC) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float sx = (m < p.M) ? __half2float(p.sx[(size_t)g * p.M + m]) : 0.f;
        const float* swg = p.sw + (size_t)g * p.N + n0;
#pragma unroll
        for (int c = 0; c < EPI_COLS / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tl + b * BN + 32 * c, r);
          tmem_ld_wait();
          if (DBG) {
            if (m < p.M) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                const int n = n0 + 32 * c + j;
                if (n < p.N)
                  *(uint4*)(p.acc_dbg + ((size_t)g * p.M + m) * p.N + n) =
                      make_uint4(r[j] - MAGIC_BITS, r[j + 1] - MAGIC_BITS, r[j + 2] - MAGIC_BITS, r[j + 3] - MAGIC_BITS);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const int n = n0 + 32 * c + j;
              const float4 w4 = (n < p.N) ? __ldg((const float4*)(swg + 32 * c + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
              float f0 = __uint_as_float(r[j]), f1 = __uint_as_float(r[j + 1]);
              float f2 = __uint_as_float(r[j + 2]), f3 = __uint_as_float(r[j + 3]);
              sub2(f0, f1, MAGIC, MAGIC);  // exact: the group's integer sums
              sub2(f2, f3, MAGIC, MAGIC);
              float s0 = w4.x, s1 = w4.y, s2 = w4.z, s3 = w4.w;
              mul2(s0, s1, sx, sx);
              mul2(s2, s3, sx, sx);
              fma2(y[32 * c + j], y[32 * c + j + 1], s0, s1, f0, f1);
              fma2(y[32 * c + j + 2], y[32 * c + j + 3], s2, s3, f2, f3);
            }
          }
        }
        tmem_fill_magic(tl + b * BN);  // re-arm this accumulator
        tmem_fill_magic(tl + b * BN + 32);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
      }
      if (!ok) break;
      if (!DBG && m < p.M) {
#pragma unroll
        for (int j8 = 0; j8 < EPI_COLS / 8; ++j8) {
          const int n = n0 + 8 * j8;
          if (n < p.N) {
            const float4 b0 = __ldg((const float4*)(p.bias + n));
            const float4 b1 = __ldg((const float4*)(p.bias + n + 4));
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h =
                  __floats2bfloat162_rn(y[8 * j8 + 2 * e] + bb[2 * e], y[8 * j8 + 2 * e + 1] + bb[2 * e + 1]);
              o[e] = *(uint32_t*)&h;
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

int sm_count_i4(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace

int launch_gemm_int4(const svdq_layer* L, int64_t M, void* Y, uint8_t* ws, const Workspace& w, int32_t* acc_dbg,
                     cudaStream_t stream) {
  I4Maps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int K = (int)L->K, N = (int)L->N, r = L->rank;
  int st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.codes, (uint64_t)K / 2, (uint64_t)M,
                          (uint64_t)K / 2, BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  maps.b = L->map_w;
  I4Params p{};
  const LowRankChunks ch = lowrank_chunks(r);
  p.n_lr = acc_dbg ? 0 : ch.n;  // the integer-path export skips the low-rank unit
  for (int i = 0; i < ch.n; ++i) {
    p.lr_off[i] = ch.off[i];
    p.lr_w[i] = ch.width[i];
  }
  if (r > 0) {
    const int widths[3] = {64, 32, 16};
    const CUtensorMapSwizzle swz[3] = {CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_SWIZZLE_64B,
                                       CU_TENSOR_MAP_SWIZZLE_32B};
    for (int i = 0; i < 3; ++i) {
      if (widths[i] > r) continue;
      st = encode_tmap_2d(&maps.t[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + w.t, (uint64_t)r, (uint64_t)M,
                          (uint64_t)r * 2, widths[i], BM, swz[i]);
      if (st != SVDQ_OK) return st;
      maps.l2[i] = L->map_l2[i];
    }
  }
  p.M = (int)M;
  p.N = N;
  p.K = K;
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = (N + BN - 1) / BN;
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.k_stages = K / BK;
  p.groups = K / 64;
  p.sx = (const __half*)(ws + w.scales);
  p.sw = (const float*)L->wscales;
  p.bias = L->bias;
  p.Y = (uint16_t*)Y;
  p.acc_dbg = acc_dbg;
  p.status = (int*)(ws + w.status);
  p.limit = wait_limit_cycles();
  const size_t smem = 1024 + (size_t)CONV_STAGES * CONV_BYTES + LR_A + LR_B + (size_t)RAW_STAGES * RAW_BYTES + 256;
  const int grid = p.num_tiles < sm_count_i4(L->device) ? p.num_tiles : sm_count_i4(L->device);
  if (acc_dbg) {
    if (cudaFuncSetAttribute(k_gemm_int4<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    k_gemm_int4<true><<<grid, THREADS, smem, stream>>>(maps, p);
  } else {
    if (cudaFuncSetAttribute(k_gemm_int4<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    k_gemm_int4<false><<<grid, THREADS, smem, stream>>>(maps, p);
  }
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace svdq
