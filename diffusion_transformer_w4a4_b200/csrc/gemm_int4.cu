// K3: INT4 W4A4 GEMM of the svdq_w4a4 layer on 5th-generation tensor cores.
//
//   Y = t . L2  +  sum_g  s_x[m,g] s_w[n,g] acc_g[m,n]  +  b,
//   acc_g[m,n] = sum_{k in group g} qx[m,k] qw[n,k]   (an exact integer)
//
// "Суть метода" ("Hugging Face встроила Nunchaku в Diffusers ...") with the INT4
// variant of the next paragraph: signed 4-bit codes in groups of 64 along K with
// fp16 group scales.  Tensor cores have no 4-bit integer kind.  Every integer
// of [-8, 7] is exact in FP8 E4M3, so the activation quantizer and the weight
// packer store each code as the E4M3 byte of its value and the group products
// run as tcgen05.mma kind::f8f6f4 with an f32 accumulator: the products are
// integers of magnitude <= 64 and a group's sum is an integer of magnitude
// <= 4096, all exact in binary32, so the accumulator holds acc_g exactly.
// Because both scales change every 64 columns of K, each group's accumulator is
// drained by the epilogue warps into an fp32 running sum held in registers,
// y += (s_x s_w) acc_g: two fp32 operations per output and group, against one
// 128 x 128 x 64 MMA.  That drain, not the tensor core, bounds the kernel.  Per
// 128 x 128 group an SM spends about 256 cycles of FMA-pipe time (128 fp32
// lanes per clock, packed f32x2 or not), about 256 cycles reading the 64 KiB
// accumulator out of tensor memory in the 16x256b shape (about 255 B/clk; the
// 32x32b shape reads about 3x faster but would need 64 weight scales per
// thread and group from shared memory, which costs more), and about 128
// cycles of shared-memory traffic for the scales.
//
// Persistent, warp-specialized CTA (one per SM), tile 128 x 128:
//   warp 0      TMA producer: E4M3 codes [128 x 128 B] (128-byte swizzle) for
//               A and B per 128-column K stage (two groups); the two groups'
//               scales (f32 s_w [2 x 128], fp16 s_x [2 x 128]) into a ring of
//               their own; the bf16 t / L2^T chunks of the low-rank branch.
//   warp 1      owns tensor memory and issues the MMAs.  Accumulator units of
//               256 columns, double-buffered: one unit per K stage holds its
//               two groups side by side (2 x kind::f8f6f4, K = 32, per group),
//               so the MMA and epilogue hand over once per two groups; the
//               low-rank product t . L2 (kind::f16) is a unit of its own, once
//               per tile, and seeds the running sum.
//   warps 2-9   epilogue (two per lane quarter, 64 columns each; a thread holds
//               4 rows x 16 columns): tcgen05.ld each group, release the unit
//               once its last group is in registers (one arrival per warp),
//               y += (s_x s_w) acc in packed f32x2 arithmetic; bias,
//               bf16 round-to-nearest-even, stores.  With a debug output
//               pointer it instead writes the group accumulators as int32
//               (integer-path parity).
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
constexpr int BK = 128;      // K codes (bytes) per stage: two groups of 64
constexpr int GPS = BK / 64;
constexpr int STAGES = 5;
constexpr int STAGE_A = BM * BK;  // 16 KiB, one 128-byte swizzled row per token
constexpr int STAGE_B = BN * BK;
constexpr int STAGE_BYTES = STAGE_A + STAGE_B;
constexpr int LR_A = BM * 128;  // one low-rank chunk: up to 64 bf16 per row
constexpr int LR_B = BN * 128;
constexpr int SC_SLOTS = 8;                   // scale ring: one slot per K stage
constexpr int SC_SW = GPS * BN * 4;           // f32 s_w [GPS][BN]
constexpr int SC_SX = GPS * BM * 2;           // fp16 s_x [GPS][BM]
constexpr int SC_BYTES = SC_SW + SC_SX;       // 1.5 KiB, a multiple of 128
constexpr int EPI_WARPS = 8;  // two per tensor-memory lane quarter, 64 columns each
constexpr int EPI_COLS = BN / 2;
constexpr int EPI_WARP0 = 2;
constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;  // 10 warps: at most 168 registers each
constexpr uint32_t TMEM_COLS = 512;
constexpr int UNIT_COLS = GPS * BN;  // one accumulator unit: the GPS groups of a K stage
constexpr int NBUF = 2;              // double-buffered units (all 512 columns)
constexpr uint32_t IDESC_E4M3 = idesc_e4m3_f32(BM, BN);
constexpr uint32_t IDESC_BF16 = idesc_bf16_f32(BM, BN);
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + LR_A + LR_B + (size_t)SC_SLOTS * SC_BYTES + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(SC_SW % 128 == 0 && SC_BYTES % 128 == 0, "TMA destinations stay 128-byte aligned");

struct I4Maps {
  CUtensorMap a, b, sw, sx, t[3], l2[3];
};

struct I4Params {
  int M, N, K, m_tiles, n_tiles, num_tiles, k_stages;
  int n_lr;
  int lr_off[4], lr_w[4];
  const float* bias;
  uint16_t* Y;
  int32_t* acc_dbg;  // [K/64, M, N] or null
  int* status;
  unsigned long long limit;
};

__device__ __forceinline__ int lr_map_index(int w) { return w == 64 ? 0 : (w == 32 ? 1 : 2); }

// Epilogue fragment of one thread (tcgen05.ld 16x256b, one load each for the
// lanes 32q..32q+15 and 32q+16..32q+31 of its quarter q): rows 32q + t/4 + 8i
// (i = 0..3) by columns c0 + 8j + e (j = 0..7, e = 0, 1), with
// c0 = 64 p + 2 (t % 4) for the warp's column half p, held in y[16 i + 2 j + e].
// (The 32x32b shape reads tensor memory about 3x faster, but gives each thread
// one row and 64 columns, so every thread would need 64 weight scales per group
// from shared memory; here a thread needs 16.)

// y += (s_x[row] s_w[col]) acc over the fragment; sw points at s_w[c0], sx[i]
// is s_x of row i.  Two packed operations per pair of outputs.
__device__ __forceinline__ void drain_frag(float2 (&y)[32], const uint32_t (&lo)[32], const uint32_t (&hi)[32],
                                           const float* sw, const float2 (&sx)[4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 w = *(const float2*)(sw + 8 * j);  // 4 distinct addresses per warp
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t(&r)[32] = i < 2 ? lo : hi;
      const int k = 4 * j + 2 * (i & 1);
      const float2 c = __fmul2_rn(w, sx[i]);  // exact: products of two fp16 values
      y[8 * i + j] = __ffma2_rn(c, make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), y[8 * i + j]);
    }
  }
}

// integer-path export of one group's fragment
__device__ __forceinline__ void export_frag(const I4Params& p, size_t g, int row0, int col0, const uint32_t (&lo)[32],
                                            const uint32_t (&hi)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = row0 + 8 * i;
    if (m >= p.M) continue;
    const uint32_t(&r)[32] = i < 2 ? lo : hi;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = col0 + 8 * j;
      const int k = 4 * j + 2 * (i & 1);
      if (n < p.N)
        *(int2*)(p.acc_dbg + (g * p.M + m) * p.N + n) =
            make_int2(__float2int_rz(__uint_as_float(r[k])), __float2int_rz(__uint_as_float(r[k + 1])));
    }
  }
}

template <bool DBG>
__global__ void __launch_bounds__(THREADS, 1) k_gemm_int4(const __grid_constant__ I4Maps maps, const __grid_constant__ I4Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;                             // [STAGES][STAGE_BYTES]  (1024-aligned)
  uint8_t* lrbuf = stages + STAGES * STAGE_BYTES;     // [LR_A + LR_B]
  uint8_t* scring = lrbuf + LR_A + LR_B;              // [SC_SLOTS][SC_BYTES]
  uint64_t* full = (uint64_t*)(scring + SC_SLOTS * SC_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* sc_full = empty + STAGES;
  uint64_t* sc_empty = sc_full + SC_SLOTS;
  uint64_t* lr_full = sc_empty + SC_SLOTS;
  uint64_t* lr_empty = lr_full + 1;
  uint64_t* acc_full = lr_empty + 1;      // [NBUF]
  uint64_t* acc_empty = acc_full + NBUF;  // [NBUF]
  uint64_t* mma_done = acc_empty + NBUF;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.status, p.limit};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < SC_SLOTS; ++s) {
      mbar_init(&sc_full[s], 1);
      mbar_init(&sc_empty[s], EPI_WARPS);
    }
    mbar_init(lr_full, 1);
    mbar_init(lr_empty, 1);
    for (int b = 0; b < NBUF; ++b) {
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
      prefetch_tmap(&maps.sw);
      prefetch_tmap(&maps.sx);
      int it = 0, sit = 0, lit = 0;  // operand stages, scale stages, low-rank chunks issued
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
        for (int ks = 0; ks < p.k_stages && ok; ++ks) {
          const int s = it % STAGES, ss = sit % SC_SLOTS;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(&maps.a, &full[s], st, ks * BK, mt * BM);
          tma_load_2d(&maps.b, &full[s], st + STAGE_A, ks * BK, nt * BN);
          ++it;
          if (!mbar_wait(&sc_empty[ss], ((sit / SC_SLOTS) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* sc = scring + ss * SC_BYTES;
          mbar_arrive_expect_tx(&sc_full[ss], SC_BYTES);
          tma_load_2d(&maps.sw, &sc_full[ss], sc, nt * BN, ks * GPS);
          tma_load_2d(&maps.sx, &sc_full[ss], sc + SC_SW, mt * BM, ks * GPS);
          ++sit;
        }
      }
      if (!ok) {  // drain copies still in flight
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, p.limit);
        for (int j = (sit > SC_SLOTS ? sit - SC_SLOTS : 0); j < sit; ++j)
          mbar_wait_drain(&sc_full[j % SC_SLOTS], (j / SC_SLOTS) & 1, p.limit);
        if (lit > 0) mbar_wait_drain(lr_full, (lit - 1) & 1, p.limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, lit = 0, unit = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        if (p.n_lr > 0) {
          const int b = unit % NBUF;
          if (!mbar_wait(&acc_empty[b], ((unit / NBUF) & 1) ^ 1, wc)) break;
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
              mma_bf16(tmem + b * UNIT_COLS, make_sdesc(a_addr + 32 * kk, 16, sbo, layout),
                       make_sdesc(b_addr + 32 * kk, 16, sbo, layout), IDESC_BF16, accum);
              accum = 1;
            }
            umma_commit(lr_empty);
          }
          if (!ok) break;
          umma_commit(&acc_full[b]);
          ++unit;
        }
        for (int ks = 0; ks < p.k_stages && ok; ++ks, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + s * STAGE_BYTES), b_addr = a_addr + STAGE_A;
          const int b = unit % NBUF;
          if (!mbar_wait(&acc_empty[b], ((unit / NBUF) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int g = 0; g < GPS; ++g) {  // each group into its own 128 columns of the unit
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {  // K = 32 codes (bytes) per instruction
              const uint32_t off = 64 * g + 32 * kk;
              mma_f8f6f4(tmem + b * UNIT_COLS + g * BN, make_sdesc(a_addr + off, 16, 1024, LAYOUT_SW128),
                         make_sdesc(b_addr + off, 16, 1024, LAYOUT_SW128), IDESC_E4M3, (uint32_t)kk);
            }
          }
          umma_commit(&acc_full[b]);
          ++unit;
          umma_commit(&empty[s]);
        }
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, p.limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int part = (warp - EPI_WARP0) >> 2;
    const int rq = 32 * q + (lane >> 2);             // fragment rows rq + 8i
    const int cq = part * EPI_COLS + 2 * (lane & 3);  // fragment columns cq + 8j + e
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(part * EPI_COLS);
    const uint32_t tq_hi = tq + (16u << 16);
    int it = 0, unit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int m0 = mt * BM + rq;
      const int n0 = nt * BN + cq;
      float2 y[32];  // y[8i + j] = columns 8j, 8j + 1 of row 8i (of this thread's fragment)
#pragma unroll
      for (int j = 0; j < 32; ++j) y[j] = make_float2(0.f, 0.f);
      if (p.n_lr > 0) {
        const int b = unit % NBUF;
        if (!mbar_wait(&acc_full[b], (unit / NBUF) & 1, wc)) break;
        tc_fence_after();
        uint32_t lo[32], hi[32];
        tmem_ld_16x256b_x8(tq + b * UNIT_COLS, lo);
        tmem_ld_16x256b_x8(tq_hi + b * UNIT_COLS, hi);
        tmem_ld_wait_regs(lo);
        reg_order(hi);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t(&r)[32] = i < 2 ? lo : hi;
            y[8 * i + j] = make_float2(__uint_as_float(r[4 * j + 2 * (i & 1)]), __uint_as_float(r[4 * j + 2 * (i & 1) + 1]));
          }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        ++unit;
      }
      // One unit per K stage: the accumulators of its GPS groups, drained one
      // group at a time; the unit is released once its last group is in
      // registers.
      for (int ks = 0; ks < p.k_stages && ok; ++ks, ++it, ++unit) {
        const int ss = it % SC_SLOTS;
        const int b = unit % NBUF;
        if (!mbar_wait(&sc_full[ss], (it / SC_SLOTS) & 1, wc) || !mbar_wait(&acc_full[b], (unit / NBUF) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* sc = scring + ss * SC_BYTES;
#pragma unroll 1
        for (int g = 0; g < GPS; ++g) {
          uint32_t lo[32], hi[32];
          tmem_ld_16x256b_x8(tq + b * UNIT_COLS + g * BN, lo);
          tmem_ld_16x256b_x8(tq_hi + b * UNIT_COLS + g * BN, hi);
          tmem_ld_wait_regs(lo);
          reg_order(hi);
          if (g == GPS - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);  // every group of the unit is in registers
          }
          if (DBG) {
            export_frag(p, (size_t)(ks * GPS + g), m0, n0, lo, hi);
          } else {
            const __half* sxs = (const __half*)(sc + SC_SW) + g * BM + rq;
            float2 sx[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sx[i].x = sx[i].y = __half2float(sxs[8 * i]);
            drain_frag(y, lo, hi, (const float*)sc + g * BN + cq, sx);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sc_empty[ss]);
      }
      if (!ok) break;
      if (!DBG) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = n0 + 8 * j;
          if (n >= p.N) continue;
          const float2 bb = __ldg((const float2*)(p.bias + n));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = m0 + 8 * i;
            if (m < p.M) {
              __nv_bfloat162 h = __floats2bfloat162_rn(y[8 * i + j].x + bb.x, y[8 * i + j].y + bb.y);
              *(__nv_bfloat162*)(p.Y + (size_t)m * p.N + n) = h;
            }
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

}  // namespace

int launch_gemm_int4(const svdq_layer* L, int64_t M, void* Y, uint8_t* ws, const Workspace& w, int32_t* acc_dbg,
                     cudaStream_t stream) {
  I4Maps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int K = (int)L->K, N = (int)L->N, r = L->rank;
  const int64_t sld = int4_scale_ld(M);
  int st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.codes, (uint64_t)K, (uint64_t)M, (uint64_t)K,
                          BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  st = encode_tmap_2d(&maps.sw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, L->wscales, (uint64_t)N, (uint64_t)K / 64,
                      (uint64_t)N * 4, BN, GPS, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != SVDQ_OK) return st;
  st = encode_tmap_2d(&maps.sx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + w.scales, (uint64_t)sld, (uint64_t)K / 64,
                      (uint64_t)sld * 2, BM, GPS, CU_TENSOR_MAP_SWIZZLE_NONE);
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
  p.bias = L->bias;
  p.Y = (uint16_t*)Y;
  p.acc_dbg = acc_dbg;
  p.status = (int*)(ws + w.status);
  p.limit = wait_limit_cycles();
  const int grid = p.num_tiles < device_sm_count(L->device) ? p.num_tiles : device_sm_count(L->device);
  if (acc_dbg) {
    if (cudaFuncSetAttribute(k_gemm_int4<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
        cudaSuccess)
      return SVDQ_ERR_CUDA;
    k_gemm_int4<true><<<grid, THREADS, SMEM_BYTES, stream>>>(maps, p);
  } else {
    if (cudaFuncSetAttribute(k_gemm_int4<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
        cudaSuccess)
      return SVDQ_ERR_CUDA;
    k_gemm_int4<false><<<grid, THREADS, SMEM_BYTES, stream>>>(maps, p);
  }
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace svdq
