// K2: NVFP4 W4A4 GEMM of the svdq_w4a4 layer on 5th-generation tensor cores,
// with the low-rank up-projection and the output epilogue fused in.
//
//   Y = g_x g_w * [ sum_blocks (s_x s_w) (qx . qw)  +  t . (L2 / (g_x g_w)) ] + b
//
// "Суть метода" ("Hugging Face встроила Nunchaku в Diffusers ..."): the 4-bit
// product of quantized activations and quantized residual weights, plus the
// 16-bit low-rank branch, plus the bias.  Because both per-tensor scales are
// powers of two, L2 / (g_x g_w) is exact in bf16 and the low-rank product can
// accumulate into the same fp32 tensor-memory accumulator as the block-scaled
// 4-bit product; the epilogue then only applies the exact power-of-two scale,
// adds the bias and rounds to bf16.
//
// Persistent, warp-specialized CTA (one per SM), tile 128 x 192:
//   warp 0      TMA producer: per stage a 128x256 activation-code tile and a
//               192x256 weight-code tile (128-byte swizzle); the t / L2^T chunks
//               of the low-rank branch ride the same ring first.
//   warp 10     scale-factor producer: the E4M3 scale-factor atoms of two K
//               stages per bulk copy (activation and weight side) into a ring of
//               their own, so they arrive ahead of the codes they scale.
//   warp 1      owns tensor memory (512 columns: two 192-column fp32
//               accumulators for ping-pong with the epilogue, and two 48-column
//               scale-factor buffers); one lane issues tcgen05.mma kind::f16
//               (low rank, K=16) and kind::mxf4nvf4 block16 (K=64).
//   warps 6-9   move each stage's E4M3 scale-factor atoms from shared memory
//               into their tensor-memory lane quarter with tcgen05.st, in the
//               replicated layout the block-scaled MMA reads, so the transfer
//               runs beside the tensor pipe instead of inside it; with their own
//               ring they finish before the stage's codes land.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator rows, scale, bias,
//               bf16 round-to-nearest-even into a 128B-swizzled shared-memory
//               staging tile, written to Y by TMA bulk-tensor stores.
// Every wait is bounded (see sm100.cuh); no load uses cluster multicast.
#include <cuda_bf16.h>

#include <cstring>

#include "sm100.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = kGemmBM;   // 128
constexpr int BN = kNvfp4BN;  // 192
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * 128;  // 256 fp4 per row
constexpr int B_BYTES = BN * 128;
constexpr int SFA_BYTES = 4 * kSfAtomBytes;      // 4 k-atoms x 128 rows
constexpr int SFB_BYTES = 4 * 2 * kSfAtomBytes;  // 4 k-atoms x 256 rows (192 used)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SF_SLOTS = 2;                                 // scale-factor ring
constexpr int SF_SLOT_BYTES = 2 * (SFA_BYTES + SFB_BYTES);  // two K stages: [SFA x2 | SFB x2]
constexpr int SF_WARP = 10;
constexpr int THREADS = 352;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL = 2 * BN;  // 384: two buffers of [SFA 16 | SFB 32] columns
constexpr uint32_t SF_BUF_COLS = 48;
constexpr int EPI_STAGE_BYTES = 32 * 128;  // one warp's 32 rows x 64 bf16, 128B-swizzled
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES + 4 * 2 * EPI_STAGE_BYTES;
constexpr uint32_t IDESC_NVF4 = idesc_nvf4_ue4m3(BM, BN);
constexpr uint32_t IDESC_BF16 = idesc_bf16_f32(BM, BN);
static_assert(STAGE_BYTES % 1024 == 0 && SF_SLOT_BYTES % 1024 == 0, "stage alignment");
static_assert(SMEM_BYTES + 1024 + 256 <= 227 * 1024, "shared memory budget");
static_assert(SF_COL + 2 * SF_BUF_COLS <= TMEM_COLS, "tensor memory budget");

struct GemmMaps {
  CUtensorMap a, b, t[3], l2[3], y;
};

struct GParams {
  int M, N, K, m_tiles, n_tiles, num_tiles, k_stages, katoms;
  int n_lr;
  int lr_off[4], lr_w[4];
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* bias;
  uint16_t* Y;
  float out_scale;       // g_x g_w (static activation scale)
  const float* gx_dev;   // dynamic activation scale: g_x left by the quantizer (else null)
  float g_w;
  int* status;
  unsigned long long limit;
  size_t sfa_bytes, sfb_bytes;  // extents of the scale-factor arrays (debug bounds checks)
};

__device__ __forceinline__ int lr_map_index(int w) { return w == 64 ? 0 : (w == 32 ? 1 : 2); }

__global__ void __launch_bounds__(THREADS, 1) k_gemm_nvfp4(const __grid_constant__ GemmMaps maps, const __grid_constant__ GParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sfring = smem + STAGES * STAGE_BYTES;                // [SF_SLOTS][SF_SLOT_BYTES]
  uint8_t* epi_stage = sfring + SF_SLOTS * SF_SLOT_BYTES;       // [4 warps][2][EPI_STAGE_BYTES]
  uint64_t* full = (uint64_t*)(smem + SMEM_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* mma_done = acc_empty + 2;   // [1]
  uint64_t* sf_ready = mma_done + 1;    // [2]
  uint64_t* sf_free = sf_ready + 2;     // [2]
  uint64_t* sfs_full = sf_free + 2;     // [SF_SLOTS]
  uint64_t* sfs_empty = sfs_full + SF_SLOTS;
  uint32_t* tmem_slot = (uint32_t*)(sfs_empty + SF_SLOTS);
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
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sf_ready[b], 4);
      mbar_init(&sf_free[b], 1);
    }
    for (int b = 0; b < SF_SLOTS; ++b) {
      mbar_init(&sfs_full[b], 1);
      mbar_init(&sfs_empty[b], 4);
    }
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
  if (threadIdx.x == 0) pdl_launch_dependents();  // the next kernel may start its prologue
  const uint32_t tmem = *tmem_slot;
  const int units = p.n_lr + p.k_stages;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&maps.a);
      prefetch_tmap(&maps.b);
      pdl_wait();  // the quantized activations come from the previous kernel
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int u = 0; u < units; ++u, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE_BYTES;
          if (u < p.n_lr) {
            const int w = p.lr_w[u], mi = lr_map_index(w);
            mbar_arrive_expect_tx(&full[s], (uint32_t)(BM + BN) * 2 * w);
            tma_load_2d(&maps.t[mi], &full[s], st, p.lr_off[u], mt * BM);
            tma_load_2d(&maps.l2[mi], &full[s], st + A_BYTES, p.lr_off[u], nt * BN);
          } else {
            const int ks = u - p.n_lr;
            mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
            tma_load_2d(&maps.a, &full[s], st, ks * 128, mt * BM);
            tma_load_2d(&maps.b, &full[s], st + A_BYTES, ks * 128, nt * BN);
          }
        }
      }
      if (!ok) {  // drain the copies still in flight
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, p.limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, local = 0, kst = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++local) {
        const int b = local & 1;
        if (!mbar_wait(&acc_empty[b], ((local >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * BN);
        uint32_t accum = 0;
        for (int u = 0; u < units; ++u, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
          if (u < p.n_lr) {
            const int w = p.lr_w[u];
            const uint32_t layout = w == 64 ? LAYOUT_SW128 : (w == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
            const uint32_t sbo = 8u * 2u * (uint32_t)w;  // 8 rows of w bf16
            for (int kk = 0; kk < w / 16; ++kk) {
              mma_bf16(d, make_sdesc(a_addr + 32 * kk, 16, sbo, layout), make_sdesc(b_addr + 32 * kk, 16, sbo, layout),
                       IDESC_BF16, accum);
              accum = 1;
            }
          } else {
            const int sb = kst & 1;
            if (!mbar_wait(&sf_ready[sb], (kst >> 1) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sfa_t = tmem + SF_COL + (uint32_t)sb * SF_BUF_COLS;
            const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvf4(d, make_sdesc(a_addr + 32 * j, 16, 1024, LAYOUT_SW128),
                       make_sdesc(b_addr + 32 * j, 16, 1024, LAYOUT_SW128), IDESC_NVF4, sfa_t + 4 * j, sfb_t + 8 * j,
                       accum);
              accum = 1;
            }
            umma_commit(&sf_free[sb]);
            ++kst;
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[b]);
      }
      umma_commit(mma_done);  // every MMA issued above has completed when this fires
      mbar_wait_drain(mma_done, 0, p.limit);
    }
  } else if (warp == SF_WARP) {
    // ------------------------------------------------------------ scale-factor producer
    // Pair j of a tile carries the atoms of K stages 2j and 2j+1 (one stage for
    // an odd tail): [SFA stage 2j | SFA 2j+1 | SFB stage 2j | SFB 2j+1].
    if (lane == 0) {
      pdl_wait();  // the activation scales come from the previous kernel
      int pit = 0;
      bool ok = true;
      const int pairs = (p.k_stages + 1) / 2;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int j = 0; j < pairs; ++j, ++pit) {
          const int slot = pit % SF_SLOTS;
          if (!mbar_wait(&sfs_empty[slot], ((pit / SF_SLOTS) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          const int ns = (2 * j + 1 < p.k_stages) ? 2 : 1;
          uint8_t* dst = sfring + slot * SF_SLOT_BYTES;
          mbar_arrive_expect_tx(&sfs_full[slot], (uint32_t)ns * (SFA_BYTES + SFB_BYTES));
          const size_t oa = ((size_t)mt * p.katoms + 8 * j) * kSfAtomBytes;
          const size_t ob = ((size_t)nt * p.katoms + 8 * j) * 2 * kSfAtomBytes;
          // (debug variant: a copy that would leave its array is not issued; the
          // stage's wait then expires, after the bounds error was recorded)
          if (SVDQ_INB(p.status, oa, ns * SFA_BYTES, p.sfa_bytes))
            bulk_load(dst, p.sfa + oa, ns * SFA_BYTES, &sfs_full[slot]);
          if (SVDQ_INB(p.status, ob, ns * SFB_BYTES, p.sfb_bytes))
            bulk_load(dst + 2 * SFA_BYTES, p.sfb + ob, ns * SFB_BYTES, &sfs_full[slot]);
        }
      }
      if (!ok) {  // drain the copies still in flight
        for (int j = (pit > SF_SLOTS ? pit - SF_SLOTS : 0); j < pit; ++j)
          mbar_wait_drain(&sfs_full[j % SF_SLOTS], (j / SF_SLOTS) & 1, p.limit);
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ scale-factor movers
    // Warp q owns tensor-memory lanes 32q..32q+31.  Lane l writes, for every
    // 128-row scale-factor atom of the stage, the atom's 16-byte row l (the
    // scales of rows l, l+32, l+64, l+96 for 4 consecutive K blocks) into 4
    // consecutive columns -- the same bytes in every lane quarter.
    const int q = warp & 3;
    int kst = 0, pit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      for (int ks = 0; ks < p.k_stages; ++ks, ++kst) {
        const int h = ks & 1, slot = pit % SF_SLOTS, sb = kst & 1;
        const bool last_of_pair = h == 1 || ks + 1 == p.k_stages;
        if (h == 0) ok = mbar_wait(&sfs_full[slot], (pit / SF_SLOTS) & 1, wc);
        ok = ok && mbar_wait(&sf_free[sb], ((kst >> 1) & 1) ^ 1, wc);
        if (!ok) break;
        const uint8_t* sfa_s = sfring + slot * SF_SLOT_BYTES + h * SFA_BYTES;
        const uint8_t* sfb_s = sfring + slot * SF_SLOT_BYTES + 2 * SFA_BYTES + h * SFB_BYTES;
        uint32_t ra[16], rb[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 a = *(const uint4*)(sfa_s + j * kSfAtomBytes + lane * 16);
          ra[4 * j] = a.x; ra[4 * j + 1] = a.y; ra[4 * j + 2] = a.z; ra[4 * j + 3] = a.w;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint4 b4 = *(const uint4*)(sfb_s + (2 * j + hh) * kSfAtomBytes + lane * 16);
            rb[8 * j + 4 * hh] = b4.x; rb[8 * j + 4 * hh + 1] = b4.y; rb[8 * j + 4 * hh + 2] = b4.z; rb[8 * j + 4 * hh + 3] = b4.w;
          }
        }
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + SF_COL + (uint32_t)sb * SF_BUF_COLS;
        tmem_st_32x32b_x16(tq, ra);
        tmem_st_32x32b_x32(tq + 16, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sf_ready[sb]);
          if (last_of_pair) mbar_arrive(&sfs_empty[slot]);  // the slot's atoms are in tensor memory
        }
        if (last_of_pair) ++pit;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();  // g_x and Y belong to the stream's order
    const float out_scale = p.gx_dev != nullptr ? *p.gx_dev * p.g_w : p.out_scale;  // exact: powers of two
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    uint8_t* stg = epi_stage + (warp - 2) * 2 * EPI_STAGE_BYTES;
    int local = 0, sbuf = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int b = local & 1;
      if (!mbar_wait(&acc_full[b], (local >> 1) & 1, wc)) break;
      tc_fence_after();
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int m0 = mt * BM + 32 * q;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c) {
        const int n0 = nt * BN + 64 * c;
        uint8_t* dst = stg + sbuf * EPI_STAGE_BYTES + lane * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float bb[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = n0 + 32 * h + 4 * j;
            const float4 v = (n < p.N) ? __ldg((const float4*)(p.bias + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
            bb[4 * j] = v.x;
            bb[4 * j + 1] = v.y;
            bb[4 * j + 2] = v.z;
            bb[4 * j + 3] = v.w;
          }
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + 64 * c + 32 * h, r);
          tmem_ld_wait();
          if (c == BN / 64 - 1 && h == 1) {
            tc_fence_before();
            mbar_arrive(&acc_empty[b]);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 16-byte chunk 4h+k of this row, swizzled
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 8 * k + 2 * e;
              const float y0 = fmaf(__uint_as_float(r[j]), out_scale, bb[j]);
              const float y1 = fmaf(__uint_as_float(r[j + 1]), out_scale, bb[j + 1]);
              __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
              o[e] = *(uint32_t*)&hv;
            }
            const int chunk = 4 * h + k;
            *(uint4*)(dst + ((chunk ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&maps.y, stg + sbuf * EPI_STAGE_BYTES, n0, m0);
          bulk_commit();
          bulk_wait_read<1>();  // the other staging buffer is free again
        }
        __syncwarp();
        sbuf ^= 1;
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------
// CTA-pair variant: a cluster of two CTAs computes a 256 x 192 tile with
// tcgen05.mma cta_group::2 (M = 256).  CTA r of the pair holds accumulator rows
// 128r..128r+127 in its own tensor memory; its shared memory holds activation
// rows 128r.. of the tile and weight rows 96r..96r+95 (each CTA loads its own
// halves -- no multicast), and the pair MMA reads the B halves of both CTAs.
// Per SM and per 256-deep K stage that is 16 KiB of activation codes and
// 12 KiB of weight codes for the same tensor work as the single-CTA tile's
// 16 + 24 KiB.  Each CTA stages the E4M3 scale-factor atoms of its own 128
// rows and of all 192 weight rows; the leader copies them into both CTAs'
// tensor memory with tcgen05.cp.cta_group::2 in the tensor pipe, in order with
// the MMAs that read them, so the scale factors need no cross-CTA handshake of
// their own.  Only CTA 0 ("leader") issues tensor-core work; its barriers count
// the bytes of both CTAs' loads and the arrivals of both CTAs' epilogues, and
// its completions are signalled to the same barrier in both CTAs.
constexpr int PB_ROWS = BN / 2;              // 96 weight rows per CTA
constexpr int P_STAGES = 6;
constexpr int P_B_BYTES = PB_ROWS * 128;     // 12 KiB
constexpr int P_STAGE_BYTES = A_BYTES + P_B_BYTES;
constexpr int P_THREADS = 224;               // warps: 0 operands, 1 MMA, 2-5 epilogue, 6 scale factors
constexpr int P_SF_WARP = 6;
constexpr uint32_t P_SF_COL = 2 * BN;        // one 48-column scale-factor buffer
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES + 4 * 2 * EPI_STAGE_BYTES;
constexpr uint32_t P_IDESC_NVF4 = idesc_nvf4_ue4m3(2 * BM, BN);
constexpr uint32_t P_IDESC_BF16 = idesc_bf16_f32(2 * BM, BN);
static_assert(P_STAGE_BYTES % 1024 == 0 && P_B_BYTES % 1024 == 0, "pair stage alignment");
static_assert(P_SMEM_BYTES + 1024 + 256 <= 227 * 1024, "pair shared memory budget");

struct PairMaps {
  CUtensorMap a, b, t[3], l2[3], y, sfa, sfb;  // sfa/sfb: scale-factor atoms as rows of 128 u32
};

__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
    k_gemm_nvfp4_pair(const __grid_constant__ PairMaps maps, const __grid_constant__ GParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sfring = smem + P_STAGES * P_STAGE_BYTES;
  uint8_t* epi_stage = sfring + SF_SLOTS * SF_SLOT_BYTES;
  uint64_t* full = (uint64_t*)(smem + P_SMEM_BYTES);  // leader: operand stages of both CTAs
  uint64_t* empty = full + P_STAGES;                  // both: released by the leader's MMAs
  uint64_t* acc_full = empty + P_STAGES;              // both [2]
  uint64_t* acc_empty = acc_full + 2;                 // leader [2]: 8 epilogue warps
  uint64_t* mma_done = acc_empty + 2;                 // leader
  uint64_t* sfs_full = mma_done + 1;                  // leader [SF_SLOTS]: both CTAs' atoms
  uint64_t* sfs_empty = sfs_full + SF_SLOTS;          // both: released by the leader's MMAs
  uint32_t* tmem_slot = (uint32_t*)(sfs_empty + SF_SLOTS);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  WaitCtl wc{abort_flag, p.status, p.limit};
  const unsigned long long drain_limit = p.limit > (1ull << 24) ? p.limit : (1ull << 24);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < SF_SLOTS; ++b) {
      mbar_init(&sfs_full[b], 1);
      mbar_init(&sfs_empty[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  if (threadIdx.x == 0) pdl_launch_dependents();  // the next kernel may start its prologue
  const uint32_t tmem = *tmem_slot;
  const int units = p.n_lr + p.k_stages;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      prefetch_tmap(&maps.a);
      prefetch_tmap(&maps.b);
      pdl_wait();  // the quantized activations come from the previous kernel
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        const int arow = mt * 2 * BM + (int)rank * BM, brow = nt * BN + (int)rank * PB_ROWS;
        for (int u = 0; u < units; ++u, ++it) {
          const int s = it % P_STAGES;
          if (!mbar_wait(&empty[s], ((it / P_STAGES) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * P_STAGE_BYTES;
          const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
          if (u < p.n_lr) {
            const int w = p.lr_w[u], mi = lr_map_index(w);
            if (leader) mbar_arrive_expect_tx(&full[s], 2u * (uint32_t)(BM + PB_ROWS) * 2 * w);
            tma_load_2d_pair(&maps.t[mi], fbar, st, p.lr_off[u], arow);
            tma_load_2d_pair(&maps.l2[mi], fbar, st + A_BYTES, p.lr_off[u], brow);
          } else {
            const int ks = u - p.n_lr;
            if (leader) mbar_arrive_expect_tx(&full[s], 2u * P_STAGE_BYTES);
            tma_load_2d_pair(&maps.a, fbar, st, ks * 128, arow);
            tma_load_2d_pair(&maps.b, fbar, st + A_BYTES, ks * 128, brow);
          }
        }
      }
      if (!ok && leader) {  // drain the copies of both CTAs still in flight
        for (int j = (it > P_STAGES ? it - P_STAGES : 0); j < it; ++j)
          mbar_wait_drain(&full[j % P_STAGES], (j / P_STAGES) & 1, drain_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int it = 0, local = 0, pit = 0;
      bool ok = true;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs, ++local) {
        const int b = local & 1;
        if (!mbar_wait_cl(&acc_empty[b], ((local >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * BN);
        uint32_t accum = 0;
        for (int u = 0; u < units; ++u, ++it) {
          const int s = it % P_STAGES;
          if (!mbar_wait(&full[s], (it / P_STAGES) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * P_STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
          if (u < p.n_lr) {
            const int w = p.lr_w[u];
            const uint32_t layout = w == 64 ? LAYOUT_SW128 : (w == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
            const uint32_t sbo = 8u * 2u * (uint32_t)w;  // 8 rows of w bf16
            for (int kk = 0; kk < w / 16; ++kk) {
              mma_bf16_pair(d, make_sdesc(a_addr + 32 * kk, 16, sbo, layout),
                            make_sdesc(b_addr + 32 * kk, 16, sbo, layout), P_IDESC_BF16, accum);
              accum = 1;
            }
          } else {
            // this stage's scale-factor atoms into tensor memory, in the tensor
            // pipe ahead of the MMAs that read them (one buffer: the pipe keeps
            // this thread's copies and MMAs in order)
            const int ks = u - p.n_lr, h = ks & 1, slot = pit % SF_SLOTS;
            const bool last_of_pair = h == 1 || ks + 1 == p.k_stages;
            if (h == 0 && !mbar_wait(&sfs_full[slot], (pit / SF_SLOTS) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sfa_s = smem_u32(sfring + slot * SF_SLOT_BYTES + h * SFA_BYTES);
            const uint32_t sfb_s = smem_u32(sfring + slot * SF_SLOT_BYTES + 2 * SFA_BYTES + h * SFB_BYTES);
            const uint32_t sfa_t = tmem + P_SF_COL, sfb_t = sfa_t + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_cp_32x128b_x4_pair(sfa_t + 4 * j, make_sdesc(sfa_s + j * kSfAtomBytes, 0, 128, LAYOUT_NONE));
              tmem_cp_32x128b_x4_pair(sfb_t + 8 * j, make_sdesc(sfb_s + 2 * j * kSfAtomBytes, 0, 128, LAYOUT_NONE));
              tmem_cp_32x128b_x4_pair(sfb_t + 8 * j + 4,
                                      make_sdesc(sfb_s + (2 * j + 1) * kSfAtomBytes, 0, 128, LAYOUT_NONE));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvf4_pair(d, make_sdesc(a_addr + 32 * j, 16, 1024, LAYOUT_SW128),
                            make_sdesc(b_addr + 32 * j, 16, 1024, LAYOUT_SW128), P_IDESC_NVF4, sfa_t + 4 * j,
                            sfb_t + 8 * j, accum);
              accum = 1;
            }
            if (last_of_pair) {  // the slot's atoms are read once these MMAs complete
              umma_commit_pair(&sfs_empty[slot], 3);
              ++pit;
            }
          }
          umma_commit_pair(&empty[s], 3);
        }
        if (ok) umma_commit_pair(&acc_full[b], 3);
      }
      umma_commit_pair(mma_done, 1);  // every pair MMA issued above has completed when this fires
      mbar_wait_drain(mma_done, 0, drain_limit);
    }
  } else if (warp == P_SF_WARP) {
    // ------------------------------------------------------------ scale-factor producer (both CTAs)
    // Two K stages per slot: [SFA 2j | SFA 2j+1 | SFB 2j | SFB 2j+1], this CTA's
    // 128 activation rows (atom tile 2 mt + rank) and all 192 weight rows; the
    // copies of both CTAs complete on the leader's barrier.
    if (lane == 0) {
      prefetch_tmap(&maps.sfa);
      prefetch_tmap(&maps.sfb);
      pdl_wait();
      int pit = 0;
      bool ok = true;
      const int pairs_k = (p.k_stages + 1) / 2;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        const int at = 2 * mt + (int)rank;
        for (int j = 0; j < pairs_k; ++j, ++pit) {
          const int slot = pit % SF_SLOTS;
          if (!mbar_wait(&sfs_empty[slot], ((pit / SF_SLOTS) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          const int ns = (2 * j + 1 < p.k_stages) ? 2 : 1;
          uint8_t* dst = sfring + slot * SF_SLOT_BYTES;
          const uint32_t fbar = mapa_shared(smem_u32(&sfs_full[slot]), 0);
          if (leader) mbar_arrive_expect_tx(&sfs_full[slot], 2u * (uint32_t)ns * (SFA_BYTES + SFB_BYTES));
          for (int h = 0; h < ns; ++h) {
            tma_load_2d_pair(&maps.sfa, fbar, dst + h * SFA_BYTES, 0, at * p.katoms + 8 * j + 4 * h);
            tma_load_2d_pair(&maps.sfb, fbar, dst + 2 * SFA_BYTES + h * SFB_BYTES, 0,
                             (nt * p.katoms + 8 * j + 4 * h) * 2);
          }
        }
      }
      if (!ok && leader) {
        for (int j = (pit > SF_SLOTS ? pit - SF_SLOTS : 0); j < pit; ++j)
          mbar_wait_drain(&sfs_full[j % SF_SLOTS], (j / SF_SLOTS) & 1, drain_limit);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    pdl_wait();  // g_x and Y belong to the stream's order
    const float out_scale = p.gx_dev != nullptr ? *p.gx_dev * p.g_w : p.out_scale;  // exact: powers of two
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    uint8_t* stg = epi_stage + (warp - 2) * 2 * EPI_STAGE_BYTES;
    const uint32_t empty_cl0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    const uint32_t empty_cl1 = mapa_shared(smem_u32(&acc_empty[1]), 0);
    int local = 0, sbuf = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++local) {
      const int b = local & 1;
      if (!mbar_wait(&acc_full[b], (local >> 1) & 1, wc)) break;
      tc_fence_after();
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int m0 = mt * 2 * BM + (int)rank * BM + 32 * q;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c) {
        const int n0 = nt * BN + 64 * c;
        uint8_t* dst = stg + sbuf * EPI_STAGE_BYTES + lane * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float bb[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = n0 + 32 * h + 4 * j;
            const float4 v = (n < p.N) ? __ldg((const float4*)(p.bias + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
            bb[4 * j] = v.x;
            bb[4 * j + 1] = v.y;
            bb[4 * j + 2] = v.z;
            bb[4 * j + 3] = v.w;
          }
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + 64 * c + 32 * h, r);
          tmem_ld_wait();
          if (c == BN / 64 - 1 && h == 1) {  // the whole accumulator is in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(b ? empty_cl1 : empty_cl0);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 16-byte chunk 4h+k of this row, swizzled
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 8 * k + 2 * e;
              const float y0 = fmaf(__uint_as_float(r[j]), out_scale, bb[j]);
              const float y1 = fmaf(__uint_as_float(r[j + 1]), out_scale, bb[j + 1]);
              __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
              o[e] = *(uint32_t*)&hv;
            }
            const int chunk = 4 * h + k;
            *(uint4*)(dst + ((chunk ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (m0 < p.M && n0 < p.N) {  // boxes wholly past the edge are skipped
            tma_store_2d(&maps.y, stg + sbuf * EPI_STAGE_BYTES, n0, m0);
            bulk_commit();
            bulk_wait_read<1>();  // the other staging buffer is free again
          } else {
            bulk_wait_read<0>();  // no store from this buffer: both buffers are free
          }
        }
        __syncwarp();
        sbuf ^= 1;
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  // Neither CTA leaves (or frees tensor memory) while the pair MMAs, the peer's
  // remote arrivals or its loads completing on the leader's barriers may still
  // touch it.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

int sm_count(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Largest number of co-resident CTA pairs of the pair kernel on a device (0 if
// the query fails), cached per device.
int pair_clusters(int dev, size_t smem) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(P_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_gemm_nvfp4_pair, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = -1;
    }
    cache[dev] = n;
  }
  return cache[dev] > 0 ? cache[dev] : 0;
}

}  // namespace

int launch_gemm_nvfp4(const svdq_layer* L, int64_t M, void* Y, uint8_t* ws, const Workspace& w, cudaStream_t stream) {
  const int K = (int)L->K, N = (int)L->N, r = L->rank;
  GParams p{};
  const LowRankChunks ch = lowrank_chunks(r);
  p.n_lr = ch.n;
  for (int i = 0; i < ch.n; ++i) {
    p.lr_off[i] = ch.off[i];
    p.lr_w[i] = ch.width[i];
  }
  p.M = (int)M;
  p.N = N;
  p.K = K;
  p.n_tiles = (N + BN - 1) / BN;
  p.k_stages = K / kKStage;
  p.katoms = K / 64;
  p.sfa = ws + w.scales;
  p.sfb = L->wscales;
  p.bias = L->bias;
  p.Y = (uint16_t*)Y;
  p.out_scale = L->g_x * L->g_w;
  p.g_w = L->g_w;
  p.gx_dev = L->dyn_gx ? (const float*)(ws + w.status + 4) : nullptr;
  p.status = (int*)(ws + w.status);
  p.limit = wait_limit_cycles();
  p.sfa_bytes = w.scales_bytes;
  p.sfb_bytes = L->off.total - L->off.wscales;

  // Token counts above one 128-row tile use the CTA-pair kernel (256-row tiles)
  // when the device can co-schedule its clusters.
  const size_t psmem = 1024 + (size_t)P_SMEM_BYTES + 256;
  if (M > BM) {
    static int attr_done[64] = {0};
    const int dev = L->device;
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
      if (cudaFuncSetAttribute(k_gemm_nvfp4_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem) !=
          cudaSuccess)
        return SVDQ_ERR_CUDA;
      attr_done[dev] = 1;
    }
    const int maxc = pair_clusters(dev, psmem);
    if (maxc > 0) {
      PairMaps maps;
      std::memset(&maps, 0, sizeof(maps));
      int st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.codes, (uint64_t)K / 2, (uint64_t)M,
                              (uint64_t)K / 2, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B);
      if (st != SVDQ_OK) return st;
      maps.b = L->map_w_half;
      if (r > 0) {
        const int widths[3] = {64, 32, 16};
        const CUtensorMapSwizzle swz[3] = {CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_SWIZZLE_64B,
                                           CU_TENSOR_MAP_SWIZZLE_32B};
        for (int i = 0; i < 3; ++i) {
          if (widths[i] > r) continue;
          st = encode_tmap_2d(&maps.t[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + w.t, (uint64_t)r, (uint64_t)M,
                              (uint64_t)r * 2, widths[i], BM, swz[i]);
          if (st != SVDQ_OK) return st;
          maps.l2[i] = L->map_l2_half[i];
        }
      }
      st = encode_tmap_2d(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 64,
                          32, CU_TENSOR_MAP_SWIZZLE_128B);
      if (st != SVDQ_OK) return st;
      // scale-factor atoms (512 B each) as rows of 128 u32: 4 k-atoms (one K
      // stage) per activation load, 8 per weight load (two atoms per k-atom)
      const uint64_t sfa_rows = (uint64_t)((M + 2 * BM - 1) / (2 * BM)) * 2 * (K / 64);
      const uint64_t sfb_rows = (uint64_t)((N + BN - 1) / BN) * (K / 64) * 2;
      st = encode_tmap_2d(&maps.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT32, ws + w.scales, 128, sfa_rows, kSfAtomBytes, 128, 4,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
      if (st != SVDQ_OK) return st;
      st = encode_tmap_2d(&maps.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT32, L->wscales, 128, sfb_rows, kSfAtomBytes, 128, 8,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
      if (st != SVDQ_OK) return st;
      p.m_tiles = (int)((M + 2 * BM - 1) / (2 * BM));
      p.num_tiles = p.m_tiles * p.n_tiles;
      const int npairs = p.num_tiles < maxc ? p.num_tiles : maxc;
      if (launch_pdl(k_gemm_nvfp4_pair, dim3(2 * npairs), dim3(P_THREADS), psmem, stream, maps, p) != cudaSuccess)
        return SVDQ_ERR_CUDA;
      return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
    }
  }

  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  int st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.codes, (uint64_t)K / 2, (uint64_t)M,
                          (uint64_t)K / 2, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  maps.b = L->map_w;
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
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.num_tiles = p.m_tiles * p.n_tiles;
  st = encode_tmap_2d(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  const size_t smem = 1024 + (size_t)SMEM_BYTES + 256;
  if (cudaFuncSetAttribute(k_gemm_nvfp4, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  const int grid = p.num_tiles < sm_count(L->device) ? p.num_tiles : sm_count(L->device);
  if (launch_pdl(k_gemm_nvfp4, dim3(grid), dim3(THREADS), smem, stream, maps, p) != cudaSuccess) return SVDQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace svdq
