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
//               192x256 weight-code tile (128-byte swizzle).  The low-rank
//               branch's t / L2^T tiles: for ranks up to 32 into a buffer of
//               their own, once per tile (a slot of the operand ring costs a
//               whole stage of the pipeline, ~7 % of a 3072-deep tile); larger
//               ranks ride the ring in chunks ahead of the K stages.
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
//               staging tile (one per warp), written to Y by TMA bulk-tensor
//               stores.
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
// Ranks up to 32 (one low-rank chunk) have a buffer of their own, loaded once per
// tile ahead of the tile's first MMA, instead of a slot of the operand ring: t
// [128 x r] and the L2^T chunk [192 x r], bf16.
constexpr int LR_MAX = 32;
constexpr int LR_T_BYTES = BM * LR_MAX * 2;
constexpr int LR_BYTES = LR_T_BYTES + BN * LR_MAX * 2;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES + 4 * EPI_STAGE_BYTES + LR_BYTES;
constexpr uint32_t IDESC_NVF4 = idesc_nvf4_ue4m3(BM, BN);
constexpr uint32_t IDESC_BF16 = idesc_bf16_f32(BM, BN);
static_assert(STAGE_BYTES % 1024 == 0 && SF_SLOT_BYTES % 1024 == 0 && LR_T_BYTES % 1024 == 0, "stage alignment");
static_assert(SMEM_BYTES + 1024 + 256 <= 227 * 1024, "shared memory budget");
static_assert(SF_COL + 2 * SF_BUF_COLS <= TMEM_COLS, "tensor memory budget");

struct GemmMaps {
  CUtensorMap a, b, t[3], l2[3], y;
};

struct GParams {
  int M, N, K, m_tiles, n_tiles, num_tiles, k_stages, katoms;
  int n_lr;
  int lr_off[4], lr_w[4];
  int lr_buf_w;  // width of the single low-rank chunk held in its own buffer (0: none / on the ring)
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

// Output tile of a persistent CTA's work index: M tiles vary fastest, so the
// CTAs running at one time share few weight tiles.
__device__ __forceinline__ void tile_coords(int tile, const GParams& p, int& mt, int& nt) {
  mt = tile % p.m_tiles;
  nt = tile / p.m_tiles;
}

__global__ void __launch_bounds__(THREADS, 1) k_gemm_nvfp4(const __grid_constant__ GemmMaps maps, const __grid_constant__ GParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sfring = smem + STAGES * STAGE_BYTES;                // [SF_SLOTS][SF_SLOT_BYTES]
  uint8_t* epi_stage = sfring + SF_SLOTS * SF_SLOT_BYTES;       // [4 warps][EPI_STAGE_BYTES]
  uint8_t* lrbuf = epi_stage + 4 * EPI_STAGE_BYTES;             // [t | L2^T chunk], 1024-aligned
  uint64_t* full = (uint64_t*)(smem + SMEM_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* mma_done = acc_empty + 2;   // [1]
  uint64_t* sf_ready = mma_done + 1;    // [2]
  uint64_t* sf_free = sf_ready + 2;     // [2]
  uint64_t* sfs_full = sf_free + 2;     // [SF_SLOTS]
  uint64_t* sfs_empty = sfs_full + SF_SLOTS;
  uint64_t* lr_full = sfs_empty + SF_SLOTS;
  uint64_t* lr_free = lr_full + 1;
  uint32_t* tmem_slot = (uint32_t*)(lr_free + 1);
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
    mbar_init(lr_full, 1);
    mbar_init(lr_free, 1);
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
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, p, mt, nt);
        if (p.lr_buf_w > 0) {  // the tile's t and L2^T chunk, once the previous tile's MMAs read theirs
          const int w = p.lr_buf_w, mi = lr_map_index(w);
          if (!mbar_wait(lr_free, (lt & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(lr_full, (uint32_t)(BM + BN) * 2 * w);
          tma_load_2d(&maps.t[mi], lr_full, lrbuf, 0, mt * BM);
          tma_load_2d(&maps.l2[mi], lr_full, lrbuf + LR_T_BYTES, 0, nt * BN);
          ++lt;
        }
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
        if (lt > 0) mbar_wait_drain(lr_full, (lt - 1) & 1, p.limit);
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
        if (p.lr_buf_w > 0) {  // the low-rank product first, from its own buffer
          if (!mbar_wait(lr_full, local & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int w = p.lr_buf_w;
          const uint32_t layout = w == 32 ? LAYOUT_SW64 : LAYOUT_SW32;
          const uint32_t sbo = 8u * 2u * (uint32_t)w;
          const uint32_t a_addr = smem_u32(lrbuf), b_addr = a_addr + LR_T_BYTES;
          for (int kk = 0; kk < w / 16; ++kk) {
            mma_bf16(d, make_sdesc(a_addr + 32 * kk, 16, sbo, layout), make_sdesc(b_addr + 32 * kk, 16, sbo, layout),
                     IDESC_BF16, accum);
            accum = 1;
          }
          umma_commit(lr_free);
        }
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
        int mt, nt;
        tile_coords(tile, p, mt, nt);
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
        if (h == 0) ok = warp_wait(&sfs_full[slot], (pit / SF_SLOTS) & 1, wc);
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
        // the atoms are in registers before the wait for the tensor-memory buffer, so
        // the shared-memory reads stay off the MMA -> mover -> MMA chain
        if (!warp_wait(&sf_free[sb], ((kst >> 1) & 1) ^ 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();  // the MMAs that read this buffer completed: order the stores after them
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + SF_COL + (uint32_t)sb * SF_BUF_COLS;
        tmem_st_32x32b_x16(tq, ra);
        tmem_st_32x32b_x32(tq + 16, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sf_ready[sb]);
          // the slot is released only after the stores that consumed the loaded
          // registers: releasing it right after the shared-memory loads let the next
          // bulk copy into the slot overtake them (wrong scales at large K)
          if (last_of_pair) mbar_arrive(&sfs_empty[slot]);
        }
        if (last_of_pair) ++pit;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();  // g_x and Y belong to the stream's order
    const float out_scale = p.gx_dev != nullptr ? *p.gx_dev * p.g_w : p.out_scale;  // exact: powers of two
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    uint8_t* stg = epi_stage + (warp - 2) * EPI_STAGE_BYTES;
    int local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int b = local & 1;
      if (!mbar_wait(&acc_full[b], (local >> 1) & 1, wc)) break;
      tc_fence_after();
      int mt, nt;
      tile_coords(tile, p, mt, nt);
      const int m0 = mt * BM + 32 * q;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c) {
        const int n0 = nt * BN + 64 * c;
        uint8_t* dst = stg + lane * 128;
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
          tma_store_2d(&maps.y, stg, n0, m0);
          bulk_commit();
          bulk_wait_read<0>();  // the staging buffer is free again
        }
        __syncwarp();
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

}  // namespace

int launch_gemm_nvfp4(const svdq_layer* L, int64_t M, void* Y, uint8_t* ws, const Workspace& w, cudaStream_t stream) {
  const int K = (int)L->K, N = (int)L->N, r = L->rank;
  GParams p{};
  const LowRankChunks ch = lowrank_chunks(r);
  if (ch.n == 1 && ch.width[0] <= LR_MAX) {  // one chunk of at most 32: its own buffer
    p.n_lr = 0;
    p.lr_buf_w = ch.width[0];
  } else {
    p.n_lr = ch.n;
    p.lr_buf_w = 0;
    for (int i = 0; i < ch.n; ++i) {
      p.lr_off[i] = ch.off[i];
      p.lr_w[i] = ch.width[i];
    }
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
  const int grid = p.num_tiles < device_sm_count(L->device) ? p.num_tiles : device_sm_count(L->device);
  if (launch_pdl(k_gemm_nvfp4, dim3(grid), dim3(THREADS), smem, stream, maps, p) != cudaSuccess) return SVDQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace svdq
