// K8: the MLP up-projection GEMM with the down-projection's activation
// quantizer fused into its epilogue (cross-layer fusion of the MLP pair).
//
//   h  = bf16( g_x g_w [ sum_blocks (s_x s_w)(qx . qw) + t . L2/(g_x g_w) ] + b )   (the up layer's y)
//   x' = bf16( GELU(h) ),  GELU(h) = h/2 (1 + erf(h / sqrt 2)) in binary32 (gelu_erf2)
//   x^' = f32(x') * inv_lambda'                                                     (the down layer's input)
//   codes', E4M3 block scales'  of x^' (blocks of 16, static g_x'),  t' = bf16( bf16(x^') . L1' )
//
// "Hugging Face встроила Nunchaku в Diffusers ..." (iitog.ru), paragraph on
// Nunchaku Lite: the original engine's speed comes from fused, model-specific
// kernels.  Here the up layer's output never goes to memory: each epilogue
// thread owns one token row of the tile, so the 16-column blocks of the down
// layer's quantizer need no cross-thread step, and the up layer's N columns
// are the down layer's K columns.  The low-rank sum t' runs over all N columns
// of a row; each tile contributes bf16(x^'_tile) . L1'[tile columns] with a
// tensor-core MMA into a 32-column tensor-memory accumulator that persists
// across the tiles of a work unit (one 128-row M tile times one of S contiguous
// groups of N tiles), and the S partial sums of a row are added in a fixed
// order by the unit that finishes last (counter per 32-row group), as the
// standalone quantizer does for its K slices.
//
// Same main loop as the single-CTA NVFP4 GEMM (k_gemm_nvfp4: 128 x 192 tile,
// block-scaled kind::mxf4nvf4, scale factors moved into tensor memory by four
// mover warps), with a 3-stage operand ring to make room for the x^' tile and
// the L1' slice.  Roles per CTA (512 threads):
//   warp 0      operand TMA producer            warp 1   tensor memory, main MMAs
//   warps 2-9   epilogue: two warps per tensor-memory lane quarter, 96 columns each
//   warps 10-13 scale-factor movers             warp 14  scale-factor producer
//   warp 15     L1'^T slice loader and t' MMA issuer, per tile
// An epilogue thread's codes and scales would be scattered stores (32 rows per
// warp instruction), so the tile's codes (128 x 96 B) and its three scale atoms
// are staged in shared memory and written by one thread with a TMA tensor store
// and one bulk copy.  Tensor memory (512 columns): two 192-column accumulators,
// two 48-column scale-factor buffers and the 32-column t' accumulator, so the
// down layer's rank is at most 32.  Every wait is bounded; no load uses cluster
// multicast.
#include <cuda_bf16.h>

#include <cstring>

#include "sm100.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = kGemmBM;   // 128
constexpr int BN = kNvfp4BN;  // 192
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * 128;
constexpr int B_BYTES = BN * 128;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SFA_BYTES = 4 * kSfAtomBytes;
constexpr int SFB_BYTES = 4 * 2 * kSfAtomBytes;
constexpr int SF_SLOTS = 3;
constexpr int SF_SLOT_BYTES = SFA_BYTES + SFB_BYTES;  // one K stage: [SFA | SFB]
constexpr int XT_BYTES = 3 * BM * 128;  // bf16 x^' tile: three 64-column blocks, 128B-swizzled
constexpr int L1_MAX_ROWS = 32;         // rank rows of L1'^T (rank <= 32)
constexpr int L1_BYTES = 3 * L1_MAX_ROWS * 128;
constexpr int CST_BYTES = BM * BN / 2;  // the tile's down-layer codes, row-major (96 B per row)
constexpr int SST_BYTES = 3 * kSfAtomBytes;  // the tile's 12 block scales per row: three atoms
constexpr int THREADS = 512;
constexpr int SF_WARP = 14, T_WARP = 15;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL = 2 * BN;     // 384: two buffers of [SFA 16 | SFB 32] columns
constexpr uint32_t SF_BUF_COLS = 48;
constexpr uint32_t TP_COL = SF_COL + 2 * SF_BUF_COLS;  // 480
constexpr int SMEM_BYTES =
    STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES + XT_BYTES + L1_BYTES + 2 * (CST_BYTES + SST_BYTES);
constexpr uint32_t IDESC_NVF4 = idesc_nvf4_ue4m3(BM, BN);
constexpr uint32_t IDESC_BF16 = idesc_bf16_f32(BM, BN);
static_assert(STAGE_BYTES % 1024 == 0 && SF_SLOT_BYTES % 1024 == 0 && XT_BYTES % 1024 == 0, "alignment");
static_assert(SMEM_BYTES + 1024 + 512 <= 227 * 1024, "shared memory budget");
static_assert(TP_COL + 32 <= TMEM_COLS, "tensor memory budget");

struct FusedMaps {
  CUtensorMap a, b, t[3], l2[3], l1dn;
  CUtensorMap codes_dn;  // the down layer's activation codes [M, N/2] bytes, box 96 x 128 (stores)
};

struct FParams {
  int M, N, K, m_tiles, n_tiles, num_units, S, k_stages, katoms;
  int n_lr;
  int lr_off[4], lr_w[4];
  int rank_dn, katoms_dn;
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* bias;        // up layer
  float out_scale;          // g_x g_w of the up layer (static)
  const float* gx_dev;      // up layer's dynamic g_x (else null)
  float g_w;
  const float* inv_lambda_dn;
  float den_dn, inv_g_dn;   // 6 g_x' and 1/g_x' of the down layer (powers of two: exact)
  uint8_t* scales_dn;       // atom layout, 128-row tiles, katoms_dn
  uint16_t* t_dn;           // [M, rank_dn]
  float* tpart;             // [S, M, rank_dn]
  int* counters;            // per 32-row group (128-row block x lane quarter)
  uint16_t* H;              // optional [M, N] bf16: bf16(GELU(h))
  int* status;
  unsigned long long limit;
  // extents in bytes (debug bounds checks)
  size_t sfa_bytes, sfb_bytes, scales_dn_bytes, t_dn_bytes, tpart_bytes, cnt_bytes, H_bytes;
};

__device__ __forceinline__ int lr_map_index(int w) { return w == 64 ? 0 : (w == 32 ? 1 : 2); }

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

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU(h) = h Phi(h) = h/2 (1 + erf(h / sqrt 2)) in binary32 for two elements,
// packed f32x2 arithmetic, no branches.  With x = |h| / sqrt 2:
//   h < 0:  (h/2) erfc(x)          h >= 0:  h (1 - erfc(x)/2)
// (no cancellation on either side).  erfc(x) = t exp(-x^2 + P(t)), t = 1/(1 + x/2):
// the Chebyshev-fit form of Press et al., "Numerical Recipes" (2nd ed., sec.
// 6.2), with P a degree-9 polynomial fitted by least squares to
// log(erfc(x) e^(x^2) / t) at Chebyshev nodes in t in (0, 1], coefficients rounded
// to binary32 (relative error of erfc below 1.2e-7 before rounding).  The
// exponential is taken in base 2 and as the square of 2^(y/2), y = log2(erfc/t):
// 2^(y/2) stays normal down to y = -252, so erfc far below the binary32 normal
// range still comes out of one rounding of t 2^(y/2) 2^(y/2), as bf16 keeps it.
// +inf gives t = 0 and 2^(y/2) = 0, so h (1 - 0) = +inf; -0 gives -0 and NaN gives
// NaN through the h >= 0 form.  Simulated in binary32 over all 65536 bf16
// inputs, bf16(result) equals the binary64 definition rounded to bf16.  (A table
// of the correctly rounded results measured slower: its random reads cost more
// than this arithmetic.)
__device__ __forceinline__ float2 gelu_erf2(float2 h) {
  constexpr float HL2E = 0.72134752044448170f;  // log2(e) / 2
  const float2 d = __ffma2_rn(make_float2(fabsf(h.x), fabsf(h.y)), make_float2(0.35355339059327376f, 0.35355339059327376f),
                              make_float2(1.0f, 1.0f));  // 1 + |h| / (2 sqrt 2)
  const float2 t = make_float2(rcp_approx(d.x), rcp_approx(d.y));
  float2 p = make_float2(1.708930433e-01f * HL2E, 1.708930433e-01f * HL2E);
#define SVDQ_H(c) p = __ffma2_rn(p, t, make_float2((c) * HL2E, (c) * HL2E))
  SVDQ_H(-8.222485185e-01f);
  SVDQ_H(1.488708496e+00f);
  SVDQ_H(-1.135414600e+00f);
  SVDQ_H(2.790049911e-01f);
  SVDQ_H(-1.863418519e-01f);
  SVDQ_H(9.679660201e-02f);
  SVDQ_H(3.740904033e-01f);
  SVDQ_H(1.000023723e+00f);
  SVDQ_H(-1.265512228e+00f);
#undef SVDQ_H
  // y/2 = (-x^2 + P(t)) log2(e) / 2 = -h^2 log2(e) / 4 + P(t) log2(e) / 2
  const float2 y2 = __ffma2_rn(__fmul2_rn(h, make_float2(-0.5f * HL2E, -0.5f * HL2E)), h, p);
  const float2 e = make_float2(ex2_approx(y2.x), ex2_approx(y2.y));
  const float2 te = __fmul2_rn(__fmul2_rn(t, e), e);  // erfc(|h| / sqrt 2)
  const float2 ht = __fmul2_rn(te, make_float2(0.5f, 0.5f));
  const float2 q = __fmul2_rn(h, ht);                                        // h < 0: h erfc / 2
  const float2 r = __fmul2_rn(h, __ffma2_rn(ht, make_float2(-1.0f, -1.0f), make_float2(1.0f, 1.0f)));  // h (1 - erfc / 2)
  return make_float2(h.x < 0.0f ? q.x : r.x, h.y < 0.0f ? q.y : r.y);  // -0, +inf, NaN: r
}

__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_gelu_quant(const __grid_constant__ FusedMaps maps, const __grid_constant__ FParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sfring = smem + STAGES * STAGE_BYTES;
  uint8_t* xt = sfring + SF_SLOTS * SF_SLOT_BYTES;  // 1024-aligned
  uint8_t* l1s = xt + XT_BYTES;                     // 1024-aligned
  uint8_t* cst = l1s + L1_BYTES;                     // codes staging [2][128][96]
  uint8_t* sst = cst + 2 * CST_BYTES;                // scale staging [2][three atoms]
  uint64_t* full = (uint64_t*)(sst + 2 * SST_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;    // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]: 8 epilogue warps
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* sf_ready = mma_done + 1;      // [2]: 4 movers
  uint64_t* sf_free = sf_ready + 2;       // [2]
  uint64_t* sfs_full = sf_free + 2;       // [SF_SLOTS]
  uint64_t* sfs_empty = sfs_full + SF_SLOTS;
  uint64_t* l1_full = sfs_empty + SF_SLOTS;
  uint64_t* xt_full = l1_full + 1;        // [2] per staging buffer, 8 epilogue warps: x^' tile and codes/scales staged
  uint64_t* xt_free = xt_full + 2;        // t' MMAs of the tile done (x^' tile and L1' slot free)
  uint64_t* tp_full = xt_free + 1;        // the unit's t' sum is complete
  uint64_t* tp_empty = tp_full + 1;       // 4 reader warps
  uint64_t* tdone = tp_empty + 1;
  uint64_t* st_free = tdone + 1;          // [2] a staging buffer's stores have read it
  uint32_t* tmem_slot = (uint32_t*)(st_free + 2);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* ticket = abort_flag + 1;  // [4] one per lane-quarter reader warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.status, p.limit};
  const unsigned long long drain_limit = p.limit > (1ull << 24) ? p.limit : (1ull << 24);
  const int units = p.n_lr + p.k_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
      mbar_init(&sf_ready[b], 4);
      mbar_init(&sf_free[b], 1);
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < SF_SLOTS; ++b) {
      mbar_init(&sfs_full[b], 1);
      mbar_init(&sfs_empty[b], 4);
    }
    mbar_init(l1_full, 1);
    mbar_init(&xt_full[0], 8);
    mbar_init(&xt_full[1], 8);
    mbar_init(xt_free, 1);
    mbar_init(tp_full, 1);
    mbar_init(tp_empty, 4);
    mbar_init(tdone, 1);
    mbar_init(&st_free[0], 1);
    mbar_init(&st_free[1], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ operand producer
    if (lane == 0) {
      prefetch_tmap(&maps.a);
      prefetch_tmap(&maps.b);
      pdl_wait();  // the quantized activations come from the previous kernel
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const int mt = u % p.m_tiles, sg = u / p.m_tiles;
        const int nt0 = sg * p.n_tiles / p.S, nt1 = (sg + 1) * p.n_tiles / p.S;
        for (int nt = nt0; nt < nt1 && ok; ++nt) {
          for (int st = 0; st < units; ++st, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, wc)) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + s * STAGE_BYTES;
            if (st < p.n_lr) {
              const int w = p.lr_w[st], mi = lr_map_index(w);
              mbar_arrive_expect_tx(&full[s], (uint32_t)(BM + BN) * 2 * w);
              tma_load_2d(&maps.t[mi], &full[s], dst, p.lr_off[st], mt * BM);
              tma_load_2d(&maps.l2[mi], &full[s], dst + A_BYTES, p.lr_off[st], nt * BN);
            } else {
              const int ks = st - p.n_lr;
              mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
              tma_load_2d(&maps.a, &full[s], dst, ks * 128, mt * BM);
              tma_load_2d(&maps.b, &full[s], dst + A_BYTES, ks * 128, nt * BN);
            }
          }
        }
      }
      if (!ok) {
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, drain_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ main MMA issuer
    if (lane == 0) {
      int it = 0, local = 0, kst = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const int sg = u / p.m_tiles;
        const int nt0 = sg * p.n_tiles / p.S, nt1 = (sg + 1) * p.n_tiles / p.S;
        for (int nt = nt0; nt < nt1 && ok; ++nt, ++local) {
          const int b = local & 1;
          if (!mbar_wait(&acc_empty[b], ((local >> 1) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(b * BN);
          uint32_t accum = 0;
          for (int st = 0; st < units; ++st, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(&full[s], (it / STAGES) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b_addr = a_addr + A_BYTES;
            if (st < p.n_lr) {
              const int w = p.lr_w[st];
              const uint32_t layout = w == 64 ? LAYOUT_SW128 : (w == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
              const uint32_t sbo = 8u * 2u * (uint32_t)w;
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
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, drain_limit);
    }
  } else if (warp == SF_WARP) {
    // ------------------------------------------------------------ scale-factor producer
    // One slot per K stage: [SFA 4 atoms | SFB 8 atoms], two bulk copies.
    if (lane == 0) {
      pdl_wait();  // the activation scales come from the previous kernel
      int pit = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const int mt = u % p.m_tiles, sg = u / p.m_tiles;
        const int nt0 = sg * p.n_tiles / p.S, nt1 = (sg + 1) * p.n_tiles / p.S;
        for (int nt = nt0; nt < nt1 && ok; ++nt) {
          for (int ks = 0; ks < p.k_stages; ++ks, ++pit) {
            const int slot = pit % SF_SLOTS;
            if (!mbar_wait(&sfs_empty[slot], ((pit / SF_SLOTS) & 1) ^ 1, wc)) {
              ok = false;
              break;
            }
            uint8_t* dst = sfring + slot * SF_SLOT_BYTES;
            mbar_arrive_expect_tx(&sfs_full[slot], SFA_BYTES + SFB_BYTES);
            const size_t oa = ((size_t)mt * p.katoms + 4 * ks) * kSfAtomBytes;
            const size_t ob = ((size_t)nt * p.katoms + 4 * ks) * 2 * kSfAtomBytes;
            if (SVDQ_INB(p.status, oa, SFA_BYTES, p.sfa_bytes)) bulk_load(dst, p.sfa + oa, SFA_BYTES, &sfs_full[slot]);
            if (SVDQ_INB(p.status, ob, SFB_BYTES, p.sfb_bytes))
              bulk_load(dst + SFA_BYTES, p.sfb + ob, SFB_BYTES, &sfs_full[slot]);
          }
        }
      }
      if (!ok) {
        for (int j = (pit > SF_SLOTS ? pit - SF_SLOTS : 0); j < pit; ++j)
          mbar_wait_drain(&sfs_full[j % SF_SLOTS], (j / SF_SLOTS) & 1, drain_limit);
      }
    }
  } else if (warp >= 10 && warp <= 13) {
    // ------------------------------------------------------------ scale-factor movers
    // Warp q owns tensor-memory lanes 32q..32q+31; lane l writes, for every
    // 128-row atom of the stage, the atom's 16-byte row l into 4 consecutive
    // columns (the replicated layout the block-scaled MMA reads).
    const int q = warp & 3;
    int kst = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
      const int sg = u / p.m_tiles;
      const int nt0 = sg * p.n_tiles / p.S, nt1 = (sg + 1) * p.n_tiles / p.S;
      for (int nt = nt0; nt < nt1 && ok; ++nt) {
        for (int ks = 0; ks < p.k_stages; ++ks, ++kst) {
          const int slot = kst % SF_SLOTS, sb = kst & 1;
          ok = warp_wait(&sfs_full[slot], (kst / SF_SLOTS) & 1, wc);
          if (!ok) break;
          const uint8_t* sfa_s = sfring + slot * SF_SLOT_BYTES;
          const uint8_t* sfb_s = sfa_s + SFA_BYTES;
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
            mbar_arrive(&sfs_empty[slot]);  // after the stores that consumed the loaded registers
          }
        }
      }
    }
  } else if (warp == T_WARP) {
    // ------------------------------------------------------------ t' MMAs and the staged stores
    // Per tile: the rank rows of L1'^T for the tile's 192 columns (three 64-column
    // boxes, 128-byte swizzle) into the slot; once the epilogue has staged the
    // tile (x^', codes, scales), t' += bf16(x^'_tile) . L1'[tile] (M = 128,
    // N = rank, K = 192) -- the x^' tile and the slot are free when those MMAs
    // complete -- then the codes (TMA tensor store, rows past M clipped) and the
    // three scale atoms (one bulk copy: contiguous in the atom layout) leave from
    // the tile's staging buffer.  The staging is double-buffered: a buffer is
    // released when the next tile's stores are issued and its own have been read.
    if (lane == 0) {
      const bool lr = p.rank_dn > 0;
      if (lr) prefetch_tmap(&maps.l1dn);
      prefetch_tmap(&maps.codes_dn);
      bool ok = true;
      int tt = 0, ut = 0;
      const uint32_t idesc_t = lr ? idesc_bf16_f32(BM, p.rank_dn) : 0u;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++ut) {
        const int mt = u % p.m_tiles, sg = u / p.m_tiles;
        const int nt0 = sg * p.n_tiles / p.S, nt1 = (sg + 1) * p.n_tiles / p.S;
        for (int nt = nt0; nt < nt1 && ok; ++nt, ++tt) {
          const int sb = tt & 1;
          if (lr) {
            if (!mbar_wait(xt_free, (tt & 1) ^ 1, wc)) {  // the previous tile's t' MMAs completed
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(l1_full, 3u * (uint32_t)p.rank_dn * 128u);
            for (int hb = 0; hb < 3; ++hb)
              tma_load_2d(&maps.l1dn, l1_full, l1s + hb * L1_MAX_ROWS * 128, nt * BN + 64 * hb, 0);
          }
          // the epilogue staged the tile (one barrier per buffer: the epilogue cannot
          // complete one twice before this wait, since it reuses the buffer only after
          // the release below)
          if (!mbar_wait(&xt_full[sb], (tt >> 1) & 1, wc)) {
            ok = false;
            break;
          }
          if (lr) {
            if (!mbar_wait(l1_full, tt & 1, wc) || (nt == nt0 && !mbar_wait(tp_empty, (ut & 1) ^ 1, wc))) {
              ok = false;  // (the unit's previous t' was read out before its first MMA)
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(xt), b0 = smem_u32(l1s);
            for (int kk = 0; kk < 12; ++kk) {
              const uint32_t hb = kk >> 2, koff = (kk & 3) * 32;
              mma_bf16(tmem + TP_COL, make_sdesc(a0 + hb * (BM * 128) + koff, 16, 1024, LAYOUT_SW128),
                       make_sdesc(b0 + hb * (L1_MAX_ROWS * 128) + koff, 16, 1024, LAYOUT_SW128), idesc_t,
                       (nt > nt0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(xt_free);
            if (nt + 1 == nt1) umma_commit(tp_full);
          }
          tma_store_2d(&maps.codes_dn, cst + sb * CST_BYTES, nt * (BN / 2), mt * BM);
          const size_t so = ((size_t)mt * p.katoms_dn + 3 * nt) * kSfAtomBytes;
          if (SVDQ_INB(p.status, so, SST_BYTES, p.scales_dn_bytes))
            bulk_store(p.scales_dn + so, sst + sb * SST_BYTES, SST_BYTES);
          bulk_commit();
          if (tt > 0) {  // the previous tile's stores have read their buffer
            bulk_wait_read<1>();
            mbar_arrive(&st_free[sb ^ 1]);
          }
        }
      }
      bulk_wait<0>();  // the stores are complete
      if (lr) {
        umma_commit(tdone);
        mbar_wait_drain(tdone, 0, drain_limit);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9)
    const int e = warp - 2;         // 0..7
    pdl_wait();  // g_x and the down layer's workspace belong to the stream's order
    const int q = warp & 3;         // tensor-memory lane quarter
    const int half = e >> 2;        // columns 96*half .. 96*half + 95 of the tile
    const float out_scale = p.gx_dev != nullptr ? *p.gx_dev * p.g_w : p.out_scale;
    const int row = 32 * q + lane;  // row of the 128-row tile
    int local = 0, tt = 0, ut = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++ut) {
      const int mt = u % p.m_tiles, sg = u / p.m_tiles;
      const int nt0 = sg * p.n_tiles / p.S, nt1 = (sg + 1) * p.n_tiles / p.S;
      const int64_t m = (int64_t)mt * BM + row;
      const bool live = m < p.M;
      for (int nt = nt0; nt < nt1 && ok; ++nt, ++local, ++tt) {
        const int b = local & 1, sb = tt & 1;
        if (!warp_wait(&acc_full[b], (local >> 1) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint8_t* cs = cst + sb * CST_BYTES;
        uint8_t* ss = sst + sb * SST_BYTES;
        const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN) + 96 * half;
        uint64_t swords = 0;  // the six block scales' of this warp's columns, one byte each
#pragma unroll 1
        for (int blk = 0; blk < 6; ++blk) {
          const int n = nt * BN + 96 * half + 16 * blk;  // first column (= the down layer's K index)
          uint32_t r[16];
          tmem_ld_32x32b_x16(tbase + 16 * blk, r);
          float bb[16], il[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 v = __ldg((const float4*)(p.bias + n) + j);
            const float4 w = __ldg((const float4*)(p.inv_lambda_dn + n) + j);
            bb[4 * j] = v.x; bb[4 * j + 1] = v.y; bb[4 * j + 2] = v.z; bb[4 * j + 3] = v.w;
            il[4 * j] = w.x; il[4 * j + 1] = w.y; il[4 * j + 2] = w.z; il[4 * j + 3] = w.w;
          }
          tmem_ld_wait();
          if (blk == 5) {  // this warp's 96 accumulator columns are in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
          }
          float2 v[8];
          uint32_t hbits[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // the up layer's bf16 output h, then x' = bf16(GELU(h)) (the down layer's input)
            const float2 y2 = __ffma2_rn(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])),
                                         make_float2(out_scale, out_scale), make_float2(bb[2 * j], bb[2 * j + 1]));
            const __nv_bfloat162 gh = __float22bfloat162_rn(gelu_erf2(__bfloat1622float2(__float22bfloat162_rn(y2))));
            hbits[j] = *(const uint32_t*)&gh;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            v[j] = __fmul2_rn(make_float2(__uint_as_float(hbits[j] << 16), __uint_as_float(hbits[j] & 0xFFFF0000u)),
                              make_float2(il[2 * j], il[2 * j + 1]));
          if (p.H != nullptr && live && SVDQ_INB(p.status, ((size_t)m * p.N + n) * 2, 32, p.H_bytes)) {
            // parity export of the down layer's input
            *(uint4*)(p.H + (size_t)m * p.N + n) = make_uint4(hbits[0], hbits[1], hbits[2], hbits[3]);
            *(uint4*)(p.H + (size_t)m * p.N + n + 8) = make_uint4(hbits[4], hbits[5], hbits[6], hbits[7]);
          }
          float mx[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) mx[j] = fmaxf(fabsf(v[j].x), fabsf(v[j].y));
#pragma unroll
          for (int j = 0; j < 4; ++j) mx[j] = fmaxf(mx[j], mx[j + 4]);
          const float amax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
          const uint32_t sc = cvt_e4m3(__fdiv_rn(amax, p.den_dn));
          // 1 / (e4m3(sc) g') = (1 / e4m3(sc)) (1 / g'), exact: g' is a power of two
          const float inv = sc != 0 ? __frcp_rn(e4m3_value(sc)) * p.inv_g_dn : 0.f;
          const float2 inv2 = make_float2(inv, inv);
          float2 qv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) qv[j] = __fmul2_rn(v[j], inv2);
          uint32_t c0 = cvt_e2m1x8(qv[0], qv[1], qv[2], qv[3]), c1 = cvt_e2m1x8(qv[4], qv[5], qv[6], qv[7]);
          if (sc == 0) c0 = c1 = 0u;  // a zero block scale: all codes +0
          if (blk == 0) {
            // the staging buffer is free once the stores of two tiles back have read it,
            // the x^' tile once the previous tile's t' MMAs completed
            if (!warp_wait(&st_free[sb], ((tt >> 1) & 1) ^ 1, wc) ||
                (p.rank_dn > 0 && !warp_wait(xt_free, (tt & 1) ^ 1, wc))) {
              ok = false;
              break;
            }
          }
          *(uint2*)(cs + row * (BN / 2) + 48 * half + 8 * blk) = make_uint2(c0, c1);
          swords |= (uint64_t)sc << (8 * blk);
          if (p.rank_dn > 0) {  // bf16(x^') into the swizzled x^' tile
            uint32_t xb[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const __nv_bfloat162 hx = __float22bfloat162_rn(v[j]);
              xb[j] = *(const uint32_t*)&hx;
            }
            const int col = 96 * half + 16 * blk;          // tile column of the block
            const int hb = col >> 6, ch = (col & 63) >> 3;  // 64-column block, 16-byte chunk in the row
            uint8_t* rowp = xt + hb * (BM * 128) + row * 128;
            *(uint4*)(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(xb[0], xb[1], xb[2], xb[3]);
            *(uint4*)(rowp + (((ch + 1) ^ (row & 7)) << 4)) = make_uint4(xb[4], xb[5], xb[6], xb[7]);
          }
        }
        if (!ok) break;
        {  // the six block scales' into the staged atoms (tile-local blocks 6*half .. 6*half + 5)
          const int lb0 = 6 * half;
          const size_t o0 = sf_offset(row, lb0, 3, kSfAtomRows);
          const size_t o1 = sf_offset(row, lb0 + (half == 0 ? 4 : 2), 3, kSfAtomRows);
          if (half == 0) {  // a whole atom word, then the first half of the next
            *(uint32_t*)(ss + o0) = (uint32_t)swords;
            *(uint16_t*)(ss + o1) = (uint16_t)(swords >> 32);
          } else {  // the second half of a word, then a whole word
            *(uint16_t*)(ss + o0) = (uint16_t)swords;
            *(uint32_t*)(ss + o1) = (uint32_t)(swords >> 16);
          }
        }
        fence_proxy_async_smem();  // x^' tile -> tensor core, staging -> bulk copies
        __syncwarp();
        if (lane == 0) mbar_arrive(&xt_full[sb]);
      }
      // ------------------------------------------------------------ the unit's t' partial
      if (ok && p.rank_dn > 0 && half == 0) {
        if (!warp_wait(tp_full, ut & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r0[16], r1[16];
        const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + TP_COL;
        tmem_ld_32x32b_x16(ta, r0);
        if (p.rank_dn > 16) tmem_ld_32x32b_x16(ta + 16, r1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tp_empty);
        float acc[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          acc[j] = __uint_as_float(r0[j]);
          acc[16 + j] = p.rank_dn > 16 ? __uint_as_float(r1[j]) : 0.f;
        }
        const int R = p.rank_dn;
        if (live && p.S > 1) {
          float* dst = p.tpart + ((size_t)sg * p.M + m) * R;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (j < R && SVDQ_INB(p.status, (((size_t)sg * p.M + m) * R + j) * 4, 16, p.tpart_bytes))
              *(float4*)(dst + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        }
        if (p.S == 1) {  // one group covers every column: the sum is complete
          if (live) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              if (j < R && SVDQ_INB(p.status, ((size_t)m * R + j) * 2, 8, p.t_dn_bytes)) {
                const __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j], acc[j + 1]);
                const __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
                *(uint2*)(p.t_dn + (size_t)m * R + j) = make_uint2(*(const uint32_t*)&h0, *(const uint32_t*)&h1);
              }
            }
          }
          continue;
        }
        __threadfence();
        __syncwarp();
        // the last of the S units to finish these 32 rows adds the partials in group order
        int* cnt = p.counters + 4 * mt + q;
        if (lane == 0)
          ticket[q] = SVDQ_INB(p.status, (size_t)(4 * mt + q) * 4, 4, p.cnt_bytes) ? atomicAdd(cnt, 1) : -1;
        __syncwarp();
        if (ticket[q] == p.S - 1) {
          __threadfence();
          if (live) {
            // the groups' partials in group order; a batch of groups' loads is issued together
            constexpr int SB = 4;
#pragma unroll 1
            for (int j = 0; j < R; j += 4) {
              float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
              for (int g0 = 0; g0 < p.S; g0 += SB) {
                float4 v[SB];
#pragma unroll
                for (int i = 0; i < SB; ++i) {
                  const size_t e = ((size_t)(g0 + i) * p.M + m) * R + j;
                  v[i] = (g0 + i < p.S && SVDQ_INB(p.status, e * 4, 16, p.tpart_bytes)) ? __ldcg((const float4*)(p.tpart + e))
                                                                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int i = 0; i < SB; ++i) {
                  if (g0 + i >= p.S) break;
                  if (g0 + i == 0) {
                    sum = v[0];
                  } else {
                    sum.x += v[i].x;
                    sum.y += v[i].y;
                    sum.z += v[i].z;
                    sum.w += v[i].w;
                  }
                }
              }
              const __nv_bfloat162 h0 = __floats2bfloat162_rn(sum.x, sum.y);
              const __nv_bfloat162 h1 = __floats2bfloat162_rn(sum.z, sum.w);
              if (SVDQ_INB(p.status, ((size_t)m * R + j) * 2, 8, p.t_dn_bytes))
                *(uint2*)(p.t_dn + (size_t)m * R + j) = make_uint2(*(const uint32_t*)&h0, *(const uint32_t*)&h1);
            }
          }
          if (lane == 0) *cnt = 0;  // every unit has arrived: ready for the next call
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

int fused_mlp_supported(const svdq_layer* up, const svdq_layer* dn) {
  if (!up || !dn) return SVDQ_ERR_INVALID_ARG;
  if (up->fmt != SVDQ_NVFP4_G16 || dn->fmt != SVDQ_NVFP4_G16) return SVDQ_ERR_INVALID_ARG;
  if (up->N != dn->K || up->device != dn->device) return SVDQ_ERR_INVALID_ARG;
  if (dn->dyn_gx || dn->rank > 32 || up->N % kNvfp4BN != 0) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

int launch_gemm_gelu_quant(const svdq_layer* L, const svdq_layer* D, int64_t M, uint8_t* ws, const Workspace& w,
                           uint8_t* wsd, const Workspace& wd, void* H, cudaStream_t stream) {
  int st = fused_mlp_supported(L, D);
  if (st != SVDQ_OK) return st;
  const int K = (int)L->K, N = (int)L->N, r = L->rank;
  FusedMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.codes, (uint64_t)K / 2, (uint64_t)M,
                      (uint64_t)K / 2, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  maps.b = L->map_w;
  FParams p{};
  const LowRankChunks ch = lowrank_chunks(r);
  p.n_lr = ch.n;
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
  st = encode_tmap_2d(&maps.codes_dn, CU_TENSOR_MAP_DATA_TYPE_UINT8, wsd + wd.codes, (uint64_t)N / 2, (uint64_t)M,
                      (uint64_t)N / 2, BN / 2, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != SVDQ_OK) return st;
  const int rd = D->rank;
  if (rd > 0) {  // L1'^T [rd, N] bf16, 64 columns per box
    st = encode_tmap_2d(&maps.l1dn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D->L1t, (uint64_t)D->K, (uint64_t)rd,
                        (uint64_t)D->K * 2, 64, (uint32_t)rd, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SVDQ_OK) return st;
  }
  p.M = (int)M;
  p.N = N;
  p.K = K;
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = N / BN;
  p.k_stages = K / kKStage;
  p.katoms = K / 64;
  p.sfa = ws + w.scales;
  p.sfb = L->wscales;
  p.bias = L->bias;
  p.out_scale = L->g_x * L->g_w;
  p.gx_dev = L->dyn_gx ? (const float*)(ws + w.status + 4) : nullptr;
  p.g_w = L->g_w;
  p.rank_dn = rd;
  p.katoms_dn = (int)(D->K / 64);
  p.inv_lambda_dn = D->inv_lambda;
  p.den_dn = 6.0f * D->g_x;
  p.inv_g_dn = 1.0f / D->g_x;  // exact: a power of two
  p.scales_dn = wsd + wd.scales;
  p.t_dn = (uint16_t*)(wsd + wd.t);
  p.tpart = (float*)(wsd + wd.tpart);
  // one counter per 32-row group in the down workspace's first-pass slots (idle:
  // the down layer has a static activation scale); zero between calls
  if (M > kFusedMlpMaxM || 4 * (int64_t)p.m_tiles > kAmaxSlots) return SVDQ_ERR_INVALID_ARG;
  p.counters = (int*)(wsd + wd.amax);
  p.H = (uint16_t*)H;
  p.status = (int*)(ws + w.status);
  p.limit = wait_limit_cycles();
  p.sfa_bytes = w.scales_bytes;
  p.sfb_bytes = L->off.total - L->off.wscales;
  p.scales_dn_bytes = wd.scales_bytes;
  p.t_dn_bytes = wd.t_bytes;
  p.tpart_bytes = wd.tpart_bytes;
  p.cnt_bytes = 4 * (size_t)kAmaxSlots;
  p.H_bytes = (size_t)M * N * 2;

  const size_t smem = 1024 + (size_t)SMEM_BYTES + 512;
  if (cudaFuncSetAttribute(k_gemm_gelu_quant, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  const int sms = device_sm_count(L->device);
  // work units: (128-row M tile) x (one of S contiguous groups of N tiles); the
  // t' partial sums of the groups land in the down layer's split-K area
  // (wd.nslices of them)
  int S = sms / p.m_tiles;  // one wave of units
  const int max_groups = rd > 0 ? wd.nslices : p.n_tiles;
  if (S > max_groups) S = max_groups;
  if (S > p.n_tiles) S = p.n_tiles;
  if (S < 1) S = 1;
  if (rd > 0 && S > 1 && wd.tpart_bytes < (size_t)S * M * rd * 4) return SVDQ_ERR_INVALID_ARG;
  p.S = S;
  p.num_units = p.m_tiles * S;
  const int grid = p.num_units < sms ? p.num_units : sms;
  if (launch_pdl(k_gemm_gelu_quant, dim3(grid), dim3(THREADS), smem, stream, maps, p) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // namespace svdq
