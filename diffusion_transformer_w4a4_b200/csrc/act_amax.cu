// First pass of the dynamic per-tensor NVFP4 activation scale: the largest
// |x^| = |fl32(x * inv_lambda)| of the activation tensor, for layers prepared
// with g_x = 0 ("Суть метода" of "Hugging Face встроила Nunchaku в Diffusers ...",
// NVFP4 variant of the following paragraph, whose per-tensor fp32 scale this
// computes per call instead of from calibration).
//
// HBM-bound: one read of X.  A CTA owns a slab of 256 column vectors (8 bf16 =
// 16 bytes each, so a vector never straddles a row since K % 64 == 0) and a
// stride of rows; a thread keeps its vector's eight 1/lambda in registers and
// walks rows, so every warp load is 512 contiguous bytes, four rows in flight
// per thread.  Streaming (evict-first) loads measured faster overall than
// default-cached ones, although the quantizer reads X again right after.  Each CTA writes its
// maximum to one slot; the activation quantizer reduces the slots (a maximum is
// exact and order-free, so the result does not depend on scheduling).
#include <cuda_bf16.h>

#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kAmaxThreads = 256;
constexpr int kUnroll = 4;

// SMOOTH: |fl32(x * inv_lambda)|; else |x| (the INT8 tensorwise layer)
template <bool SMOOTH>
__global__ void __launch_bounds__(kAmaxThreads) k_act_amax(const uint4* __restrict__ x, const float4* __restrict__ il,
                                                         int M, int kv, float* __restrict__ slots) {
  const int c = blockIdx.y * kAmaxThreads + threadIdx.x;  // column vector
  float m = 0.f;
  if (c < kv) {
    float s[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
    if constexpr (SMOOTH) {
      const float4 a = __ldg(il + 2 * c), b = __ldg(il + 2 * c + 1);
      s[0] = a.x, s[1] = a.y, s[2] = a.z, s[3] = a.w, s[4] = b.x, s[5] = b.y, s[6] = b.z, s[7] = b.w;
    }
    auto fold = [&](const uint4 v) {
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        m = fmaxf(m, fabsf(__uint_as_float(w[h] << 16) * s[2 * h]));  // binary32 products, as the quantizer's
        m = fmaxf(m, fabsf(__uint_as_float(w[h] & 0xFFFF0000u) * s[2 * h + 1]));
      }
    };
    const int g = gridDim.x;
    int row = blockIdx.x;
    for (; row + (kUnroll - 1) * g < M; row += kUnroll * g) {  // kUnroll loads in flight per thread
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) v[u] = __ldcs(x + (size_t)(row + u * g) * kv + c);  // streamed
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) fold(v[u]);
    }
    for (; row < M; row += g) fold(__ldcs(x + (size_t)row * kv + c));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[kAmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int i = 1; i < kAmaxThreads / 32; ++i) r = fmaxf(r, red[i]);
    slots[blockIdx.y * gridDim.x + blockIdx.x] = r;
  }
}

}  // namespace

void act_amax_grid(int64_t M, int64_t K, int* gx, int* gy) {
  const int64_t kv = K / 8;
  int y = (int)((kv + kAmaxThreads - 1) / kAmaxThreads);
  if (y < 1) y = 1;
  // about eight CTAs per SM of a 148-SM part, fixed so the slot count does not depend on the device
  int64_t x = (8 * kQSmCount + y - 1) / y;
  if (x > M) x = M;
  if (x < 1) x = 1;
  while (x * y > kAmaxSlots) --x;
  *gx = (int)x;
  *gy = y;
}

int launch_act_amax_raw(const void* X, int64_t M, int64_t K, const float* inv_lambda, float* slots,
                        cudaStream_t stream) {
  int gx = 0, gy = 0;
  act_amax_grid(M, K, &gx, &gy);
  if (inv_lambda)
    k_act_amax<true><<<dim3(gx, gy), kAmaxThreads, 0, stream>>>((const uint4*)X, (const float4*)inv_lambda, (int)M,
                                                               (int)(K / 8), slots);
  else
    k_act_amax<false><<<dim3(gx, gy), kAmaxThreads, 0, stream>>>((const uint4*)X, nullptr, (int)M, (int)(K / 8),
                                                                slots);
  return cudaPeekAtLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

int launch_act_amax(const svdq_layer* L, const void* X, int64_t M, uint8_t* ws, const Workspace& w,
                    cudaStream_t stream) {
  return launch_act_amax_raw(X, M, L->K, L->inv_lambda, (float*)(ws + w.amax), stream);
}

}  // namespace svdq
