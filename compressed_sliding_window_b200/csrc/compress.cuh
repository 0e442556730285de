// Block compressor: 128 raw tokens -> one cache entry.
// 'BaiduがERNIE 5.5 Flash Baseを公開' §2.1 (Latent-Gated Sparse Attention):
// every 128 tokens become one cache entry.  Entry j is the softmax(s)-weighted
// sum of the block's rows, computed separately for K and V with the same weights.
//
// The work is a pure HBM stream (each K/V byte read once, 1/128 of it
// written), so it runs on CUDA cores with 16-byte coalesced loads.  One CTA of
// 128 threads handles one (block, tensor, 128-channel quarter): 32 KB in,
// 256 B out.  That gives 8 CTAs per block, enough of them to fill all SMs at
// T = 32K (2048 CTAs).
#pragma once

#include "hca_ptx.cuh"

namespace hca {

constexpr int kD = 512;
constexpr int kBlk = 128;
constexpr int kCompressThreads = 128;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// grid.x = B * nb blocks, grid.y = 8 (tensor K/V x 4 channel quarters)
__global__ void __launch_bounds__(kCompressThreads)
    compress_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                    const uint16_t* __restrict__ s, int T, int nb, uint16_t* __restrict__ ck,
                    uint16_t* __restrict__ cv) {
  __shared__ float w[kBlk];
  __shared__ float red[2][4];
  __shared__ float part[8][kBlk + 4];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int bj = blockIdx.x;
  const int b = bj / nb;
  const int j = bj - b * nb;
  const int which = blockIdx.y >> 2;   // 0 = K, 1 = V
  const int quarter = blockIdx.y & 3;  // channels [128 * quarter, +128)
  const size_t tok0 = static_cast<size_t>(b) * T + static_cast<size_t>(j) * kBlk;

  // Within-block softmax weights of the per-token scores (fp32).
  const float sv = __uint_as_float(static_cast<uint32_t>(s[tok0 + tid]) << 16);
  float m = warp_max(sv);
  if ((tid & 31) == 0) red[0][warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  const float e = expf(sv - m);
  float z = warp_sum(e);
  if ((tid & 31) == 0) red[1][warp] = z;
  __syncthreads();
  z = red[1][0] + red[1][1] + red[1][2] + red[1][3];
  w[tid] = e / z;
  __syncthreads();

  // Weighted sum: thread (r, c) covers tokens r, r+8, ... and channels 8c..8c+7
  // of this quarter; a warp reads two 256-byte row segments per load.
  const uint16_t* src = (which ? v : k) + tok0 * kD + quarter * 128;
  const int c = tid & 15;
  const int r = tid >> 4;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  uint4 x[16];
#pragma unroll
  for (int p = 0; p < 16; ++p)
    x[p] = __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(p * 8 + r) * kD + c * 8));
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const float wi = w[p * 8 + r];
    const uint32_t u[4] = {x[p].x, x[p].y, x[p].z, x[p].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] = fmaf(wi, bf16lo_to_f32(u[q]), acc[2 * q]);
      acc[2 * q + 1] = fmaf(wi, bf16hi_to_f32(u[q]), acc[2 * q + 1]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[r][c * 8 + i] = acc[i];
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) tot += part[rr][tid];
  uint16_t* dst = (which ? cv : ck) + (static_cast<size_t>(b) * nb + j) * kD + quarter * 128;
  __nv_bfloat16 hb = __float2bfloat16_rn(tot);
  dst[tid] = *reinterpret_cast<uint16_t*>(&hb);
}

}  // namespace hca
