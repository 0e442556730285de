// Incremental decode-cache update: append one token per sequence to its raw
// window ring and, when the token completes a 128-token block, emit that
// block's compressed entry.
//
// 'BaiduがERNIE 5.5 Flash Baseを公開' §2.1: every 128 tokens become one cache
// entry, next to a window of recent raw tokens (the newest 128, xenospectrum
// analysis, section 活性140億パラメータと長文処理を支える仕組み).  In serving
// the entries are produced one block at a time as tokens arrive: the token at
// position p lives in ring slot p mod 128, so when position p = 128 j + 127
// arrives the ring holds exactly block j, and entry j is the
// softmax(s)-weighted sum of the ring's rows (K and V with the same weights,
// fp32 softmax and accumulation, bf16 result) -- the same value hca_compress
// computes from the raw sequence.
//
// One CTA per sequence, 256 threads.  The ring write is 2 KB plus a score; a
// completing block reads the ring (256 KB) once, 8-byte coalesced loads.
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace append {

constexpr int kD = 512;
constexpr int kBlk = 128;
constexpr int kThreads = 256;

// grid.x = S
__global__ void __launch_bounds__(kThreads)
    append_kernel(const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
                  const uint16_t* __restrict__ s_new, const int* __restrict__ ctx_len,
                  uint16_t* __restrict__ wk, uint16_t* __restrict__ wv, uint16_t* __restrict__ ws,
                  uint16_t* __restrict__ ck, uint16_t* __restrict__ cv, int max_nc) {
  __shared__ float w[kBlk];
  __shared__ float red[2][4];
  const int i = blockIdx.x;
  const int tid = threadIdx.x;
  const int L = ctx_len[i];
  if (L < 1) {
    if (tid == 0) record_error(DEVERR_BAD_INPUT, 200);
    return;
  }
  const int slot = (L - 1) % kBlk;
  const size_t ring = (static_cast<size_t>(i) * kBlk + slot) * kD;
  // ring write: threads 0-63 copy the K row, 64-127 the V row (16 B each)
  if (tid < 128) {
    const uint16_t* src = (tid < 64 ? k_new : v_new) + static_cast<size_t>(i) * kD;
    uint16_t* dst = (tid < 64 ? wk : wv) + ring;
    const int c = (tid & 63) * 8;
    *reinterpret_cast<uint4*>(dst + c) = __ldg(reinterpret_cast<const uint4*>(src + c));
  } else if (tid == 128) {
    ws[static_cast<size_t>(i) * kBlk + slot] = s_new[i];
  }
  if (L % kBlk != 0) return;   // uniform: no block completes
  const int j = L / kBlk - 1;
  if (j >= max_nc) {
    if (tid == 0) record_error(DEVERR_BAD_INPUT, 201);
    return;
  }
  // Block j is ring slots 0..127, the newest (slot 127) taken from the input.
  // Weights: fp32 softmax over the block's scores.
  if (tid < kBlk) {
    const uint16_t sb = tid == kBlk - 1 ? s_new[i] : ws[static_cast<size_t>(i) * kBlk + tid];
    const float sv = __uint_as_float(static_cast<uint32_t>(sb) << 16);
    float m = sv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[0][tid >> 5] = m;
    named_bar_sync(1, kBlk);
    m = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
    const float e = expf(sv - m);
    float z = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if ((tid & 31) == 0) red[1][tid >> 5] = z;
    named_bar_sync(1, kBlk);
    z = red[1][0] + red[1][1] + red[1][2] + red[1][3];
    w[tid] = e / z;
  }
  __syncthreads();
  // Weighted sums: thread t covers 4 channels of K (t < 128) or V.
  const int which = tid >> 7;
  const int ch = (tid & 127) * 4;
  const uint16_t* base = (which ? wv : wk) + static_cast<size_t>(i) * kBlk * kD + ch;
  const uint16_t* newest = (which ? v_new : k_new) + static_cast<size_t>(i) * kD + ch;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
  for (int r = 0; r < kBlk; ++r) {
    const uint2 x = r == kBlk - 1 ? __ldg(reinterpret_cast<const uint2*>(newest))
                                  : *reinterpret_cast<const uint2*>(base + static_cast<size_t>(r) * kD);
    const float wr = w[r];
    acc[0] = fmaf(wr, bf16lo_to_f32(x.x), acc[0]);
    acc[1] = fmaf(wr, bf16hi_to_f32(x.x), acc[1]);
    acc[2] = fmaf(wr, bf16lo_to_f32(x.y), acc[2]);
    acc[3] = fmaf(wr, bf16hi_to_f32(x.y), acc[3]);
  }
  uint16_t* dst = (which ? cv : ck) + (static_cast<size_t>(i) * max_nc + j) * kD + ch;
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
}

}  // namespace append
}  // namespace hca
