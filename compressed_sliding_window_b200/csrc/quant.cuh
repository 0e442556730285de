// FP8 (e4m3) storage of 512-wide cache rows: per row, scale = amax / 448 and
// code = e4m3(x / scale), round to nearest even, saturating at +-448.
//
// The pages train with FP8 mixed precision and ship FP8 weights ('Baiduが
// ERNIE 5.5 Flash Baseを公開' §3, §5); storing the decode cache the same way
// halves the bytes every decode step streams.  The row's value is
// code * scale.  Division and rounding are IEEE fp32 (no fast-math
// reciprocal), so the codes are fully determined by the bf16 inputs.
//
// One warp per row: lane l holds elements 16 l .. 16 l + 15 (32-byte loads,
// 16-byte code stores).
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace quant {

constexpr int kD = 512;
constexpr int kThreads = 256;
constexpr int kRowsPerCta = kThreads / 32;

// two fp32 values -> two e4m3 codes (lo in the low byte), RNE, saturating
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kThreads)
    quantize_e4m3_kernel(const uint16_t* __restrict__ x, long long rows, uint8_t* __restrict__ codes,
                         float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kRowsPerCta + (threadIdx.x >> 5);
  if (row >= rows) return;   // uniform per warp
  const uint4* src = reinterpret_cast<const uint4*>(x + row * kD) + 2 * lane;
  const uint4 a = __ldg(src), b = __ldg(src + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16lo_to_f32(w[i]);
    v[2 * i + 1] = bf16hi_to_f32(w[i]);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = e4m3x2(__fdiv_rn(v[4 * i], s), __fdiv_rn(v[4 * i + 1], s));
    const uint32_t hi = e4m3x2(__fdiv_rn(v[4 * i + 2], s), __fdiv_rn(v[4 * i + 3], s));
    c[i] = lo | (hi << 16);
  }
  *reinterpret_cast<uint4*>(codes + row * kD + 16 * lane) = make_uint4(c[0], c[1], c[2], c[3]);
  if (lane == 0) scale[row] = s;
}

}  // namespace quant
}  // namespace hca
