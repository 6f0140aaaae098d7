// lf_fp8.cuh — e4m3 quantisation of the attention operands for the FP8 variant of stage
// (d): queries per (token, head), keys per head, power-of-two scales (the smallest 2^e with
// max|x| <= 448 * 2^e), round to nearest, ties to the even code.  [LF-yly 五] deploys the
// video model with FP8 (weights per channel, activations per token); applying e4m3 to the
// attention's QK^T operands is this library's extension of it.
#pragma once
#include "lf_common.cuh"

namespace lf {

constexpr float kE4m3Max = 448.0f;

// The smallest e with amax <= 448 * 2^e (0 for amax == 0), by exact comparisons.
__device__ __forceinline__ int pow2_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int e;
  frexpf(amax / kE4m3Max, &e);                  // amax/448 in [2^(e-1), 2^e) up to rounding
  while (amax > ldexpf(kE4m3Max, e)) ++e;
  while (amax <= ldexpf(kE4m3Max, e - 1)) --e;
  return e;
}

// Two fp32 values (|x| <= 448) to two e4m3 codes, round to nearest even: lo -> bits 0-7,
// hi -> bits 8-15.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// x [rows, H, d] bf16 -> x8 [rows, H, d] e4m3 codes.  head_scale != null: one given scale per
// head; else a scale per (row, head) computed here and written to row_scale [rows, H].
// One warp per (row, head); d / 32 channels per lane (d in {64, 128}).
__global__ void quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, long long rows, int H,
                                     int d, const float* __restrict__ head_scale,
                                     uint8_t* __restrict__ x8, float* __restrict__ row_scale) {
  const long long unit = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (unit >= rows * H) return;
  const int h = (int)(unit % H);
  const int per = d / 32;                         // 2 or 4 channels per lane
  const __nv_bfloat16* src = x + unit * d + lane * per;
  float v[4];
  if (per == 4) {                                  // one 8-byte load (rows are 16-byte aligned)
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src));
    v[0] = a.x; v[1] = a.y;
  }
  float scale;
  if (head_scale != nullptr) {
    scale = head_scale[h];
  } else {
    float a = 0.f;
    for (int i = 0; i < per; ++i) a = fmaxf(a, fabsf(v[i]));
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    scale = ldexpf(1.0f, pow2_exponent(a));
    if (lane == 0) row_scale[unit] = scale;
  }
  const float inv = 1.0f / scale;                 // exact: a power of two
  uint8_t* dst = x8 + unit * d + lane * per;
  const uint16_t c01 = cvt_e4m3x2(v[0] * inv, v[1] * inv);
  if (per == 4) {                                  // the lane's four codes in one store
    const uint16_t c23 = cvt_e4m3x2(v[2] * inv, v[3] * inv);
    *reinterpret_cast<uint32_t*>(dst) = (uint32_t)c01 | ((uint32_t)c23 << 16);
  } else {
    *reinterpret_cast<uint16_t*>(dst) = c01;
  }
}

// Per-head max |x| over rows x d, folded into amax_bits[h] (non-negative floats order like
// their bit patterns, so an integer atomicMax is exact and order-independent).
__global__ void head_amax_kernel(const __nv_bfloat16* __restrict__ x, long long rows, int H,
                                 int d, unsigned int* __restrict__ amax_bits) {
  const int h = blockIdx.y;
  float a = 0.f;
  for (long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x; r < rows;
       r += (long long)gridDim.x * blockDim.x) {
    const __nv_bfloat16* row = x + (r * H + h) * d;
    for (int c = 0; c < d; c += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + c);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&amax_bits[h], __float_as_uint(a));
}

// head_scale[h] = 2^e for the amax in amax_bits[h].
__global__ void head_scale_kernel(const unsigned int* __restrict__ amax_bits, int H,
                                  float* __restrict__ head_scale) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) head_scale[h] = ldexpf(1.0f, pow2_exponent(__uint_as_float(amax_bits[h])));
}

}  // namespace lf
