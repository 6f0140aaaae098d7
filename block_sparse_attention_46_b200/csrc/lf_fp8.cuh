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
// d / 8 threads per (row, head), eight channels each (one 16-byte load, one 8-byte store);
// a (row, head)'s threads are consecutive lanes of one warp, which reduce its max |x|.
__global__ void quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, long long rows, int H,
                                     int d, const float* __restrict__ head_scale,
                                     uint8_t* __restrict__ x8, float* __restrict__ row_scale) {
  const int tpu = d / 8;                          // 16 or 8 threads per (row, head)
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long unit = gt / tpu;
  const int sub = (int)(gt % tpu);
  const bool valid = unit < rows * H;             // the others only join the shuffles
  const int h = (int)(unit % H);
  float v[8];
  if (valid) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + unit * d + sub * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  float scale;
  if (head_scale != nullptr) {
    scale = valid ? head_scale[h] : 1.f;
  } else {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    for (int o = tpu / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    scale = ldexpf(1.0f, pow2_exponent(a));
    if (valid && sub == 0) row_scale[unit] = scale;
  }
  if (!valid) return;
  const float inv = 1.0f / scale;                 // exact: a power of two
  uint32_t c[2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
    c[i] = (uint32_t)cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) |
           ((uint32_t)cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  *reinterpret_cast<uint2*>(x8 + unit * d + sub * 8) = make_uint2(c[0], c[1]);
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
