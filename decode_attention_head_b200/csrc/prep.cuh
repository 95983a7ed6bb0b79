// The step before the path, fused into its kernels: per-head RMSNorm (where the model has
// one) and rotary position embedding of the raw query / key projections ("WUSH-KV: KV
// Cache Quantization with Data-Adaptive Transforms", §4.1: keys are cached after
// head-wise normalisation and RoPE; §4.2: the key transform and the query compensation
// act on the post-RoPE vectors).  Textbook forms:
//   RMSNorm: y = x / sqrt(mean(x^2) + eps) * gain, over the 128 head dimensions;
//   RoPE (rotate-half): dimension i < 64 pairs with i + 64 and the pair turns by
//   pos * theta^(-i/64).
// The result is rounded once to fp16, as the path's inputs are; the arithmetic before
// that rounding is fp32, except the rotation angle, which is formed and reduced to
// [-pi, pi] in fp64 so that positions up to 2^31 keep it to ~1e-7 rad.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace wushkv {

struct PrepSpec {
  int enabled;          // 0: q and k arrive already normalised and rotated
  double log2_theta;    // log2 of the RoPE base
  const __half* q_gain; // per-dimension RMSNorm gain of queries, or nullptr: no query norm
  const __half* k_gain; // ... of keys
  float eps;
};

// theta^(-i/64) for pair index i (0..63).
__device__ __forceinline__ double rope_inv_freq(const PrepSpec& p, int i) {
  return exp2(-(double)i / 64.0 * p.log2_theta);
}

// cos / sin of pos * inv_freq: the product and its reduction modulo 2*pi in fp64 (2*pi
// split into two doubles), then the fp32 hardware sine and cosine on [-pi, pi].
__device__ __forceinline__ void rope_cs(double inv_freq, int pos, float& c, float& s) {
  constexpr double kTwoPiHi = 6.283185307179586;             // fp64(2*pi)
  constexpr double kTwoPiLo = 2.4492935982947064e-16;        // 2*pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double a = (double)pos * inv_freq;
  const double k = rint(a * kInvTwoPi);
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
  __sincosf((float)r, &s, &c);
}

// One warp takes one head vector held in shared memory as fp32 (x[0..127]): RMSNorm with
// `gain` (skipped when gain is nullptr), RoPE at `pos`, rounded to fp16, written back in
// place (as the fp32 value of that fp16).  Lane l holds dimensions l, l+32, l+64, l+96,
// i.e. the pairs (l, l+64) and (l+32, l+96).
__device__ __forceinline__ void prep_head_warp(float* x, const __half* gain, const PrepSpec& p, int pos, int lane) {
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = x[lane + 32 * k];
  if (gain != nullptr) {
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) ss = fmaf(v[k], v[k], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.0f / sqrtf(ss / 128.0f + p.eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = (v[k] * inv) * __half2float(gain[lane + 32 * k]);
  }
  float c0, s0, c1, s1;
  rope_cs(rope_inv_freq(p, lane), pos, c0, s0);
  rope_cs(rope_inv_freq(p, lane + 32), pos, c1, s1);
  const float o0 = v[0] * c0 - v[2] * s0, o2 = v[2] * c0 + v[0] * s0;
  const float o1 = v[1] * c1 - v[3] * s1, o3 = v[3] * c1 + v[1] * s1;
  x[lane] = __half2float(__float2half_rn(o0));
  x[lane + 32] = __half2float(__float2half_rn(o1));
  x[lane + 64] = __half2float(__float2half_rn(o2));
  x[lane + 96] = __half2float(__float2half_rn(o3));
}

}  // namespace wushkv
