// Per-token percentile-clipped asymmetric affine quantizer, one row over 2 or 4 lanes
// ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", §5.3: percentile
// clipping with asymmetric affine scaling and an adaptive zero point; §1: per-token
// clipped quantizers).
//
// For the 128 fp16 values x of one token's head vector:
//   lo, hi = p_lo / p_hi percentiles, linear interpolation at rank p/100*127 between
//            sorted values, P = s[i] + f*(s[i+1] - s[i]) in fp32, each op rounded alone
//   s = fp16_rn((hi - lo) / (2^bits - 1)),  z = fp16_rn(lo)
//   code = clamp(round_half_even(fp32(x - z) / s), 0, 2^bits - 1); s == 0 -> 0
// Only the NSEL smallest and NSEL largest values are needed (NSEL <= 4 covers the
// ranks of percentiles within 4 of either end); they are selected with half2 min/max
// insertion networks (exact: the values are fp16 and fp16 comparisons are exact).
// The division is done as a multiplication by the correctly rounded reciprocal; where
// that product lies within its error bound of a rounding midpoint, the exact IEEE
// division decides, so the code always equals round(fl32(fl32(x - z) / s)).
// The RMS-scaled symmetric alternative (QuEST-style, same page §4.3 and Appendix B.3)
// replaces only (s, z): sigma = sqrt(sum x^2 / 128) in fp32 in a fixed order,
// s = fp16(fp32(2 alpha / (2^bits - 1)) * sigma), z = fp16(-alpha * sigma).
#pragma once
#include <cuda_fp16.h>
#include <cstdint>
#include "ptx.cuh"

namespace wushkv {

struct QuantSpec {
  int i_lo, i_hi;   // ranks floor(p/100 * 127)
  float f_lo, f_hi; // fractional parts, fp32
  int rms;          // 1: RMS-scaled symmetric grid instead of percentiles
  float kb, alpha;  // fp32(2*alpha/(2^b-1)), fp32(alpha)
};

// Insert x into the ascending list a[0..K-1] of the K smallest seen so far (both halves
// of the half2 independently).
template <int K>
__device__ __forceinline__ void insert_small(__half2 (&a)[K], __half2 x) {
  __half2 mx[K];
#pragma unroll
  for (int j = 0; j < K - 1; ++j) mx[j] = __hmax2(a[j], x);
  a[0] = __hmin2(a[0], x);
#pragma unroll
  for (int j = 1; j < K; ++j) a[j] = __hmin2(a[j], mx[j - 1]);
}

// Insert x into the descending list b[0..K-1] of the K largest seen so far.
template <int K>
__device__ __forceinline__ void insert_large(__half2 (&b)[K], __half2 x) {
  __half2 mn[K];
#pragma unroll
  for (int j = 0; j < K - 1; ++j) mn[j] = __hmin2(b[j], x);
  b[0] = __hmax2(b[0], x);
#pragma unroll
  for (int j = 1; j < K; ++j) b[j] = __hmax2(b[j], mn[j - 1]);
}

template <int K>
__device__ __forceinline__ void merge_small(float (&a)[K], const float (&b)[K]) {
#pragma unroll
  for (int i = 0; i < K; ++i) {
    float x = b[i];
    float mx[K];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) mx[j] = fmaxf(a[j], x);
    a[0] = fminf(a[0], x);
#pragma unroll
    for (int j = 1; j < K; ++j) a[j] = fminf(a[j], mx[j - 1]);
  }
}

template <int K>
__device__ __forceinline__ void merge_large(float (&a)[K], const float (&b)[K]) {
#pragma unroll
  for (int i = 0; i < K; ++i) {
    float x = b[i];
    float mn[K];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) mn[j] = fminf(a[j], x);
    a[0] = fmaxf(a[0], x);
#pragma unroll
    for (int j = 1; j < K; ++j) a[j] = fmaxf(a[j], mn[j - 1]);
  }
}

// P = s_i + f * (s_j - s_i), three separately rounded fp32 operations.
__device__ __forceinline__ float interp(float si, float sj, float f) {
  return __fadd_rn(si, __fmul_rn(f, __fsub_rn(sj, si)));
}

template <int BITS>
__device__ __forceinline__ uint32_t quantize_one(float v, float zf, float sf, float rcp) {
  constexpr float kLevels = float((1 << BITS) - 1);
  const float t = __fsub_rn(v, zf);
  float q = __fmul_rn(t, rcp);
  float c = rintf(q);
  const float dist = fabsf(__fsub_rn(q, c));
  // |q - fl(t/s)| <= 1.8e-7 |q|: only a midpoint inside that band can change the rounding
  if (dist > 0.5f - fmaf(2.5e-7f, fabsf(q), 1e-30f)) {
    c = rintf(__fdiv_rn(t, sf));
  }
  c = fminf(fmaxf(c, 0.0f), kLevels);
  return static_cast<uint32_t>(c);
}

// The smallest fp16 x whose code under (s, z) is at least k (1 <= k <= 2^bits - 1), so that
// code(x) = #{k : x >= X_k}.  code(x) = clamp(rint_even(fl32(fl32(x - z) / s))) is a
// non-decreasing function of x, so these thresholds give exactly the codes of the reading.
//  * In t = fl32(x - z): code >= k iff t >= T_k, with T_k = (k - 1/2) s when k is even (the
//    quotient k - 1/2 is exact and ties round to the even k) and the next fp32 value above
//    it when k is odd.  (k - 1/2) s is exact in fp32 (at most 16 significant bits).
//  * In x: fl32(x - z) >= T_k iff the exact x - z reaches the midpoint between T_k and the
//    fp32 value below it (reaching it exactly counts when T_k's last mantissa bit is even:
//    the tie rounds to T_k).  x - z is exact in double for fp16 x and z, so the nearest fp16
//    value to z + mid is checked there and moved by one fp16 step at most.
// Both facts were checked exhaustively on the CPU (every positive fp16 scale for T_k, every
// fp16 z against 400 scales and every k <= 15 for X_k).  Returns +inf when no finite x
// reaches code k.
__device__ __forceinline__ __half h_step(__half x, int d) {  // the next fp16 value up (d = 1) or down (-1)
  const int b = __half_as_ushort(x);
  int key = b >= 0x8000 ? 0xFFFF - b : b + 0x8000;  // fp16 order as an integer order (-0 just below +0)
  key = min(max(key + d, 0), 0xFFFF);
  return __ushort_as_half((unsigned short)(key >= 0x8000 ? key - 0x8000 : 0xFFFF - key));
}

__device__ __forceinline__ __half code_threshold(int k, float sf, float zf) {
  const float e = __fmul_rn((float)k - 0.5f, sf);
  const float T = (k & 1) ? __uint_as_float(__float_as_uint(e) + 1u) : e;
  const double mid = 0.5 * ((double)T + (double)__uint_as_float(__float_as_uint(T) - 1u));
  const bool incl = (__float_as_uint(T) & 1u) == 0u;
  const double zd = (double)zf;
  auto reach = [&](__half x) {
    const double y = (double)__half2float(x) - zd;
    return incl ? y >= mid : y > mid;
  };
  __half v = __double2half(zd + mid);
  if (reach(v)) {
    const __half p = h_step(v, -1);
    if (reach(p)) v = p;
  } else {
    v = h_step(v, 1);
  }
  return v;
}

// Value codes are stored in groups of 16 positions laid out for the decode's PV operand:
// each 32-bit word pairs the 16-bit chunk c (codes of 16 / BITS consecutive dimensions) of
// group positions t and t + 8 (t = 0 .. 7; position t in the low half), and the four words
// one lane of the decode needs sit together, lane after lane, so that a warp reads a group
// with one conflict-free 16-byte load per lane (two at 4 bits).  Word of (t, c):
//   2 bits:  16 * (c >> 1) + 4 * (t & 3) + 2 * (c & 1) + (t >> 2)
//   4 bits: 128 * ((c >> 1) & 1) + 16 * (c >> 2) + 4 * (t & 3) + 2 * (c & 1) + (t >> 2)
// This returns the index of the 16-bit half holding chunk c of group position r (0 .. 15).
template <int BITS>
__host__ __device__ __forceinline__ int vgroup_half(int r, int c) {
  const int t = r & 7;
  const int lane_part = 4 * (t & 3) + 2 * (c & 1) + (t >> 2);
  const int word = BITS == 2 ? 16 * (c >> 1) + lane_part : 128 * ((c >> 1) & 1) + 16 * (c >> 2) + lane_part;
  return 2 * word + (r >> 3);
}

// The quantizer with one row split over P adjacent lanes (P = 2 or 4; lanes
// P*k .. P*k+P-1 of a warp, all active together): lane `part` takes values
// [part*128/P, (part+1)*128/P), keeps its own NSEL smallest / largest, the lists are merged
// over log2(P) xor-shuffle rounds (every lane ends with the same order statistics, so
// every lane computes the same s and z), and each lane quantizes and writes its own
// slice of the packed codes (16*BITS/P bytes); part 0 writes (s, z).
// vrow < 0: codes_out is the row's record (key layout); vrow >= 0: codes_out is the base of
// the row's 16-position group and vrow its position there (value layout, vgroup_half).
template <int BITS, int NSEL, int P>
__device__ __forceinline__ void quantize_row_part(const __half* __restrict__ x, int part,
                                                  uint8_t* __restrict__ codes_out,
                                                  uint32_t* __restrict__ params_out, const QuantSpec qs,
                                                  int vrow = -1) {
  static_assert(P == 2 || P == 4, "two or four lanes per row");
  constexpr int V = 128 / P;  // values of this lane
  constexpr int H = V / 2;    // half2 of this lane
  __half2 v[H];
  const uint4* src = reinterpret_cast<const uint4*>(x + part * V);
#pragma unroll
  for (int i = 0; i < V / 8; ++i) {
    uint4 u = src[i];
    v[4 * i + 0] = u32_as_h2(u.x);
    v[4 * i + 1] = u32_as_h2(u.y);
    v[4 * i + 2] = u32_as_h2(u.z);
    v[4 * i + 3] = u32_as_h2(u.w);
  }
  const int lane = threadIdx.x & 31;
  const unsigned group = ((1u << P) - 1u) << (lane & ~(P - 1));
  __half s_h, z_h;
  if (qs.rms) {
    // sigma^2: runs of 32 consecutive squares summed left to right, then (g0+g1)+(g2+g3)
    float gsum[V / 32];
#pragma unroll
    for (int r = 0; r < V / 32; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int k = 16 * r; k < 16 * r + 16; ++k) {
        const float2 f = __half22float2(v[k]);
        acc = __fadd_rn(acc, __fmul_rn(f.x, f.x));
        acc = __fadd_rn(acc, __fmul_rn(f.y, f.y));
      }
      gsum[r] = acc;
    }
    float ss = V == 64 ? __fadd_rn(gsum[0], gsum[V / 32 - 1]) : gsum[0];  // P = 2: this lane's pair
    if (P == 4) ss = __fadd_rn(ss, __shfl_xor_sync(group, ss, 1));          // g0+g1 | g2+g3
    ss = __fadd_rn(ss, __shfl_xor_sync(group, ss, P == 4 ? 2 : 1));         // (g0+g1)+(g2+g3)
    const float sigma = __fsqrt_rn(__fdiv_rn(ss, 128.0f));
    s_h = __float2half_rn(__fmul_rn(qs.kb, sigma));
    z_h = __float2half_rn(__fmul_rn(-qs.alpha, sigma));
  } else {
  const __half2 pinf = __halves2half2(__ushort_as_half(0x7C00), __ushort_as_half(0x7C00));
  const __half2 ninf = __halves2half2(__ushort_as_half(0xFC00), __ushort_as_half(0xFC00));
  __half2 a[NSEL], b[NSEL];
#pragma unroll
  for (int j = 0; j < NSEL; ++j) {
    a[j] = pinf;
    b[j] = ninf;
  }
  // Pairs of values first: of each pair (v[2m], v[2m+1]) only the smaller can be among the
  // NSEL smallest unless its partner is too, so at most NSEL / 2 pair maxima are among them
  // (and at most NSEL / 2 pair minima among the NSEL largest).  The minima go through the
  // NSEL-list of the smallest and the maxima through an (NSEL / 2)-list, and the other way
  // round for the largest; the short lists join the long ones at the end.  Exact, with 3.5
  // instead of 5 min / max per value for NSEL = 3.
  constexpr int NB = NSEL / 2;
  __half2 a2[NB], b2[NB];
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    a2[j] = pinf;
    b2[j] = ninf;
  }
  static_assert(H % 2 == 0, "values come in pairs of half2");
#pragma unroll
  for (int i = 0; i < H; i += 2) {
    const __half2 lo = __hmin2(v[i], v[i + 1]), hi = __hmax2(v[i], v[i + 1]);
    insert_small<NSEL>(a, lo);
    insert_large<NSEL>(b, hi);
    insert_small<NB>(a2, hi);
    insert_large<NB>(b2, lo);
  }
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    insert_small<NSEL>(a, a2[j]);
    insert_large<NSEL>(b, b2[j]);
  }
  float lo_s[NSEL], lo_t[NSEL], hi_s[NSEL], hi_t[NSEL];
#pragma unroll
  for (int j = 0; j < NSEL; ++j) {
    lo_s[j] = __low2float(a[j]);
    lo_t[j] = __high2float(a[j]);
    hi_s[j] = __low2float(b[j]);
    hi_t[j] = __high2float(b[j]);
  }
  merge_small<NSEL>(lo_s, lo_t);
  merge_large<NSEL>(hi_s, hi_t);
#pragma unroll
  for (int off = 1; off < P; off <<= 1) {
#pragma unroll
    for (int j = 0; j < NSEL; ++j) {
      lo_t[j] = __shfl_xor_sync(group, lo_s[j], off);
      hi_t[j] = __shfl_xor_sync(group, hi_s[j], off);
    }
    merge_small<NSEL>(lo_s, lo_t);
    merge_large<NSEL>(hi_s, hi_t);
  }
  float slo0 = 0.f, slo1 = 0.f, shi0 = 0.f, shi1 = 0.f;
  const int jh0 = 127 - qs.i_hi;
  const int jh1 = 127 - min(qs.i_hi + 1, 127);
#pragma unroll
  for (int j = 0; j < NSEL; ++j) {
    if (j == qs.i_lo) slo0 = lo_s[j];
    if (j == qs.i_lo + 1) slo1 = lo_s[j];
    if (j == jh0) shi0 = hi_s[j];
    if (j == jh1) shi1 = hi_s[j];
  }
  const float lo = interp(slo0, slo1, qs.f_lo);
  const float hi = interp(shi0, shi1, qs.f_hi);
  const float scale32 = __fdiv_rn(__fsub_rn(hi, lo), float((1 << BITS) - 1));
  s_h = __float2half_rn(scale32);
  z_h = __float2half_rn(lo);
  }
  const float sf = __half2float(s_h);
  const float zf = __half2float(z_h);

  constexpr int NW = 4 * BITS / P;  // 32-bit words of this lane's packed codes
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0u;
  if (sf != 0.0f && BITS == 2) {
    // code = #{k : x >= X_k}, three half2 comparison masks per pair of values.  The masks are
    // nested (X_1 <= X_2 <= X_3), so the code's bit 1 is the second mask and its bit 0 is
    // (m1 & ~m2) | m3; four pairs' bits are gathered in one word (values 2k at bits 4j,
    // 4j + 1 of the low half, values 2k + 1 in the high half) and folded into 16 code bits.
    const __half2 x1 = __half2half2(code_threshold(1, sf, zf));
    const __half2 x2 = __half2half2(code_threshold(2, sf, zf));
    const __half2 x3 = __half2half2(code_threshold(3, sf, zf));
    static_assert(H % 4 == 0, "four pairs per gathered word");
#pragma unroll
    for (int k0 = 0; k0 < H; k0 += 4) {
      uint32_t u = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t m1 = __hge2_mask(v[k0 + j], x1), m2 = __hge2_mask(v[k0 + j], x2);
        const uint32_t m3 = __hge2_mask(v[k0 + j], x3);
        const uint32_t b0 = (m1 & ~m2) | m3;
        u |= ((b0 & 0x00010001u) | (m2 & 0x00020002u)) << (4 * j);
      }
      w[k0 / 8] |= ((u | (u >> 14)) & 0xFFFFu) << (16 * ((k0 / 4) & 1));
    }
  } else if (sf != 0.0f) {
    const float rcp = __frcp_rn(sf);
#pragma unroll
    for (int k = 0; k < H; ++k) {
      const float2 f = __half22float2(v[k]);
      const uint32_t c0 = quantize_one<BITS>(f.x, zf, sf, rcp);
      const uint32_t c1 = quantize_one<BITS>(f.y, zf, sf, rcp);
      if (BITS == 2) {
        w[k / 8] |= (c0 | (c1 << 2)) << (4 * (k % 8));
      } else {
        w[k / 4] |= (c0 | (c1 << 4)) << (8 * (k % 4));
      }
    }
  }
  if (vrow >= 0) {
    uint16_t* grp = reinterpret_cast<uint16_t*>(codes_out);
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const int c = 2 * (part * NW + k);
      grp[vgroup_half<BITS>(vrow, c)] = (uint16_t)(w[k] & 0xFFFFu);
      grp[vgroup_half<BITS>(vrow, c + 1)] = (uint16_t)(w[k] >> 16);
    }
    if (part == 0) *params_out = h2_as_u32(__halves2half2(s_h, z_h));
    return;
  }
  uint8_t* dst = codes_out + part * (NW * 4);
  if (NW % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NW / 4; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < NW / 2; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
  }
  if (part == 0) *params_out = h2_as_u32(__halves2half2(s_h, z_h));
}

}  // namespace wushkv
