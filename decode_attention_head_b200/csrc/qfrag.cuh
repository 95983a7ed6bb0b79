// The decode query in the form the quantized-path kernel consumes ("WUSH-KV: KV Cache
// Quantization with Data-Adaptive Transforms", §4.2: the compensated query q' = T_K^{-T} q
// dotted with the dequantized keys s*c + z, so q'.k = s*(q'.c) + z*sum(q')).
//
// q'.c is taken on the integer tensor-core path (tcgen05.mma kind::i8: u8 key codes x s8
// query digits, exact int32): per query head, Q_d = rint(q'_d / (sigma * scale_d)) with
// sigma = max_d |q'_d / scale_d| / 2^30 (scale_d = 4^m or 16^m, the power of two that
// masking leaves on dimension d's key codes), split into four balanced base-256 digits
// (limbs 0..3, each in [-128, 127]).  The digits form the MMA's B operand, an
// [NQ rows][128 K-bytes] matrix (row n = 4 * head + limb, NQ = max(16, 4 * G)) stored in the
// canonical K-major, unswizzled shared-memory layout: 8-row x 16-byte core matrices, row r
// of a core matrix at +16 r, row groups 128 bytes apart, K chunks of 16 bytes NQ * 16 bytes
// apart.  K index k (byte b = k % 4 of TMEM column c = k / 4 of the key operand) carries
//   2-bit: dimension 16 (c % 8) + 4 b + c / 8 with scale 4^(c / 8)   (mask plane c / 8 of
//          packed key word c % 8);
//   4-bit: dimension 8 (c % 16) + 2 b + c / 16 with scale 16^(c / 16).
// The operand is built once per (sequence, KV head) -- by the decode prologue or by the
// fused append of a decode step -- into the workspace, and every work item of the unit
// copies it into its shared memory as it is, followed by the per-head constants
// log2e*scale*sum(q') and log2e*scale*sigma.
#pragma once
#include <cstdint>
#include "internal.h"

namespace wushkv {

constexpr float kQMax = 1073741824.0f;  // |fixed-point query| <= 2^30; four signed 8-bit limbs hold +-2.1e9

template <int G>
struct GCfg {
  static constexpr int NQ = G <= 4 ? 16 : 32;         // QK MMA N: 4 limbs per head, at least 16
  static constexpr int QBYTES = NQ * kHeadDim;        // the B operand
  static constexpr int LBO = NQ * 16;                 // bytes between 16-byte K chunks
  static constexpr int NHS = G <= 4 ? 1 : 2;          // PV n-tiles (mma.sync, 8 columns each)
};

// Per-unit bytes of the workspace's query operand: room for G = 8, then A[8], B[8] floats.
constexpr size_t kQFragBytes = 32 * kHeadDim + 16 * 4;

// Byte offset of B operand element (row n, K byte k) in the canonical layout.
template <int G>
__host__ __device__ __forceinline__ int qop_offset(int n, int k) {
  return (k >> 4) * GCfg<G>::LBO + (n >> 3) * 128 + (n & 7) * 16 + (k & 15);
}

// The dimension carried by K index k of the key operand, and the log2 of its scale.
template <int BITS>
__host__ __device__ __forceinline__ void k_dim(int k, int& dim, int& l2s) {
  const int c = k >> 2, b = k & 3;
  if (BITS == 2) {
    dim = 16 * (c & 7) + 4 * b + (c >> 3);
    l2s = 2 * (c >> 3);
  } else {
    dim = 8 * (c & 15) + 2 * b + (c >> 4);
    l2s = 4 * (c >> 4);
  }
}

// Build the unit's operand from q' (fp32 [G][128] in shared memory) with `nthr` threads
// (tid = 0 .. nthr-1, a multiple of 32, all of them calling; out 16-byte aligned).  red:
// shared scratch of 2 * 8 floats.  sync() is the barrier of those threads (a named
// barrier in a kernel whose other threads do other work).  Per head, one warp reduces
// max |q'_d / scale_d| and the sum of q' (lane l holds dimensions 4l .. 4l+3; xor-shuffle
// tree, a fixed order).
template <int BITS, int G, typename Sync>
__device__ __forceinline__ void build_query_frags(const float (*qf)[kHeadDim], int tid, int nthr, float* red,
                                                  float scale_log2, uint8_t* out, Sync sync) {
  constexpr int NQ = GCfg<G>::NQ;
  float* amax_h = red;      // [G]
  float* sum_h = red + 8;   // [G]
  const int wl = tid & 31;
  for (int hh = tid >> 5; hh < G; hh += nthr >> 5) {
    const float4 v = *reinterpret_cast<const float4*>(&qf[hh][4 * wl]);
    const float fv[4] = {v.x, v.y, v.z, v.w};
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = 4 * wl + e;  // the key-code scale depends on the dimension's low bits
      const int l2s = BITS == 2 ? 2 * (d & 3) : 4 * (d & 1);
      amax = fmaxf(amax, fabsf(fv[e]) * (1.0f / float(1 << l2s)));
    }
    float sum = (fv[0] + fv[1]) + (fv[2] + fv[3]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      sum += __shfl_xor_sync(0xffffffffu, sum, off);
    }
    if (wl == 0) {
      amax_h[hh] = amax;
      sum_h[hh] = sum;
    }
  }
  sync();
  // one 32-bit word = K bytes k0 .. k0+3 of row n (4 consecutive K bytes of one core row)
  uint32_t* words = reinterpret_cast<uint32_t*>(out);
  for (int wi = tid; wi < NQ * kHeadDim / 4; wi += nthr) {
    const int n = wi / (kHeadDim / 4), k0 = 4 * (wi % (kHeadDim / 4));
    const int hh = n >> 2, limb = n & 3;
    uint32_t word = 0u;
    if (hh < G) {
      const float amax = amax_h[hh];
      const float sigma = amax > 0.f ? amax / kQMax : 1.0f;
      const float rs = 1.0f / sigma;
#pragma unroll
      for (int byte = 0; byte < 4; ++byte) {
        int dim, l2s;
        k_dim<BITS>(k0 + byte, dim, l2s);
        const int Q = __float2int_rn(qf[hh][dim] * (rs / float(1 << l2s)));
        // balanced base-256 digits, each in [-128, 127]
        const int L0 = ((Q + 128) & 255) - 128;
        const int Q1 = (Q - L0) >> 8;
        const int L1 = ((Q1 + 128) & 255) - 128;
        const int Q2 = (Q1 - L1) >> 8;
        const int L2 = ((Q2 + 128) & 255) - 128;
        const int L3 = (Q2 - L2) >> 8;
        const int L = limb == 0 ? L0 : limb == 1 ? L1 : limb == 2 ? L2 : L3;
        word |= (uint32_t)(L & 255) << (8 * byte);
      }
    }
    words[qop_offset<G>(n, k0) >> 2] = word;
  }
  float* hc = reinterpret_cast<float*>(out + GCfg<G>::QBYTES);
  for (int i = tid; i < 16; i += nthr) {
    const int hh = i & 7;
    float v = 0.f;
    if (hh < G) {
      if (i < 8) {
        v = scale_log2 * sum_h[hh];
      } else {
        const float amax = amax_h[hh];
        v = scale_log2 * (amax > 0.f ? amax / kQMax : 1.0f);
      }
    }
    hc[i] = v;
  }
}

}  // namespace wushkv
