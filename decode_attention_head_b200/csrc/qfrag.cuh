// The decode query in the form the quantized-path kernel consumes ("WUSH-KV: KV Cache
// Quantization with Data-Adaptive Transforms", §4.2: the compensated query q' = T_K^{-T} q
// dotted with the dequantized keys s*c + z, so q'.k = s*(q'.c) + z*sum(q')).
//
// q'.c is taken on the integer tensor-core path (u8 codes x s8 query digits, exact int32):
// per query head, Q_d = rint(q'_d / (sigma * scale_d)) with sigma = max_d |q'_d / scale_d| /
// 2^30 (scale_d = 4^j or 16^j, the power of two that masking leaves on dimension d's key
// codes), split into four balanced base-256 digits (limbs 0..3, each in [-128, 127]).
// Those digits are laid out as the mma.sync m16n8k32 B fragments of the consumer warps:
// lane (g, t4) holds, for k-step j, n-tile nt and register r, the four bytes = limb
// 2*(nt / NHS) + (g & 1) of head 4*(nt % NHS) + (g >> 1) at the four dimensions that its
// key-code register carries.  The fragments are built once per (sequence, KV head) -- by
// the decode prologue, or by the fused append of a decode step -- and every work item of
// the unit loads them as they are.
#pragma once
#include <cstdint>
#include "internal.h"

namespace wushkv {

constexpr float kQMax = 1073741824.0f;  // |fixed-point query| <= 2^30; four signed 8-bit limbs hold +-2.1e9

template <int G>
struct GCfg {
  static constexpr int NHS = G <= 4 ? 1 : 2;  // head sets handled per lane
  static constexpr int NT = 2 * NHS;          // QK n-tiles: limbs {0,1} then {2,3} per head set
  static constexpr int FW = 4 * NT * 2;       // fragment words per lane: [k-step][n-tile][reg]
};

// Per-unit layout of the fragments in the decode workspace: FW/4 uint4 per lane stored as
// [FW/4][32 lanes] (coalesced), then the per-head constants A[8] = log2e*scale*sum(q'),
// B[8] = log2e*scale*sigma (zero for heads >= G).
constexpr size_t kQFragBytes = 32 * 32 * 4 + 16 * 4;  // room for G = 8

// The dimension (0..127) of byte `byte` of fragment register (k-step j, reg r) of lane
// quarter t4, and the log2 of the scale its key codes carry after masking.
template <int BITS>
__device__ __forceinline__ void frag_dim(int j, int r, int t4, int byte, int& dim, int& l2s) {
  if (BITS == 2) {  // key word w = dim / 16 holds 16 codes; mask plane j picks dims 4i + j
    dim = 32 * t4 + 16 * r + 4 * byte + j;
    l2s = 2 * j;
  } else {          // key word w = dim / 8 holds 8 codes; mask plane j & 1 picks dims 2i + (j & 1)
    const int wl = 2 * (j >> 1) + r;
    dim = 32 * t4 + 8 * wl + 2 * byte + (j & 1);
    l2s = 4 * (j & 1);
  }
}

// Build the unit's fragments from q' (fp32 [G][128] in shared memory) with `nthr` threads
// (tid = 0 .. nthr-1, all of them calling).  red: shared scratch of 2 * 8 * 4 floats.
// sync() is the barrier of those threads (a named barrier in a kernel whose other threads
// do other work).  The per-head sum is taken in the order (s0 + s1) + (s2 + s3), s_c the
// left-to-right sum over dimensions 32c .. 32c+31.
template <int BITS, int G, typename Sync>
__device__ __forceinline__ void build_query_frags(const float (*qf)[kHeadDim], int tid, int nthr, float* red,
                                                  float scale_log2, uint8_t* out, Sync sync) {
  constexpr int NHS = GCfg<G>::NHS, NT = GCfg<G>::NT, FW = GCfg<G>::FW;
  float* amax_q = red;           // [G][4]
  float* sum_q = red + 8 * 4;    // [G][4]
  for (int i = tid; i < G * 4; i += nthr) {
    const int hh = i >> 2, c = i & 3;
    float amax = 0.f, sum = 0.f;
    for (int k = 0; k < 32; ++k) {
      const float v = qf[hh][32 * c + k];
      const int l2s = BITS == 2 ? 2 * (k & 3) : 4 * (k & 1);
      amax = fmaxf(amax, fabsf(v) * (1.0f / float(1 << l2s)));
      sum += v;
    }
    amax_q[i] = amax;
    sum_q[i] = sum;
  }
  sync();
  uint32_t* words = reinterpret_cast<uint32_t*>(out);
  for (int w = tid; w < FW * 32; w += nthr) {
    const int idx = w >> 5, lane = w & 31;  // word idx of lane; idx = (j * NT + nt) * 2 + r
    const int g = lane >> 2, t4 = lane & 3;
    const int r = idx & 1, nt = (idx >> 1) % NT, j = (idx >> 1) / NT;
    const int hh = 4 * (nt % NHS) + (g >> 1);
    const int limb = 2 * (nt / NHS) + (g & 1);
    uint32_t word = 0u;
    if (hh < G) {
      const float amax = fmaxf(fmaxf(amax_q[4 * hh], amax_q[4 * hh + 1]), fmaxf(amax_q[4 * hh + 2], amax_q[4 * hh + 3]));
      const float sigma = amax > 0.f ? amax / kQMax : 1.0f;
      const float rs = 1.0f / sigma;
#pragma unroll
      for (int byte = 0; byte < 4; ++byte) {
        int dim, l2s;
        frag_dim<BITS>(j, r, t4, byte, dim, l2s);
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
    words[((idx >> 2) * 32 + lane) * 4 + (idx & 3)] = word;
  }
  float* hc = reinterpret_cast<float*>(out + FW * 32 * 4);
  for (int i = tid; i < 16; i += nthr) {
    const int hh = i & 7;
    float v = 0.f;
    if (hh < G) {
      if (i < 8) {
        v = scale_log2 * ((sum_q[4 * hh] + sum_q[4 * hh + 1]) + (sum_q[4 * hh + 2] + sum_q[4 * hh + 3]));
      } else {
        const float amax =
            fmaxf(fmaxf(amax_q[4 * hh], amax_q[4 * hh + 1]), fmaxf(amax_q[4 * hh + 2], amax_q[4 * hh + 3]));
        v = scale_log2 * (amax > 0.f ? amax / kQMax : 1.0f);
      }
    }
    hc[i] = v;
  }
}

}  // namespace wushkv
