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
// (tid = 0 .. nthr-1, a multiple of 32, all of them calling; qf 16-byte aligned).  red: shared scratch of
// 2 * 8 floats.  sync() is the barrier of those threads (a named barrier in a kernel whose
// other threads do other work).  Per head, one warp reduces max |q'_d / scale_d| and the
// sum of q' (lane l holds dimensions 4l .. 4l+3; xor-shuffle tree, a fixed order).
template <int BITS, int G, typename Sync>
__device__ __forceinline__ void build_query_frags(const float (*qf)[kHeadDim], int tid, int nthr, float* red,
                                                  float scale_log2, uint8_t* out, Sync sync) {
  constexpr int NHS = GCfg<G>::NHS, NT = GCfg<G>::NT, FW = GCfg<G>::FW;
  float* amax_h = red;      // [G]
  float* sum_h = red + 8;   // [G]
  const int wl = tid & 31;
  for (int hh = tid >> 5; hh < G; hh += nthr >> 5) {
    const float4 v = *reinterpret_cast<const float4*>(&qf[hh][4 * wl]);
    const float fv[4] = {v.x, v.y, v.z, v.w};
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 4 * wl + e;  // the key-code scale depends on the dimension's low bits
      const int l2s = BITS == 2 ? 2 * (k & 3) : 4 * (k & 1);
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
  uint32_t* words = reinterpret_cast<uint32_t*>(out);
  for (int w = tid; w < FW * 32; w += nthr) {
    const int idx = w >> 5, lane = w & 31;  // word idx of lane; idx = (j * NT + nt) * 2 + r
    const int g = lane >> 2, t4 = lane & 3;
    const int r = idx & 1, nt = (idx >> 1) % NT, j = (idx >> 1) / NT;
    const int hh = 4 * (nt % NHS) + (g >> 1);
    const int limb = 2 * (nt / NHS) + (g & 1);
    uint32_t word = 0u;
    if (hh < G) {
      const float amax = amax_h[hh];
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
