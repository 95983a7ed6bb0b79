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
// key-code register carries.  With eight query heads per KV head the query takes three
// limbs instead (sigma = max / 2^22, a 23-bit fixed point): n-tiles 0 and 1 hold limbs 0
// and 1 of heads 0..3 and 4..7 as above, n-tile 2 holds limb 2 of all eight, column g
// belonging to head (g >> 1) + 4 (g & 1) -- so that the lane that holds a head's limbs 0
// and 1 in its accumulator also holds its limb 2 -- and each slice issues 24 QK MMAs
// instead of 32.  With one query head per KV head a single n-tile holds its four limbs in
// columns 0..3 (lane t4 = 0 gets limbs 0 and 1 in its accumulator, lane t4 = 1 limbs 2 and
// 3, combined by one shuffle): 8 QK MMAs per slice instead of 16.  The fragments are built once per (sequence, KV head) -- by the decode's
// query kernel, or by the fused append of a decode step -- and every work item of the unit
// loads them as they are.
#pragma once
#include <cstdint>
#include "internal.h"

namespace wushkv {

template <int G>
struct GCfg {
  static constexpr int NHS = G <= 4 ? 1 : 2;  // head sets handled per lane
  static constexpr int LIMBS = G <= 4 ? 4 : 3;  // signed 8-bit limbs of the fixed-point query
  // QK n-tiles: limbs {0,1} then {2,3} per head set; three limbs: {0,1} per head set, then
  // limb 2; one query head: its four limbs in columns 0..3 of a single n-tile
  static constexpr int NT = G == 1 ? 1 : LIMBS == 4 ? 2 * NHS : 3;
  static constexpr int FW = 4 * NT * 2;       // fragment words per lane: [k-step][n-tile][reg]
  // |fixed-point query| bound: four limbs hold +-2.1e9, three +-8.4e6
  static constexpr float QMAX = LIMBS == 4 ? 1073741824.0f : 4194304.0f;
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

// q' = T_K^{-T} q for thread j's dimension of G query heads, the sums that every path to
// the decode's query takes: t[i] = Tinv[i][j] (row i of T_K^{-1}, column j), qs the G query
// rows; one fmaf chain per block of rows -- rows [0, 64) and [64, 128) added in that order
// when nchains = 2, one chain over all 128 rows when nchains = 1.
template <int G>
__device__ __forceinline__ void qprime_chains(const float (&t)[kHeadDim], const float (*qs)[kHeadDim], int nchains,
                                              float (&acc)[G]) {
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    if (nchains == 2) {
      float p0 = 0.f, p1 = 0.f;
#pragma unroll
      for (int i = 0; i < kHeadDim / 2; ++i) p0 = fmaf(t[i], qs[hh][i], p0);
#pragma unroll
      for (int i = kHeadDim / 2; i < kHeadDim; ++i) p1 = fmaf(t[i], qs[hh][i], p1);
      acc[hh] = p0 + p1;
    } else {
      float p0 = 0.f;
#pragma unroll
      for (int i = 0; i < kHeadDim; ++i) p0 = fmaf(t[i], qs[hh][i], p0);
      acc[hh] = p0;
    }
  }
}

// Build the unit's fragments from q' (fp32 [G][128] in shared memory) with 128 threads
// (tid = 0 .. 127, all of them calling; out 16-byte aligned).  red: shared scratch of 3 * 8
// floats.  sync() is the barrier of those threads (a named barrier in a kernel whose other
// threads do other work).  Per head, one warp reduces max |q'_d / scale_d| and the sum of
// q' (lane l holds dimensions 4l .. 4l+3; xor-shuffle tree, a fixed order); then thread d
// takes dimension d of every head: its fixed-point value, its four limbs, and the byte
// each limb occupies in the fragment words (the inverse of frag_dim), which start zeroed.
template <int BITS, int G, typename Sync>
__device__ __forceinline__ void build_query_frags(const float (*qf)[kHeadDim], int tid, int nthr, float* red,
                                                  float scale_log2, uint8_t* out, Sync sync) {
  constexpr int NHS = GCfg<G>::NHS, NT = GCfg<G>::NT, FW = GCfg<G>::FW;
  float* amax_h = red;      // [G]
  float* sum_h = red + 8;   // [G]
  float* rs_h = red + 16;   // [G]: 1 / sigma
  const int wl = tid & 31;
  for (int i = tid; i < FW * 8; i += nthr) reinterpret_cast<uint4*>(out)[i] = make_uint4(0u, 0u, 0u, 0u);
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
      const float sigma = amax > 0.f ? amax * (1.0f / GCfg<G>::QMAX) : 1.0f;
      amax_h[hh] = amax;
      sum_h[hh] = sum;
      rs_h[hh] = 1.0f / sigma;
    }
  }
  sync();
  for (int dim = tid; dim < kHeadDim; dim += nthr) {
    int j, r, t4, byte;
    if (BITS == 2) {  // dim = 32*t4 + 16*r + 4*byte + j
      j = dim & 3;
      byte = (dim >> 2) & 3;
      r = (dim >> 4) & 1;
      t4 = dim >> 5;
    } else {          // dim = 32*t4 + 8*(2*(j >> 1) + r) + 2*byte + (j & 1)
      const int rem = dim & 31, w8 = rem >> 3;
      t4 = dim >> 5;
      byte = (rem >> 1) & 3;
      j = 2 * (w8 >> 1) + (rem & 1);
      r = w8 & 1;
    }
    const int l2s = BITS == 2 ? 2 * j : 4 * (j & 1);
    const float unscale = __int_as_float((127 - l2s) << 23);  // 2^-l2s, exact
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const int Q = __float2int_rn(qf[hh][dim] * (rs_h[hh] * unscale));
      // balanced base-256 digits, each in [-128, 127] (with three limbs the top one is the
      // rest, |Q2| <= 64)
      int L[4];
      L[0] = ((Q + 128) & 255) - 128;
      const int Q1 = (Q - L[0]) >> 8;
      L[1] = ((Q1 + 128) & 255) - 128;
      const int Q2 = (Q1 - L[1]) >> 8;
      L[2] = GCfg<G>::LIMBS == 4 ? ((Q2 + 128) & 255) - 128 : Q2;
      L[3] = (Q2 - L[2]) >> 8;
      const int hs = hh >> 2, hq = hh & 3;
#pragma unroll
      for (int l = 0; l < GCfg<G>::LIMBS; ++l) {
        const bool top3 = GCfg<G>::LIMBS == 3 && l == 2;  // n-tile 2: column 2 hq + hs
        const int nt = G == 1 ? 0 : top3 ? 2 : (l >> 1) * NHS + hs;
        const int g = G == 1 ? l : top3 ? 2 * hq + hs : 2 * hq + (l & 1);
        const int lane = 4 * g + t4, idx = (j * NT + nt) * 2 + r;
        out[(((idx >> 2) * 32 + lane) * 4 + (idx & 3)) * 4 + byte] = (uint8_t)(L[l] & 255);
      }
    }
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
        v = scale_log2 * (amax > 0.f ? amax * (1.0f / GCfg<G>::QMAX) : 1.0f);
      }
    }
    hc[i] = v;
  }
}

}  // namespace wushkv
