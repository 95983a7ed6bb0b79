// Decode attention over the packed cache ("WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms", §4.1 grouped-query attention re-evaluated at each new
// length S; §4.2 query-side compensation q' = T_K^{-T} q after RoPE, so q'.k' = q.k;
// §4.4 fp16 sink / recent windows around the quantized middle region).
//
// Two launches per call:
//  1. decode_query (one 128-thread CTA per (sequence, KV head)): q'_j = T_K^{-T} q_j for its
//     g query heads in fp32 and the query's fixed-point tensor-core fragments built from it
//     (qfrag.cuh), into the workspace.  It releases the main kernel at once (programmatic
//     dependent launch), so the main kernel's KV stream starts while it runs.  (In a fused
//     step, wushkv_step, the append kernel does this work instead; the main kernel then
//     derives the post-append state itself, streams the tiles the append cannot touch at
//     once and waits for the append before reading anything else -- see DecodeArgs::fused.)
//  2. decode_main: grid (n_split, units) in clusters of C (1 or 2) consecutive work items of
//     a unit (with many items per unit the grid's clusters interleave the units instead, in
//     linear order, so that every unit has items in every round of CTAs an SM receives: the
//     rounds dispatched last run slowest, and a unit confined to them finished last).  Work
//     item s of a unit takes the s-th share of the unit's current quantized
//     region [S_sink, S_quant) (whole 128-position stages) and of its fp16 window positions
//     (sink [0, S_sink) and recent [S_quant, S)).
//   * Stream: the quantized positions pass through shared memory in 128-position stages
//     (K codes, V codes, K and V (s, z)) via bulk copies on an mbarrier ring: one producer
//     warp, four consumer warps, 32 positions per consumer warp per stage.  The consumer
//     warps take q' as a 31-bit fixed-point integer split into four signed 8-bit limbs
//     (23-bit, three limbs, for eight query heads per KV head), laid out as the mma.sync B
//     fragments they need:
//       QK  : u8 codes x s8 query limbs on tensor cores (mma m16n8k32, exact int32),
//             logit = log2e*scale*(z*sum(q') + s*sigma*D)  (dequantization folded);
//       softmax: online, base 2, with a running max that may go stale by 2^8;
//       PV  : fp16 codes x fp16 (p*s as hi + lo) on tensor cores (mma m16n8k16,
//             fp32 accumulate), plus sum(p*z) for the zero-point term.
//   * Merge: each CTA merges its warps into (m, l, o) in its own shared memory; in a
//     cluster of two, rank 1 stores its state into rank 0's shared memory and rank 0 merges
//     the two; with one cluster per unit it writes the output, else it writes the
//     cluster's partial and the last cluster of the unit to finish (an atomic counter that
//     it then resets to zero, so the workspace needs no clearing between calls) merges them
//     and writes the output.  Nobody waits on another cluster.
//
// Code unpacking needs no shifts on the key side: masking a packed 32-bit word with
// 0x03030303 << 2j leaves, in each byte, one code times 4^j -- an exact u8 operand.
// The key-side scale 4^j is divided out of the query's integer representation.  On
// the value side, pairs of 16-bit code chunks (one per token) are shifted so that one
// code sits at bits 4..9 of each half and masked: the half is then the fp16 subnormal
// c * 2^(b-24) (b = 4, 6 or 8, the code's lowest bit), an exact operand whose
// power-of-two scale is undone once per output row.  Codes are kept high in the
// subnormal range on purpose: the tensor core aligns a product by the operand's nominal
// exponent (-14 for every subnormal), so each leading zero bit of a subnormal costs one
// bit of the product's precision inside the MMA; at bits 4..9 at most 6 of 24 are lost.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <climits>
#include <cstdint>
#include <math_constants.h>
#include "internal.h"
#include "ptx.cuh"
#include "qfrag.cuh"

namespace wushkv {
namespace {

constexpr int kThreads = 160;            // 4 consumer warps + 1 producer warp
constexpr int kConsumers = 4;
constexpr int kSlice = 32;               // positions per consumer warp per stage
constexpr int kPartStride = 132;         // floats per (item, head) partial: m, l, pad, pad, o[128]
constexpr int kTau = 8;                  // log2 headroom of the stale running max
static_assert(kTileTokens == kConsumers * kSlice, "a stage holds one slice per consumer warp");

// 2^n as an fp32 bit pattern, exact for -126 <= n <= 127.
__device__ __forceinline__ float pow2i(int n) { return __int_as_float((n + 127) << 23); }

__device__ __forceinline__ float ex2(float x) {  // 2^x (hardware approximation, 2^-inf = 0)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Row (in units of 128 elements) of query head v (0..G-1) of unit (b, h) in q and out: a
// one-token decode has its G heads side by side; chunk attention's v is token t0 + v / gq
// of the chunk (t0: the first token of the virtual unit's block), head v % gq.
__device__ __forceinline__ size_t head_row(const DecodeArgs& a, int b, int h, int t0, int v) {
  const int t = v / a.gq, hh = v - t * a.gq;
  const int ntok = a.chunk_n > 0 ? a.chunk_n : 1;
  return ((size_t)b * ntok + t0 + t) * a.Hq + (size_t)h * a.gq + hh;
}

// Virtual unit vu of a launch (a grid row): its cache unit (sequence, KV head) and the first
// chunk token of its block (chunk attention takes npass blocks of G / gq tokens per launch;
// npass = 1 and t0 = 0 otherwise).
template <int G>
__device__ __forceinline__ void virtual_unit(const DecodeArgs& a, int vu, int& unit, int& t0) {
  unit = vu / a.npass;
  t0 = a.chunk_t0 + (vu - unit * a.npass) * (G / a.gq);
}

template <int BITS>
struct Cfg {
  static constexpr int CB = 16 * BITS;
  static constexpr int NSTAGE = BITS == 2 ? 4 : 2;  // 4-bit: two 17 KB stages keep four CTAs per SM
  static constexpr int STAGE = kTileTokens * (2 * CB + 8);
};

// Value-side: dimension carried by row (g or g+8) of m-tile mt for lane group g, and the
// log2 of the scale its masked codes carry.
template <int BITS>
__device__ __forceinline__ void value_row(int mt, int g, int hi, int& dim, int& log2scale) {
  if (BITS == 2) {
    constexpr int kPos[8] = {4, 6, 4, 6, 8, 4, 6, 8};  // bit position code mt is moved to
    dim = 16 * g + 8 * hi + mt;                        // code mt of the chunk
    log2scale = kPos[mt];
  } else {
    const int ws = mt >> 2, mi = mt & 3;
    dim = 16 * g + 8 * ws + 4 * hi + mi;
    log2scale = 6;  // placed at bits 6..9
  }
}

// One value-side A register: code `mt` of both 16-bit halves of x (2-bit codes).
__device__ __forceinline__ uint32_t vcode2(uint32_t x, int mt) {
  constexpr uint32_t M45 = 0x00300030u, M67 = 0x00C000C0u, M89 = 0x03000300u;
  switch (mt) {
    case 0: return (x << 4) & M45;
    case 1: return (x << 4) & M67;
    case 2: return x & M45;
    case 3: return x & M67;
    case 4: return x & M89;
    case 5: return (x >> 6) & M45;
    case 6: return (x >> 6) & M67;
    default: return (x >> 6) & M89;
  }
}

// One value-side A register: code `mi` (0..3) of both 16-bit halves of x (4-bit codes).
__device__ __forceinline__ uint32_t vcode4(uint32_t x, int mi) {
  constexpr uint32_t M = 0x03C003C0u;
  switch (mi) {
    case 0: return (x << 6) & M;
    case 1: return (x << 2) & M;
    case 2: return (x >> 2) & M;
    default: return (x >> 6) & M;
  }
}

// The query of a plain decode call, in a kernel of its own: one 128-thread CTA per unit
// loads column j = thread of T_K^{-1} (all rows in flight at once), forms q' in the chains
// every path takes (qprime_chains, with the main kernel's cluster size) and the query
// fragments (qfrag.cuh), into the workspace.  It lets the main kernel launch at once
// (programmatic dependent launch); the main kernel's KV stream does not wait for it.
template <int BITS, int G>
__global__ void __launch_bounds__(128) decode_query_kernel(const DecodeArgs a) {
  __shared__ __align__(16) float qs[G][kHeadDim];
  __shared__ float red[24];
  griddep_launch();
  const int vu = blockIdx.x, tid = threadIdx.x;
  int unit, t0;
  virtual_unit<G>(a, vu, unit, t0);
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  const float* Tcol = a.t_k_inv + (size_t)h * kHeadDim * kHeadDim + tid;
  float t[kHeadDim];
#pragma unroll
  for (int i = 0; i < kHeadDim; ++i) t[i] = __ldg(Tcol + (size_t)i * kHeadDim);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) qs[hh][tid] = __half2float(a.q[head_row(a, b, h, t0, hh) * kHeadDim + tid]);
  if (a.prep.enabled) {  // raw queries (bulk-route step): RMSNorm + RoPE at position S - 1
    __syncthreads();
    const int qpos = max(a.state[2 * unit] - 1, 0);
    for (int hh = tid >> 5; hh < G; hh += 4) prep_head_warp(qs[hh], a.prep.q_gain, a.prep, qpos, tid & 31);
  }
  __syncthreads();
  float acc[G];
  qprime_chains<G>(t, qs, a.cluster, acc);
  __syncthreads();  // every thread has read q
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    qs[hh][tid] = acc[hh];
    a.qprime[((size_t)vu * G + hh) * kHeadDim + tid] = acc[hh];
  }
  __syncthreads();
  build_query_frags<BITS, G>(qs, tid, 128, red, a.scale_log2, a.qfrag + (size_t)vu * kQFragBytes,
                             [] { __syncthreads(); });
}

// The unit's query fragments and per-head constants (built by the cluster or the fused
// append, staged in shared memory), loaded by one lane: bq[j][nt][r], and for the lane's
// logit head t4 + 4*hs the constants log2e*scale*sum(q') (zero-point term) and
// log2e*scale*sigma.
template <int G>
__device__ __forceinline__ void load_query(const uint8_t* qfs, int lane, int t4, uint32_t (&bq)[4][GCfg<G>::NT][2],
                                           float (&Ah)[GCfg<G>::NHS], float (&Bh)[GCfg<G>::NHS]) {
  constexpr int NT = GCfg<G>::NT, NHS = GCfg<G>::NHS, FW = GCfg<G>::FW;
  const uint4* src = reinterpret_cast<const uint4*>(qfs) + lane;
#pragma unroll
  for (int m = 0; m < FW / 4; ++m) {
    const uint4 u = src[32 * m];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = 4 * m + e;
      bq[(idx >> 1) / NT][(idx >> 1) % NT][idx & 1] = w[e];
    }
  }
  const float* hc = reinterpret_cast<const float*>(qfs + FW * 32 * 4);
#pragma unroll
  for (int hs = 0; hs < NHS; ++hs) {
    Ah[hs] = hc[t4 + 4 * hs];
    Bh[hs] = hc[8 + t4 + 4 * hs];
  }
}

// ---------------------------------------------------------------------------------
constexpr int kMaxCluster = 2;   // CTAs per cluster

struct __align__(16) Merge {  // per pseudo-warp (0..3 quantized path, 4..7 window path) and head
  float m[8][8], l[8][8], bias[8][8];
  float e[8][8];      // the pseudo-warps' weights 2^(m - M) in the item's merge
  float M[8], L[8];   // the item's merged max and denominator per head
  // the cluster's merge (rank 0): the CTAs' weights 2^(m_r - M) and the merged (M, L)
  float ce[kMaxCluster][8];
  float cM[8], cL[8];
  int c_abort;        // some CTA of the cluster gave up on a wait
};
static_assert(sizeof(Merge) % 16 == 0, "the regions after the Merge block stay 16-byte aligned");

// Dynamic shared memory of the main kernel, in this order: the stage ring (after the
// stream: the consumer warps' o [4][G][128], the CTA's merged state o [G][128], m [G], l [G],
// and the weights of the unit's last merge [n_split][G]), the ring's mbarriers, the Merge
// block, the window path's o [4][G][128], the query fragments, and the other rank's merged
// state o [G][128], m [G], l [G], abort word (written by that rank).
template <int BITS, int G>
struct Shared {
  static constexpr int kStages = Cfg<BITS>::NSTAGE * Cfg<BITS>::STAGE;
  static constexpr int kPv = kConsumers * G * kHeadDim * 4;
  static constexpr int kPart = ((G * kHeadDim + 2 * G + 1) * 4 + 15) / 16 * 16;  // o, m, l, abort word
  static constexpr int kWts = kMaxSplits * G * 4;
  static constexpr int kArena = kStages;
  static_assert(kPv + kPart + kWts <= kStages, "the epilogue's buffers fit the drained stage ring");
  static constexpr size_t bytes() {
    return (size_t)kArena + 2 * Cfg<BITS>::NSTAGE * 8 + sizeof(Merge) + (size_t)kPv + kQFragBytes + kPart;
  }
};

// Per-warp online-softmax state of the quantized path.
template <int NHS>
struct QState {
  float m[NHS], l[NHS], bias[NHS];
  float o[8][4];
  int kacc;
  float s_lim;
};

// One consumer warp's 32-position slice of a stage.  FULL: every position is in range.
template <int BITS, int G, bool FULL>
__device__ __forceinline__ void slice(const uint8_t* __restrict__ st, int base, int tpos, int vlo, int vhi,
                                      const uint32_t (&bq)[4][GCfg<G>::NT][2], const float (&Ah)[GCfg<G>::NHS],
                                      const float (&Bh)[GCfg<G>::NHS], const bool (&hvalid)[GCfg<G>::NHS],
                                      QState<GCfg<G>::NHS>& s, int g, int t4) {
  constexpr int NT = GCfg<G>::NT, NHS = GCfg<G>::NHS;
  constexpr int CB = 16 * BITS;
  const uint8_t* kc = st;
  const uint8_t* vc = st + kTileTokens * CB;
  const uint32_t* kpar = reinterpret_cast<const uint32_t*>(st + 2 * kTileTokens * CB);
  const uint32_t* vpar = kpar + kTileTokens;

  // ---- QK^T over two 16-position m-tiles: rows base + 16i + g (+8)
  int acc[2][NT][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[i][nt][0] = acc[i][nt][1] = acc[i][nt][2] = acc[i][nt][3] = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r0 = base + 16 * i + g, r1 = r0 + 8;
    if (BITS == 2) {
      const uint2 ka = *reinterpret_cast<const uint2*>(kc + r0 * CB + 8 * t4);
      const uint2 kb = *reinterpret_cast<const uint2*>(kc + r1 * CB + 8 * t4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t mk = 0x03030303u << (2 * j);
        const uint32_t A[4] = {ka.x & mk, kb.x & mk, ka.y & mk, kb.y & mk};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_u8s8(acc[i][nt], A, bq[j][nt]);
      }
    } else {
      const uint4 ka = *reinterpret_cast<const uint4*>(kc + r0 * CB + 16 * t4);
      const uint4 kb = *reinterpret_cast<const uint4*>(kc + r1 * CB + 16 * t4);
      const uint32_t kaw[4] = {ka.x, ka.y, ka.z, ka.w};
      const uint32_t kbw[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t mk = (j & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
        const int wa = 2 * (j >> 1);
        const uint32_t A[4] = {kaw[wa] & mk, kbw[wa] & mk, kaw[wa + 1] & mk, kbw[wa + 1] & mk};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_u8s8(acc[i][nt], A, bq[j][nt]);
      }
    }
  }

  // ---- logits (base 2) of this lane's 4 positions: rows base + 16i + g + 8u
  float2 ksz[2][2], vsz[2][2];
  bool val[2][2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = base + 16 * i + g + 8 * u;
      ksz[i][u] = __half22float2(u32_as_h2(kpar[r]));
      vsz[i][u] = __half22float2(u32_as_h2(vpar[r]));
      val[i][u] = FULL || (tpos + r >= vlo && tpos + r < vhi);
    }
  // The running max is kept stale: p = 2^(x - mref) may reach 2^kTau, and only a logit above
  // mref + kTau (a warp vote) triggers the rescale, so the common path has no reduction.
  float x[2][2][NHS], alpha[NHS];
  bool hit = false;
#pragma unroll
  for (int hs = 0; hs < NHS; ++hs) {
    float mx = -CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        // q'.c / sigma = sum_l 256^l D_l; pairs of limbs combine exactly in int32
        const int d01 = acc[i][hs][2 * u] + 256 * acc[i][hs][2 * u + 1];
        // limbs 2 and 3; with three limbs limb 2 alone, in n-tile 2 column 2 t4 + hs; with one
        // query head, the next lane's pair (t4 = 1 holds limbs 2 and 3 of the head at t4 = 0)
        int d23;
        if constexpr (G == 1)
          d23 = __shfl_xor_sync(0xffffffffu, d01, 1);
        else if constexpr (GCfg<G>::LIMBS == 4)
          d23 = acc[i][NHS + hs][2 * u] + 256 * acc[i][NHS + hs][2 * u + 1];
        else
          d23 = acc[i][NT - 1][2 * u + hs];
        const float f = fmaf(65536.0f, (float)d23, (float)d01);
        const float xv = fmaf(Bh[hs] * ksz[i][u].x, f, Ah[hs] * ksz[i][u].y);
        x[i][u][hs] = (val[i][u] && hvalid[hs]) ? xv : -CUDART_INF_F;
        mx = fmaxf(mx, x[i][u][hs]);
      }
    alpha[hs] = mx;  // lane maximum, reused below
    hit |= mx > s.m[hs] + kTau;
  }
  const bool any_hit = __any_sync(0xffffffffu, hit);
  if (any_hit) {
#pragma unroll
    for (int hs = 0; hs < NHS; ++hs) {
      float mx = alpha[hs];
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(s.m[hs], mx);
      alpha[hs] = mn > s.m[hs] ? ex2(s.m[hs] - mn) : 1.0f;
      s.m[hs] = mn;
    }
  }
  // ---- p*s enters the PV product scaled by 2^kacc: the largest weight of a slice sits below
  // 2^14 and small weights stay in fp16's normal range; kacc only decreases, and only a
  // position whose s reaches s_lim = 2^(14 - kTau - kacc) forces a (warp-wide) recomputation
  bool over = false;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int u = 0; u < 2; ++u) over |= val[i][u] && vsz[i][u].x >= s.s_lim;
  float fk = 1.0f;
  if (__any_sync(0xffffffffu, over)) {
    float smax = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u) smax = fmaxf(smax, val[i][u] ? vsz[i][u].x : 0.f);
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 4));
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 8));
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 16));
    if (smax > 0.f) {
      // p <= 2^kTau, so smax * 2^k < 2^(14 - kTau) keeps p*s*2^k below 2^14
      const int k = 13 - kTau - (((__float_as_int(smax) >> 23) & 255) - 127);
      if (k < s.kacc) {
        fk = pow2i(max(k - s.kacc, -126));
        s.kacc = k;
        s.s_lim = pow2i(14 - kTau - k);
      }
    }
  }
  if (any_hit || fk != 1.0f) {
    if (!any_hit) {
#pragma unroll
      for (int hs = 0; hs < NHS; ++hs) alpha[hs] = 1.0f;
    }
    // o columns are heads 2t4, 2t4+1 (lo parts in 4..7 when g <= 4); their alpha lives in
    // lanes 4g + (head & 3)
    float ac0 = __shfl_sync(0xffffffffu, alpha[0], 4 * g + ((2 * t4) & 3));
    float ac1 = __shfl_sync(0xffffffffu, alpha[0], 4 * g + ((2 * t4 + 1) & 3));
    if (NHS == 2) {
      const float bc0 = __shfl_sync(0xffffffffu, alpha[NHS - 1], 4 * g + ((2 * t4) & 3));
      const float bc1 = __shfl_sync(0xffffffffu, alpha[NHS - 1], 4 * g + ((2 * t4 + 1) & 3));
      if (t4 >= 2) {
        ac0 = bc0;
        ac1 = bc1;
      }
    }
    ac0 *= fk;
    ac1 *= fk;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      s.o[mt][0] *= ac0;
      s.o[mt][1] *= ac1;
      s.o[mt][2] *= ac0;
      s.o[mt][3] *= ac1;
    }
#pragma unroll
    for (int hs = 0; hs < NHS; ++hs) {
      s.l[hs] *= alpha[hs];
      s.bias[hs] *= alpha[hs];
    }
  }
  const float wscale = pow2i(s.kacc);

  // ---- PV, one 16-position k-block per m-tile pair i
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    // p*s as an fp16 pair hi + lo (hi = fp16(p*s), lo = fp16(p*s - hi)): the PV product
    // then carries ~22 bits of p*s, matching the fp32 l it is normalised by
    uint32_t pk[NHS], pkl[NHS];
#pragma unroll
    for (int hs = 0; hs < NHS; ++hs) {
      const float ms = s.m[hs] == -CUDART_INF_F ? 0.f : s.m[hs];
      const float p0 = ex2(x[i][0][hs] - ms);
      const float p1 = ex2(x[i][1][hs] - ms);
      s.l[hs] += p0 + p1;
      // masked positions may hold any bits in (s, z): never multiply them
      const float w0 = val[i][0] ? p0 * vsz[i][0].x * wscale : 0.f;
      const float w1 = val[i][1] ? p1 * vsz[i][1].x * wscale : 0.f;
      const float b0 = val[i][0] ? p0 * vsz[i][0].y : 0.f;
      const float b1 = val[i][1] ? p1 * vsz[i][1].y : 0.f;
      s.bias[hs] += b0 + b1;
      const __half2 hi2 = __floats2half2_rn(w0, w1);
      const float2 hif = __half22float2(hi2);
      pk[hs] = h2_as_u32(hi2);
      pkl[hs] = h2_as_u32(__floats2half2_rn(w0 - hif.x, w1 - hif.y));
    }
    // B operand: rows k=2t4,2t4+1 <- positions t4, t4+8; k=2t4+8,+9 <- t4+4, t4+12 (of the
    // block); column n = head n (n < 4 or g == 8); for g <= 4 columns 4..7 carry lo parts
    const int src0 = 4 * t4 + (g & 3), src1 = 4 * (t4 + 4) + (g & 3);
    uint32_t pb[2], pbl[2];
    {
      const uint32_t h0 = __shfl_sync(0xffffffffu, pk[0], src0);
      const uint32_t h1 = __shfl_sync(0xffffffffu, pk[0], src1);
      const uint32_t l0 = __shfl_sync(0xffffffffu, pkl[0], src0);
      const uint32_t l1 = __shfl_sync(0xffffffffu, pkl[0], src1);
      if (NHS == 2) {
        const uint32_t h2 = __shfl_sync(0xffffffffu, pk[NHS - 1], src0);
        const uint32_t h3 = __shfl_sync(0xffffffffu, pk[NHS - 1], src1);
        const uint32_t l2 = __shfl_sync(0xffffffffu, pkl[NHS - 1], src0);
        const uint32_t l3 = __shfl_sync(0xffffffffu, pkl[NHS - 1], src1);
        pb[0] = g < 4 ? h0 : h2;
        pb[1] = g < 4 ? h1 : h3;
        pbl[0] = g < 4 ? l0 : l2;
        pbl[1] = g < 4 ? l1 : l3;
      } else {
        pb[0] = g < 4 ? h0 : l0;
        pb[1] = g < 4 ? h1 : l1;
        pbl[0] = pbl[1] = 0u;
      }
    }
    // the V codes of k-block i are one 16-position group in the value layout (vgroup_half):
    // lane (g, t4) reads the words pairing positions (t4, t4 + 8) and (t4 + 4, t4 + 12) for
    // its chunks -- four consecutive words, one 16-byte load, the warp's loads contiguous
    const uint8_t* vgrp = vc + (size_t)(base + 16 * i) * CB;
    if (BITS == 2) {
      const uint4 vv = *reinterpret_cast<const uint4*>(vgrp + 64 * g + 16 * t4);
      const uint32_t xl1 = vv.x, xl2 = vv.y, xh1 = vv.z, xh2 = vv.w;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t A[4] = {vcode2(xl1, mt), vcode2(xh1, mt), vcode2(xl2, mt), vcode2(xh2, mt)};
        mma_f16(s.o[mt], A, pb);
        if (NHS == 2) mma_f16(s.o[mt], A, pbl);
      }
    } else {
#pragma unroll
      for (int ws = 0; ws < 2; ++ws) {
        const uint4 vv = *reinterpret_cast<const uint4*>(vgrp + 512 * ws + 64 * g + 16 * t4);
        const uint32_t xl1 = vv.x, xl2 = vv.y, xh1 = vv.z, xh2 = vv.w;
#pragma unroll
        for (int mi = 0; mi < 4; ++mi) {
          const uint32_t A[4] = {vcode4(xl1, mi), vcode4(xh1, mi), vcode4(xl2, mi), vcode4(xh2, mi)};
          mma_f16(s.o[4 * ws + mi], A, pb);
          if (NHS == 2) mma_f16(s.o[4 * ws + mi], A, pbl);
        }
      }
    }
  }
}

// fp16 window positions [wbeg, wend) of a unit, positions wbeg + warp, + 4, ...: exact
// scalar path (lane = 4 dims), written to the window pseudo-warp slots of the merge area.
// The rows of a batch of positions are loaded together (the first batch before
// the kernel waits for q'), their G x batch logits are reduced as independent
// shuffle chains, and the online softmax is updated once per batch.
template <int G>
struct WinRows {
  static constexpr int KB = G >= 8 ? 2 : 4;  // positions per batch (registers bound it at G = 8)
  uint2 k[KB], v[KB];
};

template <int G>
__device__ __forceinline__ void window_load(const DecodeArgs& a, int unit, int it0, int wend, int n_sink, int r0,
                                            int lane, WinRows<G>& w) {
#pragma unroll
  for (int u = 0; u < WinRows<G>::KB; ++u) {
    const int it = it0 + u * kConsumers;
    w.k[u] = w.v[u] = make_uint2(0u, 0u);
    if (it < wend) {
      const __half *kr, *vr;
      if (it < n_sink) {
        kr = a.k_sink + ((size_t)unit * a.sink_dim + it) * kHeadDim;
        vr = a.v_sink + ((size_t)unit * a.sink_dim + it) * kHeadDim;
      } else {
        const int p = r0 + (it - n_sink);
        kr = a.k_ring + ((size_t)unit * a.R + p % a.R) * kHeadDim;
        vr = a.v_ring + ((size_t)unit * a.R + p % a.R) * kHeadDim;
      }
      w.k[u] = *reinterpret_cast<const uint2*>(kr + 4 * lane);
      w.v[u] = *reinterpret_cast<const uint2*>(vr + 4 * lane);
    }
  }
}

// qlim: chunk attention's causal limit -- head v sees positions <= qlim + v / gq (a
// one-token decode passes INT_MAX: every cached position is visible).
template <int G>
__device__ void window_share(const DecodeArgs& a, int unit, int wbeg, int wend, int n_sink, int r0, int warp,
                             int lane, WinRows<G>& w, Merge* mg, float* wpv, int qlim, const float* qsrc) {
  constexpr int KB = WinRows<G>::KB;
  float qv[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float4 t = *reinterpret_cast<const float4*>(qsrc + hh * kHeadDim + 4 * lane);
    qv[hh][0] = t.x * a.scale_log2;
    qv[hh][1] = t.y * a.scale_log2;
    qv[hh][2] = t.z * a.scale_log2;
    qv[hh][3] = t.w * a.scale_log2;
  }
  float m[G], l[G], o[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m[hh] = -CUDART_INF_F;
    l[hh] = 0.f;
    o[hh][0] = o[hh][1] = o[hh][2] = o[hh][3] = 0.f;
  }
  for (int it0 = wbeg + warp; it0 < wend; it0 += KB * kConsumers) {
    if (it0 != wbeg + warp) window_load<G>(a, unit, it0, wend, n_sink, r0, lane, w);
    float x[KB][G];
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const float2 k01 = __half22float2(u32_as_h2(w.k[u].x)), k23 = __half22float2(u32_as_h2(w.k[u].y));
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float xx = qv[hh][0] * k01.x;
        xx = fmaf(qv[hh][1], k01.y, xx);
        xx = fmaf(qv[hh][2], k23.x, xx);
        x[u][hh] = fmaf(qv[hh][3], k23.y, xx);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < KB; ++u)
#pragma unroll
        for (int hh = 0; hh < G; ++hh) x[u][hh] += __shfl_xor_sync(0xffffffffu, x[u][hh], off);
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const int it = it0 + u * kConsumers;
      const int pos = it < n_sink ? it : r0 + (it - n_sink);
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
        if (it >= wend || pos > qlim + hh / a.gq) x[u][hh] = -CUDART_INF_F;
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float mn = m[hh];
#pragma unroll
      for (int u = 0; u < KB; ++u) mn = fmaxf(mn, x[u][hh]);
      // no visible position yet (a causally masked head): every factor below is 2^-inf = 0
      // rather than 2^(-inf - -inf) = NaN
      const float ms = mn == -CUDART_INF_F ? 0.f : mn;
      const float al = ex2(m[hh] - ms);  // 2^-inf = 0 on the first batch
      l[hh] *= al;
      o[hh][0] *= al;
      o[hh][1] *= al;
      o[hh][2] *= al;
      o[hh][3] *= al;
#pragma unroll
      for (int u = 0; u < KB; ++u) {
        const float p = ex2(x[u][hh] - ms);
        const float2 v01 = __half22float2(u32_as_h2(w.v[u].x)), v23 = __half22float2(u32_as_h2(w.v[u].y));
        l[hh] += p;
        o[hh][0] = fmaf(p, v01.x, o[hh][0]);
        o[hh][1] = fmaf(p, v01.y, o[hh][1]);
        o[hh][2] = fmaf(p, v23.x, o[hh][2]);
        o[hh][3] = fmaf(p, v23.y, o[hh][3]);
      }
      m[hh] = mn;
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    if (lane == 0) {
      mg->m[kConsumers + warp][hh] = m[hh];
      mg->l[kConsumers + warp][hh] = l[hh];
      mg->bias[kConsumers + warp][hh] = 0.f;
    }
    float* dst = wpv + ((size_t)warp * G + hh) * kHeadDim + 4 * lane;
    dst[0] = o[hh][0];
    dst[1] = o[hh][1];
    dst[2] = o[hh][2];
    dst[3] = o[hh][3];
  }
}

// Four consecutive output values (fp32, or fp16 when out_fp16) at element offset o of out.
__device__ __forceinline__ void store_out4(const DecodeArgs& a, size_t o, float4 v) {
  if (a.out_fp16) {
    __half2* oh = reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + o);
    oh[0] = __floats2half2_rn(v.x, v.y);
    oh[1] = __floats2half2_rn(v.z, v.w);
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + o) = v;
  }
}

// Merge the `count` (<= kMaxSplits) cluster partials (m, l, pad, pad, o[128] per head,
// base 2, o not yet normalised) of one virtual unit (cache unit `unit`, chunk block at t0)
// and write the normalised output rows of its G
// query heads, summing the partials in their order.  wts: shared [count][G].  The warp of
// head hh reduces the partials' (m, l) (lane i loads partials i, i + 32, ... at once); thread
// (head, quad) then sums dimensions 4*quad .. 4*quad+3 of every partial's row, row_batch
// row loads in flight at a time -- the first batch issued before the weights are known, so
// that their round trip overlaps the (m, l) one.  Every partial is finite (an empty one
// holds m = -inf, l = 0, o = 0), so no term needs skipping.
// partial rows in flight per thread (19, which brings the 37 clusters of a 74-item unit
// into two round trips, measured 2.6 us slower on the Qwen3 call)
template <int G>
__host__ __device__ constexpr int row_batch() { return 16; }
template <int G>
__device__ void merge_partials(const DecodeArgs& a, int unit, int t0, const float* src, int count, float* wts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kQuads = kHeadDim / 4;
  constexpr int kRowBatch = row_batch<G>();
  float4 ov[kRowBatch];
  auto load_rows = [&](int idx, int i0) {
    const int hh = idx / kQuads, d = 4 * (idx % kQuads);
#pragma unroll
    for (int u = 0; u < kRowBatch; ++u)
      ov[u] = i0 + u < count
                  ? __ldcg(reinterpret_cast<const float4*>(src + ((size_t)(i0 + u) * G + hh) * kPartStride + 4 + d))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  if (tid < G * kQuads) load_rows(tid, 0);
  for (int hh = warp; hh < G; hh += kThreads / 32) {
    // every (m, l) this lane needs in one round trip
    constexpr int kPer = kMaxSplits / 32;
    float mi[kPer], li[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int i = lane + 32 * k;
      mi[k] = -CUDART_INF_F;
      li[k] = 0.f;
      if (i < count) {
        const float* p = src + ((size_t)i * G + hh) * kPartStride;
        mi[k] = __ldcg(p);
        li[k] = __ldcg(p + 1);
      }
    }
    float M = mi[0];
#pragma unroll
    for (int k = 1; k < kPer; ++k) M = fmaxf(M, mi[k]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f, e[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      e[k] = (lane + 32 * k < count && M != -CUDART_INF_F) ? exp2f(mi[k] - M) : 0.f;
      L = fmaf(e[k], li[k], L);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    const float invL = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k)
      if (lane + 32 * k < count) wts[(lane + 32 * k) * G + hh] = e[k] * invL;
    if (lane == 0 && !(L > 0.f)) atomicOr(a.status, kStatusEmpty);
  }
  __syncthreads();
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  for (int idx = tid; idx < G * kQuads; idx += kThreads) {
    const int hh = idx / kQuads, d = 4 * (idx % kQuads);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < count; i0 += kRowBatch) {
      if (idx != tid || i0 != 0) load_rows(idx, i0);
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        if (i0 + u < count) {
          const float w = wts[(i0 + u) * G + hh];
          acc.x = fmaf(w, ov[u].x, acc.x);
          acc.y = fmaf(w, ov[u].y, acc.y);
          acc.z = fmaf(w, ov[u].z, acc.z);
          acc.w = fmaf(w, ov[u].w, acc.w);
        }
      }
    }
    store_out4(a, head_row(a, b, h, t0, hh) * kHeadDim + d, acc);
  }
}

// A warp-wide wait on an mbarrier phase: every lane waits (so each observes the phase), and
// the warp's verdict is uniform -- false if any lane gave up or saw the CTA's abort word.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const DecodeArgs& a,
                                          volatile int* abort) {
  const bool ok = mbar_wait_abortable(bar, parity, a.status, abort, a.wait_limit);
  return __all_sync(0xffffffffu, ok);
}

template <int BITS, int G>
__global__ void __launch_bounds__(kThreads, decode_ctas_per_sm(G)) decode_main_kernel(const DecodeArgs a) {
  using C = Cfg<BITS>;
  using SM = Shared<BITS, G>;
  constexpr int NT = GCfg<G>::NT, NHS = GCfg<G>::NHS;
  constexpr int CB = C::CB;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  float* pv = reinterpret_cast<float*>(smem);  // [4][G][128], written once the stages are drained
  float* cpo = reinterpret_cast<float*>(smem + SM::kPv);  // the CTA's merged o [G][128] (not normalised)
  float* cpm = cpo + G * kHeadDim;                        // and its m [G], l [G]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kArena);
  uint64_t* empty = full + C::NSTAGE;
  Merge* mg = reinterpret_cast<Merge*>(empty + C::NSTAGE);
  float* wpv = reinterpret_cast<float*>(mg + 1);   // window path [4][G][128]
  uint8_t* qfs = reinterpret_cast<uint8_t*>(wpv + kConsumers * G * kHeadDim);  // the unit's query fragments
  float* srecv = reinterpret_cast<float*>(qfs + kQFragBytes);  // rank 1's merged state (rank 0 only)
  float* wts = reinterpret_cast<float*>(smem + SM::kPv + SM::kPart);  // [n_split][G] (the last merge only)
  __shared__ uint32_t s_last;
  __shared__ int s_abort;  // set by a bounded wait that gave up: every role leaves its loop
  __shared__ int s_vu[4];  // vu, unit, t0, item for the epilogue (kept out of the stream's registers)
  volatile int* abort = &s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  // virtual unit (workspace index) and work item of this CTA
  int vu, item;  // (both re-read from shared memory for the epilogue)
  if (a.interleave) {
    const int lin = blockIdx.y * gridDim.x + blockIdx.x, cl = lin / a.cluster;
    vu = cl % gridDim.y;
    item = (cl / gridDim.y) * a.cluster + lin % a.cluster;
  } else {
    vu = blockIdx.y;
    item = blockIdx.x;
  }
  int unit, t0;         // its cache unit and chunk block
  virtual_unit<G>(a, vu, unit, t0);
  const int nitems = a.n_split;
  const int ncta = a.cluster;  // CTAs per cluster (consecutive items of the unit)
  int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  // fused step: the state read above is the one before the append (that kernel leaves the
  // state words to this one); the append's outcome follows from it as the append derives it
  const int sq_stable = Sq;  // quantized positions below it are not touched by the append
  int S_next = -1, Sq_next = 0;
  if (a.fused) {
    if (S >= 0 && S <= a.cap && Sq >= 0 && Sq <= S && S + a.n_new <= a.cap) {
      int lo0, nf;
      flush_bounds(Sq, S, a.s_sink, a.s_keep, a.s_flush, lo0, nf);  // the flush under the old S
      S_next = S + a.n_new;
      Sq_next = nf ? lo0 + nf : Sq;
      S = S_next;
      Sq = Sq_next;
    }  // else the append is refused (it reports why): decode the cache as it stands
  }
  if (S < 0 || S > a.cap_alloc || Sq < 0 || Sq > S) {  // never read outside the buffers
    if (tid == 0 && item == 0) atomicOr(a.status, kStatusBadState);
    S = 0;
    Sq = 0;
  }
  // chunk attention needs the chunk in the fp16 window (so the quantized positions precede
  // every chunk query); report a cache where that does not hold
  if (a.chunk_n > 0 && Sq > S - a.chunk_n && tid == 0 && item == 0) atomicOr(a.status, kStatusChunkQuantized);
  // quantized positions of this item: [lo, hi) within [qlo, qhi).  The items split the
  // region as it stands now (not the capacity), in whole 128-position stages counted from
  // the stage that holds qlo, so every item but the last streams the same number of stages.
  const int qlo = a.s_sink;
  const int qhi = Sq > a.s_sink ? Sq : a.s_sink;
  const int qbase = (qlo / kTileTokens) * kTileTokens;
  const int tiles_all = qhi > qlo ? (qhi - qbase + kTileTokens - 1) / kTileTokens : 0;
  const int per = (tiles_all + nitems - 1) / nitems * kTileTokens;
  const int ibeg = qbase + item * per, iend = ibeg + per;
  const int lo = max(ibeg, qlo), hi = min(iend, qhi);
  const int tile0 = lo < hi ? (lo / kTileTokens) * kTileTokens : 0;
  const int ntiles = lo < hi ? (hi - tile0 + kTileTokens - 1) / kTileTokens : 0;
  // fp16 window positions of the unit: sink [0, n_sink) then recent [r0, S); this item's share
  const int n_sink = min(a.s_sink, S);
  const int r0 = max(Sq, a.s_sink);
  const int n_win = n_sink + (S > r0 ? S - r0 : 0);
  const int wper = (n_win + nitems - 1) / nitems;
  const int wbeg = min(item * wper, n_win), wend = min(wbeg + wper, n_win);

  if (tid == 0) {
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    s_abort = 0;
    s_vu[0] = vu;
    s_vu[1] = unit;
    s_vu[2] = t0;
    s_vu[3] = item;
    fence_mbar_init();
  }
  __syncthreads();

  QState<NHS> qs;
  bool hvalid[NHS];
#pragma unroll
  for (int hs = 0; hs < NHS; ++hs) {
    hvalid[hs] = (G % 4 == 0) || t4 + 4 * hs < G;
    qs.m[hs] = -CUDART_INF_F;
    qs.l[hs] = 0.f;
    qs.bias[hs] = 0.f;
  }
  qs.kacc = 64;
  qs.s_lim = 0.f;  // the first position with s > 0 sets kacc

  // With clusters of two, every thread of both CTAs takes the cluster barrier once, on every
  // path: when rank 1 has stored its merged state into rank 0's shared memory.
  if (warp == kConsumers) {
    // ---------------- producer: streams the item's tiles; needs nothing from the query
    if (lane == 0 && ntiles > 0) {
      int issued = 0;
      bool waited = !a.fused;  // fused step: tiles below the old S_quant stream at once
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % C::NSTAGE;
        if (!waited && tile0 + (t + 1) * kTileTokens > sq_stable) {
          griddep_wait();
          waited = true;
        }
        if (t >= C::NSTAGE &&
            !mbar_wait_abortable(&empty[s], ((t / C::NSTAGE) - 1) & 1, a.status, abort, a.wait_limit))
          break;
        if (*abort) break;
        if (t == a.withhold_tile) continue;  // test hook: this stage is never issued
        uint8_t* st = stages + s * C::STAGE;
        const size_t rec = (size_t)unit * a.cap_alloc + tile0 + (size_t)t * kTileTokens;
        mbar_expect_tx(&full[s], C::STAGE);
        bulk_g2s(st, a.k_codes + rec * CB, kTileTokens * CB, &full[s]);
        bulk_g2s(st + kTileTokens * CB, a.v_codes + rec * CB, kTileTokens * CB, &full[s]);
        bulk_g2s(st + 2 * kTileTokens * CB, a.k_params + rec, kTileTokens * 4, &full[s]);
        bulk_g2s(st + 2 * kTileTokens * CB + kTileTokens * 4, a.v_params + rec, kTileTokens * 4, &full[s]);
        issued = t + 1;
      }
      // every issued copy has landed before the CTA may leave (issued copies always land:
      // they are plain reads of the cache)
      for (int t = max(0, issued - C::NSTAGE); t < issued; ++t)
        if (t != a.withhold_tile) mbar_wait(&full[t % C::NSTAGE], (t / C::NSTAGE) & 1, a.status);
    }
  } else {
    // ---------------- consumers
    // (a) this warp's share of the fp16 window: the first rows are loaded before the wait
    // for the query (they do not depend on it), the rest while the first tiles land
    WinRows<G> wr;
    if (a.fused) griddep_wait();  // the window holds the appended tokens
    window_load<G>(a, unit, wbeg + warp, wend, n_sink, r0, lane, wr);
    griddep_wait();  // q' and the query fragments come from the kernel before
    {  // the unit's query fragments into shared memory while the window share runs
      constexpr int n16 = GCfg<G>::FW * 8 + 4;
      const uint8_t* src = a.qfrag + (size_t)vu * kQFragBytes;
      for (int i = tid; i < n16; i += kConsumers * 32) cp_async16(qfs + 16 * i, src + 16 * i);
      cp_async_commit();
    }
    const int qlim = a.chunk_n > 0 ? S - a.chunk_n + t0 : INT_MAX;
    window_share<G>(a, unit, wbeg, wend, n_sink, r0, warp, lane, wr, mg, wpv, qlim,
                    a.qprime + (size_t)vu * G * kHeadDim);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) qs.o[mt][0] = qs.o[mt][1] = qs.o[mt][2] = qs.o[mt][3] = 0.f;
    // (b) quantized positions
    cp_async_wait_all();
    bar_sync(1, kConsumers * 32);  // every consumer thread's copies have landed
    uint32_t bq[4][NT][2];
    float Ah[NHS], Bh[NHS];
    load_query<G>(qfs, lane, t4, bq, Ah, Bh);
    const int base = kSlice * warp;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % C::NSTAGE;
      if (!warp_wait(&full[s], (t / C::NSTAGE) & 1, a, abort)) break;
      const uint8_t* st = stages + s * C::STAGE;
      const int tpos = tile0 + t * kTileTokens;
      if (tpos + base >= lo && tpos + base + kSlice <= hi)
        slice<BITS, G, true>(st, base, tpos, lo, hi, bq, Ah, Bh, hvalid, qs, g, t4);
      else if (tpos + base + kSlice > lo && tpos + base < hi)
        slice<BITS, G, false>(st, base, tpos, lo, hi, bq, Ah, Bh, hvalid, qs, g, t4);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // l and bias summed over the 8 lane groups
#pragma unroll
    for (int hs = 0; hs < NHS; ++hs) {
      float lv = qs.l[hs], bv = qs.bias[hs];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lv += __shfl_xor_sync(0xffffffffu, lv, off);
        bv += __shfl_xor_sync(0xffffffffu, bv, off);
      }
      if (g == 0 && hvalid[hs]) {
        mg->m[warp][t4 + 4 * hs] = qs.m[hs];
        mg->l[warp][t4 + 4 * hs] = lv;
        mg->bias[warp][t4 + 4 * hs] = bv;
      }
    }
    if (NHS == 1) {  // columns 4..7 (lanes t4 = 2, 3) hold the lo parts of heads 0..3
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) qs.o[mt][c] += __shfl_down_sync(0xffffffffu, qs.o[mt][c], 2);
    }
  }
  __syncthreads();  // every stage consumed and every copy landed: pv may reuse the stages
  // A CTA whose bounded wait gave up (STATUS_TIMEOUT is set) has incomplete results: it still
  // takes every step below (the cluster barrier needs it), but its unit's output and state
  // are not written, so a timeout never produces plausible-looking output.

  if (warp < kConsumers) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int hi2 = 0; hi2 < 2; ++hi2) {
        int dim, l2s;
        value_row<BITS>(mt, g, hi2, dim, l2s);
        const float unscale = pow2i(24 - l2s - qs.kacc);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int hh = 2 * t4 + c;
          if (hh < G) pv[((size_t)warp * G + hh) * kHeadDim + dim] = qs.o[mt][2 * hi2 + c] * unscale;
        }
      }
    }
  }
  __syncthreads();

  // ======================= merge the 8 pseudo-warps into the CTA's state (m, l, o): the
  // weights once per (pseudo-warp, head), then the rows.  Rank 0 of a cluster keeps its
  // state (cpo, cpm); rank 1 stores its own straight into rank 0's receive buffer.
  vu = s_vu[0];
  unit = s_vu[1];
  t0 = s_vu[2];
  item = s_vu[3];
  const int rank = ncta > 1 ? (int)cluster_rank() : 0;
  const int ncl = nitems / ncta;  // clusters of the unit
  const uint32_t peer = ncta > 1 ? cluster_map(srecv, 0) : 0u;  // rank 0's receive buffer
  if (tid < G) {
    const int hh = tid;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < 2 * kConsumers; ++w) M = fmaxf(M, mg->m[w][hh]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < 2 * kConsumers; ++w) {
      const float e = M != -CUDART_INF_F ? exp2f(mg->m[w][hh] - M) : 0.f;
      mg->e[w][hh] = e;
      L = fmaf(e, mg->l[w][hh], L);
    }
    if (rank == 0) {
      cpm[hh] = M;
      cpm[G + hh] = L;
    } else {
      st_cluster_f32(peer + 4 * (G * kHeadDim + hh), M);
      st_cluster_f32(peer + 4 * (G * kHeadDim + G + hh), L);
    }
  } else if (tid == 32 && rank != 0) {
    st_cluster_s32(peer + 4 * (G * kHeadDim + 2 * G), s_abort);
  }
  __syncthreads();
  for (int q4 = tid; q4 < G * kHeadDim / 4; q4 += kThreads) {
    const int hh = (4 * q4) / kHeadDim, d = (4 * q4) % kHeadDim;
    float O[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      O[c] = 0.f;
#pragma unroll
      for (int w = 0; w < 2 * kConsumers; ++w) {
        const float ov = w < kConsumers ? pv[((size_t)w * G + hh) * kHeadDim + d + c]
                                        : wpv[((size_t)(w - kConsumers) * G + hh) * kHeadDim + d + c];
        O[c] = fmaf(mg->e[w][hh], ov + mg->bias[w][hh], O[c]);
      }
    }
    const float4 o4 = make_float4(O[0], O[1], O[2], O[3]);
    if (rank == 0)
      *reinterpret_cast<float4*>(cpo + 4 * q4) = o4;
    else
      st_cluster_f32x4(peer + 16 * q4, o4);
  }
  // phase B: rank 0 holds both CTAs' states (rank 1 is done after it)
  __syncwarp();
  if (ncta > 1) {
    cluster_arrive();
    cluster_wait();
  } else {
    __syncthreads();
  }
  if (rank != 0) return;

  // ======================= rank 0 merges the cluster's states in rank order
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  if (tid < G) {
    const int hh = tid;
    const float m0 = cpm[hh], l0 = cpm[G + hh];
    const float m1 = ncta > 1 ? srecv[G * kHeadDim + hh] : -CUDART_INF_F;
    const float l1 = ncta > 1 ? srecv[G * kHeadDim + G + hh] : 0.f;
    const float M = fmaxf(m0, m1);
    const float e0 = M != -CUDART_INF_F ? exp2f(m0 - M) : 0.f;
    const float e1 = (M != -CUDART_INF_F && ncta > 1) ? exp2f(m1 - M) : 0.f;
    mg->ce[0][hh] = e0;
    mg->ce[1][hh] = e1;
    mg->cM[hh] = M;
    mg->cL[hh] = fmaf(e1, l1, e0 * l0);
  } else if (tid == 32) {
    mg->c_abort = s_abort | (ncta > 1 ? reinterpret_cast<const int*>(srecv)[G * kHeadDim + 2 * G] : 0);
  }
  __syncthreads();
  const bool c_abort = mg->c_abort != 0;
  float* part = a.partials + ((size_t)vu * ncl + item / ncta) * G * kPartStride;
  for (int q4 = tid; q4 < G * kHeadDim / 4; q4 += kThreads) {
    const int hh = (4 * q4) / kHeadDim, d = (4 * q4) % kHeadDim;
    const float e0 = mg->ce[0][hh], e1 = mg->ce[1][hh];
    const float4 v0 = *reinterpret_cast<const float4*>(cpo + 4 * q4);
    const float4 v1 = ncta > 1 ? *reinterpret_cast<const float4*>(srecv + 4 * q4) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 O = make_float4(fmaf(e1, v1.x, e0 * v0.x), fmaf(e1, v1.y, e0 * v0.y), fmaf(e1, v1.z, e0 * v0.z),
                                 fmaf(e1, v1.w, e0 * v0.w));
    if (ncl == 1) {  // the unit's only cluster: the output rows
      if (!c_abort) {
        const float L = mg->cL[hh];
        const float invL = L > 0.f ? 1.0f / L : 0.f;
        if (d == 0 && !(L > 0.f)) atomicOr(a.status, kStatusEmpty);
        store_out4(a, head_row(a, b, h, t0, hh) * kHeadDim + d,
                   make_float4(O.x * invL, O.y * invL, O.z * invL, O.w * invL));
      }
    } else {  // the cluster's partial, for the unit's last merge
      *reinterpret_cast<float4*>(part + hh * kPartStride + 4 + d) = O;
      if (d == 0) {
        part[hh * kPartStride + 0] = mg->cM[hh];
        part[hh * kPartStride + 1] = mg->cL[hh];
      }
    }
  }
  if (ncl == 1) {
    if (S_next >= 0 && tid == 0 && !c_abort) {  // every item of the unit has read the old state
      a.state[2 * unit] = S_next;
      a.state[2 * unit + 1] = Sq_next;
    }
    return;
  }

  // ======================= the unit's last cluster merges the clusters' partials (an
  // atomic counter, reset by that cluster for the next call; nobody waits).  A cluster that
  // gave up on a wait adds 2^16 as well, and the last one then writes nothing.
  __syncthreads();  // the partial is written; thread 0's acquire-release add publishes it
  if (tid == 0) {
    const uint32_t inc = mg->c_abort ? 0x10001u : 1u;
    const uint32_t old = atomic_add_acq_rel(&a.tickets[vu], inc);
    s_last = ((old & 0xFFFFu) == (uint32_t)(ncl - 1)) ? (((old + inc) >> 16) != 0 ? 2u : 1u) : 0u;
  }
  __syncthreads();  // (and orders the other clusters' partials before this CTA's reads of them)
  if (!s_last) return;
  if (s_last == 1u) {
    merge_partials<G>(a, unit, t0, a.partials + (size_t)vu * ncl * G * kPartStride, ncl, wts);
    if (S_next >= 0 && tid == 0) {  // every item of the unit has read the old state
      a.state[2 * unit] = S_next;
      a.state[2 * unit + 1] = Sq_next;
    }
  }
  if (tid == 0) a.tickets[vu] = 0u;
}

// One launch of the main kernel, in clusters of d.cluster consecutive work items (no
// attribute for clusters of one).  `dependent` (the fused step) makes it the programmatic
// dependent of the kernel before it in the stream, which it may overlap: whatever it reads
// from that kernel is behind griddepcontrol.wait.
template <int BITS, int G>
cudaError_t launch_main_t(const Derived& d, const DecodeArgs& a, cudaStream_t st, bool dependent) {
  constexpr size_t smem = Shared<BITS, G>::bytes();
  cudaError_t e = ensure_smem_attr<decode_main_kernel<BITS, G>>((int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(d.n_split, d.units);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (d.cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)d.cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (dependent) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  lc.attrs = attr;
  lc.numAttrs = n;
  e = cudaLaunchKernelEx(&lc, decode_main_kernel<BITS, G>, a);
  if (e != cudaSuccess && dependent) {  // without the programmatic dependency: plain stream order
    (void)cudaGetLastError();
    lc.numAttrs = n - 1;
    e = cudaLaunchKernelEx(&lc, decode_main_kernel<BITS, G>, a);
  }
  return e;
}

template <int BITS>
cudaError_t launch_main_b(const Derived& d, const DecodeArgs& a, cudaStream_t st, bool dependent) {
  switch (d.group) {
    case 1: return launch_main_t<BITS, 1>(d, a, st, dependent);
    case 2: return launch_main_t<BITS, 2>(d, a, st, dependent);
    case 4: return launch_main_t<BITS, 4>(d, a, st, dependent);
    default: return launch_main_t<BITS, 8>(d, a, st, dependent);
  }
}

}  // namespace

template <int BITS>
cudaError_t launch_query_b(const Derived& d, const DecodeArgs& a, cudaStream_t st) {
  switch (d.group) {
    case 1: decode_query_kernel<BITS, 1><<<d.units, 128, 0, st>>>(a); break;
    case 2: decode_query_kernel<BITS, 2><<<d.units, 128, 0, st>>>(a); break;
    case 4: decode_query_kernel<BITS, 4><<<d.units, 128, 0, st>>>(a); break;
    default: decode_query_kernel<BITS, 8><<<d.units, 128, 0, st>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_decode(const Derived& d, int bits, const DecodeArgs& a, cudaStream_t st) {
  // the query kernel, then the main kernel as its programmatic dependent
  const cudaError_t e = bits == 2 ? launch_query_b<2>(d, a, st) : launch_query_b<4>(d, a, st);
  if (e != cudaSuccess) return e;
  return bits == 2 ? launch_main_b<2>(d, a, st, true) : launch_main_b<4>(d, a, st, true);
}

cudaError_t launch_decode_main(const Derived& d, int bits, const DecodeArgs& a, cudaStream_t st) {
  return bits == 2 ? launch_main_b<2>(d, a, st, true) : launch_main_b<4>(d, a, st, true);
}

}  // namespace wushkv
