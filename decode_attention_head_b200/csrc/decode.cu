// Decode attention over the packed cache ("WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms", §4.1 grouped-query attention re-evaluated at each new
// length S; §4.2 query-side compensation q' = T_K^{-T} q after RoPE, so q'.k' = q.k;
// §4.4 fp16 sink / recent windows around the quantized middle region).
//
// Two launches per call:
//  1. decode_prologue (one 512-thread CTA per (sequence, KV head)): q'_j = T_K^{-T} q_j
//     for its g query heads in fp32, the query's fixed-point tensor-core operand built
//     from it (qfrag.cuh), and the reset of the unit's completion counters.  It releases
//     the main kernel at once (programmatic dependent launch), so the main kernel's KV
//     stream starts while it runs.  (In a fused step, wushkv_step, the append kernel does
//     this work instead; the main kernel then derives the post-append state itself,
//     streams the tiles the append cannot touch at once and waits for the append before
//     reading anything else -- see DecodeArgs::fused.)
//  2. decode_main: grid (n_split, units).  Work item s of a unit takes the s-th share of
//     the unit's current quantized region [S_sink, S_quant) (whole 128-position stages)
//     and of its fp16 window positions (sink [0, S_sink) and recent [S_quant, S)).
//     The quantized positions stream through shared memory in 128-position stages
//     (K codes, V codes, K and V (s, z)) via bulk copies on an mbarrier ring.  Ten warps:
//       producer  one lane issues the stages' bulk copies;
//       MMA       one lane issues, per stage, the QK^T product on the fifth-generation
//                 tensor cores: tcgen05.mma kind::i8, M = 128 positions, N = 4 limbs per
//                 query head, K = 128 masked key codes (u8, in tensor memory) x the
//                 query's signed 8-bit limbs (shared memory), exact int32 in tensor memory;
//       position warps (4)  one thread per position: mask the stage's key codes into the
//                 MMA's A operand (tensor memory), then read their row of q'.c back,
//                 form the logits log2e*scale*(z*sum(q') + s*sigma*D) (dequantization
//                 folded), run the online softmax (base 2, a running max that may go
//                 stale by 2^8) and write the PV weights p*s (fp16 hi + lo) for
//       value warps (4)  paired one to one with the position warps (the same 32 positions
//                 of every stage): PV on mma.sync m16n8k16 with the V codes unpacked in
//                 registers as exact fp16 subnormals, fp32 accumulate; before the stages
//                 they take the item's share of the fp16 window on an exact scalar path.
//     Each item merges its warps and writes (m, l, o); the last item of each group of
//     items merges the group, the last group merges the groups and writes the output
//     (atomic counters, nobody waits).
//
// Key codes: masking a packed 32-bit word with 0x03030303 << 2m leaves, in each byte, one
// code times 4^m -- an exact u8 operand; the 4^m is divided out of the query's integer
// representation.  Value codes: pairs of 16-bit code chunks (one per token) are shifted so
// that one code sits at bits 4..9 of each half and masked: the half is then the fp16
// subnormal c * 2^(b-24) (b = 4, 6 or 8, the code's lowest bit), an exact operand whose
// power-of-two scale is undone once per output row.  Codes are kept high in the subnormal
// range on purpose: the tensor core aligns a product by the operand's nominal exponent (-14
// for every subnormal), so each leading zero bit of a subnormal costs one bit of the
// product's precision inside the MMA; at bits 4..9 at most 6 of 24 are lost.
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

constexpr int kPosWarps = 4;             // one thread per position of a 128-position stage
constexpr int kValWarps = 4;             // PV partners of the position warps
constexpr int kConsumers = 4;            // pseudo-warps per path in the item merge
constexpr int kProducerWarp = kPosWarps + kValWarps;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kSlice = 32;               // positions per warp pair per stage
constexpr int kPartStride = 132;         // floats per (item, head) partial: m, l, pad, pad, o[128]
constexpr int kTau = 8;                  // log2 headroom of the stale running max
constexpr int kQkBufs = 4;               // key operands / QK results in flight (tensor memory)
constexpr uint32_t kTmemCols = 256;      // 4 key operands (32 columns each) + 4 QK results (16 or 32)
static_assert(kTileTokens == kPosWarps * kSlice, "a stage holds one slice per warp pair");

// 2^n as an fp32 bit pattern, exact for -126 <= n <= 127.
__device__ __forceinline__ float pow2i(int n) { return __int_as_float((n + 127) << 23); }

__device__ __forceinline__ float ex2(float x) {  // 2^x (hardware approximation, 2^-inf = 0)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Row (in units of 128 elements) of query head v (0..G-1) of unit (b, h) in q and out: a
// one-token decode has its G heads side by side; chunk attention's v is token v / gq of the
// launch's block of the chunk, head v % gq.
__device__ __forceinline__ size_t head_row(const DecodeArgs& a, int b, int h, int v) {
  const int t = v / a.gq, hh = v - t * a.gq;
  const int ntok = a.chunk_n > 0 ? a.chunk_n : 1;
  return ((size_t)b * ntok + a.chunk_t0 + t) * a.Hq + (size_t)h * a.gq + hh;
}

// Stage ring depth: a stage holds its shared-memory slot from the copy's issue until its PV
// is done (load latency plus three hand-offs), so each CTA keeps as many stages in flight as
// two CTAs per SM can hold (2-bit: 8 x 9 KB; 4-bit: 5 x 17 KB, 4 at eight query heads).
template <int BITS, int G>
struct Cfg {
  static constexpr int CB = 16 * BITS;
  static constexpr int NSTAGE = BITS == 2 ? 8 : (G == 8 ? 4 : 5);
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

// ---------------------------------------------------------------------------------
// Prologue: one CTA per unit, 512 threads; thread (part, j) sums 32 of the 128 terms of
// q'[j] = sum_i Tinv[i][j] q[i], the four parts are added in shared memory, and the CTA
// then builds the unit's query fragments (qfrag.cuh) for every work item of the unit.
constexpr int kPrologueThreads = 512;

template <int BITS, int G>
__global__ void __launch_bounds__(kPrologueThreads) decode_prologue_kernel(const DecodeArgs a) {
  __shared__ __align__(16) float qs[G][kHeadDim];  // q, then q'
  __shared__ float part[4][G][kHeadDim];
  __shared__ float red[64];
  griddep_launch();
  const int unit = blockIdx.x;
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  const int tid = threadIdx.x, j = tid & (kHeadDim - 1), pt = tid >> 7;
  const float* Ti = a.t_k_inv + (size_t)h * kHeadDim * kHeadDim + (size_t)(32 * pt) * kHeadDim + j;
  // all 32 of this thread's T_K^{-1} loads are in flight before q is staged: one round trip
  float t[32];
#pragma unroll
  for (int u = 0; u < 32; ++u) t[u] = __ldg(Ti + (size_t)u * kHeadDim);
  for (int i = tid; i < G * kHeadDim; i += kPrologueThreads) {
    const int hh = i / kHeadDim, cc = i % kHeadDim;
    qs[hh][cc] = __half2float(a.q[head_row(a, b, h, hh) * kHeadDim + cc]);
  }
  if (a.prep.enabled) {  // raw queries (fused step, bulk route): RMSNorm + RoPE at position S - 1
    __syncthreads();
    const int qpos = max(a.state[2 * unit] - 1, 0);
    for (int hh = tid >> 5; hh < G; hh += kPrologueThreads / 32)
      prep_head_warp(qs[hh], a.prep.q_gain, a.prep, qpos, tid & 31);
  }
  __syncthreads();
  float qp[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) qp[hh] = 0.f;
#pragma unroll
  for (int u = 0; u < 32; ++u)
#pragma unroll
    for (int hh = 0; hh < G; ++hh) qp[hh] = fmaf(t[u], qs[hh][32 * pt + u], qp[hh]);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) part[pt][hh][j] = qp[hh];
  __syncthreads();
  for (int i = tid; i < G * kHeadDim; i += kPrologueThreads) {
    const int hh = i / kHeadDim, q = i % kHeadDim;
    const float v = (part[0][hh][q] + part[1][hh][q]) + (part[2][hh][q] + part[3][hh][q]);
    qs[hh][q] = v;
    a.qprime[((size_t)unit * G + hh) * kHeadDim + q] = v;
  }
  // completion counters of the unit: its group counters, then the unit counter
  const int ngroups = (a.n_split + kMergeGroup - 1) / kMergeGroup;
  for (int i = tid; i < ngroups; i += kPrologueThreads) a.tickets[a.units + (size_t)unit * ngroups + i] = 0u;
  if (tid == 0) a.tickets[unit] = 0u;
  __syncthreads();
  build_query_frags<BITS, G>(qs, tid, kPrologueThreads, red, a.scale_log2, a.qfrag + (size_t)unit * kQFragBytes,
                             [] { __syncthreads(); });
}

// ---------------------------------------------------------------------------------
struct Merge {  // per pseudo-warp (0..3 quantized path, 4..7 window path) and head
  float m[8][8], l[8][8], bias[8][8];
  float e[8][8];      // the pseudo-warps' weights 2^(m - M) in the item's merge
  float M[8], L[8];   // the item's merged max and denominator per head
};

// PV weights handed from a position warp to its value warp, per stage (double-buffered):
// for each of the two 16-position k-blocks, NC columns (G <= 4: heads' hi parts in columns
// 0..3 and lo parts in 4..7; G = 8: hi in 0..7, lo in 8..15) of eight 32-bit words; word
// 2 * (r % 4) + (r / 4) % 2 of a column holds block positions r (low half) and r + 8, as the
// m16n8k16 B fragment of lane (g = column, t4 = r % 4) wants them.  Then a header: a flag
// and, when it is set, the factor each head's accumulator must first be multiplied by.
template <int G>
struct WB {
  static constexpr int NC = G <= 4 ? 8 : 16;
  static constexpr int KB = NC * 32 + 32;     // one k-block, padded: conflict-free stores
  static constexpr int HDR = 2 * KB;          // int flag, pad, float factor[8]
  static constexpr int BYTES = HDR + 48;
};

template <int BITS, int G>
struct Shared {
  static constexpr int kStages = Cfg<BITS, G>::NSTAGE * Cfg<BITS, G>::STAGE;
  static constexpr int kPv = kConsumers * G * kHeadDim * 4;  // [4][G][128] fp32, reuses the stages
  static constexpr int kArena = kStages > kPv ? kStages : kPv;
  static constexpr int kWbuf = kPosWarps * 2 * WB<G>::BYTES;
  static constexpr int kNumBars = 2 * Cfg<BITS, G>::NSTAGE + 2 * kQkBufs + 4 * kPosWarps;
  static constexpr size_t kFixed = (size_t)kArena + kWbuf + GCfg<G>::QBYTES + kNumBars * 8 + sizeof(Merge) +
                                   (size_t)kPv + 64;
  static size_t bytes(int nitems) { return kFixed + (size_t)nitems * G * 4; }
};

// One position thread's key record (stage row r) masked into the 32 columns of its tensor
// memory lane: column c = 8 m + w holds word w & (0x03030303 << 2 m) (2-bit), column
// c = 16 m + w holds word w & (0x0F0F0F0F << 4 m) (4-bit) -- the K order qfrag.cuh encodes.
template <int BITS>
__device__ __forceinline__ void store_key_operand(const uint8_t* st, int r, uint32_t taddr) {
  constexpr int CB = 16 * BITS;
  const uint4* rec = reinterpret_cast<const uint4*>(st + r * CB);
  uint32_t v[32];
  if (BITS == 2) {
    const uint4 u0 = rec[0], u1 = rec[1];
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 * m + i] = w[i] & (0x03030303u << (2 * m));
  } else {
    const uint4 u0 = rec[0], u1 = rec[1], u2 = rec[2], u3 = rec[3];
    const uint32_t w[16] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w,
                            u2.x, u2.y, u2.z, u2.w, u3.x, u3.y, u3.z, u3.w};
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int i = 0; i < 16; ++i) v[16 * m + i] = w[i] & (m ? 0xF0F0F0F0u : 0x0F0F0F0Fu);
  }
  tmem_st32(taddr, v);
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
                             int lane, WinRows<G>& w, Merge* mg, float* wpv, int qlim) {
  constexpr int KB = WinRows<G>::KB;
  float qv[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float4 t = *reinterpret_cast<const float4*>(a.qprime + ((size_t)unit * G + hh) * kHeadDim + 4 * lane);
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

// Merge `count` (<= kMergeMax) consecutive partials (m, l, pad, pad, o[128] per head, base 2, o not
// yet normalised) of one unit.  dst != nullptr: write the merged partial there; else write
// the normalised output rows of the unit's G query heads.  wts: shared [count][G].  Lane
// `it` of the warp of head hh reads partial it's (m, l) in one round trip.
constexpr int kMergeMax = 16;  // partials one merge level reads at most
static_assert(kMergeGroup <= kMergeMax && (kMaxSplits + kMergeGroup - 1) / kMergeGroup <= kMergeMax,
              "a merge level reads at most kMergeMax partials (one per lane of a warp)");
template <int G>
__device__ void merge_partials(const DecodeArgs& a, int unit, const float* src, int count, float* dst,
                               float* wts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // thread (hh, quad) takes dimensions 4*quad .. 4*quad+3 of head hh: every partial's row is
  // loaded at once, the first (head, quad)'s rows before the weights are known, so that
  // their round trip overlaps the (m, l) one; then they are summed in partial order.  Every
  // partial is finite (an empty one holds o = 0), so no term needs skipping.
  constexpr int kQuads = kHeadDim / 4;
  float4 ov[kMergeMax];
  auto load_rows = [&](int idx) {
    const int hh = idx / kQuads, d = 4 * (idx % kQuads);
#pragma unroll
    for (int it = 0; it < kMergeMax; ++it)
      ov[it] = it < count ? __ldcg(reinterpret_cast<const float4*>(src + ((size_t)it * G + hh) * kPartStride + 4 + d))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  if (tid < G * kQuads) load_rows(tid);
  for (int hh = warp; hh < G; hh += kThreads / 32) {
    const bool has = lane < count;
    float mi = -CUDART_INF_F, li = 0.f;
    if (has) {
      mi = __ldcg(src + ((size_t)lane * G + hh) * kPartStride);
      li = __ldcg(src + ((size_t)lane * G + hh) * kPartStride + 1);
    }
    float M = mi;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float e = (!has || M == -CUDART_INF_F) ? 0.f : exp2f(mi - M);
    if (has) wts[lane * G + hh] = e;
    float L = fmaf(e, li, 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    __syncwarp();
    if (dst) {
      if (lane == 0) {
        dst[hh * kPartStride + 0] = M;
        dst[hh * kPartStride + 1] = L;
      }
    } else {
      const float invL = L > 0.f ? 1.0f / L : 0.f;
      for (int it = lane; it < count; it += 32) wts[it * G + hh] *= invL;
      if (lane == 0 && !(L > 0.f)) atomicOr(a.status, kStatusEmpty);
    }
  }
  __syncthreads();
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  for (int idx = tid; idx < G * kQuads; idx += kThreads) {
    const int hh = idx / kQuads, d = 4 * (idx % kQuads);
    if (idx != tid) load_rows(idx);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int it = 0; it < kMergeMax; ++it) {
      if (it < count) {
        const float w = wts[it * G + hh];
        acc.x = fmaf(w, ov[it].x, acc.x);
        acc.y = fmaf(w, ov[it].y, acc.y);
        acc.z = fmaf(w, ov[it].z, acc.z);
        acc.w = fmaf(w, ov[it].w, acc.w);
      }
    }
    if (dst) {
      *reinterpret_cast<float4*>(dst + hh * kPartStride + 4 + d) = acc;
    } else {
      const size_t o = head_row(a, b, h, hh) * kHeadDim + d;
      if (a.out_fp16) {
        __half2* oh = reinterpret_cast<__half2*>(reinterpret_cast<__half*>(a.out) + o);
        oh[0] = __floats2half2_rn(acc.x, acc.y);
        oh[1] = __floats2half2_rn(acc.z, acc.w);
      } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + o) = acc;
      }
    }
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
  using C = Cfg<BITS, G>;
  using SM = Shared<BITS, G>;
  using W = WB<G>;
  constexpr int NQ = GCfg<G>::NQ, NHS = GCfg<G>::NHS, LBO = GCfg<G>::LBO;
  constexpr int CB = C::CB, NST = C::NSTAGE;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  float* pv = reinterpret_cast<float*>(smem);  // [4][G][128], written once the stages are drained
  uint8_t* wbuf = smem + SM::kArena;           // [4 warp pairs][2 buffers] PV weights
  uint8_t* qop = wbuf + SM::kWbuf;             // the QK MMA's B operand (query limbs)
  uint64_t* full = reinterpret_cast<uint64_t*>(qop + GCfg<G>::QBYTES);
  uint64_t* empty = full + NST;
  uint64_t* kready = empty + NST;              // [4] key operand of a stage in tensor memory
  uint64_t* qkdone = kready + kQkBufs;         // [4] its QK product complete
  uint64_t* wfull = qkdone + kQkBufs;          // [4][2] weights written by position warp w
  uint64_t* wempty = wfull + 2 * kPosWarps;    // [4][2] ... consumed by value warp w
  Merge* mg = reinterpret_cast<Merge*>(full + SM::kNumBars);
  float* wpv = reinterpret_cast<float*>(mg + 1);                // window path [4][G][128]
  float* wts = wpv + kConsumers * G * kHeadDim;                 // [nitems][G] (last item only)
  __shared__ uint32_t s_last, s_taddr;
  __shared__ int s_abort;
  volatile int* abort = &s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y, item = blockIdx.x;
  const int nitems = a.n_split;
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
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPosWarps + kValWarps);
    }
    for (int b = 0; b < kQkBufs; ++b) {
      mbar_init(&kready[b], kPosWarps);
      mbar_init(&qkdone[b], 1);
    }
    for (int i = 0; i < 2 * kPosWarps; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&wempty[i], 1);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < SM::kWbuf / 16; i += kThreads) reinterpret_cast<uint4*>(wbuf)[i] = make_uint4(0, 0, 0, 0);
  if (warp == kMmaWarp) tmem_alloc(&s_taddr, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = s_taddr;

  float o[8][4];  // value warps: the PV accumulators of their 32 positions per stage
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

  if (warp == kProducerWarp) {
    // ---------------- producer: streams the item's tiles; needs nothing from the prologue
    if (lane == 0) {  // warm L2 with the item's fp16 window rows, read at the end of the item
      const int s_end = min(wend, n_sink);
      if (wbeg < s_end) {
        const size_t row = (size_t)unit * a.sink_dim + wbeg;
        bulk_prefetch_l2(a.k_sink + row * kHeadDim, (uint32_t)(s_end - wbeg) * kHeadDim * 2);
        bulk_prefetch_l2(a.v_sink + row * kHeadDim, (uint32_t)(s_end - wbeg) * kHeadDim * 2);
      }
      const int rb = max(wbeg, n_sink);
      if (rb < wend) {
        const int cnt = wend - rb, slot0 = (r0 + (rb - n_sink)) % a.R;
        const int first = min(cnt, a.R - slot0);
        const size_t row = (size_t)unit * a.R;
        bulk_prefetch_l2(a.k_ring + (row + slot0) * kHeadDim, (uint32_t)first * kHeadDim * 2);
        bulk_prefetch_l2(a.v_ring + (row + slot0) * kHeadDim, (uint32_t)first * kHeadDim * 2);
        if (cnt > first) {
          bulk_prefetch_l2(a.k_ring + row * kHeadDim, (uint32_t)(cnt - first) * kHeadDim * 2);
          bulk_prefetch_l2(a.v_ring + row * kHeadDim, (uint32_t)(cnt - first) * kHeadDim * 2);
        }
      }
    }
    if (lane == 0 && ntiles > 0) {
      int issued = 0;
      bool waited = !a.fused;  // fused step: tiles below the old S_quant stream at once
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NST;
        if (!waited && tile0 + (t + 1) * kTileTokens > sq_stable) {
          griddep_wait();
          waited = true;
        }
        if (t >= NST && !mbar_wait_abortable(&empty[s], ((t / NST) - 1) & 1, a.status, abort, a.wait_limit)) break;
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
      for (int t = max(0, issued - NST); t < issued; ++t)
        if (t != a.withhold_tile) mbar_wait(&full[t % NST], (t / NST) & 1, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- tensor-core issue: the query operand into shared memory, then one
    // QK^T product per stage as soon as the position warps have stored its key operand
    griddep_wait();  // the operand comes from the prologue (or the fused append)
    const uint4* src = reinterpret_cast<const uint4*>(a.qfrag + (size_t)unit * kQFragBytes);
    for (int i = lane; i < GCfg<G>::QBYTES / 16; i += 32) reinterpret_cast<uint4*>(qop)[i] = src[i];
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8_u8s8(128, NQ);
      const uint32_t qaddr = smem_u32(qop);
      int last[kQkBufs] = {-1, -1, -1, -1};
      for (int t = 0; t < ntiles; ++t) {
        const int b = t % kQkBufs;
        if (!mbar_wait_abortable(&kready[b], (t / kQkBufs) & 1, a.status, abort, a.wait_limit)) break;
        tc_fence_after();
        const uint32_t acol = tbase + 32 * b, dcol = tbase + 32 * kQkBufs + NQ * b;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_i8_ts(dcol, acol + 8 * kk, smem_desc(qaddr + 2 * kk * LBO, LBO, 128), idesc, kk > 0);
        mma_commit(&qkdone[b]);
        last[b] = t;
      }
      // no product may still be writing tensor memory when it is released
      for (int b = 0; b < kQkBufs; ++b)
        if (last[b] >= 0) mbar_wait(&qkdone[b], (last[b] / kQkBufs) & 1, a.status);
    }
  } else if (warp < kPosWarps) {
    // ---------------- position warps: thread = position r of every stage
    const int w = warp, r = kSlice * w + lane;
    const uint32_t lrow = (uint32_t)(kSlice * w) << 16;  // this warp's tensor-memory lanes
    griddep_wait();  // the per-head constants come from the prologue (or the fused append)
    const float* hc = reinterpret_cast<const float*>(a.qfrag + (size_t)unit * kQFragBytes + GCfg<G>::QBYTES);
    float Ah[G], Bh[G], mref[G], lsum[G], bsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      Ah[h] = hc[h];
      Bh[h] = hc[8 + h];
      mref[h] = -CUDART_INF_F;
      lsum[h] = 0.f;
      bsum[h] = 0.f;
    }
    int kacc = 64;
    float s_lim = 0.f;  // the first position with s > 0 sets kacc
    // Key operands go to tensor-memory buffer u % 4 (free: the product of stage u - 4 that
    // read it, and wrote the result buffer stage u reuses, was complete and read before this
    // warp got past stage u - 4).  The stores are asynchronous: those issued at the top of an
    // iteration complete while the stage's softmax runs, and are handed to the MMA warp
    // (wait, fence, arrive) only after it.
    auto store_keys = [&](int u) {
      store_key_operand<BITS>(stages + (u % NST) * C::STAGE, r, tbase + lrow + 32 * (u % kQkBufs));
    };
    auto commit_keys = [&](int u0, int u1) {  // stages [u0, u1) stored: release them to the MMA
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int u = u0; u < u1; ++u) mbar_arrive(&kready[u % kQkBufs]);
    };
    uint32_t dn0[16], dn1[16];  // a stage's QK result, in flight from tensor memory
    auto load_result = [&](int u) {
      const uint32_t col = tbase + lrow + 32 * kQkBufs + NQ * (u % kQkBufs);
      tmem_ld16(col, dn0);
      if (NQ == 32) tmem_ld16(col + 16, dn1);
    };
    auto wait_result = [&]() {
      tmem_wait_ld16(dn0);
      if (NQ == 32) tmem_wait_ld16(dn1);
    };
    bool have_next = false;  // the result of the stage about to be processed is in flight
    int staged = 0;  // key operands stored so far: stages [0, staged)
    for (int t = 0; t < ntiles; ++t) {
      const int slot = t % NST, b = t & 1;
      const uint8_t* st = stages + slot * C::STAGE;
      if (staged == t) {  // starved: this stage's operand is needed now
        if (!warp_wait(&full[slot], (t / NST) & 1, a, abort)) break;
        store_keys(t);
        commit_keys(t, t + 1);
        staged = t + 1;
      }
      // the operands of the next stages whose data has landed, up to 3 ahead (never waits)
      const int s0 = staged;
      while (staged < ntiles && staged <= t + kQkBufs - 1 &&
             __all_sync(0xffffffffu, mbar_test_wait(&full[staged % NST], (staged / NST) & 1))) {
        store_keys(staged);
        ++staged;
      }
      // this stage's QK result: loaded ahead during the previous stage when it was ready
      if (!have_next) {
        if (!warp_wait(&qkdone[t % kQkBufs], (t / kQkBufs) & 1, a, abort)) break;
        tc_fence_after();
        load_result(t);
      }
      wait_result();
      uint32_t dq[NQ];
#pragma unroll
      for (int c = 0; c < 16; ++c) dq[c] = dn0[c];
      if (NQ == 32) {
#pragma unroll
        for (int c = 0; c < 16; ++c) dq[(16 + c) % NQ] = dn1[c];
      }
      // the next stage's result, if its product is complete, loads while this one's
      // softmax runs (its key operand was handed over in an earlier iteration)
      have_next = t + 1 < ntiles && t + 1 < s0 &&
                  __all_sync(0xffffffffu, mbar_test_wait(&qkdone[(t + 1) % kQkBufs], ((t + 1) / kQkBufs) & 1));
      if (have_next) {
        tc_fence_after();
        load_result(t + 1);
      }
      // ---- logits (base 2) of this thread's position, one per head
      const int pos = tile0 + t * kTileTokens + r;
      const bool val = pos >= lo && pos < hi;
      const uint32_t* kpar = reinterpret_cast<const uint32_t*>(st + 2 * kTileTokens * CB);
      const float2 ksz = __half22float2(u32_as_h2(kpar[r]));
      const float2 vsz = __half22float2(u32_as_h2(kpar[kTileTokens + r]));
      float x[G], fac[G];
      bool hit = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        // q'.c / sigma = sum_l 256^l D_l; pairs of limbs combine exactly in int32
        const int d01 = (int)dq[4 * h] + 256 * (int)dq[4 * h + 1];
        const int d23 = (int)dq[4 * h + 2] + 256 * (int)dq[4 * h + 3];
        const float f = fmaf(65536.0f, (float)d23, (float)d01);
        x[h] = val ? fmaf(Bh[h] * ksz.x, f, Ah[h] * ksz.y) : -CUDART_INF_F;
        hit |= x[h] > mref[h] + kTau;
        fac[h] = 1.0f;
      }
      // The running max is kept stale: p = 2^(x - mref) may reach 2^kTau, and only a logit
      // above mref + kTau (a warp vote) triggers the rescale.
      bool post = false;
      if (__any_sync(0xffffffffu, hit)) {
        post = true;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float mx = x[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float mn = fmaxf(mref[h], mx);
          const float al = mn > mref[h] ? ex2(mref[h] - mn) : 1.0f;
          mref[h] = mn;
          lsum[h] *= al;
          bsum[h] *= al;
          fac[h] = al;
        }
      }
      // p*s enters the PV product scaled by 2^kacc: the largest weight sits below 2^14 and
      // small weights stay in fp16's normal range; kacc only decreases, and only a position
      // whose s reaches s_lim = 2^(14 - kTau - kacc) forces a (warp-wide) recomputation.
      // Positions outside the item may hold any bits in (s, z): never use them.
      if (__any_sync(0xffffffffu, val && vsz.x >= s_lim)) {
        float smax = val ? vsz.x : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
        if (smax > 0.f) {
          const int k = 13 - kTau - (((__float_as_int(smax) >> 23) & 255) - 127);
          if (k < kacc) {
            const float fk = pow2i(max(k - kacc, -126));
#pragma unroll
            for (int h = 0; h < G; ++h) fac[h] *= fk;
            kacc = k;
            s_lim = pow2i(14 - kTau - k);
            post = true;
          }
        }
      }
      const float wscale = pow2i(kacc);
      // ---- PV weights for the value warp: its buffer b was read by the stage t - 2
      if (t >= 2 && !warp_wait(&wempty[2 * w + b], ((t >> 1) - 1) & 1, a, abort)) break;
      uint8_t* wb = wbuf + (2 * w + b) * W::BYTES;
      const int rr = lane & 15;
      uint8_t* wcol = wb + (lane >> 4) * W::KB + (2 * (rr & 3) + ((rr >> 2) & 1)) * 4 + (rr >> 3) * 2;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ms = mref[h] == -CUDART_INF_F ? 0.f : mref[h];
        const float p = ex2(x[h] - ms);
        lsum[h] += p;
        const float wv = val ? p * vsz.x * wscale : 0.f;
        bsum[h] += val ? p * vsz.y : 0.f;
        // p*s as an fp16 pair hi + lo: the PV product then carries ~22 bits of p*s,
        // matching the fp32 l it is normalised by
        const __half whi = __float2half_rn(wv);
        const __half wlo = __float2half_rn(wv - __half2float(whi));
        *reinterpret_cast<__half*>(wcol + h * 32) = whi;
        *reinterpret_cast<__half*>(wcol + (h + W::NC / 2) * 32) = wlo;
      }
      if (lane == 0) {
        int* hdr = reinterpret_cast<int*>(wb + W::HDR);
        hdr[0] = post ? 1 : 0;
        hdr[1] = kacc;
        if (post) {
#pragma unroll
          for (int h = 0; h < G; ++h) reinterpret_cast<float*>(hdr)[2 + h] = fac[h];
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&wfull[2 * w + b]);
        mbar_arrive(&empty[slot]);  // this warp is done with the stage's key codes and (s, z)
      }
      if (staged > s0) commit_keys(s0, staged);
    }
    // l and bias summed over the warp's positions
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float lv = lsum[h], bv = bsum[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        lv += __shfl_xor_sync(0xffffffffu, lv, off);
        bv += __shfl_xor_sync(0xffffffffu, bv, off);
      }
      if (lane == 0) {
        mg->m[w][h] = mref[h];
        mg->l[w][h] = lv;
        mg->bias[w][h] = bv;
      }
    }
  } else {
    // ---------------- value warps: the fp16 window share, then PV of the paired positions
    const int w = warp - kPosWarps;
    const int g = lane >> 2, t4 = lane & 3;
    griddep_wait();  // the window holds the appended tokens; q' comes from the prologue
    int kacc = 64;   // the weight scale of the stages seen (the position warp's, via the header)
    for (int t = 0; t < ntiles; ++t) {
      const int slot = t % NST, b = t & 1;
      if (!warp_wait(&full[slot], (t / NST) & 1, a, abort)) break;
      if (!warp_wait(&wfull[2 * w + b], (t >> 1) & 1, a, abort)) break;
      const uint8_t* wb = wbuf + (2 * w + b) * W::BYTES;
      const int* hdr = reinterpret_cast<const int*>(wb + W::HDR);
      kacc = hdr[1];
      if (hdr[0]) {  // the running max or the weight scale moved: rescale first
        const float* fac = reinterpret_cast<const float*>(hdr) + 2;
        // o columns are heads 2t4, 2t4+1 (G <= 4: lo parts in columns 4..7)
        const float c0 = fac[NHS == 1 ? (2 * t4) & 3 : 2 * t4];
        const float c1 = fac[NHS == 1 ? (2 * t4 + 1) & 3 : 2 * t4 + 1];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] *= c0;
          o[mt][1] *= c1;
          o[mt][2] *= c0;
          o[mt][3] *= c1;
        }
      }
      const uint8_t* vc = stages + slot * C::STAGE + kTileTokens * CB;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        // B operand: rows k=2t4,2t4+1 <- positions t4, t4+8; k=2t4+8,+9 <- t4+4, t4+12 (of
        // the block); column n = the lane group g
        const uint2 bw = *reinterpret_cast<const uint2*>(wb + i * W::KB + g * 32 + t4 * 8);
        const uint32_t pb[2] = {bw.x, bw.y};
        uint32_t pbl[2] = {0u, 0u};
        if (NHS == 2) {
          const uint2 bl = *reinterpret_cast<const uint2*>(wb + i * W::KB + (8 + g) * 32 + t4 * 8);
          pbl[0] = bl.x;
          pbl[1] = bl.y;
        }
        // the V codes of k-block i are one 16-position group in the value layout (vgroup_half):
        // lane (g, t4) reads the words pairing positions (t4, t4 + 8) and (t4 + 4, t4 + 12) for
        // its chunks -- four consecutive words, one 16-byte load, the warp's loads contiguous
        const uint8_t* vgrp = vc + (size_t)(kSlice * w + 16 * i) * CB;
        if (BITS == 2) {
          const uint4 vv = *reinterpret_cast<const uint4*>(vgrp + 64 * g + 16 * t4);
          const uint32_t xl1 = vv.x, xl2 = vv.y, xh1 = vv.z, xh2 = vv.w;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const uint32_t A[4] = {vcode2(xl1, mt), vcode2(xh1, mt), vcode2(xl2, mt), vcode2(xh2, mt)};
            mma_f16(o[mt], A, pb);
            if (NHS == 2) mma_f16(o[mt], A, pbl);
          }
        } else {
#pragma unroll
          for (int ws = 0; ws < 2; ++ws) {
            const uint4 vv = *reinterpret_cast<const uint4*>(vgrp + 512 * ws + 64 * g + 16 * t4);
            const uint32_t xl1 = vv.x, xl2 = vv.y, xh1 = vv.z, xh2 = vv.w;
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
              const uint32_t A[4] = {vcode4(xl1, mi), vcode4(xh1, mi), vcode4(xl2, mi), vcode4(xh2, mi)};
              mma_f16(o[4 * ws + mi], A, pb);
              if (NHS == 2) mma_f16(o[4 * ws + mi], A, pbl);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&wempty[2 * w + b]);
        mbar_arrive(&empty[slot]);
      }
    }
    if (NHS == 1) {  // columns 4..7 (lanes t4 = 2, 3) hold the lo parts of heads 0..3
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[mt][c] += __shfl_down_sync(0xffffffffu, o[mt][c], 2);
    }
    // every value warp is done with the stages (and every copy has landed: all were
    // consumed), so the accumulators may go to the stage arena
    bar_sync(1, kValWarps * 32);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int hi2 = 0; hi2 < 2; ++hi2) {
        int dim, l2s;
        value_row<BITS>(mt, g, hi2, dim, l2s);
        const float unscale = pow2i(24 - l2s - kacc);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int hh = 2 * t4 + c;
          if (hh < G) pv[((size_t)w * G + hh) * kHeadDim + dim] = o[mt][2 * hi2 + c] * unscale;
        }
      }
    }
    // the item's share of the fp16 window comes after the stages (its rows were warmed in L2
    // at the start), so that it never holds up the stage ring
    WinRows<G> wr;
    window_load<G>(a, unit, wbeg + w, wend, n_sink, r0, lane, wr);
    const int qlim = a.chunk_n > 0 ? S - a.chunk_n + a.chunk_t0 : INT_MAX;
    window_share<G>(a, unit, wbeg, wend, n_sink, r0, w, lane, wr, mg, wpv, qlim);
  }
  tc_fence_before();
  __syncthreads();  // every stage consumed, every copy landed, every product complete
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
  // a bounded wait gave up (STATUS_TIMEOUT is set): this item's results are incomplete, so
  // it writes no partial and takes no part in the merge -- the unit's output is not written
  if (s_abort) return;


  // ======================= merge the 8 pseudo-warps, write this item's partial: the
  // weights once per (pseudo-warp, head), then the rows
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
    mg->M[hh] = M;
    mg->L[hh] = L;
  }
  __syncthreads();
  float* part = a.partials + ((size_t)unit * nitems + item) * G * kPartStride;
  for (int idx = tid; idx < G * kHeadDim; idx += kThreads) {
    const int hh = idx / kHeadDim, d = idx % kHeadDim;
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < 2 * kConsumers; ++w) {
      const float ov = w < kConsumers ? pv[((size_t)w * G + hh) * kHeadDim + d]
                                      : wpv[((size_t)(w - kConsumers) * G + hh) * kHeadDim + d];
      O = fmaf(mg->e[w][hh], ov + mg->bias[w][hh], O);
    }
    part[hh * kPartStride + 4 + d] = O;
    if (d == 0) {
      part[hh * kPartStride + 0] = mg->M[hh];
      part[hh * kPartStride + 1] = mg->L[hh];
    }
  }
  // ======================= two-level merge: the last item of each group of kMergeGroup
  // items merges the group; the last group to finish merges the groups and writes the
  // output (atomic counters, nobody waits).  Neither level reads more than a few partials.
  const int ngroups = (nitems + kMergeGroup - 1) / kMergeGroup;
  const int grp = item / kMergeGroup;
  const int g0 = grp * kMergeGroup, gn = min(kMergeGroup, nitems - g0);
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    uint32_t* gt = a.tickets + a.units + (size_t)unit * ngroups + grp;
    s_last = (atomicAdd(gt, 1u) == (uint32_t)(gn - 1)) ? 1u : 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* up = a.partials + ((size_t)unit * nitems + g0) * G * kPartStride;
  if (ngroups == 1) {
    merge_partials<G>(a, unit, up, gn, nullptr, wts);
    if (S_next >= 0 && tid == 0) {  // every item of the unit has read the old state
      a.state[2 * unit] = S_next;
      a.state[2 * unit + 1] = Sq_next;
    }
    return;
  }
  float* gp = a.gpartials + ((size_t)unit * ngroups + grp) * G * kPartStride;
  merge_partials<G>(a, unit, up, gn, gp, wts);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.tickets[unit], 1u) == (uint32_t)(ngroups - 1)) ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  merge_partials<G>(a, unit, a.gpartials + (size_t)unit * ngroups * G * kPartStride, ngroups, nullptr, wts);
  if (S_next >= 0 && tid == 0) {  // every item of the unit has read the old state
    a.state[2 * unit] = S_next;
    a.state[2 * unit + 1] = Sq_next;
  }
}

// The main kernel as the programmatic dependent of the kernel before it in the stream: it
// may start before that kernel ends; whatever it reads from it is behind griddepcontrol.wait.
template <int BITS, int G>
cudaError_t launch_main_t(const Derived& d, const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = Shared<BITS, G>::bytes(d.n_split);
  cudaError_t e = ensure_smem_attr<decode_main_kernel<BITS, G>>((int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(d.n_split, d.units);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, decode_main_kernel<BITS, G>, a);
  if (e != cudaSuccess) {  // without the attribute: plain stream order
    (void)cudaGetLastError();
    decode_main_kernel<BITS, G><<<lc.gridDim, kThreads, smem, st>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

template <int BITS, int G>
cudaError_t launch_decode_t(const Derived& d, const DecodeArgs& a, cudaStream_t st) {
  decode_prologue_kernel<BITS, G><<<d.units, kPrologueThreads, 0, st>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the main kernel may start before the prologue ends; its consumers wait
  // (griddepcontrol.wait) for the prologue's results, its producer does not
  return launch_main_t<BITS, G>(d, a, st);
}

template <int BITS>
cudaError_t launch_main_b(const Derived& d, const DecodeArgs& a, cudaStream_t st) {
  switch (d.group) {
    case 1: return launch_main_t<BITS, 1>(d, a, st);
    case 2: return launch_main_t<BITS, 2>(d, a, st);
    case 4: return launch_main_t<BITS, 4>(d, a, st);
    default: return launch_main_t<BITS, 8>(d, a, st);
  }
}

template <int BITS>
cudaError_t launch_decode_b(const Derived& d, const DecodeArgs& a, cudaStream_t st) {
  switch (d.group) {
    case 1: return launch_decode_t<BITS, 1>(d, a, st);
    case 2: return launch_decode_t<BITS, 2>(d, a, st);
    case 4: return launch_decode_t<BITS, 4>(d, a, st);
    default: return launch_decode_t<BITS, 8>(d, a, st);
  }
}

}  // namespace

cudaError_t launch_decode(const Derived& d, int bits, const DecodeArgs& a, cudaStream_t st) {
  return bits == 2 ? launch_decode_b<2>(d, a, st) : launch_decode_b<4>(d, a, st);
}

cudaError_t launch_decode_main(const Derived& d, int bits, const DecodeArgs& a, cudaStream_t st) {
  return bits == 2 ? launch_main_b<2>(d, a, st) : launch_main_b<4>(d, a, st);
}

}  // namespace wushkv
