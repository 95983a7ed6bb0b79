// Quantize-on-append ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
// §4.1 new columns of K_h / V_h, §4.2 post-RoPE key transform k' = T_K k, §4.4
// "Full-Precision Cache Window" (Algorithm 2 prose), §5.3 quantizer).
//
// State per (sequence, KV head): S (cached positions) and S_quant (0 or the exclusive
// end of the quantized region [S_sink, S_quant)).  Flush under a length L:
//   lo0 = max(S_quant, S_sink); e = L - S_keep - lo0;
//   e >= S_flush -> quantize [lo0, lo0 + floor(e/S_flush)*S_flush), S_quant moves there.
//
// Small appends (n_new <= chunk_max), one CTA per (sequence, KV head), one launch:
//   flush under S (the step that closes the previous chunk, whose attention has been
//   computed by now), then transform + store the new tokens fp16, then advance S.
//   In a fused decode step (wushkv_step) a second CTA per unit prepares the decode query
//   in the same launch, and the state words are left to the decode kernel.
// Bulk appends (n_new > chunk_max), three launches in stream order:
//   flush_ring   quantize the ring entries the flush under S + n_new covers;
//   append_bulk  T_K GEMM on tensor cores (mma.sync m16n8k16, fp32 accumulate) per
//                64-token tile, then per token: sink, quantize, or ring;
//   advance      S += n_new, S_quant = the flush's new boundary.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "internal.h"
#include "ptx.cuh"
#include "quantize.cuh"
#include "qfrag.cuh"

namespace wushkv {
namespace {

struct FlushPlan {
  int lo0, nf;
};

__device__ __forceinline__ FlushPlan flush_plan(int Sq, int L, const AppendArgs& a) {
  FlushPlan f;
  flush_bounds(Sq, L, a.s_sink, a.s_keep, a.s_flush, f.lo0, f.nf);
  return f;
}

// A state entry the kernels can trust: 0 <= S_quant <= S <= capacity.
__device__ __forceinline__ bool state_ok(int S, int Sq, const AppendArgs& a) {
  return S >= 0 && S <= a.cap && Sq >= 0 && Sq <= S;
}

__device__ __forceinline__ QuantSpec spec_of(const AppendArgs& a) {
  QuantSpec q;
  q.i_lo = a.i_lo;
  q.i_hi = a.i_hi;
  q.f_lo = a.f_lo;
  q.f_hi = a.f_hi;
  q.rms = a.quant_rms;
  q.kb = a.rms_kb;
  q.alpha = a.rms_alpha;
  return q;
}

// Quantize ring positions [p_begin, p_end) of `unit` (K and V): each row is split over four
// adjacent threads (quantize_row_part), nthreads / 4 rows at a time.
template <int BITS, int NSEL>
__device__ void quantize_ring_range(const AppendArgs& a, int unit, int p_begin, int p_end, int tid = threadIdx.x,
                                    int nthreads = blockDim.x) {
  const int n = p_end - p_begin;
  if (n <= 0) return;
  constexpr int CB = 16 * BITS;
  constexpr int P = 4;
  const QuantSpec qs = spec_of(a);
  for (int item = tid / P; item < 2 * n; item += nthreads / P) {
    const int kind = item / n;  // 0 = K, 1 = V
    const int p = p_begin + item % n;
    const __half* ring = kind ? a.v_ring : a.k_ring;
    const __half* row = ring + ((size_t)unit * a.R + (p % a.R)) * kHeadDim;
    const size_t rec = (size_t)unit * a.cap_alloc + p;
    uint32_t* params = (kind ? a.v_params : a.k_params) + rec;
    // value codes go to the position's 16-position group (cap_alloc is a multiple of 16); one
    // call site, so that the quantizer is inlined once
    uint8_t* codes = kind ? a.v_codes + (rec & ~(size_t)15) * CB : a.k_codes + rec * CB;
    quantize_row_part<BITS, NSEL, P>(row, tid % P, codes, params, qs, kind ? (p & 15) : -1);
  }
}

// ---------------------------------------------------------------------------------
// q'_j = T_K^{-T} q_j (fp32) of the unit's G query heads into the decode workspace, by the
// CTA's 128 threads: thread j loads column j of T_K^{-1} (all 128 rows in flight at once)
// and sums Tinv[i][j] * q[i] in the chains every decode path takes (qprime_chains, with
// a.qchains = the decode's cluster size), so that the fused step and a plain decode see the
// same q'.  Also builds the unit's query fragments for the decode kernel (qfrag.cuh).
template <int BITS, int G>
__device__ void prepare_query(const AppendArgs& a, int unit, int tid) {
  __shared__ __align__(16) float qs[G][kHeadDim];
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  const int warp = tid >> 5, lane = tid & 31;
  const float* Tcol = a.t_k_inv + (size_t)h * kHeadDim * kHeadDim + tid;
  float t[kHeadDim];
#pragma unroll
  for (int i = 0; i < kHeadDim; ++i) t[i] = __ldg(Tcol + (size_t)i * kHeadDim);
  for (int i = tid; i < G * kHeadDim; i += 128)
    qs[i / kHeadDim][i % kHeadDim] = __half2float(a.q[((size_t)b * a.Hq + h * G) * kHeadDim + i]);
  if (a.prep.enabled) {  // raw queries: RMSNorm + RoPE at the query's position, head by head
    // the query is the newest token: position S + n_new - 1 (S - 1 if the append is refused);
    // the state is read here, after the loads above are in flight
    const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
    const bool valid = state_ok(S, Sq, a);
    const bool fits = valid && S + a.n_new <= a.cap;
    const int qpos = max((fits ? S + a.n_new : (valid ? S : 1)) - 1, 0);
    bar_sync(2, 128);
    for (int hh = warp; hh < G; hh += 4) prep_head_warp(qs[hh], a.prep.q_gain, a.prep, qpos, lane);
  }
  bar_sync(2, 128);
  float acc[G];
  qprime_chains<G>(t, qs, a.qchains, acc);
  bar_sync(2, 128);  // every thread has read q
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    qs[hh][tid] = acc[hh];
    a.qprime[((size_t)unit * G + hh) * kHeadDim + tid] = acc[hh];
  }
  bar_sync(2, 128);
  __shared__ float cred[64];
  build_query_frags<BITS, G>(qs, tid, 128, cred, a.scale_log2, a.qfrag + (size_t)unit * kQFragBytes,
                             [] { bar_sync(2, 128); });
}

// Row r (= the thread) of k' = T_K k in fp32: its 256-byte row of T_K (tr, fp16) against the
// key staged in shared memory, in four interleaved partial sums added at the end.
__device__ __forceinline__ float key_row(const uint4 (&tr)[kHeadDim / 8], const float* ks) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < kHeadDim / 8; ++i) {
    const uint32_t w[4] = {tr[i].x, tr[i].y, tr[i].z, tr[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 tf = __half22float2(u32_as_h2(w[e]));
      acc[e] = fmaf(tf.x, ks[8 * i + 2 * e], acc[e]);
      acc[e] = fmaf(tf.y, ks[8 * i + 2 * e + 1], acc[e]);
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// The small append's new tokens, one after another: k' = fp16_rn(T_K k) (fp32 accumulation;
// or the Walsh-Hadamard transform), v as given, into the sink or the ring.  Thread r owns
// output row r: its row of T_K is loaded once (16 x 16 B in flight); the token's key is
// staged in shared memory (ks) as fp32, after RMSNorm + RoPE at its position when the step
// takes raw keys.  All 128 threads of the CTA take part (named barrier 1).
__device__ void append_tokens(const AppendArgs& a, int unit, int b, int h, int S, float* ks) {
  __shared__ float hs[kHeadDim];  // Hadamard butterflies across warps
  const int r = threadIdx.x;
  const bool hadamard = a.transform == WUSHKV_TRANSFORM_HADAMARD;
  uint4 tr[kHeadDim / 8];
  if (!hadamard) {
    const uint4* Trow = reinterpret_cast<const uint4*>(a.t_k + ((size_t)h * kHeadDim + r) * kHeadDim);
#pragma unroll
    for (int i = 0; i < kHeadDim / 8; ++i) tr[i] = Trow[i];
  }
  for (int t = 0; t < a.n_new; ++t) {
    const int p = S + t;
    const size_t src = (((size_t)b * a.n_new + t) * a.Hkv + h) * kHeadDim;
    __half* kdst;
    __half* vdst;
    if (p < a.s_sink) {
      kdst = a.k_sink + ((size_t)unit * a.sink_dim + p) * kHeadDim;
      vdst = a.v_sink + ((size_t)unit * a.sink_dim + p) * kHeadDim;
    } else {
      kdst = a.k_ring + ((size_t)unit * a.R + p % a.R) * kHeadDim;
      vdst = a.v_ring + ((size_t)unit * a.R + p % a.R) * kHeadDim;
    }
    ks[r] = __half2float(a.k_new[src + r]);
    if (r < kHeadDim / 8)
      reinterpret_cast<uint4*>(vdst)[r] = reinterpret_cast<const uint4*>(a.v_new + src)[r];
    if (a.prep.enabled) {  // raw key: RMSNorm + RoPE at its position, by the first warp
      bar_sync(1, 128);
      if (r < 32) prep_head_warp(ks, a.prep.k_gain, a.prep, p, r);
    }
    bar_sync(1, 128);
    if (hadamard) {
      // fast Walsh-Hadamard transform: butterflies over bits 1..16 within the warp, 32 and
      // 64 across warps through shared memory; then the 1/sqrt(128) normalisation
      float y = ks[r];
#pragma unroll
      for (int bit = 1; bit < 32; bit <<= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, y, bit);
        y = (r & bit) ? o - y : y + o;
      }
#pragma unroll
      for (int bit = 32; bit < kHeadDim; bit <<= 1) {
        hs[r] = y;
        bar_sync(1, 128);
        const float o = hs[r ^ bit];
        y = (r & bit) ? o - y : y + o;
        bar_sync(1, 128);
      }
      kdst[r] = __float2half_rn(y * 0.08838834764831845f);
    } else {
      kdst[r] = __float2half_rn(key_row(tr, ks));
    }
    bar_sync(1, 128);  // ks is rewritten by the next token
  }
}

// Small append: one 128-thread CTA per (sequence, KV head).  G > 0: the fused step
// (wushkv_step) also prepares the decode that follows (q' and its query fragments) in a
// second CTA per unit (blockIdx.y = 1), in parallel with the append and
// for every unit, including one whose append is refused (its cache is decoded as it
// stands).  Each role synchronises on its own named barrier (1: append, 2: decode
// preparation).
template <int BITS, int NSEL, int G>
__global__ void __launch_bounds__(128) append_small_kernel(const AppendArgs a) {
  const int unit = blockIdx.x;
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  if (G > 0) {
    griddep_launch();  // the decode kernel may launch now; it waits for this whole grid
    // the fused step leaves the state words to the decode kernel (defer_state), so the two
    // roles need not order their reads of them
    if (blockIdx.y == 1) {
      prepare_query<BITS, (G > 0 ? G : 1)>(a, unit, threadIdx.x);
      return;
    }
  }
  __shared__ float ks[kHeadDim];  // the token's key (fp32), for the transform
  const int r = threadIdx.x;
  // One post-RoPE token under a dense transform (a decode step): k' = T_K k needs nothing
  // from the state, so it is formed first -- thread r loads its row of T_K and the token --
  // and the state read, the flush and the stores follow.  Same arithmetic as the general
  // path below.
  const bool early = a.n_new == 1 && !a.prep.enabled && a.transform == WUSHKV_TRANSFORM_DENSE;
  float k_early = 0.f;
  uint4 v_early = make_uint4(0u, 0u, 0u, 0u);
  if (early) {
    const size_t src = ((size_t)b * a.Hkv + h) * kHeadDim;
    uint4 tr[kHeadDim / 8];
    const uint4* Trow = reinterpret_cast<const uint4*>(a.t_k + ((size_t)h * kHeadDim + r) * kHeadDim);
#pragma unroll
    for (int i = 0; i < kHeadDim / 8; ++i) tr[i] = Trow[i];
    ks[r] = __half2float(a.k_new[src + r]);
    if (r < kHeadDim / 8) v_early = reinterpret_cast<const uint4*>(a.v_new + src)[r];
    bar_sync(1, 128);
    k_early = key_row(tr, ks);
  } else if (G > 0 && threadIdx.x == 0 && a.transform == WUSHKV_TRANSFORM_DENSE) {
    // the unit's key transform into L2 while the state is read (the rows are loaded below)
    bulk_prefetch_l2(a.t_k + (size_t)h * kHeadDim * kHeadDim, kHeadDim * kHeadDim * 2);
  }
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  const bool valid = state_ok(S, Sq, a);
  const bool fits = valid && S + a.n_new <= a.cap;
  if (!valid) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusBadState);
    return;
  }
  if (!fits) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusOverflow);
    return;
  }
  // 1. the flush that closes the previous chunk (entries still in the ring)
  const FlushPlan fp = flush_plan(Sq, S, a);
  quantize_ring_range<BITS, NSEL>(a, unit, fp.lo0, fp.lo0 + fp.nf, threadIdx.x, 128);
  bar_sync(1, 128);  // ring slots are read above before new tokens may reuse them below

  // 2. the new tokens
  if (early) {  // the one formed above
    __half* kdst;
    __half* vdst;
    if (S < a.s_sink) {
      kdst = a.k_sink + ((size_t)unit * a.sink_dim + S) * kHeadDim;
      vdst = a.v_sink + ((size_t)unit * a.sink_dim + S) * kHeadDim;
    } else {
      kdst = a.k_ring + ((size_t)unit * a.R + S % a.R) * kHeadDim;
      vdst = a.v_ring + ((size_t)unit * a.R + S % a.R) * kHeadDim;
    }
    kdst[r] = __float2half_rn(k_early);
    if (r < kHeadDim / 8) reinterpret_cast<uint4*>(vdst)[r] = v_early;
  } else {
    append_tokens(a, unit, b, h, S, ks);
  }
  // 3. state (a fused step's decode kernel writes it instead, once it has read the old one)
  if (threadIdx.x == 0 && !a.defer_state) {
    a.state[2 * unit] = S + a.n_new;
    if (fp.nf) a.state[2 * unit + 1] = fp.lo0 + fp.nf;
  }
}

// ---------------------------------------------------------------------------------
// Bulk append, launch 1: quantize the ring entries covered by the flush under S + n_new.
// CTA (slice, unit): slice c takes ring positions lo0 + [16c, 16c + 16) (32 rows, K and V,
// four lanes per row), so a long ring flush is spread over many CTAs.
constexpr int kFlushSlice = 16;

template <int BITS, int NSEL>
__global__ void __launch_bounds__(128) flush_ring_kernel(const AppendArgs a) {
  const int unit = blockIdx.y;
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  if (!state_ok(S, Sq, a) || S + a.n_new > a.cap) return;
  const FlushPlan fp = flush_plan(Sq, S + a.n_new, a);
  const int p0 = fp.lo0 + kFlushSlice * blockIdx.x;
  const int p1 = min(min(fp.lo0 + fp.nf, S), p0 + kFlushSlice);
  quantize_ring_range<BITS, NSEL>(a, unit, p0, p1);
}

// Bulk append, launch 2.  CTA = (256-token slab, unit), 8 warps; per 64-token tile:
// load k / v tiles and T_K into padded shared memory, k' = k T_K^T on tensor cores
// (warp w: tile rows 16*(w%4).., output columns 64*(w/4)..), fp16 k' back into the k tile,
// then two threads per token-head row quantize it (or store it fp16).
constexpr int kBulkTile = 64;
constexpr int kBulkSlab = 256;
constexpr int kPad = 136;  // halves per padded shared row (272 bytes: conflict-free ldmatrix)
// k / v tiles are double-buffered (the next tile's copies land while this one is
// transformed and quantized); value codes of a tile are staged by 16-position group (a
// 64-token tile spans at most 5)
template <int BITS>
constexpr size_t bulk_smem() {
  return (size_t)(kHeadDim + 4 * kBulkTile) * kPad * sizeof(__half) + 5 * 16 * 16 * BITS;
}

constexpr int kBulkThreads = 256;

// RMSNorm + RoPE of one raw key row held by 16 adjacent lanes, 8 dimensions (one uint4 of
// fp16) each: lane chunk c has dimensions col = 8c .. 8c+7, whose rotation partners are
// in chunk c ^ 8 (dimension +-64).
__device__ __forceinline__ uint4 prep_chunk16(uint4 raw, int col, int pos, const double* inv_freq,
                                              const PrepSpec& p) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  float x[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(u32_as_h2(w[e]));
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
  if (p.k_gain != nullptr) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(x[j], x[j], ss);
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.0f / sqrtf(ss / 128.0f + p.eps);
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = (x[j] * inv) * __half2float(p.k_gain[col + j]);
  }
  const bool first = col < 64;  // dimensions i < 64: out = x c - partner s; else x c + partner s
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    float r2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float partner = __shfl_xor_sync(0xffffffffu, x[j + u], 8);
      float c, sn;
      rope_cs(inv_freq[(col + j + u) & 63], pos, c, sn);
      r2[u] = first ? x[j + u] * c - partner * sn : x[j + u] * c + partner * sn;
    }
    o[j / 2] = h2_as_u32(__floats2half2_rn(r2[0], r2[1]));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int BITS, int NSEL, bool PREP>
__global__ void __launch_bounds__(kBulkThreads, 2) append_bulk_kernel(const AppendArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __half* Ts = reinterpret_cast<__half*>(smem_raw);
  __half* const kbuf = Ts + kHeadDim * kPad;               // [2][kBulkTile][kPad]
  __half* const vbuf = kbuf + 2 * kBulkTile * kPad;        // [2][kBulkTile][kPad]
  uint8_t* vstg = reinterpret_cast<uint8_t*>(vbuf + 2 * kBulkTile * kPad);  // value groups of the tile

  const int unit = blockIdx.y;
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  if (!state_ok(S, Sq, a) || S + a.n_new > a.cap) return;
  const FlushPlan fp = flush_plan(Sq, S + a.n_new, a);
  const int sq_new = fp.nf ? fp.lo0 + fp.nf : Sq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int CB = 16 * BITS;
  const QuantSpec qs = spec_of(a);

  // T_K -> shared (row r = output dim, col i = input dim); the Hadamard transform as its
  // exact +-1 pattern (the 1/sqrt(128) is applied to the fp32 products)
  const bool hadamard = a.transform == WUSHKV_TRANSFORM_HADAMARD;
  const float tscale = hadamard ? 0.08838834764831845f : 1.0f;
  const __half* T = a.t_k + (size_t)h * kHeadDim * kHeadDim;
  for (int c = tid; c < kHeadDim * 16; c += kBulkThreads) {
    const int r = c >> 4, col = (c & 15) * 8;
    uint4 v;
    if (hadamard) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = (__popc(r & (col + 2 * e)) & 1) ? 0xBC00u : 0x3C00u;  // -1 / +1
        const uint32_t hi = (__popc(r & (col + 2 * e + 1)) & 1) ? 0xBC00u : 0x3C00u;
        w[e] = lo | (hi << 16);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      v = *reinterpret_cast<const uint4*>(T + r * kHeadDim + col);
    }
    *reinterpret_cast<uint4*>(Ts + r * kPad + col) = v;
  }

  // raw keys (PREP): the 64 rotation frequencies, once per CTA
  __shared__ double inv_freq[PREP ? 64 : 1];
  if (PREP && tid < 64) inv_freq[tid] = rope_inv_freq(a.prep, tid);

  // tile tile0's k / v rows into buffer `buf` (16-byte asynchronous copies; rows past the
  // chunk are zero-filled); one commit group per call
  auto load_tile = [&](int tile0, int buf) {
    __half* kd = kbuf + buf * kBulkTile * kPad;
    __half* vd = vbuf + buf * kBulkTile * kPad;
    for (int c = tid; c < kBulkTile * 16; c += kBulkThreads) {
      const int r = c >> 4, col = (c & 15) * 8;
      const int t = tile0 + r;
      if (t < a.n_new) {
        const size_t src = (((size_t)b * a.n_new + t) * a.Hkv + h) * kHeadDim + col;
        cp_async16(kd + r * kPad + col, a.k_new + src);
        cp_async16(vd + r * kPad + col, a.v_new + src);
      } else {
        *reinterpret_cast<uint4*>(kd + r * kPad + col) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vd + r * kPad + col) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_commit();
  };
  const int slab0 = blockIdx.x * kBulkSlab;
  const int slab_end = min(slab0 + kBulkSlab, a.n_new);
  if (slab0 < slab_end) load_tile(slab0, 0);
  int buf = 0;
  for (int tile0 = slab0; tile0 < slab_end; tile0 += kBulkTile, buf ^= 1) {
    __syncthreads();  // previous tile fully consumed (and T_K stored on the first pass)
    __half* const ks = kbuf + buf * kBulkTile * kPad;
    const __half* const vs = vbuf + buf * kBulkTile * kPad;
    if (tile0 + kBulkTile < slab_end) {  // the next tile lands while this one is worked on
      load_tile(tile0 + kBulkTile, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();  // this tile's rows are in
    if (PREP) {  // raw keys: RMSNorm + RoPE in place, 16 lanes per row
      for (int c = tid; c < kBulkTile * 16; c += kBulkThreads) {
        const int r = c >> 4, col = (c & 15) * 8;
        uint4* kp = reinterpret_cast<uint4*>(ks + r * kPad + col);
        *kp = prep_chunk16(*kp, col, S + tile0 + r, inv_freq, a.prep);
      }
      __syncthreads();
    }

    // GEMM: warp w owns tile rows [16*mw, 16*mw+16) and output columns [64*nw, 64*nw+64)
    // (mw = w % 4, nw = w / 4): C[16][64] = K[16][128] * T^T
    {
      const int mw = warp & 3, nw = warp >> 2;
      float acc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
      const int arow = 16 * mw + (lane & 7) + 8 * ((lane >> 3) & 1);
      const int acol = 8 * (lane >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t A[4];
        ldmatrix_x4(A, ks + arow * kPad + 16 * kk + acol);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t Bm[4];
          const int brow = 64 * nw + 8 * (2 * np + (lane >> 4)) + (lane & 7);
          const int bcol = 16 * kk + 8 * ((lane >> 3) & 1);
          ldmatrix_x4(Bm, Ts + brow * kPad + bcol);
          const uint32_t b0[2] = {Bm[0], Bm[1]};
          const uint32_t b1[2] = {Bm[2], Bm[3]};
          mma_f16(acc[2 * np], A, b0);
          mma_f16(acc[2 * np + 1], A, b1);
        }
      }
      // every warp has read its rows of the k tile before any overwrites them with k'
      __syncthreads();
      const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int col = 64 * nw + 8 * nt + 2 * t4;
        *reinterpret_cast<__half2*>(ks + (16 * mw + g) * kPad + col) =
            __floats2half2_rn(acc[nt][0] * tscale, acc[nt][1] * tscale);
        *reinterpret_cast<__half2*>(ks + (16 * mw + g + 8) * kPad + col) =
            __floats2half2_rn(acc[nt][2] * tscale, acc[nt][3] * tscale);
      }
    }
    __syncthreads();

    // route: row = tid / 2 (rows 0..63 keys, 64..127 values), two threads per row
    {
      const int row = tid >> 1, part = tid & 1;
      const int kind = row >> 6;
      const int r = row & 63;
      const int t = tile0 + r;
      if (t < a.n_new) {
        const int p = S + t;
        const __half* src = (kind ? vs : ks) + r * kPad;
        if (p < a.s_sink) {
          __half* dst = (kind ? a.v_sink : a.k_sink) + ((size_t)unit * a.sink_dim + p) * kHeadDim;
          for (int i = 8 * part; i < 8 * part + 8; ++i)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
        } else if (p < sq_new) {
          const size_t rec = (size_t)unit * a.cap_alloc + p;
          // value codes into the tile's staged copy of the position's group; one call site, so
          // that the quantizer is inlined once
          uint8_t* codes = kind ? vstg + (size_t)((p >> 4) - ((S + tile0) >> 4)) * 16 * CB : a.k_codes + rec * CB;
          quantize_row_part<BITS, NSEL, 2>(src, part, codes, (kind ? a.v_params : a.k_params) + rec, qs,
                                           kind ? (p & 15) : -1);
        } else {
          __half* dst = (kind ? a.v_ring : a.k_ring) + ((size_t)unit * a.R + p % a.R) * kHeadDim;
          for (int i = 8 * part; i < 8 * part + 8; ++i)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
        }
      }
    }
    __syncthreads();

    // the staged value groups out, 16 bytes at a time (the four positions t4, t4 + 8,
    // t4 + 4, t4 + 12 of one decode lane's unit); halves of positions this tile does not
    // quantize (a group shared with another append or with the windows) are left alone
    {
      const int p_first = S + tile0, p_end = S + min(tile0 + kBulkTile, a.n_new);
      const int q_lo = max(p_first, a.s_sink), q_hi = min(p_end, sq_new);
      if (q_lo < q_hi) {
        const int g0 = p_first >> 4, ga = q_lo >> 4, gb = (q_hi - 1) >> 4;
        for (int u = tid; u < (gb - ga + 1) * CB; u += kBulkThreads) {  // CB 16-byte units per group
          const int gi = ga + u / CB, ul = u % CB;
          const int pb = 16 * gi, t4 = ul & 3;
          // halves 0..7 of the unit belong to positions pb + t4 + {0, 8, 4, 12, 0, 8, 4, 12}
          const unsigned own = (pb + t4 >= q_lo && pb + t4 < q_hi ? 0x11u : 0u) |
                               (pb + t4 + 8 >= q_lo && pb + t4 + 8 < q_hi ? 0x22u : 0u) |
                               (pb + t4 + 4 >= q_lo && pb + t4 + 4 < q_hi ? 0x44u : 0u) |
                               (pb + t4 + 12 >= q_lo && pb + t4 + 12 < q_hi ? 0x88u : 0u);
          const uint4* srcu = reinterpret_cast<const uint4*>(vstg + (size_t)(gi - g0) * 16 * CB) + ul;
          uint8_t* dstg = a.v_codes + ((size_t)unit * a.cap_alloc + pb) * CB;
          if (own == 0xFFu) {
            reinterpret_cast<uint4*>(dstg)[ul] = *srcu;
          } else {
            const uint16_t* sh = reinterpret_cast<const uint16_t*>(srcu);
            uint16_t* dh = reinterpret_cast<uint16_t*>(dstg) + 8 * ul;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              if (own & (1u << k)) dh[k] = sh[k];
          }
        }
      }
    }
  }
}

// Bulk append, launch 3.
__global__ void advance_state_kernel(const AppendArgs a) {
  const int unit = blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= a.B * a.Hkv) return;
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  if (!state_ok(S, Sq, a)) {
    atomicOr(a.status, kStatusBadState);
    return;
  }
  if (S + a.n_new > a.cap) {
    atomicOr(a.status, kStatusOverflow);
    return;
  }
  const FlushPlan fp = flush_plan(Sq, S + a.n_new, a);
  a.state[2 * unit] = S + a.n_new;
  if (fp.nf) a.state[2 * unit + 1] = fp.lo0 + fp.nf;
}

template <int BITS, int NSEL>
cudaError_t launch_append_t(const Derived& d, bool small, const AppendArgs& a, cudaStream_t st) {
  if (small) {
    append_small_kernel<BITS, NSEL, 0><<<d.units, 128, 0, st>>>(a);
    return cudaGetLastError();
  }
  // the ring holds at most R entries, so R / kFlushSlice slices cover any flush of it
  flush_ring_kernel<BITS, NSEL><<<dim3((d.ring + kFlushSlice - 1) / kFlushSlice, d.units), 128, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((a.n_new + kBulkSlab - 1) / kBulkSlab, d.units);
  if (a.prep.enabled) {
    e = ensure_smem_attr<append_bulk_kernel<BITS, NSEL, true>>((int)bulk_smem<BITS>());
    if (e != cudaSuccess) return e;
    append_bulk_kernel<BITS, NSEL, true><<<grid, kBulkThreads, bulk_smem<BITS>(), st>>>(a);
  } else {
    e = ensure_smem_attr<append_bulk_kernel<BITS, NSEL, false>>((int)bulk_smem<BITS>());
    if (e != cudaSuccess) return e;
    append_bulk_kernel<BITS, NSEL, false><<<grid, kBulkThreads, bulk_smem<BITS>(), st>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  advance_state_kernel<<<(d.units + 127) / 128, 128, 0, st>>>(a);
  return cudaGetLastError();
}

template <int BITS, int NSEL>
cudaError_t launch_fused_t(const Derived& d, const AppendArgs& a, cudaStream_t st) {
  switch (d.group) {
    case 1: append_small_kernel<BITS, NSEL, 1><<<dim3(d.units, 2), 128, 0, st>>>(a); break;
    case 2: append_small_kernel<BITS, NSEL, 2><<<dim3(d.units, 2), 128, 0, st>>>(a); break;
    case 4: append_small_kernel<BITS, NSEL, 4><<<dim3(d.units, 2), 128, 0, st>>>(a); break;
    default: append_small_kernel<BITS, NSEL, 8><<<dim3(d.units, 2), 128, 0, st>>>(a); break;
  }
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_fused_b(const Derived& d, const AppendArgs& a, cudaStream_t st) {
  switch (d.nsel) {
    case 2: return launch_fused_t<BITS, 2>(d, a, st);
    case 3: return launch_fused_t<BITS, 3>(d, a, st);
    default: return launch_fused_t<BITS, 4>(d, a, st);
  }
}

template <int BITS>
cudaError_t launch_append_b(const Derived& d, bool small, const AppendArgs& a, cudaStream_t st) {
  switch (d.nsel) {
    case 2: return launch_append_t<BITS, 2>(d, small, a, st);
    case 3: return launch_append_t<BITS, 3>(d, small, a, st);
    default: return launch_append_t<BITS, 4>(d, small, a, st);
  }
}

}  // namespace

cudaError_t launch_append(const Derived& d, int bits, bool small, const AppendArgs& a, cudaStream_t st) {
  return bits == 2 ? launch_append_b<2>(d, small, a, st) : launch_append_b<4>(d, small, a, st);
}

cudaError_t launch_append_fused(const Derived& d, int bits, const AppendArgs& a, cudaStream_t st) {
  return bits == 2 ? launch_fused_b<2>(d, a, st) : launch_fused_b<4>(d, a, st);
}

}  // namespace wushkv
