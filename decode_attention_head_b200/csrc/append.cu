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

namespace wushkv {
namespace {

struct FlushPlan {
  int lo0, nf;
};

__device__ __forceinline__ FlushPlan flush_plan(int Sq, int L, const AppendArgs& a) {
  FlushPlan f;
  f.lo0 = max(Sq, a.s_sink);
  const int e = L - a.s_keep - f.lo0;
  f.nf = (e >= a.s_flush) ? (e / a.s_flush) * a.s_flush : 0;
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
  return q;
}

// Quantize ring positions [p_begin, p_end) of `unit` (K and V), threads of the CTA in turn.
template <int BITS, int NSEL>
__device__ void quantize_ring_range(const AppendArgs& a, int unit, int p_begin, int p_end) {
  const int n = p_end - p_begin;
  if (n <= 0) return;
  constexpr int CB = 16 * BITS;
  const QuantSpec qs = spec_of(a);
  for (int item = threadIdx.x; item < 2 * n; item += blockDim.x) {
    const int kind = item / n;  // 0 = K, 1 = V
    const int p = p_begin + item % n;
    const __half* ring = kind ? a.v_ring : a.k_ring;
    const __half* row = ring + ((size_t)unit * a.R + (p % a.R)) * kHeadDim;
    const size_t rec = (size_t)unit * a.cap_alloc + p;
    uint8_t* codes = (kind ? a.v_codes : a.k_codes) + rec * CB;
    uint32_t* params = (kind ? a.v_params : a.k_params) + rec;
    quantize_row<BITS, NSEL>(row, codes, params, qs);
  }
}

// ---------------------------------------------------------------------------------
// Small append: one CTA (128 threads) per (sequence, KV head).
template <int BITS, int NSEL>
__global__ void __launch_bounds__(128) append_small_kernel(const AppendArgs a) {
  const int unit = blockIdx.x;
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  if (!state_ok(S, Sq, a)) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusBadState);
    return;
  }
  if (S + a.n_new > a.cap) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusOverflow);
    return;
  }
  // 1. the flush that closes the previous chunk (entries still in the ring)
  const FlushPlan fp = flush_plan(Sq, S, a);
  quantize_ring_range<BITS, NSEL>(a, unit, fp.lo0, fp.lo0 + fp.nf);
  __syncthreads();  // ring slots are read above before new tokens may reuse them below

  // 2. new tokens: k' = fp16_rn(T_K k) (fp32 accumulation), v as given
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __half* T = a.t_k + (size_t)h * kHeadDim * kHeadDim;
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
    // lane holds k[4*lane .. 4*lane+3]
    const uint2 kraw = *reinterpret_cast<const uint2*>(a.k_new + src + 4 * lane);
    const float2 k01 = __half22float2(u32_as_h2(kraw.x));
    const float2 k23 = __half22float2(u32_as_h2(kraw.y));
    float mine = 0.f;
    for (int j = 0; j < 32; ++j) {
      const int r = 32 * warp + j;
      const uint2 traw = *reinterpret_cast<const uint2*>(T + (size_t)r * kHeadDim + 4 * lane);
      const float2 t01 = __half22float2(u32_as_h2(traw.x));
      const float2 t23 = __half22float2(u32_as_h2(traw.y));
      float acc = t01.x * k01.x;
      acc = fmaf(t01.y, k01.y, acc);
      acc = fmaf(t23.x, k23.x, acc);
      acc = fmaf(t23.y, k23.y, acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == j) mine = acc;
    }
    kdst[32 * warp + lane] = __float2half_rn(mine);
    if (threadIdx.x < 32) {
      reinterpret_cast<uint2*>(vdst)[threadIdx.x] = reinterpret_cast<const uint2*>(a.v_new + src)[threadIdx.x];
    }
  }
  __syncthreads();
  // 3. state
  if (threadIdx.x == 0) {
    a.state[2 * unit] = S + a.n_new;
    if (fp.nf) a.state[2 * unit + 1] = fp.lo0 + fp.nf;
  }
}

// ---------------------------------------------------------------------------------
// Bulk append, launch 1: quantize the ring entries covered by the flush under S + n_new.
template <int BITS, int NSEL>
__global__ void __launch_bounds__(128) flush_ring_kernel(const AppendArgs a) {
  const int unit = blockIdx.x;
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  if (!state_ok(S, Sq, a) || S + a.n_new > a.cap) return;
  const FlushPlan fp = flush_plan(Sq, S + a.n_new, a);
  quantize_ring_range<BITS, NSEL>(a, unit, fp.lo0, min(fp.lo0 + fp.nf, S));
}

// Bulk append, launch 2.  CTA = (256-token slab, unit), 4 warps; per 64-token tile:
// load k / v tiles and T_K into padded shared memory, k' = k T_K^T on tensor cores,
// fp16 k' back into the k tile, then one thread per token-head quantizes or stores.
constexpr int kBulkTile = 64;
constexpr int kBulkSlab = 256;
constexpr int kPad = 136;  // halves per padded shared row (272 bytes: conflict-free ldmatrix)
constexpr size_t kBulkSmem = (size_t)(kHeadDim + 2 * kBulkTile) * kPad * sizeof(__half);

template <int BITS, int NSEL>
__global__ void __launch_bounds__(128) append_bulk_kernel(const AppendArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __half* Ts = reinterpret_cast<__half*>(smem_raw);
  __half* ks = Ts + kHeadDim * kPad;
  __half* vs = ks + kBulkTile * kPad;

  const int unit = blockIdx.y;
  const int b = unit / a.Hkv, h = unit % a.Hkv;
  const int S = a.state[2 * unit], Sq = a.state[2 * unit + 1];
  if (!state_ok(S, Sq, a) || S + a.n_new > a.cap) return;
  const FlushPlan fp = flush_plan(Sq, S + a.n_new, a);
  const int sq_new = fp.nf ? fp.lo0 + fp.nf : Sq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int CB = 16 * BITS;
  const QuantSpec qs = spec_of(a);

  // T_K -> shared (row r = output dim, col i = input dim)
  const __half* T = a.t_k + (size_t)h * kHeadDim * kHeadDim;
  for (int c = tid; c < kHeadDim * 16; c += 128) {
    const int r = c >> 4, col = (c & 15) * 8;
    *reinterpret_cast<uint4*>(Ts + r * kPad + col) = *reinterpret_cast<const uint4*>(T + r * kHeadDim + col);
  }

  const int slab0 = blockIdx.x * kBulkSlab;
  for (int tile0 = slab0; tile0 < min(slab0 + kBulkSlab, a.n_new); tile0 += kBulkTile) {
    __syncthreads();  // previous tile fully consumed (and T_K stored on the first pass)
    for (int c = tid; c < kBulkTile * 16; c += 128) {
      const int r = c >> 4, col = (c & 15) * 8;
      const int t = tile0 + r;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (t < a.n_new) {
        const size_t src = (((size_t)b * a.n_new + t) * a.Hkv + h) * kHeadDim + col;
        kv = *reinterpret_cast<const uint4*>(a.k_new + src);
        vv = *reinterpret_cast<const uint4*>(a.v_new + src);
      }
      *reinterpret_cast<uint4*>(ks + r * kPad + col) = kv;
      *reinterpret_cast<uint4*>(vs + r * kPad + col) = vv;
    }
    __syncthreads();

    // GEMM: warp w owns tile rows [16w, 16w+16): C[16][128] = K[16][128] * T^T
    {
      float acc[16][4];
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
      const int arow = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
      const int acol = 8 * (lane >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t A[4];
        ldmatrix_x4(A, ks + arow * kPad + 16 * kk + acol);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          uint32_t Bm[4];
          const int brow = 8 * (2 * np + (lane >> 4)) + (lane & 7);
          const int bcol = 16 * kk + 8 * ((lane >> 3) & 1);
          ldmatrix_x4(Bm, Ts + brow * kPad + bcol);
          const uint32_t b0[2] = {Bm[0], Bm[1]};
          const uint32_t b1[2] = {Bm[2], Bm[3]};
          mma_f16(acc[2 * np], A, b0);
          mma_f16(acc[2 * np + 1], A, b1);
        }
      }
      __syncwarp();
      const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int col = 8 * nt + 2 * t4;
        *reinterpret_cast<__half2*>(ks + (16 * warp + g) * kPad + col) = __floats2half2_rn(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<__half2*>(ks + (16 * warp + g + 8) * kPad + col) =
            __floats2half2_rn(acc[nt][2], acc[nt][3]);
      }
    }
    __syncthreads();

    // route: threads 0..63 keys, 64..127 values
    {
      const int kind = tid >> 6;
      const int r = tid & 63;
      const int t = tile0 + r;
      if (t < a.n_new) {
        const int p = S + t;
        const __half* row = (kind ? vs : ks) + r * kPad;
        if (p < a.s_sink) {
          __half* dst = (kind ? a.v_sink : a.k_sink) + ((size_t)unit * a.sink_dim + p) * kHeadDim;
          for (int i = 0; i < 16; ++i)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(row)[i];
        } else if (p < sq_new) {
          const size_t rec = (size_t)unit * a.cap_alloc + p;
          quantize_row<BITS, NSEL>(row, (kind ? a.v_codes : a.k_codes) + rec * CB,
                                   (kind ? a.v_params : a.k_params) + rec, qs);
        } else {
          __half* dst = (kind ? a.v_ring : a.k_ring) + ((size_t)unit * a.R + p % a.R) * kHeadDim;
          for (int i = 0; i < 16; ++i)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(row)[i];
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
    append_small_kernel<BITS, NSEL><<<d.units, 128, 0, st>>>(a);
    return cudaGetLastError();
  }
  flush_ring_kernel<BITS, NSEL><<<d.units, 128, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr<append_bulk_kernel<BITS, NSEL>>((int)kBulkSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.n_new + kBulkSlab - 1) / kBulkSlab, d.units);
  append_bulk_kernel<BITS, NSEL><<<grid, 128, kBulkSmem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  advance_state_kernel<<<(d.units + 127) / 128, 128, 0, st>>>(a);
  return cudaGetLastError();
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

}  // namespace wushkv
