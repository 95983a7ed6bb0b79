// Calibration statistics: the per-KV-head Gram matrices of cached vectors ("WUSH-KV: KV
// Cache Quantization with Data-Adaptive Transforms": §3, the WUSH transform is built from
// the Gram matrix of the tensor being quantized; Appendix B.1, M = X X^T with one
// quantization group -- here one token's 128-vector of one head -- per column of X; §5.2,
// Setup, a calibration pass accumulates key Gram matrices after RMS normalisation and RoPE,
// and value Gram matrices, per KV head).
//
// gram[h] += sum_t x[t][h] x[t][h]^T is a dense contraction over tokens (128 x n x 128 per
// head), run on the tensor cores: mma.sync m16n8k16 with fp16 operands and fp32
// accumulation (a product of two fp16 values is exact in fp32).
//
// Work split.  A CTA takes up to kGramTokens consecutive tokens of one head.  It stages
// kGramStage tokens at a time in shared memory, transposed to [dimension][token pair], so
// that every MMA operand is a plain conflict-free 32-bit load: for a block of 16 dimensions
// and a 16-token k-step, the four words a lane loads are at once the A fragment of that
// block as an m-tile and the B fragments of its two n-tiles.  M is symmetric, so only the
// 10 blocks of 32 x 32 on and above the diagonal are computed (of 16): each of the 5 warps
// takes two blocks that share their row block.  The next stage's global loads are issued
// before the current stage's MMAs.  At the end the CTA adds its fp32 sums into the fp64
// Gram matrix with atomics, an off-diagonal block at both (i, j) and (j, i).  A CTA's fp32
// sum covers at most kGramTokens tokens, which bounds its rounding error; the fp64
// additions across CTAs come in no fixed order.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "gram.h"
#include "internal.h"
#include "ptx.cuh"

namespace wushkv {
namespace {

constexpr int kGramWarps = 5;
constexpr int kGramThreads = 32 * kGramWarps;
constexpr int kGramStage = 64;                   // tokens per shared-memory stage
constexpr int kGramPitch = kGramStage / 2 + 4;   // words per dimension row: token pairs, then 4 words of padding

// Nibble w of a table: the 32-dimension blocks of warp w.  Row block, first and second
// column block: (0; 0, 1) (0; 2, 3) (1; 1, 2) (3; 1, 3) (2; 2, 3) -- each of the 10
// unordered pairs {i, j} once.
constexpr uint32_t kRowBlock = 0x23100u, kColBlock0 = 0x21120u, kColBlock1 = 0x33231u;
__device__ __forceinline__ int nibble(uint32_t table, int w) { return (table >> (4 * w)) & 15; }

// The four fragment words of 16-dimension block `blk` at k-step `ks` of the staged tokens:
// f[0] = dims 16 blk + g, tokens 16 ks + 2 t4 (+1); f[1] = the same eight dims further;
// f[2], f[3] = the same two rows, eight tokens further.
__device__ __forceinline__ void load_frag(uint32_t (&f)[4], const uint32_t* xt, int blk, int ks, int g, int t4) {
  const uint32_t* r0 = xt + (16 * blk + g) * kGramPitch + 8 * ks + t4;
  const uint32_t* r1 = r0 + 8 * kGramPitch;
  f[0] = r0[0];
  f[1] = r1[0];
  f[2] = r0[4];
  f[3] = r1[4];
}

__global__ void __launch_bounds__(kGramThreads) gram_kernel(const uint16_t* __restrict__ x, int64_t n_tokens,
                                                           int n_heads, double* __restrict__ gram) {
  __shared__ __align__(16) uint32_t xt[kHeadDim * kGramPitch];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int h = blockIdx.y;
  const int64_t t_begin = (int64_t)blockIdx.x * kGramTokens;
  const int64_t t_end = min(n_tokens, t_begin + (int64_t)kGramTokens);
  const int bi = nibble(kRowBlock, warp);
  const int bj[2] = {nibble(kColBlock0, warp), nibble(kColBlock1, warp)};

  // Staging: warp w moves the 8-dimension chunks q = w, w + 5, w + 10, w + 15 (those below
  // 16) of the stage's tokens; lane l moves tokens 2l and 2l + 1.  Tokens past the CTA's
  // range are zeros, which add nothing.
  uint4 pre[4][2];
  auto load_stage = [&](int64_t t0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int q = warp + kGramWarps * k;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int64_t t = t0 + 2 * lane + j;
        pre[k][j] = make_uint4(0u, 0u, 0u, 0u);
        if (q < 16 && t < t_end)
          pre[k][j] = __ldg(reinterpret_cast<const uint4*>(x + (t * n_heads + h) * kHeadDim + 8 * q));
      }
    }
  };
  auto store_stage = [&]() {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int q = warp + kGramWarps * k;
      if (q < 16) {
        const uint32_t a[4] = {pre[k][0].x, pre[k][0].y, pre[k][0].z, pre[k][0].w};
        const uint32_t b[4] = {pre[k][1].x, pre[k][1].y, pre[k][1].z, pre[k][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {  // dimension 8q + e: token 2l in the low half, 2l + 1 in the high
          const uint32_t lo = a[e >> 1], hi = b[e >> 1];
          xt[(8 * q + e) * kGramPitch + lane] =
              (e & 1) ? ((lo >> 16) | (hi & 0xffff0000u)) : ((lo & 0xffffu) | (hi << 16));
        }
      }
    }
  };

  float acc[2][2][4][4];  // [column block][m-tile][n-tile][C fragment]
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[s][mt][nt][i] = 0.f;

  int64_t t0 = t_begin;
  load_stage(t0);
  for (;;) {
    __syncthreads();  // every warp has read the previous stage
    store_stage();
    __syncthreads();
    const int64_t tn = t0 + kGramStage;
    if (tn < t_end) load_stage(tn);  // in flight during this stage's MMAs
#pragma unroll
    for (int ks = 0; ks < kGramStage / 16; ++ks) {
      uint32_t fa[2][4];
      load_frag(fa[0], xt, 2 * bi, ks, g, t4);
      load_frag(fa[1], xt, 2 * bi + 1, ks, g, t4);
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        uint32_t fb[2][4];
        load_frag(fb[0], xt, 2 * bj[s], ks, g, t4);
        load_frag(fb[1], xt, 2 * bj[s] + 1, ks, g, t4);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const uint32_t b[2] = {fb[nt >> 1][nt & 1], fb[nt >> 1][(nt & 1) + 2]};
            mma_f16(acc[s][mt][nt], fa[mt], b);
          }
      }
    }
    t0 = tn;
    if (t0 >= t_end) break;
  }

  double* G = gram + (size_t)h * kHeadDim * kHeadDim;
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = 32 * bi + 16 * mt + g + 8 * (i >> 1);
          const int col = 32 * bj[s] + 8 * nt + 2 * t4 + (i & 1);
          const double v = acc[s][mt][nt][i];
          atomicAdd(G + row * kHeadDim + col, v);
          if (bi != bj[s]) atomicAdd(G + col * kHeadDim + row, v);
        }
}

}  // namespace

cudaError_t launch_gram(const uint16_t* x, int64_t n_tokens, int n_heads, double* gram, cudaStream_t st) {
  const int64_t chunks = (n_tokens + kGramTokens - 1) / kGramTokens;
  gram_kernel<<<dim3((unsigned)chunks, (unsigned)n_heads), kGramThreads, 0, st>>>(x, n_tokens, n_heads, gram);
  return cudaGetLastError();
}

}  // namespace wushkv
