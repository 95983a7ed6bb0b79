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
// Work split.  A CTA takes a run of at most kGramTokens consecutive tokens of one head; the
// run length is chosen so that the grid fills two CTAs per SM when the input allows.  The
// tokens arrive 64 at a time through a cp.async ring of kGramStages slots, stored as they
// are in memory (one 256-byte row per token, padded to 272 bytes so that ldmatrix reads
// are conflict-free).  ldmatrix.trans turns 16 tokens x 16 dimensions into the four words
// that are at once the A fragment of that dimension block and the B fragments of its two
// n-tiles.  M is symmetric, so only the 10 blocks of 32 x 32 on and above the diagonal are
// computed (of 16): each of 5 warps takes two blocks that share their row block, and two
// such groups of 5 warps take alternate halves of every stage's k-steps.  At the end the
// two groups add their sums through shared memory, and the CTA adds its fp32 sums into the
// fp64 Gram matrix with atomics, an off-diagonal block at both (i, j) and (j, i).  A CTA's
// fp32 sum covers at most kGramTokens tokens, which bounds its rounding error; the fp64
// additions across CTAs come in no fixed order.
#include <algorithm>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "gram.h"
#include "internal.h"
#include "ptx.cuh"

namespace wushkv {
namespace {

constexpr int kGramGroupWarps = 5;                    // one warp per pair of 32 x 32 blocks
constexpr int kGramGroupThreads = 32 * kGramGroupWarps;
constexpr int kGramThreads = 2 * kGramGroupThreads;   // two groups: k-steps {0, 1} and {2, 3} of a stage
constexpr int kGramStage = 64;                        // tokens per stage
constexpr int kGramStages = 3;                        // cp.async ring slots
constexpr int kGramRowBytes = 272;                    // one token's 256 bytes + 16 bytes of padding
constexpr int kGramSlotBytes = kGramStage * kGramRowBytes;
constexpr int kGramSmem = kGramStages * kGramSlotBytes;
static_assert(2 * 32 * kGramGroupThreads * 4 <= kGramSmem, "the group exchange reuses the ring");

// Nibble w of a table: the 32-dimension blocks of warp w of a group.  Row block, first and
// second column block: (0; 0, 1) (0; 2, 3) (1; 1, 2) (3; 1, 3) (2; 2, 3) -- each of the 10
// unordered pairs {i, j} once.
constexpr uint32_t kRowBlock = 0x23100u, kColBlock0 = 0x21120u, kColBlock1 = 0x33231u;
__device__ __forceinline__ int nibble(uint32_t table, int w) { return (table >> (4 * w)) & 15; }

// Four transposed 8 x 8 fp16 matrices: lanes 8m .. 8m + 7 give the row addresses of matrix m,
// and lane (g, t4) receives rows 2 t4, 2 t4 + 1 of column g of each.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kGramThreads, 2)
    gram_kernel(const uint16_t* __restrict__ x, int64_t n_tokens, int n_heads, int64_t cta_tokens,
                double* __restrict__ gram) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int grp = warp / kGramGroupWarps, wg = warp % kGramGroupWarps;
  const int h = blockIdx.y;
  const int64_t t_begin = (int64_t)blockIdx.x * cta_tokens;
  const int64_t t_end = min(n_tokens, t_begin + cta_tokens);
  const int n_stages = (int)((t_end - t_begin + kGramStage - 1) / kGramStage);
  const int bi = nibble(kRowBlock, wg);
  const int bj0 = nibble(kColBlock0, wg), bj1 = nibble(kColBlock1, wg);
  const uint32_t smem0 = smem_u32(smem);

  // Stage s (tokens t_begin + 64 s ...) into ring slot s % kGramStages: 16-byte copies, one
  // token row per 16 threads.  Rows past the run are zero-filled, so they add nothing.  One
  // commit group per call, empty past the last stage.
  auto issue_stage = [&](int s) {
    if (s < n_stages) {
      uint8_t* slot = smem + (s % kGramStages) * kGramSlotBytes;
      const int64_t t0 = t_begin + (int64_t)s * kGramStage;
      for (int i = tid; i < kGramStage * 16; i += kGramThreads) {
        const int r = i >> 4, c = i & 15;
        const int64_t t = t0 + r;
        uint8_t* dst = slot + r * kGramRowBytes + 16 * c;
        if (t < t_end)
          cp_async16(dst, x + (t * n_heads + h) * kHeadDim + 8 * c);
        else
          *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
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

#pragma unroll
  for (int s = 0; s < kGramStages - 1; ++s) issue_stage(s);

  // ldmatrix row address of this lane within a slot: token 16 ks + (lane & 7) + 8 (lane >> 4),
  // dimensions + 8 ((lane >> 3) & 1): matrices 0..3 are (tokens +0, dims +0), (+0, +8),
  // (+8, +0), (+8, +8) of a 16 x 16 block, i.e. fragment words f[0] .. f[3].
  const uint32_t lane_off = ((lane & 7) + 8 * (lane >> 4)) * kGramRowBytes + 16 * ((lane >> 3) & 1);
  for (int s = 0; s < n_stages; ++s) {
    cp_async_wait_group<kGramStages - 2>();  // this thread's copies of stage s have landed
    __syncthreads();                          // everyone's have; everyone is done with stage s - 1
    issue_stage(s + kGramStages - 1);         // into the slot stage s - 1 used
    const uint32_t slot = smem0 + (s % kGramStages) * kGramSlotBytes + lane_off;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const uint32_t rows = slot + (16 * (2 * grp + kk)) * kGramRowBytes;
      uint32_t fa[2][4];
      ldsm_x4_trans(fa[0], rows + 32 * (2 * bi));
      ldsm_x4_trans(fa[1], rows + 32 * (2 * bi + 1));
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const int bj = cb ? bj1 : bj0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t fb[4];
          ldsm_x4_trans(fb, rows + 32 * (2 * bj + half));
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int n2 = 0; n2 < 2; ++n2) {
              const uint32_t b[2] = {fb[n2], fb[n2 + 2]};
              mma_f16(acc[cb][mt][2 * half + n2], fa[mt], b);
            }
        }
      }
    }
  }

  // The two groups add their sums: group 0 finishes column block 0, group 1 column block 1.
  cp_async_wait_group<0>();
  __syncthreads();  // the ring is free
  float* xch = reinterpret_cast<float*>(smem);  // [2][32][kGramGroupThreads]: block handed over
  const int gt = tid % kGramGroupThreads;
  auto put = [&](const float (&a)[2][4][4], int which) {
#pragma unroll
    for (int e = 0; e < 32; ++e) xch[(which * 32 + e) * kGramGroupThreads + gt] = a[e >> 4][(e >> 2) & 3][e & 3];
  };
  auto take = [&](float (&a)[2][4][4], int which) {
#pragma unroll
    for (int e = 0; e < 32; ++e) a[e >> 4][(e >> 2) & 3][e & 3] += xch[(which * 32 + e) * kGramGroupThreads + gt];
  };
  if (grp == 0)
    put(acc[1], 1);
  else
    put(acc[0], 0);
  __syncthreads();
  double* G = gram + (size_t)h * kHeadDim * kHeadDim;
  auto flush = [&](const float (&a)[2][4][4], int bj) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = 32 * bi + 16 * mt + g + 8 * (i >> 1);
          const int col = 32 * bj + 8 * nt + 2 * t4 + (i & 1);
          const double v = a[mt][nt][i];
          atomicAdd(G + row * kHeadDim + col, v);
          if (bi != bj) atomicAdd(G + col * kHeadDim + row, v);
        }
  };
  if (grp == 0) {
    take(acc[0], 0);
    flush(acc[0], bj0);
  } else {
    take(acc[1], 1);
    flush(acc[1], bj1);
  }
}

}  // namespace

cudaError_t launch_gram(const uint16_t* x, int64_t n_tokens, int n_heads, double* gram, cudaStream_t st) {
  // Runs per head for two CTAs per SM, each a whole number of stages and at most kGramTokens.
  const int64_t runs = std::max<int64_t>(1, (2 * kB200SMs + n_heads - 1) / n_heads);
  int64_t cta_tokens = (n_tokens + runs - 1) / runs;
  cta_tokens = (cta_tokens + kGramStage - 1) / kGramStage * kGramStage;
  cta_tokens = std::min<int64_t>(std::max<int64_t>(cta_tokens, kGramStage), kGramTokens);
  const int64_t chunks = (n_tokens + cta_tokens - 1) / cta_tokens;
  const cudaError_t e = ensure_smem_attr<gram_kernel>(kGramSmem);
  if (e != cudaSuccess) return e;
  gram_kernel<<<dim3((unsigned)chunks, (unsigned)n_heads), kGramThreads, kGramSmem, st>>>(x, n_tokens, n_heads,
                                                                                        cta_tokens, gram);
  return cudaGetLastError();
}

}  // namespace wushkv
