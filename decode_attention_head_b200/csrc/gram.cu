// Calibration statistics: the per-KV-head Gram matrices of cached vectors ("WUSH-KV: KV
// Cache Quantization with Data-Adaptive Transforms": §3, the WUSH transform is built from
// the Gram matrix of the tensor being quantized; Appendix B.1, M = X X^T with one
// quantization group -- here one token's 128-vector of one head -- per column of X; §5.2,
// Setup, a calibration pass accumulates key Gram matrices after RMS normalisation and RoPE,
// and value Gram matrices, per KV head).
//
// gram[h] += sum_t x[t][h] x[t][h]^T is a dense contraction over tokens (128 x n x 128 per
// head), run on the fifth-generation tensor cores: tcgen05.mma kind::f16, M = N = 128
// dimensions, K = 16 tokens per instruction, fp16 operands, the whole 128 x 128 fp32 sum in
// tensor memory (128 lanes x 128 columns).  A product of two fp16 values is exact in fp32.
//
// Both operands are the same shared-memory tile: with tokens as the K mode and dimensions
// as the M (or N) mode, a token's row of 128 dimensions is an MN-major operand row, so no
// transposition is needed.  The tile is stored in the canonical MN-major 128-byte-swizzled
// layout: dimensions 0..63 and 64..127 in two regions of [tokens][128 bytes], the 16-byte
// chunk c of token t at chunk c ^ (t % 8) of its row.  One descriptor serves as A and as B.
//
// Work split.  A CTA takes a run of at most kGramTokens consecutive tokens of one head; the
// run length is chosen so that the grid fills two CTAs per SM when the input allows.  The
// tokens arrive 64 at a time through a ring of kGramStages slots, each filled by two TMA
// tile copies (a 3-D tensor map over [tokens][heads][128 dims], boxes of 64 dimensions x 1
// head x 64 tokens, 128-byte swizzle: the copies write the MN-major layout above, and zero
// past the last token).  One thread issues the copies, another the four MMAs of a slot,
// which it commits to the slot's mbarrier; the slot is refilled only once they have read
// it.  At the end the four warps read the sum back from tensor memory (warp w: rows
// 32 w .. 32 w + 31) into a shared-memory tile and add it into the fp64 Gram matrix with
// atomics, row by row with consecutive columns across a warp's lanes (coalesced): the entry
// (i, j), i <= j, at both (i, j) and (j, i), the same value at both.  A CTA's fp32
// sum covers at most kGramTokens tokens, which bounds its rounding error; the fp64 additions
// across CTAs come in no fixed order.
#include <algorithm>
#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched through the runtime)
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "gram.h"
#include "internal.h"
#include "ptx.cuh"

namespace wushkv {
namespace {

constexpr int kGramThreads = 128;                 // four warps: copies, MMA issue, read-back
constexpr int kGramStage = 64;                    // tokens per stage (four MMAs of K = 16)
constexpr int kGramStages = 4;                    // ring slots
constexpr int kGramRegion = kGramStage * 128;     // bytes of one 64-dimension half of a slot
constexpr int kGramSlotBytes = 2 * kGramRegion;   // 16 KB
constexpr int kGramPitch = kHeadDim + 1;         // floats per row of the read-back tile (no bank conflicts)
static_assert(kHeadDim * kGramPitch * 4 <= kGramStages * kGramSlotBytes + 2048, "the read-back tile fits");
constexpr int kGramSmem = kGramStages * kGramSlotBytes + 1024 + 2048;  // + room to align to 1024, + tile pitch
constexpr uint32_t kGramTmemCols = 128;

// kind::f16 with an fp32 accumulator, A and B fp16 and MN-major, M = N = 128.
constexpr uint32_t kGramIdesc = (1u << 4) | (0u << 7) | (0u << 10) | (1u << 15) | (1u << 16) |
                                ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

// D (tensor memory) [+]= A x B with both operands from shared memory; one thread.
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// MN-major, 128-byte-swizzle descriptor of 16 tokens starting at `saddr` (1024-byte aligned):
// 8-token groups 1024 bytes apart, the two 64-dimension regions kGramRegion bytes apart.
__device__ __forceinline__ uint64_t gram_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((kGramRegion >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((1024 >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// 32 consecutive columns of this thread's tensor-memory lane, waited for inside the same
// statement (so that no use of r can be scheduled before the data is there).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// One 3-D TMA tile copy (no multicast) into shared memory, completing on an mbarrier:
// coordinates (dimension, head, token) of the box's first element.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kGramThreads)
    gram_kernel(const __grid_constant__ CUtensorMap map, int64_t n_tokens, int64_t cta_tokens,
                double* __restrict__ gram) {
  extern __shared__ uint8_t smem_raw[];
  // the swizzle pattern repeats every 1024 bytes: slots start on such a boundary
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[kGramStages];  // a slot's tokens have landed
  __shared__ __align__(8) uint64_t done[kGramStages];  // the MMAs that read a slot have completed
  __shared__ uint32_t s_taddr;
  __shared__ uint32_t s_status;  // the Gram call has no status word: a wait that gives up (a library bug) lands here
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int64_t t_begin = (int64_t)blockIdx.x * cta_tokens;
  const int64_t t_end = min(n_tokens, t_begin + cta_tokens);
  const int n_stages = (int)((t_end - t_begin + kGramStage - 1) / kGramStage);

  if (tid == 0) {
    for (int s = 0; s < kGramStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_taddr, kGramTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = s_taddr;

  if (tid == 0) {
    // producer: stage u (tokens t_begin + 64 u ...) into slot u % kGramStages once the MMAs
    // of stage u - kGramStages (the slot's previous user) have read it.  Tokens past the
    // run belong to the next CTA only where the run is a whole number of stages, so a
    // partial stage exists only at the tensor's end, where the copy fills zeros.
    int issued = 0;
    for (int u = 0; u < n_stages; ++u) {
      const int slot = u % kGramStages;
      if (u >= kGramStages && !mbar_wait(&done[slot], ((u / kGramStages) - 1) & 1, &s_status)) break;
      uint8_t* base = smem + slot * kGramSlotBytes;
      const int z = (int)(t_begin + (int64_t)u * kGramStage);
      mbar_expect_tx(&full[slot], kGramSlotBytes);
      tma_load_3d(base, &map, 0, h, z, &full[slot]);
      tma_load_3d(base + kGramRegion, &map, 64, h, z, &full[slot]);
      issued = u + 1;
    }
    // every issued copy has landed before the CTA may leave (they are plain reads of x)
    for (int u = max(0, issued - kGramStages); u < issued; ++u)
      mbar_wait(&full[u % kGramStages], (u / kGramStages) & 1, &s_status);
  } else if (tid == 32) {
    // MMA issue: four K = 16 slices of each slot, committed to the slot's `done`
    const uint32_t smem0 = smem_u32(smem);
    for (int s = 0; s < n_stages; ++s) {
      const int slot = s % kGramStages;
      if (!mbar_wait(&full[slot], (s / kGramStages) & 1, &s_status)) break;
      tc_fence_after();
      const uint32_t a = smem0 + slot * kGramSlotBytes;
#pragma unroll
      for (int j = 0; j < kGramStage / 16; ++j) {
        const uint64_t d = gram_desc(a + j * 16 * 128);
        mma_f16_ss(tbase, d, d, kGramIdesc, (s > 0 || j > 0) ? 1u : 0u);
      }
      mma_commit(&done[slot]);
    }
  }
  // every MMA complete (the last commit covers all of them; the MMA thread waits for it --
  // a thread that had not followed the barrier's phases could not), then the sum leaves
  // tensor memory into a [128][129] fp32 tile over the drained slots (warp w: rows 32 w ..
  // 32 w + 31)
  if (tid == 32 && n_stages > 0)
    mbar_wait(&done[(n_stages - 1) % kGramStages], ((n_stages - 1) / kGramStages) & 1, &s_status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  float* tile = reinterpret_cast<float*>(smem);
  const int i = 32 * warp + lane;  // this thread's row (tensor-memory lane)
#pragma unroll 1
  for (int c = 0; c < kHeadDim / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + ((uint32_t)(32 * warp) << 16) + 32 * c, r);
#pragma unroll
    for (int k = 0; k < 32; ++k) tile[i * kGramPitch + 32 * c + k] = __uint_as_float(r[k]);
  }
  tc_fence_before();
  __syncthreads();
  // G[r][c] += the CTA's (min(r, c), max(r, c)) entry, the same value at (r, c) and (c, r): a warp
  // takes a row, its lanes 32 consecutive columns, so every fp64 atomic instruction covers
  // 256 contiguous bytes
  // (the CTAs of a head start at different rows, so that they do not all add into the same
  // lines at the same time)
  double* G = gram + (size_t)h * kHeadDim * kHeadDim;
  const int shift = (int)((blockIdx.x * 8u) & (kHeadDim - 1));
#pragma unroll 1
  for (int r0 = warp; r0 < kHeadDim; r0 += kGramThreads / 32) {
    const int row = (r0 + shift) & (kHeadDim - 1);
#pragma unroll
    for (int q = 0; q < kHeadDim / 32; ++q) {
      const int col = 32 * q + lane;
      const float v = col >= row ? tile[row * kGramPitch + col] : tile[col * kGramPitch + row];
      atomicAdd(G + row * kHeadDim + col, (double)v);
    }
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kGramTmemCols);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's cuTensorMapEncodeTiled, fetched through the runtime (no link against libcuda).
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace

cudaError_t launch_gram(const uint16_t* x, int64_t n_tokens, int n_heads, double* gram, cudaStream_t st) {
  const EncodeTiledFn encode = encode_tiled();
  if (!encode) return cudaErrorNotSupported;
  cudaError_t e = ensure_smem_attr<gram_kernel>(kGramSmem);
  if (e != cudaSuccess) return e;
  // windows of at most 2^30 tokens (a tensor map's token coordinate is a 32-bit integer)
  constexpr int64_t kWindow = int64_t(1) << 30;
  for (int64_t w0 = 0; w0 < n_tokens; w0 += kWindow) {
    const int64_t nw = std::min(kWindow, n_tokens - w0);
    // runs per head for two CTAs per SM, each a whole number of stages and at most kGramTokens
    const int64_t runs = std::max<int64_t>(1, (2 * kB200SMs + n_heads - 1) / n_heads);
    int64_t cta_tokens = (nw + runs - 1) / runs;
    cta_tokens = (cta_tokens + kGramStage - 1) / kGramStage * kGramStage;
    cta_tokens = std::min<int64_t>(std::max<int64_t>(cta_tokens, kGramStage), kGramTokens);
    const int64_t chunks = (nw + cta_tokens - 1) / cta_tokens;
    // [tokens][heads][128] fp16: dimension fastest, then head, then token
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)n_heads, (cuuint64_t)nw};
    const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)n_heads * kHeadDim * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kGramStage};
    const cuuint32_t estrides[3] = {1, 1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
               const_cast<uint16_t*>(x + w0 * n_heads * kHeadDim), dims, strides, box, estrides,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    gram_kernel<<<dim3((unsigned)chunks, (unsigned)n_heads), kGramThreads, kGramSmem, st>>>(map, nw, cta_tokens,
                                                                                          gram);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace wushkv
