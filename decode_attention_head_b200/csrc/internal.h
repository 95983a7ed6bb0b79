// Internal interfaces between the C-ABI layer (abi.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include "../../include/wushkv.h"
#include "prep.cuh"

namespace wushkv {

constexpr int kHeadDim = 128;
constexpr int kTileTokens = 128;      // positions per decode pipeline stage (and cap_alloc granule)
constexpr int kB200SMs = 148;         // split policy sizes the decode grid for this many SMs
// Resident decode CTAs per SM the split policy aims at (the kernel's launch bounds hold its
// registers to this): 8 query heads per KV head need more registers than the others.
constexpr int decode_ctas_per_sm(int group) { return group == 8 ? 3 : 4; }
constexpr int kMaxSplits = 128;       // work items per (sequence, KV head): at most 16 clusters of 8

struct Derived {
  int units;        // B * H_kv
  int group;        // H_q / H_kv
  int cap_alloc;    // capacity rounded up to 128
  int ring;         // ring slots
  int sink_dim;     // max(s_sink, 1)
  int code_bytes;   // 16 * bits
  int nsel;         // extreme order statistics the quantizer keeps (2..4)
  int i_lo, i_hi;
  float f_lo, f_hi;
  int n_split, split_tokens;
  int cluster;      // decode CTAs per thread-block cluster (consecutive items of a unit; divides n_split)
  int interleave;   // 1: the decode grid's consecutive clusters belong to different units
  // workspace offsets (bytes)
  size_t ws_tickets, ws_qprime, ws_qfrag, ws_partials, ws_total;
  // cache buffer sizes (bytes)
  size_t codes_bytes, params_bytes, sink_bytes, ring_bytes, state_bytes;
};

// Validates cfg and fills d; returns WUSHKV_OK / WUSHKV_EINVAL / WUSHKV_EUNSUPPORTED.
// ticket_units: completion counters to reserve at the start of the workspace (-1: those
// of cfg's own largest chunk-attention launch, which every layout of cfg reserves alike).
int derive(const wushkv_config* cfg, Derived* d, long long ticket_units = -1);

// The flush under length L of a (sequence, KV head) whose quantized region ends at Sq:
// lo0 = max(Sq, S_sink); e = L - S_keep - lo0; e >= S_flush -> nf = floor(e / S_flush) *
// S_flush positions [lo0, lo0 + nf) are quantized and S_quant moves to lo0 + nf (else nf = 0).
__host__ __device__ __forceinline__ void flush_bounds(int Sq, int L, int s_sink, int s_keep, int s_flush, int& lo0,
                                                     int& nf) {
  lo0 = Sq > s_sink ? Sq : s_sink;
  const int e = L - s_keep - lo0;
  nf = (e >= s_flush) ? (e / s_flush) * s_flush : 0;
}

struct AppendArgs {
  int B, Hkv, cap, cap_alloc, s_sink, s_keep, s_flush, R, sink_dim, n_new;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint32_t* k_params;
  uint32_t* v_params;
  __half* k_sink;
  __half* v_sink;
  __half* k_ring;
  __half* v_ring;
  int32_t* state;
  uint32_t* status;
  const __half* k_new;
  const __half* v_new;
  const __half* t_k;
  int i_lo, i_hi;
  float f_lo, f_hi;
  // decode preparation fused into a one-token append (wushkv_step): q' = T_K^{-T} q of the
  // unit's query heads and its query fragments into the decode workspace
  const __half* q;
  const float* t_k_inv;
  float* qprime;
  uint8_t* qfrag;      // the unit's query fragments for the decode kernel (qfrag.cuh)
  float scale_log2;    // softmax_scale * log2(e)
  int Hq;
  int qchains;         // the decode's cluster size: q' is summed in that many row blocks
  PrepSpec prep;  // raw q / k (wushkv_step_prep): RMSNorm + RoPE fused in
  int defer_state;  // 1 (fused step): leave the state words to the decode kernel that follows
  int transform;  // WUSHKV_TRANSFORM_DENSE (t_k) or WUSHKV_TRANSFORM_HADAMARD (in-kernel)
  int quant_rms;            // WUSHKV_QUANT_RMS: (s, z) from the token's RMS, not its percentiles
  float rms_kb, rms_alpha;  // fp32(2*alpha/(2^b-1)), fp32(alpha)
};

struct DecodeArgs {
  int B, Hkv, Hq, cap, cap_alloc, s_sink, s_keep, s_flush, R, sink_dim, n_split, split_tokens;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint32_t* k_params;
  const uint32_t* v_params;
  const __half* k_sink;
  const __half* v_sink;
  const __half* k_ring;
  const __half* v_ring;
  int32_t* state;     // read; written only in a fused step (below)
  uint32_t* status;
  const __half* q;
  const float* t_k_inv;
  float scale_log2;  // softmax_scale * log2(e)
  void* out;
  int out_fp16;
  int units;
  // workspace, per virtual unit (units * npass of them; see chunk attention below)
  uint32_t* tickets;   // [vu] completion counters of the last merge (zero between calls)
  float* qprime;       // [vu][G][128] fp32 (fused step: written by the append kernel)
  uint8_t* qfrag;      // [vu][kQFragBytes]: query fragments and constants (qfrag.cuh; fused step)
  float* partials;     // [vu][n_split / cluster][G][132]: the clusters' merged states
  int cluster;         // CTAs per cluster
  // 1: cluster c of the grid (in linear order) is cluster c / U of unit c % U (U = gridDim.y),
  // so that every unit has work items in every round of CTAs an SM receives; 0: grid row =
  // unit, column = item
  int interleave;
  // fused step (wushkv_step's one-kernel append of n_new tokens runs just before): that
  // kernel leaves the state words alone, so this one reads the pre-append state, derives the
  // post-append (S, S_quant) from it, streams the tiles below the old S_quant before the
  // append has finished (nothing there changes), reads everything else after it, and writes
  // the new state once every item of the unit has read the old one (the final merge).
  int fused, n_new;
  // chunk attention (wushkv_chunk_attn): the kernel's G query heads per unit are gq real
  // heads of each of G / gq consecutive chunk tokens; q and out are [B][chunk_n][H_q][128];
  // chunk_n = 0 for a one-token decode (gq = G).  One launch takes npass such blocks of
  // tokens, starting at chunk token chunk_t0: its grid has a virtual unit vu = unit * npass
  // + pass for each (cache unit, block), with the workspace (tickets, q', fragments,
  // partials) indexed by vu and the cache by unit; block `pass` starts at chunk token
  // chunk_t0 + pass * G / gq.  npass = 1 outside chunk attention.
  int chunk_n, chunk_t0, gq, npass;
  PrepSpec prep;       // raw q (wushkv_step_prep, bulk route): the kernel normalises and rotates it
  // bounded waits: the cycle limit after which a wait gives up (STATUS_TIMEOUT), and a test
  // hook -- the producer never issues stage `withhold_tile` of any item (-1: off)
  int withhold_tile;
  long long wait_limit;
};

// Raise a kernel's dynamic shared-memory limit once per device (a function attribute,
// not a stream operation, so it is kept out of the launch path and of graph capture).
// One flag set per kernel (the template argument is the kernel itself).
template <auto Kernel>
cudaError_t ensure_smem_attr(int bytes) {
  static int done[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = bytes;
  return e;
}

cudaError_t launch_append(const Derived& d, int bits, bool small, const AppendArgs& a, cudaStream_t st);
cudaError_t launch_decode(const Derived& d, int bits, const DecodeArgs& a, cudaStream_t st);
// wushkv_step's one-token path: the small append fused with the decode's query preparation
// (it lets its dependents launch early), then the main decode kernel, launched as that
// kernel's programmatic dependent (it waits for it before reading what it writes).
cudaError_t launch_append_fused(const Derived& d, int bits, const AppendArgs& a, cudaStream_t st);
cudaError_t launch_decode_main(const Derived& d, int bits, const DecodeArgs& a, cudaStream_t st);

}  // namespace wushkv
