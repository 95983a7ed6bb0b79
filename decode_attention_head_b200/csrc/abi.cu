// C-ABI entry points of libwushkv (declared in include/wushkv.h): configuration
// validation, buffer layout, the host-side compensation-matrix helper, and launch.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include "internal.h"
#include "gram.h"
#include "ptx.cuh"
#include "qfrag.cuh"

namespace wushkv {

static inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
static inline size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// Chunk attention runs up to this many blocks of chunk tokens in one launch, as that many
// virtual units per cache unit (and never more virtual units than a grid column holds).
constexpr int kMaxPasses = 32;
static int max_passes(const wushkv_config* cfg, long long units) {
  long long p = kMaxPasses;
  if (cfg->chunk_max < p) p = cfg->chunk_max;
  if (65535 / units < p) p = 65535 / units;
  return p < 1 ? 1 : (int)p;
}

int derive(const wushkv_config* cfg, Derived* d, long long ticket_units) {
  if (!cfg || !d) return WUSHKV_EINVAL;
  if (cfg->head_dim != kHeadDim) return WUSHKV_EUNSUPPORTED;
  if (cfg->bits != 2 && cfg->bits != 4) return WUSHKV_EUNSUPPORTED;
  if (cfg->batch < 1 || cfg->n_kv_heads < 1 || cfg->n_q_heads < 1 || cfg->capacity < 1) return WUSHKV_EINVAL;
  if (cfg->n_q_heads % cfg->n_kv_heads) return WUSHKV_EINVAL;
  const int g = cfg->n_q_heads / cfg->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return WUSHKV_EUNSUPPORTED;
  if (cfg->s_sink < 0 || cfg->s_keep < 0 || cfg->s_flush < 1 || cfg->chunk_max < 1) return WUSHKV_EINVAL;
  if (!(cfg->p_lo >= 0.f) || !(cfg->p_hi <= 100.f) || !(cfg->p_lo < cfg->p_hi)) return WUSHKV_EINVAL;
  if (cfg->transform != WUSHKV_TRANSFORM_DENSE && cfg->transform != WUSHKV_TRANSFORM_HADAMARD) return WUSHKV_EINVAL;
  if (cfg->quantizer != WUSHKV_QUANT_PERCENTILE && cfg->quantizer != WUSHKV_QUANT_RMS) return WUSHKV_EINVAL;
  if (cfg->quantizer == WUSHKV_QUANT_RMS && !(cfg->clip_alpha > 0.f && std::isfinite(cfg->clip_alpha)))
    return WUSHKV_EINVAL;
  const long long units = (long long)cfg->batch * cfg->n_kv_heads;
  if (units > (1 << 24) || cfg->capacity > (1 << 28)) return WUSHKV_EINVAL;

  d->units = (int)units;
  d->group = g;
  d->cap_alloc = (int)round_up((size_t)cfg->capacity, kTileTokens);
  d->ring = cfg->s_keep + cfg->s_flush - 1 + cfg->chunk_max;
  d->sink_dim = cfg->s_sink > 0 ? cfg->s_sink : 1;
  d->code_bytes = 16 * cfg->bits;
  // percentile ranks: pos = p/100 * 127 in double, i = floor(pos), f = fp32(pos - i)
  const double pos_lo = (double)cfg->p_lo / 100.0 * (double)(kHeadDim - 1);
  const double pos_hi = (double)cfg->p_hi / 100.0 * (double)(kHeadDim - 1);
  d->i_lo = (int)std::floor(pos_lo);
  d->i_hi = (int)std::floor(pos_hi);
  d->f_lo = (float)(pos_lo - d->i_lo);
  d->f_hi = (float)(pos_hi - d->i_hi);
  const int need_lo = d->i_lo + 2;               // s[i_lo], s[i_lo+1]
  const int need_hi = kHeadDim - d->i_hi;        // s[i_hi] from the top
  d->nsel = need_lo > need_hi ? need_lo : need_hi;
  if (d->nsel < 2) d->nsel = 2;
  if (cfg->quantizer == WUSHKV_QUANT_RMS) d->nsel = 2;  // no order statistics
  if (d->nsel > 4) return WUSHKV_EUNSUPPORTED;

  // decode work split: n_split items per unit, chosen so that units * n_split fills whole
  // waves of the GPU's CTA slots best (the kernel divides each unit's current quantized
  // region evenly among its items at run time); an even n_split runs as clusters of two
  // CTAs (consecutive items), which share the query's preparation and merge their states
  // before the unit's last merge, and wins a near-tie (within half a percent of fill); on
  // a tie the smaller n_split wins.  (Clusters of three or more CTAs would leave SMs of a
  // B200 that no such cluster can be placed on idle.)  split_tokens is the per-item bound
  // at capacity
  {
    const int slots = kB200SMs * decode_ctas_per_sm(g);
    int n0 = slots / d->units;
    if (n0 < 1) n0 = 1;
    if (n0 > kMaxSplits) n0 = kMaxSplits;
    int best = 1;
    double best_score = -1.0;
    for (int n = n0 > 3 ? n0 - 3 : 1; n <= n0 + 3 && n <= kMaxSplits; ++n) {
      const long long items = (long long)d->units * n;
      const long long waves = (items + slots - 1) / slots;
      const double score = (double)items / (double)(waves * slots) + (n % 2 == 0 ? 0.005 : 0.0);
      if (score > best_score + 1e-9) {
        best_score = score;
        best = n;
      }
    }
    d->n_split = best;
    d->cluster = best % 2 == 0 ? 2 : 1;
    // a unit whose items fill a quarter of a round of CTAs or more (one sequence at long
    // context) would otherwise sit in the rounds an SM receives last, which run slowest
    d->interleave = best * 4 >= kB200SMs ? 1 : 0;
    const int tiles = ceil_div(d->cap_alloc, kTileTokens);
    d->split_tokens = ceil_div(tiles, d->n_split) * kTileTokens;
  }

  const size_t U = (size_t)d->units;
  d->codes_bytes = U * d->cap_alloc * d->code_bytes;
  d->params_bytes = U * d->cap_alloc * 4;
  d->sink_bytes = U * d->sink_dim * kHeadDim * 2;
  d->ring_bytes = U * (size_t)d->ring * kHeadDim * 2;
  d->state_bytes = round_up((2 * U + 1) * 4, 16);
  size_t off = 0;
  // unit counters (zero between calls): one per virtual unit of the largest chunk-attention
  // launch, in every layout, so that decode, step and chunk calls may share one workspace --
  // no call writes anything but zeros into another call's counters
  if (ticket_units < 0) ticket_units = (long long)U * max_passes(cfg, (long long)U);
  d->ws_tickets = off;
  off = round_up(off + (size_t)ticket_units * 4, 256);
  d->ws_qprime = off;
  off = round_up(off + U * g * kHeadDim * 4, 256);
  d->ws_qfrag = off;
  off = round_up(off + U * kQFragBytes, 256);
  d->ws_partials = off;  // one merged state per cluster
  off = round_up(off + U * (size_t)(d->n_split / d->cluster) * g * 132 * 4, 256);
  d->ws_total = off;
  return WUSHKV_OK;
}

static bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

static bool cache_ok(const wushkv_cache* c) {
  return c && aligned16(c->k_codes) && aligned16(c->v_codes) && aligned16(c->k_params) &&
         aligned16(c->v_params) && aligned16(c->k_sink) && aligned16(c->v_sink) && aligned16(c->k_ring) &&
         aligned16(c->v_ring) && aligned16(c->state);
}

}  // namespace wushkv

using namespace wushkv;

// Largest power of two ng with ng * g <= 8 and ng <= n: the chunk tokens one block of
// chunk attention takes (as ng * g query heads per KV head).
static int chunk_block(int g, int n) {
  int ng = 1;
  while (2 * ng * g <= 8 && 2 * ng <= n) ng *= 2;
  return ng;
}

// The decode derivation for a launch of chunk attention over np blocks of ng tokens: the
// query heads per KV head of one block, and np virtual units per cache unit (passed to the
// split policy and the workspace layout as np times the batch).
static int derive_chunk(const wushkv_config* cfg, int ng, int np, Derived* d) {
  wushkv_config c2 = *cfg;
  c2.n_q_heads = cfg->n_kv_heads * (cfg->n_q_heads / cfg->n_kv_heads) * ng;
  c2.batch = cfg->batch * np;
  const long long units = (long long)cfg->batch * cfg->n_kv_heads;
  return derive(&c2, d, units * max_passes(cfg, units));
}

// The launches of chunk attention over the chunk tokens [t0, n): the first takes the whole
// blocks of the largest size that fits, up to kMaxPasses of them (and no more virtual units
// than a grid column holds), all in one grid -- their passes over the cache run side by side,
// so the blocks of a unit read each stage at about the same time; what is left takes the
// next launch, and so on.
static void chunk_launch(int g, int units, int n, int t0, int* ng, int* np) {
  *ng = chunk_block(g, n - t0);
  int p = (n - t0) / *ng;
  const int grid_cap = 65535 / units > 1 ? 65535 / units : 1;
  if (p > kMaxPasses) p = kMaxPasses;
  if (p > grid_cap) p = grid_cap;
  *np = p;
}

// Workspace of wushkv_chunk_attn: the largest any of its launches needs, over every chunk
// length up to chunk_max (lengths above (kMaxPasses + 1) * 8 repeat launches of shorter ones).
static size_t chunk_workspace(const wushkv_config* cfg) {
  const int g = cfg->n_q_heads / cfg->n_kv_heads;
  const int units = cfg->batch * cfg->n_kv_heads;
  const int nmax = cfg->chunk_max < (kMaxPasses + 1) * 8 ? cfg->chunk_max : (kMaxPasses + 1) * 8;
  size_t best = 0;
  for (int n = 1; n <= nmax; ++n) {
    for (int t0 = 0; t0 < n;) {
      int ng, np;
      chunk_launch(g, units, n, t0, &ng, &np);
      Derived d;
      if (derive_chunk(cfg, ng, np, &d) == WUSHKV_OK && d.ws_total > best) best = d.ws_total;
      t0 += ng * np;
    }
  }
  return best;
}

extern "C" int wushkv_pack_layout(const wushkv_config* cfg, wushkv_layout* out) {
  if (!out) return WUSHKV_EINVAL;
  Derived d;
  const int rc = derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  std::memset(out, 0, sizeof(*out));
  out->codes_bytes = d.codes_bytes;
  out->params_bytes = d.params_bytes;
  out->sink_bytes = d.sink_bytes;
  out->ring_bytes = d.ring_bytes;
  out->state_bytes = d.state_bytes;
  out->workspace_bytes = d.ws_total;
  out->cap_alloc = d.cap_alloc;
  out->ring_slots = d.ring;
  out->code_bytes = d.code_bytes;
  out->n_splits = d.n_split;
  out->chunk_workspace_bytes = chunk_workspace(cfg);
  out->split_tokens = d.split_tokens;
  out->code_order = WUSHKV_CODE_ORDER_VGROUP16;
  out->decode_cluster = d.cluster;
  out->decode_interleave = d.interleave;
  return WUSHKV_OK;
}

extern "C" int wushkv_compensation(const uint16_t* t_k, int32_t n_kv_heads, float* t_k_inv) {
  if (!t_k || !t_k_inv || n_kv_heads < 1) return WUSHKV_EINVAL;
  const int n = kHeadDim;
  std::vector<double> a((size_t)n * 2 * n);
  for (int h = 0; h < n_kv_heads; ++h) {
    // [T | I], Gauss-Jordan with partial pivoting -> [I | T^{-1}]
    for (int r = 0; r < n; ++r) {
      for (int c = 0; c < n; ++c) {
        __half_raw raw;
        raw.x = t_k[((size_t)h * n + r) * n + c];
        a[(size_t)r * 2 * n + c] = (double)__half2float(__half(raw));
        a[(size_t)r * 2 * n + n + c] = (r == c) ? 1.0 : 0.0;
      }
    }
    for (int col = 0; col < n; ++col) {
      int piv = col;
      double best = std::fabs(a[(size_t)col * 2 * n + col]);
      for (int r = col + 1; r < n; ++r) {
        const double v = std::fabs(a[(size_t)r * 2 * n + col]);
        if (v > best) {
          best = v;
          piv = r;
        }
      }
      if (!(best > 0.0)) return WUSHKV_ESINGULAR;
      if (piv != col)
        for (int c = 0; c < 2 * n; ++c) std::swap(a[(size_t)piv * 2 * n + c], a[(size_t)col * 2 * n + c]);
      const double inv = 1.0 / a[(size_t)col * 2 * n + col];
      for (int c = 0; c < 2 * n; ++c) a[(size_t)col * 2 * n + c] *= inv;
      for (int r = 0; r < n; ++r) {
        if (r == col) continue;
        const double f = a[(size_t)r * 2 * n + col];
        if (f == 0.0) continue;
        for (int c = 0; c < 2 * n; ++c) a[(size_t)r * 2 * n + c] -= f * a[(size_t)col * 2 * n + c];
      }
    }
    for (int r = 0; r < n; ++r)
      for (int c = 0; c < n; ++c) t_k_inv[((size_t)h * n + r) * n + c] = (float)a[(size_t)r * 2 * n + n + c];
  }
  return WUSHKV_OK;
}

static void fill_append(const wushkv_config* cfg, const Derived& d, const wushkv_cache* cache, const void* k_new,
                        const void* v_new, int32_t n_new, const void* t_k, AppendArgs* a) {
  std::memset(a, 0, sizeof(*a));
  a->B = cfg->batch;
  a->Hkv = cfg->n_kv_heads;
  a->cap = cfg->capacity;
  a->cap_alloc = d.cap_alloc;
  a->s_sink = cfg->s_sink;
  a->s_keep = cfg->s_keep;
  a->s_flush = cfg->s_flush;
  a->R = d.ring;
  a->sink_dim = d.sink_dim;
  a->n_new = n_new;
  a->k_codes = static_cast<uint8_t*>(cache->k_codes);
  a->v_codes = static_cast<uint8_t*>(cache->v_codes);
  a->k_params = static_cast<uint32_t*>(cache->k_params);
  a->v_params = static_cast<uint32_t*>(cache->v_params);
  a->k_sink = static_cast<__half*>(cache->k_sink);
  a->v_sink = static_cast<__half*>(cache->v_sink);
  a->k_ring = static_cast<__half*>(cache->k_ring);
  a->v_ring = static_cast<__half*>(cache->v_ring);
  a->state = cache->state;
  a->status = reinterpret_cast<uint32_t*>(cache->state + 2 * (size_t)d.units);
  a->k_new = static_cast<const __half*>(k_new);
  a->v_new = static_cast<const __half*>(v_new);
  a->t_k = static_cast<const __half*>(t_k);
  a->i_lo = d.i_lo;
  a->i_hi = d.i_hi;
  a->f_lo = d.f_lo;
  a->f_hi = d.f_hi;
  a->Hq = cfg->n_q_heads;
  a->transform = cfg->transform;
  a->quant_rms = cfg->quantizer == WUSHKV_QUANT_RMS;
  a->rms_kb = (float)(2.0 * (double)cfg->clip_alpha / (double)((1 << cfg->bits) - 1));
  a->rms_alpha = cfg->clip_alpha;
}

static void fill_decode(const wushkv_config* cfg, const Derived& d, const wushkv_cache* cache, const void* q,
                        const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out, void* workspace,
                        DecodeArgs* a) {
  std::memset(a, 0, sizeof(*a));
  a->B = cfg->batch;
  a->Hkv = cfg->n_kv_heads;
  a->Hq = cfg->n_q_heads;
  a->cap = cfg->capacity;
  a->cap_alloc = d.cap_alloc;
  a->s_sink = cfg->s_sink;
  a->s_keep = cfg->s_keep;
  a->s_flush = cfg->s_flush;
  a->R = d.ring;
  a->sink_dim = d.sink_dim;
  a->n_split = d.n_split;
  a->split_tokens = d.split_tokens;
  a->k_codes = static_cast<const uint8_t*>(cache->k_codes);
  a->v_codes = static_cast<const uint8_t*>(cache->v_codes);
  a->k_params = static_cast<const uint32_t*>(cache->k_params);
  a->v_params = static_cast<const uint32_t*>(cache->v_params);
  a->k_sink = static_cast<const __half*>(cache->k_sink);
  a->v_sink = static_cast<const __half*>(cache->v_sink);
  a->k_ring = static_cast<const __half*>(cache->k_ring);
  a->v_ring = static_cast<const __half*>(cache->v_ring);
  a->state = cache->state;
  a->status = reinterpret_cast<uint32_t*>(cache->state + 2 * (size_t)d.units);
  a->q = static_cast<const __half*>(q);
  a->t_k_inv = t_k_inv;
  a->scale_log2 = softmax_scale * 1.4426950408889634f;
  a->out = out;
  a->out_fp16 = out_fp16;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a->tickets = reinterpret_cast<uint32_t*>(ws + d.ws_tickets);
  a->qprime = reinterpret_cast<float*>(ws + d.ws_qprime);
  a->qfrag = ws + d.ws_qfrag;
  a->partials = reinterpret_cast<float*>(ws + d.ws_partials);
  a->cluster = d.cluster;
  a->interleave = d.interleave;
  a->units = d.units;
  a->fused = 0;
  a->n_new = 0;
  a->gq = d.group;
  a->chunk_n = 0;
  a->chunk_t0 = 0;
  a->npass = 1;
  a->withhold_tile = -1;
  a->wait_limit = kWaitLimitCycles;
}

static int check_append(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_new, const void* v_new,
                        int32_t n_new, const void* t_k) {
  if (!cache_ok(cache) || n_new < 0) return WUSHKV_EINVAL;
  if (cfg->transform == WUSHKV_TRANSFORM_DENSE && !aligned16(t_k)) return WUSHKV_EINVAL;
  if (n_new > 0 && (!aligned16(k_new) || !aligned16(v_new))) return WUSHKV_EINVAL;
  return WUSHKV_OK;
}

static int check_decode(const wushkv_cache* cache, const void* q, const float* t_k_inv, float softmax_scale,
                        int32_t out_fp16, const void* out, const void* workspace) {
  if (!cache_ok(cache) || !aligned16(q) || !aligned16(t_k_inv) || !aligned16(out) || !aligned16(workspace))
    return WUSHKV_EINVAL;
  if (!std::isfinite(softmax_scale) || (out_fp16 != 0 && out_fp16 != 1)) return WUSHKV_EINVAL;
  return WUSHKV_OK;
}

extern "C" int wushkv_hadamard(int32_t n_kv_heads, float* t_k_inv) {
  if (!t_k_inv || n_kv_heads < 1) return WUSHKV_EINVAL;
  const float c = (float)(1.0 / std::sqrt((double)kHeadDim));
  for (int h = 0; h < n_kv_heads; ++h)
    for (int r = 0; r < kHeadDim; ++r)
      for (int i = 0; i < kHeadDim; ++i)
        t_k_inv[((size_t)h * kHeadDim + r) * kHeadDim + i] = (__builtin_popcount(r & i) & 1) ? -c : c;
  return WUSHKV_OK;
}

extern "C" int wushkv_gram_accumulate(const void* x, int64_t n_tokens, int32_t n_heads, double* gram,
                                      void* stream) {
  if (!aligned16(gram) || n_tokens < 0 || n_heads < 1 || n_heads > 65535) return WUSHKV_EINVAL;
  // keeps the kernel's element offsets (t * n_heads + h) * 128 and its grid size in range
  if (n_tokens > (INT64_C(1) << 40) / n_heads) return WUSHKV_EINVAL;
  if (n_tokens == 0) return WUSHKV_OK;
  if (!aligned16(x)) return WUSHKV_EINVAL;
  const cudaError_t e = launch_gram(static_cast<const uint16_t*>(x), n_tokens, n_heads, gram,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : WUSHKV_ECUDA;
}

extern "C" int wushkv_append(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_new,
                             const void* v_new, int32_t n_new, const void* t_k, void* stream) {
  Derived d;
  int rc = derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  rc = check_append(cfg, cache, k_new, v_new, n_new, t_k);
  if (rc != WUSHKV_OK) return rc;
  AppendArgs a;
  fill_append(cfg, d, cache, k_new, v_new, n_new, t_k, &a);
  const bool small = n_new <= cfg->chunk_max;
  const cudaError_t e = launch_append(d, cfg->bits, small, a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : WUSHKV_ECUDA;
}

extern "C" int wushkv_decode_attn(const wushkv_config* cfg, const wushkv_cache* cache, const void* q,
                                  const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                                  void* workspace, void* stream) {
  Derived d;
  int rc = derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  rc = check_decode(cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace);
  if (rc != WUSHKV_OK) return rc;
  DecodeArgs a;
  fill_decode(cfg, d, cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace, &a);
  const cudaError_t e = launch_decode(d, cfg->bits, a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : WUSHKV_ECUDA;
}

extern "C" int wushkv_decode_attn_test_timeout(const wushkv_config* cfg, const wushkv_cache* cache, const void* q,
                                               const float* t_k_inv, float softmax_scale, int32_t out_fp16,
                                               void* out, void* workspace, int32_t withhold_stage,
                                               int64_t wait_limit_cycles, void* stream) {
  Derived d;
  int rc = derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  rc = check_decode(cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace);
  if (rc != WUSHKV_OK) return rc;
  if (withhold_stage < -1 || wait_limit_cycles < 1000 || wait_limit_cycles > kWaitLimitCycles) return WUSHKV_EINVAL;
  DecodeArgs a;
  fill_decode(cfg, d, cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace, &a);
  a.withhold_tile = withhold_stage;
  a.wait_limit = wait_limit_cycles;
  const cudaError_t e = launch_decode(d, cfg->bits, a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WUSHKV_OK : WUSHKV_ECUDA;
}

static int step_impl(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_new, const void* v_new,
                     int32_t n_new, const void* t_k, const void* q, const float* t_k_inv, float softmax_scale,
                     int32_t out_fp16, void* out, void* workspace, const wushkv_prep* prep, void* stream) {
  Derived d;
  int rc = derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  rc = check_append(cfg, cache, k_new, v_new, n_new, t_k);
  if (rc != WUSHKV_OK) return rc;
  rc = check_decode(cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace);
  if (rc != WUSHKV_OK) return rc;
  PrepSpec ps;
  std::memset(&ps, 0, sizeof(ps));
  if (prep) {
    if (!(prep->rope_theta > 1.0f) || !std::isfinite(prep->rope_theta)) return WUSHKV_EINVAL;
    if ((prep->q_norm_gain || prep->k_norm_gain) && !(prep->norm_eps > 0.0f)) return WUSHKV_EINVAL;
    if ((prep->q_norm_gain && !aligned16(prep->q_norm_gain)) || (prep->k_norm_gain && !aligned16(prep->k_norm_gain)))
      return WUSHKV_EINVAL;
    ps.enabled = 1;
    ps.log2_theta = std::log2((double)prep->rope_theta);
    ps.q_gain = static_cast<const __half*>(prep->q_norm_gain);
    ps.k_gain = static_cast<const __half*>(prep->k_norm_gain);
    ps.eps = prep->norm_eps;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  AppendArgs aa;
  fill_append(cfg, d, cache, k_new, v_new, n_new, t_k, &aa);
  aa.prep = ps;
  DecodeArgs da;
  fill_decode(cfg, d, cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace, &da);
  da.prep = ps;
  cudaError_t e;
  if (n_new <= cfg->chunk_max) {
    // one kernel appends and prepares the decode (q' and its fragments); the main decode
    // kernel is its programmatic dependent and waits for it before reading the cache
    aa.defer_state = 1;
    aa.q = da.q;
    aa.t_k_inv = da.t_k_inv;
    aa.qprime = da.qprime;
    aa.qfrag = da.qfrag;
    aa.scale_log2 = da.scale_log2;
    aa.qchains = d.cluster;
    e = launch_append_fused(d, cfg->bits, aa, st);
    if (e == cudaSuccess) {
      da.fused = 1;
      da.n_new = n_new;
      e = launch_decode_main(d, cfg->bits, da, st);
    }
  } else {
    e = launch_append(d, cfg->bits, false, aa, st);
    if (e == cudaSuccess) e = launch_decode(d, cfg->bits, da, st);
  }
  return e == cudaSuccess ? WUSHKV_OK : WUSHKV_ECUDA;
}

extern "C" int wushkv_step(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_new, const void* v_new,
                           int32_t n_new, const void* t_k, const void* q, const float* t_k_inv, float softmax_scale,
                           int32_t out_fp16, void* out, void* workspace, void* stream) {
  return step_impl(cfg, cache, k_new, v_new, n_new, t_k, q, t_k_inv, softmax_scale, out_fp16, out, workspace, nullptr,
                   stream);
}

extern "C" int wushkv_step_prep(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_raw,
                                const void* v_new, int32_t n_new, const void* t_k, const void* q_raw,
                                const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                                void* workspace, const wushkv_prep* prep, void* stream) {
  if (!prep) return WUSHKV_EINVAL;
  return step_impl(cfg, cache, k_raw, v_new, n_new, t_k, q_raw, t_k_inv, softmax_scale, out_fp16, out, workspace, prep,
                   stream);
}

extern "C" int wushkv_chunk_attn(const wushkv_config* cfg, const wushkv_cache* cache, const void* q, int32_t n_q,
                                 const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                                 void* workspace, void* stream) {
  Derived d;
  int rc = derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  if (n_q < 1 || n_q > cfg->chunk_max) return WUSHKV_EINVAL;
  rc = check_decode(cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace);
  if (rc != WUSHKV_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // blocks of ng tokens (ng * g query heads per KV head share one pass over the cache); one
  // launch pair takes np blocks as np virtual units per cache unit
  for (int t0 = 0; t0 < n_q;) {
    int ng, np;
    chunk_launch(d.group, d.units, n_q, t0, &ng, &np);
    Derived d2;
    rc = derive_chunk(cfg, ng, np, &d2);
    if (rc != WUSHKV_OK) return rc;
    DecodeArgs a;
    fill_decode(cfg, d2, cache, q, t_k_inv, softmax_scale, out_fp16, out, workspace, &a);
    a.B = cfg->batch;  // the cache's units, not the virtual ones
    a.units = d.units;
    a.status = reinterpret_cast<uint32_t*>(cache->state + 2 * (size_t)d.units);
    a.Hq = cfg->n_q_heads;
    a.gq = d.group;
    a.chunk_n = n_q;
    a.chunk_t0 = t0;
    a.npass = np;
    const cudaError_t e = launch_decode(d2, cfg->bits, a, st);
    if (e != cudaSuccess) return WUSHKV_ECUDA;
    t0 += ng * np;
  }
  return WUSHKV_OK;
}
