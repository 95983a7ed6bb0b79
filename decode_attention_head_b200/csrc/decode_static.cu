// wushkv_decode_attn_static: decode attention whose scratch lives in a fixed array of
// device memory that belongs to the library, for callers that cannot allocate device
// memory at call time (an allocator-less runtime, code that must not enter the CUDA
// or PyTorch caching allocator between steps, a plugin host that owns every buffer).
//
// The attention itself is the ordinary wushkv_decode_attn path: this file only supplies
// its `workspace` argument.  The array is file-scope `static __device__`, so every
// device that loads the library holds WUSHKV_STATIC_SCRATCH_BYTES of it until the
// process exits.  It starts zero-filled (static storage), as a workspace must before its
// first use, and every call leaves the decode's completion counters in it at zero again.
// Its device address is looked up with cudaGetSymbolAddress (the host-side name is not a
// device address) on every call, in the current CUDA context.
#include <cmath>
#include <cuda_runtime.h>
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[WUSHKV_STATIC_SCRATCH_BYTES];

// The array's device address depends on the CUDA context the library's module is loaded
// in (each device's primary context, or a context the caller created), so it is looked up
// on every call, in the context current then: a cache keyed on the context handle could
// hand out a dead context's address once a destroyed context's handle is reused.  The
// lookup is a host-side table query; the first one in a context loads the module.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess) return e;
  if (!p) return cudaErrorInvalidSymbol;
  *out = p;
  return cudaSuccess;
}

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

// The argument checks of wushkv_decode_attn, repeated so that a rejected call queues
// nothing (not even the counter reset below).
bool args_ok(const wushkv_cache* c, const void* q, const float* t_k_inv, float softmax_scale, int32_t out_fp16,
             const void* out) {
  return c && aligned16(c->k_codes) && aligned16(c->v_codes) && aligned16(c->k_params) &&
         aligned16(c->v_params) && aligned16(c->k_sink) && aligned16(c->v_sink) && aligned16(c->k_ring) &&
         aligned16(c->v_ring) && aligned16(c->state) && aligned16(q) && aligned16(t_k_inv) && aligned16(out) &&
         std::isfinite(softmax_scale) && (out_fp16 == 0 || out_fp16 == 1);
}

}  // namespace

extern "C" int wushkv_decode_attn_static(const wushkv_config* cfg, const wushkv_cache* cache, const void* q,
                                         const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                                         void* stream) {
  wushkv::Derived d;
  const int rc = wushkv::derive(cfg, &d);
  if (rc != WUSHKV_OK) return rc;
  if (!args_ok(cache, q, t_k_inv, softmax_scale, out_fp16, out)) return WUSHKV_EINVAL;
  if (d.ws_total > (size_t)WUSHKV_STATIC_SCRATCH_BYTES) return WUSHKV_ESCRATCH;
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return WUSHKV_ECUDA;
  // The array keeps whatever the previous call (of any configuration) left in it.  Nothing
  // needs clearing here: the decode's own first kernel (the prologue) resets the split
  // merge's completion counters on every call, and every other part of the workspace is
  // written before it is read.
  return wushkv_decode_attn(cfg, cache, q, t_k_inv, softmax_scale, out_fp16, out, ws, stream);
}
