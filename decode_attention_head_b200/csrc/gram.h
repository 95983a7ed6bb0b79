// Internal interface of the calibration Gram-matrix kernel (gram.cu) to the C-ABI layer.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace wushkv {

constexpr int kGramTokens = 4096;  // at most this many tokens of one head per CTA (one fp32 partial sum)

// wushkv_gram_accumulate after validation (n_tokens >= 1, 1 <= n_heads <= 65535,
// n_tokens * n_heads <= 2^40, both pointers 16-byte aligned).
cudaError_t launch_gram(const uint16_t* x, int64_t n_tokens, int n_heads, double* gram, cudaStream_t st);

}  // namespace wushkv
