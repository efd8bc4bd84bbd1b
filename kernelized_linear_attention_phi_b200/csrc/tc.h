// Tensor-core (tcgen05 / TMEM / TMA) kernels for bf16 inputs, d in {64, 128}.
#pragma once

#include "internal.h"

namespace la {

// True when the tcgen05 path handles this problem (bf16, d = 64 or 128).
bool tc_supported(const Problem& p);

// The kernels below bound every wait; an expired wait sets
// tc::FLAG_TIMEOUT in *err (the workspace error word) and the kernel returns.

// Same contract as simt_kv_partial; tokens_per_split must be a multiple of 128.
cudaError_t tc_kv_partial(const Problem& p, const void* k, const void* v, int tokens_per_split,
                          int nsplit, float* part, uint32_t* err, cudaStream_t st);
// Same contract as simt_readout.
cudaError_t tc_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                       uint32_t* err, cudaStream_t st);
// True when tc_causal handles this problem.
bool tc_causal_supported(const Problem& p);
// Causal outputs of every block from its prefix state.
cudaError_t tc_causal(const Problem& p, int chunk, const void* q, const void* k, const void* v,
                      const float* prefix, int block_tokens, int nblk, void* out, uint32_t* err,
                      cudaStream_t st);

}  // namespace la
