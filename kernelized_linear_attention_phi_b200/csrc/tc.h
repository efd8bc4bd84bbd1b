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
// Chunk length the tensor-core chunked kernel runs at for a requested chunk
// (d = 128 always runs 64-token chunks: the shared-memory budget).
int tc_chunk(const Problem& p, int chunk);
// Same contract as simt_chunked, at chunk length tc_chunk(p, chunk); the
// prefix-mask inputs (perm, bins, mcl, nbins) must be binned at that length.
cudaError_t tc_chunked(const Problem& p, int chunk, const void* q, const void* k, const void* v,
                       const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                       const int32_t* bins, const int32_t* mcl, int nbins, void* out, uint32_t* err,
                       cudaStream_t st);

}  // namespace la
