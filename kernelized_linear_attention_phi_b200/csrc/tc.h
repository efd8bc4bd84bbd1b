// Tensor-core (tcgen05 / TMEM / TMA) kernels for bf16 inputs, d in {64, 128}.
#pragma once

#include <cuda.h>

#include "internal.h"
#include "plan.h"

namespace la {

// True when the tcgen05 path handles this problem (bf16, d = 64 or 128).
bool tc_supported(const Problem& p);

// Every kernel below bounds its waits; an expired wait sets
// tc::FLAG_TIMEOUT in *err (the workspace error word) and the kernel returns.

// Balanced split of the KV summary (plan::KvBalanced): a 1-D grid of G CTAs
// cuts the flattened sequence of (head, 128-token tile) pairs into G
// contiguous ranges of equal length; a range that touches several heads
// writes one partial record per head, slot (cta * K + j) holding the record
// of the j-th head the CTA touches. Planned for the current device's SMs,
// per_sm ranges per SM.
using KvBalanced = plan::KvBalanced;
KvBalanced kv_balanced_plan(const Problem& p, int per_sm = 1);

// KV summary in balanced mode: partial records into `part` (G*K slots of
// d*d + d floats), then a fixed-order reduction into S [bh][d*d], z [bh][d].
cudaError_t tc_kv_summary(const Problem& p, const void* k, const void* v, float* part, float* S,
                          float* z, uint32_t* err, cudaStream_t st);
// Non-causal attention in one kernel for small problems (tc_fused.cu): bf16,
// d = 64, N <= 8192, and one 8-CTA cluster per head all resident at once
// (B*H <= 33 on a B200). Writes
// out and, when S / z are non-null, the KV summary [bh][d*d], [bh][d]; with
// out null (q then unused) only the KV summary, into S and z (both needed).
bool tc_noncausal_fused_supported(const Problem& p);
cudaError_t tc_noncausal_fused(const Problem& p, const void* q, const void* k, const void* v, void* out, float* S,
                               float* z, uint32_t* err, cudaStream_t st);
// Sums balanced-split records of plan w (slot cta * K + j, d*d + d floats
// each) per head in CTA order into S [bh][d*d] and z [bh][d].
cudaError_t tc_reduce_records(const Problem& p, const KvBalanced& w, const float* part, float* S, float* z,
                              cudaStream_t st);
// KV summary per block: CTA (block, head) writes record (head*nblk + block)
// over tokens [block*block_tokens, ...); block_tokens must be a multiple of 128.
// Only blocks 0..nform-1 are formed (nform <= nblk; -1: all).
cudaError_t tc_kv_blocks(const Problem& p, const void* k, const void* v, int block_tokens, int nblk,
                         float* part, uint32_t* err, cudaStream_t st, int nform = -1);
// tc_kv_blocks followed by the exclusive block-state scan, in one kernel with
// a thread-block cluster per head (bf16, d = 64, nblk <= 16, every head's
// cluster resident at once, with one or two blocks per CTA): part[bh*nblk +
// blk] receives the prefix of the blocks before blk (what
// state_exclusive_scan leaves), S_total / z_total (nullable) the total.
bool tc_kv_scan_supported(const Problem& p, int block_tokens, int nblk);
cudaError_t tc_kv_blocks_scan(const Problem& p, const void* k, const void* v, int block_tokens, int nblk, float* part,
                              float* S_total, float* z_total, uint32_t* err, cudaStream_t st);
// Same contract as simt_readout.
cudaError_t tc_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                       uint32_t* err, cudaStream_t st);

// Chunk length the tensor-core chunked kernel runs at for a requested chunk
// (d = 128 always runs 64-token chunks: the shared-memory budget).
int tc_chunk(const Problem& p, int chunk);
// Same contract as simt_chunked, at chunk length tc_chunk(p, chunk); the
// prefix-mask inputs (perm, bins, msort, nbins) must be binned at that length.
cudaError_t tc_chunked(const Problem& p, int chunk, const void* q, const void* k, const void* v,
                       const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                       const int32_t* bins, const int32_t* msort, int nbins, void* out, uint32_t* err,
                       cudaStream_t st);

// The d = 128 kernel behind tc_chunked (64-token chunks, state kept as S^T).
// With raw_prefix, `prefix` holds each block's own state (as tc_kv_blocks
// writes it; the last block's record is not read) and every CTA sums the
// records of the blocks before it, so no scan runs in between.
cudaError_t tc_chunked_t(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                         int block_tokens, int nblk, const int32_t* perm, const int32_t* bins,
                         const int32_t* msort, int nbins, void* out, uint32_t* err, cudaStream_t st,
                         bool raw_prefix = false);

// Gradients of the non-causal form (tc_bwd.cu): S, z are the KV summary of
// the forward; `part` holds tc_backward_record_slots(p) records, (G, h)
// [bh][d*d], [bh][d] receive the reduced records. Writes dq, dk, dv.
size_t tc_backward_record_slots(const Problem& p);
cudaError_t tc_noncausal_backward(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                                  const float* S, const float* z, float* part, float* G, float* h, void* dq,
                                  void* dk, void* dv, uint32_t* err, cudaStream_t st);

// First sweep of the causal gradients on tensor cores (tc_bwd_causal.cu,
// tc_bwd_causal_t.cu at d = 128; bf16, d = 64 or 128, block_tokens a
// multiple of 64): from the forward's exclusive
// block prefixes, writes dq, gn (bf16 [bh][N][d]), gden (fp32 [bh][N]) and
// the blocks' own (G, h) records grec[bh*nblk + blk], as bwd_q does.
bool tc_causal_backward_supported(const Problem& p, int block_tokens);
cudaError_t tc_causal_backward_q(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                                 const float* prefix, int block_tokens, int nblk, void* dq, void* gn, float* gden,
                                 float* grec, uint32_t* err, cudaStream_t st);
// Second sweep (same support): from the blocks' suffix states (G, h)
// (grec after the reverse exclusive scan), gn and gden, writes dk and dv.
cudaError_t tc_causal_backward_kv(const Problem& p, const void* q, const void* k, const void* v, const void* gn,
                                  const float* gden, const float* suffix, int block_tokens, int nblk, void* dk,
                                  void* dv, uint32_t* err, cudaStream_t st);
// The same two sweeps at d = 128 (tc_bwd_causal_t.cu), bf16, 64-token chunks.
cudaError_t tc_causal_backward_q_t(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                                   const float* prefix, int block_tokens, int nblk, void* dq, void* gn, float* gden,
                                   float* grec, uint32_t* err, cudaStream_t st);
cudaError_t tc_causal_backward_kv_t(const Problem& p, const void* q, const void* k, const void* v, const void* gn,
                                    const float* gden, const float* suffix, int block_tokens, int nblk, void* dk,
                                    void* dv, uint32_t* err, cudaStream_t st);

// [BH, N, d] bf16 viewed as 3-D for TMA: 64-column x `rows` boxes, 128-byte
// swizzle, zero fill outside the tensor.
cudaError_t make_map(CUtensorMap* map, const void* base, int d, int N, long long bh, int rows);
// Same, for any element type: boxes of box_cols x box_rows elements (box_cols
// * elem_bytes = 128 for the 128-byte swizzle).
cudaError_t make_map_box(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes, int d,
                         int N, long long bh, int box_cols, int box_rows);

// fp32 forms at d = 64 on the tensor cores with split bf16 operands (tc_f32.cu).
bool tc_f32_supported(const Problem& p);
// (S, z) of each block of block_tokens keys: record (bh * nblk + blk) of part.
cudaError_t tc_f32_states(const Problem& p, const void* k, const void* v, int block_tokens, int nblk, float* part,
                          uint32_t* err, cudaStream_t st);
// Causal outputs of each block from its exclusive prefix record in `prefix`.
cudaError_t tc_f32_chunked(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                           int block_tokens, int nblk, void* out, uint32_t* err, cudaStream_t st);
// Prefix-mask outputs: the queries of bin c (from the binning tables perm,
// bins, msort of bin_queries with 64-token chunks) answered at chunk c from
// the block's exclusive prefix record in `prefix`.
cudaError_t tc_f32_prefix(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                          int block_tokens, int nblk, const int32_t* perm, const int32_t* bins, const int32_t* msort,
                          int nbins, void* out, uint32_t* err, cudaStream_t st);
// Non-causal outputs from each head's total S [bh][d][d] and z [bh][d].
cudaError_t tc_f32_readout(const Problem& p, const void* q, const float* S, const float* z, int block_tokens,
                           int nblk, void* out, uint32_t* err, cudaStream_t st);
// The same tensor viewed as 2-D [rows = BH * N, d] for row gathers
// (tile::gather4): 64-column x 1-row boxes, 128-byte swizzle.
cudaError_t make_row_map(CUtensorMap* map, const void* base, int d, long long rows);
// Same, for any element type: one-row boxes of box_cols elements (box_cols *
// elem_bytes = 128 for the 128-byte swizzle).
cudaError_t make_row_map_box(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes, int d,
                             long long rows, int box_cols);

}  // namespace la
