// Internal interfaces between the host API (la_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <la.h>
#include <stddef.h>
#include <stdint.h>

namespace la {

// la_kv_summary's checks of the descriptor and the four pointers (no CUDA
// call); LA_OK or the status la_kv_summary returns for them (la_api.cu).
la_status kv_summary_args(const la_desc* desc, const void* k, const void* v, const float* S_out,
                          const float* z_out);
// la_kv_summary: validation, then the KV summary with `ws` as workspace.
la_status kv_summary_checked(const la_desc* desc, const void* k, const void* v, float* S_out,
                             float* z_out, void* ws, size_t ws_bytes, cudaStream_t st);

struct Problem {
    int B, H, N, d;
    int dtype;      // DT_F32 / DT_BF16
    int phi;        // PHI_RELU1 / PHI_IDENTITY
    int normalize;  // 0 / 1
    long long bh() const { return (long long)B * H; }
    size_t elem_bytes() const { return dtype == 0 ? 4 : 2; }
    // floats in one (S, z) state record: S (d*d) followed by z (d)
    size_t state_floats() const { return (size_t)d * d + d; }
};

// ---- CUDA-core kernels (simt.cu) -------------------------------------------
// Partial KV summaries. Head bh, split s covers tokens
// [s*tokens_per_split, min(N, (s+1)*tokens_per_split)) and writes the state
// record part[(bh*nsplit + s) * state_floats()].
cudaError_t simt_kv_partial(const Problem& p, const void* k, const void* v, int tokens_per_split,
                            int nsplit, float* part, cudaStream_t st);
// Sums the nsplit records of each head in split order into S [bh][d*d] and
// z [bh][d].
cudaError_t state_reduce(const Problem& p, const float* part, int nsplit, float* S, float* z,
                         cudaStream_t st);
// In place: record b of each head becomes the sum of records 0..b-1 (zero for
// b = 0), or with `reverse` of records b+1..nblk-1. If S_total/z_total are
// non-null they receive the sum of all records.
cudaError_t state_exclusive_scan(const Problem& p, float* part, int nblk, float* S_total,
                                 float* z_total, cudaStream_t st, bool reverse = false);
// out = phi(q) S / (phi(q).z) (or numerator only) for every token.
cudaError_t simt_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                         cudaStream_t st);
// Non-causal outputs of short heads at d <= 32 in one launch (one CTA per
// head: S and z, then the readout); S_out / z_out (both or neither) also
// receive S and z. simt_noncausal_small_supported tells whether a problem
// qualifies on the current device (plan::small_noncausal).
bool simt_noncausal_small_supported(const Problem& p);
cudaError_t simt_noncausal_small(const Problem& p, const void* q, const void* k, const void* v, void* out,
                                 float* S_out, float* z_out, cudaStream_t st);
// Chunked causal / prefix-mask outputs. Block blk of head bh covers tokens
// [blk*block_tokens, ...) and starts from record blk of `prefix` (the state of
// all earlier keys). With perm == nullptr the queries of chunk c are the
// tokens of chunk c (causal); otherwise the queries answered at chunk c are
// perm[b*N + bin_start[b*(nbins+1) + c] ...] with key limits msort at the
// same positions (bin_queries).
cudaError_t simt_chunked(const Problem& p, const void* q, const void* k, const void* v,
                         const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                         const int32_t* bin_start, const int32_t* msort, int nbins, void* out,
                         cudaStream_t st);

// ---- prefix-mask binning (bin.cu) -------------------------------------------
// For each sequence b: clamp m into [0, N-1] (setting FLAG_MASK_RANGE in
// *flags when it had to), bin query i by floor((m_i + 1) / chunk) and write a
// counting-sort permutation perm[b*N ...] plus bin offsets
// bin_start[b*(nbins+1) ...] (nbins = N / chunk + 1); msort[b*N + pos] is
// the clamped m of query perm[b*N + pos] (the mask in sorted order).
cudaError_t bin_queries(const Problem& p, const int32_t* m, int chunk, int nbins, int32_t* perm,
                        int32_t* bin_start, int32_t* msort, uint32_t* flags, cudaStream_t st);

// ---- gradients (bwd.cu) -------------------------------------------------------
// Chunk length of the gradient kernels (block_tokens must be a multiple).
int bwd_chunk(const Problem& p);
// Forward sweep: per block of block_tokens tokens (causal: its state is the
// exclusive prefix (S, z) at index bh*nblk + blk; non-causal: the head totals
// at index bh; S at S + index*s_stride, z at z + index*z_stride), writes dq,
// gn [bh][N][d] and gden [bh][N] (fp32) and the block's own (G, h) record
// grec[(bh*nblk + blk)] (d*d + d floats).
cudaError_t bwd_q(const Problem& p, bool causal, const void* q, const void* k, const void* v, const void* dout,
                  const float* S, const float* z, long long s_stride, long long z_stride, int block_tokens,
                  int nblk, void* dq, float* gn, float* gden, float* grec, cudaStream_t st);
// Reverse sweep: per block, from (G, h) of all later queries (causal: suffix
// state at index bh*nblk + blk; non-causal: totals at index bh), writes dk
// and dv. gn is fp32, or bf16 with gn_bf16 (causal bf16 d = 64 only: the
// tensor-core first sweep's output).
cudaError_t bwd_kv(const Problem& p, bool causal, const void* q, const void* k, const void* v, const void* gn,
                   const float* gden, const float* G, const float* h, long long g_stride, long long h_stride,
                   int block_tokens, int nblk, void* dk, void* dv, cudaStream_t st, bool gn_bf16 = false);

// ---- decode (decode.cu) -------------------------------------------------------
cudaError_t decode_step(const Problem& p, const void* q, const void* k, const void* v, float* S,
                        float* z, void* out, cudaStream_t st);

}  // namespace la
