/*
 * la.h -- C ABI of the B200 (sm_100a) kernelized linear attention library
 *         (libla_b200.so).
 *
 * The method. A positive feature map phi is applied to queries and keys.
 * The keys and values of a head are folded into the KV summary
 *     S = sum_j phi(K_j) (x) V_j      (d x d, row-major S[a*d + b])
 *     z = sum_j phi(K_j)              (d)
 * and each query reads out
 *     out_i = phi(Q_i) S / (phi(Q_i) . z)        (normalize = 1)
 *     out_i = phi(Q_i) S                         (normalize = 0)
 * with no 1/sqrt(d) scale and no epsilon. Sources:
 *   - "nx_f32_linear_attention.nx source": header comment (definitions of phi,
 *     S, z, out), function la_phi (phi = relu(x)+1, relu by the sign bit),
 *     the KV-summary loop and the per-query loop;
 *   - "trim-transformer 0.1.0": introduction (unnormalized Q K^T V with the
 *     identity map), "Masking" (query i sees keys 0..m_i, m_i in [0, n-1];
 *     causal = arange(n)), "Key-value caching" (decode on a stored state);
 *   - "lineartile 1.0.1", "How It Works" (O = phi(Q)(phi(K)^T V)).
 *
 * Conventions shared by every entry point.
 *   - Tensors q, k, v, out are dense, contiguous [B, H, N, d] in the element
 *     type desc->dtype (out has the same type as the inputs). d_k = d_v = d.
 *   - S and z are float32: S [B, H, d, d] row-major per head, z [B, H, d].
 *   - All pointers are device pointers owned by the caller, 16-byte aligned.
 *     The library never allocates device memory and keeps no pointer after
 *     a call returns; scratch space is the caller's workspace (ws), sized by
 *     la_workspace_size(). A workspace starts with an error word that must
 *     be zero when the workspace is first used (see la_last_error); the rest
 *     needs no initialization. Calls that overlap on the GPU need distinct
 *     workspaces.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream). Buffers must stay valid until the stream
 *     reaches the call's work.
 *   - Validation is fail-closed: on any status other than LA_OK nothing was
 *     launched, except LA_ERR_CUDA, which reports a failed launch.
 *   - Supported: d in {16, 32, 64, 128}; dtype LA_F32 or LA_BF16;
 *     phi LA_PHI_RELU1, LA_PHI_IDENTITY or LA_PHI_ELU1; normalize in
 *     {0, 1}, with normalize = 1 only for the positive maps LA_PHI_RELU1 and
 *     LA_PHI_ELU1 (with the identity map the denominator phi(q).z can be
 *     zero or negative). Device: compute
 *     capability 10.x (B200).
 *   - Results are deterministic: every reduction runs in a fixed order, so
 *     repeated calls on the same inputs give bit-identical outputs.
 */
#ifndef LA_B200_H
#define LA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,  /* NULL pointer, size <= 0, unknown enum value */
    LA_ERR_UNSUPPORTED = 2,  /* valid request outside the supported set, or not a CC 10.x device */
    LA_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
    LA_ERR_WORKSPACE = 4,    /* ws is NULL or smaller than la_workspace_size() */
    LA_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
    LA_ERR_MASK_RANGE = 6,   /* (la_last_error) some m_i was outside [0, N-1] */
    LA_ERR_TIMEOUT = 7       /* (la_last_error) a kernel's bounded internal wait expired;
                                the outputs of that call are undefined (internal error) */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

typedef enum {
    LA_PHI_RELU1 = 0,    /* phi(x) = relu(x) + 1, relu by the sign bit (-0.0 -> 1) */
    LA_PHI_IDENTITY = 1, /* phi(x) = x (unnormalized Q K^T V form) */
    LA_PHI_ELU1 = 2      /* phi(x) = elu(x) + 1: x + 1 for x > 0, exp(x) otherwise
                            (lineartile 1.0.1, "How It Works"; elu with alpha = 1) */
} la_phi;

typedef enum {
    LA_OP_KV_SUMMARY = 0,
    LA_OP_NONCAUSAL = 1,
    LA_OP_CAUSAL = 2,
    LA_OP_PREFIX = 3,
    LA_OP_DECODE = 4,
    LA_OP_NONCAUSAL_BWD = 5,  /* la_noncausal_backward */
    LA_OP_CAUSAL_BWD = 6      /* la_causal_backward */
} la_op;

/* Problem description. d is both d_k and d_v. */
typedef struct {
    int32_t B, H, N, d;
    int32_t dtype;      /* la_dtype */
    int32_t phi;        /* la_phi */
    int32_t normalize;  /* 1: divide by phi(q).z; 0: unnormalized */
} la_desc;

/* Bytes of workspace `op` needs for `desc` (chunk is used by LA_OP_CAUSAL and
 * LA_OP_PREFIX only; it must be 64 or 128 for those and is ignored
 * otherwise). Returns 0 when the request is invalid or unsupported, and for
 * ops that need none (LA_OP_DECODE). A valid request that needs a workspace
 * always gets a non-zero size. Host function; launches nothing. The work is
 * split to fill the SMs of the current device, so the size is for that
 * device (with no CUDA device, for a 148-SM B200): a workspace sized on one
 * device can be too small for another, which the call then rejects with
 * LA_ERR_WORKSPACE. */
LA_API size_t la_workspace_size(const la_desc* desc, int32_t op, int32_t chunk);

/* KV summary of every head (nx source, KV-summary loop):
 *   S[b,h] = sum_j phi(K[b,h,j]) (x) V[b,h,j],  z[b,h] = sum_j phi(K[b,h,j]).
 * k, v: [B,H,N,d] inputs. S_out [B,H,d,d], z_out [B,H,d]: float32 outputs,
 * overwritten. desc->normalize is ignored. This is the prefill of a decode
 * state. */
LA_API la_status la_kv_summary(const la_desc* desc, const void* k, const void* v,
                        float* S_out, float* z_out,
                        void* ws, size_t ws_bytes, void* stream);

/* Non-causal attention: every query sees every key of its head.
 *   out_i = phi(q_i) S / (phi(q_i) . z)   (or the numerator alone).
 * q, k, v: [B,H,N,d] inputs; out: [B,H,N,d] output.
 * S_out, z_out: optional (may be NULL) float32 outputs receiving the KV
 * summary used, so that a decode can continue from it. */
LA_API la_status la_noncausal(const la_desc* desc, const void* q, const void* k,
                       const void* v, void* out, float* S_out, float* z_out,
                       void* ws, size_t ws_bytes, void* stream);

/* Causal attention: query i sees keys 0..i (inclusive; trim-transformer
 * "Masking": the causal mask is arange(n)). Computed chunk by chunk: the
 * intra-chunk part (phi(Q_c) phi(K_c)^T, lower triangle with diagonal) times
 * V_c, plus phi(Q_c) times the state of all earlier chunks.
 * chunk: 64 or 128 tokens. The result does not depend on it beyond rounding.
 * q, k, v: [B,H,N,d] inputs; out: [B,H,N,d] output. */
LA_API la_status la_causal_chunked(const la_desc* desc, int32_t chunk, const void* q,
                            const void* k, const void* v, void* out,
                            void* ws, size_t ws_bytes, void* stream);

/* Causal prefill (trim-transformer 0.1.0, "Key-value caching": the cache
 * built over a prompt is what the one-token steps continue from): the same
 * outputs as la_causal_chunked, and in the same pass the state after the last
 * token, S_out = sum_j phi(k_j)^T v_j and z_out = sum_j phi(k_j) over all N
 * keys, float32 [B,H,d,d] and [B,H,d], overwritten, ready for
 * la_decode_step. Same arguments, workspace (op LA_OP_CAUSAL) and errors as
 * la_causal_chunked, plus LA_ERR_INVALID_ARG for a NULL S_out or z_out and
 * LA_ERR_MISALIGNED when either is not 16-byte aligned. */
LA_API la_status la_causal_prefill(const la_desc* desc, int32_t chunk, const void* q,
                                   const void* k, const void* v, void* out, float* S_out,
                                   float* z_out, void* ws, size_t ws_bytes, void* stream);

/* Gradients of the non-causal and causal forms (the training path; the
 * pages list a backward pass, lineartile 1.0.1 "Project Structure":
 * core/kernels/backward.py, without its formulas, so these are the
 * derivatives of the forward definition above). Given dout = dL/dout
 * ([B,H,N,d], input dtype), writes dq, dk, dv ([B,H,N,d], input dtype,
 * overwritten) for the same desc (phi and normalize) and q, k, v as the
 * forward call. With a = phi(q), b = phi(k), g = dout:
 *   gn_i = g_i / den_i, gden_i = -(g_i . out_i) / den_i   (normalize = 1;
 *   else gn_i = g_i, gden_i = 0)
 *   dq_i = phi'(q_i) * (S_i gn_i + z_i gden_i)
 *   dk_j = phi'(k_j) * (G_j v_j + h_j),  dv_j = G_j^T b_j
 * where S_i, z_i are the state of the keys query i sees and G_j =
 * sum a_i gn_i^T, h_j = sum a_i gden_i over the queries that see key j
 * (non-causal: every query; causal: i >= j). phi' is 1 for x > 0 and 0
 * otherwise for relu+1 (relu's derivative taken as 0 at 0), 1 for the
 * identity, 1 for x > 0 and exp(x) otherwise for elu+1. Products and sums
 * are fp32. Workspace: op LA_OP_NONCAUSAL_BWD / LA_OP_CAUSAL_BWD (it holds,
 * among others, gn and gden in fp32: (d + 1) * 4 bytes per token and head).
 * Errors as for the forward calls (NULL or misaligned dout, dq, dk, dv
 * included). */
LA_API la_status la_noncausal_backward(const la_desc* desc, const void* q, const void* k,
                                       const void* v, const void* dout, void* dq, void* dk,
                                       void* dv, void* ws, size_t ws_bytes, void* stream);
LA_API la_status la_causal_backward(const la_desc* desc, const void* q, const void* k,
                                    const void* v, const void* dout, void* dq, void* dk,
                                    void* dv, void* ws, size_t ws_bytes, void* stream);

/* Prefix-mask attention (trim-transformer 0.1.0, "Masking"): query i of
 * sequence b sees keys 0..m[b*N + i], inclusive. m: int32 [B, N] device
 * array with values in [0, N-1], one mask per sequence shared by its heads.
 * An m_i outside that range is clamped into it and recorded in the
 * workspace's error word (read it with la_last_error). m = arange(N) is the
 * causal mask; m = N-1 everywhere is non-causal.
 * chunk: 64 or 128 (queries are binned by floor((m_i+1)/chunk)). */
LA_API la_status la_prefix_mask(const la_desc* desc, int32_t chunk, const void* q,
                         const void* k, const void* v, const int32_t* m,
                         void* out, void* ws, size_t ws_bytes, void* stream);

/* One recurrent decode step for every (b, h), on a cached state
 * (trim-transformer 0.1.0, "Key-value caching"; update first, so the new
 * token sees itself):
 *   S += phi(k) (x) v;  z += phi(k);  out = phi(q) S / (phi(q) . z).
 * q, k, v: [B,H,1,d] inputs (desc->N is ignored); S [B,H,d,d] and
 * z [B,H,d]: float32 state, updated in place; out: [B,H,1,d] output.
 * Zero-filled S and z are the empty cache. Needs no workspace. */
LA_API la_status la_decode_step(const la_desc* desc, const void* q, const void* k,
                         const void* v, float* S, float* z, void* out,
                         void* stream);

/* la_kv_summary without a caller workspace, for callers that cannot allocate
 * device memory: code that runs where cudaMalloc is off limits (inside a
 * stream capture, in a real-time path that must not allocate, or behind a
 * host framework that owns every device allocation and hands the caller only
 * its tensors). The pages describe no such variant; it exists for these
 * callers only.
 *
 * Same inputs, outputs, result and argument checks as la_kv_summary. The
 * scratch the KV summary needs lives in a device array of 32 MiB inside the
 * library, which every GPU that loads the library holds until the process
 * exits; a problem whose la_workspace_size(desc, LA_OP_KV_SUMMARY, 0)
 * exceeds 32 MiB is rejected with LA_ERR_WORKSPACE before anything is
 * launched. The call allocates nothing: it issues a 4-byte cudaMemsetAsync
 * (clearing the array's error word), the KV-summary kernels and one small
 * kernel that checks the error word.
 * - The first call in each CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress, with that context current) and keeps it for that
 *   context; make that first call before any stream capture. A device reset
 *   creates a new context, whose first call looks the address up again.
 * - All calls share the one array, which keeps the last call's contents:
 *   calls that may overlap on the GPU (different streams, or different host
 *   threads) race and give undefined results; serialize them.
 * - An expired bounded wait (an internal error; see LA_ERR_TIMEOUT) fills
 *   S_out and z_out with NaN: this call has no workspace that la_last_error
 *   could read. */
LA_API la_status la_kv_summary_static(const la_desc* desc, const void* k, const void* v,
                                      float* S_out, float* z_out, void* stream);

/* Waits for `stream`, then reads and clears the error word of workspace `ws`.
 * The error word is the first 4 bytes of a workspace; it is sticky: the
 * calls that use the workspace only set bits in it, so the caller zeroes it
 * once when allocating the workspace, and la_last_error reports everything
 * since the previous read. *flags_out (may be NULL) receives the raw bits:
 * bit 0 = a mask value was out of range (la_prefix_mask); bit 1 = a
 * kernel's bounded wait on its own asynchronous copies or tensor-core
 * operations expired and the kernel returned early. Returns LA_ERR_TIMEOUT
 * when bit 1 was set, else LA_ERR_MASK_RANGE when bit 0 was set, LA_OK when
 * no bit was set, LA_ERR_CUDA on a CUDA failure. */
LA_API la_status la_last_error(void* ws, void* stream, uint32_t* flags_out);

/* Per-kernel timing, a measurement aid with no counterpart in the method.
 * While enabled, every entry point records a CUDA event on its stream before
 * its first kernel and one after each kernel it launches (16 at most per
 * call). The events are the library's own, created by la_timing_enable(1) on
 * the current device (LA_ERR_CUDA if that fails); la_timing_enable(0) stops
 * the recording. Under stream capture the records become event nodes of the
 * graph and are taken again at each replay; an event node between two kernels
 * ends the overlap of the second kernel's start with the first one's end, so
 * timed calls can run slightly slower than untimed ones. The state is global
 * to the process: only one call at a time may run while timing is on.
 *
 * la_timing_read waits for the last call's (or the last replay's) final
 * event, then writes the duration in milliseconds of its kernel i (from the
 * event before it to the event after it) to ms[i] for i < capacity, and the
 * number of kernels that call launched to *count (0 if no call was recorded).
 * Returns LA_ERR_INVALID_ARG for a NULL count, a negative capacity or a NULL
 * ms with capacity > 0, LA_ERR_CUDA on a CUDA failure. */
LA_API la_status la_timing_enable(int32_t enable);
LA_API la_status la_timing_read(float* ms, int32_t capacity, int32_t* count);

/* Static string naming a status. */
LA_API const char* la_status_string(la_status status);

/* ABI version: major * 10000 + minor * 100 + patch. */
LA_API int32_t la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_B200_H */
