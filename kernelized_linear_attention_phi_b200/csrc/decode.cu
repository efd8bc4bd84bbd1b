// One recurrent decode step on a cached (S, z) state, every (b, h) at once
// ("trim-transformer 0.1.0", "Key-value caching"; update, then read out):
//   S += phi(k) (x) v;  z += phi(k);  out = phi(q) S / (phi(q) . z).
//
// Bandwidth-bound: each step must read and write the d x d fp32 state once
// (64 KiB per head at d = 128) and touches nothing else of note, so the
// kernel is one streaming read-modify-write pass over S with the readout's
// column sums formed on the way. One CTA per head; a warp covers whole
// 512-byte rows (d = 128) with 16-byte accesses.

#include "common.cuh"
#include "internal.h"
#include "launch_util.h"

namespace la {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld_cs(const float4* p) {
    float4 r;
    asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_cs(float4* p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
              float* __restrict__ S, float* __restrict__ z, T* __restrict__ out, int phi,
              int normalize) {
    constexpr int NCG = D / 4;            // float4 column groups per row
    constexpr int NRG = kThreads / NCG;   // row groups
    constexpr int RPT = (D + NRG - 1) / NRG;
    __shared__ float spk[D], spq[D], sv[D];
    __shared__ __align__(16) float red[NRG][D];
    __shared__ float sden[kThreads / 32];
    const long long bh = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_wait();
    if (tid < D) {
        spk[tid] = phi_apply(to_f32<T>(k[bh * D + tid]), phi);
        spq[tid] = phi_apply(to_f32<T>(q[bh * D + tid]), phi);
        sv[tid] = to_f32<T>(v[bh * D + tid]);
    }
    __syncthreads();
    float dpart = 0.f;
    if (tid < D) {
        const float zn = z[bh * D + tid] + spk[tid];
        z[bh * D + tid] = zn;
        dpart = spq[tid] * zn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dpart += __shfl_xor_sync(0xffffffffu, dpart, o);
    if ((tid & 31) == 0) sden[tid >> 5] = dpart;

    const int cg = tid % NCG, rg = tid / NCG;
    const float4 vv = make_float4(sv[cg * 4], sv[cg * 4 + 1], sv[cg * 4 + 2], sv[cg * 4 + 3]);
    float4* Sh = reinterpret_cast<float4*>(S + bh * (long long)D * D);
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int a = rg + r * NRG;
        if (a < D) s[r] = ld_cs(Sh + a * NCG + cg);
    }
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int a = rg + r * NRG;
        if (a < D) {
            const float pk = spk[a], pq = spq[a];
            s[r].x = fmaf(pk, vv.x, s[r].x);
            s[r].y = fmaf(pk, vv.y, s[r].y);
            s[r].z = fmaf(pk, vv.z, s[r].z);
            s[r].w = fmaf(pk, vv.w, s[r].w);
            st_cs(Sh + a * NCG + cg, s[r]);
            num.x = fmaf(pq, s[r].x, num.x);
            num.y = fmaf(pq, s[r].y, num.y);
            num.z = fmaf(pq, s[r].z, num.z);
            num.w = fmaf(pq, s[r].w, num.w);
        }
    }
    *reinterpret_cast<float4*>(&red[rg][cg * 4]) = num;
    __syncthreads();
    if (tid < D) {
        float acc = 0.f;
#pragma unroll
        for (int g = 0; g < NRG; ++g) acc += red[g][tid];
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) den += sden[w];
        out[bh * D + tid] = from_f32<T>(normalize ? acc / den : acc);
    }
}

template <typename T, int D>
cudaError_t launch_decode(const Problem& p, const void* q, const void* k, const void* v, float* S,
                          float* z, void* out, cudaStream_t st) {
    return launch_pdl(decode_kernel<T, D>, dim3((unsigned)p.bh()), dim3(kThreads), 0, st,
                      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), S, z,
                      static_cast<T*>(out), p.phi, p.normalize);
}

}  // namespace

cudaError_t decode_step(const Problem& p, const void* q, const void* k, const void* v, float* S,
                        float* z, void* out, cudaStream_t st) {
    if (p.dtype == DT_F32) {
        switch (p.d) {
            case 16: return launch_decode<float, 16>(p, q, k, v, S, z, out, st);
            case 32: return launch_decode<float, 32>(p, q, k, v, S, z, out, st);
            case 64: return launch_decode<float, 64>(p, q, k, v, S, z, out, st);
            case 128: return launch_decode<float, 128>(p, q, k, v, S, z, out, st);
        }
    } else {
        switch (p.d) {
            case 16: return launch_decode<__nv_bfloat16, 16>(p, q, k, v, S, z, out, st);
            case 32: return launch_decode<__nv_bfloat16, 32>(p, q, k, v, S, z, out, st);
            case 64: return launch_decode<__nv_bfloat16, 64>(p, q, k, v, S, z, out, st);
            case 128: return launch_decode<__nv_bfloat16, 128>(p, q, k, v, S, z, out, st);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace la
