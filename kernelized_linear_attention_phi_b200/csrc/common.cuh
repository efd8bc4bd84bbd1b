// Device helpers shared by the kernels of libla_b200.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

enum { PHI_RELU1 = 0, PHI_IDENTITY = 1, PHI_ELU1 = 2 };
enum { DT_F32 = 0, DT_BF16 = 1 };

// Error-word bits written into the workspace header.
enum : uint32_t { FLAG_MASK_RANGE = 1u };

// Bytes reserved at the start of every workspace (error word + padding).
constexpr size_t WS_HEADER = 256;

// Feature map. relu1: a value whose sign bit is set (negative numbers and
// -0.0) becomes 0, then 1 is added ("nx_f32_linear_attention.nx source",
// la_phi). identity: unchanged.
__device__ __forceinline__ float phi_relu1(float x) {
    return ((__float_as_uint(x) & 0x80000000u) ? 0.0f : x) + 1.0f;
}
// elu1: elu(x) + 1 with alpha = 1, i.e. x + 1 for x > 0 and exp(x)
// otherwise (lineartile 1.0.1, "How It Works"); -0.0 and +0.0 both map to 1.
__device__ __forceinline__ float phi_elu1(float x) { return x > 0.0f ? x + 1.0f : expf(x); }
__device__ __forceinline__ float phi_apply(float x, int phi) {
    return phi == PHI_RELU1 ? phi_relu1(x) : phi == PHI_ELU1 ? phi_elu1(x) : x;
}
// d phi / dx: relu1 1 for x > 0, else 0 (relu's derivative taken as 0 at 0);
// elu1 1 for x > 0, else exp(x); identity 1.
__device__ __forceinline__ float phi_grad(float x, int phi) {
    if (phi == PHI_RELU1) return x > 0.0f ? 1.0f : 0.0f;
    if (phi == PHI_ELU1) return x > 0.0f ? 1.0f : expf(x);
    return 1.0f;
}

// 16-byte vector <-> floats.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
        f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Programmatic dependent launch. Every kernel of the library is launched
// with programmatic stream serialization and calls pdl_wait() after its
// prologue (shared memory, barriers, TMEM), before it touches global memory.
// pdl_wait() waits for the previous kernel on the stream to complete with its
// memory visible, then lets this kernel's own dependents launch: the hardware
// starts them once every CTA of this grid has got that far, so their launch
// and prologue overlap this kernel's work, and their own pdl_wait() still
// waits for this whole grid to complete. (No CTA of this grid is left to
// start by then, so an early dependent never takes an SM from this grid;
// one that is resident on an SM where this grid still holds TMEM waits in its
// allocation until that CTA releases it.)
// A kernel may read memory before its pdl_wait() only when no earlier kernel
// still running can write it: a later kernel of a call may prefetch the
// caller's inputs (no kernel of the call writes them), but the first kernel of
// a call may not, because the kernel before it on the stream can be the last
// kernel of an earlier call whose outputs are this call's inputs.
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// For a kernel (or a warp) that reads nothing the previous kernel of the
// call writes: lets dependents launch without waiting. Memory written by
// kernels that completed before the previous kernel started waiting is
// visible all the same, which covers the caller's inputs of a library call
// (its first kernel waits for them).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Hint: moves the 128-byte line holding p towards L2 (no data returned).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Streaming 16-byte global load (read once: do not keep in L1).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// Copies `rows` rows of a [*, D] tile into a float [rows][LD] shared array,
// converting to fp32 and optionally applying phi. Rows at or beyond `valid`
// are written as 0 (after phi, so a padded key adds nothing to S or z).
template <typename T, int D, int LD>
__device__ __forceinline__ void tile_to_smem(float* dst, const T* src, int rows, int valid,
                                             bool apply_phi, int phi) {
    constexpr int EPV = Vec16<T>::N;
    constexpr int VPR = D / EPV;  // vectors per row
    const int nvec = rows * VPR;
    for (int t = threadIdx.x; t < nvec; t += blockDim.x) {
        const int row = t / VPR;
        const int col = (t % VPR) * EPV;
        float f[EPV];
        if (row < valid) {
            Vec16<T>::unpack(ldg_stream(src + (size_t)row * D + col), f);
            if (apply_phi) {
#pragma unroll
                for (int e = 0; e < EPV; ++e) f[e] = phi_apply(f[e], phi);
            }
        } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) f[e] = 0.0f;
        }
        float4* o = reinterpret_cast<float4*>(dst + row * LD + col);
#pragma unroll
        for (int e = 0; e < EPV; e += 4) o[e / 4] = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
    }
}

}  // namespace la
