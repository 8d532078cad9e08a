// la_decode.cu -- one decode token per unit, and the state initialiser.
//
// Decode is the recurrence for a single token (slides "Chunking, causality,
// and parallel prefill", "Prefill and decode": with one token the triangle
// is 1x1 and only the state read plus the local term remain):
//     S' = S + k v^T,        o = q^T S'   ( = q^T S + (q . k) v )
// The step reads the fp32 state once and writes it once, so it is bound by
// memory bandwidth.  A block owns one unit: each thread owns four adjacent
// columns of the state and a strided set of its rows, issues all of its
// 128-bit state loads before any arithmetic (so they are in flight
// together), updates the rows, stores them back, and keeps a partial
// q^T S' for its columns; the partials of the rows are summed in shared
// memory.
#include <cuda_bf16.h>

#include "la_internal.h"

namespace la {

template <typename T>
__device__ __forceinline__ float dec_in(const T* p, int64_t i);
template <>
__device__ __forceinline__ float dec_in<float>(const float* p, int64_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float dec_in<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void dec_out(T* p, int64_t i, float x);
template <>
__device__ __forceinline__ void dec_out<float>(float* p, int64_t i, float x) {
    p[i] = x;
}
template <>
__device__ __forceinline__ void dec_out<__nv_bfloat16>(__nv_bfloat16* p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

constexpr int kDecThreads = 256;
constexpr int kDecMaxRowsPerThread = 16;

// Vector form: d_v / 4 divides 256, state rows 16-byte aligned.
template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_vec_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                 const T* __restrict__ v, T* __restrict__ o,
                                                                 float* __restrict__ state, int64_t n_units,
                                                                 int dk, int dv) {
    extern __shared__ float sm[];
    float* qs = sm;
    float* ks = qs + 128;
    float* vs = ks + 128;
    float* red = vs + 128;  // [rows per pass][dv]
    const int tid = threadIdx.x;
    const int cols4 = dv >> 2;
    const int rpp = kDecThreads / cols4;
    const int c4 = tid % cols4;
    const int r0 = tid / cols4;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        for (int i = tid; i < dk; i += kDecThreads) {
            qs[i] = dec_in<T>(q, u * dk + i);
            ks[i] = dec_in<T>(k, u * dk + i);
        }
        for (int i = tid; i < dv; i += kDecThreads) vs[i] = dec_in<T>(v, u * dv + i);
        float4* S = reinterpret_cast<float4*>(state + u * static_cast<int64_t>(dk) * dv);
        float4 sv[kDecMaxRowsPerThread];
#pragma unroll
        for (int i = 0; i < kDecMaxRowsPerThread; ++i) {
            const int r = r0 + i * rpp;
            if (r < dk) sv[i] = S[r * cols4 + c4];
        }
        __syncthreads();
        const float4 vv = make_float4(vs[4 * c4], vs[4 * c4 + 1], vs[4 * c4 + 2], vs[4 * c4 + 3]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kDecMaxRowsPerThread; ++i) {
            const int r = r0 + i * rpp;
            if (r < dk) {
                const float kr = ks[r], qr = qs[r];
                float4 s = sv[i];
                s.x = fmaf(kr, vv.x, s.x);
                s.y = fmaf(kr, vv.y, s.y);
                s.z = fmaf(kr, vv.z, s.z);
                s.w = fmaf(kr, vv.w, s.w);
                S[r * cols4 + c4] = s;
                acc.x = fmaf(qr, s.x, acc.x);
                acc.y = fmaf(qr, s.y, acc.y);
                acc.z = fmaf(qr, s.z, acc.z);
                acc.w = fmaf(qr, s.w, acc.w);
            }
        }
        if (r0 < rpp) reinterpret_cast<float4*>(red + r0 * dv)[c4] = acc;
        __syncthreads();
        for (int n = tid; n < dv; n += kDecThreads) {
            float sum = 0.f;
            for (int rr = 0; rr < rpp && rr < dk; ++rr) sum += red[rr * dv + n];
            dec_out<T>(o, u * dv + n, sum);
        }
        __syncthreads();
    }
}

// Scalar form for any d_k, d_v <= 128 and any alignment.
template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_scalar_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                    const T* __restrict__ v, T* __restrict__ o,
                                                                    float* __restrict__ state, int64_t n_units,
                                                                    int dk, int dv) {
    extern __shared__ float sm[];
    float* qs = sm;
    float* ks = qs + 128;
    float* vs = ks + 128;
    float* red = vs + 128;  // [rows per pass][dv]
    const int tid = threadIdx.x;
    const int rpp = kDecThreads / dv;
    const int c = tid % dv;
    const int r0 = tid / dv;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        for (int i = tid; i < dk; i += kDecThreads) {
            qs[i] = dec_in<T>(q, u * dk + i);
            ks[i] = dec_in<T>(k, u * dk + i);
        }
        for (int i = tid; i < dv; i += kDecThreads) vs[i] = dec_in<T>(v, u * dv + i);
        __syncthreads();
        float* S = state + u * static_cast<int64_t>(dk) * dv;
        float acc = 0.f;
        if (r0 < rpp) {
            for (int r = r0; r < dk; r += rpp) {
                const float s = fmaf(ks[r], vs[c], S[r * dv + c]);
                S[r * dv + c] = s;
                acc = fmaf(qs[r], s, acc);
            }
            red[r0 * dv + c] = acc;
        }
        __syncthreads();
        for (int n = tid; n < dv; n += kDecThreads) {
            float sum = 0.f;
            for (int rr = 0; rr < rpp && rr < dk; ++rr) sum += red[rr * dv + n];
            dec_out<T>(o, u * dv + n, sum);
        }
        __syncthreads();
    }
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* state,
                          int dtype, int64_t n_units, int dk, int dv, int num_sms, cudaStream_t s) {
    (void)num_sms;
    if (n_units <= 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>(n_units < 2147483647 ? n_units : 2147483647);
    const size_t smem = sizeof(float) * (3 * 128 + 1024);
    const int cols4 = dv / 4;
    const bool vec = (dv % 4 == 0) && cols4 > 0 && (kDecThreads % cols4 == 0) &&
                     (reinterpret_cast<uintptr_t>(state) % 16 == 0) &&
                     ((dk + (kDecThreads / cols4) - 1) / (kDecThreads / cols4) <= kDecMaxRowsPerThread);
    if (dtype == 0) {
        const float *qq = static_cast<const float*>(q), *kk = static_cast<const float*>(k),
                    *vv = static_cast<const float*>(v);
        float* oo = static_cast<float*>(o);
        if (vec)
            decode_vec_kernel<float><<<grid, kDecThreads, smem, s>>>(qq, kk, vv, oo, state, n_units, dk, dv);
        else
            decode_scalar_kernel<float><<<grid, kDecThreads, smem, s>>>(qq, kk, vv, oo, state, n_units, dk, dv);
    } else {
        const __nv_bfloat16 *qq = static_cast<const __nv_bfloat16*>(q),
                            *kk = static_cast<const __nv_bfloat16*>(k),
                            *vv = static_cast<const __nv_bfloat16*>(v);
        __nv_bfloat16* oo = static_cast<__nv_bfloat16*>(o);
        if (vec)
            decode_vec_kernel<__nv_bfloat16><<<grid, kDecThreads, smem, s>>>(qq, kk, vv, oo, state, n_units, dk, dv);
        else
            decode_scalar_kernel<__nv_bfloat16><<<grid, kDecThreads, smem, s>>>(qq, kk, vv, oo, state, n_units, dk, dv);
    }
    return cudaGetLastError();
}

// S_0: copy of `src`, or zero.
__global__ void state_init_kernel(float* __restrict__ state, const float* __restrict__ src, int64_t n) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const bool vec = ((reinterpret_cast<uintptr_t>(state) | reinterpret_cast<uintptr_t>(src)) & 15) == 0;
    if (vec) {
        const int64_t n4 = n / 4;
        float4* d4 = reinterpret_cast<float4*>(state);
        const float4* s4 = reinterpret_cast<const float4*>(src);
        for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4; i += stride)
            d4[i] = src ? s4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t i = n4 * 4 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
            state[i] = src ? src[i] : 0.f;
    } else {
        for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
            state[i] = src ? src[i] : 0.f;
    }
}

cudaError_t launch_state_init(float* state, const float* src, int64_t n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    int64_t blocks = (n / 4 + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 16) blocks = 148 * 16;
    state_init_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(state, src, n);
    return cudaGetLastError();
}

}  // namespace la
