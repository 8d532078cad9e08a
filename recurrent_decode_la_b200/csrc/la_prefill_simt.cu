// la_prefill_simt.cu -- chunkwise prefill on the CUDA cores in fp32.
//
// Same chunk algebra as the tensor-core kernel (slides "Chunking, causality,
// and parallel prefill", "Split into chunks"), for any 1 <= d_k, d_v <= 128
// and any chunk size whose tiles fit in shared memory:
//     M   = tril(Q_c K_c^T)               (j <= i, diagonal kept)
//     O_c = M V_c + Q_c S_{c-1}
//     S_c = S_{c-1} + K_c^T V_c
// Inputs are widened to fp32 and every product is accumulated in fp32, so
// small integer inputs (the slides' 8-token trace) come out exact.  Used for
// fp32 inputs (where tf32 tensor cores cannot meet a 1e-4 error bound) and
// for bf16 shapes the tensor-core kernel does not cover.
#include <cuda_bf16.h>

#include "la_internal.h"

namespace la {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
    return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
    return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

size_t prefill_simt_smem_bytes(int dk, int dv, int chunk) {
    // S [dk][dv], Q_c [C][dk], K_c [C][dk], V_c [C][dv], M [C][C]
    return sizeof(float) * (static_cast<size_t>(dk) * dv + static_cast<size_t>(chunk) * (2 * dk + dv) +
                            static_cast<size_t>(chunk) * chunk);
}

template <typename T>
__global__ void __launch_bounds__(256) prefill_simt_kernel(PrefillProblem p) {
    extern __shared__ float sm[];
    const int dk = p.dk, dv = p.dv, C = p.chunk;
    float* S = sm;
    float* Qc = S + dk * dv;
    float* Kc = Qc + C * dk;
    float* Vc = Kc + C * dk;
    float* M = Vc + C * dv;
    const T* q = static_cast<const T*>(p.q);
    const T* k = static_cast<const T*>(p.k);
    const T* v = static_cast<const T*>(p.v);
    T* o = static_cast<T*>(p.o);
    const int tid = threadIdx.x, nt = blockDim.x;

    for (int64_t u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        int64_t group = u, row0 = 0, len = p.rows_per_group;
        if (p.cu) {
            const int n = static_cast<int>(u / p.H);
            group = u % p.H;
            const int a = p.cu[n], b = p.cu[n + 1];
            if (a < 0 || b < a || static_cast<int64_t>(b) > p.rows_per_group) continue;
            row0 = a;
            len = b - a;
        }
        if (len == 0) continue;
        float* st = p.state + u * static_cast<int64_t>(dk) * dv;
        for (int i = tid; i < dk * dv; i += nt) S[i] = st[i];
        const int64_t base = group * p.rows_per_group + row0;  // first row of the unit
        for (int64_t c0 = 0; c0 < len; c0 += C) {
            const int nv = static_cast<int>(len - c0 < C ? len - c0 : C);
            __syncthreads();
            for (int i = tid; i < C * dk; i += nt) {
                const int r = i / dk, d = i % dk;
                const bool in = r < nv;
                Qc[i] = in ? to_f32<T>(q[(base + c0 + r) * dk + d]) : 0.f;
                Kc[i] = in ? to_f32<T>(k[(base + c0 + r) * dk + d]) : 0.f;
            }
            for (int i = tid; i < C * dv; i += nt) {
                const int r = i / dv, d = i % dv;
                Vc[i] = r < nv ? to_f32<T>(v[(base + c0 + r) * dv + d]) : 0.f;
            }
            __syncthreads();
            // M = tril(Q_c K_c^T): entries above the diagonal are never formed.
            for (int i = tid; i < nv * nv; i += nt) {
                const int r = i / nv, j = i % nv;
                float acc = 0.f;
                if (j <= r)
                    for (int d = 0; d < dk; ++d) acc = fmaf(Qc[r * dk + d], Kc[j * dk + d], acc);
                M[r * C + j] = acc;
            }
            __syncthreads();
            // O_c = M V_c + Q_c S_{c-1}
            for (int i = tid; i < nv * dv; i += nt) {
                const int r = i / dv, n = i % dv;
                float intra = 0.f, inter = 0.f;
                for (int j = 0; j <= r; ++j) intra = fmaf(M[r * C + j], Vc[j * dv + n], intra);
                for (int d = 0; d < dk; ++d) inter = fmaf(Qc[r * dk + d], S[d * dv + n], inter);
                o[(base + c0 + r) * dv + n] = from_f32<T>(intra + inter);
            }
            __syncthreads();
            // S_c = S_{c-1} + K_c^T V_c
            for (int i = tid; i < dk * dv; i += nt) {
                const int d = i / dv, n = i % dv;
                float acc = 0.f;
                for (int j = 0; j < nv; ++j) acc = fmaf(Kc[j * dk + d], Vc[j * dv + n], acc);
                S[i] += acc;
            }
        }
        __syncthreads();
        for (int i = tid; i < dk * dv; i += nt) st[i] = S[i];
        __syncthreads();
    }
}

cudaError_t launch_prefill_simt(const PrefillProblem& p, int num_sms, cudaStream_t s) {
    const size_t smem = prefill_simt_smem_bytes(p.dk, p.dv, p.chunk);
    int64_t grid = p.n_units < 4 * static_cast<int64_t>(num_sms) ? p.n_units : 4 * static_cast<int64_t>(num_sms);
    if (grid < 1) return cudaSuccess;
    if (p.dtype == 0) {
        cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        prefill_simt_kernel<float><<<static_cast<unsigned>(grid), 256, smem, s>>>(p);
    } else {
        cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        prefill_simt_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), 256, smem, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace la
