// la_decode.cu -- one decode token per unit, and the state initialiser.
//
// Decode is the recurrence for a single token (slides "Chunking, causality,
// and parallel prefill", "Prefill and decode": with one token the triangle
// is 1x1 and only the state read plus the local term remain):
//     S' = S + k v^T,        o = q^T S'   ( = q^T S + (q . k) v )
// The step reads the fp32 state once and writes it once, so it is bound by
// memory bandwidth.  The main kernel splits a unit's d_v columns over a few
// CTAs (o[j] only needs column j of S', so no reduction crosses CTAs); each
// thread owns four adjacent columns and a strided set of rows, has all of
// its 128-bit state loads in flight before any arithmetic, reads the q, k
// and v entries it needs itself, updates the rows, stores them back, and
// keeps a partial q^T S' for its columns; the partials of the rows are
// summed by warp shuffles, then across warps in shared memory.
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

// Four consecutive entries as floats: one vector load when p is aligned for
// it (always, for d_v a multiple of 4 and a suitably aligned tensor), else
// four scalar loads.
template <typename T>
__device__ __forceinline__ float4 dec_in4(const T* p);
template <>
__device__ __forceinline__ float4 dec_in4<float>(const float* p) {
    if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) return *reinterpret_cast<const float4*>(p);
    return make_float4(p[0], p[1], p[2], p[3]);
}
template <>
__device__ __forceinline__ float4 dec_in4<__nv_bfloat16>(const __nv_bfloat16* p) {
    if ((reinterpret_cast<uintptr_t>(p) & 7) == 0) {
        const uint2 raw = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    return make_float4(__bfloat162float(p[0]), __bfloat162float(p[1]), __bfloat162float(p[2]), __bfloat162float(p[3]));
}

// Bring the 128-byte line holding p into L2 (a hint: no data is returned).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p) : "memory");
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

// Column-split form: the d_v columns of a unit's state are split over CB
// CTAs, each of which owns all d_k rows of its columns, so o[j] (a sum over
// rows of column j) needs no reduction across CTAs.
//
// Launched as a programmatic dependent of the previous kernel in the stream.
// A CTA may start while that kernel still runs: before griddepcontrol.wait it
// only prefetches its state rows and its q, k, v into L2, and it reads
// nothing before the wait returns.  A prefetch is a hint that moves no data
// into registers or shared memory, and L2 is the device's point of coherence
// for global memory, so a line the previous kernel writes after the prefetch
// is still read correctly after the wait.  The prefetch takes the HBM
// latency of the state off the critical path of a chain of decode launches
// (one per layer, say): CTAs of the next launch take the SM slots of this
// launch's CTAs as they finish, and pull their state towards the SMs while
// the rest of this launch runs.  Measured on B200 at 128 units (d = 128,
// cold state): 3.4 us per launch with the prefetch, 5.0 us without; a
// 32-register budget (eight CTAs per SM) made both the cold and the
// L2-resident step slower than four CTAs per SM.
//
// FDK / FNC fix d_k = d_v and the columns per CTA at compile time (0: taken
// from the arguments): d 64 or 128 with 16, 32 or 64 columns run one batch of
// rows per thread with every index known to the compiler.  NT threads per
// CTA: 256 (four CTAs per SM), or 1024 for few units (fewer, larger CTAs
// launch faster; each thread then holds two rows).
template <typename T, int NR, int FDK, int FNC, int NT = kDecThreads>
__global__ void __launch_bounds__(NT, (NT >= 1024 ? 1 : 4))
    decode_cols_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
                       float* __restrict__ state, int64_t n_units, int dk_arg, int dv_arg, int cb_count) {
    extern __shared__ float sm[];
    float* red = sm;  // [warps][cols of this CTA]
    const int dk = FDK > 0 ? FDK : dk_arg;
    const int dv = FDK > 0 ? FDK : dv_arg;
    const int64_t u = blockIdx.x / cb_count;
    const int cb = static_cast<int>(blockIdx.x % cb_count);
    const int ncol = FNC > 0 ? FNC : dv / cb_count;  // columns of this CTA
    const int cbeg = cb * ncol;
    const int cols4 = ncol >> 2;
    const int rpp = NT / cols4;   // rows per pass
    const int tid = threadIdx.x;
    const int c4 = tid % cols4;
    const int r0 = tid / cols4;
    float4* S = reinterpret_cast<float4*>(state + u * static_cast<int64_t>(dk) * dv + cbeg) + c4;
    const int row4 = dv >> 2;  // float4 per state row
    const T* qu = q + u * dk;
    const T* ku = k + u * dk;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int r = r0; r < dk; r += rpp) prefetch_l2(S + r * row4);
    {
        constexpr int kPer = 128 / static_cast<int>(sizeof(T));  // elements per 128-byte line
        const int i = tid * kPer;
        if (i < dk) {
            prefetch_l2(qu + i);
            prefetch_l2(ku + i);
        }
        if (i < ncol) prefetch_l2(v + u * dv + cbeg + i);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // first batch of this thread's rows: loads in flight before anything else
    float4 sv[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const int r = r0 + i * rpp;
        if (FDK > 0 || r < dk) sv[i] = S[r * row4];
    }
    // each thread reads the q and k entries of its own rows and the v entries
    // of its own columns itself (the CTA's threads share them through L1), so
    // no block barrier stands between the loads and the arithmetic
    const T* vc = v + u * dv + cbeg + 4 * c4;
    const float4 vv = dec_in4<T>(vc);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (FDK > 0) {
        // fixed form: NR rows per thread cover d_k exactly, one batch
        static_assert(NR * (NT / (FNC / 4)) == FDK, "rows per thread");
        float qr[NR], kr[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            qr[i] = dec_in<T>(qu, r0 + i * rpp);
            kr[i] = dec_in<T>(ku, r0 + i * rpp);
        }
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            const int r = r0 + i * rpp;
            float4 s4 = sv[i];
            s4.x = fmaf(kr[i], vv.x, s4.x);
            s4.y = fmaf(kr[i], vv.y, s4.y);
            s4.z = fmaf(kr[i], vv.z, s4.z);
            s4.w = fmaf(kr[i], vv.w, s4.w);
            S[r * row4] = s4;
            acc.x = fmaf(qr[i], s4.x, acc.x);
            acc.y = fmaf(qr[i], s4.y, acc.y);
            acc.z = fmaf(qr[i], s4.z, acc.z);
            acc.w = fmaf(qr[i], s4.w, acc.w);
        }
    } else
#pragma unroll 1
    for (int rb = 0; r0 + rb * rpp < dk; rb += NR) {
        if (rb > 0) {
#pragma unroll
            for (int i = 0; i < NR; ++i) {
                const int r = r0 + (rb + i) * rpp;
                if (r < dk) sv[i] = S[r * row4];
            }
        }
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            const int r = r0 + (rb + i) * rpp;
            if (r < dk) {
                const float kr = dec_in<T>(ku, r), qr = dec_in<T>(qu, r);
                float4 s4 = sv[i];
                s4.x = fmaf(kr, vv.x, s4.x);
                s4.y = fmaf(kr, vv.y, s4.y);
                s4.z = fmaf(kr, vv.z, s4.z);
                s4.w = fmaf(kr, vv.w, s4.w);
                S[r * row4] = s4;
                acc.x = fmaf(qr, s4.x, acc.x);
                acc.y = fmaf(qr, s4.y, acc.y);
                acc.z = fmaf(qr, s4.z, acc.z);
                acc.w = fmaf(qr, s4.w, acc.w);
            }
        }
    }
    // q^T S' over this CTA's rows: first across the lanes of a warp that own
    // the same columns (shuffles), then across the warps (shared memory).
    for (int off = cols4; off < 32; off <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
    }
    const int lane = tid & 31, wid = tid >> 5;
    if (lane < cols4) reinterpret_cast<float4*>(red + wid * ncol)[lane] = acc;
    __syncthreads();
    for (int n = tid; n < ncol; n += NT) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) sum += red[w * ncol + n];
        dec_out<T>(o, u * dv + cbeg + n, sum);
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

template <typename T>
static cudaError_t launch_cols(const T* q, const T* k, const T* v, T* o, float* state, int64_t n_units, int dk,
                               int dv, int cb, bool big, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units * cb), 1, 1);
    cfg.blockDim = dim3(big ? 1024 : kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = sizeof(float) * (big ? 32 * 64 : 1024);  // row partials [warps][columns]
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = tuning().decode_pdl ? 1 : 0;
    const int ncol = dv / cb;
    const bool sq = (dk == dv);
    if (big && dk == 128)  // two 1024-thread CTAs per unit, 64 columns each
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 2, 128, 64, 1024>, q, k, v, o, state, n_units, dk, dv,
                                  cb);
    if (big)  // d = 64: one 1024-thread CTA per unit
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 1, 64, 64, 1024>, q, k, v, o, state, n_units, dk, dv,
                                  cb);
    if (sq && dk == 128 && ncol == 32)
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 4, 128, 32>, q, k, v, o, state, n_units, dk, dv, cb);
    if (sq && dk == 128 && ncol == 16)
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 2, 128, 16>, q, k, v, o, state, n_units, dk, dv, cb);
    if (sq && dk == 64 && ncol == 32)
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 2, 64, 32>, q, k, v, o, state, n_units, dk, dv, cb);
    if (sq && dk == 64 && ncol == 16)
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 1, 64, 16>, q, k, v, o, state, n_units, dk, dv, cb);
    // other shapes: rows per thread held in registers at once, batches of up to 4
    const int rpp = kDecThreads / (ncol / 4);
    const int need = (dk + rpp - 1) / rpp;
    if (need <= 1)
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 1, 0, 0>, q, k, v, o, state, n_units, dk, dv, cb);
    if (need <= 2)
        return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 2, 0, 0>, q, k, v, o, state, n_units, dk, dv, cb);
    return cudaLaunchKernelEx(&cfg, decode_cols_kernel<T, 4, 0, 0>, q, k, v, o, state, n_units, dk, dv, cb);
}

// Column blocks per unit for the 256-thread form: 32 columns per CTA where
// d_v allows it (each row piece one 128-byte line; the best 256-thread shape
// measured on B200 from 128 to 8192 units), more blocks while the grid
// covers the SMs less than about three times.  Every block is a whole number
// of float4 columns.
static int decode_col_blocks(int64_t n_units, int num_sms, int dk, int dv) {
    auto ok = [&](int cb) {
        if (cb < 1 || dv % (4 * cb) != 0) return false;
        const int cols4 = dv / (4 * cb);
        return kDecThreads % cols4 == 0;
    };
    int cb = (dv % 32 == 0 && ok(dv / 32)) ? dv / 32 : 1;
    while (cb < 8 && n_units * cb < 3LL * num_sms && ok(cb * 2)) cb *= 2;
    return ok(cb) ? cb : 0;
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* state,
                          int dtype, int64_t n_units, int dk, int dv, int num_sms, cudaStream_t s) {
    if (n_units <= 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>(n_units < 2147483647 ? n_units : 2147483647);
    const size_t smem = sizeof(float) * (3 * 128 + 1024);
    const int cols4 = dv / 4;
    const bool vec = (dv % 4 == 0) && cols4 > 0 && (kDecThreads % cols4 == 0) &&
                     (reinterpret_cast<uintptr_t>(state) % 16 == 0) &&
                     ((dk + (kDecThreads / cols4) - 1) / (kDecThreads / cols4) <= kDecMaxRowsPerThread);
    // The column split launches n_units * cb CTAs (2^31 at most).
    // LINATTN_DECODE_COLBLOCKS overrides the split (0 = one CTA per unit,
    // without a programmatic launch).
    int cb = (vec && n_units <= (1LL << 27)) ? decode_col_blocks(n_units, num_sms, dk, dv) : 0;
    // Few units: 1024-thread CTAs, two per unit at d = 128 and one at d = 64,
    // when they fit in one wave of two CTAs per SM.  Measured on B200 with a
    // cold state: 128 units of d = 128 3.27 against 4.78 us per step, 32 units
    // of d = 64 2.11 against 2.69 us; at 1024 units and more the 256-thread
    // form is faster.
    bool big = vec && dk == dv &&
               ((dk == 128 && n_units * 2 <= 2LL * num_sms) || (dk == 64 && n_units <= 2LL * num_sms));
    if (big) cb = dk / 64;
    if (vec && tuning().decode_col_blocks >= 0) {
        cb = tuning().decode_col_blocks;
        big = false;
    }
    if (cb > 0 && (dv % (4 * cb) != 0 || kDecThreads % (dv / (4 * cb)) != 0)) cb = 0;
    if (cb > 0) {
        cudaError_t e;
        if (dtype == 0)
            e = launch_cols<float>(static_cast<const float*>(q), static_cast<const float*>(k),
                                   static_cast<const float*>(v), static_cast<float*>(o), state, n_units, dk, dv, cb,
                                   big, s);
        else
            e = launch_cols<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                           static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), state,
                                           n_units, dk, dv, cb, big, s);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
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
