// la_prefill_short.cu -- prefill of a few tokens per unit (T <= 16) from a
// saved state: the multi-token form of decode.
//
// The whole input is one chunk of T tokens that starts from state S (slides
// "Chunking, causality, and parallel prefill": "Causal triangle", "Incoming
// and outgoing state"), and within it the kernel follows the recurrence
// itself: with S_t = S + sum_{j <= t} k_j v_j^T,
//     o_t = q_t^T S_t,    S' = S_T
// (the same numbers as q_t^T S + sum_{j <= t} (q_t . k_j) v_j, the causal
// triangle with its diagonal, in exact arithmetic).  Like a decode step, the
// cost is one read and one write of the fp32 state; the T tokens only add
// T (d_k + d_v) inputs.  The d_v columns of a unit's state may be split
// over CB CTAs when there are fewer units than SMs (o_t[j] needs column j
// only, so there is no reduction across CTAs).
//
// One CTA: the token loads are issued first, then the state tile goes in
// flight with asynchronous copies into shared memory (the bytes in flight
// are then not limited by registers); q and k are staged transposed (a
// row's tokens contiguous) and v as is.  Each thread takes four adjacent
// columns and a strided set of rows, and copies exactly those state
// elements, in two groups, so that it starts on the first group's rows
// while the second lands.  For each row it steps through the tokens:
// S[r] += k_t[r] v_t, then o_t's partial += q_t[r] S[r], and it writes the
// final row straight back.  The partials of the rows are summed by warp
// shuffles, then across warps in shared memory.  All arithmetic is fp32.
#include <cuda_bf16.h>

#include "la_device.cuh"
#include "la_internal.h"

namespace la {

namespace {

// Threads per CTA: 256, or 128 for d_k <= 64 when the units alone cover
// the SMs (one column block per unit), where 256 threads would leave each
// thread too few rows to pay for the CTA's fixed steps.  With fewer units
// the columns are split over CTAs and the token staging, shared out over
// the threads, is the longer step: 256 threads there.
constexpr int kShortThreadsMax = 256;
constexpr int short_threads(int dk, int64_t n_units, int num_sms) {
    return dk <= 64 && n_units >= num_sms ? 128 : kShortThreadsMax;
}

template <typename E>
__device__ __forceinline__ float elem_in(const E* p, int64_t i);
template <>
__device__ __forceinline__ float elem_in<float>(const float* p, int64_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float elem_in<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
// Four consecutive outputs: one vector store when p is aligned for it, else
// four scalar stores.
template <typename E>
__device__ __forceinline__ void elem_out4(E* p, float4 x);
template <>
__device__ __forceinline__ void elem_out4<float>(float* p, float4 x) {
    if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
        *reinterpret_cast<float4*>(p) = x;
    } else {
        p[0] = x.x;
        p[1] = x.y;
        p[2] = x.z;
        p[3] = x.w;
    }
}
template <>
__device__ __forceinline__ void elem_out4<__nv_bfloat16>(__nv_bfloat16* p, float4 x) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
    if ((reinterpret_cast<uintptr_t>(p) & 7) == 0) {
        uint2 raw;
        raw.x = *reinterpret_cast<const uint32_t*>(&a);
        raw.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = raw;
    } else {
        p[0] = a.x;
        p[1] = a.y;
        p[2] = b.x;
        p[3] = b.y;
    }
}

// a += s * b, as two paired fp32 FMAs (sm_100)
__device__ __forceinline__ void fma4(float4& a, float s, const float4& b) {
    const float2 ss = make_float2(s, s);
    const float2 lo = __ffma2_rn(ss, make_float2(b.x, b.y), make_float2(a.x, a.y));
    const float2 hi = __ffma2_rn(ss, make_float2(b.z, b.w), make_float2(a.z, a.w));
    a = make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Shared memory (floats) of one CTA: the CTA's state tile [d_k][ncol], q
// and k transposed [d_k][TM] (a row's tokens are contiguous), v [TM][ncol],
// per-warp partial outputs [warps][TM][ncol].
__host__ __device__ constexpr size_t short_smem_floats(int tm, int dk, int ncol, int warps) {
    return static_cast<size_t>(dk) * ncol + 2 * static_cast<size_t>(dk) * tm +
           static_cast<size_t>(tm) * (1 + warps) * ncol;
}

// Bring the 128-byte line holding p into L2 (a hint: no data is returned).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p) : "memory");
}

__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}

// The rows of unit u: dense unit u = group u, rows 0..T-1; packed unit
// n*H + h = head h, rows cu[n] .. cu[n+1]-1 (offsets out of range: empty).
struct ShortUnit {
    int64_t rbase;  // first row in the [groups][rows_per_group] token layout
    int len;
};
__device__ __forceinline__ ShortUnit short_unit(const PrefillProblem& p, int64_t u) {
    if (p.cu == nullptr) return {u * p.rows_per_group, static_cast<int>(p.rows_per_group)};
    const int n = static_cast<int>(u / p.H);
    const int64_t group = u % p.H;
    const int a = p.cu[n], b = p.cu[n + 1];
    const bool bad = a < 0 || b < a || static_cast<int64_t>(b) > p.rows_per_group;
    return {group * p.rows_per_group + (bad ? 0 : a), bad ? 0 : b - a};
}

// Prefetch into L2 the q, k and v rows rbase .. rbase + len - 1 of a unit
// (nothing when len is out of range).
template <typename E, int NT>
__device__ __forceinline__ void short_prefetch_tokens(const PrefillProblem& p, int64_t rbase, int len, int tm,
                                                      int dv) {
    if (len < 1 || len > tm) return;
    constexpr int kPer = 128 / static_cast<int>(sizeof(E));  // elements per 128-byte line
    const E* Q = static_cast<const E*>(p.q) + rbase * p.dk;
    const E* K = static_cast<const E*>(p.k) + rbase * p.dk;
    const E* V = static_cast<const E*>(p.v) + rbase * dv;
    const int nq = len * p.dk, nv = len * dv;
    for (int i = threadIdx.x * kPer; i < nq; i += NT * kPer) {
        prefetch_l2(Q + i);
        prefetch_l2(K + i);
    }
    for (int i = threadIdx.x * kPer; i < nv; i += NT * kPer) prefetch_l2(V + i);
}

// One state row of the recurrence: for t = 0 .. TM-1, S[r] += k_t[r] v_t,
// then acc[t] += q_t[r] S[r] (tokens past the end have q = k = v = 0 and
// change nothing); the final row goes straight back to global memory.
// St / Sg: this CTA's state tile in shared / global memory, row r, this
// thread's four columns 4*c4 .. 4*c4+3.
template <int TM>
__device__ __forceinline__ void short_row(const float* St, float* Sg, int r, int ncol, int dv, int c4,
                                          const float* qT, const float* kT, const float4 (&vv)[TM],
                                          float4 (&acc)[TM]) {
    float4 s = reinterpret_cast<const float4*>(St + r * ncol)[c4];
    const float4* q4 = reinterpret_cast<const float4*>(qT + r * TM);
    const float4* k4 = reinterpret_cast<const float4*>(kT + r * TM);
#pragma unroll
    for (int t4 = 0; t4 < TM / 4; ++t4) {
        const float4 kk = k4[t4], qq = q4[t4];
        fma4(s, kk.x, vv[4 * t4 + 0]);
        fma4(acc[4 * t4 + 0], qq.x, s);
        fma4(s, kk.y, vv[4 * t4 + 1]);
        fma4(acc[4 * t4 + 1], qq.y, s);
        fma4(s, kk.z, vv[4 * t4 + 2]);
        fma4(acc[4 * t4 + 2], qq.z, s);
        fma4(s, kk.w, vv[4 * t4 + 3]);
        fma4(acc[4 * t4 + 3], qq.w, s);
    }
    reinterpret_cast<float4*>(Sg + static_cast<int64_t>(r) * dv)[c4] = s;
}

// o_t = q_t^T S_t for the CTA's columns: the partials of the rows summed by
// lanes that own the same columns (shuffles), then across the warps (shared
// memory, behind one block barrier); each thread writes four adjacent
// outputs.  O points at token 0, column 0 of the unit.
template <typename E, int TM, int NT>
__device__ __forceinline__ void short_reduce_store(float4 (&acc)[TM], float* red, int ncol, int cols4, int len,
                                                   E* O, int dv, int cbeg) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
#pragma unroll
    for (int t = 0; t < TM; ++t) {
        for (int off = cols4; off < 32; off <<= 1) {
            acc[t].x += __shfl_xor_sync(0xffffffffu, acc[t].x, off);
            acc[t].y += __shfl_xor_sync(0xffffffffu, acc[t].y, off);
            acc[t].z += __shfl_xor_sync(0xffffffffu, acc[t].z, off);
            acc[t].w += __shfl_xor_sync(0xffffffffu, acc[t].w, off);
        }
        if (lane < cols4) reinterpret_cast<float4*>(red + (wid * TM + t) * ncol)[lane] = acc[t];
    }
    __syncthreads();
    for (int i = tid; i < len * cols4; i += NT) {
        const int t = i / cols4, c = (i % cols4) * 4;
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) {
            const float4 x = *reinterpret_cast<const float4*>(red + (w * TM + t) * ncol + c);
            sum.x += x.x;
            sum.y += x.y;
            sum.z += x.z;
            sum.w += x.w;
        }
        elem_out4<E>(O + static_cast<int64_t>(t) * dv + cbeg + c, sum);
    }
}

template <typename E, int TM, int NT>
__global__ void __launch_bounds__(NT, (TM <= 8 ? 2 : 1) * (kShortThreadsMax / NT))
    prefill_short_kernel(const PrefillProblem p, int cb_count) {
    extern __shared__ float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    const int dk = p.dk, dv = p.dv;
    const int64_t u = blockIdx.x / cb_count;
    const int ncol = dv / cb_count;
    const int cbeg = static_cast<int>(blockIdx.x % cb_count) * ncol;
    const int cols4 = ncol >> 2;
    const int rpp = NT / cols4;  // rows per pass
    const int tid = threadIdx.x;
    const int c4 = tid % cols4;
    const int r0 = tid / cols4;

    // Launched as a programmatic dependent of the previous kernel in the
    // stream: nothing is read from global memory before griddepcontrol.wait
    // returns (cu_seqlens included: the previous kernel may write it).
    // Before it, a CTA of dense input, whose rows need no lookup, only
    // prefetches its tokens into L2 (a hint; L2 is the point of coherence,
    // so a line the previous kernel writes afterwards is still read
    // correctly).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (p.cu == nullptr)
        short_prefetch_tokens<E, NT>(p, u * p.rows_per_group, static_cast<int>(p.rows_per_group), TM, dv);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const ShortUnit un = short_unit(p, u);
    const int len = un.len;
    if (len == 0) return;
    if (len > TM) {
        // longer than the max_seqlen the caller promised: leave the unit
        // untouched and report it
        if (tid == 0) atomicOr(&g_error_word[0], kErrTooLong);
        return;
    }
    float* St = sm;                   // [dk][ncol]
    float* qT = St + dk * ncol;       // [dk][TM]
    float* kT = qT + dk * TM;         // [dk][TM]
    float* vs = kT + dk * TM;         // [TM][ncol]
    float* red = vs + TM * ncol;      // [NT / 32][TM][ncol]
    const int64_t rbase = un.rbase;
    const E* Q = static_cast<const E*>(p.q) + rbase * dk;
    const E* K = static_cast<const E*>(p.k) + rbase * dk;
    const E* V = static_cast<const E*>(p.v) + rbase * dv;
    E* O = static_cast<E*>(p.o) + rbase * dv;
    float* Sg = p.state + u * static_cast<int64_t>(dk) * dv + cbeg;
    // the token loads first (d_k, d_v <= 128: at most TM * 128 / NT
    // elements of each per thread), in registers until the state copies are
    // issued
    constexpr int kPer = (TM * 128 + NT - 1) / NT;
    float qv[kPer], kv[kPer], vt[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * NT;
        qv[j] = i < len * dk ? elem_in<E>(Q, i) : 0.f;
        kv[j] = i < len * dk ? elem_in<E>(K, i) : 0.f;
        const int t = i / ncol, c = i % ncol;
        vt[j] = (i < TM * ncol && t < len) ? elem_in<E>(V, static_cast<int64_t>(t) * dv + cbeg + c) : 0.f;
    }
    // then the state: this thread's rows r0, r0 + rpp, ... of columns
    // 4*c4 .. 4*c4+3 (the elements it updates), the first nh rows in one
    // group of asynchronous copies and the rest in a second
    const int nrow = (dk - r0 + rpp - 1) / rpp;
    const int nh = (nrow + 1) >> 1;
    for (int i = 0; i < nh; ++i) {
        const int r = r0 + i * rpp;
        cp_async16(St + r * ncol + 4 * c4, Sg + static_cast<int64_t>(r) * dv + 4 * c4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int i = nh; i < nrow; ++i) {
        const int r = r0 + i * rpp;
        cp_async16(St + r * ncol + 4 * c4, Sg + static_cast<int64_t>(r) * dv + 4 * c4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * NT;
        if (i < TM * dk) {  // tokens past the end are zero
            const int t = i / dk, r = i % dk;
            qT[r * TM + t] = qv[j];
            kT[r * TM + t] = kv[j];
        }
        if (i < TM * ncol) vs[i] = vt[j];
    }
    __syncthreads();
    float4 vv[TM];
#pragma unroll
    for (int t = 0; t < TM; ++t) vv[t] = reinterpret_cast<const float4*>(vs + t * ncol)[c4];
    // state pass, row by row (short_row); each thread reads only the state
    // elements it copied, so waiting for its own copies is enough
    float4 acc[TM];
#pragma unroll
    for (int t = 0; t < TM; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
#pragma unroll 1
    for (int i = 0; i < nh; ++i) short_row<TM>(St, Sg, r0 + i * rpp, ncol, dv, c4, qT, kT, vv, acc);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll 1
    for (int i = nh; i < nrow; ++i) short_row<TM>(St, Sg, r0 + i * rpp, ncol, dv, c4, qT, kT, vv, acc);
    short_reduce_store<E, TM, NT>(acc, red, ncol, cols4, len, O, dv, cbeg);
}

// Column blocks per unit: the fewest (so that each CTA stages a large state
// tile) that still give every SM a CTA, each block a whole number of float4
// columns whose count divides the block's nt threads.  0 when d_v does not
// allow it.
int short_col_blocks(int64_t n_units, int num_sms, int dv, int nt) {
    auto ok = [&](int cb) {
        if (dv % (4 * cb) != 0) return false;
        const int cols4 = dv / (4 * cb);
        return cols4 <= 32 && nt % cols4 == 0;
    };
    if (!ok(1)) return 0;
    int cb = 1;
    while (cb < 8 && n_units * cb < num_sms && ok(cb * 2)) cb *= 2;
    return cb;
}

template <typename E, int TM, int NT>
cudaError_t launch_short_tm(const PrefillProblem& p, int cb, cudaStream_t s) {
    auto kern = prefill_short_kernel<E, TM, NT>;
    const size_t smem = short_smem_floats(TM, p.dk, p.dv / cb, NT / 32) * sizeof(float);
    // raise the limit to the largest this instantiation can ask for, once
    // per device (not inside a stream capture: the first launch sets it)
    static PerDeviceOnce attrs;
    cudaError_t e = attrs.run([&] {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(short_smem_floats(TM, 128, 128, NT / 32) * sizeof(float)));
        if (r != cudaSuccess) return r;
        // all of the SM's unified L1/shared storage as shared memory, so that
        // two CTAs with large state tiles can be resident together
        return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.n_units * cb), 1, 1);
    cfg.blockDim = dim3(NT, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, p, cb);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename E, int NT>
cudaError_t launch_short_t(const PrefillProblem& p, int64_t max_tokens, int cb, cudaStream_t s) {
    if (max_tokens <= 4) return launch_short_tm<E, 4, NT>(p, cb, s);
    if (max_tokens <= 8) return launch_short_tm<E, 8, NT>(p, cb, s);
    return launch_short_tm<E, 16, NT>(p, cb, s);
}

}  // namespace

bool prefill_short_supported(int64_t max_tokens, int dk, int dv, const void* state) {
    return max_tokens >= 1 && max_tokens <= kShortMaxTokens && dk >= 1 && dk <= 128 && dv >= 4 && dv <= 128 &&
           (reinterpret_cast<uintptr_t>(state) & 15) == 0 && short_col_blocks(1, 1, dv, kShortThreadsMax) > 0;
}

cudaError_t launch_prefill_short(const PrefillProblem& p, int64_t max_tokens, int num_sms, cudaStream_t s) {
    if (p.n_units <= 0) return cudaSuccess;
    const int nt = short_threads(p.dk, p.n_units, num_sms);
    const int cb = short_col_blocks(p.n_units, num_sms, p.dv, nt);
    if (cb == 0 || p.n_units * cb > 2147483647LL) return cudaErrorInvalidValue;
    if (nt == kShortThreadsMax)
        return p.dtype == 1 ? launch_short_t<__nv_bfloat16, kShortThreadsMax>(p, max_tokens, cb, s)
                            : launch_short_t<float, kShortThreadsMax>(p, max_tokens, cb, s);
    return p.dtype == 1 ? launch_short_t<__nv_bfloat16, 128>(p, max_tokens, cb, s)
                        : launch_short_t<float, 128>(p, max_tokens, cb, s);
}

}  // namespace la
