// la_api.cu -- the C ABI of liblinattn.so (declared in include/linattn.h):
// argument checks, kernel choice, TMA descriptors and launches.  Host code
// only; every step of the computation runs in the kernels.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "../../include/linattn.h"
#include "la_device.cuh"
#include "la_internal.h"

// Scratch of la_prefill_noalloc: a static device buffer, so that entry point
// allocates nothing.  In host code this name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress (per device).
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

namespace la {

__device__ unsigned int g_error_word[2];

const Tuning& tuning() {
    // C++ guarantees this initialiser runs once, even with concurrent callers.
    static const Tuning t = [] {
        auto get = [](const char* name) -> const char* {
            const char* e = getenv(name);
            return e && *e ? e : nullptr;
        };
        Tuning v;
        const char* e = get("LINATTN_CHUNK");
        v.chunk = e ? atoi(e) : 0;
        e = get("LINATTN_SHORT");
        v.short_kernel = !(e && e[0] == '0');
        e = get("LINATTN_SPLIT");
        v.split = !(e && e[0] == '0');
        e = get("LINATTN_PREFETCH");
        v.prefetch = e ? atoi(e) : 1;  // one chunk ahead: measured best on B200 (deeper thrashes L2)
        if (v.prefetch < 0) v.prefetch = 0;
        e = get("LINATTN_DECODE_COLBLOCKS");
        v.decode_col_blocks = e ? atoi(e) : -1;
        e = get("LINATTN_DECODE_PDL");
        v.decode_pdl = !(e && e[0] == '0');
        e = get("LINATTN_WAIT_TIMEOUT_MS");
        double ms = e ? atof(e) : 4000.0;
        if (!(ms > 0)) ms = 4000.0;
        v.wait_timeout_ns = static_cast<uint64_t>(ms * 1e6);
        return v;
    }();
    return t;
}

namespace {

thread_local char g_last_cuda_error[256] = "";

la_status cuda_fail(cudaError_t e) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return LA_ERR_CUDA;
}

int current_sm_count() {
    static std::atomic<int> cache[64];  // static storage: zero-initialised
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// The calling thread's current CUDA context (nullptr if the driver entry
// point cannot be found or no context is current).
CUcontext current_context() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    });
    CUcontext c = nullptr;
    if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// 3-D bf16 view (d, rows, groups) of a [groups][rows][d] tensor, box
// (64, chunk, 1), 128-byte swizzle: one box fills one swizzled smem panel.
bool encode_bf16_map(CUtensorMap* map, const void* base, int d, int64_t rows, int64_t groups, int chunk) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(chunk), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int default_chunk(la_dtype dtype, int dk, int dv) {
    if (tuning().chunk > 0) return tuning().chunk;
    // bf16 tensor-core path: 128-token chunks run full-rate M = 128 MMAs with
    // P kept in tensor memory (the measured fastest chunk on B200).
    if (dtype == LA_BF16 && dk == dv && (dk == 64 || dk == 128)) return 128;
    return dk <= 32 && dv <= 32 ? 32 : 16;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Event-trace buffer of the tensor-core prefill; set only through the
// debugging hook of LINATTN_TRACE builds.
struct TraceBuf {
    unsigned long long* buf = nullptr;
    unsigned int* count = nullptr;
    unsigned int cap = 0;
};
TraceBuf g_trace;

// Intra-sequence split plan (dense bf16 tensor-core input with fewer units
// than SMs): seg_count segments per unit run as separate work items, each
// starting from S_0 plus the K^T V sums of the sub-segments before it.
struct SplitPlan {
    int seg_count = 1;
    int64_t seg_len = 0;
    int64_t sub_len = 0;
    int subs_per_seg = 0;
    int subs_per_unit = 0;
    size_t bytes = 0;
};

SplitPlan plan_split(int64_t n_units, int64_t T, int dk, int dv, int chunk, int sms) {
    SplitPlan sp;
    sp.seg_len = T;
    if (!tuning().split) return sp;
    if (n_units <= 0 || T <= 0) return sp;
    const int64_t nch = (T + chunk - 1) / chunk;
    int64_t P = sms / n_units;
    if (P > 8) P = 8;
    if (P > nch / 4) P = nch / 4;  // at least four chunks per segment
    if (P < 2) return sp;
    const int64_t seg_chunks = (nch + P - 1) / P;
    const int64_t seg_len = seg_chunks * chunk;
    P = (T + seg_len - 1) / seg_len;
    if (P < 2) return sp;
    // sub-segments: enough work items for the first pass to cover the SMs
    const int64_t base_items = n_units * (P - 1);
    int k = 1;
    while (k < 16 && base_items * k < 3LL * sms && seg_chunks % (2 * k) == 0) k *= 2;
    sp.seg_count = static_cast<int>(P);
    sp.seg_len = seg_len;
    sp.sub_len = seg_len / k;
    sp.subs_per_seg = k;
    sp.subs_per_unit = static_cast<int>((P - 1) * k);
    // sub-segment sums, then one start state per later segment
    sp.bytes = static_cast<size_t>(n_units) * (sp.subs_per_unit + sp.seg_count) * dk * dv * sizeof(float);
    return sp;
}

// Packed input: a 256-byte slot for the work counter, then the length order
// (one int32 per sequence, 2 to kMaxOrderedSeqs sequences).
size_t packed_ws_bytes(int num_seqs) {
    const size_t order = (num_seqs >= 2 && num_seqs <= kMaxOrderedSeqs)
                             ? (static_cast<size_t>(num_seqs) * 4 + 255) / 256 * 256
                             : 0;
    return 256 + order;
}

enum Path { kTc, kSimt, kShort, kUnsupported };

Path choose_path(la_dtype dtype, int dk, int dv, int chunk, const void* q, const void* k, const void* v,
                 const void* o) {
    if (dk < 1 || dv < 1 || dk > 128 || dv > 128 || chunk < 1) return kUnsupported;
    if (dtype == LA_BF16 && dk == dv && prefill_tc_supported(dk, chunk) && aligned16(q) && aligned16(k) &&
        aligned16(v) && aligned16(o))
        return kTc;
    if (prefill_simt_smem_bytes(dk, dv, chunk) <= 227 * 1024) return kSimt;
    return kUnsupported;
}

// The kernel a prefill runs: the few-token kernel when no unit has more than
// kShortMaxTokens rows (LINATTN_SHORT=0 turns it off), else the chunked
// tensor-core kernel, else the chunked CUDA-core kernel.
Path choose_kernel(la_dtype dtype, int64_t max_tokens, int dk, int dv, int chunk, const void* q, const void* k,
                   const void* v, const void* o, const void* state) {
    if (dk < 1 || dv < 1 || dk > 128 || dv > 128 || chunk < 1) return kUnsupported;
    if (tuning().short_kernel && prefill_short_supported(max_tokens, dk, dv, state)) return kShort;
    Path path = choose_path(dtype, dk, dv, chunk, q, k, v, o);
    // The tensor-core kernel moves state rows with 16-byte accesses.
    if (path == kTc && !aligned16(state)) path = kSimt;
    return path;
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" {

const char* la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "ok";
        case LA_ERR_INVALID_ARG: return "invalid argument";
        case LA_ERR_UNSUPPORTED: return "unsupported";
        case LA_ERR_CUDA: return "CUDA error";
        case LA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char* la_last_cuda_error(void) { return g_last_cuda_error; }

int la_resolve_chunk(la_dtype dtype, int d_k, int d_v, int chunk) {
    return chunk > 0 ? chunk : default_chunk(dtype, d_k, d_v);
}

const char* la_prefill_path(la_dtype dtype, int d_k, int d_v, int chunk, const void* q, const void* k,
                            const void* v, const void* o) {
    const int c = la_resolve_chunk(dtype, d_k, d_v, chunk);
    switch (choose_path(dtype, d_k, d_v, c, q, k, v, o)) {
        case kTc: return "tc";
        case kSimt: return "simt";
        default: return "unsupported";
    }
}

const char* la_prefill_kernel(la_dtype dtype, int64_t max_tokens, int d_k, int d_v, int chunk, const void* q,
                              const void* k, const void* v, const void* o, const float* state) {
    const int c = la_resolve_chunk(dtype, d_k, d_v, chunk);
    switch (choose_kernel(dtype, max_tokens, d_k, d_v, c, q, k, v, o, state)) {
        case kShort: return "short";
        case kTc: return "tc";
        case kSimt: return "simt";
        default: return "unsupported";
    }
}

la_status la_state_init(float* state, const float* src, int64_t n_units, int d_k, int d_v, void* stream) {
    if (n_units < 0 || d_k <= 0 || d_v <= 0) return LA_ERR_INVALID_ARG;
    if (n_units == 0) return LA_OK;
    if (!state) return LA_ERR_INVALID_ARG;
    cudaError_t e = launch_state_init(state, src, n_units * d_k * d_v, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e);
}

size_t la_prefill_workspace_size(la_dtype dtype, int B, int H, int64_t T, int d_k, int d_v, int num_seqs,
                                 int chunk) {
    // Tensor-core path only: dense input may be split (segment states);
    // packed input is walked dynamically (work counter + length order).
    if (B <= 0 || H <= 0 || T <= 0) return 0;
    const int c = la_resolve_chunk(dtype, d_k, d_v, chunk);
    if (!(dtype == LA_BF16 && d_k == d_v && prefill_tc_supported(d_k, c))) return 0;
    if (num_seqs > 0) return packed_ws_bytes(num_seqs);
    return plan_split(static_cast<int64_t>(B) * H, T, d_k, d_v, c, current_sm_count()).bytes;
}

la_status la_prefill(const void* q, const void* k, const void* v, void* o, float* state, la_dtype dtype, int B,
                     int H, int64_t T, int d_k, int d_v, const int32_t* cu_seqlens, int num_seqs,
                     int64_t max_seqlen, int chunk, void* workspace, size_t workspace_bytes, void* stream) {
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || d_k <= 0 || d_v <= 0) return LA_ERR_INVALID_ARG;
    if (T > 0x7fffffffLL) return LA_ERR_UNSUPPORTED;
    int64_t n_units, groups;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0) return LA_ERR_INVALID_ARG;
        n_units = static_cast<int64_t>(num_seqs) * H;
        groups = H;
    } else {
        n_units = static_cast<int64_t>(B) * H;
        groups = n_units;
    }
    if (n_units == 0 || T == 0) return LA_OK;
    if (!q || !k || !v || !o || !state) return LA_ERR_INVALID_ARG;
    const int c = la_resolve_chunk(dtype, d_k, d_v, chunk);
    // packed input: max_seqlen is the caller's bound on every sequence (0: unknown)
    const int64_t max_tokens = cu_seqlens ? max_seqlen : T;
    const Path path = choose_kernel(dtype, max_tokens, d_k, d_v, c, q, k, v, o, state);
    if (path == kUnsupported) return LA_ERR_UNSUPPORTED;

    PrefillProblem p;
    p.q = q; p.k = k; p.v = v; p.o = o; p.state = state;
    p.dtype = dtype == LA_BF16 ? 1 : 0;
    p.H = H > 0 ? H : 1;
    p.rows_per_group = T;
    p.n_units = n_units;
    p.dk = d_k; p.dv = d_v;
    p.cu = cu_seqlens;
    p.chunk = c;
    p.timeout_ns = tuning().wait_timeout_ns;
    p.seg_count = 1;
    p.seg_len = T;
    p.sub_len = 0;
    p.subs_per_seg = 0;
    p.subs_per_unit = 0;
    p.sub_states = nullptr;
    p.seg_states = nullptr;
    p.work_counter = nullptr;
    p.order = nullptr;
    p.prefetch = tuning().prefetch;
    p.trace = g_trace.buf;
    p.trace_count = g_trace.count;
    p.trace_cap = g_trace.cap;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int sms = current_sm_count();
    cudaError_t e;
    if (path == kShort) {
        e = launch_prefill_short(p, max_tokens, sms, s);
        return e == cudaSuccess ? LA_OK : cuda_fail(e);
    }
    if (path == kTc) {
        CUtensorMap tq, tk, tv, to;
        if (!encode_bf16_map(&tq, q, d_k, T, groups, c) || !encode_bf16_map(&tk, k, d_k, T, groups, c) ||
            !encode_bf16_map(&tv, v, d_v, T, groups, c) ||
            !encode_bf16_map(&to, o, d_v, T, groups, prefill_tc_o_box_rows(c))) {
            snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed");
            return LA_ERR_CUDA;
        }
        // Packed sequences, more units than SMs: the persistent CTAs claim
        // units from a counter (so lengths that differ, and SMs that run at
        // different speeds, even out), longest sequences first.
        if (cu_seqlens && n_units > sms && n_units < 0x7fffffffLL && workspace && workspace_bytes >= 256 &&
            aligned16(workspace)) {
            unsigned int* counter = static_cast<unsigned int*>(workspace);
            e = cudaMemsetAsync(counter, 0, sizeof(unsigned int), s);
            if (e != cudaSuccess) return cuda_fail(e);
            p.work_counter = counter;
            if (num_seqs >= 2 && num_seqs <= kMaxOrderedSeqs && workspace_bytes >= packed_ws_bytes(num_seqs)) {
                int32_t* order = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + 256);
                e = launch_length_order(cu_seqlens, num_seqs, T, order, s);
                if (e != cudaSuccess) return cuda_fail(e);
                p.order = order;
            }
        }
        // Few long sequences: split each one so that every SM gets work, when
        // the caller provided the workspace la_prefill_workspace_size asks for.
        if (!cu_seqlens) {
            const SplitPlan sp = plan_split(n_units, T, d_k, d_v, c, sms);
            if (sp.seg_count > 1 && workspace && workspace_bytes >= sp.bytes && aligned16(workspace)) {
                p.seg_count = sp.seg_count;
                p.seg_len = sp.seg_len;
                p.sub_len = sp.sub_len;
                p.subs_per_seg = sp.subs_per_seg;
                p.subs_per_unit = sp.subs_per_unit;
                float* sub = static_cast<float*>(workspace);
                float* seg = sub + static_cast<size_t>(n_units) * sp.subs_per_unit * d_k * d_v;
                p.sub_states = sub;
                p.seg_states = seg;
                e = launch_subsegment_states(p, tk, tv, sub, sms, s);
                if (e != cudaSuccess) return cuda_fail(e);
                e = launch_segment_prefix(p, seg, s);
                if (e != cudaSuccess) return cuda_fail(e);
            }
        }
        e = launch_prefill_tc(p, tq, tk, tv, to, sms, s);
    } else {
        e = launch_prefill_simt(p, sms, s);
    }
    return e == cudaSuccess ? LA_OK : cuda_fail(e);
}

la_status la_decode_step(const void* q, const void* k, const void* v, void* o, float* state, la_dtype dtype,
                         int B, int H, int d_k, int d_v, void* stream) {
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || d_k <= 0 || d_v <= 0) return LA_ERR_INVALID_ARG;
    if (d_k > 128 || d_v > 128) return LA_ERR_UNSUPPORTED;
    const int64_t n_units = static_cast<int64_t>(B) * H;
    if (n_units == 0) return LA_OK;
    if (!q || !k || !v || !o || !state) return LA_ERR_INVALID_ARG;
    cudaError_t e = launch_decode(q, k, v, o, state, dtype == LA_BF16 ? 1 : 0, n_units, d_k, d_v,
                                  current_sm_count(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e);
}

#ifdef LINATTN_TRACE
// Debugging hook of trace builds only (not part of the ABI): record events of
// CTA 0 of later tensor-core prefill launches into `buf` (`cap` records) and
// count them in `*count` (device memory, zeroed by the caller).
la_status la_debug_set_trace(unsigned long long* buf, unsigned int* count, unsigned int cap) {
    g_trace.buf = buf;
    g_trace.count = count;
    g_trace.cap = cap;
    return LA_OK;
}
#endif

la_status la_prefill_noalloc(const void* q, const void* k, const void* v, void* o, float* state, la_dtype dtype,
                             int B, int H, int64_t T, int d_k, int d_v, const int32_t* cu_seqlens, int num_seqs,
                             int64_t max_seqlen, int chunk, void* stream) {
    // Scratch this request needs (the same amount la_prefill would take from
    // a caller's workspace); refuse it up front when the static buffer is
    // too small.
    const size_t need = (B >= 0 && H >= 0 && T >= 0 && d_k > 0 && d_v > 0)
                            ? la_prefill_workspace_size(dtype, B, H, T, d_k, d_v, cu_seqlens ? num_seqs : 0, chunk)
                            : 0;
    if (need > LA_NOALLOC_SCRATCH_BYTES) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                 "la_prefill_noalloc: needs %zu bytes of scratch, the static buffer holds %u", need,
                 static_cast<unsigned>(LA_NOALLOC_SCRATCH_BYTES));
        return LA_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    if (need > 0) {
        // Device address of the static buffer, looked up once per device
        // with that device current, and again whenever the device's current
        // context is no longer the one it was looked up in (after a
        // cudaDeviceReset, say, the old address is stale).
        static void* addr[64] = {nullptr};
        static CUcontext ctx_of[64] = {nullptr};
        static std::mutex mu;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return cuda_fail(e);
        if (dev < 0 || dev >= 64) return LA_ERR_UNSUPPORTED;
        const CUcontext ctx = current_context();  // nullptr before the runtime has made one current
        std::lock_guard<std::mutex> lock(mu);
        if (!addr[dev] || ctx == nullptr || ctx != ctx_of[dev]) {
            void* ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);  // makes the primary context current
            if (e != cudaSuccess) return cuda_fail(e);
            addr[dev] = ptr;
            ctx_of[dev] = current_context();
        }
        scratch = addr[dev];
    }
    return la_prefill(q, k, v, o, state, dtype, B, H, T, d_k, d_v, cu_seqlens, num_seqs, max_seqlen, chunk, scratch,
                      scratch ? static_cast<size_t>(LA_NOALLOC_SCRATCH_BYTES) : 0, stream);
}

}  // extern "C"

namespace la {
// One thread waits on an mbarrier that nothing arrives on, through the same
// bounded wait as the prefill kernels; it gives up after timeout_ns.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
        mbar_wait(&bar, 0, &abort_flag, timeout_ns, 0xF00);
    }
}
}  // namespace la

extern "C" {

la_status la_selftest_wait_timeout(double timeout_ms, void* stream) {
    if (!(timeout_ms > 0.0) || timeout_ms > 10000.0) return LA_ERR_INVALID_ARG;
    la::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(timeout_ms * 1e6));
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LA_OK : cuda_fail(e);
}

la_status la_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int w[2] = {0, 0};
    e = cudaMemcpyFromSymbol(w, g_error_word, sizeof(w));
    if (e != cudaSuccess) return cuda_fail(e);
    if (w[0] != 0) {
        if (w[0] & kErrWaitTimeout)
            snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "device wait gave up at site 0x%x", w[1]);
        else
            snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "a packed sequence is longer than max_seqlen");
        const unsigned int z[2] = {0, 0};
        e = cudaMemcpyToSymbol(g_error_word, z, sizeof(z));
        if (e != cudaSuccess) return cuda_fail(e);
        return (w[0] & kErrWaitTimeout) ? LA_ERR_TIMEOUT : LA_ERR_INVALID_ARG;
    }
    return LA_OK;
}

}  // extern "C"
