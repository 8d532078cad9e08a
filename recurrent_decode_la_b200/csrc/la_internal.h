// la_internal.h -- host-side launch interfaces shared by the library's .cu
// files (not part of the public ABI; see include/linattn.h for that).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace la {

// Tuning switches taken from the environment once per process, on the first
// call into the library that needs one; later changes to the environment
// have no effect.  None of them changes a result, only which kernel runs or
// how it is scheduled.
//   LINATTN_CHUNK             default chunk size (0 / unset: per shape)
//   LINATTN_SHORT=0           never take the few-token prefill kernel
//   LINATTN_SPLIT=0           never split a sequence into segments
//   LINATTN_PREFETCH          chunks the prefill producer prefetches into L2
//   LINATTN_DECODE_COLBLOCKS  decode column blocks per unit (unset: per
//                             shape; 0: one CTA per unit)
//   LINATTN_DECODE_PDL=0      launch decode without programmatic dependency
//   LINATTN_WAIT_TIMEOUT_MS   bound of every device-side wait (default 4000)
struct Tuning {
    int chunk;
    bool short_kernel;
    bool split;
    int prefetch;
    int decode_col_blocks;  // -1: per shape
    bool decode_pdl;
    uint64_t wait_timeout_ns;
};
const Tuning& tuning();

// Per-device one-time set-up of a kernel's attributes (a raised shared-memory
// limit and the like).  cudaFuncSetAttribute may not run inside a stream
// capture, so the first launch on each device (made outside any capture)
// runs it; later launches skip it.  Safe to call from several host threads:
// the attribute calls are idempotent, the flags atomic.  Devices beyond the
// first 64 run the set-up on every launch.
struct PerDeviceOnce {
    std::atomic<bool> done[64];  // static storage: zero-initialised
    template <typename F>
    cudaError_t run(F&& setup) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const bool cached = dev >= 0 && dev < 64;
        if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
        e = setup();
        if (e != cudaSuccess) return e;
        if (cached) done[dev].store(true, std::memory_order_release);
        return cudaSuccess;
    }
};

// Launch `kern` as a programmatic dependent of the previous kernel in the
// stream: it may start while that kernel drains, so it must call
// griddepcontrol.wait before touching global memory the previous kernel
// writes (every kernel launched this way does).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Everything a prefill kernel needs to locate its units.  Dense input:
// groups = B*H, rows_per_group = T, unit u = group u.  Packed input:
// groups = H, rows_per_group = T_total, unit u = (seq u / H, head u % H).
struct PrefillProblem {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* state;
    int dtype;  // 0 = f32, 1 = bf16
    int H;
    int64_t rows_per_group;
    int64_t n_units;
    int dk;
    int dv;
    const int32_t* cu;  // nullptr for dense input
    int chunk;
    uint64_t timeout_ns;
    // Intra-sequence split (dense input only; seg_count = 1 means none).
    // Work item i is segment i % seg_count of unit i / seg_count: rows
    // [s * seg_len, min((s + 1) * seg_len, rows_per_group)).  Segment s
    // starts from seg_states[u][s] = S_0 plus the K^T V sums of the first
    // s * subs_per_seg sub-segments (sub_len rows each, sums kept in
    // sub_states [units][subs_per_unit][dk][dv]); only the last segment
    // writes S_T.
    int seg_count;
    int64_t seg_len;
    int64_t sub_len;
    int subs_per_seg;
    int subs_per_unit;
    const float* sub_states;
    const float* seg_states;  // [units][seg_count][dk][dv]
    // Dynamic walk (tensor-core prefill): a zeroed counter from which the
    // persistent CTAs claim work items in turn (nullptr: CTA b takes items
    // b, b + G, b + 2G, ...).  Packed input under the dynamic walk may also
    // give `order`, the sequences by decreasing length: item i is then head
    // i % H of the sequence order[i / H], so that the longest are claimed
    // first.
    unsigned int* work_counter;
    const int32_t* order;
    // Chunks ahead of the shared-memory load that the producer prefetches
    // into L2 (0 = none).
    int prefetch;
    // Event trace of CTA 0 (builds with LINATTN_TRACE only; nullptr otherwise).
    unsigned long long* trace;
    unsigned int* trace_count;
    unsigned int trace_cap;
};

cudaError_t launch_prefill_simt(const PrefillProblem& p, int num_sms, cudaStream_t s);
size_t prefill_simt_smem_bytes(int dk, int dv, int chunk);

// Tensor-core prefill (bf16, d_k == d_v == D in {64,128}, chunk in {16,32,64,128}).
bool prefill_tc_supported(int D, int chunk);
// Rows of the O tensor map's box for this chunk size (C = 128: each output
// warp stores its own 32 rows).
int prefill_tc_o_box_rows(int chunk);
cudaError_t launch_prefill_tc(const PrefillProblem& p, const CUtensorMap& tq,
                              const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& to, int num_sms, cudaStream_t s);

// Sub-segment states for the intra-sequence split: sub_states[u][j] =
// K^T V over rows [j * sub_len, (j + 1) * sub_len) of unit u, for
// j < subs_per_unit (tensor cores, bf16 in, fp32 out).
cudaError_t launch_subsegment_states(const PrefillProblem& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                     float* sub_states, int num_sms, cudaStream_t s);

// seg_states[u][s] = S_0[u] + sum of sub_states[u][0 .. s*subs_per_seg - 1]
// for s = 0 .. seg_count - 1 (one pass over the sub-segment sums).
cudaError_t launch_segment_prefix(const PrefillProblem& p, float* seg_states, cudaStream_t s);

// Prefill of at most kShortMaxTokens tokens per unit (dense T, or packed
// max_seqlen) from a saved state: one pass over the state, CUDA cores, fp32.
constexpr int kShortMaxTokens = 16;
bool prefill_short_supported(int64_t max_tokens, int dk, int dv, const void* state);
cudaError_t launch_prefill_short(const PrefillProblem& p, int64_t max_tokens, int num_sms, cudaStream_t s);

// order[r] = the sequence of rank r when sequences are sorted by decreasing
// length (ties: lower index first), for num_seqs <= kMaxOrderedSeqs.
constexpr int kMaxOrderedSeqs = 4096;
cudaError_t launch_length_order(const int32_t* cu, int num_seqs, int64_t total_rows, int32_t* order,
                                cudaStream_t s);

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* state,
                          int dtype, int64_t n_units, int dk, int dv, int num_sms,
                          cudaStream_t s);

cudaError_t launch_state_init(float* state, const float* src, int64_t n, cudaStream_t s);

}  // namespace la
