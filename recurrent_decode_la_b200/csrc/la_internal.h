// la_internal.h -- host-side launch interfaces shared by the library's .cu
// files (not part of the public ABI; see include/linattn.h for that).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

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
    // Event trace of CTA 0 (builds with LINATTN_TRACE only; nullptr otherwise).
    unsigned long long* trace;
    unsigned int* trace_count;
    unsigned int trace_cap;
};

cudaError_t launch_prefill_simt(const PrefillProblem& p, int num_sms, cudaStream_t s);
size_t prefill_simt_smem_bytes(int dk, int dv, int chunk);

// Tensor-core prefill (bf16, d_k == d_v == D in {64,128}, chunk in {64,128}).
bool prefill_tc_supported(int D, int chunk);
cudaError_t launch_prefill_tc(const PrefillProblem& p, const CUtensorMap& tq,
                              const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& to, int num_sms, cudaStream_t s);

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* state,
                          int dtype, int64_t n_units, int dk, int dv, int num_sms,
                          cudaStream_t s);

cudaError_t launch_state_init(float* state, const float* src, int64_t n, cudaStream_t s);

}  // namespace la
