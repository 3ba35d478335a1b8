// ssd_internal.h -- host-side interfaces between ssd_api.cu and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssd {

struct SeqInfo;

// Validated arguments of one ssd_chunk_scan_fwd call.
struct ScanArgs {
    int64_t b, L, H, P, N, G, S;
    int dtype;  // 0 = float32, 1 = bfloat16
    int Q;
    const void *x, *dt, *B, *C;
    const float *dt_bias, *A, *D, *init_state;
    const int32_t* seq_idx;
    void* y;
    float* final_state;
};

// Packed-sequence table: spans and chunk offsets computed on the device.
void launch_seq_table(const int32_t* seq_idx, int64_t L, int32_t S, int32_t Q, int32_t* start,
                      int32_t* end, int32_t* chunk_off, int32_t* status, cudaStream_t st);

// CUDA-core path (any supported shape, float32 or bfloat16).
size_t simt_workspace_bytes(const ScanArgs& a, int64_t max_chunks);
void launch_simt_scan(const ScanArgs& a, const SeqInfo& si, int64_t max_chunks, void* ws,
                      cudaStream_t st);

// Decode state update.
struct UpdateArgs {
    int64_t b, H, P, N, G;
    int dtype;
    float* state;
    const void *x, *dt, *B, *C;
    const float *A, *D, *dt_bias;
    void* y;
};
void launch_state_update(const UpdateArgs& a, cudaStream_t st);

// Backward of the scan (ssd_bwd.cu): the gradients' buffers of one
// ssd_chunk_scan_bwd call.
struct BwdArgs {
    const void* dy;            // (b, L, H, P), dtype of x
    const float* dfinal;       // (S, H, N, P) or null
    void *dx, *ddt, *dB, *dC;  // dtype of x
    float *ddt_bias, *dA, *dD; // (H)
    float* dinit;              // (S, H, N, P) or null
};
// Shapes the CUDA-core backward handles: P divides 256, N P a power-of-two
// multiple of 256 up to 8192.
bool bwd_supported(const ScanArgs& a);
size_t bwd_workspace_bytes(const ScanArgs& a);
// `si64` describes the sequences with 64-token blocks (chunk_off counts them).
int launch_scan_bwd(const ScanArgs& a, const BwdArgs& g, const SeqInfo& si64, void* ws, cudaStream_t st);

// Sequence-parallel state passing (ssd_seqpar.cu): the total log-decay of
// each batch row's slice, out (b, H); and h_out = exp(logdecay) h_in + F over
// bh (batch, head) pairs of N P floats.
void launch_segment_logdecay(int64_t b, int64_t L, int64_t H, int dtype, const void* dt, const float* dt_bias,
                             const float* A, float* out, cudaStream_t st);
void launch_state_chain(int64_t bh, int64_t NP, const float* h_in, const float* logdecay, const float* F,
                        float* h_out, cudaStream_t st);

// Head-sharded mixer (ssd_tp.cu): group norm of (rows, C) with C / ngroups channels per group,
// and the steps of the quantised all-reduce (int8 codes, one fp32 scale per 64 columns).
bool group_norm_supported(int64_t C, int64_t ngroups);
void launch_group_norm(int dtype, const void* x, const float* gamma, const float* beta, float eps, int64_t rows,
                       int64_t C, int64_t ngroups, void* out, cudaStream_t st);
void launch_quant_chunks(const float* x, int64_t T, int64_t D, int64_t Tp, int8_t* q, float* scale, cudaStream_t st);
void launch_dequant_sum_quant(const int8_t* qin, const float* sin, int64_t Tp, int64_t T, int64_t Dc, int8_t* qout,
                              float* sout, cudaStream_t st);
void launch_dequant_chunks(int dtype, const int8_t* q, const float* s, int64_t Tp, int64_t T, int64_t Dc, void* out,
                           cudaStream_t st);

// Debug-mode value checks around a tensor-core scan (ssd_check.cu): counters[0]
// += non-finite inputs, counters[1] += finite x / B / C / init_state values
// beyond the fp16 range, counters[2] += non-finite outputs.
void launch_range_check_inputs(const ScanArgs& a, uint32_t* counters, cudaStream_t st);
void launch_range_check_outputs(const ScanArgs& a, uint32_t* counters, cudaStream_t st);

// One thread waits, with the kernels' bounded wait and `limit_cycles`, on an
// mbarrier nothing arrives at, and writes the outcome to *status.
void launch_selftest_wait(long long limit_cycles, int32_t* status, cudaStream_t st);

}  // namespace ssd
