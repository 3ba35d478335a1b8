// ssd_tc.h -- host interface of the tensor-core (tcgen05) scan path.
#pragma once

#include "ssd_internal.h"

namespace ssd {

// True when the bf16 tensor-core path covers this call's shapes.
bool tc_supported(const ScanArgs& a);
size_t tc_workspace_bytes(const ScanArgs& a, int64_t max_chunks);
// Returns an ssd_status; launches asynchronously on `st`.
int launch_tc_scan(const ScanArgs& a, const SeqInfo& si, int64_t max_chunks, void* ws,
                   int32_t* status, cudaStream_t st);

// y += the output of the state h_in (b, H, N, P) entering every row at its start
// (ssd_state_to_output): bf16 inputs, P = 64, N = 128.
bool state_out_supported(const ScanArgs& a);
size_t state_out_workspace_bytes(const ScanArgs& a);
int launch_state_to_output(const ScanArgs& a, const float* h_in, void* ws, int32_t* status, cudaStream_t st);

// The state-to-output pass of the segment split (ssd_state_out.cu): rows W .. b - 1 of `a` are
// split into K segments of Ls tokens (`tiles` tiles); fin holds every segment's final state and
// cs the running log-decay of its tokens, c16 the fp16 copy of C; adds each later segment's
// entering-state output to y and writes those rows' final states.
int launch_state_out_split(const ScanArgs& a, const void* c16, const float* fin, const float* cs, int64_t W, int K,
                           int64_t Ls, int tiles, int32_t* status, cudaStream_t st);

}  // namespace ssd
