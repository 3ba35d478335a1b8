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

}  // namespace ssd
