// ssd_tc.cu -- tensor-core (tcgen05) path of the chunked scan (bf16 inputs).
#include "ssd_common.cuh"
#include "ssd_tc.h"

namespace ssd {

bool tc_supported(const ScanArgs&) { return false; }
size_t tc_workspace_bytes(const ScanArgs&, int64_t) { return 0; }
int launch_tc_scan(const ScanArgs&, const SeqInfo&, int64_t, void*, int32_t*, cudaStream_t) {
    return 5;
}

}  // namespace ssd
