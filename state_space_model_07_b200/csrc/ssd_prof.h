// ssd_prof.h -- launch counting and optional CUDA-event timing of each kernel.
#pragma once

#include <cuda_runtime.h>

namespace ssd {

enum KernelId : int {
    K_SEQ_BOUNDS = 0,
    K_SEQ_TABLE,
    K_SIMT_CHUNK_STATE,
    K_SIMT_STATE_PASS,
    K_SIMT_CHUNK_OUT,
    K_STATE_UPDATE,
    K_TC_PREP,
    K_TC_SCAN,
    K_SELFTEST_WAIT,
    K_SCAN_BWD,
    K_BWD_CAST,
    K_SEG_DECAY,
    K_STATE_CHAIN,
    K_STATE_OUT,
    K_TILE_DECAY,
    K_GROUP_NORM,
    K_QUANT,
    K_BWD_PASS,
    K_BWD_GRADS,
    K_COUNT
};

// Brackets one kernel launch: counts it and, while profiling is enabled,
// records a CUDA event pair on `st` around it.
class ProfScope {
  public:
    ProfScope(KernelId id, cudaStream_t st);
    ~ProfScope();
    ProfScope(const ProfScope&) = delete;
    ProfScope& operator=(const ProfScope&) = delete;

  private:
    KernelId id_;
    cudaStream_t st_;
    cudaEvent_t e0_ = nullptr, e1_ = nullptr;
};

}  // namespace ssd
