// ssd_check.cu -- debug-mode value checks around the tensor-core scan.
//
// The tensor-core path feeds the tensor cores fp16 operands (x, B, C, the
// masked score matrix and the carried state), whose largest finite value is
// 65504.  A bf16 input beyond that, or an intermediate that grows past it,
// becomes inf where the recurrence itself (and the CUDA-core path) stays
// finite.  With SSD_DEBUG_CHECK=1 the library counts, on the device:
//   [0] non-finite input values (x, dt, B, C, init_state),
//   [1] finite x, B, C or init_state values of magnitude above 65504,
//   [2] non-finite output values (y, final_state),
// and the host reports SSD_ERR_RANGE when [1] > 0, or when [2] > 0 while
// [0] == 0 (finite inputs gave a non-finite result).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kCheckThreads = 256;

__device__ __forceinline__ void block_add(uint32_t v, uint32_t* counter) {
    v = __reduce_add_sync(0xffffffffu, v);
    if ((threadIdx.x & 31) == 0 && v) atomicAdd(counter, v);
}

// bf16 words: exponent all ones = inf / NaN; otherwise |v| > 65504 is over range.
__global__ void k_check_bf16(const uint16_t* __restrict__ p, int64_t n, uint32_t* nonfinite, uint32_t* over,
                             int range) {
    uint32_t nf = 0, ov = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t a = p[i] & 0x7fffu;
        if (a >= 0x7f80u)
            ++nf;
        else if (range && __uint_as_float(a << 16) > 65504.f)
            ++ov;
    }
    block_add(nf, nonfinite);
    if (range) block_add(ov, over);
}

__global__ void k_check_f32(const float* __restrict__ p, int64_t n, uint32_t* nonfinite, uint32_t* over,
                            int range) {
    uint32_t nf = 0, ov = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = fabsf(p[i]);
        if (!(v <= 3.402823466e38f))
            ++nf;
        else if (range && v > 65504.f)
            ++ov;
    }
    block_add(nf, nonfinite);
    if (range) block_add(ov, over);
}

void check_array(const void* p, int64_t n, bool bf16, uint32_t* nonfinite, uint32_t* over, bool range,
                 cudaStream_t st) {
    if (!p || n <= 0) return;
    int64_t blocks = (n + kCheckThreads - 1) / kCheckThreads;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (bf16)
        k_check_bf16<<<(unsigned)blocks, kCheckThreads, 0, st>>>((const uint16_t*)p, n, nonfinite, over, range);
    else
        k_check_f32<<<(unsigned)blocks, kCheckThreads, 0, st>>>((const float*)p, n, nonfinite, over, range);
}

}  // namespace

void launch_range_check_inputs(const ScanArgs& a, uint32_t* counters, cudaStream_t st) {
    const int64_t ntok = a.b * a.L;
    const bool bf = a.dtype == 1;
    check_array(a.x, ntok * a.H * a.P, bf, counters, counters + 1, true, st);
    check_array(a.B, ntok * a.G * a.N, bf, counters, counters + 1, true, st);
    check_array(a.C, ntok * a.G * a.N, bf, counters, counters + 1, true, st);
    check_array(a.dt, ntok * a.H, bf, counters, counters + 1, false, st);
    check_array(a.init_state, a.S * a.H * a.N * a.P, false, counters, counters + 1, true, st);
}

void launch_range_check_outputs(const ScanArgs& a, uint32_t* counters, cudaStream_t st) {
    const int64_t ntok = a.b * a.L;
    check_array(a.y, ntok * a.H * a.P, a.dtype == 1, counters + 2, counters + 1, false, st);
    check_array(a.final_state, a.S * a.H * a.N * a.P, false, counters + 2, counters + 1, false, st);
}

}  // namespace ssd
