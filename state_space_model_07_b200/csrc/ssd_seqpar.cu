// ssd_seqpar.cu -- the two small steps of sequence-parallel state passing.
//
// "5.3 Tensor Parallelism support and large-cluster training", section 4.2,
// splits a long sequence over devices: each device scans its slice, and the
// N x P state crosses from one device to the next.  With the slice's own scan
// run from a zero state (final state F) and its total log-decay
//   D = sum over the slice of softplus(dt_t + dt_bias_h) A_h,
// the state leaving the slice is h_out = exp(D) h_in + F for the state h_in
// entering it (the recurrence is linear in the state, and the decay of the whole
// slice is the product of its per-token factors exp(d_t A_h)).
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

namespace ssd {
namespace {

constexpr int kDecayThreads = 256;

// One block per (batch row, head): out[b, h] = sum_t softplus(dt[b, t, h] + dt_bias_h) A_h.
template <typename T>
__global__ void __launch_bounds__(kDecayThreads)
k_segment_logdecay(const T* __restrict__ dt, const float* __restrict__ dt_bias, const float* __restrict__ A,
                   float* __restrict__ out, int64_t L, int H) {
    const int h = blockIdx.x % H;
    const int64_t b = blockIdx.x / H;
    const float bias = dt_bias ? dt_bias[h] : 0.f;
    float acc = 0.f;
    for (int64_t t = threadIdx.x; t < L; t += kDecayThreads) acc += softplus_f(to_f<T>(dt[(b * L + t) * H + h]) + bias);
    __shared__ float red[kDecayThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int i = 0; i < kDecayThreads / 32; ++i) s += red[i];
        out[blockIdx.x] = s * A[h];
    }
}

// h_out[b, h] = exp(logdecay[b, h]) h_in[b, h] + F[b, h] over (b, H, N P), float4 at a time.
__global__ void k_state_chain(const float4* __restrict__ h_in, const float* __restrict__ logdecay,
                              const float4* F, float4* h_out, int64_t n4, int64_t NP4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float e = expf(logdecay[i / NP4]);
        const float4 a = h_in[i], f = F[i];
        h_out[i] = make_float4(e * a.x + f.x, e * a.y + f.y, e * a.z + f.z, e * a.w + f.w);
    }
}

}  // namespace

void launch_segment_logdecay(int64_t b, int64_t L, int64_t H, int dtype, const void* dt, const float* dt_bias,
                             const float* A, float* out, cudaStream_t st) {
    ProfScope ps(K_SEG_DECAY, st);
    const unsigned grid = (unsigned)(b * H);
    if (dtype == 0)
        k_segment_logdecay<float><<<grid, kDecayThreads, 0, st>>>((const float*)dt, dt_bias, A, out, L, (int)H);
    else
        k_segment_logdecay<__nv_bfloat16><<<grid, kDecayThreads, 0, st>>>((const __nv_bfloat16*)dt, dt_bias, A, out,
                                                                          L, (int)H);
}

void launch_state_chain(int64_t bh, int64_t NP, const float* h_in, const float* logdecay, const float* F,
                        float* h_out, cudaStream_t st) {
    const int64_t n4 = bh * NP / 4;
    int64_t blocks = (n4 + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    ProfScope ps(K_STATE_CHAIN, st);
    k_state_chain<<<(unsigned)blocks, 256, 0, st>>>((const float4*)h_in, logdecay, (const float4*)F, (float4*)h_out,
                                                    n4, NP / 4);
}

}  // namespace ssd
