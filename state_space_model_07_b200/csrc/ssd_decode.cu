// ssd_decode.cu -- single-token state update on a cached fp32 state (decode).
//
// One step of the recurrence of "5.3 Tensor Parallelism support and
// large-cluster training", section 2.1, on the state carried over from the
// prefill scan ("Scaling State-Space Models on Multiple GPUs with Tensor
// Parallelism", abstract):
//   d = softplus(dt + dt_bias_h)
//   h <- exp(d A_h) h + d B x^T          (N x P, in place)
//   y  = C^T h + D_h x
// The state is read and written exactly once, so the kernel is bound by HBM
// bandwidth: every thread streams float4 columns of the state with
// evict-first loads/stores, several rows in flight at a time, and the
// per-column output is reduced across the block in shared memory.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

namespace ssd {

constexpr int kDecThreads = 256;
constexpr int kDecUnroll = 8;

template <typename T>
__global__ void __launch_bounds__(kDecThreads)
k_state_update(float* __restrict__ state, const T* __restrict__ x, const T* __restrict__ dt,
               const float* __restrict__ dt_bias, const float* __restrict__ A,
               const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D,
               T* __restrict__ y, int H, int P, int N, int G) {
    extern __shared__ float sm[];
    float* dB_s = sm;        // N
    float* C_s = sm + N;     // N
    float4* red = reinterpret_cast<float4*>(sm + 2 * N);  // kDecThreads float4

    const int64_t bh = blockIdx.x;
    const int64_t bi = bh / H;
    const int h = (int)(bh % H);
    const int g = h / (H / G);
    const int tid = threadIdx.x;
    const int P4 = P / 4;
    const int RG = kDecThreads / P4;
    const int col = tid % P4, rg = tid / P4;

    const float d = softplus_f(to_f<T>(dt[bh]) + (dt_bias ? dt_bias[h] : 0.f));
    const float dA = expf(d * A[h]);
    for (int n = tid; n < N; n += kDecThreads) {
        dB_s[n] = d * to_f<T>(B[(bi * G + g) * N + n]);
        C_s[n] = to_f<T>(C[(bi * G + g) * N + n]);
    }
    __syncthreads();

    float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 yacc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rg < RG) {
        const T* xp = x + bh * P + 4 * col;
        x4 = make_float4(to_f<T>(xp[0]), to_f<T>(xp[1]), to_f<T>(xp[2]), to_f<T>(xp[3]));
        float4* st = reinterpret_cast<float4*>(state + bh * (int64_t)N * P) + col;
        for (int n0 = rg; n0 < N; n0 += kDecUnroll * RG) {
            float4 v[kDecUnroll];
#pragma unroll
            for (int k = 0; k < kDecUnroll; ++k) {
                const int n = n0 + k * RG;
                if (n < N) v[k] = __ldcs(st + (int64_t)n * P4);
            }
#pragma unroll
            for (int k = 0; k < kDecUnroll; ++k) {
                const int n = n0 + k * RG;
                if (n < N) {
                    const float bn = dB_s[n], cn = C_s[n];
                    float4 u;
                    u.x = dA * v[k].x + bn * x4.x;
                    u.y = dA * v[k].y + bn * x4.y;
                    u.z = dA * v[k].z + bn * x4.z;
                    u.w = dA * v[k].w + bn * x4.w;
                    __stcs(st + (int64_t)n * P4, u);
                    yacc.x += cn * u.x;
                    yacc.y += cn * u.y;
                    yacc.z += cn * u.z;
                    yacc.w += cn * u.w;
                }
            }
        }
    }
    red[tid] = yacc;
    __syncthreads();
    if (tid < P4) {
        float4 s = red[tid];
        for (int r = 1; r < RG; ++r) {
            float4 o = red[r * P4 + tid];
            s.x += o.x; s.y += o.y; s.z += o.z; s.w += o.w;
        }
        const float Dh = D ? D[h] : 0.f;
        T* yp = y + bh * P + 4 * tid;
        yp[0] = from_f<T>(s.x + Dh * x4.x);
        yp[1] = from_f<T>(s.y + Dh * x4.y);
        yp[2] = from_f<T>(s.z + Dh * x4.z);
        yp[3] = from_f<T>(s.w + Dh * x4.w);
    }
}

void launch_state_update(const UpdateArgs& a, cudaStream_t st) {
    const size_t smem = sizeof(float) * 2 * a.N + sizeof(float4) * kDecThreads;
    const unsigned grid = (unsigned)(a.b * a.H);
    ProfScope ps(K_STATE_UPDATE, st);
    if (a.dtype == 0)
        k_state_update<float><<<grid, kDecThreads, smem, st>>>(
            a.state, (const float*)a.x, (const float*)a.dt, a.dt_bias, a.A, (const float*)a.B,
            (const float*)a.C, a.D, (float*)a.y, (int)a.H, (int)a.P, (int)a.N, (int)a.G);
    else
        k_state_update<__nv_bfloat16><<<grid, kDecThreads, smem, st>>>(
            a.state, (const __nv_bfloat16*)a.x, (const __nv_bfloat16*)a.dt, a.dt_bias, a.A,
            (const __nv_bfloat16*)a.B, (const __nv_bfloat16*)a.C, a.D, (__nv_bfloat16*)a.y,
            (int)a.H, (int)a.P, (int)a.N, (int)a.G);
}

}  // namespace ssd
