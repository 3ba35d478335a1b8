// ssd_bwd.cu -- gradient of the scan (backward pass), on CUDA cores in fp32.
//
// The pages train these models ("5.3 Tensor Parallelism support and
// large-cluster training", sections 6.3 and Table 5.3.1), so the backward of
// the recurrence of section 2.1 is part of the training step.  They print no
// gradient formulas; the ones below are the chain rule applied to
//   z_t = dt_t + dt_bias_h,  d_t = softplus(z_t),  a_t = exp(d_t A_h),
//   h_t = a_t h_{t-1} + d_t B_t x_t^T,  y_t = C_t^T h_t + D_h x_t
// for J = sum_t <dy_t, y_t> + <dfinal, h_last>: the adjoint state
// g_t = dJ/dh_t runs backwards, g_t = C_t dy_t^T + a_{t+1} g_{t+1} (with
// a_{last+1} g_{last+1} = dfinal), and every gradient is read off the step that
// used its input:
//   dx_t = D dy_t + d_t B_t^T g_t          dC_t = h_t dy_t
//   dB_t = d_t g_t x_t                     dD  += <dy_t, x_t>
//   u_t  = <g_t, h_{t-1}>                  dd_t = u_t a_t A + <g_t, B_t x_t^T>
//   dA  += u_t a_t d_t                     dz_t = dd_t sigmoid(z_t)
//   ddt_t = dz_t, ddt_bias += dz_t         dinit = a_first g_first
// dB and dC sum over the heads of a group, ddt_bias, dA and dD over tokens and
// sequences; every packed sequence restarts from its own initial state.
//
// Layout of the work: one 256-thread block per (sequence, head).  The N x P
// state is spread over the block, thread `tid` owning column p = tid % P of
// rows tid / P + (256 / P) k, k < E = N P / 256, in registers.  Pass 1 walks
// the sequence forward and keeps the state at the start of every 64-token
// block (checkpoints, in the workspace).  Pass 2 takes the blocks in reverse:
// it recomputes the block's per-token states into a per-(sequence, head)
// scratch area and then runs the adjoint sweep over the block's tokens, last
// to first.  Every quantity is fp32; inputs are read in their own dtype.
#include <stdio.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

namespace ssd {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdBlock = 64;         // tokens between checkpoints
constexpr int kBwdMaxE = 32;          // N P <= 8192

struct BwdParams {
    SeqInfo si;                       // spans of the sequences; chunk_off counts 64-token blocks
    int64_t ck_per_row;               // blocks per sequence when not packed
    const void *x, *dt, *B, *C, *dy;
    const float *dt_bias, *A, *D, *init_state, *dfinal;
    void *dx, *ddt;
    float *dB_acc, *dC_acc;           // (b, L, G, N) fp32, summed over the group's heads
    float *ddt_bias, *dA, *dD;        // (H), summed over tokens and sequences
    float* dinit;                     // (S, H, N, P) or null
    float* ckpt;                      // checkpoints, (blocks, H, N P)
    float* scratch;                   // per-token states of one block, (S H, 64, N P)
    int H, P, N, G;
};

__device__ __forceinline__ float sigmoid_f(float z) {
    if (z >= 0.f) return 1.f / (1.f + expf(-z));
    const float e = expf(z);
    return e / (1.f + e);
}

// Sum over the block; every thread gets the result.  `red` holds 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kBwdThreads / 32; ++i) s += red[i];
    return s;
}

template <typename T, int E>
__global__ void __launch_bounds__(kBwdThreads)
k_scan_bwd(const BwdParams p) {
    const int H = p.H, P = p.P, N = p.N, G = p.G;
    const int seq = blockIdx.x / H, h = blockIdx.x % H;
    const int g = h / (H / G);
    const int tid = threadIdx.x;
    const int RG = kBwdThreads / P;           // row groups; P divides 256
    const int col = tid % P, rg = tid / P;
    const int64_t NP = (int64_t)N * P;

    int64_t row, t0, t1;
    seq_span(p.si, seq, row, t0, t1);
    const int64_t len = t1 > t0 ? t1 - t0 : 0;
    const int nb = (int)((len + kBwdBlock - 1) / kBwdBlock);
    const int64_t ck0 = p.si.packed ? (int64_t)p.si.chunk_off[seq] : (int64_t)seq * p.ck_per_row;
    const int64_t tok0 = row * p.si.L + t0;    // flat token index of the sequence start
    float* ck = p.ckpt + (ck0 * H + h) * NP;   // block c's checkpoint at ck + c H NP
    float* scr = p.scratch + (int64_t)blockIdx.x * kBwdBlock * NP;

    extern __shared__ float sm[];
    float* sB = sm;                 // N
    float* sC = sB + N;             // N
    float* sx = sC + N;             // P
    float* sdy = sx + P;            // P
    float* red = sdy + P;           // 32
    float* sdx = red + 32;          // RG x P

    const float Ah = p.A[h];
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const float Dh = p.D ? p.D[h] : 0.f;
    const T* xg = (const T*)p.x;
    const T* dtg = (const T*)p.dt;
    const T* Bg = (const T*)p.B;
    const T* Cg = (const T*)p.C;
    const T* dyg = (const T*)p.dy;

    auto load_tok = [&](int64_t t, bool with_c_dy) {
        const int64_t tk = tok0 + t;
        for (int i = tid; i < N; i += kBwdThreads) {
            sB[i] = to_f<T>(Bg[(tk * G + g) * N + i]);
            if (with_c_dy) sC[i] = to_f<T>(Cg[(tk * G + g) * N + i]);
        }
        for (int i = tid; i < P; i += kBwdThreads) {
            sx[i] = to_f<T>(xg[(tk * H + h) * P + i]);
            if (with_c_dy) sdy[i] = to_f<T>(dyg[(tk * H + h) * P + i]);
        }
    };

    // ---- pass 1: forward, checkpoint at every block start
    float hr[E];
    {
        const float* src = p.init_state ? p.init_state + ((int64_t)seq * H + h) * NP : nullptr;
#pragma unroll
        for (int k = 0; k < E; ++k) hr[k] = src ? src[(int64_t)(rg + RG * k) * P + col] : 0.f;
    }
    for (int64_t t = 0; t < len; ++t) {
        if (t % kBwdBlock == 0) {
            float* dst = ck + (t / kBwdBlock) * H * NP;
#pragma unroll
            for (int k = 0; k < E; ++k) dst[(int64_t)(rg + RG * k) * P + col] = hr[k];
        }
        __syncthreads();
        load_tok(t, false);
        __syncthreads();
        const float d = softplus_f(to_f<T>(dtg[(tok0 + t) * H + h]) + bias);
        const float a = expf(d * Ah);
        const float dx = d * sx[col];
#pragma unroll
        for (int k = 0; k < E; ++k) hr[k] = a * hr[k] + dx * sB[rg + RG * k];
    }

    // ---- pass 2: blocks in reverse; recompute, then the adjoint sweep
    float gr[E];
    {
        const float* src = p.dfinal ? p.dfinal + ((int64_t)seq * H + h) * NP : nullptr;
#pragma unroll
        for (int k = 0; k < E; ++k) gr[k] = src ? src[(int64_t)(rg + RG * k) * P + col] : 0.f;
    }
    float a_next = 1.f;               // a_{t+1}; g arrives as a_{t+1} g_{t+1} (dfinal at the end)
    float acc_dA = 0.f, acc_dbias = 0.f, acc_dD = 0.f;
    for (int c = nb - 1; c >= 0; --c) {
        const int64_t b0 = (int64_t)c * kBwdBlock;
        const int bl = (int)(len - b0 < kBwdBlock ? len - b0 : kBwdBlock);
        const float* ckc = ck + (int64_t)c * H * NP;
        // recompute h_t, t in the block, into the scratch (row j = t - b0)
#pragma unroll
        for (int k = 0; k < E; ++k) hr[k] = ckc[(int64_t)(rg + RG * k) * P + col];
        for (int j = 0; j < bl; ++j) {
            __syncthreads();
            load_tok(b0 + j, false);
            __syncthreads();
            const float d = softplus_f(to_f<T>(dtg[(tok0 + b0 + j) * H + h]) + bias);
            const float a = expf(d * Ah);
            const float dx = d * sx[col];
#pragma unroll
            for (int k = 0; k < E; ++k) {
                hr[k] = a * hr[k] + dx * sB[rg + RG * k];
                scr[(int64_t)j * NP + tid + (int64_t)kBwdThreads * k] = hr[k];
            }
        }
        // adjoint sweep over the block, last token first
        for (int j = bl - 1; j >= 0; --j) {
            const int64_t t = b0 + j, tk = tok0 + t;
            __syncthreads();
            load_tok(t, true);
            __syncthreads();
            const float z = to_f<T>(dtg[tk * H + h]) + bias;
            const float d = softplus_f(z);
            const float a = expf(d * Ah);
            // h_t (this thread's elements) and h_{t-1}
            float hc[E], hp[E];
#pragma unroll
            for (int k = 0; k < E; ++k) {
                hc[k] = scr[(int64_t)j * NP + tid + (int64_t)kBwdThreads * k];
                hp[k] = j > 0 ? scr[(int64_t)(j - 1) * NP + tid + (int64_t)kBwdThreads * k]
                              : ckc[(int64_t)(rg + RG * k) * P + col];
            }
            const float dyp = sdy[col], xp = sx[col];
            float u = 0.f, gbx = 0.f, pdx = 0.f;
#pragma unroll
            for (int k = 0; k < E; ++k) {
                const int n = rg + RG * k;
                gr[k] = a_next * gr[k] + sC[n] * dyp;      // g_t
                u += gr[k] * hp[k];
                gbx += gr[k] * sB[n];
                pdx += gr[k] * sB[n];
            }
            gbx *= xp;
            // dC_t[n] = sum_p h_t[n, p] dy_t[p], dB_t[n] = d_t sum_p g_t[n, p] x_t[p]: reduce over the
            // P threads of each row group (P divides 256: P <= 32 is a lane segment, else whole warps)
#pragma unroll
            for (int k = 0; k < E; ++k) {
                float vc = hc[k] * dyp, vb = gr[k] * xp;
                const int w = P < 32 ? P : 32;
                for (int o = w >> 1; o > 0; o >>= 1) {
                    vc += __shfl_xor_sync(0xffffffffu, vc, o);
                    vb += __shfl_xor_sync(0xffffffffu, vb, o);
                }
                if ((tid & (w - 1)) == 0) {
                    const int n = rg + RG * k;
                    atomicAdd(&p.dC_acc[(tk * G + g) * N + n], vc);
                    atomicAdd(&p.dB_acc[(tk * G + g) * N + n], d * vb);
                }
            }
            // dx_t[p] = D dy_t[p] + d_t sum_n g_t[n, p] B_t[n]: reduce over the RG row groups
            sdx[rg * P + col] = pdx;
            const float su = block_sum(u, red);
            const float sgbx = block_sum(gbx, red);      // (its barriers also publish sdx)
            if (tid < P) {
                float s = 0.f;
                for (int r = 0; r < RG; ++r) s += sdx[r * P + tid];
                ((T*)p.dx)[tk * H * P + (int64_t)h * P + tid] = from_f<T>(Dh * sdy[tid] + d * s);
            }
            if (tid == 0) {
                const float dd = su * a * Ah + sgbx;
                const float dz = dd * sigmoid_f(z);
                ((T*)p.ddt)[tk * H + h] = from_f<T>(dz);
                acc_dA += su * a * d;
                acc_dbias += dz;
            }
            if (tid < P) acc_dD += sdy[tid] * sx[tid];
            a_next = a;
        }
    }
    // dinit = a_first g_first (zero-length sequence: dfinal passes straight through)
    if (p.dinit) {
        float* dst = p.dinit + ((int64_t)seq * H + h) * NP;
#pragma unroll
        for (int k = 0; k < E; ++k) dst[(int64_t)(rg + RG * k) * P + col] = a_next * gr[k];
    }
    const float sdD = block_sum(acc_dD, red);
    if (tid == 0) {
        atomicAdd(&p.dA[h], acc_dA);
        atomicAdd(&p.ddt_bias[h], acc_dbias);
        atomicAdd(&p.dD[h], sdD);
    }
}

template <typename T>
__global__ void k_bwd_cast(const float* __restrict__ src, T* __restrict__ dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = from_f<T>(src[i]);
}

template <typename T, int E>
void launch_e(const BwdParams& p, unsigned grid, size_t smem, cudaStream_t st) {
    k_scan_bwd<T, E><<<grid, kBwdThreads, smem, st>>>(p);
}

template <typename T>
void launch_t(const BwdParams& p, int E, unsigned grid, size_t smem, cudaStream_t st) {
    switch (E) {
        case 1: launch_e<T, 1>(p, grid, smem, st); break;
        case 2: launch_e<T, 2>(p, grid, smem, st); break;
        case 4: launch_e<T, 4>(p, grid, smem, st); break;
        case 8: launch_e<T, 8>(p, grid, smem, st); break;
        case 16: launch_e<T, 16>(p, grid, smem, st); break;
        default: launch_e<T, 32>(p, grid, smem, st); break;
    }
}

}  // namespace

bool bwd_supported(const ScanArgs& a) {
    const int64_t NP = a.N * a.P;
    if (a.P > kBwdThreads || kBwdThreads % a.P != 0) return false;
    if (NP % kBwdThreads != 0 || NP / kBwdThreads > kBwdMaxE) return false;
    const int64_t E = NP / kBwdThreads;
    return E == 1 || E == 2 || E == 4 || E == 8 || E == 16 || E == 32;
}

size_t bwd_workspace_bytes(const ScanArgs& a) {
    const int64_t blocks = a.seq_idx ? (a.L + kBwdBlock - 1) / kBwdBlock + a.S
                                     : a.b * ((a.L + kBwdBlock - 1) / kBwdBlock);
    const size_t NP = (size_t)a.N * a.P;
    auto r = [](size_t v) { return (v + 255) & ~(size_t)255; };
    return r(sizeof(float) * blocks * a.H * NP) + r(sizeof(float) * a.S * a.H * kBwdBlock * NP) +
           2 * r(sizeof(float) * a.b * a.L * a.G * a.N);
}

int launch_scan_bwd(const ScanArgs& a, const BwdArgs& g, const SeqInfo& si64, void* ws, cudaStream_t st) {
    const size_t NP = (size_t)a.N * a.P;
    auto r = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const int64_t blocks = a.seq_idx ? (a.L + kBwdBlock - 1) / kBwdBlock + a.S
                                     : a.b * ((a.L + kBwdBlock - 1) / kBwdBlock);
    char* w = (char*)ws;
    BwdParams p;
    p.si = si64;
    p.ck_per_row = (a.L + kBwdBlock - 1) / kBwdBlock;
    p.x = a.x; p.dt = a.dt; p.B = a.B; p.C = a.C; p.dy = g.dy;
    p.dt_bias = a.dt_bias; p.A = a.A; p.D = a.D; p.init_state = a.init_state; p.dfinal = g.dfinal;
    p.dx = g.dx; p.ddt = g.ddt;
    p.ckpt = (float*)w; w += r(sizeof(float) * blocks * a.H * NP);
    p.scratch = (float*)w; w += r(sizeof(float) * a.S * a.H * kBwdBlock * NP);
    const int64_t nbc = a.b * a.L * a.G * a.N;
    p.dB_acc = (float*)w; w += r(sizeof(float) * nbc);
    p.dC_acc = (float*)w;
    p.ddt_bias = g.ddt_bias; p.dA = g.dA; p.dD = g.dD; p.dinit = g.dinit;
    p.H = (int)a.H; p.P = (int)a.P; p.N = (int)a.N; p.G = (int)a.G;
    cudaError_t e = cudaMemsetAsync(p.dB_acc, 0, sizeof(float) * nbc, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.dC_acc, 0, sizeof(float) * nbc, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(g.ddt_bias, 0, sizeof(float) * a.H, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(g.dA, 0, sizeof(float) * a.H, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(g.dD, 0, sizeof(float) * a.H, st);
    if (e != cudaSuccess) return 6;
    const int E = (int)(NP / kBwdThreads);
    const size_t smem = sizeof(float) * (2 * a.N + 2 * a.P + 32 + (kBwdThreads / a.P) * a.P);
    {
        ProfScope ps(K_SCAN_BWD, st);
        if (a.dtype == 0)
            launch_t<float>(p, E, (unsigned)(a.S * a.H), smem, st);
        else
            launch_t<__nv_bfloat16>(p, E, (unsigned)(a.S * a.H), smem, st);
    }
    int64_t cb = (nbc + 255) / 256;
    if (cb > 148 * 16) cb = 148 * 16;
    if (cb < 1) cb = 1;
    {
        ProfScope ps(K_BWD_CAST, st);
        if (a.dtype == 0) {
            k_bwd_cast<float><<<(unsigned)cb, 256, 0, st>>>(p.dB_acc, (float*)g.dB, nbc);
            k_bwd_cast<float><<<(unsigned)cb, 256, 0, st>>>(p.dC_acc, (float*)g.dC, nbc);
        } else {
            k_bwd_cast<__nv_bfloat16><<<(unsigned)cb, 256, 0, st>>>(p.dB_acc, (__nv_bfloat16*)g.dB, nbc);
            k_bwd_cast<__nv_bfloat16><<<(unsigned)cb, 256, 0, st>>>(p.dC_acc, (__nv_bfloat16*)g.dC, nbc);
        }
    }
    return 0;
}

}  // namespace ssd
