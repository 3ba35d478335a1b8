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
// bandwidth.  Every thread issues its state loads (float4, evict-first)
// before it reads dt, x, B or C, so the state stream does not wait behind the
// small per-head loads, and keeps up to kBatch rows in flight.
#include <stdio.h>
#include <stdlib.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

namespace ssd {

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
    static __device__ __forceinline__ void store(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
};
template <> struct Vec4<__nv_bfloat16> {
    // 4 bf16 = 8 bytes; bf16 -> fp32 is exact (the bits move to the high half)
    static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float4 v) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&lo);
        u.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(p) = u;
    }
};

// Block (bh, cs) of a (batch, head) whose P columns are split over CS blocks:
// the block owns float4 columns [cs Pc, cs Pc + Pc), Pc = P / (4 CS), of every
// state row, so its part of y = C^T h is complete without any exchange
// between blocks.  Thread (rg, col) takes float4 column `col` of rows rg,
// rg + RG, ... (RG = kThreads / Pc), up to kBatch rows in flight at a time.
template <typename T, int kThreads, int kBatch>
__global__ void __launch_bounds__(kThreads)
k_state_update(float* __restrict__ state, const T* __restrict__ x, const T* __restrict__ dt,
               const float* __restrict__ dt_bias, const float* __restrict__ A,
               const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D,
               T* __restrict__ y, int H, int P, int N, int G, int CS) {
    extern __shared__ float4 red[];     // kThreads partial y columns
    const int cs = (int)(blockIdx.x % CS);
    const int64_t bh = blockIdx.x / CS;
    const int64_t bi = bh / H;
    const int h = (int)(bh % H);
    const int g = h / (H / G);
    const int tid = threadIdx.x;
    const int Pc = P / (4 * CS);
    const int RG = kThreads / Pc;
    const int col = tid % Pc, rg = tid / Pc;
    const int c4 = cs * Pc + col;                              // float4 column within the row
    const int nrows = rg < RG ? (N - rg + RG - 1) / RG : 0;   // rows of this thread

    float4* st = reinterpret_cast<float4*>(state + bh * N * (int64_t)P) + c4;
    const int P4 = P / 4;
    float4 v[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k)
        if (k < nrows) v[k] = __ldcs(st + (int64_t)(rg + k * RG) * P4);

    const float d = softplus_f(to_f<T>(dt[bh]) + (dt_bias ? dt_bias[h] : 0.f));
    const float dA = expf(d * A[h]);
    const float4 x4 = rg < RG ? Vec4<T>::load(x + bh * P + 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
    const T* Bg = B + (bi * G + g) * N;
    const T* Cg = C + (bi * G + g) * N;
    float4 yacc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < nrows; k0 += kBatch) {
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            if (k0 + k < nrows) {
                const int n = rg + (k0 + k) * RG;
                const float bn = d * to_f<T>(Bg[n]), cn = to_f<T>(Cg[n]);
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
        if (k0 + kBatch < nrows) {
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
                if (k0 + kBatch + k < nrows) v[k] = __ldcs(st + (int64_t)(rg + (k0 + kBatch + k) * RG) * P4);
        }
    }
    red[tid] = yacc;
    __syncthreads();
    if (tid < Pc) {
        float4 s = red[tid];
        for (int q = 1; q < RG; ++q) {
            const float4 o = red[q * Pc + tid];
            s.x += o.x; s.y += o.y; s.z += o.z; s.w += o.w;
        }
        const float Dh = D ? D[h] : 0.f;
        Vec4<T>::store(y + bh * P + 4 * c4,
                       make_float4(s.x + Dh * x4.x, s.y + Dh * x4.y, s.z + Dh * x4.z, s.w + Dh * x4.w));
    }
}

namespace {

struct DecodeCfg {
    int threads, batch, cs;
};

// SSD_DECODE_CFG="threads,batch,cs" picks one of the compiled shapes below
// (for tests and tuning); unset: the choice in decode_cfg().  Read once.
DecodeCfg forced_decode_cfg() {
    static DecodeCfg v = {-1, 0, 0};
    if (v.threads < 0) {
        v = {0, 0, 0};
        const char* e = getenv("SSD_DECODE_CFG");
        int t = 0, b = 0, c = 0;
        if (e && sscanf(e, "%d,%d,%d", &t, &b, &c) == 3) v = {t, b, c};
    }
    return v;
}

bool cfg_fits(const UpdateArgs& a, DecodeCfg c) {
    const int P4 = (int)(a.P / 4);
    if (c.cs < 1 || P4 % c.cs) return false;
    const int Pc = P4 / c.cs;
    return c.threads % Pc == 0 && c.threads / Pc >= 1;
}

// Default: 128 threads, each block owning 16 columns (64 bytes) of every state
// row, so one (batch, head) spreads over P / 16 blocks and even a small decode
// batch keeps every SM streaming; 4 rows in flight per thread.  (Measured on
// B200 against 256- and 512-thread blocks, whole rows per block and 8 or 16
// rows in flight: best or within 1% on b8 H80, b64 H64 (N 128) and b16 H128
// (N 256).)  P not a multiple of 16: whole rows per block.
DecodeCfg decode_cfg(const UpdateArgs& a) {
    const DecodeCfg f = forced_decode_cfg();
    if (f.threads && cfg_fits(a, f)) return f;
    const int P4 = (int)(a.P / 4);
    return {128, 4, P4 % 4 == 0 ? P4 / 4 : 1};
}

template <typename T, int kThreads, int kBatch>
void launch_shape(const UpdateArgs& a, int cs, cudaStream_t st) {
    const unsigned grid = (unsigned)(a.b * a.H * cs);
    k_state_update<T, kThreads, kBatch><<<grid, kThreads, sizeof(float4) * kThreads, st>>>(
        a.state, (const T*)a.x, (const T*)a.dt, a.dt_bias, a.A, (const T*)a.B, (const T*)a.C, a.D, (T*)a.y,
        (int)a.H, (int)a.P, (int)a.N, (int)a.G, cs);
}

template <typename T>
void launch_typed(const UpdateArgs& a, cudaStream_t st) {
    const DecodeCfg c = decode_cfg(a);
    if (c.threads == 128 && c.batch == 16) launch_shape<T, 128, 16>(a, c.cs, st);
    else if (c.threads == 128 && c.batch == 8) launch_shape<T, 128, 8>(a, c.cs, st);
    else if (c.threads == 128 && c.batch == 4) launch_shape<T, 128, 4>(a, c.cs, st);
    else if (c.threads == 64 && c.batch == 8) launch_shape<T, 64, 8>(a, c.cs, st);
    else if (c.threads == 512 && c.batch == 4) launch_shape<T, 512, 4>(a, c.cs, st);
    else if (c.threads == 256 && c.batch == 16) launch_shape<T, 256, 16>(a, c.cs, st);
    else if (c.threads == 256 && c.batch == 4) launch_shape<T, 256, 4>(a, c.cs, st);
    else launch_shape<T, 256, 8>(a, c.cs, st);
}

}  // namespace

void launch_state_update(const UpdateArgs& a, cudaStream_t st) {
    ProfScope ps(K_STATE_UPDATE, st);
    if (a.dtype == 0)
        launch_typed<float>(a, st);
    else
        launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace ssd
