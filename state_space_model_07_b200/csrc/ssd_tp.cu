// ssd_tp.cu -- the two local steps of the head-sharded (tensor-parallel) mixer that are not
// matrix products: the grouped normalisation of the scan's output, and the quantised
// all-reduce of the output projection's partial sums.
//
// "5.3 Tensor Parallelism support and large-cluster training", section 4.1: each of the Tp
// devices holds H / Tp heads; the input projection is split by columns, the scan runs on the
// device's own heads, the normalisation is a group norm whose groups divide among the devices
// (so it needs no communication), and the output projection is split by rows, so the layer's
// output is the sum of the devices' partial products -- its one all-reduce.  "Scaling
// State-Space Models on Multiple GPUs with Tensor Parallelism" (abstract) lowers that
// all-reduce's bandwidth by quantising it.
//
// Quantisation: symmetric int8 per block of 64 consecutive columns of a row, scale =
// amax / 127, code = rint(x * (127 / amax)) (0 for an all-zero block).  The all-reduce over Tp
// ranks is a reduce-scatter then an all-gather, both on codes:
//   1. every rank quantises its partial (T, D) into Tp column chunks (chunk j = columns
//      [j D / Tp, (j + 1) D / Tp), stored chunk-major so each is contiguous);
//   2. an all-to-all sends chunk j to rank j;
//   3. rank j dequantises the Tp chunks it received, sums them in fp32 and quantises the sum;
//   4. an all-gather of the summed chunks; every rank dequantises all of them into (T, D).
// Each rank sends and receives 2 (Tp - 1) / Tp of the codes (one byte per value plus a 4-byte
// scale per 64), against 2 bytes per value for a bf16 ring all-reduce.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

namespace ssd {
namespace {

constexpr int kQBlock = 64;   // columns per quantisation block (four per lane of a half warp)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Group norm of each row: one warp per (row, group) of gs = C / ngroups channels; mean and
// variance (biased) over the group in fp32, two passes over values held in registers, then
// gamma, beta per channel.  Vector form: 16-byte chunks (8 bf16 or 4 fp32 values), chunk m of
// the group to lane m % 32, at most kMaxChunks per lane (gs <= 2048); rows and groups must start
// on 16-byte boundaries.  Scalar form otherwise (gs <= 32 kMaxPerLane).
constexpr int kMaxPerLane = 64;
constexpr int kMaxChunks = 8;

template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int kN = 4;
    static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
    static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kN = 8;
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T, int kCh>
__global__ void k_group_norm_vec(const T* __restrict__ x, const float* __restrict__ gamma,
                                 const float* __restrict__ beta, float eps, int64_t rows, int C, int gs,
                                 T* __restrict__ out) {
    constexpr int VN = Vec16<T>::kN;
    const int lane = threadIdx.x & 31;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int ng = C / gs, nch = gs / VN;
    if (wid >= rows * ng) return;
    const int64_t row = wid / ng;
    const int c0 = (int)(wid % ng) * gs;
    const T* xr = x + row * C + c0;
    float v[kCh][VN];
    float s = 0.f;
#pragma unroll
    for (int m = 0; m < kCh; ++m) {
        const int ch = lane + 32 * m;
        if (ch < nch) {
            Vec16<T>::load(xr + ch * VN, v[m]);
#pragma unroll
            for (int i = 0; i < VN; ++i) s += v[m][i];
        }
    }
    const float mean = warp_sum(s) / gs;
    float q = 0.f;
#pragma unroll
    for (int m = 0; m < kCh; ++m)
        if (lane + 32 * m < nch) {
#pragma unroll
            for (int i = 0; i < VN; ++i) {
                const float d = v[m][i] - mean;
                q += d * d;
            }
        }
    const float rstd = rsqrtf(warp_sum(q) / gs + eps);
    T* orow = out + row * C + c0;
#pragma unroll
    for (int m = 0; m < kCh; ++m) {
        const int ch = lane + 32 * m;
        if (ch < nch) {
            float o[VN];
            const int c = c0 + ch * VN;
#pragma unroll
            for (int i = 0; i < VN; i += 4) {
                const float4 g = *reinterpret_cast<const float4*>(gamma + c + i);
                const float4 b = *reinterpret_cast<const float4*>(beta + c + i);
                o[i] = (v[m][i] - mean) * rstd * g.x + b.x;
                o[i + 1] = (v[m][i + 1] - mean) * rstd * g.y + b.y;
                o[i + 2] = (v[m][i + 2] - mean) * rstd * g.z + b.z;
                o[i + 3] = (v[m][i + 3] - mean) * rstd * g.w + b.w;
            }
            Vec16<T>::store(orow + ch * VN, o);
        }
    }
}

template <typename T>
__global__ void k_group_norm(const T* __restrict__ x, const float* __restrict__ gamma, const float* __restrict__ beta,
                             float eps, int64_t rows, int C, int gs, T* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int ng = C / gs;
    if (wid >= rows * ng) return;
    const int64_t row = wid / ng;
    const int c0 = (int)(wid % ng) * gs;
    const T* xr = x + row * C + c0;
    float v[kMaxPerLane];
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) {
        const int c = lane + 32 * k;
        v[k] = c < gs ? to_f<T>(xr[c]) : 0.f;
        s += v[k];
    }
    const float mean = warp_sum(s) / gs;
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) {
        const int c = lane + 32 * k;
        const float d = c < gs ? v[k] - mean : 0.f;
        q += d * d;
    }
    const float rstd = rsqrtf(warp_sum(q) / gs + eps);
    T* orow = out + row * C + c0;
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) {
        const int c = lane + 32 * k;
        if (c < gs) orow[c] = from_f<T>((v[k] - mean) * rstd * gamma[c0 + c] + beta[c0 + c]);
    }
}

// Quantisation: half a warp per 64-column block, four values per lane (16-byte loads of fp32,
// 4-byte loads and stores of codes).  `hl` = lane within the half warp; the 16 lanes of a half
// agree on the block's amax by shuffles within the half, so every lane of the warp takes part
// in them (a half past the end works on block 0 and stores nothing).
__device__ __forceinline__ float half_max(float v) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ signed char code_of(float v, float inv) {
    return (signed char)fmaxf(-127.f, fminf(127.f, rintf(__fmul_rn(v, inv))));
}

// Codes of four values of a block and the block's scale.
__device__ __forceinline__ char4 quant4(float a, float b, float c, float d, float& scale) {
    const float amax = half_max(fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d))));
    const float inv = amax > 0.f ? 127.f / amax : 0.f;
    scale = amax / 127.f;
    return make_char4(code_of(a, inv), code_of(b, inv), code_of(c, inv), code_of(d, inv));
}

// x (T, D) fp32 -> codes (Tp, T, Dc) and scales (Tp, T, Dc / 64), Dc = D / Tp.
// Each half warp takes blocks hid and hid + halves (both loads issued before either is used).
__global__ void k_quant_chunks(const float* __restrict__ x, int64_t T, int D, int Tp, int8_t* __restrict__ q,
                               float* __restrict__ scale) {
    const int hl = threadIdx.x & 15;
    const int64_t halves = ((int64_t)gridDim.x * blockDim.x) >> 4;
    const int64_t hid0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int nb = D / kQBlock, Dc = D / Tp, nbc = Dc / kQBlock;
    float4 u[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int64_t hid = hid0 + k * halves;
        const int64_t hb = hid < T * nb ? hid : 0;
        u[k] = *reinterpret_cast<const float4*>(x + (hb / nb) * D + (int64_t)(hb % nb) * kQBlock + 4 * hl);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int64_t hid = hid0 + k * halves;
        float sc;
        const char4 c = quant4(u[k].x, u[k].y, u[k].z, u[k].w, sc);
        if (hid < T * nb) {
            const int64_t t = hid / nb;
            const int blk = (int)(hid % nb), j = blk / nbc, bc = blk % nbc;
            const int64_t o = (int64_t)j * T + t;
            *reinterpret_cast<char4*>(q + o * Dc + (int64_t)bc * kQBlock + 4 * hl) = c;
            if (hl == 0) scale[o * nbc + bc] = sc;
        }
    }
}

// The reduce step: Tp chunks (Tp, T, Dc) of codes and scales -> their dequantised fp32 sum (in
// rank order, each product and sum rounded separately) -> codes (T, Dc) and scales (T, Dc / 64).
__global__ void k_dequant_sum_quant(const int8_t* __restrict__ qin, const float* __restrict__ sin, int Tp, int64_t T,
                                    int Dc, int8_t* __restrict__ qout, float* __restrict__ sout) {
    const int hl = threadIdx.x & 15;
    const int64_t hid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int nbc = Dc / kQBlock;
    const bool live = hid < T * nbc;
    const int64_t hb = live ? hid : 0;
    const int64_t t = hb / nbc;
    const int bc = (int)(hb % nbc);
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < Tp; ++r) {
        const float sc = sin[((int64_t)r * T + t) * nbc + bc];
        const char4 c = *reinterpret_cast<const char4*>(qin + ((int64_t)r * T + t) * Dc + (int64_t)bc * kQBlock + 4 * hl);
        a[0] = __fadd_rn(a[0], __fmul_rn(sc, (float)c.x));
        a[1] = __fadd_rn(a[1], __fmul_rn(sc, (float)c.y));
        a[2] = __fadd_rn(a[2], __fmul_rn(sc, (float)c.z));
        a[3] = __fadd_rn(a[3], __fmul_rn(sc, (float)c.w));
    }
    float sc;
    const char4 c = quant4(a[0], a[1], a[2], a[3], sc);
    if (live) {
        *reinterpret_cast<char4*>(qout + t * Dc + (int64_t)bc * kQBlock + 4 * hl) = c;
        if (hl == 0) sout[t * nbc + bc] = sc;
    }
}

// Codes (Tp, T, Dc) and scales -> out (T, D), chunk j into columns [j Dc, (j + 1) Dc).
template <typename T> __device__ __forceinline__ void store4(T* p, float a, float b, float c, float d);
template <> __device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float a, float b, float c, float d) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                              *reinterpret_cast<const uint32_t*>(&hi));
}

template <typename T>
__global__ void k_dequant_chunks(const int8_t* __restrict__ q, const float* __restrict__ s, int Tp, int64_t Tn,
                                 int Dc, T* __restrict__ out) {
    const int hl = threadIdx.x & 15;
    const int64_t hid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int nbc = Dc / kQBlock;
    if (hid >= (int64_t)Tp * Tn * nbc) return;
    const int bc = (int)(hid % nbc);
    const int64_t jt = hid / nbc;                 // j T + t
    const int j = (int)(jt / Tn);
    const int64_t t = jt % Tn;
    const float sc = s[hid];
    const char4 c = *reinterpret_cast<const char4*>(q + jt * Dc + (int64_t)bc * kQBlock + 4 * hl);
    store4<T>(out + t * ((int64_t)Dc * Tp) + (int64_t)j * Dc + (int64_t)bc * kQBlock + 4 * hl,
              __fmul_rn(sc, (float)c.x), __fmul_rn(sc, (float)c.y), __fmul_rn(sc, (float)c.z),
              __fmul_rn(sc, (float)c.w));
}

unsigned warps_grid(int64_t warps) { return (unsigned)((warps * 32 + 255) / 256); }
unsigned halves_grid(int64_t halves) { return (unsigned)((halves * 16 + 255) / 256); }

}  // namespace

bool group_norm_supported(int64_t C, int64_t ngroups) {
    return ngroups >= 1 && C % ngroups == 0 && C / ngroups <= 32 * kMaxPerLane;
}

namespace {
template <typename T>
void group_norm_typed(const T* x, const float* gamma, const float* beta, float eps, int64_t rows, int64_t C,
                      int64_t ngroups, T* out, cudaStream_t st) {
    const int gs = (int)(C / ngroups);
    const bool vec = (gs * sizeof(T)) % 16 == 0 && gs % 4 == 0 && ((uintptr_t)x & 15u) == 0 &&
                     ((uintptr_t)out & 15u) == 0 && ((uintptr_t)gamma & 15u) == 0 && ((uintptr_t)beta & 15u) == 0 &&
                     gs / (int)(16 / sizeof(T)) <= 32 * kMaxChunks;
    const unsigned grid = warps_grid(rows * ngroups);
    // chunks per lane: as few registers as the group size needs (occupancy)
    const int ch = (gs / (int)(16 / sizeof(T)) + 31) / 32;
    if (vec && ch <= 1)
        k_group_norm_vec<T, 1><<<grid, 256, 0, st>>>(x, gamma, beta, eps, rows, (int)C, gs, out);
    else if (vec && ch <= 2)
        k_group_norm_vec<T, 2><<<grid, 256, 0, st>>>(x, gamma, beta, eps, rows, (int)C, gs, out);
    else if (vec && ch <= 3)
        k_group_norm_vec<T, 3><<<grid, 256, 0, st>>>(x, gamma, beta, eps, rows, (int)C, gs, out);
    else if (vec && ch <= 4)
        k_group_norm_vec<T, 4><<<grid, 256, 0, st>>>(x, gamma, beta, eps, rows, (int)C, gs, out);
    else if (vec)
        k_group_norm_vec<T, kMaxChunks><<<grid, 256, 0, st>>>(x, gamma, beta, eps, rows, (int)C, gs, out);
    else
        k_group_norm<T><<<grid, 256, 0, st>>>(x, gamma, beta, eps, rows, (int)C, gs, out);
}
}  // namespace

void launch_group_norm(int dtype, const void* x, const float* gamma, const float* beta, float eps, int64_t rows,
                       int64_t C, int64_t ngroups, void* out, cudaStream_t st) {
    ProfScope ps(K_GROUP_NORM, st);
    if (dtype == 0)
        group_norm_typed<float>((const float*)x, gamma, beta, eps, rows, C, ngroups, (float*)out, st);
    else
        group_norm_typed<__nv_bfloat16>((const __nv_bfloat16*)x, gamma, beta, eps, rows, C, ngroups,
                                        (__nv_bfloat16*)out, st);
}

void launch_quant_chunks(const float* x, int64_t T, int64_t D, int64_t Tp, int8_t* q, float* scale, cudaStream_t st) {
    ProfScope ps(K_QUANT, st);
    k_quant_chunks<<<halves_grid((T * (D / kQBlock) + 1) / 2), 256, 0, st>>>(x, T, (int)D, (int)Tp, q, scale);
}

void launch_dequant_sum_quant(const int8_t* qin, const float* sin, int64_t Tp, int64_t T, int64_t Dc, int8_t* qout,
                              float* sout, cudaStream_t st) {
    ProfScope ps(K_QUANT, st);
    k_dequant_sum_quant<<<halves_grid(T * (Dc / kQBlock)), 256, 0, st>>>(qin, sin, (int)Tp, T, (int)Dc, qout, sout);
}

void launch_dequant_chunks(int dtype, const int8_t* q, const float* s, int64_t Tp, int64_t T, int64_t Dc, void* out,
                           cudaStream_t st) {
    ProfScope ps(K_QUANT, st);
    const unsigned grid = halves_grid(Tp * T * (Dc / kQBlock));
    if (dtype == 0)
        k_dequant_chunks<float><<<grid, 256, 0, st>>>(q, s, (int)Tp, T, (int)Dc, (float*)out);
    else
        k_dequant_chunks<__nv_bfloat16><<<grid, 256, 0, st>>>(q, s, (int)Tp, T, (int)Dc, (__nv_bfloat16*)out);
}

}  // namespace ssd
