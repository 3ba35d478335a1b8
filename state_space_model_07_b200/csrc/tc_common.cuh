// tc_common.cuh -- pieces shared by the tensor-core kernels (the scan in ssd_tc.cu and the
// state-to-output pass in ssd_state_out.cu): tile constants, the bounded mbarrier waits,
// warp-level arrivals, the fast softplus, bf16 -> fp16 packing, and on the host the tensor-map
// encoder, the SM count and the work split of the state-to-output pass.
#pragma once

#include <cuda.h>
#include <algorithm>
#include <cmath>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "ssd_common.cuh"
#include "tc_ptx.cuh"

namespace ssd {
namespace tc {

using namespace ptx;

constexpr int kT = 128;             // tokens per tile
constexpr int kP = 64;              // headdim handled by this kernel
constexpr uint32_t kTileBytesX = kT * kP * 2;     // 16 KB
constexpr uint32_t kBoxBytes = kT * 64 * 2;       // one 64-column box of a B or C tile: 16 KB

struct TcCtl {
    int abort;
};

__device__ __forceinline__ __half2 u2h(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t h2u(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Bounded wait of a single issuing thread; false once the CTA has given up.
__device__ __forceinline__ bool wait_bar(TcCtl& c, uint64_t* bar, uint32_t parity, int32_t* status) {
    if (*(volatile int*)&c.abort) return false;
    if (!mbar_wait(bar, parity)) {
        c.abort = 1;
        if (status) atomicExch(status, kStatusTimeout);
        return false;
    }
    return true;
}

// Bounded wait of a whole warp; the result is the same in every lane, so the
// warp-collective TMEM instructions that follow stay uniform even on the
// error path.  Every warp of a role polls its waits itself: a rendezvous of the
// role's warps at each wait would let one lagging warp hold the whole role back.
__device__ __forceinline__ bool wait_bar_w(TcCtl& c, uint64_t* bar, uint32_t parity, int32_t* status) {
    return __all_sync(0xffffffffu, wait_bar(c, bar, parity, status));
}

// softplus(z) = max(z, 0) + log(1 + e), e = exp(-|z|) in (0, 1], with the
// hardware base-2 exponential and logarithm; for e < 2^-7 the logarithm is
// replaced by its Taylor series e - e^2/2 + e^3/3 (truncation < e^4/4 < 2^-30,
// and no cancellation in 1 + e).  Relative error ~1e-6, which the decay and
// the update d B x^T pass through unamplified.
__device__ __forceinline__ float softplus_fast(float z) {
    const float e = ex2(-fabsf(z) * 1.4426950408889634f);
    float l;
    if (e < 0.0078125f) {
        l = e * fmaf(e, fmaf(e, 0.333333343f, -0.5f), 1.f);
    } else {
        float lg;
        asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(1.f + e));
        l = lg * 0.693147182f;
    }
    return fmaxf(z, 0.f) + l;
}

// One arrival per warp: the warp's lanes synchronise first (ordering their
// shared-memory and TMEM writes before the release of the arrival), so the
// barrier counts warps, not threads.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// bf16 -> fp16 of eight packed values.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
    return make_uint4(pack_f16x2(bf16lo(v.x), bf16hi(v.x)), pack_f16x2(bf16lo(v.y), bf16hi(v.y)),
                      pack_f16x2(bf16lo(v.z), bf16hi(v.z)), pack_f16x2(bf16lo(v.w), bf16hi(v.w)));
}

// ---- host ------------------------------------------------------------------------------------

// SMs of the current device (queried once per device).
inline int sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        cache[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
    }
    return cache[dev];
}

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// (inner, mid, outer) tensor with `inner` contiguous, box (64, 1, 128),
// 128-byte swizzle; out-of-range rows read as zero.
inline bool make_map(CUtensorMap* m, CUtensorMapDataType ty, const void* base, uint64_t inner, uint64_t mid,
              uint64_t outer) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
    cuuint32_t box[3] = {64, 1, kT}, es[3] = {1, 1, 1};
    return enc(m, ty, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Parts for k_state_out over spans of `tiles` tiles: the count whose CTAs (items per part)
// best fill whole waves of S SMs, with at least four tiles per part.
inline void plan_parts(int tiles, int64_t items, int S, int& nparts, int& tpp) {
    double best = -1.0;
    nparts = 1;
    tpp = tiles;
    for (int np = 1; np <= 32 && tiles / np >= 4; ++np) {
        const int t = (tiles + np - 1) / np;
        const int used = (tiles + t - 1) / t;
        const double x = (double)(items * used) / S;
        const double eff = x / std::ceil(x);
        if (eff > best + 0.02) {
            best = eff;
            nparts = used;
            tpp = t;
        }
    }
}

}  // namespace tc
}  // namespace ssd
