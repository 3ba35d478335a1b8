// ssd_tc.cu -- tensor-core (tcgen05) path of the chunked scan, bf16 inputs.
//
// Block decomposition of "5.3 Tensor Parallelism support and large-cluster
// training", section 3.2, mapped onto one B200 SM per (sequence, head):
//
//   * The sequence is walked in 128-token tiles (one TMEM lane per token).  A
//     chunk of 256 tokens is two tiles joined by the same N x P state hand-over
//     as two chunks are, so the result equals the chunked form up to rounding.
//   * Per tile, with d = softplus(dt + dt_bias), cs = tile-local inclusive
//     cumulative sum of d*A:
//       CB   = C B^T                               tcgen05, fp16 x fp16 -> fp32 TMEM
//       S    = CB o exp(cs_j - cs_i) d_i (i <= j)  math warps, written back to TMEM
//       Yd   = S x                                 tcgen05, A from TMEM
//       Yo   = C h_prev                            tcgen05 (low-rank term of the
//                                                  state entering the tile)
//       Sc   = B^T (w o x), w_i = d_i exp(cs_last - cs_i)     tcgen05
//       y    = Yd + exp(cs_j) Yo + D x             math warps -> bf16 -> HBM
//       h    = exp(cs_last) h_prev + Sc            math warps, fp32 in registers
//   * The operands the math warps produce (S, h_prev, w o x) are rounded to fp16
//     (11-bit significand): bf16's 8 bits miss the 1e-2 (1 + |y|) accuracy bound.
//     B and C are converted to fp16 once by k_tc_prep; x is converted in place in
//     shared memory.  C B^T on those fp16 copies is exact for normal-range
//     bf16 values.
//
// Warp roles (288 threads): warps 0-7 are two math warpgroups (thread j of
// each owns token / state row j of the tile, TMEM lane j, and one half of the
// row's columns); warp 8 lane 0 issues the TMA loads (two-stage ring) and
// every tcgen05.mma.  All waits are bounded: on a
// timeout the kernel records SSD_ERR_TIMEOUT in the status word and returns
// after freeing its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <stdio.h>

#include "ssd_common.cuh"
#include "ssd_prof.h"
#include "ssd_tc.h"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace ptx;

constexpr int kT = 128;           // tokens per tile
constexpr int kP = 64;            // headdim handled by this kernel
constexpr int kN = 128;           // dstate handled by this kernel
constexpr int kMathThreads = 256;
constexpr int kThreads = 288;
constexpr uint32_t kTmemCols = 512;
// TMEM column map
constexpr uint32_t kColCB = 0, kColS = 128, kColYd = 192, kColYo = 256, kColSc = 320;

constexpr uint32_t kTileBytesX = kT * kP * 2;        // 16 KB
constexpr uint32_t kHalfBytes = kT * 64 * 2;         // one 64-column half of a B or C tile: 16 KB
constexpr uint32_t kStageBytes = kTileBytesX + 4 * kHalfBytes;

struct __align__(1024) TcSmem {
    uint8_t x[2][kTileBytesX];        // x tile per stage (bf16 from TMA, fp16 after conversion)
    uint8_t b[2][2][kHalfBytes];      // B tile (fp16) per stage: n in [0,64) and [64,128)
    uint8_t c[2][2][kHalfBytes];      // C tile (fp16)
    uint8_t wx[kTileBytesX];          // (w o x) fp16, token rows
    uint8_t hs[kN * kP * 2];          // h_prev fp16, state rows
    float cs[kT];          // tile-local cumulative decay, base-2 exponent
    float d[kT];
    float colfac[kT];
    float wtot[2][4];
    uint64_t full[2];
    uint64_t cb_done, os_done, yd_done, ops_ready, s_ready, epi_done;
    uint32_t tmem_base;
    int abort;
};

struct TcParams {
    SeqInfo si;
    const __nv_bfloat16* dt;
    const float* dt_bias;
    const float* A;
    const float* D;
    const float* init_state;
    float* final_state;
    __nv_bfloat16* y;
    int32_t* status;
    int H, G;
};

__device__ __forceinline__ void math_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ void set_abort(TcSmem& s, int32_t* status) {
    s.abort = 1;
    if (status) atomicExch(status, kStatusTimeout);
}

// Bounded wait shared by all roles; false once the CTA has given up.
__device__ __forceinline__ bool wait_bar(TcSmem& s, uint64_t* bar, uint32_t parity, int32_t* status) {
    if (*(volatile int*)&s.abort) return false;
    if (!mbar_wait(bar, parity)) {
        set_abort(s, status);
        return false;
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
k_tc_scan(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
          const __grid_constant__ CUtensorMap tm_c, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem& s = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, G = p.G;
    const int h = blockIdx.x % H;
    const int seq = blockIdx.x / H;
    const int g = h / (H / G);

    int64_t row, t0, t1;
    seq_span(p.si, seq, row, t0, t1);
    const int64_t len = t1 > t0 ? t1 - t0 : 0;
    const int nt = (int)((len + kT - 1) / kT);
    const int64_t tok0 = row * p.si.L + t0;  // global token index of the sequence start

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) mbar_init(&s.full[i], 1);
        mbar_init(&s.cb_done, 1);
        mbar_init(&s.os_done, 1);
        mbar_init(&s.yd_done, 1);
        mbar_init(&s.ops_ready, kMathThreads);
        mbar_init(&s.s_ready, kMathThreads);
        mbar_init(&s.epi_done, kMathThreads);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&s.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------------ control
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            tma_prefetch_desc(&tm_c);
            int loads_issued = 0;
            auto issue_loads = [&](int t) {
                const int st = t & 1;
                const int tok = (int)(tok0 + (int64_t)t * kT);
                mbar_expect_tx(&s.full[st], kStageBytes);
                tma_load_3d(s.x[st], &tm_x, &s.full[st], 0, h, tok);
                for (int k = 0; k < 2; ++k) {
                    tma_load_3d(s.b[st][k], &tm_b, &s.full[st], 64 * k, g, tok);
                    tma_load_3d(s.c[st][k], &tm_c, &s.full[st], 64 * k, g, tok);
                }
                ++loads_issued;
            };
            const uint32_t id_cb = idesc_f16(128, 128, 0, 0);
            const uint32_t id_pn = idesc_f16(128, 64, 0, 1);   // K-major A, MN-major B
            const uint32_t id_mn = idesc_f16(128, 64, 1, 1);   // MN-major A and B
            auto issue_cb = [&](int t) {
                const int st = t & 1;
                const uint32_t cb = smem_u32(s.c[st][0]), bb = smem_u32(s.b[st][0]);
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                    mma_ss(tmem + kColCB, sdesc_sw128(cb + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024),
                           id_cb, k > 0);
                }
                mma_commit(&s.cb_done);
            };
            issue_loads(0);
            if (nt > 1) issue_loads(1);
            bool ok = wait_bar(s, &s.full[0], 0, p.status);
            if (ok) {
                tc_fence_after();
                issue_cb(0);
            }
            for (int t = 0; ok && t < nt; ++t) {
                const int st = t & 1;
                // low-rank term of the entering state and the tile's own state
                if (!(ok = wait_bar(s, &s.ops_ready, t & 1, p.status))) break;
                if (t > 0 && !(ok = wait_bar(s, &s.epi_done, (t - 1) & 1, p.status))) break;
                tc_fence_after();
                {
                    const uint32_t cb = smem_u32(s.c[st][0]), bb = smem_u32(s.b[st][0]);
                    const uint32_t hsb = smem_u32(s.hs), wxb = smem_u32(s.wx);
                    for (int k = 0; k < kN / 16; ++k) {
                        const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                        mma_ss(tmem + kColYo, sdesc_sw128(cb + off, 16, 1024),
                               sdesc_sw128(hsb + k * 2048, kHalfBytes, 1024), id_pn, k > 0);
                    }
                    for (int k = 0; k < kT / 16; ++k)
                        mma_ss(tmem + kColSc, sdesc_sw128(bb + k * 2048, kHalfBytes, 1024),
                               sdesc_sw128(wxb + k * 2048, kHalfBytes, 1024), id_mn, k > 0);
                    mma_commit(&s.os_done);
                }
                // intra-tile quadratic block
                if (!(ok = wait_bar(s, &s.s_ready, t & 1, p.status))) break;
                tc_fence_after();
                {
                    const uint32_t xb = smem_u32(s.x[st]);
                    for (int k = 0; k < kT / 16; ++k)
                        mma_ts(tmem + kColYd, tmem + kColS + k * 8,
                               sdesc_sw128(xb + k * 2048, kHalfBytes, 1024), id_pn, k > 0);
                    mma_commit(&s.yd_done);
                }
                if (t + 1 < nt) {
                    if (!(ok = wait_bar(s, &s.full[(t + 1) & 1], ((t + 1) >> 1) & 1, p.status))) break;
                    tc_fence_after();
                    issue_cb(t + 1);
                }
                if (t + 2 < nt) {
                    // stage st is free once every MMA of tile t has completed
                    if (!(ok = wait_bar(s, &s.yd_done, t & 1, p.status))) break;
                    issue_loads(t + 2);
                }
            }
            if (!ok) {
                // Give up: let the copies already in flight land before the CTA exits.
                for (int t = 0; t < loads_issued; ++t) mbar_wait(&s.full[t & 1], (t >> 1) & 1, 200000000ull);
            }
        }
    } else {
        // -------------------------------------------------------------- math
        // Thread (quarter, ch, lane): token / state row j = 32 quarter + lane
        // (TMEM lane j), columns [32 ch, 32 ch + 32) of its row.
        const int quarter = warp & 3, ch = warp >> 2;
        const int j = 32 * quarter + lane;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float kLog2e = 1.4426950408889634f;
        const float A2 = p.A[h] * kLog2e;     // decays are kept as base-2 exponents
        const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
        const float Dh = p.D ? p.D[h] : 0.f;
        float hreg[32];
        {
            const float* src = p.init_state
                ? p.init_state + (((int64_t)seq * H + h) * kN + j) * kP + 32 * ch : nullptr;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                float4 v = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                hreg[c] = v.x; hreg[c + 1] = v.y; hreg[c + 2] = v.z; hreg[c + 3] = v.w;
            }
        }
        float cs2_last_prev = 0.f;
        bool ok = true;
        // dt of this thread's token in the next tile, loaded one tile ahead
        float dt_next = 0.f;
        if (nt > 0 && j < len) dt_next = __bfloat162float(p.dt[(tok0 + j) * H + h]);
        for (int t = 0; t < nt; ++t) {
            const int st = t & 1;
            const int q = (int)(len - (int64_t)t * kT < kT ? len - (int64_t)t * kT : kT);
            const int64_t tok = tok0 + (int64_t)t * kT + j;
            // (1) step sizes and the tile-local cumulative log2-decay (both warpgroups
            //     compute it; warpgroup 0 publishes it)
            float dj = 0.f, a = 0.f;
            if (j < q) {
                dj = softplus_f(dt_next + bias);
                a = dj * A2;
            }
            if (t + 1 < nt && (int64_t)(t + 1) * kT + j < len)
                dt_next = __bfloat162float(p.dt[(tok + kT) * H + h]);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, a, o);
                if (lane >= o) a += u;
            }
            if (lane == 31) s.wtot[ch][quarter] = a;
            math_bar();
            for (int w = 0; w < quarter; ++w) a += s.wtot[ch][w];
            const float cs2j = a;
            // column factor of the rank-1 split 2^(cs_j - cs_i) = 2^(cs_j - cs_m) 2^(cs_m - cs_i),
            // pivot m = last token of i's 32-token block (lane 31 of this warp)
            const float cs2_pivot = __shfl_sync(0xffffffffu, cs2j, 31);
            if (ch == 0) {
                s.cs[j] = cs2j;
                s.d[j] = dj;
                s.colfac[j] = ex2(cs2_pivot - cs2j) * dj;
            }
            math_bar();
            const float cs2_last = s.cs[q - 1];

            // (2) state entering this tile -> fp16 operand of Yo = C h_prev
            if (t > 0) {
                if (!(ok = wait_bar(s, &s.os_done, (t - 1) & 1, p.status))) break;
                tc_fence_after();
                const float e = ex2(cs2_last_prev);
                uint32_t r0[16], r1[16];
                tmem_ld16(tmem + lane_base + kColSc + 32 * ch, r0);
                tmem_ld16(tmem + lane_base + kColSc + 32 * ch + 16, r1);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    hreg[k] = e * hreg[k] + __uint_as_float(r0[k]);
                    hreg[16 + k] = e * hreg[16 + k] + __uint_as_float(r1[k]);
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint4 v;
                v.x = pack_f16x2(hreg[8 * m + 0], hreg[8 * m + 1]);
                v.y = pack_f16x2(hreg[8 * m + 2], hreg[8 * m + 3]);
                v.z = pack_f16x2(hreg[8 * m + 4], hreg[8 * m + 5]);
                v.w = pack_f16x2(hreg[8 * m + 6], hreg[8 * m + 7]);
                *reinterpret_cast<uint4*>(s.hs + sw128_off(j, 4 * ch + m)) = v;
            }

            // (3) x -> fp16 in place, w o x, rows past the sequence end zeroed
            if (!(ok = wait_bar(s, &s.full[st], (t >> 1) & 1, p.status))) break;
            if (!(ok = wait_bar(s, &s.cb_done, t & 1, p.status))) break;
            uint32_t xr[16];
            {
                const float w = dj * ex2(cs2_last - cs2j);
                uint8_t* xt = s.x[st];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t off = sw128_off(j, 4 * ch + m);
                    uint4 v = *reinterpret_cast<const uint4*>(xt + off);
                    if (j >= q) v = make_uint4(0u, 0u, 0u, 0u);
                    xr[4 * m] = v.x; xr[4 * m + 1] = v.y; xr[4 * m + 2] = v.z; xr[4 * m + 3] = v.w;
                    uint4 xf, wf;
                    xf.x = pack_f16x2(bf16lo(v.x), bf16hi(v.x));
                    xf.y = pack_f16x2(bf16lo(v.y), bf16hi(v.y));
                    xf.z = pack_f16x2(bf16lo(v.z), bf16hi(v.z));
                    xf.w = pack_f16x2(bf16lo(v.w), bf16hi(v.w));
                    wf.x = pack_f16x2(w * bf16lo(v.x), w * bf16hi(v.x));
                    wf.y = pack_f16x2(w * bf16lo(v.y), w * bf16hi(v.y));
                    wf.z = pack_f16x2(w * bf16lo(v.z), w * bf16hi(v.z));
                    wf.w = pack_f16x2(w * bf16lo(v.w), w * bf16hi(v.w));
                    *reinterpret_cast<uint4*>(xt + off) = xf;
                    *reinterpret_cast<uint4*>(s.wx + off) = wf;
                }
                if (j >= q) {
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(s.b[st][ch] + sw128_off(j, c)) = z;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&s.ops_ready);

            // (4) S = CB o decay o d, causal, into TMEM as the A operand of Yd.
            //     This thread covers CB columns [32 bi + 16 ch, + 16) of each 32-block bi.
            tc_fence_after();
            {
                const int bj = j >> 5;
#pragma unroll
                for (int pair = 0; pair < 2; ++pair) {
                    uint32_t r[2][16];
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        if (2 * pair + u <= bj)
                            tmem_ld16(tmem + lane_base + kColCB + 32 * (2 * pair + u) + 16 * ch, r[u]);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int bi = 2 * pair + u;
                        uint32_t sv[8];
                        const int i0 = 32 * bi + 16 * ch;
                        if (bi > bj) {
#pragma unroll
                            for (int k = 0; k < 8; ++k) sv[k] = 0u;
                        } else if (bi < bj) {
                            const float rf = ex2(cs2j - s.cs[32 * bi + 31]);
#pragma unroll
                            for (int k = 0; k < 16; k += 4) {
                                const float4 cf = *reinterpret_cast<const float4*>(&s.colfac[i0 + k]);
                                sv[k / 2] = pack_f16x2(__uint_as_float(r[u][k]) * cf.x * rf,
                                                       __uint_as_float(r[u][k + 1]) * cf.y * rf);
                                sv[k / 2 + 1] = pack_f16x2(__uint_as_float(r[u][k + 2]) * cf.z * rf,
                                                           __uint_as_float(r[u][k + 3]) * cf.w * rf);
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < 16; k += 2) {
                                const int i = i0 + k;
                                const float e0 = ex2(cs2j - s.cs[i]) * s.d[i];
                                const float e1 = ex2(cs2j - s.cs[i + 1]) * s.d[i + 1];
                                sv[k / 2] = pack_f16x2(i <= j ? __uint_as_float(r[u][k]) * e0 : 0.f,
                                                       i + 1 <= j ? __uint_as_float(r[u][k + 1]) * e1 : 0.f);
                            }
                        }
                        tmem_st8(tmem + lane_base + kColS + 16 * bi + 8 * ch, sv);
                    }
                }
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&s.s_ready);

            // (5) epilogue: y = Yd + exp(cs_j) Yo + D x
            if (!(ok = wait_bar(s, &s.yd_done, t & 1, p.status))) break;
            tc_fence_after();
            {
                const float ej = ex2(cs2j);
                __nv_bfloat16* yrow = p.y + tok * H * kP + (int64_t)h * kP + 32 * ch;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t rd[16], ro[16];
                    tmem_ld16(tmem + lane_base + kColYd + 32 * ch + 16 * half, rd);
                    tmem_ld16(tmem + lane_base + kColYo + 32 * ch + 16 * half, ro);
                    tmem_ld_wait();
                    if (half == 1) {
                        tc_fence_before();
                        mbar_arrive(&s.epi_done);
                    }
                    uint32_t out[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t xv = xr[8 * half + k];
                        out[k] = pack_bf16x2(
                            __uint_as_float(rd[2 * k]) + ej * __uint_as_float(ro[2 * k]) + Dh * bf16lo(xv),
                            __uint_as_float(rd[2 * k + 1]) + ej * __uint_as_float(ro[2 * k + 1]) +
                                Dh * bf16hi(xv));
                    }
                    if (j < q) {
                        *reinterpret_cast<uint4*>(yrow + 16 * half) = make_uint4(out[0], out[1], out[2], out[3]);
                        *reinterpret_cast<uint4*>(yrow + 16 * half + 8) = make_uint4(out[4], out[5], out[6], out[7]);
                    }
                }
            }
            cs2_last_prev = cs2_last;
        }
        // final state after the last tile
        if (ok && nt > 0) {
            if (wait_bar(s, &s.os_done, (nt - 1) & 1, p.status)) {
                tc_fence_after();
                const float e = ex2(cs2_last_prev);
                uint32_t r0[16], r1[16];
                tmem_ld16(tmem + lane_base + kColSc + 32 * ch, r0);
                tmem_ld16(tmem + lane_base + kColSc + 32 * ch + 16, r1);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    hreg[k] = e * hreg[k] + __uint_as_float(r0[k]);
                    hreg[16 + k] = e * hreg[16 + k] + __uint_as_float(r1[k]);
                }
            }
        }
        if (p.final_state && !s.abort) {
            float* dst = p.final_state + (((int64_t)seq * H + h) * kN + j) * kP + 32 * ch;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
                *reinterpret_cast<float4*>(dst + c) = make_float4(hreg[c], hreg[c + 1], hreg[c + 2], hreg[c + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// bf16 -> fp16 copies of B and C (8 elements per thread step).
__global__ void k_tc_prep(const uint4* __restrict__ b, const uint4* __restrict__ c, uint4* __restrict__ b16,
                          uint4* __restrict__ c16, int64_t n8) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        uint4 vb = b[i], vc = c[i], ob, oc;
        ob.x = pack_f16x2(bf16lo(vb.x), bf16hi(vb.x));
        ob.y = pack_f16x2(bf16lo(vb.y), bf16hi(vb.y));
        ob.z = pack_f16x2(bf16lo(vb.z), bf16hi(vb.z));
        ob.w = pack_f16x2(bf16lo(vb.w), bf16hi(vb.w));
        oc.x = pack_f16x2(bf16lo(vc.x), bf16hi(vc.x));
        oc.y = pack_f16x2(bf16lo(vc.y), bf16hi(vc.y));
        oc.z = pack_f16x2(bf16lo(vc.z), bf16hi(vc.z));
        oc.w = pack_f16x2(bf16lo(vc.w), bf16hi(vc.w));
        b16[i] = ob;
        c16[i] = oc;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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
bool make_map(CUtensorMap* m, CUtensorMapDataType ty, const void* base, uint64_t inner, uint64_t mid,
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

}  // namespace

bool tc_supported(const ScanArgs& a) {
    return a.dtype == 1 && a.P == kP && a.N == kN && (a.Q == 128 || a.Q == 256) &&
           a.b * a.L < ((int64_t)1 << 31) && a.S * a.H < ((int64_t)1 << 31) && get_encode() != nullptr;
}

size_t tc_workspace_bytes(const ScanArgs& a, int64_t) {
    return 2 * (size_t)a.b * a.L * a.G * a.N * sizeof(__half) + 256;
}

int launch_tc_scan(const ScanArgs& a, const SeqInfo& si, int64_t, void* ws, int32_t* status, cudaStream_t st) {
    const int64_t ntok = a.b * a.L;
    __half* b16 = reinterpret_cast<__half*>(ws);
    __half* c16 = b16 + (size_t)ntok * a.G * a.N;
    {
        const int64_t n8 = ntok * a.G * a.N / 8;
        int64_t blocks = (n8 + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        ProfScope ps(K_TC_PREP, st);
        k_tc_prep<<<(unsigned)blocks, 256, 0, st>>>((const uint4*)a.B, (const uint4*)a.C, (uint4*)b16,
                                                    (uint4*)c16, n8);
    }
    CUtensorMap tm_x, tm_b, tm_c;
    if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)ntok) ||
        !make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, b16, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)ntok) ||
        !make_map(&tm_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c16, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)ntok))
        return 6;  // SSD_ERR_CUDA
    TcParams p;
    p.si = si;
    p.dt = (const __nv_bfloat16*)a.dt;
    p.dt_bias = a.dt_bias;
    p.A = a.A;
    p.D = a.D;
    p.init_state = a.init_state;
    p.final_state = a.final_state;
    p.y = (__nv_bfloat16*)a.y;
    p.status = status;
    p.H = (int)a.H;
    p.G = (int)a.G;
    const size_t smem = sizeof(TcSmem) + 1024;
    cudaFuncSetAttribute(k_tc_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    ProfScope ps(K_TC_SCAN, st);
    k_tc_scan<<<(unsigned)(a.S * a.H), kThreads, smem, st>>>(tm_x, tm_b, tm_c, p);
    return 0;
}

}  // namespace ssd
