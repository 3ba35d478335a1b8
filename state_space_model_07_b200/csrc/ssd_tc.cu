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
//     bf16 values.  The skip term D x rides on the diagonal of S, and the state
//     is accumulated in TMEM by the MMA itself: the math warps scale it by the
//     tile's total decay, then B^T (w o x) is added on the tensor core.
//
// Warp roles (576 threads), pipelined through mbarriers.  A warp can reach
// only its quarter of the 128 TMEM lanes, so each role has two warps per lane
// quarter (thread j of a quarter owns token / state row j = TMEM lane j):
//   P  (warps 0-7):   decay scan and the causal mask S of tile t; the two warps
//                     of a quarter split its 32-column blocks by parity, which
//                     evens out the triangular work.
//   E  (warps 8-15):  state hand-over and fp16 x, (w o x), h for tile t + 1,
//                     then the output epilogue of tile t (Yd, Yo are double-
//                     buffered); the two warps of a quarter split the columns.
//   W16 (lane 0):     TMA loads (two-stage ring) and the C B^T MMAs.
//   W17 (lane 0):     the C h_prev, B^T (w o x) and S x MMAs.
// Every mbarrier's next phase depends on an action its waiters take after
// waiting, so no waiter can see a barrier two phases ahead.  All waits are
// bounded: on a timeout the kernel records SSD_ERR_TIMEOUT in the status word
// and returns after freeing its TMEM.
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
constexpr int kRoleThreads = 256;   // P and E: two warps per TMEM lane quarter
constexpr int kThreads = 576;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: C B^T, S (fp16 pairs), Yd[2], Yo[2], running state H
constexpr uint32_t kColCB = 0, kColS = 128, kColYd = 192, kColYo = 320, kColH = 448;

constexpr uint32_t kTileBytesX = kT * kP * 2;        // 16 KB
constexpr uint32_t kHalfBytes = kT * 64 * 2;         // one 64-column half of a B or C tile: 16 KB
constexpr uint32_t kStageBytes = kTileBytesX + 4 * kHalfBytes;

struct __align__(1024) TcSmem {
    uint8_t x[2][kTileBytesX];        // x tile per stage (bf16 from TMA, fp16 after conversion)
    uint8_t b[2][2][kHalfBytes];      // B tile (fp16) per stage: n in [0,64) and [64,128)
    uint8_t c[2][2][kHalfBytes];      // C tile (fp16)
    uint8_t wx[2][kTileBytesX];       // (w o x) fp16, token rows, by tile parity
    uint8_t hs[kN * kP * 2];          // h_prev fp16, state rows
    float cs[2][kT];       // tile-local cumulative decay (base-2 exponent), by tile parity
    float d[2][kT];
    float colfac[2][kT];   // 2^(cs_m - cs_i) d_i with pivot m = last token of i's 16-block
    float wtot[2][4];
    uint64_t full[2];         // TMA -> E, W8            (per stage)
    uint64_t scan_done[2];    // P -> E                  (per tile parity)
    uint64_t e_done[2];       // E -> P                  (per tile parity)
    uint64_t yd_par[2];       // W9 commit -> E, P, W8   (per tile parity)
    uint64_t cb_done;         // W8 commit -> P
    uint64_t s_ready;         // P -> W8, W9
    uint64_t x_ready;         // E -> W9
    uint64_t sc_done;         // W9 commit -> E
    uint32_t tmem_base;
    int abort;
    int p_flag, e_flag;    // leader-wait results handed to the rest of a role
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

__device__ __forceinline__ void p_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ __half2 u2h(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t h2u(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

__device__ __forceinline__ void set_abort(TcSmem& s, int32_t* status) {
    s.abort = 1;
    if (status) atomicExch(status, kStatusTimeout);
}

// Bounded wait of a single issuing thread; false once the CTA has given up.
__device__ __forceinline__ bool wait_bar(TcSmem& s, uint64_t* bar, uint32_t parity, int32_t* status) {
    if (*(volatile int*)&s.abort) return false;
    if (!mbar_wait(bar, parity)) {
        set_abort(s, status);
        return false;
    }
    return true;
}

// Bounded wait of a whole warp; the result is the same in every lane, so the
// warp-collective TMEM instructions that follow stay uniform even on the
// error path.
__device__ __forceinline__ bool wait_bar_w(TcSmem& s, uint64_t* bar, uint32_t parity, int32_t* status) {
    return __all_sync(0xffffffffu, wait_bar(s, bar, parity, status));
}

// Bounded wait of a whole 8-warp role: only the role's first warp polls the
// mbarrier; the other seven sleep in a hardware named barrier, so waiting
// warps take no issue slots from the warps doing work.  `flag` carries the
// leader's result (false once the CTA has given up) to the others.
template <int kBarId>
__device__ __forceinline__ bool wait_role(TcSmem& s, uint64_t* bar, uint32_t parity, int32_t* status,
                                          bool leader, int* flag) {
    if (leader) {
        const bool ok = wait_bar_w(s, bar, parity, status);
        if ((threadIdx.x & 31) == 0) *(volatile int*)flag = ok ? 1 : 0;
    }
    asm volatile("bar.sync %0, 256;" ::"n"(kBarId) : "memory");
    return *(volatile int*)flag != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
k_tc_scan(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
          const __grid_constant__ CUtensorMap tm_c, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Align to 1024 bytes (128-byte swizzle atoms) by pointer arithmetic on the
    // shared array, so that the compiler keeps every access in the shared state
    // space (a round trip through an integer would turn them into generic ones).
    TcSmem& s = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
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
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.scan_done[i], kRoleThreads);
            mbar_init(&s.e_done[i], kRoleThreads);
            mbar_init(&s.yd_par[i], 1);
        }
        mbar_init(&s.cb_done, 1);
        mbar_init(&s.s_ready, kRoleThreads);
        mbar_init(&s.x_ready, kRoleThreads);
        mbar_init(&s.sc_done, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&s.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    const float kLog2e = 1.4426950408889634f;

    if (warp == 16) {
        // ------------------------------------------------ W16: TMA + C B^T
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
            issue_loads(0);
            if (nt > 1) issue_loads(1);
            bool ok = true;
            for (int t = 0; t < nt; ++t) {
                const int st = t & 1;
                if (!(ok = wait_bar(s, &s.full[st], (t >> 1) & 1, p.status))) break;
                // P has finished reading C B^T of the previous tile
                if (t > 0 && !(ok = wait_bar(s, &s.s_ready, (t - 1) & 1, p.status))) break;
                tc_fence_after();
                const uint32_t cb = smem_u32(s.c[st][0]), bb = smem_u32(s.b[st][0]);
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                    mma_ss(tmem + kColCB, sdesc_sw128(cb + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024),
                           id_cb, k > 0);
                }
                mma_commit(&s.cb_done);
                // stage (t + 1) & 1 is free once every MMA of tile t - 1 has completed
                if (t >= 1 && t + 1 < nt) {
                    if (!(ok = wait_bar(s, &s.yd_par[(t - 1) & 1], ((t - 1) >> 1) & 1, p.status))) break;
                    issue_loads(t + 1);
                }
            }
            if (!ok)
                for (int t = 0; t < loads_issued; ++t) mbar_wait(&s.full[t & 1], (t >> 1) & 1, 400000000ll);
        }
    } else if (warp == 17) {
        // ----------------------------------- W17: C h_prev, B^T (w o x), S x
        if (lane == 0) {
            const uint32_t id_pn = idesc_f16(128, 64, 0, 1);   // K-major A, MN-major B
            const uint32_t id_mn = idesc_f16(128, 64, 1, 1);   // MN-major A and B
            for (int t = 0; t < nt; ++t) {
                const int st = t & 1;
                if (!wait_bar(s, &s.x_ready, t & 1, p.status)) break;
                tc_fence_after();
                const uint32_t cb = smem_u32(s.c[st][0]), bb = smem_u32(s.b[st][0]);
                const uint32_t hsb = smem_u32(s.hs), wxb = smem_u32(s.wx[st]), xb = smem_u32(s.x[st]);
                // Yo = C h_prev
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                    mma_ss(tmem + kColYo + 64 * st, sdesc_sw128(cb + off, 16, 1024),
                           sdesc_sw128(hsb + k * 2048, kHalfBytes, 1024), id_pn, k > 0);
                }
                // H += B^T (w o x): needs the B rows past the sequence end zeroed by P
                if (!wait_bar(s, &s.s_ready, t & 1, p.status)) break;
                tc_fence_after();
                for (int k = 0; k < kT / 16; ++k)
                    mma_ss(tmem + kColH, sdesc_sw128(bb + k * 2048, kHalfBytes, 1024),
                           sdesc_sw128(wxb + k * 2048, kHalfBytes, 1024), id_mn, 1);
                mma_commit(&s.sc_done);
                // Yd = S x  (S carries D on its diagonal)
                for (int k = 0; k < kT / 16; ++k)
                    mma_ts(tmem + kColYd + 64 * st, tmem + kColS + k * 8,
                           sdesc_sw128(xb + k * 2048, kHalfBytes, 1024), id_pn, k > 0);
                mma_commit(&s.yd_par[st]);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------ P: decay scan and mask
        const int quarter = warp & 3, half = warp >> 2;
        const int j = 32 * quarter + lane;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float A2 = p.A[h] * kLog2e;     // decays kept as base-2 exponents
        const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
        const float Dh = p.D ? p.D[h] : 0.f;
        // S columns above this quarter's rows are zero for every tile: write them once.
        // (TMEM loads and stores are warp-collective: every choice below is uniform per warp.)
        {
            const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
            for (int pr = 0; pr < 4; ++pr)
                if (pr > quarter && (pr & 1) == half) {
                    tmem_st8(tmem + lane_base + kColS + 16 * pr, z);
                    tmem_st8(tmem + lane_base + kColS + 16 * pr + 8, z);
                }
            tmem_st_wait();
        }
        float dt_next = 0.f;
        if (nt > 0 && j < len) dt_next = __bfloat162float(p.dt[(tok0 + j) * H + h]);
        for (int t = 0; t < nt; ++t) {
            const int buf = t & 1;
            const int q = (int)(len - (int64_t)t * kT < kT ? len - (int64_t)t * kT : kT);
            // E is done with tile t - 2, whose decay arrays share this parity
            if (t >= 2 && !wait_role<1>(s, &s.e_done[buf], ((t - 2) >> 1) & 1, p.status, warp == 0, &s.p_flag)) break;
            // both warps of a quarter compute the scan; the first one publishes it
            float dj = 0.f, a = 0.f;
            if (j < q) {
                dj = softplus_f(dt_next + bias);
                a = dj * A2;
            }
            if (t + 1 < nt && (int64_t)(t + 1) * kT + j < len)
                dt_next = __bfloat162float(p.dt[(tok0 + (int64_t)(t + 1) * kT + j) * H + h]);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, a, o);
                if (lane >= o) a += u;
            }
            if (lane == 31) s.wtot[half][quarter] = a;
            p_bar();
            for (int w = 0; w < quarter; ++w) a += s.wtot[half][w];
            const float cs2j = a;
            // rank-1 split 2^(cs_j - cs_i) = 2^(cs_j - cs_m) 2^(cs_m - cs_i), pivot m = last
            // token of i's 16-token block (lane 15 or 31 of this warp)
            const float cs2_pivot = __shfl_sync(0xffffffffu, cs2j, lane | 15);
            if (half == 0) {
                s.cs[buf][j] = cs2j;
                s.d[buf][j] = dj;
                s.colfac[buf][j] = ex2(cs2_pivot - cs2j) * dj;
            }
            mbar_arrive(&s.scan_done[buf]);
            p_bar();
            if (!wait_role<1>(s, &s.cb_done, t & 1, p.status, warp == 0, &s.p_flag)) break;
            if (j >= q) {
                // C B^T has read this tile's B: zero the rows past the sequence end
                // so that B^T (w o x) sees exact zeros there (even for non-finite data)
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(s.b[buf][half] + sw128_off(j, c)) = z;
                fence_proxy_async_smem();
            }
            // S of the previous tile has been consumed by its S x
            if (t > 0 && !wait_role<1>(s, &s.yd_par[(t - 1) & 1], ((t - 1) >> 1) & 1, p.status, warp == 0, &s.p_flag)) break;
            tc_fence_after();
            // S = C B^T o 2^(cs_j - cs_i) d_i for i <= j, plus D on the diagonal.  This warp
            // handles the 32-column blocks pr <= quarter of its parity.  Blocks strictly
            // below the diagonal use the rank-1 split; the block holding the diagonal uses
            // the full exponential in every lane (exact there too), so no lane diverges.
#pragma unroll 1
            for (int b = 2 * half; b <= 2 * quarter + 1; b += (b & 1) ? 3 : 1) {
                // 16-column block b (pairs pr = b / 2 of this warp's parity)
                const int pr = b >> 1;
                const int i0 = 16 * b;
                uint32_t r[16];
                tmem_ld16(tmem + lane_base + kColCB + i0, r);
                float f[16];
                if (pr < quarter) {
                    const float rf = ex2(cs2j - s.cs[buf][i0 + 15]);
#pragma unroll
                    for (int k = 0; k < 16; k += 4) {
                        const float4 cf = *reinterpret_cast<const float4*>(&s.colfac[buf][i0 + k]);
                        f[k] = cf.x * rf; f[k + 1] = cf.y * rf; f[k + 2] = cf.z * rf; f[k + 3] = cf.w * rf;
                    }
                } else {
                    float c[16], dd[16];
#pragma unroll
                    for (int k = 0; k < 16; k += 4) {
                        const float4 cv = *reinterpret_cast<const float4*>(&s.cs[buf][i0 + k]);
                        const float4 dv = *reinterpret_cast<const float4*>(&s.d[buf][i0 + k]);
                        c[k] = cv.x; c[k + 1] = cv.y; c[k + 2] = cv.z; c[k + 3] = cv.w;
                        dd[k] = dv.x; dd[k + 1] = dv.y; dd[k + 2] = dv.z; dd[k + 3] = dv.w;
                    }
#pragma unroll
                    for (int k = 0; k < 16; ++k) f[k] = i0 + k <= j ? ex2(cs2j - c[k]) * dd[k] : 0.f;
                }
                tmem_ld_wait();
                uint32_t sv[8];
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    float v0 = __uint_as_float(r[k]) * f[k];
                    float v1 = __uint_as_float(r[k + 1]) * f[k + 1];
                    if (i0 + k == j) v0 += Dh;
                    if (i0 + k + 1 == j) v1 += Dh;
                    sv[k / 2] = pack_f16x2(v0, v1);
                }
                tmem_st8(tmem + lane_base + kColS + 8 * b, sv);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&s.s_ready);
        }
    } else if (warp < 16) {
        // ---------------------- E: state hand-over, fp16 operands, epilogue
        const int quarter = warp & 3, half = (warp >> 2) & 1;
        const int j = 32 * quarter + lane;
        const int col0 = 32 * half;           // this warp's 32 of the 64 state / x / y columns
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float* init_row = p.init_state ? p.init_state + (((int64_t)seq * H + h) * kN + j) * kP : nullptr;
        // Tile u's operands: fp16 copy of the state entering it (hs), the state in
        // TMEM pre-scaled by the tile's total decay (B^T (w o x) is then added by
        // the MMA), x in fp16 and (w o x).
        auto prepare = [&](int u, bool first) -> bool {
            const int st = u & 1;
            const int qu = (int)(len - (int64_t)u * kT < kT ? len - (int64_t)u * kT : kT);
            if (!wait_role<2>(s, &s.scan_done[st], (u >> 1) & 1, p.status, warp == 8, &s.e_flag)) return false;
            const float cs2j = s.cs[st][j], dj = s.d[st][j], cs2_last = s.cs[st][qu - 1];
            const float e = ex2(cs2_last);
            uint32_t hv[2][16];
            if (first) {
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int k = 0; k < 16; k += 4) {
                        const float4 v = init_row ? *reinterpret_cast<const float4*>(init_row + col0 + 16 * m + k)
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                        hv[m][k] = __float_as_uint(v.x); hv[m][k + 1] = __float_as_uint(v.y);
                        hv[m][k + 2] = __float_as_uint(v.z); hv[m][k + 3] = __float_as_uint(v.w);
                    }
            } else {
                tmem_ld16(tmem + lane_base + kColH + col0, hv[0]);
                tmem_ld16(tmem + lane_base + kColH + col0 + 16, hv[1]);
                tmem_ld_wait();
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                uint4 v0, v1;
                v0.x = pack_f16x2(__uint_as_float(hv[m][0]), __uint_as_float(hv[m][1]));
                v0.y = pack_f16x2(__uint_as_float(hv[m][2]), __uint_as_float(hv[m][3]));
                v0.z = pack_f16x2(__uint_as_float(hv[m][4]), __uint_as_float(hv[m][5]));
                v0.w = pack_f16x2(__uint_as_float(hv[m][6]), __uint_as_float(hv[m][7]));
                v1.x = pack_f16x2(__uint_as_float(hv[m][8]), __uint_as_float(hv[m][9]));
                v1.y = pack_f16x2(__uint_as_float(hv[m][10]), __uint_as_float(hv[m][11]));
                v1.z = pack_f16x2(__uint_as_float(hv[m][12]), __uint_as_float(hv[m][13]));
                v1.w = pack_f16x2(__uint_as_float(hv[m][14]), __uint_as_float(hv[m][15]));
                const int c = col0 + 16 * m;
                *reinterpret_cast<uint4*>(s.hs + sw128_off(j, c / 8)) = v0;
                *reinterpret_cast<uint4*>(s.hs + sw128_off(j, c / 8 + 1)) = v1;
#pragma unroll
                for (int k = 0; k < 16; ++k) hv[m][k] = __float_as_uint(e * __uint_as_float(hv[m][k]));
                tmem_st16(tmem + lane_base + kColH + c, hv[m]);
            }
            tmem_st_wait();
            if (!wait_role<2>(s, &s.full[st], (u >> 1) & 1, p.status, warp == 8, &s.e_flag)) return false;
            const __half2 w2 = __float2half2_rn(dj * ex2(cs2_last - cs2j));
            uint8_t* xt = s.x[st];
            uint4 v[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                v[m] = *reinterpret_cast<const uint4*>(xt + sw128_off(j, col0 / 8 + m));
                if (j >= qu) v[m] = make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint4 xf, wf;
                xf.x = pack_f16x2(bf16lo(v[m].x), bf16hi(v[m].x));
                xf.y = pack_f16x2(bf16lo(v[m].y), bf16hi(v[m].y));
                xf.z = pack_f16x2(bf16lo(v[m].z), bf16hi(v[m].z));
                xf.w = pack_f16x2(bf16lo(v[m].w), bf16hi(v[m].w));
                wf.x = h2u(__hmul2(u2h(xf.x), w2));
                wf.y = h2u(__hmul2(u2h(xf.y), w2));
                wf.z = h2u(__hmul2(u2h(xf.z), w2));
                wf.w = h2u(__hmul2(u2h(xf.w), w2));
                const uint32_t off = sw128_off(j, col0 / 8 + m);
                *reinterpret_cast<uint4*>(xt + off) = xf;
                *reinterpret_cast<uint4*>(s.wx[st] + off) = wf;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&s.x_ready);
            return true;
        };
        // Step k prepares tile k (once the state entering it is complete) and then
        // writes the output of tile k - 1.
        bool ok = true;
        for (int k = 0; ok && k <= nt; ++k) {
            if (k < nt) {
                // the state entering tile k is complete once B^T (w o x) of tile k - 1 has been added
                if (k > 0) {
                    if (!(ok = wait_role<2>(s, &s.sc_done, (k - 1) & 1, p.status, warp == 8, &s.e_flag))) break;
                    tc_fence_after();
                }
                if (!(ok = prepare(k, k == 0))) break;
            }
            if (k == 0) continue;
            const int t = k - 1, st = t & 1;
            const int q = (int)(len - (int64_t)t * kT < kT ? len - (int64_t)t * kT : kT);
            // epilogue of tile t: y = Yd + 2^cs_j Yo   (D x is inside Yd)
            if (!(ok = wait_role<2>(s, &s.yd_par[st], (t >> 1) & 1, p.status, warp == 8, &s.e_flag))) break;
            tc_fence_after();
            {
                const float ej = ex2(s.cs[st][j]);
                __nv_bfloat16* yrow = p.y + (tok0 + (int64_t)t * kT + j) * H * kP + (int64_t)h * kP;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int c = col0 + 16 * m;
                    uint32_t rd[16], ro[16];
                    tmem_ld16(tmem + lane_base + kColYd + 64 * st + c, rd);
                    tmem_ld16(tmem + lane_base + kColYo + 64 * st + c, ro);
                    tmem_ld_wait();
                    uint32_t out[8];
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2)
                        out[k2] = pack_bf16x2(__uint_as_float(rd[2 * k2]) + ej * __uint_as_float(ro[2 * k2]),
                                              __uint_as_float(rd[2 * k2 + 1]) + ej * __uint_as_float(ro[2 * k2 + 1]));
                    if (j < q) {
                        *reinterpret_cast<uint4*>(yrow + c) = make_uint4(out[0], out[1], out[2], out[3]);
                        *reinterpret_cast<uint4*>(yrow + c + 8) = make_uint4(out[4], out[5], out[6], out[7]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&s.e_done[st]);
        }
        // final state: H after the last tile's B^T (w o x) (or init_state for an empty sequence)
        if (p.final_state) {
            float* dst = p.final_state + (((int64_t)seq * H + h) * kN + j) * kP;
            if (nt == 0) {
#pragma unroll
                for (int c = col0; c < col0 + 32; c += 4)
                    *reinterpret_cast<float4*>(dst + c) =
                        init_row ? *reinterpret_cast<const float4*>(init_row + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            } else if (ok) {
                tc_fence_after();
#pragma unroll
                for (int c = col0; c < col0 + 32; c += 16) {
                    uint32_t hv[16];
                    tmem_ld16(tmem + lane_base + kColH + c, hv);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 16; k += 4)
                        *reinterpret_cast<float4*>(dst + c + k) =
                            make_float4(__uint_as_float(hv[k]), __uint_as_float(hv[k + 1]),
                                        __uint_as_float(hv[k + 2]), __uint_as_float(hv[k + 3]));
                }
            }
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
