// ssd_tc.cu -- tensor-core (tcgen05) path of the chunked scan, bf16 inputs.
//
// Block decomposition of "5.3 Tensor Parallelism support and large-cluster
// training", section 3.2, mapped onto one B200 SM per (sequence, head):
//
//   * The sequence is walked in 128-token tiles (one TMEM lane per token).  A
//     chunk of 256 tokens is two tiles joined by the same N x P state hand-over
//     as two chunks are, so the result equals the chunked form up to rounding.
//   * Per tile, with d = softplus(dt + dt_bias), cs = tile-local inclusive
//     cumulative sum of d*A, w_i = d_i exp(cs_last - cs_i):
//       CB   = C B^T                               tcgen05, fp16 x fp16 -> fp32 TMEM
//       S    = CB o exp(cs_j - cs_i) d_i (i <= j)  math warps, written back to TMEM
//       y    = S x + exp(cs_j) C h_prev + D x      tcgen05 (+ math warps)
//       h    = exp(cs_last) h_prev + B^T (w o x)   tcgen05 for the B^T (w o x) term
//   * The operands the math warps produce (S, h_prev, w o x) are rounded to fp16
//     (11-bit significand): bf16's 8 bits miss the 1e-2 (1 + |y|) accuracy bound.
//     B and C are converted to fp16 once by k_tc_prep; x is converted in place in
//     shared memory.  C B^T on those fp16 copies is exact for normal-range
//     bf16 values.  The skip term D x rides on the diagonal of S.
//
// Two kernels:
//   * k_tc_scan3 (N = 128, below in namespace v3): the state recurrence runs on
//     CUDA cores in fp32 registers, off the tensor core's critical path; C is
//     copied to TMEM and scaled there by exp(cs_j), so the output is one
//     accumulator; y leaves by TMA tensor stores.  Its own header comment has
//     the roles and the hand-off rules.
//   * k_tc_scan<N> (N = 256): the first design, in which the MMA accumulates
//     the state in TMEM (the math warps scale it by the tile's total decay,
//     then B^T (w o x) is added on the tensor core) and the epilogue combines
//     two accumulators.  Warp roles (608 threads): P (warps 0-7) decay scan and
//     the causal mask; E (warps 8-15) state hand-over, fp16 operands and the
//     epilogue; W16 TMA loads and C B^T; W17 C h_prev, then S x; W18
//     B^T (w o x).  A single thread issues tcgen05.mma chains at roughly one
//     instruction per 100-200 cycles whatever N is, so the three 16-instruction
//     chains of a tile come from separate warps, and each starts on the first
//     64-column box of B / C while the rest is still loading.
//
// A warp can reach only its quarter of the 128 TMEM lanes, so each math role
// has two warps per lane quarter (thread j of a quarter owns token / state row
// j = TMEM lane j).  Every mbarrier's next phase depends on an action its
// waiters take after waiting, so no waiter can see a barrier two phases ahead.
// All waits are bounded: on a timeout the kernel records SSD_ERR_TIMEOUT in the
// status word and returns after freeing its TMEM.
#include <cuda.h>
#include <algorithm>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <stdio.h>
#include <stdlib.h>

#include "ssd_common.cuh"
#include "ssd_prof.h"
#include "ssd_tc.h"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kRoleThreads = 256;   // P and E: two warps per TMEM lane quarter
constexpr uint32_t kTmemCols = 512;

// Layout constants for dstate N (the kernel is instantiated for N = 256 only):
// B and C tiles (64 KB each) single-buffered, reloaded once the tile's C B^T,
// C h_prev and B^T (w o x) MMAs are done; Yd single-buffered (its MMA waits for
// the previous epilogue), Yo double-buffered; the state takes two 128-lane TMEM
// blocks.
template <int N>
struct Cfg {
    static constexpr int kThreads = 608;                    // P 0-7, E 8-15, W16, W17, W18
    static constexpr int kBoxes = N / 64;                   // 64-column boxes per B / C tile
    static constexpr int kBCStages = N == 128 ? 2 : 1;
    static constexpr int kYdBufs = N == 128 ? 2 : 1;
    static constexpr int kHBlocks = N / 128;                // 128-row blocks of the state
    // TMEM columns: C B^T | S (fp16 pairs) | Yd[kYdBufs] | Yo[2] | H[kHBlocks]
    static constexpr uint32_t kColCB = 0, kColS = 128, kColYd = 192;
    static constexpr uint32_t kColYo = kColYd + 64 * kYdBufs;
    static constexpr uint32_t kColH = kColYo + 128;
    static_assert(kColH + 64 * kHBlocks <= kTmemCols, "TMEM columns");
};


template <int N>
struct __align__(1024) TcSmem {
    uint8_t x[2][kTileBytesX];                         // x per stage (bf16 from TMA, fp16 after conversion)
    uint8_t b[Cfg<N>::kBCStages][Cfg<N>::kBoxes][kBoxBytes];  // B (fp16), 64-column boxes
    uint8_t c[Cfg<N>::kBCStages][Cfg<N>::kBoxes][kBoxBytes];  // C (fp16)
    uint8_t wx[kTileBytesX];                           // (w o x) fp16, token rows
    uint8_t hs[N * kP * 2];                            // h_prev fp16, state rows
    float cs[2][kT];       // tile-local cumulative decay (base-2 exponent), by tile parity
    float d[2][kT];
    float colfac[2][kT];   // 2^(cs_m - cs_i) d_i with pivot m = last token of i's 16-block
    float wtot[2][4];
    // Every barrier's next phase depends on an action its waiters take after
    // waiting, so no waiter can ever see a barrier two phases ahead.
    uint64_t xfull[2];        // TMA x -> E                    (per x stage)
    uint64_t bcfull[4];       // TMA B, C box k -> W16, W17, W18  (per 64-column box)
    uint64_t scan_done[2];    // P -> E                        (per tile parity)
    uint64_t e_done[2];       // E -> P, W17                   (per tile parity)
    uint64_t x_ready[2];      // E -> W17, W18                 (per tile parity)
    uint64_t yd_par[2];       // W17 commit (S x) -> E, P, W16 (per tile parity)
    uint64_t cb_done;         // W16 commit -> P, W16
    uint64_t s_ready;         // P -> W16, W17
    uint64_t sc_done;         // W17 (C h_prev) and W18 (B^T (w o x)) commits -> E, W16
    uint64_t b_zeroed;        // P -> W18, once: B rows past the sequence end zeroed
    uint64_t fin[3];          // W16, W17, W18: own tcgen05 work drained before exit
    uint32_t tmem_base;
    TcCtl ctl;
};

// Rows split into segments (k_tc_scan3 only).  Span index s >= first is segment
// (s - first) % K of batch row row0 + (s - first) / K: tokens [k Ls, (k + 1) Ls) of the
// row, the last segment running to the row's end.  Segment 0 starts from the row's
// initial state and the others from zero; every segment's final state goes to fin
// and the running base-2 log-decay from the segment start through each of its tokens
// to cs (128 `tiles` floats per (segment, head)).  first = INT32_MAX: no split.
struct SplitSpec {
    int32_t first = 0x7fffffff, K = 0, row0 = 0, tiles = 0;
    int64_t Ls = 0;
    float* fin = nullptr;
    float* cs = nullptr;
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
    SplitSpec split;
};

__device__ __forceinline__ void p_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }


template <int N>
__global__ void __launch_bounds__(Cfg<N>::kThreads, 1)
k_tc_scan(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
          const __grid_constant__ CUtensorMap tm_c, const TcParams p) {
    using C = Cfg<N>;
    static_assert(C::kBCStages == 1 && C::kYdBufs == 1, "the hand-off below is written for N = 256");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Align to 1024 bytes (128-byte swizzle atoms) by pointer arithmetic on the
    // shared array, so that the compiler keeps every access in the shared state
    // space (a round trip through an integer would turn them into generic ones).
    TcSmem<N>& s = *reinterpret_cast<TcSmem<N>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    TcCtl& ctl = s.ctl;
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
            mbar_init(&s.xfull[i], 1);
            mbar_init(&s.scan_done[i], kRoleThreads);
            mbar_init(&s.e_done[i], kRoleThreads);
            mbar_init(&s.x_ready[i], kRoleThreads);
            mbar_init(&s.yd_par[i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&s.bcfull[i], 1);
        for (int i = 0; i < 3; ++i) mbar_init(&s.fin[i], 1);
        mbar_init(&s.cb_done, 1);
        mbar_init(&s.s_ready, kRoleThreads);
        mbar_init(&s.sc_done, 2);
        mbar_init(&s.b_zeroed, kRoleThreads);
        ctl.abort = 0;
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
            int x_issued = 0, bc_issued = 0;
            auto load_x = [&](int t) {
                const int st = t & 1;
                mbar_expect_tx(&s.xfull[st], kTileBytesX);
                tma_load_3d(s.x[st], &tm_x, &s.xfull[st], 0, h, (int)(tok0 + (int64_t)t * kT));
                ++x_issued;
            };
            // B and C land box by box, so that the MMAs of a tile start on the first 64 state
            // columns while the rest is still in flight
            auto load_bc = [&](int t) {
                const int tok = (int)(tok0 + (int64_t)t * kT);
                for (int k = 0; k < C::kBoxes; ++k) {
                    mbar_expect_tx(&s.bcfull[k], 2 * kBoxBytes);
                    tma_load_3d(s.b[0][k], &tm_b, &s.bcfull[k], 64 * k, g, tok);
                    tma_load_3d(s.c[0][k], &tm_c, &s.bcfull[k], 64 * k, g, tok);
                }
                ++bc_issued;
            };
            // x, B and C of a tile are pulled into L2 three tiles ahead of use, so that the loads on
            // the critical path (the single B / C stage is refilled only once a tile's MMAs are done)
            // read L2 rather than HBM
            auto prefetch = [&](int t) {
                const int tok = (int)(tok0 + (int64_t)t * kT);
                tma_prefetch_l2_3d(&tm_x, 0, h, tok);
                for (int k = 0; k < C::kBoxes; ++k) {
                    tma_prefetch_l2_3d(&tm_b, 64 * k, g, tok);
                    tma_prefetch_l2_3d(&tm_c, 64 * k, g, tok);
                }
            };
            const uint32_t id_cb = idesc_f16(128, 128, 0, 0);
            load_x(0);
            load_bc(0);
            if (nt > 1) load_x(1);
            if (nt > 2) prefetch(2);
            bool ok = true;
            for (int t = 0; t < nt; ++t) {
                if (t + 3 < nt) prefetch(t + 3);
                // P has finished reading C B^T of the previous tile
                if (t > 0 && !(ok = wait_bar(ctl, &s.s_ready, (t - 1) & 1, p.status))) break;
                const uint32_t cb = smem_u32(s.c[0][0]), bb = smem_u32(s.b[0][0]);
                for (int k = 0; k < N / 16; ++k) {
                    if ((k & 3) == 0) {
                        if (!(ok = wait_bar(ctl, &s.bcfull[k >> 2], (uint32_t)(t & 1), p.status))) break;
                        tc_fence_after();
                    }
                    const uint32_t off = (k >> 2) * kBoxBytes + (k & 3) * 32;
                    mma_ss(tmem + C::kColCB, sdesc_sw128(cb + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024),
                           id_cb, k > 0);
                }
                if (!ok) break;
                mma_commit(&s.cb_done);
                if (t >= 1 && t + 1 < nt) {
                    // x stage (t + 1) & 1 is free once S x of tile t - 1 has completed
                    if (!(ok = wait_bar(ctl, &s.yd_par[(t - 1) & 1], ((t - 1) >> 1) & 1, p.status))) break;
                    load_x(t + 1);
                }
                if (t + 1 < nt) {
                    // the single B/C stage is free once C B^T, C h_prev and B^T (w o x) of
                    // tile t are done
                    if (!(ok = wait_bar(ctl, &s.cb_done, t & 1, p.status))) break;
                    if (!(ok = wait_bar(ctl, &s.sc_done, t & 1, p.status))) break;
                    load_bc(t + 1);
                }
            }
            if (!ok) {
                // Give up: let the copies already in flight land before the CTA exits.
                for (int t = 0; t < x_issued; ++t) mbar_wait(&s.xfull[t & 1], (t >> 1) & 1, 400000000ll);
                for (int t = 0; t < bc_issued; ++t)
                    for (int k = 0; k < C::kBoxes; ++k) mbar_wait(&s.bcfull[k], t & 1, 400000000ll);
            }
            // every C B^T issued has completed before TMEM is freed (on a timeout nobody else
            // waits for the last ones)
            mma_commit(&s.fin[0]);
            mbar_wait(&s.fin[0], 0, 400000000ll);
        }
    } else if (warp == 17) {
        // -------------------------------------------------------- W17: C h_prev, S x
        if (lane == 0) {
            const uint32_t id_pn = idesc_f16(128, 64, 0, 1);   // K-major A, MN-major B
            bool ok = true;
            for (int t = 0; ok && t < nt; ++t) {
                const int st = t & 1;
                // E has written h_prev (fp16) and read out Yo[st] two tiles back
                if (!(ok = wait_bar(ctl, &s.x_ready[st], (uint32_t)((t >> 1) & 1), p.status))) break;
                const uint32_t cb = smem_u32(s.c[0][0]), hsb = smem_u32(s.hs);
                // Yo = C h_prev, box by box as C lands
                for (int k = 0; k < N / 16; ++k) {
                    if ((k & 3) == 0) {
                        if (!(ok = wait_bar(ctl, &s.bcfull[k >> 2], (uint32_t)(t & 1), p.status))) break;
                        tc_fence_after();
                    }
                    const uint32_t off = (k >> 2) * kBoxBytes + (k & 3) * 32;
                    mma_ss(tmem + C::kColYo + 64 * st, sdesc_sw128(cb + off, 16, 1024),
                           sdesc_sw128(hsb + k * 2048, kBoxBytes, 1024), id_pn, k > 0);
                }
                if (!ok) break;
                mma_commit(&s.sc_done);
                // Yd = S x  (S carries D on its diagonal), issued after C h_prev so that it never
                // delays the state chain: S must be written, and the single Yd buffer read out
                // by the previous epilogue
                if (!(ok = wait_bar(ctl, &s.s_ready, t & 1, p.status))) break;
                if (t > 0 && !(ok = wait_bar(ctl, &s.e_done[(t - 1) & 1], ((t - 1) >> 1) & 1, p.status))) break;
                tc_fence_after();
                const uint32_t xb = smem_u32(s.x[st]);
                for (int k = 0; k < kT / 16; ++k)
                    mma_ts(tmem + C::kColYd, tmem + C::kColS + k * 8, sdesc_sw128(xb + k * 2048, kBoxBytes, 1024),
                           id_pn, k > 0);
                mma_commit(&s.yd_par[st]);
            }
            if (nt > 0) {
                mma_commit(&s.fin[1]);
                mbar_wait(&s.fin[1], 0, 400000000ll);
            }
        }
    } else if (warp == 18) {
        // ------------------------------------------------- W18: H += B^T (w o x)
        if (lane == 0) {
            const uint32_t id_mn = idesc_f16(128, 64, 1, 1);   // MN-major A and B
            const int qlast = (int)(len - (int64_t)(nt - 1) * kT);
            bool ok = true;
            for (int t = 0; ok && t < nt; ++t) {
                // E has scaled the state in TMEM by the tile's total decay and written w o x
                if (!(ok = wait_bar(ctl, &s.x_ready[t & 1], (uint32_t)((t >> 1) & 1), p.status))) break;
                // on a partial last tile, the B rows past the sequence end must read as zeros
                if (t == nt - 1 && qlast < kT && !(ok = wait_bar(ctl, &s.b_zeroed, 0, p.status))) break;
                const uint32_t bb = smem_u32(s.b[0][0]), wxb = smem_u32(s.wx);
                // one 128-row block of the state at a time: rows 128 mb .. 128 mb + 127 are the
                // B columns of boxes 2 mb and 2 mb + 1
                for (int mb = 0; ok && mb < C::kHBlocks; ++mb) {
                    if (!(ok = wait_bar(ctl, &s.bcfull[2 * mb], (uint32_t)(t & 1), p.status))) break;
                    if (!(ok = wait_bar(ctl, &s.bcfull[2 * mb + 1], (uint32_t)(t & 1), p.status))) break;
                    tc_fence_after();
                    for (int k = 0; k < kT / 16; ++k)
                        mma_ss(tmem + C::kColH + 64 * mb,
                               sdesc_sw128(bb + 2 * mb * kBoxBytes + k * 2048, kBoxBytes, 1024),
                               sdesc_sw128(wxb + k * 2048, kBoxBytes, 1024), id_mn, 1);
                }
                if (ok) mma_commit(&s.sc_done);
            }
            if (nt > 0) {
                mma_commit(&s.fin[2]);
                mbar_wait(&s.fin[2], 0, 400000000ll);
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
                    tmem_st8(tmem + lane_base + C::kColS + 16 * pr, z);
                    tmem_st8(tmem + lane_base + C::kColS + 16 * pr + 8, z);
                }
            tmem_st_wait();
        }
        float dt_next = 0.f;
        if (nt > 0 && j < len) dt_next = __bfloat162float(p.dt[(tok0 + j) * H + h]);
        for (int t = 0; t < nt; ++t) {
            const int buf = t & 1;
            const int q = (int)(len - (int64_t)t * kT < kT ? len - (int64_t)t * kT : kT);
            // E is done with tile t - 2, whose decay arrays share this parity
            if (t >= 2 && !wait_bar_w(ctl, &s.e_done[buf], ((t - 2) >> 1) & 1, p.status))
                break;
            // both warps of a quarter compute the scan; the first one publishes it
            float dj = 0.f, a = 0.f;
            if (j < q) {
                dj = softplus_f(dt_next + bias);
                a = dj * A2;
            }
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
            // dt of the next tile: loaded only now, since an arrival (a release) waits for the
            // thread's loads in flight; the next one (s_ready) comes after C B^T of this tile
            if (t + 1 < nt && (int64_t)(t + 1) * kT + j < len)
                dt_next = __bfloat162float(p.dt[(tok0 + (int64_t)(t + 1) * kT + j) * H + h]);
            p_bar();
            if (!wait_bar_w(ctl, &s.cb_done, t & 1, p.status)) break;
            if (q < kT) {
                // (the last tile only) C B^T has read this tile's B: zero the rows past the
                // sequence end so that B^T (w o x) sees exact zeros there (even for non-finite
                // data), then let W18 issue it
                if (j >= q) {
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    for (int bx = half; bx < C::kBoxes; bx += 2)
#pragma unroll
                        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(s.b[0][bx] + sw128_off(j, c)) = z;
                    fence_proxy_async_smem();
                }
                mbar_arrive(&s.b_zeroed);
            }
            // S of the previous tile has been consumed by its S x
            if (t > 0 &&
                !wait_bar_w(ctl, &s.yd_par[(t - 1) & 1], ((t - 1) >> 1) & 1, p.status))
                break;
            tc_fence_after();
            // S = C B^T o 2^(cs_j - cs_i) d_i for i <= j, plus D on the diagonal.  This warp
            // handles the 32-column blocks pr <= quarter of its parity, 16 columns at a time.
            // Blocks strictly below the diagonal use the rank-1 split; the block holding the
            // diagonal uses the full exponential in every lane (exact there too), so no lane
            // diverges.
#pragma unroll 1
            for (int b = 2 * half; b <= 2 * quarter + 1; b += (b & 1) ? 3 : 1) {
                const int pr = b >> 1;
                const int i0 = 16 * b;
                uint32_t r[16];
                tmem_ld16(tmem + lane_base + C::kColCB + i0, r);
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
                    // a select, not a multiply by zero: C B^T above the diagonal may hold B rows
                    // of the next packed sequence (past this one's end), and inf * 0 is NaN
                    float v0 = i0 + k <= j ? __uint_as_float(r[k]) * f[k] : 0.f;
                    float v1 = i0 + k + 1 <= j ? __uint_as_float(r[k + 1]) * f[k + 1] : 0.f;
                    if (i0 + k == j) v0 += Dh;
                    if (i0 + k + 1 == j) v1 += Dh;
                    sv[k / 2] = pack_f16x2(v0, v1);
                }
                tmem_st8(tmem + lane_base + C::kColS + 8 * b, sv);
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
        const float* init_base = p.init_state ? p.init_state + ((int64_t)seq * H + h) * N * kP : nullptr;
        // Tile u's operands: fp16 copy of the state entering it (hs), the state in
        // TMEM pre-scaled by the tile's total decay (B^T (w o x) is then added by
        // the MMA), x in fp16 and (w o x).  State row n = 128 hb + j lives in TMEM
        // block hb.
        auto prepare = [&](int u, bool first) -> bool {
            const int st = u & 1;
            const int qu = (int)(len - (int64_t)u * kT < kT ? len - (int64_t)u * kT : kT);
            if (!wait_bar_w(ctl, &s.scan_done[st], (u >> 1) & 1, p.status)) return false;
            const float cs2j = s.cs[st][j], dj = s.d[st][j], cs2_last = s.cs[st][qu - 1];
            const float e = ex2(cs2_last);
#pragma unroll 1
            for (int hb = 0; hb < C::kHBlocks; ++hb) {
                const int n = 128 * hb + j;
                const uint32_t hcol = tmem + lane_base + C::kColH + 64 * hb + col0;
                uint32_t hv[2][16];
                if (first) {
                    const float* src = init_base ? init_base + (int64_t)n * kP + col0 : nullptr;
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int k = 0; k < 16; k += 4) {
                            const float4 v = src ? *reinterpret_cast<const float4*>(src + 16 * m + k)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                            hv[m][k] = __float_as_uint(v.x); hv[m][k + 1] = __float_as_uint(v.y);
                            hv[m][k + 2] = __float_as_uint(v.z); hv[m][k + 3] = __float_as_uint(v.w);
                        }
                } else {
                    tmem_ld16(hcol, hv[0]);
                    tmem_ld16(hcol + 16, hv[1]);
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
                    *reinterpret_cast<uint4*>(s.hs + sw128_off(n, c / 8)) = v0;
                    *reinterpret_cast<uint4*>(s.hs + sw128_off(n, c / 8 + 1)) = v1;
#pragma unroll
                    for (int k = 0; k < 16; ++k) hv[m][k] = __float_as_uint(e * __uint_as_float(hv[m][k]));
                    tmem_st16(hcol + 16 * m, hv[m]);
                }
            }
            tmem_st_wait();
            if (!wait_bar_w(ctl, &s.xfull[st], (u >> 1) & 1, p.status)) return false;
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
                *reinterpret_cast<uint4*>(s.wx + off) = wf;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&s.x_ready[st]);
            return true;
        };
        // Step k prepares tile k (once the state entering it is complete) and then
        // writes the output of tile k - 1.
        bool ok = true;
        for (int k = 0; ok && k <= nt; ++k) {
            // the state entering tile k is complete once B^T (w o x) of tile k - 1 has been
            // added; that also frees hs and (w o x) for tile k, and C h_prev of tile k - 1
            // (read by its epilogue below) is done
            if (k > 0) {
                if (!(ok = wait_bar_w(ctl, &s.sc_done, (k - 1) & 1, p.status))) break;
                tc_fence_after();
            }
            if (k < nt && !(ok = prepare(k, k == 0))) break;
            if (k == 0) continue;
            const int t = k - 1, st = t & 1;
            const int q = (int)(len - (int64_t)t * kT < kT ? len - (int64_t)t * kT : kT);
            // epilogue of tile t: y = Yd + 2^cs_j Yo   (D x is inside Yd)
            if (!(ok = wait_bar_w(ctl, &s.yd_par[st], (t >> 1) & 1, p.status))) break;
            tc_fence_after();
            {
                const float ej = ex2(s.cs[st][j]);
                __nv_bfloat16* yrow = p.y + (tok0 + (int64_t)t * kT + j) * H * kP + (int64_t)h * kP;
                const uint32_t yd = tmem + lane_base + C::kColYd;
                const uint32_t yo = tmem + lane_base + C::kColYo + 64 * st;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int c = col0 + 16 * m;
                    uint32_t rd[16], ro[16];
                    tmem_ld16(yd + c, rd);
                    tmem_ld16(yo + c, ro);
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
#pragma unroll 1
            for (int hb = 0; hb < C::kHBlocks; ++hb) {
                const int n = 128 * hb + j;
                float* dst = p.final_state + (((int64_t)seq * H + h) * N + n) * kP + col0;
                if (nt == 0) {
                    const float* src = init_base ? init_base + (int64_t)n * kP + col0 : nullptr;
#pragma unroll
                    for (int c = 0; c < 32; c += 4)
                        *reinterpret_cast<float4*>(dst + c) =
                            src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < 32; c += 16) {
                        uint32_t hv[16];
                        tmem_ld16(tmem + lane_base + C::kColH + 64 * hb + col0 + c, hv);
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Decoupled-state kernel (N = 128).
//
// Shared-memory bandwidth (128 B per clock per SM, shared by TMA writes, the
// MMAs' operand reads and the threads) is what bounds this kernel, so the
// design keeps bytes out of shared memory:
//   * C goes to TMEM once (tcgen05.cp); C B^T and C' h_prev take A from TMEM.
//     C' = rows of C scaled by 2^cs_j is made in place in TMEM, so the output
//     of a tile is one accumulator Y = C' h_prev + S x.
//   * x arrives by TMA and is converted in place to fp16; the E warps also
//     write w o x once.
//   * The state recurrence runs on the E warps in fp32 registers,
//     h <- 2^cs_last h + s, with s = B^T (w o x) the tile's own contribution
//     from the tensor core; only an fp16 copy of h goes to shared memory.
// Per 128-token tile that is ~320 KB of shared-memory traffic (TMA writes of
// x, B, C 80 KB; tcgen05.cp of C 32 KB; MMA operand reads 112 KB; the E
// warps 64 KB; y staging and its TMA store 32 KB), ~2.5 k cycles at 128 B/clk.
//
// No role thread keeps a global load in flight across an mbarrier arrival
// (an arrival is a release, which waits for the thread's outstanding loads):
// global inputs come in through TMA or through the scan warp, which runs up to
// four tiles ahead.
//
// Roles (768 threads):
//   P   (warps 0-7):  C' scaling and the causal mask S.  Two warps per TMEM
//                     lane quarter split the 16-column blocks of a row by
//                     parity.
//   E   (warps 8-15): x -> fp16 operands and the state update.  Two warps
//                     per lane quarter split the 64 columns.
//   Y   (warps 20-23): the epilogue, Y (TMEM) -> bf16 -> y, one warp per
//                     lane quarter.
//   W16 (lane 0):     TMA loads of x, B and C, two stages.
//   W17 (lane 0):     s, C' h_prev and S x MMAs.
//   W18 (lane 0):     C -> TMEM copies and the C B^T MMAs.
//   W19:              the decay scan (softplus, cumulative sum, mask column
//                     factors) of the coming tiles into a four-slot ring.
// Every per-tile barrier exists per tile parity, and every barrier's next
// phase (tile t + 2) depends on an action its waiters take after waiting for
// tile t, so no waiter can see a barrier two phases ahead.
namespace v3 {

constexpr int kThreads3 = 800;

// Per-tile event timestamps of CTA 0, compiled in only with -DSSD_TC_TRACE
// (performance analysis builds); a no-op otherwise.
#ifdef SSD_TC_TRACE
__device__ long long g_tc_trace[48][1024];
#define TC_TRACE(ev, t) \
    do { if (blockIdx.x == 0 && (t) >= 0 && (t) < 1024) g_tc_trace[ev][t] = clock64(); } while (0)
__device__ unsigned long long g_cta_span[8192][3];   // start, end (global ns), SM id
#else
#define TC_TRACE(ev, t) do { } while (0)
#endif
constexpr int kRoleWarps = 8;       // P and E arrive once per warp
constexpr uint32_t kColC = 0;       // two 64-column buffers: C, then C' (fp16 pairs)
constexpr uint32_t kColCB = 128;    // C B^T, fp32 128 x 128
constexpr uint32_t kColS = 256;     // S, fp16 pairs (64 columns)
constexpr uint32_t kColSt = 320;    // s, fp32 128 x 64
constexpr uint32_t kColY = 384;     // two 64-column fp32 buffers


struct __align__(1024) Smem {
    uint8_t b[2][2][kBoxBytes];       // B (fp16), two 64-column boxes per stage
    uint8_t c[2][2][kBoxBytes];       // C (fp16)
    uint8_t x[2][kTileBytesX];        // x (bf16 from TMA, fp16 after conversion), per stage
    uint8_t wx[kTileBytesX];          // w o x (fp16)
    uint8_t hs[2][kTileBytesX];       // state entering tile t (fp16), buffer t & 1
    float cs[4][kT];                  // tile-local cumulative decay (base-2 exponent), slot u & 3
    float d[4][kT];
    float colfac[4][kT];              // 2^(cs_m - cs_i) d_i, pivot m = last token of i's 16-block
    uint64_t full[2];                 // TMA x, B, C -> W18, W17, E
    uint64_t scan_done[4];            // W19 (decay scan of tile u in slot u & 3) -> P, E
    uint64_t scan_free[4];            // P, E (slot read) -> W19
    uint64_t cb_full[2];              // W18 commit (C in TMEM, C B^T) -> P
    uint64_t cb_free[2];              // P (C B^T read) -> W18
    uint64_t c_scaled[2];             // P (C' in TMEM) -> W17
    uint64_t s_ready[2];              // P (S in TMEM) -> W17
    uint64_t x_ready[2];              // E (x, w o x written) -> W17
    uint64_t hs_ready[2];             // E -> W17
    uint64_t stg_free[2];             // Y (y staged in hs[t & 1] has been stored) -> E
    uint64_t s_done[2];               // W17 commit -> E
    uint64_t y_full[2];               // W17 commit -> E, P, W16, W18
    uint64_t fin[3];                  // W18, W17, W24: own tcgen05 work drained before exit
    uint32_t tmem_base;
    TcCtl ctl;
};

// kSplit: the launch holds split segments (SplitSpec); the plain instantiation carries none
// of their bookkeeping.
template <bool kSplit>
__global__ void __launch_bounds__(kThreads3, 1)
k_tc_scan3(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, const TcParams p) {
    constexpr int N = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    TcCtl& ctl = s.ctl;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, G = p.G;
    const int h = blockIdx.x % H;
    const int seq = blockIdx.x / H;
    const int g = h / (H / G);

    int64_t row, t0, t1;
    const float* init_src = nullptr;   // state entering the span (null: zero)
    float* final_dst = nullptr;        // state leaving it (null: not wanted)
    float* tok_cs = nullptr;           // running log-decay per token (split segments only)
    bool y_f16 = false;                // y written as fp16 (a segment after the first of its row)
    if (kSplit && seq >= p.split.first) {
        const int sp = seq - p.split.first, k = sp % p.split.K;
        row = p.split.row0 + sp / p.split.K;
        t0 = (int64_t)k * p.split.Ls;
        t1 = k == p.split.K - 1 || t0 + p.split.Ls > p.si.L ? p.si.L : t0 + p.split.Ls;
        if (k == 0 && p.init_state) init_src = p.init_state + (row * H + h) * N * kP;
        final_dst = p.split.fin + ((int64_t)sp * H + h) * N * kP;
        tok_cs = p.split.cs + ((int64_t)sp * H + h) * p.split.tiles * kT;
        y_f16 = k > 0;
    } else {
        seq_span(p.si, seq, row, t0, t1);
        if (p.init_state) init_src = p.init_state + ((int64_t)seq * H + h) * N * kP;
        if (p.final_state) final_dst = p.final_state + ((int64_t)seq * H + h) * N * kP;
    }
    const int64_t len = t1 > t0 ? t1 - t0 : 0;
    const int nt = (int)((len + kT - 1) / kT);
    const int64_t tok0 = row * p.si.L + t0;
    auto tile_len = [&](int t) { return (int)(len - (int64_t)t * kT < kT ? len - (int64_t)t * kT : kT); };

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) {
            mbar_init(&s.scan_done[i], 1);
            mbar_init(&s.scan_free[i], 2 * kRoleWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.cb_full[i], 1);
            mbar_init(&s.cb_free[i], kRoleWarps);
            mbar_init(&s.c_scaled[i], kRoleWarps);
            mbar_init(&s.s_ready[i], kRoleWarps);
            mbar_init(&s.x_ready[i], kRoleWarps);
            mbar_init(&s.hs_ready[i], kRoleWarps);
            mbar_init(&s.stg_free[i], 1);
            mbar_init(&s.s_done[i], 1);
            mbar_init(&s.y_full[i], 1);
            mbar_init(&s.fin[i], 1);
        }
        mbar_init(&s.fin[2], 1);
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&s.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    const float kLog2e = 1.4426950408889634f;
    // Every warp of a role polls the mbarrier itself (no rendezvous inside the role: a warp that
    // lags its siblings does not hold the others back); the result is uniform per warp.
    auto wait_w = [&](uint64_t* bar, uint32_t par) { return wait_bar_w(ctl, bar, par, p.status); };
    auto wait_w2 = [&](uint64_t* b1, uint32_t p1, uint64_t* b2, uint32_t p2) {
        return wait_bar_w(ctl, b1, p1, p.status) && (!b2 || wait_bar_w(ctl, b2, p2, p.status));
    };
#ifdef SSD_TC_TRACE
    if (tid == 0 && blockIdx.x < 8192) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        g_cta_span[blockIdx.x][0] = globaltimer_ns();
        g_cta_span[blockIdx.x][2] = smid;
    }
#endif

#ifdef SSD_TC_TRACE
    if (warp == 16 && lane == 1) {
        // observer: timestamps of MMA completions
        if (blockIdx.x == 0) {
            int tc = 0, ts = 0, ty = 0;
            const long long t_start = clock64();
            while ((tc < nt || ts < nt || ty < nt) && clock64() - t_start < 2000000000ll) {
                if (tc < nt && mbar_test_wait(&s.cb_full[tc & 1], (tc >> 1) & 1)) { TC_TRACE(25, tc); ++tc; }
                if (ts < nt && mbar_test_wait(&s.s_done[ts & 1], (ts >> 1) & 1)) { TC_TRACE(26, ts); ++ts; }
                if (ty < nt && mbar_test_wait(&s.y_full[ty & 1], (ty >> 1) & 1)) { TC_TRACE(27, ty); ++ty; }
            }
        }
    } else
#endif
    if (warp == 19) {
        // --------------------- W19: decay scan of each tile into a four-slot ring
        // Lane l takes tokens 4l .. 4l + 3 of the tile: d = softplus(dt + dt_bias),
        // a = d A log2(e), inclusive cumulative sum over the tile (serial within the lane,
        // shuffles across lanes), and the rank-1 column factors of the decay mask.
        const float A2 = p.A[h] * kLog2e;
        const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
        // dt of the next tile is loaded right after this tile's arrival (an arrival is a
        // release and would otherwise wait for it), and lands while the warp waits
        float dtn[4];
        auto load_dt = [&](int u) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 4 * lane + i;
                dtn[i] = (int64_t)u * kT + r < len ? __bfloat162float(p.dt[(tok0 + (int64_t)u * kT + r) * H + h]) : 0.f;
            }
        };
        if (nt > 0) load_dt(0);
        float run = 0.f;   // log-decay from the span start through the tile before u
        for (int u = 0; u < nt; ++u) {
            const int sl = u & 3, qu = tile_len(u);
            // P and E have read slot sl for tile u - 4
            if (u >= 4 && !wait_bar_w(ctl, &s.scan_free[sl], ((u - 4) >> 2) & 1, p.status)) break;
            float dd[4], cs[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dd[i] = 4 * lane + i < qu ? softplus_fast(dtn[i] + bias) : 0.f;
                cs[i] = (i ? cs[i - 1] : 0.f) + dd[i] * A2;
            }
            float incl = cs[3];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const float excl = incl - cs[3];
            // pivot of token 4 lane + i: the last token of its 16-token block, held by lane | 3
            const float pivot = __shfl_sync(0xffffffffu, incl, lane | 3);
            float cf[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                cs[i] += excl;
                cf[i] = ex2(pivot - cs[i]) * dd[i];
            }

            *reinterpret_cast<float4*>(&s.cs[sl][4 * lane]) = make_float4(cs[0], cs[1], cs[2], cs[3]);
            *reinterpret_cast<float4*>(&s.d[sl][4 * lane]) = make_float4(dd[0], dd[1], dd[2], dd[3]);
            *reinterpret_cast<float4*>(&s.colfac[sl][4 * lane]) = make_float4(cf[0], cf[1], cf[2], cf[3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.scan_done[sl]);
            if (kSplit) {
                if (tok_cs)
                    *reinterpret_cast<float4*>(tok_cs + (int64_t)u * kT + 4 * lane) =
                        make_float4(run + cs[0], run + cs[1], run + cs[2], run + cs[3]);
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (u + 1 < nt) load_dt(u + 1);
        }
    } else if (warp == 16) {
        // ------------------------------------------------- W16: TMA x, B, C
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            tma_prefetch_desc(&tm_c);
            int issued = 0;
            // x comes from HBM with a latency of a few thousand cycles, more than the two stages
            // hide: each tile's x is pulled into L2 four tiles before its load
            for (int u = 0; u < 4 && u < nt; ++u) tma_prefetch_l2_3d(&tm_x, 0, h, (int)(tok0 + (int64_t)u * kT));
            for (int u = 0; u < nt; ++u) {
                const int st = u & 1;
                if (u + 4 < nt) tma_prefetch_l2_3d(&tm_x, 0, h, (int)(tok0 + (int64_t)(u + 4) * kT));
                // stage st is free once every MMA of tile u - 2 has completed: W24's output chain
                // (y_full) and W17's B^T (w o x) (s_done), issued by different threads
                if (u >= 2 && !wait_bar(ctl, &s.y_full[st], ((u - 2) >> 1) & 1, p.status)) break;
                if (u >= 2 && !wait_bar(ctl, &s.s_done[st], ((u - 2) >> 1) & 1, p.status)) break;
                const int tok = (int)(tok0 + (int64_t)u * kT);
                mbar_expect_tx(&s.full[st], kTileBytesX + 4 * kBoxBytes);
                tma_load_3d(s.x[st], &tm_x, &s.full[st], 0, h, tok);
                for (int k = 0; k < 2; ++k) {
                    tma_load_3d(s.b[st][k], &tm_b, &s.full[st], 64 * k, g, tok);
                    tma_load_3d(s.c[st][k], &tm_c, &s.full[st], 64 * k, g, tok);
                }
                ++issued;
                TC_TRACE(0, u);
            }
            if (*(volatile int*)&ctl.abort) {
                // let the copies already in flight land before the CTA exits
                for (int u = 0; u < issued; ++u) mbar_wait(&s.full[u & 1], (u >> 1) & 1, 400000000ll);
            }
        }
    } else if (warp == 18) {
        // ------------------------------------------- W18: C -> TMEM, C B^T
        if (lane == 0 && nt > 0) {
            const uint32_t id_cb = idesc_f16(128, 128, 0, 0);
            for (int t = 0; t < nt; ++t) {
                const int st = t & 1;
                if (!wait_bar(ctl, &s.full[st], (t >> 1) & 1, p.status)) break;
                // (TMEM C buffer st is free again: full(t) follows W16's wait for y_full(t - 2), which
                // follows C' h_prev of tile t - 2)
                tc_fence_after();
                // descriptors differ per K step only in the start address (low bits, in 16-byte units)
                const uint64_t dc = sdesc_sw128(smem_u32(s.c[st][0]), 16, 1024);
                const uint64_t db = sdesc_sw128(smem_u32(s.b[st][0]), 16, 1024);
                const uint32_t ct = tmem + kColC + 64 * st;
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k)
                    tmem_cp_128x256b(ct + 8 * k, dc + (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4));
                TC_TRACE(1, t);
                // P has read C B^T of tile t - 1
                if (t >= 1 && !wait_bar(ctl, &s.cb_free[st ^ 1], ((t - 1) >> 1) & 1, p.status)) break;
                tc_fence_after();
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k)
                    mma_ts(tmem + kColCB, ct + 8 * k, db + (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4), id_cb,
                           k > 0);
                mma_commit(&s.cb_full[st]);
                TC_TRACE(2, t);
            }
            mma_commit(&s.fin[0]);
            mbar_wait(&s.fin[0], 0, 400000000ll);
        }
    } else if (warp == 17) {
        // -------------------------------------------------- W17: s = B^T (w o x)
        if (lane == 0 && nt > 0) {
            const uint32_t id_st = idesc_f16(128, 64, 1, 1);   // MN-major A (B^T) and B (w o x)
            for (int t = 0; t < nt; ++t) {
                const int st = t & 1;
                const uint32_t par = (t >> 1) & 1;
                const uint64_t db = sdesc_sw128(smem_u32(s.b[st][0]), kBoxBytes, 1024);
                const uint64_t dwx = sdesc_sw128(smem_u32(s.wx), kBoxBytes, 1024);
                // (the single s buffer is free again: E loads s of tile t - 1 before it writes the
                // w o x of tile t that x_ready announces)
                if (!wait_bar(ctl, &s.x_ready[st], par, p.status)) break;
                if (!wait_bar(ctl, &s.full[st], par, p.status)) break;
                // a partial tile's B rows past the sequence end are zeroed by P before c_scaled
                if (tile_len(t) < kT && !wait_bar(ctl, &s.c_scaled[st], par, p.status)) break;
                TC_TRACE(3, t);
                tc_fence_after();
#pragma unroll 1
                for (int k = 0; k < kT / 16; ++k)
                    mma_ss(tmem + kColSt, db + (uint64_t)(k * 128), dwx + (uint64_t)(k * 128), id_st, k > 0);
                mma_commit(&s.s_done[st]);
                TC_TRACE(4, t);
            }
            mma_commit(&s.fin[1]);
            mbar_wait(&s.fin[1], 0, 400000000ll);
        }
    } else if (warp == 24) {
        // --------------------------------------------- W24: Y = C' h_prev + S x
        // A second MMA-issuing thread: an issuing thread is held for each tcgen05.mma it issues,
        // and a chain accumulating into one TMEM buffer waits for its previous step, so the
        // tile's two independent chains (s on W17, Y here) run side by side.
        if (lane == 0 && nt > 0) {
            const uint32_t id_y = idesc_f16(128, 64, 0, 1);    // A from TMEM, MN-major B
            for (int t = 0; t < nt; ++t) {
                const int st = t & 1;
                const uint32_t par = (t >> 1) & 1;
                const uint64_t dx = sdesc_sw128(smem_u32(s.x[st]), kBoxBytes, 1024);
                const uint64_t dhs = sdesc_sw128(smem_u32(s.hs[st]), kBoxBytes, 1024);
                // Y = C' h_prev: needs the state entering tile t and C'.  (The Y buffer is free
                // again: hs_ready(t) follows E's wait for stg_free(t - 2), which the epilogue
                // arrives at after reading Y of tile t - 2.)
                if (!wait_bar(ctl, &s.hs_ready[st], par, p.status)) break;
                if (!wait_bar(ctl, &s.c_scaled[st], par, p.status)) break;
                TC_TRACE(5, t);
                tc_fence_after();
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k)
                    mma_ts(tmem + kColY + 64 * st, tmem + kColC + 64 * st + 8 * k, dhs + (uint64_t)(k * 128), id_y, k > 0);
                TC_TRACE(6, t);
                // Y += S x: needs S and the converted x of tile t
                if (!wait_bar(ctl, &s.s_ready[st], par, p.status)) break;
                if (!wait_bar(ctl, &s.x_ready[st], par, p.status)) break;
                TC_TRACE(7, t);
                tc_fence_after();
#pragma unroll 1
                for (int k = 0; k < kT / 16; ++k)
                    mma_ts(tmem + kColY + 64 * st, tmem + kColS + k * 8, dx + (uint64_t)(k * 128), id_y, 1);
                mma_commit(&s.y_full[st]);
                TC_TRACE(8, t);
            }
            mma_commit(&s.fin[2]);
            mbar_wait(&s.fin[2], 0, 400000000ll);
        }
    } else if (warp < 8) {
        // -------------------------------------- P: C', decay mask, decay scan
        const int quarter = warp & 3, half = warp >> 2;
        const int j = 32 * quarter + lane;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float Dh = p.D ? p.D[h] : 0.f;
        // S blocks right of this quarter's diagonal stay zero: write them once.
        {
            const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            for (int b = 2 * quarter + 2 + half; b < 8; b += 2) tmem_st8(tmem + lane_base + kColS + 8 * b, z);
            tmem_st_wait();
        }
        for (int t = 0; t < nt; ++t) {
            const int st = t & 1;
            const uint32_t par = (t >> 1) & 1;
            const int sl = t & 3;
            if (!wait_w2(&s.scan_done[sl], (t >> 2) & 1, &s.cb_full[st], par))
                break;
            if (tid == 128) TC_TRACE(9, t);
            tc_fence_after();
            const float cs2j = s.cs[sl][j];
            {
                // C'_j = 2^cs_j C_j in place in TMEM (this warp: 32 of the 64 columns)
                const __half2 e2 = __float2half2_rn(ex2(cs2j));
                const uint32_t ct = tmem + lane_base + kColC + 64 * st + 32 * half;
                uint32_t r0[16], r1[16];
                tmem_ld16(ct, r0);
                tmem_ld16(ct + 16, r1);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    r0[i] = h2u(__hmul2(u2h(r0[i]), e2));
                    r1[i] = h2u(__hmul2(u2h(r1[i]), e2));
                }
                tmem_st16(ct, r0);
                tmem_st16(ct + 16, r1);
                tmem_st_wait();
                if (tile_len(t) < kT && j >= tile_len(t)) {
                    // C B^T has read B: zero this row past the sequence end so that B^T (w o x)
                    // meets exact zeros there even for non-finite values of the next sequence
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(s.b[st][half] + sw128_off(j, c)) = z;
                    fence_proxy_async_smem();
                }
                tc_fence_before();
                warp_arrive(&s.c_scaled[st]);
                if (tid == 128) TC_TRACE(10, t);
            }
            // S = C B^T o 2^(cs_j - cs_i) d_i (i <= j), D on the diagonal.  This warp takes the
            // 16-column blocks b = 2m + half: m < quarter lie left of the diagonal 32-block
            // (rank-1 split, one exponential per block), m = quarter holds the diagonal (one
            // exponential per element, masked with a select).  All held in registers until
            // the S buffer is free.
            uint32_t sv[4][8];
            const uint32_t cbuf = tmem + lane_base + kColCB;
#pragma unroll
            for (int m = 0; m < 3; ++m) {
                if (m < quarter) {
                    const int i0 = 16 * (2 * m + half);
                    uint32_t r[16];
                    tmem_ld16(cbuf + i0, r);
                    const float rf = ex2(cs2j - s.cs[sl][i0 + 15]);
                    const uint64_t rf2 = f2pack(rf, rf);
                    uint64_t f[8];
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        const float4 cf = *reinterpret_cast<const float4*>(&s.colfac[sl][i0 + 2 * k]);
                        f[k] = f2mul(f2pack(cf.x, cf.y), rf2);
                        f[k + 1] = f2mul(f2pack(cf.z, cf.w), rf2);
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float lo, hi;
                        f2unpack(f2mul(f2pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), f[k]), lo, hi);
                        sv[m][k] = pack_f16x2(lo, hi);
                    }
                }
            }
            {
                const int i0 = 16 * (2 * quarter + half);
                uint32_t r[16];
                tmem_ld16(cbuf + i0, r);
                float f[16];
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    const float4 cv = *reinterpret_cast<const float4*>(&s.cs[sl][i0 + k]);
                    const float4 dv = *reinterpret_cast<const float4*>(&s.d[sl][i0 + k]);
                    f[k] = ex2(cs2j - cv.x) * dv.x;
                    f[k + 1] = ex2(cs2j - cv.y) * dv.y;
                    f[k + 2] = ex2(cs2j - cv.z) * dv.z;
                    f[k + 3] = ex2(cs2j - cv.w) * dv.w;
                }
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    float v0 = i0 + k <= j ? __uint_as_float(r[k]) * f[k] : 0.f;
                    float v1 = i0 + k + 1 <= j ? __uint_as_float(r[k + 1]) * f[k + 1] : 0.f;
                    if (i0 + k == j) v0 += Dh;
                    if (i0 + k + 1 == j) v1 += Dh;
                    sv[3][k / 2] = pack_f16x2(v0, v1);
                }
            }
            tc_fence_before();
            warp_arrive(&s.cb_free[st]);
            warp_arrive(&s.scan_free[sl]);
            if (tid == 128) TC_TRACE(11, t);
            if (tid == 96) TC_TRACE(15, t);
            // the S buffer is free once S x of tile t - 1 has completed
            if (t > 0 && !wait_w(&s.y_full[st ^ 1], ((t - 1) >> 1) & 1))
                break;
            if (tid == 128) TC_TRACE(12, t);
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < 3; ++m)
                if (m < quarter) tmem_st8(tmem + lane_base + kColS + 8 * (2 * m + half), sv[m]);
            tmem_st8(tmem + lane_base + kColS + 8 * (2 * quarter + half), sv[3]);
            tmem_st_wait();
            tc_fence_before();
            warp_arrive(&s.s_ready[st]);
            if (tid == 128) TC_TRACE(13, t);
            if (tid == 96) TC_TRACE(16, t);

            if (tid == 128) TC_TRACE(14, t);
        }
    } else if (warp >= 20 && warp < 24) {
        // ---------------------------------------------- Y: epilogue, y = Y
        // A full tile is staged (bf16, 128-byte swizzled rows) in hs[u & 1], free once C' h_prev
        // of tile u has completed and until E writes the state entering tile u + 2 there, and
        // leaves by one TMA store; a partial tile (the end of a sequence) is stored row by row,
        // since the rows past its end belong to the next sequence.
        const int quarter = warp & 3;
        const int j = 32 * quarter + lane;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const bool issuer = warp == 20 && lane == 0;
        bool stored = false;
        if (issuer) tma_prefetch_desc(&tm_y);
        for (int u = 0; u < nt; ++u) {
            const int q = tile_len(u);
            if (!wait_w(&s.y_full[u & 1], (u >> 1) & 1)) break;
            tc_fence_after();
            const uint32_t ya = tmem + lane_base + kColY + 64 * (u & 1);
            uint8_t* stg = s.hs[u & 1];
            __nv_bfloat16* yrow = p.y + (tok0 + (int64_t)u * kT + j) * H * kP + (int64_t)h * kP;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[32];
                tmem_ld16(ya + 32 * hh, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16(ya + 32 * hh + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    // a split segment's partial y waits in fp16 for the state-to-output pass
                    // (11 significant bits: its later rounding to bf16 stays the only one that
                    // counts even where that pass cancels most of it)
                    auto pk = [&](int e) {
                        const float lo = __uint_as_float(r[8 * c + e]), hi = __uint_as_float(r[8 * c + e + 1]);
                        return kSplit && y_f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
                    };
                    const uint4 val = make_uint4(pk(0), pk(2), pk(4), pk(6));
                    if (q == kT)
                        *reinterpret_cast<uint4*>(stg + sw128_off(j, 4 * hh + c)) = val;
                    else if (j < q)
                        *reinterpret_cast<uint4*>(yrow + 32 * hh + 8 * c) = val;
                }
            }
            if (q == kT) fence_proxy_async_smem();
            tc_fence_before();      // the Y reads precede stg_free, hence the next MMA into this buffer
            asm volatile("bar.sync 3, 128;" ::: "memory");
            if (issuer) {
                if (q == kT) {
                    tma_store_3d(&tm_y, stg, 0, h, (int)(tok0 + (int64_t)u * kT));
                    bulk_commit();
                    bulk_wait_read0();
                    stored = true;
                }
                mbar_arrive(&s.stg_free[u & 1]);
            }
            if (lane == 0 && warp == 20) TC_TRACE(22, u);
        }
        if (issuer && stored) bulk_wait0();
    } else if (warp < 16) {
        // ------------------------------------------- E: x operands, state
        const int quarter = warp & 3, half = (warp >> 2) & 1;
        const int j = 32 * quarter + lane;     // token row (x, y) and state row (s, h)
        const int col0 = 32 * half;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        float hreg[32];
        {
            const float* src = init_src ? init_src + (int64_t)j * kP + col0 : nullptr;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 v = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                hreg[c] = v.x; hreg[c + 1] = v.y; hreg[c + 2] = v.z; hreg[c + 3] = v.w;
            }
        }
        // fp16 copy of the state entering tile u, into hs[u & 1]
        auto put_state = [&](int u) {
            uint8_t* hsu = s.hs[u & 1];
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
                uint4 v;
                v.x = pack_f16x2(hreg[c], hreg[c + 1]);
                v.y = pack_f16x2(hreg[c + 2], hreg[c + 3]);
                v.z = pack_f16x2(hreg[c + 4], hreg[c + 5]);
                v.w = pack_f16x2(hreg[c + 6], hreg[c + 7]);
                *reinterpret_cast<uint4*>(hsu + sw128_off(j, (col0 + c) / 8)) = v;
            }
            fence_proxy_async_smem();
            warp_arrive(&s.hs_ready[u & 1]);
        };
        // x of tile k -> fp16 in place (zero past the sequence end); returns the tile's total
        // decay 2^cs_last and this row's weight w_j = d_j 2^(cs_last - cs_j).
        auto convert_x = [&](int k, float& e_tot, __half2& w2) {
            const int q = tile_len(k);
            const float cs_last = s.cs[k & 3][q - 1];
            e_tot = ex2(cs_last);
            w2 = __float2half2_rn(s.d[k & 3][j] * ex2(cs_last - s.cs[k & 3][j]));
            warp_arrive(&s.scan_free[k & 3]);
            uint8_t* xt = s.x[k & 1];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t off = sw128_off(j, col0 / 8 + m);
                const uint4 xv = *reinterpret_cast<const uint4*>(xt + off);
                uint4 o;
                o.x = pack_f16x2(bf16lo(xv.x), bf16hi(xv.x));
                o.y = pack_f16x2(bf16lo(xv.y), bf16hi(xv.y));
                o.z = pack_f16x2(bf16lo(xv.z), bf16hi(xv.z));
                o.w = pack_f16x2(bf16lo(xv.w), bf16hi(xv.w));
                if (j >= q) o = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4*>(xt + off) = o;
            }
        };
        // w o x of tile k from its converted x, then x_ready
        auto write_wx = [&](int k, __half2 w2) {
            const uint8_t* xt = s.x[k & 1];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t off = sw128_off(j, col0 / 8 + m);
                const uint4 o = *reinterpret_cast<const uint4*>(xt + off);
                uint4 w;
                w.x = h2u(__hmul2(u2h(o.x), w2));
                w.y = h2u(__hmul2(u2h(o.y), w2));
                w.z = h2u(__hmul2(u2h(o.z), w2));
                w.w = h2u(__hmul2(u2h(o.w), w2));
                *reinterpret_cast<uint4*>(s.wx + off) = w;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(&s.x_ready[k & 1]);
        };
        bool ok = true;
        float e_cur = 1.f, e_next = 1.f;   // 2^cs_last of tiles t and t + 1
        __half2 w_next = __float2half2_rn(0.f);
        if (nt > 0) {
            put_state(0);
            if ((ok = wait_w2(&s.scan_done[0], 0, &s.full[0], 0))) {
                convert_x(0, e_cur, w_next);
                write_wx(0, w_next);
            }
        }
        // Tile t: x of tile t + 1 is converted while B^T (w o x) of tile t runs; once it has
        // completed, s(t) is taken into the state, and w o x of tile t + 1 (the single w o x
        // buffer is free again) and the state entering tile t + 1 are written.
        for (int t = 0; ok && t < nt; ++t) {
            if (t + 1 < nt) {
                const int k = t + 1;
                if (!(ok = wait_w2(&s.scan_done[k & 3], (k >> 2) & 1, &s.full[k & 1], (k >> 1) & 1))) break;
                if (tid == 256) TC_TRACE(19, k);
                convert_x(k, e_next, w_next);
                if (tid == 256) TC_TRACE(21, k);
            }
            // s(t) is complete (and hs[(t + 1) & 1] free again: it held y of tile t - 1 on its way out)
            if (!(ok = wait_w2(&s.s_done[t & 1], (t >> 1) & 1,
                                     (t >= 1 && t + 1 < nt) ? &s.stg_free[(t + 1) & 1] : nullptr,
                                     ((t - 1) >> 1) & 1)))
                break;
            if (tid == 256) TC_TRACE(17, t);
            tc_fence_after();
            {
                uint32_t r0[16], r1[16];
                tmem_ld16(tmem + lane_base + kColSt + col0, r0);
                tmem_ld16(tmem + lane_base + kColSt + col0 + 16, r1);
                tmem_ld_wait();
                const uint64_t e2 = f2pack(e_cur, e_cur);
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    float lo, hi;
                    f2unpack(f2fma(e2, f2pack(hreg[i], hreg[i + 1]),
                                   f2pack(__uint_as_float(r0[i]), __uint_as_float(r0[i + 1]))), lo, hi);
                    hreg[i] = lo; hreg[i + 1] = hi;
                    f2unpack(f2fma(e2, f2pack(hreg[16 + i], hreg[17 + i]),
                                   f2pack(__uint_as_float(r1[i]), __uint_as_float(r1[i + 1]))), lo, hi);
                    hreg[16 + i] = lo; hreg[17 + i] = hi;
                }
            }
            if (t + 1 < nt) {
                write_wx(t + 1, w_next);
                if (tid == 256) TC_TRACE(20, t + 1);
                put_state(t + 1);
                if (tid == 256) TC_TRACE(18, t + 1);
            }
            e_cur = e_next;
        }
        if (final_dst && (ok || nt == 0)) {
            float* dst = final_dst + (int64_t)j * kP + col0;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
                *reinterpret_cast<float4*>(dst + c) = make_float4(hreg[c], hreg[c + 1], hreg[c + 2], hreg[c + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
#ifdef SSD_TC_TRACE
    if (tid == 0 && blockIdx.x < 8192) g_cta_span[blockIdx.x][1] = globaltimer_ns();
#endif
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace v3


// bf16 -> fp16 copies of B and C (8 elements per thread step).

__global__ void k_tc_prep(const uint4* __restrict__ b, const uint4* __restrict__ c, uint4* __restrict__ b16,
                          uint4* __restrict__ c16, int64_t n8) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        b16[i] = bf16x8_to_f16x8(b[i]);
        c16[i] = bf16x8_to_f16x8(c[i]);
    }
}

// ---- Few long rows: the segment split ------------------------------------------------------
//
// One CTA scans one (row, head) from start to end, so when b H is small (few long rows) most
// SMs sit idle.  The rows from W on (all rows, unless forced otherwise) are then cut into K
// segments of Ls tokens (tile-aligned; the last runs to the row's end).  One launch of the
// scan takes the whole rows and every segment (segment 0 from the row's initial state, the
// others from zero; see SplitSpec), and k_state_out adds to every later segment the output
// of the state entering it, chained from the segments' final states and total decays
// (section 4.2 of "5.3 Tensor Parallelism support and large-cluster training", state
// passing at segment granularity), and writes the row's final state.

struct SplitPlan {
    int K = 0;                 // segments per split row; 0: no split
    int64_t W = 0;             // whole rows 0 .. W - 1; rows W .. b - 1 are split
    int64_t Ls = 0;            // tokens per segment
    int tiles = 0;             // Ls / 128
};


// SSD_TC_SPLIT="K" or "K,R", read once: split the last R rows (default: all) into K segments
// whenever a row has at least K tiles; "1": never split (for tests and tuning); "0" or unset:
// the plan below.
struct ForcedSplit {
    int K = 0, R = 0;
};
ForcedSplit forced_split() {
    static ForcedSplit v;
    static bool read = false;
    if (!read) {
        const char* e = getenv("SSD_TC_SPLIT");
        int k = 0, r = 0;
        if (e && sscanf(e, "%d,%d", &k, &r) >= 1 && k >= 1 && k <= 64) v = {k, r > 0 ? r : 0};
        read = true;
    }
    return v;
}


// The plan: split only rows that leave at least half the SMs idle (b H <= S / 2), every row
// into the most segments that still run in one wave (b H K <= S), with at least 8 tiles per
// segment.  Measured on B200 (b1 L131072 H64): K = 2 beats the single pass by 30 % and K = 3
// (two waves) by a further 40 %; three unequal segments sized to fill all 148 SMs (443 + 443 + 138
// tiles) take 1.42 ms against 1.26-1.32 ms for the two halves on 128 SMs, because a CTA's tiles
// slow down as more CTAs run at once (below).  Filling only the last, partial wave of a long batch does
// not pay: a CTA's tiles run faster when fewer CTAs share the GPU (about 1.8 us per tile
// with 48 CTAs against 2.9 us with 148 on b8 L4096 H80), so the time won in the scan (~25 us)
// goes to the state-to-output pass.
SplitPlan plan_split(const ScanArgs& a) {
    SplitPlan pl;
    const int64_t nt = (a.L + kT - 1) / kT;
    if (a.seq_idx || a.b * a.H <= 0 || a.N != 128) return pl;
    const int S = sm_count();
    const ForcedSplit f = forced_split();
    int K;
    int64_t R = a.b;   // rows split (the last R)
    if (f.K) {
        if (f.K == 1 || nt < f.K) return pl;
        K = f.K;
        if (f.R && f.R < a.b) R = f.R;
    } else {
        if (a.b * a.H * 2 > S) return pl;
        K = (int)std::min<int64_t>(8, S / (a.b * a.H));
        if (K < 2 || nt < 8 * (int64_t)K) return pl;
    }
    pl.tiles = (int)((nt + K - 1) / K);
    pl.Ls = (int64_t)pl.tiles * kT;
    if ((K - 1) * pl.Ls >= a.L) return SplitPlan();
    pl.K = K;
    pl.W = a.b - R;
    return pl;
}

size_t split_workspace_bytes(const ScanArgs& a, const SplitPlan& pl) {
    if (!pl.K) return 0;
    const size_t spans = (size_t)(a.b - pl.W) * pl.K * a.H;
    return ((spans * a.N * a.P * sizeof(float) + 255) & ~(size_t)255) +
           ((spans * pl.tiles * kT * sizeof(float) + 255) & ~(size_t)255);
}


}  // namespace

#ifdef SSD_TC_TRACE
extern "C" __attribute__((visibility("default"))) int ssd_tc_trace_read(long long* out) {
    return (int)cudaMemcpyFromSymbol(out, v3::g_tc_trace, sizeof(v3::g_tc_trace));
}
extern "C" __attribute__((visibility("default"))) int ssd_tc_span_read(unsigned long long* out) {
    return (int)cudaMemcpyFromSymbol(out, v3::g_cta_span, sizeof(v3::g_cta_span));
}
extern "C" __attribute__((visibility("default"))) int ssd_tc_poll_read(unsigned long long* out) {
    cudaMemcpyFromSymbol(out, ptx::g_poll_iters, sizeof(ptx::g_poll_iters));
    return (int)cudaMemcpyFromSymbol(out + 32, ptx::g_poll_calls, sizeof(ptx::g_poll_calls));
}
#endif

bool tc_supported(const ScanArgs& a) {
    return a.dtype == 1 && a.P == kP && (a.N == 128 || a.N == 256) && (a.Q == 128 || a.Q == 256) &&
           a.b * a.L < ((int64_t)1 << 31) && a.S * a.H < ((int64_t)1 << 31) && get_encode() != nullptr;
}

size_t tc_workspace_bytes(const ScanArgs& a, int64_t) {
    const size_t bc = (2 * (size_t)a.b * a.L * a.G * a.N * sizeof(__half) + 255) & ~(size_t)255;
    return bc + 256 + split_workspace_bytes(a, plan_split(a));
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
    CUtensorMap tm_y;
    if (!make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)ntok))
        return 6;
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
    const SplitPlan pl = a.N == 128 ? plan_split(a) : SplitPlan();
    if (pl.K) {
        const int64_t R = a.b - pl.W, spans = R * pl.K;
        const size_t states = ((size_t)spans * a.H * a.N * a.P * sizeof(float) + 255) & ~(size_t)255;
        char* w = reinterpret_cast<char*>(ws) + ((2 * (size_t)ntok * a.G * a.N * sizeof(__half) + 255) & ~(size_t)255) + 256;
        p.split.first = (int32_t)pl.W;
        p.split.K = pl.K;
        p.split.row0 = (int32_t)pl.W;
        p.split.tiles = pl.tiles;
        p.split.Ls = pl.Ls;
        p.split.fin = reinterpret_cast<float*>(w);
        p.split.cs = reinterpret_cast<float*>(w + states);
        {
            const size_t smem = sizeof(v3::Smem) + 1024;
            cudaFuncSetAttribute(v3::k_tc_scan3<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            ProfScope ps(K_TC_SCAN, st);
            v3::k_tc_scan3<true><<<(unsigned)((pl.W + spans) * a.H), v3::kThreads3, smem, st>>>(tm_x, tm_b, tm_c, tm_y, p);
        }
        return launch_state_out_split(a, c16, p.split.fin, p.split.cs, pl.W, pl.K, pl.Ls, pl.tiles, status, st);
    }
    ProfScope ps(K_TC_SCAN, st);
    if (a.N == 128) {
        const size_t smem = sizeof(v3::Smem) + 1024;
        cudaFuncSetAttribute(v3::k_tc_scan3<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        v3::k_tc_scan3<false><<<(unsigned)(a.S * a.H), v3::kThreads3, smem, st>>>(tm_x, tm_b, tm_c, tm_y, p);
    } else {
        const size_t smem = sizeof(TcSmem<256>) + 1024;
        cudaFuncSetAttribute(k_tc_scan<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_tc_scan<256><<<(unsigned)(a.S * a.H), Cfg<256>::kThreads, smem, st>>>(tm_x, tm_b, tm_c, p);
    }
    return 0;
}


}  // namespace ssd
