// ssd_state_out.cu -- the output of a state entering a span of tokens, on the tensor cores:
// the second step of the segment split of long rows (launched by launch_tc_scan) and the C ABI
// call ssd_state_to_output (the sequence-parallel ring's last step).
#include <cuda.h>
#include <algorithm>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "ssd_common.cuh"
#include "ssd_prof.h"
#include "ssd_tc.h"
#include "tc_common.cuh"

namespace ssd {
namespace {

using namespace tc;

// ---- Contribution of an entering state to the output -------------------------------------
//
// For a span of tokens entered by the state h_in (N x P) and scanned from zero, the full
// output adds, at every token j of the span,
//   y_j += 2^(cs_j) C_j^T h_in,   cs_j = sum over the span's tokens i <= j of d_i A log2(e)
// (the state term of section 3.2 of "5.3 Tensor Parallelism support and large-cluster
// training", taken from the span start instead of the chunk start).  Per 128-token tile that
// is one 128 x 64 x 128 product C h_in on the tensor core (fp16 operands, as the scan's own
// C' h_prev), scaled by 2^cs_j per row in the epilogue and added to y in place.
//
// A CTA takes `tpp` consecutive tiles of one (span, head); its entering state is either given
// (h_in) or chained from the spans before it in the row: h_in(k) = 2^D(k-1) h_in(k-1) + F(k-1),
// with F the spans' own final states and D their total log-decay (the last entry of the
// running log-decay table cs).  The CTA holding the first tiles of a row's last span writes
// the row's final state 2^D h_in + F.
//
// Roles (384 threads, one CTA per SM):
//   warps 0-7:  prologue (the fp16 copy of h_in), then the epilogue: TMEM -> registers,
//               y tile (shared memory) += 2^cs_j (C h_in)_j.  Two warps per TMEM lane
//               quarter split the 64 columns; each warp hands its part on by itself.
//   warp 8:     TMA loads of the C and y tiles and a bulk copy of the tile's running
//               log-decays cs_j (a table the scan wrote), kStagesSO deep: no epilogue thread
//               waits on a global load.
//   warps 9, 10: the MMAs of the even and of the odd tiles (an issuing thread is held for
//               each tcgen05.mma it issues, so two of them keep up with the memory rate);
//               warp 9 also owns the TMEM allocation.
//   warp 11:    the TMA store of each finished y tile, which hands the stage back as soon as
//               the store has read it.
namespace so {

constexpr int kEpiWarps = 8;
constexpr int kThreadsSO = 32 * (kEpiWarps + 4);
constexpr int kStagesSO = 4;
constexpr uint32_t kTmemColsSO = 64 * kStagesSO;

struct __align__(1024) SmemSO {
    uint8_t c[kStagesSO][2][kBoxBytes];   // C (fp16), two 64-column boxes per stage
    uint8_t y[kStagesSO][kTileBytesX];    // y (bf16), updated in place and stored from here
    uint8_t hs[kTileBytesX];              // h_in (fp16), state rows, 128-byte swizzled
    float cs[kStagesSO][kT];              // running log-decay cs_j of the tile's tokens
    uint64_t full[kStagesSO];             // TMA (C, y) -> MMA, epilogue
    uint64_t acc_full[kStagesSO];         // MMA commit -> epilogue
    uint64_t acc_free[kStagesSO];         // epilogue (accumulator read) -> MMA
    uint64_t y_ready[kStagesSO];          // epilogue warps (y tile updated) -> store warp
    uint64_t stage_free[kStagesSO];       // store warp (y stored or written) -> TMA
    uint64_t hs_ready;                    // epilogue warps (h_in in shared memory) -> MMA
    uint64_t fin[2];                      // MMA warps: own MMAs drained before exit
    uint32_t tmem_base;
    TcCtl ctl;
};

struct SOParams {
    const __nv_bfloat16* dt;
    const float* dt_bias;
    const float* A;
    const float* h_in;     // (rows, H, N, P) given entering states, or null: chain from fin
    const float* fin;      // chained mode: final state of every span, (rows K, H, N, P)
    const float* cs;       // running log-decay from the span start through each token, 128 tiles
                           // floats per (span, head)
    float* final_state;    // chained mode: the rows' final states (batch rows, H, N, P) or null
    __nv_bfloat16* y;      // (batch rows, L, H, P), updated in place
    int y_f16;             // y holds fp16 partial outputs (chained mode), written back as bf16
    int32_t* status;
    int64_t L;             // tokens per batch row
    int64_t Ls;            // tokens per span (the last span of a row runs to its end)
    int H, G;
    int K;                 // spans per row
    int k0;                // first span corrected (chained mode 1: span 0 has its own state)
    int row0;              // batch row of the first row taken
    int tiles;             // tiles of the longest span
    int nparts, tpp;       // parts per span, tiles per part
};

__global__ void __launch_bounds__(kThreadsSO, 1)
k_state_out(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, const SOParams p) {
    constexpr int N = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    SmemSO& s = *reinterpret_cast<SmemSO*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    TcCtl& ctl = s.ctl;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    const int h = blockIdx.x % H;
    int64_t rest = blockIdx.x / H;
    const int part = (int)(rest % p.nparts);
    rest /= p.nparts;
    const int nk = p.K - p.k0;
    const int k = p.k0 + (int)(rest % nk);
    const int rr = (int)(rest / nk);               // row taken, relative to row0
    const int64_t row = p.row0 + rr;
    const int g = h / (H / p.G);
    const int64_t NP = (int64_t)N * kP;

    const int64_t s0 = (int64_t)k * p.Ls;
    const int64_t s1 = k == p.K - 1 || s0 + p.Ls > p.L ? p.L : s0 + p.Ls;
    const int nts = (int)((s1 - s0 + kT - 1) / kT);           // tiles of the span
    const int ft = part * p.tpp;                              // first tile of this part
    const int nt = ft < nts ? min(p.tpp, nts - ft) : 0;       // tiles of this part
    const int64_t span = (int64_t)rr * p.K + k;
    const float* cs_span = p.cs + (span * H + h) * p.tiles * kT;   // running log-decay per token
    const int64_t tok_base = row * p.L + s0 + (int64_t)ft * kT;   // flat token of the first tile

    if (tid == 0) {
        for (int i = 0; i < kStagesSO; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_free[i], kEpiWarps);
            mbar_init(&s.y_ready[i], kEpiWarps);
            mbar_init(&s.stage_free[i], 1);
        }
        mbar_init(&s.hs_ready, kEpiWarps);
        mbar_init(&s.fin[0], 1);
        mbar_init(&s.fin[1], 1);
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) tmem_alloc(&s.tmem_base, kTmemColsSO);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kEpiWarps) {
        // ---- prologue (while the first tiles load): the entering state, and the row's final
        // state; thread = (column half, state row)
        const int n = 32 * (warp & 3) + lane, c0 = 32 * (warp >> 2);
        float hv[32];
        if (p.h_in) {
            const float* src = p.h_in + (row * H + h) * NP + (int64_t)n * kP + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 v = *reinterpret_cast<const float4*>(src + c);
                hv[c] = v.x; hv[c + 1] = v.y; hv[c + 2] = v.z; hv[c + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) hv[c] = 0.f;
            for (int j = 0; j < k; ++j) {
                const int64_t sj = (int64_t)rr * p.K + j;
                // spans before the last hold Ls tokens; the decay of span j enters from j + 1 on
                const float e = j ? ex2(p.cs[(sj * H + h) * p.tiles * kT + p.Ls - 1]) : 0.f;
                const float* f = p.fin + (sj * H + h) * NP + (int64_t)n * kP + c0;
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(f + c);
                    hv[c] = e * hv[c] + v.x; hv[c + 1] = e * hv[c + 1] + v.y;
                    hv[c + 2] = e * hv[c + 2] + v.z; hv[c + 3] = e * hv[c + 3] + v.w;
                }
            }
            if (p.final_state && k == p.K - 1 && part == 0) {
                const float e = ex2(cs_span[s1 - s0 - 1]);
                const float* f = p.fin + (span * H + h) * NP + (int64_t)n * kP + c0;
                float* dst = p.final_state + (row * H + h) * NP + (int64_t)n * kP + c0;
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(f + c);
                    *reinterpret_cast<float4*>(dst + c) = make_float4(e * hv[c] + v.x, e * hv[c + 1] + v.y,
                                                                      e * hv[c + 2] + v.z, e * hv[c + 3] + v.w);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
            uint4 v;
            v.x = pack_f16x2(hv[c], hv[c + 1]);
            v.y = pack_f16x2(hv[c + 2], hv[c + 3]);
            v.z = pack_f16x2(hv[c + 4], hv[c + 5]);
            v.w = pack_f16x2(hv[c + 6], hv[c + 7]);
            *reinterpret_cast<uint4*>(s.hs + sw128_off(n, (c0 + c) / 8)) = v;
        }
        fence_proxy_async_smem();
        warp_arrive(&s.hs_ready);
    }

    if (warp == 8) {
        // ------------------------------------------------------------ TMA: C and y tiles
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_c);
            tma_prefetch_desc(&tm_y);
            int issued = 0;
            for (int i = 0; i < nt; ++i) {
                const int st = i % kStagesSO;
                if (i >= kStagesSO && !wait_bar(ctl, &s.stage_free[st], ((i / kStagesSO) - 1) & 1, p.status)) break;
                const int tok = (int)(tok_base + (int64_t)i * kT);
                mbar_expect_tx(&s.full[st], 2 * kBoxBytes + kTileBytesX + kT * sizeof(float));
                tma_load_3d(s.c[st][0], &tm_c, &s.full[st], 0, g, tok);
                tma_load_3d(s.c[st][1], &tm_c, &s.full[st], 64, g, tok);
                tma_load_3d(s.y[st], &tm_y, &s.full[st], 0, h, tok);
                bulk_load(s.cs[st], cs_span + (int64_t)(ft + i) * kT, kT * sizeof(float), &s.full[st]);
                ++issued;
            }
            if (*(volatile int*)&ctl.abort)
                for (int i = 0; i < issued; ++i) mbar_wait(&s.full[i % kStagesSO], (i / kStagesSO) & 1, 400000000ll);
        }
    } else if (warp == 9 || warp == 10) {
        // ----------------------------------------------- MMA: C h_in, even / odd tiles
        const int par0 = warp == 9 ? 0 : 1;
        if (lane == 0 && nt > par0) {
            const uint32_t id = idesc_f16(128, 64, 0, 1);   // K-major A (C rows), MN-major B (state rows)
            const uint32_t hsb = smem_u32(s.hs);
            bool go = wait_bar(ctl, &s.hs_ready, 0, p.status);
            for (int i = par0; go && i < nt; i += 2) {
                const int st = i % kStagesSO;
                if (!wait_bar(ctl, &s.full[st], (i / kStagesSO) & 1, p.status)) break;
                if (i >= kStagesSO && !wait_bar(ctl, &s.acc_free[st], ((i / kStagesSO) - 1) & 1, p.status)) break;
                tc_fence_after();
                const uint32_t cb = smem_u32(s.c[st][0]);
                for (int kk = 0; kk < N / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    mma_ss(tmem + 64 * st, sdesc_sw128(cb + off, 16, 1024), sdesc_sw128(hsb + kk * 2048, kBoxBytes, 1024),
                           id, kk > 0);
                }
                mma_commit(&s.acc_full[st]);
            }
            mma_commit(&s.fin[par0]);
            mbar_wait(&s.fin[par0], 0, 400000000ll);
        }
    } else if (warp == 11) {
        // ------------------------------------------------------------ TMA stores of y tiles
        if (lane == 0 && nt > 0) {
            bool stored = false;
            for (int i = 0; i < nt; ++i) {
                const int st = i % kStagesSO;
                if (!wait_bar(ctl, &s.y_ready[st], (i / kStagesSO) & 1, p.status)) break;
                const int64_t left = s1 - (s0 + (int64_t)(ft + i) * kT);
                if (left >= kT) {
                    tma_store_3d(&tm_y, s.y[st], 0, h, (int)(tok_base + (int64_t)i * kT));
                    bulk_commit();
                    bulk_wait_read0();
                    stored = true;
                }
                mbar_arrive(&s.stage_free[st]);
            }
            if (stored) bulk_wait0();
        }
    }
    if (warp < kEpiWarps) {
        // ---------------------------------------------------------------------- epilogue
        const int quarter = warp & 3, half = warp >> 2;
        const int j = 32 * quarter + lane;                      // token row of the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        for (int i = 0; i < nt; ++i) {
            const int st = i % kStagesSO;
            const int64_t tok = tok_base + (int64_t)i * kT;
            const int64_t left = s1 - (s0 + (int64_t)(ft + i) * kT);
            const int q = left < kT ? (int)left : kT;
            const bool ok = wait_bar_w(ctl, &s.acc_full[st], (i / kStagesSO) & 1, p.status) &&
                            wait_bar_w(ctl, &s.full[st], (i / kStagesSO) & 1, p.status);
            const float f = j < q ? ex2(s.cs[st][j]) : 0.f;
            if (ok) {
                tc_fence_after();
                uint32_t r[32];
                uint32_t (&r0)[16] = *reinterpret_cast<uint32_t (*)[16]>(&r[0]);
                uint32_t (&r1)[16] = *reinterpret_cast<uint32_t (*)[16]>(&r[16]);
                tmem_ld16(tmem + lane_base + 64 * st + 32 * half, r0);
                tmem_ld16(tmem + lane_base + 64 * st + 32 * half + 16, r1);
                tmem_ld_wait();
                tc_fence_before();
                warp_arrive(&s.acc_free[st]);
                // a full tile goes back through shared memory and one TMA store; the rows of a
                // partial tile (a span's end) are written one by one, since the rows past its end
                // belong to the next batch row
                if (j < q) {
                    uint8_t* yrow = s.y[st];
                    __nv_bfloat16* yg = p.y + (tok + j) * H * kP + (int64_t)h * kP + 32 * half;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint4* pv = reinterpret_cast<uint4*>(yrow + sw128_off(j, 4 * half + c));
                        uint4 v = *pv;
                        uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float lo, hi;
                            if (p.y_f16) {
                                const float2 v2 = __half22float2(u2h(w[e]));
                                lo = v2.x;
                                hi = v2.y;
                            } else {
                                lo = bf16lo(w[e]);
                                hi = bf16hi(w[e]);
                            }
                            w[e] = pack_bf16x2(lo + f * __uint_as_float(r[8 * c + 2 * e]),
                                               hi + f * __uint_as_float(r[8 * c + 2 * e + 1]));
                        }
                        if (q == kT)
                            *pv = v;
                        else
                            *reinterpret_cast<uint4*>(yg + 8 * c) = v;
                    }
                }
                fence_proxy_async_smem();
            }
            if (!ok) break;
            warp_arrive(&s.y_ready[st]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, kTmemColsSO);
}

}  // namespace so

// ---- The output of a given entering state (ssd_state_to_output) --------------------------

// bf16 -> fp16 copy of one array (as k_tc_prep).
__global__ void k_to_f16(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n8) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = bf16x8_to_f16x8(src[i]);
}

// Sum of d A log2(e) over each 128-token tile of every row and head: one block per (row, tile),
// one thread per head (consecutive heads are consecutive in dt).
__global__ void k_tile_sums(const __nv_bfloat16* __restrict__ dt, const float* __restrict__ dt_bias,
                            const float* __restrict__ A, int64_t L, int H, int nt, float* __restrict__ tsum) {
    const int64_t row = blockIdx.x / nt;
    const int tile = (int)(blockIdx.x % nt);
    const int64_t t0 = (int64_t)tile * kT;
    const int q = L - t0 < kT ? (int)(L - t0) : kT;
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        const float bias = dt_bias ? dt_bias[h] : 0.f;
        const __nv_bfloat16* d = dt + (row * L + t0) * H + h;
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j < q; ++j) acc += softplus_fast(__bfloat162float(d[(int64_t)j * H]) + bias);
        tsum[(int64_t)blockIdx.x * H + h] = acc * A[h] * 1.4426950408889634f;
    }
}

// Running sums of the tile sums along each row: run[(row H + h) nt + t] = log-decay from the
// row's start through tile t.  One thread per (row, head).
__global__ void k_tile_running(const float* __restrict__ tsum, int64_t bh, int H, int nt, float* __restrict__ run) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= bh) return;
    const int64_t row = i / H;
    const int h = (int)(i % H);
    float r = 0.f;
    for (int t = 0; t < nt; ++t) {
        r += tsum[(row * nt + t) * H + h];
        run[i * nt + t] = r;
    }
}

// Per token: cs[((row H + h) nt + t) 128 + j] = log-decay from the row's start through token
// j of tile t.  One block of 128 threads (one per token) per (row, tile), heads in turn.
__global__ void __launch_bounds__(kT)
k_token_running(const __nv_bfloat16* __restrict__ dt, const float* __restrict__ dt_bias, const float* __restrict__ A,
                const float* __restrict__ run, int64_t L, int H, int nt, float* __restrict__ cs) {
    __shared__ float wsum[kT / 32];
    const int64_t row = blockIdx.x / nt;
    const int tile = (int)(blockIdx.x % nt);
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
    const int64_t t0 = (int64_t)tile * kT;
    const int q = L - t0 < kT ? (int)(L - t0) : kT;
    for (int h = 0; h < H; ++h) {
        float a = j < q ? softplus_fast(__bfloat162float(dt[(row * L + t0 + j) * H + h]) + (dt_bias ? dt_bias[h] : 0.f)) *
                              A[h] * 1.4426950408889634f
                        : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a, o);
            if (lane >= o) a += v;
        }
        if (lane == 31) wsum[warp] = a;
        __syncthreads();
        float before = tile > 0 ? run[(row * H + h) * nt + tile - 1] : 0.f;
        for (int w = 0; w < warp; ++w) before += wsum[w];
        cs[((row * H + h) * nt + tile) * kT + j] = before + a;
        __syncthreads();
    }
}

}  // namespace

bool state_out_supported(const ScanArgs& a) {
    return a.dtype == 1 && a.P == kP && a.N == 128 && a.b * a.L < ((int64_t)1 << 31) && get_encode() != nullptr;
}

size_t state_out_workspace_bytes(const ScanArgs& a) {
    const int64_t nt = (a.L + kT - 1) / kT;
    const size_t c16 = ((size_t)a.b * a.L * a.G * a.N * sizeof(__half) + 255) & ~(size_t)255;
    const size_t tab = ((size_t)a.b * nt * a.H * sizeof(float) + 255) & ~(size_t)255;
    const size_t tok = ((size_t)a.b * nt * kT * a.H * sizeof(float) + 255) & ~(size_t)255;
    return c16 + 2 * tab + tok;
}

int launch_state_to_output(const ScanArgs& a, const float* h_in, void* ws, int32_t* status, cudaStream_t st) {
    const int64_t ntok = a.b * a.L, nt = (a.L + kT - 1) / kT;
    char* w = reinterpret_cast<char*>(ws);
    __half* c16 = reinterpret_cast<__half*>(w);
    w += ((size_t)ntok * a.G * a.N * sizeof(__half) + 255) & ~(size_t)255;
    const size_t tab = ((size_t)a.b * nt * a.H * sizeof(float) + 255) & ~(size_t)255;
    float* tsum = reinterpret_cast<float*>(w);
    float* run = reinterpret_cast<float*>(w + tab);
    float* cs = reinterpret_cast<float*>(w + 2 * tab);
    {
        const int64_t n8 = ntok * a.G * a.N / 8;
        const int64_t blocks = std::min<int64_t>((n8 + 255) / 256, 148 * 16);
        ProfScope ps(K_TC_PREP, st);
        k_to_f16<<<(unsigned)blocks, 256, 0, st>>>((const uint4*)a.C, (uint4*)c16, n8);
    }
    {
        ProfScope ps(K_TILE_DECAY, st);
        const int threads = a.H < 256 ? (int)((a.H + 31) / 32 * 32) : 256;
        k_tile_sums<<<(unsigned)(a.b * nt), threads, 0, st>>>((const __nv_bfloat16*)a.dt, a.dt_bias, a.A, a.L,
                                                              (int)a.H, (int)nt, tsum);
        k_tile_running<<<(unsigned)((a.b * a.H + 127) / 128), 128, 0, st>>>(tsum, a.b * a.H, (int)a.H, (int)nt, run);
        k_token_running<<<(unsigned)(a.b * nt), kT, 0, st>>>((const __nv_bfloat16*)a.dt, a.dt_bias, a.A, run, a.L,
                                                            (int)a.H, (int)nt, cs);
    }
    CUtensorMap tm_c, tm_y;
    if (!make_map(&tm_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c16, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)ntok) ||
        !make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)ntok))
        return 6;  // SSD_ERR_CUDA
    int nparts, tpp;
    plan_parts((int)nt, a.b * a.H, sm_count(), nparts, tpp);
    so::SOParams q;
    q.dt = (const __nv_bfloat16*)a.dt;
    q.dt_bias = a.dt_bias;
    q.A = a.A;
    q.h_in = h_in;
    q.fin = nullptr;
    q.cs = cs;
    q.final_state = nullptr;
    q.y = (__nv_bfloat16*)a.y;
    q.y_f16 = 0;
    q.status = status;
    q.L = a.L;
    q.Ls = a.L;
    q.H = (int)a.H;
    q.G = (int)a.G;
    q.K = 1;
    q.k0 = 0;
    q.row0 = 0;
    q.tiles = (int)nt;
    q.nparts = nparts;
    q.tpp = tpp;
    const size_t smem = sizeof(so::SmemSO) + 1024;
    cudaFuncSetAttribute(so::k_state_out, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    ProfScope ps(K_STATE_OUT, st);
    so::k_state_out<<<(unsigned)(a.b * nparts * a.H), so::kThreadsSO, smem, st>>>(tm_c, tm_y, q);
    return 0;
}

int launch_state_out_split(const ScanArgs& a, const void* c16, const float* fin, const float* cs, int64_t W, int K,
                           int64_t Ls, int tiles, int32_t* status, cudaStream_t st) {
    const int64_t ntok = a.b * a.L;
    CUtensorMap tm_c, tm_y;
    if (!make_map(&tm_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c16, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)ntok) ||
        !make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)ntok))
        return 6;  // SSD_ERR_CUDA
    const int64_t R = a.b - W;
    int nparts, tpp;
    plan_parts(tiles, R * (K - 1) * a.H, sm_count(), nparts, tpp);
    so::SOParams q;
    q.dt = (const __nv_bfloat16*)a.dt;
    q.dt_bias = a.dt_bias;
    q.A = a.A;
    q.h_in = nullptr;
    q.fin = fin;
    q.cs = cs;
    q.final_state = a.final_state;
    q.y = (__nv_bfloat16*)a.y;
    q.y_f16 = 1;
    q.status = status;
    q.L = a.L;
    q.Ls = Ls;
    q.H = (int)a.H;
    q.G = (int)a.G;
    q.K = K;
    q.k0 = 1;
    q.row0 = (int)W;
    q.tiles = tiles;
    q.nparts = nparts;
    q.tpp = tpp;
    const size_t smem = sizeof(so::SmemSO) + 1024;
    cudaFuncSetAttribute(so::k_state_out, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    ProfScope ps(K_STATE_OUT, st);
    so::k_state_out<<<(unsigned)(R * (K - 1) * nparts * a.H), so::kThreadsSO, smem, st>>>(tm_c, tm_y, q);
    return 0;
}

}  // namespace ssd
