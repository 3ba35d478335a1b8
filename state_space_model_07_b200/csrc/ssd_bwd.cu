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
#include <algorithm>
#include <cmath>
#include <cuda_fp16.h>
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

// ---- Chunked backward (P = 64, N = 64 or 128) ---------------------------------------------
//
// The same gradients in the block-decomposed form of section 3.2, a chunk of Qb = 64 tokens at a
// time.  Inside a chunk, with a_i = d_i A (natural log-decay), chunk-local cs_j = sum_{k<=j} a_k,
// e_j = exp(cs_j), E = exp(cs_last), u_i = exp(cs_last - cs_i) d_i, the forward is
//   y_j   = sum_{i<=j} (C_j . B_i) exp(cs_j - cs_i) d_i x_i + e_j C_j^T h_prev + D x_j,
//   h_end = E h_prev + sum_i u_i B_i x_i^T,
// and with dh_end the adjoint of the state leaving the chunk:
//   dh_prev = E dh_end + sum_j e_j C_j dy_j^T                       (reverse state passing)
//   dx = D dy + W^T dy + u o (B dh_end),      W[j,i] = (C_j.B_i) L[j,i] d_i
//   dB = K^T C + u o (x dh_end^T),            K[j,i] = L[j,i] (dy_j.x_i) d_i
//   dC = K B + e o (dy h_prev^T)
// with L[j,i] = exp(cs_j - cs_i) for i <= j, else 0; and for the decays, with
// R[j,i] = (C_j.B_i)(dy_j.x_i) L[j,i], Z_i = B_i^T dh_end x_i, Y_j = C_j^T h_prev dy_j:
//   dJ/dd_i (direct) = sum_j R[j,i] + exp(cs_last - cs_i) Z_i
//   dJ/dcs_k = sum_i R[k,i] d_i - sum_j R[j,k] d_k + e_k Y_k - u_k Z_k
//              (+ E <dh_end, h_prev> + sum_i u_i Z_i at k = last)
//   dJ/da_m = sum_{k>=m} dJ/dcs_k,  dd = direct + A dJ/da,  dA += d dJ/da,  dz = dd sigmoid(z).
// fp32 inputs, three kernels: k_bwd_terms (per chunk and head: the chunk's own state term
// S = sum_i u_i B_i x_i^T and adjoint term T = sum_j e_j C_j dy_j^T, and E), k_bwd_pass (per
// state element: the state entering every chunk, forwards, and the adjoint leaving every chunk,
// backwards), and k_bwd_grads (per chunk and group: every gradient of the chunk's tokens; C B^T
// is shared by the group's heads, and dB, dC are summed over them in registers, so no atomics
// touch them).  bf16 inputs, two: k_bwd_pass_h (the pass with each chunk's term computed on the
// tensor cores as it goes, so the terms never reach HBM) and k_bwd_grads_h.

constexpr int kQb = 64;   // tokens per chunk of the chunked backward
constexpr int kPb = 64;   // headdim of the chunked backward

bool bwd_chunked(const ScanArgs& a) { return a.P == kPb && (a.N == 64 || a.N == 128); }

// Chunk-local decay quantities of tokens 2 lane, 2 lane + 1 of a chunk (one warp): d, z, cs and
// the chunk's last cs; tokens past q get d = 0.
template <typename T>
__device__ __forceinline__ void chunk_decay(const T* dt, int64_t tok0, int H, int h, int q, float bias, float Ah,
                                            float* sd, float* sz, float* scs, float* slast);

// The same from raw dt values already loaded (tokens 2 lane and 2 lane + 1; ignored past q).
__device__ __forceinline__ void chunk_decay_raw(const float (&raw)[2], int q, float bias, float Ah, float* sd,
                                                float* sz, float* scs, float* slast) {
    const int lane = threadIdx.x & 31;
    float dd[2], zz[2], cc[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int j = 2 * lane + k;
        zz[k] = j < q ? raw[k] + bias : 0.f;
        dd[k] = j < q ? softplus_f(zz[k]) : 0.f;
    }
    cc[0] = dd[0] * Ah;
    cc[1] = cc[0] + dd[1] * Ah;
    float incl = cc[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    const float excl = incl - cc[1];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        sd[2 * lane + k] = dd[k];
        sz[2 * lane + k] = zz[k];
        scs[2 * lane + k] = excl + cc[k];
    }
    if (lane == 31) *slast = incl;   // tokens past q add 0, so this is cs of token q - 1
}

// dt of tokens 2 lane and 2 lane + 1 of the chunk (0 past q).
template <typename T>
__device__ __forceinline__ void load_dt2(float (&raw)[2], const T* dt, int64_t tok0, int H, int h, int q) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int j = 2 * lane + k;
        raw[k] = j < q ? to_f<T>(dt[(tok0 + j) * H + h]) : 0.f;
    }
}

template <typename T>
__device__ __forceinline__ void chunk_decay(const T* dt, int64_t tok0, int H, int h, int q, float bias, float Ah,
                                            float* sd, float* sz, float* scs, float* slast) {
    float raw[2];
    load_dt2<T>(raw, dt, tok0, H, h, q);
    chunk_decay_raw(raw, q, bias, Ah, sd, sz, scs, slast);
}

// acc[i][j] += sum_k A(r0 + i, k) Bm(k, c0 + j), A(r, k) = A[r ar + k ak], Bm(k, c) = Bm[k bk + c bc],
// four k at a time with 16-byte shared-memory reads: AI (ar == 1) reads A along i, else along k
// (ak == 1); BJ (bc == 1) reads Bm along j, else along k (bk == 1).  r0, c0, TM, TN, K, the
// non-unit strides and every row start are multiples of 4 floats.
template <int TM, int TN, bool AI, bool BJ>
__device__ __forceinline__ void mm_acc(float (&acc)[TM][TN], const float* A, int ar, int ak, const float* Bm, int bk,
                                       int bc, int r0, int c0, int K) {
#pragma unroll 1
    for (int k = 0; k < K; k += 4) {
        float av[4][TM], bv[4][TN];
        if (AI) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int i = 0; i < TM; i += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(A + r0 + i + (k + kk) * ak);
                    av[kk][i] = v.x; av[kk][i + 1] = v.y; av[kk][i + 2] = v.z; av[kk][i + 3] = v.w;
                }
        } else {
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const float4 v = *reinterpret_cast<const float4*>(A + (r0 + i) * ar + k);
                av[0][i] = v.x; av[1][i] = v.y; av[2][i] = v.z; av[3][i] = v.w;
            }
        }
        if (BJ) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int j = 0; j < TN; j += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(Bm + (k + kk) * bk + c0 + j);
                    bv[kk][j] = v.x; bv[kk][j + 1] = v.y; bv[kk][j + 2] = v.z; bv[kk][j + 3] = v.w;
                }
        } else {
#pragma unroll
            for (int j = 0; j < TN; ++j) {
                const float4 v = *reinterpret_cast<const float4*>(Bm + (c0 + j) * bc + k);
                bv[0][j] = v.x; bv[1][j] = v.y; bv[2][j] = v.z; bv[3][j] = v.w;
            }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[kk][i], bv[kk][j], acc[i][j]);
    }
}

// Warp products on the tensor cores: mma.sync m16n8k16, fp16 operands (rounded from the fp32
// shared-memory values), fp32 accumulators.  A warp computes an (16 MT) x (8 NT) tile at rows
// r0.., columns c0.. of sum_k A(r, k) Bm(k, c), A(r, k) = A[r ar + k ak], Bm(k, c) = Bm[k bk + c bc];
// AK1 / BK1: ak == 1 / bk == 1 (the fragment's pairs of consecutive k are adjacent: one 8-byte
// read).  Fragment layout (PTX ISA, m16n8k16 with .row A and .col B), g = lane / 4, t = lane % 4:
// A regs {(g, 2t..2t+1), (g+8, 2t..), (g, 2t+8..), (g+8, 2t+8..)}; B regs {(2t..2t+1, g),
// (2t+8..2t+9, g)}; accumulator {(g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1)}.
__device__ __forceinline__ uint32_t h2pack(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// The fp16 pair of what the packed pair `hi` (the fp16 roundings of a and b) leaves of a and b.
__device__ __forceinline__ uint32_t h2lo(uint32_t hi, float a, float b) {
    const __half2 h = *reinterpret_cast<const __half2*>(&hi);
    return h2pack(a - __low2float(h), b - __high2float(h));
}

template <bool K1>
__device__ __forceinline__ uint32_t pair_k(const float* M, int64_t at, int kstride) {
    if (K1) {
        const float2 v = *reinterpret_cast<const float2*>(M + at);
        return h2pack(v.x, v.y);
    }
    return h2pack(M[at], M[at + kstride]);
}

template <int MT, int NT, bool AK1, bool BK1>
__device__ __forceinline__ void mma_tile(float (&acc)[MT][NT][4], const float* A, int ar, int ak, const float* Bm,
                                         int bk, int bc, int r0, int c0, int K) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 1
    for (int k = 0; k < K; k += 16) {
        uint32_t af[MT][4], bf[NT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int ra = r0 + 16 * mt + g;
            af[mt][0] = pair_k<AK1>(A, (int64_t)ra * ar + (k + 2 * t) * ak, ak);
            af[mt][1] = pair_k<AK1>(A, (int64_t)(ra + 8) * ar + (k + 2 * t) * ak, ak);
            af[mt][2] = pair_k<AK1>(A, (int64_t)ra * ar + (k + 2 * t + 8) * ak, ak);
            af[mt][3] = pair_k<AK1>(A, (int64_t)(ra + 8) * ar + (k + 2 * t + 8) * ak, ak);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = c0 + 8 * nt + g;
            bf[nt][0] = pair_k<BK1>(Bm, (int64_t)(k + 2 * t) * bk + n * bc, bk);
            bf[nt][1] = pair_k<BK1>(Bm, (int64_t)(k + 2 * t + 8) * bk + n * bc, bk);
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                    "{%8, %9}, {%0, %1, %2, %3};"
                    : "+f"(acc[mt][nt][0]), "+f"(acc[mt][nt][1]), "+f"(acc[mt][nt][2]), "+f"(acc[mt][nt][3])
                    : "r"(af[mt][0]), "r"(af[mt][1]), "r"(af[mt][2]), "r"(af[mt][3]), "r"(bf[nt][0]),
                      "r"(bf[nt][1]));
    }
}

// The same tile in fp32 on the CUDA cores, each thread computing the elements an m16n8k16
// accumulator would hold (fp32 inputs: their accuracy bound leaves no room for fp16 operands).
template <int MT, int NT>
__device__ __forceinline__ void fma_tile(float (&acc)[MT][NT][4], const float* A, int ar, int ak, const float* Bm,
                                         int bk, int bc, int r0, int c0, int K) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k = 0; k < K; ++k) {
        float av[MT][2], bv[NT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            av[mt][0] = A[(int64_t)(r0 + 16 * mt + g) * ar + k * ak];
            av[mt][1] = A[(int64_t)(r0 + 16 * mt + g + 8) * ar + k * ak];
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            bv[nt][0] = Bm[(int64_t)k * bk + (c0 + 8 * nt + 2 * t) * bc];
            bv[nt][1] = Bm[(int64_t)k * bk + (c0 + 8 * nt + 2 * t + 1) * bc];
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[mt][nt][e] = fmaf(av[mt][e >> 1], bv[nt][e & 1], acc[mt][nt][e]);
    }
}

// Tensor cores for bf16 inputs, fp32 CUDA cores for fp32 inputs.
template <typename T, int MT, int NT, bool AK1, bool BK1>
__device__ __forceinline__ void prod(float (&acc)[MT][NT][4], const float* A, int ar, int ak, const float* Bm, int bk,
                                     int bc, int r0, int c0, int K) {
    if constexpr (sizeof(T) == 2)
        mma_tile<MT, NT, AK1, BK1>(acc, A, ar, ak, Bm, bk, bc, r0, c0, K);
    else
        fma_tile<MT, NT>(acc, A, ar, ak, Bm, bk, bc, r0, c0, K);
}

// Row and column of accumulator element e of tile (mt, nt) of a warp tile at (r0, c0).
__device__ __forceinline__ int frag_row(int r0, int mt, int e) { return r0 + 16 * mt + ((threadIdx.x & 31) >> 2) + 8 * (e >> 1); }
__device__ __forceinline__ int frag_col(int c0, int nt, int e) { return c0 + 8 * nt + 2 * (threadIdx.x & 3) + (e & 1); }

// Sums over the lanes of an mma.sync fragment that hold one row (the four lanes of a quad) or one
// column (the same lane of the eight quads); every lane gets the sum.
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v + __shfl_xor_sync(0xffffffffu, v, 2);
}
__device__ __forceinline__ float across_quads_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    return v + __shfl_xor_sync(0xffffffffu, v, 16);
}

template <int MT, int NT>
__device__ __forceinline__ void zero_frag(float (&acc)[MT][NT][4]) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
}

template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN]) {
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

struct ChunkedBwd {
    SeqInfo si;                        // 64-token chunks
    const void *x, *dt, *B, *C, *dy;
    const float *dt_bias, *A, *D, *init_state, *dfinal;
    void *dx, *ddt, *dB, *dC;
    float *ddt_bias, *dA, *dD, *dinit;
    float *S, *T, *E;                  // (chunks, H, N P), (chunks, H, N P), (chunks, H)
    int H, N, G;
    // k_bwd_grads_h only: the heads of a group split over hsplit blocks per chunk; each part's
    // dB, dC go to fp32 partials (part p at dBp + p part_stride, laid out as dB), summed after
    int hsplit = 1;
    float *dBp = nullptr, *dCp = nullptr;
    int64_t part_stride = 0;
};

// Loads rows [0, q) of a (tokens, stride) slab of T into shared fp32 (rows, cols) with row
// stride ld, zero past q.
template <typename T>
__device__ __forceinline__ void load_rows(float* dst, const T* src, int64_t stride, int q, int rows, int cols,
                                          int ld) {
    for (int e = threadIdx.x; e < rows * cols; e += blockDim.x) {
        const int r = e / cols, c = e % cols;
        dst[r * ld + c] = r < q ? to_f<T>(src[(int64_t)r * stride + c]) : 0.f;
    }
}

// ---- k_bwd_terms: S = sum_i u_i B_i x_i^T, T = sum_j e_j C_j dy_j^T (N x 64 each), E = exp(cs_last)
template <typename T, int N>
__global__ void __launch_bounds__(256) k_bwd_terms(const ChunkedBwd p) {
    constexpr int P = kPb;
    extern __shared__ float smf[];
    float* sB = smf;                    // kQb x N
    float* sX = sB + kQb * N;           // kQb x P
    __shared__ float sd[kQb], sz[kQb], scs[kQb], slast;
    const int H = p.H, G = p.G;
    const int64_t f = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H), g = h / (H / G);
    ChunkRef r;
    if (!chunk_ref(p.si, f, r)) return;
    const int q = (int)(r.t1 - r.t0);
    const int64_t tok0 = r.row * p.si.L + r.t0;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f, Ah = p.A[h];
    if (threadIdx.x < 32) chunk_decay<T>((const T*)p.dt, tok0, H, h, q, bias, Ah, sd, sz, scs, &slast);
    __syncthreads();
    // warp tiles of the N x 64 result: (16 MT) x 32
    constexpr int MT = N / 64;
    const int warp = threadIdx.x >> 5;
    const int n0 = 16 * MT * (warp >> 1), c0 = 32 * (warp & 1);
    for (int pass = 0; pass < 2; ++pass) {
        // pass 0: B with u and x -> S; pass 1: C with e and dy -> T
        const T* mat = (const T*)(pass == 0 ? p.B : p.C) + (tok0 * G + g) * N;
        const T* vec = (const T*)(pass == 0 ? p.x : p.dy) + (tok0 * H + h) * P;
        load_rows<T>(sB, mat, (int64_t)G * N, q, kQb, N, N);
        for (int e = threadIdx.x; e < kQb * P; e += blockDim.x) {
            const int j = e / P, c = e % P;
            float w = 0.f;
            if (j < q) w = pass == 0 ? expf(slast - scs[j]) * sd[j] : expf(scs[j]);
            sX[e] = j < q ? w * to_f<T>(vec[(int64_t)j * H * P + c]) : 0.f;
        }
        __syncthreads();
        float acc[MT][4][4];
        zero_frag(acc);
        prod<T, MT, 4, false, false>(acc, sB, 1, N, sX, P, 1, n0, c0, kQb);
        float* out = (pass == 0 ? p.S : p.T) + ((int64_t)f * H + h) * N * P;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; e += 2)
                    *reinterpret_cast<float2*>(out + (int64_t)frag_row(n0, mt, e) * P + frag_col(c0, nt, e)) =
                        make_float2(acc[mt][nt][e], acc[mt][nt][e + 1]);
        __syncthreads();
    }
    if (threadIdx.x == 0) p.E[f * H + h] = expf(slast);
}

// ---- k_bwd_pass: per (sequence, head), the state entering every chunk (overwriting S) and the
// adjoint of the state leaving every chunk (overwriting T), and dinit.  One 256-thread block per
// (sequence, head) holds the N x 64 state in registers, kVec float4 per thread, and walks the
// chunks with the next two chunks' terms in flight (every chunk is one contiguous N P slab).
constexpr int kPassThreads = 256;

__device__ __forceinline__ float4 fma4(float e, float4 a, float4 b) {
    return make_float4(fmaf(e, a.x, b.x), fmaf(e, a.y, b.y), fmaf(e, a.z, b.z), fmaf(e, a.w, b.w));
}

// h (in registers) runs through nc chunks whose slabs (N P floats, indexed chunk H + head, as E)
// are first, first + dir, ...; every slab is replaced by the value entering its chunk, and h
// becomes E h + (the slab's term).
template <int kVec>
__device__ __forceinline__ void chain_block(float4* M, const float* E, int64_t first, int64_t dir, int nc,
                                            float4 (&hv)[kVec]) {
    constexpr int64_t slab4 = (int64_t)kVec * kPassThreads;
    const int tid = threadIdx.x;
    auto at = [&](int c) { return M + (first + dir * c) * slab4 + tid; };
    float4 m0[kVec], m1[kVec];
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
        if (nc > 0) m0[k] = at(0)[kPassThreads * k];
        if (nc > 1) m1[k] = at(1)[kPassThreads * k];
    }
    for (int c = 0; c < nc; c += 2) {
        {
            const float e = E[first + dir * c];
            float4* dst = at(c);
#pragma unroll
            for (int k = 0; k < kVec; ++k) {
                const float4 mv = m0[k];
                if (c + 2 < nc) m0[k] = at(c + 2)[kPassThreads * k];
                dst[kPassThreads * k] = hv[k];
                hv[k] = fma4(e, hv[k], mv);
            }
        }
        if (c + 1 < nc) {
            const float e = E[first + dir * (c + 1)];
            float4* dst = at(c + 1);
#pragma unroll
            for (int k = 0; k < kVec; ++k) {
                const float4 mv = m1[k];
                if (c + 3 < nc) m1[k] = at(c + 3)[kPassThreads * k];
                dst[kPassThreads * k] = hv[k];
                hv[k] = fma4(e, hv[k], mv);
            }
        }
    }
}

template <int kVec>
__global__ void __launch_bounds__(kPassThreads) k_bwd_pass(float* __restrict__ S, float* __restrict__ Tm,
                                                             const float* __restrict__ E,
                                                             const float* __restrict__ init,
                                                             const float* __restrict__ dfinal,
                                                             float* __restrict__ dinit, SeqInfo si, int H) {
    constexpr int64_t slab4 = (int64_t)kVec * kPassThreads;   // N P / 4
    const int64_t sh = blockIdx.x;
    const int s = (int)(sh / H), h = (int)(sh % H);
    const int nc = seq_nchunks(si, s);
    const int64_t c0 = seq_chunk0(si, s);
    const int tid = threadIdx.x;
    float4 hv[kVec];
    const float4* i4 = init ? reinterpret_cast<const float4*>(init) + sh * slab4 + tid : nullptr;
#pragma unroll
    for (int k = 0; k < kVec; ++k) hv[k] = i4 ? i4[kPassThreads * k] : make_float4(0.f, 0.f, 0.f, 0.f);
    chain_block<kVec>(reinterpret_cast<float4*>(S), E, c0 * H + h, H, nc, hv);                    // forwards
    const float4* d4 = dfinal ? reinterpret_cast<const float4*>(dfinal) + sh * slab4 + tid : nullptr;
#pragma unroll
    for (int k = 0; k < kVec; ++k) hv[k] = d4 ? d4[kPassThreads * k] : make_float4(0.f, 0.f, 0.f, 0.f);
    chain_block<kVec>(reinterpret_cast<float4*>(Tm), E, (c0 + nc - 1) * H + h, -(int64_t)H, nc, hv);  // backwards
    if (dinit) {
        float4* o4 = reinterpret_cast<float4*>(dinit) + sh * slab4 + tid;
#pragma unroll
        for (int k = 0; k < kVec; ++k) o4[kPassThreads * k] = hv[k];
    }
}

// ---- k_bwd_grads: every gradient of one chunk's tokens for one group (its heads in turn)
template <typename T, int N>
__global__ void __launch_bounds__(256, 1) k_bwd_grads(const ChunkedBwd p) {
    constexpr int P = kPb, Q = kQb;
    // warp tiles: 64 x 64 products 16 x 32 per warp; 64 x N products (16 MTN) x 32
    constexpr int WC = N / 32, MTN = WC / 2;
    // rows of the matrices read along a row by the threads of different rows (B, C, x, dy and
    // the two states) padded by 4 floats, so that those reads spread over the banks
    constexpr int LN = N + 4, LP = P + 4, LQ = Q;
    extern __shared__ float smf[];
    float* sB = smf;                  // Q x N (row stride LN)
    float* sC = sB + Q * LN;          // Q x N
    float* sCB = sC + Q * LN;         // Q x Q, C_j . B_i at [j LQ + i]
    float* sX = sCB + Q * LQ;         // Q x P (row stride LP)
    float* sDY = sX + Q * LP;         // Q x P
    float* sHP = sDY + Q * LP;        // N x P, state entering the chunk
    float* sDH = sHP + N * LP;        // N x P, adjoint of the state leaving it
    float* sW = sDH + N * LP;         // Q x Q
    float* sK = sW + Q * LQ;          // Q x Q
    float* sd = sK + Q * LQ;          // Q each below
    float* sz = sd + Q;
    float* scs = sz + Q;
    float* se = scs + Q;
    float* su = se + Q;
    float* colR = su + Q;
    float* rowRd = colR + Q;
    float* rowZ = rowRd + Q;
    float* rowY = rowZ + Q;
    float* sred = rowY + Q;           // [0] <dh_end, h_prev>, [1] sum dy x, [2] last cs
    const int H = p.H, G = p.G, HG = H / G;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t f = blockIdx.x / G;
    const int g = (int)(blockIdx.x % G);
    ChunkRef r;
    if (!chunk_ref(p.si, f, r)) return;
    const int q = (int)(r.t1 - r.t0);
    const int64_t tok0 = r.row * p.si.L + r.t0;
    const T* dtg = (const T*)p.dt;
    load_rows<T>(sB, (const T*)p.B + (tok0 * G + g) * N, (int64_t)G * N, q, Q, N, LN);
    load_rows<T>(sC, (const T*)p.C + (tok0 * G + g) * N, (int64_t)G * N, q, Q, N, LN);
    __syncthreads();
    const int warp = tid >> 5;
    const int r64 = 16 * (warp >> 1), c64 = 32 * (warp & 1);        // 64 x 64 warp tiles
    const int rN = 16 * MTN * (warp / WC), cN = 32 * (warp % WC);   // 64 x N warp tiles
    {
        float acc[1][4][4];
        zero_frag(acc);
        prod<T, 1, 4, true, true>(acc, sC, LN, 1, sB, 1, LN, r64, c64, N);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sCB[frag_row(r64, 0, e) * LQ + frag_col(c64, nt, e)] = acc[0][nt][e];
    }
    float dBa[MTN][4][4], dCa[MTN][4][4];
    zero_frag(dBa);
    zero_frag(dCa);
    for (int hh = 0; hh < HG; ++hh) {
        const int h = g * HG + hh;
        const float bias = p.dt_bias ? p.dt_bias[h] : 0.f, Ah = p.A[h], Dh = p.D ? p.D[h] : 0.f;
        load_rows<T>(sX, (const T*)p.x + (tok0 * H + h) * P, (int64_t)H * P, q, Q, P, LP);
        load_rows<T>(sDY, (const T*)p.dy + (tok0 * H + h) * P, (int64_t)H * P, q, Q, P, LP);
        {
            const float4* hp = reinterpret_cast<const float4*>(p.S + ((int64_t)f * H + h) * N * P);
            const float4* dh = reinterpret_cast<const float4*>(p.T + ((int64_t)f * H + h) * N * P);
            for (int e = tid; e < N * P / 4; e += blockDim.x) {
                const int n = e / (P / 4), c = 4 * (e % (P / 4));
                *reinterpret_cast<float4*>(sHP + n * LP + c) = hp[e];
                *reinterpret_cast<float4*>(sDH + n * LP + c) = dh[e];
            }
        }
        if (tid < Q) {
            colR[tid] = 0.f; rowRd[tid] = 0.f; rowZ[tid] = 0.f; rowY[tid] = 0.f;
        }
        if (tid < 2) sred[tid] = 0.f;      // sred[2] is written by the decay scan below
        if (tid < 32) {
            chunk_decay<T>(dtg, tok0, H, h, q, bias, Ah, sd, sz, scs, &sred[2]);
            __syncwarp();
            const float last = sred[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int j = 2 * lane + k;
                se[j] = j < q ? expf(scs[j]) : 0.f;
                su[j] = j < q ? expf(last - scs[j]) * sd[j] : 0.f;
            }
        }
        __syncthreads();
        {
            float a1 = 0.f, a2 = 0.f;
            for (int e = tid; e < N * P; e += blockDim.x) a1 += sHP[(e / P) * LP + e % P] * sDH[(e / P) * LP + e % P];
            for (int e = tid; e < Q * P; e += blockDim.x) a2 += sDY[(e / P) * LP + e % P] * sX[(e / P) * LP + e % P];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a1 += __shfl_xor_sync(0xffffffffu, a1, o);
                a2 += __shfl_xor_sync(0xffffffffu, a2, o);
            }
            if (lane == 0) {
                atomicAdd(&sred[0], a1);
                atomicAdd(&sred[1], a2);
            }
        }
        // (1) dy_j . x_i, the masked forms W, K and the sums of R
        {
            float acc[1][4][4];
            zero_frag(acc);
            prod<T, 1, 4, true, true>(acc, sDY, LP, 1, sX, 1, LP, r64, c64, P);
            float rrow[2] = {0.f, 0.f}, rcol[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = frag_row(r64, 0, e), i = frag_col(c64, nt, e);
                    const float L = (i <= j && j < q) ? expf(scs[j] - scs[i]) : 0.f;
                    const float cb = sCB[j * LQ + i], di = sd[i], dyx = acc[0][nt][e];
                    sW[j * LQ + i] = cb * L * di;
                    sK[j * LQ + i] = L * dyx * di;
                    const float R = cb * dyx * L;
                    rrow[e >> 1] += R * di;
                    rcol[nt][e & 1] += R;
                }
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float v = quad_sum(rrow[a]);
                if ((threadIdx.x & 3) == 0) atomicAdd(&rowRd[frag_row(r64, 0, 2 * a)], v);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const float v = across_quads_sum(rcol[nt][b]);
                    if ((threadIdx.x & 31) < 4) atomicAdd(&colR[frag_col(c64, nt, b)], v);
                }
        }
        __syncthreads();
        // (2) dx = D dy + W^T dy + u o (B dh_end), and Z_i = B_i^T dh_end x_i
        {
            float bd[1][4][4], wd[1][4][4];
            zero_frag(bd);
            zero_frag(wd);
            prod<T, 1, 4, true, false>(bd, sB, LN, 1, sDH, LP, 1, r64, c64, N);
            prod<T, 1, 4, false, false>(wd, sW, 1, LQ, sDY, LP, 1, r64, c64, Q);
            T* dxg = (T*)p.dx + (tok0 * H + h) * P;
            float z[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = frag_row(r64, 0, e), c = frag_col(c64, nt, e);
                    z[e >> 1] += bd[0][nt][e] * sX[i * LP + c];
                    if (i < q)
                        dxg[(int64_t)i * H * P + c] = from_f<T>(Dh * sDY[i * LP + c] + wd[0][nt][e] + su[i] * bd[0][nt][e]);
                }
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float v = quad_sum(z[a]);
                if ((threadIdx.x & 3) == 0) atomicAdd(&rowZ[frag_row(r64, 0, 2 * a)], v);
            }
        }
        // (3) Y_j = C_j^T h_prev dy_j
        {
            float ch[1][4][4];
            zero_frag(ch);
            prod<T, 1, 4, true, false>(ch, sC, LN, 1, sHP, LP, 1, r64, c64, N);
            float y[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    y[e >> 1] += ch[0][nt][e] * sDY[frag_row(r64, 0, e) * LP + frag_col(c64, nt, e)];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float v = quad_sum(y[a]);
                if ((threadIdx.x & 3) == 0) atomicAdd(&rowY[frag_row(r64, 0, 2 * a)], v);
            }
        }
        // (4) dB += K^T C + u o (x dh_end^T),  dC += K B + e o (dy h_prev^T)
        {
            float t[MTN][4][4];
            prod<T, MTN, 4, false, false>(dBa, sK, 1, LQ, sC, LN, 1, rN, cN, Q);
            zero_frag(t);
            prod<T, MTN, 4, true, true>(t, sX, LP, 1, sDH, 1, LP, rN, cN, P);
#pragma unroll
            for (int mt = 0; mt < MTN; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dBa[mt][nt][e] += su[frag_row(rN, mt, e)] * t[mt][nt][e];
            prod<T, MTN, 4, true, false>(dCa, sK, LQ, 1, sB, LN, 1, rN, cN, Q);
            zero_frag(t);
            prod<T, MTN, 4, true, true>(t, sDY, LP, 1, sHP, 1, LP, rN, cN, P);
#pragma unroll
            for (int mt = 0; mt < MTN; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dCa[mt][nt][e] += se[frag_row(rN, mt, e)] * t[mt][nt][e];
        }
        __syncthreads();
        // (5) the decays, on warp 0: tokens 2 lane, 2 lane + 1
        if (tid < 32) {
            const float last = sred[2], E = expf(last);
            float ddir[2], dcs[2], uz = 0.f;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int j = 2 * lane + k;
                const bool in = j < q;
                const float Z = rowZ[j];
                ddir[k] = in ? colR[j] + expf(last - scs[j]) * Z : 0.f;
                dcs[k] = in ? rowRd[j] - sd[j] * colR[j] + se[j] * rowY[j] - su[j] * Z : 0.f;
                uz += in ? su[j] * Z : 0.f;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) uz += __shfl_xor_sync(0xffffffffu, uz, o);
#pragma unroll
            for (int k = 0; k < 2; ++k)
                if (2 * lane + k == q - 1) dcs[k] += E * sred[0] + uz;
            // dJ/da_m = sum_{k >= m} dJ/dcs_k: suffix sums over the lanes
            const float pair = dcs[0] + dcs[1];
            float suf = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += t;
            }
            const float above = suf - pair;
            const float da[2] = {above + pair, above + dcs[1]};
            float sdA = 0.f, sbias = 0.f;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int j = 2 * lane + k;
                if (j < q) {
                    const float dd = ddir[k] + Ah * da[k];
                    const float z = sz[j];
                    const float sg = z >= 0.f ? 1.f / (1.f + expf(-z)) : expf(z) / (1.f + expf(z));
                    const float dz = dd * sg;
                    ((T*)p.ddt)[(tok0 + j) * H + h] = from_f<T>(dz);
                    sdA += sd[j] * da[k];
                    sbias += dz;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sdA += __shfl_xor_sync(0xffffffffu, sdA, o);
                sbias += __shfl_xor_sync(0xffffffffu, sbias, o);
            }
            if (lane == 0) {
                atomicAdd(&p.dA[h], sdA);
                atomicAdd(&p.ddt_bias[h], sbias);
                atomicAdd(&p.dD[h], sred[1]);
            }
        }
        __syncthreads();
    }
    T* dBg = (T*)p.dB + (tok0 * G + g) * N;
    T* dCg = (T*)p.dC + (tok0 * G + g) * N;
#pragma unroll
    for (int mt = 0; mt < MTN; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = frag_row(rN, mt, e), n = frag_col(cN, nt, e);
                if (i < q) {
                    dBg[(int64_t)i * G * N + n] = from_f<T>(dBa[mt][nt][e]);
                    dCg[(int64_t)i * G * N + n] = from_f<T>(dCa[mt][nt][e]);
                }
            }
}


// 8 packed bf16 -> 8 packed fp16 (exact for values in fp16's normal range).
__device__ __forceinline__ uint4 bf16x8_to_f16x8_bwd(uint4 v) {
    auto cv = [](uint32_t w) { return h2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); };
    return make_uint4(cv(v.x), cv(v.y), cv(v.z), cv(v.w));
}

// ---- k_bwd_grads_h: k_bwd_grads for bf16 inputs with fp16 operand tiles in shared memory ----
//
// The tensor-core operands are fp16 either way; holding them as fp16 halves the shared memory and
// lets the MMA fragments be read as packed pairs.  Every tile is row-major [rows][W] fp16 with its
// 4-byte words XOR-swizzled by row (word w of row r at w ^ 4 (r mod 8)): the eight rows and four
// word offsets a fragment read touches then fall in 32 different banks, for reads along a row
// (a pair of consecutive k in one word) and across rows (a pair in two rows) alike.
__device__ __forceinline__ int hsw(int r, int c, int W) {
    return r * W + ((((c >> 1) ^ ((r & 7) << 2))) << 1) + (c & 1);
}

// 16 bytes (8 fp16) for columns 8 c8 .. 8 c8 + 7 of row r.
__device__ __forceinline__ __half* hsw8(__half* M, int r, int c8, int W) { return M + r * W + 8 * (c8 ^ (r & 7)); }

// ldmatrix: four 8 x 8 fp16 matrices whose rows (16 bytes each) lanes 8 m .. 8 m + 7 address;
// .trans delivers each transposed.  With the swizzle above a 16-byte row chunk stays contiguous
// and eight consecutive rows of one chunk fall in eight different bank groups.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const __half* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const __half* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}

// mma_tile for fp16 tiles: A(r, k) = A[r][k] (AROWK) or A[k][r]; Bm(k, n) = Bm[n][k] (BROWK) or
// Bm[k][n]; fragments by ldmatrix (NT even).  Lane l addresses row l % 8 of matrix l / 8: for A
// the matrices are (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
// -- the m16n8k16 A registers in order; for B, (k 0-7) and (k 8-15) of columns n .. n + 7, then
// of n + 8 .. n + 15 -- the B registers of two adjacent 8-column tiles.
template <int MT, int NT, bool AROWK, bool BROWK, int kUnroll = 4>
__device__ __forceinline__ void mma_tile_h(float (&acc)[MT][NT][4], const __half* A, int WA, const __half* Bm, int WB,
                                           int r0, int c0, int K) {
    static_assert(NT % 2 == 0, "B fragments come two tiles at a time");
    const int lane = threadIdx.x & 31, m = lane >> 3, rr = lane & 7;
#pragma unroll kUnroll
    for (int k = 0; k < K; k += 16) {
        uint32_t af[MT][4], bf[NT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r = r0 + 16 * mt;
            if (AROWK)
                ldsm_x4(af[mt], hsw8(const_cast<__half*>(A), r + rr + 8 * (m & 1), (k >> 3) + (m >> 1), WA));
            else
                ldsm_x4_t(af[mt], hsw8(const_cast<__half*>(A), k + rr + 8 * (m >> 1), (r >> 3) + (m & 1), WA));
        }
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            const int n = c0 + 8 * nt;
            uint32_t t4[4];
            if (BROWK)
                ldsm_x4(t4, hsw8(const_cast<__half*>(Bm), n + rr + 8 * (m >> 1), (k >> 3) + (m & 1), WB));
            else
                ldsm_x4_t(t4, hsw8(const_cast<__half*>(Bm), k + rr + 8 * (m & 1), (n >> 3) + (m >> 1), WB));
            bf[nt][0] = t4[0];
            bf[nt][1] = t4[1];
            bf[nt + 1][0] = t4[2];
            bf[nt + 1][1] = t4[3];
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                    "{%8, %9}, {%0, %1, %2, %3};"
                    : "+f"(acc[mt][nt][0]), "+f"(acc[mt][nt][1]), "+f"(acc[mt][nt][2]), "+f"(acc[mt][nt][3])
                    : "r"(af[mt][0]), "r"(af[mt][1]), "r"(af[mt][2]), "r"(af[mt][3]), "r"(bf[nt][0]),
                      "r"(bf[nt][1]));
    }
}

// acc += A Bm + A2 Bm (kSecondA) or A Bm + A Bm2: the two products of an operand split into an fp16
// pair hi + lo, with the shared operand's fragments read once per k step.  Layouts as in mma_tile_h.
template <int MT, int NT, bool AROWK, bool BROWK, bool kSecondA>
__device__ __forceinline__ void mma_tile_h_pair(float (&acc)[MT][NT][4], const __half* A, const __half* A2, int WA,
                                                const __half* Bm, const __half* Bm2, int WB, int r0, int c0, int K) {
    static_assert(NT % 2 == 0, "B fragments come two tiles at a time");
    const int lane = threadIdx.x & 31, m = lane >> 3, rr = lane & 7;
    auto load_a = [&](uint32_t (&af)[MT][4], const __half* M, int k) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r = r0 + 16 * mt;
            if (AROWK)
                ldsm_x4(af[mt], hsw8(const_cast<__half*>(M), r + rr + 8 * (m & 1), (k >> 3) + (m >> 1), WA));
            else
                ldsm_x4_t(af[mt], hsw8(const_cast<__half*>(M), k + rr + 8 * (m >> 1), (r >> 3) + (m & 1), WA));
        }
    };
    auto load_b = [&](uint32_t (&bf)[NT][2], const __half* M, int k) {
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            const int n = c0 + 8 * nt;
            uint32_t t4[4];
            if (BROWK)
                ldsm_x4(t4, hsw8(const_cast<__half*>(M), n + rr + 8 * (m >> 1), (k >> 3) + (m & 1), WB));
            else
                ldsm_x4_t(t4, hsw8(const_cast<__half*>(M), k + rr + 8 * (m & 1), (n >> 3) + (m >> 1), WB));
            bf[nt][0] = t4[0];
            bf[nt][1] = t4[1];
            bf[nt + 1][0] = t4[2];
            bf[nt + 1][1] = t4[3];
        }
    };
    auto mma = [&](const uint32_t (&af)[MT][4], const uint32_t (&bf)[NT][2]) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                    "{%8, %9}, {%0, %1, %2, %3};"
                    : "+f"(acc[mt][nt][0]), "+f"(acc[mt][nt][1]), "+f"(acc[mt][nt][2]), "+f"(acc[mt][nt][3])
                    : "r"(af[mt][0]), "r"(af[mt][1]), "r"(af[mt][2]), "r"(af[mt][3]), "r"(bf[nt][0]),
                      "r"(bf[nt][1]));
    };
#pragma unroll 2
    for (int k = 0; k < K; k += 16) {
        uint32_t af[MT][4], bf[NT][2];
        load_a(af, A, k);
        load_b(bf, Bm, k);
        mma(af, bf);
        if (kSecondA) {
            load_a(af, A2, k);
            mma(af, bf);
        } else {
            load_b(bf, Bm2, k);
            mma(af, bf);
        }
    }
}

// Rows [0, q) of a bf16 (tokens, stride) slab -> fp16 tile [rows][W] (swizzled), zero past q.
__device__ __forceinline__ void load_rows_h(__half* dst, const __nv_bfloat16* src, int64_t stride, int q, int rows,
                                            int W) {
    const int c8n = W / 8;
    for (int e = threadIdx.x; e < rows * c8n; e += blockDim.x) {
        const int r = e / c8n, c8 = e % c8n;
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (r < q) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + (int64_t)r * stride + 8 * c8);
            o = bf16x8_to_f16x8_bwd(v);
        }
        *reinterpret_cast<uint4*>(hsw8(dst, r, c8, W)) = o;
    }
}

// 16-byte asynchronous copy global -> shared (cached at L2 only), and the wait for all of this
// thread's copies committed so far.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(a), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Layout of k_bwd_grads_h's dynamic shared memory: the fp16 tiles, the fp32 C B^T and per-token
// arrays, then (16-byte aligned) the staging area of the next head's inputs.  C B^T rows are
// kCBW = Q + 8 floats apart: a fragment's eight rows then start 8 banks apart, so its float2
// reads (four lanes per row) take the two wavefronts 256 bytes need instead of eight.
constexpr int kCBW = kQb + 8;
template <int N>
constexpr size_t grads_h_stage_offset() {
    return (2 * (2 * kQb * N + 2 * kQb * kPb + 3 * N * kPb + 3 * kQb * kQb) + sizeof(float) * (kQb * kCBW + 9 * kQb + 4) +
            15) & ~(size_t)15;
}

template <int N>
constexpr size_t grads_h_smem() {
    return grads_h_stage_offset<N>() + 2 * 2 * kQb * kPb + 2 * sizeof(float) * N * kPb;
}

// 512 threads (16 warps) per block: the 64 x 64 products in 16 x 16 warp tiles, the 64 x N
// products in 16 x (N / 4) warp tiles.
constexpr int kGradThreads = 512;

template <int N>
__global__ void __launch_bounds__(kGradThreads, 1) k_bwd_grads_h(const ChunkedBwd p) {
    using T = __nv_bfloat16;
    constexpr int P = kPb, Q = kQb;
    constexpr int NTN = N / 32;   // 8-column MMA tiles per warp in the 64 x N products
    extern __shared__ __align__(16) uint8_t smraw[];
    __half* sB = reinterpret_cast<__half*>(smraw);   // [Q][N]
    __half* sC = sB + Q * N;                         // [Q][N]
    __half* sX = sC + Q * N;                         // [Q][P]
    __half* sDY = sX + Q * P;                        // [Q][P]
    __half* sHP = sDY + Q * P;                       // [N][P] state entering the chunk
    __half* sDH = sHP + N * P;                       // [N][P] adjoint of the state leaving it
    __half* sW = sDH + N * P;                        // [Q][Q]
    __half* sK = sW + Q * Q;                         // [Q][Q] K summed over the heads (hi), at the end
    // dx = D dy + W^T dy + u o (B dh_end): its last two terms can each be many times dx itself
    // and cancel, so W and dh_end enter those products as fp16 pairs hi + lo (lo = the fp16
    // rounding of what hi leaves), which makes them exact to about 2^-22
    __half* sDHl = sK + Q * Q;                       // [N][P]
    __half* sWl = sDHl + N * P;                      // [Q][Q]
    float* sCB = reinterpret_cast<float*>(sWl + Q * Q);   // [Q][kCBW] C_j . B_i in fp32 (it enters the decays)
    float* sd = sCB + Q * kCBW;
    float* sz = sd + Q;
    float* scs = sz + Q;
    float* se = scs + Q;
    float* su = se + Q;
    float* colR = su + Q;
    float* rowRd = colR + Q;
    float* rowZ = rowRd + Q;
    float* rowY = rowZ + Q;
    float* sred = rowY + Q;           // [0] <dh_end, h_prev>, [1] sum dy x, [2] last cs
    // staging for the next head's inputs, filled by asynchronous copies while this head computes:
    // x and dy as they are in memory (bf16 rows), the two fp32 states
    uint8_t* stg = smraw + grads_h_stage_offset<N>();
    T* stX = reinterpret_cast<T*>(stg);
    T* stDY = stX + Q * P;
    float* stHP = reinterpret_cast<float*>(stDY + Q * P);
    float* stDH = stHP + N * P;
    const int H = p.H, G = p.G, HG = H / G;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t f = blockIdx.x / ((int64_t)G * p.hsplit);
    const int g = (int)((blockIdx.x / p.hsplit) % G), part = (int)(blockIdx.x % p.hsplit);
    // this block's heads of group g: hh0 .. hh1 - 1
    const int hh0 = part * (HG / p.hsplit), hh1 = hh0 + HG / p.hsplit;
    ChunkRef r;
    if (!chunk_ref(p.si, f, r)) return;
    const int q = (int)(r.t1 - r.t0);
    const int64_t tok0 = r.row * p.si.L + r.t0;
    const T* dtg = (const T*)p.dt;
    // copies of head hh's x, dy rows (those inside the chunk) and states into the staging area
    auto stage = [&](int hh) {
        const int h = g * HG + hh;
        const T* xs = (const T*)p.x + (tok0 * H + h) * P;
        const T* dys = (const T*)p.dy + (tok0 * H + h) * P;
        for (int e = tid; e < Q * P / 8; e += blockDim.x) {
            const int r = e / (P / 8), c8 = e % (P / 8);
            if (r < q) {
                cp_async16(stX + r * P + 8 * c8, xs + (int64_t)r * H * P + 8 * c8);
                cp_async16(stDY + r * P + 8 * c8, dys + (int64_t)r * H * P + 8 * c8);
            }
        }
        const float* hp = p.S + ((int64_t)f * H + h) * N * P;
        const float* dh = p.T + ((int64_t)f * H + h) * N * P;
        for (int e = tid; e < N * P / 4; e += blockDim.x) {
            cp_async16(stHP + 4 * e, hp + 4 * e);
            cp_async16(stDH + 4 * e, dh + 4 * e);
        }
        cp_async_commit();
    };
    stage(hh0);
    // warp 0 holds the raw dt of the head it prepares next (loaded a head ahead)
    float dt_raw[2] = {0.f, 0.f};
    if (tid < 32) load_dt2<T>(dt_raw, dtg, tok0, H, g * HG + hh0, q);
    load_rows_h(sB, (const T*)p.B + (tok0 * G + g) * N, (int64_t)G * N, q, Q, N);
    load_rows_h(sC, (const T*)p.C + (tok0 * G + g) * N, (int64_t)G * N, q, Q, N);
    __syncthreads();
    const int warp = tid >> 5;
    const int r64 = 16 * (warp >> 2), c64 = 16 * (warp & 3);
    const int rN = 16 * (warp >> 2), cN = (N / 4) * (warp & 3);
    {
        float acc[1][2][4];
        zero_frag(acc);
        mma_tile_h<1, 2, true, true>(acc, sC, N, sB, N, r64, c64, N);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                sCB[frag_row(r64, 0, e) * kCBW + frag_col(c64, nt, e)] = acc[0][nt][e];
    }
    // (5) the decays of head hh, on warp 0 (tokens 2 lane, 2 lane + 1): they read only the per-token
    // arrays and sums of that head, so warp 0 runs them while the other warps convert the next
    // head's operands
    auto decays = [&](int hh) {
        const int h = g * HG + hh;
        const float Ah = p.A[h];
        const float last = sred[2], E = expf(last);
        float ddir[2], dcs[2], uz = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = 2 * lane + k;
            const bool in = j < q;
            const float Z = rowZ[j];
            ddir[k] = in ? colR[j] + expf(last - scs[j]) * Z : 0.f;
            dcs[k] = in ? rowRd[j] - sd[j] * colR[j] + se[j] * rowY[j] - su[j] * Z : 0.f;
            uz += in ? su[j] * Z : 0.f;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) uz += __shfl_xor_sync(0xffffffffu, uz, o);
#pragma unroll
        for (int k = 0; k < 2; ++k)
            if (2 * lane + k == q - 1) dcs[k] += E * sred[0] + uz;
        const float pair = dcs[0] + dcs[1];
        float suf = pair;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float tt = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += tt;
        }
        const float above = suf - pair;
        const float da[2] = {above + pair, above + dcs[1]};
        float sdA = 0.f, sbias = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = 2 * lane + k;
            if (j < q) {
                const float dd = ddir[k] + Ah * da[k];
                const float z = sz[j];
                const float sg = z >= 0.f ? 1.f / (1.f + expf(-z)) : expf(z) / (1.f + expf(z));
                const float dz = dd * sg;
                ((T*)p.ddt)[(tok0 + j) * H + h] = from_f<T>(dz);
                sdA += sd[j] * da[k];
                sbias += dz;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sdA += __shfl_xor_sync(0xffffffffu, sdA, o);
            sbias += __shfl_xor_sync(0xffffffffu, sbias, o);
        }
        if (lane == 0) {
            atomicAdd(&p.dA[h], sdA);
            atomicAdd(&p.ddt_bias[h], sbias);
            atomicAdd(&p.dD[h], sred[1]);
        }
    };
    float dBa[1][NTN][4], dCa[1][NTN][4];
    zero_frag(dBa);
    zero_frag(dCa);
    // K = L o (dy x^T) o d summed over this block's heads (this thread's fragment of the 64 x 64
    // product (1)): the terms K^T C of dB and K B of dC share C and B across the group's heads,
    // so they are one product each of the sum, after the last head
    float ksum[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int hh = hh0; hh < hh1; ++hh) {
        const int h = g * HG + hh;
        const float bias = p.dt_bias ? p.dt_bias[h] : 0.f, Ah = p.A[h], Dh = p.D ? p.D[h] : 0.f;
        // this head's inputs have landed in the staging area (every thread's copies)
        cp_async_wait_all();
        __syncthreads();
        // warp 0: the previous head's decays; warps 1-15: this head's operands
        const int ct = tid - 32, cn = (int)blockDim.x - 32;
        if (warp == 0 && hh > hh0) decays(hh - 1);
        float xdy = 0.f;   // this thread's part of sum dy . x (bf16 values, exact in fp32 products)
        for (int e = warp == 0 ? Q * P / 8 : ct; e < Q * P / 8; e += cn) {
            const int r = e / (P / 8), c8 = e % (P / 8);
            uint4 ox = make_uint4(0u, 0u, 0u, 0u), od = ox;
            if (r < q) {
                const uint4 vx = *reinterpret_cast<const uint4*>(stX + r * P + 8 * c8);
                const uint4 vd = *reinterpret_cast<const uint4*>(stDY + r * P + 8 * c8);
                const uint32_t wx[4] = {vx.x, vx.y, vx.z, vx.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    xdy += __uint_as_float(wx[m] << 16) * __uint_as_float(wd[m] << 16) +
                           __uint_as_float(wx[m] & 0xffff0000u) * __uint_as_float(wd[m] & 0xffff0000u);
                ox = bf16x8_to_f16x8_bwd(vx);
                od = bf16x8_to_f16x8_bwd(vd);
            }
            *reinterpret_cast<uint4*>(hsw8(sX, r, c8, P)) = ox;
            *reinterpret_cast<uint4*>(hsw8(sDY, r, c8, P)) = od;
        }
        float hpdh = 0.f;   // <h_prev, dh_end> in fp32 from the fp32 states
        {
            const float* hp = stHP;
            const float* dh = stDH;
            for (int e = warp == 0 ? N * P / 8 : ct; e < N * P / 8; e += cn) {
                const int n = e / (P / 8), c8 = e % (P / 8);
                const float4 a0 = *reinterpret_cast<const float4*>(hp + n * P + 8 * c8);
                const float4 a1 = *reinterpret_cast<const float4*>(hp + n * P + 8 * c8 + 4);
                const float4 b0 = *reinterpret_cast<const float4*>(dh + n * P + 8 * c8);
                const float4 b1 = *reinterpret_cast<const float4*>(dh + n * P + 8 * c8 + 4);
                *reinterpret_cast<uint4*>(hsw8(sHP, n, c8, P)) =
                    make_uint4(h2pack(a0.x, a0.y), h2pack(a0.z, a0.w), h2pack(a1.x, a1.y), h2pack(a1.z, a1.w));
                const uint4 dhi =
                    make_uint4(h2pack(b0.x, b0.y), h2pack(b0.z, b0.w), h2pack(b1.x, b1.y), h2pack(b1.z, b1.w));
                *reinterpret_cast<uint4*>(hsw8(sDH, n, c8, P)) = dhi;
                *reinterpret_cast<uint4*>(hsw8(sDHl, n, c8, P)) =
                    make_uint4(h2lo(dhi.x, b0.x, b0.y), h2lo(dhi.y, b0.z, b0.w), h2lo(dhi.z, b1.x, b1.y),
                               h2lo(dhi.w, b1.z, b1.w));
                hpdh += a0.x * b0.x + a0.y * b0.y + a0.z * b0.z + a0.w * b0.w + a1.x * b1.x + a1.y * b1.y +
                        a1.z * b1.z + a1.w * b1.w;
            }
        }
        if (tid < 32) {
            // (after the previous head's decays, which read them in other lanes)
            __syncwarp();
            for (int j = lane; j < Q; j += 32) {
                colR[j] = 0.f; rowRd[j] = 0.f; rowZ[j] = 0.f; rowY[j] = 0.f;
            }
            if (lane < 2) sred[lane] = 0.f;   // sred[2] is written by the decay scan below
            __syncwarp();
            chunk_decay_raw(dt_raw, q, bias, Ah, sd, sz, scs, &sred[2]);
            if (hh + 1 < hh1) load_dt2<T>(dt_raw, dtg, tok0, H, h + 1, q);
            __syncwarp();
            const float last = sred[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int j = 2 * lane + k;
                se[j] = j < q ? expf(scs[j]) : 0.f;
                su[j] = j < q ? expf(last - scs[j]) * sd[j] : 0.f;
            }
        }
        __syncthreads();
        // every thread is done with the staging area: the next head's copies fly while this one
        // computes
        if (hh + 1 < hh1) stage(hh + 1);
        {
            float a1 = hpdh, a2 = xdy;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a1 += __shfl_xor_sync(0xffffffffu, a1, o);
                a2 += __shfl_xor_sync(0xffffffffu, a2, o);
            }
            if (lane == 0) {
                atomicAdd(&sred[0], a1);
                atomicAdd(&sred[1], a2);
            }
        }
        // (1) dy_j . x_i, the masked forms W, K and the sums of R
        {
            float acc[1][2][4];
            zero_frag(acc);
            mma_tile_h<1, 2, true, true>(acc, sDY, P, sX, P, r64, c64, P);
            float rrow[2] = {0.f, 0.f}, rcol[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                    // elements (j, i) and (j, i + 1), i even: one fp16 pair per tile
                    const int j = frag_row(r64, 0, e), i = frag_col(c64, nt, e);
                    const float2 cb = *reinterpret_cast<const float2*>(&sCB[j * kCBW + i]);
                    const float2 di = *reinterpret_cast<const float2*>(&sd[i]);
                    const float2 ci = *reinterpret_cast<const float2*>(&scs[i]);
                    // the fast exponential: this path's operands are fp16 anyway
                    const float L0 = (i <= j && j < q) ? __expf(scs[j] - ci.x) : 0.f;
                    const float L1 = (i + 1 <= j && j < q) ? __expf(scs[j] - ci.y) : 0.f;
                    const float dyx0 = acc[0][nt][e], dyx1 = acc[0][nt][e + 1];
                    const float w0 = cb.x * L0 * di.x, w1 = cb.y * L1 * di.y;
                    const __half2 whi = __floats2half2_rn(w0, w1);
                    const int at = hsw(j, i, Q);
                    *reinterpret_cast<__half2*>(&sW[at]) = whi;
                    *reinterpret_cast<__half2*>(&sWl[at]) =
                        __floats2half2_rn(w0 - __low2float(whi), w1 - __high2float(whi));
                    ksum[nt][e] += L0 * dyx0 * di.x;
                    ksum[nt][e + 1] += L1 * dyx1 * di.y;
                    const float R0 = cb.x * dyx0 * L0, R1 = cb.y * dyx1 * L1;
                    rrow[e >> 1] += R0 * di.x + R1 * di.y;
                    rcol[nt][0] += R0;
                    rcol[nt][1] += R1;
                }
            // summed in the warp first (a row's values sit in one lane quad, a column's in the
            // eight quads), then one shared atomic per row or column and warp
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float v = quad_sum(rrow[a]);
                if ((lane & 3) == 0) atomicAdd(&rowRd[frag_row(r64, 0, 2 * a)], v);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const float v = across_quads_sum(rcol[nt][b]);
                    if (lane < 4) atomicAdd(&colR[frag_col(c64, nt, b)], v);
                }
        }
        __syncthreads();
        // (2) dx = D dy + W^T dy + u o (B dh_end), and Z_i = B_i^T dh_end x_i
        {
            float bd[1][2][4], wd[1][2][4];
            zero_frag(bd);
            zero_frag(wd);
            mma_tile_h_pair<1, 2, true, false, false>(bd, sB, nullptr, N, sDH, sDHl, P, r64, c64, N);
            mma_tile_h_pair<1, 2, false, false, true>(wd, sW, sWl, Q, sDY, nullptr, P, r64, c64, Q);
            T* dxg = (T*)p.dx + (tok0 * H + h) * P;
            float z[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                    // columns c, c + 1 (c even) of row i: one fp16 pair of x and of dy, one bf16 pair out
                    const int i = frag_row(r64, 0, e), c = frag_col(c64, nt, e), at = hsw(i, c, P);
                    const float2 xv = __half22float2(*reinterpret_cast<const __half2*>(&sX[at]));
                    const float2 dv = __half22float2(*reinterpret_cast<const __half2*>(&sDY[at]));
                    z[e >> 1] += bd[0][nt][e] * xv.x + bd[0][nt][e + 1] * xv.y;
                    if (i < q) {
                        const float ui = su[i];
                        *reinterpret_cast<__nv_bfloat162*>(dxg + (int64_t)i * H * P + c) =
                            __floats2bfloat162_rn(Dh * dv.x + wd[0][nt][e] + ui * bd[0][nt][e],
                                                  Dh * dv.y + wd[0][nt][e + 1] + ui * bd[0][nt][e + 1]);
                    }
                }
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float v = quad_sum(z[a]);
                if ((lane & 3) == 0) atomicAdd(&rowZ[frag_row(r64, 0, 2 * a)], v);
            }
        }
        // (4) dB += u o (x dh_end^T),  dC += e o (dy h_prev^T)  (K^T C and K B after the last head),
        // and Y_j = C_j^T h_prev dy_j = sum_n C_jn (dy h_prev^T)_jn from the second product
        {
            float t[1][NTN][4];
            zero_frag(t);
            mma_tile_h<1, NTN, true, true>(t, sX, P, sDH, P, rN, cN, P);
#pragma unroll
            for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dBa[0][nt][e] += su[frag_row(rN, 0, e)] * t[0][nt][e];
            zero_frag(t);
            mma_tile_h<1, NTN, true, true>(t, sDY, P, sHP, P, rN, cN, P);
            float y[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                    const int j = frag_row(rN, 0, e), n = frag_col(cN, nt, e);
                    const float2 cv = __half22float2(*reinterpret_cast<const __half2*>(&sC[hsw(j, n, N)]));
                    y[e >> 1] += cv.x * t[0][nt][e] + cv.y * t[0][nt][e + 1];
                    const float ej = se[j];
                    dCa[0][nt][e] += ej * t[0][nt][e];
                    dCa[0][nt][e + 1] += ej * t[0][nt][e + 1];
                }
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float v = quad_sum(y[a]);
                if ((lane & 3) == 0) atomicAdd(&rowY[frag_row(rN, 0, 2 * a)], v);
            }
        }
        // (the barrier at the top of the next head orders these reads before its conversion)
    }
    __syncthreads();
    if (warp == 0) decays(hh1 - 1);
    // dB += (sum K)^T C, dC += (sum K) B, the sum as an fp16 pair hi + lo (lo over W's last tile)
    {
        __half* sKl = sWl;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const int at = hsw(frag_row(r64, 0, e), frag_col(c64, nt, e), Q);
                const __half2 hi = __floats2half2_rn(ksum[nt][e], ksum[nt][e + 1]);
                *reinterpret_cast<__half2*>(&sK[at]) = hi;
                *reinterpret_cast<__half2*>(&sKl[at]) =
                    __floats2half2_rn(ksum[nt][e] - __low2float(hi), ksum[nt][e + 1] - __high2float(hi));
            }
        __syncthreads();
        mma_tile_h_pair<1, NTN, false, false, true>(dBa, sK, sKl, Q, sC, nullptr, N, rN, cN, Q);
        mma_tile_h_pair<1, NTN, true, false, true>(dCa, sK, sKl, Q, sB, nullptr, N, rN, cN, Q);
    }
    if (p.hsplit > 1) {
        // this part's sums, in fp32, for k_bwd_sum_parts
        float* dBg = p.dBp + part * p.part_stride + (tok0 * G + g) * N;
        float* dCg = p.dCp + part * p.part_stride + (tok0 * G + g) * N;
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const int i = frag_row(rN, 0, e), n = frag_col(cN, nt, e);
                if (i < q) {
                    *reinterpret_cast<float2*>(dBg + (int64_t)i * G * N + n) = make_float2(dBa[0][nt][e], dBa[0][nt][e + 1]);
                    *reinterpret_cast<float2*>(dCg + (int64_t)i * G * N + n) = make_float2(dCa[0][nt][e], dCa[0][nt][e + 1]);
                }
            }
        return;
    }
    T* dBg = (T*)p.dB + (tok0 * G + g) * N;
    T* dCg = (T*)p.dC + (tok0 * G + g) * N;
#pragma unroll
    for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = frag_row(rN, 0, e), n = frag_col(cN, nt, e);
            if (i < q) {
                dBg[(int64_t)i * G * N + n] = from_f<T>(dBa[0][nt][e]);
                dCg[(int64_t)i * G * N + n] = from_f<T>(dCa[0][nt][e]);
            }
        }
}

// ---- k_bwd_pass_h: the chunk terms computed inside the sequential pass (bf16, P = Q = 64) ----
//
// Two blocks per (sequence, head) walk the sequence's chunks, one forwards, one backwards, each
// holding the N x 64 state (or its adjoint) in mma.sync accumulator fragments: warp w owns 16 state rows and
// P / NCB columns.  At every chunk it computes the chunk's own term on the tensor cores,
// S = B^T (u o x) forwards and T = C^T (e o dy) backwards (u_j = exp(cs_last - cs_j) d_j,
// e_j = exp(cs_j)), from operands staged by cp.async one chunk ahead, so no term goes through
// HBM.  It writes the state entering every chunk (forwards, over S) and the adjoint of the state
// leaving every chunk (backwards, over T) for k_bwd_grads_h, and d h0 at the end.
template <int N>
__global__ void __launch_bounds__(256, 3) k_bwd_pass_h(const ChunkedBwd p) {
    using T = __nv_bfloat16;
    constexpr int P = kPb, Q = kQb;
    constexpr int NRB = N / 16;          // 16-row blocks of the state
    constexpr int NCB = 8 / NRB;         // column blocks per row block (eight warps)
    constexpr int NT = P / NCB / 8;      // 8-column MMA tiles per warp
    static_assert(NRB * NCB == 8 && NT % 2 == 0, "eight warps cover the N x 64 state");
    extern __shared__ __align__(16) uint8_t smraw[];
    __half* sM = reinterpret_cast<__half*>(smraw);   // [Q][N] B or C, fp16 swizzled
    __half* sV = sM + Q * N;                         // [Q][P] u o x or e o dy
    T* stM = reinterpret_cast<T*>(sV + Q * P);       // [Q][N] the next chunk's raw rows
    T* stV = stM + Q * N;                            // [Q][P]
    // decay quantities of a chunk, double-buffered: warp 0 prepares chunk i + 1 while chunk i runs
    __shared__ float sd[2][kQb], sz[2][kQb], scs[2][kQb], sw[2][kQb], slast[2];
    const int H = p.H, G = p.G;
    // blocks [0, S H) run the forward sweep, [S H, 2 S H) the backward one: they are independent
    const bool fwd_block = blockIdx.x < (unsigned)(p.si.S * H);
    const int sh = (int)(fwd_block ? blockIdx.x : blockIdx.x - p.si.S * H);
    const int s = sh / H, h = sh % H, g = h / (H / G);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nc = seq_nchunks(p.si, s);
    const int64_t cf0 = seq_chunk0(p.si, s);
    int64_t row, ts, te;
    seq_span(p.si, s, row, ts, te);
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f, Ah = p.A[h];
    const int n0 = 16 * (warp % NRB), col0 = (P / NCB) * (warp / NRB);
    const T* dtg = (const T*)p.dt;
    auto chunk_q = [&](int c) {
        const int64_t t0 = ts + (int64_t)c * Q;
        return (int)(te - t0 < Q ? te - t0 : Q);
    };
    auto chunk_tok0 = [&](int c) { return row * p.si.L + ts + (int64_t)c * Q; };
    const int64_t slab = (int64_t)N * P;
    // raw rows (those inside the chunk) of M (B or C, per group) and V (x or dy, per head)
    auto stage = [&](int c, const T* Mg, const T* Vg) {
        const int q = chunk_q(c);
        const int64_t tok0 = chunk_tok0(c);
        for (int e = tid; e < Q * N / 8; e += blockDim.x) {
            const int r = e / (N / 8), c8 = e % (N / 8);
            if (r < q) cp_async16(stM + r * N + 8 * c8, Mg + ((tok0 + r) * G + g) * N + 8 * c8);
        }
        for (int e = tid; e < Q * P / 8; e += blockDim.x) {
            const int r = e / (P / 8), c8 = e % (P / 8);
            if (r < q) cp_async16(stV + r * P + 8 * c8, Vg + ((tok0 + r) * H + h) * P + 8 * c8);
        }
        cp_async_commit();
    };
    float acc[1][NT][4];
    // (N, P) fp32 row-major <-> this warp's fragment (null source: zero)
    auto load_frag = [&](const float* src) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                float2 v = make_float2(0.f, 0.f);
                if (src) v = *reinterpret_cast<const float2*>(src + frag_row(n0, 0, e) * P + frag_col(col0, nt, e));
                acc[0][nt][e] = v.x;
                acc[0][nt][e + 1] = v.y;
            }
    };
    auto store_frag = [&](float* dst) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; e += 2)
                *reinterpret_cast<float2*>(dst + frag_row(n0, 0, e) * P + frag_col(col0, nt, e)) =
                    make_float2(acc[0][nt][e], acc[0][nt][e + 1]);
    };
    auto sweep = [&](bool fwd) {
        const T* Mg = (const T*)(fwd ? p.B : p.C);
        const T* Vg = (const T*)(fwd ? p.x : p.dy);
        float* slabs = fwd ? p.S : p.T;
        const int cfirst = fwd ? 0 : nc - 1, step = fwd ? 1 : -1;
        float dt_raw[2] = {0.f, 0.f};   // warp 0: raw dt of the next chunk to prepare
        // warp 0: d, z, cs and the operand weights (u forwards, e backwards) of chunk c into buffer b
        auto decay = [&](int c, int b) {
            const int q = chunk_q(c);
            chunk_decay_raw(dt_raw, q, bias, Ah, sd[b], sz[b], scs[b], &slast[b]);
            __syncwarp();
            const float last = slast[b];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int j = 2 * lane + k;
                sw[b][j] = j < q ? (fwd ? expf(last - scs[b][j]) * sd[b][j] : expf(scs[b][j])) : 0.f;
            }
        };
        if (nc > 0) {
            stage(cfirst, Mg, Vg);
            if (tid < 32) {
                load_dt2<T>(dt_raw, dtg, chunk_tok0(cfirst), H, h, chunk_q(cfirst));
                decay(cfirst, 0);
                if (nc > 1) load_dt2<T>(dt_raw, dtg, chunk_tok0(cfirst + step), H, h, chunk_q(cfirst + step));
            }
        }
        for (int i = 0; i < nc; ++i) {
            const int c = cfirst + step * i, b = i & 1;
            const int q = chunk_q(c);
            // chunk c's rows have landed and its decay is in buffer b; every warp is done with the
            // previous chunk's operands and with buffer b ^ 1
            cp_async_wait_all();
            __syncthreads();
            if (tid < 32) {
                if (i + 1 < nc) {
                    decay(c + step, b ^ 1);
                    if (i + 2 < nc) load_dt2<T>(dt_raw, dtg, chunk_tok0(c + 2 * step), H, h, chunk_q(c + 2 * step));
                }
            } else {
                for (int e = tid - 32; e < Q * N / 8; e += blockDim.x - 32) {
                    const int r = e / (N / 8), c8 = e % (N / 8);
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if (r < q) o = bf16x8_to_f16x8_bwd(*reinterpret_cast<const uint4*>(stM + r * N + 8 * c8));
                    *reinterpret_cast<uint4*>(hsw8(sM, r, c8, N)) = o;
                }
                for (int e = tid - 32; e < Q * P / 8; e += blockDim.x - 32) {
                    const int r = e / (P / 8), c8 = e % (P / 8);
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if (r < q) {
                        const float w = sw[b][r];
                        const uint4 v = *reinterpret_cast<const uint4*>(stV + r * P + 8 * c8);
                        auto cv = [w](uint32_t u) {
                            return h2pack(w * __uint_as_float(u << 16), w * __uint_as_float(u & 0xffff0000u));
                        };
                        o = make_uint4(cv(v.x), cv(v.y), cv(v.z), cv(v.w));
                    }
                    *reinterpret_cast<uint4*>(hsw8(sV, r, c8, P)) = o;
                }
            }
            const float E = expf(slast[b]);
            __syncthreads();   // operands ready; the staging area is free again
            if (i + 1 < nc) stage(c + step, Mg, Vg);
            // the state entering chunk c (forwards) / the adjoint of the state leaving it (backwards)
            store_frag(slabs + ((cf0 + c) * H + h) * slab);
            // h <- E h + (the chunk's term): scale, then let the MMA add the term in place
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[0][nt][e] *= E;
            mma_tile_h<1, NT, false, false, 1>(acc, sM, N, sV, P, n0, col0, Q);
        }
    };
    if (fwd_block) {
        load_frag(p.init_state ? p.init_state + ((int64_t)s * H + h) * slab : nullptr);
        sweep(true);
    } else {
        load_frag(p.dfinal ? p.dfinal + ((int64_t)s * H + h) * slab : nullptr);
        sweep(false);
        if (p.dinit) store_frag(p.dinit + ((int64_t)s * H + h) * slab);
    }
}

template <int N>
constexpr size_t grads_smem() {
    return sizeof(float) * (2 * kQb * (N + 4) + 3 * kQb * kQb + 2 * kQb * (kPb + 4) + 2 * N * (kPb + 4) +
                            10 * kQb + 4);
}

// dB, dC = the sum of the gradient blocks' fp32 partials (parts in order), rounded once; 4 per step.
__global__ void k_bwd_sum_parts(const float* __restrict__ pb, const float* __restrict__ pc,
                                __nv_bfloat16* __restrict__ db, __nv_bfloat16* __restrict__ dc, int64_t n4, int parts,
                                int64_t stride) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        float4 sb = reinterpret_cast<const float4*>(pb)[i], sc = reinterpret_cast<const float4*>(pc)[i];
        for (int k = 1; k < parts; ++k) {
            const float4 ob = reinterpret_cast<const float4*>(pb + k * stride)[i];
            const float4 oc = reinterpret_cast<const float4*>(pc + k * stride)[i];
            sb.x += ob.x; sb.y += ob.y; sb.z += ob.z; sb.w += ob.w;
            sc.x += oc.x; sc.y += oc.y; sc.z += oc.z; sc.w += oc.w;
        }
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(sb.x, sb.y), b1 = __floats2bfloat162_rn(sb.z, sb.w);
        const __nv_bfloat162 c0 = __floats2bfloat162_rn(sc.x, sc.y), c1 = __floats2bfloat162_rn(sc.z, sc.w);
        reinterpret_cast<__nv_bfloat162*>(db)[2 * i] = b0;
        reinterpret_cast<__nv_bfloat162*>(db)[2 * i + 1] = b1;
        reinterpret_cast<__nv_bfloat162*>(dc)[2 * i] = c0;
        reinterpret_cast<__nv_bfloat162*>(dc)[2 * i + 1] = c1;
    }
}

// Blocks per (chunk, group) of the bf16 gradient kernel, each taking an equal share of the
// group's heads: 1, 2 or 4, whichever fills the last wave of the SMs best (by at least 3%, since
// every extra part repeats C B^T and adds the pass summing dB, dC).  With one 512-thread block
// per SM, 512 blocks on 148 SMs run as 3.46 waves (four, the last half empty); 1024 as 6.92.
int grads_hsplit(const ScanArgs& a, int64_t chunks) {
    if (a.dtype == 0 || !bwd_chunked(a)) return 1;
    const int64_t HG = a.H / a.G;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    auto fill = [&](int S) {
        const double w = (double)(chunks * a.G * S) / sms;
        return w / std::ceil(w);
    };
    int best = 1;
    double bf = fill(1);
    for (int S = 2; S <= 4; S *= 2)
        if (HG % S == 0 && fill(S) > bf + 0.03) {
            best = S;
            bf = fill(S);
        }
    return best;
}

template <typename T, int N>
void launch_chunked_t(const ChunkedBwd& p, int64_t chunks, cudaStream_t st) {
    const size_t sm_terms = sizeof(float) * (kQb * N + kQb * kPb);
    if constexpr (sizeof(T) == 4) {
        cudaFuncSetAttribute(k_bwd_terms<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_terms);
        cudaFuncSetAttribute(k_bwd_grads<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grads_smem<N>());
    }
    if constexpr (sizeof(T) == 2) {
        // bf16: the chunk terms are computed inside the pass (k_bwd_pass_h)
        ProfScope ps(K_BWD_PASS, st);
        const size_t sm_p = 2 * 2 * (kQb * N + kQb * kPb);
        cudaFuncSetAttribute(k_bwd_pass_h<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_p);
        k_bwd_pass_h<N><<<(unsigned)(2 * (int64_t)p.si.S * p.H), 256, sm_p, st>>>(p);
    } else {
        {
            ProfScope ps(K_SCAN_BWD, st);
            k_bwd_terms<T, N><<<(unsigned)(chunks * p.H), 256, sm_terms, st>>>(p);
        }
        ProfScope ps(K_BWD_PASS, st);
        constexpr int kVec = N * kPb / 4 / kPassThreads;
        k_bwd_pass<kVec><<<(unsigned)((int64_t)p.si.S * p.H), kPassThreads, 0, st>>>(p.S, p.T, p.E, p.init_state,
                                                                                    p.dfinal, p.dinit, p.si, p.H);
    }
    {
        ProfScope ps(K_BWD_GRADS, st);
        if constexpr (sizeof(T) == 2) {
            cudaFuncSetAttribute(k_bwd_grads_h<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grads_h_smem<N>());
            k_bwd_grads_h<N><<<(unsigned)(chunks * p.G * p.hsplit), kGradThreads, grads_h_smem<N>(), st>>>(p);
            if (p.hsplit > 1) {
                const int64_t n4 = p.part_stride / 4;
                const unsigned grid = (unsigned)std::min<int64_t>((n4 + 255) / 256, 148 * 8);
                k_bwd_sum_parts<<<grid, 256, 0, st>>>(p.dBp, p.dCp, (__nv_bfloat16*)p.dB, (__nv_bfloat16*)p.dC, n4,
                                                       p.hsplit, p.part_stride);
            }
        } else {
            k_bwd_grads<T, N><<<(unsigned)(chunks * p.G), 256, grads_smem<N>(), st>>>(p);
        }
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
    if (bwd_chunked(a)) {
        const int S = grads_hsplit(a, blocks);
        const size_t parts = S > 1 ? 2 * r(sizeof(float) * S * (size_t)(a.b * a.L) * a.G * a.N) : 0;
        return 2 * r(sizeof(float) * blocks * a.H * NP) + r(sizeof(float) * blocks * a.H) + parts;
    }
    return r(sizeof(float) * blocks * a.H * NP) + r(sizeof(float) * a.S * a.H * kBwdBlock * NP) +
           2 * r(sizeof(float) * a.b * a.L * a.G * a.N);
}

int launch_scan_bwd(const ScanArgs& a, const BwdArgs& g, const SeqInfo& si64, void* ws, cudaStream_t st) {
    const size_t NP = (size_t)a.N * a.P;
    auto r = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const int64_t blocks = a.seq_idx ? (a.L + kBwdBlock - 1) / kBwdBlock + a.S
                                     : a.b * ((a.L + kBwdBlock - 1) / kBwdBlock);
    char* w = (char*)ws;
    if (bwd_chunked(a)) {
        ChunkedBwd c;
        c.si = si64;
        c.x = a.x; c.dt = a.dt; c.B = a.B; c.C = a.C; c.dy = g.dy;
        c.dt_bias = a.dt_bias; c.A = a.A; c.D = a.D; c.init_state = a.init_state; c.dfinal = g.dfinal;
        c.dx = g.dx; c.ddt = g.ddt; c.dB = g.dB; c.dC = g.dC;
        c.ddt_bias = g.ddt_bias; c.dA = g.dA; c.dD = g.dD; c.dinit = g.dinit;
        c.S = (float*)w; w += r(sizeof(float) * blocks * a.H * NP);
        c.T = (float*)w; w += r(sizeof(float) * blocks * a.H * NP);
        c.E = (float*)w; w += r(sizeof(float) * blocks * a.H);
        c.H = (int)a.H; c.N = (int)a.N; c.G = (int)a.G;
        c.hsplit = grads_hsplit(a, blocks);
        if (c.hsplit > 1) {
            c.part_stride = a.b * a.L * a.G * a.N;
            c.dBp = (float*)w; w += r(sizeof(float) * c.hsplit * c.part_stride);
            c.dCp = (float*)w;
        }
        cudaError_t e = cudaMemsetAsync(g.ddt_bias, 0, sizeof(float) * a.H, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(g.dA, 0, sizeof(float) * a.H, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(g.dD, 0, sizeof(float) * a.H, st);
        if (e != cudaSuccess) return 6;
        if (a.dtype == 0) {
            if (a.N == 128) launch_chunked_t<float, 128>(c, blocks, st);
            else launch_chunked_t<float, 64>(c, blocks, st);
        } else {
            if (a.N == 128) launch_chunked_t<__nv_bfloat16, 128>(c, blocks, st);
            else launch_chunked_t<__nv_bfloat16, 64>(c, blocks, st);
        }
        return 0;
    }
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
