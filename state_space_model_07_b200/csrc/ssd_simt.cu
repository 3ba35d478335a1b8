// ssd_simt.cu -- chunked SSD scan with CUDA-core fp32 arithmetic.
//
// The general path of libssd.so: any supported P, N, chunk length, float32 or
// bfloat16 inputs.  It is the only path for float32 inputs (tensor-core tf32
// would lose the 1e-4 accuracy float32 mode promises) and for bf16 shapes the
// tensor-core path does not cover.  Three stages, following the block
// decomposition of "5.3 Tensor Parallelism support and large-cluster training",
// section 3.2:
//   1. k_simt_chunk_state: per chunk and head, the chunk's own state
//        S_c = sum_i exp(cs_last - cs_i) d_i B_i x_i^T      (N x P, fp32)
//      plus the chunk's total log-decay cs_last.
//   2. k_simt_state_pass: per sequence and head, sequentially over chunks,
//        h_c = exp(cs_last_c) h_{c-1} + S_c,  h_{-1} = init_state,
//      overwriting S_c in place with the state entering chunk c.
//   3. k_simt_chunk_out: per chunk and head, the quadratic diagonal block plus
//      the low-rank term of the entering state and the D skip:
//        y_j = sum_{i<=j} (C_j.B_i) exp(cs_j - cs_i) d_i x_i
//              + exp(cs_j) C_j^T h_prev + D x_j.
// Chunks start at each sequence's first token, so a packed sequence never
// shares a chunk with another one: the reset at sequence starts (section 4.3)
// is structural and needs no masking arithmetic.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

namespace ssd {

constexpr int kThreads = 256;

// Block-wide inclusive prefix sum of one value per thread (blockDim = 256).
__device__ __forceinline__ float block_inclusive_scan(float v, float* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float t = lane < (kThreads / 32) ? warp_tot[lane] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        if (lane < (kThreads / 32)) warp_tot[lane] = t;
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    return v;
}

// d_i = softplus(dt_i + dt_bias_h) and the chunk-local inclusive cumulative
// log-decay cs_i = sum_{k<=i} d_k A_h, for the q <= 256 tokens of one chunk.
template <typename T>
__device__ __forceinline__ void chunk_decay(const ChunkRef& r, const T* __restrict__ dt, float bias,
                                            float Ah, int64_t L, int H, int h, float* d_s,
                                            float* cs_s, float* warp_tot) {
    const int i = threadIdx.x;
    const int q = (int)(r.t1 - r.t0);
    float dv = 0.f, a = 0.f;
    if (i < q) {
        float z = to_f<T>(dt[(r.row * L + r.t0 + i) * H + h]) + bias;
        dv = softplus_f(z);
        a = dv * Ah;
    }
    float cs = block_inclusive_scan(a, warp_tot);
    d_s[i] = dv;
    cs_s[i] = cs;
    __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
k_simt_chunk_state(SeqInfo si, const T* __restrict__ x, const T* __restrict__ dt,
                   const float* __restrict__ dt_bias, const float* __restrict__ A,
                   const T* __restrict__ B, int H, int P, int N, int G,
                   float* __restrict__ ws_states, float* __restrict__ ws_cs) {
    ChunkRef r;
    if (!chunk_ref(si, blockIdx.x, r)) return;
    const int64_t f = blockIdx.x;
    const int h = blockIdx.y, g = h / (H / G);
    const int64_t L = si.L;
    __shared__ float d_s[kThreads], cs_s[kThreads], w_s[kThreads], warp_tot[8];
    __shared__ float Bs[32][65], xs[32][65];
    const int ntn = N >= 64 ? 64 : N, ntp = P >= 64 ? 64 : P;
    const int tiles_p = P / ntp;
    const int n0 = (blockIdx.z / tiles_p) * ntn, p0 = (blockIdx.z % tiles_p) * ntp;

    chunk_decay<T>(r, dt, dt_bias ? dt_bias[h] : 0.f, A[h], L, H, h, d_s, cs_s, warp_tot);
    const int q = (int)(r.t1 - r.t0);
    const float cs_last = cs_s[q - 1];
    const int tid = threadIdx.x;
    if (tid < q) w_s[tid] = d_s[tid] * expf(cs_last - cs_s[tid]);
    __syncthreads();

    const int ty = tid / 16, tx = tid % 16;
    const int na = ntn / 16, pb = ntp / 16;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

    for (int i0 = 0; i0 < q; i0 += 32) {
        for (int e = tid; e < 32 * ntn; e += kThreads) {
            int ii = e / ntn, nn = e % ntn, tok = i0 + ii;
            Bs[ii][nn] = tok < q ? to_f<T>(B[((r.row * L + r.t0 + tok) * G + g) * N + n0 + nn]) : 0.f;
        }
        for (int e = tid; e < 32 * ntp; e += kThreads) {
            int ii = e / ntp, pp = e % ntp, tok = i0 + ii;
            xs[ii][pp] = tok < q ? w_s[tok] * to_f<T>(x[((r.row * L + r.t0 + tok) * H + h) * P + p0 + pp])
                                 : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int ii = 0; ii < 32; ++ii) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                if (a < na) {
                    float bv = Bs[ii][ty + 16 * a];
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (b < pb) acc[a][b] += bv * xs[ii][tx + 16 * b];
                }
            }
        }
        __syncthreads();
    }
    float* out = ws_states + ((f * H + h) * (int64_t)N) * P;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            if (a < na && b < pb) out[(int64_t)(n0 + ty + 16 * a) * P + p0 + tx + 16 * b] = acc[a][b];
    if (blockIdx.z == 0 && tid == 0) ws_cs[f * H + h] = cs_last;
}

// One thread owns 4 consecutive state elements of one (sequence, head) and
// walks the sequence's chunks in order.
__global__ void __launch_bounds__(kThreads)
k_simt_state_pass(SeqInfo si, const float* __restrict__ init_state, float* __restrict__ ws_states,
                  const float* __restrict__ ws_cs, float* final_state, int H, int64_t NP) {
    const int s = blockIdx.x, h = blockIdx.y;
    const int64_t e = ((int64_t)blockIdx.z * kThreads + threadIdx.x) * 4;
    if (e >= NP) return;
    const int nc = seq_nchunks(si, s);
    const int64_t f0 = seq_chunk0(si, s);
    float4 hv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init_state) hv = *reinterpret_cast<const float4*>(init_state + ((int64_t)s * H + h) * NP + e);
    for (int c = 0; c < nc; ++c) {
        const int64_t f = f0 + c;
        float4* ptr = reinterpret_cast<float4*>(ws_states + (f * H + h) * NP + e);
        float4 sc = *ptr;
        *ptr = hv;  // state entering chunk c
        const float dec = expf(ws_cs[f * H + h]);
        hv.x = dec * hv.x + sc.x;
        hv.y = dec * hv.y + sc.y;
        hv.z = dec * hv.z + sc.z;
        hv.w = dec * hv.w + sc.w;
    }
    if (final_state) *reinterpret_cast<float4*>(final_state + ((int64_t)s * H + h) * NP + e) = hv;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
k_simt_chunk_out(SeqInfo si, const T* __restrict__ x, const T* __restrict__ dt,
                 const float* __restrict__ dt_bias, const float* __restrict__ A,
                 const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D,
                 const float* __restrict__ ws_hprev, T* __restrict__ y, int H, int P, int N, int G) {
    ChunkRef r;
    if (!chunk_ref(si, blockIdx.x, r)) return;
    const int64_t f = blockIdx.x;
    const int h = blockIdx.y, g = h / (H / G);
    const int64_t L = si.L;
    const int pt = P >= 64 ? 64 : P;
    const int p0 = blockIdx.z * pt;
    const int ldn = N + 1;
    extern __shared__ float smem[];
    float* d_s = smem;                 // 256
    float* cs_s = d_s + kThreads;      // 256
    float* Cs = cs_s + kThreads;       // 32 x (N+1)
    float* Bs = Cs + 32 * ldn;         // 32 x (N+1)
    float* Ss = Bs + 32 * ldn;         // 32 x 33
    float* xs = Ss + 32 * 33;          // 32 x 64
    float* hs = xs + 32 * 64;          // 32 x 64
    __shared__ float warp_tot[8];

    chunk_decay<T>(r, dt, dt_bias ? dt_bias[h] : 0.f, A[h], L, H, h, d_s, cs_s, warp_tot);
    const int q = (int)(r.t1 - r.t0);
    const int tid = threadIdx.x;
    const int jr = tid / 8, pc = tid % 8;
    const int kp = pt / 8;
    const float Dh = D ? D[h] : 0.f;
    const float* hp = ws_hprev + (f * H + h) * (int64_t)N * P;

    for (int j0 = 0; j0 < q; j0 += 32) {
        for (int e = tid; e < 32 * N; e += kThreads) {
            int jj = e / N, n = e % N, tok = j0 + jj;
            Cs[jj * ldn + n] = tok < q ? to_f<T>(C[((r.row * L + r.t0 + tok) * G + g) * N + n]) : 0.f;
        }
        float acc[8], acco[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) { acc[k] = 0.f; acco[k] = 0.f; }

        for (int i0 = 0; i0 <= j0; i0 += 32) {
            for (int e = tid; e < 32 * N; e += kThreads) {
                int ii = e / N, n = e % N, tok = i0 + ii;
                Bs[ii * ldn + n] = tok < q ? to_f<T>(B[((r.row * L + r.t0 + tok) * G + g) * N + n]) : 0.f;
            }
            for (int e = tid; e < 32 * pt; e += kThreads) {
                int ii = e / pt, pp = e % pt, tok = i0 + ii;
                xs[ii * 64 + pp] = tok < q ? to_f<T>(x[((r.row * L + r.t0 + tok) * H + h) * P + p0 + pp]) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                int e = tid + kThreads * k, jj = e / 32, ii = e % 32;
                int j = j0 + jj, i = i0 + ii;
                float v = 0.f;
                if (i <= j && j < q) {
                    float dot = 0.f;
                    for (int n = 0; n < N; ++n) dot += Cs[jj * ldn + n] * Bs[ii * ldn + n];
                    v = dot * expf(cs_s[j] - cs_s[i]) * d_s[i];
                }
                Ss[jj * 33 + ii] = v;
            }
            __syncthreads();
#pragma unroll 8
            for (int ii = 0; ii < 32; ++ii) {
                float sv = Ss[jr * 33 + ii];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < kp) acc[k] += sv * xs[ii * 64 + pc + 8 * k];
            }
            __syncthreads();
        }
        // Low-rank term of the state entering the chunk.
        for (int n0 = 0; n0 < N; n0 += 32) {
            for (int e = tid; e < 32 * pt; e += kThreads) {
                int nn = e / pt, pp = e % pt;
                hs[nn * 64 + pp] = n0 + nn < N ? hp[(int64_t)(n0 + nn) * P + p0 + pp] : 0.f;
            }
            __syncthreads();
            const int nmax = N - n0 < 32 ? N - n0 : 32;
            for (int nn = 0; nn < nmax; ++nn) {
                float cv = Cs[jr * ldn + n0 + nn];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < kp) acco[k] += cv * hs[nn * 64 + pc + 8 * k];
            }
            __syncthreads();
        }
        const int j = j0 + jr;
        if (j < q) {
            const float ej = expf(cs_s[j]);
            const int64_t base = ((r.row * L + r.t0 + j) * H + h) * P + p0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (k < kp) {
                    int p = pc + 8 * k;
                    float xv = to_f<T>(x[base + p]);
                    y[base + p] = from_f<T>(acc[k] + ej * acco[k] + Dh * xv);
                }
            }
        }
        __syncthreads();
    }
}

// ---- packed-sequence table ------------------------------------------------------

__global__ void k_seq_bounds(const int32_t* __restrict__ seq_idx, int64_t L, int32_t S,
                             int32_t* __restrict__ start, int32_t* status) {
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < L;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int32_t v = seq_idx[t];
        const int32_t prev = t > 0 ? seq_idx[t - 1] : -1;
        if (status) {
            bool bad = (t == 0 && v != 0) || (t > 0 && v != prev && v != prev + 1) ||
                       (t == L - 1 && v != S - 1);
            if (bad) atomicExch(status, kStatusSeqIdx);
        }
        const int32_t s = v < 0 ? 0 : (v >= S ? S - 1 : v);
        if (t == 0 || v != prev) start[s] = (int32_t)t;
    }
}

// One thread: turns sequence starts into [start, end) spans and chunk offsets.
// Any start that is missing or out of order (a broken seq_idx) becomes an
// empty span, so every later index stays inside [0, L].
__global__ void k_seq_table(int64_t L, int32_t S, int32_t Q, int32_t* start, int32_t* end,
                            int32_t* chunk_off) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int32_t next = (int32_t)L;
    for (int32_t s = S - 1; s >= 0; --s) {
        int32_t st = start[s];
        if (st < 0 || st > next) st = next;
        start[s] = st;
        end[s] = next;
        next = st;
    }
    int32_t off = 0;
    for (int32_t s = 0; s < S; ++s) {
        chunk_off[s] = off;
        off += (end[s] - start[s] + Q - 1) / Q;
    }
    chunk_off[S] = off;
}

void launch_seq_table(const int32_t* seq_idx, int64_t L, int32_t S, int32_t Q, int32_t* start,
                      int32_t* end, int32_t* chunk_off, int32_t* status, cudaStream_t st) {
    cudaMemsetAsync(start, 0xff, sizeof(int32_t) * S, st);
    int64_t blocks = (L + 255) / 256;
    if (blocks > 1184) blocks = 1184;
    if (blocks < 1) blocks = 1;
    {
        ProfScope ps(K_SEQ_BOUNDS, st);
        k_seq_bounds<<<(unsigned)blocks, 256, 0, st>>>(seq_idx, L, S, start, status);
    }
    {
        ProfScope ps(K_SEQ_TABLE, st);
        k_seq_table<<<1, 32, 0, st>>>(L, S, Q, start, end, chunk_off);
    }
}

template <typename T>
static void launch_simt_t(const ScanArgs& a, const SeqInfo& si, int64_t max_chunks, float* ws_states,
                          float* ws_cs, cudaStream_t st) {
    const int H = (int)a.H, P = (int)a.P, N = (int)a.N, G = (int)a.G;
    const int ntn = N >= 64 ? 64 : N, ntp = P >= 64 ? 64 : P;
    dim3 g1((unsigned)max_chunks, H, (N / ntn) * (P / ntp));
    {
        ProfScope ps(K_SIMT_CHUNK_STATE, st);
        k_simt_chunk_state<T><<<g1, kThreads, 0, st>>>(si, (const T*)a.x, (const T*)a.dt, a.dt_bias,
                                                       a.A, (const T*)a.B, H, P, N, G, ws_states, ws_cs);
    }
    const int64_t NP = (int64_t)N * P;
    dim3 g2((unsigned)si.S, H, (unsigned)((NP / 4 + kThreads - 1) / kThreads));
    {
        ProfScope ps(K_SIMT_STATE_PASS, st);
        k_simt_state_pass<<<g2, kThreads, 0, st>>>(si, a.init_state, ws_states, ws_cs, a.final_state,
                                                   H, NP);
    }
    const size_t smem = sizeof(float) * (2 * kThreads + 2 * 32 * (N + 1) + 32 * 33 + 2 * 32 * 64);
    cudaFuncSetAttribute(k_simt_chunk_out<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 g3((unsigned)max_chunks, H, P / ntp);
    {
        ProfScope ps(K_SIMT_CHUNK_OUT, st);
        k_simt_chunk_out<T><<<g3, kThreads, smem, st>>>(si, (const T*)a.x, (const T*)a.dt, a.dt_bias,
                                                        a.A, (const T*)a.B, (const T*)a.C, a.D,
                                                        ws_states, (T*)a.y, H, P, N, G);
    }
}

size_t simt_workspace_bytes(const ScanArgs& a, int64_t max_chunks) {
    return sizeof(float) * (size_t)max_chunks * a.H * (a.N * a.P + 1);
}

void launch_simt_scan(const ScanArgs& a, const SeqInfo& si, int64_t max_chunks, void* ws,
                      cudaStream_t st) {
    float* ws_states = (float*)ws;
    float* ws_cs = ws_states + (size_t)max_chunks * a.H * a.N * a.P;
    if (a.dtype == 0)
        launch_simt_t<float>(a, si, max_chunks, ws_states, ws_cs, st);
    else
        launch_simt_t<__nv_bfloat16>(a, si, max_chunks, ws_states, ws_cs, st);
}

}  // namespace ssd
