// ssd_common.cuh -- device helpers shared by the SSD kernels of libssd.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// softplus(z) = log(1 + e^z) without overflow: the step size d_t of the
// discretised recurrence is softplus(dt_t + dt_bias_h).
__device__ __forceinline__ float softplus_f(float z) {
    return z > 0.f ? z + log1pf(expf(-z)) : log1pf(expf(z));
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Where the sequences live.  Without packing, sequence s is batch row s and
// spans [0, L).  With packing (batch 1), sequence s spans [start[s], end[s])
// of row 0; chunk_off[s] is the index of its first chunk in the flat chunk
// list (chunk_off[S] = total).  Chunks are aligned to each sequence's first
// token, so no chunk ever holds two sequences.
struct SeqInfo {
    const int32_t* start;
    const int32_t* end;
    const int32_t* chunk_off;
    int64_t L;
    int32_t S;
    int32_t Q;
    int32_t packed;
    int32_t nc_row;  // chunks per row when not packed
};

struct ChunkRef {
    int64_t row, t0, t1;  // tokens [t0, t1) of batch row `row`
    int32_t s, c;         // sequence and chunk index within it
    int32_t nc;           // chunks in the sequence
};

__device__ __forceinline__ void seq_span(const SeqInfo& si, int s, int64_t& row, int64_t& t0,
                                         int64_t& t1) {
    if (!si.packed) {
        row = s; t0 = 0; t1 = si.L;
    } else {
        row = 0; t0 = si.start[s]; t1 = si.end[s];
    }
}

__device__ __forceinline__ int seq_nchunks(const SeqInfo& si, int s) {
    if (!si.packed) return si.nc_row;
    return si.chunk_off[s + 1] - si.chunk_off[s];
}

__device__ __forceinline__ int64_t seq_chunk0(const SeqInfo& si, int s) {
    if (!si.packed) return (int64_t)s * si.nc_row;
    return si.chunk_off[s];
}

// Maps a flat chunk index to its sequence and token range; false past the end.
__device__ __forceinline__ bool chunk_ref(const SeqInfo& si, int64_t f, ChunkRef& r) {
    if (!si.packed) {
        if (si.nc_row == 0) return false;
        int64_t s = f / si.nc_row;
        if (s >= si.S) return false;
        r.s = (int32_t)s; r.c = (int32_t)(f - s * si.nc_row); r.nc = si.nc_row;
        r.row = s; r.t0 = (int64_t)r.c * si.Q;
        r.t1 = r.t0 + si.Q < si.L ? r.t0 + si.Q : si.L;
        return true;
    }
    if (f >= si.chunk_off[si.S]) return false;
    int lo = 0, hi = si.S - 1;  // last s with chunk_off[s] <= f
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (si.chunk_off[mid] <= f) lo = mid; else hi = mid - 1;
    }
    r.s = lo; r.c = (int32_t)(f - si.chunk_off[lo]);
    r.nc = si.chunk_off[lo + 1] - si.chunk_off[lo];
    r.row = 0;
    r.t0 = si.start[lo] + (int64_t)r.c * si.Q;
    int64_t e = si.end[lo];
    r.t1 = r.t0 + si.Q < e ? r.t0 + si.Q : e;
    return true;
}

// Device status word codes (mirrors ssd_status in ssd.h).
enum : int32_t { kStatusOk = 0, kStatusTimeout = 7, kStatusSeqIdx = 8 };

}  // namespace ssd
