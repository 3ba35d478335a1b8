// ssd_api.cu -- the extern "C" boundary of libssd.so (declared in include/ssd.h).
//
// Host side only: argument validation (no device reads), path selection,
// stream-ordered temporary memory (from a library-owned pool), launches, error
// reporting.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_tc.h"

namespace {

thread_local char g_last_error[512];

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return code;
}

bool debug_check() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("SSD_DEBUG_CHECK");
        v = (e && e[0] == '1') ? 1 : 0;
    }
    return v == 1;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

int check_sizes(const ssd_dims* d) {
    if (d->dtype != SSD_F32 && d->dtype != SSD_BF16)
        return fail(SSD_ERR_DTYPE, "dtype %d is not SSD_F32 or SSD_BF16", (int)d->dtype);
    if (d->nheads < 1 || d->ngroups < 1 || d->nheads % d->ngroups != 0)
        return fail(SSD_ERR_SHAPE, "nheads (%lld) must be a positive multiple of ngroups (%lld)",
                    (long long)d->nheads, (long long)d->ngroups);
    if (d->headdim < 16 || d->headdim > 256 || d->headdim % 16 != 0)
        return fail(SSD_ERR_SHAPE, "headdim %lld must be a multiple of 16 in [16, 256]",
                    (long long)d->headdim);
    if (d->dstate < 16 || d->dstate > 256 || d->dstate % 16 != 0)
        return fail(SSD_ERR_SHAPE, "dstate %lld must be a multiple of 16 in [16, 256]",
                    (long long)d->dstate);
    if (d->batch < 0) return fail(SSD_ERR_SHAPE, "batch %lld < 0", (long long)d->batch);
    if (d->nheads > 65535) return fail(SSD_ERR_SHAPE, "nheads %lld > 65535", (long long)d->nheads);
    return SSD_OK;
}

// Sub-allocator over one stream-ordered block (256-byte aligned pieces).
struct Carve {
    char* base = nullptr;
    size_t off = 0;
    void* take(size_t bytes) {
        void* p = base + off;
        off += (bytes + 255) & ~(size_t)255;
        return p;
    }
    static size_t round(size_t bytes) { return (bytes + 255) & ~(size_t)255; }
};

int cuda_fail(const char* what, cudaError_t e) {
    return fail(SSD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// The library's own stream-ordered memory pool, one per device, created on
// first use with that device current.  Its release threshold is unlimited: a
// workspace freed at the end of a call stays mapped in the pool for the next
// call instead of going back to the OS at the next synchronisation (which made
// each call after a sync map the workspace again, occasionally for
// milliseconds).  The pool holds at most the largest workspace in flight at a
// time; the caller's own allocations (torch's, the default pool's) are left
// alone.  Returns nullptr if the pool cannot be made.
cudaMemPool_t workspace_pool() {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
        uint64_t keep = ~(uint64_t)0;
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return nullptr;
        }
        pools[dev] = pool;
    }
    return pools[dev];
}

// Waits for the stream and reports device-side status (debug mode only):
// the status word and, after a tensor-core scan, the value-check counters.
int debug_sync(cudaStream_t st, const int32_t* status_dev, const uint32_t* counters_dev = nullptr) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail("kernel execution", e);
    if (status_dev) {
        int32_t s = 0;
        e = cudaMemcpy(&s, status_dev, sizeof(s), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail("status read", e);
        if (s == ssd::kStatusSeqIdx) return fail(SSD_ERR_SEQIDX, "seq_idx breaks its contract");
        if (s == ssd::kStatusTimeout) return fail(SSD_ERR_TIMEOUT, "a bounded device wait gave up");
    }
    if (counters_dev) {
        uint32_t c[3] = {0, 0, 0};
        e = cudaMemcpy(c, counters_dev, sizeof(c), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail("value-check read", e);
        if (c[1])
            return fail(SSD_ERR_RANGE,
                        "%u finite x, B, C or init_state values exceed 65504, the fp16 operand range of the "
                        "tensor-core path", c[1]);
        if (c[2] && !c[0])
            return fail(SSD_ERR_RANGE,
                        "finite inputs gave %u non-finite outputs: an intermediate (score matrix or carried "
                        "state) left the fp16 operand range of the tensor-core path", c[2]);
    }
    return SSD_OK;
}

// Host-side validation shared by both scan entry points; touches no device
// memory.  On SSD_OK, `a` holds the launch arguments, `max_chunks` the number
// of chunks the scan may visit (packed input: one partial chunk more per
// sequence) and `nstate` the bytes of one (S, H, N, P) float32 state array.
int prepare_scan(const ssd_dims* dims, const void* x, const void* dt, const float* dt_bias,
                 const float* A, const void* B, const void* C, const float* D,
                 const float* init_state, const int32_t* seq_idx, int chunk, void* y,
                 float* final_state, ssd::ScanArgs& a, int64_t& max_chunks, size_t& nstate) {
    if (!dims) return fail(SSD_ERR_NULL, "dims is NULL");
    int rc = check_sizes(dims);
    if (rc) return rc;
    if (chunk < 16 || chunk > 256 || (chunk & (chunk - 1)) != 0)
        return fail(SSD_ERR_CHUNK, "chunk %d is not a power of two in [16, 256]", chunk);
    const int64_t b = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim;
    const int64_t N = dims->dstate, G = dims->ngroups;
    if (L < 0) return fail(SSD_ERR_SHAPE, "seqlen %lld < 0", (long long)L);
    if (!A) return fail(SSD_ERR_NULL, "A is NULL");
    int64_t S = b;
    if (seq_idx) {
        if (b != 1 && b * L != 0)
            return fail(SSD_ERR_SHAPE, "seq_idx requires batch == 1 (got %lld)", (long long)b);
        if (L >= ((int64_t)1 << 31)) return fail(SSD_ERR_SHAPE, "packed seqlen must be < 2^31");
        S = dims->nseqs;
        if (S < 0 || (L > 0 && (S < 1 || S > L)))
            return fail(SSD_ERR_SHAPE, "nseqs %lld must be in [1, seqlen] for packed input",
                        (long long)S);
    }
    const int64_t ntok = b * L;
    const size_t es = dims->dtype == SSD_BF16 ? 2 : 4;
    if (ntok > 0) {
        if (!x || !dt || !B || !C || !y) return fail(SSD_ERR_NULL, "x, dt, B, C and y are required");
        if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y))
            return fail(SSD_ERR_SHAPE, "x, B, C and y must be 16-byte aligned");
        const size_t nx = (size_t)ntok * H * P * es, nbc = (size_t)ntok * G * N * es;
        const size_t ndt = (size_t)ntok * H * es;
        if (overlaps(y, nx, x, nx) || overlaps(y, nx, B, nbc) || overlaps(y, nx, C, nbc) ||
            overlaps(y, nx, dt, ndt))
            return fail(SSD_ERR_SHAPE, "y overlaps an input");
    }
    nstate = (size_t)S * H * N * P * sizeof(float);
    if ((init_state && !aligned16(init_state)) || (final_state && !aligned16(final_state)))
        return fail(SSD_ERR_SHAPE, "init_state and final_state must be 16-byte aligned");
    if (init_state && final_state && init_state != final_state &&
        overlaps(init_state, nstate, final_state, nstate))
        return fail(SSD_ERR_SHAPE, "final_state partially overlaps init_state");

    a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G; a.S = S;
    a.dtype = dims->dtype; a.Q = chunk;
    a.x = x; a.dt = dt; a.B = B; a.C = C;
    a.dt_bias = dt_bias; a.A = A; a.D = D; a.init_state = init_state; a.seq_idx = seq_idx;
    a.y = y; a.final_state = final_state;
    max_chunks = seq_idx ? (L + chunk - 1) / chunk + S : b * ((L + chunk - 1) / chunk);
    return SSD_OK;
}

// A scan with no tokens (or no sequences): final_state = init_state (or zero).
int empty_scan(const ssd::ScanArgs& a, size_t nstate, cudaStream_t st) {
    if (a.final_state && a.S > 0) {
        cudaError_t e = a.init_state
            ? (a.init_state == a.final_state ? cudaSuccess
                                             : cudaMemcpyAsync(a.final_state, a.init_state, nstate,
                                                               cudaMemcpyDeviceToDevice, st))
            : cudaMemsetAsync(a.final_state, 0, nstate, st);
        if (e != cudaSuccess) return cuda_fail("empty-input state copy", e);
    }
    return debug_check() ? debug_sync(st, nullptr) : SSD_OK;
}

// Bytes of scratch a scan needs besides its path's own workspace: the status
// word and, for packed input, the sequence table (start, end, chunk offsets).
size_t scan_table_bytes(const ssd::ScanArgs& a) {
    size_t n = Carve::round(sizeof(int32_t));
    if (a.seq_idx) n += 3 * Carve::round(sizeof(int32_t) * (a.S + 1));
    return n;
}

// Carves the status word and the sequence table out of `cv` (after the path's
// workspace), fills the sequence description *out and, for packed input,
// launches the kernels that build the table.  Returns an ssd_status.
int scan_tables(const ssd::ScanArgs& a, Carve& cv, bool dbg, int32_t** status, ssd::SeqInfo* out,
                cudaStream_t st) {
    *status = (int32_t*)cv.take(sizeof(int32_t));
    if (dbg) {
        cudaError_t e = cudaMemsetAsync(*status, 0, sizeof(int32_t), st);
        if (e != cudaSuccess) return cuda_fail("status word reset", e);
    }
    ssd::SeqInfo si;
    si.L = a.L; si.S = (int32_t)a.S; si.Q = a.Q; si.packed = a.seq_idx ? 1 : 0;
    si.nc_row = (int32_t)((a.L + a.Q - 1) / a.Q);
    si.start = si.end = si.chunk_off = nullptr;
    if (a.seq_idx) {
        int32_t* start = (int32_t*)cv.take(sizeof(int32_t) * (a.S + 1));
        int32_t* end = (int32_t*)cv.take(sizeof(int32_t) * (a.S + 1));
        int32_t* off = (int32_t*)cv.take(sizeof(int32_t) * (a.S + 1));
        ssd::launch_seq_table(a.seq_idx, a.L, (int32_t)a.S, a.Q, start, end, off, dbg ? *status : nullptr, st);
        si.start = start; si.end = end; si.chunk_off = off;
    }
    *out = si;
    return SSD_OK;
}

}  // namespace

extern "C" {

const char* ssd_status_string(int s) {
    switch (s) {
        case SSD_OK: return "ok";
        case SSD_ERR_NULL: return "a required pointer is NULL";
        case SSD_ERR_SHAPE: return "sizes out of range, inconsistent, overlapping or misaligned buffers";
        case SSD_ERR_DTYPE: return "unknown dtype";
        case SSD_ERR_CHUNK: return "chunk must be a power of two in [16, 256]";
        case SSD_ERR_UNSUPPORTED: return "request not supported by this library";
        case SSD_ERR_CUDA: return "CUDA error";
        case SSD_ERR_TIMEOUT: return "bounded device wait timed out";
        case SSD_ERR_SEQIDX: return "seq_idx breaks its contract";
        case SSD_ERR_RANGE: return "values outside the fp16 operand range of the tensor-core path";
        default: return "unknown status";
    }
}

const char* ssd_last_error(void) { return g_last_error; }

int ssd_chunk_scan_fwd(const ssd_dims* dims, const void* x, const void* dt, const float* dt_bias,
                       const float* A, const void* B, const void* C, const float* D,
                       const float* init_state, const int32_t* seq_idx, int chunk, void* y,
                       float* final_state, void* stream) {
    g_last_error[0] = 0;
    ssd::ScanArgs a;
    int64_t max_chunks = 0;
    size_t nstate = 0;
    int rc = prepare_scan(dims, x, dt, dt_bias, A, B, C, D, init_state, seq_idx, chunk, y, final_state, a,
                          max_chunks, nstate);
    if (rc) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();  // clear a stale error so it is not blamed on this call
    if (a.b * a.L == 0 || a.S == 0) return empty_scan(a, nstate, st);

    const bool use_tc = ssd::tc_supported(a);
    const size_t ws_path = use_tc ? ssd::tc_workspace_bytes(a, max_chunks)
                                  : ssd::simt_workspace_bytes(a, max_chunks);
    const bool dbg = debug_check();
    const bool value_check = dbg && use_tc;
    const size_t ws_bytes = Carve::round(ws_path) + scan_table_bytes(a) + (value_check ? Carve::round(16) : 0);

    Carve cv;
    cudaMemPool_t pool = workspace_pool();
    if (!pool) return fail(SSD_ERR_CUDA, "could not create the workspace memory pool");
    cudaError_t e = cudaMallocFromPoolAsync((void**)&cv.base, ws_bytes, pool, st);
    if (e != cudaSuccess) return cuda_fail("cudaMallocFromPoolAsync(workspace)", e);
    void* ws_main = cv.take(ws_path);
    int32_t* status = nullptr;
    ssd::SeqInfo si;
    rc = scan_tables(a, cv, dbg, &status, &si, st);
    if (rc) {
        cudaFreeAsync(cv.base, st);
        return rc;
    }
    uint32_t* counters = nullptr;
    if (value_check) {
        counters = (uint32_t*)cv.take(16);
        e = cudaMemsetAsync(counters, 0, 16, st);
        if (e != cudaSuccess) rc = cuda_fail("value-check reset", e);
        else ssd::launch_range_check_inputs(a, counters, st);
    }
    if (rc == SSD_OK) {
        if (use_tc)
            rc = ssd::launch_tc_scan(a, si, max_chunks, ws_main, dbg ? status : nullptr, st);
        else
            ssd::launch_simt_scan(a, si, max_chunks, ws_main, st);
    }
    if (rc == SSD_OK && value_check) ssd::launch_range_check_outputs(a, counters, st);
    e = cudaGetLastError();
    if (rc == SSD_OK && e != cudaSuccess) rc = cuda_fail("kernel launch", e);
    if (rc == SSD_OK && dbg) rc = debug_sync(st, status, counters);
    cudaError_t ef = cudaFreeAsync(cv.base, st);
    if (rc == SSD_OK && ef != cudaSuccess) rc = cuda_fail("cudaFreeAsync(workspace)", ef);
    return rc;
}

int ssd_state_update(const ssd_dims* dims, float* state, const void* x, const void* dt,
                     const float* A, const void* B, const void* C, const float* D, void* y,
                     void* stream, const float* dt_bias) {
    g_last_error[0] = 0;
    if (!dims) return fail(SSD_ERR_NULL, "dims is NULL");
    int rc = check_sizes(dims);
    if (rc) return rc;
    const int64_t b = dims->batch, H = dims->nheads, P = dims->headdim, N = dims->dstate;
    if (b == 0) return SSD_OK;
    if (!state || !x || !dt || !A || !B || !C || !y)
        return fail(SSD_ERR_NULL, "state, x, dt, A, B, C and y are required");
    if (!aligned16(state) || !aligned16(x) || !aligned16(y))
        return fail(SSD_ERR_SHAPE, "state, x and y must be 16-byte aligned");
    const size_t es = dims->dtype == SSD_BF16 ? 2 : 4;
    if (overlaps(y, (size_t)b * H * P * es, state, (size_t)b * H * N * P * 4) ||
        overlaps(y, (size_t)b * H * P * es, x, (size_t)b * H * P * es))
        return fail(SSD_ERR_SHAPE, "y overlaps state or x");
    // the decode grid has up to b H P / 16 blocks
    if (b * H > 0x7fffffffLL / 16) return fail(SSD_ERR_SHAPE, "batch * nheads too large");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::UpdateArgs a;
    a.b = b; a.H = H; a.P = P; a.N = N; a.G = dims->ngroups; a.dtype = dims->dtype;
    a.state = state; a.x = x; a.dt = dt; a.B = B; a.C = C; a.A = A; a.D = D; a.dt_bias = dt_bias;
    a.y = y;
    ssd::launch_state_update(a, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kernel launch", e);
    if (debug_check()) return debug_sync(st, nullptr);
    return SSD_OK;
}

}  // extern "C"

// ---- Sequence-parallel state passing ---------------------------------------------------

extern "C" int ssd_segment_logdecay(const ssd_dims* dims, const void* dt, const float* dt_bias, const float* A,
                                    float* out, void* stream) {
    g_last_error[0] = 0;
    if (!dims) return fail(SSD_ERR_NULL, "dims is NULL");
    int rc = check_sizes(dims);
    if (rc) return rc;
    const int64_t b = dims->batch, L = dims->seqlen, H = dims->nheads;
    if (L < 0) return fail(SSD_ERR_SHAPE, "seqlen %lld < 0", (long long)L);
    if (b == 0) return SSD_OK;
    if (!A || !out || (L > 0 && !dt)) return fail(SSD_ERR_NULL, "dt, A and out are required");
    if (b * H > 0x7fffffffLL) return fail(SSD_ERR_SHAPE, "batch * nheads too large");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::launch_segment_logdecay(b, L, H, dims->dtype, dt, dt_bias, A, out, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kernel launch", e);
    return debug_check() ? debug_sync(st, nullptr) : SSD_OK;
}

extern "C" int ssd_state_chain(const ssd_dims* dims, const float* h_in, const float* logdecay, const float* F,
                               float* h_out, void* stream) {
    g_last_error[0] = 0;
    if (!dims) return fail(SSD_ERR_NULL, "dims is NULL");
    int rc = check_sizes(dims);
    if (rc) return rc;
    const int64_t b = dims->batch, H = dims->nheads, NP = dims->dstate * dims->headdim;
    if (b == 0) return SSD_OK;
    if (!h_in || !logdecay || !F || !h_out) return fail(SSD_ERR_NULL, "h_in, logdecay, F and h_out are required");
    if (!aligned16(h_in) || !aligned16(F) || !aligned16(h_out))
        return fail(SSD_ERR_SHAPE, "h_in, F and h_out must be 16-byte aligned");
    const size_t ns = (size_t)b * H * NP * sizeof(float);
    if ((h_out != h_in && overlaps(h_out, ns, h_in, ns)) || (h_out != F && overlaps(h_out, ns, F, ns)) ||
        overlaps(h_out, ns, logdecay, (size_t)b * H * sizeof(float)))
        return fail(SSD_ERR_SHAPE, "h_out partially overlaps an input");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::launch_state_chain(b * H, NP, h_in, logdecay, F, h_out, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kernel launch", e);
    return debug_check() ? debug_sync(st, nullptr) : SSD_OK;
}

// ---- Backward of the scan -------------------------------------------------------------

extern "C" int ssd_group_norm(int64_t rows, int64_t channels, int64_t ngroups, int dtype, const void* x,
                              const float* gamma, const float* beta, float eps, void* out, void* stream) {
    g_last_error[0] = 0;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return fail(SSD_ERR_DTYPE, "dtype %d is not SSD_F32 or SSD_BF16", dtype);
    if (rows < 0 || channels < 1) return fail(SSD_ERR_SHAPE, "rows must be >= 0 and channels >= 1");
    if (!ssd::group_norm_supported(channels, ngroups))
        return fail(SSD_ERR_SHAPE, "ngroups must divide channels, with at most 2048 channels per group");
    if (rows == 0) return SSD_OK;
    if (!x || !gamma || !beta || !out) return fail(SSD_ERR_NULL, "x, gamma, beta and out are required");
    if (!(eps >= 0.f)) return fail(SSD_ERR_SHAPE, "eps must be >= 0");
    if (rows * ngroups > 0x7fffffffLL / 32) return fail(SSD_ERR_SHAPE, "rows * ngroups too large");
    const size_t es = dtype == SSD_BF16 ? 2 : 4, n = (size_t)rows * channels * es;
    if (overlaps(out, n, x, n) && out != x) return fail(SSD_ERR_SHAPE, "out overlaps x without being x");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::launch_group_norm(dtype, x, gamma, beta, eps, rows, channels, ngroups, out, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kernel launch", e);
    return debug_check() ? debug_sync(st, nullptr) : SSD_OK;
}

namespace {
int quant_shape(int64_t T, int64_t D, int64_t Tp) {
    if (T < 0 || D < 1 || Tp < 1 || Tp > 64) return fail(SSD_ERR_SHAPE, "need T >= 0, D >= 1, 1 <= ranks <= 64");
    if (D % (64 * Tp)) return fail(SSD_ERR_SHAPE, "D (%lld) must be a multiple of 64 * ranks", (long long)D);
    if (T * (D / 64) > 0x7fffffffLL / 32) return fail(SSD_ERR_SHAPE, "T * D too large");
    return SSD_OK;
}
int launched(cudaStream_t st) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kernel launch", e);
    return debug_check() ? debug_sync(st, nullptr) : SSD_OK;
}
}  // namespace

extern "C" int ssd_quant_chunks(int64_t T, int64_t D, int64_t ranks, const float* x, int8_t* q, float* scale,
                                void* stream) {
    g_last_error[0] = 0;
    int rc = quant_shape(T, D, ranks);
    if (rc || T == 0) return rc;
    if (!x || !q || !scale) return fail(SSD_ERR_NULL, "x, q and scale are required");
    if (!aligned16(x) || !aligned16(q) || !aligned16(scale)) return fail(SSD_ERR_SHAPE, "x, q and scale must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::launch_quant_chunks(x, T, D, ranks, q, scale, st);
    return launched(st);
}

extern "C" int ssd_dequant_sum_quant(int64_t T, int64_t Dc, int64_t ranks, const int8_t* q_in, const float* scale_in,
                                     int8_t* q_out, float* scale_out, void* stream) {
    g_last_error[0] = 0;
    int rc = quant_shape(T, Dc, 1);
    if (rc || T == 0) return rc;
    if (ranks < 1 || ranks > 64) return fail(SSD_ERR_SHAPE, "1 <= ranks <= 64");
    if (!q_in || !scale_in || !q_out || !scale_out) return fail(SSD_ERR_NULL, "all buffers are required");
    if (!aligned16(q_in) || !aligned16(q_out) || !aligned16(scale_in) || !aligned16(scale_out))
        return fail(SSD_ERR_SHAPE, "codes and scales must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::launch_dequant_sum_quant(q_in, scale_in, ranks, T, Dc, q_out, scale_out, st);
    return launched(st);
}

extern "C" int ssd_dequant_chunks(int64_t T, int64_t D, int64_t ranks, int dtype, const int8_t* q, const float* scale,
                                  void* out, void* stream) {
    g_last_error[0] = 0;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return fail(SSD_ERR_DTYPE, "dtype %d is not SSD_F32 or SSD_BF16", dtype);
    int rc = quant_shape(T, D, ranks);
    if (rc || T == 0) return rc;
    if (!q || !scale || !out) return fail(SSD_ERR_NULL, "q, scale and out are required");
    if (!aligned16(q) || !aligned16(scale) || !aligned16(out)) return fail(SSD_ERR_SHAPE, "q, scale and out must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    ssd::launch_dequant_chunks(dtype, q, scale, ranks, T, D / ranks, out, st);
    return launched(st);
}

extern "C" int ssd_state_to_output(const ssd_dims* dims, const void* dt, const float* dt_bias, const float* A,
                                   const void* C, const float* h_in, void* y, void* stream) {
    g_last_error[0] = 0;
    if (!dims) return fail(SSD_ERR_NULL, "dims is NULL");
    int rc = check_sizes(dims);
    if (rc) return rc;
    if (dims->nseqs) return fail(SSD_ERR_UNSUPPORTED, "packed sequences (nseqs > 0) are not taken by this call");
    const int64_t b = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim, N = dims->dstate,
                  G = dims->ngroups;
    if (L < 0) return fail(SSD_ERR_SHAPE, "seqlen %lld < 0", (long long)L);
    if (b * L == 0) return SSD_OK;
    if (!dt || !A || !C || !h_in || !y) return fail(SSD_ERR_NULL, "dt, A, C, h_in and y are required");
    ssd::ScanArgs a{};
    a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G; a.S = b; a.dtype = dims->dtype; a.Q = 128;
    a.dt = dt; a.C = C; a.dt_bias = dt_bias; a.A = A; a.y = y;
    if (!ssd::state_out_supported(a))
        return fail(SSD_ERR_UNSUPPORTED, "needs bfloat16 inputs, headdim 64 and dstate 128 (tensor-core path)");
    if (!aligned16(C) || !aligned16(h_in) || !aligned16(y))
        return fail(SSD_ERR_SHAPE, "C, h_in and y must be 16-byte aligned");
    const size_t ny = (size_t)b * L * H * P * 2;
    if (overlaps(y, ny, dt, (size_t)b * L * H * 2) || overlaps(y, ny, C, (size_t)b * L * G * N * 2) ||
        overlaps(y, ny, h_in, (size_t)b * H * N * P * 4))
        return fail(SSD_ERR_SHAPE, "y overlaps dt, C or h_in");
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    const bool dbg = debug_check();
    const size_t ws_path = ssd::state_out_workspace_bytes(a);
    Carve cv;
    cudaMemPool_t pool = workspace_pool();
    if (!pool) return fail(SSD_ERR_CUDA, "could not create the workspace memory pool");
    cudaError_t e = cudaMallocFromPoolAsync((void**)&cv.base, Carve::round(ws_path) + Carve::round(16), pool, st);
    if (e != cudaSuccess) return cuda_fail("cudaMallocFromPoolAsync(workspace)", e);
    void* ws = cv.take(ws_path);
    int32_t* status = (int32_t*)cv.take(16);
    if (dbg) {
        e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
        if (e != cudaSuccess) rc = cuda_fail("status reset", e);
    }
    if (rc == SSD_OK) rc = ssd::launch_state_to_output(a, h_in, ws, dbg ? status : nullptr, st);
    e = cudaGetLastError();
    if (rc == SSD_OK && e != cudaSuccess) rc = cuda_fail("kernel launch", e);
    if (rc == SSD_OK && dbg) rc = debug_sync(st, status);
    cudaError_t ef = cudaFreeAsync(cv.base, st);
    if (rc == SSD_OK && ef != cudaSuccess) rc = cuda_fail("cudaFreeAsync(workspace)", ef);
    return rc;
}

extern "C" int ssd_chunk_scan_bwd(const ssd_dims* dims, const void* x, const void* dt, const float* dt_bias,
                                  const float* A, const void* B, const void* C, const float* D,
                                  const float* init_state, const int32_t* seq_idx, int chunk, const void* dy,
                                  const float* dfinal, void* dx, void* ddt, float* ddt_bias, float* dA,
                                  void* dB, void* dC, float* dD, float* dinit, void* stream) {
    g_last_error[0] = 0;
    ssd::ScanArgs a;
    int64_t max_chunks = 0;
    size_t nstate = 0;
    // the forward's validation, with dx in the place of y and dinit in that of final_state
    int rc = prepare_scan(dims, x, dt, dt_bias, A, B, C, D, init_state, seq_idx, chunk, dx, dinit, a,
                          max_chunks, nstate);
    if (rc) return rc;
    if (!ddt_bias || !dA || !dD) return fail(SSD_ERR_NULL, "ddt_bias, dA and dD are required");
    const int64_t ntok = a.b * a.L;
    const size_t es = a.dtype == SSD_BF16 ? 2 : 4;
    if (ntok > 0) {
        if (!dy || !ddt || !dB || !dC) return fail(SSD_ERR_NULL, "dy, ddt, dB and dC are required");
        if (!aligned16(dy)) return fail(SSD_ERR_SHAPE, "dy must be 16-byte aligned");
        const size_t nx = (size_t)ntok * a.H * a.P * es, nbc = (size_t)ntok * a.G * a.N * es;
        const size_t ndt = (size_t)ntok * a.H * es;
        const void* outs[4] = {dx, ddt, dB, dC};
        const size_t nout[4] = {nx, ndt, nbc, nbc};
        const void* ins[5] = {x, dt, B, C, dy};
        const size_t nin[5] = {nx, ndt, nbc, nbc, nx};
        for (int i = 0; i < 4; ++i) {
            for (int k = 0; k < 5; ++k)
                if (overlaps(outs[i], nout[i], ins[k], nin[k])) return fail(SSD_ERR_SHAPE, "a gradient overlaps an input");
            for (int k = i + 1; k < 4; ++k)
                if (overlaps(outs[i], nout[i], outs[k], nout[k])) return fail(SSD_ERR_SHAPE, "two gradients overlap");
        }
    }
    if (dfinal && !aligned16(dfinal)) return fail(SSD_ERR_SHAPE, "dfinal must be 16-byte aligned");
    if (!ssd::bwd_supported(a))
        return fail(SSD_ERR_UNSUPPORTED,
                    "the backward handles headdim dividing 256 and headdim * dstate a power-of-two multiple of "
                    "256 up to 8192 (got headdim %lld, dstate %lld)", (long long)a.P, (long long)a.N);
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (ntok == 0 || a.S == 0) {
        cudaError_t e = cudaMemsetAsync(ddt_bias, 0, sizeof(float) * a.H, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dA, 0, sizeof(float) * a.H, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dD, 0, sizeof(float) * a.H, st);
        if (e == cudaSuccess && dinit && a.S > 0)
            e = dfinal ? cudaMemcpyAsync(dinit, dfinal, nstate, cudaMemcpyDeviceToDevice, st)
                       : cudaMemsetAsync(dinit, 0, nstate, st);
        if (e != cudaSuccess) return cuda_fail("empty-input gradients", e);
        return debug_check() ? debug_sync(st, nullptr) : SSD_OK;
    }
    // sequence tables with 64-token blocks (the backward's checkpoint spacing)
    ssd::ScanArgs a64 = a;
    a64.Q = 64;
    const bool dbg = debug_check();
    const size_t ws_path = ssd::bwd_workspace_bytes(a);
    const size_t ws_bytes = Carve::round(ws_path) + scan_table_bytes(a64);
    Carve cv;
    cudaMemPool_t pool = workspace_pool();
    if (!pool) return fail(SSD_ERR_CUDA, "could not create the workspace memory pool");
    cudaError_t e = cudaMallocFromPoolAsync((void**)&cv.base, ws_bytes, pool, st);
    if (e != cudaSuccess) return cuda_fail("cudaMallocFromPoolAsync(workspace)", e);
    void* ws_main = cv.take(ws_path);
    int32_t* status = nullptr;
    ssd::SeqInfo si;
    rc = scan_tables(a64, cv, dbg, &status, &si, st);
    if (rc == SSD_OK) {
        ssd::BwdArgs g;
        g.dy = dy; g.dfinal = dfinal; g.dx = dx; g.ddt = ddt; g.dB = dB; g.dC = dC;
        g.ddt_bias = ddt_bias; g.dA = dA; g.dD = dD; g.dinit = dinit;
        rc = ssd::launch_scan_bwd(a, g, si, ws_main, st);
        if (rc) rc = fail(SSD_ERR_CUDA, "could not clear the gradient accumulators");
    }
    e = cudaGetLastError();
    if (rc == SSD_OK && e != cudaSuccess) rc = cuda_fail("kernel launch", e);
    if (rc == SSD_OK && dbg) rc = debug_sync(st, status);
    cudaError_t ef = cudaFreeAsync(cv.base, st);
    if (rc == SSD_OK && ef != cudaSuccess) rc = cuda_fail("cudaFreeAsync(workspace)", ef);
    return rc;
}

// ---- Self-test of the bounded device waits -------------------------------------------

extern "C" int ssd_selftest_bounded_wait(int64_t limit_cycles, void* stream) {
    g_last_error[0] = 0;
    if (limit_cycles < 1000 || limit_cycles > 4000000000LL)
        return fail(SSD_ERR_SHAPE, "limit_cycles %lld outside [1000, 4e9]", (long long)limit_cycles);
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    cudaMemPool_t pool = workspace_pool();
    if (!pool) return fail(SSD_ERR_CUDA, "could not create the workspace memory pool");
    int32_t* status = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync((void**)&status, 256, pool, st);
    if (e != cudaSuccess) return cuda_fail("cudaMallocFromPoolAsync(status)", e);
    int rc = SSD_OK;
    e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) rc = cuda_fail("status reset", e);
    if (rc == SSD_OK) {
        ssd::launch_selftest_wait((long long)limit_cycles, status, st);
        e = cudaGetLastError();
        if (e != cudaSuccess) rc = cuda_fail("kernel launch", e);
    }
    if (rc == SSD_OK) rc = debug_sync(st, status);   // waits for the kernel, reads the status word
    cudaError_t ef = cudaFreeAsync(status, st);
    if (rc == SSD_OK && ef != cudaSuccess) rc = cuda_fail("cudaFreeAsync(status)", ef);
    return rc;
}

// ---- Scan without any device allocation ---------------------------------------------
//
// Some callers cannot let a library allocate device memory: a serving engine
// that has already handed nearly all of HBM to its own pool (so a
// stream-ordered allocation inside the call fails or forces memory back out
// of that pool), or a caller that forbids allocation after start-up to keep latency
// predictable.  ssd_chunk_scan_fwd_noalloc serves them: it runs the CUDA-core
// scan with its scratch (per-chunk states, chunk decays, packed-sequence
// table, status word) placed in the fixed-size array below instead of a
// stream-ordered allocation.

// Scratch limit of the no-allocation scan, in bytes (32 MiB).  The array is
// part of the library's device image: every GPU that uses the entry point
// holds it from its first use until the process exits.
static constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return fail(SSD_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(no-alloc scratch)", e);
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return SSD_OK;
}

}  // namespace

extern "C" int ssd_chunk_scan_fwd_noalloc(const ssd_dims* dims, const void* x, const void* dt,
                                          const float* dt_bias, const float* A, const void* B,
                                          const void* C, const float* D, const float* init_state,
                                          const int32_t* seq_idx, int chunk, void* y,
                                          float* final_state, void* stream) {
    g_last_error[0] = 0;
    ssd::ScanArgs a;
    int64_t max_chunks = 0;
    size_t nstate = 0;
    int rc = prepare_scan(dims, x, dt, dt_bias, A, B, C, D, init_state, seq_idx, chunk, y, final_state, a,
                          max_chunks, nstate);
    if (rc) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (a.b * a.L == 0 || a.S == 0) return empty_scan(a, nstate, st);

    const size_t ws_path = ssd::simt_workspace_bytes(a, max_chunks);
    const size_t need = Carve::round(ws_path) + scan_table_bytes(a);
    if (need > kNoAllocScratchBytes)
        return fail(SSD_ERR_UNSUPPORTED,
                    "this call needs %zu bytes of scratch; the no-allocation scan is limited to %zu "
                    "bytes (32 MiB): use ssd_chunk_scan_fwd",
                    need, kNoAllocScratchBytes);

    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    cudaGetLastError();
    Carve cv;
    cv.base = (char*)scratch;
    void* ws_main = cv.take(ws_path);
    const bool dbg = debug_check();
    int32_t* status = nullptr;
    ssd::SeqInfo si;
    rc = scan_tables(a, cv, dbg, &status, &si, st);
    if (rc) return rc;
    ssd::launch_simt_scan(a, si, max_chunks, ws_main, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kernel launch", e);
    if (dbg) return debug_sync(st, status);
    return SSD_OK;
}
