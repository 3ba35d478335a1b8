/*
 * ssd.h -- C ABI of libssd.so: the selective state-space (Mamba-2 SSD) scan
 * forward and the single-token decode state update, for NVIDIA B200 (sm_100a).
 *
 * The operation (sources: "5.3 Tensor Parallelism support and large-cluster
 * training", sections 2.1, 3.1, 3.2, 4.3; "Scaling State-Space Models on
 * Multiple GPUs with Tensor Parallelism", abstract):
 *
 *   d_t  = softplus(dt_t + dt_bias_h)                    (per token, head)
 *   h_t  = exp(d_t * A_h) * h_{t-1} + d_t * B_t x_t^T    (N x P state per head;
 *                                                         A_t = a_t I, sec. 3.1)
 *   y_t  = C_t^T h_t + D_h * x_t
 *
 * ssd_chunk_scan_fwd evaluates it over whole sequences in the block-decomposed
 * (chunked) form of section 3.2: a quadratic form inside each chunk, N x P
 * states handed from chunk to chunk.  ssd_state_update applies one step to a
 * cached state (prefill -> decode state cache, second page's abstract).
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers to caller-owned, contiguous,
 *     row-major memory on the current CUDA device.  The library never frees or
 *     keeps them.  Scalar-per-head arrays (dt_bias, A, D) are float32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream and do not synchronise, except when
 *     the environment variable SSD_DEBUG_CHECK=1 is set (then each call waits
 *     for its kernels and reports device-side errors).
 *   - Argument errors are detected on the host, before anything is launched,
 *     and returned as an ssd_status; no exception crosses the ABI.
 *   - The library keeps no data between calls and is reentrant.  Temporary
 *     device memory is taken stream-ordered on `stream` (cudaMallocFromPoolAsync
 *     / cudaFreeAsync) from a memory pool the library creates per device on
 *     first use.  The pool keeps freed workspace mapped for later calls (it
 *     holds at most the largest workspace in flight, until the process exits)
 *     so that a call after a synchronisation does not map it again.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of x, dt, B, C and y.  A, D, dt_bias and all states are float32
 * in both modes; accumulation is float32. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

typedef enum {
    SSD_OK = 0,
    SSD_ERR_NULL = 1,        /* a required pointer is NULL                          */
    SSD_ERR_SHAPE = 2,       /* sizes out of the supported range or inconsistent    */
    SSD_ERR_DTYPE = 3,       /* dtype is not an ssd_dtype value                     */
    SSD_ERR_CHUNK = 4,       /* chunk is not a power of two in [16, 256]            */
    SSD_ERR_UNSUPPORTED = 5, /* valid request the library does not implement       */
    SSD_ERR_CUDA = 6,        /* a CUDA call failed; see ssd_last_error()            */
    SSD_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up (debug check)     */
    SSD_ERR_SEQIDX = 8,      /* seq_idx breaks its contract (debug check only)       */
    SSD_ERR_RANGE = 9        /* values outside the tensor-core path's fp16 operand
                                range (debug check only; see ssd_chunk_scan_fwd)    */
} ssd_status;

/* Problem sizes.  b = batch, L = seqlen, H = nheads, P = headdim, N = dstate,
 * G = ngroups (head h uses group h / (H / G)), nseqs = number of packed
 * sequences when seq_idx is given (ignored otherwise). */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, nseqs;
    int32_t dtype; /* ssd_dtype */
} ssd_dims;

/*
 * ssd_chunk_scan_fwd -- whole-sequence scan, chunked (SSD block decomposition,
 * "5.3 Tensor Parallelism ...", section 3.2).
 *
 *   x          (b, L, H, P)   dtype            required
 *   dt         (b, L, H)      dtype            required; raw, before softplus
 *   dt_bias    (H)            float32          NULL = 0
 *   A          (H)            float32          required; the per-head scalar a of A = a I
 *   B, C       (b, L, G, N)   dtype            required
 *   D          (H)            float32          NULL = no skip term
 *   init_state (S, H, N, P)   float32          NULL = zero initial state
 *   seq_idx    (L)            int32            NULL = each batch row is one sequence.
 *              Otherwise batch must be 1 and the row packs nseqs sequences:
 *              seq_idx is non-decreasing, starts at 0, moves in steps of 0 or
 *              +1 and ends at nseqs - 1.  The state is reset at the first token
 *              of every sequence ("A_t = 0" at sequence ends, section 4.3) and
 *              restarted from init_state[s].  A seq_idx that breaks the contract
 *              gives unspecified values but never an out-of-bounds access; with
 *              SSD_DEBUG_CHECK=1 it is reported as SSD_ERR_SEQIDX.
 *   chunk      power of two in [16, 256]: the block length Q of the
 *              decomposition.  Results do not depend on it beyond rounding.
 *   y          (b, L, H, P)   dtype            required; must not alias an input
 *   final_state(S, H, N, P)   float32          NULL = not written; may alias
 *              init_state exactly (in-place continuation)
 *   S = nseqs when seq_idx is given, else b.
 *
 * Supported sizes: P and N multiples of 16 with 16 <= P, N <= 256; H % G == 0;
 * b, L >= 0 (empty inputs are a no-op apart from final_state = init_state).
 *
 * Value range.  bf16 calls with P = 64, N in {128, 256} and chunk in {128, 256}
 * run on the tensor cores, whose operands are fp16 (11-bit significand, largest
 * finite value 65504) with fp32 accumulation; every other call runs on CUDA
 * cores in fp32.  On the tensor-core path:
 *   - every x, B, C and init_state value must be finite with magnitude at most
 *     65504 (a larger bf16 value cannot be represented and becomes inf);
 *   - the masked score matrix (C_j . B_i) exp(sum of d A from i+1 to j) d_i and
 *     the state carried between 128-token tiles must also stay within 65504
 *     in magnitude (for N(0,1) inputs of the sizes above they stay below ~20,
 *     so B and C may grow ~58x, x and the state ~2e4x, before this binds).
 * Outside these limits the result holds inf or NaN where the recurrence is
 * finite.  With SSD_DEBUG_CHECK=1 such calls return SSD_ERR_RANGE: an input
 * beyond 65504, or a non-finite y / final_state from finite inputs.
 * Returns an ssd_status.
 */
SSD_API int ssd_chunk_scan_fwd(const ssd_dims* dims, const void* x, const void* dt, const float* dt_bias,
                       const float* A, const void* B, const void* C, const float* D,
                       const float* init_state, const int32_t* seq_idx, int chunk, void* y,
                       float* final_state, void* stream);

/*
 * ssd_state_update -- one decode step on a cached state, in place (the
 * prefill -> decode state cache of "Scaling State-Space Models on Multiple GPUs
 * with Tensor Parallelism", abstract; same recurrence as above for one token).
 *
 *   state   (b, H, N, P)  float32   in/out, required
 *   x       (b, H, P)     dtype     required
 *   dt      (b, H)        dtype     required; raw, same meaning as in the scan
 *   A       (H)           float32   required
 *   B, C    (b, G, N)     dtype     required
 *   D       (H)           float32   NULL = no skip term
 *   y       (b, H, P)     dtype     required
 *   dt_bias (H)           float32   NULL = 0.  Last so that the leading
 *           arguments keep the order of the problem statement; it must be the
 *           same bias the prefill scan used for the continuation to be exact.
 * Uses dims->batch, nheads, headdim, dstate, ngroups, dtype (seqlen, nseqs ignored).
 * state, x and y must be 16-byte aligned (SSD_ERR_SHAPE otherwise).
 */
SSD_API int ssd_state_update(const ssd_dims* dims, float* state, const void* x, const void* dt,
                     const float* A, const void* B, const void* C, const float* D, void* y,
                     void* stream, const float* dt_bias);

/*
 * Sequence-parallel state passing ("5.3 Tensor Parallelism ...", section 4.2:
 * a long sequence split over devices, the N x P state handed from each device
 * to the next).  A slice scanned from a zero state (final state F) leaves the
 * state h_out = exp(D) h_in + F for a state h_in entering it, with D its total
 * log-decay; these two calls compute D and that step, on the device.  The
 * slice's own output then misses only the part that comes from h_in, which
 * ssd_state_to_output adds.
 *
 * ssd_segment_logdecay -- D[b, h] = sum_t softplus(dt[b, t, h] + dt_bias_h) A_h
 *   dt (b, L, H) dtype of dims; dt_bias (H) float32, NULL = 0; A (H) float32;
 *   out (b, H) float32.  Uses dims->batch, seqlen, nheads, dtype.
 * ssd_state_chain -- h_out = exp(logdecay) h_in + F per (batch, head)
 *   h_in, F, h_out (b, H, N, P) float32, 16-byte aligned; logdecay (b, H)
 *   float32.  h_out may alias h_in or F exactly.  Uses dims->batch, nheads,
 *   headdim, dstate.
 */
SSD_API int ssd_segment_logdecay(const ssd_dims* dims, const void* dt, const float* dt_bias, const float* A,
                                 float* out, void* stream);
SSD_API int ssd_state_chain(const ssd_dims* dims, const float* h_in, const float* logdecay, const float* F,
                            float* h_out, void* stream);

/*
 * ssd_state_to_output -- the output of a state entering each row at its start
 * (the state-to-output term of "5.3 Tensor Parallelism ...", section 3.2,
 * measured from the row's first token):
 *   y[b, t, h, :] += exp(sum_{i <= t} softplus(dt[b, i, h] + dt_bias_h) A_h)
 *                    * sum_n C[b, t, g, n] h_in[b, h, n, :],   g = h / (H / G)
 * so that a scan of the row from a zero state plus this call equals the scan
 * from h_in (up to rounding: y is read as bf16 and written back as bf16).
 *   dt (b, L, H), C (b, L, G, N), y (b, L, H, P): bfloat16; y is read and
 *   written in place.  h_in (b, H, N, P), A (H) float32; dt_bias (H) float32,
 *   NULL = 0.  C, h_in and y 16-byte aligned; y must not overlap the inputs.
 * Runs on the tensor cores (C and h_in rounded to fp16 operands, fp32
 * accumulation; the value range of ssd_chunk_scan_fwd applies): dtype
 * SSD_BF16, headdim 64 and dstate 128 only, SSD_ERR_UNSUPPORTED otherwise, and
 * for nseqs > 0.  Workspace (stream-ordered, from the library's pool):
 * 2 b L G N + 520 b H ceil(L / 128) bytes.  Uses dims->batch, seqlen, nheads,
 * headdim, dstate, ngroups, dtype.
 */
SSD_API int ssd_state_to_output(const ssd_dims* dims, const void* dt, const float* dt_bias, const float* A,
                                const void* C, const float* h_in, void* y, void* stream);

/*
 * Head-sharded (tensor-parallel) mixer ("5.3 Tensor Parallelism ...", section 4.1;
 * "Scaling State-Space Models on Multiple GPUs with Tensor Parallelism", abstract):
 * each of `ranks` devices holds H / ranks heads; the layer's output is the sum of
 * the devices' partial output projections, formed by a quantised all-reduce.
 *
 * ssd_group_norm -- out[r, c] = (x[r, c] - mean_g) / sqrt(var_g + eps) * gamma[c]
 *   + beta[c], mean_g and var_g (biased) over the channels of c's group in row r
 *   (ngroups groups of channels / ngroups consecutive channels, at most 2048).
 *   x, out (rows, channels) of dtype (SSD_F32 or SSD_BF16; out may be x);
 *   gamma, beta (channels) float32.  Statistics in fp32.
 *
 * The quantised all-reduce of (T, D) float32 partials over `ranks` devices, with
 * int8 codes and one float32 scale per block of 64 consecutive columns of a row
 * (scale = amax / 127 in fp32; code = rint(x * (127 / amax)) with round-half-even,
 * in [-127, 127]; 0 for an all-zero block).  Column chunk j = columns
 * [j D / ranks, (j + 1) D / ranks), Dc = D / ranks a multiple of 64:
 * ssd_quant_chunks -- x (T, D) float32 -> q (ranks, T, Dc) int8,
 *   scale (ranks, T, Dc / 64): chunk-major, so chunk j is contiguous (it goes to
 *   rank j in an all-to-all).
 * ssd_dequant_sum_quant -- the chunks from every rank, q_in (ranks, T, Dc) and
 *   scale_in (ranks, T, Dc / 64) -> their dequantised sum in float32 (added in
 *   rank order, each product and sum rounded separately) -> q_out (T, Dc),
 *   scale_out (T, Dc / 64).
 * ssd_dequant_chunks -- gathered chunks q (ranks, T, Dc), scale -> out (T, D) of
 *   dtype, out[t, j Dc + c] = scale * code (rounded once to dtype).
 * Every buffer 16-byte aligned; sizes and alignment checked on the host
 * (SSD_ERR_SHAPE).
 */
SSD_API int ssd_group_norm(int64_t rows, int64_t channels, int64_t ngroups, int dtype, const void* x,
                           const float* gamma, const float* beta, float eps, void* out, void* stream);
SSD_API int ssd_quant_chunks(int64_t T, int64_t D, int64_t ranks, const float* x, int8_t* q, float* scale,
                             void* stream);
SSD_API int ssd_dequant_sum_quant(int64_t T, int64_t Dc, int64_t ranks, const int8_t* q_in, const float* scale_in,
                                  int8_t* q_out, float* scale_out, void* stream);
SSD_API int ssd_dequant_chunks(int64_t T, int64_t D, int64_t ranks, int dtype, const int8_t* q, const float* scale,
                               void* out, void* stream);

/*
 * ssd_chunk_scan_bwd -- gradient of the scan (the backward of the training step
 * the pages describe: "5.3 Tensor Parallelism support and large-cluster
 * training", section 6.3 and Table 5.3.1; the pages print no gradient
 * formulas, these are the chain rule applied to the recurrence above).
 *
 * For the objective J = sum_t <dy_t, y_t> + <dfinal, final_state> it writes
 *   dx, ddt   dJ/dx (b, L, H, P) and dJ/d(raw dt) (b, L, H), dtype of x
 *   dB, dC    (b, L, G, N), dtype of x, summed over the heads of each group
 *   ddt_bias, dA, dD  (H) float32, summed over tokens and sequences
 *   dinit     (S, H, N, P) float32, dJ/d init_state (NULL = not written)
 * Inputs are those of ssd_chunk_scan_fwd with the same meaning, plus
 *   dy        (b, L, H, P)  dtype of x, required
 *   dfinal    (S, H, N, P)  float32, NULL = zero
 * chunk is validated as in the forward; the result does not depend on it.
 * Every output is overwritten (none is read).  Gradient buffers must not
 * overlap the inputs or each other; dy is 16-byte aligned like x (both
 * SSD_ERR_SHAPE otherwise).  blocks = the number of 64-token blocks over all
 * sequences.  headdim 64 with dstate 64 or 128: the block decomposition over
 * 64-token chunks (per-chunk terms, a sequential pass over chunk states,
 * per-chunk gradients; for bf16 the matrix products on the tensor cores with
 * fp16 operands and fp32 accumulation), workspace 8 N P H blocks + 4 H blocks
 * bytes, plus 8 K b L G N bytes of fp32 dB / dC partials when bf16 gradient
 * blocks split each group's heads K ways (K = 2 or 4, chosen from the block
 * count and the SM count to fill the last wave).  Other shapes: CUDA cores in fp32 with checkpoints of the state every
 * 64 tokens, workspace 4 N P H (blocks + 64 S) + 8 b L G N bytes; supported
 * there are headdim dividing 256 and headdim * dstate in {256, 512, ...,
 * 8192}, other shapes return SSD_ERR_UNSUPPORTED.  Workspace is stream-ordered,
 * from the library's pool (each piece rounded up to 256 bytes).
 */
SSD_API int ssd_chunk_scan_bwd(const ssd_dims* dims, const void* x, const void* dt, const float* dt_bias,
                               const float* A, const void* B, const void* C, const float* D,
                               const float* init_state, const int32_t* seq_idx, int chunk, const void* dy,
                               const float* dfinal, void* dx, void* ddt, float* ddt_bias, float* dA,
                               void* dB, void* dC, float* dD, float* dinit, void* stream);

/*
 * ssd_chunk_scan_fwd_noalloc -- the same scan, for callers that cannot let the
 * library allocate device memory (for example a serving engine that has
 * already given nearly all of HBM to its own pool, or a caller that forbids
 * allocation after start-up).  The pages have no counterpart to this call; it
 * is a deployment variant of ssd_chunk_scan_fwd.
 *
 * Arguments, layouts, ownership and validation are those of
 * ssd_chunk_scan_fwd; the caller still passes all inputs and outputs.  It
 * always runs the CUDA-core scan, whose scratch (per-chunk states, chunk
 * decays, packed-sequence table) lives in one fixed 32 MiB device array
 * inside the library instead of a stream-ordered pool block:
 *   - needed scratch = 4 * (chunks * H * (N * P + 1)) bytes plus a few KiB,
 *     rounded to 256-byte pieces, with chunks = b * ceil(L / chunk), or
 *     ceil(L / chunk) + nseqs when packed.  Larger calls are rejected with
 *     SSD_ERR_UNSUPPORTED before anything is launched (ssd_last_error() says
 *     how much was needed);
 *   - the array is part of the library's device code: every GPU on which that
 *     code is loaded holds it until the process exits (loaded at first use
 *     under CUDA's default lazy module loading, at context creation with
 *     CUDA_MODULE_LOADING=EAGER);
 *   - the first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture;
 *   - every call shares the one array, which keeps the previous call's
 *     contents.  Everything a call reads from it is written earlier by the
 *     same call, so stale contents do no harm; but calls that overlap on the
 *     GPU (concurrent streams, several host threads) race on it and must be
 *     serialised by the caller.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
SSD_API int ssd_chunk_scan_fwd_noalloc(const ssd_dims* dims, const void* x, const void* dt,
                                       const float* dt_bias, const float* A, const void* B,
                                       const void* C, const float* D, const float* init_state,
                                       const int32_t* seq_idx, int chunk, void* y,
                                       float* final_state, void* stream);

/* Static English text for an ssd_status value (never NULL). */
SSD_API const char* ssd_status_string(int status);

/* Detail of the last failure on the calling host thread (e.g. the CUDA error
 * text behind SSD_ERR_CUDA, or which argument was rejected); "" if none. */
SSD_API const char* ssd_last_error(void);

/*
 * Instrumentation.  No counterpart in the pages: these calls exist so that a
 * benchmark can time the library's own kernels on the stream they run on.
 *
 * Every kernel launch is counted.  While profiling is enabled, each launch is
 * also bracketed by two CUDA events recorded on its stream (recording adds no
 * device work, but costs a few microseconds of host time per launch).
 */
typedef struct {
    char name[48];      /* kernel name                                   */
    int64_t launches;   /* launches since the last reset                 */
    int64_t timed;      /* launches with a measured duration             */
    double total_ms;    /* summed event-measured duration of the timed   */
} ssd_kernel_stat;

/* on != 0 turns event timing on, 0 off.  Returns the previous setting. */
SSD_API int ssd_profile_enable(int on);

/*
 * Self-test of the bounded device waits.  Every mbarrier wait in the library's
 * kernels gives up after a bounded number of SM clock cycles, records the
 * timeout in a device status word and lets the kernel return.  This call runs
 * that same wait, on `stream`, in one thread waiting on an mbarrier that
 * nothing ever arrives at, with a limit of `limit_cycles` (1000 .. 4e9; about
 * 2e6 is a millisecond).  It then synchronises `stream` and reads the status
 * word.  Returns SSD_ERR_TIMEOUT when the path works (the wait ran out and was
 * reported), SSD_ERR_SHAPE for a limit out of range, SSD_ERR_CUDA on a CUDA
 * failure.  No fault, trap or hang is involved.
 */
SSD_API int ssd_selftest_bounded_wait(int64_t limit_cycles, void* stream);

/* Waits for the recorded events, folds them into the per-kernel totals and
 * copies up to max_entries entries (kernels launched at least once) into
 * out.  reset != 0 clears all counters afterwards.  Returns the number of
 * entries written, or -SSD_ERR_CUDA if an event could not be read. */
SSD_API int ssd_profile_read(ssd_kernel_stat* out, int max_entries, int reset);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
