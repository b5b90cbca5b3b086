/*
 * ssd.h -- C ABI of libssd, the Mamba-2 state space duality (SSD) layer for NVIDIA B200.
 *
 * The layer (per batch row and head h, group g = h / (nheads / ngroups)):
 *
 *     a_t      = exp(dt_t * A_h)
 *     h_t[p,n] = a_t * h_{t-1}[p,n] + dt_t * x_t[p] * B_t[g,n]
 *     y_t[p]   = sum_n C_t[g,n] * h_t[p,n] + D_h * x_t[p]
 *
 * Sources: "Engineering Hybrid State-Space Models" section 2 (the diagonal recurrence
 * h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t h_t with Abar_t = exp(dt_t A), and its
 * chunked semiseparable form Y = (M o C B^T) X); "Compiler-First State Space Duality and
 * Portable O(1) Autoregressive Caching for Inference" abstract (scalar per-head dynamics,
 * fixed-size chunking, a prefill that hands an O(1) cache to single-token decode);
 * "Mamba and Selective State Space Models" section 2 (the D x feedthrough).  The input
 * term is the Euler form dt_t * B_t (the first page's code section uses delta * x), not
 * the full zero-order-hold Bbar.
 *
 * Layouts (row-major, contiguous, no strides):
 *     x      [batch, seqlen, nheads, headdim]      dtype of the call (fp32 or bf16)
 *     dt     [batch, seqlen, nheads]               fp32, > 0 (not checked: device data)
 *     A      [nheads]                              fp32 (normally < 0)
 *     B, C   [batch, seqlen, ngroups, dstate]      dtype of the call
 *     D      [nheads]                              fp32
 *     y      [batch, seqlen, nheads, headdim]      fp32 (always, see below)
 *     state  [batch, nheads, headdim, dstate]      fp32
 * Decode drops the seqlen axis (x [batch, nheads, headdim], dt [batch, nheads], B and C
 * [batch, ngroups, dstate], y [batch, nheads, headdim]).
 *
 * y is written in fp32 for every input dtype: the layer's output is dominated by the
 * D x term, whose largest elements are many times its RMS, and rounding those to bf16
 * would by itself exceed a max-error bound of 2e-2 RMS.
 *
 * Conventions of every call:
 *   - All array pointers are DEVICE pointers on the current CUDA device, owned by the
 *     caller.  libssd never allocates or frees device memory, and keeps no state between
 *     calls that changes a result.  The one exception is ssd_prefill_noalloc: its scratch
 *     is a fixed device array inside the library (held on a device from its first use
 *     there), whose address it caches per CUDA context.  Host-side caches of encoded
 *     tensor maps and of per-device kernel attributes only save set-up time.  A pointer
 *     may be NULL only if its array has zero elements.
 *   - x, B, C, y, state, final_state and workspace must be 16-byte aligned; dt, A and D
 *     4-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream): they validate on the host, enqueue kernels and return.  On a validation
 *     error nothing is enqueued.  A launch failure is reported as SSD_ERR_CUDA.  No call
 *     aborts or prints, and none but ssd_prefill_device_status synchronises.
 *   - Inputs and outputs must not overlap, except as stated for ssd_decode_step.
 */
#ifndef LIBSSD_SSD_H_
#define LIBSSD_SSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *ssd_stream_t;

typedef enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1, /* NULL pointer, misalignment, bad sizes, nheads % ngroups != 0 */
  SSD_ERR_UNSUPPORTED = 2, /* valid but outside the compiled shape set (see below)        */
  SSD_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than ssd_prefill_workspace_size()  */
  SSD_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed                  */
  SSD_ERR_TIMEOUT = 5      /* a bounded device-side wait expired (ssd_prefill_device_status) */
} ssd_status;

typedef enum {
  SSD_F32 = 0, /* x, B, C in fp32; fp32 arithmetic throughout (no tensor cores)          */
  SSD_BF16 = 1 /* x, B, C in bf16; bf16 tensor-core products with fp32 accumulation      */
} ssd_dtype;

typedef struct {
  int64_t batch;   /* >= 0                                     */
  int64_t seqlen;  /* >= 0 (ignored by ssd_decode_step)        */
  int64_t nheads;  /* >= 1, multiple of ngroups                */
  int64_t headdim; /* P: 1 .. 256                              */
  int64_t dstate;  /* N: one of 16, 32, 64, 128, 256           */
  int64_t ngroups; /* >= 1                                     */
} ssd_dims;

/* Human-readable name of a status code (static storage; never NULL). */
SSD_API const char *ssd_status_string(ssd_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
SSD_API int ssd_version(void);

/*
 * Bytes of device workspace ssd_prefill needs for these arguments (0 if the arguments
 * are invalid or need none).  Depends only on the arguments.
 */
SSD_API size_t ssd_prefill_workspace_size(const ssd_dims *dims, ssd_dtype dtype, int chunk);

/*
 * Number of kernels one ssd_prefill call with these arguments enqueues (-1 if the
 * arguments are invalid).  For launch accounting only.
 */
SSD_API int ssd_prefill_kernel_launches(const ssd_dims *dims, ssd_dtype dtype, int chunk);

/*
 * Chunked prefill from a zero initial state.
 *
 * Computes y for every token of every sequence and writes the state after the last
 * token, h_{seqlen-1}, to final_state (all zeros when seqlen == 0).  `chunk` (Q) is the
 * chunk length of the chunked form: a power of two in [1, 256]; the result does not
 * depend on it beyond rounding ("Engineering Hybrid State-Space Models" section 2 uses
 * Q = 64).  seqlen need not be a multiple of chunk: the last chunk may be partial.
 *
 * Within each chunk the kernels compute the in-chunk cumulative log-decay, the chunk's
 * state contribution, carry the state across chunks, then form each token's output from
 * the masked decay-weighted C B^T product plus the carried-in state.
 *
 * workspace: device scratch of at least ssd_prefill_workspace_size() bytes, 16-byte
 * aligned, owned by the caller, contents on entry ignored and on return unspecified.
 * Calls that share a workspace must be ordered (same stream or synchronised).
 *
 * Errors: SSD_ERR_INVALID_ARG for NULL dims, NULL or misaligned non-empty arrays,
 * negative sizes, headdim outside 1..256, nheads % ngroups != 0, chunk not a power of
 * two in [1, 256]; SSD_ERR_UNSUPPORTED for a dstate outside {16,32,64,128,256};
 * SSD_ERR_WORKSPACE for a missing or short workspace; SSD_ERR_CUDA if a launch fails.
 */
SSD_API ssd_status ssd_prefill(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                       const float *A, const void *B, const void *C, const float *D,
                       int chunk, float *y, float *final_state, void *workspace,
                       size_t workspace_bytes, ssd_stream_t stream);

/*
 * ssd_prefill from a given initial state, optionally exporting the state at every chunk
 * boundary: the carried state of the chunked form ("Engineering Hybrid State-Space
 * Models" section 2), started from h_{-1} = initial_state instead of zero.  This lets a
 * long prompt be processed in pieces (pass one piece's final_state as the next piece's
 * initial_state) and a prefix cache keep the state at any chunk boundary.
 *
 *   initial_state  [batch, nheads, headdim, dstate] fp32, or NULL for a zero state.  It
 *                  may be the same array as final_state (then updated in place); it
 *                  must not overlap any other argument.
 *   chunk_states   [batch, nchunks, nheads, headdim, dstate] fp32 with
 *                  nchunks = ceil(seqlen / chunk), or NULL.  chunk_states[b][c] is the
 *                  state after token min((c + 1) * chunk, seqlen) - 1, so its last entry
 *                  equals final_state.  Written only when non-NULL.
 *
 * With both NULL this is exactly ssd_prefill.  When seqlen == 0, final_state is set to
 * initial_state (or zeros) and chunk_states is not touched.  Workspace, alignment (16
 * bytes for both optional arrays), asynchrony and errors as ssd_prefill;
 * SSD_ERR_INVALID_ARG also for a misaligned initial_state or chunk_states.
 */
SSD_API ssd_status ssd_prefill_ex(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                                  const float *A, const void *B, const void *C, const float *D, int chunk,
                                  const float *initial_state, float *y, float *final_state, float *chunk_states,
                                  void *workspace, size_t workspace_bytes, ssd_stream_t stream);

/*
 * ssd_prefill, with per-kernel timing for profiling harnesses.  `events` holds
 * num_events caller-created cudaEvent_t handles (cudaEventDefault flags, i.e. timing
 * enabled), num_events >= ssd_prefill_kernel_launches() + 1.  events[i] is recorded on
 * `stream` just before kernel i is enqueued and events[k] after the last of the k
 * kernels, so cudaEventElapsedTime(events[i], events[i+1]) is kernel i's duration.
 * Nothing is allocated and nothing synchronises.  Same computation, results and errors
 * as ssd_prefill, plus SSD_ERR_INVALID_ARG if events is NULL or too short.
 */
SSD_API ssd_status ssd_prefill_timed(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C, const float *D, int chunk,
                                     float *y, float *final_state, void *workspace, size_t workspace_bytes,
                                     ssd_stream_t stream, void *const *events, int num_events);

/*
 * Name of kernel i (0-based) of an ssd_prefill call with these arguments, in launch
 * order (static storage), or NULL if i is out of range or the arguments are invalid.
 */
SSD_API const char *ssd_prefill_kernel_name(const ssd_dims *dims, ssd_dtype dtype, int chunk, int i);

/*
 * Device-side status of the last ssd_prefill that used this workspace: synchronises
 * `stream`, then reads the workspace's error word.  SSD_ERR_TIMEOUT means a bounded
 * device-side wait inside the prefill kernels expired (the kernels then stop touching
 * data and exit; y and final_state are undefined); SSD_OK otherwise.  SSD_ERR_CUDA if
 * the copy or the synchronisation fails, SSD_ERR_INVALID_ARG for a NULL, misaligned or
 * too small workspace.  Unlike every other call, this one blocks the host.
 */
SSD_API ssd_status ssd_prefill_device_status(const void *workspace, size_t workspace_bytes, ssd_stream_t stream);

/*
 * ssd_prefill for callers that cannot allocate device memory.  Some callers cannot call
 * cudaMalloc or provide device memory of their own: plugins inside a host process whose
 * device allocator belongs to the host framework, and serving loops that forbid any
 * allocation once running.  This call takes no workspace: its scratch is a fixed array
 * of ssd_prefill_noalloc_max_workspace() bytes (32 MiB) compiled into the library.  It
 * computes exactly what ssd_prefill computes, with the same arguments otherwise.
 * (The pages describe no such call; it serves these callers only.)
 *
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.  The
 *     array is held on a device, until the process exits, from the first call on it.
 *   - The first call in a CUDA context (on a device, with its context current) looks
 *     up the array's device address there (cudaGetSymbolAddress) and caches it under the
 *     context's unique id; make that first call before any stream capture.  A new context
 *     (after cudaDeviceReset, or another one the caller made current) gets its own
 *     look-up, never a stale address.
 *   - A bounded device wait that expired is reported by
 *     ssd_prefill_noalloc_device_status, which reads the array's error word.
 *   - Every call shares the one array: calls whose executions overlap on the GPU (other
 *     streams, other host threads without ordering) race and give undefined results.
 *     Order them on one stream or synchronise between them.
 *   - Errors: as ssd_prefill; SSD_ERR_WORKSPACE if ssd_prefill_workspace_size() for these
 *     arguments exceeds the array (the 2.7B-shaped 4096-token layer needs more; the
 *     130M-shaped one fits).  SSD_ERR_CUDA if the address look-up fails.
 */
SSD_API ssd_status ssd_prefill_noalloc(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                                       const float *A, const void *B, const void *C, const float *D, int chunk,
                                       float *y, float *final_state, ssd_stream_t stream);

/*
 * Self-test of the bounded device-side waits (the library's own check; the pages describe
 * no such call).  Every mbarrier wait in the tensor-core prefill kernels gives up after a
 * time limit, sets the workspace's error word and lets the kernel finish, so a lost
 * producer surfaces as SSD_ERR_TIMEOUT from ssd_prefill_device_status instead of a hung
 * GPU.  This call runs that same wait in one small kernel: with `expire` non-zero nothing
 * ever arrives on the barrier and the wait runs out after `limit_ns` (1 .. 1e8 ns); with
 * `expire` zero the barrier completes at once.  It clears the error word first; read the
 * outcome with ssd_prefill_device_status (SSD_ERR_TIMEOUT, resp. SSD_OK).  Asynchronous.
 * Errors: SSD_ERR_INVALID_ARG for a NULL, misaligned or too small workspace or a limit out
 * of range; SSD_ERR_CUDA if the launch fails.
 */
SSD_API ssd_status ssd_wait_selftest(void *workspace, size_t workspace_bytes, uint64_t limit_ns, int expire,
                                     ssd_stream_t stream);

/* Size in bytes of the fixed scratch array ssd_prefill_noalloc uses (32 MiB). */
SSD_API size_t ssd_prefill_noalloc_max_workspace(void);

/*
 * ssd_prefill_device_status for ssd_prefill_noalloc, whose callers hold no workspace:
 * waits for `stream`, then reads the error word of the library's scratch array in the
 * current context.  SSD_ERR_TIMEOUT if a bounded wait of the last noalloc prefill on it
 * expired (y and final_state are then undefined), SSD_OK otherwise; SSD_ERR_CUDA if the
 * look-up, the copy or the synchronisation fails.  Allocates nothing; blocks the host.
 */
SSD_API ssd_status ssd_prefill_noalloc_device_status(ssd_stream_t stream);

/*
 * The prefill end to end, with HOST arrays: copies x, dt, A, B, C and D to the device,
 * runs ssd_prefill there, and copies y and final_state back, all enqueued on `stream`
 * in that order (one cudaMemcpyAsync per array).  Arguments, layouts and results are
 * those of ssd_prefill, except that every array pointer is a host pointer; host arrays
 * need no particular alignment.  In page-locked host memory the copies run
 * asynchronously and the call returns once they are enqueued; the host outputs are
 * complete when the stream has passed the call.  Pageable host memory also works, with
 * the copies then synchronous with the host.
 *
 * device_buffer: caller-owned device memory of at least
 * ssd_prefill_host_buffer_size(dims, dtype, chunk) bytes, 16-byte aligned: it holds the
 * device copies of the inputs and outputs and the prefill's workspace.  Calls that share
 * it must be ordered.
 *
 * Errors: as ssd_prefill; SSD_ERR_WORKSPACE if device_buffer is NULL, misaligned or
 * short.  Nothing is enqueued on an error found before the first copy.
 */
SSD_API size_t ssd_prefill_host_buffer_size(const ssd_dims *dims, ssd_dtype dtype, int chunk);
SSD_API ssd_status ssd_prefill_host(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                                    const float *A, const void *B, const void *C, const float *D, int chunk,
                                    float *y, float *final_state, void *device_buffer,
                                    size_t device_buffer_bytes, ssd_stream_t stream);

/*
 * One cached decode step (O(1) in the sequence length: "Compiler-First State Space
 * Duality ..." abstract; the recurrent mode of "Mamba and Selective State Space Models"
 * section 3).  Reads state = h_{t-1}, overwrites it in place with h_t, writes y_t.
 * dims->seqlen is ignored.  Each head's state is read once and written once.
 *
 * The state continues a prefill: pass ssd_prefill's final_state to continue that
 * sequence; any fp32 state (a saved cache) may be passed.
 *
 * Errors: as ssd_prefill, without the chunk and workspace checks.
 */
SSD_API ssd_status ssd_decode_step(const ssd_dims *dims, ssd_dtype dtype, float *state, const void *x,
                           const float *dt, const float *A, const void *B, const void *C,
                           const float *D, float *y, ssd_stream_t stream);

/*
 * The block's front end, right before the SSD layer ("Engineering Hybrid State-Space
 * Models" section 3: a width-4 1-D convolution with SiLU, Delta = Softplus(Linear(x) +
 * bias), and the convState of the last dConv - 1 = 3 inputs per channel), in one pass:
 *
 *   a[t, c]  = silu( sum_{k=0..3} conv_w[c, k] * xbc[t - 3 + k, c] + conv_b[c] )
 *   x, B, C  = a split by channel: [0, H*P) -> x, then G*N -> B, then G*N -> C
 *   dt[t, h] = softplus(dt_raw[t, h] + dt_bias[h]),  softplus(z) = log(1 + exp(z))
 *
 *   xbc            [batch, seqlen, H*P + 2*G*N] in the call's dtype (the projected
 *                  x, B and C channels; the projection itself is the caller's)
 *   conv_w         [H*P + 2*G*N, 4] fp32, 16-byte aligned (tap k = 3 multiplies token t)
 *   conv_b         [H*P + 2*G*N] fp32, or NULL for no bias
 *   conv_state_in  [batch, 3, H*P + 2*G*N] fp32: the three inputs before the first token,
 *                  oldest first, or NULL for zeros (a new sequence)
 *   conv_state_out same shape: receives the last three inputs (from conv_state_in too
 *                  when seqlen < 3), or NULL; it may be conv_state_in (updated in place)
 *   dt_raw, dt     [batch, seqlen, nheads] fp32 (dt may be dt_raw); dt_bias [nheads] fp32
 *   x, B, C        the ssd_prefill input layouts in the call's dtype (bf16: rounded to
 *                  nearest even from the fp32 result), 16-byte aligned
 *
 * With seqlen = 1 and the conv state in place this is the decode-time front end of one
 * token (x, B, C then have ssd_decode_step's layouts).  The convolution is depthwise and
 * causal, as the page's width-4 conv is read here.  Errors: as ssd_prefill for the
 * dims; SSD_ERR_INVALID_ARG for NULL or misaligned arrays, and for batch > 65535 or more
 * than 65535 * 256 channels (launch grid limits).
 */
SSD_API ssd_status ssd_frontend(const ssd_dims *dims, ssd_dtype dtype, const void *xbc, const float *conv_w,
                                const float *conv_b, const float *conv_state_in, float *conv_state_out,
                                const float *dt_raw, const float *dt_bias, void *x, void *B, void *C, float *dt,
                                ssd_stream_t stream);

/*
 * Windowed cached decode: ReplaySSM as "SketchSSM: Write to the Full State, Read from a
 * Compact Sketch" summarises it (abstract; Table 4: per state head per decode step, read
 * D and write D/W, against read D + write D for ssd_decode_step).  The state is read at
 * every step but written only when a window of up to `window` buffered tokens is folded
 * into it.  The outputs and the state after a flush are those of ssd_decode_step over
 * the same tokens (the same recurrence, unrolled over the window).
 *
 * Window buffers, caller-owned device arrays of the call's dtype (fp32 for win_dt):
 *   win_x [batch, window, nheads, headdim], win_dt [batch, window, nheads],
 *   win_B [batch, window, ngroups, dstate];  contents are managed by these two calls.
 *
 * ssd_decode_window_step: one token, with `pos` tokens (0 .. window-1) already buffered
 * since the state was last flushed.  Reads `state` (the committed state, not modified),
 * writes y (this token's output) and stores the token in buffer slot `pos`.  x, dt, B, C,
 * D, y as for ssd_decode_step.  The caller then calls ssd_decode_window_flush once the
 * window is full (pos + 1 == window), or earlier.
 *
 * ssd_decode_window_flush: folds the first `count` (0 .. window) buffered tokens into
 * `state` in place (one read and one write per head); the next window starts at pos 0.
 *
 * window: 1 .. 16.  Errors: as ssd_decode_step, plus SSD_ERR_INVALID_ARG for a window,
 * pos or count out of range or a misaligned buffer (win_x, win_B 16-byte, win_dt 4-byte).
 */
SSD_API ssd_status ssd_decode_window_step(const ssd_dims *dims, ssd_dtype dtype, int window, int pos,
                                          const float *state, void *win_x, float *win_dt, void *win_B,
                                          const void *x, const float *dt, const float *A, const void *B,
                                          const void *C, const float *D, float *y, ssd_stream_t stream);
SSD_API ssd_status ssd_decode_window_flush(const ssd_dims *dims, ssd_dtype dtype, int window, int count,
                                           float *state, const void *win_x, const float *win_dt,
                                           const void *win_B, const float *A, ssd_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBSSD_SSD_H_ */
