/*
 * sf_gdn.h — C ABI of libsf_gdn.so: forward and backward of one sequence
 * segment of a Gated DeltaNet (gated delta-rule) linear-recurrence layer with
 * an explicit boundary state, and the segment chain that runs a long sequence
 * as N segments on one GPU.
 *
 * The operations (StateFlow: Sequence Pipeline Parallelism for Long-Context
 * Modeling with Linear Recurrence, arXiv 2608.06838):
 *   - section 2.1 (the generic linear recurrence, with the Gated DeltaNet
 *     "scalar-plus-low-rank" transition), written with the state S in
 *     R^{dk x dv} per (batch, head):
 *         alpha_t = exp(g_t)
 *         S_t     = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *         o_t     = scale * S_t^T q_t
 *     and with the beta path off (the scalar-identity transition of Mamba-2):
 *         S_t     = alpha_t S_{t-1} + k_t v_t^T
 *   - section 3.1, the chunk forward  Fwd(C_in, S_in) -> (C_out, S_out)
 *     and backward Bwd(C_in, S_in, dC_out, dS_out) -> (dC_in, dS_in):
 *     sf_gdn_fwd / sf_gdn_bwd.  The backward gives the gradients of
 *         L = sum_t <o_t, dO_t> + <S_out, dS_out>
 *     with respect to q, k, v, g, beta and S_in.  It recomputes everything it
 *     needs from its inputs and S_in; nothing is saved between the calls.
 *   - section 3.1, the sequence split X = C_0 || ... || C_{N-1} with the state
 *     handed forward (S_{i+1}^in = S_i^out) and the state gradient handed
 *     backward (dS_i^out = dS_{i+1}^in): sf_segment_run.
 *
 * Layouts (row-major, contiguous unless stated):
 *   q, k, dq, dk          [B, H, T, dk]   in the I/O dtype
 *   v, o, dO, dv          [B, H, T, dv]   in the I/O dtype
 *   g, beta, dg, dbeta    [B, H, T]       fp32   (g is the log-decay, <= 0 in practice)
 *   S_in, S_out, dS_out, dS_in  [B, H, dk, dv]  fp32
 * All device pointers must be 16-byte aligned.
 *
 * Ownership: the caller owns every buffer, including the workspace; the library
 * allocates no device or host memory and keeps no state between calls, so calls
 * on different streams with different workspaces may run concurrently.  All
 * work is enqueued on `stream` (a cudaStream_t, NULL = the legacy default
 * stream); the calls return as soon as the work is enqueued.
 *
 * Errors: arguments are checked before anything is enqueued; a failed check
 * returns its status and leaves every output untouched.  A launch failure
 * returns SF_ERR_CUDA (the CUDA error string is kept per thread, see
 * sf_last_cuda_error).  No exception crosses the ABI.
 */
#ifndef SF_GDN_H_
#define SF_GDN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SF_OK = 0,
    SF_ERR_INVALID_ARG = 1,   /* null pointer where one is required, negative size, bad flag */
    SF_ERR_UNSUPPORTED = 2,   /* head size, chunk size or dtype this build does not implement */
    SF_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned */
    SF_ERR_WORKSPACE = 4,     /* workspace missing or smaller than the *_workspace_bytes query */
    SF_ERR_CUDA = 5,          /* a CUDA launch or copy failed */
    SF_ERR_TIMEOUT = 6        /* a kernel gave up waiting for one of its own asynchronous copies
                                 (reported by sf_device_check; that call's results are undefined) */
} sf_status;

typedef enum { SF_F32 = 0, SF_BF16 = 1 } sf_dtype;

/* Shape of one call.  B, H >= 0 and T >= 0 (T need not be a multiple of C:
 * the last chunk is ragged and is handled exactly).  dk, dv in {16, 32, 64, 128}.
 * C (the kernel chunk length) in {16, 32, 64, 128}.  io = dtype of q, k, v, o,
 * dO, dq, dk, dv.  use_beta = 0 selects the recurrence without the delta term
 * (beta must then be NULL).  scale multiplies q (1.0 = none). */
typedef struct {
    int B, H, T;
    int dk, dv;
    int C;
    sf_dtype io;
    int use_beta;
    float scale;
} sf_gdn_shape;

/* Human-readable name of a status. */
const char* sf_status_str(sf_status s);

/* Text of the last CUDA error seen by a call on this thread ("" if none). */
const char* sf_last_cuda_error(void);

/* Bytes of device workspace the call needs for this shape (0 when the shape
 * is invalid).  The workspace must be 16-byte aligned; its contents on entry
 * do not matter and are clobbered. */
size_t sf_gdn_fwd_workspace_bytes(const sf_gdn_shape* shape);
size_t sf_gdn_bwd_workspace_bytes(const sf_gdn_shape* shape);

/* Forward of one segment (StateFlow section 3.1, Fwd).
 *   q, k, v, g           inputs (device); beta: device [B,H,T] fp32 iff use_beta, else NULL
 *   S_in                 device state entering the segment, NULL = zeros
 *   o                    device output [B,H,T,dv] (io dtype)
 *   S_out                device state leaving the segment, NULL = not written
 *   ws, ws_bytes         device workspace of at least sf_gdn_fwd_workspace_bytes(shape)
 *   stream               cudaStream_t */
sf_status sf_gdn_fwd(const sf_gdn_shape* shape, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* S_in, void* o,
                     float* S_out, void* ws, size_t ws_bytes, void* stream);

/* Backward of one segment (StateFlow section 3.1, Bwd).  Inputs as for
 * sf_gdn_fwd plus dO [B,H,T,dv] (io dtype) and dS_out (NULL = zeros).
 * Outputs dq, dk, dv (io dtype), dg (fp32), dbeta (fp32; NULL iff !use_beta)
 * and dS_in (fp32; NULL = not written).  All outputs are overwritten. */
sf_status sf_gdn_bwd(const sf_gdn_shape* shape, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* S_in, const void* dO,
                     const float* dS_out, void* dq, void* dk, void* dv, float* dg,
                     float* dbeta, float* dS_in, void* ws, size_t ws_bytes, void* stream);

/* Workspace for sf_segment_run.  seg_len: host array of N lengths summing to
 * shape->T, or NULL for the equal split (the first T % N segments one token
 * longer).  sf_segment_workspace_bytes gives the size of the fastest mode,
 * sf_segment_min_workspace_bytes the smallest size the call accepts;
 * sf_segment_run picks the fastest mode the workspace it is given allows.
 * Two cases for the fastest mode:
 *  - tensor-core path (bf16 I/O, dk = 128, dv in {64, 128}, C = 64): the
 *    pipelined chain keeps every segment's forward intermediates for its
 *    backward, so the workspace grows with T: 8 + 4 dk + 4 C + 6 dv +
 *    4 dk dv / C bytes per token per head (2568 B at dk = dv = 128, C = 64:
 *    2.7 GB for B = 1, H = 16, T = 65536), plus the backward tiles of three
 *    pieces of 4096 tokens and the fp32 boundary states;
 *  - otherwise: the per-segment workspace of the longest segment plus N+1
 *    fp32 boundary states and two boundary state gradients. */
size_t sf_segment_workspace_bytes(const sf_gdn_shape* full, int N, const int* seg_len);

/* Bounded-memory mode of sf_segment_run (StateFlow section 3.1: each chunk's
 * activations are released after its backward; section 3.3: the retained
 * activation is bounded by the boundary states plus one chunk): the N+1 fp32
 * boundary states, two boundary state gradients and the workspace of one
 * sf_gdn_bwd call on the longest segment.  Given a workspace below
 * sf_segment_workspace_bytes but at least this size, sf_segment_run runs the
 * segments one after another, each backward recomputing its forward from the
 * saved boundary state; the results are bit-identical to the pipelined mode.
 * sf_segment_min_workspace_bytes returns the smaller of this size and the
 * pipelined one (a single long segment needs less in the pipelined mode, which
 * works in pieces of 4096 tokens).
 * At B=1, H=16, d=128 in 16 segments: 0.24 GB instead of 2.9 GB at T = 65536,
 * 0.89 GB instead of 11.0 GB at T = 262144. */
size_t sf_segment_min_workspace_bytes(const sf_gdn_shape* full, int N, const int* seg_len);

/* The segment chain on one GPU (StateFlow section 3.1): split the sequence of
 * `full` into N segments, run the forward on segments 0..N-1 with each S_out
 * handed on as the next S_in, then (when dO != NULL) the backward on segments
 * N-1..0 with each dS_in handed back as the previous dS_out.  Arguments are the
 * full-sequence tensors of sf_gdn_fwd and sf_gdn_bwd; with dO == NULL the
 * backward is skipped and dq, dk, dv, dg, dbeta, dS_in are ignored.  The
 * boundary states stay fp32 on the device, so when every segment length is a
 * multiple of C the results are bit-identical to N = 1.
 *
 * On the tensor-core path, given the workspace of sf_segment_workspace_bytes,
 * the chain is pipelined (StateFlow section 3.4, the
 * split-and-overlap of the state scan with the chunk-parallel kernels):
 * segments are further cut into pieces of 4096 tokens at chunk boundaries
 * (this changes no result); the state scans of consecutive pieces run in
 * order on an internal high-priority stream while the chunk-parallel kernels
 * of neighbouring pieces run on two lower-priority streams.  The streams and
 * their events are created for the call, forked from `stream` and joined back
 * to it before the call returns, so for the caller all work is ordered on
 * `stream` as usual; they are released asynchronously.  The backward reuses
 * the forward's intermediates instead of recomputing them; its results are
 * bit-identical to sf_gdn_fwd followed by sf_gdn_bwd on the same segment. */
sf_status sf_segment_run(const sf_gdn_shape* full, int N, const int* seg_len, const void* q,
                         const void* k, const void* v, const float* g, const float* beta,
                         const float* S_in, const void* dO, const float* dS_out, void* o,
                         float* S_out, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                         float* dS_in, void* ws, size_t ws_bytes, void* stream);

/* Synchronises the current device and reports whether any kernel of this
 * library gave up a bounded wait for its own asynchronous copies since the last
 * check (SF_ERR_TIMEOUT), then clears the flag.  No kernel waits on another
 * CTA or another launch, so this only fires if the memory system failed to
 * deliver a copy within about two seconds. */
sf_status sf_device_check(void);

/* Forward of one segment for callers that cannot allocate device memory (an
 * engine or plugin whose memory is planned up front and gives no allocation
 * hook, or code that must not call cudaMalloc on its hot path).  The paper has
 * no counterpart: this is a packaging of sf_gdn_fwd, which it runs unchanged,
 * with the workspace taken from a fixed array of SF_NOALLOC_SCRATCH_BYTES that
 * the library keeps in each GPU's memory for the life of the process.
 *   - Shapes whose forward workspace (sf_gdn_fwd_workspace_bytes) exceeds the
 *     array return SF_ERR_WORKSPACE before anything is enqueued.
 *   - All calls share the array: calls whose work overlaps on the GPU race on
 *     it, so issue them on one stream or order them with events.
 *   - The first call on a device looks up the array's address with that device
 *     current; make it outside any stream capture.
 * Other arguments, errors and results are those of sf_gdn_fwd. */
#define SF_NOALLOC_SCRATCH_BYTES (32u << 20)
sf_status sf_gdn_fwd_noalloc(const sf_gdn_shape* shape, const void* q, const void* k, const void* v,
                             const float* g, const float* beta, const float* S_in, void* o,
                             float* S_out, void* stream);

/* ---------------------------------------------------------------------------
 * Short causal convolution with a boundary state: the local-convolution state
 * a sequence chunk hands to the next beside the recurrent state (StateFlow
 * section 1: chunks must keep the boundary states of local convolution
 * modules; section 3.3: the boundary tensor B_r holds recurrent and
 * local-convolution boundary states).  The pages do not define the
 * convolution; it is the causal depthwise short convolution that Gated
 * DeltaNet-style layers apply per channel of q, k and v before the recurrence.
 * Per (batch b, head h, channel c), with taps w[h][c][j] (tap j multiplies the
 * input j steps back) and the extended input xe_p = conv_in[K-1+p] for p < 0,
 * x_p otherwise:
 *     pre_t = sum_j w_j xe_{t-j},  y_t = act(pre_t)  (act: identity or SiLU)
 *     conv_out = xe_{T-K+1} .. xe_{T-1}   (the state handed to the next segment)
 * The backward gives the gradients of sum_t <y_t, dy_t> + <conv_out, dconv_out>.
 *
 * Layouts: x, y, dy, dx [B,H,T,d] (I/O dtype); w, dw [H,d,K] fp32; conv_in,
 * conv_out [B,H,K-1,d] (I/O dtype, oldest input first); dconv_out, dconv_in
 * [B,H,K-1,d] fp32.  Pointers 8-byte aligned, the workspace 16-byte aligned;
 * conv_out must not overlap x or conv_in.  Summation orders are fixed, so a
 * sequence split into segments gives bit-identical y, conv_out, dx and
 * dconv_in for any segment lengths, and a bit-identical dw when every segment
 * length is a multiple of 64 (the weight gradient is folded per 64 tokens,
 * from the last block to the first, continuing from dw_in). */
typedef struct {
    int B, H, T;   /* batch, heads, tokens (>= 0) */
    int d;         /* channels per head: even, 2..1024 */
    int K;         /* taps: 2..8 */
    sf_dtype io;   /* dtype of x, y, dy, dx, conv_in, conv_out */
    int act;       /* 0: identity, 1: SiLU */
} sf_conv_shape;

/* Workspace of sf_conv_bwd (0 when the shape is invalid). */
size_t sf_conv_workspace_bytes(const sf_conv_shape* shape);

/* Forward of one segment.  conv_in NULL = zeros (the start of a sequence);
 * conv_out NULL = not written. */
sf_status sf_conv_fwd(const sf_conv_shape* shape, const void* x, const float* w, const void* conv_in,
                      void* y, void* conv_out, void* stream);

/* Backward of one segment: dx (I/O dtype), dconv_in (fp32; NULL = not
 * written) and dw_out = dw_in + this segment's weight gradient (dw_in NULL =
 * zeros; dw_in == dw_out is allowed).  dconv_out NULL = zeros. */
sf_status sf_conv_bwd(const sf_conv_shape* shape, const void* x, const float* w, const void* conv_in,
                      const void* dy, const float* dconv_out, void* dx, const float* dw_in, float* dw_out,
                      float* dconv_in, void* ws, size_t ws_bytes, void* stream);

/* The segment chain of the convolution (as sf_segment_run for the recurrent
 * state): forward over N segments with conv_out handed on as the next conv_in,
 * then (dy != NULL) backward in reverse with dconv_in handed back as the
 * previous dconv_out and the weight gradient accumulated into dw. */
size_t sf_conv_segment_workspace_bytes(const sf_conv_shape* full, int N, const int* seg_len);
sf_status sf_conv_segment_run(const sf_conv_shape* full, int N, const int* seg_len, const void* x,
                              const float* w, const void* conv_in, const void* dy, const float* dconv_out,
                              void* y, void* conv_out, void* dx, float* dw, float* dconv_in, void* ws,
                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Delta rule with a per-channel (diagonal) decay: the diagonal-plus-low-rank
 * transition StateFlow lists beside the scalar-plus-low-rank one (section 2.1:
 * Kimi Delta Attention), in this library's state orientation:
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t     (use_beta = 0: S_t = Diag(exp(g_t)) S_{t-1} + k_t v_t^T)
 * with a log-decay g_t per key channel.  Same layouts as sf_gdn_* except
 * g, dg: [B,H,T,dk] fp32.  With every channel's log-decay equal this is the
 * sf_gdn_* layer.  The computation is fp32 token by token on the CUDA cores
 * (see csrc/kda_kernels.cu), so splitting a sequence at any token gives
 * bit-identical results.  dk in {32, 64, 128}; dv a multiple of 32 up to 1024;
 * pointers 16-byte aligned. */
typedef struct {
    int B, H, T;
    int dk, dv;
    sf_dtype io;
    int use_beta;
    float scale;
} sf_kda_shape;

/* Workspace bytes: forward (backward = 0) needs none; the backward holds a
 * checkpoint every 64 tokens, a window scratch per CTA and the per-column-block
 * partial sums (at B=1, H=16, T=65536, dk=dv=128: about 6.5 GB). */
size_t sf_kda_workspace_bytes(const sf_kda_shape* shape, int backward);

/* Forward of one segment: o, and S_out (NULL = not written); S_in NULL = zeros. */
sf_status sf_kda_fwd(const sf_kda_shape* shape, const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* S_in, void* o, float* S_out, void* stream);

/* Backward of one segment: gradients of sum <o, dO> + <S_out, dS_out>; dS_in
 * NULL = not written; dS_out NULL = zeros. */
sf_status sf_kda_bwd(const sf_kda_shape* shape, const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* S_in, const void* dO, const float* dS_out, void* dq,
                     void* dk, void* dv, float* dg, float* dbeta, float* dS_in, void* ws, size_t ws_bytes,
                     void* stream);

/* Optional launch observer, for profiling.  When set, every kernel this
 * library launches is bracketed by hook(name, 0, stream, user) just before the
 * launch and hook(name, 1, stream, user) just after it, on the calling thread,
 * so the caller can record CUDA events on `stream` around each kernel.  NULL
 * removes the observer.  The setting is process-wide; set it while no other
 * thread is inside the library. */
typedef void (*sf_launch_hook)(const char* kernel, int after, void* stream, void* user);
void sf_set_launch_hook(sf_launch_hook hook, void* user);

/* Native launch timer, for measurement with little host overhead.  While
 * enabled, each of the next `capacity` kernel launches of this library is
 * bracketed by two CUDA events (timing enabled) recorded on the launch's own
 * stream; later launches are not timed.  sf_timer_enable creates the events
 * (and discards earlier records); sf_timer_disable stops recording and keeps
 * the records; sf_timer_count gives how many launches were recorded;
 * sf_timer_read(i, ...) waits for launch i to finish and returns its kernel
 * name (a static string) and its duration in milliseconds; sf_timer_free
 * destroys the events.  Process-wide, for one host thread at a time; the only
 * state this library keeps between calls, and only while a caller uses it. */
sf_status sf_timer_enable(int capacity);
void sf_timer_disable(void);
int sf_timer_count(void);
sf_status sf_timer_read(int i, const char** kernel, float* ms);
/* As sf_timer_read, plus the launch's start relative to the first recorded
 * launch's start (a timeline of the recorded launches). */
sf_status sf_timer_read_at(int i, const char** kernel, float* start_ms, float* ms);
void sf_timer_free(void);

/* Introspection for tests and benchmarks: the kernel family a shape runs on
 * ("tc" = tensor-core kernels, "simt" = fp32 CUDA-core kernels; NULL if the
 * shape is unsupported) and how many kernels one sf_gdn_fwd (backward = 0) or
 * sf_gdn_bwd (backward = 1) call launches. */
const char* sf_gdn_path(const sf_gdn_shape* shape);
int sf_gdn_launches(const sf_gdn_shape* shape, int backward);

#ifdef __cplusplus
}
#endif

#endif /* SF_GDN_H_ */
