/*
 * ssd.h -- C ABI of libssd.so, the B200 (sm_100a) SSD layer forward.
 *
 * The operation is the SSD layer Y = SSD(A, B, C)(X) of "Transformers are
 * SSMs: Generalized Models and Efficient Algorithms Through Structured State
 * Space Duality" (arXiv 2405.21060; analysis page, section "The SSD Layer:
 * Formal Definition"), i.e. the scalar-identity selective SSM of section "The
 * Scalar-Identity SSM":
 *
 *     h_t = exp(dt_t * A_h) * h_{t-1} + B_t x_t^T        (state [P x N] per head)
 *     y_t = C_t^T h_t + D_h * x_t
 *
 * with h_{-1} = init_state (zero when NULL), computed by the block
 * decomposition of section "The Block-Decomposition SSD Algorithm": chunks of
 * Q tokens (stage 0, ceil(T/Q) chunks, the last one may be short), the
 * quadratic masked form inside each chunk (stage 1), chunk-final states
 * (stage 2), the scalar recurrence between chunks (stage 3), the inter-chunk
 * output (stage 4) and their sum (stage 5).  The exponential discretisation,
 * the D_h skip and the place of init_state are not written on the pages; they
 * are the readings stated above.  Head h reads B/C group g = h / (H / G)
 * (grouped heads: analysis page, "The Mamba-2 Architecture", G divides H).
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *    and densely packed in the layouts given below.  The library never
 *    allocates device memory; scratch lives in the caller's workspace.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream and never synchronise the
 *    host, except ssd_fwd_check which waits for the stream.
 *  - Return values are ssd status codes (SSD_OK = 0).  Argument errors are
 *    detected on the host before anything is launched.
 *  - Stateless and thread-safe; concurrent calls must use distinct
 *    workspaces.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>

/* Every declared entry point is exported; everything else in libssd.so is hidden. */
#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of x, B, C and y.  dt, A, D and both states are always fp32. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype_t;

enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1, /* NULL required pointer, bad dimension, H % G != 0,
                                misaligned pointer, workspace too small */
    SSD_ERR_UNSUPPORTED = 2, /* valid shape outside the kernels' limits
                                (P > 128, N > 256, Q > 256) */
    SSD_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
    SSD_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (see ssd_fwd_check) */
};

/*
 * Bytes of device workspace ssd_fwd needs for this problem (256-byte
 * multiple).  Returns 0 for invalid dimensions.  The workspace holds a status
 * word and, on the CUDA-core path, the per-chunk log-decay prefix sums and the
 * chunk states (stages 0-3); on the fused tensor-core path (bf16 x, B, C;
 * Q in {128, 256}; P a multiple of 8 up to 64, or 128; N a multiple of 16 up
 * to 128, or 256), per launch, the unit counter, the inter-chunk hand-off
 * flags and L2-sized rings of the latest chunk states (fp32, and bf16 tiles
 * of them for the other row block of each chunk; fp32 local chunk states
 * instead of the tiles where a long sequence uses look-back).
 */
SSD_API size_t ssd_fwd_workspace_bytes(int batch, int T, int H, int P, int G, int N, int Q, int dtype);

/*
 * SSD layer forward.
 *
 *   x           [batch][T][H][P]   dtype      input sequence X
 *   dt          [batch][T][H]      fp32       step sizes, already positive (no softplus inside)
 *   A           [H]                fp32       per-head log-decay rate, a_t = exp(dt_t * A_h)
 *   B, C        [batch][T][G][N]   dtype      expansion / contraction vectors
 *   D           [H]                fp32       skip weight
 *   Q                                         chunk length (1 <= Q <= 256)
 *   init_state  [batch][H][P][N]   fp32       h_{-1}; NULL = zero
 *   y           [batch][T][H][P]   dtype      output (written)
 *   final_state [batch][H][P][N]   fp32       h_{T-1} (written); NULL = not written
 *   workspace   >= ssd_fwd_workspace_bytes(...) bytes of device memory, 256-byte aligned
 *
 * Limits: batch, H, G, P, N, Q >= 1, T >= 0, H % G == 0, P <= 128, N <= 256,
 * Q <= 256.  Pointers must be aligned to their element size (16 bytes for
 * the bf16 tensor-core path).  y must not alias any input.  T == 0 writes
 * final_state = init_state (or zero) and nothing else; x, dt, B, C and y are
 * not read then and may be NULL.
 *
 * Returns SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED or SSD_ERR_CUDA.
 * Device-side failures of bounded waits are reported by ssd_fwd_check.
 */
SSD_API int ssd_fwd(const void *x, const float *dt, const float *A, const void *B, const void *C,
            const float *D, int Q, const float *init_state, void *y, float *final_state,
            int batch, int T, int H, int P, int G, int N, int dtype, void *workspace,
            size_t workspace_bytes, void *stream);

/*
 * Number of main kernel launches ssd_fwd issues for these arguments, which is
 * also the number of stages ssd_fwd_timed reports (0 when the arguments are
 * invalid).  The fused path also runs one small kernel that clears the
 * workspace's counter and flags in front of its first launch (it overlaps
 * that launch's start and is timed within the first stage); the CUDA-core
 * path clears them with a memset.  Lets callers account for launches without
 * a profiler.
 */
SSD_API int ssd_fwd_launch_count(int batch, int T, int H, int P, int G, int N, int Q, int dtype);

/*
 * ssd_fwd, instrumented for measurement: records a CUDA event on `stream`
 * before the first kernel and after each kernel, waits for the stream, and
 * writes each stage's duration in milliseconds to stage_ms[0 .. k-1]
 * (k = min(ssd_fwd_launch_count(...), max_stages); a stage is one main
 * launch, on the fused path the first one together with the workspace clear
 * in front of it) and the span of the whole call to *total_ms (either pointer
 * may be NULL).  The events are created on
 * the first call in each host thread and kept until the process exits.  Same
 * arguments and results as ssd_fwd otherwise.
 */
SSD_API int ssd_fwd_timed(const void *x, const float *dt, const float *A, const void *B, const void *C,
                  const float *D, int Q, const float *init_state, void *y, float *final_state,
                  int batch, int T, int H, int P, int G, int N, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream, float *stage_ms, int max_stages,
                  float *total_ms);

/*
 * Name of kernel `i` (0-based, launch order) of the sequence ssd_fwd issues
 * for these arguments, or NULL when i is out of range.
 */
SSD_API const char *ssd_fwd_stage_name(int batch, int T, int H, int P, int G, int N, int Q, int dtype, int i);

/*
 * Waits for `stream`, then reads the status word the kernels of the last
 * ssd_fwd on this workspace left (SSD_OK or SSD_ERR_TIMEOUT).  Returns
 * SSD_ERR_CUDA if the wait or the copy fails.
 */
SSD_API int ssd_fwd_check(const void *workspace, void *stream);

/*
 * Test hook of the bounded waits (no counterpart on the pages): ssd_fwd on
 * the fused tensor-core path, except that the block owning chunk
 * `withhold_c` of sequence (withhold_b, withhold_h) never publishes its
 * outgoing state, and every wait on another block's flag gives up after
 * `flag_polls` polls (about 0.1-1 us each).  The blocks waiting for that
 * state then give up, ssd_fwd_check reports SSD_ERR_TIMEOUT, the kernel still
 * finishes (every block drains its own copies and products before it exits)
 * and the device stays usable; y and final_state are not valid.  Arguments as
 * for ssd_fwd plus the three indices (in range) and flag_polls >= 1; returns
 * SSD_ERR_UNSUPPORTED for problems that do not take the fused path.
 */
SSD_API int ssd_fwd_withhold_publish(const void *x, const float *dt, const float *A, const void *B, const void *C,
                                     const float *D, int Q, const float *init_state, void *y, float *final_state,
                                     int batch, int T, int H, int P, int G, int N, int dtype, void *workspace,
                                     size_t workspace_bytes, void *stream, int withhold_b, int withhold_h,
                                     int withhold_c, unsigned flag_polls);

/*
 * ssd_fwd for callers that cannot allocate device memory when they run the
 * layer (an engine that fixes every buffer before serving, a framework whose
 * allocator owns the device, a loop that must never reach cudaMalloc).  The
 * paper has no counterpart to this entry point; it only changes where the
 * scratch lives.
 *
 * Same arguments, results and conventions as ssd_fwd, without the workspace:
 * the library uses its own scratch, a static device array of
 * SSD_NO_ALLOC_SCRATCH_BYTES bytes present on every GPU that loads the
 * library until the process exits.  Problems whose ssd_fwd_workspace_bytes
 * exceeds that size are rejected with SSD_ERR_UNSUPPORTED before anything is
 * launched.  The first call on each device looks up the array's device
 * address (and may load the library's device code there), so make it before
 * any stream capture.  All calls on a device share the array and it keeps
 * the last call's contents (each call clears what it needs); calls whose GPU
 * work overlaps, e.g. on two streams, race on it.  Nothing is allocated.
 */
#define SSD_NO_ALLOC_SCRATCH_BYTES (32u << 20)
SSD_API int ssd_fwd_no_alloc(const void *x, const float *dt, const float *A, const void *B, const void *C,
                     const float *D, int Q, const float *init_state, void *y, float *final_state,
                     int batch, int T, int H, int P, int G, int N, int dtype, void *stream);

/*
 * ssd_fwd_check for ssd_fwd_no_alloc, whose callers hold no workspace
 * pointer: waits for `stream`, then reads the status word the last
 * ssd_fwd_no_alloc on the current device left in the library's scratch
 * (SSD_OK or SSD_ERR_TIMEOUT).  Returns SSD_ERR_CUDA if the wait or the copy
 * fails.  Allocates nothing.
 */
SSD_API int ssd_fwd_no_alloc_check(void *stream);

/*
 * One autoregressive (decode) step of the same recurrence, in place: for
 * every batch row b and head h, with g = h / (H / G),
 *
 *     state[b][h] = exp(dt[b][h] * A[h]) * state[b][h] + x[b][h] B[b][g]^T
 *     y[b][h]     = state[b][h] C[b][g] + D[h] * x[b][h]
 *
 * (the recurrent mode: "Transformers are SSMs", analysis page, section "The
 * Scalar-Identity SSM"; the English note's section "Working Through Four
 * Tokens" advances it one token at a time).  Calling it for t = 0 .. T-1 from
 * state = init_state gives the y and final_state of ssd_fwd over those T
 * tokens, up to rounding.
 *
 *   state  [batch][H][P][N]   fp32    h_{t-1} on entry, h_t on return
 *   x      [batch][H][P]      dtype   this token's input
 *   dt     [batch][H]         fp32    step sizes
 *   A, D   [H]                fp32
 *   B, C   [batch][G][N]      dtype
 *   y      [batch][H][P]      dtype   output (written)
 *
 * Limits: batch, H, G, P, N >= 1, H % G == 0, N <= 1024 (else
 * SSD_ERR_UNSUPPORTED), batch and H <= 65535.  Pointers aligned to their
 * element size; y and the state must not overlap each other or an input.  No
 * workspace, no host synchronisation.  Returns SSD_OK, SSD_ERR_INVALID_ARG,
 * SSD_ERR_UNSUPPORTED or SSD_ERR_CUDA.
 */
SSD_API int ssd_step(float *state, const void *x, const float *dt, const float *A, const void *B, const void *C,
             const float *D, void *y, int batch, int H, int P, int G, int N, int dtype, void *stream);

/*
 * The Mamba-2 block's step after the layer: the output gated by the Swish of
 * a parallel branch z, then GroupNorm ("Transformers are SSMs", analysis page,
 * section "The Mamba-2 Architecture", paragraphs "Gating" and "Extra
 * normalization").  Per token (row), with g = y * silu(z) = y * z / (1 + e^-z)
 * and the channels split into ngroups contiguous groups,
 *
 *     out = (g - mean(g)) / sqrt(var(g) + eps) * weight + bias      (per group, population variance)
 *
 *   y, z, out  [rows][channels]  dtype   y is ssd_fwd's output viewed as [batch*T][H*P]
 *   weight     [channels]        fp32    NULL = 1
 *   bias       [channels]        fp32    NULL = 0
 *
 * Limits: rows >= 0, channels >= 1, channels % ngroups == 0, channels /
 * ngroups <= 4096 (else SSD_ERR_UNSUPPORTED), eps >= 0.  out may be y
 * (in place) but must not otherwise overlap y or z.  Returns SSD_OK,
 * SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED or SSD_ERR_CUDA.
 */
SSD_API int ssd_gate_norm(const void *y, const void *z, const float *weight, const float *bias, void *out,
                  long long rows, int channels, int ngroups, float eps, int dtype, void *stream);

/*
 * The layer forward followed by the block's gate and GroupNorm with a group
 * per head ("Transformers are SSMs", analysis page, section "The Mamba-2
 * Architecture", paragraphs "Gating" and "Extra normalization"): per token
 * and head, with y the ssd_fwd output and g = y * silu(z),
 *
 *     out = (g - mean(g)) / sqrt(var(g) + eps) * norm_weight + norm_bias
 *
 * over the head's P channels (population variance), i.e. ssd_gate_norm with
 * ngroups = H on ssd_fwd's y.  Arguments as for ssd_fwd, plus
 *
 *   z            [batch][T][H][P]  dtype   the gate branch
 *   norm_weight  [H * P]           fp32    NULL = 1 (16-byte aligned)
 *   norm_bias    [H * P]           fp32    NULL = 0 (16-byte aligned)
 *   eps          >= 0
 *   out          [batch][T][H][P]  dtype   written in place of y; y itself is not returned
 *
 * On the fused tensor-core path with P = 64 and N <= 128 the gate and the norm
 * run in the kernel's drain on the fp32 y (one launch, y never reaches
 * memory); elsewhere ssd_fwd writes y into out and ssd_gate_norm runs over it
 * in place (one more launch).  z must not overlap out.  Same workspace as
 * ssd_fwd.  Returns as ssd_fwd.
 */
SSD_API int ssd_fwd_gated(const void *x, const float *dt, const float *A, const void *B, const void *C,
                  const float *D, int Q, const float *init_state, const void *z, const float *norm_weight,
                  const float *norm_bias, float eps, void *out, float *final_state, int batch, int T, int H,
                  int P, int G, int N, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/* Main kernel launches ssd_fwd_gated issues for these arguments (0 when they are invalid), counted as
 * for ssd_fwd_launch_count (the fused path's workspace-clear kernel not included). */
SSD_API int ssd_fwd_gated_launch_count(int batch, int T, int H, int P, int G, int N, int Q, int dtype);

/*
 * Sequence split: contiguous shards of one sequence (on one GPU or one per
 * worker) run ssd_fwd from a zero state at the same time and exchange only
 * their states.  Workers process contiguous shards and pass recurrent states
 * between them, communication linear in the number of workers (the paper's
 * claim summary on its reproduction page); it is the block decomposition of
 * "Transformers are SSMs" (analysis page, section "The Block-Decomposition
 * SSD Algorithm", stages 3 and 4) one level up, shards in the place of
 * chunks.  For shard k of K, with sigma_t the inclusive sum of dt_u * A_h
 * over the shard's tokens up to t:
 *
 *   1. ssd_fwd(shard, init_state = NULL)  -> y0, fin0
 *   2. ssd_split_logdecay                 -> sig [batch][H][T_shard], total [batch][H]
 *   3. exchange (fin0, total) of every shard, shard order, into
 *      fin0_all [K][batch][H][P][N] and total_all [K][batch][H]
 *   4. ssd_split_combine(k)               -> s_in = state entering shard k (fold of the
 *      earlier shards over init_state) and the shard's true final state
 *   5. ssd_split_correct                  -> y += exp(sigma_t) s_in C_t, in place
 *
 * gives the y and final_state of ssd_fwd over the whole sequence (up to
 * rounding; bf16 y is rounded once more).  Layouts as for ssd_fwd; all
 * pointers are device pointers; sig, total, s_in are fp32.
 *
 * ssd_split_logdecay: dt [batch][T][H], A [H] -> sig, total.  T >= 1.
 * ssd_split_combine: init_state and final_state may be NULL (zero / not written).
 * ssd_split_correct: y [batch][T][H][P] (dtype, updated in place), C [batch][T][G][N]
 * (dtype), sig, s_in [batch][H][P][N].  Limits P <= 128, N <= 256.
 * Each returns SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED or SSD_ERR_CUDA.
 */
SSD_API int ssd_split_logdecay(const float *dt, const float *A, float *sig, float *total, int batch, int T, int H,
                       void *stream);
SSD_API int ssd_split_combine(const float *fin0_all, const float *total_all, const float *init_state, int k,
                      int shards, float *s_in, float *final_state, int batch, int H, int P, int N, void *stream);
SSD_API int ssd_split_correct(void *y, const void *C, const float *sig, const float *s_in, int batch, int T, int H,
                      int P, int G, int N, int dtype, void *stream);

/*
 * Backward pass: the gradients of L = sum(dy * y) + sum(dfinal_state * final_state)
 * with respect to every input of ssd_fwd, for the same problem.  The pages
 * print the forward only ("Transformers are SSMs", analysis page, section
 * "The SSM as a Matrix Transformation", equation (2), and the chunked form of
 * section "The Block-Decomposition SSD Algorithm"); this is the unique
 * gradient of that function, organised by the same chunks.  Per (b, h), with
 * the adjoint g_t = dL/dh_t of the state h_t [P][N] (g_{T-1} = dfinal + dy C^T,
 * g_t = a_{t+1} g_{t+1} + dy_t C_t^T):
 *
 *   dx_t   = g_t B_t + D_h dy_t                     [batch][T][H][P], dtype
 *   dB_t   = sum over the group's heads of g_t^T x_t    [batch][T][G][N], dtype
 *   dC_t   = sum over the group's heads of h_t^T dy_t   [batch][T][G][N], dtype
 *   ddt_t  = A_h <g_t, a_t h_{t-1}>                 [batch][T][H], fp32
 *   dA_h   = sum_{b,t} dt_t <g_t, a_t h_{t-1}>      [H], fp32
 *   dD_h   = sum_{b,t} <dy_t, x_t>                  [H], fp32
 *   dinit  = a_0 g_0                                [batch][H][P][N], fp32 (NULL: not written)
 *
 * Inputs as for ssd_fwd, plus dy [batch][T][H][P] in the dtype of x and
 * dfinal_state [batch][H][P][N] fp32 (NULL: zero).  init_state NULL means
 * zero.  All pointers are device pointers, 4-byte (fp32) or 2-byte (bf16)
 * aligned; workspace 256-byte aligned with at least ssd_bwd_workspace_bytes()
 * bytes (0 there: invalid dimensions).  Outputs may not overlap any input,
 * one another or the workspace.  Every kernel runs on the CUDA cores in fp32
 * (sums over the sequence for dt, A and D in fp64), in a fixed order: results
 * are bitwise reproducible.  Same dimension limits as ssd_fwd, plus batch,
 * H <= 65535.  Asynchronous on `stream`; 11 launches (none when T == 0, where
 * dA = dD = 0 and dinit = dfinal).  Returns SSD_OK, SSD_ERR_INVALID_ARG,
 * SSD_ERR_UNSUPPORTED or SSD_ERR_CUDA.
 */
SSD_API size_t ssd_bwd_workspace_bytes(int batch, int T, int H, int P, int G, int N, int Q, int dtype);
SSD_API int ssd_bwd(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                    int Q, const float *init_state, const void *dy, const float *dfinal_state, void *dx, float *ddt,
                    float *dA, void *dB, void *dC, float *dD, float *dinit_state, int batch, int T, int H, int P,
                    int G, int N, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Waits for `stream` and returns the status word of the last ssd_bwd call on
 * this workspace: SSD_OK, or SSD_ERR_TIMEOUT when a bounded wait of the
 * tensor-core kernels gave up (a defect of the kernel, not of the inputs; the
 * gradients of that call are then not valid).  SSD_ERR_INVALID_ARG for a NULL
 * workspace, SSD_ERR_CUDA if the stream or the copy fails.
 */
SSD_API int ssd_bwd_check(const void *workspace, void *stream);

/* Static, NUL-terminated description of a status code. */
SSD_API const char *ssd_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
SSD_API int ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
