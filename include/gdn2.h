/*
 * gdn2.h -- C ABI of libgdn2.so: the Gated DeltaNet-2 chunkwise gated
 * delta-rule recurrence on one NVIDIA B200 (sm_100a).
 *
 * The operation (per batch b and head h, tokens t = 1..T, S_0 given or zero):
 *
 *     alpha_t = exp(log_alpha_t)            channel-wise decay, d_k entries
 *     S'      = Diag(alpha_t) S_{t-1}       decay first
 *     u_t     = w_t (.) v_t - S'^T (b_t (.) k_t)
 *     S_t     = S' + k_t u_t^T  =  (I - k_t (b_t (.) k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t (.) v_t)^T
 *     o_t     = S_t^T q_t
 *
 * b_t (key side, d_k entries) is the erase gate, w_t (value side, d_v
 * entries) the write gate.  Sources: aixai.ru "Gated DeltaNet-2" post, section
 * "Один скаляр не может решать два разных вопроса" (the update in prose) and
 * "Как это реализуется на практике" (chunkwise computation, gate-weighted
 * keys/values, A and T, gate-aware backward, log-decay in fp32); aiexpert.news
 * article, gate paragraph (b_t in [0,1]^{d_k}, w_t in [0,1]^{d_v}, exact
 * reduction to KDA when b_t = w_t = beta_t 1) and implementation paragraph
 * (chunkwise WY algorithm with the decay absorbed into asymmetric erase
 * factors).  No 1/sqrt(d) scale is applied: fold any scale into q.
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are caller-owned DEVICE pointers to contiguous
 *    row-major memory, 16-byte aligned (GDN2_ERR_ALIGN otherwise).  The
 *    library allocates no device memory and keeps no pointer after a call.
 *  - q, k, b: [B, T, H, Dk]; v, w, o (and their gradients): [B, T, H, Dv];
 *    element type given by `dt` (fp32 or bf16).  log_alpha and its gradient
 *    are [B, T, H, Dk] fp32 always.  States S0, S_T, dS_T, dS0 are
 *    [B, H, Dk, Dv] fp32 always (d_v contiguous).
 *  - v1 shape contract: Dk == Dv in {64, 128}; B >= 1; 1 <= H <= 65535; T >= 0
 *    (any T; T = 0 copies S0 to S_T).  Other shapes give GDN2_ERR_UNSUPPORTED.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    are asynchronous on it: a GDN2_OK return means the arguments were valid
 *    and the kernels were enqueued.  An error raised inside a kernel (a
 *    bounded wait that gave up) is recorded in a per-device status word that
 *    gdn2_sync_status() reports.
 *  - Every call validates all arguments before it launches anything; on an
 *    error nothing is launched and no output is written.  No C++ exception
 *    crosses this boundary.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_NULL = -1,        /* a required pointer is NULL */
    GDN2_ERR_SHAPE = -2,       /* a size is negative or zero where it must be positive */
    GDN2_ERR_DTYPE = -3,       /* dt is not a gdn2_dtype value */
    GDN2_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned */
    GDN2_ERR_WORKSPACE = -5,   /* workspace NULL or smaller than gdn2_workspace_size() */
    GDN2_ERR_CUDA = -6,        /* a CUDA runtime call failed (launch error, no device, ...) */
    GDN2_ERR_TIMEOUT = -7,     /* a kernel's bounded wait gave up (reported by gdn2_sync_status) */
    GDN2_ERR_UNSUPPORTED = -8, /* valid but outside the v1 shape contract */
    GDN2_ERR_TOO_LARGE = -9,   /* needs more scratch than GDN2_NOALLOC_MAX_SCRATCH_BYTES
                                  (gdn2_chunk_bwd_noalloc only) */
    GDN2_ERR_SEQLENS = -10     /* a kernel found cu_seqlens invalid (reported by gdn2_sync_status) */
} gdn2_status;

typedef enum { GDN2_F32 = 0, GDN2_BF16 = 1 } gdn2_dtype;

/*
 * Chunkwise forward (chunk length 64): o and the final state S_T.
 *   S0:  initial state, or NULL for zeros.
 *   o:   output [B,T,H,Dv] of type dt.
 *   S_T: final state, or NULL when not wanted.  May alias S0 (in-place
 *        state update), but no other argument.
 *   workspace / ws_bytes: scratch of gdn2_workspace_size(0, ...) bytes.  That is 0
 *        (NULL accepted) except for bf16 batches of at most 48 (batch, head) chains of
 *        at least 48 chunks, which run as a chunk-parallel scan over segments of each
 *        sequence when given it (the serial chain runs when it is missing or short).
 * bf16 inputs run on the tensor cores (bf16 operands, fp32 accumulation,
 * fp32 state); fp32 inputs run token by token in fp32 arithmetic throughout.
 * Any decay alpha in [0, 1] is exact: a chunk whose log-decay falls below -80
 * on some channel (where the chunkwise factor e^{-G} would leave the fp32
 * range) runs token by token instead, slower but with the same results.
 */
GDN2_API gdn2_status gdn2_chunk_fwd(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream);

/*
 * One recurrent decode step for N independent sequences (one token each).
 *   q, k, b: [N,H,Dk]; v, w, o: [N,H,Dv] of type dt; log_alpha [N,H,Dk] fp32.
 *   S: [N,H,Dk,Dv] fp32, read and overwritten in place with S_t.
 * Same update as above with T = 1; the state is read once and written once.
 */
GDN2_API gdn2_status gdn2_decode_step(gdn2_dtype dt, int N, int H, int Dk, int Dv,
                             const void *q, const void *k, const void *v, const float *log_alpha,
                             const void *b, const void *w, float *S, void *o, void *stream);

/*
 * Gate-aware backward of L = <o, d_o> + <S_T, dS_T> for the forward above.
 *   d_o: [B,T,H,Dv] of type dt.  dS_T: fp32 state gradient, or NULL for zero.
 *   Outputs: dq, dk, db [B,T,H,Dk] and dv, dw [B,T,H,Dv] of type dt;
 *            dlog_alpha [B,T,H,Dk] fp32; dS0 [B,H,Dk,Dv] fp32.
 *   S0 may be NULL (zeros).  All outputs must be distinct from the inputs.
 *   workspace: at least gdn2_workspace_size(1, ...) bytes.  bf16: chunk-boundary
 *   states and per-chunk factors (bf16), the chain's per-chunk inputs and the
 *   state gradients at chunk ends (bf16), and the scratch of the token-level
 *   gradients of chunks whose decay is too strong for the chunkwise factors
 *   (a chunk log-decay below -80 on some channel); fp32: fp32 chunk-boundary
 *   states and chunk-end state gradients, and that scratch.
 * The gates enter inside the chunk products (gate-weighted keys and values),
 * as the aixai.ru post's implementation section requires.
 */
GDN2_API gdn2_status gdn2_chunk_bwd(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream);

/*
 * The forward on HOST buffers: q, k, v, log_alpha, b, w, S0 (S0 may be NULL) are read from
 * host memory and o, S_T (S_T may be NULL) written to host memory, with the layouts of
 * gdn2_chunk_fwd.  The call pipelines slices of batch rows: the copies in, the chunk
 * kernels (on `stream`) and the copies out overlap, through three rotating staging slots
 * in the device `workspace` (gdn2_workspace_size(4, ...) bytes) and two library-owned
 * streams.  Asynchronous on `stream`: the outputs are in host memory once `stream` has
 * completed; the host buffers must stay valid until then.  Page-locked host memory
 * (cudaHostAlloc / cudaHostRegister) lets the copies overlap; pageable memory works but
 * serialises them.  The results equal gdn2_chunk_fwd's on the same values bit for bit.
 * Errors as gdn2_chunk_fwd, plus GDN2_ERR_WORKSPACE for a missing or short workspace.
 */
GDN2_API gdn2_status gdn2_chunk_fwd_host(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream);

/*
 * Training pair.  gdn2_chunk_fwd_save is gdn2_chunk_fwd (same o and S_T, bit for bit)
 * that also records the chunk-boundary states into `workspace`, the backward's
 * workspace of gdn2_workspace_size(1, ...) bytes; gdn2_chunk_bwd_saved is
 * gdn2_chunk_bwd taking those recorded states instead of running its own forward
 * pass over the batch.  Call the backward with the same inputs, S0 and workspace,
 * with nothing written to the workspace in between; the gradients equal
 * gdn2_chunk_bwd's bit for bit.  fp32 batches record nothing (the backward recomputes).
 * gdn2_chunk_fwd_save returns GDN2_ERR_WORKSPACE for a missing or short workspace.
 */
GDN2_API gdn2_status gdn2_chunk_fwd_save(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream);
GDN2_API gdn2_status gdn2_chunk_bwd_saved(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream);

/*
 * gdn2_chunk_bwd without a workspace argument, for callers that cannot
 * allocate device memory when they run the backward: code running inside a
 * custom allocator or memory pool (allocating there would recurse), runtimes
 * that fix their device-memory budget at start-up and forbid cudaMalloc
 * afterwards, and plain C hosts that have no tensor library to hand them a
 * buffer.  The operation has no counterpart in the paper: it is the same
 * backward as gdn2_chunk_bwd, with the same arguments minus the workspace and
 * the same gradients.
 *   Scratch: a file-scope device array of GDN2_NOALLOC_MAX_SCRATCH_BYTES
 *   bytes inside the library.  A problem is accepted when
 *   gdn2_workspace_size(1, ...) <= GDN2_NOALLOC_MAX_SCRATCH_BYTES (for
 *   example B*H = 2, T = 1024, d = 128 needs about 8 MiB with either dtype,
 *   B*H = 4, T = 4096, d = 128 more than 32 MiB); larger ones return
 *   GDN2_ERR_TOO_LARGE before anything is launched.  Arguments are checked by
 *   the same rules as gdn2_chunk_bwd.
 *   When the memory is taken: CUDA loads a library's code lazily by default
 *   (CUDA_MODULE_LOADING=LAZY), so the array is committed on a device at the
 *   first call of this entry point with that device current, and from then on
 *   held until the process exits.  A caller whose budget must not move makes
 *   one call on each device at start-up, before the budget is fixed and
 *   before any stream capture.
 *   Allocation: none.  No cudaMalloc, cudaFree or allocating library call.
 *   Every call looks up the array's device address (cudaGetSymbolAddress) for
 *   the device current at the call, which must be the device that holds the
 *   arguments and the stream.
 *   Sharing: all calls on one device use the same array, and it keeps what
 *   the last call left there.  Calls whose kernels overlap on the GPU (on
 *   different streams, or from different threads) race on it and give wrong
 *   gradients: order them on one stream or with events.  Nothing in the
 *   array needs to start at zero: each call writes or clears every scratch
 *   byte it reads before reading it.
 */
#define GDN2_NOALLOC_MAX_SCRATCH_BYTES ((size_t)32 << 20)

GDN2_API gdn2_status gdn2_chunk_bwd_noalloc(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *stream);

/*
 * Variable-length batches: N sequences packed along the token axis.
 *   cu_seqlens: DEVICE int32 [N + 1] with 0 = c_0 <= c_1 <= ... <= c_N = total_T;
 *               sequence n is token rows c_n .. c_{n+1} (empty sequences allowed).
 *   q, k, b, log_alpha: [total_T, H, Dk]; v, w, o (and gradients): [total_T, H, Dv];
 *   S0, S_T, dS_T, dS0: [N, H, Dk, Dv] fp32, one state per sequence and head.
 * Every sequence runs the recurrence of gdn2_chunk_fwd / gdn2_chunk_bwd on its own,
 * from its own S0.  cu_seqlens lives on the device, so the library cannot check it
 * before launching: a kernel that finds it invalid skips the affected sequences and
 * records GDN2_ERR_SEQLENS for gdn2_sync_status.  When total_T == 0 it is not read.
 * Workspace: gdn2_workspace_size(2, ...) (forward, 0) and gdn2_workspace_size(3, ...)
 * (backward), with B = N and T = total_T.
 */
GDN2_API gdn2_status gdn2_chunk_fwd_varlen(gdn2_dtype dt, int N, int total_T, int H, int Dk, int Dv,
                           const int *cu_seqlens, const void *q, const void *k, const void *v,
                           const float *log_alpha, const void *b, const void *w, const float *S0,
                           void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream);

GDN2_API gdn2_status gdn2_chunk_bwd_varlen(gdn2_dtype dt, int N, int total_T, int H, int Dk, int Dv,
                           const int *cu_seqlens, const void *q, const void *k, const void *v,
                           const float *log_alpha, const void *b, const void *w, const float *S0,
                           const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream);

/*
 * Gate layouts.  The calls above take every gate with one value per channel.  The
 * *_gated calls take a flags word that gives each gate one of three layouts:
 *   per channel (no flag): as above, [B, T, H, D];
 *   scalar (GDN2_*_SCALAR): one value per token and head, [B, T, H] (decode:
 *     [N, H]), used for every channel;
 *   absent (GDN2_*_NONE): the pointer is ignored; b and w are 1 and log_alpha is 0.
 * With b = w = beta scalar the recurrence is KDA; with a scalar decay as well it
 * is Gated DeltaNet; with no decay and scalar b = w it is DeltaNet (the
 * needhelp.icu write-up's generalisation hierarchy).  Absent b or w gives the
 * write-only and erase-only ablations of the aixai.ru post ("Абляции").
 * The results are identical to the plain calls made with the gates broadcast to
 * per-channel tensors.  The decode step reads every layout as it is.  In the bf16 chunk
 * calls the kernels read a scalar decay, and scalar b and w together (without the prologue
 * flags, in the backward), as they are, one value per token; every other scalar or absent
 * gate of the chunk calls is broadcast into the workspace first.  In the backward the gradient of a scalar gate is the sum of the per-channel
 * gradients over the channels (the order of that sum, so its last bits, depends on which
 * of the two routes ran); the other gradients are identical.  An absent gate's gradient pointer is
 * ignored (NULL allowed).  Flags outside the eight below, or scalar and absent set
 * for one gate, give GDN2_ERR_UNSUPPORTED.
 * Workspace: gdn2_workspace_size_gated(which, flags, ...) with which = 0 (forward),
 * 1 (backward), 2 (decode; B = N, T ignored).  Where it returns 0 the call needs no
 * workspace (NULL allowed): the decode step without the prologue pass, and the bf16
 * forward whose gates the kernels read as they are.  Fixed-length batches only.
 *
 * Input prologue (two more flags, combinable with the layouts above).  The aixai.ru
 * post's architecture paragraph normalises queries and keys before the recurrent update
 * and takes the erase and write gates from their own projections; log alpha is computed
 * outside the kernel, so it stays an input here.
 *   GDN2_QK_L2NORM: q and k are raw; each token's q and k (per head, over the head
 *     dimension) is replaced by x / sqrt(sum x^2 + 1e-6) in fp32.
 *   GDN2_BW_LOGITS: b and w, where present, are logits (either layout) and pass through
 *     the logistic sigmoid 1 / (1 + e^-x).
 * The bf16 forward with per-channel b and w applies both inside the tensor-core chunk
 * kernel (the sigmoid there goes through the hardware tanh, 1/2 + tanh(x/2)/2), and the
 * decode step with per-channel b and w inside its kernel; every other call writes the
 * normalised / activated inputs into its workspace first.  The
 * backward returns dq, dk for the raw q, k and db, dw for the logits.
 */
typedef enum {
    GDN2_DECAY_SCALAR = 1,
    GDN2_ERASE_SCALAR = 2,
    GDN2_WRITE_SCALAR = 4,
    GDN2_DECAY_NONE = 8,
    GDN2_ERASE_NONE = 16,
    GDN2_WRITE_NONE = 32,
    GDN2_QK_L2NORM = 64,
    GDN2_BW_LOGITS = 128
} gdn2_gate_flags;

GDN2_API gdn2_status gdn2_chunk_fwd_gated(int flags, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream);

GDN2_API gdn2_status gdn2_chunk_bwd_gated(int flags, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *S0,
                           const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream);

GDN2_API gdn2_status gdn2_decode_step_gated(int flags, gdn2_dtype dt, int N, int H, int Dk, int Dv,
                           const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, float *S, void *o,
                           void *workspace, size_t ws_bytes, void *stream);

GDN2_API size_t gdn2_workspace_size_gated(int which, int flags, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv);

/* The input prologue on its own (the pass the gated calls run before the recurrence where
 * it is not fused): for N token rows of H heads and head size D, writes
 *   q_n, k_n = x / sqrt(sum x^2 + 1e-6) per (row, head)      (flags & GDN2_QK_L2NORM)
 *   b_s, w_s = 1 / (1 + e^-x)                               (flags & GDN2_BW_LOGITS)
 * with b and w per channel [N, H, D] or per token [N, H] as GDN2_ERASE_SCALAR /
 * GDN2_WRITE_SCALAR say, or skipped with GDN2_ERASE_NONE / GDN2_WRITE_NONE.  Inputs and
 * outputs have dtype dt (bf16 results are rounded once from fp32); outputs that the flags
 * do not ask for may be NULL.  Decay flags are ignored.  Asynchronous on `stream`.
 * Errors: GDN2_ERR_SHAPE for N < 0 or H < 1, GDN2_ERR_UNSUPPORTED for D not 64 or 128 or
 * unknown flags, GDN2_ERR_NULL / GDN2_ERR_ALIGN for a missing or unaligned tensor that the
 * flags need. */
GDN2_API gdn2_status gdn2_prologue(int flags, gdn2_dtype dt, int N, int H, int D, const void *q, const void *k,
                                   const void *b, const void *w, void *q_n, void *k_n, void *b_s, void *w_s,
                                   void *stream);

/* Workspace bytes for which = 0 (gdn2_chunk_fwd), 1 (gdn2_chunk_bwd),
 * 2 (gdn2_chunk_fwd_varlen), 3 (gdn2_chunk_bwd_varlen, B = N, T = total_T) or
 * 4 (gdn2_chunk_fwd_host's device staging); 0 for invalid or unsupported arguments. */
GDN2_API size_t gdn2_workspace_size(int which, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv);

/* Static, NUL-terminated description of a status code. */
GDN2_API const char *gdn2_strerror(gdn2_status status);

/* Synchronises `stream`, then returns and clears the current device's kernel
 * status word: GDN2_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last check, GDN2_ERR_SEQLENS if a kernel found cu_seqlens invalid,
 * GDN2_ERR_CUDA if the stream reported an error, else GDN2_OK. */
GDN2_API gdn2_status gdn2_sync_status(void *stream);

/* Failure-detection self-test.  Enqueues one block whose thread waits on an mbarrier phase
 * that nothing completes, bounded by `limit_us` microseconds: the same bounded wait every
 * tensor-core kernel uses.  When the wait gives up, the kernel records a timeout in the status
 * word, as a kernel that lost a transfer would, and returns.  The next gdn2_sync_status()
 * reports GDN2_ERR_TIMEOUT (and clears it); the context stays usable.  Asynchronous on
 * `stream`.  GDN2_ERR_SHAPE for limit_us outside 1 .. 100000 (nothing is launched). */
GDN2_API gdn2_status gdn2_selftest_timeout(int limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
