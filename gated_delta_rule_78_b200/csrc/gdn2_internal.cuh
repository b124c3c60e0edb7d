// Internal declarations shared by the kernels and the C ABI layer of libgdn2.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn2.h"

namespace gdn2 {

constexpr int kChunk = 64;  // tokens per chunk

// Device status word values (written by kernels, read by gdn2_sync_status).
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadSeqlens = 2;  // cu_seqlens not non-decreasing inside [0, total_T]

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Problem description handed from the C ABI layer to the launchers.  All
// pointers are device pointers; layouts as in gdn2.h.
//
// Fixed length (cu_seqlens == null): B sequences of T tokens, tensors [B, T, H, D].
// Variable length: B sequences packed into T rows, tensors [T, H, D]; sequence n is rows
// cu_seqlens[n] .. cu_seqlens[n+1].  chunk_off (device, B + 1 entries, variable length
// only, filled by launch_chunk_offsets) is the exclusive prefix sum of the sequences'
// chunk counts; per-chunk workspace lists of (sequence n, head h) start at
// chunk_off[n] * H + h * nchunks(n), which for fixed length is (n * H + h) * nchunks.
struct Problem {
    int B, T, H, D;  // Dk == Dv == D
    const void *q, *k, *v, *b, *w;
    const float *g;   // log alpha
    const float *S0;  // may be null
    const int *cu_seqlens = nullptr;
    const int *chunk_off = nullptr;
    bool g_scalar = false;  // bf16 tensor-core paths only: log alpha is [rows, H] (one decay per head),
                            // and in the backward so is dlog alpha
    bool bw_scalar = false; // bf16 tensor-core paths only: b and w are [rows, H] (one gate value each per
                            // head), and in the backward so are db and dw
    int prologue = 0;       // tensor-core forward only: kProNorm | kProSigmoid, applied inside the kernel
};

// Fused input prologue (tensor-core forward): q and k are L2-normalised per token and head,
// x / sqrt(sum x^2 + kNormEps); b and w are logits and pass through the logistic sigmoid.
constexpr int kProNorm = 1;
constexpr int kProSigmoid = 2;
constexpr float kNormEps = 1e-6f;

// rows of the token tensors
__host__ __device__ inline size_t token_rows(const Problem &p)
{
    return p.cu_seqlens ? (size_t)p.T : (size_t)p.B * p.T;
}
// upper bound of the total number of chunks over all sequences (per head)
__host__ __device__ inline size_t chunk_bound(const Problem &p)
{
    return p.cu_seqlens ? (size_t)(p.T + kChunk - 1) / kChunk + p.B : (size_t)p.B * ((p.T + kChunk - 1) / kChunk);
}

struct SeqSpan {
    int bos, len;  // first row and token count of the sequence
};
// Span of sequence n; len = -1 marks invalid cu_seqlens (the caller reports it).
__device__ __forceinline__ SeqSpan seq_span(const Problem &p, int n)
{
    if (!p.cu_seqlens) return {n * p.T, p.T};
    const int b0 = p.cu_seqlens[n], b1 = p.cu_seqlens[n + 1];
    if (b0 < 0 || b1 < b0 || b1 > p.T) return {0, -1};
    return {b0, b1 - b0};
}
__device__ __forceinline__ int seq_chunks(int len) { return (len + kChunk - 1) / kChunk; }
// first chunk (over all sequences) of sequence n
__device__ __forceinline__ size_t chunk_first(const Problem &p, int n)
{
    return p.chunk_off ? (size_t)p.chunk_off[n] : (size_t)n * seq_chunks(p.T);
}
// index of chunk ci of (sequence n, head h) in a per-chunk workspace list
__device__ __forceinline__ size_t chunk_slot(const Problem &p, int n, int h, int nch, int ci)
{
    return chunk_first(p, n) * p.H + (size_t)h * nch + ci;
}
// index of boundary state ci (0 .. nch) of (sequence n, head h) in a per-boundary list
__device__ __forceinline__ size_t bound_slot(const Problem &p, int n, int h, int nch, int ci)
{
    return (chunk_first(p, n) + n) * p.H + (size_t)h * (nch + 1) + ci;
}
// A chunk of the chunk-parallel kernels: (chunk gc over all sequences, head h) -> sequence n,
// chunk ci of its nch, its span and its per-chunk workspace slot.  Fixed length: gc is
// sequence-major; variable length: the sequence is found in chunk_off.  False for chunk indices
// past the last chunk and for sequences with invalid cu_seqlens.
struct ChunkRef {
    int n, h, ci, nch;
    SeqSpan sp;
    size_t cidx;
};
__device__ __forceinline__ bool chunk_at(const Problem &p, int gc, int h, ChunkRef &r)
{
    r.h = h;
    if (!p.cu_seqlens) {
        const int nc = seq_chunks(p.T);
        if (nc == 0) return false;
        r.n = gc / nc;
        r.ci = gc % nc;
        if (r.n >= p.B) return false;
    } else {
        if (gc >= p.chunk_off[p.B]) return false;
        int lo = 0, hi = p.B;  // last n with chunk_off[n] <= gc
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.chunk_off[mid] <= gc) lo = mid;
            else hi = mid;
        }
        r.n = lo;
        r.ci = gc - p.chunk_off[lo];
    }
    r.sp = seq_span(p, r.n);
    if (r.sp.len < 0) return false;
    r.nch = seq_chunks(r.sp.len);
    if (r.ci >= r.nch) return false;
    r.cidx = chunk_slot(p, r.n, r.h, r.nch, r.ci);
    return true;
}
// offset of token row t of sequence span sp, head h, in a [rows, H, D] tensor
__device__ __forceinline__ size_t tok_row(const Problem &p, const SeqSpan &sp, int h, int t)
{
    return ((size_t)(sp.bos + t) * p.H + h) * p.D;
}

// Variable length: checks cu_seqlens (sets the status word to kStatusBadSeqlens if it is
// not non-decreasing inside [0, total_rows]) and writes chunk_off (n_seqs + 1 ints) when
// chunk_off is non-null.  One small launch.
cudaError_t launch_chunk_offsets(const int *cu_seqlens, int n_seqs, int total_rows, int *chunk_off, int *status,
                                 cudaStream_t s);

// Chunks whose decay is too strong for the chunkwise factors.  The tensor-core kernels form
// e^{-G} (G the cumulative log-decay inside a chunk, non-increasing) for the factor K~ = k e^{-G};
// with the chunk's total log-decay at or above -kChunkDecayLimit on every channel, e^{-G} <= e^{80}
// and all factors and products stay finite in fp32 and bf16.  Chunks past that limit run the
// token-by-token form instead (tok_util.cuh), which is exact for any decay.
constexpr float kChunkDecayLimit = 80.f;

// The token-level forward (tok.cu): the fp32 path, any head size.  `states`, when non-null,
// receives the fp32 state S ([c][j], d_k rows) at every chunk boundary, at the boundary slots
// (bound_slot).  `o` may be null (states only).
cudaError_t launch_fwd_tok(gdn2_dtype dt, const Problem &p, void *o, float *S_T, float *states, cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit on the current device (once per
// kernel and device; thread-safe).
cudaError_t set_smem_attr(const void *kernel, int bytes);

// forward on the tensor cores (bf16 operands); returns cudaErrorNotSupported when
// the shape is outside what the kernel handles.  `o` may be null (no output);
// `states`, when non-null, receives S^T in bf16 at every chunk boundary:
// [B*H][nchunks + 1][D][D], entry c the state before chunk c, the last entry S_T.
// Chunk-parallel scan of the forward (scan.cu): each sequence is cut into nseg segments, the
// first of seg0_len tokens and the others of seg_len (multiples of the chunk; the last may be
// shorter).  Pass 0 runs, in one launch, segment 0 from S0 with
// its output (end state -> send0), and for every middle segment s = 1 .. nseg-2 its local end
// state from zero (-> shat) and its transition, the state map's linear part applied to the
// identity (-> phi).  The combine gives every later segment its start state (sstart); pass 1
// runs segments 1 .. nseg-1 from those with their output, the last one writing S_T.
// Layouts, fp32 [.., H, D, D]: send0 [B], shat and phi [B][nseg-2], sstart [B][nseg-1].
struct ScanArgs {
    int nseg, seg_len, pass, seg0_len;
    float *send0, *shat, *phi;
    const float *sstart;
};

// The backward's per-chunk factors, written by the tensor-core forward in states mode for the
// dS chain and the gradient kernel (chunk slots of chunk_slot): W^T [D][C], K~ [C][D], M^T [D][C]
// with M = Q~ - P W (so that R = Q~^T dO - W^T P^T dO = M^T dO), T = (I + A)^-1 and P [C][C], all
// bf16 with D = 128; gamma [kGamStride] fp32 with the chunk's token-mode flag
// (an int) after the D values; flist[0] counts the chunks that run token by token and flist[1 ..]
// lists them as tasks gc + nchb h (gc the chunk over all sequences).
constexpr int kGamStride = 128 + 4;
struct BwdFactors {
    __nv_bfloat16 *W = nullptr, *Kt = nullptr, *Mc = nullptr, *Tm = nullptr, *Pm = nullptr;
    float *gam = nullptr;
    int *flist = nullptr;
    int nchb = 0;
};

// Workspace of the chunk-parallel scan for this problem; 0 when the scan is not used for it
// (variable length, scalar decay, prologue, more than 48 chains, or short sequences).
size_t fwd_scan_workspace_bytes(const Problem &p);
cudaError_t launch_fwd_scan(const Problem &p, void *o, float *S_T, void *ws, size_t ws_bytes, int *status,
                            cudaStream_t s);

// The forward on host buffers (host_fwd.cu): device staging bytes, and the pipelined run;
// `run` is the device forward on one slice.
size_t host_fwd_workspace_bytes(size_t elem_bytes, int B, int T, int H, int D);
cudaError_t launch_fwd_host(gdn2_dtype dt, int B, int T, int H, int D, const void *q, const void *k, const void *v,
                            const float *g, const void *b, const void *w, const float *S0, void *o, float *S_T,
                            void *ws, cudaStream_t s,
                            cudaError_t (*run)(gdn2_dtype, const Problem &, void *, float *, cudaStream_t));

// The input prologue as separate passes (prologue.cu).  rows = token rows x heads; gate modes:
// 0 untouched, 1 per channel ([rows, D]), 2 per token ([rows]).
cudaError_t launch_prologue_fwd(bool fp32, size_t rows, int D, bool norm, const void *q, const void *k, void *qn,
                                void *kn, int b_mode, const void *b, void *bs, int w_mode, const void *w, void *ws,
                                cudaStream_t s);
cudaError_t launch_prologue_bwd(bool fp32, size_t rows, int D, bool norm, const void *q, const void *k, void *dq,
                                void *dk, int b_mode, const void *b, void *db, int w_mode, const void *w, void *dw,
                                cudaStream_t s);
cudaError_t launch_fwd_tc(const Problem &p, void *o, float *S_T, __nv_bfloat16 *states, int *status,
                          cudaStream_t s,
                          const ScanArgs *scan = nullptr, const BwdFactors *bw = nullptr);

// gate_modes: two bits per gate (log alpha, b, w from bit 0 up): kGateChannel (one value per
// channel), kGateScalar (one per sequence and head), kGateAbsent (log alpha 0, b and w 1)
constexpr int kGateChannel = 0, kGateScalar = 1, kGateAbsent = 2;
cudaError_t launch_decode(gdn2_dtype dt, int N, int H, int D, const void *q, const void *k,
                          const void *v, const float *g, const void *b, const void *w, float *S,
                          void *o, cudaStream_t s, int prologue = 0, int gate_modes = 0);

struct BwdOut {
    void *dq, *dk, *dv, *db, *dw;
    float *dg, *dS0;
};
// bytes reserved at the front of a variable-length workspace for chunk_off (256-aligned)
inline size_t varlen_offsets_bytes(int n_seqs) { return ((size_t)(n_seqs + 1) * sizeof(int) + 255) / 256 * 256; }

// Backward workspace bytes (depends on the path: bf16 with D = 128 runs on the
// tensor cores, everything else on the token-level kernels).  Only the sizes and
// whether cu_seqlens is set are read from p.
size_t bwd_workspace_bytes(gdn2_dtype dt, const Problem &p);
// states_saved: the bf16 backward's chunk-boundary states are already in ws (launch_fwd_save
// wrote them with the same inputs), so its states pass is skipped; ignored for fp32.
cudaError_t launch_bwd(gdn2_dtype dt, const Problem &p, const void *d_o, const float *dS_T,
                       const BwdOut &out, void *ws, cudaStream_t s, bool states_saved = false);

// Token-level gradients of whole chunks (tok.cu), the exact path for chunks flagged by the
// tensor-core backward: given each chunk's start state (the tensor-core workspace's bf16 S^T,
// 128 x 128 per boundary slot) and its end-state gradient (bf16 dS^T, 128 x 128 per chunk slot),
// writes dq, dk, dv, db, dw and dlog alpha of the chunk's tokens.  `list` (device): list[0]
// chunk tasks follow, each gc + chunk_bound * h.  `scratch`: nblocks x tok_grad_block_bytes(D).
size_t tok_grad_block_bytes(int D);
cudaError_t launch_tok_grad_tc(const Problem &p, const void *d_o, const __nv_bfloat16 *states,
                               const __nv_bfloat16 *dSn, const int *list, float *scratch, int nblocks,
                               const BwdOut &out, cudaStream_t s);

// tensor-core backward (bf16, D = 128): the forward in states mode (which also stores the
// chunk factors), then the chain and gradient kernels, then the token-form gradients of the
// chunks past the factors' range
size_t bwd_tc_workspace_bytes(const Problem &p);
cudaError_t launch_bwd_tc(const Problem &p, const void *d_o, const float *dS_T, const BwdOut &out, void *ws,
                          int *status, cudaStream_t s, bool states_saved = false);
// the bf16 forward (o, S_T) that also records the chunk-boundary states and factors into the
// backward's workspace ws, for launch_bwd_tc(..., states_saved = true); fixed-length batches
cudaError_t launch_fwd_save(const Problem &p, void *o, float *S_T, void *ws, int *status, cudaStream_t s);

// Gate layouts (gates.cu): fill dst ([n_rows, D]) with src[row] (a per-row scalar) or,
// when src is null, with `fill`; and sum src ([n_rows, D]) over D into dst ([n_rows]).
// fp32 selects float, otherwise bf16.
cudaError_t launch_expand_gate(bool fp32, const void *src, void *dst, size_t n_rows, int D, float fill, cudaStream_t s);
cudaError_t launch_channel_sum(bool fp32, const void *src, void *dst, size_t n_rows, int D, cudaStream_t s);

// device address of the library's kernel status word on the current device
int *status_word();
// Argument checks of the backward entry points (sizes inside the contract, required pointers
// non-null, every pointer 16-byte aligned), shared by gdn2_chunk_bwd and gdn2_chunk_bwd_noalloc
// so that both reject exactly the same calls.
gdn2_status check_bwd_args(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q, const void *k,
                           const void *v, const float *log_alpha, const void *b, const void *w, const float *S0,
                           const void *d_o, const float *dS_T, const void *dq, const void *dk, const void *dv,
                           const float *dlog_alpha, const void *db, const void *dw, const float *dS0);
// Failure-detection self-test (selftest.cu): one bounded wait on a phase nothing completes.
cudaError_t launch_selftest_timeout(int limit_us, int *status, cudaStream_t s);

}  // namespace gdn2
