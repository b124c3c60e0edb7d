// C ABI of libgdn2.so: argument validation, workspace sizing, kernel dispatch.
// Declarations and the contract of every entry point are in include/gdn2.h.
#include <vector>
#include <string.h>
#include <stdint.h>

#include <mutex>

#include "gdn2_internal.cuh"

namespace gdn2 {

cudaError_t set_smem_attr(const void *kernel, int bytes)
{
    // (kernel, device) pairs already raised; a small table is enough for the handful of kernels here
    struct Entry { const void *fn; uint64_t devices; };
    static Entry table[32];
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    std::lock_guard<std::mutex> lock(mu);
    int slot = -1;
    for (int i = 0; i < 32; ++i) {
        if (table[i].fn == kernel) { slot = i; break; }
        if (!table[i].fn && slot < 0) slot = i;
    }
    if (slot >= 0 && table[slot].fn == kernel && (table[slot].devices >> dev & 1u)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && slot >= 0) {
        table[slot].fn = kernel;
        table[slot].devices |= 1ull << dev;
    }
    return e;
}

}  // namespace gdn2

// Per-device kernel status word (0 = fine).  Kernels that give up a bounded
// wait store a non-zero code here; gdn2_sync_status() reads and clears it.
__device__ int g_gdn2_status = 0;

int *gdn2::status_word()
{
    int *p = nullptr;
    return cudaGetSymbolAddress((void **)&p, g_gdn2_status) == cudaSuccess ? p : nullptr;
}

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

gdn2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA; }

// Common checks for the chunked entry points.  Returns GDN2_OK when the sizes
// are inside the v1 contract.
gdn2_status check_sizes(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv)
{
    if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (B <= 0 || H <= 0 || T < 0 || Dk <= 0 || Dv <= 0) return GDN2_ERR_SHAPE;
    if (Dk != Dv || (Dk != 64 && Dk != 128)) return GDN2_ERR_UNSUPPORTED;
    // element counts must fit comfortably in the kernels' 64-bit index math and
    // the grid's x dimension
    if ((long long)B * H > (1LL << 30) || H > 65535) return GDN2_ERR_UNSUPPORTED;
    if ((long long)B * T * H * Dk > (1LL << 40)) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

gdn2_status check_ptrs(std::initializer_list<const void *> required,
                       std::initializer_list<const void *> optional)
{
    for (const void *p : required)
        if (!p) return GDN2_ERR_NULL;
    for (const void *p : required)
        if (!aligned16(p)) return GDN2_ERR_ALIGN;
    for (const void *p : optional)
        if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
    return GDN2_OK;
}

gdn2::Problem make_problem(int B, int T, int H, int D, const void *q, const void *k, const void *v,
                           const float *g, const void *b, const void *w, const float *S0)
{
    gdn2::Problem p;
    p.B = B; p.T = T; p.H = H; p.D = D;
    p.q = q; p.k = k; p.v = v; p.b = b; p.w = w; p.g = g; p.S0 = S0;
    return p;
}

// Launch the forward of a validated problem (T > 0): bf16 with D = 128 on the tensor
// cores, everything else (fp32) on the token-level kernel.  Variable length first checks cu_seqlens.
gdn2_status run_fwd(gdn2_dtype dt, const gdn2::Problem &p, void *o, float *S_T, cudaStream_t s);
// the device forward of one host-pipeline slice
cudaError_t run_fwd_slice(gdn2_dtype dt, const gdn2::Problem &p, void *o, float *S_T, cudaStream_t s)
{
    return run_fwd(dt, p, o, S_T, s) == GDN2_OK ? cudaSuccess : cudaErrorLaunchFailure;
}

gdn2_status run_fwd(gdn2_dtype dt, const gdn2::Problem &p, void *o, float *S_T, cudaStream_t s)
{
    int *status = gdn2::status_word();
    if (!status) return GDN2_ERR_CUDA;
    if (p.cu_seqlens) {
        cudaError_t e = gdn2::launch_chunk_offsets(p.cu_seqlens, p.B, p.T, nullptr, status, s);
        if (e != cudaSuccess) return GDN2_ERR_CUDA;
    }
    if (dt == GDN2_BF16) {
        cudaError_t e = gdn2::launch_fwd_tc(p, o, S_T, nullptr, status, s);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();  // clear the sticky "not supported" code; fall through to the token-level path
    }
    return from_cuda(gdn2::launch_fwd_tok(dt, p, o, S_T, nullptr, s));
}


// ---- gate layouts (the gdn2_*_gated entry points)
// gate i: 0 = log decay, 1 = erase gate b, 2 = write gate w
bool gate_scalar(int flags, int i) { return (flags >> i) & 1; }
bool gate_none(int flags, int i) { return (flags >> (3 + i)) & 1; }
bool gate_full(int flags, int i) { return !gate_scalar(flags, i) && !gate_none(flags, i); }

gdn2_status check_gate_flags(int flags)
{
    if (flags & ~0xFF) return GDN2_ERR_UNSUPPORTED;
    for (int i = 0; i < 3; ++i)
        if (gate_scalar(flags, i) && gate_none(flags, i)) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// The input prologue: GDN2_QK_L2NORM normalises q and k, GDN2_BW_LOGITS takes b and w (where
// present) as logits.  The bf16 forward with per-channel b and w applies it inside the
// tensor-core kernel; every other call runs it as a pass into the workspace first.
bool pro_any(int flags) { return flags & (GDN2_QK_L2NORM | GDN2_BW_LOGITS); }
// b and w both one value per (token, head): the bf16 forward reads them as they are
bool bw_native(int flags, gdn2_dtype dt) { return dt == GDN2_BF16 && gate_scalar(flags, 1) && gate_scalar(flags, 2); }
// ... and the bf16 backward, without the prologue (whose backward pass wants per-channel gates)
bool bw_native_bwd(int flags, gdn2_dtype dt) { return bw_native(flags, dt) && !pro_any(flags); }
// a scalar decay: the bf16 forward and backward read it as it is (the prologue leaves log alpha alone)
bool decay_native(int flags, gdn2_dtype dt) { return dt == GDN2_BF16 && gate_scalar(flags, 0); }
bool pro_fused(int flags, gdn2_dtype dt)
{
    return dt == GDN2_BF16 && ((gate_full(flags, 1) && gate_full(flags, 2)) || bw_native(flags, dt));
}
// prologue mode of gate i (1 = b, 2 = w): 0 none, 1 per channel, 2 per token
int pro_gate_mode(int flags, int i)
{
    if (!(flags & GDN2_BW_LOGITS) || gate_none(flags, i)) return 0;
    return gate_scalar(flags, i) ? 2 : 1;
}

// [prologue outputs q_n | k_n | b_s | w_s] [expanded g | b | w]
// [full-size gradients of dg | db | dw (backward)] [core workspace]
struct GatedWs {
    size_t pro[4], off[3], grad[3], core, total;
};
// The chunk kernels keep some scalar gates as they are, which then need no broadcast copy and,
// in the backward, no full-size gradient: bw_kept (scalar b and w together) and decay_kept (a
// scalar decay, bf16).
GatedWs gated_ws(bool bwd, int flags, gdn2_dtype dt, size_t rows, int H, int D, size_t core_bytes, bool pro_pass,
                 bool bw_kept = false, bool decay_kept = false)
{
    GatedWs l;
    const size_t n = rows * H * D;
    const size_t es[3] = {4, dt == GDN2_F32 ? 4u : 2u, dt == GDN2_F32 ? 4u : 2u};
    size_t off = 0;
    for (int i = 0; i < 4; ++i) {
        l.pro[i] = off;
        if (!pro_pass) continue;
        if (i < 2 && (flags & GDN2_QK_L2NORM)) off += round256(n * es[1]);
        if (i >= 2) {
            const int m = pro_gate_mode(flags, i - 1);
            if (m) off += round256((m == 1 ? n : rows * H) * es[1]);
        }
    }
    for (int i = 0; i < 3; ++i) {
        l.off[i] = off;
        if (!gate_full(flags, i) && !(bw_kept && i > 0) && !(decay_kept && i == 0)) off += round256(n * es[i]);
    }
    for (int i = 0; i < 3; ++i) {
        l.grad[i] = off;
        if (bwd && !gate_full(flags, i) && !(bw_kept && i > 0) && !(decay_kept && i == 0)) off += round256(n * es[i]);
    }
    l.core = off;
    l.total = off + core_bytes;
    return l;
}

// Broadcast the non-per-channel gates into the workspace; gp[i] is replaced by the full
// tensor's address.  Absent gates are 0 (log decay) or 1 (b, w).
gdn2_status expand_gates(int flags, gdn2_dtype dt, const GatedWs &l, char *ws, size_t rows, int H, int D,
                         const void *gp[3], cudaStream_t s, bool bw_kept = false)
{
    for (int i = 0; i < 3; ++i) {
        if (gate_full(flags, i) || (bw_kept && i > 0)) continue;
        void *dst = ws + l.off[i];
        const bool fp32 = (i == 0) || dt == GDN2_F32;
        cudaError_t e = gdn2::launch_expand_gate(fp32, gate_none(flags, i) ? nullptr : gp[i], dst, rows * H, D,
                                                 i == 0 ? 0.f : 1.f, s);
        if (e != cudaSuccess) return GDN2_ERR_CUDA;
        gp[i] = dst;
    }
    return GDN2_OK;
}

// The prologue as a pass: q, k, b, w are replaced by the normalised / activated copies.
gdn2_status prologue_pass(int flags, gdn2_dtype dt, const GatedWs &l, char *ws, size_t rows, int H, int D,
                          const void *&q, const void *&k, const void *&b, const void *&w, cudaStream_t s)
{
    const bool norm = flags & GDN2_QK_L2NORM;
    const int bm = pro_gate_mode(flags, 1), wm = pro_gate_mode(flags, 2);
    void *qn = norm ? ws + l.pro[0] : nullptr, *kn = norm ? ws + l.pro[1] : nullptr;
    void *bs = bm ? ws + l.pro[2] : nullptr, *wsg = wm ? ws + l.pro[3] : nullptr;
    if (gdn2::launch_prologue_fwd(dt == GDN2_F32, rows * H, D, norm, q, k, qn, kn, bm, b, bs, wm, w, wsg, s) !=
        cudaSuccess)
        return GDN2_ERR_CUDA;
    if (norm) {
        q = qn;
        k = kn;
    }
    if (bm) b = bs;
    if (wm) w = wsg;
    return GDN2_OK;
}

gdn2_status check_gate_ptrs(int flags, const void *g, const void *b, const void *w)
{
    const void *gp[3] = {g, b, w};
    for (int i = 0; i < 3; ++i) {
        if (gate_none(flags, i)) continue;
        if (!gp[i]) return GDN2_ERR_NULL;
        if (!aligned16(gp[i])) return GDN2_ERR_ALIGN;
    }
    return GDN2_OK;
}
}  // namespace

gdn2_status gdn2::check_bwd_args(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q, const void *k,
                                 const void *v, const float *log_alpha, const void *b, const void *w, const float *S0,
                                 const void *d_o, const float *dS_T, const void *dq, const void *dk, const void *dv,
                                 const float *dlog_alpha, const void *db, const void *dw, const float *dS0)
{
    gdn2_status st = check_sizes(dt, B, T, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    if (T > 0) return check_ptrs({q, k, v, log_alpha, b, w, d_o, dq, dk, dv, dlog_alpha, db, dw, dS0}, {S0, dS_T});
    return check_ptrs({dS0}, {S0, dS_T});
}

namespace {
gdn2_status chunk_bwd_impl(bool saved, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q,
                           const void *k, const void *v, const float *log_alpha, const void *b,
                           const void *w, const float *S0, const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream)
{
    const gdn2_status st = gdn2::check_bwd_args(dt, B, T, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, d_o, dS_T, dq, dk,
                                                dv, dlog_alpha, db, dw, dS0);
    if (st != GDN2_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
    if (T == 0) {
        if (dS_T) return from_cuda(cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(dS0, 0, state_bytes, s));
    }
    const size_t need = gdn2::bwd_workspace_bytes(dt, make_problem(B, T, H, Dk, nullptr, nullptr, nullptr, nullptr,
                                                                    nullptr, nullptr, nullptr));
    if (!workspace || ws_bytes < need) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    gdn2::Problem p = make_problem(B, T, H, Dk, q, k, v, log_alpha, b, w, S0);
    gdn2::BwdOut out{dq, dk, dv, db, dw, dlog_alpha, dS0};
    return from_cuda(gdn2::launch_bwd(dt, p, d_o, dS_T, out, workspace, s, saved));
}

}  // namespace

extern "C" {

const char *gdn2_strerror(gdn2_status s)
{
    switch (s) {
    case GDN2_OK: return "success";
    case GDN2_ERR_NULL: return "a required pointer is NULL";
    case GDN2_ERR_SHAPE: return "invalid size (negative, or zero where positive is required)";
    case GDN2_ERR_DTYPE: return "unknown dtype";
    case GDN2_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case GDN2_ERR_WORKSPACE: return "workspace missing or too small";
    case GDN2_ERR_CUDA: return "a CUDA runtime call failed";
    case GDN2_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case GDN2_ERR_UNSUPPORTED: return "outside the supported shapes (Dk == Dv in {64, 128})";
    case GDN2_ERR_TOO_LARGE: return "problem needs more scratch than the library's static array holds";
    case GDN2_ERR_SEQLENS: return "cu_seqlens is not 0 = c_0 <= c_1 <= ... <= c_N = total_T";
    }
    return "unknown status";
}

size_t gdn2_workspace_size(int which, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv)
{
    if (check_sizes(dt, B, T, H, Dk, Dv) != GDN2_OK) return 0;
    if (T == 0 || which == 2) return 0;
    if (which == 4) return gdn2::host_fwd_workspace_bytes(dt == GDN2_F32 ? 4 : 2, B, T, H, Dk);
    if (which != 0 && which != 1 && which != 3) return 0;
    gdn2::Problem p = make_problem(B, T, H, Dk, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
    if (which == 0) return dt == GDN2_BF16 ? gdn2::fwd_scan_workspace_bytes(p) : 0;  // the chunk-parallel scan
    static const int marker = 0;
    if (which == 3) p.cu_seqlens = &marker;  // sizes only: the pointer is not read
    return gdn2::bwd_workspace_bytes(dt, p);
}

gdn2_status gdn2_chunk_fwd(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q,
                           const void *k, const void *v, const float *log_alpha, const void *b,
                           const void *w, const float *S0, void *o, float *S_T, void *workspace,
                           size_t ws_bytes, void *stream)
{
    gdn2_status st = check_sizes(dt, B, T, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    if (T > 0) st = check_ptrs({q, k, v, log_alpha, b, w, o}, {S0, S_T});
    else st = check_ptrs({}, {S0, S_T});
    if (st != GDN2_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
    if (T == 0) {
        if (!S_T) return GDN2_OK;
        if (S0) return S0 == S_T ? GDN2_OK : from_cuda(cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(S_T, 0, state_bytes, s));
    }
    gdn2::Problem p = make_problem(B, T, H, Dk, q, k, v, log_alpha, b, w, S0);
    const size_t scan_need = dt == GDN2_BF16 ? gdn2::fwd_scan_workspace_bytes(p) : 0;
    if (scan_need && workspace && ws_bytes >= scan_need && aligned16(workspace)) {  // few long chains
        int *status = gdn2::status_word();
        if (!status) return GDN2_ERR_CUDA;
        return from_cuda(gdn2::launch_fwd_scan(p, o, S_T, workspace, ws_bytes, status, s));
    }
    return run_fwd(dt, p, o, S_T, s);
}

gdn2_status gdn2_decode_step(gdn2_dtype dt, int N, int H, int Dk, int Dv, const void *q,
                             const void *k, const void *v, const float *log_alpha, const void *b,
                             const void *w, float *S, void *o, void *stream)
{
    gdn2_status st = check_sizes(dt, N, 1, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    st = check_ptrs({q, k, v, log_alpha, b, w, S, o}, {});
    if (st != GDN2_OK) return st;
    return from_cuda(gdn2::launch_decode(dt, N, H, Dk, q, k, v, log_alpha, b, w, S, o,
                                         (cudaStream_t)stream));
}

gdn2_status gdn2_chunk_bwd(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q,
                           const void *k, const void *v, const float *log_alpha, const void *b,
                           const void *w, const float *S0, const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream)
{
    return chunk_bwd_impl(false, dt, B, T, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, d_o, dS_T, dq, dk, dv, dlog_alpha, db, dw, dS0, workspace, ws_bytes, stream);
}

gdn2_status gdn2_chunk_bwd_saved(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q,
                           const void *k, const void *v, const float *log_alpha, const void *b,
                           const void *w, const float *S0, const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                           float *dS0, void *workspace, size_t ws_bytes, void *stream)
{
    return chunk_bwd_impl(true, dt, B, T, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, d_o, dS_T, dq, dk, dv, dlog_alpha, db, dw, dS0, workspace, ws_bytes, stream);
}

gdn2_status gdn2_chunk_fwd_save(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q, const void *k,
                                const void *v, const float *log_alpha, const void *b, const void *w, const float *S0,
                                void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream)
{
    gdn2_status st = check_sizes(dt, B, T, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    if (T == 0 || dt != GDN2_BF16)  // nothing to record (fp32: the backward recomputes its states)
        return gdn2_chunk_fwd(dt, B, T, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, o, S_T, nullptr, 0, stream);
    if ((st = check_ptrs({q, k, v, log_alpha, b, w, o}, {S0, S_T})) != GDN2_OK) return st;
    gdn2::Problem p = make_problem(B, T, H, Dk, q, k, v, log_alpha, b, w, S0);
    const size_t need = gdn2::bwd_workspace_bytes(dt, p);
    if (!workspace || ws_bytes < need) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    int *status = gdn2::status_word();
    if (!status) return GDN2_ERR_CUDA;
    return from_cuda(gdn2::launch_fwd_save(p, o, S_T, workspace, status, (cudaStream_t)stream));
}

gdn2_status gdn2_chunk_fwd_varlen(gdn2_dtype dt, int N, int total_T, int H, int Dk, int Dv,
                                  const int *cu_seqlens, const void *q, const void *k, const void *v,
                                  const float *log_alpha, const void *b, const void *w, const float *S0, void *o,
                                  float *S_T, void *workspace, size_t ws_bytes, void *stream)
{
    (void)workspace;
    (void)ws_bytes;
    gdn2_status st = check_sizes(dt, N, total_T, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    if (!cu_seqlens) return GDN2_ERR_NULL;
    if (((uintptr_t)cu_seqlens & 3u) != 0) return GDN2_ERR_ALIGN;
    if (total_T > 0) st = check_ptrs({q, k, v, log_alpha, b, w, o}, {S0, S_T});
    else st = check_ptrs({}, {S0, S_T});
    if (st != GDN2_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t state_bytes = (size_t)N * H * Dk * Dv * sizeof(float);
    if (total_T == 0) {  // every sequence is empty: S_T = S0
        if (!S_T) return GDN2_OK;
        if (S0) return S0 == S_T ? GDN2_OK : from_cuda(cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(S_T, 0, state_bytes, s));
    }
    gdn2::Problem p = make_problem(N, total_T, H, Dk, q, k, v, log_alpha, b, w, S0);
    p.cu_seqlens = cu_seqlens;
    return run_fwd(dt, p, o, S_T, s);
}

gdn2_status gdn2_chunk_bwd_varlen(gdn2_dtype dt, int N, int total_T, int H, int Dk, int Dv,
                                  const int *cu_seqlens, const void *q, const void *k, const void *v,
                                  const float *log_alpha, const void *b, const void *w, const float *S0,
                                  const void *d_o, const float *dS_T, void *dq, void *dk, void *dv,
                                  float *dlog_alpha, void *db, void *dw, float *dS0, void *workspace,
                                  size_t ws_bytes, void *stream)
{
    gdn2_status st = check_sizes(dt, N, total_T, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    if (!cu_seqlens) return GDN2_ERR_NULL;
    if (((uintptr_t)cu_seqlens & 3u) != 0) return GDN2_ERR_ALIGN;
    if (total_T > 0)
        st = check_ptrs({q, k, v, log_alpha, b, w, d_o, dq, dk, dv, dlog_alpha, db, dw, dS0}, {S0, dS_T});
    else
        st = check_ptrs({dS0}, {S0, dS_T});
    if (st != GDN2_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t state_bytes = (size_t)N * H * Dk * Dv * sizeof(float);
    if (total_T == 0) {
        if (dS_T) return from_cuda(cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(dS0, 0, state_bytes, s));
    }
    gdn2::Problem p = make_problem(N, total_T, H, Dk, q, k, v, log_alpha, b, w, S0);
    p.cu_seqlens = cu_seqlens;
    const size_t need = gdn2::bwd_workspace_bytes(dt, p);
    if (!workspace || ws_bytes < need) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    gdn2::BwdOut out{dq, dk, dv, db, dw, dlog_alpha, dS0};
    return from_cuda(gdn2::launch_bwd(dt, p, d_o, dS_T, out, workspace, s));
}

size_t gdn2_workspace_size_gated(int which, int flags, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv)
{
    if (check_gate_flags(flags) != GDN2_OK) return 0;
    if (which == 2) {  // decode: B sequences of one token (the prologue is fused for per-channel b and w)
        if (check_sizes(dt, B, 1, H, Dk, Dv) != GDN2_OK) return 0;
        const bool fused = gate_full(flags, 1) && gate_full(flags, 2);
        return gated_ws(false, flags, dt, (size_t)B, H, Dk, 0, pro_any(flags) && !fused, true, true).total;
    }
    if (check_sizes(dt, B, T, H, Dk, Dv) != GDN2_OK || T == 0 || (which != 0 && which != 1)) return 0;
    const size_t core = which == 1 ? gdn2::bwd_workspace_bytes(dt, make_problem(B, T, H, Dk, nullptr, nullptr, nullptr,
                                                                                nullptr, nullptr, nullptr, nullptr))
                                   : 0;
    const bool pro_pass = pro_any(flags) && (which == 1 || !pro_fused(flags, dt));
    return gated_ws(which == 1, flags, dt, (size_t)B * T, H, Dk, core, pro_pass,
                    which == 0 ? bw_native(flags, dt) : bw_native_bwd(flags, dt), decay_native(flags, dt))
        .total;
}

gdn2_status gdn2_chunk_fwd_gated(int flags, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q,
                                 const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                                 const float *S0, void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream)
{
    gdn2_status st = check_gate_flags(flags);
    if (st != GDN2_OK) return st;
    if ((st = check_sizes(dt, B, T, H, Dk, Dv)) != GDN2_OK) return st;
    if (T == 0) return gdn2_chunk_fwd(dt, B, 0, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, o, S_T, nullptr, 0, stream);
    if ((st = check_ptrs({q, k, v, o}, {S0, S_T})) != GDN2_OK) return st;
    if ((st = check_gate_ptrs(flags, log_alpha, b, w)) != GDN2_OK) return st;
    const bool fused = pro_any(flags) && pro_fused(flags, dt);
    const bool native_bw = bw_native(flags, dt);
    const bool native_decay = decay_native(flags, dt);
    const GatedWs l = gated_ws(false, flags, dt, (size_t)B * T, H, Dk, 0, pro_any(flags) && !fused, native_bw,
                               native_decay);
    if (l.total > 0 && (!workspace || ws_bytes < l.total)) return GDN2_ERR_WORKSPACE;
    if (l.total > 0 && !aligned16(workspace)) return GDN2_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = static_cast<char *>(workspace);
    const void *qq = q, *kk = k, *bq = b, *wq = w;
    if (pro_any(flags) && !fused &&
        (st = prologue_pass(flags, dt, l, ws, (size_t)B * T, H, Dk, qq, kk, bq, wq, s)) != GDN2_OK)
        return st;
    // a scalar decay, and scalar b and w together, go to the tensor-core forward as they are
    // (one exponential per token; one gate value per token)
    int expand_flags = native_decay ? (flags & ~GDN2_DECAY_SCALAR) : flags;
    if (native_bw) expand_flags &= ~(GDN2_ERASE_SCALAR | GDN2_WRITE_SCALAR);
    const void *gp[3] = {log_alpha, bq, wq};
    if ((st = expand_gates(expand_flags, dt, l, ws, (size_t)B * T, H, Dk, gp, s)) != GDN2_OK) return st;
    gdn2::Problem p = make_problem(B, T, H, Dk, qq, kk, v, static_cast<const float *>(gp[0]), gp[1], gp[2], S0);
    if (native_decay || native_bw || fused) {
        p.g_scalar = native_decay;
        p.bw_scalar = native_bw;
        if (fused)
            p.prologue = ((flags & GDN2_QK_L2NORM) ? gdn2::kProNorm : 0) | ((flags & GDN2_BW_LOGITS) ? gdn2::kProSigmoid : 0);
        int *status = gdn2::status_word();
        if (!status) return GDN2_ERR_CUDA;
        return from_cuda(gdn2::launch_fwd_tc(p, o, S_T, nullptr, status, s));
    }
    return run_fwd(dt, p, o, S_T, s);
}

gdn2_status gdn2_chunk_bwd_gated(int flags, gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q,
                                 const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                                 const float *S0, const void *d_o, const float *dS_T, void *dq, void *dk, void *dv,
                                 float *dlog_alpha, void *db, void *dw, float *dS0, void *workspace, size_t ws_bytes,
                                 void *stream)
{
    gdn2_status st = check_gate_flags(flags);
    if (st != GDN2_OK) return st;
    if ((st = check_sizes(dt, B, T, H, Dk, Dv)) != GDN2_OK) return st;
    if (T == 0)
        return gdn2_chunk_bwd(dt, B, 0, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, d_o, dS_T, dq, dk, dv, dlog_alpha, db,
                              dw, dS0, nullptr, 0, stream);
    if ((st = check_ptrs({q, k, v, d_o, dq, dk, dv, dS0}, {S0, dS_T})) != GDN2_OK) return st;
    if ((st = check_gate_ptrs(flags, log_alpha, b, w)) != GDN2_OK) return st;
    if ((st = check_gate_ptrs(flags, dlog_alpha, db, dw)) != GDN2_OK) return st;
    gdn2::Problem p = make_problem(B, T, H, Dk, q, k, v, log_alpha, b, w, S0);
    // scalar b and w together (KDA-shaped), and a scalar decay, run natively: the kernels read them
    // per token and write their gradients per token
    const bool nat = bw_native_bwd(flags, dt), nat_g = decay_native(flags, dt);
    const GatedWs l = gated_ws(true, flags, dt, (size_t)B * T, H, Dk, gdn2::bwd_workspace_bytes(dt, p), pro_any(flags),
                               nat, nat_g);
    if (!workspace || ws_bytes < l.total) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = static_cast<char *>(workspace);
    const void *qq = q, *kk = k, *bq = b, *wq = w;
    if (pro_any(flags) && (st = prologue_pass(flags, dt, l, ws, (size_t)B * T, H, Dk, qq, kk, bq, wq, s)) != GDN2_OK)
        return st;
    p.q = qq;
    p.k = kk;
    const void *gp[3] = {log_alpha, bq, wq};
    if ((st = expand_gates(nat_g ? (flags & ~GDN2_DECAY_SCALAR) : flags, dt, l, ws, (size_t)B * T, H, Dk, gp, s,
                           nat)) != GDN2_OK)
        return st;
    p.g = static_cast<const float *>(gp[0]);
    p.b = gp[1];
    p.w = gp[2];
    p.bw_scalar = nat;
    p.g_scalar = nat_g;
    void *grads[3] = {dlog_alpha, db, dw};
    for (int i = 0; i < 3; ++i)  // full-size gradients, reduced below
        if (!gate_full(flags, i) && !(nat && i > 0) && !(nat_g && i == 0)) grads[i] = ws + l.grad[i];
    gdn2::BwdOut out{dq, dk, dv, grads[1], grads[2], static_cast<float *>(grads[0]), dS0};
    if (gdn2::launch_bwd(dt, p, d_o, dS_T, out, ws + l.core, s) != cudaSuccess) return GDN2_ERR_CUDA;
    void *user[3] = {dlog_alpha, db, dw};
    for (int i = 0; i < 3; ++i) {
        if (!gate_scalar(flags, i) || (nat && i > 0) || (nat_g && i == 0)) continue;
        const bool fp32 = (i == 0) || dt == GDN2_F32;
        if (gdn2::launch_channel_sum(fp32, grads[i], user[i], (size_t)B * T * H, Dk, s) != cudaSuccess)
            return GDN2_ERR_CUDA;
    }
    if (pro_any(flags) &&  // back through the prologue, in place, against the raw inputs
        gdn2::launch_prologue_bwd(dt == GDN2_F32, (size_t)B * T * H, Dk, flags & GDN2_QK_L2NORM, q, k, dq, dk,
                                  pro_gate_mode(flags, 1), b, db, pro_gate_mode(flags, 2), w, dw, s) != cudaSuccess)
        return GDN2_ERR_CUDA;
    return GDN2_OK;
}

gdn2_status gdn2_decode_step_gated(int flags, gdn2_dtype dt, int N, int H, int Dk, int Dv, const void *q,
                                   const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                                   float *S, void *o, void *workspace, size_t ws_bytes, void *stream)
{
    gdn2_status st = check_gate_flags(flags);
    if (st != GDN2_OK) return st;
    if ((st = check_sizes(dt, N, 1, H, Dk, Dv)) != GDN2_OK) return st;
    if ((st = check_ptrs({q, k, v, S, o}, {})) != GDN2_OK) return st;
    if ((st = check_gate_ptrs(flags, log_alpha, b, w)) != GDN2_OK) return st;
    // the prologue runs inside the decode kernel when b and w are per channel; the kernel reads
    // every gate layout as it is (nothing is broadcast)
    const bool fused = pro_any(flags) && gate_full(flags, 1) && gate_full(flags, 2);
    const GatedWs l = gated_ws(false, flags, dt, (size_t)N, H, Dk, 0, pro_any(flags) && !fused, true, true);
    if (l.total > 0 && (!workspace || ws_bytes < l.total)) return GDN2_ERR_WORKSPACE;
    if (l.total > 0 && !aligned16(workspace)) return GDN2_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = static_cast<char *>(workspace);
    const void *qq = q, *kk = k, *bq = b, *wq = w;
    if (pro_any(flags) && !fused &&
        (st = prologue_pass(flags, dt, l, ws, (size_t)N, H, Dk, qq, kk, bq, wq, s)) != GDN2_OK)
        return st;
    int modes = 0;
    for (int i = 0; i < 3; ++i)
        modes |= (gate_scalar(flags, i) ? gdn2::kGateScalar : gate_none(flags, i) ? gdn2::kGateAbsent : gdn2::kGateChannel)
                 << (2 * i);
    const int pro = fused ? ((flags & GDN2_QK_L2NORM) ? gdn2::kProNorm : 0) | ((flags & GDN2_BW_LOGITS) ? gdn2::kProSigmoid : 0)
                          : 0;
    return from_cuda(gdn2::launch_decode(dt, N, H, Dk, qq, kk, v, log_alpha, bq, wq, S, o, s, pro, modes));
}

gdn2_status gdn2_prologue(int flags, gdn2_dtype dt, int N, int H, int D, const void *q, const void *k, const void *b,
                          const void *w, void *q_n, void *k_n, void *b_s, void *w_s, void *stream)
{
    gdn2_status st = check_gate_flags(flags);
    if (st != GDN2_OK) return st;
    if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (N < 0 || H < 1) return GDN2_ERR_SHAPE;
    if (D != 64 && D != 128) return GDN2_ERR_UNSUPPORTED;
    const bool norm = flags & GDN2_QK_L2NORM;
    const int bm = pro_gate_mode(flags, 1), wm = pro_gate_mode(flags, 2);
    std::vector<const void *> need;
    if (norm) need.insert(need.end(), {q, k, q_n, k_n});
    if (bm) need.insert(need.end(), {b, b_s});
    if (wm) need.insert(need.end(), {w, w_s});
    for (const void *ptr : need) {
        if (!ptr) return GDN2_ERR_NULL;
        if (!aligned16(ptr)) return GDN2_ERR_ALIGN;
    }
    if (N == 0) return GDN2_OK;
    return from_cuda(gdn2::launch_prologue_fwd(dt == GDN2_F32, (size_t)N * H, D, norm, q, k, q_n, k_n, bm, b, b_s, wm,
                                               w, w_s, (cudaStream_t)stream));
}

gdn2_status gdn2_chunk_fwd_host(gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q, const void *k,
                                const void *v, const float *log_alpha, const void *b, const void *w, const float *S0,
                                void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream)
{
    gdn2_status st = check_sizes(dt, B, T, H, Dk, Dv);
    if (st != GDN2_OK) return st;
    if (T == 0) {  // S_T = S0 (or zeros), host to host
        if (!S_T) return GDN2_OK;
        const size_t n = (size_t)B * H * Dk * Dv * sizeof(float);
        cudaStream_t s = (cudaStream_t)stream;
        if (S0) return S0 == S_T ? GDN2_OK : from_cuda(cudaMemcpyAsync(S_T, S0, n, cudaMemcpyHostToHost, s));
        memset(S_T, 0, n);
        return GDN2_OK;
    }
    for (const void *ptr : {q, k, v, static_cast<const void *>(log_alpha), b, w, static_cast<const void *>(o)})
        if (!ptr) return GDN2_ERR_NULL;
    const size_t need = gdn2::host_fwd_workspace_bytes(dt == GDN2_F32 ? 4 : 2, B, T, H, Dk);
    if (!workspace || ws_bytes < need) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    return from_cuda(gdn2::launch_fwd_host(dt, B, T, H, Dk, q, k, v, log_alpha, b, w, S0, o, S_T, workspace,
                                           (cudaStream_t)stream, run_fwd_slice));
}

gdn2_status gdn2_selftest_timeout(int limit_us, void *stream)
{
    if (limit_us < 1 || limit_us > 100000) return GDN2_ERR_SHAPE;
    int *status = gdn2::status_word();
    if (!status) return GDN2_ERR_CUDA;
    return from_cuda(gdn2::launch_selftest_timeout(limit_us, status, (cudaStream_t)stream));
}

gdn2_status gdn2_sync_status(void *stream)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gdn2_status, sizeof(int)) != cudaSuccess) return GDN2_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_gdn2_status, &zero, sizeof(int)) != cudaSuccess) return GDN2_ERR_CUDA;
        return v == gdn2::kStatusBadSeqlens ? GDN2_ERR_SEQLENS : GDN2_ERR_TIMEOUT;
    }
    return GDN2_OK;
}

}  // extern "C"
