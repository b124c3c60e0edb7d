// Gate-aware chunkwise backward of the GDN-2 recurrence (fp32 FMA arithmetic).
//
// Three launches:
//   1. the forward kernel re-run in "states" mode: the fp32 state at the start
//      of every chunk goes to the workspace;
//   2. bwd_chunk_kernel: one CTA per (batch, head, 32-column slice of d_v)
//      walks the chunks in reverse carrying its slice of dS, the gradient of the
//      loss with respect to the state at the end of the chunk;
//   3. a reduction that sums the per-slice partial gradients of the key-side
//      inputs (q, k, b, log alpha) and casts them to the output type.
//
// Chunk quantities are those of the forward (G, Q~, E~, K~, K^, gamma, A,
// W = (I+A)^-1 E~, U = (I+A)^-1 (w.V), U~ = U - W S, P = lower_incl(Q~ K~^T)).
// Reverse mode, per chunk, given dO and dS_next (all derived by hand from the
// forward; the gates stay inside the products E~ = (b.k) e^G and X = w.v, as
// the aixai.ru post's implementation section requires):
//   dP   = lower_incl(dO U~^T)          dU~ = P^T dO + K^ dS_next
//   dQ~  = dO S^T + dP K~               dK~ = dP^T Q~          dK^ = U~ dS_next^T
//   dgam = rowsum(dS_next . S)          dW  = -dU~ S^T
//   dE~W = (I+A)^-T dW                  dX  = (I+A)^-T dU~
//   dA   = -strictly_lower(dE~W W^T + dX U^T)
//   dE~  = dE~W + dA K~                 dK~ += dA^T E~
//   dS   = Q~^T dO + Diag(gamma) dS_next - W^T dU~      (carried to the previous chunk)
// then through the factors: dq = dQ~ e^G; d(b.k) = dE~ e^G; db = d(b.k) k;
// dk = d(b.k) b + dK~ e^-G + dK^ e^(G_L-G); dw = dX v; dv = dX w;
// dG = dQ~ Q~ + dE~ E~ - dK~ K~ - dK^ K^, plus sum_t dK^ K^ + dgam gamma on
// the last row; dlog alpha = reverse cumulative sum of dG inside the chunk.
// Everything that sums over d_v is linear in this CTA's slice, so each slice
// writes a partial and launch 3 adds them (no atomics, deterministic).
#include <algorithm>

#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kThreads = 256;
constexpr int kDVT = 32;

template <int D>
struct BwdSmem {
    static constexpr int LA = kChunk + 1;
    static constexpr size_t floats = 3 * (size_t)kChunk * LA + 2 * (size_t)D * kDVT +
                                     6 * (size_t)kChunk * kDVT + 2 * D;
    static constexpr size_t bytes = floats * sizeof(float);
};

// per-CTA global scratch: ten C x D fp32 matrices
constexpr int kScratchMats = 10;

struct BwdArgs {
    Problem p;
    const void *d_o;
    const float *dS_T;
    const float *states;   // [BH][NC][D][D]
    float *scratch;        // [BH * NT][kScratchMats][C][D]
    float *part;           // [4][NT][B*T*H*D]  partial dq, dk, db, dg
    void *dv, *dw;
    float *dS0;
};

template <int D, typename Tin>
__global__ void __launch_bounds__(kThreads) bwd_chunk_kernel(BwdArgs a)
{
    using SM = BwdSmem<D>;
    constexpr int C = kChunk, LA = SM::LA;
    constexpr int NT = D / kDVT;
    extern __shared__ float sm[];
    float *Am = sm;                 // [C][LA]  A, then dA
    float *Pm = Am + C * LA;        // [C][LA]
    float *dPm = Pm + C * LA;       // [C][LA]
    float *Sc = dPm + C * LA;       // [D][kDVT]
    float *dSn = Sc + D * kDVT;     // [D][kDVT]
    float *dO = dSn + D * kDVT;     // [C][kDVT]
    float *Xs = dO + C * kDVT;      // [C][kDVT]
    float *Us = Xs + C * kDVT;      // [C][kDVT]
    float *Ub = Us + C * kDVT;      // [C][kDVT]
    float *dUb = Ub + C * kDVT;     // [C][kDVT]
    float *dX = dUb + C * kDVT;     // [C][kDVT]
    float *gam = dX + C * kDVT;     // [D]
    float *dgam = gam + D;          // [D]

    const Problem &p = a.p;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, bb = bh / p.H, hh = bh % p.H;
    const int tile = blockIdx.y, j0 = tile * kDVT;
    const SeqSpan sp = seq_span(p, bb);
    if (sp.len < 0) return;  // invalid cu_seqlens (reported by the offsets pass)
    const int T = sp.len;
    const size_t tok = (size_t)p.H * D;
    const size_t base = tok_row(p, sp, hh, 0);
    const size_t total = token_rows(p) * p.H * D;
    const int nchunks = (T + C - 1) / C;
    const Tin *q = (const Tin *)p.q, *k = (const Tin *)p.k, *v = (const Tin *)p.v;
    const Tin *bg = (const Tin *)p.b, *wg = (const Tin *)p.w, *dog = (const Tin *)a.d_o;

    float *scr = a.scratch + ((size_t)bh * NT + tile) * kScratchMats * C * D;
    float *Gm = scr, *Qt = scr + 1 * C * D, *Et = scr + 2 * C * D, *Kt = scr + 3 * C * D;
    float *Kh = scr + 4 * C * D, *Wm = scr + 5 * C * D, *dQt = scr + 6 * C * D;
    float *dKt = scr + 7 * C * D, *dKh = scr + 8 * C * D, *dEw = scr + 9 * C * D;
    float *pdq = a.part + (0 * NT + tile) * total, *pdk = a.part + (1 * NT + tile) * total;
    float *pdb = a.part + (2 * NT + tile) * total, *pdg = a.part + (3 * NT + tile) * total;

    for (int idx = tid; idx < D * kDVT; idx += kThreads) {
        const int c = idx / kDVT, j = idx % kDVT;
        dSn[idx] = a.dS_T ? a.dS_T[((size_t)bh * D + c) * D + j0 + j] : 0.f;
    }

    for (int ci = nchunks - 1; ci >= 0; --ci) {
        const int c0 = ci * C;
        const int L = min(C, T - c0);
        __syncthreads();
        // ---- 1. factors (thread per key channel), value-side tiles, chunk-start state
        if (tid < D) {
            const int c = tid;
            float G = 0.f;
            for (int t = 0; t < C; ++t) {
                float qv = 0.f, kv = 0.f, bv = 0.f;
                if (t < L) {
                    const size_t off = base + (size_t)(c0 + t) * tok + c;
                    G += p.g[off];
                    qv = to_f(q[off]); kv = to_f(k[off]); bv = to_f(bg[off]);
                }
                const float eG = expf(G);
                Gm[t * D + c] = G;
                Qt[t * D + c] = qv * eG;
                Et[t * D + c] = bv * kv * eG;
                Kt[t * D + c] = kv * expf(-G);
            }
            gam[c] = expf(G);
            for (int t = 0; t < C; ++t) {
                float kv = 0.f;
                if (t < L) kv = to_f(k[base + (size_t)(c0 + t) * tok + c]);
                Kh[t * D + c] = kv * expf(G - Gm[t * D + c]);
            }
        } else {
            for (int idx = tid - D; idx < C * kDVT; idx += kThreads - D) {
                const int t = idx / kDVT, j = idx % kDVT;
                float x = 0.f, d = 0.f;
                if (t < L) {
                    const size_t off = base + (size_t)(c0 + t) * tok + j0 + j;
                    x = to_f(wg[off]) * to_f(v[off]);
                    d = to_f(dog[off]);
                }
                Xs[idx] = x;
                dO[idx] = d;
            }
        }
        {
            const float *src = a.states + chunk_slot(p, bb, hh, nchunks, ci) * D * D;
            for (int idx = tid; idx < D * kDVT; idx += kThreads) {
                const int c = idx / kDVT, j = idx % kDVT;
                Sc[idx] = src[(size_t)c * D + j0 + j];
            }
        }
        __syncthreads();
        // ---- 2. A = strictly_lower(E~ K~^T), P = lower_incl(Q~ K~^T)
        {
            const int i = tid >> 2, jb = tid & 3;
            float aa[16], pa[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) { aa[jj] = 0.f; pa[jj] = 0.f; }
            for (int c = 0; c < D; ++c) {
                const float e = Et[i * D + c], qv = Qt[i * D + c];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const float kt = Kt[(jb + 4 * jj) * D + c];
                    aa[jj] += e * kt;
                    pa[jj] += qv * kt;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = jb + 4 * jj;
                Am[i * LA + j] = (j < i) ? aa[jj] : 0.f;
                Pm[i * LA + j] = (j <= i) ? pa[jj] : 0.f;
            }
        }
        __syncthreads();
        // ---- 3. W = (I+A)^-1 E~ (global), U = (I+A)^-1 X (smem): forward substitution
        if (tid < D) {
            const int c = tid;
            for (int i = 0; i < C; ++i) {
                float s = Et[i * D + c];
                for (int m = 0; m < i; ++m) s -= Am[i * LA + m] * Wm[m * D + c];
                Wm[i * D + c] = s;
            }
        } else if (tid < D + kDVT) {
            const int j = tid - D;
            for (int i = 0; i < C; ++i) {
                float s = Xs[i * kDVT + j];
                for (int m = 0; m < i; ++m) s -= Am[i * LA + m] * Us[m * kDVT + j];
                Us[i * kDVT + j] = s;
            }
        }
        __syncthreads();
        // ---- 4. U~ = U - W S
        {
            const int j = tid & 31, ib = tid >> 5;
            for (int ii = 0; ii < C / 8; ++ii) {
                const int i = ib + 8 * ii;
                float acc = Us[i * kDVT + j];
                for (int c = 0; c < D; ++c) acc -= Wm[i * D + c] * Sc[c * kDVT + j];
                Ub[i * kDVT + j] = acc;
            }
        }
        __syncthreads();
        // ---- 5. dP = lower_incl(dO U~^T); dU~ = P^T dO + K^ dS_next
        {
            const int i = tid >> 2, jb = tid & 3;  // dP row t = i, columns m = jb + 4 jj
            float acc[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.f;
            for (int j = 0; j < kDVT; ++j) {
                const float d = dO[i * kDVT + j];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) acc[jj] += d * Ub[(jb + 4 * jj) * kDVT + j];
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int m = jb + 4 * jj;
                dPm[i * LA + m] = (m <= i) ? acc[jj] : 0.f;
            }
        }
        {
            const int j = tid & 31, ib = tid >> 5;
            for (int ii = 0; ii < C / 8; ++ii) {
                const int i = ib + 8 * ii;
                float acc = 0.f;
                for (int t = i; t < C; ++t) acc += Pm[t * LA + i] * dO[t * kDVT + j];
                for (int c = 0; c < D; ++c) acc += Kh[i * D + c] * dSn[c * kDVT + j];
                dUb[i * kDVT + j] = acc;
            }
        }
        __syncthreads();
        // ---- 6. per key channel c: dQ~, dK~ (from P), dK^, dgam, dW
        if (tid < D) {
            const int c = tid;
            float dg = 0.f;
            for (int j = 0; j < kDVT; ++j) dg += dSn[c * kDVT + j] * Sc[c * kDVT + j];
            dgam[c] = dg;
        }
        for (int idx = tid; idx < C * D; idx += kThreads) {
            const int t = idx / D, c = idx % D;
            float aq = 0.f, akt = 0.f, akh = 0.f, aw = 0.f;
            for (int j = 0; j < kDVT; ++j) {
                const float s = Sc[c * kDVT + j], ds = dSn[c * kDVT + j];
                aq += dO[t * kDVT + j] * s;
                akh += Ub[t * kDVT + j] * ds;
                aw -= dUb[t * kDVT + j] * s;
            }
            for (int i = 0; i <= t; ++i) aq += dPm[t * LA + i] * Kt[i * D + c];
            for (int s2 = t; s2 < C; ++s2) akt += dPm[s2 * LA + t] * Qt[s2 * D + c];
            dQt[idx] = aq;
            dKt[idx] = akt;
            dKh[idx] = akh;
            dEw[idx] = aw;
        }
        __syncthreads();
        // ---- 7. back substitution with (I+A)^T: dE~W (in place), dX
        if (tid < D) {
            const int c = tid;
            for (int i = C - 1; i >= 0; --i) {
                float s = dEw[i * D + c];
                for (int m = i + 1; m < C; ++m) s -= Am[m * LA + i] * dEw[m * D + c];
                dEw[i * D + c] = s;
            }
        } else if (tid < D + kDVT) {
            const int j = tid - D;
            for (int i = C - 1; i >= 0; --i) {
                float s = dUb[i * kDVT + j];
                for (int m = i + 1; m < C; ++m) s -= Am[m * LA + i] * dX[m * kDVT + j];
                dX[i * kDVT + j] = s;
            }
        }
        __syncthreads();
        // ---- 8. dA = -strictly_lower(dE~W W^T + dX U^T) into Am; dS for the previous chunk
        {
            const int i = tid >> 2, jb = tid & 3;
            float acc[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.f;
            for (int c = 0; c < D; ++c) {
                const float d = dEw[i * D + c];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) acc[jj] += d * Wm[(jb + 4 * jj) * D + c];
            }
            for (int j = 0; j < kDVT; ++j) {
                const float d = dX[i * kDVT + j];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) acc[jj] += d * Us[(jb + 4 * jj) * kDVT + j];
            }
            __syncthreads();  // every thread is done reading A (phase 7 ended above)
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int m = jb + 4 * jj;
                Am[i * LA + m] = (m < i) ? -acc[jj] : 0.f;
            }
        }
        {
            const int j = tid & 31, cb = tid >> 5;
            for (int cc = 0; cc < D / 8; ++cc) {
                const int c = cb + 8 * cc;
                float acc = gam[c] * dSn[c * kDVT + j];
                for (int t = 0; t < C; ++t)
                    acc += Qt[t * D + c] * dO[t * kDVT + j] - Wm[t * D + c] * dUb[t * kDVT + j];
                dSn[c * kDVT + j] = acc;  // each (c, j) read and written by this thread only
            }
        }
        __syncthreads();
        // ---- 9. dE~ = dE~W + dA K~, dK~ += dA^T E~, and the chain to the inputs
        if (tid < D) {
            const int c = tid;
            const float GL = Gm[(C - 1) * D + c];
            float extra = dgam[c] * gam[c];
            for (int t = 0; t < C; ++t) {
                float dE = dEw[t * D + c];
                for (int m = 0; m < t; ++m) dE += Am[t * LA + m] * Kt[m * D + c];
                float dK = dKt[t * D + c];
                for (int s2 = t + 1; s2 < C; ++s2) dK += Am[s2 * LA + t] * Et[s2 * D + c];
                const float G = Gm[t * D + c];
                const float dq_ = dQt[t * D + c], dkh = dKh[t * D + c];
                const float qt = Qt[t * D + c], et = Et[t * D + c], kt = Kt[t * D + c], kh = Kh[t * D + c];
                extra += dkh * kh;
                dEw[t * D + c] = dq_ * qt + dE * et - dK * kt - dkh * kh;  // dG_t
                if (t < L) {
                    const size_t off = base + (size_t)(c0 + t) * tok + c;
                    const float kv = to_f(k[off]), bv = to_f(bg[off]);
                    const float eG = expf(G);
                    const float de = dE * eG;
                    pdq[off] = dq_ * eG;
                    pdb[off] = de * kv;
                    pdk[off] = de * bv + dK * expf(-G) + dkh * expf(GL - G);
                }
            }
            // the last real row carries the gamma and K^ terms (padding rows have G = G_L
            // and zero factors, so they add nothing)
            dEw[(L - 1) * D + c] += extra;
            float run = 0.f;
            for (int t = L - 1; t >= 0; --t) {
                run += dEw[t * D + c];
                pdg[base + (size_t)(c0 + t) * tok + c] = run;
            }
        } else {
            for (int idx = tid - D; idx < C * kDVT; idx += kThreads - D) {
                const int t = idx / kDVT, j = idx % kDVT;
                if (t < L) {
                    const size_t off = base + (size_t)(c0 + t) * tok + j0 + j;
                    const float d = dX[idx];
                    ((Tin *)a.dw)[off] = from_f<Tin>(d * to_f(v[off]));
                    ((Tin *)a.dv)[off] = from_f<Tin>(d * to_f(wg[off]));
                }
            }
        }
    }
    __syncthreads();
    for (int idx = tid; idx < D * kDVT; idx += kThreads) {
        const int c = idx / kDVT, j = idx % kDVT;
        a.dS0[((size_t)bh * D + c) * D + j0 + j] = dSn[idx];
    }
}

template <typename Tout>
__global__ void reduce_parts_kernel(const float *__restrict__ part, int nt, size_t total,
                                    Tout *dq, Tout *dk, Tout *db, float *dg)
{
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        float s[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float acc = 0.f;
            for (int t = 0; t < nt; ++t) acc += part[((size_t)m * nt + t) * total + i];
            s[m] = acc;
        }
        dq[i] = from_f<Tout>(s[0]);
        dk[i] = from_f<Tout>(s[1]);
        db[i] = from_f<Tout>(s[2]);
        dg[i] = s[3];
    }
}

struct WsLayout {
    size_t coff, states, scratch, part, total;
};

// [chunk_off (variable length only)] [chunk-start states] [per-CTA scratch] [partials]
WsLayout ws_layout(const Problem &p, int D)
{
    const size_t nt = D / kDVT;
    WsLayout l;
    l.coff = p.cu_seqlens ? varlen_offsets_bytes(p.B) : 0;
    l.states = (size_t)p.H * chunk_bound(p) * D * D * sizeof(float);
    l.scratch = (size_t)p.B * p.H * nt * kScratchMats * kChunk * D * sizeof(float);
    l.part = 4 * nt * token_rows(p) * p.H * D * sizeof(float);
    l.total = l.coff + l.states + l.scratch + l.part;
    return l;
}

template <int D, typename Tin>
cudaError_t launch_t(const Problem &p0, const void *d_o, const float *dS_T, const BwdOut &out,
                     void *ws, int *status, cudaStream_t s)
{
    const WsLayout l = ws_layout(p0, D);
    char *base = (char *)ws;
    Problem p = p0;
    cudaError_t e;
    if (p.cu_seqlens) {
        int *coff = reinterpret_cast<int *>(base);
        if ((e = launch_chunk_offsets(p.cu_seqlens, p.B, p.T, coff, status, s)) != cudaSuccess) return e;
        p.chunk_off = coff;
    }
    base += l.coff;
    float *states = (float *)base;
    float *scratch = (float *)(base + l.states);
    float *part = (float *)(base + l.states + l.scratch);
    e = launch_fwd_simt(sizeof(Tin) == 4 ? GDN2_F32 : GDN2_BF16, p, nullptr, nullptr, states, s);
    if (e != cudaSuccess) return e;
    const size_t smem = BwdSmem<D>::bytes;
    e = cudaFuncSetAttribute(bwd_chunk_kernel<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    BwdArgs a{p, d_o, dS_T, states, scratch, part, out.dv, out.dw, out.dS0};
    bwd_chunk_kernel<D, Tin><<<dim3(p.B * p.H, D / kDVT), kThreads, smem, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t total = token_rows(p) * p.H * D;
    const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
    reduce_parts_kernel<Tin><<<blocks, 256, 0, s>>>(part, D / kDVT, total, (Tin *)out.dq,
                                                    (Tin *)out.dk, (Tin *)out.db, out.dg);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(gdn2_dtype dt, const Problem &p)
{
    if (dt == GDN2_BF16) return bwd_tc_workspace_bytes(p);  // d = 128, and d = 64 zero-padded
    return ws_layout(p, p.D).total;
}

cudaError_t launch_bwd(gdn2_dtype dt, const Problem &p, const void *d_o, const float *dS_T,
                       const BwdOut &out, void *ws, cudaStream_t s, bool states_saved)
{
    int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    if (dt == GDN2_BF16) return launch_bwd_tc(p, d_o, dS_T, out, ws, status, s, states_saved);
    if (dt == GDN2_F32)
        return p.D == 64 ? launch_t<64, float>(p, d_o, dS_T, out, ws, status, s)
                         : launch_t<128, float>(p, d_o, dS_T, out, ws, status, s);
    return p.D == 64 ? launch_t<64, __nv_bfloat16>(p, d_o, dS_T, out, ws, status, s)
                     : launch_t<128, __nv_bfloat16>(p, d_o, dS_T, out, ws, status, s);
}

}  // namespace gdn2
