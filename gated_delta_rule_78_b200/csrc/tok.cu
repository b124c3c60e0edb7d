// Token-level kernels of the GDN-2 recurrence (fp32 arithmetic, any input dtype, d = 64 or 128).
//
// They serve two purposes:
//   * the fp32 path: the forward, and the backward as three launches (the forward in states
//     mode, the reverse dS chain, the per-chunk gradients);
//   * the exact path for chunks of the bf16 tensor-core backward whose decay is too strong for
//     the chunkwise form (kChunkDecayLimit): their gradients are rewritten here.
// The recurrence is the token form of the update (tok_util.cuh): no chunk factor e^{-G} is ever
// formed, so the results are exact for any decay.
//
// Gradients of one chunk (tok_grad_kernel), given its start state S and the gradient dS of the
// state at its end, by the reverse mode of the token update:
//   forward, t = 0 .. L-1:   S'_t = Diag(alpha_t) S,  u_t = w_t.v_t - S'_t^T e_t,  S = S'_t + k_t u_t^T
//                            (S'_t and u_t kept: S'_t in a per-block scratch, u_t in shared memory)
//   reverse, t = L-1 .. 0:   S_t = S'_t + k_t u_t^T;  dS += q_t do_t^T;  dq_t = S_t do_t;
//                            dk_t = dS u_t;  du = dS^T k_t;  dv_t = du.w_t;  dw_t = du.v_t;
//                            dS' = dS - e_t du^T;  de = -S'_t du;  db_t = de.k_t;  dk_t += de.b_t;
//                            dlog alpha_t = rowsum(dS' . S'_t);  dS = Diag(alpha_t) dS'
// with e_t = b_t.k_t: the gates stay inside the erase-weighted read and the gated write, as the
// aixai.ru post's section "Как это реализуется на практике" requires of the gate-aware backward.
#include <algorithm>

#include "gdn2_internal.cuh"
#include "tok_util.cuh"

namespace gdn2 {
namespace {

constexpr int C = kChunk;

// ================================================================== forward
// One block of 2 D threads per (sequence, head), the state in the column layout of tok_util.cuh.
template <int D, typename Tin>
__global__ void __launch_bounds__(2 * D) tok_fwd_kernel(const Problem p, Tin *o, float *S_T, float *states)
{
    __shared__ __align__(16) tok::Rec<D> recs[3];
    __shared__ __align__(16) float xch[12 * D];
    const int tid = threadIdx.x, j = tid % D, hf = tid / D;
    const int bh = blockIdx.x, n = bh / p.H, h = bh % p.H;
    const SeqSpan sp = seq_span(p, n);
    if (sp.len < 0) return;  // invalid cu_seqlens (reported by the offsets pass)
    const int nch = seq_chunks(sp.len);
    const Tin *q = (const Tin *)p.q, *k = (const Tin *)p.k, *v = (const Tin *)p.v;
    const Tin *bg = (const Tin *)p.b, *wg = (const Tin *)p.w;
    constexpr int NR = D / 2;
    const int c0 = hf * NR;
    float S[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) S[i] = p.S0 ? p.S0[((size_t)bh * D + c0 + i) * D + j] : 0.f;
    auto fill = [&](int t, tok::Rec<D> &r) {
        if (tid < D) {
            const size_t off = tok_row(p, sp, h, t) + tid;
            const float kv = to_f(k[off]);
            r.q[tid] = to_f(q[off]);
            r.k[tid] = kv;
            r.e[tid] = to_f(bg[off]) * kv;
            r.a[tid] = expf(p.g[off]);
        } else {
            const size_t off = tok_row(p, sp, h, t) + j;
            r.x[j] = to_f(wg[off]) * to_f(v[off]);
        }
    };
    auto put_state = [&](int ci) {
        float *dst = states + bound_slot(p, n, h, nch, ci) * D * D;
#pragma unroll
        for (int i = 0; i < NR; ++i) dst[(size_t)(c0 + i) * D + j] = S[i];
    };
    for (int ci = 0; ci < nch; ++ci) {
        if (states) put_state(ci);
        const int t0 = ci * C, L = min(C, sp.len - t0);
        tok::fwd_tokens<D>(S, t0, L, recs, xch, j, hf, 1, fill, [&](int s, float ov) {
            if (o && hf == 0) o[tok_row(p, sp, h, t0 + s) + j] = from_f<Tin>(ov);
        });
    }
    if (states) put_state(nch);
    if (S_T) {
#pragma unroll
        for (int i = 0; i < NR; ++i) S_T[((size_t)bh * D + c0 + i) * D + j] = S[i];
    }
}

// ================================================================== the reverse dS chain
// One block of 2 D threads per (sequence, head): carries dS from dS_T to dS0 through every token
// (the state-independent reverse recurrence of tok_util.cuh) and records it at every chunk end
// (dSe, fp32 [c][j] per chunk slot).
template <int D, typename Tin>
__global__ void __launch_bounds__(2 * D)
tok_chain_kernel(const Problem p, const Tin *dO, const float *dS_T, float *dSe, float *dS0)
{
    __shared__ __align__(16) tok::Rec<D> recs[3];
    __shared__ __align__(16) float xch[4 * D];
    const int tid = threadIdx.x, j = tid % D, hf = tid / D;
    const int bh = blockIdx.x, n = bh / p.H, h = bh % p.H;
    const SeqSpan sp = seq_span(p, n);
    if (sp.len < 0) return;
    const int nch = seq_chunks(sp.len);
    const Tin *q = (const Tin *)p.q, *k = (const Tin *)p.k, *bg = (const Tin *)p.b;
    constexpr int NR = D / 2;
    const int c0 = hf * NR;
    float dS[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) dS[i] = dS_T ? dS_T[((size_t)bh * D + c0 + i) * D + j] : 0.f;
    auto fill = [&](int t, tok::Rec<D> &r) {
        if (tid < D) {
            const size_t off = tok_row(p, sp, h, t) + tid;
            const float kv = to_f(k[off]);
            r.q[tid] = to_f(q[off]);
            r.k[tid] = kv;
            r.e[tid] = to_f(bg[off]) * kv;
            r.a[tid] = expf(p.g[off]);
        } else {
            r.x[j] = to_f(dO[tok_row(p, sp, h, t) + j]);
        }
    };
    for (int ci = nch - 1; ci >= 0; --ci) {
        float *dst = dSe + chunk_slot(p, n, h, nch, ci) * D * D;
#pragma unroll
        for (int i = 0; i < NR; ++i) dst[(size_t)(c0 + i) * D + j] = dS[i];
        const int t0 = ci * C, L = min(C, sp.len - t0);
        tok::chain_tokens<D>(dS, t0 + L - 1, L, recs, xch, j, hf, 1, fill);
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) dS0[((size_t)bh * D + c0 + i) * D + j] = dS[i];
}

// ================================================================== per-chunk gradients
struct TokGradArgs {
    Problem p;            // sizes, inputs, cu_seqlens, chunk_off
    const void *dO;
    // chunk-start states (boundary slots) and chunk-end state gradients (chunk slots): fp32
    // [slot][D][D] in the [c][j] layout, or (kTcWs) the tensor-core workspace's bf16
    // [slot][128][128] in the transposed [j][c] layout
    const void *states, *dSe;
    const int *list;      // null: every chunk task 0 .. ntask-1; else list[0] tasks in list[1 ..]
    int ntask;
    float *scratch;       // per block: C x D x D fp32 (the decayed states S'_t of one chunk)
    void *dq, *dk, *dv, *db, *dw;
    float *dg;
};

// Sum of v[0 .. N) over the 32 lanes of a warp by halving exchanges: on return v[0] of lane l
// holds the total of value l / (32 / N).
template <int N>
__device__ __forceinline__ void lane_reduce(float (&v)[N], int lane)
{
    int m = 16;
#pragma unroll
    for (int n = N / 2; n >= 1; n >>= 1, m >>= 1) {
        const bool up = lane & m;
#pragma unroll
        for (int jj = 0; jj < n; ++jj) {
            const float send = up ? v[jj] : v[jj + n];
            const float keep = up ? v[jj + n] : v[jj];
            v[jj] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
#pragma unroll
    for (; m >= 1; m >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
}

template <int D>
struct TokGradSmem {
    static constexpr int NW = D / 32;  // warps per column quarter (32 rows each)
    static constexpr size_t floats = 4 * (size_t)C * D + (size_t)NW * D + D + 16 * (size_t)D + 3 * NW;
    static constexpr size_t bytes = floats * sizeof(float);
};

// 4 D threads per block, persistent over the chunk tasks.  Thread (c = tid % D, jq = tid / D)
// holds row c of S and dS at the columns j = jq D/4 .. jq D/4 + D/4 - 1 ("row layout"): the sums
// over d_v (dq, dk, de, dlog alpha) are four partials per row; the sums over d_k (u, du) reduce
// over the lanes of a warp and then across its NW warps in shared memory.
template <int D, typename Tin, bool kTcWs>
__global__ void __launch_bounds__(4 * D, 1) tok_grad_kernel(const TokGradArgs a)
{
    using SM = TokGradSmem<D>;
    constexpr int NT = 4 * D, NJ = D / 4, NW = SM::NW, WS = 128;  // WS: tensor-core workspace stride
    extern __shared__ __align__(16) float smf[];
    float *sDo = smf;                // [C][D]
    float *sV = sDo + C * D;         // [C][D]
    float *sW = sV + C * D;          // [C][D]
    float *sU = sW + C * D;          // [C][D]  u_t
    float *sRed = sU + C * D;        // [NW][D] partial sums over d_k
    float *sVec = sRed + NW * D;     // [D]     du of the current token
    float *sRow = sVec + D;          // [4 quantities][4 quarters][D]
    float *sScal = sRow + 16 * D;    // [dw | db | dlog alpha][NW] per-warp sums (scalar gates)
    const Problem &p = a.p;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = tid % D, jq = tid / D, j0 = jq * NJ, cw = warp % NW;
    const Tin *q = (const Tin *)p.q, *k = (const Tin *)p.k, *v = (const Tin *)p.v;
    const Tin *bg = (const Tin *)p.b, *wg = (const Tin *)p.w, *dOg = (const Tin *)a.dO;
    Tin *dq = (Tin *)a.dq, *dk = (Tin *)a.dk, *dv = (Tin *)a.dv, *db = (Tin *)a.db, *dw = (Tin *)a.dw;
    // scalar erase and write gates ([rows, H]): b_t, w_t read per token, db_t, dw_t summed over
    // the channels (the first D threads: a warp shuffle, then the NW warps in shared memory); a
    // scalar decay likewise (g_t per token, dlog alpha_t summed over the channels)
    const bool sg = p.bw_scalar, gs = p.g_scalar;
    auto warp_total = [&](float x) {
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
        return x;
    };
    float *Sp = a.scratch + (size_t)blockIdx.x * C * D * D;
    const int nchb = (int)chunk_bound(p);
    const int ntask = a.list ? a.list[0] : a.ntask;

    // sum over d_k of this thread's NJ values (column j0 + jj): totals land in sRed, then the
    // threads tid < D (column j = tid) add the NW partials; the caller syncs and reads
    auto colsum = [&](float (&vv)[NJ]) {
        lane_reduce<NJ>(vv, lane);
        constexpr int per = 32 / NJ;
        if (lane % per == 0) sRed[cw * D + j0 + lane / per] = vv[0];
        __syncthreads();
    };
    auto colsum_total = [&](int jj) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) s += sRed[w * D + jj];
        return s;
    };

    for (int it = blockIdx.x; it < ntask; it += gridDim.x) {
        const int task = a.list ? a.list[1 + it] : it;
        ChunkRef r;
        if (!chunk_at(p, task % nchb, task / nchb, r)) continue;  // uniform over the block
        const int h = r.h, ci = r.ci;
        const int L = min(C, r.sp.len - ci * C);
        const size_t bslot = bound_slot(p, r.n, h, r.nch, ci);
        __syncthreads();  // the previous task is done with shared memory
        for (int idx = tid; idx < C * D; idx += NT) {
            const int t = idx / D, jj = idx % D;
            float dov = 0.f, vv = 0.f, wv = 0.f;
            if (t < L) {
                const size_t off = tok_row(p, r.sp, h, ci * C + t) + jj;
                dov = to_f(dOg[off]);
                vv = to_f(v[off]);
                wv = to_f(sg ? wg[off / p.D] : wg[off]);
            }
            sDo[idx] = dov;
            sV[idx] = vv;
            sW[idx] = wv;
        }
        float S[NJ], dS[NJ];
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
            const int j = j0 + jj;
            if (kTcWs) {
                const __nv_bfloat16 *st = (const __nv_bfloat16 *)a.states + bslot * WS * WS;
                const __nv_bfloat16 *ds = (const __nv_bfloat16 *)a.dSe + r.cidx * WS * WS;
                S[jj] = __bfloat162float(st[(size_t)j * WS + c]);
                dS[jj] = __bfloat162float(ds[(size_t)j * WS + c]);
            } else {
                S[jj] = ((const float *)a.states)[(bslot * D + c) * D + j];
                dS[jj] = ((const float *)a.dSe)[(r.cidx * D + c) * D + j];
            }
        }
        __syncthreads();  // sDo, sV, sW staged
        // row scalars of token t for this thread's row c
        auto row_in = [&](int t, float &qc, float &kc, float &bc, float &ac) {
            const size_t off = tok_row(p, r.sp, h, ci * C + t) + c;
            qc = to_f(q[off]);
            kc = to_f(k[off]);
            bc = to_f(sg ? bg[off / p.D] : bg[off]);
            ac = expf(gs ? p.g[off / p.D] : p.g[off]);
        };
        // ---- forward: S'_t into the scratch, u_t into sU
        for (int t = 0; t < L; ++t) {
            float qc, kc, bc, ac;
            row_in(t, qc, kc, bc, ac);
            const float ec = bc * kc;
            float vv[NJ];
            float4 *spd = reinterpret_cast<float4 *>(Sp + ((size_t)t * D + c) * D + j0);
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj) {
                S[jj] *= ac;
                vv[jj] = ec * S[jj];
            }
#pragma unroll
            for (int jj = 0; jj < NJ; jj += 4) spd[jj / 4] = make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
            colsum(vv);
            if (tid < D) sU[t * D + tid] = sW[t * D + tid] * sV[t * D + tid] - colsum_total(tid);
            __syncthreads();
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj) S[jj] = fmaf(kc, sU[t * D + j0 + jj], S[jj]);
        }
        // ---- reverse
        for (int t = L - 1; t >= 0; --t) {
            float qc, kc, bc, ac;
            row_in(t, qc, kc, bc, ac);
            const float ec = bc * kc;
            float spv[NJ], vv[NJ];
            const float4 *sps = reinterpret_cast<const float4 *>(Sp + ((size_t)t * D + c) * D + j0);
#pragma unroll
            for (int jj = 0; jj < NJ; jj += 4) {
                const float4 f = sps[jj / 4];
                spv[jj] = f.x;
                spv[jj + 1] = f.y;
                spv[jj + 2] = f.z;
                spv[jj + 3] = f.w;
            }
            float pq = 0.f, pA = 0.f;
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj) {
                const float u = sU[t * D + j0 + jj], dov = sDo[t * D + j0 + jj];
                const float st = fmaf(kc, u, spv[jj]);
                dS[jj] = fmaf(qc, dov, dS[jj]);
                pq = fmaf(st, dov, pq);
                pA = fmaf(dS[jj], u, pA);
                vv[jj] = dS[jj] * kc;
            }
            colsum(vv);
            if (tid < D) {
                const float du = colsum_total(tid);
                sVec[tid] = du;
                const size_t off = tok_row(p, r.sp, h, ci * C + t) + tid;
                dv[off] = from_f<Tin>(du * sW[t * D + tid]);
                if (!sg) dw[off] = from_f<Tin>(du * sV[t * D + tid]);
                else {
                    const float x = warp_total(du * sV[t * D + tid]);
                    if (lane == 0) sScal[warp] = x;
                }
            }
            __syncthreads();
            if (sg && tid == 0) {
                float x = 0.f;
#pragma unroll
                for (int u = 0; u < NW; ++u) x += sScal[u];
                dw[tok_row(p, r.sp, h, ci * C + t) / p.D] = from_f<Tin>(x);
            }
            float pde = 0.f, pdg = 0.f;
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj) {
                const float du = sVec[j0 + jj];
                const float d = fmaf(-ec, du, dS[jj]);
                pde = fmaf(-spv[jj], du, pde);
                pdg = fmaf(d, spv[jj], pdg);
                dS[jj] = ac * d;
            }
            sRow[(0 * 4 + jq) * D + c] = pq;
            sRow[(1 * 4 + jq) * D + c] = pA;
            sRow[(2 * 4 + jq) * D + c] = pde;
            sRow[(3 * 4 + jq) * D + c] = pdg;
            __syncthreads();
            if (tid < D) {
                float s4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    s4[u] = sRow[(u * 4 + 0) * D + c] + sRow[(u * 4 + 1) * D + c] + sRow[(u * 4 + 2) * D + c] +
                            sRow[(u * 4 + 3) * D + c];
                const float de = s4[2];
                const size_t off = tok_row(p, r.sp, h, ci * C + t) + c;
                dq[off] = from_f<Tin>(s4[0]);
                dk[off] = from_f<Tin>(fmaf(de, bc, s4[1]));
                if (!sg) db[off] = from_f<Tin>(de * kc);
                else {
                    const float x = warp_total(de * kc);
                    if (lane == 0) sScal[NW + warp] = x;
                }
                if (!gs) a.dg[off] = s4[3];
                else {
                    const float x = warp_total(s4[3]);
                    if (lane == 0) sScal[2 * NW + warp] = x;
                }
            }
            if (sg || gs) {
                __syncthreads();
                if (tid == 0) {
                    const size_t tr = tok_row(p, r.sp, h, ci * C + t) / p.D;
                    float x = 0.f, xg = 0.f;
#pragma unroll
                    for (int u = 0; u < NW; ++u) {
                        x += sScal[NW + u];
                        xg += sScal[2 * NW + u];
                    }
                    if (sg) db[tr] = from_f<Tin>(x);
                    if (gs) a.dg[tr] = xg;
                }
            }
        }
    }
}

template <int D, typename Tin, bool kTcWs>
cudaError_t launch_grad(const TokGradArgs &a, int nblocks, cudaStream_t s)
{
    const size_t smem = TokGradSmem<D>::bytes;
    cudaError_t e = set_smem_attr(reinterpret_cast<const void *>(tok_grad_kernel<D, Tin, kTcWs>), (int)smem);
    if (e != cudaSuccess) return e;
    tok_grad_kernel<D, Tin, kTcWs><<<max(1, nblocks), 4 * D, smem, s>>>(a);
    return cudaGetLastError();
}

template <int D, typename Tin>
cudaError_t launch_fwd_t(const Problem &p, void *o, float *S_T, float *states, cudaStream_t s)
{
    tok_fwd_kernel<D, Tin><<<p.B * p.H, 2 * D, 0, s>>>(p, (Tin *)o, S_T, states);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ fp32 backward
constexpr int kGradBlocks = 148;  // blocks of the gradient kernel (one wave on a B200)

struct TokWs {
    size_t coff, states, dSe, scratch, total;
    int blocks;
};
// [chunk_off (variable length only)] [boundary states] [chunk-end dS] [gradient scratch]
TokWs tok_ws(const Problem &p)
{
    const size_t D = p.D, H = p.H, nchunk = chunk_bound(p), nbound = nchunk + p.B;
    TokWs l;
    size_t off = p.cu_seqlens ? varlen_offsets_bytes(p.B) : 0;
    l.coff = 0;
    l.states = off;  off += H * nbound * D * D * 4;
    l.dSe = off;     off += H * nchunk * D * D * 4;
    // the gradient kernel's scratch grows with the problem: as many blocks as the boundary states'
    // bytes pay for (one at least, one wave at most)
    l.blocks = (int)std::max<size_t>(1, std::min<size_t>({H * nchunk, (size_t)kGradBlocks,
                                                           (l.dSe - l.states) / tok_grad_block_bytes(p.D)}));
    l.scratch = off; off += (size_t)l.blocks * tok_grad_block_bytes(p.D);
    l.total = off;
    return l;
}

template <int D, typename Tin>
cudaError_t launch_bwd_t(const Problem &p0, const void *d_o, const float *dS_T, const BwdOut &out, void *ws,
                         int *status, cudaStream_t s)
{
    const TokWs l = tok_ws(p0);
    char *base = static_cast<char *>(ws);
    Problem p = p0;
    cudaError_t e;
    if (p.cu_seqlens) {
        int *coff = reinterpret_cast<int *>(base);
        if ((e = launch_chunk_offsets(p.cu_seqlens, p.B, p.T, coff, status, s)) != cudaSuccess) return e;
        p.chunk_off = coff;
    }
    float *states = reinterpret_cast<float *>(base + l.states);
    float *dSe = reinterpret_cast<float *>(base + l.dSe);
    tok_fwd_kernel<D, Tin><<<p.B * p.H, 2 * D, 0, s>>>(p, nullptr, nullptr, states);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    tok_chain_kernel<D, Tin><<<p.B * p.H, 2 * D, 0, s>>>(p, (const Tin *)d_o, dS_T, dSe, out.dS0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    TokGradArgs a;
    a.p = p;
    a.dO = d_o;
    a.states = states;
    a.dSe = dSe;
    a.list = nullptr;
    a.ntask = (int)(chunk_bound(p) * p.H);
    a.scratch = reinterpret_cast<float *>(base + l.scratch);
    a.dq = out.dq; a.dk = out.dk; a.dv = out.dv; a.db = out.db; a.dw = out.dw; a.dg = out.dg;
    return launch_grad<D, Tin, false>(a, l.blocks, s);
}

}  // namespace

size_t tok_grad_block_bytes(int D) { return (size_t)C * D * D * sizeof(float); }

cudaError_t launch_fwd_tok(gdn2_dtype dt, const Problem &p, void *o, float *S_T, float *states, cudaStream_t s)
{
    if (dt == GDN2_F32)
        return p.D == 64 ? launch_fwd_t<64, float>(p, o, S_T, states, s) : launch_fwd_t<128, float>(p, o, S_T, states, s);
    return p.D == 64 ? launch_fwd_t<64, __nv_bfloat16>(p, o, S_T, states, s)
                     : launch_fwd_t<128, __nv_bfloat16>(p, o, S_T, states, s);
}

cudaError_t launch_tok_grad_tc(const Problem &p, const void *d_o, const __nv_bfloat16 *states,
                               const __nv_bfloat16 *dSn, const int *list, float *scratch, int nblocks,
                               const BwdOut &out, cudaStream_t s)
{
    TokGradArgs a;
    a.p = p;
    a.dO = d_o;
    a.states = states;
    a.dSe = dSn;
    a.list = list;
    a.ntask = 0;
    a.scratch = scratch;
    a.dq = out.dq; a.dk = out.dk; a.dv = out.dv; a.db = out.db; a.dw = out.dw; a.dg = out.dg;
    return p.D == 64 ? launch_grad<64, __nv_bfloat16, true>(a, nblocks, s)
                     : launch_grad<128, __nv_bfloat16, true>(a, nblocks, s);
}

size_t bwd_workspace_bytes(gdn2_dtype dt, const Problem &p)
{
    if (dt == GDN2_BF16) return bwd_tc_workspace_bytes(p);  // d = 128, and d = 64 zero-padded
    return tok_ws(p).total;
}

cudaError_t launch_bwd(gdn2_dtype dt, const Problem &p, const void *d_o, const float *dS_T, const BwdOut &out,
                       void *ws, cudaStream_t s, bool states_saved)
{
    int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    if (dt == GDN2_BF16) return launch_bwd_tc(p, d_o, dS_T, out, ws, status, s, states_saved);
    return p.D == 64 ? launch_bwd_t<64, float>(p, d_o, dS_T, out, ws, status, s)
                     : launch_bwd_t<128, float>(p, d_o, dS_T, out, ws, status, s);
}

}  // namespace gdn2
