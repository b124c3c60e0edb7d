// Token-by-token form of the GDN-2 recurrence, shared by the token-level kernels (tok.cu: the
// fp32 path, and the exact path for chunks whose decay is too strong for the chunkwise factors)
// and by the tensor-core forward and dS chain for such chunks.
//
// The recurrence, per token t (the update as the aixai.ru post's section "Один скаляр не может
// решать два разных вопроса" describes it: decay first, an erase-weighted read of the decayed
// state, a gated write, the output read after the update):
//   S' = Diag(alpha_t) S,  u = w_t.v_t - S'^T (b_t.k_t),  S <- S' + k_t u^T,  o_t = S^T q_t
//      = S'^T q_t + (k_t . q_t) u
// and its reverse mode for the state gradient (no forward state needed):
//   dS += q_t do_t^T,  du = dS^T k_t,  dS <- Diag(alpha_t) (dS - (b_t.k_t) du^T).
// No factor here is e^{+|G|}: every product is of values no larger than the inputs, so the path
// is exact for any decay alpha in [0, 1].
//
// State layout ("column layout"): 2 D threads; thread (j = tid % D, hf = tid / D) holds column
// j (the d_v index) of S at rows c = hf D/2 .. hf D/2 + D/2 - 1 (the d_k index).  The sums over
// d_k are one exchange between the two halves.
#pragma once

#include "gdn2_internal.cuh"

namespace gdn2 {
namespace tok {

// One token's vectors in shared memory, fp32: q, k, e = b.k, a = alpha = e^g, and x = w.v (the
// forward) or do (the dS chain).  16-byte aligned rows.
template <int D>
struct Rec {
    float q[D], k[D], e[D], a[D], x[D];
};

__device__ __forceinline__ void bar_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// One forward step.  S[i] = S[hf D/2 + i][j].  xch: 6 D floats for this step's parity (three
// partial sums per half).  `hook` runs before the step's barrier (it fills the next token's
// record).  Returns o_t[j].
template <int D, typename Hook>
__device__ __forceinline__ float fwd_step(float (&S)[D / 2], const Rec<D> &r, float *xch, int j, int hf, int bar_id,
                                         Hook &&hook)
{
    constexpr int NR = D / 2;
    const int c0 = hf * NR;
    float ra = 0.f, pa = 0.f, kq = 0.f;
#pragma unroll
    for (int i = 0; i < NR; i += 4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(&r.a[c0 + i]);
        const float4 e4 = *reinterpret_cast<const float4 *>(&r.e[c0 + i]);
        const float4 q4 = *reinterpret_cast<const float4 *>(&r.q[c0 + i]);
        const float4 k4 = *reinterpret_cast<const float4 *>(&r.k[c0 + i]);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, ev[4] = {e4.x, e4.y, e4.z, e4.w};
        const float qv[4] = {q4.x, q4.y, q4.z, q4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float s = av[u] * S[i + u];
            S[i + u] = s;
            ra = fmaf(ev[u], s, ra);
            pa = fmaf(qv[u], s, pa);
            kq = fmaf(kv[u], qv[u], kq);
        }
    }
    xch[(0 * 2 + hf) * D + j] = ra;
    xch[(1 * 2 + hf) * D + j] = pa;
    xch[(2 * 2 + hf) * D + j] = kq;
    hook();
    bar_sync(bar_id, 2 * D);
    const int ot = hf ^ 1;
    ra += xch[(0 * 2 + ot) * D + j];
    pa += xch[(1 * 2 + ot) * D + j];
    kq += xch[(2 * 2 + ot) * D + j];
    const float u = r.x[j] - ra;
#pragma unroll
    for (int i = 0; i < NR; i += 4) {
        const float4 k4 = *reinterpret_cast<const float4 *>(&r.k[c0 + i]);
        S[i] = fmaf(k4.x, u, S[i]);
        S[i + 1] = fmaf(k4.y, u, S[i + 1]);
        S[i + 2] = fmaf(k4.z, u, S[i + 2]);
        S[i + 3] = fmaf(k4.w, u, S[i + 3]);
    }
    return fmaf(kq, u, pa);
}

// One reverse step of the state gradient.  dS[i] = dS[hf D/2 + i][j]; r.x holds do.  xch: 2 D
// floats for this step's parity.
template <int D, typename Hook>
__device__ __forceinline__ void chain_step(float (&dS)[D / 2], const Rec<D> &r, float *xch, int j, int hf, int bar_id,
                                           Hook &&hook)
{
    constexpr int NR = D / 2;
    const int c0 = hf * NR;
    const float dO = r.x[j];
    float du = 0.f;
#pragma unroll
    for (int i = 0; i < NR; i += 4) {
        const float4 q4 = *reinterpret_cast<const float4 *>(&r.q[c0 + i]);
        const float4 k4 = *reinterpret_cast<const float4 *>(&r.k[c0 + i]);
        const float qv[4] = {q4.x, q4.y, q4.z, q4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float d = fmaf(qv[u], dO, dS[i + u]);
            dS[i + u] = d;
            du = fmaf(d, kv[u], du);
        }
    }
    xch[hf * D + j] = du;
    hook();
    bar_sync(bar_id, 2 * D);
    du += xch[(hf ^ 1) * D + j];
#pragma unroll
    for (int i = 0; i < NR; i += 4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(&r.a[c0 + i]);
        const float4 e4 = *reinterpret_cast<const float4 *>(&r.e[c0 + i]);
        dS[i] = a4.x * fmaf(-e4.x, du, dS[i]);
        dS[i + 1] = a4.y * fmaf(-e4.y, du, dS[i + 1]);
        dS[i + 2] = a4.z * fmaf(-e4.z, du, dS[i + 2]);
        dS[i + 3] = a4.w * fmaf(-e4.w, du, dS[i + 3]);
    }
}

// Records of consecutive tokens are triple-buffered: the step on record s fills record s + 1
// before its barrier; record s + 1 was last read in step s - 2, which every thread left before
// the barrier of step s - 1.  The exchange buffers alternate by step parity.
//
// Runs `n` forward steps over tokens t0, t0 + 1, ...  `fill(t, rec)` writes this thread's part of
// token t's record; `emit(step, o)` receives o_t[j] of each step.  recs: 3 records; xch: 12 D
// floats.  The first record is filled and published here.
template <int D, typename Fill, typename Emit>
__device__ __forceinline__ void fwd_tokens(float (&S)[D / 2], int t0, int n, Rec<D> *recs, float *xch, int j, int hf,
                                           int bar_id, Fill &&fill, Emit &&emit)
{
    if (n <= 0) return;
    fill(t0, recs[0]);
    bar_sync(bar_id, 2 * D);
    for (int s = 0; s < n; ++s) {
        const float o = fwd_step<D>(S, recs[s % 3], xch + (s & 1) * 6 * D, j, hf, bar_id, [&] {
            if (s + 1 < n) fill(t0 + s + 1, recs[(s + 1) % 3]);
        });
        emit(s, o);
    }
    bar_sync(bar_id, 2 * D);  // every thread is done with the records and the exchange buffers
}

// Runs `n` reverse steps over tokens t_last, t_last - 1, ...  (records as above; xch: 4 D floats)
template <int D, typename Fill>
__device__ __forceinline__ void chain_tokens(float (&dS)[D / 2], int t_last, int n, Rec<D> *recs, float *xch, int j,
                                             int hf, int bar_id, Fill &&fill)
{
    if (n <= 0) return;
    fill(t_last, recs[0]);
    bar_sync(bar_id, 2 * D);
    for (int s = 0; s < n; ++s) {
        chain_step<D>(dS, recs[s % 3], xch + (s & 1) * 2 * D, j, hf, bar_id, [&] {
            if (s + 1 < n) fill(t_last - s - 1, recs[(s + 1) % 3]);
        });
    }
    bar_sync(bar_id, 2 * D);
}

}  // namespace tok
}  // namespace gdn2
