// Chunkwise GDN-2 forward in fp32 FMA arithmetic (the fp32 path).
//
// One CTA owns one (batch, head, 32-column slice of d_v) and walks the chunks
// of 64 tokens in order, carrying its d_k x 32 slice of the fp32 state in
// shared memory.  The columns of the state are independent (the update only
// mixes rows), so slicing d_v gives D/32 times more CTAs with no exchange.
//
// Per chunk (G = inclusive cumulative sum of log alpha inside the chunk,
// G_L its last row), following the chunkwise WY algorithm of the aiexpert.news
// article (decay absorbed into asymmetric erase factors) and the auxiliary
// matrices of the aixai.ru post ("Как это реализуется на практике"):
//   Q~ = q e^G, E~ = (b.k) e^G, K~ = k e^-G, K^ = k e^(G_L - G), gamma = e^G_L
//   A  = strictly_lower(E~ K~^T)                       erase-gated interactions
//   W  = (I + A)^-1 E~,  U = (I + A)^-1 (w.V)           forward substitution
//   U~ = U - W S
//   O  = Q~ S + lower_incl(Q~ K~^T) U~
//   S  = Diag(gamma) S + K^^T U~
// A ragged last chunk is zero-padded (k, q, b, v, w = 0 and log alpha = 0 on
// the padding), which leaves every real row unchanged.
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kThreads = 256;
constexpr int kDVT = 32;  // d_v columns per CTA

template <int D>
struct SimtSmem {
    static constexpr int LD = D + 1;  // padded row stride of the C x D factors
    static constexpr int LA = kChunk + 1;
    static constexpr size_t floats = 4 * (size_t)kChunk * LD + (size_t)kChunk * LA +
                                     (size_t)kChunk * kDVT + (size_t)D * kDVT + D;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D, typename Tin>
__global__ void __launch_bounds__(kThreads)
fwd_simt_kernel(Problem p, Tin *__restrict__ o, float *__restrict__ S_T, float *__restrict__ states)
{
    using SM = SimtSmem<D>;
    constexpr int C = kChunk, LD = SM::LD, LA = SM::LA;
    extern __shared__ float sm[];
    float *Qt = sm;                  // [C][LD]
    float *Et = Qt + C * LD;         // [C][LD]  E~, then W
    float *Kt = Et + C * LD;         // [C][LD]
    float *Kh = Kt + C * LD;         // [C][LD]
    float *Am = Kh + C * LD;         // [C][LA]  A, then P
    float *Xu = Am + C * LA;         // [C][kDVT] X, then U, then U~
    float *S = Xu + C * kDVT;        // [D][kDVT]
    float *gam = S + D * kDVT;       // [D]

    const int tid = threadIdx.x;
    const int bh = blockIdx.x, bb = bh / p.H, hh = bh % p.H;
    const int j0 = blockIdx.y * kDVT;
    const SeqSpan sp = seq_span(p, bb);
    if (sp.len < 0) return;  // invalid cu_seqlens (reported by the offsets pass)
    const int T = sp.len;
    const size_t tok = (size_t)p.H * D;                      // token stride (elements)
    const size_t base = tok_row(p, sp, hh, 0);               // (sequence bb, t = 0, h, 0)
    const Tin *q = (const Tin *)p.q, *k = (const Tin *)p.k, *v = (const Tin *)p.v;
    const Tin *bg = (const Tin *)p.b, *wg = (const Tin *)p.w;
    const int nchunks = (T + C - 1) / C;

    for (int idx = tid; idx < D * kDVT; idx += kThreads) {
        const int c = idx / kDVT, j = idx % kDVT;
        S[idx] = p.S0 ? p.S0[((size_t)bh * D + c) * D + j0 + j] : 0.f;
    }

    for (int ci = 0; ci < nchunks; ++ci) {
        const int c0 = ci * C;
        const int L = min(C, T - c0);
        __syncthreads();  // S ready; previous chunk done with every buffer
        if (states) {
            float *dst = states + chunk_slot(p, bb, hh, nchunks, ci) * D * D;
            for (int idx = tid; idx < D * kDVT; idx += kThreads) {
                const int c = idx / kDVT, j = idx % kDVT;
                dst[(size_t)c * D + j0 + j] = S[idx];
            }
        }
        // ---- decay folding: one thread per key channel walks the tokens
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
                Qt[t * LD + c] = qv * eG;
                Et[t * LD + c] = bv * kv * eG;
                Kt[t * LD + c] = kv * expf(-G);
                Kh[t * LD + c] = G;  // temporarily G_t
            }
            gam[c] = expf(G);
            for (int t = 0; t < C; ++t) {
                float kv = 0.f;
                if (t < L) kv = to_f(k[base + (size_t)(c0 + t) * tok + c]);
                Kh[t * LD + c] = kv * expf(G - Kh[t * LD + c]);
            }
        } else {
            for (int idx = tid - D; idx < C * kDVT; idx += kThreads - D) {
                const int t = idx / kDVT, j = idx % kDVT;
                float x = 0.f;
                if (t < L) {
                    const size_t off = base + (size_t)(c0 + t) * tok + j0 + j;
                    x = to_f(wg[off]) * to_f(v[off]);
                }
                Xu[idx] = x;
            }
        }
        __syncthreads();
        // ---- A = strictly_lower(E~ K~^T)
        {
            const int i = tid >> 2, jb = tid & 3;
            float acc[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.f;
            for (int c = 0; c < D; ++c) {
                const float e = Et[i * LD + c];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) acc[jj] += e * Kt[(jb + 4 * jj) * LD + c];
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = jb + 4 * jj;
                Am[i * LA + j] = (j < i) ? acc[jj] : 0.f;
            }
        }
        __syncthreads();
        // ---- W = (I+A)^-1 E~ (columns of E~), U = (I+A)^-1 X: forward substitution,
        //      one thread per column, in place
        if (tid < D + kDVT) {
            float *col = tid < D ? Et + tid : Xu + (tid - D);
            const int st = tid < D ? LD : kDVT;
            for (int i = 1; i < C; ++i) {
                float s = col[i * st];
                for (int m = 0; m < i; ++m) s -= Am[i * LA + m] * col[m * st];
                col[i * st] = s;
            }
        }
        __syncthreads();
        // ---- P = lower_incl(Q~ K~^T) into Am
        {
            const int i = tid >> 2, jb = tid & 3;
            float acc[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.f;
            for (int c = 0; c < D; ++c) {
                const float qv = Qt[i * LD + c];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) acc[jj] += qv * Kt[(jb + 4 * jj) * LD + c];
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = jb + 4 * jj;
                Am[i * LA + j] = (j <= i) ? acc[jj] : 0.f;
            }
        }
        // ---- U~ = U - W S (in place in Xu; each thread owns its entries)
        {
            const int j = tid & 31, ib = tid >> 5;
#pragma unroll
            for (int ii = 0; ii < C / 8; ++ii) {
                const int i = ib + 8 * ii;
                float acc = Xu[i * kDVT + j];
                for (int c = 0; c < D; ++c) acc -= Et[i * LD + c] * S[c * kDVT + j];
                Xu[i * kDVT + j] = acc;
            }
        }
        __syncthreads();
        // ---- O = Q~ S + P U~
        if (o) {
            const int j = tid & 31, ib = tid >> 5;
            for (int ii = 0; ii < C / 8; ++ii) {
                const int i = ib + 8 * ii;
                if (i >= L) break;
                float acc = 0.f;
                for (int c = 0; c < D; ++c) acc += Qt[i * LD + c] * S[c * kDVT + j];
                for (int m = 0; m <= i; ++m) acc += Am[i * LA + m] * Xu[m * kDVT + j];
                o[base + (size_t)(c0 + i) * tok + j0 + j] = from_f<Tin>(acc);
            }
        }
        __syncthreads();
        // ---- S = Diag(gamma) S + K^^T U~
        {
            const int j = tid & 31, cb = tid >> 5;
            for (int cc = 0; cc < D / 8; ++cc) {
                const int c = cb + 8 * cc;
                float acc = gam[c] * S[c * kDVT + j];
                for (int t = 0; t < C; ++t) acc += Kh[t * LD + c] * Xu[t * kDVT + j];
                S[c * kDVT + j] = acc;
            }
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = tid; idx < D * kDVT; idx += kThreads) {
            const int c = idx / kDVT, j = idx % kDVT;
            S_T[((size_t)bh * D + c) * D + j0 + j] = S[idx];
        }
    }
}

template <int D, typename Tin>
cudaError_t launch_t(const Problem &p, void *o, float *S_T, float *states, cudaStream_t s)
{
    const size_t smem = SimtSmem<D>::bytes;
    cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<D, Tin>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.B * p.H, D / kDVT);
    fwd_simt_kernel<D, Tin><<<grid, kThreads, smem, s>>>(p, (Tin *)o, S_T, states);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(gdn2_dtype dt, const Problem &p, void *o, float *S_T, float *states,
                            cudaStream_t s)
{
    if (dt == GDN2_F32) {
        return p.D == 64 ? launch_t<64, float>(p, o, S_T, states, s)
                         : launch_t<128, float>(p, o, S_T, states, s);
    }
    return p.D == 64 ? launch_t<64, __nv_bfloat16>(p, o, S_T, states, s)
                     : launch_t<128, __nv_bfloat16>(p, o, S_T, states, s);
}

}  // namespace gdn2
