// Single-token GDN-2 decode step: S <- (I - k (b.k)^T) Diag(alpha) S + k (w.v)^T in place,
// o = S^T q, for N sequences x H heads.
//
// The state (D x D fp32 per sequence-head, 64 KiB at D = 128) is the whole
// cost: it is read once and written once, so the kernel streams it.  One CTA
// owns one (sequence, head); its 8 warps each hold D/8 state rows in
// registers, each lane a 16-byte (D = 128) or 8-byte (D = 64) column slice,
// so every warp-wide access is one contiguous row segment.
//   S'  = Diag(alpha) S                     in registers
//   r   = S'^T (b.k),  p = S'^T q           per-warp partial sums, then a shared-memory tree
//   u   = w.v - r,     o = p + (k.q) u      since S_new^T q = S'^T q + k^T q u
//   S   = S' + k u^T                        written back with streaming stores
// Recurrent decode with constant memory per token is the property the aixai.ru
// post's opening section and its "Почему это важно" section point to.
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kWarps = 8;

template <int D> struct Vec;
template <> struct Vec<128> { using T = float4; };
template <> struct Vec<64> { using T = float2; };

__device__ __forceinline__ void scale_fma(float4 &s, float a) { s.x *= a; s.y *= a; s.z *= a; s.w *= a; }
__device__ __forceinline__ void scale_fma(float2 &s, float a) { s.x *= a; s.y *= a; }

__device__ __forceinline__ float sigmoid(float x) { return 1.f / (1.f + __expf(-x)); }

// kPro: the fused input prologue (kProNorm | kProSigmoid of gdn2_internal.cuh): q and k are
// L2-normalised in the block before use, b and w pass through the sigmoid.  `modes` gives each
// gate's layout (two bits each, kGate* of gdn2_internal.cuh): a scalar gate is read once per
// (sequence, head) and used for every channel, an absent one is not read.
template <int D, typename Tin, int kPro>
__global__ void __launch_bounds__(kWarps * 32)
decode_kernel(int H, const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ g, const Tin *__restrict__ b, const Tin *__restrict__ w,
              float *__restrict__ S, Tin *__restrict__ o, int modes)
{
    constexpr int CPT = D / 32;      // columns per lane
    constexpr int RPW = D / kWarps;  // rows per warp
    using V = typename Vec<D>::T;
    __shared__ float s_q[D], s_k[D], s_e[D], s_a[D], s_u[D];
    __shared__ float s_r[kWarps][D], s_p[kWarps][D];
    __shared__ float s_kq;
    __shared__ float s_nrm[D / 32][2];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t nh = blockIdx.x;
    const size_t vec = nh * D;
    float *Sp = S + nh * D * D;
    const int mg = modes & 3, mb = (modes >> 2) & 3, mw = (modes >> 4) & 3;
    // element of each gate this thread reads (tid < D): its channel, or the (sequence, head) scalar
    const size_t g_at = mg == kGateScalar ? nh : vec + tid, b_at = mb == kGateScalar ? nh : vec + tid,
                 w_at = mw == kGateScalar ? nh : vec + tid;

    // issue the state loads first: they are the long pole
    V sv[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const int row = warp * RPW + r;
        sv[r] = __ldcs(reinterpret_cast<const V *>(Sp + (size_t)row * D) + lane);
    }
    if (tid < D) {
        float kv = to_f(k[vec + tid]), qv = to_f(q[vec + tid]);
        if (kPro & kProNorm) {  // |q|^2, |k|^2: warp sums, combined below
            float sq = qv * qv, sk = kv * kv;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
            }
            if (lane == 0) {
                s_nrm[warp][0] = sq;
                s_nrm[warp][1] = sk;
            }
        }
        s_a[tid] = expf(mg == kGateAbsent ? 0.f : g[g_at]);
        s_q[tid] = qv;
        s_k[tid] = kv;
    }
    if (kPro & kProNorm) __syncthreads();
    if (tid < D) {
        float qv = s_q[tid], kv = s_k[tid];
        if (kPro & kProNorm) {
            float nq = 0.f, nk = 0.f;
#pragma unroll
            for (int wi = 0; wi < D / 32; ++wi) { nq += s_nrm[wi][0]; nk += s_nrm[wi][1]; }
            qv *= rsqrtf(nq + kNormEps);
            kv *= rsqrtf(nk + kNormEps);
            s_q[tid] = qv;
            s_k[tid] = kv;
        }
        const float bv = mb == kGateAbsent ? 1.f : to_f(b[b_at]);
        s_e[tid] = ((kPro & kProSigmoid) ? sigmoid(bv) : bv) * kv;
    }
    __syncthreads();
    if (warp == 0) {
        float kq = 0.f;
        for (int i = lane; i < D; i += 32) kq += s_k[i] * s_q[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (lane == 0) s_kq = kq;
    }
    float pr[CPT], pp[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) { pr[c] = 0.f; pp[c] = 0.f; }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const int row = warp * RPW + r;
        const float a = s_a[row], e = s_e[row], qq = s_q[row];
        scale_fma(sv[r], a);
        const float *x = reinterpret_cast<const float *>(&sv[r]);
#pragma unroll
        for (int c = 0; c < CPT; ++c) { pr[c] += x[c] * e; pp[c] += x[c] * qq; }
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) { s_r[warp][lane * CPT + c] = pr[c]; s_p[warp][lane * CPT + c] = pp[c]; }
    __syncthreads();
    if (tid < D) {
        float r = 0.f, pq = 0.f;
#pragma unroll
        for (int wi = 0; wi < kWarps; ++wi) { r += s_r[wi][tid]; pq += s_p[wi][tid]; }
        const float wv = mw == kGateAbsent ? 1.f : to_f(w[w_at]);
        const float u = ((kPro & kProSigmoid) ? sigmoid(wv) : wv) * to_f(v[vec + tid]) - r;
        s_u[tid] = u;
        o[vec + tid] = from_f<Tin>(pq + s_kq * u);
    }
    __syncthreads();
    float uu[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) uu[c] = s_u[lane * CPT + c];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const int row = warp * RPW + r;
        const float kk = s_k[row];
        float *x = reinterpret_cast<float *>(&sv[r]);
#pragma unroll
        for (int c = 0; c < CPT; ++c) x[c] += kk * uu[c];
        __stcs(reinterpret_cast<V *>(Sp + (size_t)row * D) + lane, sv[r]);
    }
}

template <int D, typename Tin>
cudaError_t launch_t(int N, int H, const void *q, const void *k, const void *v, const float *g,
                     const void *b, const void *w, float *S, void *o, int pro, int modes, cudaStream_t s)
{
    auto go = [&](auto kernel) {
        kernel<<<N * H, kWarps * 32, 0, s>>>(H, (const Tin *)q, (const Tin *)k, (const Tin *)v, g, (const Tin *)b,
                                             (const Tin *)w, S, (Tin *)o, modes);
        return cudaGetLastError();
    };
    switch (pro) {
    case kProNorm: return go(decode_kernel<D, Tin, kProNorm>);
    case kProSigmoid: return go(decode_kernel<D, Tin, kProSigmoid>);
    case kProNorm | kProSigmoid: return go(decode_kernel<D, Tin, kProNorm | kProSigmoid>);
    default: return go(decode_kernel<D, Tin, 0>);
    }
}

}  // namespace

cudaError_t launch_decode(gdn2_dtype dt, int N, int H, int D, const void *q, const void *k,
                          const void *v, const float *g, const void *b, const void *w, float *S,
                          void *o, cudaStream_t s, int prologue, int gate_modes)
{
    if (prologue & ~(kProNorm | kProSigmoid)) return cudaErrorInvalidValue;
    for (int i = 0; i < 3; ++i)
        if (((gate_modes >> (2 * i)) & 3) > kGateAbsent) return cudaErrorInvalidValue;
    if (gate_modes >> 6) return cudaErrorInvalidValue;
    if (dt == GDN2_F32)
        return D == 64 ? launch_t<64, float>(N, H, q, k, v, g, b, w, S, o, prologue, gate_modes, s)
                       : launch_t<128, float>(N, H, q, k, v, g, b, w, S, o, prologue, gate_modes, s);
    return D == 64 ? launch_t<64, __nv_bfloat16>(N, H, q, k, v, g, b, w, S, o, prologue, gate_modes, s)
                   : launch_t<128, __nv_bfloat16>(N, H, q, k, v, g, b, w, S, o, prologue, gate_modes, s);
}

}  // namespace gdn2
