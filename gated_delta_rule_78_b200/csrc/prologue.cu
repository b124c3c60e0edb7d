// The input prologue as separate elementwise passes.  The aixai.ru post's architecture
// paragraph ("Как это реализуется на практике") L2-normalises queries and keys before the
// recurrent update and derives the erase and write gates from their own projections (taken
// here as logits through the logistic sigmoid, which gives gates in [0, 1]); log alpha is
// computed outside the kernel.  The bf16 tensor-core forward applies the prologue inside the
// chunk kernel (fwd_tc.cu); every other path runs these passes:
//   forward: q_n = q / sqrt(|q|^2 + eps) and k_n likewise, per token and head over the head
//            dimension; b_s = sigmoid(b), w_s = sigmoid(w), per channel or per token;
//   backward (in place on the gradients of the normalised / activated inputs):
//            dq <- r (dq - q_n (q_n . dq)) with r = 1 / sqrt(|q|^2 + eps), likewise dk;
//            db <- db s (1 - s) with s = sigmoid(b), likewise dw.
// One warp per (token, head) row; each lane holds D / 32 consecutive channels.
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

__device__ __forceinline__ float bf2f(uint32_t x, int hi) { return __uint_as_float(hi ? (x & 0xffff0000u) : (x << 16)); }
__device__ __forceinline__ uint32_t f2bf2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// E consecutive elements as fp32
template <int E> __device__ __forceinline__ void ld(const float *p, float (&f)[E])
{
    if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        f[0] = v.x; f[1] = v.y;
    }
}
template <int E> __device__ __forceinline__ void ld(const __nv_bfloat16 *p, float (&f)[E])
{
    if constexpr (E == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        f[0] = bf2f(v.x, 0); f[1] = bf2f(v.x, 1); f[2] = bf2f(v.y, 0); f[3] = bf2f(v.y, 1);
    } else {
        const uint32_t v = *reinterpret_cast<const uint32_t *>(p);
        f[0] = bf2f(v, 0); f[1] = bf2f(v, 1);
    }
}
template <int E> __device__ __forceinline__ void st(float *p, const float (&f)[E])
{
    if constexpr (E == 4) *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(f[0], f[1]);
}
template <int E> __device__ __forceinline__ void st(__nv_bfloat16 *p, const float (&f)[E])
{
    if constexpr (E == 4) *reinterpret_cast<uint2 *>(p) = make_uint2(f2bf2(f[0], f[1]), f2bf2(f[2], f[3]));
    else *reinterpret_cast<uint32_t *>(p) = f2bf2(f[0], f[1]);
}
__device__ __forceinline__ float ld1(const float *p) { return *p; }
__device__ __forceinline__ float ld1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st1(float *p, float v) { *p = v; }
__device__ __forceinline__ void st1(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}
__device__ __forceinline__ float sigmoid(float x) { return 1.f / (1.f + __expf(-x)); }

struct ProArgs {
    size_t rows;           // token rows x heads
    int norm;              // q, k: normalise
    int gate_mode[2];      // b, w: 0 untouched, 1 per channel, 2 per token (one value per row)
    const void *q, *k, *b, *w;    // raw inputs
    void *qn, *kn, *bs, *ws;      // forward outputs
    void *dq, *dk, *db, *dw;      // backward: gradients, rewritten in place
};

template <typename T, int D>
__global__ void __launch_bounds__(256) prologue_fwd_kernel(const ProArgs a)
{
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const size_t nwarps = (size_t)gridDim.x * (blockDim.x >> 5);
    for (size_t row = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < a.rows; row += nwarps) {
        const size_t off = row * D + (size_t)lane * E;
        if (a.norm) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const T *src = static_cast<const T *>(which ? a.k : a.q);
                T *dst = static_cast<T *>(which ? a.kn : a.qn);
                float f[E];
                ld<E>(src + off, f);
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) ss += f[e] * f[e];
                const float r = rsqrtf(warp_sum(ss) + kNormEps);
#pragma unroll
                for (int e = 0; e < E; ++e) f[e] *= r;
                st<E>(dst + off, f);
            }
        }
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
            const T *src = static_cast<const T *>(gi ? a.w : a.b);
            T *dst = static_cast<T *>(gi ? a.ws : a.bs);
            if (a.gate_mode[gi] == 1) {
                float f[E];
                ld<E>(src + off, f);
#pragma unroll
                for (int e = 0; e < E; ++e) f[e] = sigmoid(f[e]);
                st<E>(dst + off, f);
            } else if (a.gate_mode[gi] == 2 && lane == 0) {
                st1(dst + row, sigmoid(ld1(src + row)));
            }
        }
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) prologue_bwd_kernel(const ProArgs a)
{
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const size_t nwarps = (size_t)gridDim.x * (blockDim.x >> 5);
    for (size_t row = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < a.rows; row += nwarps) {
        const size_t off = row * D + (size_t)lane * E;
        if (a.norm) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const T *x = static_cast<const T *>(which ? a.k : a.q);
                T *dx = static_cast<T *>(which ? a.dk : a.dq);
                float f[E], g[E];
                ld<E>(x + off, f);
                ld<E>(dx + off, g);
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) ss += f[e] * f[e];
                const float r = rsqrtf(warp_sum(ss) + kNormEps);
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    f[e] *= r;  // x_n
                    dot += f[e] * g[e];
                }
                dot = warp_sum(dot);
#pragma unroll
                for (int e = 0; e < E; ++e) g[e] = r * (g[e] - f[e] * dot);
                st<E>(dx + off, g);
            }
        }
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
            const T *x = static_cast<const T *>(gi ? a.w : a.b);
            T *dx = static_cast<T *>(gi ? a.dw : a.db);
            if (a.gate_mode[gi] == 1) {
                float f[E], g[E];
                ld<E>(x + off, f);
                ld<E>(dx + off, g);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float sg = sigmoid(f[e]);
                    g[e] *= sg * (1.f - sg);
                }
                st<E>(dx + off, g);
            } else if (a.gate_mode[gi] == 2 && lane == 0) {
                const float sg = sigmoid(ld1(x + row));
                st1(dx + row, ld1(dx + row) * sg * (1.f - sg));
            }
        }
    }
}

cudaError_t launch_pro(bool bwd, bool fp32, int D, const ProArgs &a, cudaStream_t s)
{
    if (a.rows == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t want = (a.rows + 7) / 8;  // 8 rows (warps) per block
    const unsigned grid = (unsigned)(want < (size_t)sms * 16 ? want : (size_t)sms * 16);
    if (D == 128) {
        if (fp32) (bwd ? prologue_bwd_kernel<float, 128> : prologue_fwd_kernel<float, 128>)<<<grid, 256, 0, s>>>(a);
        else (bwd ? prologue_bwd_kernel<__nv_bfloat16, 128> : prologue_fwd_kernel<__nv_bfloat16, 128>)<<<grid, 256, 0, s>>>(a);
    } else if (D == 64) {
        if (fp32) (bwd ? prologue_bwd_kernel<float, 64> : prologue_fwd_kernel<float, 64>)<<<grid, 256, 0, s>>>(a);
        else (bwd ? prologue_bwd_kernel<__nv_bfloat16, 64> : prologue_fwd_kernel<__nv_bfloat16, 64>)<<<grid, 256, 0, s>>>(a);
    } else {
        return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prologue_fwd(bool fp32, size_t rows, int D, bool norm, const void *q, const void *k, void *qn,
                                void *kn, int b_mode, const void *b, void *bs, int w_mode, const void *w, void *ws,
                                cudaStream_t s)
{
    ProArgs a{};
    a.rows = rows;
    a.norm = norm ? 1 : 0;
    a.gate_mode[0] = b_mode;
    a.gate_mode[1] = w_mode;
    a.q = q; a.k = k; a.b = b; a.w = w;
    a.qn = qn; a.kn = kn; a.bs = bs; a.ws = ws;
    return launch_pro(false, fp32, D, a, s);
}

cudaError_t launch_prologue_bwd(bool fp32, size_t rows, int D, bool norm, const void *q, const void *k, void *dq,
                                void *dk, int b_mode, const void *b, void *db, int w_mode, const void *w, void *dw,
                                cudaStream_t s)
{
    ProArgs a{};
    a.rows = rows;
    a.norm = norm ? 1 : 0;
    a.gate_mode[0] = b_mode;
    a.gate_mode[1] = w_mode;
    a.q = q; a.k = k; a.b = b; a.w = w;
    a.dq = dq; a.dk = dk; a.db = db; a.dw = dw;
    return launch_pro(true, fp32, D, a, s);
}

}  // namespace gdn2
