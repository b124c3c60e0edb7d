// Gate layouts other than one value per channel: a per-(token, head) scalar used for
// every channel, or an absent gate (the constant 1 for the erase and write gates, 0 for
// the log decay).  With b = w = beta scalar the recurrence is KDA; with a scalar decay as
// well it is Gated DeltaNet; without decay it is DeltaNet (the hierarchy of the
// needhelp.icu write-up's generalisation section).  The ablations of the aixai.ru post
// ("Абляции": erase gate only, write gate only) are the absent-gate cases.
//
// The chunk and decode kernels take full [rows, H, D] gate tensors; these launches
// broadcast a scalar or constant gate into such a tensor, and sum a full gradient over
// the channels back into a scalar gradient.
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

// the 32-bit word holding one fp32 value, or two copies of one bf16 value
__device__ __forceinline__ uint32_t splat32(float v) { return __float_as_uint(v); }
__device__ __forceinline__ uint32_t splat32(__nv_bfloat16 v)
{
    const uint32_t h = __bfloat16_as_ushort(v);
    return h | (h << 16);
}

template <typename T>
__global__ void expand_kernel(const T *__restrict__ src, T *__restrict__ dst, size_t n_rows, int D, float fill)
{
    // one (token, head) row of D values per iteration; 16-byte stores
    constexpr int kVec = 16 / sizeof(T);
    const int per_row = D / kVec;
    const size_t total = n_rows * per_row;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / per_row;
        const uint32_t u = splat32(src ? src[row] : from_f<T>(fill));
        reinterpret_cast<uint4 *>(dst)[i] = make_uint4(u, u, u, u);
    }
}

template <typename T>
__global__ void channel_sum_kernel(const T *__restrict__ src, T *__restrict__ dst, size_t n_rows, int D)
{
    // one warp per (token, head) row: fp32 sum of its D values
    const int lane = threadIdx.x & 31;
    const size_t warp0 = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
    const size_t nwarps = ((size_t)gridDim.x * blockDim.x) >> 5;
    for (size_t row = warp0; row < n_rows; row += nwarps) {
        float s = 0.f;
        for (int c = lane; c < D; c += 32) s += to_f(src[row * D + c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) dst[row] = from_f<T>(s);
    }
}

int grid_for(size_t work, int threads)
{
    const size_t blocks = (work + threads - 1) / threads;
    return (int)(blocks < 148 * 32 ? (blocks ? blocks : 1) : 148 * 32);
}

}  // namespace

cudaError_t launch_expand_gate(bool fp32, const void *src, void *dst, size_t n_rows, int D, float fill, cudaStream_t s)
{
    if (fp32) {
        expand_kernel<float><<<grid_for(n_rows * D / 4, 256), 256, 0, s>>>(static_cast<const float *>(src),
                                                                             static_cast<float *>(dst), n_rows, D, fill);
    } else {
        expand_kernel<__nv_bfloat16><<<grid_for(n_rows * D / 8, 256), 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(src), static_cast<__nv_bfloat16 *>(dst), n_rows, D, fill);
    }
    return cudaGetLastError();
}

cudaError_t launch_channel_sum(bool fp32, const void *src, void *dst, size_t n_rows, int D, cudaStream_t s)
{
    if (fp32) {
        channel_sum_kernel<float><<<grid_for(n_rows * 32, 256), 256, 0, s>>>(static_cast<const float *>(src),
                                                                               static_cast<float *>(dst), n_rows, D);
    } else {
        channel_sum_kernel<__nv_bfloat16><<<grid_for(n_rows * 32, 256), 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(src), static_cast<__nv_bfloat16 *>(dst), n_rows, D);
    }
    return cudaGetLastError();
}

}  // namespace gdn2
