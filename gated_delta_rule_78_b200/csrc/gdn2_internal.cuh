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

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Problem description handed from the C ABI layer to the launchers.  All
// pointers are device pointers; layouts as in gdn2.h.
struct Problem {
    int B, T, H, D;  // Dk == Dv == D
    const void *q, *k, *v, *b, *w;
    const float *g;   // log alpha
    const float *S0;  // may be null
};

// forward (SIMT fp32 FMA path).  `states`, when non-null, receives the state at
// the start of every chunk: [B*H][nchunks][D][D] fp32.  `o` may be null (states only).
cudaError_t launch_fwd_simt(gdn2_dtype dt, const Problem &p, void *o, float *S_T, float *states,
                            cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit on the current device (once per
// kernel and device; thread-safe).
cudaError_t set_smem_attr(const void *kernel, int bytes);

// forward on the tensor cores (bf16 operands); returns cudaErrorNotSupported when
// the shape is outside what the kernel handles.  `o` may be null (no output);
// `states`, when non-null, receives S^T in bf16 at every chunk boundary:
// [B*H][nchunks + 1][D][D], entry c the state before chunk c, the last entry S_T.
cudaError_t launch_fwd_tc(const Problem &p, void *o, float *S_T, __nv_bfloat16 *states, int *status,
                          cudaStream_t s);

cudaError_t launch_decode(gdn2_dtype dt, int N, int H, int D, const void *q, const void *k,
                          const void *v, const float *g, const void *b, const void *w, float *S,
                          void *o, cudaStream_t s);

struct BwdOut {
    void *dq, *dk, *dv, *db, *dw;
    float *dg, *dS0;
};
// Backward workspace bytes (depends on the path: bf16 with D = 128 runs on the
// tensor cores, everything else on the fp32 FMA kernels).
size_t bwd_workspace_bytes(gdn2_dtype dt, int B, int T, int H, int D);
cudaError_t launch_bwd(gdn2_dtype dt, const Problem &p, const void *d_o, const float *dS_T,
                       const BwdOut &out, void *ws, cudaStream_t s);

// tensor-core backward (bf16, D = 128): the forward in states mode, then the prep,
// chain and gradient kernels
size_t bwd_tc_workspace_bytes(int B, int T, int H);
cudaError_t launch_bwd_tc(const Problem &p, const void *d_o, const float *dS_T, const BwdOut &out, void *ws,
                          int *status, cudaStream_t s);

// device address of the library's kernel status word on the current device
int *status_word();

}  // namespace gdn2
