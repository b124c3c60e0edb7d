// gdn2_chunk_bwd_noalloc: the chunkwise backward with its scratch in a static
// device array instead of a caller-supplied workspace.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they run
// the backward -- code inside a custom allocator or memory pool (which would
// recurse into itself), runtimes that forbid device allocation after start-up
// so that their memory budget stays fixed, and plain C hosts with no tensor
// library around to hand them a buffer.  They pass inputs and outputs as usual;
// the scratch comes from `g_bwd_scratch` below, which is reserved once on every
// GPU that loads the library and stays reserved until the process exits.
//
// This entry point allocates nothing: no cudaMalloc, no cudaFree, no library
// routine that allocates.  It runs the same three kernels as gdn2_chunk_bwd,
// with the same workspace layout, so both give the same gradients.
#include <atomic>
#include <stdint.h>

#include "gdn2_internal.cuh"

namespace {

constexpr size_t kScratchBytes = GDN2_NOALLOC_MAX_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a handle for the runtime: its
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

// Device address of g_bwd_scratch per device ordinal (null until first use).
std::atomic<void *> g_scratch_addr[kMaxDevices];

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

gdn2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA; }

// The current device's address of g_bwd_scratch; looked up on the first call
// made with that device current.  Two threads racing here both store the same
// value, so the race is harmless.
gdn2_status scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN2_ERR_UNSUPPORTED;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return GDN2_ERR_CUDA;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return GDN2_OK;
}

}  // namespace

extern "C" GDN2_API gdn2_status gdn2_chunk_bwd_noalloc(
    gdn2_dtype dt, int B, int T, int H, int Dk, int Dv, const void *q, const void *k, const void *v,
    const float *log_alpha, const void *b, const void *w, const float *S0, const void *d_o,
    const float *dS_T, void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
    float *dS0, void *stream)
{
    // the same argument rules as gdn2_chunk_bwd
    if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (B <= 0 || H <= 0 || T < 0 || Dk <= 0 || Dv <= 0) return GDN2_ERR_SHAPE;
    if (Dk != Dv || (Dk != 64 && Dk != 128)) return GDN2_ERR_UNSUPPORTED;
    if ((long long)B * H > (1LL << 30)) return GDN2_ERR_UNSUPPORTED;
    if ((long long)B * T * H * Dk > (1LL << 40)) return GDN2_ERR_UNSUPPORTED;
    if (T > 0) {
        const void *req[] = {q, k, v, log_alpha, b, w, d_o, dq, dk, dv, dlog_alpha, db, dw, dS0};
        for (const void *p : req)
            if (!p) return GDN2_ERR_NULL;
        for (const void *p : req)
            if (!aligned16(p)) return GDN2_ERR_ALIGN;
    } else if (!dS0) {
        return GDN2_ERR_NULL;
    } else if (!aligned16(dS0)) {
        return GDN2_ERR_ALIGN;
    }
    if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T))) return GDN2_ERR_ALIGN;

    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) {
        const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
        if (dS_T) return from_cuda(cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(dS0, 0, state_bytes, s));
    }
    gdn2::Problem p;
    p.B = B; p.T = T; p.H = H; p.D = Dk;
    p.q = q; p.k = k; p.v = v; p.b = b; p.w = w; p.g = log_alpha; p.S0 = S0;
    if (gdn2::bwd_workspace_bytes(dt, p) > kScratchBytes) return GDN2_ERR_TOO_LARGE;

    void *scratch = nullptr;
    const gdn2_status st = scratch_address(&scratch);
    if (st != GDN2_OK) return st;
    // Every scratch byte the kernels read is written earlier in the same call
    // (chunk-start states, per-chunk matrices, per-slice partial gradients), so
    // nothing left by an earlier call needs clearing.
    gdn2::BwdOut out{dq, dk, dv, db, dw, dlog_alpha, dS0};
    return from_cuda(gdn2::launch_bwd(dt, p, d_o, dS_T, out, scratch, s));
}
