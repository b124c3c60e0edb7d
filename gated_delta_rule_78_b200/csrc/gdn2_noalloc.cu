// gdn2_chunk_bwd_noalloc: the chunkwise backward with its scratch in a static
// device array instead of a caller-supplied workspace.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they run
// the backward -- code inside a custom allocator or memory pool (which would
// recurse into itself), runtimes that forbid device allocation after start-up
// so that their memory budget stays fixed, and plain C hosts with no tensor
// library around to hand them a buffer.  They pass inputs and outputs as usual;
// the scratch comes from `g_bwd_scratch` below.
//
// When the array's memory is taken: CUDA loads a library's modules lazily by
// default (CUDA_MODULE_LOADING=LAZY), so the 32 MiB are committed on a device at
// the first call of this entry point with that device current, not when the
// library is loaded.  From then on they stay reserved until the process exits.
// A caller whose memory budget must not move, or that captures streams into CUDA
// graphs, makes one call on every device at start-up, before the budget is fixed
// and before any capture.
//
// This entry point allocates nothing: no cudaMalloc, no cudaFree, no library
// routine that allocates.  It runs the same three kernels as gdn2_chunk_bwd,
// with the same workspace layout, so both give the same gradients.
#include <stdint.h>

#include "gdn2_internal.cuh"

namespace {

constexpr size_t kScratchBytes = GDN2_NOALLOC_MAX_SCRATCH_BYTES;

// The scratch.  In host code this name is only a handle for the runtime: its
// device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

gdn2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA; }

// The current device's address of g_bwd_scratch, looked up on every call (a
// cheap lookup once the module is loaded), so that no address outlives the
// context it came from: after cudaDeviceReset the module is loaded anew and its
// address may change.
gdn2_status scratch_address(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return GDN2_ERR_CUDA;
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
    // the argument rules of gdn2_chunk_bwd, from the same routine
    const gdn2_status chk = gdn2::check_bwd_args(dt, B, T, H, Dk, Dv, q, k, v, log_alpha, b, w, S0, d_o, dS_T, dq,
                                                 dk, dv, dlog_alpha, db, dw, dS0);
    if (chk != GDN2_OK) return chk;

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
    // (chunk-start states, per-chunk matrices, the count of chunks that run token
    // by token, which the call clears first), so nothing left by an earlier call
    // is read.
    gdn2::BwdOut out{dq, dk, dv, db, dw, dlog_alpha, dS0};
    return from_cuda(gdn2::launch_bwd(dt, p, d_o, dS_T, out, scratch, s));
}
