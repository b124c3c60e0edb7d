// Chunk-parallel scan of the forward, for batches whose (batch, head) chains are too few to
// fill the GPU at long T.  Over a segment of chunks the state map is affine,
//   S_end = Phi S_start + S^,
// with S^ the segment's end state from a zero start and Phi (d_k x d_k) the chain's linear
// part (Diag(gamma) (I - K~^T T E~) per chunk, multiplied up) applied to the identity, which
// the chunk kernel computes as a chain with X = 0 from S = I.  Combining these maps is
// associative, so segments can run side by side:
//   pass 0 (one launch): segment 0 from S0 with its output; for each middle segment its S^
//                        and its Phi;
//   combine:             S_start(1) = S_end(0), S_start(s+1) = Phi_s S_start(s) + S^_s;
//   pass 1 (one launch): segments 1 .. nseg-1 from their start states with their output.
// Each combine step costs a d_k x d_k x d_v product, and pass 0 runs two chains per middle
// segment, so the scan pays only where the serial chain leaves SMs idle (kScanSlots: the
// B200's 148 SMs, one CTA each), for segments of at least kScanMinChunks chunks:
// * up to 48 chains: n equal segments, n the largest (up to kScanMaxSegments) whose pass 0,
//   (2n - 3) CTAs per chain, fits one wave; pass 0 and pass 1 each take one segment's time;
// * 49 to 74 chains: segment 0 twice as long as the two after it.  Pass 0 has 3 CTAs per
//   chain; the first wave holds every segment-0 CTA and half of the middle ones, and the
//   other half runs when those finish, within segment 0's time.  T = 4 L gives 2 L + L.
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kScanSlots = 148;
constexpr int kScanMaxSegments = 8;
constexpr int kScanMaxChains = kScanSlots / 3;  // equal segments: 3 CTAs per chain in pass 0
constexpr int kScanMaxChainsLong0 = kScanSlots / 2;  // long segment 0: 2 chains' worth per wave
constexpr int kScanMinChunks = 16;              // per segment

// S_start(s) for s = 1 .. nseg-1 of one (b, h), 16 state columns per block.
template <int D>
__global__ void __launch_bounds__(256) scan_combine_kernel(int H, int nseg, const float *send0, const float *shat,
                                                           const float *phi, float *sstart)
{
    constexpr int TPR = 256 / D, CPT = 16 / TPR;  // threads per row, columns per thread
    __shared__ float cur[D][16];
    const int bh = blockIdx.x, b = bh / H, h = bh % H, c0 = blockIdx.y * 16, tid = threadIdx.x;
    const int r = tid / TPR, cc = (tid % TPR) * CPT;
    const size_t dd = (size_t)D * D;
    const float *src = send0 + (size_t)bh * dd;
    float *dst = sstart + ((size_t)b * (nseg - 1) * H + h) * dd;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const float v = src[(size_t)r * D + c0 + cc + c];
        cur[r][cc + c] = v;
        dst[(size_t)r * D + c0 + cc + c] = v;
    }
    __syncthreads();
    for (int sg = 1; sg <= nseg - 2; ++sg) {
        const size_t slot = ((size_t)b * (nseg - 2) + sg - 1) * H + h;
        const float *P = phi + slot * dd + (size_t)r * D;
        const float *Sh = shat + slot * dd + (size_t)r * D + c0 + cc;
        float acc[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c] = Sh[c];
#pragma unroll 8
        for (int m = 0; m < D; ++m) {
            const float pm = __ldg(P + m);
#pragma unroll
            for (int c = 0; c < CPT; ++c) acc[c] = fmaf(pm, cur[m][cc + c], acc[c]);
        }
        __syncthreads();  // every thread has read cur
        float *d = sstart + (((size_t)b * (nseg - 1) + sg) * H + h) * dd + (size_t)r * D + c0 + cc;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            cur[r][cc + c] = acc[c];
            d[c] = acc[c];
        }
        __syncthreads();
    }
}

struct ScanLayout {
    int nseg, seg_len, seg0_len;
    size_t send0, shat, phi, sstart, total;
};

ScanLayout scan_layout(const Problem &p)
{
    ScanLayout l{};
    const int nch = (p.T + kChunk - 1) / kChunk;
    const long long chains = (long long)p.B * p.H;
    if (p.cu_seqlens || p.g_scalar || p.prologue || nch < 3 * kScanMinChunks) return l;
    if (chains <= kScanMaxChains) {
        int n = 3;
        while (n < kScanMaxSegments && chains * (2 * (n + 1) - 3) <= kScanSlots && nch >= (n + 1) * kScanMinChunks)
            ++n;
        l.nseg = n;
        l.seg_len = (nch + l.nseg - 1) / l.nseg * kChunk;
        l.seg0_len = l.seg_len;
    } else if (chains <= kScanMaxChainsLong0 && nch >= 4 * kScanMinChunks) {
        l.nseg = 3;
        const int b = (nch + 3) / 4;  // chunks of segments 1 and 2; segment 0 takes the rest
        l.seg_len = b * kChunk;
        l.seg0_len = (nch - 2 * b) * kChunk;
    } else {
        return l;
    }
    const size_t st = (size_t)p.B * p.H * p.D * p.D * sizeof(float);
    l.send0 = 0;
    l.shat = l.send0 + st;
    l.phi = l.shat + st * (l.nseg - 2);
    l.sstart = l.phi + st * (l.nseg - 2);
    l.total = l.sstart + st * (l.nseg - 1);
    return l;
}

}  // namespace

size_t fwd_scan_workspace_bytes(const Problem &p) { return scan_layout(p).total; }

cudaError_t launch_fwd_scan(const Problem &p, void *o, float *S_T, void *ws, size_t ws_bytes, int *status,
                            cudaStream_t s)
{
    const ScanLayout l = scan_layout(p);
    if (!l.nseg || !ws || ws_bytes < l.total) return cudaErrorInvalidValue;
    char *base = static_cast<char *>(ws);
    float *send0 = reinterpret_cast<float *>(base + l.send0), *shat = reinterpret_cast<float *>(base + l.shat);
    float *phi = reinterpret_cast<float *>(base + l.phi), *sstart = reinterpret_cast<float *>(base + l.sstart);
    ScanArgs a{l.nseg, l.seg_len, 0, l.seg0_len, send0, shat, phi, nullptr};
    cudaError_t e = launch_fwd_tc(p, o, S_T, nullptr, status, s, &a);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(p.B * p.H), (unsigned)(p.D / 16));
    if (p.D == 128) scan_combine_kernel<128><<<grid, 256, 0, s>>>(p.H, l.nseg, send0, shat, phi, sstart);
    else scan_combine_kernel<64><<<grid, 256, 0, s>>>(p.H, l.nseg, send0, shat, phi, sstart);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    a.pass = 1;
    a.sstart = sstart;
    return launch_fwd_tc(p, o, S_T, nullptr, status, s, &a);
}

}  // namespace gdn2
