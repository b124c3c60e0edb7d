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
// B200's 148 SMs, one CTA each).  The plan: segment 0 of k L chunks, then m middle segments and
// a last one of L chunks each (at least kScanMinChunks), with k and m chosen to minimise the
// modelled time over C chains.  Pass 0's segment-0 CTAs run first and hold C SMs for k L; the
// 2 C m middle CTAs run on the other SMs in ceil(2 C m / (148 - C)) waves of L; pass 1 runs
// C (m + 1) CTAs in ceil(C (m + 1) / 148) waves of L:
//   time = max(k, waves_0) L + waves_1 L   against the serial chain's (k + m + 1) L.
// For example 32 chains take k = 2, m = 3 (0.5 of the serial time; three equal segments give
// 0.67), 64 chains k = 2, m = 1 (0.75), and 16 chains six equal segments (0.33).
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kScanSlots = 148;
constexpr int kScanMaxSegments = 8;
constexpr int kScanMaxK = 4;                    // segment 0 at most this many segment lengths
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
    if (p.cu_seqlens || p.g_scalar || p.prologue || nch < 3 * kScanMinChunks || chains >= kScanSlots) return l;
    // modelled time in chunk steps of every plan (k, m); the serial chain takes nch
    long long best = nch;
    for (int k = 1; k <= kScanMaxK; ++k) {
        for (int m = 1; m + 2 <= kScanMaxSegments; ++m) {
            const int tm = (nch + k + m) / (k + m + 1);  // middle segments' chunks
            if (tm < kScanMinChunks) continue;
            // the rounding remainder goes to the last segment (segment 0 of k tm chunks), or else
            // to segment 0 (every later segment of tm chunks)
            for (int v = 0; v < 2; ++v) {
                const int t0 = v == 0 ? k * tm : nch - (m + 1) * tm;
                const int last = nch - t0 - m * tm;
                if (t0 < tm || last < 1 || last > tm) continue;
                const long long w0 = (2 * chains * m + (kScanSlots - chains) - 1) / (kScanSlots - chains);
                const long long w1 = (chains * (m + 1) + kScanSlots - 1) / kScanSlots;
                const long long t = (t0 > w0 * tm ? t0 : w0 * tm) + w1 * tm;
                if (t < best) {
                    best = t;
                    l.nseg = m + 2;
                    l.seg_len = tm * kChunk;
                    l.seg0_len = t0 * kChunk;
                }
            }
        }
    }
    if (!l.nseg) return l;
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
