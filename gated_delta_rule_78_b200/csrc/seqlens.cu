// Variable-length batches: check cu_seqlens and lay out per-chunk workspace lists.
//
// A packed batch of N sequences is described by cu_seqlens[0 .. N] (int32, device):
// sequence n is token rows cu_seqlens[n] .. cu_seqlens[n+1] of [total_T, H, D]
// tensors.  The contract is cu_seqlens[0] = 0, non-decreasing, cu_seqlens[N] =
// total_T (empty sequences are allowed).  chunk_off[n] is the number of 64-token
// chunks of all sequences before n, which places each (sequence, head)'s chunk list
// in the workspace.
#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) chunk_offsets_kernel(const int *cu, int n, int rows, int *coff,
                                                                     int *status)
{
    __shared__ int sbuf[kScanThreads];
    __shared__ int carry, bad;
    const int tid = threadIdx.x;
    if (tid == 0) {
        carry = 0;
        bad = 0;
    }
    __syncthreads();
    for (int base = 0; base < n; base += kScanThreads) {
        const int i = base + tid;
        int c = 0;
        if (i < n) {
            const int b0 = cu[i], b1 = cu[i + 1];
            const bool ok = b0 >= 0 && b1 >= b0 && b1 <= rows && (i > 0 || b0 == 0) && (i < n - 1 || b1 == rows);
            if (ok) c = (b1 - b0 + kChunk - 1) / kChunk;
            else atomicOr(&bad, 1);
        }
        sbuf[tid] = c;
        __syncthreads();
        for (int off = 1; off < kScanThreads; off <<= 1) {  // inclusive scan
            const int v = (tid >= off) ? sbuf[tid - off] : 0;
            __syncthreads();
            sbuf[tid] += v;
            __syncthreads();
        }
        if (coff && i < n) coff[i] = carry + sbuf[tid] - c;
        __syncthreads();
        if (tid == 0) carry += sbuf[kScanThreads - 1];
        __syncthreads();
    }
    if (tid == 0) {
        if (coff) coff[n] = carry;
        if (bad) atomicExch(status, kStatusBadSeqlens);
    }
}

}  // namespace

cudaError_t launch_chunk_offsets(const int *cu_seqlens, int n_seqs, int total_rows, int *chunk_off, int *status,
                                 cudaStream_t s)
{
    chunk_offsets_kernel<<<1, kScanThreads, 0, s>>>(cu_seqlens, n_seqs, total_rows, chunk_off, status);
    return cudaGetLastError();
}

}  // namespace gdn2
