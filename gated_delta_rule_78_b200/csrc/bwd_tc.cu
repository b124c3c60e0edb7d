// Gate-aware backward of the chunkwise GDN-2 recurrence on the tensor cores
// (bf16 operands, fp32 accumulation), d_k = d_v = 128, chunk C = 64.
//
// Forward per chunk (S the fp32 state at the chunk start; the chunkwise WY form
// with the decay folded into asymmetric factors, as in the aiexpert.news
// article's implementation paragraph and the aixai.ru post's section "Как это
// реализуется на практике"):
//   G = cumsum(log alpha), Q~ = q e^G, E~ = (b.k) e^G, K~ = k e^-G, gamma = e^G_C,
//   A = strictly_lower(E~ K~^T), P = lower_incl(Q~ K~^T), T = (I + A)^-1, X = w.v,
//   Y = X - E~ S, U~ = T Y, O = Q~ S + P U~, S' = Diag(gamma) (S + K~^T U~).
// Reverse mode (dS_n = dL/dS', dO = dL/dO), the gates staying inside the
// gate-weighted products E~ and X as the aixai.ru post requires:
//   dU~ = P^T dO + K~ Diag(gamma) dS_n        dY = T^T dU~ (= dX)
//   dP  = lower_incl(dO U~^T)                 dA = -strictly_lower(dY U~^T)
//   dQ~ = dO S^T + dP K~                      dE~ = -dY S^T + dA K~
//   dK~ = dA^T E~ + dP^T Q~ + U~ (Diag(gamma) dS_n)^T
//   gamma dgamma = rowsum(dS_n . S')          dS = gamma dS_n + Q~^T dO - E~^T dY
// and through the factors: dq = dQ~ e^G, db = dE~ e^G k, dk = dE~ e^G b + dK~ e^-G,
// dw = dY v, dv = dY w, dG = dQ~ Q~ + dE~ E~ - dK~ K~ (+ gamma dgamma on the last
// row), dlog alpha = reverse cumulative sum of dG inside the chunk.
//
// The only serial dependence is the dS chain.  With W = T E~ and K^ = K~ Diag(gamma):
//   dS = (Diag(gamma) - W^T K^) dS_n + R,   R = Q~^T dO - W^T (P^T dO),
// so the work splits into four launches:
//   1. the tensor-core forward in states mode: S^T (bf16) at every chunk boundary;
//   2. bwd_prep_tc_kernel, one CTA per chunk: factors, [A; P], T, W^T, R^T (no state
//      needed), the products as tcgen05 MMAs with TMEM accumulators;
//   3. bwd_chain_kernel, one CTA per (batch, head): the reverse dS chain,
//      two warp MMAs per chunk with dS^T kept in registers; stores dS_n per chunk;
//   4. bwd_grad_kernel, one CTA per chunk: recomputes U~ from the stored state and
//      produces every gradient of the chunk.
// The chain and gradient products are bf16 warp MMAs (m16n8k16) on ldmatrix-fed
// swizzled tiles.
#include <cuda.h>
#include <string.h>

#include "gdn2_internal.cuh"
#include "tc_util.cuh"
#include "warp_mma.cuh"

namespace gdn2 {
namespace {

using namespace tc;
using namespace wm;

constexpr int D = 128;
constexpr int C = 64;
constexpr int LDA = 68;  // fp32 row stride of the A / T scratch of the solve

// ------------------------------------------------------------------ workspace
struct BwdTcLayout {
    size_t coff, states, W, Kh, gam, Rt, Tm, Pm, dSn, total;
};

// Per (batch, head) and chunk: states S^T bf16 (nchunks + 1 entries), W^T bf16 [D][C],
// K^ bf16 [C][D], gamma fp32 [D], R^T bf16 [D][D], T and P bf16 [C][C], dS_n^T bf16 [D][D].
// Variable length puts chunk_off first; chunk lists are sized by the chunk bound.
BwdTcLayout tc_layout(const Problem &p)
{
    const size_t H = p.H, nchunk = chunk_bound(p), nbound = nchunk + p.B;
    BwdTcLayout l;
    size_t off = p.cu_seqlens ? varlen_offsets_bytes(p.B) : 0;
    l.coff = 0;
    l.states = off; off += H * nbound * D * D * 2;
    l.W = off;      off += H * nchunk * C * D * 2;
    l.Kh = off;     off += H * nchunk * C * D * 2;
    l.gam = off;    off += H * nchunk * D * 4;
    l.Rt = off;     off += H * nchunk * D * D * 2;
    l.Tm = off;     off += H * nchunk * C * C * 2;
    l.Pm = off;     off += H * nchunk * C * C * 2;
    l.dSn = off;    off += H * nchunk * D * D * 2;
    l.total = off;
    return l;
}

struct BwdTcArgs {
    Problem pr;          // sizes, cu_seqlens and chunk_off (the data pointers are below)
    int H;
    int din;             // head size of the tensors: 128, or 64 run zero-padded to 128
    const __nv_bfloat16 *q, *k, *v, *b, *w, *dO;
    const float *g;
    const float *dS_T;  // may be null
    __nv_bfloat16 *states, *W, *Kh, *Tm, *Pm, *dSn;
    float *gam;
    __nv_bfloat16 *Rt;  // R^T per chunk, bf16
    __nv_bfloat16 *dq, *dk, *dv, *db, *dw;
    float *dg, *dS0;
    int n_sm;            // multiprocessors of the device (L2 prefetch distance of the gradient kernel)
    int *status;         // kernel status word (bounded waits that gave up)
};

// ------------------------------------------------------------------ small helpers
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Row t of chunk `ci` of head hh of the sequence whose first token row is `bos`.
__device__ __forceinline__ size_t tok_off(const BwdTcArgs &a, int bos, int hh, int ci, int t)
{
    return (((size_t)bos + (size_t)ci * C + t) * a.H + hh) * a.din;
}

// The chunk a block of the chunk-parallel kernels works on: blockIdx.y is the head,
// blockIdx.x the chunk over all sequences (fixed length: sequence-major; variable
// length: found in chunk_off; blocks past the last chunk have nothing to do).
struct ChunkRef {
    int n, h, ci, nch;
    SeqSpan sp;
    size_t cidx;  // per-chunk workspace slot
};
__device__ __forceinline__ bool chunk_ref_at(const BwdTcArgs &a, int gc, int h, ChunkRef &r)
{
    const Problem &p = a.pr;
    r.h = h;
    if (!p.cu_seqlens) {
        const int nc = seq_chunks(p.T);
        r.n = gc / nc;
        r.ci = gc % nc;
    } else {
        if (gc >= p.chunk_off[p.B]) return false;
        int lo = 0, hi = p.B;  // last n with chunk_off[n] <= gc
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.chunk_off[mid] <= gc) lo = mid;
            else hi = mid;
        }
        r.n = lo;
        r.ci = gc - p.chunk_off[lo];
    }
    r.sp = seq_span(p, r.n);
    if (r.sp.len < 0) return false;
    r.nch = seq_chunks(r.sp.len);
    if (r.ci >= r.nch) return false;
    r.cidx = chunk_slot(p, r.n, r.h, r.nch, r.ci);
    return true;
}
__device__ __forceinline__ bool chunk_ref(const BwdTcArgs &a, ChunkRef &r)
{
    return chunk_ref_at(a, blockIdx.x, blockIdx.y, r);
}

// cp.async versions: the copies stay in flight until cp_async_wait; rows past the
// sequence end are zero-filled (source size 0).
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_tok_tile(uint32_t dst, const __nv_bfloat16 *src, const BwdTcArgs &a, int bb,
                                            int hh, int ci, int L, int tid, int nthreads)
{
    for (int idx = tid; idx < C * 16; idx += nthreads) {
        const int t = idx >> 4, ch = idx & 15;
        const bool ok = t < L && 8 * ch < a.din;  // channels past the head size read zeros
        cp_async16_zfill(dst + swz(t, 8 * ch, 256), src + (ok ? tok_off(a, bb, hh, ci, t) + 8 * ch : 0), ok);
    }
}
__device__ __forceinline__ void cp_dense_tile(uint32_t dst, const __nv_bfloat16 *src, int rows, int cols, int tid,
                                              int nthreads)
{
    const int cpr = cols / 8, rb = cols * 2;
    for (int idx = tid; idx < rows * cpr; idx += nthreads) {
        const int r = idx / cpr, ch = idx % cpr;
        cp_async16(dst + swz(r, 8 * ch, rb), src + (size_t)r * cols + 8 * ch);
    }
}

// store a bf16 pair at (row, col) of a swizzled tile
__device__ __forceinline__ void st_pair(uint8_t *tile, int rb, int row, int col, float lo, float hi)
{
    *reinterpret_cast<uint32_t *>(tile + swz(row, col, rb)) = pack_bf16x2(lo, hi);
}
__device__ __forceinline__ uint32_t ld_pair(const uint8_t *tile, int rb, int row, int col)
{
    return *reinterpret_cast<const uint32_t *>(tile + swz(row, col, rb));
}

// Two-channel layout of the prep and gradient kernels' elementwise work: thread (channel pair cp,
// token group g8) owns channels 2 cp, 2 cp + 1 and tokens 8 g8 .. 8 g8 + 7 (64 x 8 = 512
// threads).  log alpha of those 16 values, zero past the sequence end and the head size.
__device__ __forceinline__ void load_g8(float2 (&g)[8], const BwdTcArgs &a, int bb, int hh, int ci, int L, int cp,
                                        int g8)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = 8 * g8 + i;
        g[i] = (t < L && 2 * cp < a.din)
                   ? __ldg(reinterpret_cast<const float2 *>(a.g + tok_off(a, bb, hh, ci, t) + 2 * cp))
                   : make_float2(0.f, 0.f);
    }
}

// e^G and e^-G of this thread's 16 values (G the inclusive cumulative sum of log alpha over
// the chunk) with one exponential per value: alpha = e^g, then e^G as a running product
// forwards from the token group's start and e^-G as one backwards from its end.  The group
// totals go through sTot ([8][D] fp32); `total` is G at the chunk end.  Contains a
// __syncthreads; kWait: this thread's cp.async copies, except the newest kKeep groups,
// are waited for before it.
template <bool kWait, int kKeep = 0>
__device__ __forceinline__ void decay_pair8(const float2 (&g)[8], float2 (&eG)[8], float2 (&emG)[8], float2 &total,
                                            int cp, int g8, float *sTot)
{
    float run0 = 0.f, run1 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        run0 += g[i].x;
        run1 += g[i].y;
        eG[i] = make_float2(__expf(g[i].x), __expf(g[i].y));  // alpha for now
    }
    *reinterpret_cast<float2 *>(sTot + g8 * D + 2 * cp) = make_float2(run0, run1);
    if (kWait) cp_async_wait<kKeep>();
    __syncthreads();
    float off0 = 0.f, off1 = 0.f, tot0 = 0.f, tot1 = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const float2 v = *reinterpret_cast<const float2 *>(sTot + u * D + 2 * cp);
        if (u < g8) { off0 += v.x; off1 += v.y; }
        tot0 += v.x;
        tot1 += v.y;
    }
    float r0 = __expf(-(off0 + run0)), r1 = __expf(-(off1 + run1));
#pragma unroll
    for (int i = 7; i >= 0; --i) {
        emG[i] = make_float2(r0, r1);
        r0 *= eG[i].x;
        r1 *= eG[i].y;
    }
    float e0 = __expf(off0), e1 = __expf(off1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        e0 *= eG[i].x;
        e1 *= eG[i].y;
        eG[i] = make_float2(e0, e1);
    }
    total = make_float2(tot0, tot1);
}

// bf16x2 product, rounded to nearest even (exact before the rounding for bf16 inputs)
__device__ __forceinline__ uint32_t bmul2(uint32_t x, uint32_t y)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
    return r;
}

// L2 prefetch (bulk, no shared-memory destination)
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ================================================================== 2. prep on the tensor cores
// One 512-thread CTA per (chunk, head): the raw q, b, k, dO tiles arrive by TMA (SW128 atoms),
// the decay folds into them in place, and the four products run as tcgen05 MMAs with TMEM
// accumulators:
//   [A; P] = [E~; Q~] K~^T             M = 128 (stacked tokens), N = 64, K = 128
//   Z^T    = dO^T P                    M = 128 (d_v), N = 64, K = 64   (dO, P MN-major)
//   W^T    = E~^T T^T                  M = 128 (d_k), N = 64, K = 64   (E~ MN-major)
//   R^T    = dO^T Q~ + (-Z^T) W        M = 128 (d_v), N = 128, K = 64 + 64 (-Z^T from TMEM)
// T = (I + A)^-1 is the blocked solve on four warps, as in the forward.  Written out: K^, gamma,
// T, P, W^T (rows d_k, for the chain) and R^T (bf16).
namespace prep_tc {
// Two blocks per SM: regions are reused once their first use is over.
constexpr uint32_t QE = 0;          // [E~ a0 | Q~ a0 | E~ a1 | Q~ a1], 8 KiB each (raw b, q)
constexpr uint32_t KT = 32768;      // K~ [a0 | a1]; after [A; P]: W^T bf16 [128 rows d_k][64 tokens]
constexpr uint32_t WT = KT;
constexpr uint32_t DO = 49152;      // dO [a0 | a1]
constexpr uint32_t PP = 65536;      // P bf16 [64][64]; during the folding: decay totals [4][D] fp32
constexpr uint32_t TOT = PP;
constexpr uint32_t SA = 73728;      // A fp32 [64][LDA]; after the solve: T bf16 [64][64]
constexpr uint32_t TT = SA;
constexpr uint32_t ST = SA + 64 * LDA * 4;   // T fp32 [64][LDA]
constexpr uint32_t USED = ST + 64 * LDA * 4;
constexpr uint32_t SMEM = USED + 1024;       // slack for the 1024-byte alignment
// TMEM: [A; P] then Z^T in 0..63, W^T in 64..127, -Z^T bf16 in 128..159; R^T (issued once
// Z^T and W^T are read back) in 0..127
constexpr uint32_t TM_AP = 0, TM_ZT = 0, TM_WT = 64, TM_ZB = 128, TM_RT = 0, TM_COLS = 256;
constexpr uint32_t IDESC_AP = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_Z = tc::idesc_bf16(128, 64, 1, 1);
constexpr uint32_t IDESC_W = tc::idesc_bf16(128, 64, 1, 0);
constexpr uint32_t IDESC_R1 = tc::idesc_bf16(128, 128, 1, 1);
constexpr uint32_t IDESC_R2 = tc::idesc_bf16(128, 128, 0, 0);
constexpr int kThreads = 256;
}  // namespace prep_tc

struct PrepMaps {
    CUtensorMap q, k, b, dO, g;
};

__device__ __forceinline__ void named_bar(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__global__ void __launch_bounds__(prep_tc::kThreads, 2)
bwd_prep_tc_kernel(const __grid_constant__ PrepMaps maps, const BwdTcArgs a)
{
    using namespace prep_tc;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_in, bar_ap, bar_z, bar_w, bar_r;
    __shared__ uint32_t s_tmem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    ChunkRef cr;
    if (!chunk_ref(a, cr)) return;  // uniform over the block, before any barrier
    const int ci = cr.ci, hh = cr.h, bos = cr.sp.bos;
    const int L = min(C, cr.sp.len - ci * C);
    const size_t cidx = cr.cidx;
    const uint32_t sb = smem_u32(sm);
    float *sA = reinterpret_cast<float *>(sm + SA);
    float *sT = reinterpret_cast<float *>(sm + ST);
    float *sTot = reinterpret_cast<float *>(sm + TOT);

    if (tid == 0) {
        mbar_init(&bar_in, 1);
        mbar_init(&bar_ap, 1);
        mbar_init(&bar_z, 1);
        mbar_init(&bar_w, 1);
        mbar_init(&bar_r, 1);
        fence_mbar_init();
        prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.b); prefetch_tmap(&maps.dO);
        prefetch_tmap(&maps.g);
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, TM_COLS);
        tmem_relinquish();
    }
    for (int idx = tid; idx < 64 * LDA; idx += kThreads) sT[idx] = 0.f;  // upper blocks stay zero
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int y = bos + ci * C;
    if (tid == 0) {
        mbar_expect_tx(&bar_in, 8 * 8192);
        for (int at = 0; at < 2; ++at) {
            tma_load_3d(sm + KT + at * 8192, &maps.k, at * 64, hh, y, &bar_in);
            tma_load_3d(sm + QE + at * 16384, &maps.b, at * 64, hh, y, &bar_in);
            tma_load_3d(sm + QE + 8192 + at * 16384, &maps.q, at * 64, hh, y, &bar_in);
            tma_load_3d(sm + DO + at * 8192, &maps.dO, at * 64, hh, y, &bar_in);
        }
        for (int at = 0; at < a.din / 32; ++at) tma_prefetch_3d(&maps.g, at * 32, hh, y);
    }

    // ---- decay folding: thread (channel block cb, token group tg of 16, lane): channels
    //      64 cb + 2 lane (+1), tokens 16 tg .. 16 tg + 15
    const int cb = warp & 1, tg = warp >> 1, ch = 64 * cb + 2 * lane;
    {
        float2 gv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = 16 * tg + i;
            gv[i] = (t < L && ch < a.din)
                        ? __ldg(reinterpret_cast<const float2 *>(a.g + tok_off(a, bos, hh, ci, t) + ch))
                        : make_float2(0.f, 0.f);
        }
        float run0 = 0.f, run1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            run0 += gv[i].x;
            run1 += gv[i].y;
            gv[i] = make_float2(__expf(gv[i].x), __expf(gv[i].y));  // alpha
        }
        *reinterpret_cast<float2 *>(sTot + tg * D + ch) = make_float2(run0, run1);
        if (!mbar_wait(&bar_in, 0)) atomicExch(a.status, kStatusTimeout);
        __syncthreads();
        float off0 = 0.f, off1 = 0.f, tot0 = 0.f, tot1 = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 v = *reinterpret_cast<const float2 *>(sTot + u * D + ch);
            if (u < tg) { off0 += v.x; off1 += v.y; }
            tot0 += v.x;
            tot1 += v.y;
        }
        const float gam0 = __expf(tot0), gam1 = __expf(tot1);
        if (tg == 0) *reinterpret_cast<float2 *>(a.gam + cidx * D + ch) = make_float2(gam0, gam1);
        float2 mv[16];  // e^-G, backwards from the group's last token
        {
            float r0 = __expf(-(off0 + run0)), r1 = __expf(-(off1 + run1));
#pragma unroll
            for (int i = 15; i >= 0; --i) {
                mv[i] = make_float2(r0, r1);
                r0 *= gv[i].x;
                r1 *= gv[i].y;
            }
        }
        float e0 = __expf(off0), e1 = __expf(off1);
        uint8_t *pe = sm + QE + cb * 16384, *pq = pe + 8192, *pk = sm + KT + cb * 8192;
        __nv_bfloat16 *kh = a.Kh + cidx * C * D;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = 16 * tg + i;
            e0 *= gv[i].x;
            e1 *= gv[i].y;
            const uint32_t off = sw128(t, 4 * lane);
            uint32_t qw = *reinterpret_cast<const uint32_t *>(pq + off);
            uint32_t kw = *reinterpret_cast<const uint32_t *>(pk + off);
            uint32_t bw = *reinterpret_cast<const uint32_t *>(pe + off);
            if (t >= L) { qw = 0u; kw = 0u; bw = 0u; }
            const float k0 = bf_lo(kw), k1 = bf_hi(kw), m0 = mv[i].x, m1 = mv[i].y;
            *reinterpret_cast<uint32_t *>(pq + off) = pack_bf16x2(bf_lo(qw) * e0, bf_hi(qw) * e1);
            *reinterpret_cast<uint32_t *>(pe + off) = pack_bf16x2(bf_lo(bw) * k0 * e0, bf_hi(bw) * k1 * e1);
            *reinterpret_cast<uint32_t *>(pk + off) = pack_bf16x2(k0 * m0, k1 * m1);
            *reinterpret_cast<uint32_t *>(kh + t * D + ch) = pack_bf16x2(k0 * m0 * gam0, k1 * m1 * gam1);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    // ---- [A; P] = [E~; Q~] K~^T
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_AP, sdesc_sw128(sb + QE + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                   sdesc_sw128(sb + KT + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), IDESC_AP, ks > 0);
        mma_commit(&bar_ap);
    }
    if (!mbar_wait(&bar_ap, 0)) atomicExch(a.status, kStatusTimeout);
    tc_fence_after();
    if (warp < 8) {  // A -> fp32 scratch (strictly lower), P -> bf16 tile (lower incl.)
        const int quarter = warp & 3, half = warp >> 2;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t r[32];
        tmem_ld32(tmem + TM_AP + 32 * half + lane_off, r);
        tmem_wait_ld();
        const int row = quarter * 32 + lane;
        if (row < 64) {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int j = 32 * half + u;
                sA[row * LDA + j] = (j < row) ? __uint_as_float(r[u]) : 0.f;
            }
        } else {
            const int t = row - 64;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i0 = 32 * half + 8 * m + 2 * e;
                    w4[e] = pack_bf16x2((i0 <= t) ? __uint_as_float(r[8 * m + 2 * e]) : 0.f,
                                        (i0 + 1 <= t) ? __uint_as_float(r[8 * m + 2 * e + 1]) : 0.f);
                }
                *reinterpret_cast<uint4 *>(sm + PP + sw128(t, 64 * half + 16 * m)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- T = (I + A)^-1 on warps 0-3; Z^T = dO^T P issued meanwhile
    if (warp < 4) {
        wm::solve_unit_lower64<LDA>(sA, sT, warp, lane, [] { named_bar(1, 128); });
    } else if (tid == 128) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_ZT, sdesc_sw128(sb + DO + ks * 2048, 8192, 1024), sdesc_sw128(sb + PP + ks * 2048, 8192, 1024),
                   IDESC_Z, ks > 0);
        mma_commit(&bar_z);
    }
    __syncthreads();
    // ---- T -> bf16 tile and global (threads 0-255), P -> global (threads 256-511): 16 columns each
    {
        const int i = tid >> 2, jq = tid & 3;
        {
            uint32_t w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int j0 = 16 * jq + 2 * e;
                w8[e] = pack_bf16x2((j0 <= i) ? sT[i * LDA + j0] : 0.f, (j0 + 1 <= i) ? sT[i * LDA + j0 + 1] : 0.f);
            }
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const uint4 v = make_uint4(w8[4 * h2], w8[4 * h2 + 1], w8[4 * h2 + 2], w8[4 * h2 + 3]);
                *reinterpret_cast<uint4 *>(sm + TT + sw128(i, 32 * jq + 16 * h2)) = v;
                *reinterpret_cast<uint4 *>(a.Tm + cidx * C * C + i * C + 16 * jq + 8 * h2) = v;
            }
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
            *reinterpret_cast<uint4 *>(a.Pm + cidx * C * C + i * C + 16 * jq + 8 * h2) =
                *reinterpret_cast<const uint4 *>(sm + PP + sw128(i, 32 * jq + 16 * h2));
    }
    fence_proxy_async_smem();
    __syncthreads();
    // ---- W^T = E~^T T^T
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_WT, sdesc_sw128(sb + QE + ks * 2048, 16384, 1024), sdesc_sw128(sb + TT + ks * 32, 16, 1024),
                   IDESC_W, ks > 0);
        mma_commit(&bar_w);
    }
    // -Z^T -> bf16 A operand (warps 0-3: lanes d_v, 64 columns)
    if (!mbar_wait(&bar_z, 0)) atomicExch(a.status, kStatusTimeout);
    tc_fence_after();
    if (warp < 4) {
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t r[32], pk[16];
            tmem_ld32(tmem + TM_ZT + 32 * h2 + lane_off, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(-__uint_as_float(r[2 * e]), -__uint_as_float(r[2 * e + 1]));
            tmem_st16(tmem + TM_ZB + 16 * h2 + lane_off, pk);
        }
        tmem_wait_st();
    }
    // W^T -> bf16 tile (rows d_k, the B operand of R^T) and global (warps 4-7)
    if (!mbar_wait(&bar_w, 0)) atomicExch(a.status, kStatusTimeout);
    tc_fence_after();
    if (warp >= 4 && warp < 8) {
        const int quarter = warp & 3, c = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        __nv_bfloat16 *wg = a.W + cidx * C * D + (size_t)c * C;  // W^T [d_k][C]
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t r[32];
            tmem_ld32(tmem + TM_WT + 32 * h2 + lane_off, r);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(r[8 * m]), __uint_as_float(r[8 * m + 1])),
                                           pack_bf16x2(__uint_as_float(r[8 * m + 2]), __uint_as_float(r[8 * m + 3])),
                                           pack_bf16x2(__uint_as_float(r[8 * m + 4]), __uint_as_float(r[8 * m + 5])),
                                           pack_bf16x2(__uint_as_float(r[8 * m + 6]), __uint_as_float(r[8 * m + 7])));
                *reinterpret_cast<uint4 *>(sm + WT + sw128(c, 64 * h2 + 16 * m)) = v;
                *reinterpret_cast<uint4 *>(wg + 32 * h2 + 8 * m) = v;
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- R^T = dO^T Q~ + (-Z^T) W
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_RT, sdesc_sw128(sb + DO + ks * 2048, 8192, 1024),
                   sdesc_sw128(sb + QE + 8192 + ks * 2048, 16384, 1024), IDESC_R1, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + TM_RT, tmem + TM_ZB + 8 * ks, sdesc_sw128(sb + WT + ks * 32, 16, 1024), IDESC_R2, 1);
        mma_commit(&bar_r);
    }
    if (!mbar_wait(&bar_r, 0)) atomicExch(a.status, kStatusTimeout);
    tc_fence_after();
#pragma unroll
    for (int cq2 = 0; cq2 < 2; ++cq2) {  // R^T -> bf16, global [d_v][d_k]: warp = lane quarter x 2 column blocks
        const int quarter = warp & 3, cq = 2 * (warp >> 2) + cq2, j = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t r[32];
        tmem_ld32(tmem + TM_RT + 32 * cq + lane_off, r);
        tmem_wait_ld();
        __nv_bfloat16 *rt = a.Rt + cidx * D * D + (size_t)j * D + 32 * cq;
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<uint4 *>(rt + 8 * m) =
                make_uint4(pack_bf16x2(__uint_as_float(r[8 * m]), __uint_as_float(r[8 * m + 1])),
                           pack_bf16x2(__uint_as_float(r[8 * m + 2]), __uint_as_float(r[8 * m + 3])),
                           pack_bf16x2(__uint_as_float(r[8 * m + 4]), __uint_as_float(r[8 * m + 5])),
                           pack_bf16x2(__uint_as_float(r[8 * m + 6]), __uint_as_float(r[8 * m + 7])));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ================================================================== 3. chain
// One CTA per (batch, head); warp w owns rows 16 w .. 16 w + 15 of dS^T (d_v x d_k) and
// keeps them in fp32 registers in MMA accumulator layout.  Per chunk, newest first:
//   store dS_n^T (bf16) for the gradient kernel;
//   Z^T = dS_n^T K^^T          (16 x 64 per warp, K = 128; A operand from registers)
//   dS^T = dS_n^T Diag(gamma) + R^T - Z^T W   (K = 64; A operand = -Z^T from registers)
// W, K^, gamma and R^T of the next chunk are copied in (cp.async) during the current one.
constexpr int kChainThreads = 256;
constexpr int LDR = 136;  // bf16 row stride of the R^T tile (conflict-free fragment reads)
constexpr uint32_t CH_W = 0, CH_K = 16384, CH_G = 32768, CH_R = 33280;
constexpr uint32_t CH_BUF = CH_R + D * LDR * 2;  // per buffer
constexpr uint32_t CH_SMEM = 2 * CH_BUF;

__global__ void __launch_bounds__(kChainThreads, 1) bwd_chain_kernel(const BwdTcArgs a)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, n = bh / a.H, hh = bh % a.H;
    const int g = lane >> 2, t4 = lane & 3;
    const int j0 = 16 * warp;  // this warp's first row of dS^T
    const SeqSpan sp = seq_span(a.pr, n);
    if (sp.len < 0) return;  // invalid cu_seqlens (reported by the offsets pass)
    const int nc = seq_chunks(sp.len);
    const uint32_t sb = smem_u32(sm);

    auto prefetch = [&](int ci, int buf) {
        const size_t cidx = chunk_slot(a.pr, n, hh, nc, ci);
        const uint32_t base = sb + buf * CH_BUF;
        const __nv_bfloat16 *wsrc = a.W + cidx * C * D, *ksrc = a.Kh + cidx * C * D;
        for (int idx = tid; idx < C * 16; idx += kChainThreads) {
            const int t = idx >> 4, ch = idx & 15;
            cp_async16(base + CH_K + swz(t, 8 * ch, 256), ksrc + t * D + 8 * ch);
        }
        for (int idx = tid; idx < D * 8; idx += kChainThreads) {  // W^T: 128 rows of 64 tokens
            const int c = idx >> 3, ch = idx & 7;
            cp_async16(base + CH_W + swz(c, 8 * ch, 128), wsrc + c * C + 8 * ch);
        }
        const __nv_bfloat16 *rsrc = a.Rt + cidx * D * D;
        for (int idx = tid; idx < D * 16; idx += kChainThreads) {  // 16 x 16 bytes per bf16 row
            const int r = idx >> 4, ch = idx & 15;
            cp_async16(base + CH_R + (r * LDR + 8 * ch) * 2, rsrc + r * D + 8 * ch);
        }
        if (tid < 32) cp_async16(base + CH_G + 16 * tid, a.gam + cidx * D + 4 * tid);
        cp_async_commit();
    };

    // dS^T rows j0 + g (+8), columns 8 nt + 2 t4 (+1)
    float dS[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = j0 + g + 8 * (e >> 1), c = 8 * nt + 2 * t4 + (e & 1);
            dS[nt][e] = (a.dS_T && c < a.din && j < a.din) ? a.dS_T[((size_t)bh * a.din + c) * a.din + j] : 0.f;
        }
    if (nc > 0) prefetch(nc - 1, 0);
    for (int ci = nc - 1; ci >= 0; --ci) {
        const int buf = (nc - 1 - ci) & 1;
        const size_t cidx = chunk_slot(a.pr, n, hh, nc, ci);
        if (ci > 0) {
            prefetch(ci - 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t wb = sb + buf * CH_BUF + CH_W, kb = sb + buf * CH_BUF + CH_K;
        const float *gam = reinterpret_cast<const float *>(sm + buf * CH_BUF + CH_G);
        const __nv_bfloat16 *rt = reinterpret_cast<const __nv_bfloat16 *>(sm + buf * CH_BUF + CH_R);
        // dS_n^T for the gradient kernel, and as bf16 A fragments
        uint32_t aS[8][4];
        __nv_bfloat16 *dsn = a.dSn + cidx * D * D;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
            acc_to_a(aS[kc], dS[2 * kc], dS[2 * kc + 1], 1.f);
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const size_t row = (size_t)(j0 + g + 8 * hr) * D;
                *reinterpret_cast<uint32_t *>(dsn + row + 16 * kc + 2 * t4) = aS[kc][hr];
                *reinterpret_cast<uint32_t *>(dsn + row + 16 * kc + 8 + 2 * t4) = aS[kc][2 + hr];
            }
        }
        // Z^T = dS_n^T K^^T: B operand K^ stored [t][c] = [n][k]
        float Z[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) Z[nt][e] = 0.f;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc)
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bfr[4];
                load_b2<false>(bfr, kb, 256, 16 * kc, 16 * np, lane);
                mma_bf16(Z[2 * np], aS[kc], bfr[0], bfr[1]);
                mma_bf16(Z[2 * np + 1], aS[kc], bfr[2], bfr[3]);
            }
        // dS^T <- dS_n^T Diag(gamma) + R^T - Z^T W: B operand W stored [t][c] = [k][n]
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const float2 gm = *reinterpret_cast<const float2 *>(gam + 8 * nt + 2 * t4);
            const uint32_t r0w = *reinterpret_cast<const uint32_t *>(rt + (j0 + g) * LDR + 8 * nt + 2 * t4);
            const uint32_t r1w = *reinterpret_cast<const uint32_t *>(rt + (j0 + g + 8) * LDR + 8 * nt + 2 * t4);
            const float2 r0 = make_float2(bf_lo(r0w), bf_hi(r0w)), r1 = make_float2(bf_lo(r1w), bf_hi(r1w));
            dS[nt][0] = dS[nt][0] * gm.x + r0.x;
            dS[nt][1] = dS[nt][1] * gm.y + r0.y;
            dS[nt][2] = dS[nt][2] * gm.x + r1.x;
            dS[nt][3] = dS[nt][3] * gm.y + r1.y;
        }
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            uint32_t aZ[4];
            acc_to_a(aZ, Z[2 * kt], Z[2 * kt + 1], -1.f);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bfr[4];
                load_b2<false>(bfr, wb, 128, 16 * kt, 16 * np, lane);  // W^T stored [c][t] = [n][k]
                mma_bf16(dS[2 * np], aZ, bfr[0], bfr[1]);
                mma_bf16(dS[2 * np + 1], aZ, bfr[2], bfr[3]);
            }
        }
        __syncthreads();  // every warp is done with this buffer before it is refilled
    }
    // dS0 = dS (stored [c][j])
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = j0 + g + 8 * (e >> 1), c = 8 * nt + 2 * t4 + (e & 1);
            if (c < a.din && j < a.din) a.dS0[((size_t)bh * a.din + c) * a.din + j] = dS[nt][e];
        }
}

// ================================================================== 4. gradients
// smem map (bytes): [C][D] bf16 tiles Q~, E~, K~; S^T and (Diag(gamma) dS_n)^T [D][D] bf16;
// X -> U~, w -> Y -> dU~ -> [dP | dA], dO, -dY; T, P [C][C] bf16; scratch.  After the
// products, dQ~, dE~, dK~ (fp32 [C][LDF]) reuse the first 104 KB.
constexpr uint32_t G_Q = 0, G_E = 16384, G_K = 32768, G_S = 49152, G_DS = 81920, G_X = 114688, G_Y = 131072;
constexpr uint32_t G_DO = 147456, G_DY = 163840, G_TB = 180224, G_PB = 188416, G_TOT = 196608;
constexpr uint32_t G_GAM = G_TOT + 8 * D * 4, G_DGP = G_GAM + D * 4, G_DGF = G_DGP + 16 * D * 4;
constexpr uint32_t G_SMEM = G_DGF + D * 4;
constexpr int LDF = 136;  // fp32 row stride of the dQ~ / dE~ / dK~ tiles
constexpr uint32_t G_FQ = 0, G_FE = C * LDF * 4, G_FK = 2 * C * LDF * 4;
static_assert(G_FK + C * LDF * 4 <= G_X, "fp32 gradient tiles must fit in the dead operand tiles");
constexpr int kGradThreads = 512;

__global__ void __launch_bounds__(kGradThreads, 1) bwd_grad_kernel(const BwdTcArgs a)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    ChunkRef cr;
    if (!chunk_ref(a, cr)) return;
    const int ci = cr.ci, hh = cr.h, bb = cr.sp.bos;  // bb: the sequence's first token row
    const int L = min(C, cr.sp.len - ci * C);
    const size_t cidx = cr.cidx;
    const uint32_t sb = smem_u32(sm);
    float *sTot = reinterpret_cast<float *>(sm + G_TOT);
    float *sGam = reinterpret_cast<float *>(sm + G_GAM);
    float *sDgp = reinterpret_cast<float *>(sm + G_DGP);
    float *sDgf = reinterpret_cast<float *>(sm + G_DGF);
    const int cp = tid & 63, g8 = tid >> 6;  // elementwise mapping: channel pair, group of 8 tokens
    const __nv_bfloat16 *st_c = a.states + bound_slot(a.pr, cr.n, hh, cr.nch, ci) * D * D;
    // dS_n and the chunk-end state, for (Diag(gamma) dS_n)^T and gamma dgamma: loaded first, so
    // that their latency hides behind the operand copies and the decay folding
    const int dch = tid & 15;
    uint4 dsv[4], ssv[4];
    {
        const __nv_bfloat16 *dsn = a.dSn + cidx * D * D;
        const __nv_bfloat16 *st_n = st_c + (size_t)D * D;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = (tid >> 4) + 32 * u;
            dsv[u] = __ldg(reinterpret_cast<const uint4 *>(dsn + (size_t)j * D + 8 * dch));
            ssv[u] = __ldg(reinterpret_cast<const uint4 *>(st_n + (size_t)j * D + 8 * dch));
        }
    }

    // ---- P0: operands
    cp_tok_tile(sb + G_Q, a.q, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_K, a.k, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_E, a.b, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_X, a.v, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_Y, a.w, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_DO, a.dO, a, bb, hh, ci, L, tid, kGradThreads);
    cp_dense_tile(sb + G_S, st_c, D, D, tid, kGradThreads);
    cp_dense_tile(sb + G_TB, a.Tm + cidx * C * C, C, C, tid, kGradThreads);
    cp_dense_tile(sb + G_PB, a.Pm + cidx * C * C, C, C, tid, kGradThreads);
    cp_async_commit();
    {
        float2 gl[8], eG[8], emG[8], tot;
        load_g8(gl, a, bb, hh, ci, L, cp, g8);
        decay_pair8<true>(gl, eG, emG, tot, cp, g8, sTot);  // its barrier also publishes the tiles
        if (g8 == 0) *reinterpret_cast<float2 *>(sGam + 2 * cp) = make_float2(__expf(tot.x), __expf(tot.y));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * g8 + i;
            const uint32_t off = swz(t, 2 * cp, 256);
            uint32_t *pq = reinterpret_cast<uint32_t *>(sm + G_Q + off);
            uint32_t *pk = reinterpret_cast<uint32_t *>(sm + G_K + off);
            uint32_t *pe = reinterpret_cast<uint32_t *>(sm + G_E + off);
            uint32_t *px = reinterpret_cast<uint32_t *>(sm + G_X + off);
            const uint32_t q2 = *pq, k2 = *pk, b2 = *pe, x2 = *px, w2 = *reinterpret_cast<const uint32_t *>(sm + G_Y + off);
            const float k0 = bf_lo(k2), k1 = bf_hi(k2);
            *pq = pack_bf16x2(bf_lo(q2) * eG[i].x, bf_hi(q2) * eG[i].y);
            *pe = pack_bf16x2(bf_lo(b2) * k0 * eG[i].x, bf_hi(b2) * k1 * eG[i].y);
            *pk = pack_bf16x2(k0 * emG[i].x, k1 * emG[i].y);
            *px = bmul2(x2, w2);  // X = w.v (columns = j)
        }
    }
    __syncthreads();
    {  // (Diag(gamma) dS_n)^T tile, and gamma dgamma = rowsum(dS_n . S') partials
        const int ch = dch;
        float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float gm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) gm[e] = sGam[8 * ch + e];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = (tid >> 4) + 32 * u;
            const uint4 dv4 = dsv[u], sv4 = ssv[u];
            const uint32_t dw[4] = {dv4.x, dv4.y, dv4.z, dv4.w}, sw[4] = {sv4.x, sv4.y, sv4.z, sv4.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float d0 = bf_lo(dw[e]), d1 = bf_hi(dw[e]);
                part[2 * e] += d0 * bf_lo(sw[e]);
                part[2 * e + 1] += d1 * bf_hi(sw[e]);
                o[e] = pack_bf16x2(d0 * gm[2 * e], d1 * gm[2 * e + 1]);
            }
            *reinterpret_cast<uint4 *>(sm + G_DS + swz(j, 8 * ch, 256)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) part[e] += __shfl_xor_sync(0xffffffffu, part[e], 16);
        if (lane < 16) {
#pragma unroll
            for (int e = 0; e < 8; ++e) sDgp[warp * D + 8 * ch + e] = part[e];
        }
    }
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) s += sDgp[u * D + tid];
        sDgf[tid] = s;
    }
    {  // everything the block one wave later reads, into L2 (one bulk prefetch per thread)
        const int nblk = gridDim.x * gridDim.y, nxt = blockIdx.y * gridDim.x + blockIdx.x + a.n_sm;
        ChunkRef r;
        if (nxt < nblk && chunk_ref_at(a, nxt % gridDim.x, nxt / gridDim.x, r)) {
            const int Ln = min(C, r.sp.len - r.ci * C);
            const uint32_t rowb = (uint32_t)a.din * 2;
            if (tid < 7 * C) {
                const int which = tid / C, t = tid % C;
                if (t < Ln) {
                    const size_t off = tok_off(a, r.sp.bos, r.h, r.ci, t);
                    const __nv_bfloat16 *src = which == 0 ? a.q : which == 1 ? a.k : which == 2 ? a.b
                                             : which == 3 ? a.v : which == 4 ? a.w : a.dO;
                    if (which < 6) bulk_prefetch_l2(src + off, rowb);
                    else bulk_prefetch_l2(a.g + off, 2 * rowb);
                }
            } else if (tid == 7 * C) {
                bulk_prefetch_l2(a.states + bound_slot(a.pr, r.n, r.h, r.nch, r.ci) * D * D, 2 * D * D * 2);
            } else if (tid == 7 * C + 1) {
                bulk_prefetch_l2(a.Tm + r.cidx * C * C, C * C * 2);
            } else if (tid == 7 * C + 2) {
                bulk_prefetch_l2(a.Pm + r.cidx * C * C, C * C * 2);
            } else if (tid == 7 * C + 3) {
                bulk_prefetch_l2(a.dSn + r.cidx * D * D, D * D * 2);
            }
        }
    }
    // warp tiling of the [C][D] products: 16 rows x 32 columns
    const int mt = warp & 3, nq = warp >> 2;
    const int r0 = 16 * mt + g, c0 = 32 * nq + 2 * t4;  // + 8 hr rows, + 8 nt columns
    // ---- P1: Y = X - E~ S  -> bf16 over the raw w tile
    {
        float acc[1][4][4];
        zero_acc(acc);
        warp_gemm<1, 4, false, false, D>(acc, sb + G_E, 256, 16 * mt, sb + G_S, 256, 32 * nq, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int row = r0 + 8 * hr, col = c0 + 8 * nt;
                const uint32_t x = ld_pair(sm + G_X, 256, row, col);
                st_pair(sm + G_Y, 256, row, col, bf_lo(x) - acc[0][nt][2 * hr], bf_hi(x) - acc[0][nt][2 * hr + 1]);
            }
    }
    __syncthreads();
    // ---- P2: U~ = T Y  -> bf16 over X
    {
        float acc[1][4][4];
        zero_acc(acc);
        warp_gemm<1, 4, false, true, C>(acc, sb + G_TB, 128, 16 * mt, sb + G_Y, 256, 32 * nq, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
                st_pair(sm + G_X, 256, r0 + 8 * hr, c0 + 8 * nt, acc[0][nt][2 * hr], acc[0][nt][2 * hr + 1]);
    }
    __syncthreads();
    // ---- P3: dU~ = P^T dO + K~ (Diag(gamma) dS_n)  -> bf16 over Y
    {
        float acc[1][4][4];
        zero_acc(acc);
        warp_gemm<1, 4, true, true, C>(acc, sb + G_PB, 128, 16 * mt, sb + G_DO, 256, 32 * nq, lane);
        warp_gemm<1, 4, false, false, D>(acc, sb + G_K, 256, 16 * mt, sb + G_DS, 256, 32 * nq, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
                st_pair(sm + G_Y, 256, r0 + 8 * hr, c0 + 8 * nt, acc[0][nt][2 * hr], acc[0][nt][2 * hr + 1]);
    }
    __syncthreads();
    // ---- P4: dY = T^T dU~ -> dv = dY w, dw = dY v (global), -dY (bf16)
    {
        uint32_t vv[4][2], ww[4][2];  // all loads first, in flight during the product
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int row = r0 + 8 * hr, col = c0 + 8 * nt;
                vv[nt][hr] = ww[nt][hr] = 0u;
                if (row < L && col < a.din) {
                    const size_t off = tok_off(a, bb, hh, ci, row) + col;
                    vv[nt][hr] = __ldg(reinterpret_cast<const unsigned int *>(a.v + off));
                    ww[nt][hr] = __ldg(reinterpret_cast<const unsigned int *>(a.w + off));
                }
            }
        float acc[1][4][4];
        zero_acc(acc);
        warp_gemm<1, 4, true, true, C>(acc, sb + G_TB, 128, 16 * mt, sb + G_Y, 256, 32 * nq, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int row = r0 + 8 * hr, col = c0 + 8 * nt;
                const float d0 = acc[0][nt][2 * hr], d1 = acc[0][nt][2 * hr + 1];
                st_pair(sm + G_DY, 256, row, col, -d0, -d1);
                if (row < L && col < a.din) {
                    const size_t off = tok_off(a, bb, hh, ci, row) + col;
                    const uint32_t v2 = vv[nt][hr], w2 = ww[nt][hr];
                    *reinterpret_cast<uint32_t *>(a.dv + off) = pack_bf16x2(d0 * bf_lo(w2), d1 * bf_hi(w2));
                    *reinterpret_cast<uint32_t *>(a.dw + off) = pack_bf16x2(d0 * bf_lo(v2), d1 * bf_hi(v2));
                }
            }
    }
    __syncthreads();
    // ---- P5: [dP; dA] = [dO; -dY] U~^T (128 x 64, K = 128) -> bf16 [C][C] tiles over dU~
    {
        const int ms = warp & 7, nh = warp >> 3;
        float acc[1][4][4];
        zero_acc(acc);
        warp_gemm<1, 4, false, false, D>(acc, sb + (ms < 4 ? G_DO : G_DY), 256, 16 * (ms & 3), sb + G_X, 256, 32 * nh,
                                         lane);
        uint8_t *dst = sm + G_Y + (ms < 4 ? 0 : 8192);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int row = 16 * (ms & 3) + g + 8 * hr, col = 32 * nh + 8 * nt + 2 * t4;
                const float v0 = acc[0][nt][2 * hr], v1 = acc[0][nt][2 * hr + 1];
                if (ms < 4)
                    st_pair(dst, 128, row, col, (col <= row) ? v0 : 0.f, (col + 1 <= row) ? v1 : 0.f);
                else
                    st_pair(dst, 128, row, col, (col < row) ? v0 : 0.f, (col + 1 < row) ? v1 : 0.f);
            }
    }
    __syncthreads();
    const uint32_t dPb = sb + G_Y, dAb = sb + G_Y + 8192;
    // ---- P6-P8: dQ~, dE~, dK~ in registers
    float aq[1][4][4], ae[1][4][4], ak[1][4][4];
    zero_acc(aq);
    zero_acc(ae);
    zero_acc(ak);
    warp_gemm<1, 4, false, true, D>(aq, sb + G_DO, 256, 16 * mt, sb + G_S, 256, 32 * nq, lane);
    warp_gemm<1, 4, false, true, C>(aq, dPb, 128, 16 * mt, sb + G_K, 256, 32 * nq, lane);
    warp_gemm<1, 4, false, true, D>(ae, sb + G_DY, 256, 16 * mt, sb + G_S, 256, 32 * nq, lane);
    warp_gemm<1, 4, false, true, C>(ae, dAb, 128, 16 * mt, sb + G_K, 256, 32 * nq, lane);
    warp_gemm<1, 4, true, true, C>(ak, dAb, 128, 16 * mt, sb + G_E, 256, 32 * nq, lane);
    warp_gemm<1, 4, true, true, C>(ak, dPb, 128, 16 * mt, sb + G_Q, 256, 32 * nq, lane);
    warp_gemm<1, 4, false, true, D>(ak, sb + G_X, 256, 16 * mt, sb + G_DS, 256, 32 * nq, lane);
    __syncthreads();  // all operand tiles are dead from here on
    // raw q, k, b for the factor chain, into tiles that the fp32 gradients do not cover
    cp_tok_tile(sb + G_X, a.q, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_Y, a.k, a, bb, hh, ci, L, tid, kGradThreads);
    cp_tok_tile(sb + G_DO, a.b, a, bb, hh, ci, L, tid, kGradThreads);
    cp_async_commit();
    {
        float *fq = reinterpret_cast<float *>(sm + G_FQ), *fe = reinterpret_cast<float *>(sm + G_FE);
        float *fk = reinterpret_cast<float *>(sm + G_FK);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int o = (r0 + 8 * hr) * LDF + c0 + 8 * nt;
                *reinterpret_cast<float2 *>(fq + o) = make_float2(aq[0][nt][2 * hr], aq[0][nt][2 * hr + 1]);
                *reinterpret_cast<float2 *>(fe + o) = make_float2(ae[0][nt][2 * hr], ae[0][nt][2 * hr + 1]);
                *reinterpret_cast<float2 *>(fk + o) = make_float2(ak[0][nt][2 * hr], ak[0][nt][2 * hr + 1]);
            }
    }
    __syncthreads();
    // ---- P10: through the factors (thread: channels 2 cp, 2 cp + 1, tokens 8 g8 .. +7), fp32
    {
        const float *fq = reinterpret_cast<const float *>(sm + G_FQ), *fe = reinterpret_cast<const float *>(sm + G_FE);
        const float *fk = reinterpret_cast<const float *>(sm + G_FK);
        float2 gl[8], eG[8], emG[8], tot;
        load_g8(gl, a, bb, hh, ci, L, cp, g8);
        decay_pair8<true>(gl, eG, emG, tot, cp, g8, sTot);  // sTot is free again (P0 finished)
        const bool ch_ok = 2 * cp < a.din;
        const size_t base = tok_off(a, bb, hh, ci, 8 * g8) + 2 * cp, stride = (size_t)a.H * a.din;
        float2 dG[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * g8 + i;
            const float2 dQ = *reinterpret_cast<const float2 *>(fq + t * LDF + 2 * cp);
            const float2 dE = *reinterpret_cast<const float2 *>(fe + t * LDF + 2 * cp);
            const float2 dK = *reinterpret_cast<const float2 *>(fk + t * LDF + 2 * cp);
            const uint32_t off_s = swz(t, 2 * cp, 256);
            const uint32_t q2 = *reinterpret_cast<const uint32_t *>(sm + G_X + off_s);
            const uint32_t k2 = *reinterpret_cast<const uint32_t *>(sm + G_Y + off_s);
            const uint32_t b2 = *reinterpret_cast<const uint32_t *>(sm + G_DO + off_s);
            const float q0 = bf_lo(q2), q1 = bf_hi(q2), k0 = bf_lo(k2), k1 = bf_hi(k2), b0 = bf_lo(b2), b1 = bf_hi(b2);
            const float de0 = dE.x * eG[i].x, de1 = dE.y * eG[i].y;
            dG[i].x = dQ.x * q0 * eG[i].x + de0 * b0 * k0 - dK.x * k0 * emG[i].x;
            dG[i].y = dQ.y * q1 * eG[i].y + de1 * b1 * k1 - dK.y * k1 * emG[i].y;
            if (t < L && ch_ok) {
                const size_t off = base + (size_t)i * stride;
                *reinterpret_cast<uint32_t *>(a.dq + off) = pack_bf16x2(dQ.x * eG[i].x, dQ.y * eG[i].y);
                *reinterpret_cast<uint32_t *>(a.db + off) = pack_bf16x2(de0 * k0, de1 * k1);
                *reinterpret_cast<uint32_t *>(a.dk + off) =
                    pack_bf16x2(de0 * b0 + dK.x * emG[i].x, de1 * b1 + dK.y * emG[i].y);
            }
        }
        if (g8 == 7) {  // gamma dgamma enters at the last row of the chunk
            dG[7].x += sDgf[2 * cp];
            dG[7].y += sDgf[2 * cp + 1];
        }
        // reverse cumulative sum inside the chunk
        float run0 = 0.f, run1 = 0.f;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            run0 += dG[i].x;
            run1 += dG[i].y;
            dG[i] = make_float2(run0, run1);
        }
        __syncthreads();  // everyone has read sTot (forward cumsum) before it is reused
        *reinterpret_cast<float2 *>(sTot + g8 * D + 2 * cp) = make_float2(run0, run1);
        __syncthreads();
        float after0 = 0.f, after1 = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (u > g8) {
                after0 += sTot[u * D + 2 * cp];
                after1 += sTot[u * D + 2 * cp + 1];
            }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * g8 + i;
            if (t < L && ch_ok)
                *reinterpret_cast<float2 *>(a.dg + base + (size_t)i * stride) =
                    make_float2(dG[i].x + after0, dG[i].y + after1);
        }
    }
}

}  // namespace

size_t bwd_tc_workspace_bytes(const Problem &p) { return tc_layout(p).total; }

cudaError_t launch_fwd_save(const Problem &p, void *o, float *S_T, void *ws, int *status, cudaStream_t s)
{
    if (p.cu_seqlens || (p.D != 128 && p.D != 64)) return cudaErrorNotSupported;
    const BwdTcLayout l = tc_layout(p);
    return launch_fwd_tc(p, o, S_T, reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + l.states), status, s);
}

cudaError_t launch_bwd_tc(const Problem &p, const void *d_o, const float *dS_T, const BwdOut &out, void *ws,
                          int *status, cudaStream_t s, bool states_saved)
{
    if (p.D != 128 && p.D != 64) return cudaErrorNotSupported;
    const BwdTcLayout l = tc_layout(p);
    char *base = static_cast<char *>(ws);
    BwdTcArgs a;
    a.pr = p;
    a.H = p.H;
    a.din = p.D;
    if (p.cu_seqlens) {
        int *coff = reinterpret_cast<int *>(base);
        cudaError_t e0 = launch_chunk_offsets(p.cu_seqlens, p.B, p.T, coff, status, s);
        if (e0 != cudaSuccess) return e0;
        a.pr.chunk_off = coff;
    }
    a.q = static_cast<const __nv_bfloat16 *>(p.q);
    a.k = static_cast<const __nv_bfloat16 *>(p.k);
    a.v = static_cast<const __nv_bfloat16 *>(p.v);
    a.b = static_cast<const __nv_bfloat16 *>(p.b);
    a.w = static_cast<const __nv_bfloat16 *>(p.w);
    a.dO = static_cast<const __nv_bfloat16 *>(d_o);
    a.g = p.g;
    a.dS_T = dS_T;
    a.states = reinterpret_cast<__nv_bfloat16 *>(base + l.states);
    a.W = reinterpret_cast<__nv_bfloat16 *>(base + l.W);
    a.Kh = reinterpret_cast<__nv_bfloat16 *>(base + l.Kh);
    a.gam = reinterpret_cast<float *>(base + l.gam);
    a.Rt = reinterpret_cast<__nv_bfloat16 *>(base + l.Rt);
    a.Tm = reinterpret_cast<__nv_bfloat16 *>(base + l.Tm);
    a.Pm = reinterpret_cast<__nv_bfloat16 *>(base + l.Pm);
    a.dSn = reinterpret_cast<__nv_bfloat16 *>(base + l.dSn);
    a.dq = static_cast<__nv_bfloat16 *>(out.dq);
    a.dk = static_cast<__nv_bfloat16 *>(out.dk);
    a.dv = static_cast<__nv_bfloat16 *>(out.dv);
    a.db = static_cast<__nv_bfloat16 *>(out.db);
    a.dw = static_cast<__nv_bfloat16 *>(out.dw);
    a.dg = out.dg;
    a.dS0 = out.dS0;
    a.status = status;
    {
        int dev = 0;
        a.n_sm = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&a.n_sm, cudaDevAttrMultiProcessorCount, dev);
    }

    cudaError_t e = cudaSuccess;
    if (!states_saved || p.cu_seqlens) {  // chunk-boundary states, unless the forward recorded them
        e = launch_fwd_tc(a.pr, nullptr, nullptr, a.states, status, s);
        if (e != cudaSuccess) return e;
    }
    const dim3 nblk((unsigned)chunk_bound(p), (unsigned)p.H);
    {  // prep on the tensor cores: one block per (chunk, head)
        PrepMaps maps;
        memset(&maps, 0, sizeof(maps));
        const int rows = (int)token_rows(p);
        if (!make_map(&maps.q, p.q, false, 1, rows, p.H, p.D) || !make_map(&maps.k, p.k, false, 1, rows, p.H, p.D) ||
            !make_map(&maps.b, p.b, false, 1, rows, p.H, p.D) || !make_map(&maps.dO, d_o, false, 1, rows, p.H, p.D) ||
            !make_map(&maps.g, p.g, true, 1, rows, p.H, p.D))
            return cudaErrorInvalidValue;
        if ((e = set_smem_attr(reinterpret_cast<const void *>(bwd_prep_tc_kernel), (int)prep_tc::SMEM)) != cudaSuccess)
            return e;
        bwd_prep_tc_kernel<<<nblk, prep_tc::kThreads, prep_tc::SMEM, s>>>(maps, a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = set_smem_attr(reinterpret_cast<const void *>(bwd_chain_kernel), (int)CH_SMEM)) != cudaSuccess) return e;
    bwd_chain_kernel<<<p.B * p.H, kChainThreads, CH_SMEM, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = set_smem_attr(reinterpret_cast<const void *>(bwd_grad_kernel), (int)G_SMEM)) != cudaSuccess) return e;
    bwd_grad_kernel<<<nblk, kGradThreads, G_SMEM, s>>>(a);
    return cudaGetLastError();
}

}  // namespace gdn2
