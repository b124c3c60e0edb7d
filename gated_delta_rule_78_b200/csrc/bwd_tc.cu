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
//   gamma dgamma = rowsum(dS_n . S') = gamma rowsum(dS_n . S) + sum_t K~_t . (U~ (Diag(gamma) dS_n)^T)_t
//                                              dS = gamma dS_n + Q~^T dO - E~^T dY
// and through the factors: dq = dQ~ e^G, db = dE~ e^G k, dk = dE~ e^G b + dK~ e^-G,
// dw = dY v, dv = dY w, dG = dQ~ Q~ + dE~ E~ - dK~ K~ (+ gamma dgamma on the last
// row), dlog alpha = reverse cumulative sum of dG inside the chunk.  The terms of that sum
// cancel down to a result of the order of alpha, so dG is formed from the bf16 factors the
// products used and gamma dgamma from the state-update part of dK~ (its own accumulator): the
// cancelling pairs then cancel exactly, and dlog alpha keeps its accuracy at any decay.
//
// The only serial dependence is the dS chain.  With W = T E~ and Gm = Diag(gamma):
//   dS = Gm dS_n - W^T K~ (Gm dS_n) + R,   R = Q~^T dO - W^T (P^T dO) = M^T dO,  M = Q~ - P W,
// so the work splits into three launches:
//   1. the tensor-core forward in states mode: S^T (bf16) at every chunk boundary, and from
//      its M group the state-independent factors W^T, K~, gamma, M^T, T and P of every chunk
//      (BwdFactors), formed where the chunk's Q~, E~, K~, T and P already are;
//   2. bwd_chain_tc_kernel, one CTA per (batch, head): the reverse dS chain with dS^T
//      kept in TMEM, R^T = dO^T M formed on the tensor pipe beside it; stores dS_n per chunk;
//   3. bwd_grad_kernel, persistent over the chunks: recomputes U~ from the stored state
//      and produces every gradient of the chunk.
// Chunks whose decay is past the factors' range (kChunkDecayLimit) are flagged by the forward;
// the chain steps them token by token and tok.cu's kernel rewrites their gradients.
// Every product is a bf16 tcgen05 MMA with an fp32 TMEM accumulator, its operands
// in 128-byte swizzled shared-memory tiles (most of them loaded by TMA) or in TMEM.
#include <algorithm>
#include <climits>
#include <cuda.h>
#include <string.h>

#include "gdn2_internal.cuh"
#include "tc_util.cuh"
#include "tok_util.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int D = 128;
constexpr int C = 64;
constexpr int GSTR = kGamStride;  // per-chunk record of gamma: D floats, then the token-mode flag (int)

// ------------------------------------------------------------------ workspace
struct BwdTcLayout {
    size_t coff, states, flist, W, Kt, gam, Mc, Tm, Pm, dSn, scratch, total;
    int tok_blocks;  // blocks of the token-level gradient kernel
};

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Per (batch, head) and chunk: states S^T bf16 (nchunks + 1 entries), W^T bf16 [D][C],
// K~ bf16 [C][D], gamma and the chunk's token-mode flag [GSTR] fp32, M^T bf16 [D][C], T and P
// bf16 [C][C], (Diag(gamma) dS_n)^T bf16 [D][D] (dS_n^T as is for chunks stepped token by
// token).  flist: the count and the list of the chunk tasks that run
// token by token.  Variable length puts chunk_off first; chunk lists are sized by the chunk
// bound.  The token-level gradient kernel's scratch reuses W .. M^T, which only the chain reads
// (one block's scratch at least; past the end of the workspace when that region is smaller).
BwdTcLayout tc_layout(const Problem &p)
{
    const size_t H = p.H, nchunk = chunk_bound(p), nbound = nchunk + p.B;
    BwdTcLayout l;
    size_t off = p.cu_seqlens ? varlen_offsets_bytes(p.B) : 0;
    l.coff = 0;
    l.states = off; off += H * nbound * D * D * 2;
    l.flist = off;  off += round256((1 + H * nchunk) * 4);
    l.W = off;      off += H * nchunk * C * D * 2;
    l.Kt = off;     off += H * nchunk * C * D * 2;
    l.gam = off;    off += round256(H * nchunk * GSTR * 4);
    l.Mc = off;     off += H * nchunk * D * C * 2;
    l.Tm = off;     off += H * nchunk * C * C * 2;
    l.Pm = off;     off += H * nchunk * C * C * 2;
    l.dSn = off;    off += H * nchunk * D * D * 2;
    const size_t blk = tok_grad_block_bytes(p.D), reuse = l.Tm - l.W;
    const size_t fit = blk ? reuse / blk : 0;
    if (fit >= 1) {
        l.tok_blocks = (int)std::min<size_t>(fit, 148);
        l.scratch = l.W;
    } else {
        l.tok_blocks = 1;
        l.scratch = off;
        off += blk;
    }
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
    __nv_bfloat16 *states, *W, *Kt, *Tm, *Pm, *dSn;
    float *gam;          // [chunk][GSTR]: gamma, then the chunk's token-mode flag
    int *flist;          // flist[0]: count of the chunks that run token by token, then their tasks
    __nv_bfloat16 *Mc;  // M^T per chunk, bf16 (R^T = dO^T M)
    __nv_bfloat16 *dq, *dk, *dv, *db, *dw;
    float *dg, *dS0;
    int *status;         // kernel status word (bounded waits that gave up)
};

// ------------------------------------------------------------------ small helpers
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Row t of chunk `ci` of head hh of the sequence whose first token row is `bos`.
__device__ __forceinline__ size_t tok_off(const BwdTcArgs &a, int bos, int hh, int ci, int t)
{
    return (((size_t)bos + (size_t)ci * C + t) * a.H + hh) * a.din;
}

// The chunk a block of the chunk-parallel kernels works on: blockIdx.y is the head,
// blockIdx.x the chunk over all sequences (blocks past the last chunk have nothing to do).
__device__ __forceinline__ bool chunk_ref_at(const BwdTcArgs &a, int gc, int h, ChunkRef &r)
{
    return chunk_at(a.pr, gc, h, r);
}

// Decay folding of the gradient kernel: thread (channel pair cp, token group g8) owns channels
// 2 cp, 2 cp + 1 and tokens 8 g8 .. 8 g8 + 7 (64 x 8 = 512 threads).  e^G and e^-G of its 16
// values (G the inclusive cumulative sum of log alpha over the chunk) with one exponential per
// value: alpha = e^g, then e^G as a running product forwards from the token group's start and
// e^-G as one backwards from its end.  The group totals go through sTot ([8][D] fp32); `total`
// is G at the chunk end.  Contains a __syncthreads.
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

// barrier over `count` threads (id 0 is __syncthreads)
__device__ __forceinline__ void named_bar(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Bounded wait on an mbarrier phase.  A wait that gives up records the timeout in the status
// word and in the block's abort flag; once that is set every later wait of the block returns at
// once, so a block that lost a transfer ends (with garbage) after one wait limit instead of one
// limit per remaining wait.
__device__ __forceinline__ void wait_or_abort(uint64_t *bar, uint32_t parity, int *status, volatile int *abort)
{
    if (*abort) return;
    if (!tc::mbar_wait(bar, parity)) {
        *abort = 1;
        atomicExch(status, kStatusTimeout);
    }
}

// ================================================================== 3. chain on the tensor cores
// One CTA per (batch, head).  dS^T (d_v x d_k, fp32) lives in TMEM as an MMA accumulator, one
// row per lane.  Per chunk, newest first:
//   read dS_n^T and scale its d_k columns: (Gm dS_n)^T to global in bf16 (the gradient kernel
//     takes it as it is) and to TMEM (A operand); (Gm dS_n)^T + R^T back into the accumulator;
//   Z^T = (Gm dS_n)^T K~^T               M d_v, N 64, K d_k   (A from TMEM)
//   dS^T += (-Z^T) W                     M d_v, N d_k, K 64   (A = -Z^T bf16 from TMEM)
// with R^T = dO^T M formed a chunk ahead on the tensor pipe.  K~, W^T, dO, M^T and gamma arrive
// by TMA in a three-stage ring, two chunks ahead.
namespace chain_tc {
constexpr uint32_t ST_K = 0;          // K~ [64][128] (two 8 KiB atoms)
constexpr uint32_t ST_W = 16384;      // W^T [128 d_k][64 tokens] (one 16 KiB atom)
constexpr uint32_t ST_DO = 32768;     // dO [64 tokens][128 d_v] (two 8 KiB atoms)
constexpr uint32_t ST_M = 49152;      // M^T [128 d_k][64 tokens] (one 16 KiB atom)
constexpr uint32_t ST_G = 65536;      // gamma [128] fp32, then the token-mode flag
constexpr uint32_t STAGE = 66560;     // 65 KiB, 1024-aligned
constexpr int kStages = 3;
constexpr uint32_t SMEM = kStages * STAGE + 1024;
constexpr uint32_t STAGE_BYTES = 16384 + 16384 + 16384 + 16384 + GSTR * 4;
constexpr uint32_t TM_S = 0, TM_SB = 128, TM_Z = 192, TM_ZB = 256, TM_R = 288, TM_COLS = 512;
constexpr uint32_t IDESC_Z = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t IDESC_R = tc::idesc_bf16(128, 128, 1, 0);  // R^T = dO^T M: A (dO^T) MN-major
constexpr int kThreads = 256;
}  // namespace chain_tc

struct ChainMaps {
    CUtensorMap kt, wt, mt, dO;
};

__global__ void __launch_bounds__(chain_tc::kThreads, 1)
bwd_chain_tc_kernel(const __grid_constant__ ChainMaps maps, const BwdTcArgs a)
{
    using namespace chain_tc;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_full[kStages], bar_z, bar_s, bar_r;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, n = bh / a.H, hh = bh % a.H;
    const SeqSpan sp = seq_span(a.pr, n);
    if (sp.len < 0) return;  // invalid cu_seqlens (reported by the offsets pass)
    const int nc = seq_chunks(sp.len);
    // TMEM access: warp w reads lanes 32 (w & 3) .. + 31 (rows of dS^T) and column half w >> 2
    const int quarter = warp & 3, half = warp >> 2, row = 32 * quarter + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bar_full[s], 1);
        mbar_init(&bar_z, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_r, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    // chunk ci's K~, W^T, dO, M^T, gamma into stage s
    auto load = [&](int ci, int s) {
        const size_t cidx = chunk_slot(a.pr, n, hh, nc, ci);
        uint8_t *st = sm + s * STAGE;
        mbar_expect_tx(&bar_full[s], STAGE_BYTES);
        for (int at = 0; at < 2; ++at) {
            tma_load_2d(st + ST_K + at * 8192, &maps.kt, at * 64, (int)(cidx * C), &bar_full[s]);
            tma_load_3d(st + ST_DO + at * 8192, &maps.dO, at * 64, hh, sp.bos + ci * C, &bar_full[s]);
        }
        tma_load_2d(st + ST_W, &maps.wt, 0, (int)(cidx * D), &bar_full[s]);
        tma_load_2d(st + ST_M, &maps.mt, 0, (int)(cidx * D), &bar_full[s]);
        bulk_load(st + ST_G, a.gam + cidx * GSTR, GSTR * 4, &bar_full[s]);
    };
    // R^T = dO^T M of the chunk in stage s (state-independent) into TM_R; thread 0, after the
    // stage has landed and TM_R's last value was read
    auto issue_r = [&](int s, uint32_t par) {
        wait_or_abort(&bar_full[s], par, a.status, &s_abort);
        tc_fence_after();
        const uint32_t sb = smem_u32(sm + s * STAGE);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_R, sdesc_sw128(sb + ST_DO + ks * 2048, 8192, 1024), sdesc_sw128(sb + ST_M + ks * 32, 16, 1024),
                   IDESC_R, ks > 0);
        mma_commit(&bar_r);
    };
    if (tid == 0) {
        for (int u = 0; u < 2 && u < nc; ++u) load(nc - 1 - u, u);
        if (nc > 0) issue_r(0, 0);
    }
    // dS^T from dS_T (stored [c][j]: dS^T[j][c] = dS_T[c][j]); this thread: row j, 64 columns
    {
        uint32_t r[32];
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int c = 64 * half + 32 * h2 + u;
                r[u] = __float_as_uint((a.dS_T && c < a.din && row < a.din)
                                           ? a.dS_T[((size_t)bh * a.din + c) * a.din + row] : 0.f);
            }
            tmem_st32(tmem + TM_S + 64 * half + 32 * h2 + lane_off, r);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t ph = 0;  // phase of bar_z and bar_s (chunks stepped token by token issue no product)
    for (int it = 0; it < nc; ++it) {
        const int ci = nc - 1 - it, s = it % kStages;
        const uint32_t par = (uint32_t)(it / kStages) & 1u;
        const size_t cidx = chunk_slot(a.pr, n, hh, nc, ci);
        const uint8_t *st = sm + s * STAGE;
        if (tid == 0 && ci - 2 >= 0) load(ci - 2, (it + 2) % kStages);  // stage freed by step it - 1
        wait_or_abort(&bar_full[s], par, a.status, &s_abort);
        wait_or_abort(&bar_r, (uint32_t)it & 1u, a.status, &s_abort);  // this chunk's R^T
        tc_fence_after();
        // the next chunk's R^T, issued right after this chunk's Z^T (products below) or its tokens
        auto issue_next_r = [&]() {
            if (tid == 0 && ci >= 1) issue_r((it + 1) % kStages, (uint32_t)((it + 1) / kStages) & 1u);
        };
        if (reinterpret_cast<const int *>(st + ST_G)[D]) {
            // ---- a chunk whose decay is too strong for the factors: dS^T to registers (this
            //      thread: row `row`, columns 64 half ..), its bf16 copy to global as dS_n, then the
            //      reverse recurrence token by token; records and exchange buffers over this
            //      stage's tiles, which are not needed
            float dsr[64];
            __nv_bfloat16 *dsn = a.dSn + cidx * D * D + (size_t)row * D + 64 * half;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t r[32];
                tmem_ld32(tmem + TM_S + 64 * half + 32 * h2 + lane_off, r);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) dsr[32 * h2 + u] = __uint_as_float(r[u]);
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *reinterpret_cast<uint4 *>(dsn + 32 * h2 + 8 * m) =
                        make_uint4(pack_bf16x2(dsr[32 * h2 + 8 * m], dsr[32 * h2 + 8 * m + 1]),
                                   pack_bf16x2(dsr[32 * h2 + 8 * m + 2], dsr[32 * h2 + 8 * m + 3]),
                                   pack_bf16x2(dsr[32 * h2 + 8 * m + 4], dsr[32 * h2 + 8 * m + 5]),
                                   pack_bf16x2(dsr[32 * h2 + 8 * m + 6], dsr[32 * h2 + 8 * m + 7]));
            }
            uint8_t *stw = sm + s * STAGE;
            tok::Rec<D> *recs = reinterpret_cast<tok::Rec<D> *>(stw);
            float *xch = reinterpret_cast<float *>(stw + 3 * sizeof(tok::Rec<D>));
            const int L = min(C, sp.len - ci * C);
            const size_t row0 = (size_t)sp.bos + (size_t)ci * C;
            auto fill = [&](int t, tok::Rec<D> &rc) {
                if (tid < D) {
                    const int c = tid;
                    float qv = 0.f, kv = 0.f, bv = 0.f, gv = 0.f;
                    if (c < a.din) {
                        const size_t off = ((row0 + t) * a.H + hh) * a.din + c;
                        qv = __bfloat162float(a.q[off]);
                        kv = __bfloat162float(a.k[off]);
                        bv = __bfloat162float(a.pr.bw_scalar ? a.b[(row0 + t) * a.H + hh] : a.b[off]);
                        gv = a.pr.g_scalar ? a.g[(row0 + t) * a.H + hh] : a.g[off];
                    }
                    rc.q[c] = qv;
                    rc.k[c] = kv;
                    rc.e[c] = bv * kv;
                    rc.a[c] = expf(gv);
                } else {
                    const int jj = tid - D;
                    rc.x[jj] = jj < a.din ? __bfloat162float(a.dO[((row0 + t) * a.H + hh) * a.din + jj]) : 0.f;
                }
            };
            tok::chain_tokens<D>(dsr, L - 1, L, recs, xch, row, half, 1, fill);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t r[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(dsr[32 * h2 + u]);
                tmem_st32(tmem + TM_S + 64 * half + 32 * h2 + lane_off, r);
            }
            tmem_wait_st();
            fence_proxy_async_smem();  // the stage is refilled by TMA later
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            issue_next_r();
            continue;
        }
        // ---- (Gm dS_n)^T: bf16 to global and to TMEM; (Gm dS_n)^T + R^T back into the accumulator
        {
            const float *gam = reinterpret_cast<const float *>(st + ST_G) + 64 * half;
            __nv_bfloat16 *dsn = a.dSn + cidx * D * D + (size_t)row * D + 64 * half;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t r[32], pk[16];
                tmem_ld32(tmem + TM_S + 64 * half + 32 * h2 + lane_off, r);
                uint32_t rr[32];  // R^T row `row`, columns 64 half + 32 h2 ..
                tmem_ld32(tmem + TM_R + 64 * half + 32 * h2 + lane_off, rr);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; u += 2) {
                    const float2 g2 = *reinterpret_cast<const float2 *>(gam + 32 * h2 + u);
                    const float s0 = __uint_as_float(r[u]) * g2.x, s1 = __uint_as_float(r[u + 1]) * g2.y;
                    pk[u >> 1] = pack_bf16x2(s0, s1);
                    r[u] = __float_as_uint(s0 + __uint_as_float(rr[u]));
                    r[u + 1] = __float_as_uint(s1 + __uint_as_float(rr[u + 1]));
                }
                tmem_st16(tmem + TM_SB + 32 * half + 16 * h2 + lane_off, pk);
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *reinterpret_cast<uint4 *>(dsn + 32 * h2 + 8 * m) =
                        make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
                tmem_st32(tmem + TM_S + 64 * half + 32 * h2 + lane_off, r);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        // ---- Z^T = (Gm dS_n)^T K~^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t kb = smem_u32(st + ST_K);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ts(tmem + TM_Z, tmem + TM_SB + 8 * ks, sdesc_sw128(kb + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024),
                       IDESC_Z, ks > 0);
            mma_commit(&bar_z);
        }
        issue_next_r();  // runs on the tensor pipe while Z^T is read back
        wait_or_abort(&bar_z, ph, a.status, &s_abort);
        tc_fence_after();
        {  // -Z^T -> bf16 A operand: warp = lane quarter x 32 columns
            uint32_t r[32], pk[16];
            tmem_ld32(tmem + TM_Z + 32 * half + lane_off, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(-__uint_as_float(r[2 * e]), -__uint_as_float(r[2 * e + 1]));
            tmem_st16(tmem + TM_ZB + 16 * half + lane_off, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        // ---- dS^T += (-Z^T) W
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wb = smem_u32(st + ST_W);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ts(tmem + TM_S, tmem + TM_ZB + 8 * ks, sdesc_sw128(wb + ks * 32, 16, 1024), IDESC_S, 1);
            mma_commit(&bar_s);
        }
        wait_or_abort(&bar_s, ph, a.status, &s_abort);
        tc_fence_after();
        ph ^= 1;
    }
    // dS0 = dS (stored [c][j])
    {
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t r[32];
            tmem_ld32(tmem + TM_S + 64 * half + 32 * h2 + lane_off, r);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int c = 64 * half + 32 * h2 + u;
                if (c < a.din && row < a.din) a.dS0[((size_t)bh * a.din + c) * a.din + row] = __uint_as_float(r[u]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ================================================================== 4. gradients on the tensor cores
// Persistent: one 512-thread CTA per multiprocessor loops over the (chunk, head) tasks, loading
// the next task's tiles as this task's regions free up.  Every product runs transposed, so that
// its M side is a 128-wide feature dimension (d_v or d_k, or the two stacked 64-token tiles of
// [dP; dA]) and its TMEM accumulator holds one feature row per lane (Gm = Diag(gamma)):
//   Y^T  = X^T - S^T E~^T              M d_v, N 64, K d_k           -> bf16 A operand in TMEM
//   dU~^T = dO^T P + (Gm dS_n)^T K~^T  M d_v, N 64, K 64 + d_k      -> bf16 A operand in TMEM
//   U~^T = Y^T T^T                     A from TMEM, K 64            -> U~ tile [s][d_v]
//   dY^T = dU~^T T                     A from TMEM, K 64            -> dv, dw, -dY tile
//   [dP; dA] = [dO; -dY] U~^T          M 2 x 64 tokens, N 64, K d_v -> masked bf16 tile
//   [dQ~^T | dE~^T] = S [dO; -dY]^T + K~^T [dP; dA]^T     M d_k, N 128, K d_v + 64
//   dK~^T = [(Gm dS_n) U~^T] + [Q~^T dP + E~^T dA]        M d_k, N 64, K d_v | 128 (two accumulators)
// The tiles arrive by TMA in 128-byte swizzled atoms; a [rows][128] tile is two column atoms
// of [rows][64].  The factor chain reads dQ~^T, dE~^T, dK~^T straight from TMEM: a thread
// owns one channel of d_k (its TMEM lane) and 16 tokens (its column block).
namespace grad_tc {
constexpr uint32_t RQ = 0;        // q -> Q~ [64][128]
constexpr uint32_t RK = 16384;    // k -> K~
constexpr uint32_t RB = 32768;    // b -> E~
constexpr uint32_t GG = 49152;    // log alpha fp32 [64][128]: four 8 KiB boxes of 32 channels
constexpr uint32_t SS = 81920;    // S^T [128][128] (atoms 16 KiB apart); after the S products: raw q, k
constexpr uint32_t DS = 114688;   // (Gm dS_n)^T, as the chain stored it; after its products: raw b
constexpr uint32_t DY = 147456;   // [dO; -dY] [128][128]: atom a = dO rows 0-63 then -dY rows 64-127
constexpr uint32_t TT = 180224;   // T [64][64]; after dY: U~ [64][128] over T and P; after U~'s
constexpr uint32_t PP = 188416;   //   products: [dP; dA] [128][64]
constexpr uint32_t UU = TT;
constexpr uint32_t PA = TT;
constexpr uint32_t VV = 196608;   // v, then dw (full chunks: stored from here by TMA)
constexpr uint32_t WW = 212992;   // w, then dv
constexpr uint32_t DGF = 229376;  // gamma dgamma [D] fp32
// scalar erase and write gates: b_t and w_t of the chunk [2][64] bf16, and the four lane quarters'
// partial sums of dw_t [4][64] fp32 (those of db_t go to the first half of DS, unused then)
constexpr uint32_t SBW = DGF + D * 4;
constexpr uint32_t SDW = SBW + 256;
constexpr uint32_t USED = SDW + 1024;
constexpr uint32_t SMEM = USED + 1024;  // slack for the 1024-byte alignment
// scratch inside the -dY rows (free until dY is read back), and in DS's second half (free once
// (Gm dS_n)^T's products are done) for the factor chain
constexpr uint32_t SC_TOT = DY + 8192;           // decay group totals [8][D] fp32
constexpr uint32_t SC_DGP = DY + 16384 + 8192;   // gamma dgamma partials [16][D]
constexpr uint32_t SC_FIN = DS + 16384;          // factor chain: group sums [8][D], then [4][D] twice
// scalar decay: no log alpha tile; its region holds g_t of the chunk [64] fp32 and the four lane
// quarters' partial sums of dlog alpha_t [4][64] fp32
constexpr uint32_t SGT = GG;
constexpr uint32_t SDG = GG + 256;
// full chunks stage dq, dk, db over the reloaded raw q, k, b and dg over v, w for the TMA stores
// TMEM columns
constexpr uint32_t TM_Y = 0, TM_DU = 64, TM_YB = 128, TM_DUB = 160, TM_U = 192, TM_DY = 256, TM_PA = 320;
constexpr uint32_t TM_DQE = 384, TM_DK = 0, TM_DKU = 64, TM_COLS = 512;  // TM_DKU: dK~'s state-update part
constexpr uint32_t IDESC_KK = tc::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_MM = tc::idesc_bf16(128, 64, 1, 1);
constexpr uint32_t IDESC_KM = tc::idesc_bf16(128, 64, 0, 1);
constexpr uint32_t IDESC_MK = tc::idesc_bf16(128, 64, 1, 0);
constexpr uint32_t IDESC_MK2 = tc::idesc_bf16(128, 128, 1, 0);
constexpr int kThreads = 512;
}  // namespace grad_tc

struct GradMaps {
    CUtensorMap q, k, b, v, w, dO, g, st, dsn, tm, pm;  // loads
    CUtensorMap dq, dk, db, dv, dw, dg;                 // stores of full chunks
};


// Sums of 16 per-lane values over the 32 lanes of a warp, by halving exchanges: on return lane
// 2 i (and 2 i + 1) holds the total of value i in v[0].
__device__ __forceinline__ void warp_sum16(float (&v)[16], int lane)
{
#pragma unroll
    for (int m = 16, n = 8; m >= 2; m >>= 1, n >>= 1) {
        const bool hi = lane & m;
#pragma unroll
        for (int j = 0; j < n; ++j) {
            const float give = hi ? v[j] : v[j + n];
            v[j] = (hi ? v[j + n] : v[j]) + __shfl_xor_sync(0xffffffffu, give, m);
        }
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// bf16 element (t, c) of a [rows][128] tile whose two column atoms are `astride` bytes apart
__device__ __forceinline__ uint32_t tile_off(int t, int c, uint32_t astride)
{
    return (uint32_t)(c >> 6) * astride + tc::sw128(t, (c & 63) * 2);
}
__device__ __forceinline__ float ld_bf(const uint8_t *p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p)); }
__device__ __forceinline__ void st_bf(uint8_t *p, float x) { *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(x); }

// kSG: the erase and write gates are one value per (token, head) ([rows, H]): per-token tables
// replace the b and w tiles, and db_t, dw_t are the per-channel gradients summed over the
// channels (over the 32 lanes of a warp, then over the four lane quarters).
// kGS: the decay is one value per (token, head): g_t is read per token (registers for the
// folding, a table for the factor chain) instead of as a tile, and dlog alpha_t is the
// per-channel gradient summed over the channels in the same way.
template <bool kSG, bool kGS>
__global__ void __launch_bounds__(grad_tc::kThreads, 1)
bwd_grad_kernel(const __grid_constant__ GradMaps maps, const BwdTcArgs a)
{
    using namespace grad_tc;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_in0, bar_in1, bar_in2, bar_in3, bar_a, bar_b, bar_c, bar_d;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sb = smem_u32(sm);
    // TMEM access: warp w reads lanes 32 (w & 3) .. + 31; column block w >> 2 (16 columns)
    const int quarter = warp & 3, cg = warp >> 2, row = 32 * quarter + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
    // the block's tasks: blockIdx.x, + gridDim.x, ... over (chunk, head); chunks past a
    // sequence's end are skipped
    const int nchb = (int)chunk_bound(a.pr), ntask = nchb * a.H;
    auto find_task = [&](int from, ChunkRef &r) -> int {
        for (int t = from; t < ntask; t += gridDim.x)
            if (chunk_ref_at(a, t % nchb, t / nchb, r)) return t;
        return -1;
    };
    if (tid == 0) {
        mbar_init(&bar_in0, 1);
        mbar_init(&bar_in1, 1);
        mbar_init(&bar_in2, 1);
        mbar_init(&bar_in3, 1);
        mbar_init(&bar_a, 1);
        mbar_init(&bar_b, 1);
        mbar_init(&bar_c, 1);
        mbar_init(&bar_d, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    // A task's tile loads, in four parts as their regions free up: part 0 q, k, b, dO, T, P (and
    // the byte counts of bar_in0 and bar_in1) and part 1 log alpha (per channel), from warp 0 during the task
    // before; part 2 S^T and dS_n^T from warp 1 at the end of the task before, once the staged
    // dq, dk, db have left their tiles; part 3 v and w (bar_in3) from warp 1 during this task's
    // decay folding, once the staged dg has left its tiles.
    auto issue = [&](int part, const ChunkRef &r) {
        const int yy = r.sp.bos + r.ci * C, h = r.h, at = lane & 1;
        if (part == 0) {
            if (lane == 0) {
                mbar_expect_tx(&bar_in0, ((kSG ? 4 : 6) + (kGS ? 0 : 4)) * 8192);
                mbar_expect_tx(&bar_in1, 6 * 16384);
            }
            __syncwarp();
            if (kSG && (lane == 4 || lane == 5)) {  // b comes from the per-token table
            } else if (lane < 6) {
                const int which = lane >> 1;
                const CUtensorMap *mp = which == 0 ? &maps.q : which == 1 ? &maps.k : &maps.b;
                tma_load_3d(sm + RQ + which * 16384 + at * 8192, mp, at * 64, h, yy, &bar_in0);
            } else if (lane < 8) {
                tma_load_3d(sm + DY + at * 16384, &maps.dO, at * 64, h, yy, &bar_in1);
            } else if (lane < 10) {
                tma_load_2d(sm + (lane == 8 ? TT : PP), lane == 8 ? &maps.tm : &maps.pm, 0, (int)(r.cidx * C), &bar_in1);
            }
        } else if (part == 1) {
            if (!kGS && lane < 4) tma_load_3d(sm + GG + lane * 8192, &maps.g, lane * 32, h, yy, &bar_in0);
        } else if (part == 2) {
            const int sl = (int)(bound_slot(a.pr, r.n, r.h, r.nch, r.ci) * D);
            if (lane < 2) tma_load_2d(sm + SS + at * 16384, &maps.st, at * 64, sl, &bar_in1);
            else if (lane < 4) tma_load_2d(sm + DS + at * 16384, &maps.dsn, at * 64, (int)(r.cidx * D), &bar_in1);
        } else {
            if (lane == 0) mbar_expect_tx(&bar_in3, (kSG ? 2 : 4) * 8192);
            __syncwarp();
            if (lane < 2) tma_load_3d(sm + VV + at * 8192, &maps.v, at * 64, h, yy, &bar_in3);
            else if (!kSG && lane < 4) tma_load_3d(sm + WW + at * 8192, &maps.w, at * 64, h, yy, &bar_in3);
        }
    };
    ChunkRef cr;
    int task = find_task(blockIdx.x, cr);
    if (warp == 0 && task >= 0) {
        issue(0, cr);
        issue(1, cr);
        issue(2, cr);
        issue(3, cr);
    }
    uint32_t ph = 0;  // parity of this task's barrier phases
    bool pend3 = false;  // warp 1: this task's v, w are still to be loaded
    while (task >= 0) {
    ChunkRef nx;
    const int next = find_task(task + gridDim.x, nx);
    const int ci = cr.ci, hh = cr.h, bb = cr.sp.bos;  // bb: the sequence's first token row
    const int L = min(C, cr.sp.len - ci * C);
    const size_t slot = bound_slot(a.pr, cr.n, hh, cr.nch, ci);
    const int y = bb + ci * C;
    const bool full = L == C;  // full chunks store their gradients by TMA from shared memory
    // the chunk-start state (for gamma dgamma's part gamma rowsum(dS_n . S)), in flight during the folding
    const int dch = tid & 15;
    uint4 ssv[4];
    {
        const __nv_bfloat16 *st_n = a.states + slot * D * D;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            ssv[u] = __ldg(reinterpret_cast<const uint4 *>(st_n + (size_t)((tid >> 4) + 32 * u) * D + 8 * dch));
    }
    float gsv[8];  // kGS: g_t of the folding's 8 tokens (tokens 8 (tid >> 6) ..), in flight likewise
    if (kGS) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * (tid >> 6) + i;
            gsv[i] = t < L ? __ldg(a.g + ((size_t)y + t) * a.H + hh) : 0.f;
        }
    }
    __nv_bfloat16 *const sBt = reinterpret_cast<__nv_bfloat16 *>(sm + SBW), *const sWt = sBt + 64;
    if (kSG && tid < 128) {  // this chunk's b_t (threads 0-63) and w_t (64-127); seen after the folding's first barrier
        const int t = tid & 63;
        const __nv_bfloat16 *src = tid < 64 ? a.b : a.w;
        (tid < 64 ? sBt : sWt)[t] = t < L ? src[((size_t)y + t) * a.H + hh] : __float2bfloat16_rn(0.f);
    }

    // ---- decay folding in place: thread (channel pair cp, token group g8 of 8)
    const int cp = tid & 63, g8 = tid >> 6;
    float *sTot = reinterpret_cast<float *>(sm + SC_TOT);
    wait_or_abort(&bar_in0, ph, a.status, &s_abort);
    {
        const bool ch_ok = 2 * cp < a.din;
        float2 gl[8], eG[8], emG[8], tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * g8 + i;
            if (kGS)
                gl[i] = (t < L && ch_ok) ? make_float2(gsv[i], gsv[i]) : make_float2(0.f, 0.f);
            else
                gl[i] = (t < L && ch_ok)
                            ? *reinterpret_cast<const float2 *>(sm + GG + (cp >> 4) * 8192 + sw128(t, (cp & 15) * 8))
                            : make_float2(0.f, 0.f);
        }
        if (kGS && cp == 0) {  // the factor chain's table of g_t (the last task read it before its end)
#pragma unroll
            for (int i = 0; i < 8; ++i) reinterpret_cast<float *>(sm + SGT)[8 * g8 + i] = gsv[i];
        }
        decay_pair8(gl, eG, emG, tot, cp, g8, sTot);
        if (warp == 1 && pend3) {  // the last task's dg has left v, w's tiles by now: this task's v, w
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
            issue(3, cr);
            pend3 = false;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * g8 + i;
            const uint32_t off = (cp >> 5) * 8192 + sw128(t, (cp & 31) * 4);
            uint32_t *pq = reinterpret_cast<uint32_t *>(sm + RQ + off);
            uint32_t *pk = reinterpret_cast<uint32_t *>(sm + RK + off);
            uint32_t *pe = reinterpret_cast<uint32_t *>(sm + RB + off);
            uint32_t q2 = *pq, k2 = *pk, b2;
            if (kSG) {
                const uint32_t b16 = (uint32_t)__bfloat16_as_ushort(sBt[t]);
                b2 = b16 | (b16 << 16);
            } else {
                b2 = *pe;
            }
            if (t >= L) { q2 = 0u; k2 = 0u; b2 = 0u; }
            const float k0 = bf_lo(k2), k1 = bf_hi(k2);
            *pq = pack_bf16x2(bf_lo(q2) * eG[i].x, bf_hi(q2) * eG[i].y);
            *pe = pack_bf16x2(bf_lo(b2) * k0 * eG[i].x, bf_hi(b2) * k1 * eG[i].y);
            *pk = pack_bf16x2(k0 * emG[i].x, k1 * emG[i].y);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    // ---- Y^T = S^T E~^T (into TM_Y; X is added at the read-back)
    wait_or_abort(&bar_in1, ph, a.status, &s_abort);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_Y, sdesc_sw128(sb + SS + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                   sdesc_sw128(sb + RB + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), IDESC_KK, ks > 0);
    }
    // ---- gamma dgamma's part gamma rowsum(dS_n . S) = rowsum((Gm dS_n) . S), from the column sums
    //      of (Gm dS_n)^T . S^T (the chain stored dS_n already scaled by gamma)
    {
        float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = (tid >> 4) + 32 * u;
            const uint4 dv4 = *reinterpret_cast<const uint4 *>(sm + DS + (dch >> 3) * 16384 + sw128(j, (dch & 7) * 16));
            const uint4 sv4 = ssv[u];
            const uint32_t dw[4] = {dv4.x, dv4.y, dv4.z, dv4.w}, sw[4] = {sv4.x, sv4.y, sv4.z, sv4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                part[2 * e] += bf_lo(dw[e]) * bf_lo(sw[e]);
                part[2 * e + 1] += bf_hi(dw[e]) * bf_hi(sw[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) part[e] += __shfl_xor_sync(0xffffffffu, part[e], 16);
        float *sDgp = reinterpret_cast<float *>(sm + SC_DGP);
        if (lane < 16) {
#pragma unroll
            for (int e = 0; e < 8; ++e) sDgp[warp * D + 8 * dch + e] = part[e];
        }
        if (L < C) {  // dO rows past the sequence end belong to the next one: zero them
            for (int idx = tid; idx < (C - L) * 16; idx += kThreads) {
                const int t = L + (idx >> 4), c = idx & 15;
                *reinterpret_cast<uint4 *>(sm + DY + (c >> 3) * 16384 + sw128(t, (c & 7) * 16)) = make_uint4(0, 0, 0, 0);
            }
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < D) {
        const float *sDgp = reinterpret_cast<const float *>(sm + SC_DGP);
        float s = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) s += sDgp[u * D + tid];
        reinterpret_cast<float *>(sm + DGF)[tid] = s;
    }
    // ---- dU~^T = dO^T P + (Gm dS_n)^T K~^T
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_DU, sdesc_sw128(sb + DY + ks * 2048, 16384, 1024), sdesc_sw128(sb + PP + ks * 2048, 8192, 1024),
                   IDESC_MM, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_DU, sdesc_sw128(sb + DS + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                   sdesc_sw128(sb + RK + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), IDESC_KK, 1);
        mma_commit(&bar_a);
    }
    // ---- read back: Y^T = X^T - acc and dU~^T, as bf16 A operands (lane = d_v, 16 tokens per warp)
    wait_or_abort(&bar_a, ph, a.status, &s_abort);
    wait_or_abort(&bar_in3, ph, a.status, &s_abort);  // v, w
    tc_fence_after();
    {
        uint32_t r[16], pk[8];
        tmem_ld16(tmem + TM_Y + 16 * cg + lane_off, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float y2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = 16 * cg + 2 * e + h;
                const uint32_t so = tile_off(t, row, 8192);
                const float wt = kSG ? __bfloat162float(sWt[t]) : ld_bf(sm + WW + so);
                const float x = (t < L) ? ld_bf(sm + VV + so) * wt : 0.f;
                y2[h] = x - __uint_as_float(r[2 * e + h]);
            }
            pk[e] = pack_bf16x2(y2[0], y2[1]);
        }
        tmem_st8(tmem + TM_YB + 8 * cg + lane_off, pk);
        tmem_ld16(tmem + TM_DU + 16 * cg + lane_off, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
        tmem_st8(tmem + TM_DUB + 8 * cg + lane_off, pk);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    // ---- U~^T = Y^T T^T, dY^T = dU~^T T
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + TM_U, tmem + TM_YB + 8 * ks, sdesc_sw128(sb + TT + ks * 32, 16, 1024), IDESC_KK, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + TM_DY, tmem + TM_DUB + 8 * ks, sdesc_sw128(sb + TT + ks * 2048, 8192, 1024), IDESC_KM, ks > 0);
        mma_commit(&bar_b);
    }
    wait_or_abort(&bar_b, ph, a.status, &s_abort);
    tc_fence_after();
    // ---- read back: U~ tile [s][d_v] (over T and P, both consumed); dv = dY w, dw = dY v (full
    //      chunks: over w and v); -dY into rows 64-127 of [dO; -dY]
    {
        uint32_t r[16];
        tmem_ld16(tmem + TM_U + 16 * cg + lane_off, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) st_bf(sm + UU + tile_off(16 * cg + i, row, 8192), __uint_as_float(r[i]));
        tmem_ld16(tmem + TM_DY + 16 * cg + lane_off, r);
        tmem_wait_ld();
        const bool ch_ok = row < a.din;
        float pdw[16];  // kSG: this channel's share of dw_t
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = 16 * cg + i;
            const float d = __uint_as_float(r[i]);
            st_bf(sm + DY + tile_off(64 + t, row, 16384), -d);
            const uint32_t so = tile_off(t, row, 8192);
            const float wv = kSG ? __bfloat162float(sWt[t]) : ld_bf(sm + WW + so), vv = ld_bf(sm + VV + so);
            pdw[i] = t < L ? d * vv : 0.f;
            if (full) {
                st_bf(sm + WW + so, d * wv);
                if (!kSG) st_bf(sm + VV + so, d * vv);
            } else if (t < L && ch_ok) {
                const size_t go = tok_off(a, bb, hh, ci, t) + row;
                a.dv[go] = __float2bfloat16_rn(d * wv);
                if (!kSG) a.dw[go] = __float2bfloat16_rn(d * vv);
            }
        }
        if (kSG) {  // sum over this lane quarter's 32 channels; the quarters add up below
            warp_sum16(pdw, lane);
            if (!(lane & 1)) reinterpret_cast<float *>(sm + SDW)[quarter * 64 + 16 * cg + (lane >> 1)] = pdw[0];
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- [dP; dA] = [dO; -dY] U~^T;  [dQ~^T | dE~^T] = S [dO; -dY]^T;  dK~^T = (Gm dS_n) U~^T
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_PA, sdesc_sw128(sb + DY + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                   sdesc_sw128(sb + UU + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), IDESC_KK, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_DQE, sdesc_sw128(sb + SS + ks * 2048, 16384, 1024),
                   sdesc_sw128(sb + DY + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), IDESC_MK2, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_DKU, sdesc_sw128(sb + DS + ks * 2048, 16384, 1024),
                   sdesc_sw128(sb + UU + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), IDESC_MK, ks > 0);
        mma_commit(&bar_c);
    }
    if (tid == 32 && full) {  // dv, dw by TMA (thread 32 owns every bulk store of the block)
        for (int at = 0; at < a.din / 64; ++at) {
            tma_store_3d(&maps.dv, sm + WW + at * 8192, at * 64, hh, y);
            if (!kSG) tma_store_3d(&maps.dw, sm + VV + at * 8192, at * 64, hh, y);
        }
        bulk_commit();
    }
    if (kSG && tid < 64 && tid < L) {  // dw_t: the four lane quarters' sums
        const float *p4 = reinterpret_cast<const float *>(sm + SDW);
        a.dw[((size_t)y + tid) * a.H + hh] = __float2bfloat16_rn(p4[tid] + p4[64 + tid] + p4[128 + tid] + p4[192 + tid]);
    }
    wait_or_abort(&bar_c, ph, a.status, &s_abort);
    tc_fence_after();
    if (tid == 0) {  // S^T and (Gm dS_n)^T are consumed: the raw q, k, b for the factor chain
        mbar_expect_tx(&bar_in2, (kSG ? 4 : 6) * 8192);
        for (int at = 0; at < 2; ++at) {
            tma_load_3d(sm + SS + at * 8192, &maps.q, at * 64, hh, y, &bar_in2);
            tma_load_3d(sm + SS + 16384 + at * 8192, &maps.k, at * 64, hh, y, &bar_in2);
            if (!kSG) tma_load_3d(sm + DS + at * 8192, &maps.b, at * 64, hh, y, &bar_in2);
        }
    }
    {  // [dP; dA] -> bf16 tile [128][64] (over U~): dP lower incl., dA strictly lower
        uint32_t r[16], w8[8];
        tmem_ld16(tmem + TM_PA + 16 * cg + lane_off, r);
        tmem_wait_ld();
        const int t = row & 63, strict = row >> 6;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int s0 = 16 * cg + 2 * e;
            w8[e] = pack_bf16x2((s0 + strict <= t) ? __uint_as_float(r[2 * e]) : 0.f,
                                (s0 + 1 + strict <= t) ? __uint_as_float(r[2 * e + 1]) : 0.f);
        }
        *reinterpret_cast<uint4 *>(sm + PA + sw128(row, 32 * cg)) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        *reinterpret_cast<uint4 *>(sm + PA + sw128(row, 32 * cg + 16)) = make_uint4(w8[4], w8[5], w8[6], w8[7]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- [dQ~^T | dE~^T] += K~^T [dP; dA]^T;  dK~^T += Q~^T dP + E~^T dA
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_DQE, sdesc_sw128(sb + RK + ks * 2048, 8192, 1024), sdesc_sw128(sb + PA + ks * 32, 16, 1024),
                   IDESC_MK2, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_DK, sdesc_sw128(sb + RQ + ks * 2048, 8192, 1024), sdesc_sw128(sb + PA + ks * 2048, 8192, 1024),
                   IDESC_MM, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem + TM_DK, sdesc_sw128(sb + RB + ks * 2048, 8192, 1024),
                   sdesc_sw128(sb + PA + 8192 + ks * 2048, 8192, 1024), IDESC_MM, 1);
        mma_commit(&bar_d);
    }
    // ---- through the factors: thread = channel `row` of d_k, tokens 16 cg .. 16 cg + 15.  The
    //      terms of dG cancel down to a result of the order of alpha, so they are formed from the
    //      bf16 factors the products used (the pair terms then cancel exactly): e^G and e^-G are
    //      rebuilt here exactly as the folding built them, per 8-token group (decay_pair8), and
    //      Q~, E~, K~ rounded to bf16 as there.
    {
        float *sFin = reinterpret_cast<float *>(sm + SC_FIN);
        const bool ch_ok = row < a.din;
        float al[16];
        float run2[2] = {0.f, 0.f};  // log-decay sums of this thread's two 8-token groups
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = 16 * cg + i;
            const float gv = !(t < L && ch_ok) ? 0.f
                             : kGS ? reinterpret_cast<const float *>(sm + SGT)[t]
                                   : *reinterpret_cast<const float *>(sm + GG + (row >> 5) * 8192 + sw128(t, (row & 31) * 4));
            run2[i >> 3] += gv;
            al[i] = __expf(gv);
        }
        wait_or_abort(&bar_d, ph, a.status, &s_abort);
        tc_fence_after();
        if (warp == 0 && next >= 0) issue(0, nx);  // Q~, K~, E~, [dO; -dY], T, P are consumed
        sFin[(2 * cg) * D + row] = run2[0];
        sFin[(2 * cg + 1) * D + row] = run2[1];
        if (tid == 32) bulk_wait_read0();  // dv and dw have left v and w, which take dg below
        __syncthreads();
        if (warp == 0 && next >= 0) issue(1, nx);  // log alpha is read
        float off2[2] = {0.f, 0.f};  // G before each group: the group sums in order, as the folding added them
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (u < 2 * cg) off2[0] += sFin[u * D + row];
        off2[1] = off2[0] + run2[0];
        float emG[16];
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            float rr = __expf(-(off2[h8] + run2[h8]));
#pragma unroll
            for (int i = 7; i >= 0; --i) {
                emG[8 * h8 + i] = rr;
                rr *= al[8 * h8 + i];
            }
        }
        uint32_t rq[16], re[16], rk[16], ru[16];
        tmem_ld16(tmem + TM_DQE + 16 * cg + lane_off, rq);
        tmem_ld16(tmem + TM_DQE + 64 + 16 * cg + lane_off, re);
        tmem_ld16(tmem + TM_DK + 16 * cg + lane_off, rk);
        tmem_ld16(tmem + TM_DKU + 16 * cg + lane_off, ru);
        tmem_wait_ld();
        wait_or_abort(&bar_in2, ph, a.status, &s_abort);
        float e = 0.f, kup = 0.f;  // kup: this thread's share of sum_s K~_s . dK~_s (state-update part)
        float dG[16], pdb[16];     // pdb (kSG): this channel's share of db_t
        const size_t base = tok_off(a, bb, hh, ci, 16 * cg) + row, stride = (size_t)a.H * a.din;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = 16 * cg + i;
            if ((i & 7) == 0) e = __expf(off2[i >> 3]);
            e *= al[i];
            const uint32_t so = tile_off(t, row, 8192);
            const bool ok = t < L;
            const float q0 = ok ? ld_bf(sm + SS + so) : 0.f, k0 = ok ? ld_bf(sm + SS + 16384 + so) : 0.f;
            const float b0 = ok ? (kSG ? __bfloat162float(sBt[t]) : ld_bf(sm + DS + so)) : 0.f;
            const float dQ = __uint_as_float(rq[i]), dE = __uint_as_float(re[i]), dKu = __uint_as_float(ru[i]);
            const float dK = __uint_as_float(rk[i]) + dKu;
            const float de = dE * e;
            const uint32_t qe = pack_bf16x2(q0 * e, b0 * k0 * e);  // Q~, E~ as the folding rounded them
            const float kt = __bfloat162float(__float2bfloat16_rn(k0 * emG[i]));  // K~, likewise
            dG[i] = dQ * bf_lo(qe) + dE * bf_hi(qe) - dK * kt;
            kup = fmaf(kt, dKu, kup);
            pdb[i] = ok ? de * k0 : 0.f;
            if (full) {  // over the raw q, k, b just read
                st_bf(sm + SS + so, dQ * e);
                if (!kSG) st_bf(sm + DS + so, de * k0);
                st_bf(sm + SS + 16384 + so, de * b0 + dK * emG[i]);
            } else if (ok && ch_ok) {
                const size_t go = base + (size_t)i * stride;
                a.dq[go] = __float2bfloat16_rn(dQ * e);
                if (!kSG) a.db[go] = __float2bfloat16_rn(de * k0);
                a.dk[go] = __float2bfloat16_rn(de * b0 + dK * emG[i]);
            }
        }
        if (kSG) {  // db_t: sum over this lane quarter's 32 channels into the unused first half of DS
            warp_sum16(pdb, lane);
            if (!(lane & 1)) reinterpret_cast<float *>(sm + DS)[quarter * 64 + 16 * cg + (lane >> 1)] = pdb[0];
        }
        fence_proxy_async_smem();
        __syncthreads();  // dq, dk, db are staged: their stores go out while dg is formed
        if (tid == 32 && full) {
            for (int at = 0; at < a.din / 64; ++at) {
                tma_store_3d(&maps.dq, sm + SS + at * 8192, at * 64, hh, y);
                tma_store_3d(&maps.dk, sm + SS + 16384 + at * 8192, at * 64, hh, y);
                if (!kSG) tma_store_3d(&maps.db, sm + DS + at * 8192, at * 64, hh, y);
            }
            bulk_commit();
        }
        if (kSG && tid < 64 && tid < L) {  // db_t: the four lane quarters' sums
            const float *p4 = reinterpret_cast<const float *>(sm + DS);
            a.db[((size_t)y + tid) * a.H + hh] = __float2bfloat16_rn(p4[tid] + p4[64 + tid] + p4[128 + tid] + p4[192 + tid]);
        }
        if (cg == 3) dG[15] += reinterpret_cast<const float *>(sm + DGF)[row];  // gamma dgamma, last row
        float rs = 0.f;
#pragma unroll
        for (int i = 15; i >= 0; --i) {
            rs += dG[i];
            dG[i] = rs;
        }
        sFin[8 * D + cg * D + row] = rs;
        sFin[12 * D + cg * D + row] = kup;
        named_bar(1 + quarter, 4 * 32);  // the four warps of this TMEM lane quarter
        // later groups, and the state-update part of gamma dgamma: sum over the chunk of K~ . dK~'s
        // update part, formed from the very values dK~ and dG used, so that it cancels exactly
        float after = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u > cg) after += sFin[8 * D + u * D + row];
            after += sFin[12 * D + u * D + row];
        }
        if (kGS) {  // dlog alpha_t: sum over this lane quarter's 32 channels; the quarters add up below
            float pdg[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pdg[i] = (ch_ok && 16 * cg + i < L) ? dG[i] + after : 0.f;
            warp_sum16(pdg, lane);
            if (!(lane & 1)) reinterpret_cast<float *>(sm + SDG)[quarter * 64 + 16 * cg + (lane >> 1)] = pdg[0];
        } else if (full) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<float *>(sm + VV + (row >> 5) * 8192 + sw128(16 * cg + i, (row & 31) * 4)) =
                    dG[i] + after;
        } else if (ch_ok) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = 16 * cg + i;
                if (t < L) a.dg[base + (size_t)i * stride] = dG[i] + after;
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (kGS && tid >= 64 && tid < 64 + L) {  // dlog alpha_t: the four lane quarters' sums (warps 2, 3)
        const float *p4 = reinterpret_cast<const float *>(sm + SDG);
        const int t = tid - 64;
        a.dg[((size_t)y + t) * a.H + hh] = p4[t] + p4[64 + t] + p4[128 + t] + p4[192 + t];
    }
    if (warp == 1) {  // lane 0 owns every bulk store of the block
        if (!kGS && lane == 0 && full) {  // dq, dk, db went out before dg was formed
            for (int bx = 0; bx < a.din / 32; ++bx) tma_store_3d(&maps.dg, sm + VV + bx * 8192, bx * 32, hh, y);
            bulk_commit();
        }
        // dq, dk and db are read before S^T and dS_n^T come in (kGS: theirs is the last group)
        if (lane == 0) {
            if (kGS) bulk_wait_read0();
            else bulk_wait_read1();
        }
        __syncwarp();
        if (next >= 0) {
            issue(2, nx);  // S^T, dS_n^T into the freed tiles; v, w wait for dg (next task's folding)
            pend3 = true;
        }
    }
    task = next;
    cr = nx;
    ph ^= 1;
    }
    if (warp == 1 && lane == 0) bulk_wait0();  // the last task's gradients have been written
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace

size_t bwd_tc_workspace_bytes(const Problem &p) { return tc_layout(p).total; }

// The backward's per-chunk factors in workspace ws (layout l), written by the forward's states run.
static BwdFactors bwd_factors(const Problem &p, const BwdTcLayout &l, char *base)
{
    BwdFactors f;
    f.W = reinterpret_cast<__nv_bfloat16 *>(base + l.W);
    f.Kt = reinterpret_cast<__nv_bfloat16 *>(base + l.Kt);
    f.Mc = reinterpret_cast<__nv_bfloat16 *>(base + l.Mc);
    f.Tm = reinterpret_cast<__nv_bfloat16 *>(base + l.Tm);
    f.Pm = reinterpret_cast<__nv_bfloat16 *>(base + l.Pm);
    f.gam = reinterpret_cast<float *>(base + l.gam);
    f.flist = reinterpret_cast<int *>(base + l.flist);
    f.nchb = (int)chunk_bound(p);
    return f;
}

cudaError_t launch_fwd_save(const Problem &p, void *o, float *S_T, void *ws, int *status, cudaStream_t s)
{
    if (p.cu_seqlens || (p.D != 128 && p.D != 64)) return cudaErrorNotSupported;
    const BwdTcLayout l = tc_layout(p);
    char *base = static_cast<char *>(ws);
    const BwdFactors f = bwd_factors(p, l, base);
    cudaError_t e = cudaMemsetAsync(f.flist, 0, sizeof(int), s);  // no chunk runs token by token yet
    if (e != cudaSuccess) return e;
    return launch_fwd_tc(p, o, S_T, reinterpret_cast<__nv_bfloat16 *>(base + l.states), status, s, nullptr, &f);
}

cudaError_t launch_bwd_tc(const Problem &p, const void *d_o, const float *dS_T, const BwdOut &out, void *ws,
                          int *status, cudaStream_t s, bool states_saved)
{
    if (p.D != 128 && p.D != 64) return cudaErrorNotSupported;
    {  // TMA row coordinates are 32-bit: the state rows (slot x 128) and the token rows
        const uint64_t state_rows = (uint64_t)p.H * (chunk_bound(p) + p.B) * D;
        if (state_rows > (uint64_t)INT_MAX || (uint64_t)token_rows(p) > (uint64_t)INT_MAX)
            return cudaErrorInvalidValue;
    }
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
    a.Kt = reinterpret_cast<__nv_bfloat16 *>(base + l.Kt);
    a.gam = reinterpret_cast<float *>(base + l.gam);
    a.flist = reinterpret_cast<int *>(base + l.flist);
    a.Mc = reinterpret_cast<__nv_bfloat16 *>(base + l.Mc);
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

    cudaError_t e = cudaSuccess;
    if (!states_saved || p.cu_seqlens) {
        // the forward in states mode: chunk-boundary states and the per-chunk factors of the chain
        // and the gradient kernel, unless the forward recorded them (gdn2_chunk_fwd_save)
        const BwdFactors f = bwd_factors(a.pr, l, base);
        if ((e = cudaMemsetAsync(f.flist, 0, sizeof(int), s)) != cudaSuccess) return e;  // no chunk flagged yet
        e = launch_fwd_tc(a.pr, nullptr, nullptr, a.states, status, s, nullptr, &f);
        if (e != cudaSuccess) return e;
    }
    {  // the dS chain on the tensor cores: one block per (batch, head)
        ChainMaps cm;
        memset(&cm, 0, sizeof(cm));
        const uint64_t nchunk = (uint64_t)p.H * chunk_bound(p);
        if (!make_map_2d(&cm.kt, a.Kt, D, nchunk * C, 64, C) || !make_map_2d(&cm.wt, a.W, C, nchunk * D, 64, D) ||
            !make_map_2d(&cm.mt, a.Mc, C, nchunk * D, 64, D) ||
            !make_map(&cm.dO, d_o, false, 1, (int)token_rows(p), p.H, p.D))
            return cudaErrorInvalidValue;
        if ((e = set_smem_attr(reinterpret_cast<const void *>(bwd_chain_tc_kernel), (int)chain_tc::SMEM)) != cudaSuccess)
            return e;
        bwd_chain_tc_kernel<<<p.B * p.H, chain_tc::kThreads, chain_tc::SMEM, s>>>(cm, a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {  // gradients on the tensor cores: one block per (chunk, head)
        GradMaps maps;
        memset(&maps, 0, sizeof(maps));
        const int rows = (int)token_rows(p);
        const uint64_t nchunk = (uint64_t)p.H * chunk_bound(p), nbound = (uint64_t)p.H * (chunk_bound(p) + p.B);
        const bool sg = p.bw_scalar;  // scalar b and w ([rows, H]): no tiles of theirs, db and dw written per token
        const bool gs = p.g_scalar;   // scalar decay ([rows, H]): likewise log alpha and dlog alpha
        if (!make_map(&maps.q, p.q, false, 1, rows, p.H, p.D) || !make_map(&maps.k, p.k, false, 1, rows, p.H, p.D) ||
            (!sg && !make_map(&maps.b, p.b, false, 1, rows, p.H, p.D)) || !make_map(&maps.v, p.v, false, 1, rows, p.H, p.D) ||
            (!sg && !make_map(&maps.w, p.w, false, 1, rows, p.H, p.D)) || !make_map(&maps.dO, d_o, false, 1, rows, p.H, p.D) ||
            (!gs && !make_map(&maps.g, p.g, true, 1, rows, p.H, p.D)) ||
            !make_map_2d(&maps.st, a.states, D, nbound * D, 64, D) ||
            !make_map_2d(&maps.dsn, a.dSn, D, nchunk * D, 64, D) ||
            !make_map_2d(&maps.tm, a.Tm, C, nchunk * C, 64, C) || !make_map_2d(&maps.pm, a.Pm, C, nchunk * C, 64, C) ||
            !make_map(&maps.dq, out.dq, false, 1, rows, p.H, p.D) || !make_map(&maps.dk, out.dk, false, 1, rows, p.H, p.D) ||
            (!sg && !make_map(&maps.db, out.db, false, 1, rows, p.H, p.D)) || !make_map(&maps.dv, out.dv, false, 1, rows, p.H, p.D) ||
            (!sg && !make_map(&maps.dw, out.dw, false, 1, rows, p.H, p.D)) ||
            (!gs && !make_map(&maps.dg, out.dg, true, 1, rows, p.H, p.D)))
            return cudaErrorInvalidValue;
        int dev = 0, n_sm = 148;  // persistent: one block per multiprocessor
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
        const int ntask = (int)chunk_bound(p) * p.H;
        auto run = [&](auto kernel) -> cudaError_t {
            cudaError_t er = set_smem_attr(reinterpret_cast<const void *>(kernel), (int)grad_tc::SMEM);
            if (er != cudaSuccess) return er;
            kernel<<<max(1, min(ntask, n_sm)), grad_tc::kThreads, grad_tc::SMEM, s>>>(maps, a);
            return cudaSuccess;
        };
        e = sg ? (gs ? run(bwd_grad_kernel<true, true>) : run(bwd_grad_kernel<true, false>))
               : (gs ? run(bwd_grad_kernel<false, true>) : run(bwd_grad_kernel<false, false>));
        if (e != cudaSuccess) return e;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the chunks that run token by token: their gradients, exact, over what the gradient kernel wrote
    return launch_tok_grad_tc(a.pr, d_o, a.states, a.dSn, a.flist, reinterpret_cast<float *>(base + l.scratch),
                              l.tok_blocks, out, s);
}

}  // namespace gdn2
