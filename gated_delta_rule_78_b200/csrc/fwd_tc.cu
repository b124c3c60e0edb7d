// Chunkwise GDN-2 forward on the sm_100a tensor cores (bf16 operands, fp32
// accumulation in TMEM, fp32 state).  d_k = d_v = 128, chunk C = 64.
//
// Per chunk, with S the fp32 state at the chunk start (the chunkwise WY
// algorithm with the channel-wise decay folded into asymmetric factors, as the
// aiexpert.news article's implementation paragraph describes, and the
// auxiliary matrices of the aixai.ru post's "Как это реализуется на практике"):
//   G  = inclusive cumulative sum of log alpha over the chunk (fp32)
//   Q~ = q e^G,  E~ = (b.k) e^G,  K~ = k e^-G,  K^ = k e^(G_L - G),  gamma = e^G_L
//   [A; P] = [E~; Q~] K~^T          A strictly lower, P lower incl. (one M=128 MMA)
//   T  = (I + A)^-1                  blocked 16x16 substitution in shared memory
//   W^T = E~^T T^T,  U^T = X^T T^T  (X = w.v)
//   U~^T = U^T + S^T (-W^T)          S^T (bf16) is the TMEM A operand
//   O^T  = S^T Q~^T + U~^T P^T
//   S   <- Diag(gamma) S + (U~^T K^)^T   (update done in fp32 registers)
// Everything is formulated transposed so that every product has M = 128
// (d_k or d_v, or the stacked [E~; Q~]) and runs as a full-height tcgen05.mma.
//
// Work decomposition: one CTA per (batch, head), 8 warps.  Warp w owns TMEM
// lanes 32 (w & 3) .. +31 and column half (w >> 2) of every readback; its
// threads hold their 64 columns of S^T (row j = d_v index) in fp32 registers.
// The raw inputs of chunk c+1 are fetched by TMA (128-byte swizzle, the same
// layout the MMA descriptors read) into each buffer as soon as chunk c no
// longer needs it, so the loads overlap chunk c's compute; the elementwise pass
// converts them in place into the factors.
#include <cuda.h>

#include "gdn2_internal.cuh"
#include "tc_util.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int D = 128;
constexpr int C = 64;
constexpr int kThreads = 256;
constexpr int LDA = 68;  // fp32 row stride of the A / T scratch

// shared-memory map (bytes from a 1024-byte aligned base)
constexpr uint32_t OFF_QE = 0;          // [E~ a0 | Q~ a0 | E~ a1 | Q~ a1], 8 KiB each (raw b, q)
constexpr uint32_t OFF_K = 32768;       // K~ (raw k), 2 atoms
constexpr uint32_t OFF_KH = 49152;      // K^, 2 atoms
constexpr uint32_t OFF_G = 65536;       // log alpha fp32, 4 atoms of 32 channels
constexpr uint32_t OFF_V = 98304;       // X = w.v (raw v), 2 atoms
constexpr uint32_t OFF_W = 114688;      // raw w, 2 atoms
constexpr uint32_t OFF_WT = 131072;     // -W^T: 128 rows (d_k) x 64 tokens
constexpr uint32_t OFF_TT = 147456;     // T: 64 rows (i) x 64 (j)
constexpr uint32_t OFF_PT = 155648;     // P: 64 rows (t) x 64 (i)
constexpr uint32_t OFF_SA = 163840;     // A fp32 [64][LDA]
constexpr uint32_t OFF_ST = OFF_SA + 64 * LDA * 4;   // T fp32 [64][LDA]
constexpr uint32_t OFF_TOT = OFF_ST + 64 * LDA * 4;  // per-quarter decay totals [4][128] fp32
constexpr uint32_t OFF_GAM = OFF_TOT + 4 * 128 * 4;  // gamma [128] fp32
constexpr uint32_t SMEM_USED = OFF_GAM + 128 * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // slack for the 1024-byte alignment

// TMEM columns
constexpr uint32_t TM_SBF = 0;     // S^T bf16 (A operand), 64 columns
constexpr uint32_t TM_AP = 64;     // [A; P] fp32, 64 columns
constexpr uint32_t TM_WT = 128;    // W^T fp32
constexpr uint32_t TM_UT = 192;    // U^T, then U~^T, fp32
constexpr uint32_t TM_OT = 256;    // O^T fp32
constexpr uint32_t TM_UB = 320;    // U~^T bf16 (A operand), 32 columns
constexpr uint32_t TM_DS = 384;    // (K^^T U~)^T fp32, 128 columns
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_N64 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_N64_AMN = idesc_bf16(128, 64, 1, 0);
constexpr uint32_t IDESC_N64_BMN = idesc_bf16(128, 64, 0, 1);
constexpr uint32_t IDESC_N128_BMN = idesc_bf16(128, 128, 0, 1);

struct TcParams {
    int B, T, H;
    const float *S0;
    __nv_bfloat16 *o;
    float *S_T;
    int *status;
};

struct TcMaps {
    CUtensorMap q, k, v, b, w, g;
};

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_g, bar_k, bar_bv, bar_q, bar_mma;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hcol = warp >> 2;
    const int bh = blockIdx.x, bb = bh / p.H, hh = bh % p.H;
    const int T = p.T;
    const int nchunks = (T + C - 1) / C;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float *sA = reinterpret_cast<float *>(sm + OFF_SA);
    float *sT = reinterpret_cast<float *>(sm + OFF_ST);
    float *sTot = reinterpret_cast<float *>(sm + OFF_TOT);
    float *sGam = reinterpret_cast<float *>(sm + OFF_GAM);

    auto issue_loads = [&](int ci, int which) {
        // which: 0 = g + w, 1 = k, 2 = b + v, 3 = q
        const int y = bb * T + ci * C;
        if (which == 0) {
            mbar_expect_tx(&bar_g, 4 * 8192 + 2 * 8192);
            for (int a = 0; a < 4; ++a) tma_load_3d(sm + OFF_G + a * 8192, &maps.g, a * 32, hh, y, &bar_g);
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + OFF_W + a * 8192, &maps.w, a * 64, hh, y, &bar_g);
        } else if (which == 1) {
            mbar_expect_tx(&bar_k, 2 * 8192);
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + OFF_K + a * 8192, &maps.k, a * 64, hh, y, &bar_k);
        } else if (which == 2) {
            mbar_expect_tx(&bar_bv, 4 * 8192);
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + OFF_QE + a * 16384, &maps.b, a * 64, hh, y, &bar_bv);
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + OFF_V + a * 8192, &maps.v, a * 64, hh, y, &bar_bv);
        } else {
            mbar_expect_tx(&bar_q, 2 * 8192);
            for (int a = 0; a < 2; ++a) tma_load_3d(sm + OFF_QE + 8192 + a * 16384, &maps.q, a * 64, hh, y, &bar_q);
        }
    };
    auto fail = [&]() {
        s_abort = 1;
        atomicExch(p.status, kStatusTimeout);
    };

    if (tid == 0) {
        s_abort = 0;
        mbar_init(&bar_g, 1);
        mbar_init(&bar_k, 1);
        mbar_init(&bar_bv, 1);
        mbar_init(&bar_q, 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.v);
        prefetch_tmap(&maps.b); prefetch_tmap(&maps.w); prefetch_tmap(&maps.g);
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    if (tid == 0 && nchunks > 0)
        for (int wch = 0; wch < 4; ++wch) issue_loads(0, wch);

    // fp32 state: this thread holds S^T[j][64 hcol + i], j = 32 quarter + lane
    const int jrow = quarter * 32 + lane;
    float Sf[64];
#pragma unroll
    for (int i = 0; i < 64; ++i)
        Sf[i] = p.S0 ? p.S0[((size_t)bh * D + 64 * hcol + i) * D + jrow] : 0.f;
    {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(Sf[2 * i], Sf[2 * i + 1]);
        tmem_st32(tmem + TM_SBF + 32 * hcol + lane_off, pk);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    uint32_t mma_phase = 0;
    for (int ci = 0; ci < nchunks; ++ci) {
        const uint32_t par = ci & 1;
        const int L = min(C, T - ci * C);
        const bool has_next = ci + 1 < nchunks;
        // ---------------- wait for this chunk's inputs
        if (!mbar_wait(&bar_g, par) || !mbar_wait(&bar_k, par) || !mbar_wait(&bar_bv, par) ||
            !mbar_wait(&bar_q, par))
            fail();
        __syncthreads();
        if (s_abort) break;
        // ---------------- decay folding (elementwise, in place)
        {
            const int cb = warp & 1, tq = warp >> 1;  // channel block of 64, token quarter of 16
            float Gl[16][2];
            float run0 = 0.f, run1 = 0.f;
            const uint8_t *gatom = sm + OFF_G + (2 * cb + (lane >> 4)) * 8192;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = 16 * tq + i;
                float2 gv = *reinterpret_cast<const float2 *>(gatom + sw128(t, 8 * (lane & 15)));
                if (t >= L) gv = make_float2(0.f, 0.f);
                run0 += gv.x;
                run1 += gv.y;
                Gl[i][0] = run0;
                Gl[i][1] = run1;
            }
            const int ch = 64 * cb + 2 * lane;
            *reinterpret_cast<float2 *>(sTot + tq * 128 + ch) = make_float2(run0, run1);
            __syncthreads();
            float c0 = 0.f, c1 = 0.f, gl0 = 0.f, gl1 = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 tv = *reinterpret_cast<const float2 *>(sTot + u * 128 + ch);
                if (u < tq) { c0 += tv.x; c1 += tv.y; }
                gl0 += tv.x;
                gl1 += tv.y;
            }
            if (tq == 0) *reinterpret_cast<float2 *>(sGam + ch) = make_float2(__expf(gl0), __expf(gl1));
            uint8_t *pe = sm + OFF_QE + cb * 16384;
            uint8_t *pq = pe + 8192;
            uint8_t *pk = sm + OFF_K + cb * 8192;
            uint8_t *ph = sm + OFF_KH + cb * 8192;
            uint8_t *pv = sm + OFF_V + cb * 8192;
            const uint8_t *pw = sm + OFF_W + cb * 8192;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = 16 * tq + i;
                const uint32_t off = sw128(t, 4 * lane);
                const float G0 = c0 + Gl[i][0], G1 = c1 + Gl[i][1];
                const float e0 = __expf(G0), e1 = __expf(G1);
                const float m0 = __expf(-G0), m1 = __expf(-G1);
                const float h0 = __expf(gl0 - G0), h1 = __expf(gl1 - G1);
                uint32_t qw = *reinterpret_cast<const uint32_t *>(pq + off);
                uint32_t kw = *reinterpret_cast<const uint32_t *>(pk + off);
                uint32_t bw = *reinterpret_cast<const uint32_t *>(pe + off);
                uint32_t vw = *reinterpret_cast<const uint32_t *>(pv + off);
                uint32_t ww = *reinterpret_cast<const uint32_t *>(pw + off);
                if (t >= L) { qw = 0u; kw = 0u; bw = 0u; vw = 0u; }
                const float k0 = bf_lo(kw), k1 = bf_hi(kw);
                *reinterpret_cast<uint32_t *>(pq + off) = pack_bf16x2(bf_lo(qw) * e0, bf_hi(qw) * e1);
                *reinterpret_cast<uint32_t *>(pe + off) = pack_bf16x2(bf_lo(bw) * k0 * e0, bf_hi(bw) * k1 * e1);
                *reinterpret_cast<uint32_t *>(pk + off) = pack_bf16x2(k0 * m0, k1 * m1);
                *reinterpret_cast<uint32_t *>(ph + off) = pack_bf16x2(k0 * h0, k1 * h1);
                *reinterpret_cast<uint32_t *>(pv + off) = pack_bf16x2(bf_lo(vw) * bf_lo(ww), bf_hi(vw) * bf_hi(ww));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        // ---------------- MMA 1: [A; P] = [E~; Q~] K~^T ; prefetch g, w of the next chunk
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_QE + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(sbase + OFF_K + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                mma_ss(tmem + TM_AP, ad, bd, IDESC_N64, ks > 0);
            }
            mma_commit(&bar_mma);
            if (has_next) issue_loads(ci + 1, 0);
        }
        if (!mbar_wait(&bar_mma, mma_phase)) fail();
        mma_phase ^= 1;
        tc_fence_after();
        if (tid == 0 && has_next) issue_loads(ci + 1, 1);
        {
            uint32_t r[32];
            tmem_ld32(tmem + TM_AP + 32 * hcol + lane_off, r);
            tmem_wait_ld();
            const int row = quarter * 32 + lane;
            if (row < 64) {  // A, strictly lower
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int j = 32 * hcol + u;
                    sA[row * LDA + j] = (j < row) ? __uint_as_float(r[u]) : 0.f;
                }
            } else {  // P, lower including the diagonal -> bf16 rows of SPT
                const int t = row - 64;
                uint8_t *dst = sm + OFF_PT;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i0 = 32 * hcol + 8 * m + 2 * e;
                        const float lo = (i0 <= t) ? __uint_as_float(r[8 * m + 2 * e]) : 0.f;
                        const float hi = (i0 + 1 <= t) ? __uint_as_float(r[8 * m + 2 * e + 1]) : 0.f;
                        w4[e] = pack_bf16x2(lo, hi);
                    }
                    *reinterpret_cast<uint4 *>(dst + sw128(t, 64 * hcol + 16 * m)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (s_abort) break;
        // ---------------- T = (I + A)^-1, blocked by 16
        if (tid < 64) {  // diagonal blocks: column j of block pblk
            const int pblk = tid >> 4, j = tid & 15, r0 = 16 * pblk;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float s = 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) s += sA[(r0 + i) * LDA + r0 + m] * x[m];
                x[i] = (i > j) ? -s : (i == j ? 1.f : 0.f);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sT[(r0 + i) * LDA + r0 + j] = x[i];
        }
        __syncthreads();
        {
            const int rr = tid >> 4, ss = tid & 15;
            for (int d = 1; d < 4; ++d) {
                const int nb = 4 - d;
                float y[3];
#pragma unroll
                for (int pb = 0; pb < 3; ++pb) {
                    if (pb >= nb) break;
                    const int R = 16 * (pb + d), Cc = 16 * pb;
                    float s = 0.f;
                    for (int m = pb; m < pb + d; ++m)
#pragma unroll
                        for (int u = 0; u < 16; ++u) s += sA[(R + rr) * LDA + 16 * m + u] * sT[(16 * m + u) * LDA + Cc + ss];
                    y[pb] = s;
                }
                // stash Y in the (still empty) T block, then T_block = -T_diag Y
#pragma unroll
                for (int pb = 0; pb < 3; ++pb)
                    if (pb < nb) sT[(16 * (pb + d) + rr) * LDA + 16 * pb + ss] = y[pb];
                __syncthreads();
#pragma unroll
                for (int pb = 0; pb < 3; ++pb) {
                    if (pb >= nb) break;
                    const int R = 16 * (pb + d), Cc = 16 * pb;
                    float s = 0.f;
#pragma unroll
                    for (int u = 0; u < 16; ++u) s += sT[(R + rr) * LDA + R + u] * sT[(R + u) * LDA + Cc + ss];
                    y[pb] = -s;
                }
                __syncthreads();
#pragma unroll
                for (int pb = 0; pb < 3; ++pb)
                    if (pb < nb) sT[(16 * (pb + d) + rr) * LDA + 16 * pb + ss] = y[pb];
                __syncthreads();
            }
        }
        {  // T -> bf16 rows (i) of 64 j, zero above the diagonal
            const int i = tid >> 2, qq = tid & 3;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j0 = 16 * qq + 8 * m + 2 * e;
                    const float lo = (j0 <= i) ? sT[i * LDA + j0] : 0.f;
                    const float hi = (j0 + 1 <= i) ? sT[i * LDA + j0 + 1] : 0.f;
                    w4[e] = pack_bf16x2(lo, hi);
                }
                *reinterpret_cast<uint4 *>(sm + OFF_TT + sw128(i, 32 * qq + 16 * m)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        // ---------------- MMA 2: W^T = E~^T T^T, U^T = X^T T^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bd = sdesc_sw128(sbase + OFF_TT + ks * 32, 16, 1024);
                mma_ss(tmem + TM_WT, sdesc_sw128(sbase + OFF_QE + ks * 2048, 16384, 1024), bd, IDESC_N64_AMN, ks > 0);
                mma_ss(tmem + TM_UT, sdesc_sw128(sbase + OFF_V + ks * 2048, 8192, 1024), bd, IDESC_N64_AMN, ks > 0);
            }
            mma_commit(&bar_mma);
        }
        if (!mbar_wait(&bar_mma, mma_phase)) fail();
        mma_phase ^= 1;
        tc_fence_after();
        if (tid == 0 && has_next) {
            fence_proxy_async_smem();
            issue_loads(ci + 1, 2);
        }
        {  // -W^T -> bf16 rows (d_k) of SWT
            uint32_t r[32];
            tmem_ld32(tmem + TM_WT + 32 * hcol + lane_off, r);
            tmem_wait_ld();
            const int c = quarter * 32 + lane;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w4[e] = pack_bf16x2(-__uint_as_float(r[8 * m + 2 * e]), -__uint_as_float(r[8 * m + 2 * e + 1]));
                *reinterpret_cast<uint4 *>(sm + OFF_WT + sw128(c, 64 * hcol + 16 * m)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_abort) break;
        // ---------------- MMA 3: U~^T = U^T + S^T (-W^T);  O^T = S^T Q~^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ts(tmem + TM_UT, tmem + TM_SBF + 8 * ks, sdesc_sw128(sbase + OFF_WT + ks * 2048, 8192, 1024),
                       IDESC_N64_BMN, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ts(tmem + TM_OT, tmem + TM_SBF + 8 * ks,
                       sdesc_sw128(sbase + OFF_QE + 8192 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), IDESC_N64,
                       ks > 0);
            mma_commit(&bar_mma);
        }
        if (!mbar_wait(&bar_mma, mma_phase)) fail();
        mma_phase ^= 1;
        tc_fence_after();
        if (tid == 0 && has_next) {
            fence_proxy_async_smem();
            issue_loads(ci + 1, 3);
        }
        {  // U~^T -> bf16 TMEM operand
            uint32_t r[32];
            tmem_ld32(tmem + TM_UT + 32 * hcol + lane_off, r);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
            tmem_st16(tmem + TM_UB + 16 * hcol + lane_off, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        if (s_abort) break;
        // ---------------- MMA 4: dS^T = U~^T K^ ;  O^T += U~^T P^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ts(tmem + TM_DS, tmem + TM_UB + 8 * ks, sdesc_sw128(sbase + OFF_KH + ks * 2048, 8192, 1024),
                       IDESC_N128_BMN, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ts(tmem + TM_OT, tmem + TM_UB + 8 * ks, sdesc_sw128(sbase + OFF_PT + ks * 32, 16, 1024), IDESC_N64, 1);
            mma_commit(&bar_mma);
        }
        if (!mbar_wait(&bar_mma, mma_phase)) fail();
        mma_phase ^= 1;
        tc_fence_after();
        {  // state update in fp32 registers, bf16 copy back to TMEM
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tmem + TM_DS + 64 * hcol + 32 * half + lane_off, r);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int i = 32 * half + u;
                    Sf[i] = sGam[64 * hcol + i] * Sf[i] + __uint_as_float(r[u]);
                }
            }
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(Sf[2 * i], Sf[2 * i + 1]);
            tmem_st32(tmem + TM_SBF + 32 * hcol + lane_off, pk);
        }
        {  // O^T -> o (bf16)
            uint32_t r[32];
            tmem_ld32(tmem + TM_OT + 32 * hcol + lane_off, r);
            tmem_wait_ld();
            __nv_bfloat16 *orow = p.o + ((size_t)bb * T + (size_t)ci * C) * p.H * D + (size_t)hh * D + jrow;
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int t = 32 * hcol + u;
                if (t < L) orow[(size_t)t * p.H * D] = __float2bfloat16_rn(__uint_as_float(r[u]));
            }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
    }
    if (!s_abort && p.S_T) {
#pragma unroll
        for (int i = 0; i < 64; ++i) p.S_T[((size_t)bh * D + 64 * hcol + i) * D + jrow] = Sf[i];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// 3-D view (channel, head, token) of a [B,T,H,D] tensor; box = (inner, 1, 64 tokens), 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, bool fp32, int B, int T, int H)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t es = fp32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)B * (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es};
    cuuint32_t box[3] = {fp32 ? 32u : 64u, 1u, (cuuint32_t)C};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_fwd_tc(const Problem &pr, void *o, float *S_T, int *status, cudaStream_t s)
{
    if (pr.D != D) return cudaErrorNotSupported;
    TcMaps maps;
    if (!make_map(&maps.q, pr.q, false, pr.B, pr.T, pr.H) || !make_map(&maps.k, pr.k, false, pr.B, pr.T, pr.H) ||
        !make_map(&maps.v, pr.v, false, pr.B, pr.T, pr.H) || !make_map(&maps.b, pr.b, false, pr.B, pr.T, pr.H) ||
        !make_map(&maps.w, pr.w, false, pr.B, pr.T, pr.H) || !make_map(&maps.g, pr.g, true, pr.B, pr.T, pr.H))
        return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    TcParams prm{pr.B, pr.T, pr.H, pr.S0, (__nv_bfloat16 *)o, S_T, status};
    fwd_tc_kernel<<<pr.B * pr.H, kThreads, SMEM_BYTES, s>>>(maps, prm);
    return cudaGetLastError();
}

}  // namespace gdn2
