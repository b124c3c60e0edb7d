// Chunkwise GDN-2 forward on the sm_100a tensor cores (bf16 operands, fp32
// accumulation in TMEM, fp32 state).  d_k = d_v = 128, chunk C = 64.
//
// Per chunk, with S the fp32 state at the chunk start (the chunkwise WY
// algorithm with the channel-wise decay folded into asymmetric factors, as the
// aiexpert.news article's implementation paragraph describes, and the
// auxiliary matrices of the aixai.ru post's "Как это реализуется на практике"):
//   G  = inclusive cumulative sum of log alpha over the chunk (fp32)
//   Q~ = q e^G,  E~ = (b.k) e^G,  K~ = k e^-G,  gamma = e^G_L,  X = w.v
//                                    (one exponential per element, alpha = e^g: e^G is a
//                                    running product of alpha forwards from the token
//                                    group's start, e^-G one backwards from its end.  The
//                                    factors are bf16x2 products of the bf16 inputs and
//                                    e^+-G rounded to bf16; X is one, exact before its
//                                    single rounding)
//   [A; P] = [E~; Q~] K~^T          A strictly lower, P lower incl. (one M=128 MMA)
//   T   = (I + A)^-1                 blocked: 16x16 diagonal blocks by substitution,
//                                    the doubling levels on warp-level TF32 MMAs
//   Y   = X - E~ S                  (the gated value minus what the erase-weighted
//                                    keys read from the chunk-start state)
//   U~  = T Y                        (= (I+A)^-1 (w.V) - (I+A)^-1 E~ S)
//   O   = Q~ S + P U~
//   S  <- Diag(gamma) (S + K~^T U~)  (K~ e^G_L is the decay from token t to the
//                                    chunk end, so gamma is applied once, in fp32)
// Everything S-dependent is formulated transposed (S^T, Y^T, U~^T, O^T with
// d_v as the row index) so that every tcgen05.mma has M = 128; S^T, Y^T and
// U~^T are TMEM operands, and S^T [E~; Q~]^T is one N = 128 product.
//
// Work decomposition: one CTA per (batch, head), two warp groups that run one
// chunk apart.  The E group (warps 8-15) does the key-side work that does not
// depend on the state for chunk c+1: decay folding (log alpha is read from L2
// where a TMA prefetch has put it), the [A; P] product, and T = (I+A)^-1.  The
// M group (warps 0-7) runs chunk c's state chain: S^T [E~; Q~]^T, Y, U~, the
// state update and the output; at the end of its chunk it folds the next
// chunk's write gate into its values (X = w.v) and releases the chunk's
// buffers, into which an otherwise idle E warp then loads the chunk after.  All buffers handed from E to M are double-buffered
// by chunk parity; mbarriers, one per parity, carry the hand-offs.  Warp m of
// M owns TMEM lanes 32 (m & 3) .. +31 and column half (m >> 2) of every
// readback and holds its 64 columns of S^T in fp32 registers.  The output tile
// is staged in shared memory and written by a TMA store.
#include <climits>
#include <cuda.h>
#include <string.h>

#include <type_traits>

#include "gdn2_internal.cuh"
#include "tc_util.cuh"
#include "tok_util.cuh"
#include "warp_mma.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int D = 128;
constexpr int C = 64;
constexpr int kThreads = 512;
constexpr int kGroup = 256;  // threads per warp group
constexpr int LDA = 68;      // fp32 row stride of the A / T scratch

// shared-memory map (bytes from a 1024-byte aligned base); [2] = by chunk parity
constexpr uint32_t OFF_QE = 0;          // [2] x [E~ a0 | Q~ a0 | E~ a1 | Q~ a1], 8 KiB each (raw b, q)
constexpr uint32_t OFF_K = 65536;       // [2] x K~ (raw k), 2 atoms
constexpr uint32_t OFF_V = 98304;       // [2] x X = w.v (raw v), 2 atoms
constexpr uint32_t OFF_W = 131072;      // raw w, 2 atoms
constexpr uint32_t OFF_TP = 147456;     // [2] x [T bf16 (64 x 64) | P bf16 (64 x 64)]; the output
                                        //  tile (64 x 128 bf16, row-major) after M is done with them
constexpr uint32_t OFF_SA = 180224;     // A fp32 [64][LDA]
constexpr uint32_t OFF_ST = OFF_SA + 64 * LDA * 4;   // T fp32 [64][LDA]
constexpr uint32_t OFF_TOT = OFF_ST + 64 * LDA * 4;  // per-group decay totals [4][128] fp32
constexpr uint32_t OFF_GAM = OFF_TOT + 4 * 128 * 4;  // gamma [2][128] fp32
constexpr uint32_t OFF_NRM = OFF_GAM + 2 * 128 * 4;  // prologue: sum of squares [q|k][channel half][64] fp32
constexpr uint32_t OFF_RN = OFF_NRM + 2 * 2 * 64 * 4;  // prologue: 1/|q|, 1/|k| [2][q|k][64] fp32
constexpr uint32_t OFF_ID = (OFF_RN + 2 * 2 * 64 * 4 + 1023) / 1024 * 1024;  // kBw: identity [64][64] bf16
constexpr uint32_t SMEM_USED = OFF_ID + 8192;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // slack for the 1024-byte alignment

// TMEM columns
constexpr uint32_t TM_SBF = 0;     // S^T bf16 (A operand), 64 columns                 (M)
constexpr uint32_t TM_AP = 64;     // [A; P] fp32                                      (E)
constexpr uint32_t TM_YO = 128;    // [S^T E~^T | O^T] fp32, 128 columns               (M)
constexpr uint32_t TM_O = 192;     //   O^T half
constexpr uint32_t TM_UT = 256;    // U~^T fp32                                        (M)
constexpr uint32_t TM_YB = 320;    // Y^T bf16 (A operand), 32 columns                 (M)
constexpr uint32_t TM_UB = 352;    // U~^T bf16 (A operand), 32 columns                (M)
constexpr uint32_t TM_DS = 384;    // (K~^T U~)^T fp32, 128 columns                    (M)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_N64 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_N128 = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t IDESC_N128_BMN = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t IDESC_W = idesc_bf16(128, 64, 1, 0);  // W^T = E~^T T^T: A (E~^T) MN-major

// Register split: the launch holds 512 x 128 registers; M takes 152 per thread and
// E 104 (256 x 152 + 256 x 104 = 65536, exactly the launch's total).
constexpr int kRegM = 152;
constexpr int kRegE = 104;
static_assert(kGroup * kRegM + kGroup * kRegE == kThreads * 128, "register split must match the launch");

struct TcParams {
    int B, T, H;
    const __nv_bfloat16 *q, *k, *b, *w;  // read directly by chunks that run token by token; with
                                         // kGate, b and w are one value per (token, head) [rows, H]
    const float *S0;
    const float *g;   // log alpha [B,T,H,D] fp32
    __nv_bfloat16 *o;        // may be null (states-only run)
    float *S_T;
    __nv_bfloat16 *states;   // may be null; else S^T (d_v x d_k) at every chunk boundary, the final
                             // state last, per (sequence, head) at the boundary slots of gdn2_internal.cuh
    int *status;
    const int *cu_seqlens;   // null: B sequences of T tokens; else B packed sequences in T rows
    const int *chunk_off;    // variable length with states only: first chunk of each sequence
    int g_scalar;            // log alpha is one value per (token, head), [rows, H]: a scalar decay
    ScanArgs scan;           // chunk-parallel scan instances only (gdn2_internal.cuh)
    BwdFactors bw;           // kBw instances: the backward's per-chunk factors
};

struct TcMaps {
    CUtensorMap q, k, v, b, w, g, o;
    CUtensorMap kt, wt, mt, tm, pm;  // kBw: stores of the backward's factors (2-D, 128-byte swizzle)
    CUtensorMap st;                  // kBw: stores of the chunk-boundary states, 64 columns x 128 rows
};

// barrier over `count` threads (id 0 is __syncthreads)
__device__ __forceinline__ void named_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// bf16x2 product, rounded to nearest even
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// logistic sigmoid through the tanh unit: 1 / (1 + e^-x) = (1 + tanh(x / 2)) / 2,
// on a bf16x2 pair: the tanh unit's bf16x2 form, then 1/2 + t/2 as one bf16x2 fma (x/2 is exact)
__device__ __forceinline__ uint32_t sigmoid_bf16x2(uint32_t x)
{
    const uint32_t half2 = 0x3f003f00u;  // (0.5, 0.5) in bf16
    uint32_t h, t, r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(h) : "r"(x), "r"(half2));
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(h));
    asm("fma.rn.bf16x2 %0, %1, %2, %2;" : "=r"(r) : "r"(t), "r"(half2));
    return r;
}

// Sum over the 32 lanes of each of 16 per-lane values v[0..15], by halving exchanges (16
// shuffles instead of 80): on return lanes 2i and 2i + 1 hold the total of value i in v[0].
__device__ __forceinline__ void lane_sum16(float (&v)[16], int lane)
{
#pragma unroll
    for (int m = 16, n = 8; m >= 2; m >>= 1, n >>= 1) {
        const bool up = lane & m;
#pragma unroll
        for (int j = 0; j < n; ++j) {
            const float send = up ? v[j] : v[j + n];
            const float keep = up ? v[j + n] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// kGScalar: log alpha is one value per (token, head) (TcParams::g_scalar).
// DIN: the head size of the tensors, 128 or 64.  A d = 64 head runs as a d = 128 head
// whose channels 64..127 are zero: the TMA boxes past the tensors' channel extent are
// zero-filled, so k, q, b, v and w vanish there, the state's extra rows and columns stay
// zero, and only the first 64 channels of o, S_T are stored.
// kPro: the fused input prologue (kProNorm | kProSigmoid of gdn2_internal.cuh).  With
// normalised q_n = R_q q, k_n = R_k k (R = Diag of the per-token reciprocal norms) the chunk
// step keeps the raw-key factors and moves the scales.  The normalised A is R_k A R_k, and
// (I + R_k A R_k)^-1 = R_k^-1 (I + R_k^2 A)^-1 R_k, so with T'' = (I + R_k^2 A)^-1 (A's rows
// scaled at the readback) the product the state update K~^T U' and P U' both take is
// U' = R_k U~_n = T'' (R_k X - R_k^2 E~ S); the output is O = R_q (Q~ S + P U').  The
// squares come from the decay folding's loads; the reduction over the lanes runs while the
// [A; P] product is in flight.  The sigmoid of b is applied in the decay folding, that of w
// in the X = w.v fold.
// kGate: b and w are one value per (token, head) (the KDA and Gated DeltaNet shapes): no b, w
// tiles; E folds E~ = (b_t k) e^G with b_t from a 64-entry table per chunk, M forms X = w_t v.
// kBw: the states run of the backward, which also writes the backward's per-chunk factors
// (BwdFactors) from the M group, whose products leave it time while E prepares the next chunk.
// kScan: a pass of the chunk-parallel scan (ScanArgs): every CTA decodes its segment, its state
// source and destination, whether it writes o, and whether it runs the transition (the
// chain's linear part on the identity: X = 0, S = I at the segment start).
template <bool kGScalar, int DIN, int kPro, bool kScan = false, bool kBw = false, bool kGate = false>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    // Offset (not integer-cast) so that the compiler keeps the shared address space and
    // emits shared-memory instructions for every access through `sm`.
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    // bar_in[2]: a chunk's k, b, q have landed (E)       bar_vw[2]: its v, w have landed (M)
    // bar_emma / bar_mma: E's / M's tcgen05 batches      bar_fact[2]: E -> M, factors, P and T of a chunk
    // bar_qk[2]: M -> E, M no longer reads a chunk's E~, Q~, K~ tiles
    // bar_mdone[2]: M -> E, M is done with a chunk (its X, T / P tiles, w and per-parity values are free)
    __shared__ __align__(8) uint64_t bar_in[2], bar_vw[2], bar_emma, bar_mma, bar_fact[2], bar_qk[2], bar_mdone[2];
    __shared__ __align__(8) uint64_t bar_tfree;  // M -> E: M has read T (fp32) of the last chunk
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort_m, s_abort_e;
    // E -> M with a chunk's factors: [parity][channel half] some channel of the chunk decays past
    // kChunkDecayLimit, so the chunk runs token by token
    __shared__ int s_tok[2][2];
    __shared__ float *s_stp;  // this CTA's end-state destination (read once, at the end)
    __shared__ uint32_t s_bsc[2][kGate ? 64 : 1];  // kGate: (b_t, b_t) bf16x2 of the chunk, by chunk parity

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool is_m = warp < 8;
    const int bh = blockIdx.x, bb = bh / p.H, hh = bh % p.H;
    int bos = bb * p.T, T = p.T;  // this sequence's first token row and its length
    const float *S0p = p.S0 ? p.S0 + (size_t)bh * DIN * DIN : nullptr;  // this CTA's start state
    float *STp = p.S_T ? p.S_T + (size_t)bh * DIN * DIN : nullptr;     // and its end state
    bool o_on = p.o != nullptr, trans = false;
    if (kScan) {
        const ScanArgs &sc = p.scan;
        const int u = bh / p.H, mid = sc.nseg - 2;
        int b, sg;
        if (sc.pass == 0 && u < p.B) {  // segment 0, from S0, with its output
            b = u;
            sg = 0;
            STp = sc.send0 + ((size_t)b * p.H + hh) * DIN * DIN;
        } else if (sc.pass == 0) {  // a middle segment: local end state (even) or transition (odd)
            const int v = u - p.B, pair = v >> 1;
            b = pair / mid;
            sg = 1 + pair % mid;
            trans = v & 1;
            S0p = nullptr;
            STp = (trans ? sc.phi : sc.shat) + (((size_t)b * mid + sg - 1) * p.H + hh) * DIN * DIN;
            o_on = false;
        } else {  // segments 1 .. nseg-1 from their start states; the last one gives S_T
            b = u / (sc.nseg - 1);
            sg = 1 + u % (sc.nseg - 1);
            S0p = sc.sstart + (((size_t)b * (sc.nseg - 1) + sg - 1) * p.H + hh) * DIN * DIN;
            STp = (sg == sc.nseg - 1 && p.S_T) ? p.S_T + ((size_t)b * p.H + hh) * DIN * DIN : nullptr;
        }
        const int start = sg == 0 ? 0 : sc.seg0_len + (sg - 1) * sc.seg_len;
        bos = b * p.T + start;
        T = max(0, min(sg == 0 ? sc.seg0_len : sc.seg_len, p.T - start));
    }
    if (p.cu_seqlens) {
        const int b0 = p.cu_seqlens[bb], b1 = p.cu_seqlens[bb + 1];
        if (b0 < 0 || b1 < b0 || b1 > p.T) {  // nothing launched yet: leave before any barrier
            if (tid == 0) atomicExch(p.status, kStatusBadSeqlens);
            return;
        }
        bos = b0;
        T = b1 - b0;
    }
    const int nchunks = (T + C - 1) / C;
    const uint32_t sbase = smem_u32(sm);
    float *sA = reinterpret_cast<float *>(sm + OFF_SA);
    float *sT = reinterpret_cast<float *>(sm + OFF_ST);
    float *sTot = reinterpret_cast<float *>(sm + OFF_TOT);
    float *sGam = reinterpret_cast<float *>(sm + OFF_GAM);
    float *sNrm = reinterpret_cast<float *>(sm + OFF_NRM);  // [q|k][channel half][64]
    float *sRn = reinterpret_cast<float *>(sm + OFF_RN);    // [parity][q|k][64]

    if (tid == 0) {
        s_abort_m = 0;
        s_abort_e = 0;
        s_stp = STp;
        mbar_init(&bar_emma, 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_tfree, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_in[i], 1);
            mbar_init(&bar_vw[i], 1);
            mbar_init(&bar_qk[i], 1);
            mbar_init(&bar_fact[i], 1);
            mbar_init(&bar_mdone[i], 1);
        }
        fence_mbar_init();
        prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.v);
        prefetch_tmap(&maps.b); prefetch_tmap(&maps.w);
        if (!kGScalar) prefetch_tmap(&maps.g);  // a scalar decay has no tensor map
        if (p.o) prefetch_tmap(&maps.o);
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, TM_COLS);
        tmem_relinquish();
    }
    // T's strictly-upper blocks stay zero for the whole kernel
    for (int idx = tid; idx < 64 * LDA; idx += kThreads) sT[idx] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // TMA loads of chunk ci into the buffers of parity ci & 1 as they free up: k, b, q (E's inputs,
    // bar_in) once M's products no longer read the chunk two back (bar_qk: at its state update in
    // the plain forward), and v, w (M's, bar_vw) with log alpha into L2 once M is done with the
    // chunk before (bar_mdone; w is single-buffered and folded into X at the end of a chunk).  The
    // issuing thread may block while the TMA engine drains earlier boxes, so after the first two
    // chunks the loads go out from an E warp that is idle during the solve.
    auto issue_qbk = [&](int ci) {
        const int y = bos + ci * C, bf = ci & 1;
        fence_proxy_async_smem();
        mbar_expect_tx(&bar_in[bf], (kGate ? 4 : 6) * 8192);
        for (int a = 0; a < 2; ++a) {
            tma_load_3d(sm + OFF_K + bf * 16384 + a * 8192, &maps.k, a * 64, hh, y, &bar_in[bf]);
            if (!kGate) tma_load_3d(sm + OFF_QE + bf * 32768 + a * 16384, &maps.b, a * 64, hh, y, &bar_in[bf]);
            tma_load_3d(sm + OFF_QE + bf * 32768 + 8192 + a * 16384, &maps.q, a * 64, hh, y, &bar_in[bf]);
        }
    };
    auto issue_vw = [&](int ci) {
        const int y = bos + ci * C, bf = ci & 1;
        fence_proxy_async_smem();
        mbar_expect_tx(&bar_vw[bf], (kGate ? 2 : 4) * 8192);
        for (int a = 0; a < 2; ++a) {
            tma_load_3d(sm + OFF_V + bf * 16384 + a * 8192, &maps.v, a * 64, hh, y, &bar_vw[bf]);
            if (!kGate) tma_load_3d(sm + OFF_W + a * 8192, &maps.w, a * 64, hh, y, &bar_vw[bf]);
        }
        if (!kGScalar)
            for (int a = 0; a < DIN / 32; ++a) tma_prefetch_3d(&maps.g, a * 32, hh, y);
        if (kGate) {  // the chunk's rows of b and w ([rows, H], contiguous) into L2
            const int rows = min(C, T - ci * C);
            const uint32_t bytes = (uint32_t)(rows * p.H * 2) & ~15u;
            const size_t first = (size_t)y * p.H;
            if (bytes && ((first * 2) & 15) == 0) {
                bulk_prefetch_l2(p.b + first, bytes);
                bulk_prefetch_l2(p.w + first, bytes);
            }
        }
    };

    if (is_m) {
        // =========================== M group: the state chain of chunk ci ===========================
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegM) : "memory");
        const int mw = warp, quarter = mw & 3, half = mw >> 2;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const int jrow = quarter * 32 + lane;  // d_v index of this thread's S^T row
        auto fail = [&]() {
            s_abort_m = 1;
            atomicExch(p.status, kStatusTimeout);
        };
        // kGate: w_t of this warp's eight token rows (mw + 8 j) of a chunk, loaded one chunk ahead
        __nv_bfloat16 w_next[8];
        auto load_w = [&](int ci) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = mw + 8 * j;
                w_next[j] = (kGate && ci < nchunks && ci * C + t < T)
                                ? p.w[((size_t)bos + (size_t)ci * C + t) * p.H + hh]
                                : __float2bfloat16_rn(0.f);
            }
        };
        // X = w.v of chunk ci, in place of v (one token row of 64 channels per warp step)
        auto fold_value = [&](int ci) {
            if (kScan && trans) return;  // X = 0
            const int Lc = min(C, T - ci * C);
            uint8_t *pv = sm + OFF_V + (ci & 1) * 16384;
            const uint8_t *pw = sm + OFF_W;
#pragma unroll
            for (int it = 0; it < 2 * C / 8; ++it) {  // (atom, token) rows, one per warp step
                const int idx = mw + 8 * it;
                const int a = idx >> 6, t = idx & 63;
                const uint32_t off = a * 8192 + sw128(t, 4 * lane);
                const uint32_t vw = *reinterpret_cast<const uint32_t *>(pv + off);
                uint32_t ww;
                if (kGate) {  // one w per (token, head), the same for the whole row
                    const uint32_t w16 = (uint32_t)__bfloat16_as_ushort(w_next[it & 7]);
                    ww = w16 | (w16 << 16);
                } else {
                    ww = *reinterpret_cast<const uint32_t *>(pw + off);
                }
                const uint32_t wg = (kPro & kProSigmoid) ? sigmoid_bf16x2(ww) : ww;
                *reinterpret_cast<uint32_t *>(pv + off) = (t < Lc) ? bmul2(vw, wg) : 0u;
            }
        };
        if (kGate) load_w(0);
        if (tid == 0 && nchunks > 0) {
            issue_qbk(0);
            issue_vw(0);
            if (nchunks > 1) issue_qbk(1);
        }
        if (nchunks > 0) {
            if (!mbar_wait(&bar_vw[0], 0)) fail();
            fold_value(0);
        }
        fence_proxy_async_smem();
        named_sync(1, kGroup);
        if (tid == 0 && nchunks > 1) issue_vw(1);  // w(1) may only land after w(0) was folded
        // bf16 copy of this thread's 64 entries of S^T at chunk boundary `idx`
        auto store_state = [&](const float *Sv, int idx) {
            const size_t first = p.chunk_off ? (size_t)p.chunk_off[bb] : (size_t)bb * nchunks;
            const size_t slot = (first + bb) * p.H + (size_t)hh * (nchunks + 1) + idx;
            uint4 *dst = reinterpret_cast<uint4 *>(p.states + (slot * D + jrow) * D + 64 * half);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                dst[u] = make_uint4(pack_bf16x2(Sv[8 * u], Sv[8 * u + 1]), pack_bf16x2(Sv[8 * u + 2], Sv[8 * u + 3]),
                                    pack_bf16x2(Sv[8 * u + 4], Sv[8 * u + 5]), pack_bf16x2(Sv[8 * u + 6], Sv[8 * u + 7]));
        };
        // kBw: this thread's row of the bf16 S^T into a [128 rows][64 columns] staging tile (128-byte
        // swizzle, as the TMA store of maps.st reads it); the two column halves go out one after
        // the other through the same tile
        auto stage_state = [&](const float *Sv, uint8_t *tile) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4 *>(tile + sw128(jrow, 16 * u)) =
                    make_uint4(pack_bf16x2(Sv[8 * u], Sv[8 * u + 1]), pack_bf16x2(Sv[8 * u + 2], Sv[8 * u + 3]),
                               pack_bf16x2(Sv[8 * u + 4], Sv[8 * u + 5]), pack_bf16x2(Sv[8 * u + 6], Sv[8 * u + 7]));
        };
        // first chunk of this sequence over all sequences (the backward's per-chunk slots)
        const size_t bw_first = p.chunk_off ? (size_t)p.chunk_off[bb] : (size_t)bb * nchunks;
        // row of maps.st where the state at chunk boundary idx starts
        auto state_row = [&](int idx) { return (int)(((bw_first + bb) * p.H + (size_t)hh * (nchunks + 1) + idx) * D); };
        float Sf[64];  // S^T[jrow][64 half + i]
#pragma unroll
        for (int i = 0; i < 64; ++i)
            Sf[i] = (kScan && trans) ? ((64 * half + i == jrow && jrow < DIN) ? 1.f : 0.f)
                    : (S0p && 64 * half + i < DIN && jrow < DIN) ? S0p[(64 * half + i) * DIN + jrow] : 0.f;
        if (p.states) store_state(Sf, 0);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(Sf[32 * h2 + 2 * e], Sf[32 * h2 + 2 * e + 1]);
            tmem_st16(tmem + TM_SBF + 32 * half + 16 * h2 + lane_off, pk);
        }
        tmem_wait_st();
        if (kBw) {  // the 64 x 64 identity (B operand, 128-byte swizzle) of M^T = Q~^T I - W^T P^T
            for (int c = tid; c < 64 * 8; c += kGroup) {
                const int r = c >> 3, k8 = c & 7;
                const uint32_t one = (r >> 3) != k8 ? 0u : (r & 1) ? 0x3f800000u : 0x00003f80u, wi = (r & 7) >> 1;
                *reinterpret_cast<uint4 *>(sm + OFF_ID + sw128(r, 16 * k8)) =
                    make_uint4(wi == 0 ? one : 0u, wi == 1 ? one : 0u, wi == 2 ? one : 0u, wi == 3 ? one : 0u);
            }
            fence_proxy_async_smem();
        }
        tc_fence_before();
        named_sync(1, kGroup);
        uint32_t mma_phase = 0;
        bool qk_sent = false;  // thread 0: bar_qk of this chunk already signalled
        for (int ci = 0; ci < nchunks; ++ci) {
            const int buf = ci & 1;
            const int L = min(C, T - ci * C);
            const uint32_t oqe = OFF_QE + buf * 32768, ok = OFF_K + buf * 16384, ov = OFF_V + buf * 16384;
            const uint32_t ott = OFF_TP + buf * 16384, opt = ott + 8192;
            if (kGate) load_w(ci + 1);  // in flight during the chunk
            // ---- factors, P and T of chunk ci are ready
            if (!mbar_wait(&bar_fact[buf], (ci >> 1) & 1)) fail();
            if (s_tok[buf][0] | s_tok[buf][1]) {
                if (tid == 0) mbar_arrive(&bar_tfree);  // T is not needed
                // ---- the chunk token by token (its decay is too strong for the factors, whose
                //      products E formed all the same): q, k, b from global memory (E folded the
                //      tiles in place), X = w.v from its tile; records and exchange buffers over this
                //      parity's T / P tiles, which M alone reads from here on
                tok::Rec<128> *recs = reinterpret_cast<tok::Rec<128> *>(sm + ott);
                float *xch = reinterpret_cast<float *>(sm + ott + 3 * sizeof(tok::Rec<128>));
                const uint8_t *pxt = sm + ov;
                const __nv_bfloat16 *gq = p.q, *gk = p.k, *gb = p.b;
                const float *rqn = sRn + (buf * 2) * 64, *rkn = sRn + (buf * 2 + 1) * 64;
                const size_t row0 = (size_t)bos + (size_t)ci * C;
                auto fill = [&](int t, tok::Rec<128> &r) {
                    if (tid < 128) {
                        const int c = tid;
                        float qv = 0.f, kv = 0.f, bv = 0.f, gv = 0.f;
                        if (c < DIN) {
                            const size_t off = ((row0 + t) * p.H + hh) * DIN + c;
                            qv = __bfloat162float(gq[off]);
                            kv = __bfloat162float(gk[off]);
                            bv = __bfloat162float(kGate ? gb[(row0 + t) * p.H + hh] : gb[off]);
                            gv = kGScalar ? p.g[(row0 + t) * p.H + hh] : p.g[off];
                        }
                        if (kPro & kProNorm) {
                            qv *= rqn[t];
                            kv *= rkn[t];
                        }
                        if (kPro & kProSigmoid) bv = 1.f / (1.f + __expf(-bv));
                        r.q[c] = qv;
                        r.k[c] = kv;
                        r.e[c] = bv * kv;
                        r.a[c] = expf(gv);
                    } else {
                        const int jj = tid - 128;
                        r.x[jj] = (kScan && trans) ? 0.f
                                  : __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                                        pxt + (jj >> 6) * 8192 + sw128(t, (jj & 63) * 2)));
                    }
                };
                tok::fwd_tokens<128>(Sf, 0, L, recs, xch, jrow, half, 1, fill, [&](int s, float ov) {
                    if (o_on && half == 0 && jrow < DIN)
                        p.o[((row0 + s) * p.H + hh) * DIN + jrow] = __float2bfloat16_rn(ov);
                });
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {  // the bf16 copy of S^T for the next chunk's products
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(Sf[32 * h2 + 2 * e], Sf[32 * h2 + 2 * e + 1]);
                    tmem_st16(tmem + TM_SBF + 32 * half + 16 * h2 + lane_off, pk);
                }
                tmem_wait_st();
                if (p.states) store_state(Sf, ci + 1);
                if (kBw && tid == 128) {  // the backward steps this chunk token by token too
                    const size_t cidx = bw_first * p.H + (size_t)hh * nchunks + ci;
                    reinterpret_cast<int *>(p.bw.gam + cidx * kGamStride)[D] = 1;
                    p.bw.flist[1 + atomicAdd(p.bw.flist, 1)] = (int)(bw_first + ci + p.bw.nchb * hh);
                }
                tc_fence_before();
                named_sync(1, kGroup);
            } else {
            // ---- MMA 1: [S^T E~^T | O^T] = S^T [E~; Q~]^T
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(tmem + TM_YO, tmem + TM_SBF + 8 * ks,
                           sdesc_sw128(sbase + oqe + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), IDESC_N128, ks > 0);
                mma_commit(&bar_mma);
            }
            {  // while MMA 1 runs: T (fp32, from E's solve) -> bf16 rows i of 64 j, zero above the diagonal
                const int i = tid >> 2, q4 = tid & 3;
                uint32_t w8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j0 = 16 * q4 + 2 * e;
                    const float lo = (j0 <= i) ? sT[i * LDA + j0] : 0.f;
                    const float hi = (j0 + 1 <= i) ? sT[i * LDA + j0 + 1] : 0.f;
                    w8[e] = pack_bf16x2(lo, hi);
                }
                *reinterpret_cast<uint4 *>(sm + ott + sw128(i, 32 * q4)) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
                *reinterpret_cast<uint4 *>(sm + ott + sw128(i, 32 * q4 + 16)) = make_uint4(w8[4], w8[5], w8[6], w8[7]);
                fence_proxy_async_smem();
            }
            if (!mbar_wait(&bar_mma, mma_phase)) fail();
            mma_phase ^= 1;
            tc_fence_after();
            {  // Y^T = X^T - S^T E~^T -> bf16 TMEM operand (this warp: 32 tokens)
                const uint8_t *px = sm + ov + (jrow >> 6) * 8192;
                const uint32_t xb = (jrow & 63) * 2;
                const float *rk = sRn + (buf * 2 + 1) * 64;
                uint32_t r[32];
                tmem_ld32(tmem + TM_YO + 32 * half + lane_off, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int t = 32 * half + 2 * e;
                    float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(px + sw128(t, xb)));
                    float x1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(px + sw128(t + 1, xb)));
                    if (kScan && trans) x0 = x1 = 0.f;
                    const float a0 = __uint_as_float(r[2 * e]), a1 = __uint_as_float(r[2 * e + 1]);
                    if (kPro & kProNorm) {  // R_k X - R_k^2 E~ S
                        const float r0 = rk[t], r1 = rk[t + 1];
                        pk[e] = pack_bf16x2(r0 * (x0 - r0 * a0), r1 * (x1 - r1 * a1));
                    } else {
                        pk[e] = pack_bf16x2(x0 - a0, x1 - a1);
                    }
                }
                tmem_st16(tmem + TM_YB + 16 * half + lane_off, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            named_sync(1, kGroup);
            if (tid == 0) mbar_arrive(&bar_tfree);  // every M thread has read T
            if (s_abort_m) break;
            // ---- MMA 2: U~^T = Y^T T^T
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ts(tmem + TM_UT, tmem + TM_YB + 8 * ks, sdesc_sw128(sbase + ott + ks * 32, 16, 1024), IDESC_N64,
                           ks > 0);
                mma_commit(&bar_mma);
            }
            if (!mbar_wait(&bar_mma, mma_phase)) fail();
            mma_phase ^= 1;
            tc_fence_after();
            {  // U~^T (U' with the prologue) -> bf16 TMEM operand
                uint32_t r[32];
                tmem_ld32(tmem + TM_UT + 32 * half + lane_off, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                tmem_st16(tmem + TM_UB + 16 * half + lane_off, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            named_sync(1, kGroup);
            if (s_abort_m) break;
            // ---- MMA 3: (K~^T U~)^T = U~^T K~ ;  O^T += U~^T P^T
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    mma_ts(tmem + TM_DS, tmem + TM_UB + 8 * ks, sdesc_sw128(sbase + ok + ks * 2048, 8192, 1024),
                           IDESC_N128_BMN, ks > 0);
                    if (o_on)
                        mma_ts(tmem + TM_O, tmem + TM_UB + 8 * ks, sdesc_sw128(sbase + opt + ks * 32, 16, 1024),
                               IDESC_N64, 1);
                }
                if (kBw) {  // the backward's W^T = E~^T T^T (d_k rows) into TM_UT, read back by now
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_ss(tmem + TM_UT, sdesc_sw128(sbase + oqe + ks * 2048, 16384, 1024),
                               sdesc_sw128(sbase + ott + ks * 32, 16, 1024), IDESC_W, ks > 0);
                }
                mma_commit(&bar_mma);
            }
            if (!mbar_wait(&bar_mma, mma_phase)) fail();
            mma_phase ^= 1;
            tc_fence_after();
            {  // S = gamma (S + K~^T U~) in fp32 registers; bf16 copy back to TMEM
                const float *gam = sGam + buf * 128 + 64 * half;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t r[32];
                    tmem_ld32(tmem + TM_DS + 64 * half + 32 * h2 + lane_off, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        Sf[32 * h2 + u] = gam[32 * h2 + u] * (Sf[32 * h2 + u] + __uint_as_float(r[u]));
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(Sf[32 * h2 + 2 * e], Sf[32 * h2 + 2 * e + 1]);
                    tmem_st16(tmem + TM_SBF + 32 * half + 16 * h2 + lane_off, pk);
                }
                // the chunk-end state (kBw): column half 0 through the consumed X tile now, half 1
                // once that store has read it
                if (kBw && half == 0) stage_state(Sf, sm + ov);
            }
            // the plain forward's products are done with this parity's E~, Q~ and K~ tiles (the
            // states run still stores factors from them): chunk ci+2's k, b, q may come in
            if (!kBw && tid == 0) {
                mbar_arrive(&bar_qk[buf]);
                qk_sent = true;
            }
            if (kBw) {
                // ---- the backward's per-chunk factors, state-independent: W^T, M^T = Q~^T - W^T P^T
                //      (the chain forms R^T = dO^T M from them), K~, T, P, gamma and the token-mode
                //      flag.  W^T goes over the consumed E~ tile and M^T over Q~ (128-byte swizzled, as
                //      TMA stores read them), and TMA stores take them and the K~, T, P tiles to global.
                //      TMEM lanes are d_k channels here (jrow), columns tokens.
                const BwdFactors &bw = p.bw;
                const size_t cidx = bw_first * p.H + (size_t)hh * nchunks + ci;
                uint8_t *const pe = sm + oqe, *const pq = sm + oqe + 8192, *const pkt = sm + ok;
                const int srow = state_row(ci + 1);
                const uint32_t arow = (jrow & 63), aoff = (jrow >> 6) * 16384;  // this row in a [128][64] E~ / Q~ tile
                {  // W^T -> bf16 into the E~ tile, and -W^T as the A operand of M's product
                    uint32_t r[32], pk[16], nk[16];
                    tmem_ld32(tmem + TM_UT + 32 * half + lane_off, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float w0 = __uint_as_float(r[2 * e]), w1 = __uint_as_float(r[2 * e + 1]);
                        pk[e] = pack_bf16x2(w0, w1);
                        nk[e] = pack_bf16x2(-w0, -w1);
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        *reinterpret_cast<uint4 *>(pe + aoff + sw128(arow, 64 * half + 16 * m)) =
                            make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
                    tmem_st16(tmem + TM_YB + 16 * half + lane_off, nk);
                    tmem_wait_st();
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_sync(1, kGroup);
                if (tid == 0) {  // M^T = Q~^T I + (-W^T) P^T into TM_YO's first half (free since the Y read-back)
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_ss(tmem + TM_YO, sdesc_sw128(sbase + oqe + 8192 + ks * 2048, 16384, 1024),
                               sdesc_sw128(sbase + OFF_ID + ks * 32, 16, 1024), IDESC_W, ks > 0);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_ts(tmem + TM_YO, tmem + TM_YB + 8 * ks, sdesc_sw128(sbase + opt + ks * 32, 16, 1024), IDESC_N64, 1);
                    mma_commit(&bar_mma);
                    // the stores: state columns 0-63 as a group of its own (its tile is refilled first)
                    tma_store_2d(&maps.st, sm + ov, 0, srow);
                    bulk_commit();
                    const int wrow = (int)(cidx * D), trow = (int)(cidx * C);
                    for (int a = 0; a < 2; ++a) {
                        tma_store_2d(&maps.wt, pe + a * 16384, 0, wrow + 64 * a);
                        tma_store_2d(&maps.kt, pkt + a * 8192, 64 * a, trow);
                    }
                    tma_store_2d(&maps.tm, sm + ott, 0, trow);
                    tma_store_2d(&maps.pm, sm + opt, 0, trow);
                    bulk_commit();
                }
                if (tid < 128) bw.gam[cidx * kGamStride + tid] = sGam[buf * 128 + tid];
                if (tid == 128) {
                    const int tokm = s_tok[buf][0] | s_tok[buf][1];
                    reinterpret_cast<int *>(bw.gam + cidx * kGamStride)[D] = tokm;
                    if (tokm) bw.flist[1 + atomicAdd(bw.flist, 1)] = (int)(bw_first + ci + bw.nchb * hh);
                }
                if (!mbar_wait(&bar_mma, mma_phase)) fail();
                mma_phase ^= 1;
                tc_fence_after();
                {  // M^T -> bf16 over the Q~ tile (the product has read it)
                    uint32_t r[32], pk[16];
                    tmem_ld32(tmem + TM_YO + 32 * half + lane_off, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        *reinterpret_cast<uint4 *>(pq + aoff + sw128(arow, 64 * half + 16 * m)) =
                            make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
                }
                if (tid == 0) bulk_wait_read1();  // state columns 0-63 have left their tile
                fence_proxy_async_smem();
                tc_fence_before();
                named_sync(1, kGroup);
                if (tid == 0) {
                    for (int a = 0; a < 2; ++a) tma_store_2d(&maps.mt, pq + a * 16384, 0, (int)(cidx * D) + 64 * a);
                    bulk_commit();
                    if (o_on) bulk_wait_read0();  // T and P are read before the output tile goes over them
                }
                if (half == 1) {  // state columns 64-127 through the same tile; thread 128 owns their store
                    stage_state(Sf, sm + ov);
                    fence_proxy_async_smem();
                    named_sync(4, kGroup / 2);
                    if (tid == kGroup / 2) {
                        tma_store_2d(&maps.st, sm + ov, 64, srow);
                        bulk_commit();
                    }
                }
                if (o_on) named_sync(1, kGroup);
            }
            if (o_on) {  // O^T -> bf16 output tile (row-major [t][channel]) over this chunk's T/P tiles
                uint32_t r[32];
                tmem_ld32(tmem + TM_O + 32 * half + lane_off, r);
                tmem_wait_ld();
                __nv_bfloat16 *so = reinterpret_cast<__nv_bfloat16 *>(sm + ott);
                if (jrow < DIN) {  // row-major [t][channel] with the tensors' head size as row length
                    const float *rq = sRn + (buf * 2) * 64 + 32 * half;
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const float ov_ = (kPro & kProNorm) ? __uint_as_float(r[u]) * rq[u] : __uint_as_float(r[u]);
                        so[(32 * half + u) * DIN + jrow] = __float2bfloat16_rn(ov_);
                    }
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(1, kGroup);
            if (o_on && L == C) {
                if (tid == 0) {
                    tma_store_3d(&maps.o, sm + ott, 0, hh, bos + ci * C);
                    bulk_commit();
                }
            } else if (o_on) {  // ragged last chunk: only the valid rows (the tile would spill into the next sequence)
                const __nv_bfloat16 *so = reinterpret_cast<const __nv_bfloat16 *>(sm + ott);
                __nv_bfloat16 *dst = p.o + ((size_t)bos + (size_t)ci * C) * p.H * DIN + (size_t)hh * DIN;
                for (int idx = tid; idx < L * DIN; idx += kGroup)
                    dst[(size_t)(idx / DIN) * p.H * DIN + idx % DIN] = so[idx];
                named_sync(1, kGroup);
            }
            }  // the chunkwise products
            // ---- next chunk's values (w is single-buffered), then chunk ci+2's loads into this parity
            if (ci + 1 < nchunks) {
                if (!mbar_wait(&bar_vw[buf ^ 1], ((ci + 1) >> 1) & 1)) fail();
                fold_value(ci + 1);
            }
            if (kBw && tid == kGroup / 2) bulk_wait_read0();  // the state columns 64-127 have left their tile
            if (tid == 0) bulk_wait_read0();                  // the output and factor stores have read their tiles
            fence_proxy_async_smem();
            named_sync(1, kGroup);
            if (tid == 0) {
                if (!qk_sent) mbar_arrive(&bar_qk[buf]);
                mbar_arrive(&bar_mdone[buf]);  // this chunk's tiles, w and per-parity values are free
            }
            qk_sent = false;
        }
        float *const st_dst = s_stp;
        if (!s_abort_m && st_dst) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
                if (64 * half + i < DIN && jrow < DIN) st_dst[(64 * half + i) * DIN + jrow] = Sf[i];
        }
        if (tid == 0 || (kBw && tid == kGroup / 2)) bulk_wait0();
    } else {
        // =========== E group: decay folding, [A; P] and T = (I+A)^-1, one chunk ahead of M ===========
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegE) : "memory");
        const int ew = warp - 8, etid = tid - kGroup;
        const int quarter = ew & 3, half = ew >> 2;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const int cb = ew & 1, tg = ew >> 1;  // elementwise: channel block of 64, token group of 16
        const int ch = 64 * cb + 2 * lane;
        auto fail = [&]() {
            s_abort_e = 1;
            atomicExch(p.status, kStatusTimeout);
        };
        // kGate: b_t of chunk c, one per thread of the first 64, loaded a chunk ahead of its table
        auto load_bt = [&](int c) -> __nv_bfloat16 {
            return (kGate && etid < 64 && c < nchunks && c * C + etid < T)
                       ? p.b[((size_t)bos + (size_t)c * C + etid) * p.H + hh]
                       : __float2bfloat16_rn(0.f);
        };
        __nv_bfloat16 bt_next = load_bt(0);
        for (int ci = 0; ci < nchunks; ++ci) {
            const int buf = ci & 1;
            const int L = min(C, T - ci * C);
            const uint32_t oqe = OFF_QE + buf * 32768, ok = OFF_K + buf * 16384;
            const uint32_t ott = OFF_TP + buf * 16384, opt = ott + 8192;
            const __nv_bfloat16 bt = bt_next;
            bt_next = load_bt(ci + 1);
            // log alpha of this warp's 16 tokens x 2 channels, straight from L2
            float2 gv[16];
            if (kGScalar) {  // one decay per (token, head), the same for both channels
                const float *gsrc = p.g + ((size_t)bos + (size_t)ci * C + 16 * tg) * p.H + hh;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float gs = (16 * tg + i < L) ? __ldg(gsrc + (size_t)i * p.H) : 0.f;
                    gv[i] = make_float2(gs, gs);
                }
            } else {
                const float *gsrc =
                    p.g + ((size_t)bos + (size_t)ci * C + 16 * tg) * p.H * DIN + (size_t)hh * DIN + ch;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    gv[i] = (16 * tg + i < L && ch < DIN)
                                ? __ldg(reinterpret_cast<const float2 *>(gsrc + (size_t)i * p.H * DIN))
                                : make_float2(0.f, 0.f);
            }
            if (!mbar_wait(&bar_in[buf], (ci >> 1) & 1)) fail();
            // M is done with chunk ci-2, whose T / P tiles and per-parity values this chunk reuses
            if (ci >= 2 && !mbar_wait(&bar_mdone[buf], ((ci - 2) >> 1) & 1)) fail();
            float run0 = 0.f, run1 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                run0 += gv[i].x;
                run1 += gv[i].y;
                const float a0 = __expf(gv[i].x);
                gv[i] = make_float2(a0, kGScalar ? a0 : __expf(gv[i].y));  // alpha
            }
            *reinterpret_cast<float2 *>(sTot + tg * 128 + ch) = make_float2(run0, run1);
            if (kGate && etid < 64) {
                const uint32_t b16 = (uint32_t)__bfloat16_as_ushort(bt);
                s_bsc[buf][etid] = b16 | (b16 << 16);
            }
            named_sync(2, kGroup);
            if (s_abort_e) break;
            float sqq[16], sqk[16];  // prologue: this thread's share of |q|^2, |k|^2 per token
            {  // decay folding, in place
                float c0 = 0.f, c1 = 0.f, gl0 = 0.f, gl1 = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 tv = *reinterpret_cast<const float2 *>(sTot + u * 128 + ch);
                    if (u < tg) { c0 += tv.x; c1 += tv.y; }
                    gl0 += tv.x;
                    gl1 += tv.y;
                }
                if (tg == 0) {  // warps 8 and 9: gamma, and whether e^{-G} stays in range on every channel
                    *reinterpret_cast<float2 *>(sGam + buf * 128 + ch) = make_float2(__expf(gl0), __expf(gl1));
                    const bool out_of_range = __any_sync(0xffffffffu, gl0 < -kChunkDecayLimit || gl1 < -kChunkDecayLimit);
                    if (lane == 0) s_tok[buf][cb] = out_of_range;
                }
                uint8_t *pe = sm + oqe + cb * 16384;
                uint8_t *pq = pe + 8192;
                uint8_t *pk = sm + ok + cb * 8192;
                float2 mv[16];  // e^-G of each token: backwards from the group's last token
                {
                    float r0 = __expf(-(c0 + run0)), r1 = kGScalar ? r0 : __expf(-(c1 + run1));
#pragma unroll
                    for (int i = 15; i >= 0; --i) {
                        mv[i] = make_float2(r0, r1);
                        r0 *= gv[i].x;
                        r1 *= gv[i].y;
                    }
                }
                float e0 = __expf(c0), e1 = kGScalar ? e0 : __expf(c1);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = 16 * tg + i;
                    const uint32_t off = sw128(t, 4 * lane);
                    e0 *= gv[i].x;
                    e1 *= gv[i].y;
                    const float m0 = mv[i].x, m1 = mv[i].y;
                    uint32_t qw = *reinterpret_cast<const uint32_t *>(pq + off);
                    uint32_t kw = *reinterpret_cast<const uint32_t *>(pk + off);
                    uint32_t bw;
                    if (kGate) {
                        bw = s_bsc[buf][t];
                    } else {
                        bw = *reinterpret_cast<const uint32_t *>(pe + off);
                    }
                    if (t >= L) { qw = 0u; kw = 0u; bw = 0u; }
                    if (kPro & kProNorm) {
                        const float q0 = __uint_as_float(qw << 16), q1 = __uint_as_float(qw & 0xffff0000u);
                        const float k0 = __uint_as_float(kw << 16), k1 = __uint_as_float(kw & 0xffff0000u);
                        sqq[i] = fmaf(q0, q0, q1 * q1);
                        sqk[i] = fmaf(k0, k0, k1 * k1);
                    }
                    const uint32_t e01 = pack_bf16x2(e0, e1), m01 = pack_bf16x2(m0, m1);
                    if (kPro & kProSigmoid) bw = sigmoid_bf16x2(bw);  // kw is 0 past the sequence end
                    *reinterpret_cast<uint32_t *>(pq + off) = bmul2(qw, e01);
                    *reinterpret_cast<uint32_t *>(pe + off) = bmul2(bmul2(bw, kw), e01);
                    *reinterpret_cast<uint32_t *>(pk + off) = bmul2(kw, m01);
                }
            }
            fence_proxy_async_smem();
            named_sync(2, kGroup);
            // ---- [A; P] = [E~; Q~] K~^T on the tensor core
            if (etid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(tmem + TM_AP, sdesc_sw128(sbase + oqe + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                           sdesc_sw128(sbase + ok + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), IDESC_N64, ks > 0);
                mma_commit(&bar_emma);
            }
            if (kPro & kProNorm) {  // while the product runs: |q|^2, |k|^2 of this chunk's tokens
                lane_sum16(sqq, lane);
                lane_sum16(sqk, lane);
                if (!(lane & 1)) {
                    sNrm[cb * 64 + 16 * tg + (lane >> 1)] = sqq[0];
                    sNrm[(2 + cb) * 64 + 16 * tg + (lane >> 1)] = sqk[0];
                }
                named_sync(2, kGroup);
            }
            if (!mbar_wait(&bar_emma, ci & 1)) fail();
            tc_fence_after();
            {  // A -> fp32 scratch (strictly lower), P -> bf16 operand rows (lower incl.)
                uint32_t r[32];
                tmem_ld32(tmem + TM_AP + 32 * half + lane_off, r);
                tmem_wait_ld();
                const int row = quarter * 32 + lane;
                float rr2 = 1.f;  // prologue: 1/|k_row|^2 (A rows)
                if (kPro & kProNorm) {
                    const int which = row < 64 ? 1 : 0, t = row & 63;
                    const float n2 = sNrm[(which * 2) * 64 + t] + sNrm[(which * 2 + 1) * 64 + t] + kNormEps;
                    rr2 = __frcp_rn(n2);
                    if (half == 0) sRn[(buf * 2 + which) * 64 + t] = rsqrtf(n2);  // for M: 1/|k|, 1/|q|
                }
                if (row < 64) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int j = 32 * half + u;
                        const float av = (kPro & kProNorm) ? __uint_as_float(r[u]) * rr2 : __uint_as_float(r[u]);
                        sA[row * LDA + j] = (j < row) ? av : 0.f;
                    }
                } else {
                    const int t = row - 64;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i0 = 32 * half + 8 * m + 2 * e;
                            const float lo = (i0 <= t) ? __uint_as_float(r[8 * m + 2 * e]) : 0.f;
                            const float hi = (i0 + 1 <= t) ? __uint_as_float(r[8 * m + 2 * e + 1]) : 0.f;
                            w4[e] = pack_bf16x2(lo, hi);
                        }
                        *reinterpret_cast<uint4 *>(sm + opt + sw128(t, 64 * half + 16 * m)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            tc_fence_before();
            named_sync(2, kGroup);
            if (s_abort_e) break;
            // ---- T = (I + A)^-1 on warps 8-11: diagonal 16x16 blocks, then the doubling levels on
            //      warp-level TF32 MMAs
            if (ew < 4) {
                // M converts the last chunk's T to bf16 from sT: wait until it has
                if (ci >= 1 && !mbar_wait(&bar_tfree, (ci - 1) & 1)) fail();
                wm::solve_unit_lower64<LDA>(sA, sT, ew, lane, [] { named_sync(3, 128); });
            } else if (ew == 4 && lane == 0 && ci >= 1 && ci + 1 < nchunks) {
                // chunk ci+1's loads go to the buffers chunk ci-1 used
                if (!mbar_wait(&bar_qk[buf ^ 1], ((ci - 1) >> 1) & 1)) fail();
                issue_qbk(ci + 1);
                if (!mbar_wait(&bar_mdone[buf ^ 1], ((ci - 1) >> 1) & 1)) fail();
                issue_vw(ci + 1);
            }
            named_sync(2, kGroup);
            if (etid == 0) mbar_arrive(&bar_fact[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
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

// 3-D view (channel, head, token) of a [B,T,H,din] tensor.  Loads: box = (one 128-byte
// row of channels, 1 head, 64 tokens) with the 128-byte swizzle (a box past the channel
// extent reads zeros); the output store: box = (all din channels, 1, 64 tokens), no swizzle.
bool make_map(CUtensorMap *m, const void *ptr, bool fp32, int B, int T, int H, int din, bool store)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t es = fp32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)din, (cuuint64_t)H, (cuuint64_t)B * (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)din * es, (cuuint64_t)H * din * es};
    cuuint32_t box[3] = {store ? (cuuint32_t)din : (fp32 ? 32u : 64u), 1u, (cuuint32_t)kChunk};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               store ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D view of a row-major bf16 matrix [rows][cols]: box = (box_cols, box_rows) with the 128-byte
// swizzle (box_cols * 2 must be 128).
bool make_map_2d(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc || box_cols * 2 != 128 || box_rows == 0 || box_rows > 256) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_fwd_tc(const Problem &pr, void *o, float *S_T, __nv_bfloat16 *states, int *status,
                          cudaStream_t s, const ScanArgs *scan, const BwdFactors *bw)
{
    // d = 64 runs zero-padded to 128 (see the kernel); chunk-boundary states keep the padded
    // 128 x 128 layout (they are the backward's internal workspace)
    if (pr.D != 128 && pr.D != 64) return cudaErrorNotSupported;
    const int din = pr.D;
    TcMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int rows = (int)token_rows(pr);  // the maps view every tensor as [rows, H, din]
    if (!make_map(&maps.q, pr.q, false, 1, rows, pr.H, din) || !make_map(&maps.k, pr.k, false, 1, rows, pr.H, din) ||
        !make_map(&maps.v, pr.v, false, 1, rows, pr.H, din) ||
        (!pr.bw_scalar && !make_map(&maps.b, pr.b, false, 1, rows, pr.H, din)) ||
        (!pr.bw_scalar && !make_map(&maps.w, pr.w, false, 1, rows, pr.H, din)) ||
        (!pr.g_scalar && !make_map(&maps.g, pr.g, true, 1, rows, pr.H, din)) ||
        (o && !make_map(&maps.o, o, false, 1, rows, pr.H, din, true)))
        return cudaErrorInvalidValue;
    TcParams prm{pr.B, pr.T, pr.H, (const __nv_bfloat16 *)pr.q, (const __nv_bfloat16 *)pr.k, (const __nv_bfloat16 *)pr.b,
                 (const __nv_bfloat16 *)pr.w, pr.S0, pr.g, (__nv_bfloat16 *)o, S_T, states, status, pr.cu_seqlens, pr.chunk_off,
                 pr.g_scalar ? 1 : 0, ScanArgs{}, BwdFactors{}};
    if (bw) {  // the backward's factors: states runs without the prologue only
        if (!states || pr.prologue || scan) return cudaErrorInvalidValue;
        prm.bw = *bw;
        const uint64_t nchunk = (uint64_t)pr.H * chunk_bound(pr);
        const uint64_t state_rows = (uint64_t)pr.H * (chunk_bound(pr) + pr.B) * D;  // TMA coordinates are 32-bit
        if (state_rows > (uint64_t)INT_MAX ||
            !make_map_2d(&maps.kt, bw->Kt, D, nchunk * C, 64, C) || !make_map_2d(&maps.wt, bw->W, C, nchunk * D, 64, 64) ||
            !make_map_2d(&maps.mt, bw->Mc, C, nchunk * D, 64, 64) || !make_map_2d(&maps.tm, bw->Tm, C, nchunk * C, 64, C) ||
            !make_map_2d(&maps.pm, bw->Pm, C, nchunk * C, 64, C) || !make_map_2d(&maps.st, states, D, state_rows, 64, D))
            return cudaErrorInvalidValue;
    }
    int grid = pr.B * pr.H;
    if (scan) {  // plain gates, fixed length, no prologue; one CTA per (segment task, head)
        if (pr.g_scalar || pr.bw_scalar || pr.prologue || pr.cu_seqlens || states || scan->nseg < 3 || scan->seg_len % C ||
            scan->seg0_len % C)
            return cudaErrorInvalidValue;
        prm.scan = *scan;
        grid = (scan->pass == 0 ? pr.B * (1 + 2 * (scan->nseg - 2)) : pr.B * (scan->nseg - 1)) * pr.H;
    }
    auto run = [&](auto kernel) -> cudaError_t {
        cudaError_t e = set_smem_attr(reinterpret_cast<const void *>(kernel), (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        kernel<<<grid, kThreads, SMEM_BYTES, s>>>(maps, prm);
        return cudaGetLastError();
    };
    using T1 = std::true_type;
    using F1 = std::false_type;
    using D128 = std::integral_constant<int, 128>;
    using D64 = std::integral_constant<int, 64>;
    if (scan) return din == 128 ? run(fwd_tc_kernel<false, 128, 0, true>) : run(fwd_tc_kernel<false, 64, 0, true>);
    if (bw) {  // a scalar decay, and scalar erase and write gates, read as they are
        auto by_gate = [&](auto gs, auto dn) -> cudaError_t {
            constexpr bool kGS = decltype(gs)::value;
            constexpr int kDin = decltype(dn)::value;
            if (pr.bw_scalar) return run(fwd_tc_kernel<kGS, kDin, 0, false, true, true>);
            return run(fwd_tc_kernel<kGS, kDin, 0, false, true>);
        };
        if (din == 128) return pr.g_scalar ? by_gate(T1{}, D128{}) : by_gate(F1{}, D128{});
        return pr.g_scalar ? by_gate(T1{}, D64{}) : by_gate(F1{}, D64{});
    }
    if (pr.prologue & ~(kProNorm | kProSigmoid)) return cudaErrorInvalidValue;
    auto by_pro = [&](auto gs, auto dn) -> cudaError_t {
        constexpr bool kGS = decltype(gs)::value;
        constexpr int kDin = decltype(dn)::value;
        if (pr.bw_scalar) {
            switch (pr.prologue) {
            case kProNorm: return run(fwd_tc_kernel<kGS, kDin, kProNorm, false, false, true>);
            case kProSigmoid: return run(fwd_tc_kernel<kGS, kDin, kProSigmoid, false, false, true>);
            case kProNorm | kProSigmoid: return run(fwd_tc_kernel<kGS, kDin, kProNorm | kProSigmoid, false, false, true>);
            default: return run(fwd_tc_kernel<kGS, kDin, 0, false, false, true>);
            }
        }
        switch (pr.prologue) {
        case kProNorm: return run(fwd_tc_kernel<kGS, kDin, kProNorm>);
        case kProSigmoid: return run(fwd_tc_kernel<kGS, kDin, kProSigmoid>);
        case kProNorm | kProSigmoid: return run(fwd_tc_kernel<kGS, kDin, kProNorm | kProSigmoid>);
        default: return run(fwd_tc_kernel<kGS, kDin, 0>);
        }
    };
    if (din == 128) return pr.g_scalar ? by_pro(T1{}, D128{}) : by_pro(F1{}, D128{});
    return pr.g_scalar ? by_pro(T1{}, D64{}) : by_pro(F1{}, D64{});
}

}  // namespace gdn2
