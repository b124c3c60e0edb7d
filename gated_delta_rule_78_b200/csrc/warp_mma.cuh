// Warp-level tensor-core building block of the forward kernel (and so of the backward's
// states pass): the 64 x 64 unit lower-triangular inverse T = (I + A)^-1 that every chunk
// needs (closed-form 4x4 blocks, in-warp doubling to 16x16, then two doubling levels on
// TF32 warp MMAs).
#pragma once

#include <stdint.h>

#include "tc_util.cuh"

namespace gdn2 {
namespace wm {

using tc::mma_tf32_16x8x8;
using tc::to_tf32;

// ------------------------------------------------------------------ 64 x 64 unit lower-triangular inverse
// One warp inverts the 16x16 unit lower-triangular diagonal block (I + A_pp) that
// starts at row/column r0: closed-form 4x4 inverses, then two doubling steps
// T21 = -T22 (A21 T11) inside the warp.  Only lower blocks of sT are written.
template <int LD>
__device__ __forceinline__ void invert_diag16(const float *sA, float *sT, int r0, int lane)
{
    if (lane < 4) {
        const int b = r0 + 4 * lane;
        const float *a = sA + b * LD + b;
        const float a10 = a[1 * LD + 0], a20 = a[2 * LD + 0], a21 = a[2 * LD + 1];
        const float a30 = a[3 * LD + 0], a31 = a[3 * LD + 1], a32 = a[3 * LD + 2];
        const float t10 = -a10, t21 = -a21, t32 = -a32;
        const float t20 = -(a20 + a21 * t10);
        const float t31 = -(a31 + a32 * t21);
        const float t30 = -(a30 + a31 * t10 + a32 * t20);
        float *t = sT + b * LD + b;
        t[0 * LD + 0] = 1.f;
        t[1 * LD + 0] = t10; t[1 * LD + 1] = 1.f;
        t[2 * LD + 0] = t20; t[2 * LD + 1] = t21; t[2 * LD + 2] = 1.f;
        t[3 * LD + 0] = t30; t[3 * LD + 1] = t31; t[3 * LD + 2] = t32; t[3 * LD + 3] = 1.f;
    }
    __syncwarp();
    {  // 4 -> 8: two 4x4 blocks, one output per lane
        const int q = lane >> 4, r = (lane >> 2) & 3, c = lane & 3;
        const int R = r0 + 8 * q + 4, Cc = r0 + 8 * q;
        float y = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) y += sA[(R + r) * LD + Cc + u] * sT[(Cc + u) * LD + Cc + c];
        __syncwarp();
        sT[(R + r) * LD + Cc + c] = y;
        __syncwarp();
        float x = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) x += sT[(R + r) * LD + R + u] * sT[(R + u) * LD + Cc + c];
        __syncwarp();
        sT[(R + r) * LD + Cc + c] = -x;
        __syncwarp();
    }
    {  // 8 -> 16: one 8x8 block, two outputs per lane
        const int r = lane >> 2, c = 2 * (lane & 3);
        const int R = r0 + 8, Cc = r0;
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float a = sA[(R + r) * LD + Cc + u];
            y0 += a * sT[(Cc + u) * LD + Cc + c];
            y1 += a * sT[(Cc + u) * LD + Cc + c + 1];
        }
        __syncwarp();
        sT[(R + r) * LD + Cc + c] = y0;
        sT[(R + r) * LD + Cc + c + 1] = y1;
        __syncwarp();
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float t = sT[(R + r) * LD + R + u];
            x0 += t * sT[(R + u) * LD + Cc + c];
            x1 += t * sT[(R + u) * LD + Cc + c + 1];
        }
        __syncwarp();
        sT[(R + r) * LD + Cc + c] = -x0;
        sT[(R + r) * LD + Cc + c + 1] = -x1;
    }
}

// acc (16x8 tile) += X[0:16, 0:K] * Y[0:K, 0:8] for fp32 shared-memory operands with
// row stride LD (X and Y point at the tile origins), rounded to TF32 on load.
template <int K, int LD>
__device__ __forceinline__ void tile_mma_tf32(const float *X, const float *Y, float (&acc)[4], int lane)
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a[4] = {to_tf32(X[g * LD + k0 + t]), to_tf32(X[(g + 8) * LD + k0 + t]),
                               to_tf32(X[g * LD + k0 + t + 4]), to_tf32(X[(g + 8) * LD + k0 + t + 4])};
        const uint32_t b[2] = {to_tf32(Y[(k0 + t) * LD + g]), to_tf32(Y[(k0 + t + 4) * LD + g])};
        mma_tf32_16x8x8(acc, a, b);
    }
}
template <int LD>
__device__ __forceinline__ void tile_store(float *Z, const float (&acc)[4], float sign, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    Z[g * LD + 2 * t] = sign * acc[0];
    Z[g * LD + 2 * t + 1] = sign * acc[1];
    Z[(g + 8) * LD + 2 * t] = sign * acc[2];
    Z[(g + 8) * LD + 2 * t + 1] = sign * acc[3];
}

// T = (I + A)^-1 for the strictly lower 64 x 64 fp32 matrix in sA (row stride LD), on
// four warps (w4 = 0..3).  sT must hold zeros above the diagonal blocks on entry; its
// lower triangle (diagonal included) is written.  `sync()` is a barrier over exactly
// those four warps; it is called an equal number of times by each of them.
template <int LD, typename Sync>
__device__ __forceinline__ void solve_unit_lower64(const float *sA, float *sT, int w4, int lane, Sync sync)
{
    invert_diag16<LD>(sA, sT, 16 * w4, lane);
    sync();
    if (w4 < 2) {  // 32x32 level: T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22)
        const int R = 32 * w4 + 16, Cc = 32 * w4;
        float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma_tf32<16, LD>(sA + R * LD + Cc, sT + Cc * LD + Cc, y0, lane);
        tile_mma_tf32<16, LD>(sA + R * LD + Cc, sT + Cc * LD + Cc + 8, y1, lane);
        tile_store<LD>(sT + R * LD + Cc, y0, 1.f, lane);
        tile_store<LD>(sT + R * LD + Cc + 8, y1, 1.f, lane);
        __syncwarp();
        float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma_tf32<16, LD>(sT + R * LD + R, sT + R * LD + Cc, x0, lane);
        tile_mma_tf32<16, LD>(sT + R * LD + R, sT + R * LD + Cc + 8, x1, lane);
        __syncwarp();
        tile_store<LD>(sT + R * LD + Cc, x0, -1.f, lane);
        tile_store<LD>(sT + R * LD + Cc + 8, x1, -1.f, lane);
    }
    sync();
    {  // 64x64 level: T_BA = -T_BB (A_BA T_AA); warp: one 16-row tile, two 8-col tiles
        const int mt = w4 & 1, n0 = 16 * (w4 >> 1);
        float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma_tf32<32, LD>(sA + (32 + 16 * mt) * LD, sT + n0, y0, lane);
        tile_mma_tf32<32, LD>(sA + (32 + 16 * mt) * LD, sT + n0 + 8, y1, lane);
        tile_store<LD>(sT + (32 + 16 * mt) * LD + n0, y0, 1.f, lane);
        tile_store<LD>(sT + (32 + 16 * mt) * LD + n0 + 8, y1, 1.f, lane);
        sync();
        float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma_tf32<32, LD>(sT + (32 + 16 * mt) * LD + 32, sT + 32 * LD + n0, x0, lane);
        tile_mma_tf32<32, LD>(sT + (32 + 16 * mt) * LD + 32, sT + 32 * LD + n0 + 8, x1, lane);
        sync();
        tile_store<LD>(sT + (32 + 16 * mt) * LD + n0, x0, -1.f, lane);
        tile_store<LD>(sT + (32 + 16 * mt) * LD + n0 + 8, x1, -1.f, lane);
    }
    sync();
}

}  // namespace wm
}  // namespace gdn2
