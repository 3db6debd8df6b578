// Inverse of a 64 x 64 unit lower-triangular matrix, T = (I + A)^{-1}, with A
// strictly lower (the UT/WY transform of the chunkwise delta rule, and the
// same transform in the chunk form of the preconditioner recurrence).
//
// Blocked in 16 x 16 blocks (block indices 0..3):
//   level 0: T_ii = (I + A_ii)^{-1} by forward substitution, one warp per block;
//   level 1: T_10 = -T_11 A_10 T_00 and T_32 = -T_33 A_32 T_22
//            (the two 32 x 32 diagonal blocks are then complete);
//   level 2: X = A_[23][01] T_[01]  (the 32 x 32 lower-left block, 4 warps);
//   level 3: T_[23][01] = -T_[23] X.
// The 16 x 16 x 16 block products run on mma.sync m16n8k8 with tf32 inputs
// and fp32 accumulation; the diagonal blocks are exact fp32 FFMA.
// Executed by the 128 threads (4 warps) of one group; sync() must be a barrier
// over exactly those threads. A and T are fp32 in shared memory with row
// stride LD (68 keeps the fragment loads free of bank conflicts); T may not
// alias A. The blocks of T above the diagonal blocks are never written: the
// caller zeroes them once (tril_zero_upper) before the first call. On return T
// holds the full 64 x 64 inverse and every thread of the group has passed a
// final sync().
#pragma once
#include "common.cuh"

namespace osdn {
namespace tri {

constexpr int LD = 68;

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// c += X Y for 16 x 16 blocks X (row-major at X, stride LD) and Y; one warp.
// c[nh] holds output columns nh*8 .. nh*8+7 in the m16n8 accumulator layout.
__device__ __forceinline__ void blk_mma(float (&c)[2][4], const float* X, const float* Y, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const int k0 = ks * 8;
        const uint32_t a0 = to_tf32(X[g * LD + k0 + t]);
        const uint32_t a1 = to_tf32(X[(g + 8) * LD + k0 + t]);
        const uint32_t a2 = to_tf32(X[g * LD + k0 + t + 4]);
        const uint32_t a3 = to_tf32(X[(g + 8) * LD + k0 + t + 4]);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            const uint32_t b0 = to_tf32(Y[(k0 + t) * LD + nh * 8 + g]);
            const uint32_t b1 = to_tf32(Y[(k0 + t + 4) * LD + nh * 8 + g]);
            mma_tf32(c[nh], a0, a1, a2, a3, b0, b1);
        }
    }
}

// Same product with the fp32 bit patterns passed as tf32 operands: the tensor
// core reads the upper 19 bits (truncation instead of round-to-nearest, one
// tf32 ulp at most), which saves the conversions.
__device__ __forceinline__ void blk_mma_trunc(float (&c)[2][4], const float* X, const float* Y, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const int k0 = ks * 8;
        const uint32_t a0 = __float_as_uint(X[g * LD + k0 + t]);
        const uint32_t a1 = __float_as_uint(X[(g + 8) * LD + k0 + t]);
        const uint32_t a2 = __float_as_uint(X[g * LD + k0 + t + 4]);
        const uint32_t a3 = __float_as_uint(X[(g + 8) * LD + k0 + t + 4]);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            const uint32_t b0 = __float_as_uint(Y[(k0 + t) * LD + nh * 8 + g]);
            const uint32_t b1 = __float_as_uint(Y[(k0 + t + 4) * LD + nh * 8 + g]);
            mma_tf32(c[nh], a0, a1, a2, a3, b0, b1);
        }
    }
}

__device__ __forceinline__ void blk_zero(float (&c)[2][4]) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) c[i][j] = 0.f;
}

// Store s * c into the 16 x 16 block at D (stride LD).
__device__ __forceinline__ void blk_store(float* D, const float (&c)[2][4], float s, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        D[g * LD + nh * 8 + 2 * t] = s * c[nh][0];
        D[g * LD + nh * 8 + 2 * t + 1] = s * c[nh][1];
        D[(g + 8) * LD + nh * 8 + 2 * t] = s * c[nh][2];
        D[(g + 8) * LD + nh * 8 + 2 * t + 1] = s * c[nh][3];
    }
}

// Zero the 16 x 16 blocks of T above its diagonal blocks (threads `tid` of `n`).
__device__ __forceinline__ void tril_zero_upper(float* T, int tid, int n) {
    for (int idx = tid; idx < 64 * 64; idx += n) {
        const int r = idx >> 6, c = idx & 63;
        if ((c >> 4) > (r >> 4)) T[r * LD + c] = 0.f;
    }
}

template <class Sync>
__device__ __forceinline__ void tril_inv64(const float* A, float* T, int warp, int lane, Sync sync) {
    auto blkA = [&](int i, int j) { return A + (i * 16) * LD + j * 16; };
    auto blkT = [&](int i, int j) { return T + (i * 16) * LD + j * 16; };

    {   // level 0: diagonal block `warp`, lane j (< 16) owns column j
        const int j = lane & 15, o = warp * 16;
        float c[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) c[t] = (t == j) ? 1.f : 0.f;
#pragma unroll
        for (int t = 1; t < 16; ++t) {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int m = 0; m < t; m += 2) {
                s0 = fmaf(A[(o + t) * LD + o + m], c[m], s0);
                if (m + 1 < t) s1 = fmaf(A[(o + t) * LD + o + m + 1], c[m + 1], s1);
            }
            if (t > j) c[t] = -(s0 + s1);
        }
        if (lane < 16) {
#pragma unroll
            for (int t = 0; t < 16; ++t) T[(o + t) * LD + o + j] = c[t];
        }
    }
    sync();
    // level 1: warps 0 and 1 build T_10 and T_32 (two products each, through a block of T as scratch)
    if (warp < 2) {
        const int i = warp * 2 + 1, j = warp * 2;     // (1,0) or (3,2)
        float c[2][4];
        blk_zero(c);
        blk_mma(c, blkA(i, j), blkT(j, j), lane);     // W = A_ij T_jj
        blk_store(blkT(i, j), c, 1.f, lane);
        __syncwarp();
        blk_zero(c);
        blk_mma(c, blkT(i, i), blkT(i, j), lane);     // T_ii W
        __syncwarp();
        blk_store(blkT(i, j), c, -1.f, lane);
    }
    sync();
    // level 2: X_ab = sum_m A_am T_mb for a in {2,3}, b in {0,1} (m in {0,1}, T_01 = 0)
    {
        const int a = 2 + (warp >> 1), bb = warp & 1;
        float c[2][4];
        blk_zero(c);
        if (bb == 0) {
            blk_mma(c, blkA(a, 0), blkT(0, 0), lane);
            blk_mma(c, blkA(a, 1), blkT(1, 0), lane);
        } else {
            blk_mma(c, blkA(a, 1), blkT(1, 1), lane);
        }
        blk_store(blkT(a, bb), c, 1.f, lane);
    }
    sync();
    // level 3: T_ab = -(T_a2 X_2b + T_a3 X_3b), T_23 = 0; all products read X before any write
    {
        const int a = 2 + (warp >> 1), bb = warp & 1;
        float c[2][4];
        blk_zero(c);
        blk_mma(c, blkT(a, 2), blkT(2, bb), lane);
        if (a == 3) blk_mma(c, blkT(3, 3), blkT(3, bb), lane);
        sync();
        blk_store(blkT(a, bb), c, -1.f, lane);
    }
    sync();
}

// Forward substitution for column j of (I + L)^{-1}, L the strictly lower
// 16 x 16 block at Lb (row stride LD). Row t's entries 0..t-1 are read with
// 16-byte loads: row starts are 16-byte aligned (LD * 4 and the block offsets
// are multiples of 16 bytes, the matrix base is 16-byte aligned).
__device__ __forceinline__ void diag16_inverse_column(const float* Lb, int j, float (&c)[16]) {
#pragma unroll
    for (int t = 0; t < 16; ++t) c[t] = (t == j) ? 1.f : 0.f;
#pragma unroll
    for (int t = 1; t < 16; ++t) {
        float l[16];
#pragma unroll
        for (int m4 = 0; m4 < t; m4 += 4) {
            const float4 x = *reinterpret_cast<const float4*>(Lb + t * LD + m4);
            l[m4] = x.x; l[m4 + 1] = x.y; l[m4 + 2] = x.z; l[m4 + 3] = x.w;
        }
        float s[4] = {0.f, 0.f, 0.f, 0.f};   // four partial sums shorten the dependent FMA chain
#pragma unroll
        for (int m = 0; m < t; ++m) s[m & 3] = fmaf(l[m], c[m], s[m & 3]);
        if (t > j) c[t] = -((s[0] + s[1]) + (s[2] + s[3]));
    }
}

// In-place variant: on entry A holds the strictly lower 64 x 64 matrix (every
// entry on and above the diagonal zero, the blocks above the diagonal blocks
// included); on return it holds T = (I + A)^{-1}. Same blocking and arithmetic
// as tril_inv64 except that the block products truncate their operands to
// tf32 (blk_mma_trunc); each level computes its blocks into registers before
// any warp overwrites an operand another warp still reads.
template <class Sync>
__device__ __forceinline__ void tril_inv64_inplace(float* A, int warp, int lane, Sync sync) {
    auto blk = [&](int i, int j) { return A + (i * 16) * LD + j * 16; };
    {   // level 0: diagonal block `warp`
        const int j = lane & 15;
        float c[16];
        diag16_inverse_column(blk(warp, warp), j, c);
        __syncwarp();
        if (lane < 16) {
#pragma unroll
            for (int t = 0; t < 16; ++t) blk(warp, warp)[t * LD + j] = c[t];
        }
    }
    sync();
    if (warp < 2) {   // level 1: T_10 and T_32 (each warp owns its block)
        const int i = warp * 2 + 1, j = warp * 2;
        float c[2][4];
        blk_zero(c);
        blk_mma_trunc(c, blk(i, j), blk(j, j), lane);       // W = A_ij T_jj
        __syncwarp();
        blk_store(blk(i, j), c, 1.f, lane);
        __syncwarp();
        blk_zero(c);
        blk_mma_trunc(c, blk(i, i), blk(i, j), lane);       // T_ii W
        __syncwarp();
        blk_store(blk(i, j), c, -1.f, lane);
    }
    sync();
    {   // level 2: X_ab = sum_m A_am T_mb, a in {2,3}, b in {0,1}; stored over A_ab
        const int a = 2 + (warp >> 1), bb = warp & 1;
        float c[2][4];
        blk_zero(c);
        if (bb == 0) {
            blk_mma_trunc(c, blk(a, 0), blk(0, 0), lane);
            blk_mma_trunc(c, blk(a, 1), blk(1, 0), lane);
        } else {
            blk_mma_trunc(c, blk(a, 1), blk(1, 1), lane);
        }
        sync();
        blk_store(blk(a, bb), c, 1.f, lane);
    }
    sync();
    {   // level 3: T_ab = -(T_a2 X_2b + T_a3 X_3b), T_23 = 0
        const int a = 2 + (warp >> 1), bb = warp & 1;
        float c[2][4];
        blk_zero(c);
        blk_mma_trunc(c, blk(a, 2), blk(2, bb), lane);
        if (a == 3) blk_mma_trunc(c, blk(3, 3), blk(3, bb), lane);
        sync();
        blk_store(blk(a, bb), c, -1.f, lane);
    }
    sync();
}

// Byte offset of element (row r, column j) in a 128-byte-swizzled K-major bf16 tile whose
// 8-row groups are 1024 bytes apart (64 columns of 2 bytes per row).
__device__ __forceinline__ uint32_t sw128_elem(int r, int j) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((((j >> 3) ^ (r & 7))) << 4) + (j & 7) * 2);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// bf16 of sgn * c * sc[column] into block (a, b) of a swizzled 64 x 64 tile, from the m16n8
// accumulator layout of blk_mma (4-byte stores; the 8 rows of a store hit 8 distinct 16-byte
// bank groups).
__device__ __forceinline__ void blk_store_bf16(uint8_t* tile, const float (&c)[2][4], float sgn, const float* sc,
                                               int a, int b, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int col = 16 * b + 8 * nh + 2 * t;
        const float s0 = sgn * sc[col], s1 = sgn * sc[col + 1];
        *reinterpret_cast<uint32_t*>(tile + sw128_elem(16 * a + g, col)) = pack_bf16x2(s0 * c[nh][0], s1 * c[nh][1]);
        *reinterpret_cast<uint32_t*>(tile + sw128_elem(16 * a + g + 8, col)) = pack_bf16x2(s0 * c[nh][2], s1 * c[nh][3]);
    }
}

// bf16 of the fp32 block (a, b) of T (stride LD) times sc[column], into the swizzled tile; one warp,
// lane L takes row L / 2 and columns 8 (L % 2) .. + 7 of the block (one 16-byte store).
__device__ __forceinline__ void blk_convert_bf16(uint8_t* tile, const float* T, const float* sc, int a, int b,
                                                 int lane) {
    const int r = lane >> 1, j0 = 16 * b + 8 * (lane & 1);
    const float* src = T + (16 * a + r) * LD + j0;
    const float4 x0 = *reinterpret_cast<const float4*>(src), x1 = *reinterpret_cast<const float4*>(src + 4);
    const float4 s0 = *reinterpret_cast<const float4*>(sc + j0), s1 = *reinterpret_cast<const float4*>(sc + j0 + 4);
    uint4 pk;
    pk.x = pack_bf16x2(x0.x * s0.x, x0.y * s0.y);
    pk.y = pack_bf16x2(x0.z * s0.z, x0.w * s0.w);
    pk.z = pack_bf16x2(x1.x * s1.x, x1.y * s1.y);
    pk.w = pack_bf16x2(x1.z * s1.z, x1.w * s1.w);
    *reinterpret_cast<uint4*>(tile + sw128_elem(16 * a + r, j0)) = pk;
}

// T = (I + A)^{-1} for a strictly lower 64 x 64 A (fp32, stride LD, 16-byte aligned rows), written
// only as the bf16 tile tb = T diag(sc) (128-byte-swizzled K-major, row t, column j; 16 x 16 blocks
// above the diagonal blocks are not written and must hold zeros). A's lower blocks are overwritten by intermediates. The same blocking as tril_inv64 in three
// barrier-separated phases after the diagonal blocks:
//   phase 0: T_ii = (I + A_ii)^{-1}, right-looking forward substitution, one warp per block;
//   phase 1: T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22) (warps 0, 1);
//            Y_a0 = A_a0 T_00, X_a1 = A_a1 T_11 for a = 2, 3 (warp a, kept in registers);
//   phase 2: X_a0 = Y_a0 + A_a1 T_10 (warp a; X_a0, X_a1 stored over A_a0, A_a1), while warps 0
//            and 1 convert the finished blocks T_00, T_10, T_11 / T_22, T_32, T_33;
//   phase 3: T_2b = -T_22 X_2b, T_3b = -(T_32 X_2b + T_33 X_3b) (one block per warp), straight to bf16.
// Executed by the 4 warps of one group; sync() is a barrier over exactly those threads.
// tiles_free() is called by every thread after phase 1, before the first tile write; it must act
// as a barrier of the group and return true on every thread when the group is to stop (the
// function then returns false right away). Returns true after a final sync().
template <class Sync, class TilesFree>
__device__ __forceinline__ bool tril_inv64_to_bf16(float* A, uint8_t* tb, const float* sc, int warp, int lane,
                                                   Sync sync, TilesFree tiles_free) {
    auto blk = [&](int i, int j) { return A + (i * 16) * LD + j * 16; };
    {   // phase 0: column j of T_ww by right-looking substitution (lanes 16-31 repeat lanes 0-15)
        const int j = lane & 15;
        const float* Ab = blk(warp, warp);
        float c[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) c[t] = (t == j) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
#pragma unroll
            for (int t = m + 1; t < 16; ++t) c[t] = fmaf(-Ab[t * LD + m], c[m], c[t]);
        }
        __syncwarp();
        if (lane < 16) {
            float* Tb = blk(warp, warp);
#pragma unroll
            for (int t = 0; t < 16; ++t) Tb[t * LD + j] = c[t];
        }
    }
    sync();
    float y[2][4], x1[2][4];
    blk_zero(y);
    blk_zero(x1);
    if (warp < 2) {   // phase 1: T_10 (warp 0), T_32 (warp 1)
        const int i = 2 * warp + 1, j = 2 * warp;
        blk_mma_trunc(y, blk(i, j), blk(j, j), lane);       // W = A_ij T_jj
        __syncwarp();
        blk_store(blk(i, j), y, 1.f, lane);
        __syncwarp();
        blk_zero(y);
        blk_mma_trunc(y, blk(i, i), blk(i, j), lane);       // T_ii W
        __syncwarp();
        blk_store(blk(i, j), y, -1.f, lane);
    } else {          // Y_a0 = A_a0 T_00, X_a1 = A_a1 T_11
        blk_mma_trunc(y, blk(warp, 0), blk(0, 0), lane);
        blk_mma_trunc(x1, blk(warp, 1), blk(1, 1), lane);
    }
    if (tiles_free()) return false;
    if (warp >= 2) {  // phase 2: X_a0 = Y_a0 + A_a1 T_10
        blk_mma_trunc(y, blk(warp, 1), blk(1, 0), lane);
        __syncwarp();
        blk_store(blk(warp, 0), y, 1.f, lane);
        blk_store(blk(warp, 1), x1, 1.f, lane);
    } else {          // finished blocks of T to bf16
        const int o = 2 * warp;
        blk_convert_bf16(tb, A, sc, o, o, lane);
        blk_convert_bf16(tb, A, sc, o + 1, o, lane);
        blk_convert_bf16(tb, A, sc, o + 1, o + 1, lane);
    }
    sync();
    {                 // phase 3: block (a, b) of T, a = 2 + warp / 2, b = warp % 2
        const int a = 2 + (warp >> 1), bb = warp & 1;
        float c[2][4];
        blk_zero(c);
        blk_mma_trunc(c, blk(a, 2), blk(2, bb), lane);
        if (a == 3) blk_mma_trunc(c, blk(3, 3), blk(3, bb), lane);
        blk_store_bf16(tb, c, -1.f, sc, a, bb, lane);
    }
    sync();
    return true;
}

}  // namespace tri
}  // namespace osdn
