// Chunkwise OSDN forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1: the DeltaNet chunkwise WY
// pipeline with the scaled write key Kw = D (.) K substituted in the block
// Gram matrix and the intra-block scores; the read/erase key K unchanged.
// Per chunk of C = 64 tokens with chunk-start state S (dv x dk, fp32):
//   A = strict_tril(diag(beta) K Kw^T),   T = (I + A)^{-1},
//   U = T diag(beta) (V - K S^T),
//   O = Q S^T + tril(Q Kw^T) U,           S <- S + U^T Kw.
//
// Every contraction is issued as a tcgen05 MMA with M = 128 by putting the
// value dimension (dv = 128) or the stacked [K; Q] rows (2 x 64 tokens) on M:
//   MMA1  D1[128 x 64]  = [K; Q] Kw^T          (Gram rows 0-63, scores rows 64-127)
//   MMA2  D2[128 x 128] = S [K; Q]^T           (S K^T | S Q^T, transposed)
//   MMA3  D3[128 x 64]  = Xh^T T^T             (U^T, Xh = diag(beta) (V - K S^T))
//   MMA4  D2[:, 64:]   += U^T P^T              (O^T = S Q^T + U^T P^T)
//   MMA5  DS[128 x 128]+= U^T Kw               (state carry, Kw read MN-major)
// bf16 operands in 128-byte-swizzled shared memory (TMA-filled for Q, K, Kw;
// written by the CTA for S, Xh, U, T, P), fp32 accumulators in TMEM. The
// state S stays in TMEM for the whole sequence; its bf16 copy for MMA2 is
// refreshed once per chunk. T = (I + A)^{-1} is a blocked 16 x 16 inverse on CUDA cores (fp32 diagonal
// blocks, mma.sync tf32 block products).
//
// One CTA (128 threads = the 128 TMEM lanes) owns one (sequence, head).
// Thread i owns TMEM lane i: row v = i of S, U^T and O^T; in the epilogues of
// MMA1 it owns Gram row i (i < 64) or score row i - 64. Requires dk = dv = 128,
// bf16 inputs. Every mbarrier wait is bounded; a wait that gives up sets the
// library status word (OSDN_ERR_TIMEOUT via osdn_sync_status) and the CTA
// leaves after a bounded drain, releasing its TMEM.
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct TcSmem {
    static constexpr uint32_t QK = 0;                 // [K;Q] K-halves of 16 KB: K rows (8 KB) then Q rows (8 KB)
    static constexpr uint32_t KW = 32768;             // scaled keys (even chunks), two K-halves of 8 KB
    static constexpr uint32_t V = 49152;              // V [64 t][128 v] bf16, unswizzled
    static constexpr uint32_t SB = 65536;             // S bf16 [128 v][128 i], two K-halves of 16 KB
    static constexpr uint32_t XU = 98304;             // Xh^T, then U^T: [128 v][64 t] bf16
    static constexpr uint32_t TB = 114688;            // T [64 t][64 j] bf16
    static constexpr uint32_t PB = 122880;            // P [64 t][64 j] bf16
    static constexpr int LDF = tri::LD;               // fp32 row stride of A and T
    static constexpr uint32_t AF = 131072;            // A fp32 [64][LDF]
    static constexpr uint32_t TF = AF + 64 * LDF * 4;  // T fp32 [64][LDF]
    static constexpr uint32_t KW1 = 165888;           // second scaled-key buffer (odd chunks)
    static constexpr uint32_t OS = KW1 + 16384;       // O [64 t][128 v] bf16 staging for the TMA store
    static constexpr uint32_t BETA = OS + 16384;
    static constexpr uint32_t BAR = BETA + 256;       // tma_bar, mma_bar, tmem base address
    static constexpr uint32_t END = BAR + 64;
    static constexpr size_t kBytes = END + 1024;      // + slack to align the base to 1024
    static constexpr uint32_t kTxBytes = 6 * 8192 + 16384;   // TMA bytes per chunk
};

template <int kUnused = 0>
__global__ void __launch_bounds__(128, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_kw, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_out, const __nv_bfloat16* __restrict__ beta,
                const float* __restrict__ S0, float* __restrict__ S_final, int B, int T, int H,
                unsigned long long wait_limit_ns)
{
    constexpr int C = 64, DK = 128, DV = 128;
    constexpr uint32_t COL_S = 0, COL_D2 = 128, COL_D1 = 256, COL_D3 = 320, NCOLS = 512;
    constexpr uint32_t ID_N64 = tc::idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_N128 = tc::idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t ID_N128_BMN = tc::idesc_bf16(128, 128, 0, 1);
    using L = TcSmem;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = tc::smem_u32(sm);
    float* AF = reinterpret_cast<float*>(sm + L::AF);
    float* TF = reinterpret_cast<float*>(sm + L::TF);
    float* betas = reinterpret_cast<float*>(sm + L::BETA);
    const __nv_bfloat16* Vs = reinterpret_cast<const __nv_bfloat16*>(sm + L::V);
    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint64_t* mma_bar = tma_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tma_bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;

    if (tid == 0) {
        tc::mbar_init(tma_bar, 1);
        tc::mbar_init(mma_bar, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_kw);
        tc::prefetch_tmap(&tm_v);
        tc::prefetch_tmap(&tm_out);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, NCOLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's TMEM lane quarter
    const int v = tid;                                           // row of S / U^T / O^T owned

    {   // initial state into TMEM
        const float* srow = S0 ? S0 + ((size_t)unit * DV + v) * DK : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 x = srow ? *reinterpret_cast<const float4*>(srow + c * 32 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                r[i] = __float_as_uint(x.x); r[i + 1] = __float_as_uint(x.y);
                r[i + 2] = __float_as_uint(x.z); r[i + 3] = __float_as_uint(x.w);
            }
            tc::tmem_st32(tl + COL_S + c * 32, r);
        }
        tc::tmem_wait_st();
    }

    // TMA of chunk ci: K, Q (two 64-column halves each) into the [K;Q] tile, its
    // scaled keys into the buffer of its parity, V
    auto issue_loads = [&](int ci) {
        const int tt = ci * C;
        const uint32_t kwb = (ci & 1) ? L::KW1 : L::KW;
        tc::mbar_arrive_expect_tx(tma_bar, L::kTxBytes);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tc::tma_load_4d(sm + L::QK + half * 16384, &tm_k, half * 64, h, tt, b, tma_bar);
            tc::tma_load_4d(sm + L::QK + half * 16384 + 8192, &tm_q, half * 64, h, tt, b, tma_bar);
            tc::tma_load_4d(sm + kwb + half * 8192, &tm_kw, half * 64, h, tt, b, tma_bar);
        }
        tc::tma_load_4d(sm + L::V, &tm_v, 0, h, tt, b, tma_bar);
    };
    uint32_t tma_phase = 0, mma_phase = 0;
    const int nchunks = (T + C - 1) / C;
    bool failed = false, tma_pending = nchunks > 0, mma_pending = false;
    if (tid == 0 && nchunks > 0) issue_loads(0);
    for (int ci = 0; ci < nchunks; ++ci) {
        const int t0 = ci * C, Tc = min(C, T - t0);

        // (0) bf16 copy of the chunk-start state (A operand of MMA2), and beta
        tc::tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t r[32];
                tc::tmem_ld32(tl + COL_S + half * 64 + q * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 pk;
                    pk.x = tc::pack_bf16(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    pk.y = tc::pack_bf16(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    pk.z = tc::pack_bf16(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    pk.w = tc::pack_bf16(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4*>(sm + L::SB + half * 16384 + tc::sw128_off(v, q * 4 + cc)) = pk;
                }
            }
        }
        if (tid < C) betas[tid] = (tid < Tc) ? __bfloat162float(beta[((size_t)b * T + t0 + tid) * H + h]) : 0.f;
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // (1) this chunk's tiles (issued in the prologue or after the previous chunk's MMA1/MMA2 epilogue)
        const uint32_t KWc = (ci & 1) ? L::KW1 : L::KW;
        if (!tc::mbar_wait(tma_bar, tma_phase, wait_limit_ns)) failed = true;
        else { tma_phase ^= 1; tma_pending = false; }
        if (__syncthreads_or(failed)) break;

        // (2) MMA1: D1 = [K;Q] Kw^T   MMA2: D2 = S [K;Q]^T
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                tc::umma_bf16(tmem + COL_D1, tc::sdesc_sw128(sb + L::QK + half * 16384 + koff, 16, 1024),
                              tc::sdesc_sw128(sb + KWc + half * 8192 + koff, 16, 1024), ID_N64, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                tc::umma_bf16(tmem + COL_D2, tc::sdesc_sw128(sb + L::SB + half * 16384 + koff, 16, 1024),
                              tc::sdesc_sw128(sb + L::QK + half * 16384 + koff, 16, 1024), ID_N128, ks > 0);
            }
            tc::umma_commit(mma_bar);
        }
        mma_pending = true;
        if (!tc::mbar_wait(mma_bar, mma_phase, wait_limit_ns)) failed = true;
        else { mma_phase ^= 1; mma_pending = false; }
        if (__syncthreads_or(failed)) break;
        tc::tc_fence_after();

        // (3) epilogue of MMA1/MMA2: Xh^T = diag(beta)(V - K S^T)^T -> bf16 smem;
        //     Gram -> A (fp32, strict lower, row-scaled by beta); scores -> P (bf16, lower incl. diagonal)
        {
            uint32_t r[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tl + COL_D2 + q * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = q * 32 + cc * 8 + e;
                        x[e] = betas[t] * (__bfloat162float(Vs[t * DV + v]) - __uint_as_float(r[cc * 8 + e]));
                    }
                    uint4 pk;
                    pk.x = tc::pack_bf16(x[0], x[1]); pk.y = tc::pack_bf16(x[2], x[3]);
                    pk.z = tc::pack_bf16(x[4], x[5]); pk.w = tc::pack_bf16(x[6], x[7]);
                    *reinterpret_cast<uint4*>(sm + L::XU + tc::sw128_off(v, q * 4 + cc)) = pk;
                }
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tl + COL_D1 + q * 32, r);
                tc::tmem_wait_ld();
                if (tid < C) {
                    const int t = tid;
                    const float bt = betas[t];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = q * 32 + e;
                        AF[t * L::LDF + j] = (j < t) ? bt * __uint_as_float(r[e]) : 0.f;
                    }
                } else {
                    const int t = tid - C;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = q * 32 + cc * 8 + e;
                            x[e] = (j <= t) ? __uint_as_float(r[cc * 8 + e]) : 0.f;
                        }
                        uint4 pk;
                        pk.x = tc::pack_bf16(x[0], x[1]); pk.y = tc::pack_bf16(x[2], x[3]);
                        pk.z = tc::pack_bf16(x[4], x[5]); pk.w = tc::pack_bf16(x[6], x[7]);
                        *reinterpret_cast<uint4*>(sm + L::PB + tc::sw128_off(t, q * 4 + cc)) = pk;
                    }
                }
            }
        }
        __syncthreads();
        // Q, K and V of this chunk are consumed (MMA1, MMA2 done, V read): start the next chunk's loads
        if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);
        tma_pending = ci + 1 < nchunks;

        // (4) T = (I + A)^{-1}: blocked 16 x 16 inverse (fp32 diagonal blocks, tf32 block products)
        tri::tril_inv64(AF, TF, warp, tid & 31, [] { __syncthreads(); });
        if (tid < C) {   // T -> bf16 K-major swizzled (B operand of MMA3)
            const int t = tid;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 pk;
                const float* row = TF + t * L::LDF + c * 8;
                pk.x = tc::pack_bf16(row[0], row[1]); pk.y = tc::pack_bf16(row[2], row[3]);
                pk.z = tc::pack_bf16(row[4], row[5]); pk.w = tc::pack_bf16(row[6], row[7]);
                *reinterpret_cast<uint4*>(sm + L::TB + tc::sw128_off(t, c)) = pk;
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // (5) MMA3: D3 = Xh^T T^T = U^T
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::umma_bf16(tmem + COL_D3, tc::sdesc_sw128(sb + L::XU + ks * 32, 16, 1024),
                              tc::sdesc_sw128(sb + L::TB + ks * 32, 16, 1024), ID_N64, ks > 0);
            tc::umma_commit(mma_bar);
        }
        mma_pending = true;
        if (!tc::mbar_wait(mma_bar, mma_phase, wait_limit_ns)) failed = true;
        else { mma_phase ^= 1; mma_pending = false; }
        if (__syncthreads_or(failed)) break;
        tc::tc_fence_after();

        // (6) U^T -> bf16 smem (overwrites Xh^T, which MMA3 has consumed)
        {
            uint32_t r[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tl + COL_D3 + q * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 pk;
                    pk.x = tc::pack_bf16(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    pk.y = tc::pack_bf16(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    pk.z = tc::pack_bf16(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    pk.w = tc::pack_bf16(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4*>(sm + L::XU + tc::sw128_off(v, q * 4 + cc)) = pk;
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // (7) MMA4: D2[:, 64:] += U^T P^T (O^T)   MMA5: DS += U^T Kw (state carry)
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::umma_bf16(tmem + COL_D2 + 64, tc::sdesc_sw128(sb + L::XU + ks * 32, 16, 1024),
                              tc::sdesc_sw128(sb + L::PB + ks * 32, 16, 1024), ID_N64, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::umma_bf16(tmem + COL_S, tc::sdesc_sw128(sb + L::XU + ks * 32, 16, 1024),
                              tc::sdesc_sw128(sb + KWc + ks * 2048, 8192, 1024), ID_N128_BMN, true);
            tc::umma_commit(mma_bar);
        }
        mma_pending = true;
        if (!tc::mbar_wait(mma_bar, mma_phase, wait_limit_ns)) failed = true;
        else { mma_phase ^= 1; mma_pending = false; }
        if (__syncthreads_or(failed)) break;
        tc::tc_fence_after();

        // (8) O^T row v -> staging O[t][v] -> TMA store of the chunk (rows past T clipped)
        if (tid == 0) tc::bulk_wait_read<0>();   // the previous chunk's store has left the staging tile
        __syncthreads();
        {
            __nv_bfloat16* Os = reinterpret_cast<__nv_bfloat16*>(sm + L::OS);
            uint32_t r[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tl + COL_D2 + 64 + q * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) Os[(q * 32 + e) * DV + v] = __float2bfloat16_rn(__uint_as_float(r[e]));
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_4d(&tm_out, sm + L::OS, 0, h, t0, b);
            tc::bulk_commit();
        }
    }

    if (tid == 0) tc::bulk_wait<0>();
    if (!failed && S_final) {
        tc::tc_fence_after();
        float* srow = S_final + ((size_t)unit * DV + v) * DK;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tc::tmem_ld32(tl + COL_S + c * 32, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(srow + c * 32 + i) =
                    make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                __uint_as_float(r[i + 3]));
        }
    }
    if (failed) {
        // Drain: one more bounded wait for the copy or MMAs still in flight, so
        // nothing lands in shared memory or TMEM after the CTA releases them.
        if (tid == 0) {
            atomicOr(&g_osdn_status, kStatusTimeout);
            const unsigned long long drain_ns = wait_limit_ns > 1000000000ull ? wait_limit_ns : 1000000000ull;
            if (tma_pending) tc::mbar_wait(tma_bar, tma_phase, drain_ns);
            if (mma_pending) tc::mbar_wait(mma_bar, mma_phase, drain_ns);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, NCOLS);
    }
}

}  // namespace osdn
