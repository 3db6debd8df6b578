// Chunkwise OSDN forward on sm_100a, warp-specialized (tcgen05 + TMEM + TMA).
//
// Same mathematics and MMA set as the single-group chunk kernel ("OSDN:
// Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1; per chunk of C = 64 tokens):
//   MMA1  D1 = [K; Q] Kw^T        Gram (rows 0-63) and scores (rows 64-127)
//   MMA2  D2 = S [K; Q]^T         S K^T | S Q^T (transposed)
//   MMA3  D3 = Xh^T T^T = U^T     Xh = diag(beta)(V - K S^T), T = (I + A)^{-1}
//   MMA4  D2[:, 64:] += U^T P^T   O^T
//   MMA5  DS += U^T Kw            state carry, fp32 in TMEM for the whole sequence
// but split over five roles that run concurrently, so the work that does not
// depend on the state (Gram epilogue, T = (I + A)^{-1}) for chunk c + 1
// overlaps the state chain of chunk c:
//   warp 0      TMA producer: [K; Q] and Kw of chunk c into stage c % 2
//   warp 1      MMA issuer (one thread), in the order MMA2(c), MMA1(c+1),
//               MMA3(c), MMA5(c) + MMA4(c); warps 2-3 idle. This warpgroup
//               gives registers back (setmaxnreg 56) to the two below (224).
//   warps 4-7   chain group (128 threads, TMEM lane = value row v):
//               S -> bf16, Xh epilogue (V prefetched a chunk ahead from global
//               into registers), U epilogue, O staged in the Xh/U tile (free
//               between MMA5/MMA4 and the next Xh) and written by one TMA store
//   warps 8-11  prep group (128 threads, TMEM lane = Gram / score row):
//               A (fp32) and P (bf16) from D1, T = (I + A)^{-1}, T -> bf16
// Hand-offs are mbarriers (one arrival each: an elected thread, a TMA
// transaction count or a tcgen05.commit). Every wait is bounded; a wait that
// gives up sets the library status word and a shared abort flag, every role
// then stops at its next wait, the MMA and TMA threads drain what they
// issued, and the CTA releases its TMEM. Group members take that decision
// together through a barrier-OR, so no named barrier is left half-arrived.
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct WsSmem {
    static constexpr uint32_t STAGE = 49152;            // [K;Q] 32 KB + Kw 16 KB per stage
    static constexpr uint32_t QK0 = 0;
    static constexpr uint32_t KW0 = 32768;
    static constexpr uint32_t SB = 2 * STAGE;           // S bf16 [128 v][128 i], two K-halves of 16 KB
    static constexpr uint32_t XU = SB + 32768;          // Xh^T, then U^T [128 v][64 t] bf16
    static constexpr uint32_t TB = XU + 16384;          // T bf16 [64][64], two buffers of 8 KB
    static constexpr uint32_t PB = TB + 16384;          // P bf16 [64][64], two buffers of 8 KB
    static constexpr int LDF = tri::LD;
    static constexpr uint32_t AF = PB + 16384;          // A fp32 [64][LDF]
    static constexpr uint32_t TF = AF + 64 * LDF * 4;   // T fp32 [64][LDF]
    static constexpr uint32_t BETA_C = TF + 64 * LDF * 4;   // chain group's beta of its chunk
    static constexpr uint32_t BETA_P = BETA_C + 256;        // prep group's beta of its chunk
    static constexpr uint32_t BAR = BETA_P + 256;
    // mbarriers (8 bytes each)
    enum {
        B_FULL = 0, B_EMPTY = 2, B_D1FULL = 4, B_D1FREE = 6, B_TPREADY = 8,
        B_SB = 10, B_D2 = 11, B_XU = 12, B_D3 = 13, B_U = 14, B_S = 15, B_DRAIN = 16, NBAR = 17
    };
    static constexpr uint32_t TSLOT = BAR + NBAR * 8;   // TMEM base address
    static constexpr uint32_t ABORT = TSLOT + 4;        // abort flag
    static constexpr uint32_t END = ABORT + 4;
    static constexpr size_t kBytes = END + 1024;
    static constexpr uint32_t kTxBytes = 6 * 8192;      // TMA bytes per chunk (K, Q, Kw halves)
};

__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier with an OR over a predicate of the participating threads.
__device__ __forceinline__ bool named_sync_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

template <uint32_t N>
__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N>
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

template <int kUnused = 0>
__global__ void __launch_bounds__(384, 1)
chunk_ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_kw, const __grid_constant__ CUtensorMap tm_out,
                const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ beta,
                const float* __restrict__ S0, float* __restrict__ S_final, int B, int T, int H,
                unsigned long long wait_limit_ns)
{
    constexpr int C = 64, DK = 128, DV = 128;
    constexpr uint32_t COL_S = 0, COL_D2 = 128, COL_D1 = 256, COL_D3 = 384, NCOLS = 512;
    constexpr uint32_t ID_N64 = tc::idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_N128 = tc::idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t ID_N128_BMN = tc::idesc_bf16(128, 128, 0, 1);
    constexpr int GRP_CHAIN = 1, GRP_PREP = 2;   // named barrier ids (0 is __syncthreads)
    using L = WsSmem;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays a shared pointer
    const uint32_t sb = tc::smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::TSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::ABORT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int nchunks = (T + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < L::NBAR; ++i) tc::mbar_init(bars + i, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, NCOLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // bounded wait that also stops when another role has aborted
    auto wait = [&](int bi, uint32_t parity) -> bool {
        uint64_t* bar = bars + bi;
        if (tc::mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = tc::globaltimer_ns();
        while (true) {
            if (tc::mbar_try_wait(bar, parity)) return true;
            if (*abort_flag) return false;
            if (tc::globaltimer_ns() - t0 > wait_limit_ns) {
                *abort_flag = 1;
                atomicOr(&g_osdn_status, kStatusTimeout);
                return false;
            }
        }
    };

    if (warp < 4) regs_dec<56>();   // control warpgroup: one instruction for all four warps
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tm_q);
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_kw);
            int issued = 0, consumed_wait_ok = 1;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                if (c >= 2 && !wait(L::B_EMPTY + s, ((c >> 1) - 1) & 1)) { consumed_wait_ok = 0; break; }
                const int t0 = c * C;
                uint8_t* qk = sm + s * L::STAGE + L::QK0;
                uint8_t* kwb = sm + s * L::STAGE + L::KW0;
                tc::mbar_arrive_expect_tx(bars + L::B_FULL + s, L::kTxBytes);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tc::tma_load_4d(qk + half * 16384, &tm_k, half * 64, h, t0, b, bars + L::B_FULL + s);
                    tc::tma_load_4d(qk + half * 16384 + 8192, &tm_q, half * 64, h, t0, b, bars + L::B_FULL + s);
                    tc::tma_load_4d(kwb + half * 8192, &tm_kw, half * 64, h, t0, b, bars + L::B_FULL + s);
                }
                issued = c + 1;
            }
            (void)consumed_wait_ok;
            if (*abort_flag) {
                // drain: the loads of the last (up to) two chunks may still be in flight
                for (int c = (issued >= 2 ? issued - 2 : 0); c < issued; ++c)
                    tc::mbar_wait(bars + L::B_FULL + (c & 1), (c >> 1) & 1, 1000000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            auto mma1 = [&](int c) {   // D1[c % 2] = [K;Q] Kw^T
                const int s = c & 1;
                const uint32_t qk = sb + s * L::STAGE + L::QK0, kwb = sb + s * L::STAGE + L::KW0;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                    tc::umma_bf16(tmem + COL_D1 + s * 64, tc::sdesc_sw128(qk + half * 16384 + koff, 16, 1024),
                                  tc::sdesc_sw128(kwb + half * 8192 + koff, 16, 1024), ID_N64, ks > 0);
                }
                tc::umma_commit(bars + L::B_D1FULL + s);
            };
            bool ok = true;
            if (nchunks > 0) {
                ok = wait(L::B_FULL, 0);
                if (ok) { tc::tc_fence_after(); mma1(0); }
            }
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t qk = sb + s * L::STAGE + L::QK0, kwb = sb + s * L::STAGE + L::KW0;
                // MMA2(c): D2 = S [K;Q]^T
                if (!(ok = wait(L::B_SB, c & 1))) break;
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                    tc::umma_bf16(tmem + COL_D2, tc::sdesc_sw128(sb + L::SB + half * 16384 + koff, 16, 1024),
                                  tc::sdesc_sw128(qk + half * 16384 + koff, 16, 1024), ID_N128, ks > 0);
                }
                tc::umma_commit(bars + L::B_D2);
                // MMA1(c + 1), so the prep group can start on the next chunk
                if (c + 1 < nchunks) {
                    const int s1 = (c + 1) & 1;
                    if (!(ok = wait(L::B_FULL + s1, ((c + 1) >> 1) & 1))) break;
                    if (c + 1 >= 2 && !(ok = wait(L::B_D1FREE + s1, (((c + 1) >> 1) - 1) & 1))) break;
                    tc::tc_fence_after();
                    mma1(c + 1);
                }
                // MMA3(c): D3 = Xh^T T^T
                if (!(ok = wait(L::B_XU, c & 1))) break;
                if (!(ok = wait(L::B_TPREADY + s, (c >> 1) & 1))) break;
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16(tmem + COL_D3, tc::sdesc_sw128(sb + L::XU + ks * 32, 16, 1024),
                                  tc::sdesc_sw128(sb + L::TB + s * 8192 + ks * 32, 16, 1024), ID_N64, ks > 0);
                tc::umma_commit(bars + L::B_D3);
                // MMA5(c): DS += U^T Kw, then MMA4(c): D2[:, 64:] += U^T P^T
                if (!(ok = wait(L::B_U, c & 1))) break;
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16(tmem + COL_S, tc::sdesc_sw128(sb + L::XU + ks * 32, 16, 1024),
                                  tc::sdesc_sw128(kwb + ks * 2048, 8192, 1024), ID_N128_BMN, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16(tmem + COL_D2 + 64, tc::sdesc_sw128(sb + L::XU + ks * 32, 16, 1024),
                                  tc::sdesc_sw128(sb + L::PB + s * 8192 + ks * 32, 16, 1024), ID_N64, true);
                tc::umma_commit(bars + L::B_S);
                tc::umma_commit(bars + L::B_EMPTY + s);
            }
            // drain every MMA issued before TMEM is released
            tc::umma_commit(bars + L::B_DRAIN);
            tc::mbar_wait(bars + L::B_DRAIN, 0, 1000000000ull);
        }
        __syncwarp();
    } else if (warp < 4) {
        // warps 2-3: no role
    } else if (warp < 8) {
        // ------------------------------------------------------------ chain group
        regs_inc<224>();
        const int q4 = warp & 3;                   // TMEM lane quarter of this warp
        const int vrow = q4 * 32 + lane;           // value row of S owned
        const int gtid = tid - 128;                // 0..127 inside the group
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        float* betac = reinterpret_cast<float*>(sm + L::BETA_C);
        {   // initial state: TMEM fp32 and the bf16 copy for MMA2(0)
            const float* srow = S0 ? S0 + ((size_t)unit * DV + vrow) * DK : nullptr;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t r[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 x = srow ? *reinterpret_cast<const float4*>(srow + c4 * 32 + i)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    r[i] = __float_as_uint(x.x); r[i + 1] = __float_as_uint(x.y);
                    r[i + 2] = __float_as_uint(x.z); r[i + 3] = __float_as_uint(x.w);
                }
                tc::tmem_st32(tl + COL_S + c4 * 32, r);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 pk;
                    pk.x = tc::pack_bf16(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    pk.y = tc::pack_bf16(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    pk.z = tc::pack_bf16(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    pk.w = tc::pack_bf16(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    const int chunk16 = (c4 & 1) * 4 + cc;   // 16-byte chunk within the 64-column half
                    *reinterpret_cast<uint4*>(sm + L::SB + (c4 >> 1) * 16384 + tc::sw128_off(vrow, chunk16)) = pk;
                }
            }
            tc::tmem_wait_st();
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        named_sync(GRP_CHAIN, 128);
        if (gtid == 0 && nchunks > 0) mbar_arrive1(bars + L::B_SB);

        // V[t][v] of a chunk as raw 16-bit values, loaded one chunk ahead
        const unsigned short* vbase = reinterpret_cast<const unsigned short*>(v) + (size_t)h * DV + vrow;
        auto load_v = [&](int c, uint32_t (&raw)[C]) {
            const int tt0 = c * C, n = min(C, T - tt0);
            const unsigned short* vp = vbase + ((size_t)b * T + tt0) * H * DV;
#pragma unroll
            for (int t = 0; t < C; ++t) raw[t] = (t < n) ? (uint32_t)vp[(size_t)t * H * DV] : 0u;
        };
        uint32_t vraw[C];
        if (nchunks > 0) load_v(0, vraw);

        for (int c = 0; c < nchunks; ++c) {
            const int t0 = c * C, Tc = min(C, T - t0);
            if (gtid < C) betac[gtid] = gtid < Tc ? __bfloat162float(beta[((size_t)b * T + t0 + gtid) * H + h]) : 0.f;
            uint32_t vv[C / 2];   // this chunk's V packed as bf16 pairs; then the next chunk's loads go out
#pragma unroll
            for (int i = 0; i < C / 2; ++i) vv[i] = vraw[2 * i] | (vraw[2 * i + 1] << 16);
            if (c + 1 < nchunks) load_v(c + 1, vraw);
            // the previous chunk's O store must have left the Xh/U tile
            if (gtid == 0) tc::bulk_wait_read<0>();
            // Xh^T row v = beta_t (V[t][v] - (S K^T)^T[v][t])  -> bf16 smem
            bool fail = !wait(L::B_D2, c & 1);
            if (named_sync_or(GRP_CHAIN, 128, fail)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
                uint32_t r[32];
                tc::tmem_ld32(tl + COL_D2 + qh * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = qh * 32 + cc * 8 + e;
                        const float vt = __uint_as_float((t & 1) ? (vv[t >> 1] & 0xFFFF0000u) : (vv[t >> 1] << 16));
                        x[e] = betac[t] * (vt - __uint_as_float(r[cc * 8 + e]));
                    }
                    uint4 pk;
                    pk.x = tc::pack_bf16(x[0], x[1]); pk.y = tc::pack_bf16(x[2], x[3]);
                    pk.z = tc::pack_bf16(x[4], x[5]); pk.w = tc::pack_bf16(x[6], x[7]);
                    *reinterpret_cast<uint4*>(sm + L::XU + tc::sw128_off(vrow, qh * 4 + cc)) = pk;
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            named_sync(GRP_CHAIN, 128);
            if (gtid == 0) mbar_arrive1(bars + L::B_XU);
            // U^T row v -> bf16 smem (MMA3 has consumed Xh^T)
            fail = !wait(L::B_D3, c & 1);
            if (named_sync_or(GRP_CHAIN, 128, fail)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
                uint32_t r[32];
                tc::tmem_ld32(tl + COL_D3 + qh * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 pk;
                    pk.x = tc::pack_bf16(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    pk.y = tc::pack_bf16(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    pk.z = tc::pack_bf16(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    pk.w = tc::pack_bf16(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4*>(sm + L::XU + tc::sw128_off(vrow, qh * 4 + cc)) = pk;
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            named_sync(GRP_CHAIN, 128);
            if (gtid == 0) mbar_arrive1(bars + L::B_U);
            // state S_{c+1} and O_c are ready: O^T row to registers, S to the bf16 copy (or out)
            fail = !wait(L::B_S, c & 1);
            if (named_sync_or(GRP_CHAIN, 128, fail)) break;
            tc::tc_fence_after();
            {   // O^T row v -> O[t][v] staged in the Xh/U tile (MMA5/MMA4 have consumed U^T)
                __nv_bfloat16* Os = reinterpret_cast<__nv_bfloat16*>(sm + L::XU);
#pragma unroll
                for (int qh = 0; qh < 2; ++qh) {
                    uint32_t r[32];
                    tc::tmem_ld32(tl + COL_D2 + 64 + qh * 32, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) Os[(qh * 32 + e) * DV + vrow] = __float2bfloat16_rn(__uint_as_float(r[e]));
                }
            }
            if (c + 1 < nchunks) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int qh = 0; qh < 2; ++qh) {
                        uint32_t r[32];
                        tc::tmem_ld32(tl + COL_S + half * 64 + qh * 32, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            uint4 pk;
                            pk.x = tc::pack_bf16(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                            pk.y = tc::pack_bf16(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                            pk.z = tc::pack_bf16(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                            pk.w = tc::pack_bf16(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                            *reinterpret_cast<uint4*>(sm + L::SB + half * 16384 + tc::sw128_off(vrow, qh * 4 + cc)) = pk;
                        }
                    }
                }
                tc::fence_proxy_async_smem();
                tc::tc_fence_before();
                named_sync(GRP_CHAIN, 128);
                if (gtid == 0) {
                    mbar_arrive1(bars + L::B_SB);
                    tc::tma_store_4d(&tm_out, sm + L::XU, 0, h, t0, b);
                    tc::bulk_commit();
                }
            } else {
                tc::fence_proxy_async_smem();
                named_sync(GRP_CHAIN, 128);
                if (gtid == 0) {
                    tc::tma_store_4d(&tm_out, sm + L::XU, 0, h, t0, b);
                    tc::bulk_commit();
                }
                if (S_final) {
                float* srow = S_final + ((size_t)unit * DV + vrow) * DK;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t r[32];
                    tc::tmem_ld32(tl + COL_S + c4 * 32, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(srow + c4 * 32 + i) =
                            make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                        __uint_as_float(r[i + 3]));
                }
                }
            }
        }
        if (gtid == 0) tc::bulk_wait<0>();
        tc::tc_fence_before();
    } else {
        // ------------------------------------------------------------ prep group
        regs_inc<224>();
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;            // D1 row: Gram row (< 64) or score row
        const int gtid = tid - 256;                // 0..127 inside the group
        const int gw = warp - 8;                   // warp index inside the group
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        float* betap = reinterpret_cast<float*>(sm + L::BETA_P);
        float* AF = reinterpret_cast<float*>(sm + L::AF);
        float* TF = reinterpret_cast<float*>(sm + L::TF);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1, t0 = c * C, Tc = min(C, T - t0);
            if (gtid < C) betap[gtid] = gtid < Tc ? __bfloat162float(beta[((size_t)b * T + t0 + gtid) * H + h]) : 0.f;
            bool fail = !wait(L::B_D1FULL + s, (c >> 1) & 1);
            if (named_sync_or(GRP_PREP, 128, fail)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
                uint32_t r[32];
                tc::tmem_ld32(tl + COL_D1 + s * 64 + qh * 32, r);
                tc::tmem_wait_ld();
                if (row < C) {   // A[t][j] = beta_t <k_t, kw_j> for j < t
                    const float bt = betap[row];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = qh * 32 + e;
                        AF[row * L::LDF + j] = (j < row) ? bt * __uint_as_float(r[e]) : 0.f;
                    }
                } else {         // P[t][j] = <q_t, kw_j> for j <= t
                    const int t = row - C;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = qh * 32 + cc * 8 + e;
                            x[e] = (j <= t) ? __uint_as_float(r[cc * 8 + e]) : 0.f;
                        }
                        uint4 pk;
                        pk.x = tc::pack_bf16(x[0], x[1]); pk.y = tc::pack_bf16(x[2], x[3]);
                        pk.z = tc::pack_bf16(x[4], x[5]); pk.w = tc::pack_bf16(x[6], x[7]);
                        *reinterpret_cast<uint4*>(sm + L::PB + s * 8192 + tc::sw128_off(t, qh * 4 + cc)) = pk;
                    }
                }
            }
            tc::tc_fence_before();
            named_sync(GRP_PREP, 128);
            if (gtid == 0) mbar_arrive1(bars + L::B_D1FREE + s);
            tri::tril_inv64(AF, TF, gw, lane, [] { named_sync(2, 128); });
            if (gtid < C) {   // T -> bf16 K-major swizzled (B operand of MMA3)
                const int t = gtid;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 pk;
                    const float* rw = TF + t * L::LDF + cc * 8;
                    pk.x = tc::pack_bf16(rw[0], rw[1]); pk.y = tc::pack_bf16(rw[2], rw[3]);
                    pk.z = tc::pack_bf16(rw[4], rw[5]); pk.w = tc::pack_bf16(rw[6], rw[7]);
                    *reinterpret_cast<uint4*>(sm + L::TB + s * 8192 + tc::sw128_off(t, cc)) = pk;
                }
            }
            tc::fence_proxy_async_smem();
            named_sync(GRP_PREP, 128);
            if (gtid == 0) mbar_arrive1(bars + L::B_TPREADY + s);
        }
        tc::tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, NCOLS);
    }
}

}  // namespace osdn
