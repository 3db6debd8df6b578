// Chunkwise OSDN forward on sm_100a: two warp groups sharing one tensor core.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1: the DeltaNet chunkwise WY
// pipeline with the scaled write key Kw = D (.) K substituted in the block
// Gram matrix and the intra-block scores; the read/erase key K unchanged.
// Per chunk of C = 64 tokens with chunk-start state S (dv x dk, fp32):
//   A = strict_tril(diag(beta) K Kw^T),   T = (I + A)^{-1},
//   U = T diag(beta) (V - K S^T),
//   O = Q S^T + tril(Q Kw^T) U,           S <- S + U^T Kw.
// Every contraction is a tcgen05 MMA with M = 128 (value rows of S or the
// stacked [K; Q] tokens on M), bf16 operands in 128-byte-swizzled shared
// memory, fp32 accumulators in TMEM:
//   MMA1  D1[c%2] = [K; Q] Kw^T       Gram (rows 0-63) and scores (rows 64-127)
//   (MMA2-MMA5 take their A operand from TMEM)
//   MMA2  D2 = S K^T | S Q^T          (transposed; S K^T issued and committed first)
//   MMA3  D3 = Xh^T T^T = U^T         Xh = diag(beta)(V - K S^T)
//   MMA5  DS += U^T Kw                state carry; S stays in TMEM all sequence
//   MMA4  D2[:, 64:] += U^T P^T       O^T
//
// One CTA (256 threads) per (sequence, head), two groups of four warps:
//   chain group (warps 0-3, TMEM lane = value row v): owns the state. Its
//     elected thread issues the TMA loads (chunk c + 2 into stage c % 2 once
//     chunk c has consumed it) and MMA2, MMA3, MMA5 + MMA4, each right after
//     the group has written that MMA's A operand. Those A operands live in
//     TMEM (bf16, two per column): the bf16 copy of S, Xh^T written over the
//     S K^T columns it was formed from, U^T written over its own fp32 columns;
//     only the B operands (TMA tiles, T, P) are read from shared memory. O
//     leaves through a staging tile and one TMA store.
//   prep group (warps 4-7, TMEM lane = Gram / score row): everything that does
//     not depend on the state, one chunk ahead: A (fp32) and P (bf16) from D1,
//     T = (I + A)^{-1} (blocked inverse), T -> bf16; its elected thread then
//     issues MMA1 of the next chunk into the other D1 buffer.
// Hand-offs between the groups and with the tensor core are mbarriers (a TMA
// transaction count, a tcgen05.commit, or one elected arrival). Every wait is
// bounded: a wait that gives up sets the library status word and a shared
// abort flag; each group leaves at its next group-wide wait, taking that
// decision together through a barrier-OR; issued MMAs and loads are drained
// before TMEM is released.
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct WsSmem {
    static constexpr uint32_t STAGE = 65536;            // per stage: [K;Q] 32 KB, Kw 16 KB, V 16 KB
    static constexpr uint32_t QK0 = 0;
    static constexpr uint32_t KW0 = 32768;
    static constexpr uint32_t V0 = 49152;               // V [64 t][128 v] bf16, unswizzled
    static constexpr uint32_t OST = 2 * STAGE;          // O staging [64 t][128 v] bf16 for the TMA store
    static constexpr uint32_t TB = OST + 16384;         // T bf16 [64][64], two buffers of 8 KB
    static constexpr uint32_t PB = TB + 16384;          // P bf16 [64][64], two buffers of 8 KB
    static constexpr int LDF = tri::LD;
    static constexpr uint32_t AF = PB + 16384;          // A fp32 [64][LDF]
    static constexpr uint32_t TF = AF + 64 * LDF * 4;   // T fp32 [64][LDF]
    static constexpr uint32_t BETA_C = TF + 64 * LDF * 4;   // chain group's beta of its chunk
    static constexpr uint32_t BETA_P = BETA_C + 256;        // prep group's beta of its chunk
    static constexpr uint32_t BAR = BETA_P + 256;
    enum { B_FULL = 0, B_D1FULL = 2, B_TPREADY = 4, B_D2 = 6, B_D3 = 7, B_S = 8, B_DRAIN = 9, NBAR = 11 };
    static constexpr uint32_t TSLOT = BAR + NBAR * 8;   // TMEM base address
    static constexpr uint32_t ABORT = TSLOT + 4;        // abort flag
    static constexpr uint32_t END = ABORT + 4;
    static constexpr size_t kBytes = END + 1024;
    static constexpr uint32_t kTxBytes = 6 * 8192 + 16384;   // TMA bytes per chunk (K, Q, Kw halves, V)
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

__device__ __forceinline__ uint4 pack8_bf16(const uint32_t* r) {
    uint4 pk;
    pk.x = tc::pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1]));
    pk.y = tc::pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3]));
    pk.z = tc::pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5]));
    pk.w = tc::pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7]));
    return pk;
}

template <int kUnused = 0>
__global__ void __launch_bounds__(256, 1)
chunk_ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_kw, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_out, const __nv_bfloat16* __restrict__ beta,
                const float* __restrict__ S0, float* __restrict__ S_final, int B, int T, int H,
                unsigned long long wait_limit_ns)
{
    constexpr int C = 64, DK = 128, DV = 128;
    // TMEM columns: state fp32 | D2 (S K^T, then Xh^T bf16 in its first 32 columns | O^T) |
    // D1 x 2 | D3 (U^T fp32, then U^T bf16 in its first 32 columns) | bf16 copy of the state
    constexpr uint32_t COL_S = 0, COL_D2 = 128, COL_D1 = 256, COL_D3 = 384, COL_SB = 448, NCOLS = 512;
    constexpr uint32_t ID_N64 = tc::idesc_bf16(128, 64, 0, 0);
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

    // bounded wait that also stops when the other group has aborted
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
    // TMA of chunk c (K, Q halves into the [K;Q] tile, Kw halves) into stage c % 2
    auto issue_loads = [&](int c) {
        const int s = c & 1, t0 = c * C;
        uint8_t* qk = sm + s * L::STAGE + L::QK0;
        uint8_t* kwb = sm + s * L::STAGE + L::KW0;
        uint64_t* fb = bars + L::B_FULL + s;
        tc::mbar_arrive_expect_tx(fb, L::kTxBytes);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tc::tma_load_4d(qk + half * 16384, &tm_k, half * 64, h, t0, b, fb);
            tc::tma_load_4d(qk + half * 16384 + 8192, &tm_q, half * 64, h, t0, b, fb);
            tc::tma_load_4d(kwb + half * 8192, &tm_kw, half * 64, h, t0, b, fb);
        }
        tc::tma_load_4d(sm + s * L::STAGE + L::V0, &tm_v, 0, h, t0, b, fb);
    };
    // shared-memory descriptors of the fixed tiles; a byte offset within a tile adds (off >> 4)
    const uint64_t dQK[2] = {tc::sdesc_sw128(sb + L::QK0, 16, 1024), tc::sdesc_sw128(sb + L::STAGE + L::QK0, 16, 1024)};
    const uint64_t dKW[2] = {tc::sdesc_sw128(sb + L::KW0, 16, 1024), tc::sdesc_sw128(sb + L::STAGE + L::KW0, 16, 1024)};

    if (warp < 4) {
        // ================================================================ chain group
        const int gtid = tid;                      // 0..127
        const int vrow = tid;                      // value row of S owned (TMEM lane)
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        float* betac = reinterpret_cast<float*>(sm + L::BETA_C);
        const uint64_t dKWmn[2] = {tc::sdesc_sw128(sb + L::KW0, 8192, 1024),
                                   tc::sdesc_sw128(sb + L::STAGE + L::KW0, 8192, 1024)};
        const uint64_t dTB = tc::sdesc_sw128(sb + L::TB, 16, 1024);
        const uint64_t dPB = tc::sdesc_sw128(sb + L::PB, 16, 1024);
        // bf16 copy of a 128-column fp32 state row, packed two per TMEM column (the A operand of MMA2)
        auto store_state_bf16 = [&](const uint32_t (&row)[128]) {
            uint32_t w[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    w[i] = tc::pack_bf16(__uint_as_float(row[half * 64 + 2 * i]), __uint_as_float(row[half * 64 + 2 * i + 1]));
                tc::tmem_st32(tl + COL_SB + half * 32, w);
            }
        };

        // gtid 0 issues the MMAs, gtid 32 (another warp) the TMA loads and stores, so
        // neither waits behind the other
        constexpr int kMmaThread = 0, kTmaThread = 32;
        int issued = 0;   // chunks whose loads were issued (TMA thread)
        if (gtid == kTmaThread) {
            if (nchunks > 0) issue_loads(issued++);
            if (nchunks > 1) issue_loads(issued++);
        }
        // MMA2(c): S K^T (commit) then S Q^T; A = bf16 state in TMEM, B = chunk c's [K;Q] tile
        auto mma2 = [&](int c) -> bool {
            const int sc = c & 1;
            if (!wait(L::B_FULL + sc, (c >> 1) & 1)) return false;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::umma_bf16_ts(tmem + COL_D2, tmem + COL_SB + ks * 8, dQK[sc] + (off >> 4), ID_N64, ks > 0);
            }
            tc::umma_commit(bars + L::B_D2);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::umma_bf16_ts(tmem + COL_D2 + 64, tmem + COL_SB + ks * 8, dQK[sc] + ((off + 8192) >> 4), ID_N64,
                                 ks > 0);
            }
            return true;
        };
        {   // initial state: TMEM fp32 and its bf16 copy
            const float* srow = S0 ? S0 + ((size_t)unit * DV + vrow) * DK : nullptr;
            uint32_t row[128];
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
                float4 x = srow ? *reinterpret_cast<const float4*>(srow + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                row[i] = __float_as_uint(x.x); row[i + 1] = __float_as_uint(x.y);
                row[i + 2] = __float_as_uint(x.z); row[i + 3] = __float_as_uint(x.w);
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) tc::tmem_st32(tl + COL_S + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(row + c4 * 32));
            store_state_bf16(row);
            tc::tmem_wait_st();
        }
        auto load_beta = [&](int c) -> float {
            const int tt0 = c * C;
            return (gtid < C && gtid < T - tt0) ? __bfloat162float(beta[((size_t)b * T + tt0 + gtid) * H + h]) : 0.f;
        };
        float bnext = nchunks > 0 ? load_beta(0) : 0.f;
        tc::tc_fence_before();
        named_sync(GRP_CHAIN, 128);
        if (gtid == kMmaThread && nchunks > 0) mma2(0);

        bool fail = false;
        int c = 0;
        for (; c < nchunks; ++c) {
            const int s = c & 1, t0 = c * C;
            if (gtid < C) betac[gtid] = bnext;
            if (c + 1 < nchunks) bnext = load_beta(c + 1);

            // Xh^T row v = beta_t (V[t][v] - (S K^T)^T[v][t]) -> bf16 over D2 columns 0-31; then MMA3(c)
            fail = !wait(L::B_D2, c & 1) || !wait(L::B_FULL + s, (c >> 1) & 1);   // the V tile is this stage's
            if (named_sync_or(GRP_CHAIN, 128, fail)) break;
            tc::tc_fence_after();
            {
                const unsigned short* Vs = reinterpret_cast<const unsigned short*>(sm + s * L::STAGE + L::V0);
                uint32_t x1[64];
                tc::tmem_ld32(tl + COL_D2, *reinterpret_cast<uint32_t(*)[32]>(x1));
                tc::tmem_ld32(tl + COL_D2 + 32, *reinterpret_cast<uint32_t(*)[32]>(x1 + 32));
                tc::tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = 2 * i;
                    const float v0 = __uint_as_float((uint32_t)Vs[t * DV + vrow] << 16);
                    const float v1 = __uint_as_float((uint32_t)Vs[(t + 1) * DV + vrow] << 16);
                    w[i] = tc::pack_bf16(betac[t] * (v0 - __uint_as_float(x1[t])),
                                         betac[t + 1] * (v1 - __uint_as_float(x1[t + 1])));
                }
                tc::tmem_st32(tl + COL_D2, w);
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            named_sync(GRP_CHAIN, 128);
            if (gtid == kMmaThread) {
                if (wait(L::B_TPREADY + s, (c >> 1) & 1)) {
                    tc::tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc::umma_bf16_ts(tmem + COL_D3, tmem + COL_D2 + ks * 8, dTB + ((s * 8192 + ks * 32) >> 4), ID_N64,
                                         ks > 0);
                    tc::umma_commit(bars + L::B_D3);
                }
            }

            // U^T row v -> bf16 over D3 columns 0-31; then MMA5(c) and MMA4(c)
            fail = !wait(L::B_D3, c & 1);
            if (named_sync_or(GRP_CHAIN, 128, fail)) break;
            tc::tc_fence_after();
            {
                uint32_t u[64], w[32];
                tc::tmem_ld32(tl + COL_D3, *reinterpret_cast<uint32_t(*)[32]>(u));
                tc::tmem_ld32(tl + COL_D3 + 32, *reinterpret_cast<uint32_t(*)[32]>(u + 32));
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = tc::pack_bf16(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
                tc::tmem_st32(tl + COL_D3, w);
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            named_sync(GRP_CHAIN, 128);
            if (gtid == kMmaThread) {
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16_ts(tmem + COL_S, tmem + COL_D3 + ks * 8, dKWmn[s] + ks * 128, ID_N128_BMN, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16_ts(tmem + COL_D2 + 64, tmem + COL_D3 + ks * 8, dPB + ((s * 8192 + ks * 32) >> 4), ID_N64,
                                     true);
                tc::umma_commit(bars + L::B_S);
            }

            // S_{c+1} and O_c are ready; stage s is consumed
            fail = !wait(L::B_S, c & 1);
            if (named_sync_or(GRP_CHAIN, 128, fail)) break;
            tc::tc_fence_after();
            uint32_t orow[C];   // O^T row v, read before MMA2 of the next chunk overwrites D2
            tc::tmem_ld32(tl + COL_D2 + 64, *reinterpret_cast<uint32_t(*)[32]>(orow));
            tc::tmem_ld32(tl + COL_D2 + 96, *reinterpret_cast<uint32_t(*)[32]>(orow + 32));
            {
                uint32_t row[128];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) tc::tmem_ld32(tl + COL_S + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(row + c4 * 32));
                tc::tmem_wait_ld();
                if (c + 1 < nchunks) {
                    store_state_bf16(row);   // A operand of MMA2 of the next chunk
                    tc::tmem_wait_st();
                } else if (S_final) {
                    float* srow = S_final + ((size_t)unit * DV + vrow) * DK;
#pragma unroll
                    for (int i = 0; i < 128; i += 4)
                        *reinterpret_cast<float4*>(srow + i) = make_float4(__uint_as_float(row[i]), __uint_as_float(row[i + 1]),
                                                                           __uint_as_float(row[i + 2]), __uint_as_float(row[i + 3]));
                }
            }
            if (gtid == kTmaThread) tc::bulk_wait_read<0>();   // the previous O store has left the staging tile
            tc::tc_fence_before();
            named_sync(GRP_CHAIN, 128);
            if (gtid == kMmaThread && c + 1 < nchunks) mma2(c + 1);   // the next chunk starts on the tensor core now
            {   // O[t][v] into the staging tile; one TMA store
                unsigned short* Os = reinterpret_cast<unsigned short*>(sm + L::OST);
#pragma unroll
                for (int t = 0; t < C; ++t) {
                    const __nv_bfloat16 ob = __float2bfloat16_rn(__uint_as_float(orow[t]));
                    Os[t * DV + vrow] = *reinterpret_cast<const unsigned short*>(&ob);
                }
            }
            tc::fence_proxy_async_smem();
            named_sync(GRP_CHAIN, 128);
            if (gtid == kTmaThread) {
                tc::tma_store_4d(&tm_out, sm + L::OST, 0, h, t0, b);
                tc::bulk_commit();
                if (c + 2 < nchunks) issue_loads(issued++);   // stage s is consumed
            }
        }
        if (gtid == kMmaThread) {   // drain every MMA this thread issued before TMEM is released
            tc::umma_commit(bars + L::B_DRAIN);
            tc::mbar_wait(bars + L::B_DRAIN, 0, 1000000000ull);
        }
        if (gtid == kTmaThread) {   // stores done; loads of chunks the loop did not reach have landed
            tc::bulk_wait<0>();
            for (int cc = c; cc < issued; ++cc)
                tc::mbar_wait(bars + L::B_FULL + (cc & 1), (cc >> 1) & 1, 1000000000ull);
        }
        tc::tc_fence_before();
    } else {
        // ================================================================ prep group
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;            // D1 row: Gram row (< 64) or score row
        const int gtid = tid - 128;                // 0..127 inside the group
        const int gw = warp - 4;                   // warp index inside the group
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        float* betap = reinterpret_cast<float*>(sm + L::BETA_P);
        float* AF = reinterpret_cast<float*>(sm + L::AF);
        float* TF = reinterpret_cast<float*>(sm + L::TF);
        auto mma1 = [&](int c) {   // D1[c % 2] = [K;Q] Kw^T, after chunk c's tiles have landed
            const int s = c & 1;
            if (!wait(L::B_FULL + s, (c >> 1) & 1)) return;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                tc::umma_bf16(tmem + COL_D1 + s * 64, dQK[s] + ((half * 16384 + koff) >> 4),
                              dKW[s] + ((half * 8192 + koff) >> 4), ID_N64, ks > 0);
            }
            tc::umma_commit(bars + L::B_D1FULL + s);
        };
        auto load_beta = [&](int c) -> float {
            const int tt0 = c * C;
            return (gtid < C && gtid < T - tt0) ? __bfloat162float(beta[((size_t)b * T + tt0 + gtid) * H + h]) : 0.f;
        };
        if (gtid == 0 && nchunks > 0) mma1(0);
        float bnext = nchunks > 0 ? load_beta(0) : 0.f;
        tri::tril_zero_upper(TF, gtid, 128);   // the inverse never writes those blocks
        named_sync(GRP_PREP, 128);
        int mma1_next = 1;                     // next chunk whose MMA1 is not issued yet
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            if (gtid < C) betap[gtid] = bnext;
            if (c + 1 < nchunks) bnext = load_beta(c + 1);
            bool fail = !wait(L::B_D1FULL + s, (c >> 1) & 1);
            if (named_sync_or(GRP_PREP, 128, fail)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
                uint32_t r[32];
                tc::tmem_ld32(tl + COL_D1 + s * 64 + qh * 32, r);
                tc::tmem_wait_ld();
                if (row < C) {   // A[t][j] = beta_t <k_t, kw_j> for j < t (row stride 68: conflict-free 16-byte stores)
                    const float bt = betap[row];
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const int j = qh * 32 + e;
                        *reinterpret_cast<float4*>(AF + row * L::LDF + j) =
                            make_float4((j < row) ? bt * __uint_as_float(r[e]) : 0.f,
                                        (j + 1 < row) ? bt * __uint_as_float(r[e + 1]) : 0.f,
                                        (j + 2 < row) ? bt * __uint_as_float(r[e + 2]) : 0.f,
                                        (j + 3 < row) ? bt * __uint_as_float(r[e + 3]) : 0.f);
                    }
                } else {         // P[t][j] = <q_t, kw_j> for j <= t  (MMA4 of chunk c - 2 has read P[s])
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
            // MMA1 of the next chunk now if its tiles have landed (D1[(c+1) % 2] was read in chunk c - 1),
            // so it runs under the inverse; otherwise after it
            if (gtid == 0 && mma1_next == c + 1 && c + 1 < nchunks &&
                tc::mbar_test(bars + L::B_FULL + ((c + 1) & 1), ((c + 1) >> 1) & 1)) {
                mma1(c + 1);
                mma1_next = c + 2;
            }
            tri::tril_inv64(AF, TF, gw, lane, [] { named_sync(2, 128); });
            {   // T -> bf16 K-major swizzled (B operand of MMA3): thread -> half a row
                const int t = gtid & 63, hf = gtid >> 6;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const float4 lo = *reinterpret_cast<const float4*>(TF + t * L::LDF + hf * 32 + cc * 8);
                    const float4 hi = *reinterpret_cast<const float4*>(TF + t * L::LDF + hf * 32 + cc * 8 + 4);
                    uint4 pk;
                    pk.x = tc::pack_bf16(lo.x, lo.y); pk.y = tc::pack_bf16(lo.z, lo.w);
                    pk.z = tc::pack_bf16(hi.x, hi.y); pk.w = tc::pack_bf16(hi.z, hi.w);
                    *reinterpret_cast<uint4*>(sm + L::TB + s * 8192 + tc::sw128_off(t, hf * 4 + cc)) = pk;
                }
            }
            tc::fence_proxy_async_smem();
            named_sync(GRP_PREP, 128);
            if (gtid == 0) {
                mbar_arrive1(bars + L::B_TPREADY + s);
                if (mma1_next == c + 1 && c + 1 < nchunks) {
                    mma1(c + 1);
                    mma1_next = c + 2;
                }
            }
        }
        if (gtid == 0) {   // drain this thread's MMAs
            tc::umma_commit(bars + L::B_DRAIN + 1);
            tc::mbar_wait(bars + L::B_DRAIN + 1, 0, 1000000000ull);
        }
        tc::tc_fence_before();
    }

    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, NCOLS);
    }
}

}  // namespace osdn
