// Chunkwise OSDN forward on sm_100a: WY form with the state-independent parts
// (W, U0, scores) prepared ahead of a short state chain.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1: the DeltaNet chunkwise WY
// pipeline with the scaled write key Kw = D (.) K substituted in the block
// Gram matrix and the intra-block scores; the read/erase key K unchanged.
// Per chunk of C = 64 tokens with chunk-start state S (dv x dk, fp32):
//   A = strict_tril(diag(beta) K Kw^T),   T = (I + A)^{-1},
//   W = T diag(beta) K,   U0 = T diag(beta) V          (no state in them)
//   Vn = U0 - W S^T                                    (= T diag(beta)(V - K S^T))
//   O = Q S^T + tril(Q Kw^T) Vn,          S <- S + Vn^T Kw.
// Only Vn -> S -> next Vn is serial in the chunk index.
//
// Every contraction is a tcgen05 MMA with M = 128 and fp32 TMEM accumulators,
// bf16 operands in 128-byte-swizzled shared memory or (A only) in TMEM. The
// state-side products are transposed so that value row v of S is TMEM lane v:
//   G1  R1[c%3]  = [K; Q] Kw^T        Gram rows (lanes 0-63), score rows (64-127)
//   GW  R1[c%3]  = K^T (T diag(beta))^T = W^T            lane = key feature
//   GU  D[0,64)  = V^T (T diag(beta))^T = U0^T           lane = value row
//   GA  D       += S_bf16 [-W; Q]^T   D[0,64) = Vn^T, D[64,128) = (Q S^T)^T
//   GB  S       += Vn^T Kw;   D[64,128) += Vn^T P^T  ->  O^T   (P = tril(Q Kw^T))
//
// One CTA (288 threads) per (sequence, head):
//   state group (warps 0-3, lane v): owns S. Writes the TMEM A operands of the
//     chain (bf16 S, bf16 Vn over its own fp32 columns), turns W^T into -W rows
//     of the next chunk's [-W; Q] tile (over K, which G1 and GW have consumed),
//     stages O and stores it by TMA. Thread 32 issues all TMA traffic.
//   prep group (warps 4-7): for a chunk up to two ahead, A (fp32) and P (bf16)
//     from G1, T = (I + A)^{-1} in place, T diag(beta) -> bf16.
//   issuer warp (warp 8, one lane): every MMA, in a fixed order per chunk that
//     puts the state chain first, so that issuing (which stalls the issuing
//     thread while the tensor pipe is busy) never holds up a group; between
//     issues it sleeps in mbarrier waits rather than spinning.
// Shared memory: a three-stage ring of [K; Q] + Kw tiles (the next loads go out
// as soon as a chunk's GB completes), two V tiles (the older one doubles as
// the O staging tile), T diag(beta), two P tiles, the fp32 Gram / inverse.
// Hand-offs are mbarriers (TMA transaction counts, tcgen05.commit, one elected
// arrival). Every wait is bounded: a wait that gives up sets the library status
// word and a shared abort flag; the groups leave at their next group-wide wait
// (a barrier-OR), issued MMAs and loads are drained before TMEM is released.
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct WyLayout {
    static constexpr uint32_t STAGE = 49152, NSTAGE = 3;   // [K0|Q0|K1|Q1] (8 KB each) + [Kw0|Kw1]
    static constexpr uint32_t QK = 0, KW = 32768;
    static constexpr uint32_t VB = NSTAGE * STAGE;          // two V tiles [V0|V1], 16 KB each
    static constexpr uint32_t TB = VB + 2 * 16384;          // T diag(beta) bf16 [64 t][64 j]
    static constexpr uint32_t TB2 = TB + 8192;              // gated: T diag(beta / gamma) bf16 (B operand of GU)
    static constexpr uint32_t PB = TB2 + 8192;              // two P tiles bf16 [64 t][64 j]
    static constexpr int LDF = tri::LD;
    static constexpr uint32_t AF = PB + 2 * 8192;           // A, then T, fp32 [64][LDF]
    static constexpr uint32_t BETA = AF + 64 * LDF * 4;     // prep group's beta of its chunk
    static constexpr uint32_t BETAG = BETA + 256;           // gated: beta / gamma of the prep group's chunk
    static constexpr uint32_t GSCR = BETAG + 256;           // gated: prep scratch (gamma_31)
    static constexpr uint32_t BAR = GSCR + 16;
    enum {
        FULLQ = 0,   // 3: K, Q, Kw of a stage landed
        FULLV = 3,   // 2: V tile landed
        D1 = 5,      // 3: G1 into R1[i] done
        BW = 8,      // GW done
        BA = 9,      // GA done
        BS = 10,     // 2: GB done (by chunk parity)
        ETB = 12,    // prep: T diag(beta) and P of its chunk written
        EWE = 13,    // state: -W of its chunk written
        ESB = 14,    // state: bf16 S written, O^T columns read and zeroed
        EVN = 15,    // state: bf16 Vn written
        DRAIN = 16,
        NBAR = 17
    };
    static constexpr uint32_t TSLOT = BAR + NBAR * 8;       // TMEM base address
    static constexpr uint32_t ABORT = TSLOT + 4;
    static constexpr uint32_t END = ABORT + 4;
    static constexpr size_t kBytes = END + 1024;
    static constexpr uint32_t kTxQ = 6 * 8192;              // K, Q, Kw halves
    static constexpr uint32_t kTxV = 2 * 8192;
};

__device__ __forceinline__ unsigned short bf16_bits(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<const unsigned short*>(&h);
}

// Transposing epilogue, one warp: TMEM lanes m0..m0+31 (matrix row index m)
// x 64 columns (token t), fp32, become bf16 rows t of a 128-byte-swizzled
// K-major tile: element (t, m) at tile + (m / 64) * half_stride, row t, 16-byte
// chunk (m % 64) / 8. The load uses the 16x256b shape (two adjacent columns per
// thread); the store writes 8 x 8 tiles transposed with stmatrix, 16 bytes per
// row per tile.
struct ColsToRows {
    uint32_t lo[32], hi[32];
    __device__ __forceinline__ void load(uint32_t taddr) {   // wait with tcgen05.wait::ld before store()
        tc::tmem_ld16x256b_x8(taddr, lo);                   // lanes m0 + 0..15
        tc::tmem_ld16x256b_x8(taddr + (16u << 16), hi);     // lanes m0 + 16..31
    }
    // Column (token) t = 8j + 2(lane % 4) + e of the thread's values is scaled by sc[2j + e].
    __device__ __forceinline__ void store(uint8_t* tile, uint32_t half_stride, int m0, const float (&sc)[16],
                                          int lane) const {
        const int k = lane >> 3, c = lane & 7;              // this thread addresses row c of 8 x 8 tile k
        const int mk = m0 + 8 * k;                          // first matrix row index of tile k
        uint8_t* base = tile + (mk >> 6) * half_stride;
        const int ch = (mk & 63) >> 3;
#pragma unroll
        for (int j = 0; j < 8; ++j) {                       // tokens 8j..8j+7
            const float s0 = sc[2 * j], s1 = sc[2 * j + 1];
            const uint32_t p0 = tc::pack_bf16(s0 * __uint_as_float(lo[4 * j]), s1 * __uint_as_float(lo[4 * j + 1]));
            const uint32_t p1 = tc::pack_bf16(s0 * __uint_as_float(lo[4 * j + 2]), s1 * __uint_as_float(lo[4 * j + 3]));
            const uint32_t p2 = tc::pack_bf16(s0 * __uint_as_float(hi[4 * j]), s1 * __uint_as_float(hi[4 * j + 1]));
            const uint32_t p3 = tc::pack_bf16(s0 * __uint_as_float(hi[4 * j + 2]), s1 * __uint_as_float(hi[4 * j + 3]));
            tc::stmatrix_x4_trans(tc::smem_u32(base + tc::sw128_off(8 * j + c, ch)), p0, p1, p2, p3);
        }
    }
    __device__ __forceinline__ void store(uint8_t* tile, uint32_t half_stride, int m0, float scale, int lane) const {
        float sc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) sc[i] = scale;
        store(tile, half_stride, m0, sc, lane);
    }
};

// Inclusive prefix product over the 32 lanes of a warp.
__device__ __forceinline__ float warp_prefix_product(float x, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x *= y;
    }
    return x;
}

// GATED: the gated delta rule backbone, S_t = alpha_t S_{t-1}(I - beta_t k_t kw_t^T) + beta_t v_t kw_t^T.
// With gamma_t = prod_{m<=t} alpha_m inside the chunk and Th the inverse above (no decay in it), the
// chunk is exactly
//   Ut = Th diag(beta / gamma) V - W S^T,   O = diag(gamma) (Q S^T + P Ut),   S <- gamma_C (S + Ut^T Kw)
// (T of the decayed Gram = diag(gamma) Th diag(1/gamma)), so only GU's B operand (T diag(beta / gamma)),
// the O epilogue (x gamma_t) and the state carry (x gamma_C) change. It needs the decay within any
// chunk to stay in the fp32 range (prod of 64 alphas above ~1e-30).
template <bool GATED>
__global__ void __launch_bounds__(288, 1)
chunk_wy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_kw, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_out, const __nv_bfloat16* __restrict__ beta,
                const __nv_bfloat16* __restrict__ alpha, const float* __restrict__ S0, float* __restrict__ S_final,
                int B, int T, int H, unsigned long long wait_limit_ns)
{
    constexpr int C = 64, DK = 128, DV = 128;
    // TMEM columns: state fp32 | bf16 state | D (U0^T -> Vn^T, bf16 Vn^T in its first 32 columns | O^T) | R1 x 3
    constexpr uint32_t COL_S = 0, COL_SB = 128, COL_D = 192, COL_R1 = 320, NCOLS = 512;
    constexpr uint32_t ID_N64 = tc::idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_N64_AMN = tc::idesc_bf16(128, 64, 1, 0);
    constexpr uint32_t ID_N128 = tc::idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t ID_N128_BMN = tc::idesc_bf16(128, 128, 0, 1);
    constexpr int BAR_STATE = 1, BAR_PREP = 2;   // named barrier ids (0 is __syncthreads)
    using L = WyLayout;

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

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(&g_osdn_status, kStatusTimeout);
    };
    // bounded wait that also stops when another role has aborted
    auto wait = [&](int bi, uint32_t parity) -> bool {
        uint64_t* bar = bars + bi;
        // the hardware suspend of one try is capped by the limit, so a short limit ends a wait promptly
        const uint32_t hint = wait_limit_ns < 20000ull ? (uint32_t)wait_limit_ns : 20000u;
        if (tc::mbar_try_wait(bar, parity, hint)) return true;
        const uint64_t t0 = tc::globaltimer_ns();
        while (true) {
            if (tc::mbar_try_wait(bar, parity, hint)) return true;
            if (*abort_flag) return false;
            if (tc::globaltimer_ns() - t0 > wait_limit_ns) {
                give_up();
                return false;
            }
        }
    };

    if (warp < 4) {
        // ================================================================ state group
        const int v = tid;                                   // TMEM lane: value row of S / key feature
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        constexpr int kTmaThread = 32, kPrefetchThread = 64;
        int issuedQ = 0, issuedV = 0;
        auto load_qk = [&](int c) {   // K, Q, Kw of chunk c into stage c % 3
            uint8_t* st = sm + (c % 3) * L::STAGE;
            uint64_t* fb = bars + L::FULLQ + c % 3;
            tc::mbar_arrive_expect_tx(fb, L::kTxQ);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tma_load_4d(st + L::QK + half * 16384, &tm_k, half * 64, h, c * C, b, fb);
                tc::tma_load_4d(st + L::QK + half * 16384 + 8192, &tm_q, half * 64, h, c * C, b, fb);
                tc::tma_load_4d(st + L::KW + half * 8192, &tm_kw, half * 64, h, c * C, b, fb);
            }
        };
        auto prefetch_l2 = [&](int c) {   // chunk c's tiles into L2, two ring slots ahead of their shared-memory load
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tma_prefetch_4d(&tm_k, half * 64, h, c * C, b);
                tc::tma_prefetch_4d(&tm_q, half * 64, h, c * C, b);
                tc::tma_prefetch_4d(&tm_kw, half * 64, h, c * C, b);
                tc::tma_prefetch_4d(&tm_v, half * 64, h, c * C, b);
            }
        };
        auto load_v = [&](int c) {    // V of chunk c into V tile c % 2
            uint8_t* vt = sm + L::VB + (c & 1) * 16384;
            uint64_t* fb = bars + L::FULLV + (c & 1);
            tc::mbar_arrive_expect_tx(fb, L::kTxV);
            tc::tma_load_4d(vt, &tm_v, 0, h, c * C, b, fb);
            tc::tma_load_4d(vt + 8192, &tm_v, 64, h, c * C, b, fb);
        };
        if (tid == kTmaThread) {
            while (issuedQ < 3 && issuedQ < nchunks) load_qk(issuedQ++);
            while (issuedV < 2 && issuedV < nchunks) load_v(issuedV++);
        }
        if (tid == kPrefetchThread) {
            if (nchunks > 3) prefetch_l2(3);
            if (nchunks > 4) prefetch_l2(4);
        }
        {   // initial state: fp32 S, its bf16 copy (A operand of GA), zeroed O^T columns
            const float* srow = S0 ? S0 + ((size_t)unit * DV + v) * DK : nullptr;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t x[64], w[32];
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    const float4 f = srow ? *reinterpret_cast<const float4*>(srow + half * 64 + i)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    x[i] = __float_as_uint(f.x); x[i + 1] = __float_as_uint(f.y);
                    x[i + 2] = __float_as_uint(f.z); x[i + 3] = __float_as_uint(f.w);
                }
                tc::tmem_st32(tl + COL_S + half * 64, *reinterpret_cast<uint32_t(*)[32]>(x));
                tc::tmem_st32(tl + COL_S + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = tc::pack_bf16(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                tc::tmem_st32(tl + COL_SB + half * 32, w);
            }
            uint32_t z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0u;
            tc::tmem_st32(tl + COL_D + 64, z);
            tc::tmem_st32(tl + COL_D + 96, z);
            tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        tc::named_sync(BAR_STATE, 128);
        if (tid == 0 && nchunks > 0) tc::mbar_arrive1(bars + L::ESB);

        // -W of chunk c (from W^T in R1[c % 3], lane = key feature) into the K rows of its stage
        auto w_epilogue = [&](int c) -> bool {
            if (tc::named_sync_or(BAR_STATE, 128, !wait(L::BW, c & 1))) return false;
            tc::tc_fence_after();
            ColsToRows w;
            w.load(tl + COL_R1 + (c % 3) * 64);
            tc::tmem_wait_ld();
            w.store(sm + (c % 3) * L::STAGE + L::QK, 16384, warp * 32, -1.f, lane);
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::named_sync(BAR_STATE, 128);
            if (tid == 0) tc::mbar_arrive1(bars + L::EWE);
            return true;
        };

        // gated: alpha of tokens 2 lane, 2 lane + 1 of a chunk (1 past T), one chunk ahead
        auto load_alpha = [&](int cc, float& a0, float& a1) {
            const int t = cc * C + 2 * lane;
            a0 = t < T ? __bfloat162float(alpha[((size_t)b * T + t) * H + h]) : 1.f;
            a1 = t + 1 < T ? __bfloat162float(alpha[((size_t)b * T + t + 1) * H + h]) : 1.f;
        };
        float an0 = 1.f, an1 = 1.f;
        if (GATED && nchunks > 0) load_alpha(0, an0, an1);

        bool ok = nchunks == 0 || w_epilogue(0);
        int c = 0;
        for (; ok && c < nchunks; ++c) {
            const int s2 = c & 1;
            // gated: gamma_t = prod_{m<=t} alpha_m of this chunk (every warp computes all 64), the O scales
            // for this thread's token columns, and gamma_C
            float osc[16], gamma_c = 1.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) osc[i] = 1.f;
            if (GATED) {
                const float a0 = an0, a1 = an1;
                if (c + 1 < nchunks) load_alpha(c + 1, an0, an1);
                const float incl = warp_prefix_product(a0 * a1, lane);     // gamma_{2 lane + 1}
                float excl = __shfl_up_sync(0xffffffffu, incl, 1);
                if (lane == 0) excl = 1.f;
                const float g0 = excl * a0;                                  // gamma_{2 lane}
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int src = 4 * j + (lane & 3);                      // owner of tokens 8j + 2(lane % 4), +1
                    osc[2 * j] = __shfl_sync(0xffffffffu, g0, src);
                    osc[2 * j + 1] = __shfl_sync(0xffffffffu, incl, src);
                }
                gamma_c = __shfl_sync(0xffffffffu, incl, 31);
            }
            // Vn^T = U0^T - S W^T (D columns 0-63) -> bf16 over columns 0-31 (A operand of GB)
            if (tc::named_sync_or(BAR_STATE, 128, !wait(L::BA, c & 1))) break;
            tc::tc_fence_after();
            {
                uint32_t x[64], w[32];
                tc::tmem_ld32(tl + COL_D, *reinterpret_cast<uint32_t(*)[32]>(x));
                tc::tmem_ld32(tl + COL_D + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = tc::pack_bf16(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                tc::tmem_st32(tl + COL_D, w);
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            tc::named_sync(BAR_STATE, 128);
            if (tid == 0) tc::mbar_arrive1(bars + L::EVN);

            // -W of the next chunk while GB runs
            if (c + 1 < nchunks && !w_epilogue(c + 1)) break;

            // S_{c+1} and O_c are complete; stage c % 3 is free
            if (tc::named_sync_or(BAR_STATE, 128, !wait(L::BS + s2, (c >> 1) & 1))) break;
            tc::tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t x[64];
                tc::tmem_ld32(tl + COL_S + half * 64, *reinterpret_cast<uint32_t(*)[32]>(x));
                tc::tmem_ld32(tl + COL_S + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
                tc::tmem_wait_ld();
                if (GATED) {   // S_{c+1} = gamma_C (S_c + Ut^T Kw): decay the fp32 state in place
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = __float_as_uint(gamma_c * __uint_as_float(x[i]));
                    if (c + 1 < nchunks) {
                        tc::tmem_st32(tl + COL_S + half * 64, *reinterpret_cast<uint32_t(*)[32]>(x));
                        tc::tmem_st32(tl + COL_S + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
                    }
                }
                if (c + 1 < nchunks) {
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        w[i] = tc::pack_bf16(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                    tc::tmem_st32(tl + COL_SB + half * 32, w);
                } else if (S_final) {
                    float* srow = S_final + ((size_t)unit * DV + v) * DK + half * 64;
#pragma unroll
                    for (int i = 0; i < 64; i += 4)
                        *reinterpret_cast<float4*>(srow + i) = make_float4(__uint_as_float(x[i]), __uint_as_float(x[i + 1]),
                                                                           __uint_as_float(x[i + 2]), __uint_as_float(x[i + 3]));
                }
            }
            ColsToRows o;   // O^T columns, read before they are zeroed for the next chunk
            o.load(tl + COL_D + 64);
            tc::tmem_wait_ld();
            if (c + 1 < nchunks) {
                uint32_t z[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = 0u;
                tc::tmem_st32(tl + COL_D + 64, z);
                tc::tmem_st32(tl + COL_D + 96, z);
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            tc::named_sync(BAR_STATE, 128);
            if (tid == 0 && c + 1 < nchunks) tc::mbar_arrive1(bars + L::ESB);
            // stage c % 3 is free (GB(c) has completed): chunk c + 3's tiles, and chunk c + 5's into L2;
            // issued after the hand-off so that their issue time stays off the state chain
            if (tid == kTmaThread && issuedQ < nchunks) load_qk(issuedQ++);
            if (tid == kPrefetchThread && c + 5 < nchunks) prefetch_l2(c + 5);

            // O_c -> the V tile of this chunk (free since GU(c) completed) -> TMA store
            uint8_t* ob = sm + L::VB + s2 * 16384;
            o.store(ob, 8192, warp * 32, osc, lane);   // gated: O = diag(gamma) (...); else all ones
            tc::fence_proxy_async_smem();
            tc::named_sync(BAR_STATE, 128);
            if (tid == kTmaThread) {
                tc::tma_store_4d(&tm_out, ob, 0, h, c * C, b);
                tc::tma_store_4d(&tm_out, ob + 8192, 64, h, c * C, b);
                tc::bulk_commit();
                if (issuedV < nchunks) {   // V of chunk c + 2 reuses the staging tile once the store has read it
                    tc::bulk_wait_read<0>();
                    load_v(issuedV++);
                }
            }
        }
        if (tid == kTmaThread) {   // stores complete; loads that were issued have landed
            tc::bulk_wait<0>();
            for (int cc = issuedQ > 3 ? issuedQ - 3 : 0; cc < issuedQ; ++cc)
                tc::mbar_wait(bars + L::FULLQ + cc % 3, (cc / 3) & 1, 1000000000ull);
            for (int cc = issuedV > 2 ? issuedV - 2 : 0; cc < issuedV; ++cc)
                tc::mbar_wait(bars + L::FULLV + (cc & 1), (cc >> 1) & 1, 1000000000ull);
        }
        tc::tc_fence_before();
    } else if (warp < 8) {
        // ================================================================ prep group
        const int q4 = warp & 3;
        const int gtid = tid - 128;                // 0..127; also the TMEM lane (R1 row) it reads
        const int gw = warp - 4;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        float* betas = reinterpret_cast<float*>(sm + L::BETA);
        float* AF = reinterpret_cast<float*>(sm + L::AF);
        auto load_beta = [&](int c) -> float {
            const int t = c * C + gtid;
            return (gtid < C && t < T) ? __bfloat162float(beta[((size_t)b * T + t) * H + h]) : 0.f;
        };
        float bnext = nchunks > 0 ? load_beta(0) : 0.f;
        auto load_alpha_p = [&](int c) -> float {
            const int t = c * C + gtid;
            return (GATED && gtid < C && t < T) ? __bfloat162float(alpha[((size_t)b * T + t) * H + h]) : 1.f;
        };
        float anext = nchunks > 0 ? load_alpha_p(0) : 1.f;
        float* betag = reinterpret_cast<float*>(sm + L::BETAG);
        float* gscr = reinterpret_cast<float*>(sm + L::GSCR);
        for (int c = 0; c < nchunks; ++c) {
            const int s2 = c & 1;
            const float bt = bnext;
            if (c + 1 < nchunks) bnext = load_beta(c + 1);
            float gam = 1.f;   // gated: gamma_t of token gtid (< 64), within its warp so far
            if (GATED) {
                const float at = anext;
                if (c + 1 < nchunks) anext = load_alpha_p(c + 1);
                if (gtid < C) {
                    gam = warp_prefix_product(at, lane);
                    if (gtid == 31) *gscr = gam;                  // gamma_31, for the second warp
                }
            }
            bool fail = !wait(L::D1 + c % 3, (c / 3) & 1);
            if (!fail && c >= 2) fail = !wait(L::BS + s2, ((c - 2) >> 1) & 1);   // GB(c-2) has read P tile s2
            if (tc::named_sync_or(BAR_PREP, 128, fail)) break;
            tc::tc_fence_after();
            if (gtid < C) betas[gtid] = bt;
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
                uint32_t r[32];
                tc::tmem_ld32(tl + COL_R1 + (c % 3) * 64 + qh * 32, r);
                tc::tmem_wait_ld();
                if (gtid < C) {   // A[t][j] = beta_t <k_t, kw_j> for j < t, zero elsewhere (full rows)
                    const int t = gtid;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const int j = qh * 32 + e;
                        *reinterpret_cast<float4*>(AF + t * L::LDF + j) =
                            make_float4((j < t) ? bt * __uint_as_float(r[e]) : 0.f,
                                        (j + 1 < t) ? bt * __uint_as_float(r[e + 1]) : 0.f,
                                        (j + 2 < t) ? bt * __uint_as_float(r[e + 2]) : 0.f,
                                        (j + 3 < t) ? bt * __uint_as_float(r[e + 3]) : 0.f);
                    }
                } else {          // P[t][j] = <q_t, kw_j> for j <= t
                    const int t = gtid - C;
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
                        *reinterpret_cast<uint4*>(sm + L::PB + s2 * 8192 + tc::sw128_off(t, qh * 4 + cc)) = pk;
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::named_sync(BAR_PREP, 128);
            if (GATED && gtid < C) {   // beta_t / gamma_t (read by the T diag(beta / gamma) write below)
                if (gtid >= 32) gam *= *gscr;
                betag[gtid] = bt / gam;
            }
            tri::tril_inv64_inplace(AF, gw, lane, [] { tc::named_sync(BAR_PREP, 128); });
            // T diag(beta) -> bf16 K-major (B operand of GW and GU), once GW(c-1) and GU(c-1) have read it
            fail = c >= 1 && !wait(L::BA, (c - 1) & 1);
            if (tc::named_sync_or(BAR_PREP, 128, fail)) break;
            {
                const int t = gtid & 63, hf = gtid >> 6;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int j = hf * 32 + cc * 8;
                    const float4 lo = *reinterpret_cast<const float4*>(AF + t * L::LDF + j);
                    const float4 hi = *reinterpret_cast<const float4*>(AF + t * L::LDF + j + 4);
                    const float4 blo = *reinterpret_cast<const float4*>(betas + j);
                    const float4 bhi = *reinterpret_cast<const float4*>(betas + j + 4);
                    uint4 pk;
                    pk.x = tc::pack_bf16(lo.x * blo.x, lo.y * blo.y); pk.y = tc::pack_bf16(lo.z * blo.z, lo.w * blo.w);
                    pk.z = tc::pack_bf16(hi.x * bhi.x, hi.y * bhi.y); pk.w = tc::pack_bf16(hi.z * bhi.z, hi.w * bhi.w);
                    *reinterpret_cast<uint4*>(sm + L::TB + tc::sw128_off(t, hf * 4 + cc)) = pk;
                    if (GATED) {   // T diag(beta / gamma), the B operand of GU
                        const float4 glo = *reinterpret_cast<const float4*>(betag + j);
                        const float4 ghi = *reinterpret_cast<const float4*>(betag + j + 4);
                        uint4 pg;
                        pg.x = tc::pack_bf16(lo.x * glo.x, lo.y * glo.y); pg.y = tc::pack_bf16(lo.z * glo.z, lo.w * glo.w);
                        pg.z = tc::pack_bf16(hi.x * ghi.x, hi.y * ghi.y); pg.w = tc::pack_bf16(hi.z * ghi.z, hi.w * ghi.w);
                        *reinterpret_cast<uint4*>(sm + L::TB2 + tc::sw128_off(t, hf * 4 + cc)) = pg;
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::named_sync(BAR_PREP, 128);
            if (gtid == 0) tc::mbar_arrive1(bars + L::ETB);
        }
        tc::tc_fence_before();
    } else {
        // ================================================================ issuer warp
        if (lane == 0) {
            const uint64_t dTB = tc::sdesc_sw128(sb + L::TB, 16, 1024);
            const uint64_t dTBU = tc::sdesc_sw128(sb + (GATED ? L::TB2 : L::TB), 16, 1024);   // B of GU
            auto st = [&](int c) { return sb + (uint32_t)(c % 3) * L::STAGE; };
            auto G1 = [&](int c) {   // R1[c%3] = [K; Q] Kw^T
                const uint64_t a = tc::sdesc_sw128(st(c) + L::QK, 16, 1024), bk = tc::sdesc_sw128(st(c) + L::KW, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                    tc::umma_bf16(tmem + COL_R1 + (c % 3) * 64, a + ((half * 16384 + koff) >> 4),
                                  bk + ((half * 8192 + koff) >> 4), ID_N64, ks > 0);
                }
                tc::umma_commit(bars + L::D1 + c % 3);
            };
            auto GW = [&](int c) {   // R1[c%3] = K^T (T diag(beta))^T; K^T read MN-major (feature halves 16 KB apart)
                const uint64_t a = tc::sdesc_sw128(st(c) + L::QK, 16384, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16(tmem + COL_R1 + (c % 3) * 64, a + ((ks * 2048) >> 4), dTB + ((ks * 32) >> 4), ID_N64_AMN,
                                  ks > 0);
                tc::umma_commit(bars + L::BW);
            };
            auto GU = [&](int c) {   // D[0,64) = V^T (T diag(beta))^T; V^T read MN-major (value halves 8 KB apart)
                const uint64_t a = tc::sdesc_sw128(sb + L::VB + (c & 1) * 16384, 8192, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16(tmem + COL_D, a + ((ks * 2048) >> 4), dTBU + ((ks * 32) >> 4), ID_N64_AMN, ks > 0);
            };
            auto GA = [&](int c) {   // D += S_bf16 [-W; Q]^T
                const uint64_t bq = tc::sdesc_sw128(st(c) + L::QK, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                    tc::umma_bf16_ts(tmem + COL_D, tmem + COL_SB + ks * 8, bq + ((half * 16384 + koff) >> 4), ID_N128, true);
                }
                tc::umma_commit(bars + L::BA);
            };
            auto GB = [&](int c) {   // S += Vn^T Kw (Kw MN-major);  O^T += Vn^T P^T
                const uint64_t bkw = tc::sdesc_sw128(st(c) + L::KW, 8192, 1024);
                const uint64_t bp = tc::sdesc_sw128(sb + L::PB + (c & 1) * 8192, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16_ts(tmem + COL_S, tmem + COL_D + ks * 8, bkw + ((ks * 2048) >> 4), ID_N128_BMN, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16_ts(tmem + COL_D + 64, tmem + COL_D + ks * 8, bp + ((ks * 32) >> 4), ID_N64, true);
                tc::umma_commit(bars + L::BS + (c & 1));
            };
            // Static order per chunk c (each wait sleeps in hardware until its phase completes):
            //   GA(c) | GW(c+1), G1(c+2) if their inputs are ready | GB(c) | the rest of GW(c+1), G1(c+2) | GU(c+1)
            // GW and G1 fill the tensor pipe while the state group forms bf16 Vn after GA. G1(c+2) reuses
            // R1[(c+2)%3], whose W^T(c-1) was consumed before GA(c-1); GU(c+1) overwrites D[0,64) once GB(c)
            // has read bf16 Vn from it.
            auto issue_gu = [&](int c) -> bool {
                if (c > 0 && !wait(L::BS + ((c - 1) & 1), ((c - 1) >> 1) & 1)) return false;
                if (!wait(L::FULLV + (c & 1), (c >> 1) & 1)) return false;
                tc::tc_fence_after();
                GU(c);
                return true;
            };
            auto issue_g1 = [&](int c) -> bool {
                if (!wait(L::FULLQ + c % 3, (c / 3) & 1)) return false;
                G1(c);
                return true;
            };
            auto issue_gw = [&](int c) -> bool {
                if (!wait(L::ETB, c & 1)) return false;
                tc::tc_fence_after();
                GW(c);
                return true;
            };
            bool ok = nchunks == 0 ||
                      (issue_g1(0) && (nchunks < 2 || issue_g1(1)) && issue_gw(0) && issue_gu(0));
            for (int c = 0; ok && c < nchunks; ++c) {
                ok = wait(L::ESB, c & 1) && wait(L::EWE, c & 1);
                if (!ok) break;
                tc::tc_fence_after();
                GA(c);
                bool gw_done = c + 1 >= nchunks, g1_done = c + 2 >= nchunks;
                if (!gw_done && tc::mbar_test(bars + L::ETB, (c + 1) & 1)) {
                    tc::tc_fence_after();
                    GW(c + 1);
                    gw_done = true;
                }
                if (!g1_done && tc::mbar_test(bars + L::FULLQ + (c + 2) % 3, ((c + 2) / 3) & 1)) {
                    G1(c + 2);
                    g1_done = true;
                }
                if (!(ok = wait(L::EVN, c & 1))) break;
                tc::tc_fence_after();
                GB(c);
                if (!gw_done && !(ok = issue_gw(c + 1))) break;
                if (!g1_done && !(ok = issue_g1(c + 2))) break;
                if (c + 1 < nchunks && !(ok = issue_gu(c + 1))) break;
            }
            tc::umma_commit(bars + L::DRAIN);   // every MMA issued above has completed before TMEM is released
            tc::mbar_wait(bars + L::DRAIN, 0, 1000000000ull);
        }
        __syncwarp();
        tc::tc_fence_before();
    }

    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, NCOLS);
    }
}

}  // namespace osdn
