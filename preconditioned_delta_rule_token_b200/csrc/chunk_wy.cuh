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
//   G1   R1[c%3]  = [K; Q] Kw^T        Gram rows (lanes 0-63), score rows (64-127)
//   GW   R1[c%3]  = K^T (T diag(beta))^T = W^T            lane = key feature
//   GU   D[0,64)  = V^T (T diag(beta))^T = U0^T           lane = value row
//   GA   D       += S_bf16 [-W; Q]^T   D[0,64) = Vn^T, D[64,128) = (Q S^T)^T
//   GBS  S       += Vn^T Kw
//   GBO  D[64,128) += Vn^T P^T  ->  O^T                    (P = tril(Q Kw^T))
//
// One CTA (416 threads) per (sequence, head), four roles:
//   state group (warps 0-3, lane v): the chain only. Vn^T -> bf16 in TMEM (A
//     operand of GBS/GBO), -W rows of the next chunk over its K rows (from W^T,
//     between GA and GBS, while the tensor pipe runs GBS), S -> bf16 in TMEM
//     (A operand of the next GA).
//   prep group (warps 4-7): for the chunk two ahead, A (fp32) and P (bf16)
//     from G1, then T = (I + A)^{-1} by blocks, written straight out as bf16
//     T diag(beta) (the B operand of GW and GU; two such tiles by chunk parity).
//   epilogue group (warps 8-11): reads O^T out of TMEM as soon as GBO completes
//     and zeroes its columns for the next GA, stages O in the chunk's V tile
//     and stores it by TMA; issues every TMA load and L2 prefetch.
//   issuer warp (warp 12, one lane): every MMA. The tensor pipe runs MMAs in
//     issue order and an issuing thread stalls while the pipe is full, so the
//     order per chunk keeps the chain first and fills the chain's epilogue
//     windows with work that fits them:
//       GA(c) | GW(c+1), G1(c+2) | (bf16 Vn) GBS(c), GBO(c) | GU(c+1)
// Shared memory: a three-stage ring of [K; Q] + Kw tiles (a stage is reloaded
// once its chunk's GBO has completed), two V tiles (the older one doubles as
// the O staging tile), T diag(beta), two P tiles, the fp32 Gram / inverse.
// Hand-offs are mbarriers (TMA transaction counts, tcgen05.commit, one elected
// arrival). Every wait is bounded: a wait that gives up sets the library status
// word and a shared abort flag; the groups leave at their next group-wide wait
// (a barrier-OR), issued MMAs and loads are drained before TMEM is released.
//
// GATED: the gated delta rule backbone, S_t = alpha_t S_{t-1}(I - beta_t k_t kw_t^T) + beta_t v_t kw_t^T.
// With gamma_t = prod_{m<=t} alpha_m inside the chunk (gamma_0 = 1 before it), every decay factor
// the chunk needs is a ratio gamma_t / gamma_j with t >= j, at most 1:
//   A_g[t][j] = beta_t (gamma_t / gamma_j) <k_t, kw_j> (j < t),  T = (I + A_g)^{-1},
//   W = T diag(beta gamma) K,  U0 = T diag(beta) V,  U = U0 - W S^T,
//   O = diag(gamma) Q S^T + P_g U,  P_g[t][j] = (gamma_t / gamma_j) <q_t, kw_j> (j <= t),
//   S <- gamma_C S + sum_j (gamma_C / gamma_j) u_j kw_j^T.
// The ratios are exp2 of differences of the in-chunk cumulative log2(alpha) (each log2 clamped at
// -120, so alpha = 0 restarts the state to within 2^-120), which keeps every gate value in [0, 1]
// in range. The kernel applies them in the prep (A_g and P_g), in the epilogue group (the chunk's K
// and Q rows x gamma_t, so that GW forms W^T = (diag(gamma) K)^T (T diag(beta))^T from the same T
// tile as GU and GA forms diag(gamma) Q S^T, and its Kw rows x gamma_C / gamma_t, so that GBS adds
// U^T diag(gamma_C / gamma) Kw; done two chunks ahead, once G1 has read the three tiles), and in the
// state group (the fp32 state x gamma_C of the next chunk when it is converted to bf16).
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct WyLayout {
    static constexpr uint32_t STAGE = 49152, NSTAGE = 3;   // [K0|Q0|K1|Q1] (8 KB each) + [Kw0|Kw1]
    static constexpr uint32_t QK = 0, KW = 32768;
    static constexpr uint32_t VB = NSTAGE * STAGE;          // two V tiles [V0|V1], 16 KB each
    static constexpr uint32_t TB = VB + 2 * 16384;          // two T diag(beta) tiles bf16 (B of GU, GW), by parity
    static constexpr uint32_t PB = TB + 2 * 8192;           // two P tiles bf16 [64 t][64 j]
    static constexpr int LDF = tri::LD;
    static constexpr uint32_t AF = PB + 2 * 8192;           // A, then T, fp32 [64][LDF]
    static constexpr uint32_t BETA = AF + 64 * LDF * 4;     // prep: beta of its chunk
    static constexpr uint32_t GLOG = BETA + 256;            // prep, gated: log2 gamma_t of its chunk
    static constexpr uint32_t BAR = GLOG + 256;
    enum {
        FULLQ = 0,   // 3: K, Q, Kw of a stage landed
        FULLV = 3,   // 2: V tile landed
        D1 = 5,      // 3: G1 into R1[i] done
        BW = 8,      // GW done
        BA = 9,      // GA done
        BS = 10,     // GBS done
        BO = 11,     // 2: GBO done (by chunk parity)
        ETB = 13,    // prep: T diag(beta) and P of its chunk written
        EWE = 14,    // state: -W (and gated: gamma Q) of its chunk written
        ESB = 15,    // state: bf16 S written
        EVN = 16,    // state: bf16 Vn written
        EOR = 17,    // epilogue: O^T columns read and zeroed
        BAP = 18,    // 2: GA done (by chunk parity; the prep reuses T diag(beta) tile c % 2)
        ESC = 20,    // 2, gated, epilogue: K, Q and Kw of a chunk scaled by its gates (by chunk parity: the
                     // epilogue may finish chunk c + 2 before the issuer has consumed chunk c + 1)
        DRAIN = 22,
        NBAR = 23
    };
    static constexpr uint32_t TSLOT = BAR + NBAR * 8;       // TMEM base address
    static constexpr uint32_t ABORT = TSLOT + 4;
    static constexpr uint32_t END = ABORT + 4;
    static constexpr size_t kBytes = END + 1024;
    static constexpr uint32_t kTxQ = 6 * 8192;              // K, Q, Kw halves
    static constexpr uint32_t kTxV = 2 * 8192;
    static constexpr int kThreads = 416;
    static_assert(kBytes <= 232448, "dynamic shared memory above the 227 KB per-block limit");
};

// Transposing epilogue, one warp: TMEM lanes m0..m0+31 (matrix row index m)
// x 32 columns (tokens t0..t0+31), fp32, become bf16 rows t of a
// 128-byte-swizzled K-major tile: element (t, m) at tile + (m / 64) *
// half_stride, row t, 16-byte chunk (m % 64) / 8. The load uses the 16x256b
// shape (two adjacent columns per thread); the store writes 8 x 8 tiles
// transposed with stmatrix, 16 bytes per row per tile.
struct ColsToRows {
    uint32_t lo[16], hi[16];
    __device__ __forceinline__ void load(uint32_t taddr) {   // wait with tcgen05.wait::ld before store()
        tc::tmem_ld16x256b_x4(taddr, lo);                   // lanes m0 + 0..15
        tc::tmem_ld16x256b_x4(taddr + (16u << 16), hi);     // lanes m0 + 16..31
    }
    __device__ __forceinline__ void store(uint8_t* tile, uint32_t half_stride, int m0, int t0, float s,
                                          int lane) const {
        const int k = lane >> 3, c = lane & 7;              // this thread addresses row c of 8 x 8 tile k
        const int mk = m0 + 8 * k;                          // first matrix row index of tile k
        uint8_t* base = tile + (mk >> 6) * half_stride;
        const int ch = (mk & 63) >> 3;
#pragma unroll
        for (int j = 0; j < 4; ++j) {                       // tokens t0 + 8j .. t0 + 8j + 7
            const uint32_t p0 = tc::pack_bf16(s * __uint_as_float(lo[4 * j]), s * __uint_as_float(lo[4 * j + 1]));
            const uint32_t p1 = tc::pack_bf16(s * __uint_as_float(lo[4 * j + 2]), s * __uint_as_float(lo[4 * j + 3]));
            const uint32_t p2 = tc::pack_bf16(s * __uint_as_float(hi[4 * j]), s * __uint_as_float(hi[4 * j + 1]));
            const uint32_t p3 = tc::pack_bf16(s * __uint_as_float(hi[4 * j + 2]), s * __uint_as_float(hi[4 * j + 3]));
            tc::stmatrix_x4_trans(tc::smem_u32(base + tc::sw128_off(t0 + 8 * j + c, ch)), p0, p1, p2, p3);
        }
    }
    // both halves of a 64-column block (tokens 0..63), one after the other
    __device__ __forceinline__ void copy64(uint32_t taddr, uint8_t* tile, uint32_t half_stride, int m0, float s,
                                           int lane) {
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
            load(taddr + 32 * part);
            tc::tmem_wait_ld();
            store(tile, half_stride, m0, 32 * part, s, lane);
        }
    }
};

// 2^x and log2(x) by the special-function unit (about 2 ulp; 2^x flushes results below the
// normal range to 0, log2(0) = -inf).
__device__ __forceinline__ float sfu_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sfu_log2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A scale factor as the sum of two bf16 values, hi = bf16(s) and lo = bf16(s - hi), so that
// x * s is x * lo + x * hi with one fused rounding at the end.
struct Bf16Scale {
    __nv_bfloat162 hi, lo;
    __device__ __forceinline__ explicit Bf16Scale(float s) {
        const __nv_bfloat16 h = __float2bfloat16_rn(s);
        hi = __bfloat162bfloat162(h);
        lo = __bfloat162bfloat162(__float2bfloat16_rn(s - __bfloat162float(h)));
    }
};

// Eight bf16 values at p (16-byte aligned shared memory) multiplied by s in place, in packed
// bf16x2 arithmetic.
__device__ __forceinline__ void scale_bf16x8(uint8_t* p, const Bf16Scale& s) {
    uint4 u = *reinterpret_cast<uint4*>(p);
    __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) e[q] = __hfma2(e[q], s.hi, __hmul2(e[q], s.lo));
    *reinterpret_cast<uint4*>(p) = u;
}

// Gate values of one chunk: log2 gamma_t (inclusive prefix sum of log2 alpha within the chunk,
// each term clamped at -120; tokens past T have alpha = 1) for tokens 2 lane and 2 lane + 1,
// computed by every lane of a warp.
struct ChunkGates {
    float g0, g1;   // log2 gamma of tokens 2 lane, 2 lane + 1
    // log2 alpha of one token from its raw value (RawAlpha); tokens past T count as alpha = 1
    __device__ __forceinline__ static float log2_of(__nv_bfloat16 a, bool valid) {
        return valid ? fmaxf(sfu_log2(__bfloat162float(a)), -120.f) : 0.f;
    }
    // la0, la1: log2 alpha of the lane's two tokens (from log2_of)
    __device__ __forceinline__ void scan(float la0, float la1, int lane) {
        float x = la0 + la1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        g1 = x;
        g0 = x - la1;
    }
    // log2 gamma of token t (0..63) of the chunk, from any lane
    __device__ __forceinline__ float at(int t) const {
        const float a = __shfl_sync(0xffffffffu, g0, t >> 1), b = __shfl_sync(0xffffffffu, g1, t >> 1);
        return (t & 1) ? b : a;
    }
    __device__ __forceinline__ float last() const { return __shfl_sync(0xffffffffu, g1, 31); }
};

// alpha of a lane's two tokens of one chunk as loaded (bf16 bits): loaded a chunk or more ahead and
// first used by ChunkGates::log2_of, so that the load's latency is not waited for where it is issued.
struct RawAlpha {
    __nv_bfloat16 a0, a1;
};

template <bool GATED>
__global__ void __launch_bounds__(WyLayout::kThreads, 1)
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
    constexpr int BAR_STATE = 1, BAR_PREP = 2, BAR_EPI = 3;   // named barrier ids (0 is __syncthreads)
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
    auto alpha_idx = [&](int t) { return ((size_t)b * T + t) * H + h; };
    auto load_raw = [&](int cc) -> RawAlpha {   // gated: alpha of tokens 2 lane, 2 lane + 1 of chunk cc
        const int t = cc * C + 2 * lane;
        const __nv_bfloat16 one = __float2bfloat16(1.f);
        return RawAlpha{t < T ? alpha[alpha_idx(t)] : one, t + 1 < T ? alpha[alpha_idx(t + 1)] : one};
    };
    auto gates_from = [&](const RawAlpha& ra, int cc, ChunkGates& g) {   // gated: the gates of chunk cc
        const int t = cc * C + 2 * lane;
        g.scan(ChunkGates::log2_of(ra.a0, t < T), ChunkGates::log2_of(ra.a1, t + 1 < T), lane);
    };

    if (warp < 4) {
        // ================================================================ state group
        const int v = tid;                                   // TMEM lane: value row of S / key feature
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        // gated: gates of the current chunk (cur) and of the next one (nxt), every warp all 64 tokens;
        // alpha of the chunk after nxt is loaded an iteration ahead (pa)
        ChunkGates cur{0.f, 0.f}, nxt{0.f, 0.f};
        RawAlpha pa{};
        auto gates_of = [&](int cc, ChunkGates& g) { gates_from(load_raw(cc), cc, g); };
        if (GATED && nchunks > 0) gates_of(0, nxt);
        {   // initial state: fp32 S (gated: x gamma_C of chunk 0), its bf16 copy (A operand of GA), zeroed O^T
            const float* srow = S0 ? S0 + ((size_t)unit * DV + v) * DK : nullptr;
            const float g = GATED ? sfu_exp2(nxt.last()) : 1.f;
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) {
                uint32_t x[32], w[16];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 f = srow ? *reinterpret_cast<const float4*>(srow + qt * 32 + i)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    x[i] = __float_as_uint(f.x); x[i + 1] = __float_as_uint(f.y);
                    x[i + 2] = __float_as_uint(f.z); x[i + 3] = __float_as_uint(f.w);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = tc::pack_bf16(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                tc::tmem_st16(tl + COL_SB + qt * 16, w);
                if (GATED) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = __float_as_uint(g * __uint_as_float(x[i]));
                }
                tc::tmem_st32(tl + COL_S + qt * 32, x);
            }
            tc::tmem_zero32(tl + COL_D + 64);
            tc::tmem_zero32(tl + COL_D + 96);
            tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        tc::named_sync(BAR_STATE, 128);
        if (tid == 0 && nchunks > 0) tc::mbar_arrive1(bars + L::ESB);

        // -W of chunk c (from W^T in R1[c % 3], lane = key feature) into the K rows of its stage
        auto w_epilogue = [&](int c) -> bool {
            if (tc::named_sync_or(BAR_STATE, 128, !wait(L::BW, c & 1))) return false;
            tc::tc_fence_after();
            uint8_t* st = sm + (c % 3) * L::STAGE + L::QK;
            ColsToRows w;
            w.copy64(tl + COL_R1 + (c % 3) * 64, st, 16384, warp * 32, -1.f, lane);
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::named_sync(BAR_STATE, 128);
            if (tid == 0) tc::mbar_arrive1(bars + L::EWE);
            return true;
        };

        bool ok = true;
        if (nchunks > 0) {
            cur = nxt;
            if (GATED) {
                if (nchunks > 1) gates_of(1, nxt);
                if (nchunks > 2) pa = load_raw(2);
            }
            ok = w_epilogue(0);
        }
        int c = 0;
        for (; ok && c < nchunks; ++c) {
            // Vn^T = U0^T - S W^T (D columns 0-63) -> bf16 over columns 0-31 (A operand of GBS and GBO)
            if (tc::named_sync_or(BAR_STATE, 128, !wait(L::BA, c & 1))) break;
            tc::tc_fence_after();
#pragma unroll 1
            for (int hv = 0; hv < 2; ++hv) {   // in place, 32 columns at a time (the bf16 half lands on consumed columns)
                uint32_t x[32], w[16];
                tc::tmem_ld32(tl + COL_D + 32 * hv, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = tc::pack_bf16(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                tc::tmem_st16(tl + COL_D + 16 * hv, w);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::named_sync(BAR_STATE, 128);
            if (tid == 0) tc::mbar_arrive1(bars + L::EVN);

            // -W of the next chunk while GBS runs
            if (c + 1 < nchunks && !w_epilogue(c + 1)) break;

            // S_{c+1} is complete: its bf16 copy for GA(c + 1) (gated: the fp32 state x gamma_C of chunk c + 1)
            if (tc::named_sync_or(BAR_STATE, 128, !wait(L::BS, c & 1))) break;
            tc::tc_fence_after();
            const float gnext = (GATED && c + 1 < nchunks) ? sfu_exp2(nxt.last()) : 1.f;
#pragma unroll 1
            for (int qt = 0; qt < 4; ++qt) {
                uint32_t x[32];
                tc::tmem_ld32(tl + COL_S + qt * 32, x);
                tc::tmem_wait_ld();
                if (c + 1 < nchunks) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = tc::pack_bf16(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                    tc::tmem_st16(tl + COL_SB + qt * 16, w);
                    if (GATED) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) x[i] = __float_as_uint(gnext * __uint_as_float(x[i]));
                        tc::tmem_st32(tl + COL_S + qt * 32, x);
                    }
                } else if (S_final) {
                    float* srow = S_final + ((size_t)unit * DV + v) * DK + qt * 32;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(srow + i) = make_float4(__uint_as_float(x[i]), __uint_as_float(x[i + 1]),
                                                                           __uint_as_float(x[i + 2]), __uint_as_float(x[i + 3]));
                }
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::named_sync(BAR_STATE, 128);
            if (tid == 0 && c + 1 < nchunks) tc::mbar_arrive1(bars + L::ESB);
            if (GATED) {
                cur = nxt;
                if (c + 2 < nchunks) gates_from(pa, c + 2, nxt);
                if (c + 3 < nchunks) pa = load_raw(c + 3);
            }
        }
        tc::tc_fence_before();
    } else if (warp < 8) {
        // ================================================================ prep group
        const int q4 = warp & 3;
        const int gtid = tid - 128;                // 0..127; also the TMEM lane (R1 row) it reads
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        float* betas = reinterpret_cast<float*>(sm + L::BETA);
        float* glog = reinterpret_cast<float*>(sm + L::GLOG);
        float* AF = reinterpret_cast<float*>(sm + L::AF);
        // beta of the next chunk, loaded a chunk ahead as bf16 and converted where it is used
        auto load_beta = [&](int c) -> __nv_bfloat16 {
            const int t = c * C + gtid;
            return (gtid < C && t < T) ? beta[((size_t)b * T + t) * H + h] : __float2bfloat16(0.f);
        };
        __nv_bfloat16 bnext = nchunks > 0 ? load_beta(0) : __float2bfloat16(0.f);
        // gated: alpha of the next chunk, loaded a chunk ahead (every prep warp)
        RawAlpha la{};
        if (GATED && nchunks > 0) la = load_raw(0);
        for (int i = gtid; i < 2 * 8192 / 16; i += 128)   // the T tiles' blocks above the diagonal stay zero
            reinterpret_cast<uint4*>(sm + L::TB)[i] = make_uint4(0u, 0u, 0u, 0u);
        for (int c = 0; c < nchunks; ++c) {
            const int s2 = c & 1;
            const __nv_bfloat16 braw = bnext;
            if (c + 1 < nchunks) bnext = load_beta(c + 1);
            ChunkGates g{0.f, 0.f};
            if (GATED) {
                gates_from(la, c, g);
                if (c + 1 < nchunks) la = load_raw(c + 1);
            }
            bool fail = !wait(L::D1 + c % 3, (c / 3) & 1);
            if (!fail && c >= 2) fail = !wait(L::BO + s2, ((c - 2) >> 1) & 1);   // GBO(c-2) has read P tile s2
            if (tc::named_sync_or(BAR_PREP, 128, fail)) break;
            tc::tc_fence_after();
            const float bt = __bfloat162float(braw);
            if (gtid < C) betas[gtid] = bt;
            if (GATED && q4 == 0) {
                glog[2 * lane] = g.g0;
                glog[2 * lane + 1] = g.g1;
            }
            if (GATED) tc::named_sync(BAR_PREP, 128);
            const float gt = GATED ? glog[gtid & 63] : 0.f;
            // 8 columns per TMEM load in a rolled loop (small code: the four roles share an instruction cache)
#pragma unroll 1
            for (int jb = 0; jb < 64; jb += 8) {
                uint32_t r8[8];
                tc::tmem_ld8(tl + COL_R1 + (c % 3) * 64 + jb, r8);
                tc::tmem_wait_ld();
                float sj[8], x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) sj[u] = GATED ? sfu_exp2(gt - glog[jb + u]) : 1.f;
                if (gtid < C) {   // A[t][j] = beta_t <k_t, kw_j> for j < t, zero elsewhere; gated x gamma_t / gamma_j
                    const int t = gtid;
#pragma unroll
                    for (int u = 0; u < 8; ++u) x[u] = (jb + u < t) ? bt * sj[u] * __uint_as_float(r8[u]) : 0.f;
                    *reinterpret_cast<float4*>(AF + t * L::LDF + jb) = make_float4(x[0], x[1], x[2], x[3]);
                    *reinterpret_cast<float4*>(AF + t * L::LDF + jb + 4) = make_float4(x[4], x[5], x[6], x[7]);
                } else {          // P[t][j] = <q_t, kw_j> for j <= t; gated x gamma_t / gamma_j
                    const int t = gtid - C;
#pragma unroll
                    for (int u = 0; u < 8; ++u) x[u] = (jb + u <= t) ? sj[u] * __uint_as_float(r8[u]) : 0.f;
                    uint4 pk;
                    pk.x = tc::pack_bf16(x[0], x[1]); pk.y = tc::pack_bf16(x[2], x[3]);
                    pk.z = tc::pack_bf16(x[4], x[5]); pk.w = tc::pack_bf16(x[6], x[7]);
                    *reinterpret_cast<uint4*>(sm + L::PB + s2 * 8192 + tc::sw128_off(t, jb >> 3)) = pk;
                }
            }
            tc::tc_fence_before();
            tc::named_sync(BAR_PREP, 128);
            // T = (I + A)^{-1}, written as bf16 T diag(beta) straight into tile c % 2, the B operand of GU and
            // GW, once GW and GU of chunk c - 2, the tile's last readers, have read it (GA(c - 2) completes
            // after both).
            auto tiles_free = [&]() -> bool {
                const bool f = c >= 2 && !wait(L::BAP + s2, ((c - 2) >> 1) & 1);
                return tc::named_sync_or(BAR_PREP, 128, f);
            };
            uint8_t* tb = sm + L::TB + (uint32_t)s2 * 8192u;
            if (!tri::tril_inv64_to_bf16(AF, tb, betas, q4, lane,
                                         [] { tc::named_sync(BAR_PREP, 128); }, tiles_free))
                break;
            tc::fence_proxy_async_smem();   // P and the T tiles -> the tensor core (async proxy)
            tc::named_sync(BAR_PREP, 128);
            if (gtid == 0) tc::mbar_arrive1(bars + L::ETB);
        }
        tc::tc_fence_before();
    } else if (warp < 12) {
        // ================================================================ epilogue group
        const int q4 = warp & 3, et = tid - 256;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        constexpr int kTmaThread = 0, kPrefetchThread = 32;
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
        if (et == kTmaThread) {
            while (issuedQ < 3 && issuedQ < nchunks) load_qk(issuedQ++);
            while (issuedV < 2 && issuedV < nchunks) load_v(issuedV++);
        }
        if (et == kPrefetchThread) {
            if (nchunks > 3) prefetch_l2(3);
            if (nchunks > 4) prefetch_l2(4);
        }
        // gated: chunk c's K and Q rows x gamma_t (GW then forms (diag(gamma) K)^T (T diag(beta))^T, GA
        // diag(gamma) Q S^T) and Kw rows x gamma_C / gamma_t (GBS then adds U^T diag(gamma_C / gamma) Kw), once
        // G1(c), their other reader, has completed; the issuer waits for it before GW(c)
        RawAlpha ea{};   // gated: alpha of the next chunk to scale, loaded a call ahead
        if (GATED && nchunks > 0) ea = load_raw(0);
        auto gate_scale = [&](int c) -> bool {
            const RawAlpha ra = ea;
            if (c + 1 < nchunks) ea = load_raw(c + 1);
            if (tc::named_sync_or(BAR_EPI, 128, !wait(L::D1 + c % 3, (c / 3) & 1))) return false;
            ChunkGates g;
            gates_from(ra, c, g);
            uint8_t* st = sm + (c % 3) * L::STAGE + L::QK;
            {   // thread (et % 8) takes 16-byte chunk et % 8 of rows t = et / 8 + 16 i of each tile
                const int ch = et & 7;
                const float gl = g.last();
                uint8_t* kw = sm + (c % 3) * L::STAGE + L::KW;
#pragma unroll 1
                for (int i = 0; i < 4; ++i) {
                    const int t = (et >> 3) + 16 * i;
                    const float gt = g.at(t);
                    const Bf16Scale sq(sfu_exp2(gt)), sk(sfu_exp2(gl - gt));
                    const uint32_t row = (t >> 3) * 1024 + (t & 7) * 128 + ch * 16;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        scale_bf16x8(st + half * 16384 + row, sq);          // K
                        scale_bf16x8(st + half * 16384 + 8192 + row, sq);   // Q
                        scale_bf16x8(kw + half * 8192 + row, sk);           // Kw
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::named_sync(BAR_EPI, 128);
            if (et == 0) tc::mbar_arrive1(bars + L::ESC + (c & 1));
            return true;
        };
        bool ok = true;
        if (GATED)
            for (int c = 0; ok && c < 2 && c < nchunks; ++c) ok = gate_scale(c);
        for (int c = 0; ok && c < nchunks; ++c) {
            // O_c = (Q S^T + P Vn)^T complete: read it out and zero the columns for GA(c + 1)
            if (tc::named_sync_or(BAR_EPI, 128, !wait(L::BO + (c & 1), (c >> 1) & 1))) { ok = false; break; }
            tc::tc_fence_after();
            ColsToRows o0, o1;
            o0.load(tl + COL_D + 64);
            o1.load(tl + COL_D + 96);
            tc::tmem_wait_ld();
            if (c + 1 < nchunks) {
                tc::tmem_zero32(tl + COL_D + 64);
                tc::tmem_zero32(tl + COL_D + 96);
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            tc::named_sync(BAR_EPI, 128);
            if (et == 0 && c + 1 < nchunks) tc::mbar_arrive1(bars + L::EOR);
            // stage c % 3 is free (GBO(c), the last reader, has completed): chunk c + 3's tiles, and
            // chunk c + 5's into L2
            if (et == kTmaThread && issuedQ < nchunks) load_qk(issuedQ++);
            if (et == kPrefetchThread && c + 5 < nchunks) prefetch_l2(c + 5);
            // O_c -> the V tile of this chunk (free since GU(c) completed) -> TMA store
            uint8_t* ob = sm + L::VB + (c & 1) * 16384;
            o0.store(ob, 8192, q4 * 32, 0, 1.f, lane);
            o1.store(ob, 8192, q4 * 32, 32, 1.f, lane);
            tc::fence_proxy_async_smem();
            tc::named_sync(BAR_EPI, 128);
            if (et == kTmaThread) {
                tc::tma_store_4d(&tm_out, ob, 0, h, c * C, b);
                tc::tma_store_4d(&tm_out, ob + 8192, 64, h, c * C, b);
                tc::bulk_commit();
                if (issuedV < nchunks) {   // V of chunk c + 2 reuses the staging tile once the store has read it
                    tc::bulk_wait_read<0>();
                    load_v(issuedV++);
                }
            }
            if (GATED && c + 2 < nchunks && !(ok = gate_scale(c + 2))) break;
        }
        if (et == kTmaThread) {   // stores complete; loads that were issued have landed
            tc::bulk_wait<0>();
            for (int cc = issuedQ > 3 ? issuedQ - 3 : 0; cc < issuedQ; ++cc)
                tc::mbar_wait(bars + L::FULLQ + cc % 3, (cc / 3) & 1, 1000000000ull);
            for (int cc = issuedV > 2 ? issuedV - 2 : 0; cc < issuedV; ++cc)
                tc::mbar_wait(bars + L::FULLV + (cc & 1), (cc >> 1) & 1, 1000000000ull);
        }
        tc::tc_fence_before();
    } else {
        // ================================================================ issuer warp
        if (lane == 0) {
            // T diag(beta) of chunk c, the B operand of GU and GW
            auto dTB = [&](int c) { return tc::sdesc_sw128(sb + L::TB + (uint32_t)(c & 1) * 8192u, 16, 1024); };
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
                    tc::umma_bf16(tmem + COL_R1 + (c % 3) * 64, a + ((ks * 2048) >> 4), dTB(c) + ((ks * 32) >> 4),
                                  ID_N64_AMN, ks > 0);
                tc::umma_commit(bars + L::BW);
            };
            auto GU = [&](int c) {   // D[0,64) = V^T (T diag(beta))^T; V^T read MN-major (value halves 8 KB apart)
                const uint64_t a = tc::sdesc_sw128(sb + L::VB + (c & 1) * 16384, 8192, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16(tmem + COL_D, a + ((ks * 2048) >> 4), dTB(c) + ((ks * 32) >> 4), ID_N64_AMN, ks > 0);
            };
            auto GA = [&](int c) {   // D += S_bf16 [-W; Q]^T
                const uint64_t bq = tc::sdesc_sw128(st(c) + L::QK, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                    tc::umma_bf16_ts(tmem + COL_D, tmem + COL_SB + ks * 8, bq + ((half * 16384 + koff) >> 4), ID_N128, true);
                }
                tc::umma_commit(bars + L::BA);
                tc::umma_commit(bars + L::BAP + (c & 1));
            };
            auto GBS = [&](int c) {   // S += Vn^T Kw (Kw MN-major)
                const uint64_t bkw = tc::sdesc_sw128(st(c) + L::KW, 8192, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16_ts(tmem + COL_S, tmem + COL_D + ks * 8, bkw + ((ks * 2048) >> 4), ID_N128_BMN, true);
                tc::umma_commit(bars + L::BS);
            };
            auto GBO = [&](int c) {   // O^T += Vn^T P^T
                const uint64_t bp = tc::sdesc_sw128(sb + L::PB + (c & 1) * 8192, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::umma_bf16_ts(tmem + COL_D + 64, tmem + COL_D + ks * 8, bp + ((ks * 32) >> 4), ID_N64, true);
                tc::umma_commit(bars + L::BO + (c & 1));
            };
            auto issue_g1 = [&](int c) -> bool {
                if (!wait(L::FULLQ + c % 3, (c / 3) & 1)) return false;
                G1(c);
                return true;
            };
            auto issue_gw = [&](int c) -> bool {
                if (!wait(L::ETB, c & 1)) return false;
                if (GATED && !wait(L::ESC + (c & 1), (c >> 1) & 1)) return false;
                tc::tc_fence_after();
                GW(c);
                return true;
            };
            // GU(c) overwrites D[0,64), which holds bf16 Vn(c-1) until GBO(c-1), its last reader, completes
            auto issue_gu = [&](int c) -> bool {
                if (c > 0 && !wait(L::BO + ((c - 1) & 1), ((c - 1) >> 1) & 1)) return false;
                if (!wait(L::FULLV + (c & 1), (c >> 1) & 1)) return false;
                tc::tc_fence_after();
                GU(c);
                return true;
            };
            bool ok = nchunks == 0 ||
                      (issue_g1(0) && (nchunks < 2 || issue_g1(1)) && issue_gw(0) && issue_gu(0));
            for (int c = 0; ok && c < nchunks; ++c) {
                // GA(c) needs bf16 S_c, -W(c) and (c > 0) the O^T columns read out and zeroed
                ok = wait(L::ESB, c & 1) && wait(L::EWE, c & 1) && (c == 0 || wait(L::EOR, (c - 1) & 1));
                if (!ok) break;
                tc::tc_fence_after();
                GA(c);
                // window while the state group converts Vn: GW(c+1), G1(c+2) when their inputs are ready
                bool gw_done = c + 1 >= nchunks, g1_done = c + 2 >= nchunks;
                if (!gw_done && tc::mbar_test(bars + L::ETB, (c + 1) & 1) &&
                    (!GATED || tc::mbar_test(bars + L::ESC + ((c + 1) & 1), ((c + 1) >> 1) & 1))) {
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
                GBS(c);
                GBO(c);
                // window while the state group converts S: what is left of GW(c+1) / G1(c+2), then GU(c+1)
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
