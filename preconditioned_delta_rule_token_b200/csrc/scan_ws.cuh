// Preconditioner scan in chunk form (bf16 inputs, dk = 128) on sm_100a.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary sections 2.2-2.3: d_{t+1} = r_t d_t + x_t u_t
// with x_t = eta beta_t (1 - beta_t <d_t, a_t>), a_t = k_t^2, u_t = a_t/||k_t||^2,
// and the scaled write key kw_t = d_t (.) k_t. The recurrence is affine in d,
// which the APF section states is what keeps the two-phase scan possible; per
// sub-chunk of L = 64 tokens with carry d_c it unrolls to
//   (I + M) x = c,  M_tj = g_t beta_t R_{t,j+1} <a_j, a_t> / ||k_j||^2 (j < t),
//   c_t = g_t (1 - beta_t R_{t,0} <d_c, a_t>),   g_t = eta beta_t,
//   d_t = R_{t,0} d_c + sum_{j<t} R_{t,j+1} x_j u_j,   R_{t,j} = prod_{m=j}^{t-1} r_m,
// so the serial dependence shrinks from one 128-wide reduction per token to
// three small matrix-vector steps per 64 tokens; everything that does not
// involve the carry (M and N = (I + M)^{-1}) is prepared a block ahead.
//
// One CTA (384 threads) per (sequence, head), blocks of 128 tokens:
//   prep groups P0 (warps 4-7) and P1 (warps 8-11), one block ahead of the
//     chain: beta, r, a_t = k_t^2 as a bf16 tile and ||k_t||^2 (each group
//     half of the features); one tcgen05 MMA (M = N = K = 128, A = B = the a
//     tile) gives <a_t, a_j> for the whole block, whose two 64 x 64 diagonal
//     blocks are the sub-chunk Grams; row t of M (decay products walked right
//     to left; P0 takes columns 32-63 of the row, P1 columns 0-31); then
//     P0 inverts sub-chunk 0 and P1 sub-chunk 1 at the same time, in place.
//   chain group (warps 0-3): the carry. Per sub-chunk: b_t = <d_c, a_t> and
//     c_t, x = N c, then thread i runs feature i through the sub-chunk, writing
//     kw_t[i] = d_t[i] k_t[i] over k_t[i] and carrying d; then one TMA store of
//     the block's scaled keys; its buffer takes the block three ahead once the
//     store has read it (issued at the start of the next block).
// Anchored APF (retention toward d0): with e = d - d0 the recurrence is the
// plain one, e_{t+1} = r_t e_t + x_t u_t, and <d_t, a_t> = <e_t, a_t> + <d0, a_t>;
// the chain carries e and adds <d0, a_t> to the chunk-start term of c_t (the
// plain case is d0 -> 0 in both).
// Optional diagnostic (sections 4-5): the residual ratio of each write,
// rho_t = (1 - beta_t <d_t, k_t^2>)^2 = f_t(S_t)/f_t(S_{t-1}), into rho [B, T, H]
// and q_geo = exp(mean_t log rho_t) per (sequence, head). Since
// x_t = g_t (1 - beta_t <d_t, k_t^2>), 1 - beta_t <d_t, k_t^2> = x_t / g_t when
// g_t != 0; with g_t = 0 and a write (eta = 0) the x are all zero, d_t = R_{t,0} d_c
// and the factor is 1 - beta_t R_{t,0} b_t; with no write (beta_t = 0 or k_t = 0)
// rho_t = 1.
// K blocks are triple-buffered; N, the per-token vectors and the hand-offs are
// double-buffered by block parity. Bounded mbarrier waits with a shared abort
// flag, as in the chunk kernel.
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct ScanLayout {
    static constexpr int NKB = 3;
    static constexpr uint32_t KB = 0;                        // K blocks [128 t][128 i] bf16 (two 16 KB halves);
                                                             // the scaled keys overwrite K in place
    static constexpr uint32_t AS = NKB * 32768;              // a = k^2 bf16, same layout (Gram operand)
    static constexpr int LD = tri::LD;
    static constexpr uint32_t MAT = 64 * LD * 4;
    static constexpr uint32_t MF = AS + 32768;               // [block parity][sub-chunk] M, then N, fp32
    static constexpr uint32_t VEC = MF + 4 * MAT;            // per block parity: beta, r, g, 1/||k||^2, R_{t,0}
    enum { V_BETA = 0, V_R = 128, V_G = 256, V_INVN = 384, V_R0 = 512, V_PAR = 640 };
    static constexpr uint32_t NP = VEC + 2 * V_PAR * 4;      // prep: ||k_t||^2 halves [2][128]
    static constexpr uint32_t CV = NP + 256 * 4;             // chain: c (64), x / ||k||^2 (64), d (128)
    // c, x / ||k||^2, the carry e = d - d_anchor, the chunk-start part of <d_t, a_t>, log-rho sums (4),
    // the retention target d_anchor (d0 under anchored APF, else 0)
    enum { C_C = 0, C_X = 64, C_D = 128, C_B = 256, C_LR = 320, C_DA = 324, C_N = 452 };
    static constexpr uint32_t BAR = CV + C_N * 4;
    enum {
        FULL = 0,    // 3: K block landed
        GRAM = 3,    // Gram MMA done
        NRDY = 4,    // 2: N of both sub-chunks and the vectors of a block parity ready (one arrival per group)
        MFREE = 6,   // 2: the chain has finished with a block parity
        DRAIN = 8,   // the Gram MMA of an abandoned block has completed
        NBAR = 9
    };
    static constexpr uint32_t TSLOT = BAR + NBAR * 8;
    static constexpr uint32_t ABORT = TSLOT + 4;
    static constexpr uint32_t END = ABORT + 4;
    static constexpr size_t kBytes = END + 1024;
    static constexpr uint32_t kTx = 2 * 16384;
};

// TRAJ = 1 also writes d_t (fp32, before token t's own update) of every token to
// d_traj [B, T, H, DK], the trajectory the backward differentiates through.
template <int TRAJ = 0>
__global__ void __launch_bounds__(384, 1)
scan_ws_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kw,
               const __nv_bfloat16* __restrict__ beta, const __nv_bfloat16* __restrict__ r,
               const float* __restrict__ d0, float* __restrict__ d_final, float* __restrict__ rho,
               float* __restrict__ q_geo, float* __restrict__ d_traj, int B, int T, int H, float eta, int anchor,
               unsigned long long wait_limit_ns)
{
    constexpr int DK = 128, BLK = 128, SUB = 64;
    constexpr uint32_t NCOLS = 128;
    constexpr uint32_t ID_GRAM = tc::idesc_bf16(128, 128, 0, 0);
    constexpr int BAR_CHAIN = 1, BAR_PREP = 2, BAR_P0 = 3;   // BAR_P0 + g: prep group g alone
    using L = ScanLayout;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays a shared pointer
    const uint32_t sb = tc::smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::TSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::ABORT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int nblk = (T + BLK - 1) / BLK;

    if (tid == 0) {
        for (int i = 0; i < L::NBAR; ++i) tc::mbar_init(bars + i, (i == L::NRDY || i == L::NRDY + 1) ? 2 : 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_kw);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, NCOLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto wait = [&](int bi, uint32_t parity) -> bool {   // bounded; stops when another role has aborted
        uint64_t* bar = bars + bi;
        // the hardware suspend of one try is capped by the limit, so a short limit ends a wait promptly
        const uint32_t hint = wait_limit_ns < 20000ull ? (uint32_t)wait_limit_ns : 20000u;
        if (tc::mbar_try_wait(bar, parity, hint)) return true;
        const uint64_t t0 = tc::globaltimer_ns();
        while (true) {
            if (tc::mbar_try_wait(bar, parity, hint)) return true;
            if (*abort_flag) return false;
            if (tc::globaltimer_ns() - t0 > wait_limit_ns) {
                *abort_flag = 1;
                atomicOr(&g_osdn_status, kStatusTimeout);
                return false;
            }
        }
    };
    auto kblock = [&](int blk) { return sm + L::KB + (blk % L::NKB) * 32768; };
    auto vecs = [&](int blk) { return reinterpret_cast<float*>(sm + L::VEC) + (blk & 1) * L::V_PAR; };

    if (warp < 4) {
        // ================================================================ chain group
        float* cv = reinterpret_cast<float*>(sm + L::CV);
        float* s_c = cv + L::C_C;
        float* s_x = cv + L::C_X;
        float* s_d = cv + L::C_D;
        float* s_b = cv + L::C_B;
        float* s_da = cv + L::C_DA;
        const bool diag = rho != nullptr || q_geo != nullptr;
        float log_rho = 0.f;   // this thread's share of sum_t log rho_t
        constexpr int kTmaThread = 32;
        int issued = 0;   // K blocks whose load was issued
        auto load_k = [&](int blk) {
            uint64_t* fb = bars + L::FULL + blk % L::NKB;
            tc::mbar_arrive_expect_tx(fb, L::kTx);
            tc::tma_load_4d(kblock(blk), &tm_k, 0, h, blk * BLK, b, fb);
            tc::tma_load_4d(kblock(blk) + 16384, &tm_k, 64, h, blk * BLK, b, fb);
        };
        if (tid == kTmaThread)
            while (issued < L::NKB && issued < nblk) load_k(issued++);
        {
            const float d_init = d0 ? d0[(size_t)unit * DK + tid] : 1.f;
            s_da[tid] = anchor ? d_init : 0.f;
            s_d[tid] = d_init - s_da[tid];   // the carry e = d - d_anchor
        }
        tc::named_sync(BAR_CHAIN, 128);

        int blk = 0;
        for (; blk < nblk; ++blk) {
            const int Tb = min(BLK, T - blk * BLK);
            uint8_t* KS = kblock(blk);
            const float* vb = vecs(blk);
            if (tc::named_sync_or(BAR_CHAIN, 128, !wait(L::NRDY + (blk & 1), (blk >> 1) & 1))) break;
            for (int s = 0; s < 2 && s * SUB < Tb; ++s) {
                const float* Nm = reinterpret_cast<const float*>(sm + L::MF + ((blk & 1) * 2 + s) * L::MAT);
                {   // b_t = <e_c, a_t>; c_t = g_t (1 - beta_t (R_{t,0} b_t + <d_anchor, a_t>)); two threads per token
                    const int tl_ = tid >> 1, half = tid & 1, t = s * SUB + tl_;
                    float acc = 0.f, acc_a = 0.f;
#pragma unroll
                    for (int c0 = 0; c0 < 8; ++c0) {
                        // the two halves walk their 16-byte chunks four apart, so the two threads of a
                        // token never hit the same bank group
                        const int c = (c0 + 4 * half) & 7;
                        const uint4 raw = *reinterpret_cast<const uint4*>(KS + half * 16384 + tc::sw128_off(t, c));
                        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
                        const float4 dlo = *reinterpret_cast<const float4*>(s_d + half * 64 + c * 8);
                        const float4 dhi = *reinterpret_cast<const float4*>(s_d + half * 64 + c * 8 + 4);
                        const float dd[8] = {dlo.x, dlo.y, dlo.z, dlo.w, dhi.x, dhi.y, dhi.z, dhi.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(p2[e]);
                            acc = fmaf(f.x * f.x, dd[2 * e], acc);
                            acc = fmaf(f.y * f.y, dd[2 * e + 1], acc);
                        }
                        if (anchor) {
                            const float4 alo = *reinterpret_cast<const float4*>(s_da + half * 64 + c * 8);
                            const float4 ahi = *reinterpret_cast<const float4*>(s_da + half * 64 + c * 8 + 4);
                            const float da[8] = {alo.x, alo.y, alo.z, alo.w, ahi.x, ahi.y, ahi.z, ahi.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = __bfloat1622float2(p2[e]);
                                acc_a = fmaf(f.x * f.x, da[2 * e], acc_a);
                                acc_a = fmaf(f.y * f.y, da[2 * e + 1], acc_a);
                            }
                        }
                    }
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
                    if (half == 0) {
                        const float known = vb[L::V_R0 + t] * acc + acc_a;   // <d_t, a_t> without the x terms
                        s_c[tl_] = vb[L::V_G + t] * (1.f - vb[L::V_BETA + t] * known);
                        s_b[tl_] = known;
                    }
                }
                if (s == 0 && tid == kTmaThread && blk > 0 && issued < nblk) {
                    // the buffer of block blk - 1 takes block blk + 2 once its store has read it (issued
                    // here, a step after that store, so that the wait is normally over already)
                    tc::bulk_wait_read<0>();
                    load_k(issued++);
                }
                tc::named_sync(BAR_CHAIN, 128);
                {   // x = N c (two threads per row), kept as x_t / ||k_t||^2
                    const int tl_ = tid >> 1, half = tid & 1;
                    // half h takes columns 16h + 32m + 4i (m < 2, i < 4): with the 68-float row stride the
                    // eight threads of a quarter warp then read eight different 16-byte bank groups
                    const float* Nrow = Nm + tl_ * L::LD + half * 16;
                    const float* cc = s_c + half * 16;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int col = 32 * (m >> 2) + 4 * (m & 3);
                        const float4 n4 = *reinterpret_cast<const float4*>(Nrow + col);
                        const float4 c4 = *reinterpret_cast<const float4*>(cc + col);
                        acc = fmaf(n4.x, c4.x, fmaf(n4.y, c4.y, fmaf(n4.z, c4.z, fmaf(n4.w, c4.w, acc))));
                    }
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    const int t = s * SUB + tl_;
                    if (half == 0) s_x[tl_] = acc * vb[L::V_INVN + t];
                    if (diag && half == 0 && t < Tb) {   // residual ratio of token t (acc = x_t)
                        const float gt = vb[L::V_G + t], bt = vb[L::V_BETA + t];
                        float f = 1.f;
                        if (gt != 0.f) f = acc / gt;
                        else if (bt != 0.f && vb[L::V_INVN + t] > 0.f) f = 1.f - bt * s_b[tl_];
                        const float rt = f * f;
                        if (rho) rho[((size_t)b * T + blk * BLK + t) * H + h] = rt;
                        log_rho += logf(rt);
                    }
                }
                tc::named_sync(BAR_CHAIN, 128);
                {   // feature i through the sub-chunk, 32 tokens at a time from registers:
                    // kw_t = d_t (.) k_t over k_t, d_{t+1} = r_t d_t + (x_t / ||k_t||^2) k_t^2.
                    // Tokens past T have k = 0, r = 1, x = 0 and leave d unchanged (their rows are not stored).
                    const int i = tid;
                    uint8_t* colbase = KS + (i >> 6) * 16384 + 2 * (i & 7);
                    const int cidx = (i & 63) >> 3;
                    const float da = s_da[i];
                    float d = s_d[i];   // the carry e = d - d_anchor
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {   // rolled: smaller code
                        const int tb = s * SUB + hh * 32;   // multiple of 8
                        uint8_t* rowbase = colbase + (tb >> 3) * 1024;
                        float kk[32], rr[32], xx[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            kk[j] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                rowbase + (j >> 3) * 1024 + (j & 7) * 128 + ((cidx ^ (j & 7)) << 4)));
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 r4 = *reinterpret_cast<const float4*>(vb + L::V_R + tb + j);
                            const float4 x4 = *reinterpret_cast<const float4*>(s_x + hh * 32 + j);
                            rr[j] = r4.x; rr[j + 1] = r4.y; rr[j + 2] = r4.z; rr[j + 3] = r4.w;
                            xx[j] = x4.x; xx[j + 1] = x4.y; xx[j + 2] = x4.z; xx[j + 3] = x4.w;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float kv = kk[j];
                            if constexpr (TRAJ != 0) {
                                const int t = blk * BLK + tb + j;
                                if (t < T) d_traj[(((size_t)b * T + t) * H + h) * DK + i] = d + da;
                            }
                            kk[j] = (d + da) * kv;                           // scaled key, with d before token j
                            d = fmaf(rr[j], d, xx[j] * (kv * kv));
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            *reinterpret_cast<__nv_bfloat16*>(rowbase + (j >> 3) * 1024 + (j & 7) * 128 +
                                                              ((cidx ^ (j & 7)) << 4)) = __float2bfloat16_rn(kk[j]);
                    }
                    s_d[i] = d;
                }
                tc::named_sync(BAR_CHAIN, 128);
            }
            if (tid == 0) tc::mbar_arrive1(bars + L::MFREE + (blk & 1));   // N and vectors of this parity consumed
            tc::fence_proxy_async_smem();
            tc::named_sync(BAR_CHAIN, 128);
            if (tid == kTmaThread) {   // the scaled keys leave
                tc::tma_store_4d(&tm_kw, KS, 0, h, blk * BLK, b);
                tc::tma_store_4d(&tm_kw, KS + 16384, 64, h, blk * BLK, b);
                tc::bulk_commit();
            }
        }
        if (tid == kTmaThread) {   // stores complete; loads that were issued have landed
            tc::bulk_wait<0>();
            for (int q = issued > L::NKB ? issued - L::NKB : 0; q < issued; ++q)
                tc::mbar_wait(bars + L::FULL + q % L::NKB, (q / L::NKB) & 1, 1000000000ull);
        }
        if (blk == nblk && !*abort_flag && d_final) d_final[(size_t)unit * DK + tid] = s_d[tid] + s_da[tid];
        if (q_geo) {   // q_geo = exp(mean log rho): warp sums, then one thread
            float* lr = cv + L::C_LR;
            const float ws = warp_sum(log_rho);
            if (lane == 0) lr[warp] = ws;
            tc::named_sync(BAR_CHAIN, 128);
            if (tid == 0 && blk == nblk && !*abort_flag)
                q_geo[unit] = T > 0 ? expf((lr[0] + lr[1] + lr[2] + lr[3]) / (float)T) : 1.f;
        }
    } else {
        // ================================================================ prep groups
        const int tp = tid - 128;              // 0..255
        const int g = tp >> 7;                 // group: 0 = warps 4-7, 1 = warps 8-11
        const int row = tp & 127;              // token of the block and TMEM lane this thread serves
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        float* np = reinterpret_cast<float*>(sm + L::NP);
        // group 0: beta, group 1: r (1 past T or without APF); loaded a block ahead as bf16 and
        // converted where it is used, so that the load is not waited for where it is issued
        auto load_pv = [&](int blk) -> __nv_bfloat16 {
            const int tok = blk * BLK + row;
            const size_t gi = ((size_t)b * T + tok) * H + h;
            if (g == 0) return tok < T ? beta[gi] : __float2bfloat16(0.f);
            return (tok < T && r) ? r[gi] : __float2bfloat16(1.f);
        };
        __nv_bfloat16 pv = nblk > 0 ? load_pv(0) : __float2bfloat16(0.f);
        for (int blk = 0; blk < nblk; ++blk) {
            uint8_t* KS = kblock(blk);
            float* vb = vecs(blk);
            bool fail = !wait(L::FULL + blk % L::NKB, (blk / L::NKB) & 1);
            if (!fail && blk >= 2) fail = !wait(L::MFREE + (blk & 1), ((blk - 2) >> 1) & 1);
            if (tc::named_sync_or(BAR_PREP, 256, fail)) break;
            // beta (group 0) or r (group 1) of token `row`, loaded one block ahead
            const float bt = __bfloat162float(pv);
            if (g == 0) vb[L::V_BETA + row] = bt;
            else vb[L::V_R + row] = bt;
            if (blk + 1 < nblk) pv = load_pv(blk + 1);
            {   // a = k^2 (bf16 tile) over this group's half of the features; partial ||k||^2
                float nrm = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t off = g * 16384 + tc::sw128_off(row, q);
                    const uint4 raw = *reinterpret_cast<const uint4*>(KS + off);
                    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
                    uint4 pa;
                    uint32_t* wa = reinterpret_cast<uint32_t*>(&pa);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(p2[e]);
                        const float ax = f.x * f.x, ay = f.y * f.y;
                        nrm += ax + ay;
                        wa[e] = tc::pack_bf16(ax, ay);
                    }
                    *reinterpret_cast<uint4*>(sm + L::AS + off) = pa;
                }
                np[g * 128 + row] = nrm;
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::named_sync(BAR_PREP, 256);
            if (tp == 0) {   // the block Gram <a_t, a_j>
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                    const uint64_t d = tc::sdesc_sw128(sb + L::AS + half * 16384 + koff, 16, 1024);
                    tc::umma_bf16(tmem, d, d, ID_GRAM, ks > 0);
                }
                tc::umma_commit(bars + L::GRAM);
            }
            if (g == 0) {
                const float nrm = np[row] + np[128 + row];
                vb[L::V_INVN + row] = nrm > 0.f ? 1.f / nrm : 0.f;
                vb[L::V_G + row] = nrm > 0.f ? eta * bt : 0.f;
            }
            fail = !wait(L::GRAM, blk & 1);
            if (tc::named_sync_or(BAR_PREP, 256, fail)) break;
            tc::tc_fence_after();
            {   // row `row` of M for its sub-chunk; group 0 columns 32-63, group 1 columns 0-31
                const int s = row >> 6, tl_ = row & 63, jb = g == 0 ? 32 : 0;
                uint32_t gr[32];
                tc::tmem_ld32(tl + s * 64 + jb, gr);
                tc::tmem_wait_ld();
                const float coef = vb[L::V_G + row] * vb[L::V_BETA + row];
                const float* rr = vb + L::V_R + s * SUB;
                const float* iv = vb + L::V_INVN + s * SUB;
                float rj[32], ivj[32];
#pragma unroll
                for (int j4 = 0; j4 < 32; j4 += 4) {
                    const float4 r4 = *reinterpret_cast<const float4*>(rr + jb + j4);
                    const float4 i4 = *reinterpret_cast<const float4*>(iv + jb + j4);
                    rj[j4] = r4.x; rj[j4 + 1] = r4.y; rj[j4 + 2] = r4.z; rj[j4 + 3] = r4.w;
                    ivj[j4] = i4.x; ivj[j4 + 1] = i4.y; ivj[j4 + 2] = i4.z; ivj[j4 + 3] = i4.w;
                }
                float R = 1.f;   // R_{tl, jb + 32} when the walk enters this group's columns
                if (g == 1) {    // product of r over columns 32..tl-1, from the other half
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const float4 r4 = *reinterpret_cast<const float4*>(rr + 32 + j4);
                        if (32 + j4 < tl_) R *= r4.x;
                        if (33 + j4 < tl_) R *= r4.y;
                        if (34 + j4 < tl_) R *= r4.z;
                        if (35 + j4 < tl_) R *= r4.w;
                    }
                }
                float mrow[32];
#pragma unroll
                for (int jj = 31; jj >= 0; --jj) {
                    const int j = jb + jj;
                    mrow[jj] = 0.f;
                    if (j < tl_) {
                        mrow[jj] = coef * R * __uint_as_float(gr[jj]) * ivj[jj];
                        R *= rj[jj];
                    }
                }
                float* Mrow = reinterpret_cast<float*>(sm + L::MF + ((blk & 1) * 2 + s) * L::MAT) + tl_ * L::LD + jb;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4*>(Mrow + j) = make_float4(mrow[j], mrow[j + 1], mrow[j + 2], mrow[j + 3]);
                if (g == 1) vb[L::V_R0 + row] = R;   // R_{tl, 0}
            }
            tc::tc_fence_before();
            tc::named_sync(BAR_PREP, 256);
            // N = (I + M)^{-1} of sub-chunk g, in place, by group g
            tri::tril_inv64_inplace(reinterpret_cast<float*>(sm + L::MF + ((blk & 1) * 2 + g) * L::MAT), warp & 3, lane,
                                    [g] { tc::named_sync(BAR_P0 + g, 128); });
            if (row == 0) tc::mbar_arrive1(bars + L::NRDY + (blk & 1));
        }
        if (tp == 0) {   // an issued Gram MMA completes before TMEM is released
            tc::umma_commit(bars + L::DRAIN);
            tc::mbar_wait(bars + L::DRAIN, 0, 1000000000ull);
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
