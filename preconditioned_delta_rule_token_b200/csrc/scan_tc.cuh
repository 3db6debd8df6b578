// Preconditioner scan in chunk form (bf16 inputs, dk = 128) on sm_100a.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary sections 2.2-2.3: d_{t+1} = r_t d_t + x_t u_t
// with x_t = eta beta_t (1 - beta_t <d_t, a_t>), a_t = k_t^2, u_t = a_t/||k_t||^2,
// and the scaled write key kw_t = d_t (.) k_t. The recurrence is affine in d,
// which the APF section states is what keeps the two-phase scan possible; per
// sub-chunk of L = 64 tokens with carry d_c it unrolls to
//   (I + M) x = c,  M_tj = g_t beta_t R_{t,j+1} <u_j, a_t> (j < t),
//   c_t = g_t (1 - beta_t R_{t,0} <d_c, a_t>),   g_t = eta beta_t,
//   d_t = R_{t,0} d_c + sum_{j<t} R_{t,j+1} x_j u_j,   R_{t,j} = prod_{m=j}^{t-1} r_m,
// so the serial dependence shrinks from one 128-wide reduction per token to
// one small solve per 64 tokens.
//
// One CTA (128 threads) per (sequence, head); blocks of 128 tokens:
//   TMA loads K [128 t][128 i] (128-byte swizzle); thread t forms a_t, u_t;
//   one tcgen05 MMA (M = N = K = 128) gives <a_t, u_j> for the whole block
//   (the two 64 x 64 diagonal blocks are the sub-chunk Grams);
//   thread t builds row t of M (decay products walked right to left);
//   per sub-chunk: N = (I + M)^{-1} (blocked inverse), b_t = <d_c, a_t>,
//   x = N c, then thread i runs feature i through the sub-chunk, writing
//   kw_t[i] = d_t[i] k_t[i] over k_t[i] and carrying d to the next sub-chunk.
// K blocks are triple-buffered (the next block loads while this one is
// processed and the previous one's store drains); the scaled keys overwrite K in shared memory and leave with one
// TMA store per block. Bounded mbarrier waits as in the chunk kernel.
#pragma once
#include "tc_ptx.cuh"
#include "tril_inv.cuh"

namespace osdn {

struct ScanSmem {
    static constexpr int NBUF = 3;                        // K blocks in flight: load b+1 while b is processed
                                                          // and the store of b-1 drains
    static constexpr uint32_t KS = 0;                     // K blocks [128 t][128 i] bf16 (two 16 KB halves
                                                          // each); the scaled keys overwrite K in place
    static constexpr uint32_t AS = NBUF * 32768;          // a = k^2 (bf16), same layout
    static constexpr uint32_t US = AS + 32768;            // u = a / ||k||^2 (bf16), same layout
    static constexpr int LD = tri::LD;
    static constexpr uint32_t MF = US + 32768;            // M, two sub-chunks [64][LD] fp32
    static constexpr uint32_t NF = MF + 2 * 64 * LD * 4;  // N [64][LD] fp32
    static constexpr uint32_t VEC = NF + 64 * LD * 4;     // per-token / per-feature vectors
    // vector slots (floats), each 128 long
    static constexpr int V_BETA = 0, V_R = 128, V_G = 256, V_INVN = 384, V_R0 = 512, V_C = 640, V_X = 768,
                         V_D = 896, V_N = 1024;
    static constexpr uint32_t BAR = VEC + V_N * 4;        // tma_bar[NBUF], mma_bar, tmem base address
    static constexpr uint32_t END = BAR + 64;
    static constexpr size_t kBytes = END + 1024;
    static constexpr uint32_t kTxBytes = 2 * 16384;
};

template <int kUnused = 0>
__global__ void __launch_bounds__(128, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kw,
               const __nv_bfloat16* __restrict__ beta, const __nv_bfloat16* __restrict__ r,
               const float* __restrict__ d0, float* __restrict__ d_final, int B, int T, int H, float eta,
               unsigned long long wait_limit_ns)
{
    constexpr int DK = 128, BLK = 128, SUB = 64;
    constexpr uint32_t NCOLS = 128;
    constexpr uint32_t ID_GRAM = tc::idesc_bf16(128, 128, 0, 0);
    using L = ScanSmem;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);   // stays a shared pointer
    const uint32_t sb = tc::smem_u32(sm);
    float* MF = reinterpret_cast<float*>(sm + L::MF);
    float* NF = reinterpret_cast<float*>(sm + L::NF);
    float* vec = reinterpret_cast<float*>(sm + L::VEC);
    float* s_beta = vec + L::V_BETA;
    float* s_r = vec + L::V_R;
    float* s_g = vec + L::V_G;
    float* s_invn = vec + L::V_INVN;
    float* s_R0 = vec + L::V_R0;
    float* s_c = vec + L::V_C;
    float* s_x = vec + L::V_X;
    float* s_d = vec + L::V_D;
    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + L::BAR);   // one per K buffer
    uint64_t* mma_bar = tma_bar + L::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tma_bar + L::NBUF + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;

    if (tid == 0) {
        for (int q = 0; q < L::NBUF; ++q) tc::mbar_init(tma_bar + q, 1);
        tc::mbar_init(mma_bar, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_kw);
        if (T > 0) {   // first K block
            tc::mbar_arrive_expect_tx(tma_bar, L::kTxBytes);
            tc::tma_load_4d(sm + L::KS, &tm_k, 0, h, 0, b, tma_bar);
            tc::tma_load_4d(sm + L::KS + 16384, &tm_k, 64, h, 0, b, tma_bar);
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, NCOLS);
        tc::tmem_relinquish();
    }
    s_d[tid] = d0 ? d0[(size_t)unit * DK + tid] : 1.f;
    tri::tril_zero_upper(NF, tid, 128);   // the inverse never writes those blocks
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);

    uint32_t tma_phase = 0, mma_phase = 0;     // tma_phase: bit per K buffer
    bool failed = false, tma_pending = (T > 0), mma_pending = false;
    for (int t0 = 0, blk = 0; t0 < T; t0 += BLK, ++blk) {
        const int Tb = min(BLK, T - t0);
        const int buf = blk % L::NBUF;
        uint8_t* KS = sm + L::KS + buf * 32768;
        // (1) prefetch the next K block into the buffer of block blk - 2 once that block's
        //     store has read it (the store of blk - 1 may still be in flight); beta and r
        if (tid == 0 && t0 + BLK < T) {
            tc::bulk_wait_read<1>();
            const int nbuf = (blk + 1) % L::NBUF;
            uint64_t* nb = tma_bar + nbuf;
            uint8_t* nK = sm + L::KS + nbuf * 32768;
            tc::mbar_arrive_expect_tx(nb, L::kTxBytes);
            tc::tma_load_4d(nK, &tm_k, 0, h, t0 + BLK, b, nb);
            tc::tma_load_4d(nK + 16384, &tm_k, 64, h, t0 + BLK, b, nb);
        }
        {
            const bool in = tid < Tb;
            const size_t tok = ((size_t)b * T + t0 + tid) * H + h;
            s_beta[tid] = in ? __bfloat162float(beta[tok]) : 0.f;
            s_r[tid] = (in && r) ? __bfloat162float(r[tok]) : 1.f;
        }
        if (!tc::mbar_wait(tma_bar + buf, (tma_phase >> buf) & 1, wait_limit_ns)) failed = true;
        else { tma_phase ^= 1u << buf; tma_pending = (t0 + BLK < T); }
        if (__syncthreads_or(failed)) break;

        // (2) thread t: a_t = k_t^2 and u_t = a_t / ||k_t||^2 as bf16 MMA operands (one read of row t)
        {
            const int t = tid;
            uint4 raw[16];
            float nrm = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                raw[q] = *reinterpret_cast<const uint4*>(KS + (q >> 3) * 16384 + tc::sw128_off(t, q & 7));
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[q]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(p2[e]);
                    nrm = fmaf(f.x, f.x, fmaf(f.y, f.y, nrm));
                }
            }
            const float invn = nrm > 0.f ? 1.f / nrm : 0.f;
            s_invn[t] = invn;
            s_g[t] = nrm > 0.f ? eta * s_beta[t] : 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const uint32_t off = (q >> 3) * 16384 + tc::sw128_off(t, q & 7);
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[q]);
                uint4 pa, pu;
                uint32_t* wa = reinterpret_cast<uint32_t*>(&pa);
                uint32_t* wu = reinterpret_cast<uint32_t*>(&pu);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(p2[e]);
                    const float ax = f.x * f.x, ay = f.y * f.y;
                    wa[e] = tc::pack_bf16(ax, ay);
                    wu[e] = tc::pack_bf16(ax * invn, ay * invn);
                }
                *reinterpret_cast<uint4*>(sm + L::AS + off) = pa;
                *reinterpret_cast<uint4*>(sm + L::US + off) = pu;
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // (3) Gram of the block: D[t][j] = <a_t, u_j>
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
                tc::umma_bf16(tmem, tc::sdesc_sw128(sb + L::AS + half * 16384 + koff, 16, 1024),
                              tc::sdesc_sw128(sb + L::US + half * 16384 + koff, 16, 1024), ID_GRAM, ks > 0);
            }
            tc::umma_commit(mma_bar);
        }
        mma_pending = true;
        if (!tc::mbar_wait(mma_bar, mma_phase, wait_limit_ns)) failed = true;
        else { mma_phase ^= 1; mma_pending = false; }
        if (__syncthreads_or(failed)) break;
        tc::tc_fence_after();

        // (4) row t of M for its sub-chunk: M[tl][j] = g_t beta_t R_{tl,j+1} <u_j, a_t> (j < tl)
        {
            const int t = tid, s = t >> 6, tl_ = t & 63;
            uint32_t gr[64];
            {
                uint32_t r0[32], r1[32];
                tc::tmem_ld32(tl + s * 64, r0);
                tc::tmem_ld32(tl + s * 64 + 32, r1);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) { gr[e] = r0[e]; gr[32 + e] = r1[e]; }
            }
            const float coef = s_g[t] * s_beta[t];
            const float* rr = s_r + s * SUB;
            float* Mrow = MF + s * 64 * L::LD + tl_ * L::LD;
            float R = 1.f;                       // R_{tl, j+1}, walked from j = tl - 1 down
            float m[SUB];
#pragma unroll
            for (int j = SUB - 1; j >= 0; --j) {
                m[j] = 0.f;
                if (j < tl_) {
                    m[j] = coef * R * __uint_as_float(gr[j]);
                    R *= rr[j];
                }
            }
#pragma unroll
            for (int j = 0; j < SUB; j += 4)   // row stride 68 floats: conflict-free 16-byte stores
                *reinterpret_cast<float4*>(Mrow + j) = make_float4(m[j], m[j + 1], m[j + 2], m[j + 3]);
            s_R0[t] = R;                         // R_{tl, 0}
        }
        tc::tc_fence_before();
        __syncthreads();

        // (5) the two sub-chunks in order: solve, then carry the preconditioner
        for (int s = 0; s < 2 && s * SUB < Tb; ++s) {
            tri::tril_inv64(MF + s * 64 * L::LD, NF, warp, lane, [] { __syncthreads(); });
            {   // b_t = <d_c, a_t>; c_t = g_t (1 - beta_t R_{t,0} b_t); two threads per token
                const int tl_ = tid >> 1, half = tid & 1, t = s * SUB + tl_;
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(KS + half * 16384 + tc::sw128_off(t, c));
                    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
                    const float* dd = s_d + half * 64 + c * 8;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(p2[e]);
                        acc = fmaf(f.x * f.x, dd[2 * e], acc);
                        acc = fmaf(f.y * f.y, dd[2 * e + 1], acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (half == 0) s_c[tl_] = s_g[t] * (1.f - s_beta[t] * s_R0[t] * acc);
            }
            __syncthreads();
            {   // x = N c
                const int tl_ = tid >> 1, half = tid & 1;
                const float* Nrow = NF + tl_ * L::LD + half * 32;
                const float* cc = s_c + half * 32;
                float acc = 0.f;
#pragma unroll
                for (int k2 = 0; k2 < 32; ++k2) acc = fmaf(Nrow[k2], cc[k2], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (half == 0) s_x[s * SUB + tl_] = acc * s_invn[s * SUB + tl_];   // x_t / ||k_t||^2
            }
            __syncthreads();
            {   // feature i through the sub-chunk, 32 tokens at a time from registers:
                // kw_t = d_t (.) k_t written over k_t in place, d_{t+1} = r_t d_t + (x_t / ||k_t||^2) k_t^2.
                // Tokens past T have k = 0, r = 1, x = 0 and leave d unchanged (their rows are not stored).
                const int i = tid;
                uint8_t* colbase = KS + (i >> 6) * 16384 + 2 * (i & 7);
                const int cidx = (i & 63) >> 3;
                float d = s_d[i];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int tb = s * SUB + hh * 32;                    // multiple of 8
                    uint8_t* rowbase = colbase + (tb >> 3) * 1024;
                    float kk[32], rr[32], xx[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        kk[j] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                            rowbase + (j >> 3) * 1024 + (j & 7) * 128 + ((cidx ^ (j & 7)) << 4)));
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 r4 = *reinterpret_cast<const float4*>(s_r + tb + j);
                        const float4 x4 = *reinterpret_cast<const float4*>(s_x + tb + j);
                        rr[j] = r4.x; rr[j + 1] = r4.y; rr[j + 2] = r4.z; rr[j + 3] = r4.w;
                        xx[j] = x4.x; xx[j + 1] = x4.y; xx[j + 2] = x4.z; xx[j + 3] = x4.w;
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float kv = kk[j];
                        kk[j] = d * kv;                                  // scaled key, with d before token j
                        d = fmaf(rr[j], d, xx[j] * (kv * kv));
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        *reinterpret_cast<__nv_bfloat16*>(rowbase + (j >> 3) * 1024 + (j & 7) * 128 +
                                                          ((cidx ^ (j & 7)) << 4)) = __float2bfloat16_rn(kk[j]);
                }
                s_d[i] = d;
            }
            __syncthreads();
        }
        // (6) the block now holds the scaled keys: one TMA store (rows past T are clipped)
        tc::fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_4d(&tm_kw, KS, 0, h, t0, b);
            tc::tma_store_4d(&tm_kw, KS + 16384, 64, h, t0, b);
            tc::bulk_commit();
        }
    }
    if (tid == 0) tc::bulk_wait<0>();
    if (!failed && d_final) d_final[(size_t)unit * DK + tid] = s_d[tid];
    if (failed && tid == 0) {
        atomicOr(&g_osdn_status, kStatusTimeout);
        const unsigned long long drain_ns = wait_limit_ns > 1000000000ull ? wait_limit_ns : 1000000000ull;
        for (int q = 0; q < L::NBUF; ++q)   // any K block still in flight
            if (tma_pending) tc::mbar_wait(tma_bar + q, (tma_phase >> q) & 1, drain_ns);
        if (mma_pending) tc::mbar_wait(mma_bar, mma_phase, drain_ns);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, NCOLS);
    }
}

}  // namespace osdn
