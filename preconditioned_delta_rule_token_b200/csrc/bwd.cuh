// OSDN backward: gradients of L = <dO, O> + <dS_T, S_T> + <dd_T, d_T> with
// respect to q, k, v, beta, r, d0 and S0 (training).
//
// The pages give no backward pass; this is the reverse-mode derivative of the
// chunkwise forward of "OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention" (technical summary section 2.1, the
// DeltaNet chunk pipeline with the scaled write key Kw = D (.) K; section 2.3,
// the APF recurrence of d).  Per chunk of C = 64 tokens with chunk-start state S:
//   forward:  Kb = diag(beta) K,  A = strict_tril(Kb Kw^T),  T = (I + A)^{-1},
//             W = T Kb,  U0 = T diag(beta) V,  Vn = U0 - W S^T,
//             P = tril(Q Kw^T),  O = Q S^T + P Vn,  S' = S + Vn^T Kw;
//   backward, with dS' = dL/dS' (from the later chunks):
//             dVn = P^T dO + Kw dS'^T,           dS  = dS' + dO^T Q - dVn^T W,
//             dP  = tril(dO Vn^T),               dQ  = dO S + dP Kw,
//             dKw = Vn dS' + dP^T Q + dAb^T K,   dW  = -dVn S,
//             dT  = (dW K^T + dVn V^T) diag(beta),
//             dA  = -strict_tril(T^T dT T^T),    dAb = diag(beta) dA,
//             dV  = diag(beta) T^T dVn,          dK  = diag(beta) T^T dW + dAb Kw + dKw (.) D,
//             dbeta = rowdot(T^T dW, K) + rowdot(T^T dVn, V) + rowsum(dA (.) K Kw^T),
//             dD  = dKw (.) K   (the adjoint of d_t through the write key).
// The d recurrence d_{t+1} = r d + (1 - r) d0 [anchored] + x a, with a = k^2,
// n = ||k||^2, s = <d, a>, x = eta beta (1 - beta s) / n, is then walked backward
// token by token with Ld = dL/dd_{t+1}:
//   dx = <a, Ld>,  dr = <d - d0 [anchored], Ld>,  dbeta += dx eta (1 - 2 beta s) / n,
//   dk += 2 k (.) (x Ld - dx (eta beta^2 / n) d - dx x / n),
//   dL/dd_t = r Ld + dD_t - dx (eta beta^2 / n) a,   dd0 += (1 - r) Ld [anchored].
//
// Kernels, in launch order (every chunk quantity lives in the workspace in a
// chunk-block layout [unit][chunk][row][col], fp32):
//   bwd_dtraj   d_t for every token (token-serial, one warp per unit);
//   bwd_prep    per chunk: Kw, T, W, U0, P;
//   bwd_state_f per (unit, dv tile): S at every chunk start, Vn;
//   bwd_state_b per (unit, dv tile), chunks in reverse: dS' at every chunk end, dVn, dS0;
//   bwd_grads_a per chunk, dv tiles in turn: dQ, dV, dW, dT, the dv-summed part of dKw and dbeta;
//   bwd_grads_b per chunk: dA, dK, dKw, dD and the rest of dbeta;
//   bwd_dchain  token-serial reverse of the d recurrence: dk, dbeta, dr, dd0.
// Rows of S are independent given the chunk matrices, so the two state passes
// split dv into tiles with no exchange.  The contractions run on mma.sync
// m16n8k8 tf32 with fp32 accumulation; for fp32 inputs every product uses the
// three-pass split a = a_hi + a_lo (a_hi b_hi + a_hi b_lo + a_lo b_hi), which
// keeps fp32 accuracy.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace osdn {
namespace bwd {

constexpr int C = 64;         // chunk length
constexpr int NTHR = 256;     // threads of the per-chunk and per-tile kernels (8 warps)
constexpr int LDC = C + 4;    // row stride of C x C tiles (68 = 4 mod 32: conflict-free fragments)

// X(i, j) = p[i * s0 + j * s1], fp32 in shared or global memory.
struct Mat {
    const float* p;
    int s0, s1;
    __device__ __forceinline__ float operator()(int i, int j) const { return p[i * s0 + j * s1]; }
};

__device__ __forceinline__ uint32_t tf32_rna(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma8(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// c += a b for one m16n8k8 step; SPLIT: three tf32 products that recover fp32 accuracy.
template <bool SPLIT>
__device__ __forceinline__ void mma_step(float (&c)[4], const float (&a)[4], const float (&b)[2]) {
    uint32_t ah[4], bh[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) ah[i] = tf32_rna(a[i]);
#pragma unroll
    for (int i = 0; i < 2; ++i) bh[i] = tf32_rna(b[i]);
    if (SPLIT) {
        uint32_t al[4], bl[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) al[i] = tf32_rna(a[i] - __uint_as_float(ah[i]));
#pragma unroll
        for (int i = 0; i < 2; ++i) bl[i] = tf32_rna(b[i] - __uint_as_float(bh[i]));
        mma8(c, al, bh);
        mma8(c, ah, bl);
    }
    mma8(c, ah, bh);
}

// One warp: acc[j] += sum_{k < K} A(m0 + ., k) B(k, n0 + 8 j + .) for a 16 x 8 NT tile.
// Fragment element e of acc[j] sits at row m0 + g + 8 (e >> 1), column n0 + 8 j + 2 t + (e & 1),
// with g = lane / 4, t = lane % 4.
template <int NT, bool SPLIT>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], Mat A, Mat B, int m0, int n0, int K, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float a[4] = {A(m0 + g, k0 + t), A(m0 + g + 8, k0 + t), A(m0 + g, k0 + t + 4),
                            A(m0 + g + 8, k0 + t + 4)};
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const float b[2] = {B(k0 + t, n0 + 8 * j + g), B(k0 + t + 4, n0 + 8 * j + g)};
            mma_step<SPLIT>(acc[j], a, b);
        }
    }
}

template <int NT>
__device__ __forceinline__ void frag_zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
}

template <int NT, typename F>
__device__ __forceinline__ void frag_each(float (&acc)[NT][4], int m0, int n0, int lane, F f) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) f(m0 + g + 8 * (e >> 1), n0 + 8 * j + 2 * t + (e & 1), acc[j][e]);
}

// The CTA computes the M x N product sum_k A(m, k) B(k, n) (plus, for the two-term
// form, a second product over K2) in 16 x 32 warp tiles taken round-robin, and calls
// epi(m, n, value) once per output element on the thread that holds it.
template <bool SPLIT, typename Epi>
__device__ __forceinline__ void cta_gemm(int M, int N, int K, Mat A, Mat B, Epi epi) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tn = N / 32, tiles = (M / 16) * tn;
    for (int tile = warp; tile < tiles; tile += nw) {
        const int m0 = (tile / tn) * 16, n0 = (tile % tn) * 32;
        float acc[4][4];
        frag_zero(acc);
        warp_mma<4, SPLIT>(acc, A, B, m0, n0, K, lane);
        frag_each(acc, m0, n0, lane, epi);
    }
}

template <bool SPLIT, typename Epi>
__device__ __forceinline__ void cta_gemm2(int M, int N, int K1, Mat A1, Mat B1, int K2, Mat A2, Mat B2, Epi epi) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tn = N / 32, tiles = (M / 16) * tn;
    for (int tile = warp; tile < tiles; tile += nw) {
        const int m0 = (tile / tn) * 16, n0 = (tile % tn) * 32;
        float acc[4][4];
        frag_zero(acc);
        warp_mma<4, SPLIT>(acc, A1, B1, m0, n0, K1, lane);
        warp_mma<4, SPLIT>(acc, A2, B2, m0, n0, K2, lane);
        frag_each(acc, m0, n0, lane, epi);
    }
}

// Workspace layout of one backward call (fp32 regions, 256-byte aligned).
struct Layout {
    size_t d_all, kw, tinv, w, u0, p, ckS, ckdS, vn, dvn, dkwa, dw, dt, dba, dd, dkp, dbp, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

inline Layout make_layout(int B, int T, int H, int DK, int DV) {
    const size_t units = (size_t)B * H, nc = (size_t)(T + C - 1) / C, ch = units * nc;
    const size_t f = sizeof(float);
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
    L.d_all = take(f * (size_t)B * T * H * DK);
    L.kw = take(f * ch * C * DK);
    L.tinv = take(f * ch * C * C);
    L.w = take(f * ch * C * DK);
    L.u0 = take(f * ch * C * DV);
    L.p = take(f * ch * C * C);
    L.ckS = take(f * ch * DV * DK);
    L.ckdS = take(f * ch * DV * DK);
    L.vn = take(f * ch * C * DV);
    L.dvn = take(f * ch * C * DV);
    L.dkwa = take(f * ch * C * DK);
    L.dw = take(f * ch * C * DK);
    L.dt = take(f * ch * C * C);
    L.dba = take(f * ch * C);
    L.dd = take(f * ch * C * DK);
    L.dkp = take(f * ch * C * DK);
    L.dbp = take(f * ch * C);
    L.total = o;
    return L;
}

template <typename Tin>
__device__ __forceinline__ float ld_or0(const Tin* p, size_t i, bool ok) { return ok ? to_f32(p[i]) : 0.f; }

// ---------------------------------------------------------------------------
// d_t (before the token's own update) for every token: one warp per unit.
template <int DK, typename Tin>
__global__ void __launch_bounds__(128)
bwd_dtraj_kernel(const Tin* __restrict__ k, const Tin* __restrict__ beta, const Tin* __restrict__ r,
                 const float* __restrict__ d0, float* __restrict__ d_all, int B, int T, int H, float eta, int anchor)
{
    constexpr int PER = DK / 32;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= B * H) return;
    const int b = unit / H, h = unit % H;
    float d[PER], da[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) d[i] = d0 ? d0[(size_t)unit * DK + lane * PER + i] : 1.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) da[i] = anchor ? d[i] : 0.f;
    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)b * T + t) * H + h;
        float kk[PER], a[PER];
        VecIO<PER, Tin>::load(k + tok * DK + lane * PER, kk);
        VecIO<PER, float>::store(d_all + tok * DK + lane * PER, d);
        const float bt = to_f32(beta[tok]), rt = r ? to_f32(r[tok]) : 1.f;
        float n = 0.f, s = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            a[i] = kk[i] * kk[i];
            n += a[i];
            s += d[i] * a[i];
        }
        n = warp_sum(n);
        s = warp_sum(s);
        const float x = (n > 0.f) ? eta * bt * (1.f - bt * s) / n : 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) d[i] = rt * d[i] + (1.f - rt) * da[i] + x * a[i];
    }
}

// ---------------------------------------------------------------------------
// Per chunk: Kw = D (.) K, T = (I + strict_tril(Kb Kw^T))^{-1}, W = T Kb,
// U0 = T diag(beta) V, P = tril(Q Kw^T).  One CTA per (unit, chunk).
template <int DK, int DV>
struct PrepSmem {
    static constexpr int LDK = DK + 4, LDX = (DK > DV ? DK : DV) + 4;
    static constexpr size_t kBytes = sizeof(float) * (size_t)(2 * C * LDK + C * LDX + 2 * C * LDC + C);
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_prep_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                const Tin* __restrict__ beta, float* __restrict__ ws, Layout L, int B, int T, int H, int NC)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    using SM = PrepSmem<DK, DV>;
    constexpr int LDK = SM::LDK, LDX = SM::LDX;
    extern __shared__ float sm[];
    float* Kb = sm;                  // [C][LDK] diag(beta) K
    float* Kw = Kb + C * LDK;        // [C][LDK] D (.) K
    float* X = Kw + C * LDK;         // [C][LDX] diag(beta) V, then Q
    float* As = X + C * LDX;         // [C][LDC] strict_tril(Kb Kw^T)
    float* Ts = As + C * LDC;        // [C][LDC] (I + A)^{-1}
    float* bs = Ts + C * LDC;        // [C] beta

    const int tid = threadIdx.x;
    const size_t cid = blockIdx.x;                 // unit * NC + chunk
    const int unit = (int)(cid / NC), c = (int)(cid % NC), b = unit / H, h = unit % H;
    const int c0 = c * C, Tc = min(C, T - c0);
    const float* d_all = ws + L.d_all / sizeof(float);
    float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
    float* t_g = ws + L.tinv / sizeof(float) + cid * C * C;
    float* w_g = ws + L.w / sizeof(float) + cid * C * DK;
    float* u_g = ws + L.u0 / sizeof(float) + cid * C * DV;
    float* p_g = ws + L.p / sizeof(float) + cid * C * C;

    if (tid < C) bs[tid] = ld_or0(beta, ((size_t)b * T + c0 + tid) * H + h, tid < Tc);
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int t = idx / DK, i = idx % DK;
        const bool ok = t < Tc;
        const size_t tok = ((size_t)b * T + c0 + t) * H + h;
        const float kv = ld_or0(k, tok * DK + i, ok);
        const float w = ok ? d_all[tok * DK + i] * kv : 0.f;
        Kb[t * LDK + i] = bs[t] * kv;
        Kw[t * LDK + i] = w;
        kw_g[idx] = w;
    }
    for (int idx = tid; idx < C * DV; idx += NTHR) {
        const int t = idx / DV, j = idx % DV;
        X[t * LDX + j] = bs[t] * ld_or0(v, (((size_t)b * T + c0 + t) * H + h) * DV + j, t < Tc);
    }
    __syncthreads();
    cta_gemm<SPLIT>(C, C, DK, Mat{Kb, LDK, 1}, Mat{Kw, 1, LDK},
                    [&](int m, int n, float x) { As[m * LDC + n] = n < m ? x : 0.f; });
    __syncthreads();
    {   // (I + A) T = I by forward substitution: column j on 4 threads that split the inner sum
        const int j = tid >> 2, part = tid & 3;
        for (int i = 0; i < C; ++i) {
            float s = 0.f;
            for (int l = j + part; l < i; l += 4) s = fmaf(As[i * LDC + l], Ts[l * LDC + j], s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            __syncwarp();
            if (part == 0) Ts[i * LDC + j] = (i < j) ? 0.f : (i == j ? 1.f : -s);
            __syncwarp();
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NTHR) t_g[idx] = Ts[(idx / C) * LDC + idx % C];
    cta_gemm<SPLIT>(C, DK, C, Mat{Ts, LDC, 1}, Mat{Kb, LDK, 1},
                    [&](int m, int n, float x) { w_g[m * DK + n] = x; });
    cta_gemm<SPLIT>(C, DV, C, Mat{Ts, LDC, 1}, Mat{X, LDX, 1},
                    [&](int m, int n, float x) { u_g[m * DV + n] = x; });
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int t = idx / DK, i = idx % DK;
        X[t * LDX + i] = ld_or0(q, (((size_t)b * T + c0 + t) * H + h) * DK + i, t < Tc);
    }
    __syncthreads();
    cta_gemm<SPLIT>(C, C, DK, Mat{X, LDX, 1}, Mat{Kw, 1, LDK},
                    [&](int m, int n, float x) { p_g[m * C + n] = n <= m ? x : 0.f; });
}

// ---------------------------------------------------------------------------
// Forward state pass for DVT rows of S: S at every chunk start (ckS) and Vn.
template <int DK, int DVT>
struct StateSmem {
    static constexpr int LDK = DK + 4, LDT = DVT + 4;
    static constexpr size_t kFwdBytes = sizeof(float) * (size_t)(DVT * LDK + 2 * C * LDK + C * LDT);
    static constexpr size_t kBwdBytes = sizeof(float) * (size_t)(DVT * LDK + C * LDC + 2 * C * LDT + 2 * C * LDK);
};

template <int DK, int DV, int DVT, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_state_f_kernel(const float* __restrict__ S0, float* __restrict__ ws, Layout L, int NC)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    using SM = StateSmem<DK, DVT>;
    constexpr int LDK = SM::LDK, LDT = SM::LDT, NTILE = DV / DVT;
    extern __shared__ float sm[];
    float* Ss = sm;                  // [DVT][LDK] rows v0 .. v0 + DVT - 1 of S
    float* Ws = Ss + DVT * LDK;      // [C][LDK] W
    float* Kws = Ws + C * LDK;       // [C][LDK] Kw
    float* Vs = Kws + C * LDK;       // [C][LDT] U0, then Vn (columns of the tile)

    const int tid = threadIdx.x;
    const int unit = blockIdx.x / NTILE, v0 = (blockIdx.x % NTILE) * DVT;
    for (int idx = tid; idx < DVT * DK; idx += NTHR) {
        const int row = idx / DK, i = idx % DK;
        Ss[row * LDK + i] = S0 ? S0[((size_t)unit * DV + v0 + row) * DK + i] : 0.f;
    }
    for (int c = 0; c < NC; ++c) {
        const size_t cid = (size_t)unit * NC + c;
        const float* w_g = ws + L.w / sizeof(float) + cid * C * DK;
        const float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
        const float* u_g = ws + L.u0 / sizeof(float) + cid * C * DV;
        float* s_g = ws + L.ckS / sizeof(float) + cid * DV * DK;
        float* vn_g = ws + L.vn / sizeof(float) + cid * C * DV;
        __syncthreads();
        for (int idx = tid; idx < DVT * DK; idx += NTHR) {
            const int row = idx / DK, i = idx % DK;
            s_g[(size_t)(v0 + row) * DK + i] = Ss[row * LDK + i];
        }
        for (int idx = tid; idx < C * DK; idx += NTHR) {
            const int t = idx / DK, i = idx % DK;
            Ws[t * LDK + i] = w_g[idx];
            Kws[t * LDK + i] = kw_g[idx];
        }
        for (int idx = tid; idx < C * DVT; idx += NTHR) {
            const int t = idx / DVT, j = idx % DVT;
            Vs[t * LDT + j] = u_g[t * DV + v0 + j];
        }
        __syncthreads();
        cta_gemm<SPLIT>(C, DVT, DK, Mat{Ws, LDK, 1}, Mat{Ss, 1, LDK}, [&](int m, int n, float x) {
            const float vn = Vs[m * LDT + n] - x;
            Vs[m * LDT + n] = vn;
            vn_g[m * DV + v0 + n] = vn;
        });
        __syncthreads();
        cta_gemm<SPLIT>(DVT, DK, C, Mat{Vs, 1, LDT}, Mat{Kws, LDK, 1},
                        [&](int m, int n, float x) { Ss[m * LDK + n] += x; });
    }
}

// Reverse state pass for DVT rows of dS: dS' at every chunk end (ckdS), dVn, and dS0.
template <int DK, int DV, int DVT, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_state_b_kernel(const Tin* __restrict__ dout, const Tin* __restrict__ q, const float* __restrict__ dS_final,
                   float* __restrict__ dS0, float* __restrict__ ws, Layout L, int B, int T, int H, int NC)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    using SM = StateSmem<DK, DVT>;
    constexpr int LDK = SM::LDK, LDT = SM::LDT, NTILE = DV / DVT;
    extern __shared__ float sm[];
    float* dSs = sm;                 // [DVT][LDK] rows v0 .. of dS
    float* Ps = dSs + DVT * LDK;     // [C][LDC] P
    float* dOs = Ps + C * LDC;       // [C][LDT] dO (columns of the tile)
    float* dVs = dOs + C * LDT;      // [C][LDT] -dVn
    float* B1 = dVs + C * LDT;       // [C][LDK] Kw, then W
    float* B2 = B1 + C * LDK;        // [C][LDK] Q

    const int tid = threadIdx.x;
    const int unit = blockIdx.x / NTILE, v0 = (blockIdx.x % NTILE) * DVT, b = unit / H, h = unit % H;
    for (int idx = tid; idx < DVT * DK; idx += NTHR) {
        const int row = idx / DK, i = idx % DK;
        dSs[row * LDK + i] = dS_final ? dS_final[((size_t)unit * DV + v0 + row) * DK + i] : 0.f;
    }
    for (int c = NC - 1; c >= 0; --c) {
        const size_t cid = (size_t)unit * NC + c;
        const int c0 = c * C, Tc = min(C, T - c0);
        const float* p_g = ws + L.p / sizeof(float) + cid * C * C;
        const float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
        const float* w_g = ws + L.w / sizeof(float) + cid * C * DK;
        float* ds_g = ws + L.ckdS / sizeof(float) + cid * DV * DK;
        float* dvn_g = ws + L.dvn / sizeof(float) + cid * C * DV;
        __syncthreads();
        for (int idx = tid; idx < DVT * DK; idx += NTHR) {
            const int row = idx / DK, i = idx % DK;
            ds_g[(size_t)(v0 + row) * DK + i] = dSs[row * LDK + i];
        }
        for (int idx = tid; idx < C * C; idx += NTHR) Ps[(idx / C) * LDC + idx % C] = p_g[idx];
        for (int idx = tid; idx < C * DVT; idx += NTHR) {
            const int t = idx / DVT, j = idx % DVT;
            dOs[t * LDT + j] = ld_or0(dout, (((size_t)b * T + c0 + t) * H + h) * DV + v0 + j, t < Tc);
        }
        for (int idx = tid; idx < C * DK; idx += NTHR) {
            const int t = idx / DK, i = idx % DK;
            B1[t * LDK + i] = kw_g[idx];
            B2[t * LDK + i] = ld_or0(q, (((size_t)b * T + c0 + t) * H + h) * DK + i, t < Tc);
        }
        __syncthreads();
        // dVn = P^T dO + Kw dS'^T
        cta_gemm2<SPLIT>(C, DVT, C, Mat{Ps, 1, LDC}, Mat{dOs, LDT, 1}, DK, Mat{B1, LDK, 1}, Mat{dSs, 1, LDK},
                         [&](int m, int n, float x) {
                             dVs[m * LDT + n] = -x;
                             dvn_g[m * DV + v0 + n] = x;
                         });
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += NTHR) B1[(idx / DK) * LDK + idx % DK] = w_g[idx];
        __syncthreads();
        // dS = dS' + dO^T Q + (-dVn)^T W
        cta_gemm2<SPLIT>(DVT, DK, C, Mat{dOs, 1, LDT}, Mat{B2, LDK, 1}, C, Mat{dVs, 1, LDT}, Mat{B1, LDK, 1},
                         [&](int m, int n, float x) { dSs[m * LDK + n] += x; });
    }
    __syncthreads();
    if (dS0)
        for (int idx = tid; idx < DVT * DK; idx += NTHR) {
            const int row = idx / DK, i = idx % DK;
            dS0[((size_t)unit * DV + v0 + row) * DK + i] = dSs[row * LDK + i];
        }
}

// ---------------------------------------------------------------------------
// Per chunk, over the dv tiles in turn: dP, dQ, dV, dW, dT (V part), the
// dv-summed part of dKw (Vn dS' + dP^T Q) and of dbeta (rowdot(T^T dVn, V)).
// dQ, dKw and dW stay in registers: warp w owns rows 16 (w % 4) .. + 15 and
// columns (DK / 2) (w / 4) .. + DK / 2 - 1 of each.
constexpr int J = 32;           // dv tile of the gradient kernel
constexpr int LDJ = J + 4;

template <int DK>
struct GradSmem {
    static constexpr int LDK = DK + 4;
    static constexpr size_t kABytes =
        sizeof(float) * (size_t)(2 * C * LDK + 3 * C * LDC + 4 * C * LDJ + 2 * J * LDK + 2 * C);
    static constexpr size_t kBBytes = sizeof(float) * (size_t)(3 * C * LDK + 4 * C * LDC + 2 * C);
};

template <int NT, typename F>
__device__ __forceinline__ void frag_apply(float (&acc)[NT][4], int m0, int n0, int lane, F f) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) f(m0 + g + 8 * (e >> 1), n0 + 8 * j + 2 * t + (e & 1), acc[j][e]);
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_grads_a_kernel(const Tin* __restrict__ q, const Tin* __restrict__ v, const Tin* __restrict__ beta,
                   const Tin* __restrict__ dout, Tin* __restrict__ dq, Tin* __restrict__ dv,
                   float* __restrict__ ws, Layout L, int B, int T, int H, int NC)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    constexpr int LDK = GradSmem<DK>::LDK, NT = DK / 16;
    extern __shared__ float sm[];
    float* Qs = sm;                  // [C][LDK] Q
    float* Kws = Qs + C * LDK;       // [C][LDK] Kw
    float* Ts = Kws + C * LDK;       // [C][LDC] T
    float* dPs = Ts + C * LDC;       // [C][LDC] dP of the current tile
    float* dTs = dPs + C * LDC;      // [C][LDC] dT (V part), summed over the tiles
    float* dOs = dTs + C * LDC;      // [C][LDJ] dO columns of the tile
    float* Vns = dOs + C * LDJ;      // [C][LDJ] Vn
    float* dVns = Vns + C * LDJ;     // [C][LDJ] dVn
    float* Vs = dVns + C * LDJ;      // [C][LDJ] V
    float* SJ = Vs + C * LDJ;        // [J][LDK] rows of S (chunk start)
    float* dSJ = SJ + J * LDK;       // [J][LDK] rows of dS' (chunk end)
    float* bs = dSJ + J * LDK;       // [C] beta
    float* dbs = bs + C;             // [C] dbeta (this kernel's part)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t cid = blockIdx.x;
    const int unit = (int)(cid / NC), c = (int)(cid % NC), b = unit / H, h = unit % H;
    const int c0 = c * C, Tc = min(C, T - c0);
    const float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
    const float* t_g = ws + L.tinv / sizeof(float) + cid * C * C;
    const float* vn_g = ws + L.vn / sizeof(float) + cid * C * DV;
    const float* dvn_g = ws + L.dvn / sizeof(float) + cid * C * DV;
    const float* s_g = ws + L.ckS / sizeof(float) + cid * DV * DK;
    const float* ds_g = ws + L.ckdS / sizeof(float) + cid * DV * DK;
    float* dkwa_g = ws + L.dkwa / sizeof(float) + cid * C * DK;
    float* dw_g = ws + L.dw / sizeof(float) + cid * C * DK;
    float* dt_g = ws + L.dt / sizeof(float) + cid * C * C;
    float* dba_g = ws + L.dba / sizeof(float) + cid * C;
    auto tok = [&](int t) { return ((size_t)b * T + c0 + t) * H + h; };

    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int t = idx / DK, i = idx % DK;
        Qs[t * LDK + i] = ld_or0(q, tok(t) * DK + i, t < Tc);
        Kws[t * LDK + i] = kw_g[idx];
    }
    for (int idx = tid; idx < C * C; idx += NTHR) {
        Ts[(idx / C) * LDC + idx % C] = t_g[idx];
        dTs[(idx / C) * LDC + idx % C] = 0.f;
    }
    if (tid < C) {
        bs[tid] = ld_or0(beta, tok(tid), tid < Tc);
        dbs[tid] = 0.f;
    }

    const int m0 = 16 * (warp & 3), n0 = (DK / 2) * (warp >> 2);
    float aQ[NT][4], aKw[NT][4], aW[NT][4];
    frag_zero(aQ);
    frag_zero(aKw);
    frag_zero(aW);
    for (int v0 = 0; v0 < DV; v0 += J) {
        __syncthreads();
        for (int idx = tid; idx < C * J; idx += NTHR) {
            const int t = idx / J, j = idx % J;
            dOs[t * LDJ + j] = ld_or0(dout, tok(t) * DV + v0 + j, t < Tc);
            Vs[t * LDJ + j] = ld_or0(v, tok(t) * DV + v0 + j, t < Tc);
            Vns[t * LDJ + j] = vn_g[t * DV + v0 + j];
            dVns[t * LDJ + j] = dvn_g[t * DV + v0 + j];
        }
        for (int idx = tid; idx < J * DK; idx += NTHR) {
            const int row = idx / DK, i = idx % DK;
            SJ[row * LDK + i] = s_g[(size_t)(v0 + row) * DK + i];
            dSJ[row * LDK + i] = ds_g[(size_t)(v0 + row) * DK + i];
        }
        __syncthreads();
        // dP = tril(dO Vn^T) for this tile
        cta_gemm<SPLIT>(C, C, J, Mat{dOs, LDJ, 1}, Mat{Vns, 1, LDJ},
                        [&](int m, int n, float x) { dPs[m * LDC + n] = n <= m ? x : 0.f; });
        // dT += (dVn V^T) diag(beta)
        cta_gemm<SPLIT>(C, C, J, Mat{dVns, LDJ, 1}, Mat{Vs, 1, LDJ},
                        [&](int m, int n, float x) { dTs[m * LDC + n] += bs[n] * x; });
        // dV = diag(beta) T^T dVn;  dbeta += rowdot(T^T dVn, V)
        cta_gemm<SPLIT>(C, J, C, Mat{Ts, 1, LDC}, Mat{dVns, LDJ, 1}, [&](int m, int n, float x) {
            if (m < Tc) dv[tok(m) * DV + v0 + n] = from_f32<Tin>(bs[m] * x);
            atomicAdd(&dbs[m], x * Vs[m * LDJ + n]);
        });
        __syncthreads();
        warp_mma<NT, SPLIT>(aQ, Mat{dOs, LDJ, 1}, Mat{SJ, LDK, 1}, m0, n0, J, lane);     // dO S
        warp_mma<NT, SPLIT>(aQ, Mat{dPs, LDC, 1}, Mat{Kws, LDK, 1}, m0, n0, C, lane);    // dP Kw
        warp_mma<NT, SPLIT>(aKw, Mat{Vns, LDJ, 1}, Mat{dSJ, LDK, 1}, m0, n0, J, lane);   // Vn dS'
        warp_mma<NT, SPLIT>(aKw, Mat{dPs, 1, LDC}, Mat{Qs, LDK, 1}, m0, n0, C, lane);    // dP^T Q
        warp_mma<NT, SPLIT>(aW, Mat{dVns, LDJ, 1}, Mat{SJ, LDK, 1}, m0, n0, J, lane);    // dVn S
    }
    frag_each(aQ, m0, n0, lane, [&](int m, int n, float x) {
        if (m < Tc) dq[tok(m) * DK + n] = from_f32<Tin>(x);
    });
    frag_each(aKw, m0, n0, lane, [&](int m, int n, float x) { dkwa_g[m * DK + n] = x; });
    frag_each(aW, m0, n0, lane, [&](int m, int n, float x) { dw_g[m * DK + n] = -x; });
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NTHR) dt_g[idx] = dTs[(idx / C) * LDC + idx % C];
    if (tid < C) dba_g[tid] = dbs[tid];
}

// Per chunk: dT += (dW K^T) diag(beta), dA = -strict_tril(T^T dT T^T), the
// dbeta terms of T^T dW and of dA, dK, the rest of dKw, then dD = dKw (.) K and
// the chunk part of dk, dK + dKw (.) D.
template <int DK, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_grads_b_kernel(const Tin* __restrict__ k, const Tin* __restrict__ beta, float* __restrict__ ws, Layout L,
                   int B, int T, int H, int NC)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    constexpr int LDK = GradSmem<DK>::LDK, NT = DK / 16;
    extern __shared__ float sm[];
    float* Ks = sm;                  // [C][LDK] K
    float* Kws = Ks + C * LDK;       // [C][LDK] Kw
    float* dWs = Kws + C * LDK;      // [C][LDK] dW
    float* Ts = dWs + C * LDK;       // [C][LDC] T
    float* dTs = Ts + C * LDC;       // [C][LDC] dT, then diag(beta) dA
    float* Xs = dTs + C * LDC;       // [C][LDC] dT T^T
    float* Gs = Xs + C * LDC;        // [C][LDC] K Kw^T
    float* bs = Gs + C * LDC;        // [C] beta
    float* dbs = bs + C;             // [C] dbeta (chunk part)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t cid = blockIdx.x;
    const int unit = (int)(cid / NC), c = (int)(cid % NC), b = unit / H, h = unit % H;
    const int c0 = c * C, Tc = min(C, T - c0);
    const float* d_all = ws + L.d_all / sizeof(float);
    const float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
    const float* t_g = ws + L.tinv / sizeof(float) + cid * C * C;
    const float* dkwa_g = ws + L.dkwa / sizeof(float) + cid * C * DK;
    const float* dw_g = ws + L.dw / sizeof(float) + cid * C * DK;
    const float* dt_g = ws + L.dt / sizeof(float) + cid * C * C;
    const float* dba_g = ws + L.dba / sizeof(float) + cid * C;
    float* dd_g = ws + L.dd / sizeof(float) + cid * C * DK;
    float* dkp_g = ws + L.dkp / sizeof(float) + cid * C * DK;
    float* dbp_g = ws + L.dbp / sizeof(float) + cid * C;
    auto tok = [&](int t) { return ((size_t)b * T + c0 + t) * H + h; };

    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int t = idx / DK, i = idx % DK;
        Ks[t * LDK + i] = ld_or0(k, tok(t) * DK + i, t < Tc);
        Kws[t * LDK + i] = kw_g[idx];
        dWs[t * LDK + i] = dw_g[idx];
    }
    for (int idx = tid; idx < C * C; idx += NTHR) {
        Ts[(idx / C) * LDC + idx % C] = t_g[idx];
        dTs[(idx / C) * LDC + idx % C] = dt_g[idx];
    }
    if (tid < C) {
        bs[tid] = ld_or0(beta, tok(tid), tid < Tc);
        dbs[tid] = dba_g[tid];
    }
    __syncthreads();
    cta_gemm<SPLIT>(C, C, DK, Mat{dWs, LDK, 1}, Mat{Ks, 1, LDK},
                    [&](int m, int n, float x) { dTs[m * LDC + n] += bs[n] * x; });
    cta_gemm<SPLIT>(C, C, DK, Mat{Ks, LDK, 1}, Mat{Kws, 1, LDK},
                    [&](int m, int n, float x) { Gs[m * LDC + n] = x; });
    __syncthreads();
    cta_gemm<SPLIT>(C, C, C, Mat{dTs, LDC, 1}, Mat{Ts, 1, LDC},
                    [&](int m, int n, float x) { Xs[m * LDC + n] = x; });
    __syncthreads();
    cta_gemm<SPLIT>(C, C, C, Mat{Ts, 1, LDC}, Mat{Xs, LDC, 1}, [&](int m, int n, float x) {
        float ab = 0.f;
        if (n < m) {
            const float a = -x;                      // dA (strictly lower)
            atomicAdd(&dbs[m], a * Gs[m * LDC + n]);
            ab = bs[m] * a;
        }
        dTs[m * LDC + n] = ab;                       // diag(beta) dA
    });
    __syncthreads();
    const int m0 = 16 * (warp & 3), n0 = (DK / 2) * (warp >> 2);
    float aK[NT][4], aKw[NT][4];
    frag_zero(aK);
    warp_mma<NT, SPLIT>(aK, Mat{Ts, 1, LDC}, Mat{dWs, LDK, 1}, m0, n0, C, lane);        // T^T dW
    frag_apply(aK, m0, n0, lane, [&](int m, int n, float& x) {
        atomicAdd(&dbs[m], x * Ks[m * LDK + n]);
        x *= bs[m];
    });
    warp_mma<NT, SPLIT>(aK, Mat{dTs, LDC, 1}, Mat{Kws, LDK, 1}, m0, n0, C, lane);       // + dAb Kw
    frag_apply(aKw, m0, n0, lane, [&](int m, int n, float& x) { x = dkwa_g[m * DK + n]; });
    warp_mma<NT, SPLIT>(aKw, Mat{dTs, 1, LDC}, Mat{Ks, LDK, 1}, m0, n0, C, lane);       // + dAb^T K
    #pragma unroll
    for (int jj = 0; jj < NT; ++jj)
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = m0 + (lane >> 2) + 8 * (e >> 1), n = n0 + 8 * jj + 2 * (lane & 3) + (e & 1);
            const float dkw = aKw[jj][e];
            const float dval = m < Tc ? d_all[tok(m) * DK + n] : 0.f;
            dd_g[m * DK + n] = dkw * Ks[m * LDK + n];
            dkp_g[m * DK + n] = aK[jj][e] + dkw * dval;
        }
    __syncthreads();
    if (tid < C) dbp_g[tid] = dbs[tid];
}

// ---------------------------------------------------------------------------
// Reverse of the d recurrence, token by token: one warp per unit, lane l owns
// features l * DK / 32 ..; writes the final dk, dbeta, dr and dd0.
template <int DK, typename Tin>
__global__ void __launch_bounds__(128)
bwd_dchain_kernel(const Tin* __restrict__ k, const Tin* __restrict__ beta, const Tin* __restrict__ r,
                  const float* __restrict__ d0, const float* __restrict__ dd_final,
                  Tin* __restrict__ dk, Tin* __restrict__ dbeta, Tin* __restrict__ dr, float* __restrict__ dd0,
                  const float* __restrict__ ws, Layout L, int B, int T, int H, int NC, float eta, int anchor)
{
    constexpr int PER = DK / 32;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= B * H) return;
    const int b = unit / H, h = unit % H;
    const float* d_all = ws + L.d_all / sizeof(float);
    const float* dd_g = ws + L.dd / sizeof(float);
    const float* dkp_g = ws + L.dkp / sizeof(float);
    const float* dbp_g = ws + L.dbp / sizeof(float);

    float lam[PER], anc[PER], dda[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int f = lane * PER + i;
        lam[i] = dd_final ? dd_final[(size_t)unit * DK + f] : 0.f;
        anc[i] = anchor ? (d0 ? d0[(size_t)unit * DK + f] : 1.f) : 0.f;
        dda[i] = 0.f;
    }
    for (int t = T - 1; t >= 0; --t) {
        const size_t tok = ((size_t)b * T + t) * H + h;
        const size_t crow = ((size_t)unit * NC + t / C) * C + t % C;   // chunk-block row
        float kk[PER], d[PER], dD[PER], dkp[PER], a[PER];
        VecIO<PER, Tin>::load(k + tok * DK + lane * PER, kk);
        VecIO<PER, float>::load(d_all + tok * DK + lane * PER, d);
        VecIO<PER, float>::load(dd_g + crow * DK + lane * PER, dD);
        VecIO<PER, float>::load(dkp_g + crow * DK + lane * PER, dkp);
        const float bt = to_f32(beta[tok]), rt = r ? to_f32(r[tok]) : 1.f;
        float n = 0.f, s = 0.f, dx = 0.f, drv = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            a[i] = kk[i] * kk[i];
            n += a[i];
            s += d[i] * a[i];
            dx += a[i] * lam[i];
            drv += (d[i] - anc[i]) * lam[i];
        }
        n = warp_sum(n);
        s = warp_sum(s);
        dx = warp_sum(dx);
        drv = warp_sum(drv);
        float db = dbp_g[crow], x = 0.f, ds = 0.f, dn = 0.f;
        if (n > 0.f) {
            x = eta * bt * (1.f - bt * s) / n;
            db += dx * eta * (1.f - 2.f * bt * s) / n;
            ds = -dx * eta * bt * bt / n;
            dn = -dx * x / n;
        }
        float gk[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            gk[i] = dkp[i] + 2.f * kk[i] * (x * lam[i] + ds * d[i] + dn);
            if (anchor) dda[i] += (1.f - rt) * lam[i];
            lam[i] = rt * lam[i] + dD[i] + ds * a[i];
        }
        VecIO<PER, Tin>::store(dk + tok * DK + lane * PER, gk);
        if (lane == 0) {
            dbeta[tok] = from_f32<Tin>(db);
            if (r && dr) dr[tok] = from_f32<Tin>(drv);
        }
    }
    if (dd0) {
#pragma unroll
        for (int i = 0; i < PER; ++i) dd0[(size_t)unit * DK + lane * PER + i] = lam[i] + dda[i];
    }
}

}  // namespace bwd
}  // namespace osdn
