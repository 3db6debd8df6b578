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
//   bwd_dtraj   d_t for every token (token-serial: one CTA per unit, a chain warp
//               and three warps that stage the next slab of tokens);
//   bwd_prep    per chunk: Kw, T, W, U0, P (gated: and log2 gamma);
//   bwd_state_f per (unit, dv tile): S at every chunk start, Vn;
//   bwd_state_b per (unit, dv tile), chunks in reverse: dS' at every chunk end, dVn, dS0;
//   bwd_grads   per chunk: dQ, dV (dv tiles in turn), then dA, dK, dKw, dD and the
//               chunk part of dbeta (gated: and dalpha);
//   bwd_dchain  token-serial reverse of the d recurrence, staged as bwd_dtraj:
//               dk, dbeta, dr, dd0.
// Gated OSDN (alpha given; the state decayed by alpha_t before token t's write):
// with gamma the cumulative gate within the chunk, R_tj = gamma_t / gamma_j and
// rho_j = gamma_C / gamma_j (every factor at most 1, taken as 2 to differences of
// the in-chunk cumulative log2 alpha, each term clamped at -120, as in the forward),
//   forward:  A = strict_tril(Kb Kw^T) (.) R, W = T diag(gamma) Kb, P = tril(Q Kw^T) (.) R,
//             O = diag(gamma) Q S^T + P Vn, S' = gamma_C S + Vn^T diag(rho) Kw;
//   backward: dVn = P^T dO + diag(rho) Kw dS'^T, dS = gamma_C dS' + dO^T diag(gamma) Q - dVn^T W,
//             dQ = diag(gamma) dO S + (dP (.) R) Kw, dKw = diag(rho) Vn dS' + (dP (.) R)^T Q + ...,
//             dT = dW (diag(gamma) Kb)^T + ..., dA (.) R in place of dA downstream,
//             dK = diag(beta gamma) T^T dW + ..., dbeta gets gamma (.) rowdot(T^T dW, K),
//   and the adjoint of G = ln gamma,
//     dG_t = gamma_t <(dO S)_t, Q_t> + gamma_t beta_t <(T^T dW)_t, K_t> + sum_j X_tj - sum_j X_jt
//            - Y_t + [t = last] (gamma_C <dS', S> + sum_j Y_j),
//     X = dA (.) diag(beta) K Kw^T (.) R + dP (.) P,  Y_j = rho_j <(Vn dS')_j, Kw_j>,
//   gives dalpha_m = (sum_{t >= m} dG_t) / alpha_m (chunk-local: gamma restarts every chunk).
// Rows of S are independent given the chunk matrices, so the two state passes
// split dv into tiles with no exchange.  The contractions run on mma.sync
// m16n8k8 tf32 with fp32 accumulation; for fp32 inputs every product uses the
// three-pass split a = a_hi + a_lo (a_hi b_hi + a_hi b_lo + a_lo b_hi), which
// keeps fp32 accuracy.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "tril_inv.cuh"

namespace osdn {
namespace bwd {

constexpr int C = 64;         // chunk length
constexpr int NTHR = 512;     // threads of the per-chunk and per-tile kernels (16 warps)
constexpr int LDC = C + 4;    // row stride of C x C tiles (68 = 4 mod 32: conflict-free fragments)

// X(i, j) = p[i * S0 + j * S1], fp32 in shared memory; compile-time strides keep every
// fragment load a single instruction with an immediate offset.
template <int S0, int S1>
struct Mat {
    const float* p;
    __device__ __forceinline__ float operator()(int i, int j) const { return p[i * S0 + j * S1]; }
    // X(i, j) and X(i, j + 1), one 8-byte load when the second index is contiguous (j even)
    __device__ __forceinline__ float2 pair_j(int i, int j) const {
        if constexpr (S1 == 1) return *reinterpret_cast<const float2*>(p + i * S0 + j);
        else return make_float2(p[i * S0 + j * S1], p[i * S0 + (j + 1) * S1]);
    }
    // X(i, j) and X(i + 1, j), one 8-byte load when the first index is contiguous (i even)
    __device__ __forceinline__ float2 pair_i(int i, int j) const {
        if constexpr (S0 == 1) return *reinterpret_cast<const float2*>(p + i + j * S1);
        else return make_float2(p[i * S0 + j * S1], p[(i + 1) * S0 + j * S1]);
    }
};

__device__ __forceinline__ void mma8(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// c += a b for one m16n8k8 step. The fp32 bit patterns go to the tensor core as they
// are: it reads the upper 19 bits (tf32 truncation, one tf32 ulp at most). SPLIT: a =
// a_hi + a_lo with a_hi the truncated value and a_lo = a - a_hi (exact in fp32), and
// c += a_lo b_hi + a_hi b_lo + a_hi b_hi, which recovers fp32 accuracy.
template <bool SPLIT>
__device__ __forceinline__ void mma_step(float (&c)[4], const float (&a)[4], const float (&b)[2]) {
    uint32_t ah[4], bh[2];
    if (SPLIT) {
        uint32_t al[4], bl[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ah[i] = __float_as_uint(a[i]) & 0xffffe000u;
            al[i] = __float_as_uint(a[i] - __uint_as_float(ah[i]));
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            bh[i] = __float_as_uint(b[i]) & 0xffffe000u;
            bl[i] = __float_as_uint(b[i] - __uint_as_float(bh[i]));
        }
        mma8(c, al, bh);
        mma8(c, ah, bl);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) ah[i] = __float_as_uint(a[i]);
#pragma unroll
        for (int i = 0; i < 2; ++i) bh[i] = __float_as_uint(b[i]);
    }
    mma8(c, ah, bh);
}

// One warp: acc[j] += sum_{k < K} A(m0 + ., k) B(k, n0 + 8 j + .) for a 16 x 8 NT tile.
// Fragment element e of acc[j] sits at row m0 + g + 8 (e >> 1), column n0 + 8 j + 2 t + (e & 1),
// with g = lane / 4, t = lane % 4. Within each step of 8, the instruction's k slots t and t + 4
// carry k0 + 2t and k0 + 2t + 1 in both operands (a permutation of the summation index), so a
// lane's two k values are adjacent and load as one pair where the layout allows.
template <int NT, bool SPLIT, class MA, class MB>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], MA A, MB B, int m0, int n0, int K, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 4
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float2 lo = A.pair_j(m0 + g, k0 + 2 * t), hi = A.pair_j(m0 + g + 8, k0 + 2 * t);
        const float a[4] = {lo.x, hi.x, lo.y, hi.y};
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const float2 bb = B.pair_i(k0 + 2 * t, n0 + 8 * j + g);
            const float b[2] = {bb.x, bb.y};
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

// Calls f(m, n, value) for every element a thread holds, or f(m, n, v_n, v_{n+1}) once per
// pair of adjacent columns (n even) when f takes two values, so that a store can be 8 bytes.
template <int NT, typename F>
__device__ __forceinline__ void frag_each(float (&acc)[NT][4], int m0, int n0, int lane, F f) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int m = m0 + g + 8 * hh, n = n0 + 8 * j + 2 * t;
            if constexpr (std::is_invocable_v<F, int, int, float, float>) {
                f(m, n, acc[j][2 * hh], acc[j][2 * hh + 1]);
            } else {
                f(m, n, acc[j][2 * hh]);
                f(m, n + 1, acc[j][2 * hh + 1]);
            }
        }
}

__device__ __forceinline__ void store2(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
__device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void add2(float* p, float a, float b) {
    float2 v = *reinterpret_cast<float2*>(p);
    v.x += a;
    v.y += b;
    *reinterpret_cast<float2*>(p) = v;
}

// The CTA computes the M x N product sum_k A(m, k) B(k, n) (plus, for the two-term
// form, a second product over K2) in warp tiles of 16 x 8 NT taken round-robin, and
// calls epi(m, n, value) once per output element on the thread that holds it.
template <int NT, bool SPLIT, class MA1, class MB1, class MA2, class MB2, typename Epi>
__device__ __forceinline__ void cta_gemm_nt(int M, int N, int K1, MA1 A1, MB1 B1, int K2, MA2 A2, MB2 B2, Epi epi) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tn = N / (8 * NT), tiles = (M / 16) * tn;
    for (int tile = warp; tile < tiles; tile += nw) {
        const int m0 = (tile / tn) * 16, n0 = (tile % tn) * 8 * NT;
        float acc[NT][4];
        frag_zero(acc);
        warp_mma<NT, SPLIT>(acc, A1, B1, m0, n0, K1, lane);
        if (K2 > 0) warp_mma<NT, SPLIT>(acc, A2, B2, m0, n0, K2, lane);
        frag_each(acc, m0, n0, lane, epi);
    }
}

// The widest of 16 x 32, 16 x 16 and 16 x 8 tiles that still gives every warp one.
template <bool SPLIT, class MA1, class MB1, class MA2, class MB2, typename Epi>
__device__ __forceinline__ void cta_gemm2(int M, int N, int K1, MA1 A1, MB1 B1, int K2, MA2 A2, MB2 B2, Epi epi) {
    const int nw = (int)(blockDim.x >> 5);
    if ((M / 16) * (N / 32) >= nw) cta_gemm_nt<4, SPLIT>(M, N, K1, A1, B1, K2, A2, B2, epi);
    else if ((M / 16) * (N / 16) >= nw) cta_gemm_nt<2, SPLIT>(M, N, K1, A1, B1, K2, A2, B2, epi);
    else cta_gemm_nt<1, SPLIT>(M, N, K1, A1, B1, K2, A2, B2, epi);
}

template <bool SPLIT, class MA, class MB, typename Epi>
__device__ __forceinline__ void cta_gemm(int M, int N, int K, MA A, MB B, Epi epi) {
    cta_gemm2<SPLIT>(M, N, K, A, B, 0, A, B, epi);
}

// L2 prefetch hint for rows [0, rows) of row_bytes bytes each, stride_bytes apart from p.
__device__ __forceinline__ void prefetch_rows(const void* p, size_t stride_bytes, int rows, int row_bytes) {
    const int lines = (row_bytes + 127) / 128, n = rows * lines;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const char* a = static_cast<const char*>(p) + (size_t)(i / lines) * stride_bytes + (size_t)(i % lines) * 128;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
}

// Workspace layout of one backward call (fp32 regions, 256-byte aligned).
struct Layout {
    size_t d_all, kw, tinv, w, u0, p, ckS, ckdS, vn, dvn, dd, dkp, dbp, lg, total;
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
    L.dd = take(f * ch * C * DK);
    L.dkp = take(f * ch * C * DK);
    L.dbp = take(f * ch * C);
    L.lg = take(f * ch * C);   // gated: log2 gamma_t of every chunk
    L.total = o;
    return L;
}

template <typename Tin>
__device__ __forceinline__ float ld_or0(const Tin* p, size_t i, bool ok) { return ok ? to_f32(p[i]) : 0.f; }

// 2^x (the special-function unit; results below the normal range flush to 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Warp 0 of the CTA: gs[t] = sum_{m <= t} max(log2 alpha_m, -120) over the C tokens of a chunk
// (alpha = 1 past its Tc valid tokens), the in-chunk cumulative log2 gate of the forward.
template <typename Tin>
__device__ __forceinline__ void chunk_log2_gates(float* gs, const Tin* alpha, size_t tok0, size_t tstride, int Tc,
                                                 int lane, float* ls = nullptr) {
    static_assert(C == 64, "two tokens per lane");
    float l[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        l[e] = t < Tc ? fmaxf(log2f(to_f32(alpha[tok0 + t * tstride])), -120.f) : 0.f;
    }
    float x = l[0] + l[1];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    gs[2 * lane] = x - l[1];
    gs[2 * lane + 1] = x;
    if (ls) {   // and the clamped log2 alpha_t of every token
        ls[2 * lane] = l[0];
        ls[2 * lane + 1] = l[1];
    }
}

// 16-byte vector load of 4 fp32 or 8 bf16 values as fp32.
__device__ __forceinline__ void load16(const float* p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// The CTA copies a ROWS x COLS tile, dst[r * ldd + c] = src[r * lds + c] as fp32, with
// rows r >= valid set to zero and every element scaled by scale[r] when scale is given.
// COLS is a multiple of 16 / sizeof(Tsrc); src rows and dst rows are 16-byte aligned.
// Every thread issues all of its loads before its first shared-memory store, so the
// tile costs one memory round trip.
template <int ROWS, int COLS, typename Tsrc>
__device__ __forceinline__ void load_tile(float* dst, int ldd, const Tsrc* src, size_t lds, int valid,
                                          const float* scale = nullptr) {
    constexpr int V = 16 / sizeof(Tsrc), VPR = COLS / V, N = ROWS * VPR;
    constexpr int PER = (N + NTHR - 1) / NTHR;
    float x[PER][V];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int idx = threadIdx.x + u * NTHR, r = idx / VPR, c = (idx % VPR) * V;
        if (idx < N && r < valid) {
            load16(src + (size_t)r * lds + c, x[u]);
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i) x[u][i] = 0.f;
        }
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int idx = threadIdx.x + u * NTHR, r = idx / VPR, c = (idx % VPR) * V;
        if (idx < N) {
            const float sc = scale ? scale[r] : 1.f;
#pragma unroll
            for (int i = 0; i < V; i += 4)
                *reinterpret_cast<float4*>(dst + r * ldd + c + i) =
                    make_float4(sc * x[u][i], sc * x[u][i + 1], sc * x[u][i + 2], sc * x[u][i + 3]);
        }
    }
}

// Asynchronous copy (cp.async, 16 bytes per request) of a ROWS x COLS fp32 tile,
// dst[r * ldd + c] = src[r * lds + c]; rows r >= valid are zero-filled (no global read).
// Completes at cp_async_wait_all() followed by a CTA barrier.
__device__ __forceinline__ void cp_async16(float* dst, const float* src, bool fill) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(fill ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int ROWS, int COLS>
__device__ __forceinline__ void async_tile(float* dst, int ldd, const float* src, size_t lds, int valid = ROWS) {
    constexpr int VPR = COLS / 4, N = ROWS * VPR;
    for (int idx = threadIdx.x; idx < N; idx += NTHR) {
        const int r = idx / VPR, c = (idx % VPR) * 4;
        const bool ok = r < valid;
        cp_async16(dst + r * ldd + c, ok ? src + (size_t)r * lds + c : src, ok);
    }
}

// 16-byte stores of a ROWS x COLS fp32 tile from shared memory (row stride lds, rows
// 16-byte aligned) to global memory (row stride ldd).
template <int ROWS, int COLS>
__device__ __forceinline__ void store_rows(float* dst, size_t ldd, const float* src, int lds) {
    constexpr int VPR = COLS / 4, N = ROWS * VPR;
    for (int idx = threadIdx.x; idx < N; idx += NTHR) {
        const int r = idx / VPR, c = (idx % VPR) * 4;
        *reinterpret_cast<float4*>(dst + (size_t)r * ldd + c) = *reinterpret_cast<const float4*>(src + r * lds + c);
    }
}

// dst[r * ldd + c] = src[r * COLS + c] for a dense fp32 ROWS x COLS block (the workspace layout).
template <int ROWS, int COLS>
__device__ __forceinline__ void async_block(float* dst, int ldd, const float* src) {
    async_tile<ROWS, COLS>(dst, ldd, src, (size_t)COLS);
}

// ---------------------------------------------------------------------------
// The two token-serial kernels run one CTA of 128 threads per unit: warp 0
// carries the recurrence, warps 1-3 stage the next slab of SLAB tokens into
// shared memory meanwhile (double buffer), so no global load sits on the chain.
constexpr int SLAB = 32;
constexpr int SERIAL_THREADS = 128;

// Warp w of warps 1-3 takes rows w - 1, w + 2, ... of a slab; per row, lane l copies
// the l-th 16-byte piece of each staged row and the warp reduces what the chain needs.
constexpr int HELPERS = SERIAL_THREADS / 32 - 1;
static_assert(SLAB <= SERIAL_THREADS - 32, "one helper thread per token of a slab");

// Asynchronous copy of the lane-th 16-byte piece of a row (zero-filled when !ok); the
// helpers issue every piece of a slab before waiting once.
template <typename T>
__device__ __forceinline__ void stage_piece(T* dst, const T* src, int lane, int width, bool ok) {
    constexpr int V = 16 / sizeof(T);
    if (lane * V < width) {
        const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst + lane * V);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(ok ? src + lane * V : src),
                     "r"(ok ? 16 : 0)
                     : "memory");
    }
}

// Barrier over the three helper warps only (named barrier 1).
__device__ __forceinline__ void helpers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(SERIAL_THREADS - 32) : "memory");
}

// sum over the row's features of f(k_i, d_i) for the piece this lane staged
template <int DK, typename Tin>
__device__ __forceinline__ float k2_piece(const Tin* krow, int lane) {
    constexpr int V = 16 / sizeof(Tin);
    float acc = 0.f;
    if (lane * V < DK) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const float kv = to_f32(krow[lane * V + i]);
            acc = fmaf(kv, kv, acc);
        }
    }
    return acc;
}

template <int DK, typename Tin>
struct DtrajSmem {
    static constexpr size_t kBytes = 2 * (SLAB * DK * sizeof(Tin) + 3 * SLAB * sizeof(float));
};

// d_t (before the token's own update) for every token. Per token the helpers stage
// k and precompute c0 = eta beta / ||k||^2 and c1 = eta beta^2 / ||k||^2 (0 when k = 0),
// so that x = c0 - c1 <d, k^2> and the chain carries one reduction per token.
template <int DK, typename Tin>
__global__ void __launch_bounds__(SERIAL_THREADS, 1)
bwd_dtraj_kernel(const Tin* __restrict__ k, const Tin* __restrict__ beta, const Tin* __restrict__ r,
                 const float* __restrict__ d0, float* __restrict__ d_all, int B, int T, int H, float eta, int anchor)
{
    constexpr int PER = DK / 32;
    extern __shared__ __align__(16) unsigned char smraw[];
    Tin* ks = reinterpret_cast<Tin*>(smraw);                                        // [2][SLAB][DK]
    float* c0s = reinterpret_cast<float*>(smraw + 2 * SLAB * DK * sizeof(Tin));     // [2][SLAB]
    float* c1s = c0s + 2 * SLAB;                                                    // [2][SLAB]
    float* rs = c1s + 2 * SLAB;                                                     // [2][SLAB]
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nslab = (T + SLAB - 1) / SLAB;
    auto stage = [&](int sl, int buf) {   // warps 1-3
        const int t0 = sl * SLAB, n = min(SLAB, T - t0);
        for (int t = warp - 1; t < SLAB; t += HELPERS) {
            const size_t tok = ((size_t)b * T + t0 + t) * H + h;
            stage_piece(ks + (buf * SLAB + t) * DK, k + tok * DK, lane, DK, t < n);
        }
        const int ht = threadIdx.x - 32;                  // one helper thread per token: beta, r
        if (ht < SLAB) {
            const bool ok = ht < n;
            const size_t tok = ((size_t)b * T + t0 + ht) * H + h;
            c0s[buf * SLAB + ht] = ok ? to_f32(beta[tok]) : 0.f;      // beta for now
            rs[buf * SLAB + ht] = (ok && r) ? to_f32(r[tok]) : 1.f;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        helpers_sync();
        for (int t = warp - 1; t < SLAB; t += HELPERS) {
            const float n2 = warp_sum(k2_piece<DK>(ks + (buf * SLAB + t) * DK, lane));
            if (lane == 0) {
                const float bt = c0s[buf * SLAB + t];
                const float inv = n2 > 0.f ? eta / n2 : 0.f;
                c0s[buf * SLAB + t] = bt * inv;
                c1s[buf * SLAB + t] = bt * bt * inv;
            }
        }
    };
    float d[PER], da[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) d[i] = d0 ? d0[(size_t)unit * DK + lane * PER + i] : 1.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) da[i] = anchor ? d[i] : 0.f;
    if (warp != 0 && nslab > 0) stage(0, 0);
    __syncthreads();
    for (int sl = 0; sl < nslab; ++sl) {
        const int buf = sl & 1;
        if (warp != 0) {
            if (sl + 1 < nslab) stage(sl + 1, buf ^ 1);
        } else {
            const int t0 = sl * SLAB, n = min(SLAB, T - t0);
#pragma unroll 2
            for (int t = 0; t < n; ++t) {
                const size_t tok = ((size_t)b * T + t0 + t) * H + h;
                float kk[PER], a[PER];
                VecIO<PER, Tin>::load(ks + (buf * SLAB + t) * DK + lane * PER, kk);
                const float c0 = c0s[buf * SLAB + t], c1 = c1s[buf * SLAB + t], rt = rs[buf * SLAB + t];
                VecIO<PER, float>::store(d_all + tok * DK + lane * PER, d);
                float sd = 0.f;
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    a[i] = kk[i] * kk[i];
                    sd = fmaf(d[i], a[i], sd);
                }
                sd = warp_sum(sd);
                const float x = fmaf(-c1, sd, c0);
#pragma unroll
                for (int i = 0; i < PER; ++i) d[i] = rt * d[i] + (1.f - rt) * da[i] + x * a[i];
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Per chunk: Kw = D (.) K, T = (I + strict_tril(Kb Kw^T))^{-1}, W = T Kb,
// U0 = T diag(beta) V, P = tril(Q Kw^T).  Persistent CTAs, one chunk at a time.
template <int DK, int DV>
struct PrepSmem {
    static constexpr int LDK = DK + 4, LDX = (DK > DV ? DK : DV) + 4;
    static constexpr size_t kBytes = sizeof(float) * (size_t)(2 * C * LDK + C * LDX + 2 * C * LDC + 2 * C);
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_prep_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                const Tin* __restrict__ beta, const Tin* __restrict__ alpha, float* __restrict__ ws, Layout L, int B,
                int T, int H, int NC)
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
    float* gs = bs + C;              // [C] gated: log2 gamma_t
    const bool gated = alpha != nullptr;

    const int tid = threadIdx.x;
    const size_t nchunks = (size_t)B * H * NC;
    const float* d_all = ws + L.d_all / sizeof(float);
    // persistent: chunk cid, then cid + gridDim.x, ...; the next chunk's inputs are
    // prefetched into L2 while this one is computed
    for (size_t cid = blockIdx.x; cid < nchunks; cid += gridDim.x) {
    const int unit = (int)(cid / NC), c = (int)(cid % NC), b = unit / H, h = unit % H;
    const int c0 = c * C, Tc = min(C, T - c0);
    float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
    float* t_g = ws + L.tinv / sizeof(float) + cid * C * C;
    float* w_g = ws + L.w / sizeof(float) + cid * C * DK;
    float* u_g = ws + L.u0 / sizeof(float) + cid * C * DV;
    float* p_g = ws + L.p / sizeof(float) + cid * C * C;

    const size_t tok0 = ((size_t)b * T + c0) * H + h;     // token c0 of this (b, h)
    const size_t tstride = (size_t)H;                     // token step in [B, T, H] order
    __syncthreads();
    if (cid + gridDim.x < nchunks) {
        const size_t nx = cid + gridDim.x;
        const int un = (int)(nx / NC), cn = (int)(nx % NC), bn = un / H, hn = un % H;
        const int tcn = min(C, T - cn * C);
        const size_t tokn = ((size_t)bn * T + cn * C) * H + hn;
        prefetch_rows(k + tokn * DK, tstride * DK * sizeof(Tin), tcn, DK * sizeof(Tin));
        prefetch_rows(q + tokn * DK, tstride * DK * sizeof(Tin), tcn, DK * sizeof(Tin));
        prefetch_rows(v + tokn * DV, tstride * DV * sizeof(Tin), tcn, DV * sizeof(Tin));
        prefetch_rows(d_all + tokn * DK, tstride * DK * sizeof(float), tcn, DK * sizeof(float));
    }
    if (tid < C) bs[tid] = ld_or0(beta, tok0 + tid * tstride, tid < Tc);
    if (gated && tid < 32) {
        chunk_log2_gates(gs, alpha, tok0, tstride, Tc, tid);
        __syncwarp();
        ws[L.lg / sizeof(float) + cid * C + 2 * tid] = gs[2 * tid];
        ws[L.lg / sizeof(float) + cid * C + 2 * tid + 1] = gs[2 * tid + 1];
    }
    async_tile<C, DK>(Kw, LDK, d_all + tok0 * DK, tstride * DK, Tc);     // d_t for now
    load_tile<C, DK>(Kb, LDK, k + tok0 * DK, tstride * DK, Tc);
    cp_async_wait_all();
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int t = idx / DK, i = idx % DK;
        const float kv = Kb[t * LDK + i], w = Kw[t * LDK + i] * kv;
        Kb[t * LDK + i] = bs[t] * kv;
        Kw[t * LDK + i] = w;
    }
    load_tile<C, DV>(X, LDX, v + tok0 * DV, tstride * DV, Tc, bs);
    __syncthreads();
    store_rows<C, DK>(kw_g, DK, Kw, LDK);
    cta_gemm<SPLIT>(C, C, DK, Mat<LDK, 1>{Kb}, Mat<1, LDK>{Kw},
                    [&](int m, int n, float x0, float x1) {
                        if (gated) {   // x R_mn = gamma_m / gamma_n
                            x0 *= ex2(gs[m] - gs[n]);
                            x1 *= ex2(gs[m] - gs[n + 1]);
                        }
                        store2(As + m * LDC + n, n < m ? x0 : 0.f, n + 1 < m ? x1 : 0.f);
                    });
    __syncthreads();
    // T = (I + A)^{-1}. fp32 mode: exact forward substitution into Ts, column j on 8
    // threads that split the inner sum. bf16 inputs: the blocked inverse in place over A
    // on warps 0-3 (16 x 16 diagonal blocks by substitution, the rest on tf32 mma.sync),
    // the same routine as the forward chunk kernel's.
    const float* Tm = SPLIT ? Ts : As;
    if (SPLIT) {
        const int j = tid >> 3, part = tid & 7;
        for (int i = 0; i < C; ++i) {
            float sum = 0.f;
            for (int l = j + part; l < i; l += 8) sum = fmaf(As[i * LDC + l], Ts[l * LDC + j], sum);
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            sum += __shfl_xor_sync(0xffffffffu, sum, 4);
            __syncwarp();
            if (part == 0) Ts[i * LDC + j] = (i < j) ? 0.f : (i == j ? 1.f : -sum);
            __syncwarp();
        }
    } else if (tid < 128) {
        static_assert(LDC == tri::LD, "the blocked inverse takes the 68-float row stride");
        tri::tril_inv64_inplace(As, tid >> 5, tid & 31, [] { asm volatile("bar.sync 1, 128;" ::: "memory"); });
    }
    if (gated) {   // W = T diag(gamma) Kb: Kb rows x gamma_t (the Gram above used them unscaled)
        if (tid < C) bs[tid] = ex2(gs[tid]);   // beta is no longer needed: gamma_t in its place
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += NTHR) Kb[(idx / DK) * LDK + idx % DK] *= bs[idx / DK];
    }
    __syncthreads();
    store_rows<C, C>(t_g, C, Tm, LDC);
    cta_gemm<SPLIT>(C, DK, C, Mat<LDC, 1>{Tm}, Mat<LDK, 1>{Kb},
                    [&](int m, int n, float x0, float x1) { store2(w_g + m * DK + n, x0, x1); });
    cta_gemm<SPLIT>(C, DV, C, Mat<LDC, 1>{Tm}, Mat<LDX, 1>{X},
                    [&](int m, int n, float x0, float x1) { store2(u_g + m * DV + n, x0, x1); });
    __syncthreads();
    load_tile<C, DK>(X, LDX, q + tok0 * DK, tstride * DK, Tc);
    __syncthreads();
    cta_gemm<SPLIT>(C, C, DK, Mat<LDX, 1>{X}, Mat<1, LDK>{Kw},
                    [&](int m, int n, float x0, float x1) {
                        if (gated) {
                            x0 *= ex2(gs[m] - gs[n]);
                            x1 *= ex2(gs[m] - gs[n + 1]);
                        }
                        store2(p_g + m * C + n, n <= m ? x0 : 0.f, n + 1 <= m ? x1 : 0.f);
                    });
    }
}

// ---------------------------------------------------------------------------
// Forward state pass for DVT rows of S: S at every chunk start (ckS) and Vn.
template <int DK, int DVT>
struct StateSmem {
    static constexpr int LDK = DK + 4, LDT = DVT + 4;
    static constexpr size_t kFwdBytes = sizeof(float) * (size_t)(DVT * LDK + 2 * C * LDK + C * LDT + 2 * C);
    static constexpr size_t kBwdBytes =
        sizeof(float) * (size_t)(DVT * LDK + C * LDC + 2 * C * LDT + 2 * C * LDK + 3 * C);
};

template <int DK, int DV, int DVT, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_state_f_kernel(const float* __restrict__ S0, float* __restrict__ ws, Layout L, int NC, int gated)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    using SM = StateSmem<DK, DVT>;
    constexpr int LDK = SM::LDK, LDT = SM::LDT, NTILE = DV / DVT;
    extern __shared__ float sm[];
    float* Ss = sm;                  // [DVT][LDK] rows v0 .. v0 + DVT - 1 of S
    float* Ws = Ss + DVT * LDK;      // [C][LDK] W
    float* Kws = Ws + C * LDK;       // [C][LDK] Kw
    float* Vs = Kws + C * LDK;       // [C][LDT] U0, then Vn (columns of the tile)
    float* gs = Vs + C * LDT;        // [C] gated: log2 gamma_t
    float* rh = gs + C;              // [C] gated: rho_t = gamma_C / gamma_t

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
        if (c + 1 < NC) {   // L2 prefetch of the next chunk's blocks
            prefetch_rows(w_g + C * DK, 0, 1, C * DK * 4);
            prefetch_rows(kw_g + C * DK, 0, 1, C * DK * 4);
            prefetch_rows(u_g + C * DV + v0, (size_t)DV * 4, C, DVT * 4);
        }
        store_rows<DVT, DK>(s_g + (size_t)v0 * DK, DK, Ss, LDK);
        async_block<C, DK>(Ws, LDK, w_g);
        async_block<C, DK>(Kws, LDK, kw_g);
        async_tile<C, DVT>(Vs, LDT, u_g + v0, (size_t)DV);
        if (gated && tid < C) gs[tid] = ws[L.lg / sizeof(float) + cid * C + tid];
        cp_async_wait_all();
        __syncthreads();
        cta_gemm<SPLIT>(C, DVT, DK, Mat<LDK, 1>{Ws}, Mat<1, LDK>{Ss}, [&](int m, int n, float x0, float x1) {
            const float vn0 = Vs[m * LDT + n] - x0, vn1 = Vs[m * LDT + n + 1] - x1;
            Vs[m * LDT + n] = vn0;
            Vs[m * LDT + n + 1] = vn1;
            store2(vn_g + m * DV + v0 + n, vn0, vn1);
        });
        __syncthreads();
        if (gated) {   // S' = gamma_C S + Vn^T diag(rho) Kw
            const float gl = gs[C - 1], gc = ex2(gl);
            if (tid < C) rh[tid] = ex2(gl - gs[tid]);
            for (int idx = tid; idx < DVT * DK; idx += NTHR) Ss[(idx / DK) * LDK + idx % DK] *= gc;
            __syncthreads();
            for (int idx = tid; idx < C * DK; idx += NTHR) Kws[(idx / DK) * LDK + idx % DK] *= rh[idx / DK];
            __syncthreads();
        }
        cta_gemm<SPLIT>(DVT, DK, C, Mat<1, LDT>{Vs}, Mat<LDK, 1>{Kws},
                        [&](int m, int n, float x0, float x1) { add2(Ss + m * LDK + n, x0, x1); });
    }
}

// Reverse state pass for DVT rows of dS: dS' at every chunk end (ckdS), dVn, and dS0.
template <int DK, int DV, int DVT, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_state_b_kernel(const Tin* __restrict__ dout, const Tin* __restrict__ q, const float* __restrict__ dS_final,
                   float* __restrict__ dS0, float* __restrict__ ws, Layout L, int B, int T, int H, int NC, int gated)
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
    float* gs = B2 + C * LDK;        // [C] gated: log2 gamma_t
    float* rh = gs + C;              // [C] gated: rho_t = gamma_C / gamma_t
    float* gm = rh + C;              // [C] gated: gamma_t

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
        if (c > 0) {   // L2 prefetch of the previous chunk's blocks and rows (chunk c - 1 is full)
            const size_t tokp = ((size_t)b * T + c0 - C) * H + h;
            prefetch_rows(p_g - C * C, 0, 1, C * C * 4);
            prefetch_rows(kw_g - C * DK, 0, 1, C * DK * 4);
            prefetch_rows(w_g - C * DK, 0, 1, C * DK * 4);
            prefetch_rows(dout + tokp * DV + v0, (size_t)H * DV * sizeof(Tin), C, DVT * sizeof(Tin));
            prefetch_rows(q + tokp * DK, (size_t)H * DK * sizeof(Tin), C, DK * sizeof(Tin));
        }
        store_rows<DVT, DK>(ds_g + (size_t)v0 * DK, DK, dSs, LDK);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        async_block<C, C>(Ps, LDC, p_g);
        async_block<C, DK>(B1, LDK, kw_g);
        load_tile<C, DVT>(dOs, LDT, dout + tok0 * DV + v0, (size_t)H * DV, Tc);
        load_tile<C, DK>(B2, LDK, q + tok0 * DK, (size_t)H * DK, Tc);
        if (gated && tid < C) gs[tid] = ws[L.lg / sizeof(float) + cid * C + tid];
        cp_async_wait_all();
        __syncthreads();
        if (gated) {   // Kw rows x rho_t and Q rows x gamma_t
            if (tid < C) {
                rh[tid] = ex2(gs[C - 1] - gs[tid]);
                gm[tid] = ex2(gs[tid]);
            }
            __syncthreads();
            for (int idx = tid; idx < C * DK; idx += NTHR) {
                const int t = idx / DK, i = idx % DK;
                B1[t * LDK + i] *= rh[t];
                B2[t * LDK + i] *= gm[t];
            }
            __syncthreads();
        }
        // dVn = P^T dO + diag(rho) Kw dS'^T
        cta_gemm2<SPLIT>(C, DVT, C, Mat<1, LDC>{Ps}, Mat<LDT, 1>{dOs}, DK, Mat<LDK, 1>{B1}, Mat<1, LDK>{dSs},
                         [&](int m, int n, float x0, float x1) {
                             dVs[m * LDT + n] = -x0;
                             dVs[m * LDT + n + 1] = -x1;
                             store2(dvn_g + m * DV + v0 + n, x0, x1);
                         });
        __syncthreads();
        async_block<C, DK>(B1, LDK, w_g);
        if (gated) {   // gamma_C dS'
            const float gc = ex2(gs[C - 1]);
            for (int idx = tid; idx < DVT * DK; idx += NTHR) dSs[(idx / DK) * LDK + idx % DK] *= gc;
        }
        cp_async_wait_all();
        __syncthreads();
        // dS = gamma_C dS' + dO^T diag(gamma) Q + (-dVn)^T W
        cta_gemm2<SPLIT>(DVT, DK, C, Mat<1, LDT>{dOs}, Mat<LDK, 1>{B2}, C, Mat<1, LDT>{dVs}, Mat<LDK, 1>{B1},
                         [&](int m, int n, float x0, float x1) { add2(dSs + m * LDK + n, x0, x1); });
    }
    __syncthreads();
    if (dS0) store_rows<DVT, DK>(dS0 + ((size_t)unit * DV + v0) * DK, DK, dSs, LDK);
}

// ---------------------------------------------------------------------------
// Every gradient of one chunk. Value side, over the dv tiles in turn: dP and dT
// (V part) summed over the tiles, dV, the tile terms of dQ (dO S), dKw (Vn dS')
// and dW (-dVn S), the dbeta term rowdot(T^T dVn, V); then dQ += dP Kw and
// dKw += dP^T Q once. Key side, as written below. dQ, dKw, dW and dK stay in
// registers: warp w (of 16) owns rows 16 (w % 4) .. + 15 and columns
// (DK / 4) (w / 4) .. + DK / 4 - 1 of each.
// Gated: the gate factors enter as the header states, and dalpha_m is taken as the sum of
// the terms whose gate product holds alpha_m, each divided by alpha_m in the exponent
// (2^(sum of the other clamped log2 alphas)): the pair (t, j) of A and P for j < m <= t,
// the rows t >= m of dO S and of T^T dW, the rows j < m of Vn dS', and <dS', S>. No
// difference of large terms is taken, so dalpha keeps its relative accuracy for gates
// near 0 (where the chunk-local dG form, a reverse cumulative sum over 1 / alpha_m,
// cancels). With G the in-chunk cumulative clamped log2 alpha (G_{-1} = 0), the factor of
// pair (t, j) is 2^(G_t - G_j - l_m) = 2^(G_t - G_m) 2^(G_{m-1} - G_j), both at most 1, so
//   dalpha_m = sum_{t >= m} 2^(G_t - G_m) (Y_tm + a_t 2^G_{m-1})
//              + 2^(G_C - G_m) (sum_{j < m} W_mj y_j + <dS', S> 2^G_{m-1}),
// with W_mj = 2^(G_{m-1} - G_j) (j < m) and Y = X' W^T, one 64 x 64 x 64 product.
constexpr int J = 32;           // dv tile of the gradient kernel
constexpr int LDJ = J + 4;

template <int DK>
struct GradSmem {
    static constexpr int LDK = DK + 4;
    static constexpr size_t kBytes =
        sizeof(float) * (size_t)(2 * C * LDK + 4 * C * LDC + 4 * C * LDJ + 2 * J * LDK + 8 * C);
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(NTHR, 1)
bwd_grads_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const Tin* __restrict__ beta, const Tin* __restrict__ alpha, const Tin* __restrict__ dout,
                 Tin* __restrict__ dq, Tin* __restrict__ dv, Tin* __restrict__ dalpha, float* __restrict__ ws,
                 Layout L, int B, int T, int H, int NC)
{
    constexpr bool SPLIT = std::is_same<Tin, float>::value;
    constexpr int LDK = GradSmem<DK>::LDK, NT = DK / 32;
    extern __shared__ float sm[];
    float* Qs = sm;                  // [C][LDK] Q
    float* Kws = Qs + C * LDK;       // [C][LDK] Kw
    float* Ts = Kws + C * LDK;       // [C][LDC] T
    float* dPs = Ts + C * LDC;       // [C][LDC] dP, summed over the tiles
    float* dTs = dPs + C * LDC;      // [C][LDC] dT (V part), summed over the tiles
    float* dOs = dTs + C * LDC;      // [C][LDJ] dO columns of the tile
    float* Vns = dOs + C * LDJ;      // [C][LDJ] Vn
    float* dVns = Vns + C * LDJ;     // [C][LDJ] dVn
    float* Vs = dVns + C * LDJ;      // [C][LDJ] V
    float* SJ = Vs + C * LDJ;        // [J][LDK] rows of S (chunk start)
    float* dSJ = SJ + J * LDK;       // [J][LDK] rows of dS' (chunk end)
    float* bs = dSJ + J * LDK;       // [C] beta
    float* dbs = bs + C;             // [C] dbeta (the chunk part)
    // gated only:
    float* Xg = dbs + C;             // [C][LDC] the pair terms of d log gamma with R divided out
    float* gsm = Xg + C * LDC;       // [C] log2 gamma_t
    float* lsm = gsm + C;            // [C] clamped log2 alpha_t
    float* gam = lsm + C;            // [C] gamma_t
    float* av = gam + C;             // [C] <(dO S)_t, Q_t> + beta_t <(T^T dW)_t, K_t>
    float* yr = av + C;              // [C] <(Vn dS')_t, Kw_t>
    float* csd = yr + C;             // [1] <dS', S>
    const bool gated = alpha != nullptr;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t nchunks = (size_t)B * H * NC;
    const float* d_all = ws + L.d_all / sizeof(float);
    for (size_t cid = blockIdx.x; cid < nchunks; cid += gridDim.x) {   // persistent, as bwd_prep
    const int unit = (int)(cid / NC), c = (int)(cid % NC), b = unit / H, h = unit % H;
    const int c0 = c * C, Tc = min(C, T - c0);
    const float* kw_g = ws + L.kw / sizeof(float) + cid * C * DK;
    const float* t_g = ws + L.tinv / sizeof(float) + cid * C * C;
    const float* vn_g = ws + L.vn / sizeof(float) + cid * C * DV;
    const float* dvn_g = ws + L.dvn / sizeof(float) + cid * C * DV;
    const float* s_g = ws + L.ckS / sizeof(float) + cid * DV * DK;
    const float* ds_g = ws + L.ckdS / sizeof(float) + cid * DV * DK;
    float* dd_g = ws + L.dd / sizeof(float) + cid * C * DK;
    float* dkp_g = ws + L.dkp / sizeof(float) + cid * C * DK;
    float* dbp_g = ws + L.dbp / sizeof(float) + cid * C;
    auto tok = [&](int t) { return ((size_t)b * T + c0 + t) * H + h; };

    const size_t tok0 = tok(0);
    __syncthreads();
    async_block<C, DK>(Kws, LDK, kw_g);        // waited for with the first tile's copies
    async_block<C, C>(Ts, LDC, t_g);
    load_tile<C, DK>(Qs, LDK, q + tok0 * DK, (size_t)H * DK, Tc);
    for (int idx = tid; idx < C * C; idx += NTHR) {
        dTs[(idx / C) * LDC + idx % C] = 0.f;
        dPs[(idx / C) * LDC + idx % C] = 0.f;
    }
    if (tid < C) {
        bs[tid] = ld_or0(beta, tok(tid), tid < Tc);
        dbs[tid] = 0.f;
        av[tid] = 0.f;
        yr[tid] = 0.f;
    }
    if (gated) {
        if (tid < 32) chunk_log2_gates(gsm, alpha, tok0, (size_t)H, Tc, tid, lsm);
        if (tid == 0) *csd = 0.f;
        __syncthreads();
        if (tid < C) gam[tid] = ex2(gsm[tid]);
    }
    float sds = 0.f;   // gated: this thread's part of <dS', S>

    const int m0 = 16 * (warp & 3), n0 = (DK / 4) * (warp >> 2);
    float aQ[NT][4], aKw[NT][4], aW[NT][4];
    frag_zero(aQ);
    frag_zero(aKw);
    frag_zero(aW);
    for (int v0 = 0; v0 < DV; v0 += J) {
        __syncthreads();
        async_tile<C, J>(Vns, LDJ, vn_g + v0, (size_t)DV);
        async_tile<C, J>(dVns, LDJ, dvn_g + v0, (size_t)DV);
        async_block<J, DK>(SJ, LDK, s_g + (size_t)v0 * DK);
        async_block<J, DK>(dSJ, LDK, ds_g + (size_t)v0 * DK);
        load_tile<C, J>(dOs, LDJ, dout + tok0 * DV + v0, (size_t)H * DV, Tc);
        load_tile<C, J>(Vs, LDJ, v + tok0 * DV + v0, (size_t)H * DV, Tc);
        cp_async_wait_all();
        __syncthreads();
        // dP += tril(dO Vn^T) of this tile
        cta_gemm<SPLIT>(C, C, J, Mat<LDJ, 1>{dOs}, Mat<1, LDJ>{Vns},
                        [&](int m, int n, float x0, float x1) {
                            if (n <= m) add2(dPs + m * LDC + n, x0, n + 1 <= m ? x1 : 0.f);
                        });
        // dT += (dVn V^T) diag(beta)
        cta_gemm<SPLIT>(C, C, J, Mat<LDJ, 1>{dVns}, Mat<1, LDJ>{Vs},
                        [&](int m, int n, float x0, float x1) { add2(dTs + m * LDC + n, bs[n] * x0, bs[n + 1] * x1); });
        {   // dV = diag(beta) T^T dVn, one 16 x 8 tile per warp; dbeta += rowdot(T^T dVn, V), the
            // 4 lanes that share a row reducing before one atomic
            static_assert(NTHR == 512 && J == 32, "16 warps cover the 64 x 32 tile as 4 x 4 tiles of 16 x 8");
            const int mv = 16 * (warp & 3), nv = 8 * (warp >> 2), t4 = lane & 3;
            float acc[1][4];
            frag_zero(acc);
            warp_mma<1, SPLIT>(acc, Mat<1, LDC>{Ts}, Mat<LDJ, 1>{dVns}, mv, nv, C, lane);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int m = mv + (lane >> 2) + 8 * hh, n = nv + 2 * t4;
                const float x0 = acc[0][2 * hh], x1 = acc[0][2 * hh + 1];
                if (m < Tc) store2(dv + tok(m) * DV + v0 + n, bs[m] * x0, bs[m] * x1);
                float part = x0 * Vs[m * LDJ + n] + x1 * Vs[m * LDJ + n + 1];
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                if (t4 == 0) atomicAdd(&dbs[m], part);
            }
        }
        warp_mma<NT, SPLIT>(aQ, Mat<LDJ, 1>{dOs}, Mat<LDK, 1>{SJ}, m0, n0, J, lane);     // dO S
        warp_mma<NT, SPLIT>(aKw, Mat<LDJ, 1>{Vns}, Mat<LDK, 1>{dSJ}, m0, n0, J, lane);   // Vn dS'
        warp_mma<NT, SPLIT>(aW, Mat<LDJ, 1>{dVns}, Mat<LDK, 1>{SJ}, m0, n0, J, lane);    // dVn S
        if (gated)
            for (int idx = tid; idx < J * DK; idx += NTHR)
                sds = fmaf(SJ[(idx / DK) * LDK + idx % DK], dSJ[(idx / DK) * LDK + idx % DK], sds);
    }
    __syncthreads();
    if (gated) {
        // <dS', S>; the rows of the ungated dO S and Vn dS' against Q and Kw; then
        // dQ's dO S part x gamma_t and dKw's Vn dS' part x rho_t = gamma_C / gamma_t
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sds += __shfl_xor_sync(0xffffffffu, sds, off);
        if (lane == 0) atomicAdd(csd, sds);
        const int t4 = lane & 3;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int m = m0 + (lane >> 2) + 8 * hh;
            const float gm = gam[m], rho = ex2(gsm[C - 1] - gsm[m]);
            float pq = 0.f, pk = 0.f;
#pragma unroll
            for (int jj = 0; jj < NT; ++jj) {
                const int n = n0 + 8 * jj + 2 * t4;
                pq = fmaf(aQ[jj][2 * hh], Qs[m * LDK + n], pq);
                pq = fmaf(aQ[jj][2 * hh + 1], Qs[m * LDK + n + 1], pq);
                pk = fmaf(aKw[jj][2 * hh], Kws[m * LDK + n], pk);
                pk = fmaf(aKw[jj][2 * hh + 1], Kws[m * LDK + n + 1], pk);
                aQ[jj][2 * hh] *= gm;
                aQ[jj][2 * hh + 1] *= gm;
                aKw[jj][2 * hh] *= rho;
                aKw[jj][2 * hh + 1] *= rho;
            }
            pq += __shfl_xor_sync(0xffffffffu, pq, 1);
            pq += __shfl_xor_sync(0xffffffffu, pq, 2);
            pk += __shfl_xor_sync(0xffffffffu, pk, 1);
            pk += __shfl_xor_sync(0xffffffffu, pk, 2);
            if (t4 == 0) {
                atomicAdd(&av[m], pq);
                atomicAdd(&yr[m], pk);
            }
        }
        // the P pair terms dP (.) strict_tril(Q Kw^T), then dP <- dP (.) R
        cta_gemm<SPLIT>(C, C, DK, Mat<LDK, 1>{Qs}, Mat<1, LDK>{Kws}, [&](int m, int n, float x0, float x1) {
            store2(Xg + m * LDC + n, n < m ? dPs[m * LDC + n] * x0 : 0.f,
                   n + 1 < m ? dPs[m * LDC + n + 1] * x1 : 0.f);
        });
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += NTHR) {
            const int m = idx / C, n = idx % C;
            if (n <= m) dPs[m * LDC + n] *= ex2(gsm[m] - gsm[n]);
        }
        __syncthreads();
    }
    warp_mma<NT, SPLIT>(aQ, Mat<LDC, 1>{dPs}, Mat<LDK, 1>{Kws}, m0, n0, C, lane);        // dP Kw
    warp_mma<NT, SPLIT>(aKw, Mat<1, LDC>{dPs}, Mat<LDK, 1>{Qs}, m0, n0, C, lane);        // dP^T Q
    frag_each(aQ, m0, n0, lane, [&](int m, int n, float x0, float x1) {
        if (m < Tc) store2(dq + tok(m) * DK + n, x0, x1);
    });
    if (cid + gridDim.x < nchunks) {   // L2 prefetch of the next chunk's inputs, issued here rather than
        // at the chunk start: it keeps about one chunk per CTA in flight instead of two
        const size_t nx = cid + gridDim.x;
        const int un = (int)(nx / NC), cn = (int)(nx % NC), bn = un / H, hn = un % H;
        const int tcn = min(C, T - cn * C);
        const size_t tokn = ((size_t)bn * T + cn * C) * H + hn;
        prefetch_rows(q + tokn * DK, (size_t)H * DK * sizeof(Tin), tcn, DK * sizeof(Tin));
        prefetch_rows(k + tokn * DK, (size_t)H * DK * sizeof(Tin), tcn, DK * sizeof(Tin));
        prefetch_rows(d_all + tokn * DK, (size_t)H * DK * sizeof(float), tcn, DK * sizeof(float));
        prefetch_rows(v + tokn * DV, (size_t)H * DV * sizeof(Tin), tcn, DV * sizeof(Tin));
        prefetch_rows(dout + tokn * DV, (size_t)H * DV * sizeof(Tin), tcn, DV * sizeof(Tin));
        prefetch_rows(ws + L.kw / sizeof(float) + nx * C * DK, 0, 1, C * DK * 4);
        prefetch_rows(ws + L.tinv / sizeof(float) + nx * C * C, 0, 1, C * C * 4);
        prefetch_rows(ws + L.vn / sizeof(float) + nx * C * DV, 0, 1, C * DV * 4);
        prefetch_rows(ws + L.dvn / sizeof(float) + nx * C * DV, 0, 1, C * DV * 4);
        prefetch_rows(ws + L.ckS / sizeof(float) + nx * DV * DK, 0, 1, DV * DK * 4);
        prefetch_rows(ws + L.ckdS / sizeof(float) + nx * DV * DK, 0, 1, DV * DK * 4);
    }

    // Key side: dT += (dW K^T) diag(beta), dA = -strict_tril(T^T dT T^T), the dbeta terms
    // of T^T dW and of dA, dK and the rest of dKw (still in registers), then dD = dKw (.) K
    // and the chunk part of dk, dK + dKw (.) D. Q's buffer and the dv-tile buffers are reused.
    float* Ks = Qs;                  // [C][LDK] K
    float* dWs = dOs;                // [C][LDK] dW, over the four dv-tile buffers
    float* Xs = dPs;                 // [C][LDC] dT T^T
    float* Gs = SJ;                  // [C][LDC] K Kw^T, over the rows of S and dS'
    static_assert(C * LDK <= 4 * C * LDJ && C * LDC <= 2 * J * LDK, "key-side buffers fit the reused ones");
    __syncthreads();                 // every warp is done with Q, dP and the dv tiles
    frag_each(aW, m0, n0, lane, [&](int m, int n, float x0, float x1) { store2(dWs + m * LDK + n, -x0, -x1); });
    load_tile<C, DK>(Ks, LDK, k + tok0 * DK, (size_t)H * DK, Tc);
    __syncthreads();
    cta_gemm<SPLIT>(C, C, DK, Mat<LDK, 1>{dWs}, Mat<1, LDK>{Ks}, [&](int m, int n, float x0, float x1) {
        // x diag(beta gamma) (W = T diag(beta gamma) K when gated)
        const float f0 = gated ? bs[n] * gam[n] : bs[n], f1 = gated ? bs[n + 1] * gam[n + 1] : bs[n + 1];
        add2(dTs + m * LDC + n, f0 * x0, f1 * x1);
    });
    cta_gemm<SPLIT>(C, C, DK, Mat<LDK, 1>{Ks}, Mat<1, LDK>{Kws},
                    [&](int m, int n, float x0, float x1) { store2(Gs + m * LDC + n, x0, x1); });
    __syncthreads();
    cta_gemm<SPLIT>(C, C, C, Mat<LDC, 1>{dTs}, Mat<1, LDC>{Ts},
                    [&](int m, int n, float x0, float x1) { store2(Xs + m * LDC + n, x0, x1); });
    __syncthreads();
    cta_gemm<SPLIT>(C, C, C, Mat<1, LDC>{Ts}, Mat<LDC, 1>{Xs}, [&](int m, int n, float x0, float x1) {
        float a0 = n < m ? -x0 : 0.f, a1 = n + 1 < m ? -x1 : 0.f;   // dA (strictly lower)
        if (gated && n < m) {   // the A pair terms beta_m dA (.) K Kw^T, then dA <- dA (.) R
            // (R only below the diagonal: above it the ratio may overflow)
            Xg[m * LDC + n] += bs[m] * a0 * Gs[m * LDC + n];
            Xg[m * LDC + n + 1] += bs[m] * a1 * Gs[m * LDC + n + 1];
            a0 *= ex2(gsm[m] - gsm[n]);
            if (n + 1 < m) a1 *= ex2(gsm[m] - gsm[n + 1]);
        }
        if (n < m) atomicAdd(&dbs[m], a0 * Gs[m * LDC + n] + a1 * Gs[m * LDC + n + 1]);
        dTs[m * LDC + n] = bs[m] * a0;                                    // diag(beta) dA
        dTs[m * LDC + n + 1] = bs[m] * a1;
    });
    __syncthreads();
    float aK[NT][4];
    frag_zero(aK);
    warp_mma<NT, SPLIT>(aK, Mat<1, LDC>{Ts}, Mat<LDK, 1>{dWs}, m0, n0, C, lane);        // T^T dW
    {   // dbeta += gamma_m rowdot(T^T dW, K): the 4 lanes that share a row reduce before one
        // atomic (gamma = 1 ungated); gated, the row's d log gamma term beta_m rowdot(T^T dW, K)
        const int t4 = lane & 3;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int m = m0 + (lane >> 2) + 8 * hh;
            const float gm = gated ? gam[m] : 1.f, fk = bs[m] * gm;
            float part = 0.f;
#pragma unroll
            for (int jj = 0; jj < NT; ++jj) {
                const int n = n0 + 8 * jj + 2 * t4;
                part = fmaf(aK[jj][2 * hh], Ks[m * LDK + n], part);
                part = fmaf(aK[jj][2 * hh + 1], Ks[m * LDK + n + 1], part);
                aK[jj][2 * hh] *= fk;
                aK[jj][2 * hh + 1] *= fk;
            }
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (t4 == 0) {
                atomicAdd(&dbs[m], gm * part);
                if (gated) atomicAdd(&av[m], bs[m] * part);
            }
        }
    }
    warp_mma<NT, SPLIT>(aK, Mat<LDC, 1>{dTs}, Mat<LDK, 1>{Kws}, m0, n0, C, lane);       // + dAb Kw
    warp_mma<NT, SPLIT>(aKw, Mat<1, LDC>{dTs}, Mat<LDK, 1>{Ks}, m0, n0, C, lane);       // + dAb^T K
#pragma unroll
    for (int jj = 0; jj < NT; ++jj)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // columns n, n + 1 of row m
            const int m = m0 + (lane >> 2) + 8 * hh, n = n0 + 8 * jj + 2 * (lane & 3);
            const float w0 = aKw[jj][2 * hh], w1 = aKw[jj][2 * hh + 1];
            float2 dval = make_float2(0.f, 0.f);
            if (m < Tc) dval = *reinterpret_cast<const float2*>(d_all + tok(m) * DK + n);
            store2(dd_g + m * DK + n, w0 * Ks[m * LDK + n], w1 * Ks[m * LDK + n + 1]);
            store2(dkp_g + m * DK + n, aK[jj][2 * hh] + w0 * dval.x, aK[jj][2 * hh + 1] + w1 * dval.y);
        }
    __syncthreads();
    if (tid < C) dbp_g[tid] = dbs[tid];
    if (gated) {   // dalpha: W over the key-side buffers, Y = X' W^T, then warp w takes tokens w, w + 16, ..
        float* Wm = Xs;              // [C][LDC] W_mj
        float* Ym = Gs;              // [C][LDC] Y_tm
        for (int idx = tid; idx < C * C; idx += NTHR) {
            const int m = idx / C, j = idx % C;
            Wm[m * LDC + j] = j < m ? ex2((m > 0 ? gsm[m - 1] : 0.f) - gsm[j]) : 0.f;
        }
        __syncthreads();
        cta_gemm<SPLIT>(C, C, C, Mat<LDC, 1>{Xg}, Mat<1, LDC>{Wm},
                        [&](int t, int m, float x0, float x1) { store2(Ym + t * LDC + m, x0, x1); });
        __syncthreads();
        const float gl = gsm[C - 1];
        for (int m = warp; m < Tc; m += NTHR / 32) {
            const float gmm = gsm[m], gp = ex2(m > 0 ? gsm[m - 1] : 0.f);
            float s = 0.f, u = 0.f;
            for (int t = m + lane; t < C; t += 32) s = fmaf(ex2(gsm[t] - gmm), fmaf(av[t], gp, Ym[t * LDC + m]), s);
            for (int j = lane; j < m; j += 32) u = fmaf(Wm[m * LDC + j], yr[j], u);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, off);
                u += __shfl_xor_sync(0xffffffffu, u, off);
            }
            if (lane == 0) dalpha[tok(m)] = from_f32<Tin>(fmaf(ex2(gl - gmm), fmaf(*csd, gp, u), s));
        }
    }
    }
}

// ---------------------------------------------------------------------------
// Reverse of the d recurrence, token by token, in slabs staged by warps 1-3;
// lane l of warp 0 owns features l * DK / 32 ..; writes the final dk, dbeta, dr
// and dd0.
template <int DK, typename Tin>
struct DchainSmem {
    static constexpr size_t kBytes = 2 * (SLAB * DK * (sizeof(Tin) + 3 * sizeof(float)) + 6 * SLAB * sizeof(float));
};

// Per token the helpers stage k, d_t, dD_t and the chunk part of dk and precompute the
// scalars of the step that do not depend on Ld: x, eta (1 - 2 beta s) / n,
// -eta beta^2 / n and -x / n (all 0 when k = 0), with s = <d_t, k^2> and n = ||k||^2.
// The chain then carries one reduction, <k^2, Ld>, per token (the <d - d0, Ld> of dr
// is reduced alongside it but feeds nothing back).
template <int DK, typename Tin>
__global__ void __launch_bounds__(SERIAL_THREADS, 1)
bwd_dchain_kernel(const Tin* __restrict__ k, const Tin* __restrict__ beta, const Tin* __restrict__ r,
                  const float* __restrict__ d0, const float* __restrict__ dd_final,
                  Tin* __restrict__ dk, Tin* __restrict__ dbeta, Tin* __restrict__ dr, float* __restrict__ dd0,
                  const float* __restrict__ ws, Layout L, int B, int T, int H, int NC, float eta, int anchor)
{
    constexpr int PER = DK / 32;
    extern __shared__ __align__(16) unsigned char smraw[];
    float* ds_ = reinterpret_cast<float*>(smraw);          // [2][SLAB][DK] d_t
    float* dDs = ds_ + 2 * SLAB * DK;                      // [2][SLAB][DK] dL/dd_t through the write key
    float* dks = dDs + 2 * SLAB * DK;                      // [2][SLAB][DK] chunk part of dk
    float* sc = dks + 2 * SLAB * DK;                       // [2][SLAB][6] x, c1, c2, c3, r, chunk dbeta
    Tin* ks = reinterpret_cast<Tin*>(sc + 2 * SLAB * 6);   // [2][SLAB][DK] k
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nslab = (T + SLAB - 1) / SLAB;
    const float* d_all = ws + L.d_all / sizeof(float);
    const float* dd_g = ws + L.dd / sizeof(float);
    const float* dkp_g = ws + L.dkp / sizeof(float);
    const float* dbp_g = ws + L.dbp / sizeof(float);
    // slab sl covers tokens [sl * SLAB, ...); SLAB divides the chunk length, so a token's
    // rows of the chunk-block arrays are at crow0 + t
    auto stage = [&](int sl, int buf) {   // warps 1-3
        const int t0 = sl * SLAB, n = min(SLAB, T - t0);
        const size_t crow0 = ((size_t)unit * NC + t0 / C) * C + t0 % C;
        for (int t = warp - 1; t < SLAB; t += HELPERS) {
            const bool ok = t < n;
            const size_t tok = ((size_t)b * T + t0 + t) * H + h;
            const int row = buf * SLAB + t;
            stage_piece(ks + row * DK, k + tok * DK, lane, DK, ok);
            stage_piece(ds_ + row * DK, d_all + tok * DK, lane, DK, ok);
            stage_piece(dDs + row * DK, dd_g + (crow0 + t) * DK, lane, DK, ok);
            stage_piece(dks + row * DK, dkp_g + (crow0 + t) * DK, lane, DK, ok);
        }
        const int ht = threadIdx.x - 32;                  // one helper thread per token: beta, r, dbeta
        if (ht < SLAB) {
            const bool ok = ht < n;
            const size_t tok = ((size_t)b * T + t0 + ht) * H + h;
            float* q6 = sc + (buf * SLAB + ht) * 6;
            q6[0] = ok ? to_f32(beta[tok]) : 0.f;          // beta for now
            q6[4] = (ok && r) ? to_f32(r[tok]) : 1.f;
            q6[5] = ok ? dbp_g[crow0 + ht] : 0.f;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        helpers_sync();
        for (int t = warp - 1; t < SLAB; t += HELPERS) {
            const int row = buf * SLAB + t;
            float n2 = 0.f, sd = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const float kv = to_f32(ks[row * DK + lane * PER + i]);
                n2 = fmaf(kv, kv, n2);
                sd = fmaf(ds_[row * DK + lane * PER + i], kv * kv, sd);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                n2 += __shfl_xor_sync(0xffffffffu, n2, o);
                sd += __shfl_xor_sync(0xffffffffu, sd, o);
            }
            if (lane == 0) {
                float* q6 = sc + row * 6;
                const float bt = q6[0];
                float x = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
                if (n2 > 0.f) {
                    x = eta * bt * (1.f - bt * sd) / n2;
                    c1 = eta * (1.f - 2.f * bt * sd) / n2;
                    c2 = -eta * bt * bt / n2;
                    c3 = -x / n2;
                }
                q6[0] = x; q6[1] = c1; q6[2] = c2; q6[3] = c3;
            }
        }
    };

    float lam[PER], anc[PER], dda[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int f = lane * PER + i;
        lam[i] = dd_final ? dd_final[(size_t)unit * DK + f] : 0.f;
        anc[i] = anchor ? (d0 ? d0[(size_t)unit * DK + f] : 1.f) : 0.f;
        dda[i] = 0.f;
    }
    if (warp != 0 && nslab > 0) stage(nslab - 1, (nslab - 1) & 1);
    __syncthreads();
    for (int sl = nslab - 1; sl >= 0; --sl) {
        const int buf = sl & 1;
        if (warp != 0) {
            if (sl > 0) stage(sl - 1, buf ^ 1);
        } else {
            const int t0 = sl * SLAB, n = min(SLAB, T - t0);
#pragma unroll 2
            for (int t = n - 1; t >= 0; --t) {
                const size_t tok = ((size_t)b * T + t0 + t) * H + h;
                const int row = buf * SLAB + t;
                float kk[PER], dc[PER], dD[PER], dkp[PER], a[PER];
                VecIO<PER, Tin>::load(ks + row * DK + lane * PER, kk);
                VecIO<PER, float>::load(ds_ + row * DK + lane * PER, dc);
                VecIO<PER, float>::load(dDs + row * DK + lane * PER, dD);
                VecIO<PER, float>::load(dks + row * DK + lane * PER, dkp);
                const float* q6 = sc + row * 6;
                const float x = q6[0], c1 = q6[1], c2 = q6[2], c3 = q6[3], rt = q6[4], dbc = q6[5];
                float dx = 0.f, drv = 0.f;
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    a[i] = kk[i] * kk[i];
                    dx = fmaf(a[i], lam[i], dx);
                    drv = fmaf(dc[i] - anc[i], lam[i], drv);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    dx += __shfl_xor_sync(0xffffffffu, dx, o);
                    drv += __shfl_xor_sync(0xffffffffu, drv, o);
                }
                const float dsv = c2 * dx, dnv = c3 * dx;
                float gk[PER];
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    gk[i] = dkp[i] + 2.f * kk[i] * (x * lam[i] + dsv * dc[i] + dnv);
                    if (anchor) dda[i] += (1.f - rt) * lam[i];
                    lam[i] = rt * lam[i] + dD[i] + dsv * a[i];
                }
                VecIO<PER, Tin>::store(dk + tok * DK + lane * PER, gk);
                if (lane == 0) {
                    dbeta[tok] = from_f32<Tin>(fmaf(c1, dx, dbc));
                    if (r && dr) dr[tok] = from_f32<Tin>(drv);
                }
            }
        }
        __syncthreads();
    }
    if (warp == 0 && dd0) {
#pragma unroll
        for (int i = 0; i < PER; ++i) dd0[(size_t)unit * DK + lane * PER + i] = lam[i] + dda[i];
    }
}

}  // namespace bwd
}  // namespace osdn
