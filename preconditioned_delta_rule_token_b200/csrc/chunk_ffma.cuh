// Chunkwise OSDN forward on CUDA cores (FP32 FFMA, no tensor cores).
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1: the DeltaNet chunkwise WY
// pipeline run with the scaled write key Kw = D (.) K in the block Gram matrix
// and in the intra-block scores, the read/erase key K unchanged.  Per chunk of
// C tokens with the chunk-start state S (dv x dk), the per-token recurrence
// S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) kw_t^T unrolls to
//   A = strict_tril(diag(beta) K Kw^T),   (I + A) U = diag(beta) (V - K S^T),
//   O = Q S^T + tril(Q Kw^T) U,           S <- S + U^T Kw.
// This kernel is the fp32 mode of the library (tolerance 1e-4 against the
// float64 oracle) and the reference implementation of the same algebra for
// any dtype.  One CTA owns one (sequence, head, dv tile of DVT rows of S);
// rows of S are independent given Kw, so the dv split needs no exchange.
#pragma once
#include "common.cuh"

namespace osdn {

// acc[i][j] (+)= sum_kk A(m_i, kk) * B(n_j, kk) for m_i = ty + 16 i and
// n_j = tx + 16 j, with A(m, kk) = A[m * am + kk * ak], B(n, kk) = B[n * bn + kk * bk].
template <int MI, int NJ, bool ZERO>
__device__ __forceinline__ void ffma_tile(float (&acc)[MI][NJ], const float* A, int am, int ak,
                                          const float* Bm, int bn, int bk, int K, int tx, int ty)
{
    if (ZERO) {
#pragma unroll
        for (int i = 0; i < MI; ++i)
#pragma unroll
            for (int j = 0; j < NJ; ++j) acc[i][j] = 0.f;
    }
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float a[MI], b[NJ];
#pragma unroll
        for (int i = 0; i < MI; ++i) a[i] = A[(ty + 16 * i) * am + kk * ak];
#pragma unroll
        for (int j = 0; j < NJ; ++j) b[j] = Bm[(tx + 16 * j) * bn + kk * bk];
#pragma unroll
        for (int i = 0; i < MI; ++i)
#pragma unroll
            for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
}

template <int DK, int DVT>
struct FfmaSmem {
    static constexpr int C = 64;
    static constexpr int LDK = DK + 1;
    static constexpr int LDV = DVT + 1;
    static constexpr int LDC = C + 1;
    static constexpr int kFloats = 3 * C * LDK + C * LDV + DVT * LDK + 2 * C * LDC + C;
    static constexpr size_t kBytes = sizeof(float) * (size_t)kFloats;
};

// Element strides of q, k, v and out over (b, t, h) (the scaled keys in the workspace are dense).
struct FfmaStrides {
    Tok3 q, k, v, o;
};

template <int DK, int DVT, typename Tin>
__global__ void __launch_bounds__(256, 1)
chunk_ffma_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ kw,
                  const Tin* __restrict__ v, const Tin* __restrict__ beta, const float* __restrict__ S0,
                  Tin* __restrict__ out, float* __restrict__ S_final, int B, int T, int H, int DV, FfmaStrides st)
{
    using L = FfmaSmem<DK, DVT>;
    constexpr int C = L::C, LDK = L::LDK, LDV = L::LDV, LDC = L::LDC;
    constexpr int NT = 256;
    extern __shared__ float sm[];
    float* Qs = sm;                    // [C][LDK] queries
    float* Ks = Qs + C * LDK;          // [C][LDK] read/erase keys
    float* Ws = Ks + C * LDK;          // [C][LDK] scaled write keys
    float* Xs = Ws + C * LDK;          // [C][LDV] V, then V - K S^T, then U
    float* Ss = Xs + C * LDV;          // [DVT][LDK] state tile (rows v0 .. v0 + DVT - 1)
    float* As = Ss + DVT * LDK;        // [C][LDC] strict_tril(diag(beta) K Kw^T)
    float* Ps = As + C * LDC;          // [C][LDC] tril(Q Kw^T)
    float* bs = Ps + C * LDC;          // [C] beta

    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int v0 = blockIdx.y * DVT;

    for (int idx = tid; idx < DVT * DK; idx += NT) {
        const int vv = idx / DK, i = idx % DK;
        Ss[vv * LDK + i] = S0 ? S0[((size_t)unit * DV + v0 + vv) * DK + i] : 0.f;
    }

    for (int c0 = 0; c0 < T; c0 += C) {
        const int Tc = min(C, T - c0);
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int t = idx / DK, i = idx % DK;
            float qv = 0.f, kv = 0.f, wv = 0.f;
            if (t < Tc) {
                const size_t tok = ((size_t)b * T + c0 + t) * H + h;   // the scaled keys are dense
                qv = to_f32(q[st.q.at(b, c0 + t, h) + i]);
                kv = to_f32(k[st.k.at(b, c0 + t, h) + i]);
                wv = to_f32(kw[tok * DK + i]);
            }
            Qs[t * LDK + i] = qv; Ks[t * LDK + i] = kv; Ws[t * LDK + i] = wv;
        }
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int t = idx / DVT, j = idx % DVT;
            float vv = 0.f;
            if (t < Tc) vv = to_f32(v[st.v.at(b, c0 + t, h) + v0 + j]);
            Xs[t * LDV + j] = vv;
        }
        if (tid < C) bs[tid] = (tid < Tc) ? to_f32(beta[((size_t)b * T + c0 + tid) * H + h]) : 0.f;
        __syncthreads();

        {   // Gram and scores: A = strict_tril(diag(beta) K Kw^T), P = tril(Q Kw^T)
            float acc[4][4];
            ffma_tile<4, 4, true>(acc, Ks, LDK, 1, Ws, LDK, 1, DK, tx, ty);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = ty + 16 * i, jj = tx + 16 * j;
                    As[t * LDC + jj] = (jj < t) ? bs[t] * acc[i][j] : 0.f;
                }
            ffma_tile<4, 4, true>(acc, Qs, LDK, 1, Ws, LDK, 1, DK, tx, ty);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = ty + 16 * i, jj = tx + 16 * j;
                    Ps[t * LDC + jj] = (jj <= t) ? acc[i][j] : 0.f;
                }
        }
        {   // X = V - K S^T
            float acc[4][DVT / 16];
            ffma_tile<4, DVT / 16, true>(acc, Ks, LDK, 1, Ss, LDK, 1, DK, tx, ty);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < DVT / 16; ++j) {
                    const int t = ty + 16 * i, vv = tx + 16 * j;
                    Xs[t * LDV + vv] -= acc[i][j];
                }
        }
        __syncthreads();

        {   // (I + A) U = diag(beta) X by forward substitution; columns are
            // independent, 4 threads share one column and split the inner sum.
            const int col = tid >> 2, part = tid & 3;
            for (int cb = col; cb < DVT; cb += NT / 4) {
                for (int t = 0; t < C; ++t) {
                    float s = 0.f;
                    for (int j = part; j < t; j += 4) s = fmaf(As[t * LDC + j], Xs[j * LDV + cb], s);
                    s += __shfl_xor_sync(0xffffffffu, s, 1);
                    s += __shfl_xor_sync(0xffffffffu, s, 2);
                    const float u = bs[t] * Xs[t * LDV + cb] - s;
                    __syncwarp();
                    if (part == 0) Xs[t * LDV + cb] = u;
                    __syncwarp();
                }
            }
        }
        __syncthreads();

        {   // O = Q S^T + tril(Q Kw^T) U
            float acc[4][DVT / 16];
            ffma_tile<4, DVT / 16, true>(acc, Qs, LDK, 1, Ss, LDK, 1, DK, tx, ty);
            ffma_tile<4, DVT / 16, false>(acc, Ps, LDC, 1, Xs, 1, LDV, C, tx, ty);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = ty + 16 * i;
                if (t < Tc) {
                    const int64_t o = st.o.at(b, c0 + t, h);
#pragma unroll
                    for (int j = 0; j < DVT / 16; ++j)
                        out[o + v0 + tx + 16 * j] = from_f32<Tin>(acc[i][j]);
                }
            }
        }
        __syncthreads();

        {   // S <- S + U^T Kw
            float acc[DVT / 16][DK / 16];
            ffma_tile<DVT / 16, DK / 16, true>(acc, Xs, 1, LDV, Ws, 1, LDK, C, tx, ty);
#pragma unroll
            for (int i = 0; i < DVT / 16; ++i)
#pragma unroll
                for (int j = 0; j < DK / 16; ++j) Ss[(ty + 16 * i) * LDK + tx + 16 * j] += acc[i][j];
        }
    }
    __syncthreads();
    if (S_final) {
        for (int idx = tid; idx < DVT * DK; idx += NT) {
            const int vv = idx / DK, i = idx % DK;
            S_final[((size_t)unit * DV + v0 + vv) * DK + i] = Ss[vv * LDK + i];
        }
    }
}

}  // namespace osdn
