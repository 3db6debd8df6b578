// Preconditioner scan, token-serial form: one warp per (sequence, head).
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.2 (phase 1 of the two-phase plan: a
// light O(dk) scan over the key stream that yields the scaled write keys) and
// section 2.3 (APF retention r_t on d only):
//   k~_t = d_t (.) k_t,
//   d_{t+1} = r_t d_t + eta beta_t (1 - beta_t <d_t, k_t^2>) k_t^2 / ||k_t||^2,
// or with anchored APF r_t d_t + (1 - r_t) d0 + (the same step).
// Each lane holds DK/32 consecutive features of d in registers; the two
// per-token reductions (<d, k^2> and ||k||^2) are warp shuffles.  This form is
// latency-bound (one warp reduction per token); it serves fp32 mode and short
// sequences, and is the reference layout for the chunk-parallel scan.
// Optional diagnostic (sections 4-5): the residual ratio of each write,
// rho_t = (1 - beta_t <d_t, k_t^2>)^2 = f_t(S_t)/f_t(S_{t-1}) into rho [B, T, H],
// and q_geo = exp(mean_t log rho_t) per (sequence, head) into q_geo [B, H].
#pragma once
#include "common.cuh"

namespace osdn {

template <int DK, typename Tin>
__global__ void __launch_bounds__(128)
scan_seq_kernel(const Tin* __restrict__ k, Tok3 sk, const Tin* __restrict__ beta, const Tin* __restrict__ r,
                const float* __restrict__ d0, Tin* __restrict__ kw, float* __restrict__ d_final,
                float* __restrict__ rho, float* __restrict__ q_geo, int B, int T, int H, float eta, int anchor)
{
    constexpr int PER = DK / 32;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= B * H) return;
    const int b = unit / H, h = unit % H;

    float d[PER];
    if (d0) {
        VecIO<PER, float>::load(d0 + (size_t)unit * DK + lane * PER, d);
    } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) d[i] = 1.f;
    }

    float da[PER];                                   // retention target: d0 (anchored APF) or 0
#pragma unroll
    for (int i = 0; i < PER; ++i) da[i] = anchor ? d[i] : 0.f;
    const size_t tok_stride = (size_t)H;             // [B, T, H] index step per token
    size_t tok = (size_t)b * T * H + h;              // token (b, 0, h)
    float kc[PER], kn[PER];
    float bc = 0.f, rc = 1.f, bn = 0.f, rn = 1.f;
    float log_rho = 0.f;                             // sum over tokens of log rho_t
    if (T > 0) {
        VecIO<PER, Tin>::load(k + sk.at(b, 0, h) + lane * PER, kc);
        bc = to_f32(beta[tok]);
        if (r) rc = to_f32(r[tok]);
    }
    for (int t = 0; t < T; ++t) {
        const size_t nxt = tok + tok_stride;
        if (t + 1 < T) {                               // prefetch the next token
            VecIO<PER, Tin>::load(k + sk.at(b, t + 1, h) + lane * PER, kn);
            bn = to_f32(beta[nxt]);
            if (r) rn = to_f32(r[nxt]);
        }
        float a[PER], kwv[PER];
        float n = 0.f, s = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            a[i] = kc[i] * kc[i];
            n += a[i];
            s += d[i] * a[i];
            kwv[i] = d[i] * kc[i];
        }
        VecIO<PER, Tin>::store(kw + tok * DK + lane * PER, kwv);
        n = warp_sum(n);
        s = warp_sum(s);
        const float x = (n > 0.f) ? eta * bc * (1.f - bc * s) / n : 0.f;
        if (rho || q_geo) {
            const float rt = (1.f - bc * s) * (1.f - bc * s);
            if (rho && lane == 0) rho[tok] = rt;
            log_rho += logf(rt);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) d[i] = rc * d[i] + (1.f - rc) * da[i] + x * a[i];
        tok = nxt;
#pragma unroll
        for (int i = 0; i < PER; ++i) kc[i] = kn[i];
        bc = bn; rc = rn;
    }
    if (d_final) VecIO<PER, float>::store(d_final + (size_t)unit * DK + lane * PER, d);
    if (q_geo && lane == 0) q_geo[unit] = T > 0 ? expf(log_rho / (float)T) : 1.f;
}

}  // namespace osdn
