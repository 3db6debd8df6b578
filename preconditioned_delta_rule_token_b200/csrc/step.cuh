// Single-token recurrent decode: one CTA per (sequence, head), S streamed from
// HBM once (read) and written once, kept in registers in between.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1 (scaled write key) and sections
// 2.2-2.3 (preconditioner step), for one token:
//   kw = d (.) k,  e = S k - v,  S' = S - beta e kw^T,
//   o  = S' q = S q - beta e <kw, q>,
//   d' = r d + eta beta (1 - beta <d, k^2>) k^2 / ||k||^2
//   (anchored APF: r d + (1 - r) d_anchor + the same step);
// gated (alpha non-NULL): S is first decayed, S <- alpha S, then the step above.
// Warp w owns rows w, w + 8, ... of S; lane l owns columns [l*PER, l*PER+PER).
// The kernel is HBM-bound: 2 * dv * dk * 4 bytes of state per head and token.
#pragma once
#include "common.cuh"

namespace osdn {

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256)
step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
            const Tin* __restrict__ beta, const Tin* __restrict__ r,
            float* __restrict__ S, float* __restrict__ d, Tin* __restrict__ out, float eta,
            int anchor, const float* __restrict__ d_anchor, const Tin* __restrict__ alpha)
{
    constexpr int PER = DK / 32;
    constexpr int NW = 8;
    constexpr int ROWS = DV / NW;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t unit = blockIdx.x;
    float* Su = S + unit * (size_t)DV * DK;

    float Sr[ROWS][PER];
#pragma unroll
    for (int j = 0; j < ROWS; ++j)
        VecIO<PER, float>::load(Su + (size_t)(warp + NW * j) * DK + lane * PER, Sr[j]);

    if (alpha) {   // gated: the write applies to the decayed state alpha S
        const float a = to_f32(alpha[unit]);
#pragma unroll
        for (int j = 0; j < ROWS; ++j)
#pragma unroll
            for (int i = 0; i < PER; ++i) Sr[j][i] *= a;
    }

    float kk[PER], qq[PER], dd[PER];
    VecIO<PER, Tin>::load(k + unit * DK + lane * PER, kk);
    VecIO<PER, Tin>::load(q + unit * DK + lane * PER, qq);
    VecIO<PER, float>::load(d + unit * DK + lane * PER, dd);
    const float bt = to_f32(beta[unit]);
    const float rt = r ? to_f32(r[unit]) : 1.f;

    float n = 0.f, s = 0.f, wq = 0.f, kw[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const float a = kk[i] * kk[i];
        n += a;
        s += dd[i] * a;
        kw[i] = dd[i] * kk[i];
        wq += kw[i] * qq[i];
    }
    n = warp_sum(n);
    s = warp_sum(s);
    wq = warp_sum(wq);

#pragma unroll
    for (int j = 0; j < ROWS; ++j) {
        const int row = warp + NW * j;
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            sk = fmaf(Sr[j][i], kk[i], sk);
            sq = fmaf(Sr[j][i], qq[i], sq);
        }
        sk = warp_sum(sk);
        sq = warp_sum(sq);
        const float be = bt * (sk - to_f32(v[unit * DV + row]));
#pragma unroll
        for (int i = 0; i < PER; ++i) Sr[j][i] = fmaf(-be, kw[i], Sr[j][i]);
        if (lane == 0) out[unit * DV + row] = from_f32<Tin>(sq - be * wq);
        VecIO<PER, float>::store(Su + (size_t)row * DK + lane * PER, Sr[j]);
    }

    __syncthreads();   // every warp has read d before warp 0 overwrites it
    if (warp == 0) {
        const float x = (n > 0.f) ? eta * bt * (1.f - bt * s) / n : 0.f;
        float da[PER];   // retention target: d_anchor (ones when NULL) under anchored APF, else 0
        if (anchor && d_anchor) {
            VecIO<PER, float>::load(d_anchor + unit * DK + lane * PER, da);
        } else {
#pragma unroll
            for (int i = 0; i < PER; ++i) da[i] = anchor ? 1.f : 0.f;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) dd[i] = rt * dd[i] + (1.f - rt) * da[i] + x * (kk[i] * kk[i]);
        VecIO<PER, float>::store(d + unit * DK + lane * PER, dd);
    }
}

}  // namespace osdn
