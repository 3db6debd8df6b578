// Phase 2 split along the sequence for shapes with few (sequence, head) units.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary section 2.1: per chunk the state update is
// S <- S + (U0 - W S^T)^T Kw = S (I - W^T Kw) + U0^T Kw, affine in S (gated:
// S <- gamma_C S (...) + ..., still affine). Over a segment of chunks, then,
//   S_end = S_start E + L,
// with L the segment's end state when it starts from S = 0 and E its end state
// when it starts from S = I with V = 0. A sequence cut into P segments of equal
// length is P independent sequences in memory ([B, T, H, d] is
// [B P, T / P, H, d]), so the chunk kernel runs all segments at once, three
// times: for L (S0 = 0), for E (S0 = I, V read as zeros) and, once the start
// states S_start(p + 1) = S_start(p) E_p + L_p are combined, for the outputs.
// With one sequence (B = 1) any run of consecutive segments is itself a dense
// [n, T / P, H, d] tensor, so the passes can also go batch by batch while the
// scan is still working on later segments. With enough SMs for both phases at
// once, the phases can also simply alternate over the segments on two streams
// (phase 2 of a segment from the state the previous one ended with, beside the
// scan of the next): no transfer passes, only the per-token tensors [B, T, H]
// reordered so that each segment of every sequence is one dense block.
#pragma once
#include <cstddef>
#include <cstdint>

namespace osdn {
namespace seg {

// S [units][D][D] = I for every unit.
__global__ void identity_kernel(float* __restrict__ S, size_t units, int D) {
    const size_t n = units * (size_t)D * D;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        S[i] = ((i / D) % D == i % D) ? 1.f : 0.f;
}

// Up to three per-token tensors [B, T, H] (bf16) reordered segment-major, [P][B][T / P][H], so that
// segment s of every sequence is the dense [B, T / P, H] block at s B (T / P) H. Rows of T / P H
// elements are whole 16-byte words (T / P a multiple of 64): copied as uint4.
struct SegGather {
    const uint4* src[3];   // NULL entries are skipped
    uint4* dst[3];
};
__global__ void gather_kernel(SegGather g, int B, int T, int H, int P) {
    const size_t row = (size_t)(T / P) * H / 8;           // words of one (segment, sequence) row
    const size_t n = (size_t)B * T * H / 8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t r = i / row, w = i % row;            // destination row r = s B + b
        const size_t s = r / B, b = r % B;
        const size_t j = (b * P + s) * row + w;           // word w of segment s of sequence b in [B, T, H]
#pragma unroll
        for (int a = 0; a < 3; ++a)
            if (g.src[a]) g.dst[a][i] = g.src[a][j];
    }
}

constexpr int kRows = 16;       // rows of S per CTA of the combine
constexpr int kThreads = 256;

template <int D>
struct CombineSmem {
    static constexpr size_t kBytes = sizeof(float) * (size_t)(D * D + kRows * D);
};

// Start states of segments p0 .. p0 + n - 1 of every sequence and the state after them:
//   S_start(p0) = S0 (zeros when NULL),  S_start(p + 1) = S_start(p) E_p + L_p,
//   S_after = S_start(p0 + n - 1) E + L of that segment  (skipped when NULL).
// S0 and S_after are [B, H, D, D]; E, L and S_start are [B P, H, D, D] with segment p of
// sequence b at index b P + p. (p0 = 0, n = P: every start state and the final state.)
// Rows of S are independent, so CTA (unit, y) takes rows 16 y .. 16 y + 15 of unit b H + h;
// every thread owns one row and 8 columns of the product.
template <int D>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const float* __restrict__ S0, const float* __restrict__ E, const float* __restrict__ L,
               float* __restrict__ S_start, float* __restrict__ S_after, int H, int P, int p0, int n)
{
    static_assert(kThreads == kRows * (D / 8), "one thread per row and 8 columns");
    extern __shared__ float sm[];
    float* Es = sm;                  // [D][D] E_p
    float* Ss = Es + D * D;          // [kRows][D] rows of the running state
    const int unit = blockIdx.x, b = unit / H, h = unit % H, r0 = blockIdx.y * kRows;
    const int tid = threadIdx.x, r = tid / (D / 8), c0 = (tid % (D / 8)) * 8;
    for (int i = tid; i < kRows * D; i += kThreads)
        Ss[i] = S0 ? S0[((size_t)unit * D + r0 + i / D) * D + i % D] : 0.f;
    for (int p = p0; p < p0 + n; ++p) {
        const size_t su = ((size_t)b * P + p) * H + h;
        __syncthreads();             // Ss holds S_start(p); every thread is done with Es
        for (int i = tid; i < kRows * D; i += kThreads) S_start[(su * D + r0 + i / D) * D + i % D] = Ss[i];
        const float4* eg = reinterpret_cast<const float4*>(E + su * D * D);
        for (int i = tid; i < D * D / 4; i += kThreads) reinterpret_cast<float4*>(Es)[i] = eg[i];
        __syncthreads();
        float acc[8];
        const float* lrow = L + (su * D + r0 + r) * D + c0;
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = lrow[j];
#pragma unroll 4
        for (int kk = 0; kk < D; ++kk) {
            const float s = Ss[r * D + kk];
            const float4 e0 = *reinterpret_cast<const float4*>(Es + kk * D + c0);
            const float4 e1 = *reinterpret_cast<const float4*>(Es + kk * D + c0 + 4);
            acc[0] = fmaf(s, e0.x, acc[0]); acc[1] = fmaf(s, e0.y, acc[1]);
            acc[2] = fmaf(s, e0.z, acc[2]); acc[3] = fmaf(s, e0.w, acc[3]);
            acc[4] = fmaf(s, e1.x, acc[4]); acc[5] = fmaf(s, e1.y, acc[5]);
            acc[6] = fmaf(s, e1.z, acc[6]); acc[7] = fmaf(s, e1.w, acc[7]);
        }
        __syncthreads();             // every thread has read its row of Ss
#pragma unroll
        for (int j = 0; j < 8; ++j) Ss[r * D + c0 + j] = acc[j];
    }
    __syncthreads();
    if (S_after)
        for (int i = tid; i < kRows * D; i += kThreads) S_after[((size_t)unit * D + r0 + i / D) * D + i % D] = Ss[i];
}

}  // namespace seg
}  // namespace osdn
