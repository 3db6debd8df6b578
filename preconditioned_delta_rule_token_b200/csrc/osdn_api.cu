// Host side of libosdn.so: argument checks, workspace layout and kernel
// launches behind the C ABI declared in include/osdn.h.  Nothing here
// allocates device memory or synchronises the host (except osdn_sync_status).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstddef>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>
#include <type_traits>

#include "osdn.h"

#include "bwd.cuh"
#include "chunk_ffma.cuh"
#include "chunk_wy.cuh"
#include "scan_ws.cuh"
#include "scan_seq.cuh"
#include "segments.cuh"
#include "step.cuh"

namespace {

thread_local std::string t_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(OSDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t elem_size(int dtype) { return dtype == OSDN_BF16 ? 2 : 4; }

// Common checks of the parameter block. need_T: the forward (T used).
// Versions 1 and 2 of osdn_params ended after eta and after apf_anchor; their callers get the fields
// added since at their defaults.
constexpr size_t kParamsV1Size = offsetof(osdn_params, apf_anchor);
constexpr size_t kParamsV2Size = offsetof(osdn_params, stride_q);
int anchor_of(const osdn_params* p) {
    return p->struct_size >= offsetof(osdn_params, apf_anchor) + sizeof(int32_t) && p->apf_anchor ? 1 : 0;
}

// Element strides of a token tensor [B, T, H, width] over (b, t, h), the caller's or the dense ones.
int64_t all_zero(const int64_t (&s)[3]) { return !(s[0] | s[1] | s[2]); }
osdn::Tok3 dense_tok3(const osdn_params* p, int width) {
    return {(int64_t)p->T * p->H * width, (int64_t)p->H * width, (int64_t)width};
}
osdn::Tok3 tok3_of(const osdn_params* p, const int64_t (&s)[3], int width) {
    if (p->struct_size < sizeof(osdn_params) || all_zero(s)) return dense_tok3(p, width);
    return {s[0], s[1], s[2]};
}
struct TokStrides {
    osdn::Tok3 q, k, v, o;
};
TokStrides strides_of(const osdn_params* p) {
    return {tok3_of(p, p->stride_q, p->dk), tok3_of(p, p->stride_k, p->dk), tok3_of(p, p->stride_v, p->dv),
            tok3_of(p, p->stride_o, p->dv)};
}
// True when every stride the caller gave is the dense one (or none was given).
bool dense_layout(const osdn_params* p) {
    const TokStrides s = strides_of(p);
    auto same = [](const osdn::Tok3& a, const osdn::Tok3& b) { return a.b == b.b && a.t == b.t && a.h == b.h; };
    return same(s.q, dense_tok3(p, p->dk)) && same(s.k, dense_tok3(p, p->dk)) && same(s.v, dense_tok3(p, p->dv)) &&
           same(s.o, dense_tok3(p, p->dv));
}

int check_params(const osdn_params* p, bool need_T) {
    if (!p) return fail(OSDN_ERR_INVALID_ARG, "params is NULL");
    if (p->struct_size != sizeof(osdn_params) && p->struct_size != kParamsV2Size && p->struct_size != kParamsV1Size)
        return fail(OSDN_ERR_INVALID_ARG, "params.struct_size is %u, expected %zu (or %zu, %zu: versions 2, 1)",
                    p->struct_size, sizeof(osdn_params), kParamsV2Size, kParamsV1Size);
    if (p->B < 1 || p->H < 1) return fail(OSDN_ERR_INVALID_ARG, "B and H must be >= 1 (got %d, %d)", p->B, p->H);
    if (need_T && p->T < 0) return fail(OSDN_ERR_INVALID_ARG, "T must be >= 0 (got %d)", p->T);
    if (p->dtype != OSDN_BF16 && p->dtype != OSDN_FP32)
        return fail(OSDN_ERR_INVALID_ARG, "unknown dtype %d", p->dtype);
    if (p->dk <= 0 || p->dv <= 0) return fail(OSDN_ERR_INVALID_ARG, "dk and dv must be positive");
    if ((p->dk != 64 && p->dk != 128) || (p->dv != 64 && p->dv != 128))
        return fail(OSDN_ERR_UNSUPPORTED, "dk, dv must be 64 or 128 (got %d, %d)", p->dk, p->dv);
    if (need_T && p->chunk != 64) return fail(OSDN_ERR_UNSUPPORTED, "chunk must be 64 (got %d)", p->chunk);
    if (!(p->eta == p->eta)) return fail(OSDN_ERR_INVALID_ARG, "eta is NaN");
    const double tokens = (double)p->B * (double)(need_T ? p->T : 1) * (double)p->H;
    if (tokens * (double)(p->dk > p->dv ? p->dk : p->dv) > 9.0e18)
        return fail(OSDN_ERR_INVALID_ARG, "tensor sizes overflow 64-bit indexing");
    if ((double)p->B * p->H > 2147483647.0) return fail(OSDN_ERR_INVALID_ARG, "B * H exceeds the grid limit");
    if (p->struct_size >= sizeof(osdn_params)) {
        const int64_t* all[4] = {p->stride_q, p->stride_k, p->stride_v, p->stride_o};
        for (const int64_t* st : all)
            for (int i = 0; i < 3; ++i)
                if (st[i] < 0 || (st[i] & 7) || st[i] > ((int64_t)1 << 38))
                    return fail(OSDN_ERR_INVALID_ARG,
                                "strides must be non-negative multiples of 8 elements below 2^38 (got %lld)",
                                (long long)st[i]);
    }
    return OSDN_OK;
}

// Number of segments phase 2 cuts each sequence into (1: none). Only the tensor-core path
// (bf16, dk = dv = 128, dense tensors) splits, and only when the (b, h) units leave most SMs idle:
// P is the largest power of two up to 16 with units * P <= SMs, then lowered until the segments
// are whole 64-token chunks of at least 512 tokens; below 4 segments the three passes cost more
// than they save.
int sm_count() {
    int sms = 148, dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        sms = n;
    else
        (void)cudaGetLastError();   // no device (host-only use): keep the B200 count
    return sms;
}

// Segments per batch of the overlapped forward (one sequence, H heads): its own-end-state and
// transfer passes run side by side next to the scan, so 2 n H + H CTAs must fit the SMs.
int overlap_batch(int H, int P) {
    const int nb = (sm_count() - H) / (2 * H);
    return nb < P / 2 ? nb : P / 2;
}

int seg_count(const osdn_params* p) {
    if (p->dtype != OSDN_BF16 || p->dk != 128 || p->dv != 128 || p->T <= 0 || !dense_layout(p)) return 1;
    const int sms = sm_count();
    if (p->B == 1 && !anchor_of(p) && p->T % 1024 == 0 && p->T / 16 >= 512 && overlap_batch(p->H, 16) >= 1)
        return 16;   // one sequence, overlapped with the scan: short segments keep the tail after the scan short
    const long long units = (long long)p->B * p->H;
    int P = 1;
    while (P < 16 && units * P * 2 <= sms) P *= 2;
    while (P >= 4 && (p->T % (64 * P) != 0 || p->T / P < 512)) P /= 2;
    return P >= 4 ? P : 1;
}

// Segments of the pipelined forward (1: none). When phase 2 is not split and the (b, h) units
// take at most half the SMs, osdn_fwd cuts each sequence into P segments and runs the scan of
// segment s + 1 beside phase 2 of segment s, each on its own SMs; phase 2 of a segment starts
// from the state the previous one ended with, so no transfer passes are needed. Every launch of
// phase 2 pays its own pipeline fill and drain (about three chunks), so segments stay long: four
// when each keeps at least 1024 tokens, else two of at least 512. Not with the anchored
// preconditioner (its anchor is the d of the whole sequence's start).
constexpr int kMaxPipe = 4;
int pipe_count(const osdn_params* p) {
    if (p->dtype != OSDN_BF16 || p->dk != 128 || p->dv != 128 || p->T <= 0 || !dense_layout(p) || anchor_of(p))
        return 1;
    if (seg_count(p) > 1 || 2LL * p->B * p->H > sm_count()) return 1;
    for (int P = kMaxPipe; P >= 2; P /= 2)
        if (p->T % (64 * P) == 0 && p->T / P >= (P > 2 ? 1024 : 512)) return P;
    return 1;
}

// The forward's workspace: the scaled write keys, then (segmented phase 2 only) the start
// states, end states and transfers of every segment, fp32 [B P, H, dv, dk] each, and a 64-token
// tile of zeros that the transfer pass reads as V. When osdn_fwd also overlaps the scan with
// phase 2 (one sequence, plain APF): identity start states for the transfer passes of one batch,
// d after every segment, and an output tile for the transfer passes of one batch. When it
// pipelines the scan with phase 2 instead (few units, phase 2 not split): beta, r and alpha
// segment-major, and two buffers each for the state and d handed from segment to segment (the
// scaled write keys are then segment-major too).
struct WorkspaceLayout {
    size_t kw_off, kw_bytes, total;
    int seg;                       // segments per sequence (1: phase 2 is not split)
    size_t seg_S, seg_L, seg_E, seg_Z;
    bool overlap;                  // osdn_fwd runs the scan segment by segment, phase 2 alongside
    int ov_batch;                  // segments per batch of the overlapped passes
    size_t ov_I, ov_D, ov_O;
    int pipe;                      // segments of the pipelined forward (1: not pipelined)
    size_t pp_in[3];               // beta, r, alpha segment-major [P][B][T / P][H]
    size_t pp_S, pp_D;             // two state and two d buffers [B, H, dv, dk], [B, H, dk] fp32
};

WorkspaceLayout layout_of(const osdn_params* p) {
    WorkspaceLayout L{};
    L.kw_off = 0;
    L.kw_bytes = (size_t)p->B * (size_t)p->T * (size_t)p->H * (size_t)p->dk * elem_size(p->dtype);
    L.total = round_up(L.kw_bytes, 256);
    L.seg = seg_count(p);
    if (L.seg > 1) {
        const size_t st = (size_t)p->B * L.seg * p->H * p->dv * p->dk * sizeof(float);
        L.seg_S = L.total;
        L.seg_L = L.seg_S + st;
        L.seg_E = L.seg_L + st;
        L.seg_Z = L.seg_E + st;
        L.total = L.seg_Z + 64 * 128 * sizeof(__nv_bfloat16);
        L.ov_batch = p->B == 1 && !anchor_of(p) ? overlap_batch(p->H, L.seg) : 0;
        L.overlap = L.ov_batch >= 1;
        if (L.overlap) {
            const size_t seg_tokens = (size_t)p->T / L.seg * p->H;
            const size_t batch_states = (size_t)L.ov_batch * p->H * p->dv * p->dk * sizeof(float);
            L.ov_I = round_up(L.total, 256);
            L.ov_D = L.ov_I + batch_states;
            L.ov_O = round_up(L.ov_D + (size_t)L.seg * p->H * p->dk * sizeof(float), 256);
            L.total = L.ov_O + (size_t)L.ov_batch * seg_tokens * p->dv * sizeof(__nv_bfloat16);
        }
    }
    L.pipe = pipe_count(p);
    if (L.pipe > 1) {
        const size_t units = (size_t)p->B * p->H;
        for (int a = 0; a < 3; ++a) {
            L.pp_in[a] = L.total;
            L.total = round_up(L.total + (size_t)p->B * p->T * p->H * sizeof(__nv_bfloat16), 256);
        }
        L.pp_S = L.total;
        L.pp_D = L.pp_S + 2 * units * p->dv * p->dk * sizeof(float);
        L.total = round_up(L.pp_D + 2 * units * p->dk * sizeof(float), 256);
    }
    if (L.total == 0) L.total = 256;
    return L;
}

__global__ void fill_ones_kernel(float* x, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        x[i] = 1.f;
}

int copy_initial_state(const osdn_params* p, const float* d0, const float* S0, float* final_S, float* final_d,
                       bool want_S, bool want_d, cudaStream_t st) {
    const size_t units = (size_t)p->B * p->H;
    cudaError_t e;
    if (want_S && final_S) {
        const size_t bytes = units * p->dv * p->dk * sizeof(float);
        e = S0 ? cudaMemcpyAsync(final_S, S0, bytes, cudaMemcpyDeviceToDevice, st)
               : cudaMemsetAsync(final_S, 0, bytes, st);
        if (e != cudaSuccess) return cuda_fail(e, "initial state copy");
    }
    if (want_d && final_d) {
        const size_t n = units * p->dk;
        if (d0) {
            e = cudaMemcpyAsync(final_d, d0, n * sizeof(float), cudaMemcpyDeviceToDevice, st);
        } else {
            const size_t blocks = (n + 255) / 256;
            fill_ones_kernel<<<(unsigned)(blocks > 1024 ? 1024 : blocks), 256, 0, st>>>(final_d, n);
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) return cuda_fail(e, "initial preconditioner copy");
    }
    return OSDN_OK;
}

// Upper bound on any single device-side wait of the tensor-core kernels.
std::atomic<unsigned long long> g_wait_limit_ns{4000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 4-D bf16 tensor map over [B, T, H, width] (dims listed innermost first) with element strides s
// over (b, t, h), box {box0, 1, box_tokens, 1}. The token dimension is its own dimension, so a box
// that runs past T reads zeros instead of the next sequence.
int make_token_map(CUtensorMap* m, const void* base, int B, int T, int H, int width, int box0,
                   CUtensorMapSwizzle swizzle, int box_tokens, osdn::Tok3 s) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(OSDN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[4] = {(cuuint64_t)width, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)s.h * 2, (cuuint64_t)s.t * 2, (cuuint64_t)s.b * 2};
    const cuuint32_t box[4] = {(cuuint32_t)box0, 1, (cuuint32_t)box_tokens, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OSDN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return OSDN_OK;
}

// Phase 2 on the tensor cores (WY form, state chain fed by prepared W and U0): bf16, dk = dv = 128.
// v_zero: v is one 64-token tile of zeros [64][128] and V is read as zeros everywhere (the map
// covers only that tile; every other chunk and head lies outside it and is filled with zeros).
int launch_chunk_wy(const osdn_params* p, const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                    const __nv_bfloat16* beta, const float* S0, __nv_bfloat16* out, float* final_S,
                    const __nv_bfloat16* kw, cudaStream_t st, const __nv_bfloat16* alpha = nullptr,
                    bool v_zero = false) {
    CUtensorMap mq, mk, mkw, mv, mo;
    const TokStrides s = strides_of(p);
    const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
    int rc;
    if ((rc = make_token_map(&mq, q, p->B, p->T, p->H, 128, 64, sw, 64, s.q))) return rc;
    if ((rc = make_token_map(&mk, k, p->B, p->T, p->H, 128, 64, sw, 64, s.k))) return rc;
    if ((rc = make_token_map(&mkw, kw, p->B, p->T, p->H, 128, 64, sw, 64, dense_tok3(p, 128)))) return rc;
    if (v_zero) rc = make_token_map(&mv, v, 1, 64, 1, 128, 64, sw, 64, osdn::Tok3{64 * 128, 128, 128});
    else rc = make_token_map(&mv, v, p->B, p->T, p->H, 128, 64, sw, 64, s.v);
    if (rc) return rc;
    if ((rc = make_token_map(&mo, out, p->B, p->T, p->H, 128, 64, sw, 64, s.o))) return rc;
    auto kern = alpha ? osdn::chunk_wy_kernel<true> : osdn::chunk_wy_kernel<false>;
    const size_t smem = osdn::WyLayout::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core chunk kernel attribute");
    kern<<<p->B * p->H, osdn::WyLayout::kThreads, smem, st>>>(mq, mk, mkw, mv, mo, beta, alpha, S0, final_S, p->B,
                                                             p->T, p->H,
                                         g_wait_limit_ns.load());
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tensor-core chunk launch");
    return OSDN_OK;
}

// Phase 2 on the tensor cores with each sequence cut into L.seg segments (segments.cuh): the
// chunk kernel over [B P, T / P] for the segments' own end states (S0 = 0) and transfers
// (S0 = I, V = 0), the combine of the start states and final states, and the chunk kernel
// again from those start states for the outputs. The first two passes also write out; the
// last one overwrites it.
int launch_chunk_wy_segmented(const osdn_params* p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                              const __nv_bfloat16* v, const __nv_bfloat16* beta, const __nv_bfloat16* alpha,
                              const float* S0, __nv_bfloat16* out, float* final_S, const __nv_bfloat16* kw,
                              char* ws, const WorkspaceLayout& L, cudaStream_t st) {
    const int P = L.seg;
    osdn_params ps = *p;                       // the segments as B P sequences of T / P tokens (dense)
    ps.B = p->B * P;
    ps.T = p->T / P;
    if (ps.struct_size >= sizeof(osdn_params))
        for (int i = 0; i < 3; ++i) ps.stride_q[i] = ps.stride_k[i] = ps.stride_v[i] = ps.stride_o[i] = 0;
    float* Sst = reinterpret_cast<float*>(ws + L.seg_S);
    float* Lb = reinterpret_cast<float*>(ws + L.seg_L);
    float* Eb = reinterpret_cast<float*>(ws + L.seg_E);
    auto* Z = reinterpret_cast<__nv_bfloat16*>(ws + L.seg_Z);
    const size_t units_s = (size_t)ps.B * ps.H;
    cudaError_t e = cudaMemsetAsync(Z, 0, 64 * 128 * sizeof(__nv_bfloat16), st);
    if (e != cudaSuccess) return cuda_fail(e, "segment zero tile");
    osdn::seg::identity_kernel<<<1024, 256, 0, st>>>(Sst, units_s, 128);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "segment identity launch");
    int rc;
    if ((rc = launch_chunk_wy(&ps, q, k, v, beta, nullptr, out, Lb, kw, st, alpha))) return rc;
    if ((rc = launch_chunk_wy(&ps, q, k, Z, beta, Sst, out, Eb, kw, st, alpha, true))) return rc;
    auto comb = osdn::seg::combine_kernel<128>;
    const size_t smem = osdn::seg::CombineSmem<128>::kBytes;
    if ((e = cudaFuncSetAttribute(comb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return cuda_fail(e, "segment combine attribute");
    comb<<<dim3((unsigned)(p->B * p->H), 128 / osdn::seg::kRows), osdn::seg::kThreads, smem, st>>>(
        S0, Eb, Lb, Sst, final_S, p->H, P, 0, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "segment combine launch");
    return launch_chunk_wy(&ps, q, k, v, beta, Sst, out, nullptr, kw, st, alpha);
}

// Two non-blocking streams per device for the overlapped forward, created on first use and
// kept for the life of the process (a fork from and a join back to the caller's stream by
// events around every use).
int side_streams(cudaStream_t out[2]) {
    static std::mutex mu;
    static cudaStream_t streams[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "current device");
    if (dev < 0 || dev >= 64) return fail(OSDN_ERR_UNSUPPORTED, "device index %d above 63", dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 2; ++i)
        if (!streams[dev][i] && (e = cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "side stream");
    out[0] = streams[dev][0];
    out[1] = streams[dev][1];
    return OSDN_OK;
}

template <typename Tin>
int launch_scan(const osdn_params* p, const Tin* k, const Tin* beta, const Tin* r, const float* d0, float* final_d,
                Tin* kw, cudaStream_t st, float* rho = nullptr, float* q_geo = nullptr);

// osdn_fwd for one sequence (B = 1) split into P segments, with the scan overlapped with phase 2
// (segments.cuh). Segments 0 .. P - 2 go in batches of L.ov_batch. The caller's stream runs the
// scan batch by batch and then over the last segment, each launch from the d the previous one
// ended with. As soon as the scan has covered a batch, two side streams run its passes for the
// own end states and the transfers
// side by side, then the first side stream combines the batch's start states and runs its output
// pass; the output pass of the last batch also covers the last segment, after the scan ends, and
// that segment's end state is the final state. Consecutive segments of one sequence are a dense
// [n, T / P, H, d] tensor, so every launch is the existing scan or chunk kernel on such a view.
int launch_fwd_overlapped(const osdn_params* p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const __nv_bfloat16* beta, const __nv_bfloat16* r,
                          const __nv_bfloat16* alpha, const float* d0, const float* S0, __nv_bfloat16* out,
                          float* final_S, float* final_d, char* ws, const WorkspaceLayout& L, cudaStream_t st) {
    using T = __nv_bfloat16;
    const int P = L.seg, nb = L.ov_batch, H = p->H, D = 128;
    const int nbatch = (P - 1 + nb - 1) / nb;             // batches over segments 0 .. P - 2
    const int Ls = p->T / P;
    const size_t segtok = (size_t)Ls * H;                 // token-heads per segment
    const size_t sstate = (size_t)H * D * D;               // floats of one segment's states
    auto view = [&](int nseg) {                            // nseg consecutive segments as a dense tensor
        osdn_params v_ = *p;
        v_.B = nseg;
        v_.T = Ls;
        if (v_.struct_size >= sizeof(osdn_params))
            for (int i = 0; i < 3; ++i) v_.stride_q[i] = v_.stride_k[i] = v_.stride_v[i] = v_.stride_o[i] = 0;
        return v_;
    };
    T* kw = reinterpret_cast<T*>(ws + L.kw_off);
    float* Sst = reinterpret_cast<float*>(ws + L.seg_S);
    float* Lb = reinterpret_cast<float*>(ws + L.seg_L);
    float* Eb = reinterpret_cast<float*>(ws + L.seg_E);
    T* Z = reinterpret_cast<T*>(ws + L.seg_Z);
    float* Sid = reinterpret_cast<float*>(ws + L.ov_I);
    float* dseg = reinterpret_cast<float*>(ws + L.ov_D);
    T* Oe = reinterpret_cast<T*>(ws + L.ov_O);
    auto at = [&](auto* base, int seg, int width) { return base + (size_t)seg * segtok * width; };
    auto tok = [&](const T* base, int seg) { return base ? base + (size_t)seg * segtok : nullptr; };

    cudaStream_t side[2];
    int rc = side_streams(side);
    if (rc) return rc;
    // events: fork, scan end, join, and per batch: scanned, transfers done
    const int nev = 3 + 2 * nbatch;
    cudaEvent_t ev[3 + 2 * 16];
    cudaError_t e = cudaSuccess;
    int made = 0;
    for (; made < nev; ++made)
        if ((e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming)) != cudaSuccess) break;
    if (e != cudaSuccess) {
        for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
        return cuda_fail(e, "event");
    }
    cudaEvent_t ev_fork = ev[0], ev_scanned_all = ev[1], ev_join = ev[2];
    auto ev_scanned = [&](int bt) { return ev[3 + 2 * bt]; };
    auto ev_transfers = [&](int bt) { return ev[4 + 2 * bt]; };
    auto chk = [&](cudaError_t x, const char* what) { return x == cudaSuccess ? OSDN_OK : cuda_fail(x, what); };
    do {
        // fork: the side streams start after everything before this call on the caller's stream
        if ((rc = chk(cudaEventRecord(ev_fork, st), "fork"))) break;
        if ((rc = chk(cudaStreamWaitEvent(side[0], ev_fork, 0), "fork"))) break;
        if ((rc = chk(cudaStreamWaitEvent(side[1], ev_fork, 0), "fork"))) break;
        if ((rc = chk(cudaMemsetAsync(Z, 0, 64 * 128 * sizeof(T), side[1]), "segment zero tile"))) break;
        osdn::seg::identity_kernel<<<1024, 256, 0, side[1]>>>(Sid, (size_t)nb * H, D);
        if ((rc = chk(cudaGetLastError(), "segment identity launch"))) break;
        // the scan on the caller's stream: one launch per batch (its segments as one run of tokens),
        // then one for the last segment; d after each launch goes to the next, an event after each batch
        for (int bt = 0; bt <= nbatch && !rc; ++bt) {
            const int s0 = bt == nbatch ? P - 1 : bt * nb;
            const int s1 = bt == nbatch ? P : (s0 + nb < P - 1 ? s0 + nb : P - 1);
            osdn_params run = view(1);
            run.T = (s1 - s0) * Ls;
            const float* din = bt == 0 ? d0 : dseg + (size_t)(bt - 1) * H * D;
            float* dout = bt == nbatch ? final_d : dseg + (size_t)bt * H * D;
            rc = launch_scan<T>(&run, at(k, s0, D), tok(beta, s0), tok(r, s0), din, dout, at(kw, s0, D), st);
            if (!rc && bt < nbatch) rc = chk(cudaEventRecord(ev_scanned(bt), st), "scan event");
        }
        if (rc) break;
        if ((rc = chk(cudaEventRecord(ev_scanned_all, st), "scan event"))) break;
        auto comb = osdn::seg::combine_kernel<128>;
        const size_t csm = osdn::seg::CombineSmem<128>::kBytes;
        if ((rc = chk(cudaFuncSetAttribute(comb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csm),
                      "segment combine attribute")))
            break;
        for (int bt = 0; bt < nbatch && !rc; ++bt) {
            const int s0 = bt * nb, s1 = s0 + nb < P - 1 ? s0 + nb : P - 1;
            const osdn_params vw = view(s1 - s0);
            // own end states (side 0) and transfers (side 1) once the batch is scanned
            if ((rc = chk(cudaStreamWaitEvent(side[0], ev_scanned(bt), 0), "segment wait"))) break;
            if ((rc = chk(cudaStreamWaitEvent(side[1], ev_scanned(bt), 0), "segment wait"))) break;
            if ((rc = launch_chunk_wy(&vw, at(q, s0, D), at(k, s0, D), at(v, s0, D), tok(beta, s0), nullptr,
                                      at(out, s0, D), Lb + s0 * sstate, at(kw, s0, D), side[0], tok(alpha, s0))))
                break;
            if ((rc = launch_chunk_wy(&vw, at(q, s0, D), at(k, s0, D), Z, tok(beta, s0), Sid, Oe, Eb + s0 * sstate,
                                      at(kw, s0, D), side[1], tok(alpha, s0), true)))
                break;
            if ((rc = chk(cudaEventRecord(ev_transfers(bt), side[1]), "segment event"))) break;
            if ((rc = chk(cudaStreamWaitEvent(side[0], ev_transfers(bt), 0), "segment wait"))) break;
            // start states of the batch from S_start(s0) (S0 for the first), and S_start(s1) after it
            comb<<<dim3((unsigned)H, D / osdn::seg::kRows), osdn::seg::kThreads, csm, side[0]>>>(
                bt == 0 ? S0 : Sst + s0 * sstate, Eb, Lb, Sst, Sst + s1 * sstate, H, P, s0, s1 - s0);
            if ((rc = chk(cudaGetLastError(), "segment combine launch"))) break;
            // the batch's outputs; the last batch also takes the last segment once the scan is done,
            // with end states over the consumed own end states (the last one is the final state)
            const bool last = bt == nbatch - 1;
            if (last && (rc = chk(cudaStreamWaitEvent(side[0], ev_scanned_all, 0), "segment wait"))) break;
            const osdn_params vo = view(last ? P - s0 : s1 - s0);
            rc = launch_chunk_wy(&vo, at(q, s0, D), at(k, s0, D), at(v, s0, D), tok(beta, s0), Sst + s0 * sstate,
                                 at(out, s0, D), last ? Lb + s0 * sstate : nullptr, at(kw, s0, D), side[0],
                                 tok(alpha, s0));
        }
        if (rc) break;
        if (final_S &&
            (rc = chk(cudaMemcpyAsync(final_S, Lb + (P - 1) * sstate, sstate * sizeof(float),
                                      cudaMemcpyDeviceToDevice, side[0]),
                      "final state copy")))
            break;
        // join: the caller's stream waits for side 0, which has waited for every event of side 1
        if ((rc = chk(cudaEventRecord(ev_join, side[0]), "join"))) break;
        rc = chk(cudaStreamWaitEvent(st, ev_join, 0), "join");
    } while (false);
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
    return rc;
}

// osdn_fwd with each sequence cut into L.pipe segments (pipe_count): the caller's stream
// reorders beta, r and alpha segment-major and scans segment after segment, each launch from
// the d the previous one ended with; a side stream runs phase 2 of each segment once its scan
// is done, from the state the previous segment ended with. Phase 2 of segment s thus runs
// beside the scan of segment s + 1. Segment s of q, k, v and out is the [B, T / P, H, 128] view
// at token s T / P with the whole sequence's strides; its scaled write keys, beta, r and alpha
// are dense blocks of the workspace, so every launch is the existing scan or chunk kernel.
int launch_fwd_pipelined(const osdn_params* p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                         const __nv_bfloat16* v, const __nv_bfloat16* beta, const __nv_bfloat16* r,
                         const __nv_bfloat16* alpha, const float* d0, const float* S0, __nv_bfloat16* out,
                         float* final_S, float* final_d, char* ws, const WorkspaceLayout& L, cudaStream_t st) {
    using T = __nv_bfloat16;
    const int P = L.pipe, H = p->H, D = 128;
    const int Ls = p->T / P;
    const size_t segtok = (size_t)p->B * Ls * H;           // token-heads of one segment of every sequence
    const size_t units = (size_t)p->B * H;
    osdn_params vw{};                                      // one segment of every sequence
    std::memcpy(&vw, p, p->struct_size < sizeof(vw) ? p->struct_size : sizeof(vw));
    vw.struct_size = sizeof(vw);
    vw.T = Ls;
    const int64_t full[3] = {(int64_t)p->T * H * D, (int64_t)H * D, D};
    for (int i = 0; i < 3; ++i) vw.stride_q[i] = vw.stride_k[i] = vw.stride_v[i] = vw.stride_o[i] = full[i];
    auto view_at = [&](auto* base, int seg) { return base + (size_t)seg * Ls * H * D; };
    T* kw = reinterpret_cast<T*>(ws + L.kw_off);
    T* in[3] = {reinterpret_cast<T*>(ws + L.pp_in[0]), r ? reinterpret_cast<T*>(ws + L.pp_in[1]) : nullptr,
                alpha ? reinterpret_cast<T*>(ws + L.pp_in[2]) : nullptr};
    auto seg_of = [&](T* base, int seg) { return base ? base + (size_t)seg * segtok : nullptr; };
    float* Sb = reinterpret_cast<float*>(ws + L.pp_S);
    float* db = reinterpret_cast<float*>(ws + L.pp_D);

    cudaStream_t side[2];
    int rc = side_streams(side);
    if (rc) return rc;
    if (P < 2 || P > kMaxPipe) return fail(OSDN_ERR_UNSUPPORTED, "%d pipelined segments", P);
    const int nev = 2 + P;                                 // fork, join, per segment: scanned
    cudaEvent_t ev[2 + kMaxPipe];
    cudaError_t e = cudaSuccess;
    int made = 0;
    for (; made < nev; ++made)
        if ((e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming)) != cudaSuccess) break;
    if (e != cudaSuccess) {
        for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
        return cuda_fail(e, "event");
    }
    auto chk = [&](cudaError_t x, const char* what) { return x == cudaSuccess ? OSDN_OK : cuda_fail(x, what); };
    do {
        osdn::seg::SegGather g{};
        const void* src[3] = {beta, r, alpha};
        for (int a = 0; a < 3; ++a) {
            g.src[a] = in[a] ? reinterpret_cast<const uint4*>(src[a]) : nullptr;
            g.dst[a] = reinterpret_cast<uint4*>(in[a]);
        }
        const size_t words = (size_t)p->B * p->T * H / 8, blocks = (words + 255) / 256;
        osdn::seg::gather_kernel<<<(unsigned)(blocks > 1024 ? 1024 : blocks), 256, 0, st>>>(g, p->B, p->T, H, P);
        if ((rc = chk(cudaGetLastError(), "segment gather launch"))) break;
        // fork after the gather: the side stream reads the reordered beta and alpha
        if ((rc = chk(cudaEventRecord(ev[0], st), "fork"))) break;
        if ((rc = chk(cudaStreamWaitEvent(side[0], ev[0], 0), "fork"))) break;
        // enqueued segment by segment, so that phase 2 of a segment is queued as soon as its scan is
        for (int sg = 0; sg < P && !rc; ++sg) {
            const float* din = sg == 0 ? d0 : db + (size_t)((sg - 1) & 1) * units * D;
            float* dout = sg == P - 1 ? final_d : db + (size_t)(sg & 1) * units * D;
            if ((rc = launch_scan<T>(&vw, view_at(k, sg), seg_of(in[0], sg), seg_of(in[1], sg), din, dout,
                                     kw + (size_t)sg * segtok * D, st)))
                break;
            if ((rc = chk(cudaEventRecord(ev[2 + sg], st), "scan event"))) break;
            if ((rc = chk(cudaStreamWaitEvent(side[0], ev[2 + sg], 0), "segment wait"))) break;
            const float* sin = sg == 0 ? S0 : Sb + (size_t)((sg - 1) & 1) * units * D * D;
            float* sout = sg == P - 1 ? final_S : Sb + (size_t)(sg & 1) * units * D * D;
            rc = launch_chunk_wy(&vw, view_at(q, sg), view_at(k, sg), view_at(v, sg), seg_of(in[0], sg), sin,
                                 view_at(out, sg), sout, kw + (size_t)sg * segtok * D, side[0], seg_of(in[2], sg));
        }
        if (rc) break;
        if ((rc = chk(cudaEventRecord(ev[1], side[0]), "join"))) break;
        rc = chk(cudaStreamWaitEvent(st, ev[1], 0), "join");
    } while (false);
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
    return rc;
}

// Phase 1 in chunk form on the tensor cores: bf16, dk = 128.
// d_traj non-NULL: the instance that also writes d_t of every token (fp32 [B, T, H, 128]).
int launch_scan_tc(const osdn_params* p, const __nv_bfloat16* k, const __nv_bfloat16* beta,
                   const __nv_bfloat16* r, const float* d0, float* final_d, __nv_bfloat16* kw, float* rho,
                   float* q_geo, cudaStream_t st, float* d_traj = nullptr) {
    CUtensorMap mk, mkw;
    int rc = make_token_map(&mk, k, p->B, p->T, p->H, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B, 128, strides_of(p).k);
    if (rc) return rc;
    rc = make_token_map(&mkw, kw, p->B, p->T, p->H, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B, 128, dense_tok3(p, 128));
    if (rc) return rc;
    auto kern = d_traj ? osdn::scan_ws_kernel<1> : osdn::scan_ws_kernel<0>;
    const size_t smem = osdn::ScanLayout::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core scan kernel attribute");
    kern<<<p->B * p->H, 384, smem, st>>>(mk, mkw, beta, r, d0, final_d, rho, q_geo, d_traj, p->B, p->T, p->H, p->eta,
                                         anchor_of(p), g_wait_limit_ns.load());
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tensor-core scan launch");
    return OSDN_OK;
}


// Phase 1: preconditioner scan -> scaled write keys (workspace) and final d.
template <typename Tin>
int launch_scan(const osdn_params* p, const Tin* k, const Tin* beta, const Tin* r, const float* d0, float* final_d,
                Tin* kw, cudaStream_t st, float* rho, float* q_geo) {
    if (p->T == 0) {
        if (q_geo) {   // empty sequences: the geometric mean of no ratios is 1
            const size_t n = (size_t)p->B * p->H, blocks = (n + 255) / 256;
            fill_ones_kernel<<<(unsigned)(blocks > 1024 ? 1024 : blocks), 256, 0, st>>>(q_geo, n);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return cuda_fail(e, "q_geo fill");
        }
        return copy_initial_state(p, d0, nullptr, nullptr, final_d, false, true, st);
    }
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        if (p->dk == 128) return launch_scan_tc(p, k, beta, r, d0, final_d, kw, rho, q_geo, st);
    }
    const int units = p->B * p->H;
    const dim3 grid((units + 3) / 4);
    const osdn::Tok3 sk = strides_of(p).k;
    if (p->dk == 128)
        osdn::scan_seq_kernel<128, Tin><<<grid, 128, 0, st>>>(k, sk, beta, r, d0, kw, final_d, rho, q_geo, p->B, p->T,
                                                               p->H, p->eta, anchor_of(p));
    else
        osdn::scan_seq_kernel<64, Tin><<<grid, 128, 0, st>>>(k, sk, beta, r, d0, kw, final_d, rho, q_geo, p->B, p->T,
                                                              p->H, p->eta, anchor_of(p));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    return OSDN_OK;
}

// Phase 2: chunkwise delta rule with the scaled write key.
// ws: the whole workspace when phase 2 may use its segment scratch (NULL: never split).
template <typename Tin>
int launch_chunk(const osdn_params* p, const Tin* q, const Tin* k, const Tin* v, const Tin* beta, const float* S0,
                 Tin* out, float* final_S, const Tin* kw, cudaStream_t st, char* ws = nullptr) {
    if (p->T == 0) return copy_initial_state(p, nullptr, S0, final_S, nullptr, true, false, st);
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        if (p->dk == 128 && p->dv == 128) {
            const WorkspaceLayout L = layout_of(p);
            if (ws && L.seg > 1)
                return launch_chunk_wy_segmented(p, q, k, v, beta, nullptr, S0, out, final_S, kw, ws, L, st);
            return launch_chunk_wy(p, q, k, v, beta, S0, out, final_S, kw, st);
        }
    }
    const int units = p->B * p->H;
    constexpr int DVT = 64;
    const dim3 grid(units, p->dv / DVT);
    const TokStrides ts = strides_of(p);
    const osdn::FfmaStrides s{ts.q, ts.k, ts.v, ts.o};
    cudaError_t e;
    if (p->dk == 128) {
        auto kern = osdn::chunk_ffma_kernel<128, DVT, Tin>;
        const size_t smem = osdn::FfmaSmem<128, DVT>::kBytes;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return cuda_fail(e, "chunk kernel attribute");
        kern<<<grid, 256, smem, st>>>(q, k, kw, v, beta, S0, out, final_S, p->B, p->T, p->H, p->dv, s);
    } else {
        auto kern = osdn::chunk_ffma_kernel<64, DVT, Tin>;
        const size_t smem = osdn::FfmaSmem<64, DVT>::kBytes;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return cuda_fail(e, "chunk kernel attribute");
        kern<<<grid, 256, smem, st>>>(q, k, kw, v, beta, S0, out, final_S, p->B, p->T, p->H, p->dv, s);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "chunk launch");
    return OSDN_OK;
}

// Phase 2 of the gated variant: the tensor-core kernel only (bf16, dk = dv = 128).
int launch_chunk_gated(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta,
                       const void* alpha, const float* S0, void* out, float* final_S, const void* kw, cudaStream_t st,
                       char* ws = nullptr) {
    if (p->dtype != OSDN_BF16 || p->dk != 128 || p->dv != 128)
        return fail(OSDN_ERR_UNSUPPORTED, "the gated forward needs bf16 inputs with dk = dv = 128");
    if (p->T == 0) return copy_initial_state(p, nullptr, S0, final_S, nullptr, true, false, st);
    using T = __nv_bfloat16;
    const WorkspaceLayout L = layout_of(p);
    if (ws && L.seg > 1)
        return launch_chunk_wy_segmented(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)alpha,
                                         S0, (T*)out, final_S, (const T*)kw, ws, L, st);
    return launch_chunk_wy(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, S0, (T*)out, final_S,
                           (const T*)kw, st, (const T*)alpha);
}

// Pointer and workspace checks shared by the forward entry points.
// keys_only: the workspace needs to hold only the scaled keys (phase 2 is never split).
int check_fwd_args(const osdn_params* p, std::initializer_list<const void*> required,
                   std::initializer_list<const void*> all, const void* workspace, size_t ws_bytes,
                   bool keys_only = false) {
    if (p->T > 0) {
        for (const void* x : required)
            if (!x) return fail(OSDN_ERR_INVALID_ARG, "a required pointer (q, k, v, beta, out) is NULL");
        if (!workspace) return fail(OSDN_ERR_INVALID_ARG, "workspace is NULL");
    }
    for (const void* x : all)
        if (x && !aligned16(x)) return fail(OSDN_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    if (workspace && !aligned16(workspace)) return fail(OSDN_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    const WorkspaceLayout L = layout_of(p);
    const size_t need = keys_only ? L.kw_bytes : L.total;
    if (p->T > 0 && ws_bytes < need)
        return fail(OSDN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
    return OSDN_OK;
}

template <typename Tin>
int launch_step(const osdn_params* p, const Tin* q, const Tin* k, const Tin* v, const Tin* beta, const Tin* r,
                const float* d_anchor, float* S, float* d, Tin* out, cudaStream_t st, const Tin* alpha = nullptr) {
    const unsigned units = (unsigned)(p->B * p->H);
    const int an = anchor_of(p);
    if (p->dk == 128 && p->dv == 128)
        osdn::step_kernel<128, 128, Tin><<<units, 256, 0, st>>>(q, k, v, beta, r, S, d, out, p->eta, an, d_anchor, alpha);
    else if (p->dk == 128)
        osdn::step_kernel<128, 64, Tin><<<units, 256, 0, st>>>(q, k, v, beta, r, S, d, out, p->eta, an, d_anchor, alpha);
    else if (p->dv == 128)
        osdn::step_kernel<64, 128, Tin><<<units, 256, 0, st>>>(q, k, v, beta, r, S, d, out, p->eta, an, d_anchor, alpha);
    else
        osdn::step_kernel<64, 64, Tin><<<units, 256, 0, st>>>(q, k, v, beta, r, S, d, out, p->eta, an, d_anchor, alpha);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "step launch");
    return OSDN_OK;
}

// Forward and reverse state passes of the backward with a dv tile of DVT rows.
template <typename Tin, int DK, int DV, int DVT>
int launch_state_passes(const osdn_params* p, const Tin* q, const Tin* dout, const float* S0, const float* dS_final,
                        float* dS0, float* ws, const osdn::bwd::Layout& L, int NC, int gated, cudaStream_t st) {
    namespace B = osdn::bwd;
    const unsigned ntiles = (unsigned)(p->B * p->H * (DV / DVT));
    const size_t s_sf = B::StateSmem<DK, DVT>::kFwdBytes, s_sb = B::StateSmem<DK, DVT>::kBwdBytes;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(B::bwd_state_f_kernel<DK, DV, DVT, Tin>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_sf)) != cudaSuccess)
        return cuda_fail(e, "backward state attribute");
    B::bwd_state_f_kernel<DK, DV, DVT, Tin><<<ntiles, B::NTHR, s_sf, st>>>(S0, ws, L, NC, gated);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward state launch");
    if ((e = cudaFuncSetAttribute(B::bwd_state_b_kernel<DK, DV, DVT, Tin>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_sb)) != cudaSuccess)
        return cuda_fail(e, "backward adjoint state attribute");
    B::bwd_state_b_kernel<DK, DV, DVT, Tin><<<ntiles, B::NTHR, s_sb, st>>>(dout, q, dS_final, dS0, ws, L, p->B,
                                                                           p->T, p->H, NC, gated);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward adjoint state launch");
    return OSDN_OK;
}

// Backward: six launches on one stream (see bwd.cuh for what each computes); alpha
// non-NULL selects the gated form inside the same kernels.
template <typename Tin, int DK, int DV>
int launch_bwd_t(const osdn_params* p, const Tin* q, const Tin* k, const Tin* v, const Tin* beta, const Tin* r,
                 const float* d0, const float* S0, const Tin* dout, const float* dS_final, const float* dd_final,
                 Tin* dq, Tin* dk, Tin* dv, Tin* dbeta, Tin* dr, float* dd0, float* dS0, float* ws,
                 const Tin* alpha, Tin* dalpha, cudaStream_t st) {
    namespace B = osdn::bwd;
    const B::Layout L = B::make_layout(p->B, p->T, p->H, DK, DV);
    const int units = p->B * p->H, NC = (p->T + B::C - 1) / B::C, an = anchor_of(p);
    const long long nchunks = (long long)units * NC;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned pgrid = (unsigned)(nchunks < sms ? nchunks : sms);   // persistent per-chunk kernels
    cudaError_t e;
    auto attr = [](const void* kern, size_t smem) {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    };
    const size_t s_dt = B::DtrajSmem<DK, Tin>::kBytes, s_dc = B::DchainSmem<DK, Tin>::kBytes;
    bool traj_done = false;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && DK == 128) {
        // d_t of every token from the forward's chunk-form scan on the tensor cores; its scaled keys
        // (bf16) land in the Kw region, which bwd_prep writes next
        const int rc = launch_scan_tc(p, k, beta, r, d0, nullptr,
                                      reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(ws) + L.kw), nullptr,
                                      nullptr, st, ws + L.d_all / sizeof(float));
        if (rc) return rc;
        traj_done = true;
    }
    if (!traj_done) {   // token-serial trajectory (fp32 inputs, dk = 64)
        if ((e = attr((const void*)B::bwd_dtraj_kernel<DK, Tin>, s_dt)) != cudaSuccess)
            return cuda_fail(e, "backward d trajectory attribute");
        B::bwd_dtraj_kernel<DK, Tin><<<(unsigned)units, B::SERIAL_THREADS, s_dt, st>>>(
            k, beta, r, d0, ws + L.d_all / sizeof(float), p->B, p->T, p->H, p->eta, an);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward d trajectory launch");
    }

    const size_t s_prep = B::PrepSmem<DK, DV>::kBytes;
    if ((e = attr((const void*)B::bwd_prep_kernel<DK, DV, Tin>, s_prep)) != cudaSuccess)
        return cuda_fail(e, "backward prep attribute");
    B::bwd_prep_kernel<DK, DV, Tin><<<pgrid, B::NTHR, s_prep, st>>>(q, k, v, beta, alpha, ws, L, p->B, p->T, p->H,
                                                                  NC);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward prep launch");

    // The two state passes are serial over the chunks; their dv tile is the widest of
    // DV, DV / 2, ... (down to 32 rows) whose (unit, tile) CTAs still fit one wave, or
    // the full DV when even that is more than one wave.
    int dvt = DV;
    while (dvt > 32 && (long long)units * (DV / dvt) * 2 <= sms) dvt /= 2;
    int rcs;
    const int gated = alpha != nullptr;
    if (dvt == 32) rcs = launch_state_passes<Tin, DK, DV, 32>(p, q, dout, S0, dS_final, dS0, ws, L, NC, gated, st);
    else if (dvt == 64)
        rcs = launch_state_passes<Tin, DK, DV, 64>(p, q, dout, S0, dS_final, dS0, ws, L, NC, gated, st);
    else rcs = launch_state_passes<Tin, DK, DV, DV>(p, q, dout, S0, dS_final, dS0, ws, L, NC, gated, st);
    if (rcs) return rcs;

    const size_t s_g = B::GradSmem<DK>::kBytes;
    if ((e = attr((const void*)B::bwd_grads_kernel<DK, DV, Tin>, s_g)) != cudaSuccess)
        return cuda_fail(e, "backward gradient attribute");
    B::bwd_grads_kernel<DK, DV, Tin><<<pgrid, B::NTHR, s_g, st>>>(q, k, v, beta, alpha, dout, dq, dv, dalpha, ws, L,
                                                                   p->B, p->T, p->H, NC);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward gradient launch");

    if ((e = attr((const void*)B::bwd_dchain_kernel<DK, Tin>, s_dc)) != cudaSuccess)
        return cuda_fail(e, "backward d chain attribute");
    B::bwd_dchain_kernel<DK, Tin><<<(unsigned)units, B::SERIAL_THREADS, s_dc, st>>>(
        k, beta, r, d0, dd_final, dk, dbeta, dr, dd0, ws, L, p->B, p->T, p->H, NC, p->eta, an);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward d chain launch");
    return OSDN_OK;
}

template <typename Tin>
int launch_bwd(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
               const float* d0, const float* S0, const void* dout, const float* dS_final, const float* dd_final,
               void* dq, void* dk, void* dv, void* dbeta, void* dr, float* dd0, float* dS0, float* ws,
               const void* alpha, void* dalpha, cudaStream_t st) {
#define OSDN_BWD_ARGS                                                                                        \
    p, (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)beta, (const Tin*)r, d0, S0, (const Tin*)dout, \
        dS_final, dd_final, (Tin*)dq, (Tin*)dk, (Tin*)dv, (Tin*)dbeta, (Tin*)dr, dd0, dS0, ws, (const Tin*)alpha, \
        (Tin*)dalpha, st
    if (p->dk == 128 && p->dv == 128) return launch_bwd_t<Tin, 128, 128>(OSDN_BWD_ARGS);
    if (p->dk == 128) return launch_bwd_t<Tin, 128, 64>(OSDN_BWD_ARGS);
    if (p->dv == 128) return launch_bwd_t<Tin, 64, 128>(OSDN_BWD_ARGS);
    return launch_bwd_t<Tin, 64, 64>(OSDN_BWD_ARGS);
#undef OSDN_BWD_ARGS
}

size_t bwd_workspace_bytes(const osdn_params* p) {
    const size_t n = osdn::bwd::make_layout(p->B, p->T, p->H, p->dk, p->dv).total;
    return n ? n : 256;
}

// Scratch for osdn_fwd_noalloc: a fixed array in device memory, sized by
// OSDN_NOALLOC_SCRATCH_BYTES. In host code the symbol is only a handle; its
// device address comes from cudaGetSymbolAddress with the device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[OSDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. Outside stream capture the
// address is looked up again on every call (a device reset can move the array); during a
// capture, where the lookup may not run, the address of this device's last lookup is used.
int noalloc_scratch(cudaStream_t st, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(OSDN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if ((e = cudaStreamIsCapturing(st, &cs)) != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (cs == cudaStreamCaptureStatusNone) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the scratch array");
        g_noalloc_ptr[dev] = ptr;
    } else if (!g_noalloc_ptr[dev]) {
        return fail(OSDN_ERR_INVALID_ARG,
                    "osdn_fwd_noalloc: the first call on a device must come before any stream capture");
    }
    *out = g_noalloc_ptr[dev];
    return OSDN_OK;
}

}  // namespace

extern "C" {

int osdn_abi_version(void) { return OSDN_ABI_VERSION; }

void osdn_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns.store(ns ? ns : 4000000000ull); }

const char* osdn_get_last_error(void) { return t_last_error.c_str(); }

int osdn_fwd_workspace_size(const osdn_params* p, size_t* bytes) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!bytes) return fail(OSDN_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = layout_of(p).total;
    return OSDN_OK;
}

int osdn_fwd_segments(const osdn_params* p, int* segments) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!segments) return fail(OSDN_ERR_INVALID_ARG, "segments is NULL");
    *segments = layout_of(p).seg;
    return OSDN_OK;
}

int osdn_fwd_launches(const osdn_params* p, int* launches) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!launches) return fail(OSDN_ERR_INVALID_ARG, "launches is NULL");
    const WorkspaceLayout L = layout_of(p);
    if (p->T == 0) *launches = 1;                    // at most the fill of d with ones
    else if (L.pipe > 1) *launches = 1 + 2 * L.pipe; // gather, per segment a scan and a chunk pass
    else if (L.seg == 1) *launches = 2;              // scan, chunk
    else if (!L.overlap) *launches = 6;              // scan, identity, three chunk passes, combine
    else   // identity, last-segment scan, per batch a scan, two passes, combine, output pass
        *launches = 2 + 5 * ((L.seg - 1 + L.ov_batch - 1) / L.ov_batch);
    return OSDN_OK;
}

int osdn_fwd(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
             const float* d0, const float* S0, void* out, float* final_S, float* final_d, void* workspace,
             size_t workspace_bytes, void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    rc = check_fwd_args(p, {q, k, v, beta, out}, {q, k, v, beta, r, d0, S0, out, final_S, final_d}, workspace,
                        workspace_bytes);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    char* ws = reinterpret_cast<char*>(workspace);
    const size_t kw_off = layout_of(p).kw_off;
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        T* kw = (T*)(ws ? ws + kw_off : nullptr);
        const WorkspaceLayout L = layout_of(p);
        if (L.overlap)
            return launch_fwd_overlapped(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)r,
                                         nullptr, d0, S0, (T*)out, final_S, final_d, ws, L, st);
        if (L.pipe > 1)
            return launch_fwd_pipelined(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)r,
                                        nullptr, d0, S0, (T*)out, final_S, final_d, ws, L, st);
        rc = launch_scan<T>(p, (const T*)k, (const T*)beta, (const T*)r, d0, final_d, kw, st);
        if (rc) return rc;
        return launch_chunk<T>(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, S0, (T*)out, final_S, kw, st,
                               ws);
    }
    using T = float;
    T* kw = (T*)(ws ? ws + kw_off : nullptr);
    rc = launch_scan<T>(p, (const T*)k, (const T*)beta, (const T*)r, d0, final_d, kw, st);
    if (rc) return rc;
    return launch_chunk<T>(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, S0, (T*)out, final_S, kw, st);
}

int osdn_fwd_gated(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
                   const void* alpha, const float* d0, const float* S0, void* out, float* final_S, float* final_d,
                   void* workspace, size_t workspace_bytes, void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (p->T > 0 && !alpha) return fail(OSDN_ERR_INVALID_ARG, "alpha is NULL");
    rc = check_fwd_args(p, {q, k, v, beta, out}, {q, k, v, beta, r, alpha, d0, S0, out, final_S, final_d}, workspace,
                        workspace_bytes);
    if (rc) return rc;
    if (p->dtype != OSDN_BF16 || p->dk != 128 || p->dv != 128)
        return fail(OSDN_ERR_UNSUPPORTED, "the gated forward needs bf16 inputs with dk = dv = 128");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    using T = __nv_bfloat16;
    T* kw = (T*)(workspace ? reinterpret_cast<char*>(workspace) + layout_of(p).kw_off : nullptr);
    const WorkspaceLayout L = layout_of(p);
    if (L.overlap)
        return launch_fwd_overlapped(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)r,
                                     (const T*)alpha, d0, S0, (T*)out, final_S, final_d,
                                     reinterpret_cast<char*>(workspace), L, st);
    if (L.pipe > 1)
        return launch_fwd_pipelined(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)r,
                                    (const T*)alpha, d0, S0, (T*)out, final_S, final_d,
                                    reinterpret_cast<char*>(workspace), L, st);
    rc = launch_scan<T>(p, (const T*)k, (const T*)beta, (const T*)r, d0, final_d, kw, st);
    if (rc) return rc;
    return launch_chunk_gated(p, q, k, v, beta, alpha, S0, out, final_S, kw, st, reinterpret_cast<char*>(workspace));
}

int osdn_fwd_chunk_gated(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta,
                         const void* alpha, const float* S0, void* out, float* final_S, void* workspace,
                         size_t workspace_bytes, void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (p->T > 0 && !alpha) return fail(OSDN_ERR_INVALID_ARG, "alpha is NULL");
    rc = check_fwd_args(p, {q, k, v, beta, out}, {q, k, v, beta, alpha, S0, out, final_S}, workspace, workspace_bytes);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    char* ws = reinterpret_cast<char*>(workspace);
    return launch_chunk_gated(p, q, k, v, beta, alpha, S0, out, final_S, ws ? ws + layout_of(p).kw_off : nullptr, st,
                              ws);
}

int osdn_fwd_scan(const osdn_params* p, const void* k, const void* beta, const void* r, const float* d0,
                  float* final_d, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    rc = check_fwd_args(p, {k, beta}, {k, beta, r, d0, final_d}, workspace, workspace_bytes);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    char* ws = reinterpret_cast<char*>(workspace) + layout_of(p).kw_off;
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        return launch_scan<T>(p, (const T*)k, (const T*)beta, (const T*)r, d0, final_d, (T*)ws, st);
    }
    return launch_scan<float>(p, (const float*)k, (const float*)beta, (const float*)r, d0, final_d, (float*)ws, st);
}

int osdn_fwd_scan_diag(const osdn_params* p, const void* k, const void* beta, const void* r, const float* d0,
                       float* final_d, float* rho, float* q_geo, void* workspace, size_t workspace_bytes,
                       void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    rc = check_fwd_args(p, {k, beta}, {k, beta, r, d0, final_d, rho, q_geo}, workspace, workspace_bytes);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    char* ws = reinterpret_cast<char*>(workspace) + layout_of(p).kw_off;
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        return launch_scan<T>(p, (const T*)k, (const T*)beta, (const T*)r, d0, final_d, (T*)ws, st, rho, q_geo);
    }
    return launch_scan<float>(p, (const float*)k, (const float*)beta, (const float*)r, d0, final_d, (float*)ws, st,
                              rho, q_geo);
}

int osdn_fwd_chunk(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta,
                   const float* S0, void* out, float* final_S, void* workspace, size_t workspace_bytes,
                   void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    rc = check_fwd_args(p, {q, k, v, beta, out}, {q, k, v, beta, S0, out, final_S}, workspace, workspace_bytes);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    char* wsb = reinterpret_cast<char*>(workspace);
    const char* ws = wsb ? wsb + layout_of(p).kw_off : nullptr;
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        return launch_chunk<T>(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, S0, (T*)out, final_S,
                               (const T*)ws, st, wsb);
    }
    return launch_chunk<float>(p, (const float*)q, (const float*)k, (const float*)v, (const float*)beta, S0,
                               (float*)out, final_S, (const float*)ws, st);
}

int osdn_fwd_noalloc(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta,
                     const void* r, const float* d0, const float* S0, void* out, float* final_S, float* final_d,
                     void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    const size_t need = layout_of(p).kw_bytes;
    if (need > (size_t)OSDN_NOALLOC_SCRATCH_BYTES)
        return fail(OSDN_ERR_INVALID_ARG, "scratch needed (%zu bytes) exceeds OSDN_NOALLOC_SCRATCH_BYTES (%zu bytes)",
                    need, (size_t)OSDN_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    if (p->T > 0) {
        rc = noalloc_scratch(reinterpret_cast<cudaStream_t>(cuda_stream), &scratch);
        if (rc) return rc;
    }
    rc = check_fwd_args(p, {q, k, v, beta, out}, {q, k, v, beta, r, d0, S0, out, final_S, final_d}, scratch,
                        (size_t)OSDN_NOALLOC_SCRATCH_BYTES, true);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        T* kw = (T*)scratch;
        rc = launch_scan<T>(p, (const T*)k, (const T*)beta, (const T*)r, d0, final_d, kw, st);
        if (rc) return rc;
        return launch_chunk<T>(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, S0, (T*)out, final_S, kw, st);
    }
    float* kw = (float*)scratch;
    rc = launch_scan<float>(p, (const float*)k, (const float*)beta, (const float*)r, d0, final_d, kw, st);
    if (rc) return rc;
    return launch_chunk<float>(p, (const float*)q, (const float*)k, (const float*)v, (const float*)beta, S0,
                               (float*)out, final_S, kw, st);
}

int osdn_step_ex(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
                 const float* d_anchor, float* S, float* d, void* out, void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, false);
    if (rc) return rc;
    if (p->struct_size >= sizeof(osdn_params) &&
        !(all_zero(p->stride_q) && all_zero(p->stride_k) && all_zero(p->stride_v) && all_zero(p->stride_o)))
        return fail(OSDN_ERR_UNSUPPORTED, "the decode step takes dense tensors only (strides must be zero)");
    if (!q || !k || !v || !beta || !S || !d || !out)
        return fail(OSDN_ERR_INVALID_ARG, "q, k, v, beta, S, d and out must not be NULL");
    const void* ptrs[] = {q, k, v, beta, r, d_anchor, S, d, out};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return fail(OSDN_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        return launch_step<T>(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)r, d_anchor, S, d,
                              (T*)out, st);
    }
    return launch_step<float>(p, (const float*)q, (const float*)k, (const float*)v, (const float*)beta,
                              (const float*)r, d_anchor, S, d, (float*)out, st);
}

int osdn_step_gated(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta,
                    const void* r, const void* alpha, const float* d_anchor, float* S, float* d, void* out,
                    void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, false);
    if (rc) return rc;
    if (p->struct_size >= sizeof(osdn_params) &&
        !(all_zero(p->stride_q) && all_zero(p->stride_k) && all_zero(p->stride_v) && all_zero(p->stride_o)))
        return fail(OSDN_ERR_UNSUPPORTED, "the decode step takes dense tensors only (strides must be zero)");
    if (!q || !k || !v || !beta || !alpha || !S || !d || !out)
        return fail(OSDN_ERR_INVALID_ARG, "q, k, v, beta, alpha, S, d and out must not be NULL");
    const void* ptrs[] = {q, k, v, beta, r, alpha, d_anchor, S, d, out};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return fail(OSDN_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    if (p->dtype == OSDN_BF16) {
        using T = __nv_bfloat16;
        return launch_step<T>(p, (const T*)q, (const T*)k, (const T*)v, (const T*)beta, (const T*)r, d_anchor, S, d,
                              (T*)out, st, (const T*)alpha);
    }
    return launch_step<float>(p, (const float*)q, (const float*)k, (const float*)v, (const float*)beta,
                              (const float*)r, d_anchor, S, d, (float*)out, st, (const float*)alpha);
}

int osdn_step(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
              float* S, float* d, void* out, void* cuda_stream) {
    return osdn_step_ex(p, q, k, v, beta, r, nullptr, S, d, out, cuda_stream);
}

int osdn_bwd_workspace_size(const osdn_params* p, size_t* bytes) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!bytes) return fail(OSDN_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = bwd_workspace_bytes(p);
    return OSDN_OK;
}

}  // extern "C"

namespace {
int bwd_impl(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
             const void* alpha, const float* d0, const float* S0, const void* dout, const float* dS_final,
             const float* dd_final, void* dq, void* dk, void* dv, void* dbeta, void* dr, void* dalpha, float* dd0,
             float* dS0, void* workspace, size_t workspace_bytes, void* cuda_stream, bool gated) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!dense_layout(p)) return fail(OSDN_ERR_UNSUPPORTED, "the backward takes dense tensors only");
    const void* ptrs[] = {q, k, v, beta, r, alpha, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta, dr, dalpha,
                          dd0, dS0, workspace};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return fail(OSDN_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    const size_t units = (size_t)p->B * p->H;
    if (p->T == 0) {   // no tokens: the gradients of the initial state are those of the final state
        cudaError_t e = cudaSuccess;
        if (dS0) {
            const size_t bytes = units * p->dv * p->dk * sizeof(float);
            e = dS_final ? cudaMemcpyAsync(dS0, dS_final, bytes, cudaMemcpyDeviceToDevice, st)
                         : cudaMemsetAsync(dS0, 0, bytes, st);
            if (e != cudaSuccess) return cuda_fail(e, "initial state gradient copy");
        }
        if (dd0) {
            const size_t bytes = units * p->dk * sizeof(float);
            e = dd_final ? cudaMemcpyAsync(dd0, dd_final, bytes, cudaMemcpyDeviceToDevice, st)
                         : cudaMemsetAsync(dd0, 0, bytes, st);
            if (e != cudaSuccess) return cuda_fail(e, "initial preconditioner gradient copy");
        }
        return OSDN_OK;
    }
    if (!q || !k || !v || !beta || !dout || !dq || !dk || !dv || !dbeta)
        return fail(OSDN_ERR_INVALID_ARG, "q, k, v, beta, dout, dq, dk, dv and dbeta must not be NULL");
    if (gated && (!alpha || !dalpha)) return fail(OSDN_ERR_INVALID_ARG, "alpha and dalpha must not be NULL");
    if (!workspace) return fail(OSDN_ERR_INVALID_ARG, "workspace is NULL");
    const size_t need = bwd_workspace_bytes(p);
    if (workspace_bytes < need)
        return fail(OSDN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
    if ((double)units * (double)((p->T + 63) / 64) > 2147483647.0)
        return fail(OSDN_ERR_INVALID_ARG, "B * H * ceil(T / 64) exceeds the grid limit");
    float* ws = reinterpret_cast<float*>(workspace);
    if (!gated) alpha = dalpha = nullptr;
    if (p->dtype == OSDN_BF16)
        return launch_bwd<__nv_bfloat16>(p, q, k, v, beta, r, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta,
                                         dr, dd0, dS0, ws, alpha, dalpha, st);
    return launch_bwd<float>(p, q, k, v, beta, r, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta, dr, dd0, dS0,
                             ws, alpha, dalpha, st);
}
}  // namespace

extern "C" {

int osdn_bwd(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
             const float* d0, const float* S0, const void* dout, const float* dS_final, const float* dd_final,
             void* dq, void* dk, void* dv, void* dbeta, void* dr, float* dd0, float* dS0, void* workspace,
             size_t workspace_bytes, void* cuda_stream) {
    return bwd_impl(p, q, k, v, beta, r, nullptr, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta, dr, nullptr,
                    dd0, dS0, workspace, workspace_bytes, cuda_stream, false);
}

int osdn_bwd_gated(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta,
                   const void* r, const void* alpha, const float* d0, const float* S0, const void* dout,
                   const float* dS_final, const float* dd_final, void* dq, void* dk, void* dv, void* dbeta, void* dr,
                   void* dalpha, float* dd0, float* dS0, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    return bwd_impl(p, q, k, v, beta, r, alpha, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta, dr, dalpha,
                    dd0, dS0, workspace, workspace_bytes, cuda_stream, true);
}

int osdn_sync_status(void* cuda_stream) {
    t_last_error.clear();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int status = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&status, osdn::g_osdn_status, sizeof(status))) != cudaSuccess)
        return cuda_fail(e, "status read");
    if (status && (e = cudaMemcpyToSymbol(osdn::g_osdn_status, &zero, sizeof(zero))) != cudaSuccess)
        return cuda_fail(e, "status clear");
    if (status & osdn::kStatusTimeout) return fail(OSDN_ERR_TIMEOUT, "a bounded device-side wait gave up");
    return OSDN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------- host buffers
namespace {

// Two non-blocking copy streams per device (host to device, device to host) for osdn_fwd_host,
// apart from the streams the forward itself forks to, so that copies never queue behind its
// kernels. Created on first use and kept for the life of the process.
int copy_streams(cudaStream_t out[2]) {
    static std::mutex mu;
    static cudaStream_t streams[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "current device");
    if (dev < 0 || dev >= 64) return fail(OSDN_ERR_UNSUPPORTED, "device index %d above 63", dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 2; ++i)
        if (!streams[dev][i] && (e = cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "copy stream");
    out[0] = streams[dev][0];
    out[1] = streams[dev][1];
    return OSDN_OK;
}

constexpr int kMaxHostGroups = 16;

// The device region of osdn_fwd_host: the whole problem's inputs, outputs and initial states,
// then the forward workspace of the largest group, each 256-byte aligned.
struct HostLayout {
    int groups, per;   // groups of `per` consecutive sequences (the last may hold fewer)
    size_t q, k, v, beta, r, out, S, d, d0, S0, ws, ws_bytes, total;
};

osdn_params full_params(const osdn_params* p) {   // a version-3 copy of any accepted version
    osdn_params f{};
    std::memcpy(&f, p, p->struct_size < sizeof(f) ? p->struct_size : sizeof(f));
    f.struct_size = sizeof(f);
    return f;
}

HostLayout host_layout_of(const osdn_params* p, int groups) {
    HostLayout L{};
    int g = groups <= 0 ? 8 : groups;
    if (g > p->B) g = p->B;
    if (g > kMaxHostGroups) g = kMaxHostGroups;
    L.per = (p->B + g - 1) / g;
    L.groups = (p->B + L.per - 1) / L.per;
    const size_t es = elem_size(p->dtype), tok = (size_t)p->B * p->T * p->H, units = (size_t)p->B * p->H;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    L.q = take(tok * p->dk * es);
    L.k = take(tok * p->dk * es);
    L.v = take(tok * p->dv * es);
    L.beta = take(tok * es);
    L.r = take(tok * es);
    L.out = take(tok * p->dv * es);
    L.S = take(units * p->dv * p->dk * sizeof(float));
    L.d = take(units * p->dk * sizeof(float));
    L.S0 = take(units * p->dv * p->dk * sizeof(float));
    L.d0 = take(units * p->dk * sizeof(float));
    osdn_params gp = full_params(p);
    gp.B = L.per;
    size_t ws = layout_of(&gp).total;
    const int last = p->B - (L.groups - 1) * L.per;   // the last group's sequences
    if (last != L.per) {
        gp.B = last;
        const size_t w2 = layout_of(&gp).total;
        if (w2 > ws) ws = w2;
    }
    L.ws_bytes = ws;
    L.ws = take(ws);
    L.total = off;
    return L;
}

}  // namespace

extern "C" {

int osdn_fwd_host_buffer_size(const osdn_params* p, int groups, size_t* bytes) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!bytes) return fail(OSDN_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = host_layout_of(p, groups).total;
    return OSDN_OK;
}

int osdn_fwd_host(const osdn_params* p, const void* q, const void* k, const void* v, const void* beta, const void* r,
                  const float* d0, const float* S0, void* out, float* final_S, float* final_d, void* device_buffer,
                  size_t device_bytes, int groups, void* cuda_stream) {
    t_last_error.clear();
    int rc = check_params(p, true);
    if (rc) return rc;
    if (!dense_layout(p)) return fail(OSDN_ERR_UNSUPPORTED, "osdn_fwd_host takes dense host tensors only");
    if (p->T > 0 && (!q || !k || !v || !beta || !out))
        return fail(OSDN_ERR_INVALID_ARG, "a required pointer (q, k, v, beta, out) is NULL");
    if (!device_buffer) return fail(OSDN_ERR_INVALID_ARG, "device_buffer is NULL");
    if (!aligned16(device_buffer)) return fail(OSDN_ERR_INVALID_ARG, "device_buffer must be 16-byte aligned");
    const HostLayout L = host_layout_of(p, groups);
    if (device_bytes < L.total)
        return fail(OSDN_ERR_INVALID_ARG, "device_buffer too small: %zu bytes given, %zu needed", device_bytes, L.total);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    cudaStream_t cs[2];
    if ((rc = copy_streams(cs))) return rc;
    char* dbuf = reinterpret_cast<char*>(device_buffer);
    const size_t es = elem_size(p->dtype);
    const size_t seq_tok = (size_t)p->T * p->H;               // token-heads of one sequence
    const size_t seq_S = (size_t)p->H * p->dv * p->dk, seq_d = (size_t)p->H * p->dk;

    const int nev = 2 + 2 * L.groups;                          // fork, join, per group: inputs in, computed
    cudaEvent_t ev[2 + 2 * kMaxHostGroups];
    cudaError_t e = cudaSuccess;
    int made = 0;
    for (; made < nev; ++made)
        if ((e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming)) != cudaSuccess) break;
    if (e != cudaSuccess) {
        for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
        return cuda_fail(e, "event");
    }
    auto chk = [&](cudaError_t x, const char* what) -> int { return x == cudaSuccess ? OSDN_OK : cuda_fail(x, what); };
    // n bytes from host src + off to device region dst + off (or back), on stream s; src may be NULL
    auto h2d = [&](size_t dst, const void* src, size_t off, size_t n, cudaStream_t s) -> int {
        if (!src || n == 0) return OSDN_OK;
        return chk(cudaMemcpyAsync(dbuf + dst + off, static_cast<const char*>(src) + off, n, cudaMemcpyHostToDevice, s),
                   "host to device copy");
    };
    auto d2h = [&](void* dst, size_t src, size_t off, size_t n, cudaStream_t s) -> int {
        if (!dst || n == 0) return OSDN_OK;
        return chk(cudaMemcpyAsync(static_cast<char*>(dst) + off, dbuf + src + off, n, cudaMemcpyDeviceToHost, s),
                   "device to host copy");
    };
    do {
        if ((rc = chk(cudaEventRecord(ev[0], st), "fork"))) break;
        if ((rc = chk(cudaStreamWaitEvent(cs[0], ev[0], 0), "fork"))) break;
        if ((rc = chk(cudaStreamWaitEvent(cs[1], ev[0], 0), "fork"))) break;
        for (int gi = 0; gi < L.groups && !rc; ++gi) {
            const int b0 = gi * L.per, nb = p->B - b0 < L.per ? p->B - b0 : L.per;
            const size_t t0 = (size_t)b0 * seq_tok, tn = (size_t)nb * seq_tok;
            // inputs of the group's sequences (contiguous in every [B, ...] tensor) on the copy-in stream
            if ((rc = h2d(L.q, q, t0 * p->dk * es, tn * p->dk * es, cs[0]))) break;
            if ((rc = h2d(L.k, k, t0 * p->dk * es, tn * p->dk * es, cs[0]))) break;
            if ((rc = h2d(L.v, v, t0 * p->dv * es, tn * p->dv * es, cs[0]))) break;
            if ((rc = h2d(L.beta, beta, t0 * es, tn * es, cs[0]))) break;
            if ((rc = h2d(L.r, r, t0 * es, tn * es, cs[0]))) break;
            if ((rc = h2d(L.S0, S0, (size_t)b0 * seq_S * 4, (size_t)nb * seq_S * 4, cs[0]))) break;
            if ((rc = h2d(L.d0, d0, (size_t)b0 * seq_d * 4, (size_t)nb * seq_d * 4, cs[0]))) break;
            if ((rc = chk(cudaEventRecord(ev[2 + 2 * gi], cs[0]), "inputs event"))) break;
            // the group's forward on the caller's stream, once its inputs are in
            if ((rc = chk(cudaStreamWaitEvent(st, ev[2 + 2 * gi], 0), "inputs wait"))) break;
            osdn_params gp = full_params(p);
            gp.B = nb;
            auto at = [&](size_t base, size_t off) { return static_cast<void*>(dbuf + base + off); };
            rc = osdn_fwd(&gp, at(L.q, t0 * p->dk * es), at(L.k, t0 * p->dk * es), at(L.v, t0 * p->dv * es),
                          at(L.beta, t0 * es), r ? at(L.r, t0 * es) : nullptr,
                          d0 ? static_cast<const float*>(at(L.d0, (size_t)b0 * seq_d * 4)) : nullptr,
                          S0 ? static_cast<const float*>(at(L.S0, (size_t)b0 * seq_S * 4)) : nullptr,
                          at(L.out, t0 * p->dv * es), static_cast<float*>(at(L.S, (size_t)b0 * seq_S * 4)),
                          static_cast<float*>(at(L.d, (size_t)b0 * seq_d * 4)), dbuf + L.ws, L.ws_bytes, st);
            if (rc) break;
            if ((rc = chk(cudaEventRecord(ev[3 + 2 * gi], st), "compute event"))) break;
            // its results back on the copy-out stream
            if ((rc = chk(cudaStreamWaitEvent(cs[1], ev[3 + 2 * gi], 0), "compute wait"))) break;
            if ((rc = d2h(out, L.out, t0 * p->dv * es, tn * p->dv * es, cs[1]))) break;
            if ((rc = d2h(final_S, L.S, (size_t)b0 * seq_S * 4, (size_t)nb * seq_S * 4, cs[1]))) break;
            if ((rc = d2h(final_d, L.d, (size_t)b0 * seq_d * 4, (size_t)nb * seq_d * 4, cs[1]))) break;
        }
        if (rc) break;
        // join: the caller's stream waits for the last copies back (it already waited for every copy in)
        if ((rc = chk(cudaEventRecord(ev[1], cs[1]), "join"))) break;
        rc = chk(cudaStreamWaitEvent(st, ev[1], 0), "join");
    } while (false);
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
    return rc;
}

}  // extern "C"
