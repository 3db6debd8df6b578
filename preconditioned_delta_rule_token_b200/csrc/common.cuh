// Shared device helpers for the OSDN kernels (element conversion, reductions,
// the status word that bounded waits report into).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace osdn {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load N consecutive elements starting at p (p aligned to N * sizeof(T)) as fp32.
template <int N, typename T> struct VecIO;

template <> struct VecIO<4, float> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        float4 v = *reinterpret_cast<const float4*>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* o) {
        *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
    }
};
template <> struct VecIO<2, float> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        float2 v = *reinterpret_cast<const float2*>(p);
        o[0] = v.x; o[1] = v.y;
    }
    static __device__ __forceinline__ void store(float* p, const float* o) {
        *reinterpret_cast<float2*>(p) = make_float2(o[0], o[1]);
    }
};
template <> struct VecIO<4, __nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        uint2 u = *reinterpret_cast<const uint2*>(p);
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* o) {
        __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(o[2], o[3]);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = u;
    }
};
template <> struct VecIO<2, __nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(p);
        float2 fa = __bfloat1622float2(a);
        o[0] = fa.x; o[1] = fa.y;
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* o) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(o[0], o[1]);
    }
};

// Element strides of a token tensor [B, T, H, width] over (b, t, h); the last dimension is contiguous.
struct Tok3 {
    int64_t b, t, h;
    __host__ __device__ __forceinline__ int64_t at(int64_t bb, int64_t tt, int64_t hh) const {
        return bb * b + tt * t + hh * h;
    }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Status word shared by all kernels of the library: a bounded wait that gives
// up ORs a code into it; osdn_sync_status() reads and clears it.  The library
// is one translation unit (osdn_api.cu includes every kernel header), so this
// definition exists once.
__device__ unsigned int g_osdn_status = 0;

enum : unsigned int { kStatusTimeout = 1u };

}  // namespace osdn
