// common.cuh -- device helpers shared by the sm_100a kernels of libssm_causal.
//
// dtype-generic scalar access (f32 / f16 / bf16 widened to f32, stores rounded
// to nearest even), 128-bit streaming access for the state caches, and the
// activations of the method (SiLU, softplus, exp of the discretised decay)
// built on the SFU instructions ex2.approx / rcp.approx.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace ssm {

enum : int { kF32 = 0, kF16 = 1, kBF16 = 2, kI32 = 3 };

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- scalars --
__device__ __forceinline__ float ld_f(const void* p, int64_t i, int dt) {
    if (dt == kF16) return __half2float(static_cast<const __half*>(p)[i]);
    if (dt == kBF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    return static_cast<const float*>(p)[i];
}

__device__ __forceinline__ void st_f(void* p, int64_t i, int dt, float v) {
    if (dt == kF16) {
        static_cast<__half*>(p)[i] = __float2half_rn(v);
    } else if (dt == kBF16) {
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    } else {
        static_cast<float*>(p)[i] = v;
    }
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// -------------------------------------------------- 16-byte state vectors --
// VE elements of type T in one 16-byte vector.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int VE = 4;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};
template <> struct Vec16<__half> {
    static constexpr int VE = 8;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            float2 v = __half22float2(h);
            f[2 * i] = v.x;
            f[2 * i + 1] = v.y;
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int VE = 8;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
            float2 v = __bfloat1622float2(h);
            f[2 * i] = v.x;
            f[2 * i + 1] = v.y;
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// Streaming (evict-first) 128-bit load/store for data touched once per call.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    return __ldcs(static_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream16(void* p, const uint4& v) {
    __stcs(static_cast<uint4*>(p), v);
}

// ------------------------------------------------------------ activations --
// 2^x on the SFU (ex2.approx, flush-to-zero): relative error ~2 ulp.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float exp_fast(float x) { return ex2_approx(x * kLog2e); }

// SiLU(v) = v * sigmoid(v) = v / (1 + e^-v).  For v -> -inf the quotient
// tends to -0; __fdividef returns 0 when the divisor overflows.
__device__ __forceinline__ float silu_f(float v) {
    return __fdividef(v, 1.0f + exp_fast(-v));
}

// softplus(v) = log(1 + e^v); above 20 the correction e^-v is below 2^-28 * v.
__device__ __forceinline__ float softplus_f(float v) {
    return v > 20.0f ? v : log1pf(exp_fast(v));
}

}  // namespace ssm
