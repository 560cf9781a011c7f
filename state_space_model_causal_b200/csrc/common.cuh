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

// Record that a bounded wait ran out: code 1, the reporting kernel, and the
// lowest work item that did not complete (see DeviceError in problem.h).
template <typename E>
__device__ __forceinline__ void report_device_error(E* err, int kernel, long long first_item) {
    atomicExch(&err->code, 1);
    atomicExch(&err->kernel, kernel);
    atomicMin(&err->first_item, first_item);
}

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

// ------------------------------------------------------ cp.async staging --
// 16-byte asynchronous copy global -> shared (zero-filled when !valid)
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename IoT>
__device__ __forceinline__ void store8(IoT* p, const float* f) {
    if constexpr (sizeof(IoT) == 2) {
        __stcs(reinterpret_cast<uint4*>(p), Vec16<IoT>::pack(f));
    } else {
        __stcs(reinterpret_cast<uint4*>(p), Vec16<float>::pack(f));
        __stcs(reinterpret_cast<uint4*>(p) + 1, Vec16<float>::pack(f + 4));
    }
}

// ------------------------------------------------------- packed f32x2 math --
// Two fp32 lanes in one 64-bit register pair; sm_100 executes add/mul/fma on
// both halves with one instruction.
typedef unsigned long long u64;

__device__ __forceinline__ u64 pk(float lo, float hi) {
    u64 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(u64 v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ u64 fmul2(u64 a, u64 b) {
    u64 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 ffma2(u64 a, u64 b, u64 c) {
    u64 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ u64 fadd2(u64 a, u64 b) {
    u64 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 fsub2(u64 a, u64 b) {
    u64 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ------------------------------------------------------------ activations --
// 2^x on the SFU (ex2.approx, flush-to-zero): relative error ~2 ulp.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x for a pair, on the FMA pipe.  Cody-Waite split x = j + f with j the
// nearest integer (via the 1.5*2^23 rounding constant) and f in [-1/2, 1/2];
// 2^f from the degree-5 minimax polynomial for relative error on that
// interval (coefficients fitted for this kernel by a Remez exchange, max
// relative error 7.5e-8 before rounding); 2^j applied by adding j to the
// exponent field.  x is clamped to [-125, 126] so the result stays normal.
__device__ __forceinline__ u64 exp2_pair_fma(u64 x) {
    float x0, x1;
    upk(x, x0, x1);
    x0 = fminf(fmaxf(x0, -125.0f), 126.0f);
    x1 = fminf(fmaxf(x1, -125.0f), 126.0f);
    const u64 xc = pk(x0, x1);
    const u64 magic = pk(12582912.0f, 12582912.0f);
    const u64 t = fadd2(xc, magic);
    const u64 f = fsub2(xc, fsub2(t, magic));
    u64 p = ffma2(pk(0.0013276472454890609f, 0.0013276472454890609f), f,
                  pk(0.009675540961325169f, 0.009675540961325169f));
    p = ffma2(p, f, pk(0.05550713092088699f, 0.05550713092088699f));
    p = ffma2(p, f, pk(0.24022120237350464f, 0.24022120237350464f));
    p = ffma2(p, f, pk(0.6931469440460205f, 0.6931469440460205f));
    p = ffma2(p, f, pk(1.0000001192092896f, 1.0000001192092896f));
    float p0, p1, t0, t1;
    upk(p, p0, p1);
    upk(t, t0, t1);
    const float r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    const float r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
    return pk(r0, r1);
}

__device__ __forceinline__ u64 exp2_pair_sfu(u64 x) {
    float x0, x1;
    upk(x, x0, x1);
    return pk(ex2_approx(x0), ex2_approx(x1));
}

// 1/d for a pair of d >= 1 (up to +inf) on the FMA pipe, so that the SFU
// keeps its issue slots for the exponentials.  Newton's iteration for the
// reciprocal, r <- r + r (1 - d r), from the integer-subtraction seed
// r0 = as_float(K - bits(d)): K = 0x7ef311c2 was chosen here by a search that
// minimises the seed's relative error over a binade (5.1%); each step squares
// the relative error, so two steps leave < 7e-6 and three reach fp32 rounding
// (~1 ulp).  d is clamped to 2^125 first, so the seed stays a normal number
// and 1/d tends to 0 as d grows.
template <int STEPS>
__device__ __forceinline__ u64 rcp_pair_fma(u64 d) {
    float d0, d1;
    upk(d, d0, d1);
    d0 = fminf(d0, 4.2535295865117308e37f);  // 2^125
    d1 = fminf(d1, 4.2535295865117308e37f);
    u64 r = pk(__int_as_float(0x7ef311c2 - __float_as_int(d0)), __int_as_float(0x7ef311c2 - __float_as_int(d1)));
    const u64 nd = pk(-d0, -d1);
#pragma unroll
    for (int k = 0; k < STEPS; ++k) r = ffma2(r, ffma2(nd, r, pk(1.0f, 1.0f)), r);
    return r;
}

// SiLU on a pair, v / (1 + 2^(-v log2 e)): one SFU exponential per value,
// the reciprocal on the FMA pipe.
template <int STEPS>
__device__ __forceinline__ u64 silu_pair(u64 v) {
    const u64 den = fadd2(exp2_pair_sfu(fmul2(v, pk(-kLog2e, -kLog2e))), pk(1.0f, 1.0f));
    return fmul2(v, rcp_pair_fma<STEPS>(den));
}

__device__ __forceinline__ float exp_fast(float x) { return ex2_approx(x * kLog2e); }

// SiLU(v) = v * sigmoid(v) = v / (1 + e^-v).  For v -> -inf the quotient
// tends to -0; __fdividef returns 0 when the divisor overflows.
__device__ __forceinline__ float silu_f(float v) {
    return __fdividef(v, 1.0f + exp_fast(-v));
}

// softplus(v) = log(1 + e^v).  Above v = 20 the correction e^-v is below
// 2^-28 * v, so v is returned.  With e = e^v <= 1/16 (v <= -2.77, where the
// discretisation step of a selective SSM usually lives) log(1 + e) is the
// alternating series e - e^2/2 + e^3/3 - ... cut after e^7/7: the remainder
// is below e^8/8 <= 2^-35, i.e. < 2^-31 relative to the result.  In between,
// log1pf.
__device__ __forceinline__ float softplus_f(float v) {
    if (v > 20.0f) return v;
    const float e = exp_fast(v);
    if (e <= 0.0625f) {
        float s = fmaf(e, 1.0f / 7.0f, -1.0f / 6.0f);
        s = fmaf(s, e, 0.2f);
        s = fmaf(s, e, -0.25f);
        s = fmaf(s, e, 1.0f / 3.0f);
        s = fmaf(s, e, -0.5f);
        s = fmaf(s, e, 1.0f);
        return e * s;
    }
    return log1pf(e);
}

}  // namespace ssm
