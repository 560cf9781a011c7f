// scan_vec.cu -- the fast fused prefill for sm_100a (d_state <= 16, time
// dimension contiguous and 16-byte aligned): causal conv1d -> SiLU ->
// softplus(dt + dt_bias) -> selective scan -> D skip -> SiLU(z) gate, the
// operator chain "causal-conv1d, selective-scan, silu, element-mul" of
// "feat(llama.cu): 适配 mamba 模型" (section 2.1), reading and writing the conv
// and SSM state caches of section 3.1.
//
//   u     = silu(bias[d] + sum_k w[d,k] * x[t-(W-1)+k])
//   delta = softplus(dt[t] + dt_bias[d])
//   h[n]  = exp(delta * A[d,n]) * h[n] + delta * B[n,t] * u
//   out   = (sum_n C[n,t] * h[n] + D[d] * u) * silu(z[t])
//
// What bounds it: one exp(delta*A) per (b, t, d, n) element plus five more
// transcendentals per (b, t, d).  At d_state 16 that is ~22 SFU operations per
// 8 bytes of HBM traffic, so the kernel is SFU/issue bound, not HBM bound.
// Every exponential is computed exactly once (no split of the sequence across
// CTAs), and the instruction count per element is kept minimal:
//   * a CTA owns 16 channels of one batch entry for the whole sequence; 4
//     threads share a channel, each holding 4 state entries in registers;
//   * the chunk of 32 steps a thread will load next is fetched with 16-byte
//     loads into registers while the current chunk is scanned;
//   * the thread that loads x/dt/z for (channel, 8 steps) also computes their
//     conv, SiLU, softplus and gate in registers -- the W-1 history values come
//     from the neighbouring lane by shuffle, not from shared memory;
//   * delta and delta*u are stored as duplicated pairs so the scan's multiply
//     and fma run as packed f32x2 operations on two state entries at once;
//   * the readouts of the 4 threads of a channel are summed by a butterfly
//     reduce-scatter (3 shuffles per 4 steps);
//   * optionally SW of the thread's 2 state-entry pairs take their exponential
//     from a Cody-Waite + degree-5 minimax polynomial on the FMA pipe instead
//     of the SFU, balancing the two pipes.
// Two barriers per chunk: after the prologue writes, and after the scan.
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

namespace ssm {
namespace {

constexpr int kDT = 16;       // channels per CTA
constexpr int kT = 32;        // time steps per chunk
constexpr int kThreads = 64;  // 16 channels x 4 threads
constexpr int kV = 8;         // time steps per thread per chunk (one 16-byte vector of 16-bit I/O)
constexpr int kPairStride = kT + 2;  // float2 row stride of the delta tiles
constexpr int kYStride = kT + 4;
constexpr int kMaxHist = 7;

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

// eight consecutive I/O values = one 16-byte vector (16-bit types) or two (fp32)
template <typename IoT> struct Raw8 {
    static constexpr int NV = sizeof(IoT) == 2 ? 1 : 2;
    uint4 v[NV];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = make_uint4(0, 0, 0, 0);
    }
    __device__ __forceinline__ void load_stream(const IoT* p) {
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = __ldcs(reinterpret_cast<const uint4*>(p) + i);
    }
    __device__ __forceinline__ void load_cached(const IoT* p) {
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
    }
    __device__ __forceinline__ void unpack(float* f) const {
        if constexpr (sizeof(IoT) == 2) {
            Vec16<IoT>::unpack(v[0], f);
        } else {
            Vec16<float>::unpack(v[0], f);
            Vec16<float>::unpack(v[1], f + 4);
        }
    }
};

template <typename IoT>
__device__ __forceinline__ void store8(IoT* p, const float* f) {
    if constexpr (sizeof(IoT) == 2) {
        __stcs(reinterpret_cast<uint4*>(p), Vec16<IoT>::pack(f));
    } else {
        __stcs(reinterpret_cast<uint4*>(p), Vec16<float>::pack(f));
        __stcs(reinterpret_cast<uint4*>(p) + 1, Vec16<float>::pack(f + 4));
    }
}

struct __align__(16) VecSmem {
    float2 dl[kDT][kPairStride];  // (delta, delta)
    float2 du[kDT][kPairStride];  // (delta*u, delta*u)
    float y[kDT][kYStride];       // D*u, then + sum_n C h
    float g[kDT][kYStride];       // silu(z)
    float B[kT][16];
    float C[kT][16];
};

template <typename IoT, int W, int SW>
__global__ void __launch_bounds__(kThreads, 10) scan_vec_kernel(const ScanProblem p) {
    __shared__ VecSmem sm;
    const int tid = threadIdx.x;
    const int ch = tid >> 2;  // channel within the tile
    const int q = tid & 3;    // time vector (prologue/epilogue) and state slice (scan)
    const int lane = tid & 31;
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * kDT;
    const int64_t d = d0 + ch;
    const bool d_ok = d < p.D;
    const int64_t dd = d_ok ? d : d0;  // safe row for address arithmetic
    const int64_t g = d0 / p.ch_per_group;

    const IoT* xrow = static_cast<const IoT*>(p.x) + b * p.x_b + dd * p.x_d;
    const IoT* dtrow = static_cast<const IoT*>(p.dt) + b * p.dt_b + dd * p.dt_d;
    const IoT* zrow = p.z ? static_cast<const IoT*>(p.z) + b * p.z_b + dd * p.z_d : nullptr;
    IoT* orow = static_cast<IoT*>(p.out) + b * p.o_b + dd * p.o_d;
    // B/C rows loaded by this thread: state entry n = ch (the tile has 16 threads rows)
    const bool n_ok = ch < p.N;
    const int64_t nl = n_ok ? ch : 0;
    const IoT* brow = static_cast<const IoT*>(p.Bm) + b * p.B_b + g * p.B_g + nl * p.B_n;
    const IoT* crow = static_cast<const IoT*>(p.Cm) + b * p.C_b + g * p.C_g + nl * p.C_n;

    // per-channel parameters
    float w[W > 0 ? W : 1];
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = d_ok ? p.conv_w[dd * p.cw_d + k * p.cw_k] : 0.0f;
    const float cbias = (W > 0 && p.conv_b && d_ok) ? p.conv_b[dd * p.cb_d] : 0.0f;
    const float dbias = (p.dt_bias && d_ok) ? p.dt_bias[dd * p.db_d] : 0.0f;
    const float dskip = (p.Dp && d_ok) ? p.Dp[dd * p.D_d] : 0.0f;

    // state entries n = 4q + j, A pre-scaled by log2(e)
    float hs[4];
    u64 A01, A23;
    {
        float a2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = 4 * q + j;
            const bool ok = d_ok && n < p.N;
            a2[j] = ok ? p.A[dd * p.A_d + n * p.A_n] * kLog2e : 0.0f;
            hs[j] = (ok && p.ssm_state) ? p.ssm_state[b * p.ss_b + dd * p.ss_d + n * p.ss_n] : 0.0f;
        }
        A01 = pk(a2[0], a2[1]);
        A23 = pk(a2[2], a2[3]);
    }
    u64 h01 = pk(hs[0], hs[1]);
    u64 h23 = pk(hs[2], hs[3]);

    // conv history: hist[i] = raw input at (chunk start) - (W-1) + i
    float hist[W > 1 ? W - 1 : 1];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        // conv_state entry 1 + i holds time -(W-1) + i
        hist[i] = (p.conv_state && d_ok)
                      ? ld_f(p.conv_state, b * p.cs_b + dd * p.cs_d + (1 + i) * p.cs_k, p.cs_dt)
                      : 0.0f;
    }

    const int64_t L = p.L;
    const int nchunks = (int)((L + kT - 1) / kT);
    Raw8<IoT> rx, rdt, rz, rb, rc;
    auto fetch = [&](int c) {
        const int64_t t = (int64_t)c * kT + kV * q;
        const bool v_ok = t < L;  // L is a multiple of 8: a vector is all in or all out
        if (v_ok) {
            rx.load_stream(xrow + t);
            rdt.load_stream(dtrow + t);
            if (zrow) rz.load_stream(zrow + t); else rz.zero();
            if (n_ok) {
                rb.load_cached(brow + t);
                rc.load_cached(crow + t);
            } else {
                rb.zero();
                rc.zero();
            }
        } else {
            rx.zero(); rdt.zero(); rz.zero(); rb.zero(); rc.zero();
        }
    };
    fetch(0);

    for (int c = 0; c < nchunks; ++c) {
        const int64_t t0 = (int64_t)c * kT;
        const bool v_ok = d_ok && (t0 + kV * q < L);
        // ---- prologue in registers: conv + SiLU, softplus, gate
        float xs[kV], dts[kV], zs[kV], bv[kV], cv[kV];
        rx.unpack(xs);
        rdt.unpack(dts);
        rz.unpack(zs);
        rb.unpack(bv);
        rc.unpack(cv);
        float u[kV];
        if constexpr (W > 0) {
            float prev[W > 1 ? W - 1 : 1];
#pragma unroll
            for (int i = 0; i < W - 1; ++i) {
                const float left = __shfl_up_sync(0xffffffffu, xs[kV - (W - 1) + i], 1);
                prev[i] = q == 0 ? hist[i] : left;
            }
#pragma unroll
            for (int i = 0; i < W - 1; ++i)
                hist[i] = __shfl_sync(0xffffffffu, xs[kV - (W - 1) + i], lane | 3);
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                float acc = cbias;
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const int j = i - (W - 1) + k;
                    acc = fmaf(w[k], j >= 0 ? xs[j] : prev[W - 1 + j], acc);
                }
                u[i] = silu_f(acc);
            }
        } else {
#pragma unroll
            for (int i = 0; i < kV; ++i) u[i] = xs[i];
        }
        float dl[kV], du[kV], gate[kV];
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const float v = dts[i] + dbias;
            dl[i] = v_ok ? (p.softplus ? softplus_f(v) : v) : 0.0f;
            du[i] = v_ok ? dl[i] * u[i] : 0.0f;
            gate[i] = zrow ? silu_f(zs[i]) : 1.0f;
        }
        {
            float4* dlp = reinterpret_cast<float4*>(&sm.dl[ch][kV * q]);
            float4* dup = reinterpret_cast<float4*>(&sm.du[ch][kV * q]);
#pragma unroll
            for (int i = 0; i < kV; i += 2) {
                dlp[i / 2] = make_float4(dl[i], dl[i], dl[i + 1], dl[i + 1]);
                dup[i / 2] = make_float4(du[i], du[i], du[i + 1], du[i + 1]);
            }
            float4* yp = reinterpret_cast<float4*>(&sm.y[ch][kV * q]);
            yp[0] = make_float4(dskip * u[0], dskip * u[1], dskip * u[2], dskip * u[3]);
            yp[1] = make_float4(dskip * u[4], dskip * u[5], dskip * u[6], dskip * u[7]);
            float4* gp = reinterpret_cast<float4*>(&sm.g[ch][kV * q]);
            gp[0] = make_float4(gate[0], gate[1], gate[2], gate[3]);
            gp[1] = make_float4(gate[4], gate[5], gate[6], gate[7]);
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                sm.B[kV * q + i][ch] = bv[i];
                sm.C[kV * q + i][ch] = cv[i];
            }
        }
        // ---- next chunk's loads fly during the scan
        if (c + 1 < nchunks) fetch(c + 1);
        __syncthreads();

        // ---- scan: thread (ch, q) owns state entries 4q .. 4q+3
        const float4* dlr = reinterpret_cast<const float4*>(&sm.dl[ch][0]);
        const float4* dur = reinterpret_cast<const float4*>(&sm.du[ch][0]);
#pragma unroll 2
        for (int tt = 0; tt < kT; tt += 4) {
            float yv[4];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const float4 dl4 = dlr[(tt >> 1) + half];
                const float4 du4 = dur[(tt >> 1) + half];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int t = tt + 2 * half + k;
                    const u64 dd2 = k == 0 ? pk(dl4.x, dl4.y) : pk(dl4.z, dl4.w);
                    const u64 uu2 = k == 0 ? pk(du4.x, du4.y) : pk(du4.z, du4.w);
                    const float4 b4 = *reinterpret_cast<const float4*>(&sm.B[t][4 * q]);
                    const float4 c4 = *reinterpret_cast<const float4*>(&sm.C[t][4 * q]);
                    const u64 x01 = fmul2(dd2, A01);
                    const u64 x23 = fmul2(dd2, A23);
                    const u64 a01 = SW >= 1 ? exp2_pair_fma(x01) : exp2_pair_sfu(x01);
                    const u64 a23 = SW >= 2 ? exp2_pair_fma(x23) : exp2_pair_sfu(x23);
                    h01 = ffma2(a01, h01, fmul2(uu2, pk(b4.x, b4.y)));
                    h23 = ffma2(a23, h23, fmul2(uu2, pk(b4.z, b4.w)));
                    const u64 y2 = ffma2(pk(c4.z, c4.w), h23, fmul2(pk(c4.x, c4.y), h01));
                    float ya, yb;
                    upk(y2, ya, yb);
                    yv[2 * half + k] = ya + yb;
                }
            }
            // butterfly reduce-scatter over the 4 threads of the channel
            {
                const bool up2 = (q & 2) != 0;
                float s0 = up2 ? yv[0] : yv[2];
                float s1 = up2 ? yv[1] : yv[3];
                float k0 = up2 ? yv[2] : yv[0];
                float k1 = up2 ? yv[3] : yv[1];
                k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
                k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                const bool up1 = (q & 1) != 0;
                const float s = up1 ? k0 : k1;
                float kk = up1 ? k1 : k0;
                kk += __shfl_xor_sync(0xffffffffu, s, 1);
                sm.y[ch][tt + q] += kk;
            }
        }
        __syncthreads();

        // ---- epilogue: gate and store this thread's 8 steps
        if (v_ok) {
            const float4 y0 = *reinterpret_cast<const float4*>(&sm.y[ch][kV * q]);
            const float4 y1 = *reinterpret_cast<const float4*>(&sm.y[ch][kV * q + 4]);
            const float4 g0 = *reinterpret_cast<const float4*>(&sm.g[ch][kV * q]);
            const float4 g1 = *reinterpret_cast<const float4*>(&sm.g[ch][kV * q + 4]);
            float o[kV] = {y0.x * g0.x, y0.y * g0.y, y0.z * g0.z, y0.w * g0.w,
                           y1.x * g1.x, y1.y * g1.y, y1.z * g1.z, y1.w * g1.w};
            store8<IoT>(orow + t0 + kV * q, o);
        }
    }

    // ---- final caches
    if (p.ssm_state && d_ok) {
        float hv[4];
        upk(h01, hv[0], hv[1]);
        upk(h23, hv[2], hv[3]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = 4 * q + j;
            if (n < p.N) p.ssm_state[b * p.ss_b + dd * p.ss_d + n * p.ss_n] = hv[j];
        }
    }
    if (W > 0 && p.conv_state && d_ok && q == 0) {
        // last W raw inputs (L is a multiple of 8, so L >= 8 >= W)
#pragma unroll
        for (int k = 0; k < W; ++k)
            st_f(p.conv_state, b * p.cs_b + dd * p.cs_d + k * p.cs_k, p.cs_dt,
                 to_f(xrow[L - W + k]));
    }
}

template <typename IoT, int W>
cudaError_t launch_w(const ScanProblem& p, int sw, cudaStream_t s) {
    dim3 grid((unsigned)((p.D + kDT - 1) / kDT), (unsigned)p.Bn);
    switch (sw) {
        case 0: scan_vec_kernel<IoT, W, 0><<<grid, kThreads, 0, s>>>(p); break;
        case 1: scan_vec_kernel<IoT, W, 1><<<grid, kThreads, 0, s>>>(p); break;
        case 2: scan_vec_kernel<IoT, W, 2><<<grid, kThreads, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename IoT>
cudaError_t launch_io(const ScanProblem& p, int sw, cudaStream_t s) {
    switch (p.W) {
        case 0: return launch_w<IoT, 0>(p, sw, s);
        case 4: return launch_w<IoT, 4>(p, sw, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool scan_vec_supported(const ScanProblem& p) {
    return p.N <= 16 && (p.W == 0 || p.W == 4) && p.L % kV == 0 && p.Bn <= 65535 &&
           (p.G == 1 || p.ch_per_group % kDT == 0);
}

int scan_vec_threads() { return kThreads; }
int scan_vec_channels_per_cta() { return kDT; }

cudaError_t launch_scan_vec(const ScanProblem& p, int sw, cudaStream_t s) {
    switch (p.io_dt) {
        case kF32: return launch_io<float>(p, sw, s);
        case kF16: return launch_io<__half>(p, sw, s);
        case kBF16: return launch_io<__nv_bfloat16>(p, sw, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssm
