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
// transcendentals per (b, t, d) -- ~22 SFU operations per 8 bytes of HBM
// traffic at d_state 16 -- and the shared-memory bytes each element pulls.
// So the kernel is SFU / shared-memory bound, not HBM bound.  Every
// exponential is computed exactly once (the sequence is not split across
// CTAs), and shared-memory traffic per element is cut by register reuse:
//   * a CTA is one warp owning 16 channels of one batch entry for the whole
//     sequence; thread (pr, q) owns channels 2pr and 2pr+1 and state entries
//     4q..4q+3 of both, so each B/C value read from shared memory serves two
//     channels and the packed f32x2 operations run across the channel pair;
//   * the next 32-step chunk is staged with 16-byte cp.async copies into
//     shared memory while the current one is scanned (each thread copies the
//     words it reads back itself, so its own wait_group is the only sync);
//   * the thread that loads x/dt/z for (channel, 8 steps) computes their conv,
//     SiLU, softplus and gate in registers -- the W-1 history values come from
//     the neighbouring lane by shuffle;
//   * (delta, delta*u) of a channel pair for one step is one 16-byte word;
//   * the 8 partial readouts of a 4-step group are summed over the 4 threads
//     of the pair by a butterfly reduce-scatter (6 shuffles per 4 steps);
//   * optionally SW of the 4 state entries take their exponential from a
//     Cody-Waite + degree-5 minimax polynomial on the FMA pipe, balancing the
//     SFU against the FMA pipe.
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

namespace ssm {
namespace {

constexpr int kDT = 16;       // channels per CTA
constexpr int kPairs = 8;     // channel pairs per CTA
constexpr int kT = 32;        // time steps per chunk
constexpr int kThreads = 32;  // one warp: 8 channel pairs x 4 threads
constexpr int kV = 8;         // time steps per thread per chunk (one 16-byte vector of 16-bit I/O)
constexpr int kYStride = kT + 4;

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

// raw I/O of one chunk as staged by cp.async: x, dt, z of the 16 channels and
// B, C of the 16 state entries, each [row][32 steps]
template <typename IoT> struct __align__(16) RawStage {
    IoT x[kDT][kT];
    IoT dt[kDT][kT];
    IoT z[kDT][kT];
    IoT B[16][kT];
    IoT C[16][kT];
};

template <typename IoT> struct __align__(16) VecSmem {
    RawStage<IoT> raw;          // the chunk's inputs, refilled for the next chunk once read
    float4 dd[kPairs][kT + 1];  // (delta_c0, delta_c1, delta*u_c0, delta*u_c1) per channel pair
    float y[kDT][kYStride];     // D*u, then + sum_n C h
    float g[kDT][kYStride];     // silu(z)
    float B[kT][16];
    float C[kT][16];
};

// per-channel state of the prologue: conv weights, biases, conv history
template <int W> struct ChanParams {
    float w[W > 0 ? W : 1];
    float cbias, dbias, dskip;
    float hist[W > 1 ? W - 1 : 1];  // raw inputs at (chunk start) - (W-1) + i
};

// conv + SiLU, softplus and gate for 8 steps of one channel, in registers
template <int W>
__device__ __forceinline__ void prologue8(const ScanProblem& p, ChanParams<W>& cp, const float* xs,
                                          const float* dts, const float* zs, bool has_z, bool v_ok,
                                          int q, int lane, float* dl, float* du, float* u,
                                          float* gate) {
    if constexpr (W > 0) {
        float prev[W > 1 ? W - 1 : 1];
#pragma unroll
        for (int i = 0; i < W - 1; ++i) {
            const float left = __shfl_up_sync(0xffffffffu, xs[kV - (W - 1) + i], 1);
            prev[i] = q == 0 ? cp.hist[i] : left;
        }
#pragma unroll
        for (int i = 0; i < W - 1; ++i)
            cp.hist[i] = __shfl_sync(0xffffffffu, xs[kV - (W - 1) + i], lane | 3);
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            float acc = cp.cbias;
#pragma unroll
            for (int k = 0; k < W; ++k) {
                const int j = i - (W - 1) + k;
                acc = fmaf(cp.w[k], j >= 0 ? xs[j] : prev[W - 1 + j], acc);
            }
            u[i] = silu_f(acc);
        }
    } else {
#pragma unroll
        for (int i = 0; i < kV; ++i) u[i] = xs[i];
    }
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        const float v = dts[i] + cp.dbias;
        dl[i] = v_ok ? (p.softplus ? softplus_f(v) : v) : 0.0f;
        du[i] = v_ok ? dl[i] * u[i] : 0.0f;
        gate[i] = has_z ? silu_f(zs[i]) : 1.0f;
    }
}

// Thread layout of a CTA (one warp, 16 channels): thread (pr, q) with pr =
// tid / 4 the channel pair (channels 2pr, 2pr+1) and q = tid % 4.  In the
// prologue and epilogue q selects the 8-step vector [8q, 8q+8) of the chunk;
// in the scan it selects the state entries n = 4q .. 4q+3 of both channels.
// The same thread also loads B/C rows n = pr and pr + 8 (vector q).
template <typename IoT, int W, int SW>
__global__ void __launch_bounds__(kThreads, 12) scan_vec_kernel(const ScanProblem p) {
    __shared__ VecSmem<IoT> sm;
    const int tid = threadIdx.x;
    const int pr = tid >> 2;
    const int q = tid & 3;
    const int lane = tid;
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * kDT;
    const int64_t g = d0 / p.ch_per_group;
    const bool has_z = p.z != nullptr;

    int64_t dch[2];
    bool ok[2];
    const IoT* xrow[2];
    const IoT* dtrow[2];
    const IoT* zrow[2];
    IoT* orow[2];
    ChanParams<W> cp[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int64_t d = d0 + 2 * pr + c;
        ok[c] = d < p.D;
        dch[c] = ok[c] ? d : d0;  // safe row for address arithmetic
        xrow[c] = static_cast<const IoT*>(p.x) + b * p.x_b + dch[c] * p.x_d;
        dtrow[c] = static_cast<const IoT*>(p.dt) + b * p.dt_b + dch[c] * p.dt_d;
        zrow[c] = has_z ? static_cast<const IoT*>(p.z) + b * p.z_b + dch[c] * p.z_d : nullptr;
        orow[c] = static_cast<IoT*>(p.out) + b * p.o_b + dch[c] * p.o_d;
#pragma unroll
        for (int k = 0; k < W; ++k) cp[c].w[k] = ok[c] ? p.conv_w[dch[c] * p.cw_d + k * p.cw_k] : 0.0f;
        cp[c].cbias = (W > 0 && p.conv_b && ok[c]) ? p.conv_b[dch[c] * p.cb_d] : 0.0f;
        cp[c].dbias = (p.dt_bias && ok[c]) ? p.dt_bias[dch[c] * p.db_d] : 0.0f;
        cp[c].dskip = (p.Dp && ok[c]) ? p.Dp[dch[c] * p.D_d] : 0.0f;
#pragma unroll
        for (int i = 0; i < W - 1; ++i)
            cp[c].hist[i] = (p.conv_state && ok[c])
                                ? ld_f(p.conv_state, b * p.cs_b + dch[c] * p.cs_d + (1 + i) * p.cs_k, p.cs_dt)
                                : 0.0f;
    }
    // B/C rows this thread loads
    const IoT* brow[2];
    const IoT* crow[2];
    bool nok[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int n = pr + 8 * r;
        nok[r] = n < p.N;
        const int64_t nl = nok[r] ? n : 0;
        brow[r] = static_cast<const IoT*>(p.Bm) + b * p.B_b + g * p.B_g + nl * p.B_n;
        crow[r] = static_cast<const IoT*>(p.Cm) + b * p.C_b + g * p.C_g + nl * p.C_n;
    }
    // state entries n = 4q + j of both channels, as pairs (channel 0, channel 1);
    // A pre-scaled by log2(e)
    u64 hp[4], Ap[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = 4 * q + j;
        float a[2], h[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const bool v = ok[c] && n < p.N;
            a[c] = v ? p.A[dch[c] * p.A_d + n * p.A_n] * kLog2e : 0.0f;
            h[c] = (v && p.ssm_state) ? p.ssm_state[b * p.ss_b + dch[c] * p.ss_d + n * p.ss_n] : 0.0f;
        }
        Ap[j] = pk(a[0], a[1]);
        hp[j] = pk(h[0], h[1]);
    }

    const int64_t L = p.L;
    const int nchunks = (int)((L + kT - 1) / kT);
    constexpr int kVB = kV * (int)sizeof(IoT) / 16;  // 16-byte copies per 8-step vector
    // each thread stages exactly the vectors it reads back in the prologue
    auto fetch = [&](int ci) {
        RawStage<IoT>& st = sm.raw;
        const int64_t t = (int64_t)ci * kT + kV * q;
        const bool v_ok = t < L;  // L is a multiple of 8: a vector is all in or all out
        const int64_t ts = v_ok ? t : 0;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int ch = 2 * pr + c;
#pragma unroll
            for (int k = 0; k < kVB; ++k) {
                cp_async16(&st.x[ch][kV * q] + k * 16 / sizeof(IoT), xrow[c] + ts + k * 16 / sizeof(IoT), v_ok);
                cp_async16(&st.dt[ch][kV * q] + k * 16 / sizeof(IoT), dtrow[c] + ts + k * 16 / sizeof(IoT), v_ok);
                cp_async16(&st.z[ch][kV * q] + k * 16 / sizeof(IoT),
                           (has_z ? zrow[c] : xrow[c]) + ts + k * 16 / sizeof(IoT), v_ok && has_z);
                cp_async16(&st.B[pr + 8 * c][kV * q] + k * 16 / sizeof(IoT), brow[c] + ts + k * 16 / sizeof(IoT),
                           v_ok && nok[c]);
                cp_async16(&st.C[pr + 8 * c][kV * q] + k * 16 / sizeof(IoT), crow[c] + ts + k * 16 / sizeof(IoT),
                           v_ok && nok[c]);
            }
        }
        cp_async_commit();
    };
    auto unpack8 = [](const IoT* src, float* f) {
        if constexpr (sizeof(IoT) == 2) {
            Vec16<IoT>::unpack(*reinterpret_cast<const uint4*>(src), f);
        } else {
            Vec16<float>::unpack(*reinterpret_cast<const uint4*>(src), f);
            Vec16<float>::unpack(*(reinterpret_cast<const uint4*>(src) + 1), f + 4);
        }
    };
    fetch(0);

    for (int ci = 0; ci < nchunks; ++ci) {
        const int64_t t0 = (int64_t)ci * kT;
        const bool vec_ok = t0 + kV * q < L;
        // ---- this chunk's staged inputs (copied during the previous scan)
        cp_async_wait<0>();
        const RawStage<IoT>& st = sm.raw;
        // ---- prologue in registers for both channels, results to shared memory
        float dlc[2][kV], duc[2][kV];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float xs[kV], dts[kV], zs[kV], u[kV], gate[kV];
            unpack8(&st.x[2 * pr + c][kV * q], xs);
            unpack8(&st.dt[2 * pr + c][kV * q], dts);
            unpack8(&st.z[2 * pr + c][kV * q], zs);
            prologue8<W>(p, cp[c], xs, dts, zs, has_z, vec_ok && ok[c], q, lane, dlc[c], duc[c], u, gate);
            const int ch = 2 * pr + c;
            float4* yp = reinterpret_cast<float4*>(&sm.y[ch][kV * q]);
            yp[0] = make_float4(cp[c].dskip * u[0], cp[c].dskip * u[1], cp[c].dskip * u[2], cp[c].dskip * u[3]);
            yp[1] = make_float4(cp[c].dskip * u[4], cp[c].dskip * u[5], cp[c].dskip * u[6], cp[c].dskip * u[7]);
            float4* gp = reinterpret_cast<float4*>(&sm.g[ch][kV * q]);
            gp[0] = make_float4(gate[0], gate[1], gate[2], gate[3]);
            gp[1] = make_float4(gate[4], gate[5], gate[6], gate[7]);
        }
#pragma unroll
        for (int i = 0; i < kV; ++i)
            sm.dd[pr][kV * q + i] = make_float4(dlc[0][i], dlc[1][i], duc[0][i], duc[1][i]);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            float bv[kV], cv[kV];
            unpack8(&st.B[pr + 8 * r][kV * q], bv);
            unpack8(&st.C[pr + 8 * r][kV * q], cv);
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                sm.B[kV * q + i][pr + 8 * r] = bv[i];
                sm.C[kV * q + i][pr + 8 * r] = cv[i];
            }
        }
        // each thread re-fills only the staging words it has just read, so the
        // next chunk's copies can start now and fly during the scan
        if (ci + 1 < nchunks) fetch(ci + 1);
        __syncwarp();

        // ---- scan: thread (pr, q) updates state entries 4q..4q+3 of both
        // channels; packed pairs run across the two channels
#pragma unroll 2
        for (int tt = 0; tt < kT; tt += 4) {
            float v[8];  // v[2k + c]: partial readout of step tt+k, channel c
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 dd = sm.dd[pr][tt + k];
                const float4 b4 = *reinterpret_cast<const float4*>(&sm.B[tt + k][4 * q]);
                const float4 c4 = *reinterpret_cast<const float4*>(&sm.C[tt + k][4 * q]);
                const u64 dl2 = pk(dd.x, dd.y);
                const u64 du2 = pk(dd.z, dd.w);
                const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
                const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
                u64 y2 = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const u64 x2 = fmul2(dl2, Ap[j]);
                    const u64 a2 = j < SW ? exp2_pair_fma(x2) : exp2_pair_sfu(x2);
                    hp[j] = ffma2(a2, hp[j], fmul2(du2, pk(bb[j], bb[j])));
                    y2 = j == 0 ? fmul2(pk(cc[j], cc[j]), hp[j]) : ffma2(pk(cc[j], cc[j]), hp[j], y2);
                }
                upk(y2, v[2 * k], v[2 * k + 1]);
            }
            // butterfly reduce-scatter of the 8 partials over the 4 threads of
            // the pair: thread q ends with both channels' totals for step tt+q
            {
                const bool up2 = (q & 2) != 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float send = up2 ? v[i] : v[i + 4];
                    const float keep = up2 ? v[i + 4] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                }
                const bool up1 = (q & 1) != 0;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float send = up1 ? v[i] : v[i + 2];
                    const float keep = up1 ? v[i + 2] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                }
                sm.y[2 * pr][tt + q] += v[0];
                sm.y[2 * pr + 1][tt + q] += v[1];
            }
        }
        __syncwarp();

        // ---- epilogue: gate and store 8 steps of both channels
        if (vec_ok) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (!ok[c]) continue;
                const int ch = 2 * pr + c;
                const float4 y0 = *reinterpret_cast<const float4*>(&sm.y[ch][kV * q]);
                const float4 y1 = *reinterpret_cast<const float4*>(&sm.y[ch][kV * q + 4]);
                const float4 g0 = *reinterpret_cast<const float4*>(&sm.g[ch][kV * q]);
                const float4 g1 = *reinterpret_cast<const float4*>(&sm.g[ch][kV * q + 4]);
                const float o[kV] = {y0.x * g0.x, y0.y * g0.y, y0.z * g0.z, y0.w * g0.w,
                                     y1.x * g1.x, y1.y * g1.y, y1.z * g1.z, y1.w * g1.w};
                store8<IoT>(orow[c] + t0 + kV * q, o);
            }
        }
        __syncwarp();
    }

    // ---- final caches
    if (p.ssm_state) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = 4 * q + j;
            float h[2];
            upk(hp[j], h[0], h[1]);
#pragma unroll
            for (int c = 0; c < 2; ++c)
                if (ok[c] && n < p.N) p.ssm_state[b * p.ss_b + dch[c] * p.ss_d + n * p.ss_n] = h[c];
        }
    }
    if (W > 0 && p.conv_state && q == 0) {
        // last W raw inputs (L is a multiple of 8, so L >= 8 >= W)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            if (!ok[c]) continue;
#pragma unroll
            for (int k = 0; k < W; ++k)
                st_f(p.conv_state, b * p.cs_b + dch[c] * p.cs_d + k * p.cs_k, p.cs_dt,
                     to_f(xrow[c][L - W + k]));
        }
    }
}

template <typename IoT, int W>
cudaError_t launch_w(const ScanProblem& p, int sw, cudaStream_t s) {
    dim3 grid((unsigned)((p.D + kDT - 1) / kDT), (unsigned)p.Bn);
    auto run = [&](auto kern) -> cudaError_t {
        // many small CTAs per SM: ask for the largest shared-memory carveout
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, 0, s>>>(p);
        return cudaGetLastError();
    };
    switch (sw) {
        case 0: return run(scan_vec_kernel<IoT, W, 0>);
        case 1: return run(scan_vec_kernel<IoT, W, 1>);
        case 2: return run(scan_vec_kernel<IoT, W, 2>);
        case 3: return run(scan_vec_kernel<IoT, W, 3>);
        default: return cudaErrorInvalidValue;
    }
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
