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

// x, dt, z of one chunk as staged by cp.async: [channel][32 steps].  Each
// thread copies, and later reads back, only its own 8-step vectors.
template <typename IoT> struct __align__(16) RawXZ {
    IoT x[kDT][kT];
    IoT dt[kDT][kT];
    IoT z[kDT][kT];
};

// B, C of one chunk: [state entry n][32 steps], read by every thread of the
// CTA during the scan (so double-buffered).  The 16-byte pieces of row n are
// stored XOR-swizzled by (n / 4) mod 4, so the four rows 4q + j that the four
// q-groups read at once fall in distinct banks.
template <typename IoT> struct __align__(16) RawBC {
    IoT B[16][kT];
    IoT C[16][kT];
};
template <typename IoT> constexpr int kCE = 16 / (int)sizeof(IoT);  // elements per 16-byte piece
__device__ __forceinline__ int bc_swz(int n, int piece) { return piece ^ ((n >> 2) & 3); }

template <typename IoT> struct __align__(16) VecSmem {
    RawXZ<IoT> xz;
    RawBC<IoT> bc[2];
    float4 dd[kPairs][kT + 1];  // (delta_c0, delta_c1, delta*u_c0, delta*u_c1) per channel pair
    float y[kDT][kYStride];     // sum_n C h per (channel, step)
};

// 8 bytes of a B or C row (4 steps of 16-bit I/O, 2 of fp32), widened on use
template <typename IoT> __device__ __forceinline__ float elt8(const uint2& w, int k);
template <> __device__ __forceinline__ float elt8<float>(const uint2& w, int k) {
    return __uint_as_float(k == 0 ? w.x : w.y);
}
template <> __device__ __forceinline__ float elt8<__half>(const uint2& w, int k) {
    const uint32_t h = k < 2 ? w.x : w.y;
    return __half2float(__ushort_as_half((unsigned short)((k & 1) ? (h >> 16) : (h & 0xffffu))));
}
template <> __device__ __forceinline__ float elt8<__nv_bfloat16>(const uint2& w, int k) {
    const uint32_t h = k < 2 ? w.x : w.y;
    return __uint_as_float((k & 1) ? (h & 0xffff0000u) : (h << 16));
}

// per-channel state of the prologue: conv weights, biases, conv history
template <int W> struct ChanParams {
    float w[W > 0 ? W : 1];
    float cbias, dbias, dskip;
    float hist[W > 1 ? W - 1 : 1];  // raw inputs at (chunk start) - (W-1) + i
};

// conv + SiLU, softplus and gate for 8 steps of one channel, in registers;
// the softplus and the gate run on packed step pairs
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
    for (int i = 0; i < kV; i += 2) {
        const u64 v2 = fadd2(pk(dts[i], dts[i + 1]), pk(cp.dbias, cp.dbias));
        float v0, v1;
        upk(v2, v0, v1);
        if (p.softplus) {
            // softplus as in softplus_f, on a pair: log1p series for e^v <= 1/16
            const u64 l2 = fmul2(v2, pk(kLog2e, kLog2e));
            float l0, l1;
            upk(l2, l0, l1);
            const u64 e2 = pk(ex2_approx(l0), ex2_approx(l1));
            u64 s2 = ffma2(e2, pk(1.0f / 7.0f, 1.0f / 7.0f), pk(-1.0f / 6.0f, -1.0f / 6.0f));
            s2 = ffma2(s2, e2, pk(0.2f, 0.2f));
            s2 = ffma2(s2, e2, pk(-0.25f, -0.25f));
            s2 = ffma2(s2, e2, pk(1.0f / 3.0f, 1.0f / 3.0f));
            s2 = ffma2(s2, e2, pk(-0.5f, -0.5f));
            s2 = ffma2(s2, e2, pk(1.0f, 1.0f));
            s2 = fmul2(s2, e2);
            float e0, e1, r0, r1;
            upk(e2, e0, e1);
            upk(s2, r0, r1);
            if (e0 > 0.0625f) r0 = v0 > 20.0f ? v0 : log1pf(e0);
            if (e1 > 0.0625f) r1 = v1 > 20.0f ? v1 : log1pf(e1);
            v0 = r0;
            v1 = r1;
        }
        dl[i] = v_ok ? v0 : 0.0f;
        dl[i + 1] = v_ok ? v1 : 0.0f;
        const u64 du2 = fmul2(pk(dl[i], dl[i + 1]), pk(u[i], u[i + 1]));
        upk(du2, du[i], du[i + 1]);
        if (has_z) {
            // SiLU(z) = z / (1 + 2^(-z log2 e)) on a pair
            const u64 zn = fmul2(pk(zs[i], zs[i + 1]), pk(-kLog2e, -kLog2e));
            float a0, a1;
            upk(zn, a0, a1);
            const u64 den = fadd2(pk(ex2_approx(a0), ex2_approx(a1)), pk(1.0f, 1.0f));
            float d0, d1;
            upk(den, d0, d1);
            const u64 g2 = fmul2(pk(zs[i], zs[i + 1]), pk(__fdividef(1.0f, d0), __fdividef(1.0f, d1)));
            upk(g2, gate[i], gate[i + 1]);
        } else {
            gate[i] = gate[i + 1] = 1.0f;
        }
    }
}

// Thread layout of a CTA (one warp, 16 channels): thread (pr, q) with pr =
// tid / 4 the channel pair (channels 2pr, 2pr+1) and q = tid % 4.  In the
// prologue and epilogue q selects the 8-step vector [8q, 8q+8) of the chunk;
// in the scan it selects the state entries n = 4q .. 4q+3 of both channels.
// The same thread stages B/C rows n = pr and pr + 8 (vector q).  Gate and
// D*u of a thread's prologue vectors stay in its registers until its
// epilogue, which covers the same (channel, step) vectors.
template <typename IoT, int W, int SW>
__global__ void __launch_bounds__(kThreads, 9) scan_vec_kernel(const ScanProblem p) {
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
    // B/C rows this thread stages
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
    constexpr int kE = kCE<IoT>;
    constexpr int kVB = kV / kE;  // 16-byte copies per 8-step vector
    auto fetch = [&](int ci) {
        const int64_t t = (int64_t)ci * kT + kV * q;
        const bool v_ok = t < L;  // L is a multiple of 8: a vector is all in or all out
        const int64_t ts = v_ok ? t : 0;
        RawXZ<IoT>& xz = sm.xz;
        RawBC<IoT>& bc = sm.bc[ci & 1];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int ch = 2 * pr + c;
            const int n = pr + 8 * c;
#pragma unroll
            for (int k = 0; k < kVB; ++k) {
                const int e = kV * q + k * kE;  // first step of the piece
                cp_async16(&xz.x[ch][e], xrow[c] + ts + k * kE, v_ok);
                cp_async16(&xz.dt[ch][e], dtrow[c] + ts + k * kE, v_ok);
                cp_async16(&xz.z[ch][e], (has_z ? zrow[c] : xrow[c]) + ts + k * kE, v_ok && has_z);
                const int sp = bc_swz(n, e / kE) * kE;
                cp_async16(&bc.B[n][sp], brow[c] + ts + k * kE, v_ok && nok[c]);
                cp_async16(&bc.C[n][sp], crow[c] + ts + k * kE, v_ok && nok[c]);
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

    constexpr int kQ = 8 / (int)sizeof(IoT);  // steps per 8-byte B/C read
    for (int ci = 0; ci < nchunks; ++ci) {
        const int64_t t0 = (int64_t)ci * kT;
        const bool vec_ok = t0 + kV * q < L;
        // ---- this chunk's staged inputs (copied during the previous scan)
        cp_async_wait<0>();
        // ---- prologue in registers for both channels; (delta, delta*u) to
        // shared memory, gate and D*u kept for the epilogue
        float gk[2][kV], duk[2][kV];
        {
            float dlc[2][kV], duc[2][kV];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float xs[kV], dts[kV], zs[kV], u[kV];
                unpack8(&sm.xz.x[2 * pr + c][kV * q], xs);
                unpack8(&sm.xz.dt[2 * pr + c][kV * q], dts);
                unpack8(&sm.xz.z[2 * pr + c][kV * q], zs);
                prologue8<W>(p, cp[c], xs, dts, zs, has_z, vec_ok && ok[c], q, lane, dlc[c], duc[c], u, gk[c]);
#pragma unroll
                for (int i = 0; i < kV; ++i) duk[c][i] = cp[c].dskip * u[i];
            }
#pragma unroll
            for (int i = 0; i < kV; ++i)
                sm.dd[pr][kV * q + i] = make_float4(dlc[0][i], dlc[1][i], duc[0][i], duc[1][i]);
        }
        // every thread has waited for its own copies of this chunk: after the
        // barrier all B/C rows are visible.  x/dt/z words were read back by
        // their own thread, so the next chunk's copies can start now and fly
        // during the scan (B/C into the other buffer).
        __syncwarp();
        if (ci + 1 < nchunks) fetch(ci + 1);
        const RawBC<IoT>& bc = sm.bc[ci & 1];

        // ---- scan: thread (pr, q) updates state entries 4q..4q+3 of both
        // channels; packed pairs run across the two channels
#pragma unroll 2
        for (int tt = 0; tt < kT; tt += 4) {
            float v[8];  // v[2k + c]: partial readout of step tt+k, channel c
#pragma unroll
            for (int s0 = 0; s0 < 4; s0 += kQ) {
                // B/C of rows 4q + j for steps tt+s0 .. tt+s0+kQ-1
                uint2 wb[4], wc[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = 4 * q + j;
                    const int e = tt + s0;
                    const int off = bc_swz(n, e / kE) * kE + e % kE;
                    wb[j] = *reinterpret_cast<const uint2*>(&bc.B[n][off]);
                    wc[j] = *reinterpret_cast<const uint2*>(&bc.C[n][off]);
                }
#pragma unroll
                for (int kk = 0; kk < kQ; ++kk) {
                    const int k = s0 + kk;
                    const float4 dd = sm.dd[pr][tt + k];
                    const u64 dl2 = pk(dd.x, dd.y);
                    const u64 du2 = pk(dd.z, dd.w);
                    u64 y2 = 0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float bj = elt8<IoT>(wb[j], kk);
                        const float cj = elt8<IoT>(wc[j], kk);
                        const u64 x2 = fmul2(dl2, Ap[j]);
                        const u64 a2 = j < SW ? exp2_pair_fma(x2) : exp2_pair_sfu(x2);
                        hp[j] = ffma2(a2, hp[j], fmul2(du2, pk(bj, bj)));
                        y2 = j == 0 ? fmul2(pk(cj, cj), hp[j]) : ffma2(pk(cj, cj), hp[j], y2);
                    }
                    upk(y2, v[2 * k], v[2 * k + 1]);
                }
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
                sm.y[2 * pr][tt + q] = v[0];
                sm.y[2 * pr + 1][tt + q] = v[1];
            }
        }
        __syncwarp();

        // ---- epilogue: D skip, gate and store 8 steps of both channels
        if (vec_ok) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (!ok[c]) continue;
                const int ch = 2 * pr + c;
                const float4 y0 = *reinterpret_cast<const float4*>(&sm.y[ch][kV * q]);
                const float4 y1 = *reinterpret_cast<const float4*>(&sm.y[ch][kV * q + 4]);
                const float ys[kV] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                float o[kV];
#pragma unroll
                for (int i = 0; i < kV; ++i) o[i] = (ys[i] + duk[c][i]) * gk[c][i];
                store8<IoT>(orow[c] + t0 + kV * q, o);
            }
        }
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
        // (once per kernel and device)
        int unused = 0;
        cudaError_t e = prepared_launch(
            reinterpret_cast<const void*>(kern), 0, kThreads, &unused,
            [&](int) {
                return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                            cudaSharedmemCarveoutMaxShared);
            },
            [](int* n) {
                *n = 0;
                return cudaSuccess;
            });
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
