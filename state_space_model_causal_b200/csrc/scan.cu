// scan.cu -- fused prefill for sm_100a: causal conv1d -> SiLU -> softplus(dt +
// dt_bias) -> selective scan -> D skip -> SiLU(z) gate, the operator chain
// "causal-conv1d, selective-scan, silu, element-mul" of "feat(llama.cu): 适配
// mamba 模型" (section 2.1), with the conv and SSM state caches read at the
// start and written at the end (same page, section 3.1).
//
// Per channel d (of batch b) and per time step t:
//     u     = silu(bias[d] + sum_k w[d,k] * x[t-(W-1)+k])      (u = x without conv)
//     delta = softplus(dt[t] + dt_bias[d])
//     h[n]  = exp(delta * A[d,n]) * h[n] + delta * B[n,t] * u
//     out   = (sum_n C[n,t] * h[n] + D[d] * u) * silu(z[t])
//
// Design.  B*D*N independent recurrences give enough parallelism on their own
// (327,680 for a 2.8B-shaped layer at batch 4), so the sequence is NOT split
// across CTAs: each exp(delta*A) is evaluated exactly once, which matters
// because the scan is bound by the SFU's exponential throughput, not by HBM.
// A CTA owns DT channels of one batch entry for the whole sequence.  NS threads
// share a channel, each holding 4 of its state entries h[n] in registers.
// Time is processed in smem-staged chunks of T steps, four phases each:
//   stage     raw x (with a W-1 halo), B and C tiles -> shared memory
//   prologue  conv + SiLU, softplus(dt) per (channel, t) -> shared memory
//   scan      the recurrence; the per-thread partial readouts of NS threads
//             are summed with a butterfly reduce-scatter (NS-1 shuffles per NS
//             steps), leaving one full y per lane
//   epilogue  D skip, SiLU(z) gate, store
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

namespace ssm {
namespace {

constexpr int kHalo = 8;  // history slots in front of each staged x row (W <= 8)
constexpr int kNPT = 4;   // state entries per thread

template <int DT, int T, int NS>
struct ScanSmem {
    static constexpr int NP = NS * kNPT;  // padded d_state
    static constexpr int XS = T + kHalo;  // row stride of sX
    static constexpr int TS = T + 4;      // row stride of the other tiles
    static constexpr int X = 0;
    static constexpr int DL = X + DT * XS;
    static constexpr int U = DL + DT * TS;
    static constexpr int Y = U + DT * TS;
    static constexpr int BB = Y + DT * TS;
    static constexpr int CC = BB + NP * TS;
    static constexpr int FLOATS = CC + NP * TS;
    static constexpr int BYTES = FLOATS * 4;
};

template <typename IoT, int NS, int DT, int T>
__global__ void __launch_bounds__(DT * NS) scan_chunked_kernel(const ScanProblem p) {
    using S = ScanSmem<DT, T, NS>;
    static_assert(T % NS == 0 && T >= kHalo, "chunk must hold whole reduce groups and a halo");
    extern __shared__ float smem[];
    float* sX = smem + S::X;
    float* sDl = smem + S::DL;
    float* sU = smem + S::U;
    float* sY = smem + S::Y;
    float* sB = smem + S::BB;
    float* sC = smem + S::CC;

    constexpr int NT = DT * NS;
    const int tid = threadIdx.x;
    const int ch = tid / NS;
    const int ns = tid % NS;
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * DT;
    const int64_t d = d0 + ch;
    const bool d_ok = d < p.D;
    const int64_t g = d0 / p.ch_per_group;
    const int W = (int)p.W;
    const IoT* __restrict__ xg = static_cast<const IoT*>(p.x);
    const IoT* __restrict__ dtg = static_cast<const IoT*>(p.dt);
    const IoT* __restrict__ zg = static_cast<const IoT*>(p.z);
    const IoT* __restrict__ Bg = static_cast<const IoT*>(p.Bm);
    const IoT* __restrict__ Cg = static_cast<const IoT*>(p.Cm);
    IoT* __restrict__ og = static_cast<IoT*>(p.out);

    // state entries owned by this thread: n = ns*4 + j
    float h[kNPT], A2[kNPT];
#pragma unroll
    for (int j = 0; j < kNPT; ++j) {
        const int64_t n = ns * kNPT + j;
        const bool ok = d_ok && n < p.N;
        A2[j] = ok ? p.A[d * p.A_d + n * p.A_n] * kLog2e : 0.0f;
        h[j] = (ok && p.ssm_state) ? p.ssm_state[b * p.ss_b + d * p.ss_d + n * p.ss_n] : 0.0f;
    }

    // initial conv history: slot k holds time k - kHalo; conv_state entry
    // e = W - kHalo + k (entries 1..W-1 are the W-1 most recent raw inputs)
    for (int i = tid; i < DT * kHalo; i += NT) {
        const int c = i / kHalo, k = i % kHalo;
        const int64_t dd = d0 + c;
        const int e = W - kHalo + k;
        float v = 0.0f;
        if (W > 0 && p.conv_state && dd < p.D && e >= 1)
            v = ld_f(p.conv_state, b * p.cs_b + dd * p.cs_d + e * p.cs_k, p.cs_dt);
        sX[c * S::XS + k] = v;
    }

    int valid = 0;
    for (int64_t t0 = 0; t0 < p.L; t0 += T) {
        valid = (int)(p.L - t0 < (int64_t)T ? p.L - t0 : (int64_t)T);
        const bool last = t0 + T >= p.L;
        // ---- stage: raw x, B and C tiles
        for (int i = tid; i < DT * T; i += NT) {
            const int c = i / T, t = i % T;
            const int64_t dd = d0 + c;
            float v = 0.0f;
            if (dd < p.D && t < valid) v = to_f(xg[b * p.x_b + dd * p.x_d + (t0 + t) * p.x_t]);
            sX[c * S::XS + kHalo + t] = v;
        }
        for (int i = tid; i < S::NP * T; i += NT) {
            const int n = i / T, t = i % T;
            float vb = 0.0f, vc = 0.0f;
            if (n < p.N && t < valid) {
                vb = to_f(Bg[b * p.B_b + g * p.B_g + n * p.B_n + (t0 + t) * p.B_t]);
                vc = to_f(Cg[b * p.C_b + g * p.C_g + n * p.C_n + (t0 + t) * p.C_t]);
            }
            sB[n * S::TS + t] = vb;
            sC[n * S::TS + t] = vc;
        }
        __syncthreads();
        // ---- prologue: u and delta per (channel, t)
        for (int i = tid; i < DT * T; i += NT) {
            const int c = i / T, t = i % T;
            const int64_t dd = d0 + c;
            float u = 0.0f, dl = 0.0f;
            if (dd < p.D && t < valid) {
                const float* xr = sX + c * S::XS + kHalo + t;
                if (W > 0) {
                    float acc = p.conv_b ? p.conv_b[dd * p.cb_d] : 0.0f;
                    for (int k = 0; k < W; ++k)
                        acc = fmaf(p.conv_w[dd * p.cw_d + k * p.cw_k], xr[k - (W - 1)], acc);
                    u = silu_f(acc);
                } else {
                    u = xr[0];
                }
                float v = to_f(dtg[b * p.dt_b + dd * p.dt_d + (t0 + t) * p.dt_t]);
                if (p.dt_bias) v += p.dt_bias[dd * p.db_d];
                dl = p.softplus ? softplus_f(v) : v;
            }
            sU[c * S::TS + t] = u;
            sDl[c * S::TS + t] = dl;
        }
        __syncthreads();
        // ---- scan (plus the halo hand-over to the next chunk)
        if (!last && ns == 0) {
#pragma unroll
            for (int k = 0; k < kHalo; ++k) sX[ch * S::XS + k] = sX[ch * S::XS + T + k];
        }
        {
            const float* dlr = sDl + ch * S::TS;
            const float* ur = sU + ch * S::TS;
            const float* Br = sB + (ns * kNPT) * S::TS;
            const float* Cr = sC + (ns * kNPT) * S::TS;
            for (int tt = 0; tt < T; tt += NS) {
                float yv[NS];
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    const int t = tt + q;
                    const float dl = dlr[t];
                    const float du = dl * ur[t];
                    float y = 0.0f;
#pragma unroll
                    for (int j = 0; j < kNPT; ++j) {
                        const float a = ex2_approx(dl * A2[j]);
                        h[j] = fmaf(a, h[j], du * Br[j * S::TS + t]);
                        y = fmaf(Cr[j * S::TS + t], h[j], y);
                    }
                    yv[q] = y;
                }
                // butterfly reduce-scatter: lane ns ends with the sum for t = tt + ns
#pragma unroll
                for (int s = NS / 2; s >= 1; s >>= 1) {
                    const bool upper = (ns & s) != 0;
#pragma unroll
                    for (int i = 0; i < s; ++i) {
                        const float send = upper ? yv[i] : yv[i + s];
                        const float keep = upper ? yv[i + s] : yv[i];
                        yv[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                    }
                }
                sY[ch * S::TS + tt + ns] = yv[0];
            }
        }
        __syncthreads();
        // ---- epilogue: D skip, gate, store
        for (int i = tid; i < DT * T; i += NT) {
            const int c = i / T, t = i % T;
            const int64_t dd = d0 + c;
            if (dd < p.D && t < valid) {
                float y = sY[c * S::TS + t];
                if (p.Dp) y = fmaf(p.Dp[dd * p.D_d], sU[c * S::TS + t], y);
                if (p.z) y *= silu_f(to_f(zg[b * p.z_b + dd * p.z_d + (t0 + t) * p.z_t]));
                og[b * p.o_b + dd * p.o_d + (t0 + t) * p.o_t] = from_f<IoT>(y);
            }
        }
    }

    // ---- final caches
    if (p.ssm_state && d_ok) {
#pragma unroll
        for (int j = 0; j < kNPT; ++j) {
            const int64_t n = ns * kNPT + j;
            if (n < p.N) p.ssm_state[b * p.ss_b + d * p.ss_d + n * p.ss_n] = h[j];
        }
    }
    if (W > 0 && p.conv_state && d_ok && ns == 0) {
        // last W raw inputs of (history ++ x): positions valid-W .. valid-1 of the last chunk
        for (int k = 0; k < W; ++k)
            st_f(p.conv_state, b * p.cs_b + d * p.cs_d + k * p.cs_k, p.cs_dt,
                 sX[ch * S::XS + kHalo + valid - W + k]);
    }
}

// ------------------------------------------------------------------------
// Generic prefill: one thread per (b, d), sequential over t, state in local
// memory.  Any strides, any group layout, d_state <= 256.
// ------------------------------------------------------------------------
constexpr int kGenericMaxN = 256;
constexpr int kMaxW = 8;

__global__ void __launch_bounds__(128) scan_generic_kernel(const ScanProblem p) {
    const int64_t total = p.Bn * p.D;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = idx / p.D;
        const int64_t d = idx - b * p.D;
        const int64_t g = d / p.ch_per_group;
        const int W = (int)p.W;
        float h[kGenericMaxN];
        for (int64_t n = 0; n < p.N; ++n)
            h[n] = p.ssm_state ? p.ssm_state[b * p.ss_b + d * p.ss_d + n * p.ss_n] : 0.0f;
        // win[k] = raw input at time t - W + k (the W most recent before t)
        float win[kMaxW];
        for (int k = 0; k < kMaxW; ++k) win[k] = 0.0f;
        if (W > 0 && p.conv_state)
            for (int k = 0; k < W; ++k)
                win[k] = ld_f(p.conv_state, b * p.cs_b + d * p.cs_d + k * p.cs_k, p.cs_dt);
        for (int64_t t = 0; t < p.L; ++t) {
            const float xv = ld_f(p.x, b * p.x_b + d * p.x_d + t * p.x_t, p.io_dt);
            float u = xv;
            if (W > 0) {
                for (int k = 0; k < W - 1; ++k) win[k] = win[k + 1];
                win[W - 1] = xv;
                float acc = p.conv_b ? p.conv_b[d * p.cb_d] : 0.0f;
                for (int k = 0; k < W; ++k) acc = fmaf(p.conv_w[d * p.cw_d + k * p.cw_k], win[k], acc);
                u = silu_f(acc);
            }
            float v = ld_f(p.dt, b * p.dt_b + d * p.dt_d + t * p.dt_t, p.io_dt);
            if (p.dt_bias) v += p.dt_bias[d * p.db_d];
            const float dl = p.softplus ? softplus_f(v) : v;
            const float dl2 = dl * kLog2e;
            const float du = dl * u;
            float y = 0.0f;
            for (int64_t n = 0; n < p.N; ++n) {
                const float a = ex2_approx(dl2 * p.A[d * p.A_d + n * p.A_n]);
                const float bn = ld_f(p.Bm, b * p.B_b + g * p.B_g + n * p.B_n + t * p.B_t, p.io_dt);
                const float cn = ld_f(p.Cm, b * p.C_b + g * p.C_g + n * p.C_n + t * p.C_t, p.io_dt);
                h[n] = fmaf(a, h[n], du * bn);
                y = fmaf(cn, h[n], y);
            }
            if (p.Dp) y = fmaf(p.Dp[d * p.D_d], u, y);
            if (p.z) y *= silu_f(ld_f(p.z, b * p.z_b + d * p.z_d + t * p.z_t, p.io_dt));
            st_f(p.out, b * p.o_b + d * p.o_d + t * p.o_t, p.io_dt, y);
        }
        if (p.ssm_state)
            for (int64_t n = 0; n < p.N; ++n) p.ssm_state[b * p.ss_b + d * p.ss_d + n * p.ss_n] = h[n];
        if (W > 0 && p.conv_state)
            for (int k = 0; k < W; ++k)
                st_f(p.conv_state, b * p.cs_b + d * p.cs_d + k * p.cs_k, p.cs_dt, win[k]);
    }
}

template <typename IoT, int NS, int DT, int T>
cudaError_t launch_chunked_t(const ScanProblem& p, const ScanPlan& plan, cudaStream_t s) {
    using S = ScanSmem<DT, T, NS>;
    auto kern = scan_chunked_kernel<IoT, NS, DT, T>;
    if (S::BYTES > 48 * 1024) {
        int unused = 0;
        cudaError_t e = prepared_launch(
            reinterpret_cast<const void*>(kern), S::BYTES, DT * NS, &unused,
            [&](int limit) { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, limit); },
            [](int* n) {
                *n = 0;
                return cudaSuccess;
            });
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((p.D + DT - 1) / DT), (unsigned)p.Bn);
    kern<<<grid, DT * NS, S::BYTES, s>>>(p);
    return cudaGetLastError();
}

template <typename IoT>
cudaError_t launch_chunked(const ScanProblem& p, const ScanPlan& plan, cudaStream_t s) {
    constexpr int T = 32;
    switch (plan.ns) {
        case 1: return launch_chunked_t<IoT, 1, 64, T>(p, plan, s);
        case 2: return launch_chunked_t<IoT, 2, 32, T>(p, plan, s);
        case 4: return launch_chunked_t<IoT, 4, 16, T>(p, plan, s);
        case 8: return launch_chunked_t<IoT, 8, 8, T>(p, plan, s);
        case 16: return launch_chunked_t<IoT, 16, 4, T>(p, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int scan_chunked_smem_bytes(int ns) {
    switch (ns) {
        case 1: return ScanSmem<64, 32, 1>::BYTES;
        case 2: return ScanSmem<32, 32, 2>::BYTES;
        case 4: return ScanSmem<16, 32, 4>::BYTES;
        case 8: return ScanSmem<8, 32, 8>::BYTES;
        case 16: return ScanSmem<4, 32, 16>::BYTES;
        default: return 0;
    }
}

cudaError_t launch_scan(const ScanProblem& p, const ScanPlan& plan, cudaStream_t s) {
    if (plan.kernel == SSM_KERNEL_SCAN_VEC) return launch_scan_vec(p, plan.sw_pairs, s);
    if (plan.kernel == SSM_KERNEL_SCAN_CHUNKED) {
        switch (p.io_dt) {
            case kF32: return launch_chunked<float>(p, plan, s);
            case kF16: return launch_chunked<__half>(p, plan, s);
            case kBF16: return launch_chunked<__nv_bfloat16>(p, plan, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.kernel == SSM_KERNEL_SCAN_GENERIC) {
        scan_generic_kernel<<<plan.grid, plan.block, 0, s>>>(p);
        return cudaGetLastError();
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssm
