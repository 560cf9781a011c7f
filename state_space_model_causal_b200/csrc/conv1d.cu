// conv1d.cu -- depthwise causal conv1d (+ optional SiLU) for sm_100a, the
// "causal-conv1d" operator of "feat(llama.cu): 适配 mamba 模型" (section 2.1),
// with the conv-state cache read before and written after the sequence
// (section 3.1 of the same page).
//
//     out[b,d,t] = act(bias[d] + sum_{k<W} w[d,k] * x[b,d,t-(W-1)+k])
//
// x at t < 0 comes from the incoming conv state (its last W-1 entries).  The
// outgoing conv state is the last W raw inputs of (incoming state ++ x).
//
// Two kernels.  conv1d_vec_kernel takes the time-contiguous layout with
// 16-byte aligned rows (units of 4 or 8 512-byte blocks of a row; below).
// conv1d_kernel takes any strides: one warp owns one (b, d) row for the whole
// sequence, so the incoming state is read before the outgoing state is
// written with no cross-CTA ordering; each lane handles kVPT consecutive
// steps per segment, the W-1 history values a lane needs come from its left
// neighbour by shuffle, and lane 0 takes them from the previous segment's
// last lane.  The op is HBM-bound (2 or 4 bytes in and out per element, W
// FMAs).
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

#include <type_traits>

namespace ssm {
namespace {

constexpr int kVPT = 8;        // steps per lane per segment (>= W - 1)
constexpr int kWarpsPerCta = 4;
constexpr int kMaxW = 8;

template <typename IoT>
__global__ void __launch_bounds__(32 * kWarpsPerCta) conv1d_kernel(const Conv1dProblem p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    if (row >= p.Bn * p.D) return;  // whole warp leaves together
    const int64_t b = row / p.D;
    const int64_t d = row - b * p.D;
    const int W = (int)p.W;
    const IoT* __restrict__ xr = static_cast<const IoT*>(p.x) + b * p.x_b + d * p.x_d;
    IoT* __restrict__ orow = static_cast<IoT*>(p.out) + b * p.o_b + d * p.o_d;
    const int64_t cs_off = b * p.cs_b + d * p.cs_d;

    float w[kMaxW];
#pragma unroll
    for (int k = 0; k < kMaxW; ++k) w[k] = k < W ? p.w[d * p.w_d + k * p.w_k] : 0.0f;
    const float bias = p.bias ? p.bias[d * p.b_d] : 0.0f;

    // lane k < W keeps incoming conv-state entry k for the final hand-over
    float cs_in = 0.0f;
    if (p.conv_state && lane < W) cs_in = ld_f(p.conv_state, cs_off + lane * p.cs_k, p.cs_dt);
    // carry[j] = raw input at time (segment start) - (W-1) + j, j < W-1
    float carry[kMaxW];
#pragma unroll
    for (int j = 0; j < kMaxW; ++j) carry[j] = __shfl_sync(0xffffffffu, cs_in, (j + 1) & 31);

    for (int64_t seg = 0; seg < p.L; seg += 32 * kVPT) {
        const int64_t t_base = seg + (int64_t)lane * kVPT;
        float xv[kVPT];
#pragma unroll
        for (int i = 0; i < kVPT; ++i) {
            const int64_t t = t_base + i;
            xv[i] = t < p.L ? to_f(xr[t * p.x_t]) : 0.0f;
        }
        // history from the left neighbour: its last W-1 values
        float hist[kMaxW];
#pragma unroll
        for (int j = 0; j < kMaxW - 1; ++j) {
            const float from_left = __shfl_up_sync(0xffffffffu, xv[kVPT - (kMaxW - 1) + j], 1);
            hist[j] = from_left;
        }
        // hist[j] (j < kMaxW-1) = input at t_base - (kMaxW-1) + j; lane 0 uses the carry
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < kMaxW - 1; ++j) {
                const int jj = j - (kMaxW - 1) + (W - 1);  // index into carry
                hist[j] = (jj >= 0 && jj < W - 1) ? carry[jj] : 0.0f;
            }
        }
#pragma unroll
        for (int i = 0; i < kVPT; ++i) {
            float acc = bias;
#pragma unroll
            for (int k = 0; k < kMaxW; ++k) {
                if (k < W) {
                    const int pos = i - (W - 1) + k;  // relative to t_base
                    const float v = pos >= 0 ? xv[pos < kVPT ? pos : 0] : hist[(kMaxW - 1) + pos];
                    acc = fmaf(w[k], v, acc);
                }
            }
            const int64_t t = t_base + i;
            if (t < p.L) orow[t * p.o_t] = from_f<IoT>(p.silu ? silu_f(acc) : acc);
        }
        // next segment's carry: the last W-1 inputs of this segment (lane 31)
#pragma unroll
        for (int j = 0; j < kMaxW - 1; ++j) {
            const int src_i = kVPT - (W - 1) + j;  // may be negative when unused
            const float v = __shfl_sync(0xffffffffu, xv[src_i >= 0 && src_i < kVPT ? src_i : 0], 31);
            if (j < W - 1) carry[j] = v;
        }
    }

    if (p.conv_state) {
        // final state entry k = raw input at time L - W + k (from x or the incoming state)
        float v = 0.0f;
        const int64_t pos = p.L - W + lane;
        if (pos >= 0 && pos < p.L) v = to_f(xr[pos * p.x_t]);
        const int src = (int)(W + pos);  // incoming-state entry when pos < 0
        const float from_state = __shfl_sync(0xffffffffu, cs_in, (src >= 0 && src < 32) ? src : 0);
        if (pos < 0) v = from_state;
        __syncwarp();
        if (lane < W) st_f(p.conv_state, cs_off + lane * p.cs_k, p.cs_dt, v);
    }
}

// The time-contiguous layout with 16-byte aligned rows and L a multiple of V
// (V = 8 steps at 16-bit, 4 at fp32), W - 1 <= V.  The work is cut into units
// of U consecutive 32V-step blocks (U x 512 bytes) of one (b, d) row, numbered
// row-major, and the persistent warps take units gw, gw + nw, ... (nw warps in
// the grid): at any moment neighbouring warps read and write neighbouring
// stretches of memory, one contiguous front through the tensor as in a copy,
// not one front per row.  A warp issues all U block loads of its unit at
// once, then computes the blocks in order.  A lane holds one 16-byte vector
// of V steps per block; the W-1 inputs before a lane's steps come from the
// lane below by shuffle, before lane 0's from the previous block's lane 31,
// and at the unit's start from the 16-byte vector ahead of it (or, at a row's
// start, the incoming state).  A row's incoming state is read only by the warp
// on its first unit, and that warp writes the outgoing state (the last W raw
// inputs, read back from the row) after its lanes have read.
//
// U (U x 512 bytes of loads in flight per warp) is 8 for fp16 and fp32 up to
// W = 4 and 4 otherwise (at 8, bf16 and the larger widths spill); 3 CTAs of
// 256 threads per SM (the launch bounds' register cap).  Measured at the 2.8B
// conv shape: 8 blocks 40.9-41.5 us, 4 blocks 42.4-43.1 us, 2 blocks (at 4
// CTAs per SM) 47.9 us.
template <typename IoT>
constexpr int unroll_of(int W) {
    return (sizeof(IoT) == 4 || std::is_same<IoT, __half>::value) && W <= 4 ? 8 : 4;
}
constexpr int kVecCtasPerSm = 3;

template <typename IoT, int W, int U = unroll_of<IoT>(W)>
__global__ void __launch_bounds__(256, kVecCtasPerSm) conv1d_vec_kernel(const Conv1dProblem p, int64_t nbs, int64_t units) {
    constexpr int V = 16 / (int)sizeof(IoT);
    constexpr int H = W > 1 ? W - 1 : 1;
    constexpr int64_t kSeg = (int64_t)U * 32 * V;  // steps per unit
    static_assert(W - 1 <= V, "the history must come from one lane below");
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * 8;
    const uint4 zero = make_uint4(0, 0, 0, 0);

    int64_t u = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (u >= units) return;  // whole warps
    // the unit's (b, d, segment), advanced by nw units per step without
    // division: nw = q nbs + rs units, q = qd D + qr rows
    const int64_t q = nw / nbs, rs = nw - q * nbs;
    const int64_t qd = q / p.D, qr = q - qd * p.D;
    int64_t sg = u % nbs, d = (u / nbs) % p.D, b = (u / nbs) / p.D;
    for (; u < units; u += nw) {
        const IoT* __restrict__ xr = static_cast<const IoT*>(p.x) + b * p.x_b + d * p.x_d;
        IoT* __restrict__ orow = static_cast<IoT*>(p.out) + b * p.o_b + d * p.o_d;
        const int64_t cs0 = b * p.cs_b + d * p.cs_d;
        const int64_t t0 = sg * kSeg;
        uint4 xv[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int64_t t = t0 + i * 32 * V + lane * V;
            xv[i] = t < p.L ? *reinterpret_cast<const uint4*>(xr + t) : zero;
        }
        float w[W];
#pragma unroll
        for (int k = 0; k < W; ++k) w[k] = p.w[d * p.w_d + k * p.w_k];
        const float bias = p.bias ? p.bias[d * p.b_d] : 0.0f;
        // carry[k] = input at t0 - (W-1) + k (lane 0's history), then the
        // previous block's last W-1 inputs
        float carry[H];
        if (sg > 0) {
            float hv[V];
            Vec16<IoT>::unpack(*reinterpret_cast<const uint4*>(xr + t0 - V), hv);
#pragma unroll
            for (int k = 0; k < W - 1; ++k) carry[k] = hv[V - (W - 1) + k];
        } else {
#pragma unroll
            for (int k = 0; k < W - 1; ++k)
                carry[k] = p.conv_state ? ld_f(p.conv_state, cs0 + (k + 1) * p.cs_k, p.cs_dt) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            if (t0 + i * 32 * V >= p.L) break;  // uniform: the row ends before this block
            const int64_t t = t0 + i * 32 * V + lane * V;
            float v[V], o[V];
            Vec16<IoT>::unpack(xv[i], v);  // zero past the row's end
            float prev[H];
#pragma unroll
            for (int k = 0; k < W - 1; ++k) {
                const float up = __shfl_up_sync(0xffffffffu, v[V - (W - 1) + k], 1);
                prev[k] = lane == 0 ? carry[k] : up;
            }
#pragma unroll
            for (int k = 0; k < W - 1; ++k) carry[k] = __shfl_sync(0xffffffffu, v[V - (W - 1) + k], 31);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                float acc = bias;
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const int idx = j - (W - 1) + k;
                    acc = fmaf(w[k], idx >= 0 ? v[idx] : prev[W - 1 + idx], acc);
                }
                o[j] = p.silu ? silu_f(acc) : acc;
            }
            if (t < p.L) *reinterpret_cast<uint4*>(orow + t) = Vec16<IoT>::pack(o);
        }
        if (sg == 0 && p.conv_state) {
            float nv = 0.0f;
            if (lane < W) {
                const int64_t tt = p.L - W + lane;
                nv = tt >= 0 ? to_f(xr[tt]) : ld_f(p.conv_state, cs0 + (p.L + lane) * p.cs_k, p.cs_dt);
            }
            __syncwarp();
            if (lane < W) st_f(p.conv_state, cs0 + lane * p.cs_k, p.cs_dt, nv);
        }
        // next unit
        sg += rs;
        int64_t c = 0;
        if (sg >= nbs) {
            sg -= nbs;
            c = 1;
        }
        d += qr + c;
        b += qd;
        if (d >= p.D) {
            d -= p.D;
            ++b;
        }
    }
}

template <typename IoT>
cudaError_t launch_vec(const Conv1dProblem& p, const Conv1dPlan& plan, cudaStream_t s) {
    constexpr int V = 16 / (int)sizeof(IoT);
    const int64_t nbs = plan.units_per_row, units = plan.units;
    switch (p.W) {
        case 1: conv1d_vec_kernel<IoT, 1><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break;
        case 2: conv1d_vec_kernel<IoT, 2><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break;
        case 3: conv1d_vec_kernel<IoT, 3><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break;
        case 4: conv1d_vec_kernel<IoT, 4><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break;
        case 5: conv1d_vec_kernel<IoT, 5><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break;
        case 6: if constexpr (V >= 5) { conv1d_vec_kernel<IoT, (V >= 5 ? 6 : 1)><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break; }
                return cudaErrorInvalidValue;
        case 7: if constexpr (V >= 6) { conv1d_vec_kernel<IoT, (V >= 6 ? 7 : 1)><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break; }
                return cudaErrorInvalidValue;
        case 8: if constexpr (V >= 7) { conv1d_vec_kernel<IoT, (V >= 7 ? 8 : 1)><<<plan.grid, plan.block, 0, s>>>(p, nbs, units); break; }
                return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

int conv1d_vec_ctas_per_sm() { return kVecCtasPerSm; }
int conv1d_vec_unroll(int io_dt, int64_t W) {
    if (W < 1 || W > 8) return 4;
    const int w = (int)W;
    return io_dt == kF32 ? unroll_of<float>(w) : io_dt == kF16 ? unroll_of<__half>(w) : unroll_of<__nv_bfloat16>(w);
}

cudaError_t launch_conv1d(const Conv1dProblem& p, const Conv1dPlan& plan, cudaStream_t s) {
    if (plan.kernel == SSM_KERNEL_CONV1D) {
        switch (p.io_dt) {
            case kF32: return launch_vec<float>(p, plan, s);
            case kF16: return launch_vec<__half>(p, plan, s);
            case kBF16: return launch_vec<__nv_bfloat16>(p, plan, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.kernel != SSM_KERNEL_CONV1D_GENERIC) return cudaErrorInvalidValue;
    switch (p.io_dt) {
        case kF32: conv1d_kernel<float><<<plan.grid, plan.block, 0, s>>>(p); break;
        case kF16: conv1d_kernel<__half><<<plan.grid, plan.block, 0, s>>>(p); break;
        case kBF16: conv1d_kernel<__nv_bfloat16><<<plan.grid, plan.block, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ssm
