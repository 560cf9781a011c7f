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
// 16-byte aligned rows (a lane holds one 16-byte vector of steps; below).
// conv1d_kernel takes any strides: one warp owns one (b, d) row for the whole
// sequence, so the incoming state is read before the outgoing state is
// written with no cross-CTA ordering.
// Each lane handles kVPT consecutive steps per segment; the W-1 history values
// a lane needs come from its left neighbour by shuffle, and lane 0 takes them
// from the previous segment's last lane.  The op is HBM-bound (2 or 4 bytes in
// and out per element, W FMAs).
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

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
// (V = 8 steps at 16-bit, 4 at fp32), W - 1 <= V: a warp takes a segment of
// whole 32V-step blocks of one (b, d) row, a lane one 16-byte vector of V
// consecutive steps.  The W-1 inputs before a lane's steps come from the lane
// below by shuffle, before lane 0's from the previous block's lane 31, or at
// a segment start from the row itself (or the incoming state); the next
// block's load (or the next two blocks') is issued before the current one is
// computed.  Only the first
// segment of a row reads the incoming state (a segment is >= 32V > W-1
// steps), and its warp writes the outgoing state after all its lanes read.
template <typename IoT, int W, int Depth>
__global__ void __launch_bounds__(256) conv1d_vec_kernel(const Conv1dProblem p, int64_t S, int64_t nseg) {
    constexpr int V = 16 / (int)sizeof(IoT);
    constexpr int H = W > 1 ? W - 1 : 1;
    static_assert(W - 1 <= V, "the history must come from one lane below");
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= p.Bn * p.D * nseg) return;  // whole warps
    const int64_t row = gw / nseg, seg = gw % nseg;
    const int64_t b = row / p.D, d = row - b * p.D;
    const int64_t t0 = seg * S;
    const int64_t t1 = t0 + S < p.L ? t0 + S : p.L;
    const IoT* __restrict__ xr = static_cast<const IoT*>(p.x) + b * p.x_b + d * p.x_d;
    IoT* __restrict__ orow = static_cast<IoT*>(p.out) + b * p.o_b + d * p.o_d;
    const int64_t cs0 = b * p.cs_b + d * p.cs_d;

    float w[W];
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = p.w[d * p.w_d + k * p.w_k];
    const float bias = p.bias ? p.bias[d * p.b_d] : 0.0f;
    float carry[H];  // raw input at (block start) - (W-1) + i
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const int64_t t = t0 - (W - 1) + i;
        carry[i] = t >= 0 ? to_f(xr[t])
                          : (p.conv_state ? ld_f(p.conv_state, cs0 + (W + t) * p.cs_k, p.cs_dt) : 0.0f);
    }
    // loads run Depth blocks ahead of the arithmetic
    uint4 nx[Depth];
#pragma unroll
    for (int i = 0; i < Depth; ++i) {
        const int64_t t = t0 + lane * V + i * 32 * V;
        nx[i] = t < t1 ? *reinterpret_cast<const uint4*>(xr + t) : make_uint4(0, 0, 0, 0);
    }
    for (int64_t tb = t0; tb < t1; tb += 32 * V) {
        const int64_t t = tb + lane * V;
        const bool valid = t < t1;
        const uint4 cx = nx[0];
#pragma unroll
        for (int i = 0; i + 1 < Depth; ++i) nx[i] = nx[i + 1];
        if (t + Depth * 32 * V < t1) nx[Depth - 1] = *reinterpret_cast<const uint4*>(xr + t + Depth * 32 * V);
        float v[V], o[V];
        Vec16<IoT>::unpack(cx, v);
#pragma unroll
        for (int j = 0; j < V; ++j) v[j] = valid ? v[j] : 0.0f;
        float prev[H];
#pragma unroll
        for (int i = 0; i < W - 1; ++i) {
            const float up = __shfl_up_sync(0xffffffffu, v[V - (W - 1) + i], 1);
            prev[i] = lane == 0 ? carry[i] : up;
        }
#pragma unroll
        for (int i = 0; i < W - 1; ++i) carry[i] = __shfl_sync(0xffffffffu, v[V - (W - 1) + i], 31);
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
        if (valid) *reinterpret_cast<uint4*>(orow + t) = Vec16<IoT>::pack(o);
    }
    if (p.conv_state && seg == 0) {
        float nv = 0.0f;
        if (lane < W) {
            const int64_t t = p.L - W + lane;
            nv = t >= 0 ? to_f(xr[t]) : ld_f(p.conv_state, cs0 + (p.L + lane) * p.cs_k, p.cs_dt);
        }
        __syncwarp();
        if (lane < W) st_f(p.conv_state, cs0 + lane * p.cs_k, p.cs_dt, nv);
    }
}

template <typename IoT, int D>
cudaError_t launch_vec(const Conv1dProblem& p, const Conv1dPlan& plan, cudaStream_t s) {
    constexpr int V = 16 / (int)sizeof(IoT);
    const int64_t S = plan.seg_steps, nseg = plan.nseg;
    switch (p.W) {
        case 1: conv1d_vec_kernel<IoT, 1, D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break;
        case 2: conv1d_vec_kernel<IoT, 2, D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break;
        case 3: conv1d_vec_kernel<IoT, 3, D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break;
        case 4: conv1d_vec_kernel<IoT, 4, D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break;
        case 5: conv1d_vec_kernel<IoT, 5, D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break;
        case 6: if constexpr (V >= 5) { conv1d_vec_kernel<IoT, (V >= 5 ? 6 : 1), D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break; }
                return cudaErrorInvalidValue;
        case 7: if constexpr (V >= 6) { conv1d_vec_kernel<IoT, (V >= 6 ? 7 : 1), D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break; }
                return cudaErrorInvalidValue;
        case 8: if constexpr (V >= 7) { conv1d_vec_kernel<IoT, (V >= 7 ? 8 : 1), D><<<plan.grid, plan.block, 0, s>>>(p, S, nseg); break; }
                return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv1d(const Conv1dProblem& p, const Conv1dPlan& plan, cudaStream_t s) {
    if (plan.kernel == SSM_KERNEL_CONV1D) {
        const bool d2 = plan.depth == 2;
        switch (p.io_dt) {
            case kF32: return d2 ? launch_vec<float, 2>(p, plan, s) : launch_vec<float, 1>(p, plan, s);
            case kF16: return d2 ? launch_vec<__half, 2>(p, plan, s) : launch_vec<__half, 1>(p, plan, s);
            case kBF16:
                return d2 ? launch_vec<__nv_bfloat16, 2>(p, plan, s) : launch_vec<__nv_bfloat16, 1>(p, plan, s);
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
