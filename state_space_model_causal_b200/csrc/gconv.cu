// gconv.cu -- the double-gated short causal conv for sm_100a: the convolution
// of the "double-gated LIV convolution blocks" named in
// "LFM2.5-1.2B-Thinking性能优化CUDA核心编程技巧" (section 2.1).  The page prints
// no equation; the reading is two input-dependent gates around a depthwise
// causal conv, no activation:
//
//     v[t]   = Bg[t] * x[t]
//     out[t] = Cg[t] * (bias + sum_{k<W} w[k] * v[t-(W-1)+k])
//
// v at t < 0 comes from the incoming conv state (the last W gated inputs,
// oldest first); the outgoing state is the last W entries of (state ++ v).
// One call serves a prefill (L tokens) and a decode step (L = 1).
//
// What bounds it: HBM.  Per (b, t, d) it reads x, Bg, Cg and writes out (8
// bytes at 16-bit I/O) for W + 2 FP32 operations.  The design streams those
// bytes with 16-byte accesses:
//
//   * A thread owns V channels that sit next to each other in memory (one
//     16-byte vector: 8 at 16-bit, 4 at fp32) and a segment of S steps.  In the
//     layout a token-major projection writes (channels contiguous, tokens
//     strided), the 32 lanes of a warp read 512 contiguous bytes per tensor and
//     step.  Consecutive threads take consecutive vectors, then segments, then
//     batch entries; the segments are sized so that the grid is one wave of
//     kCtasPerSm CTAs on every SM.
//   * Each thread keeps the next kP steps of its three input vectors in flight
//     through its own ring in shared memory (16-byte cp.async, one commit
//     group per step, L1 bypassed): the bytes in flight cost shared memory,
//     not registers, and no thread waits on another (a thread only reads the
//     slots it filled itself, after cp.async.wait_group).
//   * The W-1 gated inputs before a segment are re-read from the sequence (or
//     the incoming state); a segment is at least W-1 steps long, so only the
//     first segment of a row ever reads the state.  That segment's thread also
//     writes the outgoing state, after its reads, in ascending entry order:
//     new entry k reads old entry L + k > k, so nothing it still needs is
//     overwritten, and no other thread touches the state.
//   * In the time-contiguous layout ((B, D, L) rows, as the Mamba tensors
//     are laid out) a warp takes a segment of one row and a lane 16-byte
//     vectors of consecutive steps, the history passed between lanes by
//     shuffle (gconv_rows_kernel).
//   * Any other layout runs a plain kernel (one channel per thread, scalar
//     loads at any strides, U steps of loads issued together).
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

#include <type_traits>

namespace ssm {
namespace {

// V consecutive channels of one step: loaded raw (one 16-byte vector, or one
// element when V = 1), widened only when used
template <typename IoT, int V> struct Lane {
    using Raw = typename std::conditional<V == 1, IoT, uint4>::type;
    __device__ __forceinline__ static Raw load(const IoT* p, int64_t i) {
        if constexpr (V == 1) {
            return p[i];
        } else {
            return *reinterpret_cast<const uint4*>(p + i);
        }
    }
    __device__ __forceinline__ static void widen(const Raw& r, float* f) {
        if constexpr (V == 1) {
            f[0] = to_f(r);
        } else {
            Vec16<IoT>::unpack(r, f);
        }
    }
    __device__ __forceinline__ static void store(IoT* p, int64_t i, const float* f) {
        if constexpr (V == 1) {
            p[i] = from_f<IoT>(f[0]);
        } else {
            *reinterpret_cast<uint4*>(p + i) = Vec16<IoT>::pack(f);
        }
    }
    // the gated input b * x of V channels at element offsets xi, bi
    __device__ __forceinline__ static void gated(const IoT* x, int64_t xi, const IoT* b, int64_t bi, float* v) {
        float xf[V], bf[V];
        widen(load(x, xi), xf);
        widen(load(b, bi), bf);
#pragma unroll
        for (int c = 0; c < V; ++c) v[c] = bf[c] * xf[c];
    }
};

constexpr int kBlock = 256;     // threads per CTA
constexpr int kP = 8;           // steps in flight per thread (vector kernel)
constexpr int kCtasPerSm = 2;   // vector kernel: 96 KB of ring per CTA, <= 128 registers

// any strides: one channel per thread, scalar loads, U steps of loads issued
// together
template <typename IoT, int W>
__global__ void __launch_bounds__(kBlock) gconv_kernel(const GatedConvProblem p) {
    constexpr int V = 1;
    using LN = Lane<IoT, V>;
    constexpr int U = 8;
    const int64_t nv = p.D / V;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= p.Bn * p.nseg * nv) return;
    const int64_t dv = idx % nv;
    const int64_t rest = idx / nv;
    const int64_t seg = rest % p.nseg;
    const int64_t b = rest / p.nseg;
    const int64_t d0 = dv * V;
    const int64_t t0 = seg * p.S;
    const int64_t t1 = t0 + p.S < p.L ? t0 + p.S : p.L;

    const int64_t xo = b * p.x_b + d0 * p.x_d, bo = b * p.bg_b + d0 * p.bg_d;
    const int64_t co = b * p.cg_b + d0 * p.cg_d, oo = b * p.o_b + d0 * p.o_d;
    const IoT* __restrict__ xp = static_cast<const IoT*>(p.x);
    const IoT* __restrict__ bp = static_cast<const IoT*>(p.bg);
    const IoT* __restrict__ cp = static_cast<const IoT*>(p.cg);
    IoT* __restrict__ op = static_cast<IoT*>(p.out);

    float w[V][W], bias[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
#pragma unroll
        for (int k = 0; k < W; ++k) w[c][k] = p.w[(d0 + c) * p.w_d + k * p.w_k];
        bias[c] = p.bias ? p.bias[(d0 + c) * p.b_d] : 0.0f;
    }

    // window: hv[k] = gated input at step (t - (W-1) + k) for the step t about to run
    float hv[W][V];
#pragma unroll
    for (int k = 0; k < W - 1; ++k) {
        const int64_t t = t0 - (W - 1) + k;
        if (t >= 0) {
            LN::gated(xp, xo + t * p.x_t, bp, bo + t * p.bg_t, hv[k]);
        } else {
#pragma unroll
            for (int c = 0; c < V; ++c)
                hv[k][c] = p.conv_state
                               ? ld_f(p.conv_state, b * p.cs_b + (d0 + c) * p.cs_d + (W + t) * p.cs_k, p.cs_dt)
                               : 0.0f;
        }
    }

    for (int64_t tb = t0; tb < t1; tb += U) {
        typename LN::Raw xr[U], br[U], cr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = tb + u;
            if (t < t1) {
                xr[u] = LN::load(xp, xo + t * p.x_t);
                br[u] = LN::load(bp, bo + t * p.bg_t);
                cr[u] = LN::load(cp, co + t * p.cg_t);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = tb + u;
            if (t < t1) {
                float xf[V], bf[V], cf[V], o[V];
                LN::widen(xr[u], xf);
                LN::widen(br[u], bf);
                LN::widen(cr[u], cf);
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    hv[W - 1][c] = bf[c] * xf[c];
                    float acc = bias[c];
#pragma unroll
                    for (int k = 0; k < W; ++k) acc = fmaf(w[c][k], hv[k][c], acc);
                    o[c] = cf[c] * acc;
                }
                LN::store(op, oo + t * p.o_t, o);
#pragma unroll
                for (int k = 0; k < W - 1; ++k)
#pragma unroll
                    for (int c = 0; c < V; ++c) hv[k][c] = hv[k + 1][c];
            }
        }
    }

    // outgoing state, by the first segment's thread: entry k = gated input at
    // step L - W + k, from the sequence or (step < 0) old entry L + k
    if (p.conv_state && seg == 0 && p.L > 0) {
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const int64_t t = p.L - W + k;
            float v[V];
            if (t >= 0) {
                LN::gated(xp, xo + t * p.x_t, bp, bo + t * p.bg_t, v);
            } else {
#pragma unroll
                for (int c = 0; c < V; ++c)
                    v[c] = ld_f(p.conv_state, b * p.cs_b + (d0 + c) * p.cs_d + (p.L + k) * p.cs_k, p.cs_dt);
            }
#pragma unroll
            for (int c = 0; c < V; ++c) st_f(p.conv_state, b * p.cs_b + (d0 + c) * p.cs_d + k * p.cs_k, p.cs_dt, v[c]);
        }
    }
}

// the vector layout: V = 16 / sizeof(IoT) channels per thread, unit channel
// stride, 16-byte aligned vectors; a per-thread cp.async ring of kP steps
template <typename IoT, int W>
__global__ void __launch_bounds__(kBlock, kCtasPerSm) gconv_ring_kernel(const GatedConvProblem p) {
    constexpr int V = 16 / (int)sizeof(IoT);
    using LN = Lane<IoT, V>;
    extern __shared__ uint4 ring[];  // [kP][3][kBlock]: slot s, tensor k, thread
    const int tid = threadIdx.x;
    const int64_t nv = p.D / V;
    const int64_t idx = (int64_t)blockIdx.x * kBlock + tid;
    if (idx >= p.Bn * p.nseg * nv) return;  // no barrier below: a thread may leave
    const int64_t dv = idx % nv;
    const int64_t rest = idx / nv;
    const int64_t seg = rest % p.nseg;
    const int64_t b = rest / p.nseg;
    const int64_t d0 = dv * V;
    const int64_t t0 = seg * p.S;
    const int64_t t1 = t0 + p.S < p.L ? t0 + p.S : p.L;
    const IoT* __restrict__ xp = static_cast<const IoT*>(p.x) + b * p.x_b + d0;
    const IoT* __restrict__ bp = static_cast<const IoT*>(p.bg) + b * p.bg_b + d0;
    const IoT* __restrict__ cp = static_cast<const IoT*>(p.cg) + b * p.cg_b + d0;
    IoT* __restrict__ op = static_cast<IoT*>(p.out) + b * p.o_b + d0;

    // step t's three vectors into ring slot sl (an empty group past the segment)
    auto issue = [&](int64_t t, int sl) {
        if (t < t1) {
            cp_async16(&ring[(sl * 3 + 0) * kBlock + tid], xp + t * p.x_t, true);
            cp_async16(&ring[(sl * 3 + 1) * kBlock + tid], bp + t * p.bg_t, true);
            cp_async16(&ring[(sl * 3 + 2) * kBlock + tid], cp + t * p.cg_t, true);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int sl = 0; sl < kP; ++sl) issue(t0 + sl, sl);

    float w[V][W], bias[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
#pragma unroll
        for (int k = 0; k < W; ++k) w[c][k] = p.w[(d0 + c) * p.w_d + k * p.w_k];
        bias[c] = p.bias ? p.bias[(d0 + c) * p.b_d] : 0.0f;
    }
    // window: hv[k] = gated input at step (t - (W-1) + k) for the step t about to run
    float hv[W][V];
#pragma unroll
    for (int k = 0; k < W - 1; ++k) {
        const int64_t t = t0 - (W - 1) + k;
        if (t >= 0) {
            LN::gated(xp, t * p.x_t, bp, t * p.bg_t, hv[k]);
        } else {
#pragma unroll
            for (int c = 0; c < V; ++c)
                hv[k][c] = p.conv_state
                               ? ld_f(p.conv_state, b * p.cs_b + (d0 + c) * p.cs_d + (W + t) * p.cs_k, p.cs_dt)
                               : 0.0f;
        }
    }

    int sl = 0;
    for (int64_t t = t0; t < t1; ++t) {
        cp_async_wait<kP - 1>();  // this thread's copies of step t have landed
        float xf[V], bf[V], cf[V], o[V];
        LN::widen(ring[(sl * 3 + 0) * kBlock + tid], xf);
        LN::widen(ring[(sl * 3 + 1) * kBlock + tid], bf);
        LN::widen(ring[(sl * 3 + 2) * kBlock + tid], cf);
#pragma unroll
        for (int c = 0; c < V; ++c) {
            hv[W - 1][c] = bf[c] * xf[c];
            float acc = bias[c];
#pragma unroll
            for (int k = 0; k < W; ++k) acc = fmaf(w[c][k], hv[k][c], acc);
            o[c] = cf[c] * acc;
        }
        LN::store(op, t * p.o_t, o);
#pragma unroll
        for (int k = 0; k < W - 1; ++k)
#pragma unroll
            for (int c = 0; c < V; ++c) hv[k][c] = hv[k + 1][c];
        // the slot's values are in registers and used above: refill it
        issue(t + kP, sl);
        sl = sl + 1 == kP ? 0 : sl + 1;
    }
    cp_async_wait<0>();  // the groups past the segment are empty; nothing stays in flight

    // outgoing state, by the first segment's thread: entry k = gated input at
    // step L - W + k, from the sequence or (step < 0) old entry L + k
    if (p.conv_state && seg == 0) {
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const int64_t t = p.L - W + k;
            float v[V];
            if (t >= 0) {
                LN::gated(xp, t * p.x_t, bp, t * p.bg_t, v);
            } else {
#pragma unroll
                for (int c = 0; c < V; ++c)
                    v[c] = ld_f(p.conv_state, b * p.cs_b + (d0 + c) * p.cs_d + (p.L + k) * p.cs_k, p.cs_dt);
            }
#pragma unroll
            for (int c = 0; c < V; ++c) st_f(p.conv_state, b * p.cs_b + (d0 + c) * p.cs_d + k * p.cs_k, p.cs_dt, v[c]);
        }
    }
}

template <typename IoT>
cudaError_t launch_ring(const GatedConvProblem& p, int grid, cudaStream_t s) {
    auto run = [&](auto kern) -> cudaError_t {
        const int smem = gated_conv_ring_smem_bytes();
        int unused = 0;
        cudaError_t e = prepared_launch(
            reinterpret_cast<const void*>(kern), smem, kBlock, &unused,
            [&](int bytes) { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes); },
            [](int* n) {
                *n = 0;
                return cudaSuccess;
            });
        if (e != cudaSuccess) return e;
        kern<<<grid, kBlock, smem, s>>>(p);
        return cudaGetLastError();
    };
    switch (p.W) {
        case 1: return run(gconv_ring_kernel<IoT, 1>);
        case 2: return run(gconv_ring_kernel<IoT, 2>);
        case 3: return run(gconv_ring_kernel<IoT, 3>);
        case 4: return run(gconv_ring_kernel<IoT, 4>);
        case 5: return run(gconv_ring_kernel<IoT, 5>);
        case 6: return run(gconv_ring_kernel<IoT, 6>);
        case 7: return run(gconv_ring_kernel<IoT, 7>);
        case 8: return run(gconv_ring_kernel<IoT, 8>);
        default: return cudaErrorInvalidValue;
    }
}

template <typename IoT>
cudaError_t launch_generic(const GatedConvProblem& p, int grid, int block, cudaStream_t s) {
    switch (p.W) {
        case 1: gconv_kernel<IoT, 1><<<grid, block, 0, s>>>(p); break;
        case 2: gconv_kernel<IoT, 2><<<grid, block, 0, s>>>(p); break;
        case 3: gconv_kernel<IoT, 3><<<grid, block, 0, s>>>(p); break;
        case 4: gconv_kernel<IoT, 4><<<grid, block, 0, s>>>(p); break;
        case 5: gconv_kernel<IoT, 5><<<grid, block, 0, s>>>(p); break;
        case 6: gconv_kernel<IoT, 6><<<grid, block, 0, s>>>(p); break;
        case 7: gconv_kernel<IoT, 7><<<grid, block, 0, s>>>(p); break;
        case 8: gconv_kernel<IoT, 8><<<grid, block, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// the time-contiguous layout: x, b_gate, c_gate and out rows of L contiguous
// steps (16-byte aligned, L a multiple of V).  A warp takes a segment of S
// steps of one (b, d) row, a lane 16-byte vectors of V consecutive steps; the
// W-1 gated inputs before a lane's first step come from the lane below by
// shuffle (W - 1 <= V), before lane 0's from the previous block's lane 31, or
// at the segment start from the row itself (or the incoming state).  The
// next block's loads are issued before the current one is computed.
template <typename IoT, int W>
__global__ void __launch_bounds__(kBlock) gconv_rows_kernel(const GatedConvProblem p) {
    constexpr int V = 16 / (int)sizeof(IoT);
    constexpr int H = W > 1 ? W - 1 : 1;
    static_assert(W - 1 <= V, "the history must come from one lane below");
    using LN = Lane<IoT, V>;
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (kBlock / 32) + (threadIdx.x >> 5);
    if (gw >= p.Bn * p.D * p.nseg) return;  // whole warps
    const int64_t row = gw / p.nseg, seg = gw % p.nseg;
    const int64_t b = row / p.D, d = row - b * p.D;
    const int64_t t0 = seg * p.S;
    const int64_t t1 = t0 + p.S < p.L ? t0 + p.S : p.L;
    const IoT* __restrict__ xr = static_cast<const IoT*>(p.x) + b * p.x_b + d * p.x_d;
    const IoT* __restrict__ br = static_cast<const IoT*>(p.bg) + b * p.bg_b + d * p.bg_d;
    const IoT* __restrict__ cr = static_cast<const IoT*>(p.cg) + b * p.cg_b + d * p.cg_d;
    IoT* __restrict__ orow = static_cast<IoT*>(p.out) + b * p.o_b + d * p.o_d;
    const int64_t cs0 = b * p.cs_b + d * p.cs_d;

    float w[W];
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = p.w[d * p.w_d + k * p.w_k];
    const float bias = p.bias ? p.bias[d * p.b_d] : 0.0f;
    // carry[i] = gated input at step (block start) - (W-1) + i
    float carry[H];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const int64_t t = t0 - (W - 1) + i;
        carry[i] = t >= 0 ? to_f(br[t]) * to_f(xr[t])
                          : (p.conv_state ? ld_f(p.conv_state, cs0 + (W + t) * p.cs_k, p.cs_dt) : 0.0f);
    }

    uint4 nx = make_uint4(0, 0, 0, 0), nb = nx, nc = nx;
    {
        const int64_t t = t0 + lane * V;
        if (t < t1) {
            nx = LN::load(xr, t);
            nb = LN::load(br, t);
            nc = LN::load(cr, t);
        }
    }
    for (int64_t tb = t0; tb < t1; tb += 32 * V) {
        const int64_t t = tb + lane * V;
        const bool valid = t < t1;
        const uint4 cx = nx, cb = nb, cc = nc;
        const int64_t tn = t + 32 * V;  // the next block, in flight while this one is computed
        if (tn < t1) {
            nx = LN::load(xr, tn);
            nb = LN::load(br, tn);
            nc = LN::load(cr, tn);
        }
        float xf[V], bf[V], cf[V], v[V], o[V];
        LN::widen(cx, xf);
        LN::widen(cb, bf);
        LN::widen(cc, cf);
#pragma unroll
        for (int j = 0; j < V; ++j) v[j] = valid ? bf[j] * xf[j] : 0.0f;
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
            o[j] = cf[j] * acc;
        }
        if (valid) LN::store(orow, t, o);
    }

    // outgoing state, by the first segment's warp: lane k < W computes entry k
    // (the gated input at step L - W + k, or old entry L + k), all lanes read
    // before any writes
    if (p.conv_state && seg == 0) {
        float nv = 0.0f;
        if (lane < W) {
            const int64_t t = p.L - W + lane;
            nv = t >= 0 ? to_f(br[t]) * to_f(xr[t]) : ld_f(p.conv_state, cs0 + (p.L + lane) * p.cs_k, p.cs_dt);
        }
        __syncwarp();
        if (lane < W) st_f(p.conv_state, cs0 + lane * p.cs_k, p.cs_dt, nv);
    }
}

template <typename IoT>
cudaError_t launch_rows(const GatedConvProblem& p, int grid, cudaStream_t s) {
    constexpr int V = 16 / (int)sizeof(IoT);
    switch (p.W) {
        case 1: gconv_rows_kernel<IoT, 1><<<grid, kBlock, 0, s>>>(p); break;
        case 2: gconv_rows_kernel<IoT, 2><<<grid, kBlock, 0, s>>>(p); break;
        case 3: gconv_rows_kernel<IoT, 3><<<grid, kBlock, 0, s>>>(p); break;
        case 4: gconv_rows_kernel<IoT, 4><<<grid, kBlock, 0, s>>>(p); break;
        case 5: gconv_rows_kernel<IoT, 5><<<grid, kBlock, 0, s>>>(p); break;
        case 6: if constexpr (V >= 5) { gconv_rows_kernel<IoT, (V >= 5 ? 6 : 1)><<<grid, kBlock, 0, s>>>(p); break; }
                return cudaErrorInvalidValue;
        case 7: if constexpr (V >= 6) { gconv_rows_kernel<IoT, (V >= 6 ? 7 : 1)><<<grid, kBlock, 0, s>>>(p); break; }
                return cudaErrorInvalidValue;
        case 8: if constexpr (V >= 7) { gconv_rows_kernel<IoT, (V >= 7 ? 8 : 1)><<<grid, kBlock, 0, s>>>(p); break; }
                return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename IoT>
cudaError_t launch_io(const GatedConvProblem& p, int kernel, int grid, int block, cudaStream_t s) {
    if (kernel == SSM_KERNEL_GATED_CONV) return launch_ring<IoT>(p, grid, s);
    if (kernel == SSM_KERNEL_GATED_CONV_ROWS) return launch_rows<IoT>(p, grid, s);
    return launch_generic<IoT>(p, grid, block, s);
}

}  // namespace

int gated_conv_ring_smem_bytes() { return kP * 3 * kBlock * 16; }
int gated_conv_ctas_per_sm() { return kCtasPerSm; }
int gated_conv_block() { return kBlock; }

cudaError_t launch_gated_conv(const GatedConvProblem& p, int kernel, int grid, int block, cudaStream_t s) {
    if (kernel != SSM_KERNEL_GATED_CONV && kernel != SSM_KERNEL_GATED_CONV_ROWS &&
        kernel != SSM_KERNEL_GATED_CONV_GENERIC)
        return cudaErrorInvalidValue;
    if (block != kBlock) return cudaErrorInvalidValue;
    switch (p.io_dt) {
        case kF32: return launch_io<float>(p, kernel, grid, block, s);
        case kF16: return launch_io<__half>(p, kernel, grid, block, s);
        case kBF16: return launch_io<__nv_bfloat16>(p, kernel, grid, block, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssm
