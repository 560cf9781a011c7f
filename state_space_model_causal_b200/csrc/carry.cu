// carry.cu -- the two small kernels that join the pieces of a prefill split
// along the sequence (context parallelism, across calls, devices or ranks).
//
// The selective scan is a first-order linear recurrence in h: over a piece of
// steps, h_out = exp(A * S) * h_in + h_end, where S is the sum of the piece's
// delta and h_end the state the piece reaches from a zero start.  So a
// sequence cut into consecutive pieces can be scanned piece by piece from zero
// states at the same time, and the true state entering each piece composed
// afterwards: h_in(j+1) = exp(A * S(j)) * h_in(j) + h_end(j).  This serves the
// long-context case of "feat(llama.cu): 适配 mamba 模型" (section 6.1: the scan
// is linear in the sequence length).
//
//   delta_sum_kernel   S[b,d] = sum_t delta(dt[b,d,t] + dt_bias[d]); one warp per
//                      (b, d) row, lanes over t, the sum in double; delta is the
//                      prefill kernels' own softplus
//   carry_fold_kernel  state <- exp(A * S) * state + h_end, elementwise, grid-stride;
//                      the Mamba-1 layout (A per channel and state entry, S per
//                      channel) or the Mamba-2 layout (A and S per head)
//
// Both are tiny next to the prefill (B*D*L reads of dt; 3 * B*D*N floats),
// HBM-bound, and run once per piece.
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

namespace ssm {
namespace {

__global__ void __launch_bounds__(256) delta_sum_kernel(const DeltaSumProblem p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (row >= p.Bn * p.D) return;  // warp-uniform
    const int64_t b = row / p.D, d = row - b * p.D;
    const float bias = p.dt_bias ? p.dt_bias[d * p.db_d] : 0.0f;
    const int64_t base = b * p.dt_b + d * p.dt_d;
    double sum = 0.0;
    for (int64_t t = lane; t < p.L; t += 32) {
        const float v = ld_f(p.dt, base + t * p.dt_t, p.dt_dt) + bias;
        sum += (double)(p.softplus ? softplus_f(v) : v);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) p.out[b * p.o_b + d * p.o_d] = (float)sum;
}

__global__ void __launch_bounds__(256) carry_fold_kernel(const CarryFoldProblem p) {
    const int64_t total = p.Bn * p.H * p.P * p.N;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r = i;
        const int64_t n = r % p.N;
        r /= p.N;
        const int64_t pp = r % p.P;
        r /= p.P;
        const int64_t h = r % p.H, b = r / p.H;
        const float a = p.A[h * p.A_h + pp * p.A_p + n * p.A_n] * kLog2e;
        const float S = p.S[b * p.S_b + h * p.S_h];
        float* st = p.state + b * p.s_b + h * p.s_h + pp * p.s_p + n * p.s_n;
        *st = fmaf(ex2_approx(a * S), *st, p.h_end[b * p.h_b + h * p.h_h + pp * p.h_p + n * p.h_n]);
    }
}

}  // namespace

cudaError_t launch_delta_sum(const DeltaSumProblem& p, int grid, int block, cudaStream_t s) {
    delta_sum_kernel<<<grid, block, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_carry_fold(const CarryFoldProblem& p, int grid, int block, cudaStream_t s) {
    carry_fold_kernel<<<grid, block, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace ssm
