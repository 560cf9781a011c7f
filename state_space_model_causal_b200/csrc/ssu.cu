// ssu.cu -- single-token selective_state_update for sm_100a.
//
// One decode step of the selective SSM for every row r = (b, h, p) of the
// state cache:
//     delta = softplus(dt + dt_bias)
//     state[r, n] = exp(delta * A) * state[r, n] + delta * B[g, n] * u
//     out[r]      = (sum_n C[g, n] * state[r, n] + D * u) * silu(z)
// with u = x, or u = silu(conv) after the fused conv-state roll of the
// Mamba-1 decode path.  The argument list follows the selective_state_update
// call of "[XPU] Add tuned Mamba SSU configs for Intel Arc Pro B70" (section
// 关键源码片段); the cache read-modify-write follows the Mamba state cache of
// "feat(llama.cu): 适配 mamba 模型" (section 3.1).
//
// The update is HBM-bound: every state element is read once and written once,
// with ~3 FP32 operations in between.  The vector kernel therefore streams
// the state with 16-byte evict-first loads and stores, keeps RPT rows per
// thread in flight, and reads B/C once per work item into registers.  A work
// item is a run of rows of one batch entry; the grid is a persistent
// multiple of the SM count walking the items.
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

namespace ssm {
namespace {

constexpr int kRowsPerThread = 4;  // rows each thread keeps in flight
constexpr int kMaxConvW = 8;

struct RowScalars {
    float u;      // input to the SSM (x or silu(conv))
    float delta;  // discretisation step
    float dl2;    // delta * log2(e), so that exp(delta*A) = 2^(dl2 * A)
};

// Per-row prologue shared by both kernels: Delta and u (u = silu(conv) over
// the rolled conv window when the conv is fused).  Reads only.
__device__ __forceinline__ RowScalars row_prologue(const SsuProblem& p, int64_t b, int64_t slot,
                                                   int64_t h, int64_t pp) {
    RowScalars rs;
    float xv = ld_f(p.x, b * p.x_b + h * p.x_h + pp * p.x_p, p.x_dt);
    if (p.W > 0) {
        const int64_t c = h * p.P + pp;
        const int64_t cs_off = slot * p.cs_b + c * p.cs_c;
        float acc = p.conv_b ? p.conv_b[c * p.cb_c] : 0.0f;
#pragma unroll
        for (int k = 0; k < kMaxConvW; ++k) {
            if (k < p.W) {
                // rolled window: old entries 1..W-1, then the new input
                const float v = (k == p.W - 1) ? xv : ld_f(p.conv_state, cs_off + (k + 1) * p.cs_w, p.cs_dt);
                acc = fmaf(p.conv_w[c * p.cw_c + k * p.cw_w], v, acc);
            }
        }
        xv = silu_f(acc);
    }
    float v = ld_f(p.dt, b * p.dt_b + h * p.dt_h + pp * p.dt_p, p.dt_dt);
    if (p.dt_bias) v += p.dt_bias[h * p.db_h + pp * p.db_p];
    rs.delta = p.softplus ? softplus_f(v) : v;
    rs.dl2 = rs.delta * kLog2e;
    rs.u = xv;
    return rs;
}

// Roll the channel's conv state left by one and append the raw input.  Called
// by one thread per row, after every lane of the row has read the old state.
__device__ __forceinline__ void conv_roll_store(const SsuProblem& p, int64_t b, int64_t slot,
                                                int64_t h, int64_t pp) {
    const int64_t c = h * p.P + pp;
    const int64_t cs_off = slot * p.cs_b + c * p.cs_c;
    const float xv = ld_f(p.x, b * p.x_b + h * p.x_h + pp * p.x_p, p.x_dt);
    float win[kMaxConvW];
#pragma unroll
    for (int k = 0; k < kMaxConvW; ++k)
        if (k < p.W - 1) win[k] = ld_f(p.conv_state, cs_off + (k + 1) * p.cs_w, p.cs_dt);
#pragma unroll
    for (int k = 0; k < kMaxConvW; ++k)
        if (k < p.W) st_f(p.conv_state, cs_off + k * p.cs_w, p.cs_dt, (k == p.W - 1) ? xv : win[k]);
}

__device__ __forceinline__ void row_epilogue(const SsuProblem& p, int64_t b, int64_t h, int64_t pp,
                                             float acc, float u) {
    float y = acc;
    if (p.Dp) y = fmaf(p.Dp[h * p.D_h + pp * p.D_p], u, y);
    if (p.z) y *= silu_f(ld_f(p.z, b * p.z_b + h * p.z_h + pp * p.z_p, p.z_dt));
    st_f(p.out, b * p.o_b + h * p.o_h + pp * p.o_p, p.out_dt, y);
}

// ------------------------------------------------------------------------
// Vector kernel.  Each state row (N contiguous elements, 16-byte aligned) is
// split into 16-byte chunks; `lpr` lanes share a row and each lane owns CPL
// chunks at n = (lane + lpr * j) * VE.  Rows per pass = blockDim / lpr.
// ------------------------------------------------------------------------
template <typename ST, int CPL, bool A_FULL>
__global__ void __launch_bounds__(256) ssu_vec_kernel(const SsuProblem p, const SsuPlan plan) {
    using V = Vec16<ST>;
    constexpr int VE = V::VE;
    constexpr int RPT = kRowsPerThread;
    const int lpr = plan.lpr;
    const int lane_r = threadIdx.x % lpr;
    const int row_slot = threadIdx.x / lpr;
    const int rows_per_pass = blockDim.x / lpr;
    const int64_t HP = p.H * p.P;
    const int64_t es = sizeof(ST);

    for (int64_t item = blockIdx.x; item < plan.n_items; item += gridDim.x) {
        const int64_t b = item / plan.items_per_b;
        const int64_t blk = item - b * plan.items_per_b;
        int64_t slot = b;
        if (p.slot_idx) {
            slot = p.slot_idx[b * p.si_b];
            if (slot < 0 || slot >= p.n_slots) continue;  // padding row: uniform across the CTA
        }
        const int64_t r_begin = blk * plan.rows_per_item;
        const int64_t r_end = min(r_begin + plan.rows_per_item, HP);
        const int64_t g = (r_begin / p.P) / p.heads_per_group;

        float Bv[CPL][VE], Cv[CPL][VE];
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                const int64_t n = (int64_t)(lane_r + lpr * j) * VE + e;
                Bv[j][e] = ld_f(p.Bm, b * p.B_b + g * p.B_g + n * p.B_n, p.B_dt);
                Cv[j][e] = ld_f(p.Cm, b * p.C_b + g * p.C_g + n * p.C_n, p.C_dt);
            }
        }

        // trip count is the same for every thread of the CTA (the shuffles
        // below need whole warps); rows past r_end are masked
        for (int64_t rb = r_begin; rb < r_end; rb += (int64_t)rows_per_pass * RPT) {
            uint4 sv[RPT][CPL];
            int64_t hh[RPT], pp[RPT];
            bool ok[RPT];
            // issue every state load of the batch first
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const int64_t r = rb + row_slot + (int64_t)k * rows_per_pass;
                ok[k] = r < r_end;
                const int64_t rr = ok[k] ? r : r_begin;
                hh[k] = rr / p.P;
                pp[k] = rr - hh[k] * p.P;
                const char* sp = static_cast<const char*>(p.state) +
                                 (slot * p.st_b + hh[k] * p.st_h + pp[k] * p.st_p) * es;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    sv[k][j] = ok[k] ? ld_stream16(sp + (int64_t)(lane_r + lpr * j) * 16)
                                     : make_uint4(0, 0, 0, 0);
                }
            }
            float acc[RPT];
            RowScalars rs[RPT];
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                acc[k] = 0.0f;
                if (!ok[k]) {
                    rs[k].u = rs[k].delta = rs[k].dl2 = 0.0f;
                    continue;
                }
                rs[k] = row_prologue(p, b, slot, hh[k], pp[k]);
                float dA = 0.0f;
                if (!A_FULL) dA = ex2_approx(rs[k].dl2 * p.A[hh[k] * p.A_h]);
                const float du = rs[k].delta * rs[k].u;
                char* sp = static_cast<char*>(p.state) +
                           (slot * p.st_b + hh[k] * p.st_h + pp[k] * p.st_p) * es;
                const float* Arow = p.A + hh[k] * p.A_h + pp[k] * p.A_p;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    float s[VE];
                    V::unpack(sv[k][j], s);
                    float a[VE];
                    if (A_FULL) {
                        const float* ap = Arow + (int64_t)(lane_r + lpr * j) * VE;
#pragma unroll
                        for (int e = 0; e < VE; e += 4) {
                            const float4 a4 = __ldg(reinterpret_cast<const float4*>(ap + e));
                            a[e] = a4.x;
                            a[e + 1] = a4.y;
                            a[e + 2] = a4.z;
                            a[e + 3] = a4.w;
                        }
                    }
#pragma unroll
                    for (int e = 0; e < VE; ++e) {
                        const float decay = A_FULL ? ex2_approx(rs[k].dl2 * a[e]) : dA;
                        s[e] = fmaf(decay, s[e], du * Bv[j][e]);
                        acc[k] = fmaf(Cv[j][e], s[e], acc[k]);
                    }
                    st_stream16(sp + (int64_t)(lane_r + lpr * j) * 16, V::pack(s));
                }
            }
            // row sums across the lpr lanes of each row (whole warp takes part)
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                for (int off = lpr >> 1; off >= 1; off >>= 1)
                    acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
            }
            // The shuffles above consume values computed from every lane's conv
            // reads, so the whole row has read the old conv state by now.
            if (lane_r == 0) {
#pragma unroll
                for (int k = 0; k < RPT; ++k) {
                    if (!ok[k]) continue;
                    row_epilogue(p, b, hh[k], pp[k], acc[k], rs[k].u);
                    if (p.W > 0) conv_roll_store(p, b, slot, hh[k], pp[k]);
                }
            }
        }
    }
}

// ------------------------------------------------------------------------
// Generic kernel: one thread per row, any strides, any dstate, any dtypes.
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(128) ssu_generic_kernel(const SsuProblem p) {
    const int64_t HP = p.H * p.P;
    const int64_t total = p.Bn * HP;
    for (int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; row < total;
         row += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = row / HP;
        const int64_t r = row - b * HP;
        const int64_t h = r / p.P;
        const int64_t pp = r - h * p.P;
        int64_t slot = b;
        if (p.slot_idx) {
            slot = p.slot_idx[b * p.si_b];
            if (slot < 0 || slot >= p.n_slots) continue;
        }
        const int64_t g = h / p.heads_per_group;
        const RowScalars rs = row_prologue(p, b, slot, h, pp);
        if (p.W > 0) conv_roll_store(p, b, slot, h, pp);
        const float du = rs.delta * rs.u;
        const float dA = p.A_full ? 0.0f : ex2_approx(rs.dl2 * p.A[h * p.A_h]);
        const int64_t soff = slot * p.st_b + h * p.st_h + pp * p.st_p;
        float acc = 0.0f;
        for (int64_t n = 0; n < p.N; ++n) {
            const float decay =
                p.A_full ? ex2_approx(rs.dl2 * p.A[h * p.A_h + pp * p.A_p + n * p.A_n]) : dA;
            float s = ld_f(p.state, soff + n * p.st_n, p.state_dt);
            const float bn = ld_f(p.Bm, b * p.B_b + g * p.B_g + n * p.B_n, p.B_dt);
            const float cn = ld_f(p.Cm, b * p.C_b + g * p.C_g + n * p.C_n, p.C_dt);
            s = fmaf(decay, s, du * bn);
            acc = fmaf(cn, s, acc);
            st_f(p.state, soff + n * p.st_n, p.state_dt, s);
        }
        row_epilogue(p, b, h, pp, acc, rs.u);
    }
}

template <typename ST>
cudaError_t launch_vec(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    if (plan.cpl == 1) {
        if (p.A_full) ssu_vec_kernel<ST, 1, true><<<plan.grid, plan.block, 0, s>>>(p, plan);
        else ssu_vec_kernel<ST, 1, false><<<plan.grid, plan.block, 0, s>>>(p, plan);
    } else if (plan.cpl == 2) {
        if (p.A_full) ssu_vec_kernel<ST, 2, true><<<plan.grid, plan.block, 0, s>>>(p, plan);
        else ssu_vec_kernel<ST, 2, false><<<plan.grid, plan.block, 0, s>>>(p, plan);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ssu(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    if (plan.kernel == SSM_KERNEL_SSU_VEC) {
        switch (p.state_dt) {
            case kF32: return launch_vec<float>(p, plan, s);
            case kF16: return launch_vec<__half>(p, plan, s);
            case kBF16: return launch_vec<__nv_bfloat16>(p, plan, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.kernel == SSM_KERNEL_SSU_GENERIC) {
        ssu_generic_kernel<<<plan.grid, plan.block, 0, s>>>(p);
        return cudaGetLastError();
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssm
