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
#include "tma.cuh"

namespace ssm {

// Error word shared by the kernels of this file: 0 = none, 1 = a bounded wait
// on a bulk copy timed out (the kernel then exited early).  Read and cleared
// by ssm_device_error() through the host helpers at the end of this file.
__device__ int g_ssm_device_error = 0;

namespace {

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
// Per-head decay kernel (Mamba-2 layout, A one scalar per head, no conv).
// A work item is a block of rows of one (b, h): Delta and exp(Delta*A) are
// computed once per item, B/C once per item into registers.  `lpr` lanes
// share a row, each owning CPL 16-byte chunks at chunk index lane + lpr*j
// (coalesced across the lanes); every thread keeps RPT rows in flight.
// ------------------------------------------------------------------------
template <typename ST, int CPL, int RPT>
__global__ void __launch_bounds__(256, 3) ssu_head_kernel(const SsuProblem p, const SsuPlan plan) {
    using V = Vec16<ST>;
    constexpr int VE = V::VE;
    const unsigned lpr = (unsigned)plan.lpr;
    const unsigned lane_r = threadIdx.x & (lpr - 1);
    const unsigned row_slot = threadIdx.x / lpr;
    const unsigned rows_per_pass = blockDim.x / lpr;
    const unsigned P = (unsigned)p.P;
    const unsigned rb = (unsigned)plan.rows_per_item;
    const unsigned iph = (unsigned)((P + rb - 1) / rb);  // items per head
    const unsigned items_per_b = (unsigned)p.H * iph;
    const unsigned n_items = (unsigned)plan.n_items;
    const bool dt_row = p.dt_p != 0;
    const int64_t es = sizeof(ST);

    for (unsigned item = blockIdx.x; item < n_items; item += gridDim.x) {
        const unsigned b = item / items_per_b;
        const unsigned rem = item - b * items_per_b;
        const unsigned h = rem / iph;
        const unsigned p0 = (rem - h * iph) * rb;
        const unsigned p1 = min(p0 + rb, P);
        int64_t slot = b;
        if (p.slot_idx) {
            slot = p.slot_idx[b * p.si_b];
            if (slot < 0 || slot >= p.n_slots) continue;  // uniform across the CTA
        }
        const unsigned g = h / (unsigned)p.heads_per_group;
        const float a2 = p.A[h * p.A_h] * kLog2e;
        float delta = 0.0f, dA = 0.0f;
        if (!dt_row) {
            float v = ld_f(p.dt, b * p.dt_b + h * p.dt_h, p.dt_dt);
            if (p.dt_bias) v += p.dt_bias[h * p.db_h];
            delta = p.softplus ? softplus_f(v) : v;
            dA = ex2_approx(delta * a2);
        }
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
        char* sbase = static_cast<char*>(p.state) + (slot * p.st_b + (int64_t)h * p.st_h) * es;

        for (unsigned pb = p0; pb < p1; pb += rows_per_pass * RPT) {  // uniform trip count
            uint4 sv[RPT][CPL];
            float xv[RPT];
            bool ok[RPT];
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const unsigned pp = pb + row_slot + k * rows_per_pass;
                ok[k] = pp < p1;
                const char* sp = sbase + (int64_t)pp * p.st_p * es;
#pragma unroll
                for (int j = 0; j < CPL; ++j)
                    sv[k][j] = ok[k] ? ld_stream16(sp + (int64_t)(lane_r + lpr * j) * 16)
                                     : make_uint4(0, 0, 0, 0);
                xv[k] = ok[k] ? ld_f(p.x, b * p.x_b + h * p.x_h + pp * p.x_p, p.x_dt) : 0.0f;
            }
            float acc[RPT];
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const unsigned pp = pb + row_slot + k * rows_per_pass;
                float dl = delta, da = dA;
                if (dt_row && ok[k]) {
                    float v = ld_f(p.dt, b * p.dt_b + h * p.dt_h + pp * p.dt_p, p.dt_dt);
                    if (p.dt_bias) v += p.dt_bias[h * p.db_h + pp * p.db_p];
                    dl = p.softplus ? softplus_f(v) : v;
                    da = ex2_approx(dl * a2);
                }
                const float du = dl * xv[k];
                // packed pairs: s = dA*s + du*B ; acc += C*s
                const u64 da2 = pk(da, da), du2 = pk(du, du);
                u64 acc2 = pk(0.0f, 0.0f);
                char* sp = sbase + (int64_t)pp * p.st_p * es;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    float s[VE];
                    V::unpack(sv[k][j], s);
#pragma unroll
                    for (int e = 0; e < VE; e += 2) {
                        const u64 s2 = ffma2(da2, pk(s[e], s[e + 1]),
                                             fmul2(du2, pk(Bv[j][e], Bv[j][e + 1])));
                        acc2 = ffma2(pk(Cv[j][e], Cv[j][e + 1]), s2, acc2);
                        upk(s2, s[e], s[e + 1]);
                    }
                    if (ok[k]) st_stream16(sp + (int64_t)(lane_r + lpr * j) * 16, V::pack(s));
                }
                float a0, a1;
                upk(acc2, a0, a1);
                acc[k] = a0 + a1;
            }
#pragma unroll
            for (int k = 0; k < RPT; ++k)
                for (unsigned off = lpr >> 1; off >= 1; off >>= 1)
                    acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
            if (lane_r == 0) {
#pragma unroll
                for (int k = 0; k < RPT; ++k) {
                    if (!ok[k]) continue;
                    const unsigned pp = pb + row_slot + k * rows_per_pass;
                    row_epilogue(p, b, h, pp, acc[k], xv[k]);
                }
            }
        }
    }
}

// ------------------------------------------------------------------------
// Per-head decay kernel fed by bulk copies (TMA) -- the main Mamba-2 decode
// path.  A work item is a block of rows of one (b, h); with dense rows it is
// one contiguous range of the cache, which one thread copies into a shared
// memory stage with cp.async.bulk (completion counted on an mbarrier).  Each
// CTA walks a contiguous range of items and keeps kTmaStages copies in flight,
// so the bytes in flight per SM no longer depend on registers; the threads
// update from shared memory and stream the new state back with 16-byte
// stores.  B/C are reloaded only when (b, group) changes, Delta and
// exp(Delta*A) once per item, x before the wait so its latency overlaps the
// copy.
// ------------------------------------------------------------------------
constexpr int kTmaStages = 4;
constexpr int kTmaMaxRows = 8;                 // rows per thread per item
constexpr long long kWaitBudget = 4000000000LL;  // cycles before a wait gives up (~2 s)

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <typename ST, int CPL>
__global__ void __launch_bounds__(256, 3) ssu_head_tma_kernel(const SsuProblem p, const SsuPlan plan) {
    using V = Vec16<ST>;
    constexpr int VE = V::VE;
    extern __shared__ __align__(128) unsigned char tma_stage[];
    __shared__ __align__(8) uint64_t full[kTmaStages];

    const unsigned tid = threadIdx.x;
    const unsigned lpr = (unsigned)plan.lpr;
    const unsigned lane_r = tid & (lpr - 1);
    const unsigned row_slot = tid / lpr;
    const unsigned rows_per_pass = blockDim.x / lpr;
    const unsigned P = (unsigned)p.P;
    const unsigned rb = (unsigned)plan.rows_per_item;
    const unsigned iph = (P + rb - 1) / rb;
    const unsigned items_per_b = (unsigned)p.H * iph;
    const unsigned n_items = (unsigned)plan.n_items;
    const unsigned per = (n_items + gridDim.x - 1) / gridDim.x;
    const unsigned i0 = blockIdx.x * per;
    const unsigned i1 = min(i0 + per, n_items);
    if (i0 >= i1) return;  // uniform
    const unsigned cnt = i1 - i0;
    const unsigned stage_bytes = (unsigned)plan.stage_bytes;
    const int64_t es = sizeof(ST);
    const unsigned row_bytes = (unsigned)(p.N * es);
    const bool dt_row = p.dt_p != 0;

    auto decode = [&](unsigned item, unsigned& b, unsigned& h, unsigned& p0, unsigned& p1) {
        b = item / items_per_b;
        const unsigned rem = item - b * items_per_b;
        h = rem / iph;
        p0 = (rem - h * iph) * rb;
        p1 = min(p0 + rb, P);
    };
    auto slot_of = [&](unsigned b) -> int64_t {
        if (!p.slot_idx) return b;
        const int64_t sl = p.slot_idx[b * p.si_b];
        return (sl < 0 || sl >= p.n_slots) ? -1 : sl;
    };
    // thread 0: start the copy of local item k into stage k % kTmaStages; a
    // padding row completes the stage's phase without data
    auto issue = [&](unsigned k) {
        unsigned b, h, p0, p1;
        decode(i0 + k, b, h, p0, p1);
        uint64_t* bar = &full[k % kTmaStages];
        const int64_t slot = slot_of(b);
        if (slot < 0) {
            mbar_arrive(bar);
            return;
        }
        const char* src = static_cast<const char*>(p.state) +
                          (slot * p.st_b + (int64_t)h * p.st_h + (int64_t)p0 * p.st_p) * es;
        const uint32_t bytes = (p1 - p0) * row_bytes;
        mbar_arrive_expect_tx(bar, bytes);
        tma_load_1d(tma_stage + (k % kTmaStages) * stage_bytes, src, bytes, bar);
    };

    if (tid == 0) {
        for (int s = 0; s < kTmaStages; ++s) mbar_init(&full[s], 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0)
        for (unsigned k = 0; k < min(cnt, (unsigned)kTmaStages); ++k) issue(k);

    int64_t cached_key = -1;
    float Bv[CPL][VE], Cv[CPL][VE];
    for (unsigned k = 0; k < cnt; ++k) {
        unsigned b, h, p0, p1;
        decode(i0 + k, b, h, p0, p1);
        const int64_t slot = slot_of(b);
        const unsigned stage = k % kTmaStages;
        const uint32_t parity = (k / kTmaStages) & 1u;
        const unsigned g = h / (unsigned)p.heads_per_group;
        float delta = 0.0f, dA = 0.0f, a2 = 0.0f;
        float xv[kTmaMaxRows];
        if (slot >= 0) {
            const int64_t key = (int64_t)b * p.G + g;
            if (key != cached_key) {
                cached_key = key;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
#pragma unroll
                    for (int e = 0; e < VE; ++e) {
                        const int64_t n = (int64_t)(lane_r + lpr * j) * VE + e;
                        Bv[j][e] = ld_f(p.Bm, b * p.B_b + g * p.B_g + n * p.B_n, p.B_dt);
                        Cv[j][e] = ld_f(p.Cm, b * p.C_b + g * p.C_g + n * p.C_n, p.C_dt);
                    }
                }
            }
            a2 = p.A[h * p.A_h] * kLog2e;
            if (!dt_row) {
                float v = ld_f(p.dt, b * p.dt_b + h * p.dt_h, p.dt_dt);
                if (p.dt_bias) v += p.dt_bias[h * p.db_h];
                delta = p.softplus ? softplus_f(v) : v;
                dA = ex2_approx(delta * a2);
            }
#pragma unroll
            for (int r = 0; r < kTmaMaxRows; ++r) {
                const unsigned pp = p0 + row_slot + r * rows_per_pass;
                xv[r] = pp < p1 ? ld_f(p.x, b * p.x_b + h * p.x_h + pp * p.x_p, p.x_dt) : 0.0f;
            }
        }
        const bool ok = mbar_wait_bounded(&full[stage], parity, kWaitBudget);
        if (__syncthreads_or(!ok)) {
            // give up: wait (bounded) for this CTA's copies still in flight, flag, exit
            if (tid == 0) {
                for (unsigned kk = k; kk < min(cnt, k + kTmaStages); ++kk)
                    mbar_wait_bounded(&full[kk % kTmaStages], (kk / kTmaStages) & 1u, kWaitBudget);
                atomicExch(&g_ssm_device_error, 1);
            }
            return;
        }
        if (slot >= 0) {
            const unsigned char* st = tma_stage + stage * stage_bytes;
            char* gbase = static_cast<char*>(p.state) + (slot * p.st_b + (int64_t)h * p.st_h) * es;
#pragma unroll
            for (int r = 0; r < kTmaMaxRows; ++r) {
                if (r * rows_per_pass >= rb) break;  // uniform
                const unsigned pp = p0 + row_slot + r * rows_per_pass;
                const bool rok = pp < p1;
                float dl = delta, da = dA;
                if (dt_row && rok) {
                    float v = ld_f(p.dt, b * p.dt_b + h * p.dt_h + pp * p.dt_p, p.dt_dt);
                    if (p.dt_bias) v += p.dt_bias[h * p.db_h + pp * p.db_p];
                    dl = p.softplus ? softplus_f(v) : v;
                    da = ex2_approx(dl * a2);
                }
                const float du = dl * xv[r];
                const u64 da2 = pk(da, da), du2 = pk(du, du);
                u64 acc2 = pk(0.0f, 0.0f);
                const unsigned char* srow = st + (pp - p0) * row_bytes;
                char* grow = gbase + (int64_t)pp * p.st_p * es;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    const unsigned off = (lane_r + lpr * j) * 16;
                    uint4 raw = rok ? *reinterpret_cast<const uint4*>(srow + off) : make_uint4(0, 0, 0, 0);
                    float sv[VE];
                    V::unpack(raw, sv);
#pragma unroll
                    for (int e = 0; e < VE; e += 2) {
                        const u64 s2 = ffma2(da2, pk(sv[e], sv[e + 1]),
                                             fmul2(du2, pk(Bv[j][e], Bv[j][e + 1])));
                        acc2 = ffma2(pk(Cv[j][e], Cv[j][e + 1]), s2, acc2);
                        upk(s2, sv[e], sv[e + 1]);
                    }
                    if (rok) st_stream16(grow + off, V::pack(sv));
                }
                float a0, a1;
                upk(acc2, a0, a1);
                float acc = a0 + a1;
                for (unsigned o = lpr >> 1; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (rok && lane_r == 0) row_epilogue(p, b, h, pp, acc, xv[r]);
            }
        }
        __syncthreads();  // every thread is done reading this stage
        if (tid == 0 && k + kTmaStages < cnt) {
            fence_proxy_async_smem();
            issue(k + kTmaStages);
        }
    }
}

// ------------------------------------------------------------------------
// Per-row decay kernel (A per element: Mamba-1 layout, or full A), with the
// optional fused conv-state roll.  Each row costs a conv, a softplus, a gate
// and N exponentials, so rows are not split finely: `lpr` lanes share a row
// (1 for rows of <= 64 bytes), each lane owning CPT consecutive 16-byte
// chunks and doing the row prologue itself.  B and C are the same for every
// row of an item, so they are staged once per item in shared memory and read
// back as broadcasts.
// ------------------------------------------------------------------------
constexpr int kRowKernelMaxN = 64;  // rows of <= 16 chunks of 16 bytes

template <typename ST, int CPT>
__global__ void __launch_bounds__(256, 4) ssu_row_kernel(const SsuProblem p, const SsuPlan plan) {
    using V = Vec16<ST>;
    __shared__ __align__(16) float sB[kRowKernelMaxN];
    __shared__ __align__(16) float sC[kRowKernelMaxN];
    constexpr int VE = V::VE;
    const unsigned lpr = (unsigned)plan.lpr;
    const unsigned lane_r = threadIdx.x & (lpr - 1);
    const unsigned row_slot = threadIdx.x / lpr;
    const unsigned rows_per_pass = blockDim.x / lpr;
    const unsigned HP = (unsigned)(p.H * p.P);
    const unsigned P = (unsigned)p.P;
    const unsigned rb = (unsigned)plan.rows_per_item;
    const unsigned items_per_b = (unsigned)plan.items_per_b;
    const unsigned n_items = (unsigned)plan.n_items;
    const int64_t es = sizeof(ST);

    for (unsigned item = blockIdx.x; item < n_items; item += gridDim.x) {
        const unsigned b = item / items_per_b;
        const unsigned r0 = (item - b * items_per_b) * rb;
        const unsigned r1 = min(r0 + rb, HP);
        int64_t slot = b;
        if (p.slot_idx) {
            slot = p.slot_idx[b * p.si_b];
            if (slot < 0 || slot >= p.n_slots) continue;
        }
        const unsigned g = (r0 / P) / (unsigned)p.heads_per_group;
        __syncthreads();  // the previous item's readers are done with sB/sC
        for (int n = threadIdx.x; n < p.N; n += blockDim.x) {
            sB[n] = ld_f(p.Bm, b * p.B_b + g * p.B_g + n * p.B_n, p.B_dt);
            sC[n] = ld_f(p.Cm, b * p.C_b + g * p.C_g + n * p.C_n, p.C_dt);
        }
        __syncthreads();
        for (unsigned rbase = r0; rbase < r1; rbase += rows_per_pass) {  // uniform trip count
            const unsigned r = rbase + row_slot;
            const bool ok = r < r1;
            const unsigned rr = ok ? r : r0;
            const unsigned h = P == 1 ? rr : rr / P;
            const unsigned pp = rr - h * P;
            char* sp = static_cast<char*>(p.state) +
                       (slot * p.st_b + (int64_t)h * p.st_h + (int64_t)pp * p.st_p) * es;
            const float* ap = p.A + h * p.A_h + pp * p.A_p;
            uint4 sv[CPT];
#pragma unroll
            for (int j = 0; j < CPT; ++j)
                sv[j] = ok ? *reinterpret_cast<const uint4*>(sp + (int64_t)(lane_r * CPT + j) * 16)
                           : make_uint4(0, 0, 0, 0);
            RowScalars rs{0.0f, 0.0f, 0.0f};
            if (ok) rs = row_prologue(p, b, slot, h, pp);
            const float du = rs.delta * rs.u;
            float acc = 0.0f;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                float s[VE];
                V::unpack(sv[j], s);
                const int n0 = (int)(lane_r * CPT + j) * VE;
#pragma unroll
                for (int e = 0; e < VE; e += 4) {
                    const float4 a4 = ok ? __ldg(reinterpret_cast<const float4*>(ap + n0 + e))
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 b4 = *reinterpret_cast<const float4*>(&sB[n0 + e]);
                    const float4 c4 = *reinterpret_cast<const float4*>(&sC[n0 + e]);
                    s[e] = fmaf(ex2_approx(rs.dl2 * a4.x), s[e], du * b4.x);
                    s[e + 1] = fmaf(ex2_approx(rs.dl2 * a4.y), s[e + 1], du * b4.y);
                    s[e + 2] = fmaf(ex2_approx(rs.dl2 * a4.z), s[e + 2], du * b4.z);
                    s[e + 3] = fmaf(ex2_approx(rs.dl2 * a4.w), s[e + 3], du * b4.w);
                    acc = fmaf(c4.x, s[e], acc);
                    acc = fmaf(c4.y, s[e + 1], acc);
                    acc = fmaf(c4.z, s[e + 2], acc);
                    acc = fmaf(c4.w, s[e + 3], acc);
                }
                if (ok) *reinterpret_cast<uint4*>(sp + (int64_t)(lane_r * CPT + j) * 16) = V::pack(s);
            }
            for (unsigned off = lpr >> 1; off >= 1; off >>= 1)
                acc += __shfl_xor_sync(0xffffffffu, acc, off);
            // the shuffles consume values computed from every lane's conv reads,
            // so the row's old conv state has been read by all its lanes
            if (ok && lane_r == 0) {
                row_epilogue(p, b, h, pp, acc, rs.u);
                if (p.W > 0) conv_roll_store(p, b, slot, h, pp);
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
cudaError_t launch_head(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    switch (plan.cpl) {
        case 1: ssu_head_kernel<ST, 1, 2><<<plan.grid, plan.block, 0, s>>>(p, plan); break;
        case 2: ssu_head_kernel<ST, 2, 2><<<plan.grid, plan.block, 0, s>>>(p, plan); break;
        case 4: ssu_head_kernel<ST, 4, 1><<<plan.grid, plan.block, 0, s>>>(p, plan); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// Opt the kernel into its dynamic shared memory and the largest shared-memory
// carveout, and return how many of its CTAs fit on one SM.
template <typename K>
cudaError_t prepare_tma_kernel(K kern, int block, int smem, int* per_sm) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, kern, block, smem);
}

template <typename ST>
cudaError_t launch_head_tma(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    const int smem = kTmaStages * plan.stage_bytes;
    auto run = [&](auto kern) -> cudaError_t {
        int per_sm = 0;
        cudaError_t e = prepare_tma_kernel(kern, plan.block, smem, &per_sm);
        if (e != cudaSuccess) return e;
        // persistent grid: every CTA resident at once (the item ranges are static)
        const int64_t cap = (int64_t)plan.sms * (per_sm > 0 ? per_sm : 1);
        const int grid = (int)(plan.n_items < cap ? plan.n_items : cap);
        kern<<<grid, plan.block, smem, s>>>(p, plan);
        return cudaGetLastError();
    };
    switch (plan.cpl) {
        case 1: return run(ssu_head_tma_kernel<ST, 1>);
        case 2: return run(ssu_head_tma_kernel<ST, 2>);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST>
cudaError_t launch_row(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    switch (plan.cpl) {
        case 1: ssu_row_kernel<ST, 1><<<plan.grid, plan.block, 0, s>>>(p, plan); break;
        case 2: ssu_row_kernel<ST, 2><<<plan.grid, plan.block, 0, s>>>(p, plan); break;
        case 4: ssu_row_kernel<ST, 4><<<plan.grid, plan.block, 0, s>>>(p, plan); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ssu(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    if (plan.kernel == SSM_KERNEL_SSU_TMA) {
        switch (p.state_dt) {
            case kF32: return launch_head_tma<float>(p, plan, s);
            case kF16: return launch_head_tma<__half>(p, plan, s);
            case kBF16: return launch_head_tma<__nv_bfloat16>(p, plan, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.kernel == SSM_KERNEL_SSU_VEC || plan.kernel == SSM_KERNEL_SSU_ROW) {
        const bool head = plan.kernel == SSM_KERNEL_SSU_VEC;
        switch (p.state_dt) {
            case kF32: return head ? launch_head<float>(p, plan, s) : launch_row<float>(p, plan, s);
            case kF16: return head ? launch_head<__half>(p, plan, s) : launch_row<__half>(p, plan, s);
            case kBF16:
                return head ? launch_head<__nv_bfloat16>(p, plan, s)
                            : launch_row<__nv_bfloat16>(p, plan, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.kernel == SSM_KERNEL_SSU_GENERIC) {
        ssu_generic_kernel<<<plan.grid, plan.block, 0, s>>>(p);
        return cudaGetLastError();
    }
    return cudaErrorInvalidValue;
}

int ssu_tma_stages() { return kTmaStages; }
int ssu_tma_max_rows_per_thread() { return kTmaMaxRows; }

// Read the device error word into *code (after the stream's work so far) and
// clear it.
cudaError_t read_and_clear_device_error(int* code, cudaStream_t s) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_ssm_device_error, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    *code = v;
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_ssm_device_error, &zero, sizeof(int), 0,
                                    cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    return e;
}

}  // namespace ssm
