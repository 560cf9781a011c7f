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

#include <atomic>

namespace ssm {

// The device error record of the library (DeviceError in problem.h): set by
// a kernel whose bounded wait on a bulk copy (or a hand-over) ran out, read
// and cleared by ssm_device_error() / ssm_device_error_info() through the
// host helpers at the end of this file.  Kernels in other files are handed
// its address (device_error_ptr).
__device__ DeviceError g_ssm_device_error = {0, 0, kNoItem};
__device__ DeviceError g_ssm_device_error_snap = {0, 0, kNoItem};

// Budget of the wait for copies still in flight after a stage wait gave up:
// always the full one, whatever the stage budget, so that a CTA never exits
// while bulk copies still write into its shared memory.
constexpr long long kCleanupBudget = 4000000000LL;

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
// path.  A work item is a block of rb rows of one (b, h); with dense rows it
// is one contiguous range of the cache, and its rb x values are contiguous
// too, so one thread copies both into a shared-memory stage with
// cp.async.bulk (completion counted in bytes on an mbarrier).  Each CTA walks
// a contiguous range of items (decoded incrementally), keeps plan.stages
// copies in flight, and its threads update from shared memory and stream the
// new state back with 16-byte stores.  `lpr` lanes share a row, each owning
// CPL 16-byte chunks; a thread owns RPT rows of an item, and the RPT partial
// readouts of a thread are summed over the row's lanes by a butterfly
// reduce-scatter.  I/O dtype IoT is a template parameter.  With one dt per
// head, the items' scalars (Delta, exp(Delta*A), D, the B/C group) are
// computed 32 items at a time, one item per lane of the CTA's last warp, into
// a ring in shared memory that the per-item barrier publishes; the other
// threads only read them.  The warp loads a batch's inputs 32 items before it
// computes them, so no barrier waits on those loads.
// ------------------------------------------------------------------------
constexpr int kTmaStagesMax = 4;
constexpr int kScBatch = 32;  // items per batch of scalars (one per lane)

struct ItemScalars {
    float delta, dA, dskip;
    int g;
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Sum v[0..R) over the lpr lanes of a row.  Afterwards lane r of the row holds
// the total of row k = r / (lpr / R) in v[0].  Needs R <= lpr.
template <int R>
__device__ __forceinline__ void row_reduce_scatter(float* v, unsigned lane_r, unsigned lpr) {
    unsigned off = lpr >> 1;
#pragma unroll
    for (int w = R; w > 1; w >>= 1) {
        const bool upper = (lane_r & off) != 0;
#pragma unroll
        for (int i = 0; i < w / 2; ++i) {
            const float send = upper ? v[i] : v[i + w / 2];
            const float keep = upper ? v[i + w / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
        off >>= 1;
    }
    for (; off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
}

template <typename ST, typename IoT, int CPL, int RPT>
__global__ void __launch_bounds__(256, 3) ssu_head_tma_kernel(const SsuProblem p, const SsuPlan plan) {
    using V = Vec16<ST>;
    constexpr int VE = V::VE;
    extern __shared__ __align__(128) unsigned char tma_stage[];
    __shared__ __align__(8) uint64_t full[kTmaStagesMax];
    __shared__ __align__(16) ItemScalars item_sc[2 * kScBatch];  // two batches

    const unsigned tid = threadIdx.x;
    const unsigned lpr = (unsigned)plan.lpr;
    const unsigned lane_r = tid & (lpr - 1);
    const unsigned row_slot = tid / lpr;
    const unsigned rows_per_pass = blockDim.x / lpr;
    const unsigned P = (unsigned)p.P;
    const unsigned H = (unsigned)p.H;
    const unsigned rb = (unsigned)plan.rows_per_item;
    const unsigned iph = (P + rb - 1) / rb;
    const unsigned n_items = (unsigned)plan.n_items;
    const unsigned per = (n_items + gridDim.x - 1) / gridDim.x;
    const unsigned i0 = blockIdx.x * per;
    const unsigned i1 = min(i0 + per, n_items);
    if (i0 >= i1) return;  // uniform
    const unsigned cnt = i1 - i0;
    const unsigned S = (unsigned)plan.stages;
    const unsigned stage_bytes = (unsigned)plan.stage_bytes;
    const unsigned row_bytes = (unsigned)(p.N * (int64_t)sizeof(ST));
    const unsigned x_off = rb * row_bytes;  // x values follow the rows in a stage
    const bool dt_row = p.dt_p != 0;
    const IoT* __restrict__ xg = static_cast<const IoT*>(p.x);
    const IoT* __restrict__ dtg = static_cast<const IoT*>(p.dt);
    const IoT* __restrict__ Bg = static_cast<const IoT*>(p.Bm);
    const IoT* __restrict__ Cg = static_cast<const IoT*>(p.Cm);
    const IoT* __restrict__ zg = static_cast<const IoT*>(p.z);
    IoT* __restrict__ og = static_cast<IoT*>(p.out);

    // item index -> (b, h, first row); advanced incrementally
    struct Pos { unsigned b, h, pb; };
    auto first = [&](unsigned item) {
        Pos q;
        q.b = item / (H * iph);
        const unsigned rem = item - q.b * H * iph;
        q.h = rem / iph;
        q.pb = rem - q.h * iph;
        return q;
    };
    auto next = [&](Pos& q) {
        if (++q.pb == iph) {
            q.pb = 0;
            if (++q.h == H) {
                q.h = 0;
                ++q.b;
            }
        }
    };
    auto slot_of = [&](unsigned b) -> int64_t {
        if (!p.slot_idx) return b;
        const int64_t sl = p.slot_idx[b * p.si_b];
        return (sl < 0 || sl >= p.n_slots) ? -1 : sl;
    };
    // thread 0: start the copies of local item k (at `q`) into stage `sg`,
    // with the item's scalars (one dt per head); a padding row completes the
    // stage's phase without data
    auto issue = [&](unsigned k, unsigned sg, const Pos& q) {
        uint64_t* bar = &full[sg];
#ifdef SSM_TEST_HOOKS
        if ((int64_t)(i0 + k) == plan.drop_item) return;  // failure test: never completes
#endif
        const int64_t slot = slot_of(q.b);
        if (slot < 0) {
            mbar_arrive(bar);
            return;
        }
        const unsigned p0 = q.pb * rb;
        const unsigned nr = min(rb, P - p0);
        const char* src = static_cast<const char*>(p.state) +
                          (slot * p.st_b + (int64_t)q.h * p.st_h + (int64_t)p0 * p.st_p) * (int64_t)sizeof(ST);
        const IoT* xs = xg + q.b * p.x_b + (int64_t)q.h * p.x_h + p0;
        const uint32_t sbytes = nr * row_bytes;
        const uint32_t xbytes = (nr * (unsigned)sizeof(IoT) + 15u) & ~15u;
        unsigned char* dst = tma_stage + sg * stage_bytes;
        mbar_arrive_expect_tx(bar, sbytes + xbytes);
        tma_load_1d(dst, src, sbytes, bar);
        tma_load_1d(dst + x_off, xs, xbytes, bar);
    };

    // last warp: the inputs of local items 32*j .. 32*j+31 (one per lane) are
    // loaded into registers by sc_load(j) and turned into ring entries
    // (item & 63) by sc_store(j).  Padding rows get entries too (x and dt are
    // indexed by batch row, not by cache slot); nobody reads them.
    // (measured: the ring pays for 16-bit caches, whose kernels are
    // issue-bound; fp32-cache items keep per-thread scalars, loaded before the
    // stage wait)
    const bool ring = sizeof(ST) == 2 && !dt_row;
    const bool sc_lane = ring && tid / 32 == blockDim.x / 32 - 1;
    float sc_v = 0.0f, sc_a = 0.0f, sc_d = 0.0f;
    int sc_g = 0;
    auto sc_load = [&](unsigned j) {
        const unsigned k = j * kScBatch + (tid & 31u);
        if (k >= cnt) return;
        const Pos q = first(i0 + k);
        sc_v = to_f(dtg[q.b * p.dt_b + q.h * p.dt_h]);
        if (p.dt_bias) sc_v += p.dt_bias[q.h * p.db_h];
        sc_a = p.A[q.h * p.A_h] * kLog2e;
        sc_d = p.Dp ? p.Dp[q.h * p.D_h] : 0.0f;
        sc_g = p.G == 1 ? 0 : (int)(q.h / (unsigned)p.heads_per_group);
    };
    auto sc_store = [&](unsigned j) {
        const unsigned k = j * kScBatch + (tid & 31u);
        if (k >= cnt) return;
        ItemScalars sc;
        sc.delta = p.softplus ? softplus_f(sc_v) : sc_v;
        sc.dA = ex2_approx(sc.delta * sc_a);
        sc.dskip = sc_d;
        sc.g = sc_g;
        item_sc[k & (2 * kScBatch - 1)] = sc;
    };
    if (sc_lane) {
        sc_load(0);
        sc_store(0);
        sc_load(1);
    }
    if (tid == 0) {
        for (unsigned s2 = 0; s2 < S; ++s2) mbar_init(&full[s2], 1);
        mbar_fence_init();
    }
    __syncthreads();
    Pos cur = first(i0);
    if (tid == 0) {
        Pos q = cur;
        for (unsigned k = 0; k < min(cnt, S); ++k) {
            issue(k, k, q);
            next(q);
        }
    }
    Pos ahead = cur;  // position of item k + S (thread 0's refill cursor)
    for (unsigned k = 0; k < S; ++k) next(ahead);
    // lpr and RPT are powers of two: the epilogue lanes by shift and mask
    const unsigned group = lpr / RPT;
    const unsigned gshift = __ffs(group) - 1;

    int64_t cached_key = -1;
    float Bv[CPL][VE], Cv[CPL][VE];
    // B and C of (b, group g) into registers, when they change
    auto load_bc = [&](unsigned b, unsigned g) {
        const int64_t key = (int64_t)b * p.G + g;
        if (key == cached_key) return;
        cached_key = key;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                const int64_t n = (int64_t)(lane_r + lpr * j) * VE + e;
                Bv[j][e] = to_f(Bg[b * p.B_b + g * p.B_g + n * p.B_n]);
                Cv[j][e] = to_f(Cg[b * p.C_b + g * p.C_g + n * p.C_n]);
            }
        }
    };
    unsigned stage = 0;
    uint32_t parity = 0;
    for (unsigned k = 0; k < cnt; ++k, next(cur)) {
        const unsigned b = cur.b, h = cur.h;
        const unsigned p0 = cur.pb * rb;
        const unsigned p1 = min(p0 + rb, P);
        const int64_t slot = slot_of(b);
        float delta = 0.0f, dA = 0.0f, a2 = 0.0f, dskip = 0.0f;
        if (slot >= 0 && !ring) {
            // per-thread scalars and B/C, loaded before the wait
            load_bc(b, p.G == 1 ? 0u : h / (unsigned)p.heads_per_group);
            a2 = p.A[h * p.A_h] * kLog2e;
            dskip = p.Dp ? p.Dp[h * p.D_h] : 0.0f;
            if (!dt_row) {
                float v = to_f(dtg[b * p.dt_b + h * p.dt_h]);
                if (p.dt_bias) v += p.dt_bias[h * p.db_h];
                delta = p.softplus ? softplus_f(v) : v;
                dA = ex2_approx(delta * a2);
            }
        }
        const bool ok = mbar_wait_bounded(&full[stage], parity, plan.wait_budget);
        if (__syncthreads_or(!ok)) {
            // give up: wait for this CTA's copies still in flight (items k ..
            // k+S-1 were issued, all but a dropped one), record, exit
            if (tid == 0) {
                for (unsigned kk = k; kk < min(cnt, k + S); ++kk) {
#ifdef SSM_TEST_HOOKS
                    if ((int64_t)(i0 + kk) == plan.drop_item) continue;  // never issued
#endif
                    mbar_wait_bounded(&full[kk % S], (kk / S) & 1u, kCleanupBudget);
                }
                report_device_error(&g_ssm_device_error, SSM_KERNEL_SSU_TMA, (long long)(i0 + k));
            }
            return;
        }
        if (slot >= 0) {
            if (ring) {
                const ItemScalars sc = item_sc[k & (2 * kScBatch - 1)];
                delta = sc.delta;
                dA = sc.dA;
                dskip = sc.dskip;
                load_bc(b, (unsigned)sc.g);
            }
            const unsigned char* st = tma_stage + stage * stage_bytes;
            const IoT* xsm = reinterpret_cast<const IoT*>(st + x_off);
            char* gbase = static_cast<char*>(p.state) +
                          (slot * p.st_b + (int64_t)h * p.st_h) * (int64_t)sizeof(ST);
            float acc[RPT], xr[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const unsigned pl = row_slot + r * rows_per_pass;  // row within the item
                const unsigned pp = p0 + pl;
                const bool rok = pp < p1;
                xr[r] = rok ? to_f(xsm[pl]) : 0.0f;
                float dl = delta, da = dA;
                if (dt_row && rok) {
                    float v = to_f(dtg[b * p.dt_b + h * p.dt_h + pp * p.dt_p]);
                    if (p.dt_bias) v += p.dt_bias[h * p.db_h + pp * p.db_p];
                    dl = p.softplus ? softplus_f(v) : v;
                    da = ex2_approx(dl * a2);
                }
                const float du = dl * xr[r];
                const u64 da2 = pk(da, da), du2 = pk(du, du);
                u64 acc2 = pk(0.0f, 0.0f);
                const unsigned char* srow = st + pl * row_bytes;
                char* grow = gbase + (int64_t)pp * p.st_p * (int64_t)sizeof(ST);
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    const unsigned off = (lane_r + lpr * j) * 16;
                    const uint4 raw = rok ? *reinterpret_cast<const uint4*>(srow + off) : make_uint4(0, 0, 0, 0);
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
                acc[r] = a0 + a1;
            }
            row_reduce_scatter<RPT>(acc, lane_r, lpr);
            if ((lane_r & (group - 1)) == 0) {
                const unsigned r = lane_r >> gshift;
                const unsigned pl = row_slot + r * rows_per_pass;
                const unsigned pp = p0 + pl;
                if (pp < p1) {
                    float xv = 0.0f;
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr)
                        if (rr == (int)r) xv = xr[rr];
                    float y = fmaf(dskip, xv, acc[0]);
                    if (zg) y *= silu_f(to_f(zg[b * p.z_b + h * p.z_h + pp * p.z_p]));
                    og[b * p.o_b + h * p.o_h + pp * p.o_p] = from_f<IoT>(y);
                }
            }
        }
        // halfway through batch j: batch j + 1 into the ring (its entries were
        // last read by batch j - 1, and 16 barriers publish it before its first
        // item), then the loads of batch j + 2
        if (sc_lane && (k & (kScBatch - 1)) == kScBatch / 2) {
            sc_store(k / kScBatch + 1);
            sc_load(k / kScBatch + 2);
        }
        __syncthreads();  // every thread is done reading this stage
        if (tid == 0 && k + S < cnt) {
            fence_proxy_async_smem();
            issue(k + S, stage, ahead);
        }
        next(ahead);
        if (++stage == S) {
            stage = 0;
            parity ^= 1u;
        }
    }
}

// ------------------------------------------------------------------------
// Per-row decay kernel fed by bulk copies -- the Mamba-1 decode path (A per
// (channel, state entry), fused conv-state roll).  Every warp runs its own
// pipeline over a contiguous range of work items, an item being (32 channels,
// batch row b).  The warp's lane 0 moves each item through a ring of
// kWarpStages shared-memory stages with 1-D bulk copies: state rows, conv
// rows, x/dt/z slices and the row's B and C in (completion counted on the
// stage's mbarrier); the updated state and conv rows, written back into the
// stage in place, out again as bulk stores.  A stage is refilled once its
// store has read it, one step later, so kWarpStages - 1 loads run ahead of
// the compute.  No CTA-wide barrier sits in the loop: warps never wait for
// each other.  Items are ordered channel-block-major, so a warp's
// consecutive items reuse A and the conv weights from L1.  A lane owns one
// whole row (CPT 16-byte chunks = the full d_state): conv, SiLU, softplus
// and gate once per row, no cross-lane reduction.  Lane l walks its chunks
// starting at chunk (l / (8/CPT)) mod CPT so that the 16-byte shared-memory
// accesses of neighbouring rows hit distinct banks; A, B and C are taken in
// the same rotated order.
// ------------------------------------------------------------------------
#ifndef SSM_ROW_TMA_STAGES
#define SSM_ROW_TMA_STAGES 3
#endif
#ifndef SSM_ROW_TMA_WARPS
#define SSM_ROW_TMA_WARPS 4
#endif
constexpr int kWarpStages = SSM_ROW_TMA_STAGES;  // items in flight per warp
constexpr int kRowWarps = SSM_ROW_TMA_WARPS;     // warps per CTA
// register cap: enough for 20 resident warps per SM
constexpr int kRowMinBlocks = 20 / kRowWarps > 0 ? 20 / kRowWarps : 1;

template <typename ST, typename IoT, int W, int CPT>
__global__ void __launch_bounds__(32 * kRowWarps, kRowMinBlocks) ssu_row_tma_kernel(const SsuProblem p, const SsuPlan plan) {
    using V = Vec16<ST>;
    constexpr int VE = V::VE;
    constexpr int NS = CPT * VE;  // d_state
    extern __shared__ __align__(128) unsigned char tma_stage[];
    __shared__ __align__(8) uint64_t full[kRowWarps][kWarpStages];
    __shared__ __align__(16) float bcw[kRowWarps][2 * NS];  // the item's B, C widened once

    const unsigned lane = threadIdx.x & 31u;
    const unsigned warp = threadIdx.x >> 5;
    const unsigned Dch = (unsigned)p.H;  // channels (rows)
    const unsigned Bn = (unsigned)p.Bn;
    constexpr unsigned rb = 32;          // rows per item: one per lane
    const unsigned n_items = (unsigned)plan.n_items;
    const unsigned nw = gridDim.x * kRowWarps;
    const unsigned per = (n_items + nw - 1) / nw;
    const unsigned i0 = (blockIdx.x * kRowWarps + warp) * per;
    const unsigned i1 = min(i0 + per, n_items);
    const unsigned cnt = i0 < i1 ? i1 - i0 : 0u;
    const unsigned stage_bytes = (unsigned)plan.stage_bytes;
    unsigned char* ring = tma_stage + warp * kWarpStages * stage_bytes;
    uint64_t* bars = full[warp];
    const unsigned row_bytes = (unsigned)(NS * sizeof(ST));
    const unsigned cs_es = p.cs_dt == kF32 ? 4u : 2u;
    const unsigned pad16 = 15u;
    // stage layout: state rows | conv rows | x | dt | z | B | C
    const unsigned off_cs = rb * row_bytes;
    const unsigned off_x = off_cs + ((rb * (unsigned)W * cs_es + pad16) & ~pad16);
    const unsigned io_bytes = (rb * (unsigned)sizeof(IoT) + pad16) & ~pad16;
    const unsigned off_dt = off_x + io_bytes;
    const unsigned off_z = off_dt + io_bytes;
    const unsigned off_B = off_z + io_bytes;
    const unsigned bc_bytes = (NS * (unsigned)sizeof(IoT) + pad16) & ~pad16;
    const unsigned off_C = off_B + bc_bytes;
    const IoT* __restrict__ xg = static_cast<const IoT*>(p.x);
    const IoT* __restrict__ dtg = static_cast<const IoT*>(p.dt);
    const IoT* __restrict__ zg = static_cast<const IoT*>(p.z);
    const IoT* __restrict__ Bg = static_cast<const IoT*>(p.Bm);
    const IoT* __restrict__ Cg = static_cast<const IoT*>(p.Cm);
    IoT* __restrict__ og = static_cast<IoT*>(p.out);
    const unsigned rot = (lane / (8u / CPT)) & (CPT - 1u);

    auto slot_of = [&](unsigned b) -> int64_t {
        if (!p.slot_idx) return b;
        const int64_t sl = p.slot_idx[b * p.si_b];
        return (sl < 0 || sl >= p.n_slots) ? -1 : sl;
    };
    // lane 0: start the copies of local item k; a padding row completes the
    // stage's phase without data
    auto issue = [&](unsigned k) {
        const unsigned item = i0 + k;
#ifdef SSM_TEST_HOOKS
        if ((int64_t)item == plan.drop_item) return;  // failure test: never completes
#endif
        const unsigned cb = item / Bn, b = item - cb * Bn;
        uint64_t* bar = &bars[k % kWarpStages];
        const int64_t slot = slot_of(b);
        if (slot < 0) {
            mbar_arrive(bar);
            return;
        }
        const unsigned c0 = cb * rb;
        const unsigned nr = min(rb, Dch - c0);
        unsigned char* dst = ring + (k % kWarpStages) * stage_bytes;
        const uint32_t sbytes = nr * row_bytes;
        const uint32_t cbytes = W > 0 ? nr * (unsigned)W * cs_es : 0u;
        const uint32_t ibytes = nr * (unsigned)sizeof(IoT);
        mbar_arrive_expect_tx(bar, sbytes + cbytes + ibytes * (zg ? 3u : 2u) + 2u * bc_bytes);
        tma_load_1d(dst, static_cast<const char*>(p.state) +
                             (slot * p.st_b + (int64_t)c0 * p.st_h) * (int64_t)sizeof(ST), sbytes, bar);
        if (W > 0)
            tma_load_1d(dst + off_cs, static_cast<const char*>(p.conv_state) +
                                          (slot * p.cs_b + (int64_t)c0 * p.cs_c) * (int64_t)cs_es, cbytes, bar);
        tma_load_1d(dst + off_x, xg + b * p.x_b + c0, ibytes, bar);
        tma_load_1d(dst + off_dt, dtg + b * p.dt_b + c0, ibytes, bar);
        if (zg) tma_load_1d(dst + off_z, zg + b * p.z_b + c0, ibytes, bar);
        tma_load_1d(dst + off_B, Bg + b * p.B_b, bc_bytes, bar);
        tma_load_1d(dst + off_C, Cg + b * p.C_b, bc_bytes, bar);
    };

    if (lane == 0) {
        for (unsigned s2 = 0; s2 < kWarpStages; ++s2) mbar_init(&bars[s2], 1);
        mbar_fence_init();
    }
    __syncwarp();
    if (lane == 0)
        for (unsigned k = 0; k < min(cnt, (unsigned)kWarpStages); ++k) issue(k);

    for (unsigned k = 0; k < cnt; ++k) {
        const unsigned item = i0 + k;
        const unsigned cb = item / Bn, b = item - cb * Bn;
        const unsigned c0 = cb * rb;
        const unsigned c = c0 + lane;
        const int64_t slot = slot_of(b);
        const bool rok = slot >= 0 && c < Dch;
        const unsigned cc = rok ? c : 0u;
        // this lane's channel parameters, loaded before the stage wait so their
        // latency overlaps the copy; A in the lane's rotated chunk order
        float wv[W > 0 ? W : 1];
        float cbias = 0.0f, dbias = 0.0f, dskip = 0.0f;
        float4 a4[NS / 4];
        if (rok) {
#pragma unroll
            for (int kk = 0; kk < W; ++kk) wv[kk] = p.conv_w[cc * p.cw_c + kk * p.cw_w];
            cbias = (W > 0 && p.conv_b) ? p.conv_b[cc * p.cb_c] : 0.0f;
            dbias = p.dt_bias ? p.dt_bias[cc * p.db_h] : 0.0f;
            dskip = p.Dp ? p.Dp[cc * p.D_h] : 0.0f;
            const float* ap = p.A + cc * p.A_h;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const unsigned cj = (j + rot) & (CPT - 1u);
#pragma unroll
                for (int e = 0; e < VE; e += 4) a4[(j * VE + e) / 4] = __ldg(reinterpret_cast<const float4*>(ap + cj * VE + e));
            }
        }
        const unsigned stage = k % kWarpStages;
        const bool ok = mbar_wait_bounded(&bars[stage], (k / kWarpStages) & 1u, plan.wait_budget);
        if (__any_sync(0xffffffffu, !ok)) {
            // give up: wait (bounded) for this warp's copies still in flight, flag, exit
            if (lane == 0) {
                // items issued so far: up to k + kWarpStages - 2 (the first
                // kWarpStages before the loop, one refill per later step)
                const unsigned hi = min(cnt, k == 0 ? (unsigned)kWarpStages : k + kWarpStages - 1);
                for (unsigned kk = k; kk < hi; ++kk) {
#ifdef SSM_TEST_HOOKS
                    if ((int64_t)(i0 + kk) == plan.drop_item) continue;  // never issued
#endif
                    mbar_wait_bounded(&bars[kk % kWarpStages], (kk / kWarpStages) & 1u, kCleanupBudget);
                }
                bulk_wait_all();
                report_device_error(&g_ssm_device_error, SSM_KERNEL_SSU_ROW_TMA, (long long)(i0 + k));
            }
            return;
        }
        {
            // widen the item's B and C once for the warp (every lane reads all of them)
            const unsigned char* st0 = ring + stage * stage_bytes;
            for (int i = (int)lane; i < 2 * NS; i += 32)
                bcw[warp][i] = to_f(reinterpret_cast<const IoT*>(st0 + (i < NS ? off_B : off_C))[i < NS ? i : i - NS]);
            __syncwarp();
        }
        if (rok) {
            unsigned char* st = ring + stage * stage_bytes;
            const unsigned cl = lane;
            const float xv = to_f(reinterpret_cast<const IoT*>(st + off_x)[cl]);
            float u = xv;
            float win[W > 0 ? W : 1];
            if constexpr (W > 0) {
                const unsigned char* crow = st + off_cs + cl * (unsigned)W * cs_es;
                if (cs_es == 4 && W == 4) {
                    // one 16-byte read per row: conflict-free across the warp
                    const float4 q = *reinterpret_cast<const float4*>(crow);
                    win[0] = q.y;
                    win[1] = q.z;
                    win[2] = q.w;
                } else {
#pragma unroll
                    for (int kk = 0; kk < W - 1; ++kk) win[kk] = ld_f(crow, kk + 1, p.cs_dt);
                }
                win[W - 1] = xv;
                float acc_c = cbias;
#pragma unroll
                for (int kk = 0; kk < W; ++kk) acc_c = fmaf(wv[kk], win[kk], acc_c);
                u = silu_f(acc_c);
            }
            const float v = to_f(reinterpret_cast<const IoT*>(st + off_dt)[cl]) + dbias;
            const float dl = p.softplus ? softplus_f(v) : v;
            const float dl2 = dl * kLog2e;
            const float du = dl * u;
            unsigned char* srow = st + cl * row_bytes;
            const float* bw = bcw[warp];
            const u64 dl2d = pk(dl2, dl2), dud = pk(du, du);
            u64 acc2 = 0;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const unsigned cj = (j + rot) & (CPT - 1u);
                float sv[VE];
                V::unpack(*reinterpret_cast<const uint4*>(srow + cj * 16), sv);
                // packed pairs: decay exp on the SFU per element, the rest f32x2
#pragma unroll
                for (int e = 0; e < VE; e += 4) {
                    const float4 a = a4[(j * VE + e) / 4];
                    const float4 b4 = *reinterpret_cast<const float4*>(bw + cj * VE + e);
                    const float4 c4 = *reinterpret_cast<const float4*>(bw + NS + cj * VE + e);
                    float e0, e1, e2, e3;
                    upk(fmul2(dl2d, pk(a.x, a.y)), e0, e1);
                    upk(fmul2(dl2d, pk(a.z, a.w)), e2, e3);
                    const u64 s01 = ffma2(pk(ex2_approx(e0), ex2_approx(e1)), pk(sv[e], sv[e + 1]),
                                          fmul2(dud, pk(b4.x, b4.y)));
                    const u64 s23 = ffma2(pk(ex2_approx(e2), ex2_approx(e3)), pk(sv[e + 2], sv[e + 3]),
                                          fmul2(dud, pk(b4.z, b4.w)));
                    acc2 = ffma2(pk(c4.x, c4.y), s01, acc2);
                    acc2 = ffma2(pk(c4.z, c4.w), s23, acc2);
                    upk(s01, sv[e], sv[e + 1]);
                    upk(s23, sv[e + 2], sv[e + 3]);
                }
                // new state back into the stage, in place; bulk-stored below
                *reinterpret_cast<uint4*>(srow + cj * 16) = V::pack(sv);
            }
            float acc_lo, acc_hi;
            upk(acc2, acc_lo, acc_hi);
            float y = fmaf(dskip, u, acc_lo + acc_hi);
            if (zg) y *= silu_f(to_f(reinterpret_cast<const IoT*>(st + off_z)[cl]));
            og[b * p.o_b + (int64_t)c * p.o_h] = from_f<IoT>(y);
            if constexpr (W > 0) {
                // rolled conv state (old entries 1..W-1, then x), in place
                unsigned char* crow = st + off_cs + cl * (unsigned)W * cs_es;
                if (cs_es == 4 && W == 4) {
                    *reinterpret_cast<float4*>(crow) = make_float4(win[0], win[1], win[2], win[3]);
                } else {
#pragma unroll
                    for (int kk = 0; kk < W; ++kk) st_f(crow, kk, p.cs_dt, win[kk]);
                }
            }
        }
        // each lane orders its shared-memory accesses of this stage before the
        // bulk copies that read (store) and later overwrite (refill) it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            // stream the item's state and conv rows out of the stage, then refill
            // the stage of the previous item once its own store has read it
            if (slot >= 0) {
                const unsigned nr = min(rb, Dch - c0);
                const unsigned char* st = ring + stage * stage_bytes;
                tma_store_1d(static_cast<char*>(p.state) + (slot * p.st_b + (int64_t)c0 * p.st_h) * (int64_t)sizeof(ST),
                             st, nr * row_bytes);
                if (W > 0)
                    tma_store_1d(static_cast<char*>(p.conv_state) + (slot * p.cs_b + (int64_t)c0 * p.cs_c) * (int64_t)cs_es,
                                 st + off_cs, nr * (unsigned)W * cs_es);
            }
            bulk_commit();
            if (k >= 1 && k - 1 + kWarpStages < cnt) {
                bulk_wait_read<1>();
                issue(k - 1 + kWarpStages);
            }
        }
    }
    if (lane == 0) bulk_wait_all();
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
// Done once per kernel, device and size (prepared_launch).
template <typename K>
cudaError_t prepare_tma_kernel(K kern, int block, int smem, int* per_sm) {
    return prepared_launch(
        reinterpret_cast<const void*>(kern), smem, block, per_sm,
        [&](int limit) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
            if (e != cudaSuccess) return e;
            return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                        cudaSharedmemCarveoutMaxShared);
        },
        [&](int* n) { return cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, kern, block, smem); });
}

template <typename ST, typename IoT>
cudaError_t launch_head_tma_io(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    const int smem = plan.stages * plan.stage_bytes;
    auto run = [&](auto kern) -> cudaError_t {
        int per_sm = 0;
        cudaError_t e = prepare_tma_kernel(kern, plan.block, smem, &per_sm);
        if (e != cudaSuccess) return e;
        if (plan.ctas_per_sm > 0 && plan.ctas_per_sm < per_sm) per_sm = plan.ctas_per_sm;
        // persistent grid: every CTA resident at once (the item ranges are
        // static), and every CTA given the same number of items
        const int64_t cap = (int64_t)plan.sms * (per_sm > 0 ? per_sm : 1);
        const int64_t per_cta = (plan.n_items + cap - 1) / cap;
        const int grid = (int)((plan.n_items + per_cta - 1) / per_cta);
        kern<<<grid, plan.block, smem, s>>>(p, plan);
        return cudaGetLastError();
    };
    const int key = plan.cpl * 10 + plan.rpt;
    switch (key) {
        case 11: return run(ssu_head_tma_kernel<ST, IoT, 1, 1>);
        case 12: return run(ssu_head_tma_kernel<ST, IoT, 1, 2>);
        case 14: return run(ssu_head_tma_kernel<ST, IoT, 1, 4>);
        case 21: return run(ssu_head_tma_kernel<ST, IoT, 2, 1>);
        case 22: return run(ssu_head_tma_kernel<ST, IoT, 2, 2>);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST, typename IoT>
cudaError_t launch_row_tma_io(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    const int smem = kRowWarps * kWarpStages * plan.stage_bytes;
    auto run = [&](auto kern) -> cudaError_t {
        int per_sm = 0;
        cudaError_t e = prepare_tma_kernel(kern, plan.block, smem, &per_sm);
        if (e != cudaSuccess) return e;
        // every CTA resident at once; each warp takes a contiguous item range
        const int64_t cap = (int64_t)plan.sms * (per_sm > 0 ? per_sm : 1);
        const int64_t want = (plan.n_items + kRowWarps - 1) / kRowWarps;
        const int grid = (int)(want < cap ? want : cap);
        kern<<<grid, plan.block, smem, s>>>(p, plan);
        return cudaGetLastError();
    };
    const int key = (int)p.W * 10 + plan.cpl;
    switch (key) {
        case 1: return run(ssu_row_tma_kernel<ST, IoT, 0, 1>);
        case 2: return run(ssu_row_tma_kernel<ST, IoT, 0, 2>);
        case 4: return run(ssu_row_tma_kernel<ST, IoT, 0, 4>);
        case 41: return run(ssu_row_tma_kernel<ST, IoT, 4, 1>);
        case 42: return run(ssu_row_tma_kernel<ST, IoT, 4, 2>);
        case 44: return run(ssu_row_tma_kernel<ST, IoT, 4, 4>);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST>
cudaError_t launch_row_tma(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    switch (p.x_dt) {
        case kF32: return launch_row_tma_io<ST, float>(p, plan, s);
        case kF16: return launch_row_tma_io<ST, __half>(p, plan, s);
        case kBF16: return launch_row_tma_io<ST, __nv_bfloat16>(p, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST>
cudaError_t launch_head_tma(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s) {
    switch (p.x_dt) {
        case kF32: return launch_head_tma_io<ST, float>(p, plan, s);
        case kF16: return launch_head_tma_io<ST, __half>(p, plan, s);
        case kBF16: return launch_head_tma_io<ST, __nv_bfloat16>(p, plan, s);
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
    if (plan.kernel == SSM_KERNEL_SSU_ROW_TMA) {
        switch (p.state_dt) {
            case kF32: return launch_row_tma<float>(p, plan, s);
            case kF16: return launch_row_tma<__half>(p, plan, s);
            case kBF16: return launch_row_tma<__nv_bfloat16>(p, plan, s);
            default: return cudaErrorInvalidValue;
        }
    }
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

int ssu_tma_max_stages() { return kTmaStagesMax; }
int ssu_row_tma_warps() { return kRowWarps; }
int ssu_row_tma_stages() { return kWarpStages; }

// Device address of the error record on device `dev` (the current device),
// looked up once per device so that kernels in other translation units can
// be handed it.  NULL if the lookup fails.
DeviceError* device_error_ptr(int dev) {
    static std::atomic<DeviceError*> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    DeviceError* ptr = cache[dev].load(std::memory_order_acquire);
    if (ptr) return ptr;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_ssm_device_error) != cudaSuccess) return nullptr;
    ptr = static_cast<DeviceError*>(addr);
    cache[dev].store(ptr, std::memory_order_release);
    return ptr;
}

namespace {
// Moves the error record into the snapshot and clears it, field by field
// with atomic exchanges: a report that lands while this runs is either in
// the snapshot or left for the next read, never lost.
__global__ void take_device_error_kernel() {
    g_ssm_device_error_snap.code = atomicExch(&g_ssm_device_error.code, 0);
    g_ssm_device_error_snap.kernel = atomicExch(&g_ssm_device_error.kernel, 0);
    g_ssm_device_error_snap.first_item =
        (long long)atomicExch(reinterpret_cast<unsigned long long*>(&g_ssm_device_error.first_item),
                              (unsigned long long)kNoItem);
}
}  // namespace

// After the work enqueued on `s`, take the current device's error record
// (read and clear in one step on the device) and copy it to *out.
cudaError_t read_and_clear_device_error(DeviceError* out, cudaStream_t s) {
    take_device_error_kernel<<<1, 1, 0, s>>>();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    DeviceError v{};
    e = cudaMemcpyFromSymbolAsync(&v, g_ssm_device_error_snap, sizeof(DeviceError), 0,
                                  cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    *out = v;
    return cudaSuccess;
}

}  // namespace ssm
