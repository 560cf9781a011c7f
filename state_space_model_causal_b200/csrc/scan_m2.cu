// scan_m2.cu -- prefill in the Mamba-2 layout for sm_100a: the selective scan
// over (nheads, headdim, dstate) with one scalar A and one Delta per head and
// step, B and C shared by the heads of a group, then the D skip and the SiLU(z)
// gate.  The Mamba-2 shape (batch, nheads, headdim, dstate, ngroups) is the one
// of "[XPU] Add tuned Mamba SSU configs for Intel Arc Pro B70" (vLLM PR #50534
// report), section 实现拆解; per (b, h), sequentially over t:
//
//   delta   = softplus(dt[b,h,t] + dt_bias[h])          (dt + dt_bias without softplus)
//   s[p,n]  = exp(delta * A[h]) * s[p,n] + delta * x[b,h,p,t] * B[b,g,n,t]
//   out     = (sum_n C[b,g,n,t] * s[p,n] + D[h] * x[b,h,p,t]) * silu(z[b,h,p,t])
//
// with g = h / (H / G).  The decay is one exponential per (b, h, t), so the
// work is FP32 arithmetic per state element and step: the kernel is bound by
// the FMA pipe, not by the SFU like the Mamba-1 prefill.  Because the decay
// is one scalar per (b, h, t), a chunk can run in a rescaled form: with P_t
// the product of the chunk's decays up to step t, g = s / P_t obeys
// g += (delta x / P_t) B, one FMA per element instead of a multiply and an
// FMA, and the readout is P_t (C . g).  Chunks whose decay product would
// leave the safe fp32 range run the direct recurrence.
//
// Fast kernel (time-major rows: headdim contiguous in x, z, out, and a
// multiple of 8; dstate 64, 128 or 256, contiguous in B, C; 16-byte aligned
// rows):
//   * a CTA is 128 threads on one (b, h) and a block of RPC = 512 / NG
//     headdim rows, NG = dstate / 16 (thread count, chunk length and the
//     register budget are build-time parameters; the defaults measured best).  Thread (pg, ng) owns rows 4pg..4pg+3 of
//     the block and state entries 16ng..16ng+15: a 4 x 16 register tile of the
//     state, updated with packed f32x2 operations across n, one 16-byte piece
//     of B and C at a time so that the tile fits with room to schedule;
//   * 16-step chunks of x, z, B, C are staged by 16-byte cp.async copies while
//     the previous chunk is scanned (x, z double-buffered for the epilogue;
//     B, C single-buffered, refilled once widened); dt is prefetched into a
//     register one chunk ahead;
//   * per chunk the CTA computes once per step delta and the decay (the
//     chunk's decay prefix products P_t by a warp prefix scan of delta * A, in
//     log2), delta * x per (step, row) -- divided by P_t in the rescaled form --
//     and the fp32 B, C rows (16-byte pieces XOR-swizzled so the NG groups of a
//     quarter-warp read distinct banks);
//   * the readout partials of 4 steps x 4 rows are summed over the NG threads
//     of a row block by a butterfly reduce-scatter; the epilogue applies the D
//     skip and the gate to 8 consecutive rows per thread and stores 16 bytes.
// Generic kernel: one warp per (b, h, p) row, any strides, dstate <= 256.
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

#include <atomic>
#include <type_traits>

namespace ssm {
namespace {

#ifndef SSM_M2_THREADS
#define SSM_M2_THREADS 128
#endif
#ifndef SSM_M2_STEPS
#define SSM_M2_STEPS 16
#endif
#ifndef SSM_M2_MIN_CTAS
#define SSM_M2_MIN_CTAS 3
#endif
constexpr int kM2Threads = SSM_M2_THREADS;  // threads per CTA
constexpr int kM2T = SSM_M2_STEPS;          // steps per chunk
constexpr int kM2MinCtas = SSM_M2_MIN_CTAS; // register budget: CTAs resident per SM
// A chunk runs in the rescaled form while every partial decay product P of
// the chunk lies within 2^+-64 (so that P and 1 / P stay far inside the fp32
// range); otherwise directly.
constexpr float kRescaleLog2 = 64.0f;

// (16-byte piece u of a B/C row) -> stored piece: the pieces a quarter-warp's
// NG groups read at once (u = 4 ng + k) land in distinct banks
__device__ __forceinline__ int m2_swz(int u) { return u ^ ((u >> 3) & 7); }

template <typename IoT, int NG> struct M2Smem {
    static constexpr int RPC = 4 * kM2Threads / NG;  // headdim rows per CTA
    static constexpr int N = 16 * NG;
    struct RawXZ {
        IoT x[kM2T][RPC];
        IoT z[kM2T][RPC];
    };
    RawXZ raw[2];      // x, z: read again by the epilogue, so double-buffered
    IoT rawB[kM2T][N];  // B, C: widened right after arrival, single buffer
    IoT rawC[kM2T][N];
    float2 dd[kM2T];           // per step: (decay, delta), or rescaled (P_t, delta / P_t)
    float dx[kM2T][RPC];       // delta * x
    float B[kM2T][N];          // swizzled fp32 rows
    float C[kM2T][N];
    float y[kM2T][RPC];        // sum_n C s
};

__device__ __forceinline__ void cp_async16_m2(void* dst, const void* src, bool valid) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

template <typename IoT, int NG>
__global__ void __launch_bounds__(kM2Threads, kM2MinCtas) scan_m2_kernel(const ScanM2Problem p, const M2Plan mp);

// Per device: the shared-memory attributes of the fast kernel, set once, and
// the CTAs that fit on one SM (0 = not queried yet, else count + 1).
template <typename IoT, int NG>
int m2_ctas_per_sm(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 0;
    int v = cache[dev].load(std::memory_order_acquire);
    if (v == 0) {
        auto kern = scan_m2_kernel<IoT, NG>;
        const int smem = (int)sizeof(M2Smem<IoT, NG>);
        int n = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kM2Threads, smem) != cudaSuccess)
            return 0;
        v = n + 1;
        cache[dev].store(v, std::memory_order_release);
    }
    return v - 1;
}

__device__ __forceinline__ unsigned m2_ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void m2_st_release(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned m2_atom_inc(unsigned* p, unsigned lim) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(lim) : "memory");
    return old;
}

// A unit is one (b, h, row block) over the whole sequence in 16-step chunks.
// CTA w takes the slice [w * total / workers, (w + 1) * total / workers) of
// the flattened (unit, chunk) list: the head of the unit the slice ends in
// first (its state handed to CTA w + 1 through the workspace), then whole
// units, then the tail of the unit the slice starts in (from the state CTA
// w - 1 handed over).  Without a workspace, workers == units and every CTA
// runs one whole unit.
template <typename IoT, int NG>
__global__ void __launch_bounds__(kM2Threads, kM2MinCtas) scan_m2_kernel(const ScanM2Problem p, const M2Plan mp) {
    using S = M2Smem<IoT, NG>;
    constexpr int RPC = S::RPC;
    constexpr int N = S::N;
    constexpr int E = 16 / (int)sizeof(IoT);  // elements per 16-byte copy
    extern __shared__ __align__(16) unsigned char m2_smem[];
    S& sm = *reinterpret_cast<S*>(m2_smem);
    __shared__ unsigned s_gen;
    __shared__ int s_got;
    __shared__ int s_rescale;

    const int tid = threadIdx.x;
    const int ng = tid % NG;
    const int pg = tid / NG;
    const int64_t w = blockIdx.x;
    const int64_t L = p.L;
    const int64_t nck = mp.nck;
    const int64_t total = mp.units * nck;
    const int64_t s0 = w * total / mp.workers;
    const int64_t e0 = (w + 1) * total / mp.workers;
    const bool has_head = (e0 % nck) != 0;
    const bool has_tail = (s0 % nck) != 0;
    const int64_t first_full = (s0 + nck - 1) / nck;
    const int64_t n_full = e0 / nck - first_full;
    const int64_t nseg = (has_head ? 1 : 0) + n_full + (has_tail ? 1 : 0);
    auto seg_of = [&](int64_t i, int64_t& u, int64_t& k0, int64_t& k1) -> int {
        if (has_head) {
            if (i == 0) {
                u = e0 / nck; k0 = 0; k1 = e0 % nck;
                return 2;  // emits a hand-over
            }
            --i;
        }
        if (i < n_full) {
            u = first_full + i; k0 = 0; k1 = nck;
            return 0;
        }
        u = s0 / nck; k0 = s0 % nck; k1 = nck;
        return 1;  // receives a hand-over
    };
    if (mp.ws_head) {
        if (tid == 0) s_gen = *reinterpret_cast<volatile unsigned*>(mp.ws_head);
        __syncthreads();
    }
    const unsigned gen = mp.ws_head ? s_gen : 0u;

    // unit -> (b, h, first row); per-unit base pointers
    struct Unit {
        int64_t b, h, p0;
        int rows;
        const IoT *xg, *zg, *Bg, *Cg, *dtg;
        IoT* og;
    };
    auto unit = [&](int64_t uu) {
        Unit r;
        const int64_t pb = uu % mp.nblk;
        const int64_t bh = uu / mp.nblk;
        r.h = bh % p.H;
        r.b = bh / p.H;
        r.p0 = pb * RPC;
        const int64_t g = r.h / (p.H / p.G);
        r.rows = (int)(p.P - r.p0 < RPC ? p.P - r.p0 : RPC);
        r.xg = static_cast<const IoT*>(p.x) + r.b * p.x_b + r.h * p.x_h + r.p0;
        r.zg = p.z ? static_cast<const IoT*>(p.z) + r.b * p.z_b + r.h * p.z_h + r.p0 : nullptr;
        r.Bg = static_cast<const IoT*>(p.Bm) + r.b * p.B_b + g * p.B_g;
        r.Cg = static_cast<const IoT*>(p.Cm) + r.b * p.C_b + g * p.C_g;
        r.dtg = static_cast<const IoT*>(p.dt) + r.b * p.dt_b + r.h * p.dt_h;
        r.og = static_cast<IoT*>(p.out) + r.b * p.o_b + r.h * p.o_h + r.p0;
        return r;
    };

    // x, z of chunk ck of unit U: kM2T x RPC elements each, into raw[bi]
    auto fetch_xz = [&](const Unit& U, int64_t ck, int bi) {
        typename S::RawXZ& rw = sm.raw[bi];
        const int64_t t0 = ck * kM2T;
        constexpr int XC = kM2T * RPC / E;
        for (int i = tid; i < XC; i += kM2Threads) {
            const int t = i / (RPC / E), e = (i % (RPC / E)) * E;
            const bool v = t0 + t < L && e < U.rows;
            const int64_t ts = v ? t0 + t : 0;
            cp_async16_m2(&rw.x[t][e], U.xg + ts * p.x_t + (v ? e : 0), v);
            cp_async16_m2(&rw.z[t][e], (U.zg ? U.zg : U.xg) + ts * (U.zg ? p.z_t : p.x_t) + (v ? e : 0), v && U.zg);
        }
    };
    // B, C of chunk ck: kM2T x N elements each
    auto fetch_bc = [&](const Unit& U, int64_t ck) {
        const int64_t t0 = ck * kM2T;
        constexpr int BC = kM2T * N / E;
        for (int i = tid; i < BC; i += kM2Threads) {
            const int t = i / (N / E), e = (i % (N / E)) * E;
            const bool v = t0 + t < L;
            const int64_t ts = v ? t0 + t : 0;
            cp_async16_m2(&sm.rawB[t][e], U.Bg + ts * p.B_t + e, v);
            cp_async16_m2(&sm.rawC[t][e], U.Cg + ts * p.C_t + e, v);
        }
    };
    auto commit = []() { asm volatile("cp.async.commit_group;" ::: "memory"); };
    // dt of a chunk, one step per thread of the first warp
    auto load_dt = [&](const Unit& U, int64_t ck) -> float {
        const int64_t t = ck * kM2T + tid;
        return (tid < kM2T && t < L) ? to_f(U.dtg[t * p.dt_t]) : 0.0f;
    };

    // this thread's B/C pieces: u = 4ng + k, stored at m2_swz(u)
    int boff[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) boff[k] = m2_swz(4 * ng + k) * 4;

    int64_t seg = 0, u = 0, k0 = 0, k1 = 0;
    int kind = seg_of(0, u, k0, k1);
    Unit cu = unit(u);
    float A2 = 0.0f, dbias = 0.0f, dskip = 0.0f;
    u64 hs[4][8];
    // state tile of a segment's start: rows 4pg + r, entries 16ng + 2j, 16ng + 2j + 1 as pairs
    auto setup = [&]() {
        A2 = p.A[cu.h * p.A_h] * kLog2e;
        dbias = p.dt_bias ? p.dt_bias[cu.h * p.db_h] : 0.0f;
        dskip = p.Dp ? p.Dp[cu.h * p.D_h] : 0.0f;
        if (kind == 1) {
            if (tid == 0) {
                int got = 1;
                if (mp.ws_flags) {
                    const unsigned* flag = mp.ws_flags + (w - 1);
                    const long long t_start = clock64();
                    while (m2_ld_acquire(flag) != gen + 1u) {
                        if (clock64() - t_start > mp.wait_budget) {
                            got = 0;
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                if (!got) report_device_error(mp.err, SSM_KERNEL_SCAN_M2, (long long)u);
                s_got = got;
            }
            __syncthreads();
            const bool got = s_got != 0;
            const float* slot = mp.ws_slots + (w - 1) * (int64_t)(RPC * N);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float2 v = make_float2(0.0f, 0.0f);
                    if (got) v = __ldcg(reinterpret_cast<const float2*>(slot + (4 * pg + r) * N + 16 * ng + 2 * j));
                    hs[r][j] = pk(v.x, v.y);
                }
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = 4 * pg + r;
                const bool v = row < cu.rows;
                const float* src = p.ssm_state ? p.ssm_state + cu.b * p.ss_b + cu.h * p.ss_h +
                                                     (cu.p0 + (v ? row : 0)) * p.ss_p + 16 * ng * p.ss_n
                                               : nullptr;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float a = 0.0f, c = 0.0f;
                    if (src && v) {
                        a = src[(2 * j) * p.ss_n];
                        c = src[(2 * j + 1) * p.ss_n];
                    }
                    hs[r][j] = pk(a, c);
                }
            }
        }
    };
    setup();

    int bi = 0;
    fetch_xz(cu, k0, bi);
    fetch_bc(cu, k0);
    commit();
    float dt_next = load_dt(cu, k0);
    int64_t k = k0;
    for (;;) {
        // the chunk after this one, possibly in the next segment
        int64_t nu = u, nk = k + 1, nk0 = k0, nk1 = k1;
        int nkind = kind;
        bool more = true, newseg = false;
        if (nk >= k1) {
            if (seg + 1 < nseg) {
                nkind = seg_of(seg + 1, nu, nk0, nk1);
                nk = nk0;
                newseg = true;
            } else {
                more = false;
            }
        }
        const Unit nuu = newseg ? unit(nu) : cu;
        const int64_t t0 = k * kM2T;
        const int steps = (int)(L - t0 < kM2T ? L - t0 : kM2T);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        // ---- per step (first warp, one step per lane): delta and the decay,
        // steps past L keep the state.  The chunk's log2 decays are summed by
        // a prefix scan: P_t = 2^cum_t is the decay from the chunk start to
        // the end of step t.
        if (tid < 32) {
            float delta = 0.0f, l2 = 0.0f;
            if (tid < steps) {
                const float v = dt_next + dbias;
                delta = p.softplus ? softplus_f(v) : v;
                l2 = delta * A2;
            }
            float cum = l2;
#pragma unroll
            for (int o = 1; o < kM2T; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, cum, o);
                if (tid >= o) cum += up;
            }
            // rescaled only while every P_t and 1 / P_t stays within 2^+-64
            // (delta * A can be positive without the softplus)
            float lo = tid < kM2T ? cum : 0.0f, hi = lo;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            }
            const bool rs = lo >= -kRescaleLog2 && hi <= kRescaleLog2;
            if (tid < kM2T)
                sm.dd[tid] = rs ? make_float2(ex2_approx(cum), delta * ex2_approx(-cum))
                                : make_float2(ex2_approx(l2), delta);
            if (tid == 0) s_rescale = rs;
        }
        __syncthreads();  // dd and this chunk's staged rows visible to all
        const bool rescale = s_rescale != 0;
        if (more) {
            fetch_xz(nuu, nk, bi ^ 1);
            dt_next = load_dt(nuu, nk);
        }
        const typename S::RawXZ& rw = sm.raw[bi];
        // ---- widen: delta * x per (step, row), fp32 B / C rows (swizzled)
        for (int i = tid; i < kM2T * RPC / 8; i += kM2Threads) {
            const int t = i / (RPC / 8), e = (i % (RPC / 8)) * 8;
            float xv[8];
            if constexpr (sizeof(IoT) == 2) {
                Vec16<IoT>::unpack(*reinterpret_cast<const uint4*>(&rw.x[t][e]), xv);
            } else {
                Vec16<float>::unpack(*reinterpret_cast<const uint4*>(&rw.x[t][e]), xv);
                Vec16<float>::unpack(*reinterpret_cast<const uint4*>(&rw.x[t][e + 4]), xv + 4);
            }
            const float dl = sm.dd[t].y;
            *reinterpret_cast<float4*>(&sm.dx[t][e]) = make_float4(dl * xv[0], dl * xv[1], dl * xv[2], dl * xv[3]);
            *reinterpret_cast<float4*>(&sm.dx[t][e + 4]) = make_float4(dl * xv[4], dl * xv[5], dl * xv[6], dl * xv[7]);
        }
        for (int i = tid; i < kM2T * N / 4; i += kM2Threads) {
            const int t = i / (N / 4), uq = i % (N / 4);  // 16-byte fp32 piece uq of row t
            float bv[4], cv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                bv[q] = to_f(sm.rawB[t][4 * uq + q]);
                cv[q] = to_f(sm.rawC[t][4 * uq + q]);
            }
            const int su = m2_swz(uq) * 4;
            *reinterpret_cast<float4*>(&sm.B[t][su]) = make_float4(bv[0], bv[1], bv[2], bv[3]);
            *reinterpret_cast<float4*>(&sm.C[t][su]) = make_float4(cv[0], cv[1], cv[2], cv[3]);
        }
        __syncthreads();
        // the raw B/C rows are widened: the next chunk's may land now
        if (more) fetch_bc(nuu, nk);
        commit();

        // ---- scan: 4 groups of 4 steps.  Direct form: s = decay * s + dx * B.
        // Rescaled form: the tile holds g = s / P_t, updated by g += (dx / P_t) * B
        // (dd carries delta / P_t, so dx does too); the readout C . g is scaled by
        // P_t, and at the chunk's end the tile is scaled back, s = P_end * g.
        // Both give s_t = sum_{u<=t} (P_t / P_u) dx_u B_u + P_t s_start; the
        // rescaled one in two FP32 operations per element and step instead of
        // three.
        auto scan_chunk = [&](auto rescaled) {
            constexpr bool RS = decltype(rescaled)::value;
#pragma unroll 1
            for (int tt = 0; tt < kM2T; tt += 4) {
                float v[16];  // v[4r + kk]: partial readout of row r at step tt + kk
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int t = tt + kk;
                    const float decay = sm.dd[t].x;
                    const u64 dA2 = pk(decay, decay);
                    const float4 dx4 = *reinterpret_cast<const float4*>(&sm.dx[t][4 * pg]);
                    const u64 dx2[4] = {pk(dx4.x, dx4.x), pk(dx4.y, dx4.y), pk(dx4.z, dx4.z), pk(dx4.w, dx4.w)};
                    u64 y2[4];
                    // one 16-byte piece of B and C at a time (short live ranges)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 bq = *reinterpret_cast<const float4*>(&sm.B[t][boff[q]]);
                        const float4 cq = *reinterpret_cast<const float4*>(&sm.C[t][boff[q]]);
                        const u64 b2[2] = {pk(bq.x, bq.y), pk(bq.z, bq.w)};
                        const u64 c2[2] = {pk(cq.x, cq.y), pk(cq.z, cq.w)};
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                const int j = 2 * q + jj;
                                if constexpr (RS)
                                    hs[r][j] = ffma2(dx2[r], b2[jj], hs[r][j]);
                                else
                                    hs[r][j] = ffma2(dA2, hs[r][j], fmul2(dx2[r], b2[jj]));
                                y2[r] = j == 0 ? fmul2(c2[jj], hs[r][j]) : ffma2(c2[jj], hs[r][j], y2[r]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        float lo, hi;
                        upk(y2[r], lo, hi);
                        v[4 * r + kk] = RS ? (lo + hi) * decay : lo + hi;  // decay holds P_t
                    }
                }
                // butterfly reduce-scatter over the NG threads of the row group:
                // thread ng ends with v[i], i = ng * (16 / NG) + local
#pragma unroll
                for (int m = NG / 2, S2 = 8; m >= 1; m >>= 1, S2 >>= 1) {
                    const bool up = (ng & m) != 0;
#pragma unroll
                    for (int i = 0; i < S2; ++i) {
                        const float send = up ? v[i] : v[i + S2];
                        const float keep = up ? v[i + S2] : v[i];
                        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                    }
                }
#pragma unroll
                for (int l = 0; l < 16 / NG; ++l) {
                    const int i = ng * (16 / NG) + l;
                    sm.y[tt + (i & 3)][4 * pg + (i >> 2)] = v[l];
                }
            }
            if constexpr (RS) {
                const u64 pe = pk(sm.dd[kM2T - 1].x, sm.dd[kM2T - 1].x);  // P at the chunk's end
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 8; ++j) hs[r][j] = fmul2(pe, hs[r][j]);
            }
        };
        if (rescale)
            scan_chunk(std::true_type{});
        else
            scan_chunk(std::false_type{});
        __syncthreads();

        // ---- epilogue: D skip and gate on 8 consecutive rows, 16-byte stores
        for (int i = tid; i < kM2T * RPC / 8; i += kM2Threads) {
            const int t = i / (RPC / 8), e = (i % (RPC / 8)) * 8;
            if (t >= steps || e >= cu.rows) continue;
            float xv[8], zv[8], o[8];
            if constexpr (sizeof(IoT) == 2) {
                Vec16<IoT>::unpack(*reinterpret_cast<const uint4*>(&rw.x[t][e]), xv);
                Vec16<IoT>::unpack(*reinterpret_cast<const uint4*>(&rw.z[t][e]), zv);
            } else {
                Vec16<float>::unpack(*reinterpret_cast<const uint4*>(&rw.x[t][e]), xv);
                Vec16<float>::unpack(*reinterpret_cast<const uint4*>(&rw.x[t][e + 4]), xv + 4);
                Vec16<float>::unpack(*reinterpret_cast<const uint4*>(&rw.z[t][e]), zv);
                Vec16<float>::unpack(*reinterpret_cast<const uint4*>(&rw.z[t][e + 4]), zv + 4);
            }
            const float4 y0 = *reinterpret_cast<const float4*>(&sm.y[t][e]);
            const float4 y1 = *reinterpret_cast<const float4*>(&sm.y[t][e + 4]);
            const float ys[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                o[q] = fmaf(dskip, xv[q], ys[q]);
                if (cu.zg) o[q] *= silu_f(zv[q]);
            }
            IoT* dst = cu.og + (t0 + t) * p.o_t + e;
            if constexpr (sizeof(IoT) == 2) {
                __stcs(reinterpret_cast<uint4*>(dst), Vec16<IoT>::pack(o));
            } else {
                __stcs(reinterpret_cast<uint4*>(dst), Vec16<float>::pack(o));
                __stcs(reinterpret_cast<uint4*>(dst) + 1, Vec16<float>::pack(o + 4));
            }
        }
        // the next chunk overwrites dd / dx / B / C / y only after its own
        // first barrier, which every thread reaches after this epilogue

        // ---- end of a segment: hand the tile over, or write the final state
        if (k + 1 == k1) {
            if (kind == 2) {
                float* slot = mp.ws_slots + w * (int64_t)(RPC * N);
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float a, c;
                        upk(hs[r][j], a, c);
                        __stcg(reinterpret_cast<float2*>(slot + (4 * pg + r) * N + 16 * ng + 2 * j), make_float2(a, c));
                    }
                __threadfence();
                __syncthreads();
                if (tid == 0) m2_st_release(mp.ws_flags + w, gen + 1u);
            } else if (p.ssm_state) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int row = 4 * pg + r;
                    if (row >= cu.rows) continue;
                    float* dst = p.ssm_state + cu.b * p.ss_b + cu.h * p.ss_h + (cu.p0 + row) * p.ss_p + 16 * ng * p.ss_n;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float a, c;
                        upk(hs[r][j], a, c);
                        dst[(2 * j) * p.ss_n] = a;
                        dst[(2 * j + 1) * p.ss_n] = c;
                    }
                }
            }
        }
        if (!more) break;
        if (newseg) {
            ++seg;
            u = nu;
            k0 = nk0;
            k1 = nk1;
            kind = nkind;
            cu = nuu;
            __syncthreads();  // every thread is done with this segment's tile
            setup();
        }
        k = nk;
        bi ^= 1;
    }

    // ---- the last CTA to finish advances the workspace generation
    if (mp.ws_head) {
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const unsigned old = m2_atom_inc(mp.ws_head + 1, (unsigned)(mp.workers - 1));
            if (old == (unsigned)(mp.workers - 1)) atomicAdd(mp.ws_head, 1u);
        }
    }
}

// One warp per (b, h, p) row, any strides, dstate <= 256: lane l owns entries
// n = l + 32 i.
template <typename IoT>
__global__ void __launch_bounds__(128) scan_m2_generic_kernel(const ScanM2Problem p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= p.Bn * p.H * p.P) return;
    const int64_t pp = row % p.P, h = (row / p.P) % p.H, b = row / (p.P * p.H);
    const int64_t g = h / (p.H / p.G);
    const float A = p.A[h * p.A_h];
    const float dbias = p.dt_bias ? p.dt_bias[h * p.db_h] : 0.0f;
    const float dskip = p.Dp ? p.Dp[h * p.D_h] : 0.0f;
    float s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = lane + 32 * i;
        s[i] = (n < p.N && p.ssm_state) ? p.ssm_state[b * p.ss_b + h * p.ss_h + pp * p.ss_p + n * p.ss_n] : 0.0f;
    }
    for (int64_t t = 0; t < p.L; ++t) {
        const float v = ld_f(p.dt, b * p.dt_b + h * p.dt_h + t * p.dt_t, p.io_dt) + dbias;
        const float delta = p.softplus ? softplus_f(v) : v;
        const float decay = exp_fast(delta * A);
        const float xv = ld_f(p.x, b * p.x_b + h * p.x_h + pp * p.x_p + t * p.x_t, p.io_dt);
        const float dx = delta * xv;
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t n = lane + 32 * i;
            if (n < p.N) {
                const float bv = ld_f(p.Bm, b * p.B_b + g * p.B_g + n * p.B_n + t * p.B_t, p.io_dt);
                const float cv = ld_f(p.Cm, b * p.C_b + g * p.C_g + n * p.C_n + t * p.C_t, p.io_dt);
                s[i] = fmaf(decay, s[i], dx * bv);
                acc = fmaf(cv, s[i], acc);
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            float y = fmaf(dskip, xv, acc);
            if (p.z) y *= silu_f(ld_f(p.z, b * p.z_b + h * p.z_h + pp * p.z_p + t * p.z_t, p.io_dt));
            st_f(p.out, b * p.o_b + h * p.o_h + pp * p.o_p + t * p.o_t, p.io_dt, y);
        }
    }
    if (p.ssm_state) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t n = lane + 32 * i;
            if (n < p.N) p.ssm_state[b * p.ss_b + h * p.ss_h + pp * p.ss_p + n * p.ss_n] = s[i];
        }
    }
}

template <typename IoT, int NG>
cudaError_t launch_m2_ng(const ScanM2Problem& p, const M2Plan& mp, cudaStream_t s) {
    using Sm = M2Smem<IoT, NG>;
    auto kern = scan_m2_kernel<IoT, NG>;
    const int smem = (int)sizeof(Sm);
    if (m2_ctas_per_sm<IoT, NG>(mp.dev) <= 0) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)mp.grid);
    cfg.blockDim = dim3(kM2Threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = mp.cooperative ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p, mp);
}

template <typename IoT>
cudaError_t launch_m2_io(const ScanM2Problem& p, const M2Plan& mp, cudaStream_t s, int* ctas) {
    switch (p.N / 16) {
#define SSM_M2_CASE(ng)                                              \
    case ng:                                                         \
        if (ctas) {                                                  \
            *ctas = m2_ctas_per_sm<IoT, ng>(mp.dev);                 \
            return cudaSuccess;                                      \
        }                                                            \
        return launch_m2_ng<IoT, ng>(p, mp, s);
        SSM_M2_CASE(4)
        SSM_M2_CASE(8)
        SSM_M2_CASE(16)
#undef SSM_M2_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// the fast kernel's dstate values (NG = 4, 8, 16): 0 for any other dstate
int scan_m2_rows_per_cta(int64_t N) {
    return N == 64 || N == 128 || N == 256 ? (int)(4 * kM2Threads / (N / 16)) : 0;
}
int scan_m2_threads() { return kM2Threads; }

int scan_m2_smem_bytes(int io_dt, int64_t N) {
    auto pick = [&](auto tag) -> int {
        using T = decltype(tag);
        switch (N / 16) {
            case 1: return (int)sizeof(M2Smem<T, 1>);
            case 2: return (int)sizeof(M2Smem<T, 2>);
            case 4: return (int)sizeof(M2Smem<T, 4>);
            case 8: return (int)sizeof(M2Smem<T, 8>);
            case 16: return (int)sizeof(M2Smem<T, 16>);
            default: return 0;
        }
    };
    if (io_dt == kF32) return pick(float{});
    if (io_dt == kF16) return pick(__half{});
    return pick(__nv_bfloat16{});
}

int scan_m2_ctas_per_sm(const ScanM2Problem& p, int dev) {
    M2Plan mp{};
    mp.dev = dev;
    int n = 0;
    cudaError_t e = cudaErrorInvalidValue;
    switch (p.io_dt) {
        case kF32: e = launch_m2_io<float>(p, mp, nullptr, &n); break;
        case kF16: e = launch_m2_io<__half>(p, mp, nullptr, &n); break;
        case kBF16: e = launch_m2_io<__nv_bfloat16>(p, mp, nullptr, &n); break;
        default: break;
    }
    return e == cudaSuccess ? n : 0;
}

cudaError_t launch_scan_m2(const ScanM2Problem& p, int kernel, const M2Plan& mp, cudaStream_t s) {
    if (kernel == SSM_KERNEL_SCAN_M2) {
        switch (p.io_dt) {
            case kF32: return launch_m2_io<float>(p, mp, s, nullptr);
            case kF16: return launch_m2_io<__half>(p, mp, s, nullptr);
            case kBF16: return launch_m2_io<__nv_bfloat16>(p, mp, s, nullptr);
            default: return cudaErrorInvalidValue;
        }
    }
    const int64_t rows = p.Bn * p.H * p.P;
    const unsigned grid = (unsigned)((rows + 3) / 4);  // generic kernel: 4 warps of 32
    switch (p.io_dt) {
        case kF32: scan_m2_generic_kernel<float><<<grid, 128, 0, s>>>(p); break;
        case kF16: scan_m2_generic_kernel<__half><<<grid, 128, 0, s>>>(p); break;
        case kBF16: scan_m2_generic_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ssm
