// scan_bal.cu -- the load-balanced fused prefill for sm_100a (d_state <= 16,
// time dimension contiguous and 16-byte aligned, L % 8 == 0): causal conv1d
// -> SiLU -> softplus(dt + dt_bias) -> selective scan -> D skip -> SiLU(z)
// gate, the operator chain "causal-conv1d, selective-scan, silu,
// element-mul" of "feat(llama.cu): 适配 mamba 模型" (section 2.1), reading and
// writing the conv and SSM state caches of its section 3.1.
//
//   u     = silu(bias[d] + sum_k w[d,k] * x[t-(W-1)+k])
//   delta = softplus(dt[t] + dt_bias[d])
//   h[n]  = exp(delta * A[d,n]) * h[n] + delta * B[n,t] * u
//   out   = (sum_n C[n,t] * h[n] + D[d] * u) * silu(z[t])
//
// What bounds it: the SFU.  Every (b, t, d, n) element needs one
// exp(delta * A) and every (b, t, d) three more SFU operations (the
// exponentials of the conv SiLU, the softplus and the gate; their reciprocals
// run on the FMA pipe); the four FP32 operations per element and the HBM
// traffic (8 bytes per (b, t, d)) are far below their own ceilings.  The
// design keeps the SFU fed evenly on every SM sub-partition:
//
//   * Work is split into units (batch entry, 16 channels) x the whole
//     sequence, each cut into 32-step chunks.  A warp is a worker; the workers
//     are persistent (two per sub-partition) and each takes an equal,
//     contiguous slice of the flattened (unit, chunk) list, so every
//     sub-partition gets the same number of chunks to within one -- whole
//     units per warp would leave some sub-partitions with one unit more than
//     others for the whole kernel.  A slice is [tail of unit U][whole units]
//     [head of unit V]; the worker runs the head first and publishes the state
//     it reaches (1 KB) to its successor, then its whole units, then the tail,
//     which starts from the state its predecessor published at the very
//     beginning of its own run.  The hand-over needs a caller-supplied
//     workspace; without one every worker takes whole units.  All waits are
//     bounded.
//   * With few units (short batches) the sequence is cut into pieces run in
//     two passes (context-parallel mode, see BalPlan): pieces from zero states
//     with end-state records, then re-scans from the states the records
//     compose to.
//   * In a warp, lane (cp, q) holds channels 2cp, 2cp+1 x state entries
//     4q..4q+3; the packed f32x2 operations run across state entries, so
//     B[n], B[n+1] form one operand straight from the widened fp32 [t][n] rows.
//   * The lane that stages 16 steps of a channel computes their conv, SiLU,
//     softplus, D*u and gate in registers (history by shuffle), writes
//     (delta, delta*u) for the scan lanes and later applies D*u and the gate
//     to the same steps.
//   * Readout partials go to shared memory once per 4-step group, after the
//     next group's first operands are loaded (a store ahead of the loads
//     would hold them back); the epilogue lane sums the four partials of a
//     (step, channel).  Padded and swizzled layouts keep every shared-memory
//     access conflict-free.
//   * The next chunk's x/dt/z/B/C tiles are copied by cp.async while the
//     current one is computed (double buffer).
//   * Optionally SW of every eight exponential pairs take their value from the
//     Cody-Waite + minimax polynomial on the FMA pipe instead of the SFU.
#include "../../include/ssm_causal.h"
#include "common.cuh"
#include "problem.h"

#include <atomic>

namespace ssm {
namespace {

constexpr int kCH = 16;        // channels per unit
constexpr int kT = 32;         // steps per chunk
constexpr int kSPL = kT / 2;   // prologue / epilogue steps per lane (two lanes per channel)
constexpr int kWarps = 4;      // independent workers per CTA (one per SM sub-partition)
constexpr int kDdRow = kT + 2;      // (delta, delta*u) words per channel pair (two pads)
constexpr int kYpRow = kCH + 1;     // readout words per step (one pad)
constexpr int kSlot = kCH * 16 + kCH;  // hand-over slot: 16 x 16 state, 16 partial sums of delta

// One warp's shared memory.  Raw tiles are double-buffered (the next chunk's
// copies fly during the whole current chunk); the widened B/C rows, the
// (delta, delta*u) words and the readout partials are rewritten per chunk.
template <typename IoT> struct __align__(16) BalSmem {
    IoT xr[2][kCH][kT];   // raw x tiles
    IoT dtr[2][kCH][kT];  // raw dt
    IoT zr[2][kCH][kT];   // raw z
    IoT br[2][16][kT];    // raw B rows [n][t]
    IoT cr[2][16][kT];    // raw C rows
    float bf[kT][16];     // B widened, [t][n]
    float cf[kT][16];     // C widened
    float4 dd[kCH / 2][kDdRow];  // (delta, delta*u) of channels 2cp and 2cp+1 per step
    float4 yp[kT * kYpRow + 4];  // readout partials of the four lanes q per (step, channel)
};

// (delta, delta*u) row of a channel pair: steps 16..31 sit one word further
// on, so that the two prologue halves of a pair write distinct banks.
__device__ __forceinline__ int dd_at(int t) { return t + (t >> 4); }
// Readout partials of (step t, channel c), one 16-byte word each: one row of
// kYpRow words per step, channels 8..15 one word further on (the 32 lanes of
// a store hit 32 distinct banks), and steps 16..31 four words further on, so
// that the two halves of an epilogue quarter-warp (steps t and t + 16, four
// channels each) read eight distinct 16-byte bank groups.
__device__ __forceinline__ int yp_at(int t, int c) { return t * kYpRow + (t >> 4) * 4 + c + (c >> 3); }
// Raw tiles hold 16-byte pieces of each row XOR-swizzled by row, so that the
// pieces the prologue (and the B/C widening) read at once fall in distinct
// banks: rows are 4 pieces (16-bit) or 8 pieces (fp32) long.
template <typename IoT> __device__ __forceinline__ int piece_at(int row, int piece) {
    return sizeof(IoT) == 2 ? (piece ^ ((row >> 1) & 1)) : (piece ^ (row & 3));
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_inc_acq_rel(unsigned* p, unsigned lim) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(lim) : "memory");
    return old;
}

// 8 consecutive elements of a staged row, widened
template <typename IoT>
__device__ __forceinline__ void unpack8(const IoT* src, float* f) {
    if constexpr (sizeof(IoT) == 2) {
        Vec16<IoT>::unpack(*reinterpret_cast<const uint4*>(src), f);
    } else {
        Vec16<float>::unpack(*reinterpret_cast<const uint4*>(src), f);
        Vec16<float>::unpack(*(reinterpret_cast<const uint4*>(src) + 1), f + 4);
    }
}

// 8 consecutive steps s0 .. s0+7 (s0 a multiple of 8) of a swizzled raw row
template <typename IoT>
__device__ __forceinline__ void row8(const IoT* row, int r, int s0, float* f) {
    constexpr int E = 16 / (int)sizeof(IoT);
    if constexpr (sizeof(IoT) == 2) {
        unpack8(row + piece_at<IoT>(r, s0 / E) * E, f);
    } else {
        Vec16<float>::unpack(*reinterpret_cast<const uint4*>(row + piece_at<IoT>(r, s0 / E) * E), f);
        Vec16<float>::unpack(*reinterpret_cast<const uint4*>(row + piece_at<IoT>(r, s0 / E + 1) * E), f + 4);
    }
}

// Four consecutive B or C values of a [t][n] row as two packed fp32 pairs.
__device__ __forceinline__ void bc4(const float* row, u64* pr) {
    const float4 v = *reinterpret_cast<const float4*>(row);
    pr[0] = pk(v.x, v.y);
    pr[1] = pk(v.z, v.w);
}

// Parameters of the channel whose prologue a lane computes.
template <int W> struct BalChan {
    float w[W > 0 ? W : 1];
    float cbias, dbias, dskip;
    float hist[W > 1 ? W - 1 : 1];  // raw inputs at (chunk start) - (W-1) + i
};

// SP: delta = softplus(dt + dt_bias) (else dt + dt_bias); HZ: gate by SiLU(z).
template <typename IoT, int W, int SW, bool SP, bool HZ>
__global__ void __launch_bounds__(32 * kWarps, 2) scan_bal_kernel(const ScanProblem p, const BalPlan bp) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    // Newton steps of the SiLU reciprocals: 2 (< 7e-6 relative) for 16-bit
    // outputs, 3 (fp32 rounding) for fp32 outputs
    constexpr int kRcpSteps = sizeof(IoT) == 2 ? 2 : 3;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * kWarps + warp;
    if (w >= bp.workers) return;
    BalSmem<IoT>& sm = reinterpret_cast<BalSmem<IoT>*>(smem_raw)[warp];
    // scan role: lane (cp, q) holds channels 2cp, 2cp+1 x state entries 4q..4q+3
    const int cp = lane >> 2;
    const int q = lane & 3;
    // prologue / epilogue role: channel pc = 2cp + (q & 1), steps 16*(q>>1) .. +15
    const int pc = 2 * cp + (q & 1);
    const int ph = q >> 1;
    const int64_t nck = bp.nck;
    const int64_t total = bp.units * nck;
    const int64_t s = w * total / bp.workers;
    const int64_t e = (w + 1) * total / bp.workers;

    // ---- this worker's segments, in the order they run: head of the unit the
    // slice ends in (hand-over out), whole units, tail of the unit the slice
    // starts in (hand-over in)
    const bool has_head = (e % nck) != 0;
    const bool has_tail = (s % nck) != 0;
    const int64_t first_full = (s + nck - 1) / nck;
    const int64_t n_full = e / nck - first_full;
    const int64_t nseg = (has_head ? 1 : 0) + n_full + (has_tail ? 1 : 0);
    auto seg_of = [&](int64_t i, int64_t& u, int64_t& k0, int64_t& k1) -> int {
        if (has_head) {
            if (i == 0) {
                u = e / nck; k0 = 0; k1 = e % nck;
                return 2;  // emits a hand-over
            }
            --i;
        }
        if (i < n_full) {
            u = first_full + i; k0 = 0; k1 = nck;
            return 0;
        }
        u = s / nck; k0 = s % nck; k1 = nck;
        return 1;  // receives a hand-over
    };

    unsigned gen = 0;
    if (bp.ws_head) {
        if (lane == 0) gen = *reinterpret_cast<volatile unsigned*>(bp.ws_head);
        gen = __shfl_sync(0xffffffffu, gen, 0);
    }

    // ---- staging of one chunk's raw tiles (all lanes), one cp.async group.
    // Each lane copies the same pieces of every chunk: its row pointers are
    // worked out once per unit and advanced by the chunk's first step.
    constexpr int E = 16 / (int)sizeof(IoT);  // elements per 16-byte piece
    constexpr int PPR = kT / E;               // pieces per row
    constexpr int NXP = kCH * PPR / 32;       // x/dt/z pieces per lane per tensor
    constexpr int NBP = 16 * PPR / 32;        // B/C pieces per lane per tensor
    int64_t fu_cached = -1;
    const IoT *fx[NXP], *fdt[NXP], *fz[NXP], *fB[NBP], *fC[NBP];
    bool frow[NXP], fn[NBP];
    // unit -> (base unit: batch entry x channel block, piece, first chunk)
    auto unit_of = [&](int64_t uu, int64_t& ub, int& piece) -> int64_t {
        if (bp.cp_pieces > 1) {
            ub = uu / (bp.cp_pieces - 1);
            piece = (int)(uu % (bp.cp_pieces - 1)) + (bp.cp_pass == 2 ? 1 : 0);
            return (int64_t)piece * bp.piece_chunks;
        }
        ub = uu;
        piece = 0;
        return 0;
    };
    int64_t fkc0 = 0;
    auto fetch = [&](int64_t fu, int64_t fk, int fb) {
        if (fu != fu_cached) {
            fu_cached = fu;
            int64_t ub;
            int pce;
            fkc0 = unit_of(fu, ub, pce);
            const int64_t b = ub / bp.nblk;
            const int64_t d0 = (ub % bp.nblk) * kCH;
            const int64_t g = d0 / p.ch_per_group;
#pragma unroll
            for (int j = 0; j < NXP; ++j) {
                const int64_t d = d0 + (lane + 32 * j) / PPR;
                frow[j] = d < p.D;
                const int64_t ds = frow[j] ? d : 0;
                fx[j] = static_cast<const IoT*>(p.x) + b * p.x_b + ds * p.x_d;
                fdt[j] = static_cast<const IoT*>(p.dt) + b * p.dt_b + ds * p.dt_d;
                fz[j] = HZ ? static_cast<const IoT*>(p.z) + b * p.z_b + ds * p.z_d : nullptr;
            }
#pragma unroll
            for (int j = 0; j < NBP; ++j) {
                const int n = (lane + 32 * j) / PPR;
                fn[j] = n < p.N;
                const int64_t ns = fn[j] ? n : 0;
                fB[j] = static_cast<const IoT*>(p.Bm) + b * p.B_b + g * p.B_g + ns * p.B_n;
                fC[j] = static_cast<const IoT*>(p.Cm) + b * p.C_b + g * p.C_g + ns * p.C_n;
            }
        }
        const int64_t t0 = (fkc0 + fk) * kT;
#pragma unroll
        for (int j = 0; j < NXP; ++j) {
            const int i = lane + 32 * j, row = i / PPR, pcs = i % PPR;
            const int64_t t = t0 + pcs * E;
            const bool v = frow[j] && t < p.L;  // L % 8 == 0: a piece is all in or all out
            const int64_t ts = v ? t : 0;
            const int sp = piece_at<IoT>(row, pcs) * E;
            cp_async16(&sm.xr[fb][row][sp], fx[j] + ts, v);
            cp_async16(&sm.dtr[fb][row][sp], fdt[j] + ts, v);
            if (HZ) cp_async16(&sm.zr[fb][row][sp], fz[j] + ts, v);
        }
#pragma unroll
        for (int j = 0; j < NBP; ++j) {
            const int i = lane + 32 * j, n = i / PPR, pcs = i % PPR;
            const int64_t t = t0 + pcs * E;
            const bool v = fn[j] && t < p.L;
            const int64_t ts = v ? t : 0;
            const int sp = piece_at<IoT>(n, pcs) * E;
            cp_async16(&sm.br[fb][n][sp], fB[j] + ts, v);
            cp_async16(&sm.cr[fb][n][sp], fC[j] + ts, v);
        }
        cp_async_commit();
    };

    // ---- per-segment registers
    int64_t seg = 0, u = 0, k0 = 0, k1 = 0;
    int kind = seg_of(0, u, k0, k1);
    int64_t b = 0;
    int64_t sd[2];     // the scan lane's two channels (clamped to a valid row)
    bool sok[2];
    int64_t pd = 0;    // the prologue lane's channel (clamped)
    bool pok = false;
    BalChan<W> ch;
    u64 A2[2][2], h2[2][2];  // [channel][pair of state entries]
    const IoT* pxrow = nullptr;
    IoT* porow = nullptr;
    int64_t ub = 0;     // base unit of the segment
    int piece = 0;      // its piece (context-parallel mode)
    int64_t kc0 = 0;    // its first chunk in the whole sequence
    double sdl = 0.0;   // the prologue lane's sum of delta over its steps of the piece so far
                        // (fp64: exp(A * sum) must match the product of the steps' decays)
    bool store_out = true;

    auto setup = [&]() {
        kc0 = unit_of(u, ub, piece);
        store_out = !(bp.cp_pass == 1 && piece > 0);  // pass 1 keeps only piece 0's outputs
        b = ub / bp.nblk;
        const int64_t d0 = (ub % bp.nblk) * kCH;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int64_t d = d0 + 2 * cp + c;
            sok[c] = d < p.D;
            sd[c] = sok[c] ? d : d0;
        }
        pok = d0 + pc < p.D;
        pd = pok ? d0 + pc : d0;
        pxrow = static_cast<const IoT*>(p.x) + b * p.x_b + pd * p.x_d;
        porow = static_cast<IoT*>(p.out) + b * p.o_b + pd * p.o_d;
#pragma unroll
        for (int k = 0; k < W; ++k) ch.w[k] = pok ? p.conv_w[pd * p.cw_d + k * p.cw_k] : 0.0f;
        ch.cbias = (W > 0 && p.conv_b && pok) ? p.conv_b[pd * p.cb_d] : 0.0f;
        ch.dbias = (p.dt_bias && pok) ? p.dt_bias[pd * p.db_d] : 0.0f;
        ch.dskip = (p.Dp && pok) ? p.Dp[pd * p.D_d] : 0.0f;
        float h[2][4];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float a[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = 4 * q + j;
                const bool v = sok[c] && n < p.N;
                a[j] = v ? p.A[sd[c] * p.A_d + n * p.A_n] * kLog2e : 0.0f;
                h[c][j] = 0.0f;
            }
            A2[c][0] = pk(a[0], a[1]);
            A2[c][1] = pk(a[2], a[3]);
        }
        if (kind == 1) {
            // tail: the state the predecessor reached at chunk k0
            bool got = true;
            if (bp.ws_flags) {
                const unsigned* flag = bp.ws_flags + (w - 1);
                const long long t_start = clock64();
                while (ld_acquire_u32(flag) != gen + 1u) {
                    if (clock64() - t_start > bp.wait_budget) {
                        got = false;
                        break;
                    }
                    __nanosleep(128);
                }
            }
            sdl = 0.0;
            if (got) {
                const float* slot = bp.ws_slots + (w - 1) * kSlot;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(slot + (2 * cp + c) * 16 + 4 * q));
                    h[c][0] = v.x; h[c][1] = v.y; h[c][2] = v.z; h[c][3] = v.w;
                }
                if (ph == 0) sdl = (double)__ldcg(slot + kCH * 16 + pc);
            } else if (lane == 0) {
                // the tail of unit u starts from a zero state instead
                report_device_error(bp.err, SSM_KERNEL_SCAN_BAL, (long long)u);
            }
        } else {
            sdl = 0.0;
            if (piece == 0) {
                if (p.ssm_state) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int n = 4 * q + j;
                            if (sok[c] && n < p.N) h[c][j] = p.ssm_state[b * p.ss_b + sd[c] * p.ss_d + n * p.ss_n];
                        }
                }
            } else if (bp.cp_pass == 2) {
                // the state at the piece's start, composed from the pass-1
                // records: h_in(1) = h_end(0); h_in(j+1) = exp(A * sum delta(j)) * h_in(j) + h_end(j)
                const int64_t rec0 = ub * (bp.cp_pieces - 1);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int ch_ = 2 * cp + c;
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(bp.carry_h + (rec0 * kCH + ch_) * 16 + 4 * q));
                    h[c][0] = v.x; h[c][1] = v.y; h[c][2] = v.z; h[c][3] = v.w;
                    for (int j = 1; j < piece; ++j) {
                        const float sj = __ldcg(bp.carry_sdl + (rec0 + j) * kCH + ch_);
                        const float4 e = __ldcg(reinterpret_cast<const float4*>(
                            bp.carry_h + ((rec0 + j) * kCH + ch_) * 16 + 4 * q));
                        float a[4];
                        upk(A2[c][0], a[0], a[1]);
                        upk(A2[c][1], a[2], a[3]);
                        h[c][0] = fmaf(ex2_approx(a[0] * sj), h[c][0], e.x);
                        h[c][1] = fmaf(ex2_approx(a[1] * sj), h[c][1], e.y);
                        h[c][2] = fmaf(ex2_approx(a[2] * sj), h[c][2], e.z);
                        h[c][3] = fmaf(ex2_approx(a[3] * sj), h[c][3], e.w);
                    }
                }
            }
            // pass 1, pieces >= 1: zero state
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            h2[c][0] = pk(h[c][0], h[c][1]);
            h2[c][1] = pk(h[c][2], h[c][3]);
        }
        // conv history before the segment's first step (used by the ph == 0 lanes)
#pragma unroll
        for (int i = 0; i < W - 1; ++i) {
            float v = 0.0f;
            if (pok) {
                if (kc0 + k0 == 0) {
                    if (p.conv_state) v = ld_f(p.conv_state, b * p.cs_b + pd * p.cs_d + (1 + i) * p.cs_k, p.cs_dt);
                } else {
                    v = to_f(pxrow[(kc0 + k0) * kT - (W - 1) + i]);
                }
            }
            ch.hist[i] = v;
        }
    };
    setup();

    fetch(u, k0, 0);
    int buf = 0;
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
        cp_async_wait<0>();
        __syncwarp();  // this chunk's tiles are visible; the other buffer is free
        if (more) fetch(nu, nk, buf ^ 1);

        const int64_t t0 = (kc0 + k) * kT;
        // ---- widen B/C into [t][n] rows: lane (row n, half hh) converts 16
        // steps; the two halves write rows of opposite parity at each store so
        // that the 32 lanes hit 32 distinct banks
        {
            const int n = lane >> 1, hh = lane & 1;
            float bv[16], cv[16];
            row8(sm.br[buf][n], n, 16 * hh, bv);
            row8(sm.br[buf][n], n, 16 * hh + 8, bv + 8);
            row8(sm.cr[buf][n], n, 16 * hh, cv);
            row8(sm.cr[buf][n], n, 16 * hh + 8, cv + 8);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = i ^ (17 * hh);  // hh = 1: row 16 + (i ^ 1)
                sm.bf[r][n] = hh ? bv[i ^ 1] : bv[i];
                sm.cf[r][n] = hh ? cv[i ^ 1] : cv[i];
            }
        }
        // ---- prologue: steps 16ph .. 16ph+15 of channel pc
        float Du[kSPL], gate[kSPL];
        const int64_t tl = t0 + kSPL * ph;
        const bool vv[2] = {tl < p.L && pok, tl + 8 < p.L && pok};
        {
            float xs[kSPL], dts[kSPL], zs[kSPL], uu[kSPL];
            row8(sm.xr[buf][pc], pc, kSPL * ph, xs);
            row8(sm.xr[buf][pc], pc, kSPL * ph + 8, xs + 8);
            row8(sm.dtr[buf][pc], pc, kSPL * ph, dts);
            row8(sm.dtr[buf][pc], pc, kSPL * ph + 8, dts + 8);
            if (HZ) {
                row8(sm.zr[buf][pc], pc, kSPL * ph, zs);
                row8(sm.zr[buf][pc], pc, kSPL * ph + 8, zs + 8);
            }
            if constexpr (W > 0) {
                // history: the lane two below (same channel, first half) or the
                // channel's values before this chunk
                float prev[W > 1 ? W - 1 : 1];
#pragma unroll
                for (int i = 0; i < W - 1; ++i) {
                    const float left = __shfl_up_sync(0xffffffffu, xs[kSPL - (W - 1) + i], 2);
                    prev[i] = ph == 0 ? ch.hist[i] : left;
                }
#pragma unroll
                for (int i = 0; i < W - 1; ++i)
                    ch.hist[i] = __shfl_sync(0xffffffffu, xs[kSPL - (W - 1) + i], lane | 2);
#pragma unroll
                for (int i = 0; i < kSPL; i += 2) {
                    float acc[2];
#pragma unroll
                    for (int s1 = 0; s1 < 2; ++s1) {
                        acc[s1] = ch.cbias;
#pragma unroll
                        for (int kk = 0; kk < W; ++kk) {
                            const int j = i + s1 - (W - 1) + kk;
                            acc[s1] = fmaf(ch.w[kk], j >= 0 ? xs[j] : prev[W - 1 + j], acc[s1]);
                        }
                    }
                    upk(silu_pair<kRcpSteps>(pk(acc[0], acc[1])), uu[i], uu[i + 1]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < kSPL; ++i) uu[i] = xs[i];
            }
            // delta = softplus(dt + dt_bias): e = e^v on the SFU, then log(1 + e)
            // by the alternating series of log1p (remainder < 2^-31 relative
            // for e <= 1/16, where the step of a selective SSM usually lives);
            // only when some lane holds a larger e does the warp take the
            // slow path: v itself above 20, log1pf(e) between
            float dl[kSPL];
#pragma unroll
            for (int i = 0; i < kSPL; i += 2) {
                const u64 v2 = fadd2(pk(dts[i], dts[i + 1]), pk(ch.dbias, ch.dbias));
                upk(v2, dl[i], dl[i + 1]);
            }
            if constexpr (SP) {
                bool big = false;
#pragma unroll
                for (int i = 0; i < kSPL; i += 2) {
                    const u64 e2 = exp2_pair_sfu(fmul2(pk(dl[i], dl[i + 1]), pk(kLog2e, kLog2e)));
                    u64 s2 = ffma2(e2, pk(1.0f / 7.0f, 1.0f / 7.0f), pk(-1.0f / 6.0f, -1.0f / 6.0f));
                    s2 = ffma2(s2, e2, pk(0.2f, 0.2f));
                    s2 = ffma2(s2, e2, pk(-0.25f, -0.25f));
                    s2 = ffma2(s2, e2, pk(1.0f / 3.0f, 1.0f / 3.0f));
                    s2 = ffma2(s2, e2, pk(-0.5f, -0.5f));
                    s2 = ffma2(s2, e2, pk(1.0f, 1.0f));
                    s2 = fmul2(s2, e2);
                    float e0, e1;
                    upk(e2, e0, e1);
                    big |= (e0 > 0.0625f) | (e1 > 0.0625f);
                    upk(s2, dl[i], dl[i + 1]);
                }
                if (__any_sync(0xffffffffu, big)) {
                    // recompute v and e exactly as above for the items past 1/16
#pragma unroll
                    for (int i = 0; i < kSPL; ++i) {
                        const float v = dts[i] + ch.dbias;
                        const float e = ex2_approx(v * kLog2e);
                        if (e > 0.0625f) dl[i] = v > 20.0f ? v : log1pf(e);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kSPL; i += 2) {
                const bool vo = vv[i / 8];
                const float dl0 = vo ? dl[i] : 0.0f, dl1 = vo ? dl[i + 1] : 0.0f;
                sdl += (double)dl0 + (double)dl1;
                const u64 du2 = fmul2(pk(dl0, dl1), pk(uu[i], uu[i + 1]));
                float du0, du1;
                upk(du2, du0, du1);
                // this lane's channel is component (q & 1) of the pair's word
                float2* dw = reinterpret_cast<float2*>(&sm.dd[cp][dd_at(kSPL * ph + i)]) + (q & 1);
                dw[0] = make_float2(dl0, du0);
                dw[2] = make_float2(dl1, du1);  // next step: one word further (i even: same half)
                const u64 Du2 = fmul2(pk(ch.dskip, ch.dskip), pk(uu[i], uu[i + 1]));
                upk(Du2, Du[i], Du[i + 1]);
                if constexpr (HZ) {
                    upk(silu_pair<kRcpSteps>(pk(zs[i], zs[i + 1])), gate[i], gate[i + 1]);
                } else {
                    gate[i] = gate[i + 1] = 1.0f;
                }
            }
        }
        __syncwarp();  // pair rows and (delta, delta*u) words written

        // ---- scan: lane (cp, q) updates state entries 4q..4q+3 of channels
        // 2cp and 2cp+1; its readout partials go to word (step, channel) of yp,
        // component q.  The
        // next step's (delta, delta*u) word and B/C pieces are loaded before
        // this step's partials are stored, so that the loads (and the
        // exponentials behind them) are not held back behind the stores.
        {
            float4 d4 = sm.dd[cp][dd_at(0)];  // (dl0, du0, dl1, du1)
            float4 bq = *reinterpret_cast<const float4*>(&sm.bf[0][4 * q]);
            float4 cq = *reinterpret_cast<const float4*>(&sm.cf[0][4 * q]);
#pragma unroll 2
            for (int tt = 0; tt < kT; tt += 4) {
                float yv[2][4];
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int t = tt + s4;
                    const int tn = t + 1 < kT ? t + 1 : t;
                    const float4 d4n = sm.dd[cp][dd_at(tn)];
                    const float4 bqn = *reinterpret_cast<const float4*>(&sm.bf[tn][4 * q]);
                    const float4 cqn = *reinterpret_cast<const float4*>(&sm.cf[tn][4 * q]);
                    u64 Bp[2], Cp[2];
                    bc4(reinterpret_cast<const float*>(&bq), Bp);
                    bc4(reinterpret_cast<const float*>(&cq), Cp);
                    const float dls[2] = {d4.x, d4.z}, dus[2] = {d4.y, d4.w};
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const u64 dl2 = pk(dls[c], dls[c]), du2 = pk(dus[c], dus[c]);
                        const u64 x0 = fmul2(dl2, A2[c][0]), x1 = fmul2(dl2, A2[c][1]);
                        const int sidx = (t & 1) * 4 + 2 * c;  // exponential pair index within 2 steps
                        const u64 a0 = (sidx < SW) ? exp2_pair_fma(x0) : exp2_pair_sfu(x0);
                        const u64 a1 = (sidx + 1 < SW) ? exp2_pair_fma(x1) : exp2_pair_sfu(x1);
                        h2[c][0] = ffma2(a0, h2[c][0], fmul2(du2, Bp[0]));
                        h2[c][1] = ffma2(a1, h2[c][1], fmul2(du2, Bp[1]));
                        const u64 y2 = ffma2(Cp[1], h2[c][1], fmul2(Cp[0], h2[c][0]));
                        float lo, hi;
                        upk(y2, lo, hi);
                        yv[c][s4] = lo + hi;
                    }
                    d4 = d4n;
                    bq = bqn;
                    cq = cqn;
                }
                // the group's partials, stored after the next group's first
                // operands were loaded
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    reinterpret_cast<float*>(&sm.yp[yp_at(tt + s4, 2 * cp)])[q] = yv[0][s4];
                    reinterpret_cast<float*>(&sm.yp[yp_at(tt + s4, 2 * cp + 1)])[q] = yv[1][s4];
                }
            }
        }
        __syncwarp();

        // ---- epilogue: sum the four partials, D skip, gate; store steps
        // 16ph .. 16ph+15 of channel pc
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            if (vv[v] && store_out) {
                float o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 y4 = sm.yp[yp_at(kSPL * ph + 8 * v + i, pc)];
                    o[i] = ((y4.x + y4.y) + (y4.z + y4.w) + Du[8 * v + i]) * gate[8 * v + i];
                }
                store8<IoT>(porow + tl + 8 * v, o);
            }
        }

        // ---- end of a segment: hand the state over, or write the final caches
        if (k + 1 == k1) {
            // the channel's sum of delta over the piece so far (both halves)
            const float sdl_ch = (float)(sdl + __shfl_xor_sync(0xffffffffu, sdl, 2));
            if (kind == 2) {
                float* slot = bp.ws_slots + w * kSlot;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float hv[4];
                    upk(h2[c][0], hv[0], hv[1]);
                    upk(h2[c][1], hv[2], hv[3]);
                    __stcg(reinterpret_cast<float4*>(slot + (2 * cp + c) * 16 + 4 * q),
                           make_float4(hv[0], hv[1], hv[2], hv[3]));
                }
                if (ph == 0) __stcg(slot + kCH * 16 + pc, sdl_ch);
                __threadfence();
                __syncwarp();
#ifdef SSM_TEST_HOOKS
                if (lane == 0 && (int64_t)w != bp.drop_worker)  // failure test: never published
                    st_release_u32(bp.ws_flags + w, gen + 1u);
#else
                if (lane == 0) st_release_u32(bp.ws_flags + w, gen + 1u);
#endif
            } else if (bp.cp_pass == 1) {
                // the piece's end state and sum of delta, for pass 2
                const int64_t rec = ub * (bp.cp_pieces - 1) + piece;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float hv[4];
                    upk(h2[c][0], hv[0], hv[1]);
                    upk(h2[c][1], hv[2], hv[3]);
                    __stcg(reinterpret_cast<float4*>(bp.carry_h + (rec * kCH + 2 * cp + c) * 16 + 4 * q),
                           make_float4(hv[0], hv[1], hv[2], hv[3]));
                }
                if (ph == 0) __stcg(bp.carry_sdl + rec * kCH + pc, sdl_ch);
            } else if (bp.cp_pass == 0 || piece == bp.cp_pieces - 1) {
                if (p.ssm_state) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float hv[4];
                        upk(h2[c][0], hv[0], hv[1]);
                        upk(h2[c][1], hv[2], hv[3]);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int n = 4 * q + j;
                            if (sok[c] && n < p.N) p.ssm_state[b * p.ss_b + sd[c] * p.ss_d + n * p.ss_n] = hv[j];
                        }
                    }
                }
                if (W > 0 && p.conv_state && pok && ph == 0) {
                    // last W raw inputs (L is a multiple of 8, so L >= 8 >= W)
#pragma unroll
                    for (int kk = 0; kk < W; ++kk)
                        st_f(p.conv_state, b * p.cs_b + pd * p.cs_d + kk * p.cs_k, p.cs_dt,
                             to_f(pxrow[p.L - W + kk]));
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
            setup();
        }
        k = nk;
        buf ^= 1;
    }

    // ---- the last worker to finish advances the workspace generation
    if (bp.ws_head) {
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            const unsigned old = atom_inc_acq_rel(bp.ws_head + 1, (unsigned)(bp.workers - 1));
            if (old == (unsigned)(bp.workers - 1)) atomicAdd(bp.ws_head, 1u);
        }
    }
}

// Per-device, per-instance launch set-up: the dynamic shared-memory limit and
// the CTAs that fit on one SM, queried once and cached.
template <typename IoT, int W, int SW, bool SP, bool HZ> struct BalInstance {
    // 0 = not queried yet, else CTAs per SM + 1 (setting the attribute and
    // querying twice from two threads is harmless: both store the same value)
    static int ctas_per_sm(int dev) {
        static std::atomic<int> cache[kMaxDevices];
        if (dev < 0 || dev >= kMaxDevices) return 0;
        int v = cache[dev].load(std::memory_order_acquire);
        if (v == 0) {
            auto kern = scan_bal_kernel<IoT, W, SW, SP, HZ>;
            const int smem = (int)(kWarps * sizeof(BalSmem<IoT>));
            int n = 0;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * kWarps, smem) != cudaSuccess)
                return 0;  // not cached: a later call retries
            v = n + 1;
            cache[dev].store(v, std::memory_order_release);
        }
        return v - 1;
    }
    static cudaError_t launch(const ScanProblem& p, const BalPlan& bp, cudaStream_t s) {
        auto kern = scan_bal_kernel<IoT, W, SW, SP, HZ>;
        const int smem = (int)(kWarps * sizeof(BalSmem<IoT>));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)bp.grid);
        cfg.blockDim = dim3(32 * kWarps);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = bp.cooperative ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, kern, p, bp);
    }
};

template <typename IoT, int W, int SW, bool SP, bool HZ>
cudaError_t run_instance(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int* ctas, int dev) {
    using I = BalInstance<IoT, W, SW, SP, HZ>;
    if (ctas) {
        *ctas = I::ctas_per_sm(dev);
        return cudaSuccess;
    }
    if (I::ctas_per_sm(dev) <= 0) return cudaErrorInvalidConfiguration;
    return I::launch(p, bp, s);
}

template <typename IoT, int W, int SW>
cudaError_t dispatch_flags(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int* ctas, int dev) {
    const bool sp = p.softplus != 0, hz = p.z != nullptr;
    if (sp && hz) return run_instance<IoT, W, SW, true, true>(p, bp, s, ctas, dev);
    if (sp) return run_instance<IoT, W, SW, true, false>(p, bp, s, ctas, dev);
    if (hz) return run_instance<IoT, W, SW, false, true>(p, bp, s, ctas, dev);
    return run_instance<IoT, W, SW, false, false>(p, bp, s, ctas, dev);
}

template <typename IoT, int W>
cudaError_t dispatch_sw(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int* ctas, int dev) {
    switch (bp.sw) {
        case 0: return dispatch_flags<IoT, W, 0>(p, bp, s, ctas, dev);
        case 1: return dispatch_flags<IoT, W, 1>(p, bp, s, ctas, dev);
        default: return cudaErrorInvalidValue;
    }
}

template <typename IoT>
cudaError_t dispatch_w(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int* ctas, int dev) {
    switch (p.W) {
        case 0: return dispatch_sw<IoT, 0>(p, bp, s, ctas, dev);
        case 4: return dispatch_sw<IoT, 4>(p, bp, s, ctas, dev);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t dispatch(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int* ctas, int dev) {
    switch (p.io_dt) {
        case kF32: return dispatch_w<float>(p, bp, s, ctas, dev);
        case kF16: return dispatch_w<__half>(p, bp, s, ctas, dev);
        case kBF16: return dispatch_w<__nv_bfloat16>(p, bp, s, ctas, dev);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// Allocation-free variant: the hand-over scratch lives in this fixed device
// array instead of a caller-supplied workspace.  It is zero at module load,
// every device that loads the library holds its own copy until the process
// exits, and all calls on a device share it.  Host code may not use the
// array's name as an address (it names a host-side stand-in): the device
// address is obtained with cudaGetSymbolAddress, once per device, with that
// device current.
static __device__ __align__(256) unsigned char g_scan_static_ws[kStaticWorkspaceBytes];

void* scan_static_workspace(int dev) {
    static std::atomic<void*> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    void* ptr = cache[dev].load(std::memory_order_acquire);
    if (ptr) return ptr;
    if (cudaGetSymbolAddress(&ptr, g_scan_static_ws) != cudaSuccess || !ptr) return nullptr;
    cache[dev].store(ptr, std::memory_order_release);
    return ptr;
}

bool scan_bal_supported(const ScanProblem& p) {
    return p.N <= 16 && (p.W == 0 || p.W == 4) && p.L % 8 == 0 && (p.G == 1 || p.ch_per_group % kCH == 0);
}
int scan_bal_channels_per_unit() { return kCH; }
int scan_bal_steps_per_chunk() { return kT; }
int scan_bal_warps_per_cta() { return kWarps; }
int scan_bal_smem_bytes(int io_dt) {
    return kWarps * (int)(io_dt == kF32 ? sizeof(BalSmem<float>) : sizeof(BalSmem<__half>));
}

int scan_bal_ctas_per_sm(const ScanProblem& p, int sw, int dev) {
    BalPlan bp{};
    bp.sw = sw;
    int n = 0;
    if (dispatch(p, bp, nullptr, &n, dev) != cudaSuccess) return 0;
    return n;
}

cudaError_t launch_scan_bal(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int dev) {
    return dispatch(p, bp, s, nullptr, dev);
}

}  // namespace ssm
