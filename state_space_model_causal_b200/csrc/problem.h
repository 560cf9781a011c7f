// problem.h -- normalised problem descriptors passed from the C-ABI layer
// (api.cpp) to the kernel launchers.  Host and device share these PODs; all
// strides are in elements, all offsets are 64-bit.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace ssm {

constexpr int kMaxDevices = 64;  // per-device host caches hold this many devices

// The library's device-side error record (one per device).  code: 0 = none,
// 1 = a bounded wait ran out; kernel: the ssm_kernel_id that reported last;
// first_item: the lowest work item (in the reporting kernel's numbering) that
// did not complete.  Kernels set it with atomics; ssm_device_error_info()
// reads and clears every field with atomic exchanges.
struct DeviceError {
    int code;
    int kernel;
    long long first_item;
};
constexpr long long kNoItem = 0x7fffffffffffffffLL;

// Single-token state update in the normalised (B, H, P, N) form.  A Mamba-1
// problem (d_inner channels) is mapped to H = d_inner heads of headdim P = 1,
// so that channel c = h * P + p and group g = h / (H / G) hold in both layouts.
struct SsuProblem {
    int64_t Bn, H, P, N, G, W;  // W = 0: no fused conv
    int64_t heads_per_group;    // H / G
    void* state;  int state_dt;  int64_t st_b, st_h, st_p, st_n;
    const void* x;  int x_dt;  int64_t x_b, x_h, x_p;
    const void* dt; int dt_dt; int64_t dt_b, dt_h, dt_p;
    const float* A; int64_t A_h, A_p, A_n; int A_full;  // A_full = 0: A[h * A_h] per head
    const void* Bm; int B_dt; int64_t B_b, B_g, B_n;
    const void* Cm; int C_dt; int64_t C_b, C_g, C_n;
    const float* Dp; int64_t D_h, D_p;
    const void* z;  int z_dt;  int64_t z_b, z_h, z_p;
    const float* dt_bias; int64_t db_h, db_p;
    int softplus;
    void* conv_state; int cs_dt; int64_t cs_b, cs_c, cs_w;
    const float* conv_w; int64_t cw_c, cw_w;
    const float* conv_b; int64_t cb_c;
    const int32_t* slot_idx; int64_t si_b;  // NULL: batch row b uses cache slot b
    int64_t n_slots;                        // dim 0 of the caches; other indices are padding
    void* out; int out_dt; int64_t o_b, o_h, o_p;
};

struct SsuPlan {
    int kernel;          // ssm_kernel_id
    int block;           // threads per CTA
    int grid;            // CTAs
    int lpr;             // lanes per state row (vector kernel)
    int cpl;             // 16-byte chunks per lane per row (vector kernel)
    int64_t rows_per_item;
    int64_t items_per_b;
    int64_t n_items;
    int stage_bytes;     // bulk-copy kernel: bytes of one shared-memory stage
    int stages;          // bulk-copy kernel: stages in flight per CTA
    int rpt;             // bulk-copy kernel: rows per thread per item
    int sms;             // SMs of the device (persistent grids)
    int ctas_per_sm;        // bulk-copy head kernel: CTAs per SM (0: as many as fit)
    long long wait_budget;  // bulk-copy kernels: cycles before a wait gives up
    int64_t drop_item;      // failure tests only: work item whose copies are never
                            // started, so its wait runs out (-1: none)
};

// Fused prefill (Mamba-1 layout): x, dt, z, out (B, D, L); B, C (B, G, N, L).
struct ScanProblem {
    int64_t Bn, D, L, N, G, W;  // W = 0: no fused conv (u = x)
    int64_t ch_per_group;       // D / G
    int io_dt;
    const void* x;  int64_t x_b, x_d, x_t;
    const void* dt; int64_t dt_b, dt_d, dt_t;
    const float* A; int64_t A_d, A_n;
    const void* Bm; int64_t B_b, B_g, B_n, B_t;
    const void* Cm; int64_t C_b, C_g, C_n, C_t;
    const float* Dp; int64_t D_d;
    const void* z;  int64_t z_b, z_d, z_t;
    const float* dt_bias; int64_t db_d;
    int softplus;
    const float* conv_w; int64_t cw_d, cw_k;
    const float* conv_b; int64_t cb_d;
    void* conv_state; int cs_dt; int64_t cs_b, cs_d, cs_k;
    float* ssm_state; int64_t ss_b, ss_d, ss_n;
    void* out; int64_t o_b, o_d, o_t;
};

struct ScanPlan {
    int kernel;
    int block;
    int grid;
    int ns;         // threads per channel (chunked kernel)
    int dt_tile;    // channels per CTA
    int t_chunk;    // time steps per smem chunk
    int smem;       // dynamic shared memory bytes
    int sw_pairs;   // vector kernel: state-entry pairs per thread whose exp runs on the FMA pipe
};

// Launch of the load-balanced prefill (scan_bal.cu).  Units are (batch entry,
// 16-channel block) x the whole sequence in 32-step chunks; `workers` warps
// split the flattened (unit, chunk) list into equal contiguous slices.  With
// more units than workers the slices hand states over through the workspace
// (ws_* non-NULL, cooperative launch); otherwise workers == units.
struct BalPlan {
    int64_t units;       // batch entries x channel blocks
    int64_t nblk;        // channel blocks per batch entry
    int64_t nck;         // chunks per unit (ceil(L / 32))
    int64_t workers;     // warps that take work
    int grid;            // CTAs
    int sw;              // exponentials per 8 evaluated on the FMA pipe
    int cooperative;     // all CTAs co-resident (required when slices hand over)
    unsigned* ws_head;   // workspace header: generation, finished-worker count
    unsigned* ws_flags;  // one flag per worker: its hand-over is published
    float* ws_slots;     // one hand-over state per worker (16 x 16 floats)
    DeviceError* err;    // device error record
    long long wait_budget;  // cycles before a hand-over wait gives up
    int64_t drop_worker;    // failure tests only: worker whose hand-over is never
                            // published, so its successor's wait runs out (-1: none)
    // Context-parallel mode (cp_pieces >= 3): every sequence is cut into
    // cp_pieces pieces of piece_chunks chunks; a unit is (batch entry, channel
    // block, piece).  Pass 1 runs pieces 0..S-2 -- piece 0 from the initial
    // state with its outputs, the others from zero states without outputs --
    // and records each piece's end state and per-channel sum of delta.  Pass
    // 2 runs pieces 1..S-1 again from the states composed from those records,
    // with outputs; the last piece writes the final caches.
    int cp_pieces;       // S (0: off)
    int cp_pass;         // 1 or 2
    int64_t base_units;  // batch entries x channel blocks
    int64_t piece_chunks;
    float* carry_h;      // [base unit][piece 0..S-2][16 channels][16 state entries]
    float* carry_sdl;    // [base unit][piece 0..S-2][16 channels]
};

// Prefill in the Mamba-2 layout: x, z, out (Bn, H, P, L); dt (Bn, H, L);
// A, D, dt_bias (H); B, C (Bn, G, N, L); ssm_state (Bn, H, P, N).  Strides in
// elements; head h reads group h / (H / G).
struct ScanM2Problem {
    int64_t Bn, H, P, N, G, L;
    int io_dt;
    const void* x;  int64_t x_b, x_h, x_p, x_t;
    const void* dt; int64_t dt_b, dt_h, dt_t;
    const float* A; int64_t A_h;
    const void* Bm; int64_t B_b, B_g, B_n, B_t;
    const void* Cm; int64_t C_b, C_g, C_n, C_t;
    const float* Dp; int64_t D_h;
    const void* z;  int64_t z_b, z_h, z_p, z_t;
    const float* dt_bias; int64_t db_h;
    int softplus;
    float* ssm_state; int64_t ss_b, ss_h, ss_p, ss_n;
    void* out; int64_t o_b, o_h, o_p, o_t;
};

// Launch of the fast Mamba-2-layout prefill: units are (b, h, row block) over
// the whole sequence in 16-step chunks; `workers` CTAs split the flattened
// (unit, chunk) list into equal slices, handing 32 KB state tiles over
// through the workspace when there are more units than resident CTAs
// (ws_* non-NULL, cooperative launch); otherwise workers == units.
struct M2Plan {
    int64_t units, nblk, nck, workers;
    int grid, cooperative, dev;
    unsigned* ws_head;
    unsigned* ws_flags;
    float* ws_slots;     // one state tile (rows per CTA x dstate floats) per worker
    DeviceError* err;
    long long wait_budget;
};

struct Conv1dProblem {
    int64_t Bn, D, L, W;
    int io_dt;
    const void* x; int64_t x_b, x_d, x_t;
    const float* w; int64_t w_d, w_k;
    const float* bias; int64_t b_d;
    void* conv_state; int cs_dt; int64_t cs_b, cs_d, cs_k;
    int silu;
    void* out; int64_t o_b, o_d, o_t;
};

// Double-gated short causal conv: x, bg, cg, out (Bn, D, L) any strides (the
// vector kernel needs unit channel strides); the rows are cut into nseg
// segments of S steps (S >= W - 1 when nseg > 1).
struct GatedConvProblem {
    int64_t Bn, D, L, W;
    int io_dt;
    const void* x;  int64_t x_b, x_d, x_t;
    const void* bg; int64_t bg_b, bg_d, bg_t;
    const void* cg; int64_t cg_b, cg_d, cg_t;
    const float* w; int64_t w_d, w_k;
    const float* bias; int64_t b_d;
    void* conv_state; int cs_dt; int64_t cs_b, cs_d, cs_k;
    void* out; int64_t o_b, o_d, o_t;
    int64_t S, nseg;
};

// Sum of a sequence piece's delta: dt (Bn, D, L) any strides; out (Bn, D) f32.
struct DeltaSumProblem {
    int64_t Bn, D, L;
    int dt_dt;
    const void* dt; int64_t dt_b, dt_d, dt_t;
    const float* dt_bias; int64_t db_d;
    int softplus;
    float* out; int64_t o_b, o_d;
};

// State entering the next sequence piece: state, h_end (Bn, H, P, N); A
// indexed (H, P, N) by strides (Mamba-1 layout: H channels, P = 1; Mamba-2
// layout: A per head, strides 0 over P and N); S (Bn, H); all f32.
struct CarryFoldProblem {
    int64_t Bn, H, P, N;
    float* state; int64_t s_b, s_h, s_p, s_n;
    const float* A; int64_t A_h, A_p, A_n;
    const float* S; int64_t S_b, S_h;
    const float* h_end; int64_t h_b, h_h, h_p, h_n;
};

struct Conv1dPlan {
    int kernel;
    int block;
    int grid;
    int64_t units_per_row;   // vector kernel: ceil(32-vector blocks per row / conv1d_vec_unroll(io, W))
    int64_t units;           // vector kernel: rows x units_per_row
};
int conv1d_vec_ctas_per_sm();
int conv1d_vec_unroll(int io_dt, int64_t W);  // 32-vector blocks per unit of the vector kernel

cudaError_t launch_ssu(const SsuProblem& p, const SsuPlan& plan, cudaStream_t s);
int ssu_tma_max_stages();
int ssu_row_tma_warps();
int ssu_row_tma_stages();
cudaError_t read_and_clear_device_error(DeviceError* out, cudaStream_t s);
DeviceError* device_error_ptr(int dev);
bool scan_bal_supported(const ScanProblem& p);
int scan_bal_channels_per_unit();
int scan_bal_steps_per_chunk();
int scan_bal_warps_per_cta();
int scan_bal_smem_bytes(int io_dt);
int scan_bal_ctas_per_sm(const ScanProblem& p, int sw, int dev);
// Size of the fixed device array behind ssm_selective_scan_fwd_noalloc, and
// its device address on device `dev` (the current device; NULL on failure).
constexpr unsigned long long kStaticWorkspaceBytes = 2ull << 20;
void* scan_static_workspace(int dev);
cudaError_t launch_scan_bal(const ScanProblem& p, const BalPlan& bp, cudaStream_t s, int dev);
cudaError_t launch_scan(const ScanProblem& p, const ScanPlan& plan, cudaStream_t s);
bool scan_vec_supported(const ScanProblem& p);
int scan_vec_threads();
int scan_vec_channels_per_cta();
cudaError_t launch_scan_vec(const ScanProblem& p, int sw_pairs, cudaStream_t s);
cudaError_t launch_conv1d(const Conv1dProblem& p, const Conv1dPlan& plan, cudaStream_t s);
cudaError_t launch_gated_conv(const GatedConvProblem& p, int kernel, int grid, int block, cudaStream_t s);
int gated_conv_ring_smem_bytes();  // dynamic shared memory of the vector kernel's CTA
int gated_conv_ctas_per_sm();      // CTAs of the vector kernel resident per SM
int gated_conv_block();            // threads per CTA of both kernels
cudaError_t launch_delta_sum(const DeltaSumProblem& p, int grid, int block, cudaStream_t s);
cudaError_t launch_carry_fold(const CarryFoldProblem& p, int grid, int block, cudaStream_t s);
int scan_m2_rows_per_cta(int64_t N);
int scan_m2_threads();
int scan_m2_smem_bytes(int io_dt, int64_t N);
cudaError_t launch_scan_m2(const ScanM2Problem& p, int kernel, const M2Plan& mp, cudaStream_t s);
int scan_m2_ctas_per_sm(const ScanM2Problem& p, int dev);

// Launch preparation, done once and remembered (thread-safe):
//   * per (kernel, device), `attrs(smem)` opts the kernel into `smem` bytes of
//     dynamic shared memory (and any other attribute it needs).  The limit
//     only ever grows -- it is raised when a launch needs more than any
//     before -- so that a launch never meets a limit set for a smaller one;
//   * per (kernel, device, shared memory, block), `occupancy(&n)` gives the
//     CTAs per SM.
// The tables hold far more entries than the library has kernel instances.
template <typename Attrs, typename Occupancy>
cudaError_t prepared_launch(const void* fn, int smem, int block, int* per_sm, Attrs attrs,
                            Occupancy occupancy) {
    struct Limit { const void* fn; int dev, smem; };
    struct Fit { const void* fn; int dev, smem, block, per_sm; };
    static std::mutex mu;
    static Limit limits[1024];
    static Fit fits[1024];
    static int n_limits = 0, n_fits = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(mu);
    int li = -1;
    for (int i = 0; i < n_limits; ++i)
        if (limits[i].fn == fn && limits[i].dev == dev) li = i;
    if (li < 0 || limits[li].smem < smem) {
        e = attrs(smem);
        if (e != cudaSuccess) return e;
        if (li >= 0) limits[li].smem = smem;
        else if (n_limits < 1024) limits[n_limits++] = Limit{fn, dev, smem};
        else return cudaErrorUnknown;  // never: more kernels than the table
    }
    for (int i = 0; i < n_fits; ++i)
        if (fits[i].fn == fn && fits[i].dev == dev && fits[i].smem == smem && fits[i].block == block) {
            *per_sm = fits[i].per_sm;
            return cudaSuccess;
        }
    int v = 0;
    e = occupancy(&v);
    if (e != cudaSuccess) return e;
    *per_sm = v;
    if (n_fits < 1024) fits[n_fits++] = Fit{fn, dev, smem, block, v};
    return cudaSuccess;
}

}  // namespace ssm
