// api.cpp -- the C ABI of libssm_causal.so: argument validation, layout
// normalisation, launch planning and dispatch to the sm_100a kernels.
//
// Everything here runs on the host before any CUDA call: a rejected call
// launches nothing and writes nothing.  The only CUDA calls are the SM-count
// query used for grid sizing (skipped in dry-run mode) and the launches.
#include "../../include/ssm_causal.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "problem.h"

namespace ssm {
int scan_chunked_smem_bytes(int ns);
}

namespace {

using namespace ssm;

constexpr int kDefaultSms = 148;  // B200
constexpr int kMaxN = 256;
constexpr int kMaxConvW = 8;

// ------------------------------------------------------------ tensor checks --
bool present(const ssm_tensor& t) { return t.data != nullptr; }

int esize(int dt) {
    switch (dt) {
        case SSM_F32: return 4;
        case SSM_F16: return 2;
        case SSM_BF16: return 2;
        case SSM_I32: return 4;
        default: return 0;
    }
}

bool is_float(int dt) { return dt == SSM_F32 || dt == SSM_F16 || dt == SSM_BF16; }

// Largest element count and byte span a tensor may describe: far above any
// device memory, low enough that no size, offset or extent computed from the
// tensor overflows int64.
constexpr int64_t kMaxSpan = (int64_t)1 << 56;

// rank, non-negative sizes and strides, element-aligned pointer, element
// count and byte span within kMaxSpan
ssm_status basic(const ssm_tensor& t) {
    if (!t.data) return SSM_ERR_NULL;
    if (t.ndim < 1 || t.ndim > SSM_MAX_DIMS) return SSM_ERR_SHAPE;
    if (esize(t.dtype) == 0) return SSM_ERR_DTYPE;
    for (int i = 0; i < t.ndim; ++i) {
        if (t.shape[i] < 0) return SSM_ERR_SHAPE;
        if (t.stride[i] < 0) return SSM_ERR_STRIDE;
    }
    if (reinterpret_cast<uintptr_t>(t.data) % esize(t.dtype) != 0) return SSM_ERR_STRIDE;
    for (int i = 0; i < t.ndim; ++i)
        if (t.shape[i] == 0) return SSM_OK;  // empty: touches no memory
    int64_t count = 1, last = 0;
    for (int i = 0; i < t.ndim; ++i)
        if (__builtin_mul_overflow(count, t.shape[i], &count) || count > kMaxSpan)
            return SSM_ERR_UNSUPPORTED;
    for (int i = 0; i < t.ndim; ++i) {
        int64_t step = 0;
        if (__builtin_mul_overflow(t.shape[i] - 1, t.stride[i], &step) ||
            __builtin_add_overflow(last, step, &last) || last > kMaxSpan)
            return SSM_ERR_UNSUPPORTED;
    }
    if ((last + 1) * esize(t.dtype) > kMaxSpan) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

ssm_status want_shape(const ssm_tensor& t, int nd, const int64_t* dims) {
    if (t.ndim != nd) return SSM_ERR_SHAPE;
    for (int i = 0; i < nd; ++i)
        if (t.shape[i] != dims[i]) return SSM_ERR_SHAPE;
    return SSM_OK;
}

ssm_status want(const ssm_tensor& t, std::initializer_list<int64_t> dims) {
    return want_shape(t, (int)dims.size(), dims.begin());
}

int64_t numel(const ssm_tensor& t) {
    int64_t n = 1;
    for (int i = 0; i < t.ndim; ++i) n *= t.shape[i];
    return n;
}

// Byte range [lo, hi) the tensor touches (empty tensors touch nothing).
void extent(const ssm_tensor& t, uintptr_t* lo, uintptr_t* hi) {
    const uintptr_t base = reinterpret_cast<uintptr_t>(t.data);
    if (!t.data || numel(t) == 0) {
        *lo = *hi = base;
        return;
    }
    int64_t last = 0;
    for (int i = 0; i < t.ndim; ++i) last += (t.shape[i] - 1) * t.stride[i];
    *lo = base;
    *hi = base + (uintptr_t)((last + 1) * esize(t.dtype));
}

bool overlap(const ssm_tensor& a, const ssm_tensor& b) {
    uintptr_t al, ah, bl, bh;
    extent(a, &al, &ah);
    extent(b, &bl, &bh);
    if (al == ah || bl == bh) return false;
    return al < bh && bl < ah;
}

// An output must not write one address twice: sort the non-trivial dims by
// stride and require each stride to clear the span of the smaller ones.
bool non_overlapping(const ssm_tensor& t) {
    if (numel(t) == 0) return true;  // writes nothing
    int64_t st[SSM_MAX_DIMS], sh[SSM_MAX_DIMS];
    int n = 0;
    for (int i = 0; i < t.ndim; ++i) {
        if (t.shape[i] <= 1) continue;
        st[n] = t.stride[i];
        sh[n] = t.shape[i];
        ++n;
    }
    for (int i = 0; i < n; ++i)
        for (int j = i + 1; j < n; ++j)
            if (st[j] < st[i]) {
                std::swap(st[i], st[j]);
                std::swap(sh[i], sh[j]);
            }
    int64_t span = 1;
    for (int i = 0; i < n; ++i) {
        if (st[i] < span) return false;
        span = st[i] * (sh[i] - 1) + span;
    }
    return true;
}

// stride of dim i, with size-1 dims reading as 0 (never stepped)
int64_t sd(const ssm_tensor& t, int i) { return t.shape[i] == 1 ? 0 : t.stride[i]; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An integer environment switch: only a whole decimal number counts; anything
// else (unset, empty, trailing characters) leaves the caller's default.
bool env_int(const char* name, long long* v) {
    const char* e = std::getenv(name);
    if (!e || !*e) return false;
    char* end = nullptr;
    const long long x = std::strtoll(e, &end, 10);
    if (!end || *end != '\0') return false;
    *v = x;
    return true;
}

// The current device (0 in dry-run mode, which makes no CUDA call).
int current_device(bool dry_run) {
    int dev = 0;
    if (!dry_run && cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    return dev;
}

// SM count of a device, queried once per device (dry-run mode assumes a B200).
int sm_count(bool dry_run, int dev) {
    if (dry_run) return kDefaultSms;
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return kDefaultSms;
    int n = cache[dev].load(std::memory_order_acquire);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return kDefaultSms;
    cache[dev].store(n, std::memory_order_release);
    return n;
}
int sm_count(bool dry_run) { return sm_count(dry_run, current_device(dry_run)); }

// Tuning switches for measurement sweeps, read from the environment once per
// process (never needed in normal use):
//   SSM_SCAN_KERNEL=vec    prefill on the whole-unit kernel instead of the balanced one
//   SSM_SCAN_SW=k          balanced prefill: k of every 8 exponential pairs on the FMA pipe (0..1)
//   SSM_SCAN_SW_PAIRS=k    whole-unit prefill: k of 4 state pairs on the FMA pipe (0..3)
//   SSM_SSU_ROWS_PER_ITEM, SSM_SSU_CTAS_PER_SM   Mamba-2 update launch shape
struct Tuning {
    bool scan_vec = false;
    int scan_sw = 0;
    int scan_vec_sw = 0;
    long long ssu_rows = 0;
    int ssu_ctas = 0;
};

Tuning read_tuning() {
    Tuning t;
    const char* k = std::getenv("SSM_SCAN_KERNEL");
    t.scan_vec = k && std::strcmp(k, "vec") == 0;
    long long v = 0;
    if (env_int("SSM_SCAN_SW", &v) && v >= 0 && v <= 1) t.scan_sw = (int)v;
    if (env_int("SSM_SCAN_SW_PAIRS", &v) && v >= 0 && v <= 3) t.scan_vec_sw = (int)v;
    if (env_int("SSM_SSU_ROWS_PER_ITEM", &v) && v > 0) t.ssu_rows = v;
    if (env_int("SSM_SSU_CTAS_PER_SM", &v) && v > 0 && v <= 32) t.ssu_ctas = (int)v;
    return t;
}

const Tuning& tuning() {
    static const Tuning t = read_tuning();  // thread-safe one-time initialisation
    return t;
}

void fill_info(ssm_launch_info* info, int kernel, int grid, int block, int smem, int64_t rows,
               int64_t items) {
    if (!info) return;
    info->kernel = kernel;
    info->grid = grid;
    info->block = block;
    info->smem_bytes = smem;
    info->rows_per_item = (int32_t)rows;
    info->work_items = items;
}

ssm_status info_ok(const ssm_launch_info* info) {
    if (info && info->struct_size != sizeof(ssm_launch_info)) return SSM_ERR_VERSION;
    return SSM_OK;
}

#define SSM_TRY(expr)                  \
    do {                               \
        ssm_status _s = (expr);        \
        if (_s != SSM_OK) return _s;   \
    } while (0)

// ------------------------------------------------------------------ conv1d --
ssm_status conv1d_impl(const ssm_conv1d_args* a, cudaStream_t stream) {
    if (!a) return SSM_ERR_NULL;
    if (a->struct_size != sizeof(ssm_conv1d_args)) return SSM_ERR_VERSION;
    SSM_TRY(info_ok(a->info));
    SSM_TRY(basic(a->x));
    SSM_TRY(basic(a->weight));
    SSM_TRY(basic(a->out));
    if (a->x.ndim != 3) return SSM_ERR_SHAPE;
    const int64_t B = a->x.shape[0], D = a->x.shape[1], L = a->x.shape[2];
    if (a->weight.ndim != 2 || a->weight.shape[0] != D) return SSM_ERR_SHAPE;
    const int64_t W = a->weight.shape[1];
    if (!is_float(a->x.dtype)) return SSM_ERR_DTYPE;
    if (a->weight.dtype != SSM_F32 || a->out.dtype != a->x.dtype) return SSM_ERR_DTYPE;
    SSM_TRY(want(a->out, {B, D, L}));
    if (W < 1) return SSM_ERR_SHAPE;
    if (W > kMaxConvW) return SSM_ERR_UNSUPPORTED;
    if (present(a->bias)) {
        SSM_TRY(basic(a->bias));
        SSM_TRY(want(a->bias, {D}));
        if (a->bias.dtype != SSM_F32) return SSM_ERR_DTYPE;
    }
    if (present(a->conv_state)) {
        SSM_TRY(basic(a->conv_state));
        SSM_TRY(want(a->conv_state, {B, D, W}));
        if (a->conv_state.dtype != SSM_F32 && a->conv_state.dtype != a->x.dtype) return SSM_ERR_DTYPE;
        if (!non_overlapping(a->conv_state)) return SSM_ERR_STRIDE;
    }
    if (!non_overlapping(a->out)) return SSM_ERR_STRIDE;
    const ssm_tensor* ins[] = {&a->x, &a->weight, &a->bias};
    for (const ssm_tensor* t : ins) {
        if (overlap(a->out, *t)) return SSM_ERR_ALIAS;
        if (present(a->conv_state) && overlap(a->conv_state, *t)) return SSM_ERR_ALIAS;
    }
    if (present(a->conv_state) && overlap(a->out, a->conv_state)) return SSM_ERR_ALIAS;

    Conv1dProblem p{};
    p.Bn = B; p.D = D; p.L = L; p.W = W; p.io_dt = a->x.dtype;
    p.x = a->x.data; p.x_b = sd(a->x, 0); p.x_d = sd(a->x, 1); p.x_t = sd(a->x, 2);
    p.w = static_cast<const float*>(a->weight.data); p.w_d = sd(a->weight, 0); p.w_k = sd(a->weight, 1);
    p.bias = static_cast<const float*>(a->bias.data);
    p.b_d = present(a->bias) ? sd(a->bias, 0) : 0;
    p.conv_state = a->conv_state.data;
    if (present(a->conv_state)) {
        p.cs_dt = a->conv_state.dtype;
        p.cs_b = sd(a->conv_state, 0); p.cs_d = sd(a->conv_state, 1); p.cs_k = sd(a->conv_state, 2);
    }
    p.silu = a->silu != 0;
    p.out = a->out.data; p.o_b = sd(a->out, 0); p.o_d = sd(a->out, 1); p.o_t = sd(a->out, 2);

    Conv1dPlan plan{};
    const int64_t rows = B * D;
    const bool empty = rows == 0 || (L == 0 && !present(a->conv_state));
    // L == 0 with a conv state: the state is unchanged, nothing to do
    if (empty || L == 0) {
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }
    // the vector kernel: time-contiguous, 16-byte aligned rows, L a multiple
    // of V, the history within one lane below
    const int es = esize(p.io_dt);
    const int V = 16 / es;
    bool vec = L % V == 0 && W - 1 <= V;
    for (const ssm_tensor* t : {&a->x, &a->out})
        vec = vec && t->stride[2] == 1 && aligned16(t->data) && (sd(*t, 0) * es) % 16 == 0 &&
              (sd(*t, 1) * es) % 16 == 0;
    if (vec) {
        // units of U 32-vector blocks of a row (U = 8 or 4 by dtype and
        // width); persistent CTAs of 8 warps
        const bool dry = (a->flags & SSM_FLAG_DRY_RUN) != 0;
        const int U = conv1d_vec_unroll(p.io_dt, W);
        const int64_t nb = (L + 32 * V - 1) / (32 * V);
        const int64_t nbs = (nb + U - 1) / U;
        const int64_t units = rows * nbs;
        const int64_t grid = std::min<int64_t>((units + 7) / 8, (int64_t)sm_count(dry) * conv1d_vec_ctas_per_sm());
        plan.kernel = SSM_KERNEL_CONV1D;
        plan.block = 256;
        plan.grid = (int)grid;
        plan.units_per_row = nbs;
        plan.units = units;
        fill_info(a->info, plan.kernel, plan.grid, plan.block, 0, 1, units);
        if (dry) return SSM_OK;
        return launch_conv1d(p, plan, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    plan.kernel = SSM_KERNEL_CONV1D_GENERIC;
    plan.block = 128;
    const int64_t grid = (rows + 3) / 4;
    if (grid > INT32_MAX) return SSM_ERR_UNSUPPORTED;
    plan.grid = (int)grid;
    fill_info(a->info, plan.kernel, plan.grid, plan.block, 0, 1, rows);
    if (a->flags & SSM_FLAG_DRY_RUN) return SSM_OK;
    return launch_conv1d(p, plan, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// --------------------------------------------------------- sequence pieces --
ssm_status delta_sum_impl(const ssm_delta_sum_args* a, cudaStream_t stream) {
    if (!a) return SSM_ERR_NULL;
    if (a->struct_size != sizeof(ssm_delta_sum_args)) return SSM_ERR_VERSION;
    SSM_TRY(info_ok(a->info));
    SSM_TRY(basic(a->dt));
    SSM_TRY(basic(a->out));
    if (a->dt.ndim != 3) return SSM_ERR_SHAPE;
    const int64_t B = a->dt.shape[0], D = a->dt.shape[1], L = a->dt.shape[2];
    if (!is_float(a->dt.dtype) || a->out.dtype != SSM_F32) return SSM_ERR_DTYPE;
    SSM_TRY(want(a->out, {B, D}));
    if (!non_overlapping(a->out)) return SSM_ERR_STRIDE;
    if (present(a->dt_bias)) {
        SSM_TRY(basic(a->dt_bias));
        SSM_TRY(want(a->dt_bias, {D}));
        if (a->dt_bias.dtype != SSM_F32) return SSM_ERR_DTYPE;
    }
    if (overlap(a->out, a->dt) || overlap(a->out, a->dt_bias)) return SSM_ERR_ALIAS;
    const int64_t rows = B * D;
    if (rows == 0) {
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }
    constexpr int kBlock = 256;
    const int64_t grid = (rows + kBlock / 32 - 1) / (kBlock / 32);  // one warp per row
    if (grid > INT32_MAX) return SSM_ERR_UNSUPPORTED;
    fill_info(a->info, SSM_KERNEL_DELTA_SUM, (int)grid, kBlock, 0, 1, rows);
    if (a->flags & SSM_FLAG_DRY_RUN) return SSM_OK;
    DeltaSumProblem p{};
    p.Bn = B; p.D = D; p.L = L; p.dt_dt = a->dt.dtype;
    p.dt = a->dt.data; p.dt_b = sd(a->dt, 0); p.dt_d = sd(a->dt, 1); p.dt_t = sd(a->dt, 2);
    p.dt_bias = static_cast<const float*>(a->dt_bias.data);
    p.db_d = present(a->dt_bias) ? sd(a->dt_bias, 0) : 0;
    p.softplus = a->dt_softplus != 0;
    p.out = static_cast<float*>(a->out.data); p.o_b = sd(a->out, 0); p.o_d = sd(a->out, 1);
    return launch_delta_sum(p, (int)grid, kBlock, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status carry_fold_impl(const ssm_carry_fold_args* a, cudaStream_t stream) {
    if (!a) return SSM_ERR_NULL;
    if (a->struct_size != sizeof(ssm_carry_fold_args)) return SSM_ERR_VERSION;
    SSM_TRY(info_ok(a->info));
    SSM_TRY(basic(a->state));
    SSM_TRY(basic(a->A));
    SSM_TRY(basic(a->delta_sum));
    SSM_TRY(basic(a->h_end));
    CarryFoldProblem p{};
    if (a->state.ndim == 3) {
        // Mamba-1 layout: (B, D, N), A (D, N), S (B, D)
        const int64_t B = a->state.shape[0], D = a->state.shape[1], N = a->state.shape[2];
        SSM_TRY(want(a->A, {D, N}));
        SSM_TRY(want(a->delta_sum, {B, D}));
        SSM_TRY(want(a->h_end, {B, D, N}));
        p.Bn = B; p.H = D; p.P = 1; p.N = N;
        p.s_b = sd(a->state, 0); p.s_h = sd(a->state, 1); p.s_p = 0; p.s_n = sd(a->state, 2);
        p.A_h = sd(a->A, 0); p.A_p = 0; p.A_n = sd(a->A, 1);
        p.h_b = sd(a->h_end, 0); p.h_h = sd(a->h_end, 1); p.h_p = 0; p.h_n = sd(a->h_end, 2);
    } else if (a->state.ndim == 4) {
        // Mamba-2 layout: (B, H, P, N), A (H) per head, S (B, H)
        const int64_t B = a->state.shape[0], H = a->state.shape[1], P = a->state.shape[2],
                      N = a->state.shape[3];
        SSM_TRY(want(a->A, {H}));
        SSM_TRY(want(a->delta_sum, {B, H}));
        SSM_TRY(want(a->h_end, {B, H, P, N}));
        p.Bn = B; p.H = H; p.P = P; p.N = N;
        p.s_b = sd(a->state, 0); p.s_h = sd(a->state, 1); p.s_p = sd(a->state, 2); p.s_n = sd(a->state, 3);
        p.A_h = sd(a->A, 0); p.A_p = 0; p.A_n = 0;
        p.h_b = sd(a->h_end, 0); p.h_h = sd(a->h_end, 1); p.h_p = sd(a->h_end, 2); p.h_n = sd(a->h_end, 3);
    } else {
        return SSM_ERR_SHAPE;
    }
    const ssm_tensor* all[] = {&a->state, &a->A, &a->delta_sum, &a->h_end};
    for (const ssm_tensor* t : all)
        if (t->dtype != SSM_F32) return SSM_ERR_DTYPE;
    if (!non_overlapping(a->state)) return SSM_ERR_STRIDE;
    if (overlap(a->state, a->A) || overlap(a->state, a->delta_sum) || overlap(a->state, a->h_end))
        return SSM_ERR_ALIAS;
    const int64_t total = p.Bn * p.H * p.P * p.N;
    if (total == 0) {
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }
    constexpr int kBlock = 256;
    const bool dry = (a->flags & SSM_FLAG_DRY_RUN) != 0;
    // grid-stride: at most 16 CTAs of 256 threads per SM
    const int64_t grid = std::min<int64_t>((total + kBlock - 1) / kBlock, (int64_t)sm_count(dry) * 16);
    fill_info(a->info, SSM_KERNEL_CARRY_FOLD, (int)grid, kBlock, 0, p.P * p.N, p.Bn * p.H);
    if (dry) return SSM_OK;
    p.state = static_cast<float*>(a->state.data);
    p.A = static_cast<const float*>(a->A.data);
    p.S = static_cast<const float*>(a->delta_sum.data);
    p.S_b = sd(a->delta_sum, 0); p.S_h = sd(a->delta_sum, 1);
    p.h_end = static_cast<const float*>(a->h_end.data);
    return launch_carry_fold(p, (int)grid, kBlock, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// ------------------------------------------------------------ gated conv --
ssm_status gated_conv_impl(const ssm_gated_conv1d_args* a, cudaStream_t stream) {
    if (!a) return SSM_ERR_NULL;
    if (a->struct_size != sizeof(ssm_gated_conv1d_args)) return SSM_ERR_VERSION;
    SSM_TRY(info_ok(a->info));
    SSM_TRY(basic(a->x));
    SSM_TRY(basic(a->b_gate));
    SSM_TRY(basic(a->c_gate));
    SSM_TRY(basic(a->weight));
    SSM_TRY(basic(a->out));
    if (a->x.ndim != 3) return SSM_ERR_SHAPE;
    const int64_t B = a->x.shape[0], D = a->x.shape[1], L = a->x.shape[2];
    SSM_TRY(want(a->b_gate, {B, D, L}));
    SSM_TRY(want(a->c_gate, {B, D, L}));
    SSM_TRY(want(a->out, {B, D, L}));
    if (a->weight.ndim != 2 || a->weight.shape[0] != D) return SSM_ERR_SHAPE;
    const int64_t W = a->weight.shape[1];
    if (W < 1) return SSM_ERR_SHAPE;
    if (W > kMaxConvW) return SSM_ERR_UNSUPPORTED;
    const int io = a->x.dtype;
    if (!is_float(io) || a->b_gate.dtype != io || a->c_gate.dtype != io || a->out.dtype != io)
        return SSM_ERR_DTYPE;
    if (a->weight.dtype != SSM_F32) return SSM_ERR_DTYPE;
    if (present(a->bias)) {
        SSM_TRY(basic(a->bias));
        SSM_TRY(want(a->bias, {D}));
        if (a->bias.dtype != SSM_F32) return SSM_ERR_DTYPE;
    }
    const bool has_cs = present(a->conv_state);
    if (has_cs) {
        SSM_TRY(basic(a->conv_state));
        SSM_TRY(want(a->conv_state, {B, D, W}));
        if (a->conv_state.dtype != SSM_F32 && a->conv_state.dtype != io) return SSM_ERR_DTYPE;
        if (!non_overlapping(a->conv_state)) return SSM_ERR_STRIDE;
    }
    if (!non_overlapping(a->out)) return SSM_ERR_STRIDE;
    const ssm_tensor* ins[] = {&a->x, &a->b_gate, &a->c_gate, &a->weight, &a->bias};
    for (const ssm_tensor* t : ins) {
        if (overlap(a->out, *t)) return SSM_ERR_ALIAS;
        if (has_cs && overlap(a->conv_state, *t)) return SSM_ERR_ALIAS;
    }
    if (has_cs && overlap(a->out, a->conv_state)) return SSM_ERR_ALIAS;
    if (B * D == 0 || L == 0) {  // nothing to compute; a conv state stays as it is
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }

    // the vector kernel: 16-byte vectors of V channels with unit channel stride
    const int es = esize(io);
    const int V = 16 / es;
    bool vec = D % V == 0;
    const ssm_tensor* io_t[] = {&a->x, &a->b_gate, &a->c_gate, &a->out};
    for (const ssm_tensor* t : io_t) {
        vec = vec && t->stride[1] == 1 && aligned16(t->data) && (sd(*t, 0) * es) % 16 == 0 &&
              (sd(*t, 2) * es) % 16 == 0;
    }
    // else the time-contiguous kernel: rows of L contiguous steps, 16-byte
    // aligned, L a multiple of V, the history within one lane below
    bool rows_vec = !vec && L % V == 0 && W - 1 <= V;
    for (const ssm_tensor* t : io_t) {
        rows_vec = rows_vec && t->stride[2] == 1 && aligned16(t->data) && (sd(*t, 0) * es) % 16 == 0 &&
                   (sd(*t, 1) * es) % 16 == 0;
    }
    if (rows_vec) {
        // one warp per (row, segment of whole 32-lane blocks), about 32 warps per SM
        const bool dry_r = (a->flags & SSM_FLAG_DRY_RUN) != 0;
        const int64_t rows = B * D, blk = 32 * (int64_t)V;
        const int64_t want = (int64_t)sm_count(dry_r) * 32;
        int64_t nseg = std::min<int64_t>(std::max<int64_t>((want + rows - 1) / rows, 1), (L + blk - 1) / blk);
        int64_t S = ((L + nseg - 1) / nseg + blk - 1) / blk * blk;
        nseg = (L + S - 1) / S;
        const int block = gated_conv_block();
        const int64_t warps = rows * nseg;
        const int64_t grid = (warps + block / 32 - 1) / (block / 32);
        if (grid > INT32_MAX) return SSM_ERR_UNSUPPORTED;
        fill_info(a->info, SSM_KERNEL_GATED_CONV_ROWS, (int)grid, block, 0, 1, warps);
        if (dry_r) return SSM_OK;
        GatedConvProblem p{};
        p.Bn = B; p.D = D; p.L = L; p.W = W; p.io_dt = io;
        p.x = a->x.data; p.x_b = sd(a->x, 0); p.x_d = sd(a->x, 1); p.x_t = 1;
        p.bg = a->b_gate.data; p.bg_b = sd(a->b_gate, 0); p.bg_d = sd(a->b_gate, 1); p.bg_t = 1;
        p.cg = a->c_gate.data; p.cg_b = sd(a->c_gate, 0); p.cg_d = sd(a->c_gate, 1); p.cg_t = 1;
        p.w = static_cast<const float*>(a->weight.data); p.w_d = sd(a->weight, 0); p.w_k = sd(a->weight, 1);
        p.bias = static_cast<const float*>(a->bias.data);
        p.b_d = present(a->bias) ? sd(a->bias, 0) : 0;
        p.conv_state = a->conv_state.data;
        if (has_cs) {
            p.cs_dt = a->conv_state.dtype;
            p.cs_b = sd(a->conv_state, 0); p.cs_d = sd(a->conv_state, 1); p.cs_k = sd(a->conv_state, 2);
        }
        p.out = a->out.data; p.o_b = sd(a->out, 0); p.o_d = sd(a->out, 1); p.o_t = 1;
        p.S = S; p.nseg = nseg;
        return launch_gated_conv(p, SSM_KERNEL_GATED_CONV_ROWS, (int)grid, block, stream) == cudaSuccess
                   ? SSM_OK : SSM_ERR_CUDA;
    }
    const int64_t nv = vec ? D / V : D;
    // segments of S >= 8 steps (so >= W - 1): as many as make one wave of the
    // vector kernel (2 CTAs of 256 threads per SM), or about 1024 threads per
    // SM for the generic one
    const bool dry = (a->flags & SSM_FLAG_DRY_RUN) != 0;
    const int block = gated_conv_block();
    const int64_t wave = (int64_t)sm_count(dry) * (vec ? gated_conv_ctas_per_sm() * block : 1024);
    // at most L / 8 segments, so that S = ceil(L / nseg) >= 8 >= W - 1: only the
    // first segment of a row reads the incoming state, which its own thread
    // then overwrites
    int64_t nseg = std::min<int64_t>(std::max<int64_t>((wave + B * nv - 1) / (B * nv), 1),
                                     std::max<int64_t>(L / 8, 1));
    int64_t S = L;
    if (nseg > 1) {
        S = (L + nseg - 1) / nseg;
        nseg = (L + S - 1) / S;
    }
    const int64_t threads = B * nv * nseg;
    const int64_t grid = (threads + block - 1) / block;
    if (grid > INT32_MAX) return SSM_ERR_UNSUPPORTED;
    const int kernel = vec ? SSM_KERNEL_GATED_CONV : SSM_KERNEL_GATED_CONV_GENERIC;
    fill_info(a->info, kernel, (int)grid, block, vec ? gated_conv_ring_smem_bytes() : 0, vec ? V : 1, threads);
    if (dry) return SSM_OK;

    GatedConvProblem p{};
    p.Bn = B; p.D = D; p.L = L; p.W = W; p.io_dt = io;
    p.x = a->x.data; p.x_b = sd(a->x, 0); p.x_d = sd(a->x, 1); p.x_t = sd(a->x, 2);
    p.bg = a->b_gate.data; p.bg_b = sd(a->b_gate, 0); p.bg_d = sd(a->b_gate, 1); p.bg_t = sd(a->b_gate, 2);
    p.cg = a->c_gate.data; p.cg_b = sd(a->c_gate, 0); p.cg_d = sd(a->c_gate, 1); p.cg_t = sd(a->c_gate, 2);
    p.w = static_cast<const float*>(a->weight.data); p.w_d = sd(a->weight, 0); p.w_k = sd(a->weight, 1);
    p.bias = static_cast<const float*>(a->bias.data);
    p.b_d = present(a->bias) ? sd(a->bias, 0) : 0;
    p.conv_state = a->conv_state.data;
    if (has_cs) {
        p.cs_dt = a->conv_state.dtype;
        p.cs_b = sd(a->conv_state, 0); p.cs_d = sd(a->conv_state, 1); p.cs_k = sd(a->conv_state, 2);
    }
    p.out = a->out.data; p.o_b = sd(a->out, 0); p.o_d = sd(a->out, 1); p.o_t = sd(a->out, 2);
    p.S = S; p.nseg = nseg;
    return launch_gated_conv(p, kernel, (int)grid, block, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// ------------------------------------------------------------- workspace --
// Balanced prefill workspace: a 256-byte header (generation, finished-worker
// count), one 32-bit flag per worker (rounded up to 256 bytes), then one
// hand-over state of 16 channels x 16 state entries (1 KB) per worker.
constexpr long long kWaitBudget = 4000000000LL;  // cycles (~2 s) before a bounded wait gives up
constexpr long long kMinTestBudget = 10000000LL; // shortest wait a failure test may ask for

// A failure test's wait budget, never below kMinTestBudget.
long long clamp_test_budget(long long v) { return v < kMinTestBudget ? kMinTestBudget : v; }
uint64_t bal_flag_bytes(int64_t workers) { return ((uint64_t)workers * 4 + 255) / 256 * 256; }
// bytes of one hand-over slot: a unit's 16 x 16 state and 16 partial sums of delta
uint64_t bal_slot_bytes() { return (uint64_t)scan_bal_channels_per_unit() * 17 * 4; }
uint64_t bal_workspace_bytes(int64_t workers) {
    return 256 + bal_flag_bytes(workers) + (uint64_t)workers * bal_slot_bytes();
}
// context-parallel records: per (base unit, piece 0..S-2) a 16 x 16 end state
// and 16 sums of delta
uint64_t cp_record_bytes(int64_t base_units, int pieces) {
    return (uint64_t)base_units * (uint64_t)(pieces - 1) * bal_slot_bytes();
}

// Pieces per sequence for the context-parallel prefill: used when the
// sequences alone (base units) would fill fewer than 60% of the resident
// warps.  S - 1 pieces per pass give the warps enough units; a piece is at
// least 2 chunks and the last one is never empty.  0: off.
int cp_pieces(int64_t base_units, int64_t slots, int64_t chunks) {
    if (base_units <= 0 || base_units * 10 >= slots * 6 || chunks < 6) return 0;
    int64_t per_pass = std::min<int64_t>((slots + base_units - 1) / base_units, 15);
    for (; per_pass >= 2; --per_pass) {
        const int64_t S = per_pass + 1;
        const int64_t pc = (chunks + S - 1) / S;
        if (pc >= 2 && (S - 1) * pc < chunks) return (int)S;
    }
    return 0;
}

bool present_ws(const ssm_scan_args* a) { return a->workspace != nullptr && a->workspace_bytes > 0; }

// Does the workspace overlap any tensor of the call?
bool overlaps_any(const ssm_scan_args* a) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(a->workspace);
    const uintptr_t hi = lo + (uintptr_t)a->workspace_bytes;
    const ssm_tensor* all[] = {&a->x, &a->dt, &a->A, &a->B, &a->C, &a->D, &a->z, &a->dt_bias,
                               &a->conv_weight, &a->conv_bias, &a->conv_state, &a->ssm_state, &a->out};
    for (const ssm_tensor* t : all) {
        uintptr_t tl, th;
        extent(*t, &tl, &th);
        if (tl != th && tl < hi && lo < th) return true;
    }
    return false;
}

// -------------------------------------------------------------------- scan --
// Prefill in the Mamba-2 layout (x of rank 4); arguments past the common
// checks of scan_impl.
ssm_status scan_m2_impl(const ssm_scan_args* a, cudaStream_t stream, uint64_t* ws_query) {
    const int64_t Bn = a->x.shape[0], H = a->x.shape[1], P = a->x.shape[2], L = a->x.shape[3];
    const int io = a->x.dtype;
    if (!is_float(io)) return SSM_ERR_DTYPE;
    if (present(a->conv_weight) || present(a->conv_bias) || present(a->conv_state)) return SSM_ERR_UNSUPPORTED;
    if (a->A.dtype != SSM_F32) return SSM_ERR_DTYPE;
    SSM_TRY(want(a->A, {H}));
    for (const ssm_tensor* t : {&a->dt, &a->B, &a->C, &a->out})
        if (t->dtype != io) return SSM_ERR_DTYPE;
    SSM_TRY(want(a->dt, {Bn, H, L}));
    SSM_TRY(want(a->out, {Bn, H, P, L}));
    int64_t G = 1, N = 0;
    int64_t bs[4], cs[4];  // strides of B, C as (b, g, n, t)
    if (a->B.ndim == 4) {
        G = a->B.shape[1];
        N = a->B.shape[2];
        SSM_TRY(want(a->B, {Bn, G, N, L}));
        SSM_TRY(want(a->C, {Bn, G, N, L}));
        for (int i = 0; i < 4; ++i) { bs[i] = sd(a->B, i); cs[i] = sd(a->C, i); }
    } else if (a->B.ndim == 3) {
        N = a->B.shape[1];
        SSM_TRY(want(a->B, {Bn, N, L}));
        SSM_TRY(want(a->C, {Bn, N, L}));
        bs[0] = sd(a->B, 0); bs[1] = 0; bs[2] = sd(a->B, 1); bs[3] = sd(a->B, 2);
        cs[0] = sd(a->C, 0); cs[1] = 0; cs[2] = sd(a->C, 1); cs[3] = sd(a->C, 2);
    } else {
        return SSM_ERR_SHAPE;
    }
    if (G < 1 || (H > 0 && H % G != 0)) return SSM_ERR_SHAPE;
    if (N < 1) return SSM_ERR_SHAPE;
    if (N > kMaxN) return SSM_ERR_UNSUPPORTED;
    for (const ssm_tensor* t : {&a->D, &a->dt_bias}) {
        if (!present(*t)) continue;
        SSM_TRY(basic(*t));
        SSM_TRY(want(*t, {H}));
        if (t->dtype != SSM_F32) return SSM_ERR_DTYPE;
    }
    if (present(a->z)) {
        SSM_TRY(basic(a->z));
        SSM_TRY(want(a->z, {Bn, H, P, L}));
        if (a->z.dtype != io) return SSM_ERR_DTYPE;
    }
    if (present(a->ssm_state)) {
        SSM_TRY(basic(a->ssm_state));
        SSM_TRY(want(a->ssm_state, {Bn, H, P, N}));
        if (a->ssm_state.dtype != SSM_F32) return SSM_ERR_DTYPE;
        if (!non_overlapping(a->ssm_state)) return SSM_ERR_STRIDE;
    }
    if (!non_overlapping(a->out)) return SSM_ERR_STRIDE;
    const ssm_tensor* ins[] = {&a->x, &a->dt, &a->A, &a->B, &a->C, &a->D, &a->z, &a->dt_bias};
    for (const ssm_tensor* o : {&a->out, &a->ssm_state}) {
        if (!present(*o)) continue;
        for (const ssm_tensor* t : ins)
            if (present(*t) && overlap(*o, *t)) return SSM_ERR_ALIAS;
    }
    if (overlap(a->out, a->ssm_state)) return SSM_ERR_ALIAS;

    ScanM2Problem p{};
    p.Bn = Bn; p.H = H; p.P = P; p.N = N; p.G = G; p.L = L;
    p.io_dt = io;
    p.x = a->x.data; p.x_b = sd(a->x, 0); p.x_h = sd(a->x, 1); p.x_p = sd(a->x, 2); p.x_t = sd(a->x, 3);
    p.dt = a->dt.data; p.dt_b = sd(a->dt, 0); p.dt_h = sd(a->dt, 1); p.dt_t = sd(a->dt, 2);
    p.A = static_cast<const float*>(a->A.data); p.A_h = sd(a->A, 0);
    p.Bm = a->B.data; p.B_b = bs[0]; p.B_g = bs[1]; p.B_n = bs[2]; p.B_t = bs[3];
    p.Cm = a->C.data; p.C_b = cs[0]; p.C_g = cs[1]; p.C_n = cs[2]; p.C_t = cs[3];
    p.Dp = static_cast<const float*>(a->D.data); p.D_h = present(a->D) ? sd(a->D, 0) : 0;
    p.z = a->z.data;
    if (present(a->z)) { p.z_b = sd(a->z, 0); p.z_h = sd(a->z, 1); p.z_p = sd(a->z, 2); p.z_t = sd(a->z, 3); }
    p.dt_bias = static_cast<const float*>(a->dt_bias.data); p.db_h = present(a->dt_bias) ? sd(a->dt_bias, 0) : 0;
    p.softplus = a->dt_softplus != 0;
    p.ssm_state = static_cast<float*>(a->ssm_state.data);
    if (present(a->ssm_state)) {
        p.ss_b = sd(a->ssm_state, 0); p.ss_h = sd(a->ssm_state, 1); p.ss_p = sd(a->ssm_state, 2);
        p.ss_n = sd(a->ssm_state, 3);
    }
    p.out = a->out.data; p.o_b = sd(a->out, 0); p.o_h = sd(a->out, 1); p.o_p = sd(a->out, 2); p.o_t = sd(a->out, 3);
    if (present_ws(a) && overlaps_any(a)) return SSM_ERR_ALIAS;
    if (Bn == 0 || H == 0 || P == 0 || L == 0) {  // nothing to compute, caches unchanged
        if (ws_query) {
            *ws_query = 0;
            return SSM_OK;
        }
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }
    const bool dry = (a->flags & SSM_FLAG_DRY_RUN) != 0;
    // fast kernel: headdim / dstate contiguous, 16-byte aligned rows and steps
    const int es = esize(io);
    const int64_t rpc = scan_m2_rows_per_cta(N);
    auto al16 = [](const void* ptr) { return ptr == nullptr || aligned16(ptr); };
    auto m16 = [es](int64_t st) { return (st * es) % 16 == 0; };
    const bool fast = rpc > 0 && P % 8 == 0 && p.x_p == 1 && p.o_p == 1 &&
                      (!p.z || p.z_p == 1) && p.B_n == 1 && p.C_n == 1 &&
                      al16(p.x) && al16(p.out) && al16(p.z) && al16(p.Bm) && al16(p.Cm) &&
                      m16(p.x_b) && m16(p.x_h) && m16(p.x_t) && m16(p.o_b) && m16(p.o_h) && m16(p.o_t) &&
                      (!p.z || (m16(p.z_b) && m16(p.z_h) && m16(p.z_t))) && m16(p.B_b) && m16(p.B_g) &&
                      m16(p.B_t) && m16(p.C_b) && m16(p.C_g) && m16(p.C_t) && H <= 65535 && Bn <= 65535;
    int kernel, grid, block, smem;
    int64_t items;
    M2Plan mp{};
    if (fast) {
        kernel = SSM_KERNEL_SCAN_M2;
        const int64_t blocks = (P + rpc - 1) / rpc;
        if (blocks * H * Bn > INT32_MAX) return SSM_ERR_UNSUPPORTED;
        block = scan_m2_threads();
        smem = scan_m2_smem_bytes(io, N);
        items = blocks * H * Bn;
        // balanced slices when there are more units than resident CTAs
        const int dev = current_device(dry);
        const int per_sm = dry ? std::min(3, (228 * 1024) / (smem + 1024)) : scan_m2_ctas_per_sm(p, dev);
        if (per_sm <= 0) return dry ? SSM_ERR_UNSUPPORTED : SSM_ERR_CUDA;
        const int64_t slots = (int64_t)sm_count(dry, dev) * per_sm;
        mp.units = items;
        mp.nblk = blocks;
        mp.nck = (L + 15) / 16;
        mp.dev = dev;
        const bool split = items > slots;
        const uint64_t tile = (uint64_t)rpc * N * 4;  // one CTA's state tile
        const uint64_t need = split ? 256 + bal_flag_bytes(slots) + (uint64_t)slots * tile : 0;
        if (ws_query) {
            *ws_query = need;
            return SSM_OK;
        }
        if (mp.units > ((int64_t)1 << 40) / std::max<int64_t>(mp.nck, 1)) return SSM_ERR_UNSUPPORTED;
        if (split && a->workspace) {
            if (a->workspace_bytes < need || (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
                return SSM_ERR_WORKSPACE;
            unsigned char* ws = static_cast<unsigned char*>(a->workspace);
            mp.ws_head = reinterpret_cast<unsigned*>(ws);
            mp.ws_flags = reinterpret_cast<unsigned*>(ws + 256);
            mp.ws_slots = reinterpret_cast<float*>(ws + 256 + bal_flag_bytes(slots));
            mp.workers = slots;
            mp.cooperative = 1;
        } else {
            mp.workers = items;  // one whole unit per CTA
        }
        grid = (int)mp.workers;
        mp.grid = grid;
        mp.wait_budget = kWaitBudget;
        if (!dry) {
            mp.err = device_error_ptr(dev);
            if (!mp.err) return SSM_ERR_CUDA;
        }
    } else {
        if (ws_query) {
            *ws_query = 0;
            return SSM_OK;
        }
        kernel = SSM_KERNEL_SCAN_M2_GENERIC;
        const int64_t rows = Bn * H * P;
        if ((rows + 3) / 4 > INT32_MAX) return SSM_ERR_UNSUPPORTED;
        grid = (int)((rows + 3) / 4);
        block = 128;
        smem = 0;
        items = rows;
    }
    fill_info(a->info, kernel, grid, block, smem, fast ? rpc : 1, items);
    if (a->flags & SSM_FLAG_DRY_RUN) return SSM_OK;
    return launch_scan_m2(p, kernel, mp, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status scan_impl(const ssm_scan_args* a, cudaStream_t stream, uint64_t* ws_query) {
    if (!a) return SSM_ERR_NULL;
    if (a->struct_size != sizeof(ssm_scan_args)) return SSM_ERR_VERSION;
    SSM_TRY(info_ok(a->info));
    SSM_TRY(basic(a->x));
    SSM_TRY(basic(a->dt));
    SSM_TRY(basic(a->A));
    SSM_TRY(basic(a->B));
    SSM_TRY(basic(a->C));
    SSM_TRY(basic(a->out));
    if (a->x.ndim == 4) return scan_m2_impl(a, stream, ws_query);
    if (a->x.ndim != 3) return SSM_ERR_SHAPE;
    const int64_t Bn = a->x.shape[0], D = a->x.shape[1], L = a->x.shape[2];
    if (a->A.ndim != 2 || a->A.shape[0] != D) return SSM_ERR_SHAPE;
    const int64_t N = a->A.shape[1];
    const int io = a->x.dtype;
    if (!is_float(io)) return SSM_ERR_DTYPE;
    if (a->A.dtype != SSM_F32) return SSM_ERR_DTYPE;
    for (const ssm_tensor* t : {&a->dt, &a->B, &a->C, &a->out})
        if (t->dtype != io) return SSM_ERR_DTYPE;
    SSM_TRY(want(a->dt, {Bn, D, L}));
    SSM_TRY(want(a->out, {Bn, D, L}));
    int64_t G = 1;
    int64_t bs[4], cs[4];  // strides of B, C as (b, g, n, t)
    if (a->B.ndim == 4) {
        G = a->B.shape[1];
        SSM_TRY(want(a->B, {Bn, G, N, L}));
        SSM_TRY(want(a->C, {Bn, G, N, L}));
        for (int i = 0; i < 4; ++i) { bs[i] = sd(a->B, i); cs[i] = sd(a->C, i); }
    } else if (a->B.ndim == 3) {
        SSM_TRY(want(a->B, {Bn, N, L}));
        SSM_TRY(want(a->C, {Bn, N, L}));
        bs[0] = sd(a->B, 0); bs[1] = 0; bs[2] = sd(a->B, 1); bs[3] = sd(a->B, 2);
        cs[0] = sd(a->C, 0); cs[1] = 0; cs[2] = sd(a->C, 1); cs[3] = sd(a->C, 2);
    } else {
        return SSM_ERR_SHAPE;
    }
    if (G < 1 || (D > 0 && D % G != 0)) return SSM_ERR_SHAPE;
    if (N < 1) return SSM_ERR_SHAPE;
    if (N > kMaxN) return SSM_ERR_UNSUPPORTED;
    const ssm_tensor* opt1[] = {&a->D, &a->dt_bias, &a->conv_bias};
    for (const ssm_tensor* t : opt1) {
        if (!present(*t)) continue;
        SSM_TRY(basic(*t));
        SSM_TRY(want(*t, {D}));
        if (t->dtype != SSM_F32) return SSM_ERR_DTYPE;
    }
    if (present(a->z)) {
        SSM_TRY(basic(a->z));
        SSM_TRY(want(a->z, {Bn, D, L}));
        if (a->z.dtype != io) return SSM_ERR_DTYPE;
    }
    int64_t W = 0;
    if (present(a->conv_weight)) {
        SSM_TRY(basic(a->conv_weight));
        if (a->conv_weight.ndim != 2 || a->conv_weight.shape[0] != D) return SSM_ERR_SHAPE;
        if (a->conv_weight.dtype != SSM_F32) return SSM_ERR_DTYPE;
        W = a->conv_weight.shape[1];
        if (W < 1) return SSM_ERR_SHAPE;
        if (W > kMaxConvW) return SSM_ERR_UNSUPPORTED;
    } else if (present(a->conv_bias) || present(a->conv_state)) {
        return SSM_ERR_NULL;  // conv bias / state without conv weight
    }
    if (present(a->conv_state)) {
        SSM_TRY(basic(a->conv_state));
        SSM_TRY(want(a->conv_state, {Bn, D, W}));
        if (a->conv_state.dtype != SSM_F32 && a->conv_state.dtype != io) return SSM_ERR_DTYPE;
        if (!non_overlapping(a->conv_state)) return SSM_ERR_STRIDE;
    }
    if (present(a->ssm_state)) {
        SSM_TRY(basic(a->ssm_state));
        SSM_TRY(want(a->ssm_state, {Bn, D, N}));
        if (a->ssm_state.dtype != SSM_F32) return SSM_ERR_DTYPE;
        if (!non_overlapping(a->ssm_state)) return SSM_ERR_STRIDE;
    }
    if (!non_overlapping(a->out)) return SSM_ERR_STRIDE;
    const ssm_tensor* ins[] = {&a->x, &a->dt, &a->A, &a->B, &a->C, &a->D, &a->z, &a->dt_bias,
                               &a->conv_weight, &a->conv_bias};
    const ssm_tensor* outs[] = {&a->out, &a->conv_state, &a->ssm_state};
    for (const ssm_tensor* o : outs) {
        if (!present(*o)) continue;
        for (const ssm_tensor* t : ins)
            if (present(*t) && overlap(*o, *t)) return SSM_ERR_ALIAS;
    }
    if (overlap(a->out, a->conv_state) || overlap(a->out, a->ssm_state) ||
        overlap(a->conv_state, a->ssm_state))
        return SSM_ERR_ALIAS;

    ScanProblem p{};
    p.Bn = Bn; p.D = D; p.L = L; p.N = N; p.G = G; p.W = W;
    p.ch_per_group = G > 0 && D > 0 ? D / G : 1;
    p.io_dt = io;
    p.x = a->x.data; p.x_b = sd(a->x, 0); p.x_d = sd(a->x, 1); p.x_t = sd(a->x, 2);
    p.dt = a->dt.data; p.dt_b = sd(a->dt, 0); p.dt_d = sd(a->dt, 1); p.dt_t = sd(a->dt, 2);
    p.A = static_cast<const float*>(a->A.data); p.A_d = sd(a->A, 0); p.A_n = sd(a->A, 1);
    p.Bm = a->B.data; p.B_b = bs[0]; p.B_g = bs[1]; p.B_n = bs[2]; p.B_t = bs[3];
    p.Cm = a->C.data; p.C_b = cs[0]; p.C_g = cs[1]; p.C_n = cs[2]; p.C_t = cs[3];
    p.Dp = static_cast<const float*>(a->D.data); p.D_d = present(a->D) ? sd(a->D, 0) : 0;
    p.z = a->z.data;
    if (present(a->z)) { p.z_b = sd(a->z, 0); p.z_d = sd(a->z, 1); p.z_t = sd(a->z, 2); }
    p.dt_bias = static_cast<const float*>(a->dt_bias.data);
    p.db_d = present(a->dt_bias) ? sd(a->dt_bias, 0) : 0;
    p.softplus = a->dt_softplus != 0;
    if (W > 0) {
        p.conv_w = static_cast<const float*>(a->conv_weight.data);
        p.cw_d = sd(a->conv_weight, 0); p.cw_k = sd(a->conv_weight, 1);
        p.conv_b = static_cast<const float*>(a->conv_bias.data);
        p.cb_d = present(a->conv_bias) ? sd(a->conv_bias, 0) : 0;
        p.conv_state = a->conv_state.data;
        if (present(a->conv_state)) {
            p.cs_dt = a->conv_state.dtype;
            p.cs_b = sd(a->conv_state, 0); p.cs_d = sd(a->conv_state, 1); p.cs_k = sd(a->conv_state, 2);
        }
    }
    p.ssm_state = static_cast<float*>(a->ssm_state.data);
    if (present(a->ssm_state)) {
        p.ss_b = sd(a->ssm_state, 0); p.ss_d = sd(a->ssm_state, 1); p.ss_n = sd(a->ssm_state, 2);
    }
    p.out = a->out.data; p.o_b = sd(a->out, 0); p.o_d = sd(a->out, 1); p.o_t = sd(a->out, 2);

    if (present_ws(a) && overlaps_any(a)) return SSM_ERR_ALIAS;
    if (Bn == 0 || D == 0 || L == 0) {  // nothing to compute, caches unchanged
        if (ws_query) {
            *ws_query = 0;
            return SSM_OK;
        }
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }
    // a workspace query sizes against the live device unless it is a dry run
    const bool dry = (a->flags & SSM_FLAG_DRY_RUN) != 0;
    ScanPlan plan{};
    const int es = esize(io);
    auto al16 = [](const void* ptr) { return ptr == nullptr || aligned16(ptr); };
    auto m16 = [es](int64_t st) { return (st * es) % 16 == 0; };
    const bool vec_layout =
        p.x_t == 1 && p.dt_t == 1 && p.o_t == 1 && p.B_t == 1 && p.C_t == 1 &&
        (!p.z || p.z_t == 1) && al16(p.x) && al16(p.dt) && al16(p.out) && al16(p.Bm) &&
        al16(p.Cm) && al16(p.z) && m16(p.x_b) && m16(p.x_d) && m16(p.dt_b) && m16(p.dt_d) &&
        m16(p.o_b) && m16(p.o_d) && m16(p.B_b) && m16(p.B_g) && m16(p.B_n) && m16(p.C_b) &&
        m16(p.C_g) && m16(p.C_n) && (!p.z || (m16(p.z_b) && m16(p.z_d)));
    if (vec_layout && scan_bal_supported(p) && !tuning().scan_vec) {
        // balanced persistent prefill: equal slices of the (unit, chunk) list
        const int kch = scan_bal_channels_per_unit();
        const int warps = scan_bal_warps_per_cta();
        const int dev = current_device(dry);
        BalPlan bp{};
        bp.nblk = (D + kch - 1) / kch;
        bp.units = Bn * bp.nblk;
        bp.nck = (L + scan_bal_steps_per_chunk() - 1) / scan_bal_steps_per_chunk();
        bp.sw = tuning().scan_sw;
        const int smem = scan_bal_smem_bytes(io);
        // CTAs per SM: the occupancy query when live; in dry-run mode the
        // shared-memory bound (228 KB per SM, 1 KB reserved per CTA), at most
        // the 2 that the register budget allows
        int per_sm = dry ? std::min(2, (228 * 1024) / (smem + 1024)) : scan_bal_ctas_per_sm(p, bp.sw, dev);
        if (per_sm <= 0) return dry ? SSM_ERR_UNSUPPORTED : SSM_ERR_CUDA;
        const int64_t slots = (int64_t)sm_count(dry, dev) * per_sm * warps;
        const int64_t base_units = bp.units;
        // context-parallel mode when the sequences alone leave most warps idle
        const int S = cp_pieces(base_units, slots, bp.nck);
        const int64_t pass_units = S ? base_units * (S - 1) : base_units;
        const bool split = pass_units > slots;
        const uint64_t need = (split || S) ? bal_workspace_bytes(slots) + (S ? cp_record_bytes(base_units, S) : 0) : 0;
        if (ws_query) {
            *ws_query = need;
            return SSM_OK;
        }
        // the slice bounds w * units * chunks / workers stay far inside int64
        if (bp.units > ((int64_t)1 << 40) / std::max<int64_t>(bp.nck, 1)) return SSM_ERR_UNSUPPORTED;
        const bool use_ws = a->workspace && (split || S);
        if (use_ws) {
            if (a->workspace_bytes < need || (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
                return SSM_ERR_WORKSPACE;
            unsigned char* ws = static_cast<unsigned char*>(a->workspace);
            bp.ws_head = reinterpret_cast<unsigned*>(ws);
            bp.ws_flags = reinterpret_cast<unsigned*>(ws + 256);
            bp.ws_slots = reinterpret_cast<float*>(ws + 256 + bal_flag_bytes(slots));
            if (S) {
                bp.cp_pieces = S;
                bp.base_units = base_units;
                bp.piece_chunks = (bp.nck + S - 1) / S;
                bp.nck = bp.piece_chunks;
                bp.units = pass_units;
                bp.carry_h = reinterpret_cast<float*>(ws + bal_workspace_bytes(slots));
                bp.carry_sdl = bp.carry_h + (size_t)base_units * (S - 1) * scan_bal_channels_per_unit() * 16;
            }
            bp.workers = split ? slots : bp.units;
            bp.cooperative = split ? 1 : 0;
        } else {
            bp.workers = bp.units;  // whole units, no hand-over, no pieces
        }
        const int64_t grid = (bp.workers + warps - 1) / warps;
        if (grid > INT32_MAX) return SSM_ERR_UNSUPPORTED;
        bp.grid = (int)grid;
        bp.wait_budget = kWaitBudget;
        bp.drop_worker = -1;
#ifdef SSM_TEST_HOOKS
        // Test build only: a worker whose hand-over is never published, and a
        // shorter wait (never below kMinTestBudget cycles)
        {
            long long v = 0;
            if (env_int("SSM_TEST_WAIT_CYCLES", &v) && v > 0) bp.wait_budget = clamp_test_budget(v);
            if (env_int("SSM_TEST_DROP_WORKER", &v) && v >= 0) bp.drop_worker = v;
        }
#endif
        fill_info(a->info, SSM_KERNEL_SCAN_BAL, bp.grid, 32 * warps, smem, kch, bp.units);
        if (a->flags & SSM_FLAG_DRY_RUN) return SSM_OK;
        bp.err = device_error_ptr(dev);
        if (!bp.err) return SSM_ERR_CUDA;
        if (!bp.cp_pieces) return launch_scan_bal(p, bp, stream, dev) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
        // context-parallel: pass 1 (pieces 0..S-2, records), then pass 2
        // (pieces 1..S-1 from the composed states), in order on the stream
        bp.cp_pass = 1;
        if (launch_scan_bal(p, bp, stream, dev) != cudaSuccess) return SSM_ERR_CUDA;
        bp.cp_pass = 2;
        return launch_scan_bal(p, bp, stream, dev) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    if (vec_layout && scan_vec_supported(p)) {
        if (ws_query) {
            *ws_query = 0;
            return SSM_OK;
        }
        plan.kernel = SSM_KERNEL_SCAN_VEC;
        plan.block = scan_vec_threads();
        const int64_t tiles = (D + scan_vec_channels_per_cta() - 1) / scan_vec_channels_per_cta();
        if (tiles * Bn > INT32_MAX) return SSM_ERR_UNSUPPORTED;
        plan.grid = (int)(tiles * Bn);
        plan.sw_pairs = tuning().scan_vec_sw;
        fill_info(a->info, plan.kernel, plan.grid, plan.block, 0, scan_vec_channels_per_cta(),
                  tiles * Bn);
        if (a->flags & SSM_FLAG_DRY_RUN) return SSM_OK;
        return launch_scan(p, plan, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    if (ws_query) {
        *ws_query = 0;
        return SSM_OK;
    }
    int ns = 1;
    while (ns * 4 < N) ns *= 2;
    const int dtile = 64 / (ns <= 16 ? ns : 16);
    const bool groups_fit = G == 1 || (p.ch_per_group % dtile == 0);
    if (ns <= 16 && groups_fit && Bn <= 65535) {
        plan.kernel = SSM_KERNEL_SCAN_CHUNKED;
        plan.ns = ns;
        plan.dt_tile = dtile;
        plan.t_chunk = 32;
        plan.block = dtile * ns;
        const int64_t grid = ((D + dtile - 1) / dtile) * Bn;
        if (grid > INT32_MAX) return SSM_ERR_UNSUPPORTED;
        plan.grid = (int)grid;
        plan.smem = scan_chunked_smem_bytes(ns);
        fill_info(a->info, plan.kernel, plan.grid, plan.block, plan.smem, dtile,
                  ((D + dtile - 1) / dtile) * Bn);
    } else {
        plan.kernel = SSM_KERNEL_SCAN_GENERIC;
        plan.block = 128;
        const int64_t rows = Bn * D;
        plan.grid = (int)std::min<int64_t>((rows + 127) / 128, (int64_t)sm_count(a->flags & SSM_FLAG_DRY_RUN) * 16);
        fill_info(a->info, plan.kernel, plan.grid, plan.block, 0, 1, rows);
    }
    if (a->flags & SSM_FLAG_DRY_RUN) return SSM_OK;
    return launch_scan(p, plan, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// --------------------------------------------------------------------- ssu --
// Per-head parameter (D, dt_bias): (Hm) or, in the Mamba-2 layout, (H, P).
ssm_status head_param(const ssm_tensor& t, bool m2, int64_t H, int64_t P, int64_t* sh, int64_t* sp) {
    SSM_TRY(basic(t));
    if (t.dtype != SSM_F32) return SSM_ERR_DTYPE;
    if (t.ndim == 1) {
        SSM_TRY(want(t, {H}));
        *sh = sd(t, 0);
        *sp = 0;
        return SSM_OK;
    }
    if (m2 && t.ndim == 2) {
        SSM_TRY(want(t, {H, P}));
        *sh = sd(t, 0);
        *sp = sd(t, 1);
        return SSM_OK;
    }
    return SSM_ERR_SHAPE;
}

ssm_status ssu_impl(const ssm_ssu_args* a, cudaStream_t stream) {
    if (!a) return SSM_ERR_NULL;
    if (a->struct_size != sizeof(ssm_ssu_args)) return SSM_ERR_VERSION;
    SSM_TRY(info_ok(a->info));
    for (const ssm_tensor* t : {&a->state, &a->x, &a->dt, &a->A, &a->B, &a->C, &a->out})
        SSM_TRY(basic(*t));
    const bool m2 = a->state.ndim == 4;
    if (a->state.ndim != 3 && !m2) return SSM_ERR_SHAPE;
    const int64_t slots = a->state.shape[0];
    int64_t H, P, N;
    if (m2) {
        H = a->state.shape[1]; P = a->state.shape[2]; N = a->state.shape[3];
    } else {
        H = a->state.shape[1]; P = 1; N = a->state.shape[2];  // channel = head, headdim 1
    }
    const int64_t Bn = a->x.shape[0];
    if (!is_float(a->state.dtype)) return SSM_ERR_DTYPE;
    for (const ssm_tensor* t : {&a->x, &a->dt, &a->B, &a->C, &a->out})
        if (!is_float(t->dtype)) return SSM_ERR_DTYPE;
    if (a->A.dtype != SSM_F32) return SSM_ERR_DTYPE;

    SsuProblem p{};
    p.Bn = Bn; p.H = H; p.P = P; p.N = N;
    p.n_slots = slots;
    // x / out / z
    auto row3 = [&](const ssm_tensor& t, int64_t* b, int64_t* h, int64_t* pp) -> ssm_status {
        if (m2) {
            SSM_TRY(want(t, {Bn, H, P}));
            *b = sd(t, 0); *h = sd(t, 1); *pp = sd(t, 2);
        } else {
            SSM_TRY(want(t, {Bn, H}));
            *b = sd(t, 0); *h = sd(t, 1); *pp = 0;
        }
        return SSM_OK;
    };
    SSM_TRY(row3(a->x, &p.x_b, &p.x_h, &p.x_p));
    SSM_TRY(row3(a->out, &p.o_b, &p.o_h, &p.o_p));
    if (present(a->z)) {
        SSM_TRY(basic(a->z));
        if (!is_float(a->z.dtype)) return SSM_ERR_DTYPE;
        SSM_TRY(row3(a->z, &p.z_b, &p.z_h, &p.z_p));
        p.z = a->z.data; p.z_dt = a->z.dtype;
    }
    // dt: (B, H) per head/channel, or (B, H, P) per row in the Mamba-2 layout
    if (a->dt.ndim == 2) {
        SSM_TRY(want(a->dt, {Bn, H}));
        p.dt_b = sd(a->dt, 0); p.dt_h = sd(a->dt, 1); p.dt_p = 0;
    } else if (m2 && a->dt.ndim == 3) {
        SSM_TRY(want(a->dt, {Bn, H, P}));
        p.dt_b = sd(a->dt, 0); p.dt_h = sd(a->dt, 1); p.dt_p = sd(a->dt, 2);
    } else {
        return SSM_ERR_SHAPE;
    }
    // A: Mamba-1 (D, N); Mamba-2 (H) or (H, P, N)
    if (!m2) {
        SSM_TRY(want(a->A, {H, N}));
        p.A_full = 1; p.A_h = sd(a->A, 0); p.A_p = 0; p.A_n = sd(a->A, 1);
    } else if (a->A.ndim == 1) {
        SSM_TRY(want(a->A, {H}));
        p.A_full = 0; p.A_h = sd(a->A, 0);
    } else if (a->A.ndim == 3) {
        SSM_TRY(want(a->A, {H, P, N}));
        p.A_h = sd(a->A, 0); p.A_p = sd(a->A, 1); p.A_n = sd(a->A, 2);
        p.A_full = (p.A_p != 0 || p.A_n != 0) ? 1 : 0;  // fully broadcast = one scalar per head
    } else {
        return SSM_ERR_SHAPE;
    }
    // B, C: (B, G, N) or (B, N)
    int64_t G = 1;
    if (a->B.ndim == 3) {
        G = a->B.shape[1];
        SSM_TRY(want(a->B, {Bn, G, N}));
        SSM_TRY(want(a->C, {Bn, G, N}));
        p.B_b = sd(a->B, 0); p.B_g = sd(a->B, 1); p.B_n = sd(a->B, 2);
        p.C_b = sd(a->C, 0); p.C_g = sd(a->C, 1); p.C_n = sd(a->C, 2);
    } else if (a->B.ndim == 2) {
        SSM_TRY(want(a->B, {Bn, N}));
        SSM_TRY(want(a->C, {Bn, N}));
        p.B_b = sd(a->B, 0); p.B_g = 0; p.B_n = sd(a->B, 1);
        p.C_b = sd(a->C, 0); p.C_g = 0; p.C_n = sd(a->C, 1);
    } else {
        return SSM_ERR_SHAPE;
    }
    if (N < 1 || H < 1 || P < 1) return SSM_ERR_SHAPE;
    if (G < 1 || H % G != 0) return SSM_ERR_SHAPE;
    if (N > kMaxN) return SSM_ERR_UNSUPPORTED;
    p.G = G;
    p.heads_per_group = H / G;
    if (present(a->D)) {
        SSM_TRY(head_param(a->D, m2, H, P, &p.D_h, &p.D_p));
        p.Dp = static_cast<const float*>(a->D.data);
    }
    if (present(a->dt_bias)) {
        SSM_TRY(head_param(a->dt_bias, m2, H, P, &p.db_h, &p.db_p));
        p.dt_bias = static_cast<const float*>(a->dt_bias.data);
    }
    // state: (slots, H, P, N) / (slots, D, N)
    p.state = a->state.data; p.state_dt = a->state.dtype;
    p.st_b = sd(a->state, 0);
    if (m2) {
        p.st_h = sd(a->state, 1); p.st_p = sd(a->state, 2); p.st_n = sd(a->state, 3);
    } else {
        p.st_h = sd(a->state, 1); p.st_p = 0; p.st_n = sd(a->state, 2);
    }
    if (!non_overlapping(a->state)) return SSM_ERR_STRIDE;
    // slot indices
    if (present(a->state_batch_indices)) {
        SSM_TRY(basic(a->state_batch_indices));
        if (a->state_batch_indices.dtype != SSM_I32) return SSM_ERR_DTYPE;
        SSM_TRY(want(a->state_batch_indices, {Bn}));
        p.slot_idx = static_cast<const int32_t*>(a->state_batch_indices.data);
        p.si_b = sd(a->state_batch_indices, 0);
    } else if (slots != Bn) {
        return SSM_ERR_SHAPE;
    }
    // conv
    const int64_t Cch = H * P;
    if (present(a->conv_weight)) {
        SSM_TRY(basic(a->conv_weight));
        if (a->conv_weight.ndim != 2 || a->conv_weight.shape[0] != Cch) return SSM_ERR_SHAPE;
        if (a->conv_weight.dtype != SSM_F32) return SSM_ERR_DTYPE;
        const int64_t W = a->conv_weight.shape[1];
        if (W < 1) return SSM_ERR_SHAPE;
        if (W > kMaxConvW) return SSM_ERR_UNSUPPORTED;
        if (!present(a->conv_state)) return SSM_ERR_NULL;
        SSM_TRY(basic(a->conv_state));
        SSM_TRY(want(a->conv_state, {slots, Cch, W}));
        if (!is_float(a->conv_state.dtype)) return SSM_ERR_DTYPE;
        if (!non_overlapping(a->conv_state)) return SSM_ERR_STRIDE;
        p.W = W;
        p.conv_w = static_cast<const float*>(a->conv_weight.data);
        p.cw_c = sd(a->conv_weight, 0); p.cw_w = sd(a->conv_weight, 1);
        p.conv_state = a->conv_state.data; p.cs_dt = a->conv_state.dtype;
        p.cs_b = sd(a->conv_state, 0); p.cs_c = sd(a->conv_state, 1); p.cs_w = sd(a->conv_state, 2);
        if (present(a->conv_bias)) {
            SSM_TRY(basic(a->conv_bias));
            SSM_TRY(want(a->conv_bias, {Cch}));
            if (a->conv_bias.dtype != SSM_F32) return SSM_ERR_DTYPE;
            p.conv_b = static_cast<const float*>(a->conv_bias.data);
            p.cb_c = sd(a->conv_bias, 0);
        }
    } else if (present(a->conv_state) || present(a->conv_bias)) {
        return SSM_ERR_NULL;
    }
    if (!non_overlapping(a->out)) return SSM_ERR_STRIDE;
    // aliasing: outputs vs inputs and vs each other
    const ssm_tensor* ins[] = {&a->x, &a->dt, &a->A, &a->B, &a->C, &a->D, &a->z, &a->dt_bias,
                               &a->conv_weight, &a->conv_bias, &a->state_batch_indices};
    const ssm_tensor* outs[] = {&a->out, &a->state, &a->conv_state};
    for (const ssm_tensor* o : outs) {
        if (!present(*o)) continue;
        for (const ssm_tensor* t : ins)
            if (present(*t) && overlap(*o, *t)) return SSM_ERR_ALIAS;
    }
    if (overlap(a->out, a->state) || overlap(a->out, a->conv_state) ||
        overlap(a->state, a->conv_state))
        return SSM_ERR_ALIAS;
    p.x = a->x.data; p.x_dt = a->x.dtype;
    p.dt = a->dt.data; p.dt_dt = a->dt.dtype;
    p.A = static_cast<const float*>(a->A.data);
    p.Bm = a->B.data; p.B_dt = a->B.dtype;
    p.Cm = a->C.data; p.C_dt = a->C.dtype;
    p.softplus = a->dt_softplus != 0;
    p.out = a->out.data; p.out_dt = a->out.dtype;

    const bool dry = (a->flags & SSM_FLAG_DRY_RUN) != 0;
    const int64_t HP = H * P;
    if (Bn == 0) {
        fill_info(a->info, SSM_KERNEL_NONE, 0, 0, 0, 0, 0);
        return SSM_OK;
    }
    if (HP > INT32_MAX) return SSM_ERR_UNSUPPORTED;

    // ---- plan: streaming kernels when the state rows are 16-byte addressable
    SsuPlan plan{};
    // bulk-copy waits give up after ~2 s of cycles
    plan.wait_budget = kWaitBudget;
    plan.drop_item = -1;
#ifdef SSM_TEST_HOOKS
    // Test build only (libssm_causal_testhooks.so): the failure tests name one
    // work item whose copies are never started, so that its wait runs out,
    // and shorten the wait (never below kMinTestBudget cycles, ~5 ms).
    {
        long long v = 0;
        if (env_int("SSM_TEST_WAIT_CYCLES", &v) && v > 0) plan.wait_budget = clamp_test_budget(v);
        if (env_int("SSM_TEST_DROP_ITEM", &v) && v >= 0) plan.drop_item = v;
    }
#endif
    const int es = esize(p.state_dt);
    const bool vec_rows = p.st_n == 1 && (N * es) % 16 == 0 && aligned16(p.state) &&
                          (p.st_b * es) % 16 == 0 && (p.st_h * es) % 16 == 0 &&
                          (p.st_p * es) % 16 == 0;
    const int64_t cpr = vec_rows ? N * es / 16 : 0;  // 16-byte chunks per row
    const int sms = sm_count(dry);
    const int64_t ctas = (int64_t)sms * (p.A_full || p.W ? 4 : 3);  // resident CTAs of 256 threads
    const int64_t row_bytes = N * es;
    auto pow2 = [](int64_t v) { return v > 0 && (v & (v - 1)) == 0; };
    const bool dense_rows = p.st_p == N || P == 1;
    // one I/O dtype for x, dt, B, C, z, out lets the bulk-copy kernel use typed access
    const int io = p.x_dt;
    const bool one_io = p.dt_dt == io && p.B_dt == io && p.C_dt == io && p.out_dt == io &&
                        (!p.z || p.z_dt == io);
    const int es_io = esize(io);
    const bool x_rows = p.x_p == 1 && aligned16(p.x) && (p.x_b * es_io) % 16 == 0 &&
                        (p.x_h * es_io) % 16 == 0;
    if (vec_rows && dense_rows && !p.A_full && p.W == 0 && one_io && x_rows && P >= 2) {
        // bulk-copy pipeline: items are contiguous row blocks of one head; one
        // 16-byte chunk per lane for 16-bit states of up to 16 chunks keeps B/C
        // in 16 registers; longer 16-bit rows (dstate 256) take two chunks per
        // lane (measured: 8% faster at R = 2048, the same at R = 65536)
        int cpl = 0;
        int64_t lpr = 0;
        const bool one_chunk = es == 2 && cpr <= 16;
        const int order[2] = {one_chunk ? 1 : 2, one_chunk ? 2 : 1};
        for (int c : order) {
            if (cpr % c) continue;
            if (cpr / c <= 32 && pow2(cpr / c)) {
                cpl = c;
                lpr = cpr / c;
                break;
            }
        }
        if (cpl) {
            const int64_t rows_per_pass = 256 / lpr;
            // rows per thread: up to 4 (reduce-scatter needs rpt <= lpr), stage <= 24 KB
            int rpt = 4;
            while (rpt > 1 && (rpt > lpr || rpt * rows_per_pass * row_bytes > 24 * 1024)) rpt /= 2;
            if (cpl == 2 && rpt > 2) rpt = 2;
            const int64_t xalign = 16 / es_io;  // rows per item keep x 16-byte aligned
            int64_t rb = std::min<int64_t>(rpt * rows_per_pass, P);
            rb = std::max<int64_t>(xalign, rb / xalign * xalign);
            // the largest items measured fastest at every effective batch
            // (per-item work dominates; smaller items only add items), so
            // items are split only while there are fewer of them than SMs
            while (rb > xalign && Bn * H * ((P + rb - 1) / rb) < sms)
                rb = std::max<int64_t>(xalign, (rb / 2) / xalign * xalign);
            // tuning switches (sweeps): rows per item, CTAs per SM
            const long long t = tuning().ssu_rows;
            if (t >= xalign && t % xalign == 0 && t <= rpt * rows_per_pass)
                rb = std::min<int64_t>(t, P / xalign * xalign);
            if (tuning().ssu_ctas > 0) plan.ctas_per_sm = tuning().ssu_ctas;
            if (rb <= rpt * rows_per_pass && P % xalign == 0) {
                plan.kernel = SSM_KERNEL_SSU_TMA;
                plan.block = 256;
                plan.lpr = (int)lpr;
                plan.cpl = cpl;
                plan.rpt = rpt;
                plan.rows_per_item = rb;
                plan.items_per_b = H * ((P + rb - 1) / rb);
                plan.n_items = Bn * plan.items_per_b;
                plan.stage_bytes = (int)((rb * row_bytes + rb * es_io + 127) / 128 * 128);
                plan.stages = (int)std::max<int64_t>(
                    2, std::min<int64_t>(ssu_tma_max_stages(), (72 * 1024) / plan.stage_bytes));
            }
        }
    }
    // Mamba-1 layout through bulk copies: channel rows, their conv rows, the
    // x/dt/z slices and the batch row's B/C are contiguous and 16-byte aligned;
    // one thread per row (d_state of at most 4 chunks of 16 bytes)
    if (plan.kernel == 0 && vec_rows && P == 1 && p.A_full && one_io && cpr <= 4 && pow2(cpr) &&
        (p.W == 0 || p.W == 4) && p.st_h == N && p.A_n == 1 && p.A_p == 0 && aligned16(p.A) &&
        (p.A_h * 4) % 16 == 0 && (16 / es) % 4 == 0 && p.G == 1) {
        const int cs_es = p.W ? esize(p.cs_dt) : 4;
        const bool io_ok = p.x_h == 1 && p.dt_h == 1 && (!p.z || p.z_h == 1) && aligned16(p.x) &&
                           aligned16(p.dt) && (!p.z || aligned16(p.z)) && (p.x_b * es_io) % 16 == 0 &&
                           (p.dt_b * es_io) % 16 == 0 && (!p.z || (p.z_b * es_io) % 16 == 0);
        const bool bc_ok = p.B_n == 1 && p.C_n == 1 && aligned16(p.Bm) && aligned16(p.Cm) &&
                           (p.B_b * es_io) % 16 == 0 && (p.C_b * es_io) % 16 == 0 &&
                           (N * es_io) % 16 == 0 && (cpr * 16 / es) % (16 / es_io) == 0;
        const bool cs_ok = p.W == 0 || (p.cs_w == 1 && p.cs_c == p.W && aligned16(p.conv_state) &&
                                        (p.cs_b * cs_es) % 16 == 0);
        // channels % 8 == 0: every copy of a (possibly ragged) last block is a
        // whole number of 16-byte units, so no copy reads past its tensor
        if (io_ok && bc_ok && cs_ok && H % 8 == 0) {
            // items of 32 channels (one per lane), one pipeline per warp
            const int64_t rb = 32;
            plan.kernel = SSM_KERNEL_SSU_ROW_TMA;
            plan.block = 32 * ssu_row_tma_warps();
            plan.lpr = 1;
            plan.cpl = (int)cpr;
            plan.rpt = 1;
            plan.rows_per_item = rb;
            plan.items_per_b = (H + rb - 1) / rb;
            plan.n_items = Bn * plan.items_per_b;
            const int64_t io_bytes = (rb * es_io + 15) / 16 * 16;
            const int64_t cs_bytes = (rb * p.W * cs_es + 15) / 16 * 16;
            const int64_t bc_bytes = (N * es_io + 15) / 16 * 16;
            plan.stage_bytes =
                (int)((rb * row_bytes + cs_bytes + 3 * io_bytes + 2 * bc_bytes + 127) / 128 * 128);
            plan.stages = ssu_row_tma_stages();
        }
    }
    if (plan.kernel == 0 && vec_rows && !p.A_full && p.W == 0) {
        // one decay per head: lanes split each row, per-head work once per item
        int cpl = 0;
        int64_t lpr = 0;
        for (int c : {2, 4, 1}) {
            if (cpr % c) continue;
            if (cpr / c <= 32 && pow2(cpr / c)) {
                cpl = c;
                lpr = cpr / c;
                break;
            }
        }
        if (cpl) {
            plan.kernel = SSM_KERNEL_SSU_VEC;
            plan.block = 256;
            plan.lpr = (int)lpr;
            plan.cpl = cpl;
            // ~32 KB of state per item, halved while the items cannot fill the GPU
            int64_t rb = std::max<int64_t>(1, std::min<int64_t>(P, (32 * 1024) / row_bytes));
            while (rb > 8 && Bn * H * ((P + rb - 1) / rb) < 2 * ctas) rb = (rb + 1) / 2;
            plan.rows_per_item = rb;
            plan.items_per_b = H * ((P + rb - 1) / rb);
            plan.n_items = Bn * plan.items_per_b;
        }
    } else if (plan.kernel == 0 && vec_rows && cpr <= 16 && N <= 64) {
        // a decay per element (and the conv): whole rows per thread when small
        const int cpt = cpr % 4 == 0 ? 4 : (cpr % 2 == 0 ? 2 : 1);
        const int64_t lpr = cpr / cpt;
        const int ve = 16 / es;
        const bool a_vec = p.A_n == 1 && aligned16(p.A) && (p.A_h * 4) % 16 == 0 &&
                           (p.A_p * 4) % 16 == 0 && ve % 4 == 0;
        if (a_vec && pow2(lpr) && lpr <= 32) {
            plan.kernel = SSM_KERNEL_SSU_ROW;
            plan.block = 256;
            plan.lpr = (int)lpr;
            plan.cpl = cpt;
            const int64_t rows_per_pass = plan.block / lpr;
            int64_t rb = std::max<int64_t>(rows_per_pass, (16 * 1024) / row_bytes);
            rb = (rb + rows_per_pass - 1) / rows_per_pass * rows_per_pass;
            while (rb > rows_per_pass && Bn * ((HP + rb - 1) / rb) < 2 * ctas) rb -= rows_per_pass;
            if (G > 1) {
                // an item must not straddle a group: largest divisor of the
                // group's row count not above rb
                const int64_t rg = p.heads_per_group * P;
                int64_t best = 1;
                for (int64_t dv = 1; dv * dv <= rg; ++dv) {
                    if (rg % dv) continue;
                    if (dv <= rb) best = std::max(best, dv);
                    if (rg / dv <= rb) best = std::max(best, rg / dv);
                }
                rb = best;
            }
            plan.rows_per_item = std::min<int64_t>(rb, HP);
            plan.items_per_b = (HP + plan.rows_per_item - 1) / plan.rows_per_item;
            plan.n_items = Bn * plan.items_per_b;
        }
    }
    plan.sms = sms;
    if (plan.kernel == SSM_KERNEL_SSU_ROW_TMA && plan.n_items < (int64_t)1 << 31) {
        // one pipeline per warp; the launcher caps the CTAs at what fits at once
        plan.grid = (int)std::min<int64_t>((plan.n_items + ssu_row_tma_warps() - 1) / ssu_row_tma_warps(),
                                           (int64_t)sms * 5);
    } else if (plan.kernel == SSM_KERNEL_SSU_TMA && plan.n_items < (int64_t)1 << 31) {
        // the launcher caps it at the CTAs that fit at once (occupancy query)
        plan.grid = (int)std::min<int64_t>(plan.n_items, (int64_t)sms * 3);
    } else if (plan.kernel != 0 && plan.n_items < (int64_t)1 << 31) {
        plan.grid = (int)std::min<int64_t>(plan.n_items, ctas);
    } else {
        plan = SsuPlan{};
        plan.sms = sms;
        plan.kernel = SSM_KERNEL_SSU_GENERIC;
        plan.block = 128;
        const int64_t rows = Bn * HP;
        plan.rows_per_item = 1;
        plan.n_items = rows;
        plan.grid = (int)std::min<int64_t>((rows + 127) / 128, (int64_t)sms * 16);
    }
    fill_info(a->info, plan.kernel, plan.grid, plan.block,
              plan.kernel == SSM_KERNEL_SSU_TMA ? plan.stages * plan.stage_bytes
              : plan.kernel == SSM_KERNEL_SSU_ROW_TMA ? ssu_row_tma_warps() * plan.stages * plan.stage_bytes
                                                      : 0,
              plan.rows_per_item, plan.n_items);
    if (dry) return SSM_OK;
    return launch_ssu(p, plan, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace

extern "C" {

ssm_status ssm_causal_conv1d_fwd(const ssm_conv1d_args* args, void* stream) {
    return conv1d_impl(args, static_cast<cudaStream_t>(stream));
}

ssm_status ssm_selective_scan_fwd(const ssm_scan_args* args, void* stream) {
    return scan_impl(args, static_cast<cudaStream_t>(stream), nullptr);
}

ssm_status ssm_selective_scan_fwd_noalloc(const ssm_scan_args* args, void* stream) {
    if (!args) return SSM_ERR_NULL;
    if (args->struct_size != sizeof(ssm_scan_args)) return SSM_ERR_VERSION;
    // the scratch is the library's own fixed array: no caller workspace
    if (args->workspace || args->workspace_bytes) return SSM_ERR_WORKSPACE;
    // The Mamba-2-layout prefill needs no scratch for its results (its
    // hand-overs only balance the GPU, with 32 KB per CTA, more than the
    // array): it runs here with one whole unit per CTA.
    if (args->x.ndim == 4) return scan_impl(args, static_cast<cudaStream_t>(stream), nullptr);
    // check the arguments and size the scratch exactly as the workspace query does
    uint64_t need = 0;
    SSM_TRY(scan_impl(args, static_cast<cudaStream_t>(stream), &need));
    if (need > kStaticWorkspaceBytes) return SSM_ERR_WORKSPACE;
    ssm_scan_args a = *args;
    if (need > 0 && !(args->flags & SSM_FLAG_DRY_RUN)) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
        void* ws = scan_static_workspace(dev);
        if (!ws) return SSM_ERR_CUDA;
        // The array keeps whatever the last call left.  The header and the
        // hand-over flags must start at zero: clear them on the call's stream
        // (the hand-over states behind them are written before they are read).
        const uint64_t flags_max = bal_flag_bytes((int64_t)(kStaticWorkspaceBytes / 1024));
        if (cudaMemsetAsync(ws, 0, 256 + flags_max, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return SSM_ERR_CUDA;
        a.workspace = ws;
        a.workspace_bytes = kStaticWorkspaceBytes;
    }
    return scan_impl(&a, static_cast<cudaStream_t>(stream), nullptr);
}

ssm_status ssm_selective_scan_workspace_size(const ssm_scan_args* args, uint64_t* bytes) {
    if (!bytes) return SSM_ERR_NULL;
    return scan_impl(args, nullptr, bytes);
}

ssm_status ssm_selective_state_update(const ssm_ssu_args* args, void* stream) {
    return ssu_impl(args, static_cast<cudaStream_t>(stream));
}

ssm_status ssm_scan_delta_sum(const ssm_delta_sum_args* args, void* stream) {
    return delta_sum_impl(args, static_cast<cudaStream_t>(stream));
}

ssm_status ssm_scan_carry_fold(const ssm_carry_fold_args* args, void* stream) {
    return carry_fold_impl(args, static_cast<cudaStream_t>(stream));
}

ssm_status ssm_gated_conv1d_fwd(const ssm_gated_conv1d_args* args, void* stream) {
    return gated_conv_impl(args, static_cast<cudaStream_t>(stream));
}

const char* ssm_status_string(int status) {
    switch (status) {
        case SSM_OK: return "SSM_OK";
        case SSM_ERR_NULL: return "SSM_ERR_NULL: a required pointer is NULL";
        case SSM_ERR_SHAPE: return "SSM_ERR_SHAPE: rank or sizes inconsistent";
        case SSM_ERR_DTYPE: return "SSM_ERR_DTYPE: unsupported dtype or dtype combination";
        case SSM_ERR_STRIDE: return "SSM_ERR_STRIDE: negative, overlapping or unaddressable layout";
        case SSM_ERR_UNSUPPORTED: return "SSM_ERR_UNSUPPORTED: outside the implemented range";
        case SSM_ERR_CUDA: return "SSM_ERR_CUDA: the CUDA launch failed";
        case SSM_ERR_INTERNAL: return "SSM_ERR_INTERNAL: library invariant failed";
        case SSM_ERR_VERSION: return "SSM_ERR_VERSION: struct_size does not match the library";
        case SSM_ERR_ALIAS: return "SSM_ERR_ALIAS: an output overlaps an input";
        case SSM_ERR_WORKSPACE: return "SSM_ERR_WORKSPACE: workspace too small or not 256-byte aligned";
        default: return "unknown ssm_status";
    }
}

ssm_status ssm_device_error_info(ssm_device_error_report* report, void* stream) {
    if (!report) return SSM_ERR_NULL;
    if (report->struct_size != sizeof(ssm_device_error_report)) return SSM_ERR_VERSION;
    DeviceError e{};
    if (read_and_clear_device_error(&e, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SSM_ERR_CUDA;
    report->code = e.code;
    report->kernel = e.code ? e.kernel : 0;
    report->first_item = e.code ? e.first_item : -1;
    return SSM_OK;
}

ssm_status ssm_device_error(int* code, void* stream) {
    if (!code) return SSM_ERR_NULL;
    DeviceError e{};
    if (read_and_clear_device_error(&e, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SSM_ERR_CUDA;
    *code = e.code;
    return SSM_OK;
}

long long ssm_test_clamp_wait_budget(long long cycles) { return clamp_test_budget(cycles); }

int ssm_abi_version(void) { return SSM_CAUSAL_ABI_VERSION; }

size_t ssm_struct_size(int which) {
    switch (which) {
        case 0: return sizeof(ssm_tensor);
        case 1: return sizeof(ssm_conv1d_args);
        case 2: return sizeof(ssm_scan_args);
        case 3: return sizeof(ssm_ssu_args);
        case 4: return sizeof(ssm_launch_info);
        case 5: return sizeof(ssm_device_error_report);
        case 6: return sizeof(ssm_delta_sum_args);
        case 7: return sizeof(ssm_carry_fold_args);
        case 8: return sizeof(ssm_gated_conv1d_args);
        default: return 0;
    }
}

}  // extern "C"
