/*
 * ssm_causal.h -- C ABI of libssm_causal.so, the B200 (sm_100a) Mamba hot path.
 *
 * Three operations, each one call:
 *
 *   ssm_causal_conv1d_fwd       depthwise causal conv1d (+ optional SiLU) over a
 *                               sequence, reading and writing the conv-state cache.
 *   ssm_selective_scan_fwd      fused prefill: causal conv1d -> SiLU ->
 *                               Delta = softplus(dt + dt_bias) -> selective scan
 *                               -> D skip -> SiLU(z) gate, state caches in/out.
 *   ssm_selective_state_update  single-token decode update of the state caches,
 *                               Mamba-1 layout (d_inner x d_state, optional fused
 *                               conv-state roll) and Mamba-2 layout (nheads x
 *                               headdim x dstate, scalar A per head, ngroups).
 *
 * Beside them: ssm_scan_delta_sum and ssm_scan_carry_fold join a prefill split
 * along the sequence, and ssm_gated_conv1d_fwd is the double-gated short causal
 * conv of an LFM2-style conv block (prefill or one decode step).
 *
 * Sources.  The operators "causal-conv1d, selective-scan, silu, element-mul"
 * and the Mamba state cache that is read and updated by capturing the conv and
 * scan operators come from "feat(llama.cu): 适配 mamba 模型" (InfiniLM-Rust PR
 * #48), sections 2.1 and 3.1.  The update's argument list and order
 * (state, x, dt, A, B, C, D, z, dt_bias, dt_softplus, out), the Mamba-2 shape
 * (batch, nheads, headdim, dstate, ngroups) and the effective batch
 * batch x nheads come from "[XPU] Add tuned Mamba SSU configs for Intel Arc Pro
 * B70" (vLLM PR #50534 report), sections 实现拆解 (item 2) and 关键源码片段.
 * The pages do not print the equations.  The definitions used are:
 *
 *   conv    xc[t] = bias + sum_{k<W} w[k] * x[t-(W-1)+k]   (x[t<0] from conv_state)
 *   SiLU    silu(v) = v * sigmoid(v)
 *   Delta   delta = softplus(dt + dt_bias)  (dt + dt_bias when dt_softplus == 0)
 *   scan    h[n] = exp(delta * A[n]) * h[n] + delta * B[n] * u
 *   output  y = (sum_n C[n] * h[n] + D * u) * silu(z)   (no gate without z)
 *
 * where u is silu(xc) when the conv is fused and x otherwise.  The conv state
 * of a channel holds its last W raw inputs, oldest first; a decode step rolls
 * it left by one and appends the new input before the dot product.
 *
 * Tensors.  Every tensor is an ssm_tensor: a DEVICE pointer, a dtype, a rank
 * and per-dimension sizes and strides counted in ELEMENTS.  Strides must be
 * >= 0; a stride of 0 broadcasts an input along that dimension (never allowed
 * for outputs or in/out caches).  An optional tensor is absent when its data
 * pointer is NULL (its other fields are then ignored).  A non-empty tensor
 * whose element count or byte span (from its first to its last element)
 * exceeds 2^56 is rejected with SSM_ERR_UNSUPPORTED.  Parameters (A, D,
 * dt_bias, conv weight and bias) are float32.  Arithmetic is float32 in every
 * kernel; 16-bit inputs are widened on load and 16-bit outputs and caches are
 * rounded to nearest even on store.
 *
 * Ownership and threading.  The caller owns every buffer, including the
 * prefill's optional workspace.  The library never allocates or frees device
 * memory, keeps no pointer after a call returns and never synchronises the
 * stream (except ssm_device_error / ssm_device_error_info).  Every entry point
 * is reentrant: the only state the library keeps is the device-side error
 * record that the kernels set when they give up a bounded wait (see
 * ssm_device_error_info) and per-device values it queries once and caches
 * (SM count, occupancy of the prefill kernel, the error record's address).  The environment variables
 * SSM_SCAN_KERNEL, SSM_SCAN_SW, SSM_SCAN_SW_PAIRS, SSM_SSU_ROWS_PER_ITEM and
 * SSM_SSU_CTAS_PER_SM select launch variants for measurement sweeps; they are
 * read once, at the first call, and are never needed in normal use.  Work is
 * enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 * runs asynchronously.
 *
 * Errors.  Every argument is checked before anything is launched; on an error
 * nothing is launched and nothing is written, and the status says which check
 * failed.  SSM_ERR_CUDA means the launch itself reported an error.  No entry
 * point aborts, throws or traps on the device.  Outputs must not overlap any
 * input (SSM_ERR_ALIAS); the in/out caches are updated in place.
 */
#ifndef SSM_CAUSAL_H
#define SSM_CAUSAL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSM_CAUSAL_ABI_VERSION 4
#define SSM_MAX_DIMS 5

typedef enum ssm_dtype {
    SSM_F32 = 0,
    SSM_F16 = 1,
    SSM_BF16 = 2,
    SSM_I32 = 3 /* index tensors only */
} ssm_dtype;

typedef enum ssm_status {
    SSM_OK = 0,
    SSM_ERR_NULL = 1,        /* a required pointer (args, tensor data) is NULL */
    SSM_ERR_SHAPE = 2,       /* rank or sizes inconsistent with the others */
    SSM_ERR_DTYPE = 3,       /* unsupported dtype or dtype combination */
    SSM_ERR_STRIDE = 4,      /* negative stride, zero stride on an output, or a
                                layout the kernels cannot address */
    SSM_ERR_UNSUPPORTED = 5, /* valid but outside the implemented range (e.g.
                                d_state > 256, conv width > 8) */
    SSM_ERR_CUDA = 6,        /* the CUDA launch returned an error */
    SSM_ERR_INTERNAL = 7,    /* a library invariant failed */
    SSM_ERR_VERSION = 8,     /* struct_size does not match this library */
    SSM_ERR_ALIAS = 9,       /* an output overlaps an input */
    SSM_ERR_WORKSPACE = 10   /* the workspace is smaller than required or not
                                256-byte aligned */
} ssm_status;

/* Flags for the `flags` field of every args struct. */
#define SSM_FLAG_DRY_RUN 0x1u /* check arguments and choose the launch, but launch nothing */

typedef struct ssm_tensor {
    void* data;                    /* device pointer; NULL = absent (optional tensors) */
    int32_t dtype;                 /* ssm_dtype */
    int32_t ndim;                  /* rank, 1..SSM_MAX_DIMS */
    int64_t shape[SSM_MAX_DIMS];   /* sizes, >= 0 */
    int64_t stride[SSM_MAX_DIMS];  /* in elements, >= 0 */
} ssm_tensor;

/* Optional report of the launch an entry point chose (filled on SSM_OK, also
 * in dry-run mode).  Set struct_size = sizeof(ssm_launch_info). */
typedef struct ssm_launch_info {
    uint32_t struct_size;
    int32_t kernel;          /* ssm_kernel_id */
    int32_t grid;            /* CTAs launched (0 when there is no work) */
    int32_t block;           /* threads per CTA */
    int32_t smem_bytes;      /* dynamic shared memory per CTA */
    int32_t rows_per_item;   /* state rows (or channels) one work item covers */
    int64_t work_items;      /* independent work items in the problem */
} ssm_launch_info;

typedef enum ssm_kernel_id {
    SSM_KERNEL_NONE = 0,            /* empty problem: nothing launched */
    SSM_KERNEL_CONV1D = 1,          /* conv1d, 16-byte vectors of steps: L contiguous, 16-byte aligned
                                       rows, L a multiple of 8 (16-bit) or 4 (fp32), W - 1 at most that */
    SSM_KERNEL_CONV1D_GENERIC = 2,  /* conv1d, any strides: a warp per row */
    SSM_KERNEL_SCAN_CHUNKED = 3,    /* fused prefill, smem-staged chunks of L */
    SSM_KERNEL_SCAN_GENERIC = 4,    /* fused prefill, any strides / group layout */
    SSM_KERNEL_SSU_VEC = 5,         /* 128-bit streaming state update, one decay per
                                       head (Mamba-2 layout, scalar A, no conv) */
    SSM_KERNEL_SSU_GENERIC = 6,     /* state update, any strides / dstate */
    SSM_KERNEL_SCAN_VEC = 7,        /* fused prefill, 16-byte prefetched loads, packed
                                       f32x2 scan; d_state <= 16, conv width 0 or 4,
                                       time contiguous, L % 8 == 0, 16-byte aligned rows */
    SSM_KERNEL_SSU_ROW = 8,         /* 128-bit state update with a decay per element
                                       (Mamba-1 layout or full A), fused conv roll */
    SSM_KERNEL_SSU_TMA = 9,         /* state update fed by bulk copies (TMA) into
                                       shared-memory stages: one decay per head, dense
                                       rows (Mamba-2 layout, scalar A, no conv) */
    SSM_KERNEL_SSU_ROW_TMA = 10,    /* state update fed by bulk copies: a decay per
                                       element, fused conv roll (Mamba-1 layout) */
    SSM_KERNEL_SCAN_M2 = 11,        /* Mamba-2-layout prefill: register tiles of the
                                       (headdim x dstate) state per head, staged
                                       16-step chunks; headdim and dstate contiguous,
                                       dstate 64, 128 or 256, headdim % 8 == 0 */
    SSM_KERNEL_SCAN_M2_GENERIC = 12, /* Mamba-2-layout prefill, any strides, warp per row */
    SSM_KERNEL_SCAN_BAL = 13,       /* fused prefill, persistent warps that each take an
                                       equal slice of the (16-channel unit, 32-step
                                       chunk) list and hand states over through the
                                       workspace; d_state <= 16, conv width 0 or 4,
                                       time contiguous, L % 8 == 0, 16-byte aligned rows */
    SSM_KERNEL_DELTA_SUM = 14,      /* sum of a sequence piece's delta, warp per (b, d) */
    SSM_KERNEL_CARRY_FOLD = 15,     /* state entering the next sequence piece, elementwise */
    SSM_KERNEL_GATED_CONV = 16,     /* double-gated conv, 16-byte vectors of channels that
                                       are contiguous in memory */
    SSM_KERNEL_GATED_CONV_GENERIC = 17, /* double-gated conv, any strides */
    SSM_KERNEL_GATED_CONV_ROWS = 18 /* double-gated conv, (B, D, L) rows with contiguous time:
                                       16-byte vectors of steps, history by shuffle */
} ssm_kernel_id;

/* ------------------------------------------------------------------------ *
 * ssm_causal_conv1d_fwd
 *
 *   x          (B, D, L)  f32 | f16 | bf16                       input
 *   weight     (D, W)     f32, 1 <= W <= 8                        required
 *   bias       (D)        f32                                     optional
 *   conv_state (B, D, W)  f32 or x's dtype, in/out                optional:
 *              read as the W raw inputs preceding x[:, :, 0] (oldest first),
 *              then overwritten with the last W raw inputs of (state ++ x).
 *              Absent: zeros are used and nothing is written.
 *   silu       nonzero: apply SiLU to the conv output
 *   out        (B, D, L)  x's dtype                               output
 *
 * out[b,d,t] = act(bias[d] + sum_k weight[d,k] * x[b,d,t-(W-1)+k]): the
 * "causal-conv1d" operator of "feat(llama.cu): 适配 mamba 模型" (section 2.1),
 * with the conv-state cache of its section 3.1 read before and written after
 * the sequence.  L = 0 leaves conv_state unchanged.
 *
 * Any strides.  Time-contiguous rows (unit step stride, 16-byte aligned data
 * and row strides for x and out, L a multiple of 8 at 16-bit or 4 at fp32,
 * W - 1 at most that multiple) run on SSM_KERNEL_CONV1D; other layouts on
 * SSM_KERNEL_CONV1D_GENERIC.  out may not overlap x, weight, bias or the
 * state, nor the state x, weight or bias (SSM_ERR_ALIAS); an out or
 * conv_state whose elements overlap one another (a broadcast view) is
 * SSM_ERR_STRIDE.
 * ------------------------------------------------------------------------ */
typedef struct ssm_conv1d_args {
    uint32_t struct_size; /* = sizeof(ssm_conv1d_args) */
    uint32_t flags;       /* SSM_FLAG_* */
    ssm_tensor x;
    ssm_tensor weight;
    ssm_tensor bias;
    ssm_tensor conv_state;
    int32_t silu;
    ssm_tensor out;
    ssm_launch_info* info; /* optional */
} ssm_conv1d_args;

ssm_status ssm_causal_conv1d_fwd(const ssm_conv1d_args* args, void* stream);

/* ------------------------------------------------------------------------ *
 * ssm_selective_scan_fwd -- fused prefill over L tokens (Mamba-1 layout).
 *
 *   x           (B, D, L)            f32 | f16 | bf16    input (raw when the conv is fused)
 *   dt          (B, D, L)            x's dtype
 *   A           (D, N)               f32, 1 <= N <= 256
 *   B, C        (B, G, N, L) or (B, N, L)  x's dtype; channel d reads group d / (D/G)
 *   D           (D)                  f32                 optional (absent = 0)
 *   z           (B, D, L)            x's dtype           optional (absent = no gate)
 *   dt_bias     (D)                  f32                 optional (absent = 0)
 *   dt_softplus nonzero: delta = softplus(dt + dt_bias)
 *   conv_weight (D, W)               f32, 1 <= W <= 8    optional: fuses conv + SiLU
 *   conv_bias   (D)                  f32                 optional
 *   conv_state  (B, D, W)            f32 or x's dtype    optional in/out, only with
 *               conv_weight (as in ssm_causal_conv1d_fwd)
 *   ssm_state   (B, D, N)            f32                 optional in/out: read as h0
 *               and overwritten with the state after the last token.  Absent:
 *               h0 = 0 and the final state is not written.
 *   out         (B, D, L)            x's dtype           output
 *
 * The time dimension (last) of x, dt, z, B, C and out may have any stride; the
 * fast kernel needs it to be 1.  L = 0 leaves every cache unchanged.
 *
 * Mamba-2 layout (x of rank 4): one Delta and one scalar A per head,
 *   x, z, out   (B, H, P, L)         f32 | f16 | bf16    (z optional)
 *   dt          (B, H, L)            x's dtype
 *   A           (H)                  f32
 *   B, C        (B, G, N, L) or (B, N, L)  x's dtype; head h reads group h / (H/G)
 *   D, dt_bias  (H)                  f32, optional
 *   ssm_state   (B, H, P, N)         f32, optional in/out as above
 *   conv_*      must be absent (SSM_ERR_UNSUPPORTED): the Mamba-2 conv runs
 *               over the concatenated x/B/C channels before they are split, as
 *               its own ssm_causal_conv1d_fwd call.
 * For every (b, h, p, t): delta = softplus(dt[b,h,t] + dt_bias[h]);
 * s[n] = exp(delta * A[h]) * s[n] + delta * B[b,g,n,t] * x[b,h,p,t];
 * out = (sum_n C[b,g,n,t] * s[n] + D[h] * x[b,h,p,t]) * silu(z[b,h,p,t]).
 * The fast kernel wants the time-major memory of the Mamba-2 model: P
 * contiguous in x, z and out, N contiguous in B and C (e.g. x stored as
 * (B, L, H, P) and described with the strides of its (B, H, P, L) view),
 * 16-byte aligned rows, P a multiple of 8 and N = 64, 128 or 256.
 * ------------------------------------------------------------------------ */
typedef struct ssm_scan_args {
    uint32_t struct_size; /* = sizeof(ssm_scan_args) */
    uint32_t flags;
    ssm_tensor x;
    ssm_tensor dt;
    ssm_tensor A;
    ssm_tensor B;
    ssm_tensor C;
    ssm_tensor D;
    ssm_tensor z;
    ssm_tensor dt_bias;
    int32_t dt_softplus;
    ssm_tensor conv_weight;
    ssm_tensor conv_bias;
    ssm_tensor conv_state;
    ssm_tensor ssm_state;
    ssm_tensor out;
    ssm_launch_info* info; /* optional */
    void* workspace;          /* optional device scratch, see below */
    uint64_t workspace_bytes; /* its size in bytes */
} ssm_scan_args;

ssm_status ssm_selective_scan_fwd(const ssm_scan_args* args, void* stream);

/* Workspace of the fast prefill.  On a problem with more (batch entry,
 * 16-channel) units than the GPU runs warps at once, the fast kernel splits
 * the work into equal slices per warp; a slice that starts or ends inside a
 * unit hands its running state to the neighbouring warp through `workspace`.
 * With few units (under 60% of the warps) it instead cuts every sequence into
 * pieces scanned in two passes, and the workspace also holds each piece's end
 * state and sum of delta.  The fast Mamba-2-layout prefill likewise splits
 * its (batch, head, row block) units over its CTAs, handing 32 KB state tiles
 * over through the workspace.
 * ssm_selective_scan_workspace_size() returns in *bytes how much workspace a
 * call with these arguments can use on the current device (0 when it needs
 * none); it checks the arguments as ssm_selective_scan_fwd does and launches
 * nothing.  A workspace is a device buffer of at least that size, 256-byte
 * aligned, ZERO-FILLED BEFORE ITS FIRST USE; every call leaves it in a state
 * the next call accepts (a generation counter in its first bytes advances per
 * call), so it is allocated and zeroed once and then reused.  Calls that share
 * a workspace must be ordered on one stream: two that run at the same time
 * race.  workspace == NULL runs the prefill without hand-overs (one whole unit
 * per warp: correct, slower when the units do not divide evenly over the
 * SMs); a workspace smaller than required, or misaligned, is
 * SSM_ERR_WORKSPACE.  Returns SSM_ERR_NULL for a NULL `bytes`. */
ssm_status ssm_selective_scan_workspace_size(const ssm_scan_args* args, uint64_t* bytes);

/* ssm_selective_scan_fwd_noalloc -- the same prefill as ssm_selective_scan_fwd
 * for callers that cannot allocate device memory.  It has no counterpart in
 * the method's description: it exists for callers such as a plugin or
 * custom-operator interface that is handed its input and output tensors but
 * no allocator, or a serving loop that must not allocate once it is running
 * (an allocation there can synchronise the device, fail under memory
 * pressure, or is simply not permitted).  Such callers cannot provide the
 * hand-over workspace of the fast prefill.
 *
 * The call takes the same arguments as ssm_selective_scan_fwd, with workspace
 * NULL and workspace_bytes 0 (else SSM_ERR_WORKSPACE), and computes the same
 * results.  (The Mamba-2-layout prefill, x of rank 4, needs no scratch for
 * its results: it runs here as it does without a workspace.)  The scratch it needs comes from a fixed 2 MiB device array inside
 * the library, which every GPU that loads the library holds until the
 * process exits; a problem that would need more than 2 MiB of scratch is
 * rejected with SSM_ERR_WORKSPACE before anything is launched (the prefill
 * needs 256 bytes + 1 KB and 4 bytes per resident warp: about 1.2 MB on a
 * B200).  It calls no allocating routine: the first call on a device looks
 * up that array's device address (once per device, kept for later calls), so
 * make that first call before any stream capture; every call then clears the
 * array's header and flags with an asynchronous memset on `stream` before
 * the prefill kernel.  All calls on a device share the one array and find it
 * as the previous call left it, so two calls whose work overlaps on the GPU
 * (for example on two streams) race and their results are undefined: order
 * them on one stream. */
ssm_status ssm_selective_scan_fwd_noalloc(const ssm_scan_args* args, void* stream);

/* ------------------------------------------------------------------------ *
 * Sequence pieces: a prefill split along L across calls, devices or ranks
 * (context parallelism; the scan is linear in the sequence length, the
 * long-context point of "feat(llama.cu): 适配 mamba 模型" section 6.1).
 *
 * The scan is a first-order linear recurrence in h, so a sequence cut into
 * consecutive pieces j = 0, 1, ... composes: run piece j from a zero ssm
 * state (conv_state = the raw inputs just before it) with
 * ssm_selective_scan_fwd to get its end state h_end(j), and its sum of steps
 * S(j) with ssm_scan_delta_sum; then the state entering piece j+1 is
 *
 *     h_in(j+1)[b,d,n] = exp(A[d,n] * S(j)[b,d]) * h_in(j)[b,d,n] + h_end(j)[b,d,n]
 *
 * from h_in(0) = the sequence's initial state (ssm_scan_carry_fold applies
 * one such step), and piece j run from h_in(j) gives the whole prefill's
 * outputs over its steps.  In the Mamba-2 layout (x of rank 4) the same holds
 * per head: S(j)[b,h] from dt (B, H, L), and
 * h_in(j+1)[b,h,p,n] = exp(A[h] * S(j)[b,h]) * h_in(j)[b,h,p,n] + h_end(j)[b,h,p,n].
 *
 * ssm_scan_delta_sum
 *   dt          (B, D, L)  f32 | f16 | bf16
 *   dt_bias     (D)        f32, optional (absent = 0)
 *   dt_softplus nonzero: delta = softplus(dt + dt_bias), else dt + dt_bias
 *   out         (B, D)     f32: sum over t of delta, accumulated in double
 *                          (the prefill kernels' delta, rounded once)
 * L = 0 writes zeros.
 *
 * ssm_scan_carry_fold
 *   state       (B, D, N) or (B, H, P, N)  f32, in/out: h_in(j) in, h_in(j+1) out
 *   A           (D, N)    or (H)           f32
 *   delta_sum   (B, D)    or (B, H)        f32: S(j)
 *   h_end       like state                 f32: h_end(j); may not overlap state
 * ------------------------------------------------------------------------ */
typedef struct ssm_delta_sum_args {
    uint32_t struct_size; /* = sizeof(ssm_delta_sum_args) */
    uint32_t flags;       /* SSM_FLAG_* */
    ssm_tensor dt;
    ssm_tensor dt_bias;
    int32_t dt_softplus;
    ssm_tensor out;
    ssm_launch_info* info; /* optional */
} ssm_delta_sum_args;

typedef struct ssm_carry_fold_args {
    uint32_t struct_size; /* = sizeof(ssm_carry_fold_args) */
    uint32_t flags;       /* SSM_FLAG_* */
    ssm_tensor state;
    ssm_tensor A;
    ssm_tensor delta_sum;
    ssm_tensor h_end;
    ssm_launch_info* info; /* optional */
} ssm_carry_fold_args;

ssm_status ssm_scan_delta_sum(const ssm_delta_sum_args* args, void* stream);
ssm_status ssm_scan_carry_fold(const ssm_carry_fold_args* args, void* stream);

/* ------------------------------------------------------------------------ *
 * ssm_gated_conv1d_fwd -- double-gated short causal conv, the convolution of
 * the "double-gated LIV convolution blocks" that "LFM2.5-1.2B-Thinking性能优化
 * CUDA核心编程技巧" (section 2.1) names next to its GQA blocks.  The page
 * prints no equation; the definition taken is two input-dependent gates
 * around a depthwise causal conv, with no activation:
 *
 *   v[b,d,t]   = b_gate[b,d,t] * x[b,d,t]
 *   out[b,d,t] = c_gate[b,d,t] * (bias[d] + sum_{k<W} weight[d,k] * v[b,d,t-(W-1)+k])
 *
 *   x, b_gate, c_gate (B, D, L)  f32 | f16 | bf16, one dtype   inputs
 *   weight     (D, W)     f32, 1 <= W <= 8                      required
 *   bias       (D)        f32                                   optional
 *   conv_state (B, D, W)  f32 or x's dtype, in/out              optional:
 *              read as the W gated inputs v preceding step 0 (oldest first),
 *              then overwritten with the last W entries of (state ++ v).
 *              Absent: zeros are used and nothing is written.
 *   out        (B, D, L)  x's dtype                             output
 *
 * L = 1 with a conv state is one decode step.  L = 0 leaves the state
 * unchanged.  Any strides; the fast kernel (SSM_KERNEL_GATED_CONV) takes the
 * layout a token-major projection writes: x, b_gate, c_gate and out with unit
 * channel stride, D a multiple of 8 (16-bit) or 4 (fp32), 16-byte aligned
 * data pointers, and batch and step strides that keep every 16 bytes aligned
 * (for example the three D-wide slices of one (B, L, 3D) projection output).
 * The time-contiguous layout ((B, D, L) rows with unit step stride, 16-byte
 * aligned rows, L a multiple of 8 at 16-bit or 4 at fp32, W - 1 at most that
 * multiple) runs on SSM_KERNEL_GATED_CONV_ROWS.  Other layouts run on
 * SSM_KERNEL_GATED_CONV_GENERIC.  out may not overlap an
 * input or the state.
 * ------------------------------------------------------------------------ */
typedef struct ssm_gated_conv1d_args {
    uint32_t struct_size; /* = sizeof(ssm_gated_conv1d_args) */
    uint32_t flags;       /* SSM_FLAG_* */
    ssm_tensor x;
    ssm_tensor b_gate;
    ssm_tensor c_gate;
    ssm_tensor weight;
    ssm_tensor bias;
    ssm_tensor conv_state;
    ssm_tensor out;
    ssm_launch_info* info; /* optional */
} ssm_gated_conv1d_args;

ssm_status ssm_gated_conv1d_fwd(const ssm_gated_conv1d_args* args, void* stream);

/* ------------------------------------------------------------------------ *
 * ssm_selective_state_update -- one decode token, caches updated in place.
 *
 * Mamba-1 layout (state rank 3):
 *   state   (B, D, N)        f32 | f16 | bf16   in/out
 *   x, z, out (B, D)         f32 | f16 | bf16   (z optional)
 *   dt      (B, D)
 *   A       (D, N)           f32
 *   B, C    (B, G, N) or (B, N); channel d reads group d / (D/G)
 *   D, dt_bias (D)           f32, optional
 *   conv_weight (D, W), conv_bias (D), conv_state (B, D, W) in/out: optional
 *           fused conv update.  When given, x is the raw input: the channel's
 *           conv state is rolled left by one, x appended, and
 *           u = silu(conv_bias + sum_k conv_weight[k] * conv_state[k]) replaces x.
 *
 * Mamba-2 layout (state rank 4):
 *   state   (B, H, P, N)     f32 | f16 | bf16   in/out
 *   x, z, out (B, H, P)
 *   dt      (B, H) per head, or (B, H, P)
 *   A       (H) scalar per head, or (H, P, N)   f32
 *   B, C    (B, G, N); head h reads group h / (H/G)
 *   D, dt_bias (H) or (H, P) f32, optional
 *   conv_*  as above with D = H*P channels, channel c = h*P + p
 *
 * For every row r = (b, h, p): delta = softplus(dt + dt_bias);
 * state[r, n] = exp(delta * A) * state[r, n] + delta * B[n] * u;
 * out[r] = (sum_n C[n] * state[r, n] + D * u) * silu(z).  The readout uses the
 * float32 updated state before it is rounded into a 16-bit cache.
 *
 * state_batch_indices (B) int32, optional: row b reads and writes cache slot
 * state_batch_indices[b]; state and conv_state then both hold the pool's slot
 * count in dim 0, which may differ from B.  A negative index marks a padding
 * row, which is skipped entirely (its out row is left untouched); an index at
 * or past the slot count is skipped the same way.  Two rows that name the
 * same slot race: that slot's caches and both rows' outputs are then
 * undefined, so a batch names each slot at most once.  Without
 * indices, dim 0 of the caches must equal B.
 * ------------------------------------------------------------------------ */
typedef struct ssm_ssu_args {
    uint32_t struct_size; /* = sizeof(ssm_ssu_args) */
    uint32_t flags;
    ssm_tensor state;
    ssm_tensor x;
    ssm_tensor dt;
    ssm_tensor A;
    ssm_tensor B;
    ssm_tensor C;
    ssm_tensor D;
    ssm_tensor z;
    ssm_tensor dt_bias;
    int32_t dt_softplus;
    ssm_tensor conv_weight;
    ssm_tensor conv_bias;
    ssm_tensor conv_state;
    ssm_tensor state_batch_indices;
    ssm_tensor out;
    ssm_launch_info* info; /* optional */
} ssm_ssu_args;

ssm_status ssm_selective_state_update(const ssm_ssu_args* args, void* stream);

/* Device-side error record.  Every kernel wait that can only end when
 * something else happens (a bulk copy landing in shared memory, a hand-over
 * published by another warp) is bounded; when one runs out the kernel records
 * it here instead of trapping or hanging:
 *
 *   ssm_selective_state_update (bulk-copy kernels SSM_KERNEL_SSU_TMA and
 *     SSM_KERNEL_SSU_ROW_TMA): the CTA or warp that gave up exits; the work
 *     items it had not finished are left as they were (their cache rows not
 *     advanced, their outputs not written), every item it finished before is
 *     complete.  first_item is the lowest work item any giving-up CTA or warp
 *     had not finished; work items are numbered as in ssm_launch_info
 *     (rows_per_item rows each): for SSU_TMA batch-major, then head, then row
 *     block; for SSU_ROW_TMA channel-block-major, then batch row.
 *   ssm_selective_scan_fwd (SSM_KERNEL_SCAN_BAL): a warp that waited in vain
 *     for its predecessor's hand-over scans its piece of that unit from a
 *     zero state instead; first_item is the lowest such unit
 *     (batch * ceil(D / 16) + channel / 16); in the context-parallel mode
 *     it is unit * (pieces - 1) + piece, less 1 in the second pass.  That
 *     unit's later outputs and final state are wrong, all other units are
 *     complete.
 *   ssm_selective_scan_fwd, x of rank 4 (SSM_KERNEL_SCAN_M2): the same for a
 *     CTA that waited in vain for its predecessor's state tile; first_item is
 *     the unit (b * H + h) * ceil(P / rows per CTA) + row block.
 *
 * The record belongs to the CURRENT device: call these with that device
 * current and a stream of that device.  Both wait for the work enqueued on
 * `stream` so far, then read and clear the record in one step on the device
 * (a report landing meanwhile is kept for the next read, never lost).
 * ssm_device_error() stores only the code (0 = none, 1 = a wait ran out) in
 * *code; ssm_device_error_info() fills a report (set its struct_size).  They
 * return SSM_ERR_NULL for a NULL pointer, SSM_ERR_VERSION for a wrong
 * struct_size, SSM_ERR_CUDA if the stream or the copy fails. */
typedef struct ssm_device_error_report {
    uint32_t struct_size; /* = sizeof(ssm_device_error_report) */
    int32_t code;         /* 0 = none, 1 = a bounded wait ran out */
    int32_t kernel;       /* ssm_kernel_id of the last kernel that reported (0: none) */
    int32_t reserved;
    int64_t first_item;   /* lowest unfinished work item as described above (-1: none) */
} ssm_device_error_report;

ssm_status ssm_device_error(int* code, void* stream);
ssm_status ssm_device_error_info(ssm_device_error_report* report, void* stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char* ssm_status_string(int status);

/* SSM_CAUSAL_ABI_VERSION of the loaded library. */
int ssm_abi_version(void);

/* sizeof() of the args structs and of ssm_tensor / ssm_launch_info /
 * ssm_device_error_report as compiled into the library, so that bindings can
 * check their layouts: which = 0 tensor, 1 conv1d args, 2 scan args, 3 ssu
 * args, 4 launch info, 5 error report, 6 delta-sum args, 7 carry-fold args,
 * 8 gated-conv args. */
size_t ssm_struct_size(int which);

/* The wait budget, in cycles, that a failure test's request of `cycles`
 * becomes: requests below 10^7 cycles are raised to 10^7.  Only the test
 * build of the library (libssm_causal_testhooks.so, compiled with
 * SSM_TEST_HOOKS) reads the failure-test switches from the environment:
 * SSM_TEST_DROP_ITEM (a state-update work item whose copies are never
 * started), SSM_TEST_DROP_WORKER (a prefill worker whose hand-over is never
 * published) and SSM_TEST_WAIT_CYCLES (the budget of the waits they leave
 * unanswered); the product library ignores them and always waits the full
 * budget. */
long long ssm_test_clamp_wait_budget(long long cycles);

#ifdef __cplusplus
}
#endif

#endif /* SSM_CAUSAL_H */
