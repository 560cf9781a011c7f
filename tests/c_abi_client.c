/* A plain C client of libssm_causal: fills the args structs with ssm_tensor
 * descriptors (fake, never dereferenced device addresses) and calls the entry
 * points in dry-run mode, which checks and plans without launching.  Built
 * and run by tests/test_abi_host.py; prints one line per check. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ssm_causal.h"

static uintptr_t next_addr = (uintptr_t)1 << 40;

static ssm_tensor dense(int dtype, int ndim, const int64_t* shape) {
    ssm_tensor t;
    memset(&t, 0, sizeof t);
    t.data = (void*)next_addr;
    next_addr += (uintptr_t)1 << 36;
    t.dtype = dtype;
    t.ndim = ndim;
    int64_t acc = 1;
    for (int i = ndim - 1; i >= 0; --i) {
        t.shape[i] = shape[i];
        t.stride[i] = acc;
        acc *= shape[i] > 0 ? shape[i] : 1;
    }
    return t;
}

int main(void) {
    int fails = 0;
    printf("abi_version %d\n", ssm_abi_version());
    if (ssm_struct_size(2) != sizeof(ssm_scan_args)) ++fails;

    /* Mamba-1 prefill, 2.8B shape, fp16 I/O */
    const int64_t BDL[3] = {4, 5120, 2048}, DN[2] = {5120, 16}, BNL[3] = {4, 16, 2048}, D1[1] = {5120};
    ssm_scan_args a;
    memset(&a, 0, sizeof a);
    a.struct_size = sizeof a;
    a.flags = SSM_FLAG_DRY_RUN;
    a.x = dense(SSM_F16, 3, BDL);
    a.dt = dense(SSM_F16, 3, BDL);
    a.A = dense(SSM_F32, 2, DN);
    a.B = dense(SSM_F16, 3, BNL);
    a.C = dense(SSM_F16, 3, BNL);
    a.D = dense(SSM_F32, 1, D1);
    a.out = dense(SSM_F16, 3, BDL);
    a.dt_softplus = 1;
    ssm_launch_info info;
    memset(&info, 0, sizeof info);
    info.struct_size = sizeof info;
    a.info = &info;
    int st = ssm_selective_scan_fwd(&a, NULL);
    printf("scan %s kernel %d grid %d\n", ssm_status_string(st), info.kernel, info.grid);
    if (st != SSM_OK || info.kernel != SSM_KERNEL_SCAN_BAL) ++fails;

    /* the workspace the balanced prefill asks for, then the plan that uses it */
    uint64_t need = 0;
    st = ssm_selective_scan_workspace_size(&a, &need);
    printf("scan workspace %s %llu bytes\n", ssm_status_string(st), (unsigned long long)need);
    if (st != SSM_OK || need == 0) ++fails;
    a.workspace = (void*)next_addr;
    next_addr += (uintptr_t)1 << 36;
    a.workspace_bytes = need;
    st = ssm_selective_scan_fwd(&a, NULL);
    printf("scan with workspace %s grid %d\n", ssm_status_string(st), info.grid);
    if (st != SSM_OK || info.kernel != SSM_KERNEL_SCAN_BAL) ++fails;
    a.workspace_bytes = need - 1;
    if (ssm_selective_scan_fwd(&a, NULL) != SSM_ERR_WORKSPACE) ++fails;
    a.workspace = NULL;
    a.workspace_bytes = 0;

    /* error paths: wrong struct size, NULL args, output aliasing an input */
    a.struct_size = sizeof a - 8;
    if (ssm_selective_scan_fwd(&a, NULL) != SSM_ERR_VERSION) ++fails;
    a.struct_size = sizeof a;
    if (ssm_selective_scan_fwd(NULL, NULL) != SSM_ERR_NULL) ++fails;
    a.out = a.x;
    if (ssm_selective_scan_fwd(&a, NULL) != SSM_ERR_ALIAS) ++fails;

    /* Mamba-2 decode, H=80 P=64 N=128 */
    const int64_t BHPN[4] = {16, 80, 64, 128}, BHP[3] = {16, 80, 64}, BH[2] = {16, 80}, H1[1] = {80},
                  BGN[3] = {16, 1, 128};
    ssm_ssu_args u;
    memset(&u, 0, sizeof u);
    u.struct_size = sizeof u;
    u.flags = SSM_FLAG_DRY_RUN;
    u.state = dense(SSM_F16, 4, BHPN);
    u.x = dense(SSM_F16, 3, BHP);
    u.dt = dense(SSM_F16, 2, BH);
    u.A = dense(SSM_F32, 1, H1);
    u.B = dense(SSM_F16, 3, BGN);
    u.C = dense(SSM_F16, 3, BGN);
    u.out = dense(SSM_F16, 3, BHP);
    u.dt_softplus = 1;
    memset(&info, 0, sizeof info);
    info.struct_size = sizeof info;
    u.info = &info;
    st = ssm_selective_state_update(&u, NULL);
    printf("ssu %s kernel %d grid %d\n", ssm_status_string(st), info.kernel, info.grid);
    if (st != SSM_OK || info.kernel != SSM_KERNEL_SSU_TMA) ++fails;

    /* double-gated short conv, token-major: x, b_gate, c_gate are the three
       D-wide slices of one (B, L, 3D) projection output, out is (B, L, D) */
    {
        const int64_t Bn = 4, L = 2048, D = 2048, W = 3;
        const int64_t proj_shape[3] = {Bn, L, 3 * D}, out_shape[3] = {Bn, L, D}, wshape[2] = {D, W},
                      dshape[1] = {D}, csshape[3] = {Bn, D, W};
        const ssm_tensor proj = dense(SSM_F16, 3, proj_shape), outs = dense(SSM_F16, 3, out_shape);
        ssm_gated_conv1d_args g;
        memset(&g, 0, sizeof g);
        g.struct_size = sizeof g;
        g.flags = SSM_FLAG_DRY_RUN;
        ssm_tensor* views[3] = {&g.b_gate, &g.c_gate, &g.x};
        for (int i = 0; i < 3; ++i) {
            ssm_tensor v = proj;  /* (B, D, L) view: channel stride 1, step stride 3D */
            v.data = (char*)proj.data + (size_t)(i * D) * 2;
            v.shape[0] = Bn; v.shape[1] = D; v.shape[2] = L;
            v.stride[0] = L * 3 * D; v.stride[1] = 1; v.stride[2] = 3 * D;
            *views[i] = v;
        }
        g.out = outs;
        g.out.shape[0] = Bn; g.out.shape[1] = D; g.out.shape[2] = L;
        g.out.stride[0] = L * D; g.out.stride[1] = 1; g.out.stride[2] = D;
        g.weight = dense(SSM_F32, 2, wshape);
        g.bias = dense(SSM_F32, 1, dshape);
        g.conv_state = dense(SSM_F32, 3, csshape);
        memset(&info, 0, sizeof info);
        info.struct_size = sizeof info;
        g.info = &info;
        st = ssm_gated_conv1d_fwd(&g, NULL);
        printf("gated conv %s kernel %d grid %d\n", ssm_status_string(st), info.kernel, info.grid);
        if (st != SSM_OK || info.kernel != SSM_KERNEL_GATED_CONV) ++fails;
        if (ssm_struct_size(8) != sizeof(ssm_gated_conv1d_args)) ++fails;
        g.out = g.x;  /* an output over an input */
        if (ssm_gated_conv1d_fwd(&g, NULL) != SSM_ERR_ALIAS) ++fails;
    }

    printf("fails %d\n", fails);
    return fails == 0 ? 0 : 1;
}
