/*
 * A plain C99 caller of the library, compiled against include/ssm_causal.h
 * and linked with libssm_causal.so by tests/test_abi_c_program.py. It calls
 * every entry point the header declares with arguments that the host-side
 * checks reject (fake, aligned addresses; nothing reaches a device), so it
 * runs without a GPU. A signature that drifts from the header stops it from
 * compiling; a status code or a size rule that drifts makes it exit non-zero.
 */
#include <stdio.h>
#include <string.h>

#include "ssm_causal.h"

static int failures = 0;

static void expect(const char *what, int got, int want)
{
    if (got != want) {
        printf("%s: got %d, want %d (%s)\n", what, got, want, ssm_last_error());
        ++failures;
    } else if (want != SSM_OK && ssm_last_error()[0] == '\0') {
        printf("%s: rejected without a message\n", what);
        ++failures;
    }
}

static void check(const char *what, int ok)
{
    if (!ok) {
        printf("%s: does not hold\n", what);
        ++failures;
    }
}

int main(void)
{
    char *base = (char *)0x10000; /* 16-byte aligned; never dereferenced */
    void *p = base, *q = base + 0x200000, *r = base + 0x400000;
    const float *fp = (const float *)p;
    float *wf = (float *)p;
    int32_t *ip = (int32_t *)p;
    uint32_t *up = (uint32_t *)p;
    int a = 0, b = 0;

    check("version", ssm_version() > 0);
    {
        const unsigned long long before = ssm_launch_count();
        expect("rejected calls launch nothing", ssm_set_scan_variant(3, 1),
               SSM_ERR_INVALID_ARGUMENT);
        check("launch count unchanged", ssm_launch_count() == before);
    }

    /* sizing and host-side checks */
    check("dense scan needs no workspace", ssm_scan_workspace_size(100, 64, 16, 1) == 0);
    check("packed scan workspace is 256-byte rounded",
          ssm_scan_workspace_size(65536, 5120, 16, 34) % 256 == 0 &&
              ssm_scan_workspace_size(65536, 5120, 16, 34) >= 34 * 4);
    check("backward workspace", ssm_scan_bwd_workspace_size(64, 32, 16, 1) > 0);
    {
        const int32_t good[4] = {0, 3, 3, 10}, bad[3] = {0, 5, 3};
        expect("cu_seqlens accepted", ssm_check_cu_seqlens(good, 3, 10), SSM_OK);
        expect("cu_seqlens decreasing", ssm_check_cu_seqlens(bad, 2, 3), SSM_ERR_BAD_SEQLENS);
    }
    expect("scan variant knob", ssm_set_scan_variant(3, 1), SSM_ERR_INVALID_ARGUMENT);
    expect("scan variant choice", ssm_scan_variant_for(0, 16, &a, &b), SSM_ERR_INVALID_ARGUMENT);
    expect("backward variant knob", ssm_set_scan_bwd_variant(5), SSM_ERR_INVALID_ARGUMENT);
    expect("backward variant choice", ssm_scan_bwd_variant_for(4, 0, &a),
           SSM_ERR_INVALID_ARGUMENT);

    /* the three operations */
    expect("conv K out of range",
           ssm_causal_conv1d(p, q, fp, NULL, 64, 32, 5, NULL, 1, NULL, NULL, 1, SSM_BF16,
                             SSM_BF16, NULL),
           SSM_ERR_INVALID_ARGUMENT);
    expect("conv misaligned output",
           ssm_causal_conv1d(p, base + 0x100001, fp, NULL, 64, 32, 4, NULL, 1, NULL, NULL, 1,
                             SSM_BF16, SSM_BF16, NULL),
           SSM_ERR_MISALIGNED);
    expect("scan N unsupported",
           ssm_selective_scan_fwd(p, q, fp, p, p, NULL, NULL, NULL, 1, NULL, NULL, 1, r, NULL,
                                  64, 32, 8, SSM_BF16, NULL, 0, NULL),
           SSM_ERR_INVALID_ARGUMENT);
    expect("scan bad dtype",
           ssm_selective_scan_fwd(p, q, fp, p, p, NULL, NULL, NULL, 1, NULL, NULL, 1, r, NULL,
                                  64, 32, 16, (ssm_dtype)7, NULL, 0, NULL),
           SSM_ERR_UNSUPPORTED_DTYPE);
    expect("scan workspace too small",
           ssm_selective_scan_fwd(p, q, fp, p, p, NULL, NULL, NULL, 1, NULL, ip, 4, r, NULL, 64,
                                  32, 16, SSM_BF16, p, 8, NULL),
           SSM_ERR_WORKSPACE);
    expect("decode K out of range",
           ssm_selective_state_update(p, wf, p, p, p, p, NULL, fp, NULL, fp, NULL, NULL, 1, NULL,
                                      8, q, 8, 32, 16, 6, SSM_BF16, SSM_BF16, NULL),
           SSM_ERR_INVALID_ARGUMENT);

    /* the rest of the surface */
    expect("fused conv -> scan, no A",
           ssm_conv_scan_fwd(p, fp, NULL, NULL, NULL, NULL, 4, SSM_BF16, q, NULL, p, p, NULL,
                             NULL, NULL, 1, NULL, NULL, 1, r, NULL, 64, 32, 16, SSM_BF16, NULL),
           SSM_ERR_INVALID_ARGUMENT);
    expect("backward N unsupported",
           ssm_selective_scan_bwd(p, q, fp, p, p, NULL, NULL, NULL, 1, NULL, NULL, 1, r, NULL,
                                  base + 0x600000, base + 0x800000, NULL, wf, wf, wf, NULL, NULL,
                                  NULL, 64, 32, 8, SSM_BF16, p, 1 << 20, NULL),
           SSM_ERR_INVALID_ARGUMENT);
    expect("replay window out of range",
           ssm_replay_state_update(p, wf, p, wf, wf, ip, up, 0, p, p, p, p, NULL, fp, NULL, fp,
                                   NULL, NULL, 1, NULL, 8, q, 8, 32, 16, 4, SSM_BF16, SSM_BF16,
                                   NULL),
           SSM_ERR_INVALID_ARGUMENT);
    expect("replay reset N unsupported",
           ssm_replay_reset(fp, p, ip, up, NULL, 8, 8, 32, 4, NULL), SSM_ERR_INVALID_ARGUMENT);
    expect("replay flush window out of range",
           ssm_replay_flush(wf, p, fp, fp, ip, up, fp, 9, NULL, 8, 8, 32, 16, NULL),
           SSM_ERR_INVALID_ARGUMENT);
    expect("no-allocation scan, 4097 packed sequences",
           ssm_selective_scan_fwd_noalloc(p, q, fp, p, p, NULL, NULL, NULL, 1, NULL, ip, 4097,
                                          r, NULL, 4097, 32, 16, SSM_BF16, NULL),
           SSM_ERR_INVALID_ARGUMENT);

    {
        double ops = 0.0;
        expect("probe kind out of range", ssm_probe_rate(9, 10, 64, wf, 1 << 20, &ops, NULL),
               SSM_ERR_INVALID_ARGUMENT);
        expect("probe occupancy not a multiple of 8 warps",
               ssm_probe_rate(0, 10, 12, wf, 1 << 20, &ops, NULL), SSM_ERR_INVALID_ARGUMENT);
        expect("probe without a sink", ssm_probe_rate(0, 10, 64, NULL, 0, &ops, NULL),
               SSM_ERR_INVALID_ARGUMENT);
    }

    expect("wait self-test limit out of range", ssm_selftest_wait_timeout(0, NULL),
           SSM_ERR_INVALID_ARGUMENT);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
