/* A plain C99 client of libss2d: include/ss2d.h must compile as C, and the library must
 * link and answer from C.  Host-only calls (no GPU needed): version, status strings, the
 * argument checks and the workspace queries of the fused core with fake, never-dereferenced
 * device pointers.  Prints one "key value" line per result for tests/test_c_abi.py. */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ss2d.h"

#define FAKE(k) ((void *)(uintptr_t)(0x7F0000000000ull + ((uint64_t)(k) << 20)))

static ss2d_core_args core(void)
{
    ss2d_core_args a;
    memset(&a, 0, sizeof(a));
    a.struct_size = sizeof(a);
    a.B = 1;
    a.D = 16;
    a.H = 8;
    a.W = 8;
    a.N = 16;
    a.x = FAKE(0);
    a.x_dtype = SS2D_BF16;
    a.dts = FAKE(1);
    a.dts_dtype = SS2D_BF16;
    a.Bs = (const float *)FAKE(2);
    a.Cs = (const float *)FAKE(3);
    a.A_logs = (const float *)FAKE(4);
    a.Ds = (const float *)FAKE(5);
    a.dt_bias = (const float *)FAKE(6);
    a.delta_softplus = 1;
    a.y = FAKE(8);
    return a;
}

int main(void)
{
    ss2d_core_args a = core();
    printf("version %d\n", ss2d_version());
    printf("status_ok %s\n", ss2d_status_string(SS2D_OK));
    printf("status_device %s\n", ss2d_status_string(SS2D_ERR_DEVICE));
    printf("sizeof_args %zu\n", sizeof(ss2d_core_args));
    printf("sizeof_grads %zu\n", sizeof(ss2d_core_grads));
    printf("offset_ckpt %zu\n", offsetof(ss2d_core_args, ckpt));
    printf("offset_layout %zu\n", offsetof(ss2d_core_args, layout));
    printf("offset_merge_order %zu\n", offsetof(ss2d_core_args, merge_order));
    printf("sizeof_block %zu\n", sizeof(ss2d_block_args));
    printf("offset_block_eps %zu\n", offsetof(ss2d_block_args, out_norm_eps));
    printf("offset_block_out_dtype %zu\n", offsetof(ss2d_block_args, out_dtype));
    printf("fwd_ws %zu\n", ss2d_forward_core_workspace(&a));
    printf("bwd_ws %zu\n", ss2d_forward_core_backward_workspace(&a));
    a.N = 5;
    printf("bad_n %d\n", ss2d_forward_core(&a, NULL, 0, NULL));
    printf("bad_n_msg %s\n", ss2d_last_error());
    a = core();
    a.x = (const char *)FAKE(0) + 8;
    printf("misaligned %d\n", ss2d_forward_core(&a, NULL, 0, NULL));
    a = core();
    printf("device_status_direct %d\n", ss2d_device_status(&a, NULL, 0, NULL));
    return 0;
}
