/* A plain C11 consumer of include/iabn.h: compiled and linked against
 * libiabn.so by tests/test_c_consumer.py, as C and as C++, with warnings as
 * errors.  It calls only host-side entry points (workspace sizing, plan
 * description with explicit device limits, argument rejection), so it runs
 * with or without a GPU, and prints one "key value" line per result. */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>

#include "iabn.h"

static void print_plan(const char* tag, const iabn_plan_info* p) {
    printf("%s.plan %d\n", tag, (int)p->plan);
    printf("%s.launches %d\n", tag, (int)p->launches);
    printf("%s.grid %d\n", tag, (int)p->grid);
    printf("%s.threads %d\n", tag, (int)p->threads);
    printf("%s.smem_bytes %d\n", tag, (int)p->smem_bytes);
    printf("%s.tile_bytes %d\n", tag, (int)p->tile_bytes);
    printf("%s.slots %d\n", tag, (int)p->slots);
    printf("%s.ring %d\n", tag, (int)p->ring);
    printf("%s.vectors_per_row %d\n", tag, (int)p->vectors_per_row);
    printf("%s.cols_per_thread %d\n", tag, (int)p->cols_per_thread);
    printf("%s.row_phases %d\n", tag, (int)p->row_phases);
    printf("%s.planes_per_unit %d\n", tag, (int)p->planes_per_unit);
    printf("%s.stash_rows %d\n", tag, (int)p->stash_rows);
    printf("%s.stash_copy_engine %d\n", tag, (int)p->stash_copy_engine);
}

int main(void) {
    iabn_desc trunk = {64, 256, 56, 56, IABN_NHWC, IABN_BF16};
    iabn_desc many = {128, 2048, 7, 7, IABN_NCHW, IABN_F16};
    iabn_desc bad = {0, 256, 56, 56, IABN_NHWC, IABN_BF16};
    iabn_plan_info info;
    float dummy[4];

    printf("sizeof_desc %zu\n", sizeof(iabn_desc));
    printf("sizeof_plan_info %zu\n", sizeof(iabn_plan_info));
    printf("ws_trunk %zu\n", iabn_workspace_size(&trunk));
    printf("ws_many %zu\n", iabn_workspace_size(&many));
    printf("ws_bad %zu\n", iabn_workspace_size(&bad));
    printf("describe_fwd_status %d\n", (int)iabn_describe_plan(&trunk, 0, 148, 232448, &info));
    print_plan("trunk_fwd", &info);
    printf("describe_bwd_status %d\n", (int)iabn_describe_plan(&trunk, 1, 148, 232448, &info));
    print_plan("trunk_bwd", &info);
    printf("describe_many_status %d\n", (int)iabn_describe_plan(&many, 0, 148, 232448, &info));
    print_plan("many_fwd", &info);
    printf("describe_std_bwd_status %d\n",
           (int)iabn_describe_plan(&trunk, IABN_CALL_BACKWARD_STANDARD, 148, 232448, &info));
    print_plan("trunk_std_bwd", &info);
    printf("describe_ckpt_fwd_status %d\n",
           (int)iabn_describe_plan(&trunk, IABN_CALL_FORWARD_CHECKPOINT, 148, 232448, &info));
    print_plan("trunk_ckpt_fwd", &info);
    printf("describe_bad_call %d\n", (int)iabn_describe_plan(&trunk, 6, 148, 232448, &info));
    /* rejected on the host before any CUDA call */
    printf("forward_null_x %d\n",
           (int)iabn_forward(&trunk, NULL, dummy, dummy, 1e-5f, IABN_ACT_LEAKY_RELU, 0.01f,
                             dummy, dummy, NULL, 0, NULL));
    printf("backward_bad_desc %d\n",
           (int)iabn_backward(&bad, dummy, dummy, dummy, dummy, dummy, 1e-5f,
                              IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, NULL, 0, NULL));
    printf("inference_bad_act %d\n",
           (int)iabn_inference(&trunk, dummy, dummy, dummy, dummy, dummy, 1e-5f, 9, 0.01f,
                               NULL, 0, NULL));
    printf("forward_standard_null_z %d\n",
           (int)iabn_forward_standard(&trunk, dummy, NULL, dummy, dummy, 1e-5f,
                                      IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, NULL, 0, NULL));
    printf("backward_standard_null_mean %d\n",
           (int)iabn_backward_standard(&trunk, dummy, dummy + 2, dummy, dummy, NULL, dummy, 1e-5f,
                                       IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, NULL, 0, NULL));
    printf("forward_checkpoint_bad_eps %d\n",
           (int)iabn_forward_checkpoint(&trunk, dummy, dummy, dummy, dummy, -1.f,
                                        IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, NULL, 0, NULL));
    printf("backward_checkpoint_bad_desc %d\n",
           (int)iabn_backward_checkpoint(&bad, dummy, dummy, dummy, dummy, dummy, 1e-5f,
                                         IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, NULL, 0,
                                         NULL));
    printf("recompute_null_xhat %d\n",
           (int)iabn_checkpoint_recompute(&trunk, NULL, dummy, dummy, dummy,
                                          IABN_ACT_LEAKY_RELU, 0.01f, NULL));
    printf("forward_running_null_rmean %d\n",
           (int)iabn_forward_with_running_stats(&trunk, dummy, dummy, dummy, 1e-5f,
                                                IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, NULL,
                                                dummy, 0.1f, NULL, 0, NULL));
    printf("sync_forward_stats_null_stats %d\n",
           (int)iabn_sync_forward_stats(&trunk, dummy, NULL, dummy, 1 << 30, NULL));
    printf("sync_forward_apply_bad_world %d\n",
           (int)iabn_sync_forward_apply(&trunk, dummy, (const double*)dummy, 0, dummy, dummy,
                                        1e-5f, IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, dummy,
                                        (size_t)1 << 30, NULL));
    printf("sync_backward_stats_bad_act %d\n",
           (int)iabn_sync_backward_stats(&trunk, dummy, dummy, dummy, dummy, 7, 0.01f,
                                         (double*)dummy, dummy, (size_t)1 << 30, NULL));
    printf("sync_backward_apply_null_gathered %d\n",
           (int)iabn_sync_backward_apply(&trunk, dummy, dummy + 2, NULL, 2, dummy, dummy, dummy,
                                         1e-5f, IABN_ACT_LEAKY_RELU, 0.01f, dummy, dummy, dummy,
                                         (size_t)1 << 30, NULL));
    printf("running_bad_count %d\n",
           (int)iabn_update_running_stats(256, 1, dummy, dummy, dummy, dummy, 0.1f, NULL));
    printf("status_null_ws %d\n", (int)iabn_get_device_status(NULL, NULL));
    printf("launches %llu\n", (unsigned long long)iabn_kernel_launches());
    return 0;
}
