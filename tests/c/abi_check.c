/*
 * The C ABI of include/msda.h used from plain C99 (no CUDA or C++ headers):
 * host-side queries and argument checks only, so it runs without a GPU.
 * Prints one line per check and exits non-zero on the first failure.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "msda.h"

static int failures = 0;

static void check(int ok, const char *what)
{
    printf("%s %s\n", ok ? "ok  " : "FAIL", what);
    if (!ok)
        failures++;
}

int main(void)
{
    msda_problem p;
    size_t bytes = 0;
    void *fake = (void *)(uintptr_t)0x100000; /* aligned, never dereferenced */

    memset(&p, 0, sizeof p);
    p.batch = 2;
    p.num_keys = 80;
    p.num_queries = 16;
    p.num_heads = 4;
    p.head_dim = 32;
    p.num_levels = 2;
    p.num_points = 4;
    p.value_dtype = MSDA_BF16;
    p.flags = MSDA_GRAD_VALUE_BF16;

    check(strcmp(msda_version(), "0.1.0") == 0, "version");
    check(strlen(msda_status_string(MSDA_ERR_DEVICE_BOUNDS)) > 0, "status string");
    check(msda_backward_workspace_size(&p, &bytes) == MSDA_OK && bytes == 2 * 80 * 4 * 32 * 4,
          "bf16 grad_value workspace = B*S*M*D float32");
    check(msda_forward(NULL, fake, fake, fake, fake, fake, fake, NULL) == MSDA_ERR_INVALID_ARG,
          "null problem");
    p.head_dim = 24;
    check(msda_forward(&p, fake, fake, fake, fake, fake, fake, NULL) == MSDA_ERR_UNSUPPORTED,
          "head_dim 24 unsupported");
    p.head_dim = 32;
    check(msda_forward(&p, NULL, fake, fake, fake, fake, fake, NULL) == MSDA_ERR_INVALID_ARG,
          "null value");
    p.value_dtype = MSDA_S8;
    check(msda_forward(&p, fake, fake, fake, fake, fake, fake, NULL) == MSDA_ERR_INVALID_ARG,
          "int8 value without value_scale");
    p.value_dtype = MSDA_F32;
    p.query_order = (const int32_t *)(uintptr_t)0x100002;
    check(msda_forward(&p, fake, fake, fake, fake, fake, fake, NULL) == MSDA_ERR_INVALID_ARG,
          "misaligned query_order");
    p.query_order = NULL;

    {
        msda_dcn_problem d;
        int64_t ho = 0, wo = 0;
        memset(&d, 0, sizeof d);
        d.batch = 1;
        d.height = 56;
        d.width = 56;
        d.groups = 4;
        d.group_channels = 16;
        d.kernel_h = d.kernel_w = 7;
        d.stride_h = d.stride_w = 2;
        d.pad_h = d.pad_w = 3;
        d.dilation_h = d.dilation_w = 1;
        d.value_dtype = MSDA_F32;
        check(msda_dcn_output_size(&d, &ho, &wo) == MSDA_OK && ho == 28 && wo == 28,
              "DCN output size 7x7 / 2");
        d.stride_w = 0;
        check(msda_dcn_output_size(&d, &ho, &wo) == MSDA_ERR_INVALID_ARG, "DCN stride 0");
    }
    printf("%d failure(s)\n", failures);
    return failures ? 1 : 0;
}
