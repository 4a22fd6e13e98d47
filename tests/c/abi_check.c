/* A plain C caller of the library: compiled with gcc against include/moe_b200.h and linked
 * against libmoe_b200.so.  Exercises the calls that need no GPU -- status strings, plan
 * validation of unsupported or invalid dimensions (checked before any device call), and the
 * rejection of NULL plans and oversize static routing -- prints the weight struct's layout,
 * and prints "c abi ok" on success. */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "moe_b200.h"

static int fails = 0;
#define CHECK(c)                                                        \
    do {                                                                \
        if (!(c)) {                                                     \
            printf("FAIL line %d: %s\n", __LINE__, #c);                 \
            ++fails;                                                    \
        }                                                               \
    } while (0)

int main(void)
{
    CHECK(strcmp(moe_strerror(MOE_OK), "MOE_OK") == 0);
    CHECK(strcmp(moe_strerror(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE") == 0);
    CHECK(strcmp(moe_strerror(MOE_ERR_DEVICE_TIMEOUT), "MOE_ERR_DEVICE_TIMEOUT") == 0);

    moe_dims d = {512, 4096, 512, 1024, 10, 1024, MOE_W_FP8_SC512};
    moe_plan_t *p = (moe_plan_t *)&d; /* must be reset to NULL on failure */
    size_t ws = 0;
    CHECK(moe_plan(NULL, &p, &ws) == MOE_ERR_INVALID_ARG);
    d.k = 0;
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_INVALID_ARG && p == NULL);
    d.k = 11;
    d.E = 10; /* k > E */
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_INVALID_ARG);
    d.k = 10;
    d.E = 512;
    d.H = 4000; /* not a multiple of 128 */
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_UNSUPPORTED);
    d.H = 4096;
    d.E = 2048; /* above 1024 experts */
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_UNSUPPORTED);
    d.E = 512;
    d.k = 33; /* above 32 experts per token */
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_UNSUPPORTED);
    d.k = 10;
    d.wfmt = 7; /* unknown weight format */
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_INVALID_ARG);
    d.H = 4000; /* the 4-bit formats need whole 128-element groups too */
    d.wfmt = MOE_W_MXFP4_G32;
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_UNSUPPORTED);
    d.wfmt = MOE_W_NVFP4_G16;
    CHECK(moe_plan(&d, &p, &ws) == MOE_ERR_UNSUPPORTED);
    d.H = 4096;
    /* struct layout, compared by the test with the Python binding's ctypes mirror */
    printf("layout moe_weights %zu %zu moe_dims %zu\n", sizeof(moe_weights), offsetof(moe_weights, t_gate),
           sizeof(moe_dims));

    CHECK(moe_forward(NULL, 1, NULL, NULL, NULL, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG);
    CHECK(moe_forward_x(NULL, 1, NULL, NULL, NULL, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG);
    CHECK(moe_router_logits(NULL, 1, NULL, NULL, NULL, NULL) == MOE_ERR_INVALID_ARG);
    CHECK(moe_router_topk(NULL, 1, NULL, NULL, NULL, NULL, NULL, NULL) == MOE_ERR_INVALID_ARG);
    CHECK(moe_route(NULL, 1, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG);
    CHECK(moe_launch_count(NULL) == 0);
    CHECK(moe_set_checked(NULL, 1) == MOE_ERR_INVALID_ARG);
    moe_destroy(NULL); /* accepted */
    /* static routing beyond its fixed scratch: rejected before any device work */
    CHECK(moe_route_static(1 << 18, 512, 10, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != MOE_OK);

    if (fails) {
        printf("c abi: %d failure(s)\n", fails);
        return 1;
    }
    printf("c abi ok\n");
    return 0;
}
