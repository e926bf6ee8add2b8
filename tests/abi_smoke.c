/* Plain C99 user of include/muon.h, built and run by test_c_header_cpu.py on a
 * machine without a GPU: the header compiles as C, the library links, and the
 * host-only calls behave as documented. */
#include <stdio.h>
#include <string.h>

#include "muon.h"

static int failures = 0;
#define EXPECT(cond)                                            \
    do {                                                        \
        if (!(cond)) {                                          \
            printf("FAIL line %d: %s\n", __LINE__, #cond);      \
            ++failures;                                         \
        }                                                       \
    } while (0)

int main(void) {
    muon_config cfg;
    muon_config_default(&cfg);
    EXPECT(cfg.ns_steps == 5);
    EXPECT(cfg.ns_a == 3.4445f && cfg.ns_b == -4.7750f && cfg.ns_c == 2.0315f);
    EXPECT(muon_validate_config(&cfg) == MUON_OK);
    cfg.momentum = 1.5f;
    EXPECT(muon_validate_config(&cfg) == MUON_ERR_INVALID);
    muon_config_default(&cfg);

    float* w[1] = {0};
    const void* g[1] = {0};
    float* b[1] = {0};
    muon_group grp;
    memset(&grp, 0, sizeof(grp));
    grp.rows = 4; grp.cols = 8; grp.count = 1; grp.grad_dtype = MUON_BF16;
    grp.W = w; grp.G = g; grp.B = b;
    EXPECT(muon_validate_groups(&grp, 1) == MUON_ERR_INVALID);     /* null matrix pointers */

    int shapes[3] = {768, 3072, 2};
    int n = 0;
    EXPECT(muon_plan_tiles(shapes, 1, MUON_NS_UPDATE, NULL, 0, &n) == MUON_ERR_INVALID && n > 0);

    muon_handle* h = NULL;
    const muon_status st = muon_create(&cfg, 0, &h);
    EXPECT(h == NULL && st != MUON_OK);                            /* no GPU here */
    EXPECT(muon_step(NULL, &grp, 1, NULL) == MUON_ERR_INVALID);
    EXPECT(muon_set_memory_limit(NULL, 0) == MUON_ERR_INVALID);
    EXPECT(strcmp(muon_status_string(MUON_ERR_OOM), "MUON_ERR_OOM") == 0);
    printf(failures == 0 ? "c abi ok\n" : "c abi: %d failures\n", failures);
    return failures == 0 ? 0 : 1;
}
