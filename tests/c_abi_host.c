/* A plain C consumer of include/qem.h: the header compiles as C99, and the
 * library's host-only entry points answer through it without a GPU
 * (ABI string, status names, the interaction index's polar layout, the model
 * tables, argument errors).  Prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "qem.h"

#define CHECK(c)                                                     \
    do {                                                             \
        if (!(c)) {                                                  \
            fprintf(stderr, "check failed line %d: %s\n", __LINE__, #c); \
            return 1;                                                \
        }                                                            \
    } while (0)

int main(void)
{
    CHECK(strcmp(qem_abi(), "qem-pair-v2") == 0);
    CHECK(qem_status_string(QEM_ERR_MALFORMED) != NULL);

    /* polar layout of a 17 x 17 detector about its centre: every pixel once */
    int32_t nl = 0, nr = 0;
    CHECK(qem_polar_layout(17, 17, NULL, 8.0, 8.0, NULL, NULL, &nl, &nr) == QEM_OK);
    CHECK(nl >= 16 && nr >= 16 && nr <= nl);
    uint32_t *slots = (uint32_t *)malloc(sizeof(uint32_t) * 64 * (size_t)nl);
    int32_t *r0 = (int32_t *)malloc(sizeof(int32_t) * ((size_t)nr + 1));
    CHECK(qem_polar_layout(17, 17, NULL, 8.0, 8.0, slots, r0, &nl, &nr) == QEM_OK);
    int seen[289];
    memset(seen, 0, sizeof(seen));
    for (int i = 0; i < 64 * nl; ++i)
        if (slots[i] < 289)
            seen[slots[i]]++;
    for (int p = 0; p < 289; ++p)
        CHECK(seen[p] == 1);
    CHECK(r0[0] == 0 && r0[nr] == nl);
    free(slots);
    free(r0);

    /* argument errors are reported, not faulted */
    CHECK(qem_polar_layout(0, 5, NULL, 0.0, 0.0, NULL, NULL, &nl, &nr) == QEM_ERR_ARG);
    CHECK(qem_masked_sum(NULL, NULL, 1, 0, NULL, NULL, 1, NULL) == QEM_ERR_ARG);
    CHECK(qem_finish(NULL, NULL) == QEM_ERR_ARG);
    qem_info_t info;
    CHECK(qem_info(NULL, &info) == QEM_ERR_ARG);
    qem_free(NULL);

    /* model tables: 32 models x 256 pair symbols, frequencies of each model sum to 1024 */
    uint16_t *freq = (uint16_t *)malloc(sizeof(uint16_t) * 32 * 256);
    uint8_t amax[32];
    uint32_t *cost = (uint32_t *)malloc(sizeof(uint32_t) * 32 * 16);
    CHECK(qem_model_tables(freq, amax, cost) == QEM_OK);
    for (int m = 0; m < 32; ++m) {
        unsigned s = 0;
        for (int k = 0; k < 256; ++k)
            s += freq[m * 256 + k];
        CHECK(s == 1024u);
    }
    free(freq);
    free(cost);
    printf("ok\n");
    return 0;
}
