/* The C ABI used from plain C (no C++, no Python): include/hxq.h compiles
 * as C99, libhxq links, and every entry point rejects bad arguments with
 * HXQ_EINVAL before touching a GPU. Prints "ok" and exits 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "hxq.h"

static int failures = 0;
#define EXPECT(cond)                                                      \
    do {                                                                  \
        if (!(cond)) {                                                    \
            fprintf(stderr, "%s:%d: failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                   \
        }                                                                 \
    } while (0)

int main(void) {
    float cb[256] = {0};
    uint8_t idx[64] = {0};
    uint16_t x[16] = {0};
    float y[16] = {0};
    int64_t pos = 1, count = 0;
    float val = 1.0f;
    hxq_linear_t h = (hxq_linear_t)0;
    hxq_group_t g = (hxq_group_t)0;
    hxq_linear_t none[2] = {0, 0};
    void* ys[2] = {y, y};

    EXPECT(hxq_linear_create(cb, idx, HXQ_MODE_SCALAR8, &pos, &val, 1, 8, 8, NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_create(NULL, idx, HXQ_MODE_SCALAR8, NULL, NULL, 0, 8, 8, &h) == HXQ_EINVAL);
    EXPECT(hxq_linear_create(cb, idx, 7, NULL, NULL, 0, 8, 8, &h) == HXQ_EINVAL);
    EXPECT(hxq_linear_create(cb, idx, HXQ_MODE_VQ2D12, NULL, NULL, 0, 8, 10, &h) == HXQ_EINVAL);
    EXPECT(hxq_linear_create(cb, idx, HXQ_MODE_SCALAR8, NULL, NULL, 0, 8, 0, &h) == HXQ_EINVAL);
    EXPECT(h == NULL);
    EXPECT(hxq_linear_forward(NULL, x, y, 1, NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_forward_ex(NULL, x, y, 1, HXQ_KERNEL_AUTO, 0, NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_forward_out(NULL, x, NULL, y, HXQ_OUT_F32, 1, NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_forward_noalloc(NULL, x, y, 1, NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_forward_host(NULL, x, x, y, y, 1, NULL) == HXQ_EINVAL);
    EXPECT(hxq_decode(NULL, y, NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_check(NULL) == HXQ_EINVAL);
    EXPECT(hxq_linear_info(NULL, NULL, NULL, NULL, NULL) == HXQ_EINVAL);
    EXPECT(hxq_group_create(none, 2, &g) == HXQ_EINVAL);
    EXPECT(hxq_group_create(none, HXQ_MAX_GROUP + 1, &g) == HXQ_EINVAL);
    EXPECT(g == NULL);
    EXPECT(hxq_group_forward(NULL, x, NULL, ys, HXQ_OUT_F32, 1, NULL) == HXQ_EINVAL);
    EXPECT(hxq_assign(NULL, 16, 1, cb, 8, x, NULL) == HXQ_EINVAL);
    EXPECT(hxq_kmeans(y, 16, 3, 8, 1, cb, NULL, NULL) == HXQ_EINVAL);
    EXPECT(hxq_encode(y, HXQ_MODE_SCALAR8, 2, 8, cb, -1.0f, idx, NULL, NULL, 0, &count, NULL) == HXQ_EINVAL);
    hxq_linear_destroy(NULL);
    hxq_group_destroy(NULL);
    EXPECT(strlen(hxq_strerror(HXQ_EINVAL)) > 0);
    if (failures) return 1;
    printf("ok\n");
    return 0;
}
