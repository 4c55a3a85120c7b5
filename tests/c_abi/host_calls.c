/*
 * A plain C program against include/atlas.h and libatlas.so: the boundary
 * used with no Python and no torch. Host-only calls (no GPU needed):
 * version, status names, the window offsets of a cube order and of the
 * aligned order, each checked against a count written out here from the
 * definitions, and an argument error that the library reports before any
 * device work. Exit status 0 and "ok" on success.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "atlas.h"

static int fail(const char *what) {
    fprintf(stderr, "FAIL: %s\n", what);
    return 1;
}

/* Extent of cube b along an axis of E tokens cut into cubes of c. */
static int64_t extent(int64_t E, int64_t c, int64_t b) {
    int64_t e = E - b * c;
    return e < c ? e : c;
}

int main(void) {
    if (atlas_version() <= 0) return fail("version");
    for (int s = 0; s <= 9; ++s)
        if (atlas_status_string((atlas_status)s) == NULL) return fail("status string");

    /* Cube order of a 5x7x9 grid in 2x3x4 cubes (partial cubes on every axis). */
    atlas_grid3 grid = {5, 7, 9};
    atlas_cube3 cube = {2, 3, 4};
    int64_t n = 0;
    if (atlas_cube_window_offsets(grid, cube, NULL, 0, &n) != ATLAS_OK) return fail("count");
    const int64_t nt = 3, nh = 3, nw = 3;
    if (n != nt * nh * nw) return fail("window count");
    int32_t *off = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
    if (atlas_cube_window_offsets(grid, cube, off, 4, &n) != ATLAS_ERR_CAPACITY)
        return fail("capacity error");
    if (atlas_cube_window_offsets(grid, cube, off, n + 1, &n) != ATLAS_OK) return fail("offsets");
    int64_t acc = 0, w = 0;
    for (int64_t bt = 0; bt < nt; ++bt)
        for (int64_t bh = 0; bh < nh; ++bh)
            for (int64_t bw = 0; bw < nw; ++bw, ++w) {
                if (off[w] != acc) return fail("cube offsets");
                acc += extent(5, 2, bt) * extent(7, 3, bh) * extent(9, 4, bw);
            }
    if (off[n] != acc || acc != 5 * 7 * 9) return fail("cube offsets end");

    /* Aligned order of a 2x3x4 global grid: token x of an axis of e sits at
     * detail position x*E/e, in detail cube floor(x*E/(c*e)). */
    atlas_grid3 gg = {2, 3, 4};
    int32_t *goff = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
    int64_t gn = 0;
    if (atlas_aligned_global_offsets(grid, cube, gg, goff, n + 1, &gn) != ATLAS_OK || gn != n)
        return fail("aligned offsets");
    int64_t *count = (int64_t *)calloc((size_t)n, sizeof(int64_t));
    for (int64_t t = 0; t < 2; ++t)
        for (int64_t h = 0; h < 3; ++h)
            for (int64_t x = 0; x < 4; ++x) {
                const int64_t bt = t * 5 / (2 * 2), bh = h * 7 / (3 * 3), bw = x * 9 / (4 * 4);
                count[(bt * nh + bh) * nw + bw] += 1;
            }
    acc = 0;
    for (w = 0; w < n; ++w) {
        if (goff[w] != acc) return fail("aligned ranges");
        acc += count[w];
    }
    if (goff[n] != 2 * 3 * 4) return fail("aligned end");

    /* Argument errors come back before any device work. */
    if (atlas_cube_reorder(NULL, NULL, grid, cube, 2, 64, ATLAS_FP32, NULL, NULL) !=
        ATLAS_ERR_NULL)
        return fail("null pointer");

    free(off);
    free(goff);
    free(count);
    printf("ok\n");
    return 0;
}
