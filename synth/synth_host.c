/* synth_host.c — host side of the seeded input generator (see philox.h). */
#include <stddef.h>
#include <stdint.h>

#include "philox.h"

void syn_philox_block(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
    syn_philox4x64_10(ctr, key[0], key[1], out);
}

/* out[j] = value(offset + j) of stream st, j < n. */
void syn_fill_normal(float* out, uint64_t n, uint64_t seed, uint64_t st, uint64_t offset, float c) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j) {
        int32_t s = syn_ih_int(seed, st, offset + (uint64_t)j);
        out[j] = (float)s * c;
    }
}

/* Raw 64-bit words (block words in order) for shuffles and selections. */
void syn_fill_u64(uint64_t* out, uint64_t n, uint64_t seed, uint64_t st) {
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < (int64_t)((n + 3) / 4); ++b) {
        uint64_t ctr[4] = {(uint64_t)b, st, 1, 0};
        uint64_t o[4];
        syn_philox4x64_10(ctr, seed, 0, o);
        for (int j = 0; j < 4; ++j)
            if ((uint64_t)b * 4 + j < n) out[b * 4 + j] = o[j];
    }
}
