/*
 * philox.h — Philox4x64-10 counter-based generator (Salmon, Moraes, Dror, Shaw, "Parallel
 * random numbers: as easy as 1, 2, 3", SC'11), written from its published definition, and
 * the seeded synthetic-value recipe used by the tests and the benchmark. Input generation
 * only: nothing here is part of the method. Compiled both by gcc (host side) and by nvcc
 * (device side), so both sides produce bit-identical values.
 *
 * Value recipe (a normal-shaped value computed with integer arithmetic and one binary32
 * multiply, so host and device agree exactly): value i of stream `st` under seed `seed` is
 *   block = Philox4x64-10(counter = {i >> 1, st, 0, 0}, key = {seed, 0}); take the two
 *   64-bit words 2*(i&1), 2*(i&1)+1 as eight 16-bit integers u_0..u_7;
 *   S = sum u_j - 4*65535   (an Irwin-Hall sum of 8 uniforms, centred; |S| <= 262140)
 *   value = (float)S * c    (c = sigma / sqrt(8 * (65536^2 - 1) / 12), rounded to binary32)
 * so the value has mean 0 and standard deviation sigma, with a bell shape bounded at
 * about 4.9 sigma.
 */
#ifndef SYN_PHILOX_H
#define SYN_PHILOX_H
#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_HD __host__ __device__ __forceinline__
#else
#define SYN_HD static inline
#endif

#define SYN_M0 0xD2E7470EE14C6C93ULL
#define SYN_M1 0xCA5A826395121157ULL
#define SYN_W0 0x9E3779B97F4A7C15ULL
#define SYN_W1 0xBB67AE8584CAA73BULL

SYN_HD void syn_mulhilo(uint64_t a, uint64_t b, uint64_t* hi, uint64_t* lo) {
#if defined(__CUDA_ARCH__)
    *lo = a * b;
    *hi = __umul64hi(a, b);
#else
    unsigned __int128 p = (unsigned __int128)a * b;
    *lo = (uint64_t)p;
    *hi = (uint64_t)(p >> 64);
#endif
}

/* One Philox4x64 block: 10 rounds, key bumped by the Weyl constants between rounds. */
SYN_HD void syn_philox4x64_10(const uint64_t ctr[4], uint64_t k0, uint64_t k1, uint64_t out[4]) {
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    for (int r = 0; r < 10; ++r) {
        uint64_t hi0, lo0, hi1, lo1;
        syn_mulhilo(SYN_M0, c0, &hi0, &lo0);
        syn_mulhilo(SYN_M1, c2, &hi1, &lo1);
        uint64_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += SYN_W0;
        k1 += SYN_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Centred Irwin-Hall integer of value i (see the recipe above). */
SYN_HD int32_t syn_ih_int(uint64_t seed, uint64_t st, uint64_t i) {
    uint64_t ctr[4] = {i >> 1, st, 0, 0};
    uint64_t o[4];
    syn_philox4x64_10(ctr, seed, 0, o);
    uint64_t a = o[2 * (i & 1)], b = o[2 * (i & 1) + 1];
    int32_t s = 0;
    for (int j = 0; j < 4; ++j) {
        s += (int32_t)((a >> (16 * j)) & 0xffff);
        s += (int32_t)((b >> (16 * j)) & 0xffff);
    }
    return s - 4 * 65535;
}

#endif
