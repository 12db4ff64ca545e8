/*
 * Drives the oracle with the workload of the demo program tree.ts on page "How
 * does a tree of summaries search a context? How ZHA works" (learn.chabulab.com),
 * section "Run a small tree yourself", and prints one line per tree size:
 *     <n keys> <mean comparisons per query> <mean % of attention kept>
 * The page prints the result of that program; tests/golden/demo_tree_output.txt
 * holds those values and test_oracle_demo.py compares.
 *
 * The workload generator below is written to give the same numbers as the demo,
 * so it follows JavaScript number semantics: every Float32Array store rounds to
 * fp32, arithmetic and dot products run in double, random numbers are drawn in
 * program order. The tree arithmetic itself is the oracle's (zha_oracle.c).
 *
 * Demo constants: 32 dimensions, chunks of 4, 4 reference queries (the first is
 * the zero vector, the others half of a random direction), sharpness 20, walks
 * start from the level of at most 64 nodes, p = 0.9, 12 queries per size.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "../oracle/zha_oracle.h"

enum { DIM = 32, CHUNK = 4, NREF = 4, QUERIES = 12, TOP = 64 };
static const double SHARPNESS = 20.0;
static const double PI = 3.141592653589793; /* the double nearest pi */

/* A 32-bit generator: add a Weyl constant, then two multiply-xorshift rounds
 * (known as mulberry32); seed 1; output in [0, 1). */
static uint32_t state = 1;
static double uniform01(void) {
    state += 0x6d2b79f5u;
    uint32_t t = state;
    t = (t ^ (t >> 15)) * (t | 1u);
    t ^= t + (t ^ (t >> 7)) * (t | 61u);
    return (double)(t ^ (t >> 14)) / 4294967296.0;
}

/* fp32 vector -> unit length (double norm, fp32 result); zero stays zero */
static void to_unit(float *v) {
    double ss = 0.0;
    for (int i = 0; i < DIM; ++i) ss += (double)v[i] * (double)v[i];
    double len = sqrt(ss);
    if (len == 0.0) len = 1.0;
    for (int i = 0; i < DIM; ++i) v[i] = (float)((double)v[i] / len);
}

/* random unit direction from Box-Muller normals (the log draw comes first) */
static void direction(float *v) {
    for (int i = 0; i < DIM; ++i) {
        double a = uniform01();
        double r = sqrt(-2.0 * log(1.0 - a));
        double b = uniform01();
        v[i] = (float)(r * cos(2.0 * PI * b));
    }
    to_unit(v);
}

/* unit(v + amount * random direction) */
static void nudge(const float *v, double amount, float *out) {
    float noise[DIM];
    direction(noise);
    for (int i = 0; i < DIM; ++i) out[i] = (float)((double)v[i] + amount * (double)noise[i]);
    to_unit(out);
}

/* nested topics: groups of 4096, 1024, 256, 64 and 16 neighbouring keys */
static void text_keys(long long n, float *keys) {
    static const long long sizes[5] = {4096, 1024, 256, 64, 16};
    float stack[5][DIM];
    for (int l = 0; l < 5; ++l) direction(stack[l]);
    for (long long i = 0; i < n; ++i) {
        for (int l = 0; l < 5; ++l) {
            if (i % sizes[l] == 0) {
                float base[DIM];
                if (l == 0)
                    direction(base);
                else
                    memcpy(base, stack[l - 1], sizeof base);
                nudge(base, 0.5, stack[l]);
            }
        }
        nudge(stack[4], 0.35, keys + i * DIM);
    }
}

int main(int argc, char **argv) {
    int store = argc > 1 ? atoi(argv[1]) : 1; /* the demo keeps keys fp32, biases double */
    double refs[NREF * DIM];
    memset(refs, 0, sizeof refs);
    for (int r = 1; r < NREF; ++r) {
        float v[DIM];
        direction(v);
        for (int i = 0; i < DIM; ++i) refs[r * DIM + i] = (double)(float)(v[i] * 0.5f);
    }
    static const long long sizes[4] = {1024, 4096, 16384, 65536};
    for (int si = 0; si < 4; ++si) {
        long long n = sizes[si];
        float *kf = (float *)malloc(sizeof(float) * (size_t)(n * DIM));
        double *K = (double *)malloc(sizeof(double) * (size_t)(n * DIM));
        text_keys(n, kf);
        for (long long i = 0; i < n * DIM; ++i) K[i] = kf[i];

        /* levels until at most TOP nodes remain, as the demo builds them */
        long long nn[ORC_MAX_LEVELS] = {0};
        double *lk[ORC_MAX_LEVELS] = {0}, *lb[ORC_MAX_LEVELS] = {0};
        nn[0] = n;
        int depth = 0;
        long long cur = n;
        do {
            ++depth;
            cur /= CHUNK;
            nn[depth] = cur;
            lk[depth] = (double *)malloc(sizeof(double) * (size_t)(cur * NREF * DIM));
            lb[depth] = (double *)malloc(sizeof(double) * (size_t)(cur * NREF));
            int rc = depth == 1
                         ? orc_build_level1(n, DIM, K, NREF, refs, CHUNK, SHARPNESS, store, 0, cur,
                                            lk[1], lb[1], 0)
                         : orc_build_level_up(DIM, NREF, lk[depth - 1], lb[depth - 1], refs, CHUNK,
                                              SHARPNESS, store, 0, cur, lk[depth], lb[depth], 0);
            if (rc) return 2;
        } while (cur > TOP);

        long long work = 0;
        double kept = 0.0;
        long long *sel = (long long *)malloc(sizeof(long long) * (size_t)nn[1]);
        for (int qi = 0; qi < QUERIES; ++qi) {
            long long at = (long long)floor(uniform01() * (double)n);
            float qf[DIM];
            nudge(kf + at * DIM, 0.2, qf);
            double q[DIM];
            for (int i = 0; i < DIM; ++i) q[i] = qf[i];
            long long n_sel = 0, fr[ORC_MAX_LEVELS], op[ORC_MAX_LEVELS], kr = 0, wk = 0;
            int s = 0;
            double tg, ts;
            if (orc_search(depth, nn, (const double *const *)lk, (const double *const *)lb, NREF, DIM,
                           CHUNK, SHARPNESS, TOP, q, ORC_TOP_P, 0.9, 0, sel, nn[1], &n_sel, fr, op,
                           &s, &kr, &wk, &tg, &ts))
                return 3;
            work += wk;
            kept += orc_kept_mass(n, DIM, SHARPNESS, K, q, sel, n_sel, CHUNK, nn[1]);
        }
        printf("%lld %.0f %.0f\n", n, floor((double)work / QUERIES + 0.5),
               floor(kept / QUERIES * 100.0 + 0.5));
        for (int l = 1; l <= depth; ++l) {
            free(lk[l]);
            free(lb[l]);
        }
        free(sel);
        free(kf);
        free(K);
    }
    return 0;
}
