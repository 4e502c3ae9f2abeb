/*
 * Exhaustive checks of the E2M1 and E4M3 encoding rules over all 2^32 fp32
 * bit patterns.  TEST INFRASTRUCTURE ONLY: built by the package build step,
 * run by tests/test_oracle_formats.py, never linked into the product.
 *
 * Two independent restatements of each rule are compared on every finite
 * input:
 *   (a) brute force: the nearest value of the format's own value list, ties
 *       to the even code, saturating at the largest finite value (the rule
 *       the oracle module uses, written again here in C);
 *   (b) arithmetic: an integer round-half-even on the fp32 significand,
 *       derived from where each format's grid spacing changes.
 * E2M1 follows the value table of "DeepSeek-V4.1-Flash-NVFP4" §二.
 *
 * Usage:  sweep e2m1|e4m3 [nthreads]   -> prints "mismatches=<n> checked=<n>"
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
static double kE4M3[127];

/* Nearest entry of the ascending list vals[0..n-1]; ties to the even index;
 * saturate at the last entry.  The bracket is found by bisection. */
static int nearest_even(double a, const double *vals, int n) {
  if (a >= vals[n - 1]) return n - 1;
  int lo = 0, hi = n - 1; /* invariant: vals[lo] <= a < vals[hi] */
  if (a < vals[0]) return 0;
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (vals[mid] <= a) lo = mid; else hi = mid;
  }
  double dl = a - vals[lo], dh = vals[hi] - a;
  if (dl < dh) return lo;
  if (dh < dl) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

/* Round |a| to a multiple of 2^q with round-half-even, working on the exact
 * binary value a = M * 2^E (M integer): returns the multiple count. */
static uint64_t rhe_units(double a, int q) {
  /* a and 2^q are exact doubles; a / 2^q is exact (power-of-two scaling). */
  double u = ldexp(a, -q);
  double f = floor(u);
  double rem = u - f;
  uint64_t n = (uint64_t)f;
  if (rem > 0.5 || (rem == 0.5 && (n & 1))) n += 1;
  return n;
}

/* E2M1 magnitude code by arithmetic: grid 0.5 on [0,2), 1 on [2,4), 2 on [4,6]. */
static int e2m1_arith(double a) {
  if (a >= 6.0) return 7;
  if (a < 2.0) {
    uint64_t n = rhe_units(a, -1); /* multiples of 0.5, n in 0..4 */
    /* n=4 means 2.0, which is code 4 */
    static const int code_of_half[5] = {0, 1, 2, 3, 4};
    return code_of_half[n];
  }
  if (a < 4.0) {
    uint64_t n = rhe_units(a, 0); /* 2,3,4 */
    return n == 2 ? 4 : n == 3 ? 5 : 6;
  }
  /* [4, 6): grid 2, values 4 or 6; half-even on units of 2: 4 -> 2 (even), 6 -> 3 (odd) */
  uint64_t n = rhe_units(a, 1);
  return n == 2 ? 6 : 7;
}

/* E4M3 code by arithmetic: exponent of a decides the grid 2^(e-3), subnormal grid 2^-9. */
static int e4m3_arith(double a) {
  if (a >= 448.0) return 0x7E;
  int e;
  (void)frexp(a, &e); /* a = m 2^e, m in [0.5,1): floor(log2 a) = e-1 */
  int fl = (a == 0.0) ? -100 : e - 1;
  if (fl < -6) { /* subnormal range, grid 2^-9, codes 0..8 (8 == 2^-6 normal) */
    uint64_t n = rhe_units(a, -9);
    return (int)n; /* n == 8 -> code 0x08 which is 2^-6: consistent encoding */
  }
  uint64_t n = rhe_units(a, fl - 3); /* 8..16 units of 2^(fl-3) */
  int ef = fl + 7;
  if (n == 16) { n = 8; ef += 1; }
  int code = (ef << 3) | (int)(n - 8);
  if (code > 0x7E) code = 0x7E;
  return code;
}

typedef struct { int which; uint64_t lo, hi, mism, checked; } job_t;

static void *work(void *p) {
  job_t *j = (job_t *)p;
  for (uint64_t b = j->lo; b < j->hi; ++b) {
    uint32_t bits = (uint32_t)b;
    float f;
    memcpy(&f, &bits, 4);
    if (!isfinite(f)) continue;
    double a = fabs((double)f);
    int x, y;
    if (j->which == 0) { x = nearest_even(a, kE2M1, 8); y = e2m1_arith(a); }
    else { if (bits >> 31) continue; x = nearest_even(a, kE4M3, 127); y = e4m3_arith(a); }
    j->checked++;
    if (x != y) {
      if (j->mism < 5) fprintf(stderr, "mismatch bits=%08x a=%.9g brute=%d arith=%d\n", bits, a, x, y);
      j->mism++;
    }
  }
  return NULL;
}

int main(int argc, char **argv) {
  if (argc < 2) { fprintf(stderr, "usage: sweep e2m1|e4m3 [threads]\n"); return 2; }
  int which = strcmp(argv[1], "e4m3") == 0 ? 1 : 0;
  int nt = argc > 2 ? atoi(argv[2]) : 8;
  if (nt < 1 || nt > 256) nt = 8;
  for (int c = 0; c < 127; ++c) {
    int e = c >> 3, m = c & 7;
    kE4M3[c] = e == 0 ? m * ldexp(1.0, -9) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  }
  pthread_t th[256];
  job_t jobs[256];
  uint64_t total = 1ull << 32, step = total / nt;
  for (int i = 0; i < nt; ++i) {
    jobs[i].which = which; jobs[i].lo = i * step; jobs[i].hi = (i == nt - 1) ? total : (i + 1) * step;
    jobs[i].mism = jobs[i].checked = 0;
    pthread_create(&th[i], NULL, work, &jobs[i]);
  }
  uint64_t mism = 0, checked = 0;
  for (int i = 0; i < nt; ++i) { pthread_join(th[i], NULL); mism += jobs[i].mism; checked += jobs[i].checked; }
  printf("mismatches=%llu checked=%llu\n", (unsigned long long)mism, (unsigned long long)checked);
  return mism ? 1 : 0;
}
