/*
 * Exhaustive brute-force check of the oracle's BF16 and E4M3 encoders over
 * all 2^32 binary32 bit patterns.
 *
 * The brute force works differently from the oracle: it tabulates every
 * finite value of the target format from its closed-form decoding, finds the
 * two values around |x| by search, and picks the nearer one by comparing |x|
 * with their exact midpoint (ties to the even code).  E4M3 saturates: the
 * nearest FINITE value is chosen, so everything past 448 (infinity included)
 * lands on 448.  NaN must stay NaN.
 *
 * usage: brute_encoders {e4m3|bf16} [threads]   -> prints "mismatches=N"
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "fqr_oracle.h"

static double e4m3_val[127]; /* codes 0x00..0x7E, ascending */

static void init_e4m3(void) {
  for (int c = 0; c < 127; ++c) {
    int E = c >> 3, M = c & 7;
    e4m3_val[c] = E == 0 ? M * ldexp(1.0, -9) : (1.0 + M / 8.0) * ldexp(1.0, E - 7);
  }
}

static uint8_t brute_e4m3(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs((double)x);
  int lo = 0, hi = 126; /* largest c with val[c] <= a */
  if (a >= e4m3_val[126]) return sign | 126;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (e4m3_val[mid] <= a) lo = mid; else hi = mid - 1;
  }
  int c = lo;
  double m = (e4m3_val[c] + e4m3_val[c + 1]) * 0.5; /* exact */
  int pick;
  if (a < m) pick = c;
  else if (a > m) pick = c + 1;
  else pick = (c % 2 == 0) ? c : c + 1;
  return (uint8_t)(sign | pick);
}

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* returns 1 if the oracle's code is acceptable for x */
static int bf16_ok(float x, uint16_t got) {
  uint32_t u; memcpy(&u, &x, 4);
  if (isnan(x)) return ((got & 0x7F80u) == 0x7F80u) && (got & 0x007Fu);
  uint32_t sign = u & 0x80000000u, mag = u & 0x7FFFFFFFu;
  uint32_t lower = mag & 0xFFFF0000u, upper = lower + 0x10000u;
  uint16_t want;
  if (mag == lower) {
    want = (uint16_t)(lower >> 16);
  } else {
    double lv = (double)f_of(lower);
    double uv = (upper >= 0x7F800000u) ? ldexp(1.0, 128) : (double)f_of(upper);
    double a = (double)f_of(mag), m = (lv + uv) * 0.5;
    uint32_t pick;
    if (a < m) pick = lower;
    else if (a > m) pick = upper;
    else pick = ((lower >> 16) % 2 == 0) ? lower : upper;
    want = (uint16_t)(pick >> 16);  /* upper == 0x7F800000 is infinity */
  }
  want |= (uint16_t)(sign >> 16);
  return got == want;
}

typedef struct { int mode; uint64_t lo, hi; uint64_t bad; uint32_t first_bad; } job_t;

static void* run(void* p) {
  job_t* j = (job_t*)p;
  for (uint64_t i = j->lo; i < j->hi; ++i) {
    float x = f_of((uint32_t)i);
    int ok;
    if (j->mode == 0) ok = fqro_f32_to_e4m3_rn_satfinite(x) == brute_e4m3(x);
    else ok = bf16_ok(x, fqro_f32_to_bf16_rne(x));
    if (!ok) { if (!j->bad) j->first_bad = (uint32_t)i; j->bad++; }
  }
  return NULL;
}

int main(int argc, char** argv) {
  if (argc < 2) { fprintf(stderr, "usage: %s {e4m3|bf16} [threads]\n", argv[0]); return 2; }
  int mode = strcmp(argv[1], "e4m3") == 0 ? 0 : 1;
  int nt = argc > 2 ? atoi(argv[2]) : 8;
  if (nt < 1) nt = 1;
  if (nt > 256) nt = 256;
  init_e4m3();
  pthread_t th[256];
  job_t jobs[256];
  uint64_t total = 1ull << 32, step = (total + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    jobs[t].mode = mode; jobs[t].lo = t * step;
    jobs[t].hi = (t + 1) * step < total ? (t + 1) * step : total;
    jobs[t].bad = 0; jobs[t].first_bad = 0;
    pthread_create(&th[t], NULL, run, &jobs[t]);
  }
  uint64_t bad = 0; uint32_t first = 0; int have = 0;
  for (int t = 0; t < nt; ++t) {
    pthread_join(th[t], NULL);
    if (jobs[t].bad && !have) { first = jobs[t].first_bad; have = 1; }
    bad += jobs[t].bad;
  }
  printf("mismatches=%llu checked=%llu first_bad=0x%08x\n",
         (unsigned long long)bad, (unsigned long long)total, first);
  return bad ? 1 : 0;
}
