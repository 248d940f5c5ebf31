// Exhaustive CPU check of the converter's two encoders (test code).
//
// The GPU converter encodes a 128 x 128 block with divisor d = RN(amax / 448)
// as E4M3(RN(v * c)) for a multiplier c that it first checks on the 128 BF16
// mantissas: for v_m = 1.m x 2^-e(c), E4M3 of RN(v_m / d) and of RN(v_m * c),
// both scaled by 2^0 and by 2^-7 ... 2^-12, must agree; candidates are
// RN(1/d), its upper neighbour, then its lower one; blocks with d < 2^-100 or
// no passing candidate use another encoder. This program repeats that
// selection in FP32 (SSE, round to nearest even, no contraction) for every
// positive finite BF16 block maximum, and for each block with a passing c
// compares E4M3(RN(v * c)) with E4M3(RN(v / d)) for every BF16 v with
// |v| <= amax, both signs. It also checks the converter's other encoder,
// the product bracket, for every block with d >= 2^-125: with y = RN(1/d),
// ylo = RN(y (1 - 2^-21)) and yhi = RN(y (1 + 2^-21)), whenever the codes of
// RN(v * ylo) and RN(v * yhi) agree they must equal the quotient's code (the
// other elements, the straddles, are divided exactly). It prints the counts
// and exits 1 on any mismatch.
// The E4M3 rounding here is its own: the nearest of the 127 finite
// magnitudes, ties to the even code, saturating at 448.
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float f_of(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t b_of(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

static double mag[127];  // finite E4M3 magnitudes by code 0..126
static void init_mag(void) {
  for (int c = 0; c < 127; ++c) {
    const int e = (c >> 3) & 15, m = c & 7;
    mag[c] = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp(m / 8.0, -6);
  }
}
static uint8_t e4m3(float f) {
  const uint8_t s = (uint8_t)((b_of(f) >> 24) & 0x80);
  const double a = fabs((double)f);
  if (isnan(f)) return 0x7F;
  if (a >= 448.0) return s | 0x7E;
  int lo = 0, hi = 126;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (mag[mid] <= a) lo = mid; else hi = mid;
  }
  const double dl = a - mag[lo], dh = mag[hi] - a;
  const int c = dl < dh ? lo : (dh < dl ? hi : ((lo & 1) ? hi : lo));
  return s | (uint8_t)c;
}

static int passes(float d, float c) {
  const int ec = (int)((b_of(c) >> 23) & 0xFF) - 127;
  for (int m = 0; m < 128; ++m) {
    volatile float vm = f_of(((uint32_t)(127 - ec) << 23) | ((uint32_t)m << 16));
    volatile float r = vm / d, rp = vm * c;
    if (e4m3(r) != e4m3(rp)) return 0;
    float s = 0.0078125f;  // 2^-7
    for (int k = 0; k < 6; ++k, s *= 0.5f) {
      volatile float a = r * s, b = rp * s;
      if (e4m3(a) != e4m3(b)) return 0;
    }
  }
  return 1;
}

typedef struct {
  int t, nt;
  long long blocks, chosen[3], none, pairs, bad;
  long long bracket_pairs, straddles, bracket_bad;
} Job;

// The bracket over every BF16 v of the block with maximum bits ab (d >= 2^-125).
static void bracket(Job* J, uint32_t ab, float d) {
  volatile float y = 1.0f / d;
  volatile float ylo = y * 0.99999952316284180f;  // 1 - 2^-21
  volatile float yhi = y * 1.00000047683715820f;  // 1 + 2^-21
  for (uint32_t vb = 0; vb <= ab; ++vb)
    for (int sg = 0; sg < 2; ++sg) {
      volatile float v = f_of((vb | (sg ? 0x8000u : 0u)) << 16);
      volatile float plo = v * ylo, phi = v * yhi, q = v / d;
      const uint8_t clo = e4m3(plo), chi = e4m3(phi);
      ++J->bracket_pairs;
      if (clo != chi) { ++J->straddles; continue; }
      if (clo != e4m3(q)) {
        if (J->bracket_bad < 5) printf("bracket mismatch: amax bits %04x, v bits %04x\n", ab, vb);
        ++J->bracket_bad;
      }
    }
}

static void* run(void* arg) {
  Job* J = (Job*)arg;
  for (uint32_t ab = 1 + (uint32_t)J->t; ab < 0x7F80u; ab += (uint32_t)J->nt) {
    volatile float amax = f_of(ab << 16);
    volatile float d = amax / 448.0f;
    if (d >= 2.35098870e-38f) bracket(J, ab, d);  // 2^-125: the bracket's range
    if (d < 7.88860905e-31f) continue;  // 2^-100: not a multiplier block
    ++J->blocks;
    volatile float c0 = 1.0f / d;
    const float cand[3] = {c0, f_of(b_of(c0) + 1u), f_of(b_of(c0) - 1u)};
    int k = 0;
    while (k < 3 && !passes(d, cand[k])) ++k;
    if (k == 3) { ++J->none; continue; }
    ++J->chosen[k];
    const float c = cand[k];
    for (uint32_t vb = 0; vb <= ab; ++vb)
      for (int sg = 0; sg < 2; ++sg) {
        volatile float v = f_of((vb | (sg ? 0x8000u : 0u)) << 16);
        volatile float p = v * c, q = v / d;
        ++J->pairs;
        if (e4m3(p) != e4m3(q)) {
          if (J->bad < 5) printf("mismatch: amax bits %04x, v bits %04x\n", ab, vb | (sg ? 0x8000u : 0u));
          ++J->bad;
        }
      }
  }
  return NULL;
}

int main(int argc, char** argv) {
  int nt = argc > 1 ? atoi(argv[1]) : 8;
  if (nt < 1 || nt > 64) nt = 8;
  init_mag();
  pthread_t th[64];
  Job job[64];
  memset(job, 0, sizeof job);
  for (int t = 0; t < nt; ++t) {
    job[t].t = t;
    job[t].nt = nt;
    pthread_create(&th[t], NULL, run, &job[t]);
  }
  long long blocks = 0, chosen[3] = {0, 0, 0}, none = 0, pairs = 0, bad = 0;
  long long bpairs = 0, straddles = 0, bbad = 0;
  for (int t = 0; t < nt; ++t) {
    pthread_join(th[t], NULL);
    blocks += job[t].blocks;
    for (int k = 0; k < 3; ++k) chosen[k] += job[t].chosen[k];
    none += job[t].none;
    pairs += job[t].pairs;
    bad += job[t].bad;
    bpairs += job[t].bracket_pairs;
    straddles += job[t].straddles;
    bbad += job[t].bracket_bad;
  }
  printf("blocks %lld rn %lld up %lld down %lld none %lld pairs %lld mismatches %lld "
         "bracket_pairs %lld straddles %lld bracket_mismatches %lld\n",
         blocks, chosen[0], chosen[1], chosen[2], none, pairs, bad, bpairs, straddles, bbad);
  return bad != 0 || bbad != 0;
}
