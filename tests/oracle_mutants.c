/*
 * Planted mistakes for the oracle's pins (test-only).
 *
 * ssd_mutant_recurrence() is the oracle's sequential recurrence with ONE plausible
 * mistake, chosen by `which`.  test_oracle_pins.py runs every pin against each mutant
 * and requires at least one pin to fail, showing that the pins can tell a wrong
 * recurrence from the right one.  Nothing outside the tests builds or loads this file.
 *
 *   1  D x feedthrough dropped           2  decay exponent with the wrong sign
 *   3  y read from the state before the update   4  B and C swapped
 *   5  wrong head -> group map (h % G)   6  dt missing from the input term
 *   7  decay applied after the input is added    8  x indexed by the wrong head (h+1)
 */
#include <math.h>
#include <stdint.h>

int ssd_mutant_recurrence(int which, int64_t b, int64_t L, int64_t H, int64_t P, int64_t N,
                          int64_t G, const double *x, const double *dt, const double *A,
                          const double *B, const double *C, const double *D, double *state,
                          double *y) {
  if (H % G) return 1;
  for (int64_t bi = 0; bi < b; ++bi)
    for (int64_t h = 0; h < H; ++h) {
      const int64_t g = (which == 5) ? (h % G) : h / (H / G);
      const int64_t hx = (which == 8) ? (h + 1) % H : h;
      double *hs = state + (bi * H + h) * P * N;
      for (int64_t t = 0; t < L; ++t) {
        const double dtv = dt[(bi * L + t) * H + h];
        const double a = exp((which == 2 ? -1.0 : 1.0) * dtv * A[h]);
        const double *Bt = ((which == 4) ? C : B) + ((bi * L + t) * G + g) * N;
        const double *Ct = ((which == 4) ? B : C) + ((bi * L + t) * G + g) * N;
        for (int64_t p = 0; p < P; ++p) {
          const double xv = x[((bi * L + t) * H + hx) * P + p];
          double acc = 0.0;
          for (int64_t n = 0; n < N; ++n) {
            double *e = hs + p * N + n;
            const double in = (which == 6 ? 1.0 : dtv) * xv * Bt[n];
            if (which == 3) acc += Ct[n] * *e;
            if (which == 7)
              *e = a * (*e + in);
            else
              *e = a * *e + in;
            if (which != 3) acc += Ct[n] * *e;
          }
          y[((bi * L + t) * H + h) * P + p] = acc + (which == 1 ? 0.0 : D[h] * xv);
        }
      }
    }
  return 0;
}
