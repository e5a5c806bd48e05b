/* Exhaustive check of the oracle's E4M3 encoder: every binary32 bit pattern whose
 * magnitude is at most 480 (both signs: about 2.3e9 values, the whole
 * round-to-nearest range plus the saturation band above 448), against a nearest-
 * value search written from the OCP E4M3 definition (codes E<<3 | m: E == 0 gives
 * m * 2^-9, else (1 + m/8) * 2^(E-7); 0x7F is NaN).  Ties go to the even code;
 * magnitudes above 448 saturate to 448 (0x7E); the sign bit is kept (-0 -> 0x80).
 *
 * Test infrastructure: built and run by tests/test_oracle_e4m3_sweep.py against
 * oracle/libep_oracle.so.  Prints the number of patterns checked and of
 * mismatches (with the first few) and exits non-zero on any mismatch. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

uint8_t oracle_e4m3_from_f32(float v);

static double table[127]; /* magnitude of code c, c = 0 .. 0x7E, increasing */

static void build_table(void) {
    for (int c = 0; c < 127; ++c) {
        const int E = c >> 3, m = c & 7;
        double v;
        if (E == 0) {
            v = m / 512.0; /* m * 2^-9 */
        } else {
            v = 1.0 + m / 8.0;
            for (int i = 0; i < E - 7; ++i) v *= 2.0;
            for (int i = 0; i < 7 - E; ++i) v /= 2.0;
        }
        table[c] = v;
    }
}

/* nearest code of a non-negative magnitude a <= 480 */
static uint8_t nearest(double a) {
    if (a > 448.0) return 0x7E;
    int lo = 0, hi = 126; /* largest c with table[c] <= a, by bisection */
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (table[mid] <= a) lo = mid; else hi = mid - 1;
    }
    if (lo == 126 || table[lo] == a) return (uint8_t)lo;
    const double dl = a - table[lo], dh = table[lo + 1] - a; /* exact in binary64 */
    if (dl < dh) return (uint8_t)lo;
    if (dh < dl) return (uint8_t)(lo + 1);
    return (uint8_t)((lo & 1) == 0 ? lo : lo + 1); /* tie: the even code */
}

int main(void) {
    build_table();
    float f480 = 480.0f;
    uint32_t top;
    memcpy(&top, &f480, 4);
    long long checked = 0, bad = 0;
#pragma omp parallel for schedule(static, 1 << 16) reduction(+ : checked, bad)
    for (long long i = 0; i <= (long long)top; ++i) {
        for (int s = 0; s < 2; ++s) {
            const uint32_t u = (uint32_t)i | ((uint32_t)s << 31);
            float v;
            memcpy(&v, &u, 4);
            double a = (double)v;
            if (a < 0) a = -a;
            const uint8_t want = (uint8_t)(nearest(a) | (s ? 0x80 : 0x00));
            const uint8_t got = oracle_e4m3_from_f32(v);
            ++checked;
            if (got != want) {
                ++bad;
                if (bad <= 5) {
#pragma omp critical
                    printf("mismatch bits %08x value %.9g: oracle %02x, nearest %02x\n", u, v, got,
                           want);
                }
            }
        }
    }
    printf("checked %lld mismatches %lld\n", checked, bad);
    return bad == 0 ? 0 : 1;
}
