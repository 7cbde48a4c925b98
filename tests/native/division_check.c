/* Host check of the chunk quantizer's division: for finite x and a divisor d in [2^-96, 2^100],
 * the correctly rounded reciprocal y = RN(1/d) followed by two FMA remainder corrections
 * (Markstein 1990) and the sign of x,
 *     q0 = RN(x*y); r0 = RN(x - d*q0); q1 = RN(q0 + r0*y); r1 = RN(x - d*q1); q = RN(q1 + r1*y),
 * must equal RN(x/d) bit for bit where |x/d| >= 1/16 (where an E2M1 code can be nonzero), and
 * have |q| < 1/4 with the sign of x where |x/d| < 1/16 (code 0 of that sign on both sides).
 * Domain: every finite bf16 x; d = RN(e4m3(s) * a_g) for every positive finite E4M3 s, with
 * a_g = RN(amax / 2688) for the amax values given (quotients up to 64; the quantizer's reach
 * at most ~13).  Exit status 0 when no case differs.
 * Usage: division_check <n_amax> <seed> */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float e4m3(int b) {
    const int e = (b >> 3) & 15, m = b & 7;
    return e == 0 ? ldexpf((float)m, -9) : ldexpf(1.0f + m / 8.0f, e - 7);
}

int main(int argc, char** argv) {
    const int n_amax = argc > 1 ? atoi(argv[1]) : 8;
    srand(argc > 2 ? (unsigned)atoi(argv[2]) : 1u);
    unsigned long long checked = 0, bad = 0;
    for (int t = 0; t < n_amax; ++t) {
        float amax;
        if (t == 0) amax = 1.0f;
        else if (t == 1) amax = 3.3895e38f;
        else amax = ldexpf(1.0f + rand() / (float)RAND_MAX, rand() % 200 - 100);
        const float ag = amax / 2688.0f;
        for (int sb = 1; sb < 127; ++sb) {
            volatile float dv = e4m3(sb) * ag;
            const float d = dv;
            if (!(d >= 0x1p-96f && d <= 0x1p100f)) continue;
            const float y = 1.0f / d;
            for (uint32_t h = 0; h < 65536; ++h) {
                const float x = f_of(h << 16);
                if (!isfinite(x)) continue;
                const float ref = x / d;
                if (!(fabsf(ref) <= 64.0f)) continue;
                const float q0 = x * y;
                const float r0 = fmaf(-q0, d, x);
                const float q1 = fmaf(r0, y, q0);
                const float r1 = fmaf(-q1, d, x);
                const float q = copysignf(fmaf(r1, y, q1), x);
                ++checked;
                const int ok = fabsf(ref) < 0.0625f ? (fabsf(q) < 0.25f && signbit(q) == signbit(ref))
                                                     : (u_of(q) == u_of(ref));
                if (!ok) {
                    if (bad < 5) printf("differs: x=%a d=%a x/d=%a q=%a\n", x, d, ref, q);
                    ++bad;
                }
            }
        }
    }
    printf("checked %llu cases, %llu differ\n", checked, bad);
    return bad != 0;
}
