// log u, the log of the probability that a token is sampled, for the
// sampled-attention kernels.
#pragma once

#include <math.h>

namespace mp {

// u = P[Binomial(L, x) >= 2] is the probability that a key collides with the
// query in at least 2 of the L tables, x = p^K the per-table collision
// probability and p = 1 - arccos(c)/pi the SimHash per-bit collision
// probability at cosine c.  Small x: u = C(L,2) x^2 (1-x)^(L-2) (1 + a3 r (1 +
// a4 r (1 + a5 r (1 + a6 r)))) with r = x / (1-x), a_j = (L-j+1)/j (ratios of
// consecutive binomial terms), truncated after j = 6: the first dropped term,
// a3 a4 a5 a6 a7 r^5, is below 4e-7 for x < 1e-3 and L <= 255.  Otherwise
// u = 1 - exp(y), y = (L-1) log1p(-x) + log1p((L-1) x) (the closed form
// 1 - (1-x)^L - L x (1-x)^(L-1) rearranged so that expm1 keeps u's relative
// precision).
struct LogU {
    float K, L, lnC2, a3, a4, a5, a6;
};

// log u (natural log) at cosine c.  The plain log and exp are the hardware
// approximations (__logf, __expf: a few ulp, a few 1e-6 relative at these
// arguments), which moves log u by ~1e-5 at most, far inside the output
// tolerance; acos and the log1p / expm1 terms, where cancellation matters,
// keep the accurate library functions.  Both forms share one log1p of (-x) and one
// log1p of a form-dependent argument, so a warp whose lanes take different
// forms evaluates log1p twice, not three times.
__device__ __forceinline__ float log_sampling_prob(float c, const LogU &u)
{
    c = fminf(1.f, fmaxf(-1.f, c));
    float p = 1.f - acosf(c) * 0.318309886183790671538f;
    p = fmaxf(p, 1e-30f);
    const float lx = u.K * __logf(p);
    const float x = __expf(lx);
    const bool small = x < 1e-3f;
    const float r = __fdividef(x, 1.f - x);
    const float tail = u.a3 * r * (1.f + u.a4 * r * (1.f + u.a5 * r * (1.f + u.a6 * r)));
    const float l1 = log1pf(-x);
    const float l2 = log1pf(small ? tail : (u.L - 1.f) * x);
    if (small) return u.lnC2 + 2.f * lx + (u.L - 2.f) * l1 + l2;
    return __logf(-expm1f((u.L - 1.f) * l1 + l2));
}

}  // namespace mp
