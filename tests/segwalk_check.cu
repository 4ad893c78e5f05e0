// Host-side check of the tensor-core kernel's work split (SegWalk and
// split_owners, compiled from the kernel's own header for the host): for many
// tile counts, chunk counts and grid sizes (one CTA per SM, and T * (SMs div
// T) CTAs when there are fewer tiles T than SMs), every (tile, K chunk) unit is
// walked by exactly one CTA, the CTAs' unit counts differ by at most one,
// segments stay inside one tile, and for every tile walked by more than one
// CTA the owner range [bf, bl] is exactly its set of contributors, with a
// distinct first owner per split tile (it indexes the arrival counter).
// Prints "ok" and exits 0, or prints the first violation and exits 1.
#include <cstdio>
#include <cstdint>
#include <map>
#include <set>
#include <vector>

#include "tc_gemm.cuh"

using sherry::tc::Params;
using sherry::tc::SegWalk;
using sherry::tc::split_owners;

static int check(int64_t TM, int64_t TN, int64_t Kc, int64_t G0)
{
    Params p{};
    p.TM = TM;
    p.TN = TN;
    p.Kc = Kc;
    p.U = TM * TN * Kc;
    const int64_t G = G0 < p.U ? G0 : p.U;
    std::vector<int64_t> owner(p.U, -1);
    int64_t lo = INT64_MAX, hi = 0;
    for (int64_t b = 0; b < G; ++b) {
        int64_t units = 0;
        for (SegWalk w(p, b, G); !w.done(); w.next()) {
            if (w.tile < 0 || w.tile >= TM * TN || w.cb < 0 || w.cb >= w.ce || w.ce > Kc) {
                std::printf("bad segment TM=%lld TN=%lld Kc=%lld G=%lld b=%lld\n", (long long)TM, (long long)TN,
                            (long long)Kc, (long long)G, (long long)b);
                return 1;
            }
            for (int64_t c = w.cb; c < w.ce; ++c) {
                int64_t& o = owner[w.tile * Kc + c];
                if (o != -1) {
                    std::printf("unit walked twice TM=%lld TN=%lld Kc=%lld G=%lld\n", (long long)TM, (long long)TN,
                                (long long)Kc, (long long)G);
                    return 1;
                }
                o = b;
                ++units;
            }
        }
        lo = units < lo ? units : lo;
        hi = units > hi ? units : hi;
    }
    for (int64_t u = 0; u < p.U; ++u)
        if (owner[u] == -1) {
            std::printf("unit not walked TM=%lld TN=%lld Kc=%lld G=%lld\n", (long long)TM, (long long)TN,
                        (long long)Kc, (long long)G);
            return 1;
        }
    if (hi - lo > 1) {
        std::printf("unbalanced (%lld..%lld) TM=%lld TN=%lld Kc=%lld G=%lld\n", (long long)lo, (long long)hi,
                    (long long)TM, (long long)TN, (long long)Kc, (long long)G);
        return 1;
    }
    std::set<int64_t> firsts;
    for (int64_t t = 0; t < TM * TN; ++t) {
        std::set<int64_t> contrib;
        for (int64_t c = 0; c < Kc; ++c) contrib.insert(owner[t * Kc + c]);
        if (contrib.size() < 2) continue;
        int64_t bf = 0, bl = 0;
        split_owners(p, t, G, &bf, &bl);
        std::set<int64_t> range;
        for (int64_t b = bf; b <= bl; ++b) range.insert(b);
        if (range != contrib || !firsts.insert(bf).second) {
            std::printf("owner range wrong TM=%lld TN=%lld Kc=%lld G=%lld tile=%lld\n", (long long)TM,
                        (long long)TN, (long long)Kc, (long long)G, (long long)t);
            return 1;
        }
    }
    return 0;
}

int main()
{
    const int64_t tms[] = {1, 2, 3, 16, 64};
    const int64_t tns[] = {1, 2, 32, 112, 149};
    const int64_t kcs[] = {1, 2, 5, 7, 32, 112};
    const int64_t smss[] = {148, 132, 5, 1};
    int n = 0;
    for (int64_t TM : tms)
        for (int64_t TN : tns)
            for (int64_t Kc : kcs)
                for (int64_t sms : smss) {
                    // one CTA per SM, and the launch's grid for few tiles:
                    // T * (SMs div T) when T < SMs
                    const int64_t T = TM * TN;
                    if (check(TM, TN, Kc, sms)) return 1;
                    if (T < sms && check(TM, TN, Kc, T * (sms / T))) return 1;
                    n += T < sms ? 2 : 1;
                }
    std::printf("ok %d shapes\n", n);
    return 0;
}
