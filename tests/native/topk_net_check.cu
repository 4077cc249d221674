// Host-side check of the register Top-K level merge (sort_codes_desc + topk_level_net in
// topk.cuh, the pruned merge tree) against a plain sort of all candidates.  Built and run by tests/test_topk_net_host.py; prints
// "checked <n> mismatches <m>" and exits non-zero on any mismatch.
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <random>
#include <vector>

#include "../../sparse_slot_recurrent_b200/csrc/topk.cuh"

template <int N, int DPMAX>
static long check(std::mt19937_64& rng, long trials, long& n)
{
    long bad = 0;
    for (long trial = 0; trial < trials; ++trial) {
        const int d_p = 2 + static_cast<int>(rng() % (DPMAX - 1));
        const int K = 1 + static_cast<int>(rng() % N);
        const int nk = 1 + static_cast<int>(rng() % K);
        // distinct kept words, descending (score field well inside the packed range)
        std::vector<uint64_t> kv;
        while (static_cast<int>(kv.size()) < nk) {
            const uint64_t sc = (rng() % 2000000) + (1ull << 40);
            const uint64_t w = (sc << 16) | (rng() % 4096);
            if (std::find(kv.begin(), kv.end(), w) == kv.end()) kv.push_back(w);
        }
        std::sort(kv.rbegin(), kv.rend());
        uint64_t kept[N] = {0};
        for (int i = 0; i < nk; ++i) kept[i] = kv[i];
        // digit codes, with repeated scores to exercise the index tie-break
        uint64_t e[DPMAX];
        for (int d = 0; d < DPMAX; ++d) e[d] = 0x8000000000000000ull;  // digits beyond d_p
        for (int d = 0; d < d_p; ++d) {
            int64_t q = static_cast<int64_t>(rng() % 200001) - 100000;
            if (d > 0 && rng() % 6 == 0) q = static_cast<int64_t>(e[d - 1]) >> 16;
            e[d] = (static_cast<uint64_t>(q) << 16) + static_cast<uint64_t>(d_p - 1 - d);
        }
        std::vector<uint64_t> cand;
        for (int i = 0; i < nk; ++i)
            for (int d = 0; d < d_p; ++d)
                cand.push_back(kept[i] + (kept[i] & 0xFFFFull) * static_cast<uint64_t>(d_p - 1) + e[d]);
        std::sort(cand.rbegin(), cand.rend());
        const int nout = std::min(K, nk * d_p);
        ramnet::sort_codes_desc<DPMAX>(e);
        ramnet::topk_level_net<N, DPMAX>(kept, nk, e, d_p);
        for (int i = 0; i < nout; ++i) {
            ++n;
            if (kept[i] != cand[i]) ++bad;
        }
    }
    return bad;
}

int main()
{
    std::mt19937_64 rng(12345);
    long n = 0, bad = 0;
    bad += check<8, 4>(rng, 20000, n);
    bad += check<8, 8>(rng, 20000, n);
    bad += check<16, 4>(rng, 20000, n);
    bad += check<16, 8>(rng, 20000, n);
    bad += check<16, 16>(rng, 20000, n);
    bad += check<8, 16>(rng, 20000, n);
    bad += check<32, 4>(rng, 20000, n);
    bad += check<32, 8>(rng, 10000, n);
    std::printf("checked %ld mismatches %ld\n", n, bad);
    return bad != 0;
}
