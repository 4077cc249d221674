// topk.cuh -- exact Product-Softmax Top-K address search for one token, one thread.
//
// RAM-Net project page, Product Softmax paragraph and the exactness paragraph after the
// five views: a slot's weight is the product of its U digit probabilities, so the K
// best slots can be found one digit at a time, keeping the K best partial addresses per
// level and extending each by the d_p digit values.
//
// Ranking.  prod_u softmax(x_u)[d_u] = exp(sum_u x_u[d_u]) / prod_u Z_u, and prod_u Z_u
// is common to all slots, so slots rank by the sum of their digit logits.  Each logit is
// mapped to the integer q(x) = round_half_even(clamp(x, +-4095) * 2^32), which makes the
// sum exact and order independent.  A candidate is packed into one unsigned 64-bit word
//     P = (score + 2^47) << 16 | low,    low = (d_p^u - 1) - partial_index
// so that a larger P means a higher score, and on equal scores a lower partial index.
// |score| < 8 * 4095 * 2^32 < 2^47 and partial indices are < M <= 2^16, so the fields
// never overlap.  Extending P by digit d gives
//     (score + q_d + 2^47) << 16 | (low * d_p + d_p - 1 - d),
// computed as P + low*(d_p-1) + e_d with e_d = (q_d << 16) + (d_p - 1 - d); this map is
// strictly increasing in P, so the candidates of one digit keep the order of the kept
// prefixes, and the level's Top-K is a d_p-way merge of sorted lists.
#pragma once

#include "common.cuh"

namespace ramnet {

constexpr uint64_t kKeyBias = 1ull << 47;
constexpr float kInvScale = 2.3283064365386963e-10f;  // 2^-32

__device__ __forceinline__ int64_t digit_score(float x)
{
    x = fminf(fmaxf(x, -4095.0f), 4095.0f);  // fmaxf returns -4095 for NaN
    return __float2ll_rn(x * 4294967296.0f);  // exact scaling, round half to even
}

// Bring the token's logit row (U*d_p elements from element `off`) into L1 before the search
// reads it level by level, so the U levels do not each wait for a DRAM round trip.
__device__ __forceinline__ void prefetch_logits(const void* logits, size_t off, int is_bf16, int L)
{
    const char* b = static_cast<const char*>(logits) + off * (is_bf16 ? 2 : 4);
    const char* e = b + static_cast<size_t>(L) * (is_bf16 ? 2 : 4) - 1;
    asm volatile("prefetch.global.L1 [%0];" ::"l"(b));
    if ((reinterpret_cast<uintptr_t>(b) >> 7) != (reinterpret_cast<uintptr_t>(e) >> 7))
        asm volatile("prefetch.global.L1 [%0];" ::"l"(e));
}

__device__ __forceinline__ uint64_t digit_code(float x, int d, int d_p)
{
    return (static_cast<uint64_t>(digit_score(x)) << 16) + static_cast<uint64_t>(d_p - 1 - d);
}

// Exact Top-K of one token.  Logits are read as elements [off, off + U*d_p) of `logits`
// (fp32 or bf16).  `kept` is this thread's scratch list in shared memory: KMAX words at
// stride `stride` (words).  On return out[0..K) hold the packed winners, best first.
template <int KMAX, int DPMAX>
__device__ __forceinline__ void topk_search(const void* logits, size_t off, int is_bf16, int d_p, int U, int K,
                                            uint64_t* kept, int stride, uint64_t (&out)[KMAX])
{
    prefetch_logits(logits, off, is_bf16, U * d_p);
    int nk = 1;
    kept[0] = kKeyBias << 16;  // the empty prefix: score 0, low 0
    for (int u = 0; u < U; ++u) {
        // digit codes of this level, sorted best first (ties: lower digit first)
        uint64_t e[DPMAX];
#pragma unroll
        for (int d = 0; d < DPMAX; ++d) e[d] = d < d_p ? digit_code(load_in(logits, off + u * d_p + d, is_bf16), d, d_p) : 0ull;
#pragma unroll
        for (int i = 1; i < DPMAX; ++i)
#pragma unroll
            for (int j = i; j > 0; --j)
                if (e[j] > e[j - 1]) {
                    uint64_t t = e[j];
                    e[j] = e[j - 1];
                    e[j - 1] = t;
                }
        // d_p-way merge: list j = kept prefixes (best first) extended by digit e[j]
        const uint64_t mul = static_cast<uint64_t>(d_p - 1);
        int h[DPMAX];
        uint64_t c[DPMAX];
        {
            const uint64_t p0 = kept[0];
            const uint64_t f0 = p0 + (p0 & 0xFFFFull) * mul;
#pragma unroll
            for (int j = 0; j < DPMAX; ++j) {
                h[j] = 0;
                c[j] = j < d_p ? f0 + e[j] : 0ull;
            }
        }
        const int n_out = min(K, nk * d_p);
#pragma unroll
        for (int s = 0; s < KMAX; ++s) {
            if (s < n_out) {
                uint64_t best = c[0];
                int bj = 0;
#pragma unroll
                for (int j = 1; j < DPMAX; ++j)
                    if (c[j] > best) {
                        best = c[j];
                        bj = j;
                    }
                out[s] = best;
                int hb = 0;
                uint64_t eb = 0;
#pragma unroll
                for (int j = 0; j < DPMAX; ++j)
                    if (j == bj) {
                        hb = h[j] + 1;
                        eb = e[j];
                    }
                uint64_t nv = 0;
                if (hb < nk) {
                    const uint64_t p = kept[hb * stride];
                    nv = p + (p & 0xFFFFull) * mul + eb;
                }
#pragma unroll
                for (int j = 0; j < DPMAX; ++j)
                    if (j == bj) {
                        h[j] = hb;
                        c[j] = nv;
                    }
            }
        }
        if (u + 1 < U) {
#pragma unroll
            for (int s = 0; s < KMAX; ++s)
                if (s < n_out) kept[s * stride] = out[s];
        }
        nk = n_out;
    }
}

// Compare-exchange keeping the larger word in a.
__host__ __device__ __forceinline__ void cx_desc(uint64_t& a, uint64_t& b)
{
    const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
    a = hi;
    b = lo;
}

// The N largest of two descending lists of N, descending, into a: the element-wise
// maximum of a and reversed b is a bitonic sequence holding the N largest, and a bitonic
// merge sorts it.
template <int N>
__host__ __device__ __forceinline__ void merge_top(uint64_t (&a)[N], const uint64_t (&b)[N])
{
#pragma unroll
    for (int i = 0; i < N; ++i) a[i] = a[i] > b[N - 1 - i] ? a[i] : b[N - 1 - i];
#pragma unroll
    for (int d = N / 2; d > 0; d >>= 1)
#pragma unroll
        for (int i = 0; i < N; ++i)
            if ((i & d) == 0) cx_desc(a[i], a[i + d]);
}

// Both descending lists of N merged into one descending list of 2N: a followed by reversed
// b is bitonic, and the bitonic merge of size 2N sorts it.
template <int N>
__host__ __device__ __forceinline__ void merge_full(const uint64_t (&a)[N], const uint64_t (&b)[N], uint64_t (&out)[2 * N])
{
#pragma unroll
    for (int i = 0; i < N; ++i) {
        out[i] = a[i];
        out[N + i] = b[N - 1 - i];
    }
#pragma unroll
    for (int d = N; d > 0; d >>= 1)
#pragma unroll
        for (int i = 0; i < 2 * N; ++i)
            if ((i & d) == 0) cx_desc(out[i], out[i + d]);
}

constexpr int pow2_at_least(int x) { return x <= 1 ? 1 : 2 * pow2_at_least((x + 1) / 2); }
constexpr int int_max(int a, int b) { return a > b ? a : b; }

// Pruned merge of one level.  With the digit codes e sorted best first and the extended
// kept prefixes f best first, candidate (i, j) = f[i] + e[j] is beaten by every (i', j')
// with i' <= i, j' <= j, so it can be among the N best only if (i + 1)(j + 1) <= N: digit
// list j needs only its first N / (j + 1) entries, and lists j >= N none.  The N best form
// a staircase (n_0 >= n_1 >= ... entries taken from lists 0, 1, ...), so of DE lists the
// lists j..DE-1 together hold at most N (DE - j) / DE of them.  The lists are merged from
// the last one backwards, each partial result cut to that bound.  Sizes are powers of two;
// missing entries are 0, below every real candidate word.  DP is the size of e, DE =
// min(DP, N) the number of lists that can contribute.
template <int N, int DP, int DE, int J>
struct TailMerge {
    static constexpr int LEN = pow2_at_least(int_max(1, N / (J + 1)));  // entries of list J used
    static constexpr int SUB = TailMerge<N, DP, DE, J + 1>::SZ;            // size of the merged lists J+1..DE-1
    static constexpr int X = LEN > SUB ? LEN : SUB;
    static constexpr int CAP = pow2_at_least(int_max(1, N * (DE - J) / DE));
    static constexpr bool FULL = 2 * X <= CAP;
    static constexpr int SZ = FULL ? 2 * X : X;

    __host__ __device__ __forceinline__ static void run(const uint64_t (&f)[N], int nk, const uint64_t (&e)[DP], int d_p,
                                                        uint64_t (&out)[SZ])
    {
        uint64_t sub[X];
        {
            uint64_t s[SUB];
            TailMerge<N, DP, DE, J + 1>::run(f, nk, e, d_p, s);
#pragma unroll
            for (int i = 0; i < X; ++i) sub[i] = i < SUB ? s[i < SUB ? i : 0] : 0ull;
        }
        uint64_t lst[X];
#pragma unroll
        for (int i = 0; i < X; ++i) lst[i] = (i < LEN && i < nk && J < d_p) ? f[i < N ? i : 0] + e[J] : 0ull;
        if constexpr (FULL) {
            merge_full<X>(lst, sub, out);
        } else {
#pragma unroll
            for (int i = 0; i < X; ++i) out[i] = lst[i];
            merge_top<X>(out, sub);
        }
    }
};

template <int N, int DP, int DE>
struct TailMerge<N, DP, DE, DE - 1> {
    static constexpr int LEN = pow2_at_least(int_max(1, N / DE));
    static constexpr int SZ = LEN;
    __host__ __device__ __forceinline__ static void run(const uint64_t (&f)[N], int nk, const uint64_t (&e)[DP], int d_p,
                                                        uint64_t (&out)[SZ])
    {
#pragma unroll
        for (int i = 0; i < LEN; ++i) out[i] = (i < nk && DE - 1 < d_p) ? f[i < N ? i : 0] + e[DE - 1] : 0ull;
    }
};

// Digit codes of one level sorted best first.  A code is (score << 16) + (d_p - 1 - d) taken
// as a signed 64-bit number, so that signed order is (score, lower digit) order; digits
// d >= d_p get INT64_MIN and sort last.  Bitonic sort, DPMAX a power of two.
template <int DPMAX>
__host__ __device__ __forceinline__ void sort_codes_desc(uint64_t (&e)[DPMAX])
{
#pragma unroll
    for (int k = 2; k <= DPMAX; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < DPMAX; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const int64_t a = static_cast<int64_t>(e[i]), b = static_cast<int64_t>(e[l]);
                    const bool swap = ((i & k) == 0) ? (a < b) : (a > b);
                    if (swap) {
                        e[i] = static_cast<uint64_t>(b);
                        e[l] = static_cast<uint64_t>(a);
                    }
                }
            }
}

// One level of the search with the kept list in registers (N >= K, a power of two).  `e`
// holds this level's digit codes sorted best first (sort_codes_desc), `kept` the nk best
// prefixes of the previous level, best first, 0 beyond nk.  On return kept holds the N best
// candidates of the level, best first (0 where there are fewer).
template <int N, int DPMAX>
__host__ __device__ __forceinline__ void topk_level_net(uint64_t (&kept)[N], int nk, const uint64_t (&e)[DPMAX], int d_p)
{
    const uint64_t mul = static_cast<uint64_t>(d_p - 1);
    uint64_t f[N];
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = kept[i] + (kept[i] & 0xFFFFull) * mul;
    TailMerge<N, DPMAX, (DPMAX < N ? DPMAX : N), 0>::run(f, nk, e, d_p, kept);
}

// Exact Top-K (K <= N) with the kept list in registers: the same result as topk_search,
// since the candidate words are distinct and the N best are therefore unique.  Level 0's
// candidates are the empty prefix extended by each digit, i.e. the sorted digit codes.
template <int N, int DPMAX>
__device__ __forceinline__ void topk_search_net(const void* logits, size_t off, int is_bf16, int d_p, int U, int K,
                                                uint64_t (&out)[N])
{
    prefetch_logits(logits, off, is_bf16, U * d_p);
    uint64_t kept[N];
    int nk;
    {
        uint64_t e[DPMAX];
#pragma unroll
        for (int d = 0; d < DPMAX; ++d)
            e[d] = d < d_p ? digit_code(load_in(logits, off + d, is_bf16), d, d_p) : 0x8000000000000000ull;
        sort_codes_desc<DPMAX>(e);
        nk = min(K, d_p);
#pragma unroll
        for (int i = 0; i < N; ++i) kept[i] = (i < DPMAX && i < nk) ? (kKeyBias << 16) + e[i < DPMAX ? i : 0] : 0ull;
    }
    for (int u = 1; u < U; ++u) {
        uint64_t e[DPMAX];
#pragma unroll
        for (int d = 0; d < DPMAX; ++d)
            e[d] = d < d_p ? digit_code(load_in(logits, off + u * d_p + d, is_bf16), d, d_p) : 0x8000000000000000ull;
        sort_codes_desc<DPMAX>(e);
        topk_level_net<N, DPMAX>(kept, nk, e, d_p);
        nk = min(K, nk * d_p);
#pragma unroll
        for (int i = 0; i < N; ++i)
            if (i >= nk) kept[i] = 0ull;  // only the K best prefixes are kept
    }
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = kept[i];
}

// Winner j's slot index (before CAPE) and score.
__device__ __forceinline__ int32_t packed_index(uint64_t p, int32_t M) { return (M - 1) - static_cast<int32_t>(p & 0xFFFFull); }
__device__ __forceinline__ int64_t packed_score(uint64_t p) { return static_cast<int64_t>((p >> 16) - kKeyBias); }

// Weights of the K winners (rank order) per the page's Product Softmax: renorm != 0 gives
// exp(s_j - s_0) / sum_k exp(s_k - s_0); renorm == 0 gives prod_u softmax(x_u)[d_u] =
// exp(s_j - sum_u logsumexp(x_u)).  s_j - s_0 is taken exactly from the integer scores.
template <int KMAX>
__device__ __forceinline__ void topk_weights(const uint64_t (&out)[KMAX], int K, int renorm, const void* logits,
                                             size_t off, int is_bf16, int d_p, int U, float (&w)[KMAX])
{
    const int64_t s0 = packed_score(out[0]);
    float base = 0.0f;
    if (!renorm) {
        float lse = 0.0f;
        for (int u = 0; u < U; ++u) {
            float mx = -INFINITY;
            for (int d = 0; d < d_p; ++d) mx = fmaxf(mx, fminf(fmaxf(load_in(logits, off + u * d_p + d, is_bf16), -4095.f), 4095.f));
            float z = 0.0f;
            for (int d = 0; d < d_p; ++d)
                z += expf(fminf(fmaxf(load_in(logits, off + u * d_p + d, is_bf16), -4095.f), 4095.f) - mx);
            lse += mx + logf(z);
        }
        base = static_cast<float>(s0) * kInvScale - lse;
    }
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < K) {
            const float dj = static_cast<float>(packed_score(out[j]) - s0) * kInvScale;
            w[j] = expf(base + dj);
            sum += w[j];
        } else {
            w[j] = 0.0f;
        }
    }
    if (renorm) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) w[j] = w[j] / sum;
    }
}

// Gated Sparse Update, step 1 (retention): (1 - w)^(g/(1-g)) with the write gate g
// clamped to [0,1] (NaN -> 0); 1 when w <= 0 or g == 0, 0 when w >= 1 or g == 1.
__device__ __forceinline__ float gsu_alpha(float w, float g)
{
    g = fminf(fmaxf(g, 0.0f), 1.0f);
    const float c = g / (1.0f - g);
    if (w <= 0.0f || c <= 0.0f) return 1.0f;
    if (w >= 1.0f) return 0.0f;
    return expf(c * log1pf(-w));
}

// CAPE: (idx + pos) mod M, pos any 64-bit position.
__device__ __forceinline__ int32_t cape_shift(int32_t idx, int64_t pos, int32_t M)
{
    int64_t pm = pos % M;
    if (pm < 0) pm += M;
    int64_t r = idx + pm;
    if (r >= M) r -= M;
    return static_cast<int32_t>(r);
}

}  // namespace ramnet
