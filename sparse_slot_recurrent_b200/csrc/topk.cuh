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

// One level of the search with the kept list in registers (N = 8 or 16 >= K).  Digit j's
// candidates f_i + e_j (f_i the extended kept prefix i < nk, descending in i) form a
// descending list; invalid entries are 0, below every real candidate (a real word is at
// least 2^48).  The lists are merged one after another into the N best, descending.
template <int N, int DPMAX>
__host__ __device__ __forceinline__ void topk_level_net(uint64_t (&kept)[N], int nk, const uint64_t (&e)[DPMAX], int d_p)
{
    const uint64_t mul = static_cast<uint64_t>(d_p - 1);
    uint64_t f[N];
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = kept[i] + (kept[i] & 0xFFFFull) * mul;
    uint64_t acc[N];
#pragma unroll
    for (int i = 0; i < N; ++i) acc[i] = i < nk ? f[i] + e[0] : 0ull;
#pragma unroll
    for (int j = 1; j < DPMAX; ++j) {
        if (j < d_p) {
            uint64_t l[N];
#pragma unroll
            for (int i = 0; i < N; ++i) l[i] = i < nk ? f[i] + e[j] : 0ull;
            merge_top<N>(acc, l);
        }
    }
#pragma unroll
    for (int i = 0; i < N; ++i) kept[i] = acc[i];
}

// Exact Top-K (K <= N) with the kept list in registers: the same result as topk_search,
// since the candidate words are distinct and the N best are therefore unique.
template <int N, int DPMAX>
__device__ __forceinline__ void topk_search_net(const void* logits, size_t off, int is_bf16, int d_p, int U, int K,
                                                uint64_t (&out)[N])
{
    uint64_t kept[N];
    kept[0] = kKeyBias << 16;  // the empty prefix: score 0, low 0
#pragma unroll
    for (int i = 1; i < N; ++i) kept[i] = 0ull;
    int nk = 1;
    for (int u = 0; u < U; ++u) {
        uint64_t e[DPMAX];
#pragma unroll
        for (int d = 0; d < DPMAX; ++d) e[d] = d < d_p ? digit_code(load_in(logits, off + u * d_p + d, is_bf16), d, d_p) : 0ull;
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
