/*
 * ramnet_oracle.c -- plain, slow, double-precision CPU oracle for the RAM-Net layer core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: it exists so that tests/, the smoke check and the CPU-baseline leg of the
 * benchmark can compare the CUDA library against an independent statement of what the
 * method computes.  It shares no code, header, table or helper with the CUDA path.
 *
 * Source of every step: the RAM-Net project page ("RAM-Net: Linear-Time Sequence
 * Modeling with Sparsely Addressable State", muoncat.github.io/ramnet_web), cited below
 * by its paragraph names, and for the name of the decay form the "AI Radio" episode page
 * on the same paper.  The page prints no equations; where it is silent the reading taken
 * is named R1..R11 and stated at the function that uses it.
 *
 * Everything here is straight-line loops in double.  The only library routines used
 * are qsort, exp, log1p, sqrt and llrint.  There is no blocking, fusion or reordering
 * beyond what the page's description states.
 *
 * Pins (tests/test_oracle_pins.py): the digit factorisation against torch.softmax of the
 * summed logits, Top-K against fp64 products and against the level-by-level search, U = 1
 * against a stable sort, digit regrouping, a hand-worked 2x2 address, the CAPE
 * permutation and relative-position equivariance, the GSU limits g = 0 / g = 1 in closed
 * form, unselected slots bit-identical, bounded averages, read-after-write, the RMSNorm
 * identities and the page's state-access figures.
 * Parity unpinned (the page is silent, so no test can tell whether the authors chose the
 * same): the renormalisation of the K weights (R5), the CAPE stride and sign (R6), the
 * exact retention form (R7), and the two epsilon values (R8, R11).  The code that
 * implements each of these readings is itself pinned by the tests above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------------------
 * Reading R3: the ranking score of one digit value.
 *
 * Product Softmax paragraph: the weight of slot i is prod_u softmax(x_u)[d_u(i)].  Since
 * prod_u exp(x_u[d_u]) / Z_u = exp(sum_u x_u[d_u]) / prod_u Z_u and prod_u Z_u is the
 * same for every slot, ranking slots by that product is ranking them by the plain sum
 * of their digit logits.  To make that sum exact (so that "exact Top-K" and the
 * lower-index tie-break are well defined and identical for every search order), each
 * logit is put on the grid 2^-32 with round-half-to-even, after clamping to +-4095, and
 * summed as a 64-bit integer.  For bf16 logits with |x| >= 2^-25, and fp32 logits with
 * |x| >= 2^-9, the grid value is the logit itself, so the integer sum is the exact real
 * sum.  NaN ranks as -4095 (lowest).
 * ---------------------------------------------------------------------------------- */
#define RO_CLAMP 4095.0
#define RO_SCALE 4294967296.0 /* 2^32 */

int64_t ro_digit_score(double x)
{
    if (isnan(x)) x = -RO_CLAMP;
    if (x > RO_CLAMP) x = RO_CLAMP;
    if (x < -RO_CLAMP) x = -RO_CLAMP;
    return (int64_t)llrint(x * RO_SCALE); /* default rounding mode: nearest-even */
}

/* Reading R1 + R2: logits of one token are U contiguous groups of d_p scores, group u
 * holding digit u; group 0 is the most significant digit of the slot index
 *   i = sum_u d_u * d_p^(U-1-u)
 * (Product Softmax paragraph: "each slot index can be written as U digits with d_p
 * values each"; "Waveform Modulation": low-order digits change at every slot). */
static int digit_of(int64_t slot, int u, int d_p, int U)
{
    for (int k = U - 1; k > u; --k) slot /= d_p;
    return (int)(slot % d_p);
}

typedef struct {
    int64_t key;
    int64_t idx;
} ro_cand;

/* Reading R4: the better of two candidates has the larger score; equal scores are
 * ordered by the smaller (pre-shift) slot index. */
static int cand_cmp(const void* pa, const void* pb)
{
    const ro_cand* a = (const ro_cand*)pa;
    const ro_cand* b = (const ro_cand*)pb;
    if (a->key != b->key) return a->key > b->key ? -1 : 1;
    if (a->idx != b->idx) return a->idx < b->idx ? -1 : 1;
    return 0;
}

/* Top-K by brute force: score all M = d_p^U slots and sort them (Multilevel Decision
 * Tree paragraph: the naive selection "scores all M").  idx_out/key_out get K entries
 * in rank order. */
int ro_topk_bruteforce(const double* x, int d_p, int U, int K, int32_t* idx_out, int64_t* key_out)
{
    int64_t M = 1;
    for (int u = 0; u < U; ++u) M *= d_p;
    if (K < 1 || K > M) return -1;
    ro_cand* all = (ro_cand*)malloc(sizeof(ro_cand) * (size_t)M);
    if (!all) return -2;
    for (int64_t i = 0; i < M; ++i) {
        int64_t key = 0;
        for (int u = 0; u < U; ++u) key += ro_digit_score(x[u * d_p + digit_of(i, u, d_p, U)]);
        all[i].key = key;
        all[i].idx = i;
    }
    qsort(all, (size_t)M, sizeof(ro_cand), cand_cmp);
    for (int k = 0; k < K; ++k) {
        idx_out[k] = (int32_t)all[k].idx;
        if (key_out) key_out[k] = all[k].key;
    }
    free(all);
    return 0;
}

/* Top-K by the level-by-level prefix-tree search of the page's exactness paragraph
 * ("fixes the digits one level at a time and keeps only the K most probable partial
 * addresses at each level", evaluating K*d_p candidates per level).  Used only to
 * check that it returns the brute-force result. */
int ro_topk_tree(const double* x, int d_p, int U, int K, int32_t* idx_out, int64_t* key_out)
{
    int64_t M = 1;
    for (int u = 0; u < U; ++u) M *= d_p;
    if (K < 1 || K > M) return -1;
    ro_cand* kept = (ro_cand*)malloc(sizeof(ro_cand) * (size_t)K);
    ro_cand* cand = (ro_cand*)malloc(sizeof(ro_cand) * (size_t)K * (size_t)d_p);
    if (!kept || !cand) { free(kept); free(cand); return -2; }
    int nkept = 1;
    kept[0].key = 0; /* the empty prefix */
    kept[0].idx = 0;
    for (int u = 0; u < U; ++u) {
        int n = 0;
        for (int p = 0; p < nkept; ++p)
            for (int d = 0; d < d_p; ++d) {
                cand[n].key = kept[p].key + ro_digit_score(x[u * d_p + d]);
                cand[n].idx = kept[p].idx * d_p + d;
                ++n;
            }
        qsort(cand, (size_t)n, sizeof(ro_cand), cand_cmp);
        nkept = n < K ? n : K;
        memcpy(kept, cand, sizeof(ro_cand) * (size_t)nkept);
    }
    for (int k = 0; k < K; ++k) {
        idx_out[k] = (int32_t)kept[k].idx;
        if (key_out) key_out[k] = kept[k].key;
    }
    free(kept);
    free(cand);
    return 0;
}

/* Slot weights (Product Softmax paragraph): weight = product over digits of the
 * per-group softmax probability of the slot's digit.
 * Reading R5: with renorm != 0 the K selected weights are divided by their sum (the
 * Top-K truncated distribution, renormalised); with renorm == 0 they are the raw
 * product-softmax values. */
void ro_weights(const double* x, int d_p, int U, int K, const int32_t* idx, int renorm, double* w_out)
{
    double* prob = (double*)malloc(sizeof(double) * (size_t)U * (size_t)d_p);
    for (int u = 0; u < U; ++u) {
        double mx = -INFINITY;
        for (int d = 0; d < d_p; ++d) if (x[u * d_p + d] > mx) mx = x[u * d_p + d];
        double z = 0.0;
        for (int d = 0; d < d_p; ++d) z += exp(x[u * d_p + d] - mx);
        for (int d = 0; d < d_p; ++d) prob[u * d_p + d] = exp(x[u * d_p + d] - mx) / z;
    }
    double total = 0.0;
    for (int k = 0; k < K; ++k) {
        double p = 1.0;
        for (int u = 0; u < U; ++u) p *= prob[u * d_p + digit_of(idx[k], u, d_p, U)];
        w_out[k] = p;
        total += p;
    }
    if (renorm)
        for (int k = 0; k < K; ++k) w_out[k] /= total;
    free(prob);
}

/* Reading R6 (CAPE paragraphs): a token at absolute position pos has its read and write
 * slot indices shifted cyclically by +pos along the slot array, on heads whose CAPE flag
 * is set; "the shift only permutes slot indices". */
int64_t ro_cape(int64_t idx, int64_t pos, int64_t M)
{
    int64_t r = (idx + pos) % M;
    return r < 0 ? r + M : r;
}

/* Reading R7 (Gated Sparse Update, step 1 "Retention"; decay form named "Power Decay
 * Moving Average" on the AI Radio page): alpha = (1 - w)^c with c = e^gamma.  The gate
 * input is the activated g = sigmoid(gamma) in [0,1], so c = g / (1 - g).  Edge rules:
 * w <= 0 or c <= 0 -> 1; w >= 1 (with c > 0) -> 0; g is clamped to [0,1] (NaN -> 0). */
double ro_alpha(double w, double g)
{
    g = fmin(fmax(g, 0.0), 1.0);
    double c = g / (1.0 - g); /* g == 1 gives +inf */
    if (w <= 0.0 || c <= 0.0) return 1.0;
    if (w >= 1.0) return 0.0;
    return exp(c * log1p(-w));
}

typedef struct {
    int32_t d_p, U, K, d_v;
    double eps_gsu, eps_norm;
    int32_t renorm;
} ro_config;

static int64_t num_slots(const ro_config* c)
{
    int64_t M = 1;
    for (int u = 0; u < c->U; ++u) M *= c->d_p;
    return M;
}

/* Address decoder for one token of one head: Top-K (brute force), weights, then CAPE.
 * The returned indices are in rank order. */
static void decode_one(const ro_config* c, const double* x, int cape_on, int64_t pos,
                       int32_t* idx, double* w)
{
    int64_t M = num_slots(c);
    ro_topk_bruteforce(x, c->d_p, c->U, c->K, idx, NULL);
    ro_weights(x, c->d_p, c->U, c->K, idx, c->renorm, w);
    if (cape_on)
        for (int k = 0; k < c->K; ++k) idx[k] = (int32_t)ro_cape(idx[k], pos, M);
}

/* ro_decode_addresses: logits [B,T,H,U*d_p] -> idx, w [B,T,H,K]; token (b,t,h) sits at
 * position pos0[b] + t (pos0 NULL = 0); cape_mask [H] (NULL = CAPE off). */
int ro_decode_addresses(const ro_config* c, int B, int T, int H, const double* logits,
                        const int32_t* pos0, const uint8_t* cape_mask, int32_t* idx_out,
                        double* w_out)
{
    const int L = c->U * c->d_p;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                size_t th = ((size_t)b * T + t) * H + h;
                int64_t pos = (pos0 ? pos0[b] : 0) + (int64_t)t;
                decode_one(c, logits + th * L, cape_mask ? cape_mask[h] : 0, pos,
                           idx_out + th * c->K, w_out + th * c->K);
            }
    return 0;
}

/* One token of one head, given that head's state S [M,d_v] and mass m [M]:
 *   Address Decoder on key (write set) and query (read set), CAPE, then the Gated Sparse
 *   Update of each selected write slot, then the weighted read, RMSNorm and output gate.
 * Reading R8: eps in the update rate is cfg->eps_gsu.  Reading R10: the read uses the
 * state after this token's write (the page: GSU writes, "then" the read slots are
 * combined).  Reading R11: y = o / sqrt(mean(o^2) + eps_norm) * norm_w * z. */
static void token_step(const ro_config* c, const double* kx, const double* qx, const double* v,
                       double g, const double* z, const double* norm_w, int cape_on, int64_t pos,
                       double* S, double* m, double* y, int32_t* wi, double* ww, int32_t* ri,
                       double* rw, double* o)
{
    const int K = c->K, dv = c->d_v;
    decode_one(c, kx, cape_on, pos, wi, ww);
    decode_one(c, qx, cape_on, pos, ri, rw);

    /* Gated Sparse Update, steps 1-4, on the selected write slots only (distinct). */
    for (int k = 0; k < K; ++k) {
        int64_t i = wi[k];
        double w = ww[k];
        double alpha = ro_alpha(w, g);                 /* 1. retention   */
        m[i] = alpha * m[i] + w;                       /* 2. mass        */
        double lam = w / (m[i] + c->eps_gsu);          /* 3. update rate */
        for (int d = 0; d < dv; ++d)                   /* 4. content     */
            S[i * dv + d] = S[i * dv + d] + lam * (v[d] - S[i * dv + d]);
    }

    /* Sparse read: the K read slots combined by their weights. */
    for (int d = 0; d < dv; ++d) o[d] = 0.0;
    for (int k = 0; k < K; ++k)
        for (int d = 0; d < dv; ++d) o[d] += rw[k] * S[(int64_t)ri[k] * dv + d];

    /* RMSNorm over d_v, then the output gate. */
    double ms = 0.0;
    for (int d = 0; d < dv; ++d) ms += o[d] * o[d];
    double inv = 1.0 / sqrt(ms / dv + c->eps_norm);
    for (int d = 0; d < dv; ++d) y[d] = o[d] * inv * (norm_w ? norm_w[d] : 1.0) * z[d];
}

typedef struct {
    const ro_config* c;
    int B, T, H;
    const double *k, *q, *v, *g, *z, *norm_w;
    const uint8_t* cape_mask;
    const int32_t* pos0;
    const double *S_in, *m_in;
    double *y, *S_out, *m_out;
    int next;
    pthread_mutex_t lock;
} scan_job;

static void scan_unit(scan_job* j, int unit)
{
    const ro_config* c = j->c;
    const int b = unit / j->H, h = unit % j->H;
    const int T = j->T, H = j->H, L = c->U * c->d_p, K = c->K, dv = c->d_v;
    const int64_t M = num_slots(c);
    double* S = j->S_out + (size_t)unit * M * dv;
    double* m = j->m_out + (size_t)unit * M;
    if (j->S_in) memcpy(S, j->S_in + (size_t)unit * M * dv, sizeof(double) * M * dv);
    else memset(S, 0, sizeof(double) * M * dv);
    if (j->m_in) memcpy(m, j->m_in + (size_t)unit * M, sizeof(double) * M);
    else memset(m, 0, sizeof(double) * M);
    int32_t* wi = (int32_t*)malloc(sizeof(int32_t) * K);
    int32_t* ri = (int32_t*)malloc(sizeof(int32_t) * K);
    double* ww = (double*)malloc(sizeof(double) * K);
    double* rw = (double*)malloc(sizeof(double) * K);
    double* o = (double*)malloc(sizeof(double) * dv);
    const int cape_on = j->cape_mask ? j->cape_mask[h] : 0;
    for (int t = 0; t < T; ++t) {
        size_t th = ((size_t)b * T + t) * H + h;
        int64_t pos = (j->pos0 ? j->pos0[b] : 0) + (int64_t)t;
        token_step(c, j->k + th * L, j->q + th * L, j->v + th * dv, j->g[th], j->z + th * dv,
                   j->norm_w, cape_on, pos, S, m, j->y + th * dv, wi, ww, ri, rw, o);
    }
    free(wi); free(ri); free(ww); free(rw); free(o);
}

static void* scan_worker(void* arg)
{
    scan_job* j = (scan_job*)arg;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        int unit = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (unit >= j->B * j->H) break;
        scan_unit(j, unit);
    }
    return NULL;
}

/* ro_scan_forward: the prefill scan.  Per (b,h), tokens t = 0..T-1 in order.
 * Layouts (contiguous): k,q [B,T,H,U*d_p]; v,z,y [B,T,H,d_v]; g [B,T,H];
 * S [B,H,M,d_v]; m [B,H,M]; norm_w [d_v] or NULL (ones); cape_mask [H] or NULL (off);
 * pos0 [B] or NULL (0).  S_in/m_in NULL = zero initial state (reading R9).
 * nthreads <= 0 uses every online core; the (b,h) units are independent. */
int ro_scan_forward(const ro_config* c, int B, int T, int H, const double* k, const double* q,
                    const double* v, const double* g, const double* z, const double* norm_w,
                    const uint8_t* cape_mask, const int32_t* pos0, const double* S_in,
                    const double* m_in, double* y, double* S_out, double* m_out, int nthreads)
{
    scan_job j = {c, B, T, H, k, q, v, g, z, norm_w, cape_mask, pos0, S_in, m_in, y, S_out, m_out, 0};
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads > B * H) nthreads = B * H;
    if (nthreads < 1) nthreads = 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, scan_worker, &j);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j.lock);
    return 0;
}

/* ro_decode_step: one autoregressive token per (b,h) with the state updated in place
 * (GPU-execution paragraph: decoding accesses only the current token's slots).
 * k,q [B,H,U*d_p]; v,z,y [B,H,d_v]; g [B,H]; pos [B] = this token's position;
 * S [B,H,M,d_v], m [B,H,M] in/out.  head_begin/head_end select a subset of the B*H
 * (b,h) units (flattened as b*H + h) so that a bounded sample can be timed; units
 * outside it are left untouched. */
int ro_decode_step(const ro_config* c, int B, int H, const double* k, const double* q,
                   const double* v, const double* g, const double* z, const double* norm_w,
                   const uint8_t* cape_mask, const int32_t* pos, double* S, double* m, double* y,
                   int unit_begin, int unit_end)
{
    const int L = c->U * c->d_p, K = c->K, dv = c->d_v;
    const int64_t M = num_slots(c);
    int32_t* wi = (int32_t*)malloc(sizeof(int32_t) * K);
    int32_t* ri = (int32_t*)malloc(sizeof(int32_t) * K);
    double* ww = (double*)malloc(sizeof(double) * K);
    double* rw = (double*)malloc(sizeof(double) * K);
    double* o = (double*)malloc(sizeof(double) * dv);
    if (unit_end > B * H || unit_end < 0) unit_end = B * H;
    for (int unit = unit_begin; unit < unit_end; ++unit) {
        int b = unit / H, h = unit % H;
        token_step(c, k + (size_t)unit * L, q + (size_t)unit * L, v + (size_t)unit * dv, g[unit],
                   z + (size_t)unit * dv, norm_w, cape_mask ? cape_mask[h] : 0, pos ? pos[b] : 0,
                   S + (size_t)unit * M * dv, m + (size_t)unit * M, y + (size_t)unit * dv, wi, ww,
                   ri, rw, o);
    }
    free(wi); free(ri); free(ww); free(rw); free(o);
    return 0;
}
