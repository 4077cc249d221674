// decode_step.cu -- one autoregressive token per (b,h) against an HBM-resident state.
//
// RAM-Net project page, GPU-execution paragraph on decoding: the step touches only the
// slots its token selects and never scans the whole state.  Per (b,h) unit: decode the key
// and query addresses (Product Softmax Top-K + CAPE), apply the Gated Sparse Update to the
// K write rows of S and their masses, read the K read rows (after the write), RMSNorm,
// gate, store y.
//
// One CTA per SM, each over a contiguous range of units, in groups of kGroup units:
//   decoder warps  lane l decodes stream l / kGroup (key, query) of unit l % kGroup of a
//                  group: slots, weights and (writes) the retention alpha into a shared-
//                  memory ring of group slots; the two decoder warps take alternate groups,
//                  so all decodes of a CTA start at once;
//   row warps      row warp r takes unit r of every group: it loads the unit's K write
//                  rows and their K masses together (one DRAM round trip, K rows in flight
//                  per warp, lane l owning channels [l*CPL, l*CPL + CPL)), runs GSU steps
//                  1-4 and stores them, then loads the K read rows (a read row equal to a
//                  write row is the value this lane just stored: same address, program
//                  order), sums them by weight, RMSNorm, norm weight, gate, y.
// kRowWarps rows per lane in flight per warp and kRowWarps warps per SM keep about
// 128 KB of loads outstanding per SM, which is what HBM needs to run at its rate.
// Write rows of one unit are distinct slots (Top-K without repeats, CAPE a bijection).
// Group slots are handed over with mbarriers (bounded waits, timeout recorded in the
// status word).
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

constexpr int kGroup = 16;       // units per group = lanes per stream of a decoder warp
constexpr int kRowWarps = kGroup;
constexpr int kDecWarps = 2;
constexpr int kSlots = 4;        // group slots in the ring
constexpr int kStepThreads = (kRowWarps + kDecWarps) * 32;

__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(100000u)
        : "memory");
    return ok != 0;
}

// Bounded wait (about 2 s); on expiry records kDevTimeout and raises the CTA's abort flag.
// Between polls the thread sleeps (32 ns doubling to 512 ns), so the row warps waiting for a
// group leave the issue slots to the decoder warps.
__device__ __forceinline__ void step_wait(uint32_t bar, uint32_t parity, uint32_t* status, volatile int* abort_flag)
{
    if (mbar_try(bar, parity)) return;
    if (*abort_flag) return;
    const uint64_t t_end = now_ns() + 2000000000ull;
    uint32_t nap = 32;
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        if (mbar_try(bar, parity)) return;
        if (now_ns() > t_end || *abort_flag) break;
        __nanosleep(nap);
        nap = nap < 512 ? 2 * nap : 512;
    }
    *abort_flag = 1;
    set_status(status, kDevTimeout);
}

__device__ __forceinline__ void mbar_arrive_local(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One group slot: per unit the K write slots, weights and retentions, the K read slots and
// weights.
template <int KMAX>
struct GroupSlot {
    int32_t wi[kGroup][KMAX];
    float ww[kGroup][KMAX];
    float wa[kGroup][KMAX];
    int32_t ri[kGroup][KMAX];
    float rw[kGroup][KMAX];
};

template <int KMAX, int DPMAX, int CPL>
__global__ void __launch_bounds__(kStepThreads, 1) k_decode_step(StepParams p)
{
    constexpr int kRowBatch = CPL >= 8 ? 8 : 16;  // rows per lane in flight
    extern __shared__ __align__(16) unsigned char step_smem[];
    GroupSlot<KMAX>* ring = reinterpret_cast<GroupSlot<KMAX>*>(step_smem);
    // K > 32 only: the decoders' kept lists, [kDecWarps][KMAX][32]
    uint64_t* kept_s = reinterpret_cast<uint64_t*>(step_smem + sizeof(GroupSlot<KMAX>) * kSlots);
    __shared__ uint64_t full[kSlots], empty[kSlots];
    __shared__ int abort_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = p.K, dv = p.d_v, M = p.M;
    const int units = p.B * p.H;
    // this CTA's contiguous unit range and its groups
    const int u_beg = static_cast<int>((static_cast<long long>(units) * blockIdx.x) / gridDim.x);
    const int u_end = static_cast<int>((static_cast<long long>(units) * (blockIdx.x + 1)) / gridDim.x);
    const int ngroups = (u_end - u_beg + kGroup - 1) / kGroup;
    volatile int* abort_flag = &abort_s;

    if (tid == 0) {
        abort_s = 0;
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kRowWarps);
        }
        fence_mbar_init_cluster();
    }
    __syncthreads();

    if (warp >= kRowWarps) {
        // ------------------------------------------------------------ decoder warps
        const int dw = warp - kRowWarps;
        const int ul = lane & (kGroup - 1), stream = lane / kGroup;
        const int L = p.U * p.d_p;
        for (int g = dw; g < ngroups; g += kDecWarps) {
            const int slot = g % kSlots, use = g / kSlots;
            if (use >= 1) step_wait(smem_addr(&empty[slot]), (use - 1) & 1, p.status, abort_flag);
            const int bh = u_beg + g * kGroup + ul;
            if (bh < u_end && !*abort_flag) {
                const void* lg = stream == 0 ? p.k_logits : p.q_logits;
                const size_t off = static_cast<size_t>(bh) * L;
                uint64_t out[KMAX];
                if constexpr (KMAX <= 32)
                    topk_search_net<KMAX, DPMAX>(lg, off, p.in_bf16, p.d_p, p.U, K, out);  // kept list in registers
                else
                    topk_search<KMAX, DPMAX>(lg, off, p.in_bf16, p.d_p, p.U, K, kept_s + (dw * KMAX) * 32 + lane, 32,
                                             out);
                float w[KMAX];
                topk_weights<KMAX>(out, K, p.renorm, lg, off, p.in_bf16, p.d_p, p.U, w);
                const int h = bh % p.H, b = bh / p.H;
                const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
                const int32_t pm = cape ? cape_shift(0, p.pos != nullptr ? p.pos[b] : 0, M) : 0;
                const float gg = stream == 0 ? load_in(p.g, bh, p.in_bf16) : 0.0f;
                GroupSlot<KMAX>& gs = ring[slot];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < K) {
                        int32_t idx = packed_index(out[j], M) + pm;
                        if (idx >= M) idx -= M;
                        if (!dcheck(idx >= 0 && idx < M, p.status)) idx = 0;
                        if (stream == 0) {
                            gs.wi[ul][j] = idx;
                            gs.ww[ul][j] = w[j];
                            gs.wa[ul][j] = gsu_alpha(w[j], gg);
                        } else {
                            gs.ri[ul][j] = idx;
                            gs.rw[ul][j] = w[j];
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_local(smem_addr(&full[slot]));
        }
    } else {
        // ------------------------------------------------------------ row warps
        const int LW = (CPL > 1 || dv >= 32) ? 32 : dv;  // lanes holding channels
        const bool act = lane < LW;
        const int ch0 = (act ? lane : 0) * CPL;
        float nw[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) nw[c] = p.norm_w != nullptr ? p.norm_w[ch0 + c] : 1.0f;
        for (int g = 0; g < ngroups; ++g) {
            const int slot = g % kSlots, use = g / kSlots;
            step_wait(smem_addr(&full[slot]), use & 1, p.status, abort_flag);
            const int bh = u_beg + g * kGroup + warp;
            if (bh < u_end && !*abort_flag) {
                const GroupSlot<KMAX>& gs = ring[slot];
                float* S = p.S + static_cast<size_t>(bh) * M * dv;
                float* mrow = p.m + static_cast<size_t>(bh) * M;
                float vv[CPL], zz[CPL], o[CPL];
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    vv[c] = act ? load_in(p.v, static_cast<size_t>(bh) * dv + ch0 + c, p.in_bf16) : 0.0f;
                    zz[c] = act ? load_in(p.z, static_cast<size_t>(bh) * dv + ch0 + c, p.in_bf16) : 0.0f;
                    o[c] = 0.0f;
                }
                for (int j0 = 0; j0 < K; j0 += kRowBatch) {
                    // write rows and their masses in flight together; lane j owns mass j0 + j
                    float s[kRowBatch][CPL];
#pragma unroll
                    for (int k = 0; k < kRowBatch; ++k)
                        if (j0 + k < K && act) load_row_g<CPL>(S + static_cast<size_t>(gs.wi[warp][j0 + k]) * dv + ch0, s[k]);
                    const int jm = j0 + lane;
                    float lam = 0.0f;
                    if (lane < kRowBatch && jm < K) {
                        const int sl = gs.wi[warp][jm];
                        const float w = gs.ww[warp][jm];
                        const float mn = gs.wa[warp][jm] * mrow[sl] + w;  // GSU steps 1-2
                        mrow[sl] = mn;
                        lam = w / (mn + p.eps_gsu);  // step 3
                    }
#pragma unroll
                    for (int k = 0; k < kRowBatch; ++k) {
                        const float lk = __shfl_sync(0xffffffffu, lam, k);
                        if (j0 + k < K && act) {
#pragma unroll
                            for (int c = 0; c < CPL; ++c) s[k][c] = fmaf(lk, vv[c] - s[k][c], s[k][c]);  // step 4
                            store_row_g<CPL>(S + static_cast<size_t>(gs.wi[warp][j0 + k]) * dv + ch0, s[k]);
                        }
                    }
                }
                for (int j0 = 0; j0 < K; j0 += kRowBatch) {
                    float s[kRowBatch][CPL];
#pragma unroll
                    for (int k = 0; k < kRowBatch; ++k)
                        if (j0 + k < K && act) load_row_g<CPL>(S + static_cast<size_t>(gs.ri[warp][j0 + k]) * dv + ch0, s[k]);
#pragma unroll
                    for (int k = 0; k < kRowBatch; ++k) {
                        if (j0 + k < K && act) {
                            const float r = gs.rw[warp][j0 + k];
#pragma unroll
                            for (int c = 0; c < CPL; ++c) o[c] = fmaf(r, s[k][c], o[c]);
                        }
                    }
                }
                float ss = 0.0f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) ss = fmaf(o[c], o[c], ss);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = 1.0f / sqrtf(ss / dv + p.eps_norm);
                if (act) {
#pragma unroll
                    for (int c = 0; c < CPL; ++c)
                        store_out(p.y, static_cast<size_t>(bh) * dv + ch0 + c, o[c] * inv * nw[c] * zz[c], p.out_bf16);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_local(smem_addr(&empty[slot]));
        }
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_step(const StepParams& p, cudaStream_t s)
{
    int dev = 0, nsm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int units = p.B * p.H;
    // one CTA per SM, never fewer than one unit per CTA
    const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
    const size_t smem = sizeof(GroupSlot<KMAX>) * kSlots + (KMAX > 32 ? sizeof(uint64_t) * kDecWarps * KMAX * 32 : 0);
    void (*kern)(StepParams) = nullptr;
    switch (p.d_v < 32 ? 1 : p.d_v / 32) {
        case 1: kern = k_decode_step<KMAX, DPMAX, 1>; break;
        case 2: kern = k_decode_step<KMAX, DPMAX, 2>; break;
        case 4: kern = k_decode_step<KMAX, DPMAX, 4>; break;
        case 8: kern = k_decode_step<KMAX, DPMAX, 8>; break;
        default: return cudaErrorInvalidValue;
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kStepThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int DPMAX>
cudaError_t step_k(const StepParams& p, cudaStream_t s)
{
    if (p.K <= 8) return launch_step<8, DPMAX>(p, s);
    if (p.K <= 16) return launch_step<16, DPMAX>(p, s);
    if (p.K <= 32) return launch_step<32, DPMAX>(p, s);
    return launch_step<64, DPMAX>(p, s);
}


// ------------------------------------------------------------------ one warp per unit
//
// For K <= 16 and d_p <= 8 (the batched decode shapes) the step runs one warp per (b,h)
// unit, with every unit of the batch resident at once (4 warps per CTA, up to 7 CTAs per
// SM), so the address decode, the only long dependency chain of the step, takes one Top-K
// search of latency and not a queue of them.
//
// Address decode: lanes 0-15 search the key (write) addresses, lanes 16-31 the query (read)
// addresses, each 16-lane half on its own logits.  Lane i of a half holds the i-th best
// prefix of the current level (the packed 64-bit candidate word of the prefix-tree search).
// A level extends the kept prefixes by every digit: column j of the candidates is the kept
// list shifted by digit code e[j] (codes sorted best first), so every column is sorted, and
// the columns are merged pairwise by bitonic top-16 merges over warp shuffles (the element-
// wise maximum of one list and the other reversed is bitonic and holds the 16 best; a
// bitonic merge sorts it).  The kept words are distinct, so the 16 best, and the K best
// among them, are unique: the result equals the one-thread search of the other kernels.
// Then lane i computes winner i's weight, slot (after CAPE) and, for writes, retention.
//
// Rows: lane l owns channels [l*CPL, l*CPL + CPL) of every row; the K write rows are
// loaded kStepRows at a time, updated by GSU step 4 and stored, then the K read rows are
// loaded (a read row equal to a write row is the value this lane just stored: same address,
// program order) and summed by weight; RMSNorm, norm weight, gate, y.

constexpr int kWarpStepWarps = 4;

// top-16 (best first) of two best-first 16-lists held one entry per lane of a 16-lane
// segment; `b_rev` is the other list's entry at position 15 - li
__device__ __forceinline__ uint64_t merge16(uint64_t a, uint64_t b_rev, int li)
{
    uint64_t x = a > b_rev ? a : b_rev;
#pragma unroll
    for (int d = 8; d > 0; d >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, x, d, 16);
        // the lower lane of a pair keeps the larger word, the upper one the smaller
        const bool take = (y > x) != ((li & d) != 0);
        x = take ? y : x;
    }
    return x;
}

template <int DPMAX, int CPL>
__global__ void __launch_bounds__(kWarpStepWarps * 32, 7) k_step_warp(StepParams p)
{
    constexpr int kStepRows = CPL >= 8 ? 4 : (CPL >= 4 ? 8 : 16);  // rows per lane in flight
    const int lane = threadIdx.x & 31;
    const int bh = static_cast<int>(blockIdx.x) * kWarpStepWarps + static_cast<int>(threadIdx.x >> 5);
    if (bh >= p.B * p.H) return;  // whole warps only
    const int half = lane >> 4, li = lane & 15;
    const int K = p.K, dv = p.d_v, M = p.M, d_p = p.d_p, U = p.U;
    const int L = U * d_p;
    const void* lg = half == 0 ? p.k_logits : p.q_logits;
    const size_t off = static_cast<size_t>(bh) * L;
    const int h = bh % p.H, b = bh / p.H;

    const int LW = (CPL > 1 || dv >= 32) ? 32 : dv;  // lanes holding channels
    const bool act = lane < LW;
    const int ch0 = (act ? lane : 0) * CPL;
    prefetch_logits(lg, off, p.in_bf16, L);

    // ---- digit codes, computed once per half: in a round, lane li of a half takes digit
    // li mod DPMAX of level (round * LPR + li / DPMAX); each level's DPMAX lanes sort their
    // codes best first (bitonic, by signed value as sort_codes_desc) and, for the raw product
    // softmax, reduce the level's logsumexp.  A level's sorted codes reach every lane of the
    // half by shuffles.
    constexpr int LPR = 16 / DPMAX;  // levels per round
    const int dpos = li % DPMAX, dseg = (li / DPMAX) * DPMAX;
    uint64_t cs = 0ull;  // this lane's sorted code of its level in the current round
    float lse = 0.0f;    // sum over levels of logsumexp (renorm == 0)
    auto code_round = [&](int r) {
        const int u = r * LPR + li / DPMAX;
        const bool valid = u < U && dpos < d_p;
        const float x = valid ? load_in(lg, off + u * d_p + dpos, p.in_bf16) : 0.0f;
        uint64_t c = valid ? digit_code(x, dpos, d_p) : 0x8000000000000000ull;
#pragma unroll
        for (int k = 2; k <= DPMAX; k <<= 1)
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
                const int64_t o = static_cast<int64_t>(__shfl_xor_sync(0xffffffffu, c, j, 16));
                const int64_t v = static_cast<int64_t>(c);
                const bool keep_max = ((dpos & j) == 0) == ((dpos & k) == 0);
                c = static_cast<uint64_t>(keep_max ? (v > o ? v : o) : (v < o ? v : o));
            }
        cs = c;
        if (!p.renorm) {
            const float xc = fminf(fmaxf(x, -4095.f), 4095.f);
            float mx = valid ? xc : -INFINITY;
#pragma unroll
            for (int j = DPMAX / 2; j > 0; j >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, j, 16));
            float zs = valid ? expf(xc - mx) : 0.0f;
#pragma unroll
            for (int j = DPMAX / 2; j > 0; j >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, j, 16);
            float l = (u < U) ? mx + logf(zs) : 0.0f;  // this level's logsumexp (every lane of the level)
            // add the round's levels: one value per DPMAX-lane segment of the half
            float acc = l;
#pragma unroll
            for (int j = DPMAX; j < 16; j <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, j, 16);
            lse += acc;
        }
    };
    auto level_codes = [&](int u, uint64_t (&e)[DPMAX]) {
        if (u % LPR == 0) code_round(u / LPR);
        const int base = (u % LPR) * DPMAX;
#pragma unroll
        for (int d = 0; d < DPMAX; ++d) e[d] = __shfl_sync(0xffffffffu, cs, base + d, 16);
    };

    // ---- exact Top-K by levels, one kept prefix per lane
    uint64_t kept;
    int nk;
    {
        uint64_t e[DPMAX];
        level_codes(0, e);
        nk = min(K, d_p);
        kept = 0ull;
#pragma unroll
        for (int d = 0; d < DPMAX; ++d)
            if (d == li && d < nk) kept = (kKeyBias << 16) + e[d];
    }
    const uint64_t mul = static_cast<uint64_t>(d_p - 1);
    for (int u = 1; u < U; ++u) {
        uint64_t e[DPMAX];
        level_codes(u, e);
        const uint64_t f = kept + (kept & 0xFFFFull) * mul;               // this lane's prefix, extended
        const uint64_t fr = __shfl_sync(0xffffffffu, f, 15 - li, 16);   // the prefix at position 15 - li
        const bool ok = li < nk, okr = 15 - li < nk;
        uint64_t t[DPMAX / 2];
#pragma unroll
        for (int q = 0; q < DPMAX / 2; ++q) {
            const uint64_t a = (ok && 2 * q < d_p) ? f + e[2 * q] : 0ull;
            const uint64_t br = (okr && 2 * q + 1 < d_p) ? fr + e[2 * q + 1] : 0ull;
            t[q] = merge16(a, br, li);
        }
#pragma unroll
        for (int n = DPMAX / 2; n > 1; n >>= 1)
#pragma unroll
            for (int q = 0; q < n / 2; ++q)
                t[q] = merge16(t[2 * q], __shfl_sync(0xffffffffu, t[2 * q + 1], 15 - li, 16), li);
        nk = min(K, nk * d_p);
        kept = li < nk ? t[0] : 0ull;  // only the K best prefixes are kept
    }
    // (every round of levels 0..U-1 was reached above, so lse covers all U levels)

    // ---- winner li of this half: weight, slot after CAPE, retention (writes)
    const bool win = li < K;
    const int64_t s0 = packed_score(__shfl_sync(0xffffffffu, kept, 0, 16));
    const float base = p.renorm ? 0.0f : static_cast<float>(s0) * kInvScale - lse;
    float w = win ? expf(base + static_cast<float>(packed_score(kept) - s0) * kInvScale) : 0.0f;
    if (p.renorm) {
        float sum = w;
#pragma unroll
        for (int d = 8; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d, 16);
        w = w / sum;
    }
    const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
    const int32_t pm = cape ? cape_shift(0, p.pos != nullptr ? p.pos[b] : 0, M) : 0;
    int32_t idx = packed_index(kept, M) + pm;
    if (idx >= M) idx -= M;
    if (!dcheck(!win || (idx >= 0 && idx < M), p.status) || !win) idx = 0;

    // ---- GSU steps 1-3 on the K write masses (lane j < K of the key half)
    float* S = p.S + static_cast<size_t>(bh) * M * dv;
    float* mrow = p.m + static_cast<size_t>(bh) * M;
    float vv[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) vv[c] = act ? load_in(p.v, static_cast<size_t>(bh) * dv + ch0 + c, p.in_bf16) : 0.0f;
    float lam = 0.0f;
    if (half == 0 && win) {
        const float gg = load_in(p.g, bh, p.in_bf16);
        const float mn = gsu_alpha(w, gg) * mrow[idx] + w;
        mrow[idx] = mn;
        lam = w / (mn + p.eps_gsu);
    }
    // ---- GSU step 4 on the K write rows
    for (int j0 = 0; j0 < K; j0 += kStepRows) {
        float sr[kStepRows][CPL];
        int ri[kStepRows];
#pragma unroll
        for (int k = 0; k < kStepRows; ++k) {
            ri[k] = __shfl_sync(0xffffffffu, idx, (j0 + k) & 15);
            if (j0 + k < K && act) load_row_g<CPL>(S + static_cast<size_t>(ri[k]) * dv + ch0, sr[k]);
        }
#pragma unroll
        for (int k = 0; k < kStepRows; ++k) {
            const float lk = __shfl_sync(0xffffffffu, lam, (j0 + k) & 15);
            if (j0 + k < K && act) {
#pragma unroll
                for (int c = 0; c < CPL; ++c) sr[k][c] = fmaf(lk, vv[c] - sr[k][c], sr[k][c]);
                store_row_g<CPL>(S + static_cast<size_t>(ri[k]) * dv + ch0, sr[k]);
            }
        }
    }
    // ---- read rows (after the writes), weighted sum
    float o[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = 0.0f;
    for (int j0 = 0; j0 < K; j0 += kStepRows) {
        float sr[kStepRows][CPL];
#pragma unroll
        for (int k = 0; k < kStepRows; ++k) {
            const int rj = __shfl_sync(0xffffffffu, idx, 16 + ((j0 + k) & 15));
            if (j0 + k < K && act) load_row_g<CPL>(S + static_cast<size_t>(rj) * dv + ch0, sr[k]);
        }
#pragma unroll
        for (int k = 0; k < kStepRows; ++k) {
            const float r = __shfl_sync(0xffffffffu, w, 16 + ((j0 + k) & 15));
            if (j0 + k < K && act) {
#pragma unroll
                for (int c = 0; c < CPL; ++c) o[c] = fmaf(r, sr[k][c], o[c]);
            }
        }
    }
    float ss = 0.0f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) ss = fmaf(o[c], o[c], ss);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, d);
    const float inv = 1.0f / sqrtf(ss / dv + p.eps_norm);
    if (act) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const float zc = load_in(p.z, static_cast<size_t>(bh) * dv + ch0 + c, p.in_bf16);
            const float nc = p.norm_w != nullptr ? p.norm_w[ch0 + c] : 1.0f;
            store_out(p.y, static_cast<size_t>(bh) * dv + ch0 + c, o[c] * inv * nc * zc, p.out_bf16);
        }
    }
}

template <int DPMAX>
cudaError_t launch_step_warp(const StepParams& p, cudaStream_t s)
{
    const int units = p.B * p.H;
    const unsigned grid = static_cast<unsigned>((units + kWarpStepWarps - 1) / kWarpStepWarps);
    void (*kern)(StepParams) = nullptr;
    switch (p.d_v < 32 ? 1 : p.d_v / 32) {
        case 1: kern = k_step_warp<DPMAX, 1>; break;
        case 2: kern = k_step_warp<DPMAX, 2>; break;
        case 4: kern = k_step_warp<DPMAX, 4>; break;
        case 8: kern = k_step_warp<DPMAX, 8>; break;
        default: return cudaErrorInvalidValue;
    }
    kern<<<grid, kWarpStepWarps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_step(const StepParams& p, cudaStream_t stream)
{
    if (p.d_v > 256) return cudaErrorInvalidValue;
    // one warp per unit where the kept list fits a 16-lane half and a level's columns fit the
    // merge tree; the persistent kernel otherwise
    if (p.K <= 16 && p.d_p <= 4) return launch_step_warp<4>(p, stream);
    if (p.K <= 16 && p.d_p <= 8) return launch_step_warp<8>(p, stream);
    if (p.d_p <= 4) return step_k<4>(p, stream);
    if (p.d_p <= 8) return step_k<8>(p, stream);
    return step_k<16>(p, stream);
}

}  // namespace ramnet
