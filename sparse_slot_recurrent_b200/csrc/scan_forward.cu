// scan_forward.cu -- second launch of the prefill scan: the recurrence of the RAM-Net layer
// core (Gated Sparse Update, sparse read, RMSNorm, output gate) over the events that the
// route kernel grouped by owner.
//
// RAM-Net project page: the three-stage paragraph (decode, CAPE, GSU, then read, normalise,
// gate), the Gated Sparse Update paragraphs (four steps; unselected slots unchanged) and the
// GPU-execution paragraph (events grouped by slot, each slot's events walked in causal
// order, slots and channels in parallel, slots without events cost nothing).
//
// State layout.  One head's slot array S [M, d_v] fp32 lives in tensor memory (TMEM) for
// the whole sequence, spread over a cluster of `ncta` CTAs, one per SM.  Slot i belongs to
// CTA rank (i mod ncta) as local slot s = i / ncta, which sits in TMEM lane quadrant
// (s mod 4), columns [(s/4)*CPL, (s/4)*CPL + CPL); lane l of the quadrant holds channels
// [l*CPL, l*CPL + CPL).  One slot row is one tcgen05.ld/st of CPL columns by a warp of that
// quadrant.  Scan warp w owns the local slots with s mod nw == w.
//
// Warps of a CTA:
//   loader      bulk-copies each chunk's header, this CTA's events and the chunk's value
//               rows into a ring of `stages` shared-memory stages;
//   scan warps  each walks its own event list of the chunk (token order, a token's writes
//               before its reads) in batches of up to kBatch events on distinct slots: one
//               tcgen05.ld per event, one wait per batch (a TMEM load takes a few hundred
//               cycles), then per write GSU steps 1-4 (mass m = alpha*m + w, rate
//               lambda = w/(m + eps), row S <- S + lambda (v - S), stored back with
//               tcgen05.st) and per read the weighted row r*S, stored into this CTA's
//               read-partial ring at (token, q), q = the read's rank among the token's
//               reads held by this CTA;
//   finishers   per token, the sum of the CTA's read partials in q order; the CTA that
//               finishes the chunk (rank = chunk mod ncta) adds the peers' sums in rank
//               order (peers store theirs into its shared memory: one row per token), then
//               RMSNorm over d_v, norm weight, output gate, y.
// Every sum has a fixed order, so y is the same from run to run.
// Every wait is bounded (about 2 s); a wait that gives up records RAMNET_ERR_TIMEOUT in the
// status word and raises the CTA's abort flag, after which its waits return at once, scan
// warps skip their events and the loader stops copying, so the kernel ends within seconds.
// Event fields are clamped into their ranges before use; the RAMNET_DEBUG build also records
// out-of-range fields (RAMNET_ERR_DEVICE_CHECK).
#include "common.cuh"
#include "kernels.h"

namespace ramnet {

namespace {


__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

// mbarrier indices
struct Bars {
    int sfull, sfree, ldone, lfree, xfull, xfree, count;
};
__host__ __device__ inline Bars bar_index(int S, int P, int X, int ncta)
{
    Bars b;
    b.sfull = 0;            // [S] stage landed (loader arrive + bulk-copy bytes)
    b.sfree = S;            // [S] every scan warp left the stage
    b.ldone = 2 * S;        // [P] every scan warp stored its read partials of the chunk
    b.lfree = 2 * S + P;    // [P] the finishers summed the chunk's partials
    b.xfull = 2 * S + 2 * P;          // [X] every peer stored its sums of a chunk this CTA finishes
    b.xfree = 2 * S + 2 * P + X;      // [ncta][X] finisher CTA f released its exchange slot
    b.count = 2 * S + 2 * P + X + ncta * X;
    return b;
}

struct Layout {
    size_t bars, misc, m, nloc, stage, stage_bytes, ev_off, v_off, lring, lring_bytes, xbuf, xbuf_bytes, total;
};

// Shared memory of the scan kernel.
__host__ __device__ inline Layout scan_layout(int Ml, int C, int K, int dv, int es, int S, int P, int X, int ncta,
                                              int hw)
{
    Layout L;
    const Bars b = bar_index(S, P, X, ncta);
    size_t o = 0;
    L.bars = o;
    o += align16(8 * static_cast<size_t>(b.count));
    L.misc = o;
    o += 16;
    L.m = o;
    o += align16(sizeof(float) * Ml);
    L.nloc = o;
    o += align16(static_cast<size_t>(P) * C);
    L.ev_off = align16(static_cast<size_t>(hw) * 4);
    L.v_off = L.ev_off + static_cast<size_t>(C) * 2 * K * sizeof(uint4);
    L.stage_bytes = L.v_off + align16(static_cast<size_t>(C) * dv * es);
    L.stage = o;
    o += static_cast<size_t>(S) * L.stage_bytes;
    L.lring_bytes = static_cast<size_t>(C) * K * dv * sizeof(float);
    L.lring = o;
    o += static_cast<size_t>(P) * L.lring_bytes;
    L.xbuf_bytes = static_cast<size_t>(ncta > 1 ? ncta - 1 : 0) * C * dv * sizeof(float);
    L.xbuf = o;
    o += static_cast<size_t>(X) * L.xbuf_bytes;
    L.total = o;
    return L;
}

__host__ __device__ inline int hdr_words_of(int nw, int C) { return (4 + nw + 1 + (C + 3) / 4 + 3) & ~3; }

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// One try_wait on phase `parity`: the thread may be suspended in hardware until the phase
// completes or about `hint_ns` (at most kSuspendNs) have passed.  CLUSTER selects acquire at cluster scope (for
// barriers that peers of the cluster arrive on after writing into this CTA's shared memory);
// otherwise the default CTA scope.
constexpr uint32_t kSuspendNs = 100000;

template <bool CLUSTER>
__device__ __forceinline__ bool try_wait_phase(uint32_t bar, uint32_t parity, uint32_t hint_ns = kSuspendNs)
{
    uint32_t ok;
    if constexpr (CLUSTER) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(hint_ns)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(hint_ns)
            : "memory");
    }
    return ok != 0;
}

// Bounded wait for phase `parity` of the mbarrier at shared address `bar`: at most
// kSpinLimit polls and `limit_ns` (2 s unless given; the prefill recurrence passes its
// launch's limit).  Between polls the thread sleeps
// (32 ns doubling to 256 ns), so waiting warps leave the issue slots to working ones.  On
// expiry the status word gets kDevTimeout and the CTA's abort flag is raised, after which
// every later wait of the CTA returns at once, so a kernel that lost a signal still ends
// within a few seconds.
template <bool CLUSTER>
__device__ __forceinline__ void wait_bounded(uint32_t bar, uint32_t parity, uint32_t* status, volatile int* abort_flag,
                                             uint64_t limit_ns = 2000000000ull)
{
    // a hardware suspension never outlasts the limit itself
    const uint32_t hint = limit_ns < kSuspendNs ? static_cast<uint32_t>(limit_ns) : kSuspendNs;
    if (try_wait_phase<CLUSTER>(bar, parity, hint)) return;
    if (*abort_flag) return;
    const uint64_t t_end = global_ns() + limit_ns;
    uint32_t nap = 32;
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        if (try_wait_phase<CLUSTER>(bar, parity, hint)) return;
        if (global_ns() > t_end || *abort_flag) break;
        __nanosleep(nap);
        nap = nap < 256 ? 2 * nap : 256;
    }
    *abort_flag = 1;
    set_status(status, kDevTimeout);
}

// Before exit: wait (bounded, ignoring the abort flag) until the bulk copies this CTA
// issued into its own shared memory have landed.
__device__ __noinline__ void drain_copies(uint32_t bar, uint32_t parity)
{
    const uint64_t t_end = global_ns() + 2000000000ull;
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        if (try_wait_phase<false>(bar, parity)) return;
        if (global_ns() > t_end) return;
        __nanosleep(256);
    }
}

// Arrive (release, CTA scope) on a barrier of this CTA.
__device__ __forceinline__ void arrive_local(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on mbarrier `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// CPL consecutive input elements (fp32 or bf16) from shared memory, as fp32.
template <int CPL>
__device__ __forceinline__ void load_row(const unsigned char* base, int elem, int is_bf16, float (&v)[CPL])
{
    if (is_bf16) {
        const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(base) + elem;
        if constexpr (CPL % 4 == 0) {
#pragma unroll
            for (int c = 0; c < CPL; c += 4) {
                const uint2 u = *reinterpret_cast<const uint2*>(pb + c);
                v[c + 0] = __uint_as_float(u.x << 16);
                v[c + 1] = __uint_as_float(u.x & 0xFFFF0000u);
                v[c + 2] = __uint_as_float(u.y << 16);
                v[c + 3] = __uint_as_float(u.y & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) v[c] = __bfloat162float(pb[c]);
        }
    } else {
        const float* pf = reinterpret_cast<const float*>(base) + elem;
        if constexpr (CPL % 4 == 0) {
#pragma unroll
            for (int c = 0; c < CPL; c += 4) {
                const float4 u = *reinterpret_cast<const float4*>(pf + c);
                v[c] = u.x;
                v[c + 1] = u.y;
                v[c + 2] = u.z;
                v[c + 3] = u.w;
            }
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) v[c] = pf[c];
        }
    }
}

// CPL consecutive elements of a global [.., d_v] input row as fp32.
template <int CPL>
__device__ __forceinline__ void load_row_in(const void* base, size_t elem, int is_bf16, float (&v)[CPL])
{
    if (is_bf16) {
        const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(base) + elem;
        if constexpr (CPL % 4 == 0) {
#pragma unroll
            for (int c = 0; c < CPL; c += 4) {
                const uint2 u = *reinterpret_cast<const uint2*>(pb + c);
                v[c + 0] = __uint_as_float(u.x << 16);
                v[c + 1] = __uint_as_float(u.x & 0xFFFF0000u);
                v[c + 2] = __uint_as_float(u.y << 16);
                v[c + 3] = __uint_as_float(u.y & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) v[c] = __bfloat162float(pb[c]);
        }
    } else {
        load_row_g<CPL>(reinterpret_cast<const float*>(base) + elem, v);
    }
}

template <int CPL>
__device__ __forceinline__ void lds_row(const float* p, float (&v)[CPL])
{
    load_row_g<CPL>(p, v);  // generic vector loads of shared memory
}

template <int CPL>
__device__ __forceinline__ void sts_row(float* p, const float (&v)[CPL])
{
    store_row_g<CPL>(p, v);
}

// CPL values into a peer CTA's shared memory at shared::cluster address `caddr`.
template <int CPL>
__device__ __forceinline__ void st_cluster_row(uint32_t caddr, const float (&v)[CPL])
{
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int c = 0; c < CPL; c += 4) st_cluster_v4(caddr + 4 * c, v[c], v[c + 1], v[c + 2], v[c + 3]);
    } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(caddr + 4 * c), "f"(v[c]) : "memory");
    }
}

// CPL outputs of consecutive channels to global memory (bf16 or fp32), vectorised.
template <int CPL>
__device__ __forceinline__ void store_y(void* y, size_t elem, const float (&v)[CPL], int out_bf16)
{
    if (out_bf16) {
        __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(y) + elem;
        if constexpr (CPL % 4 == 0) {
#pragma unroll
            for (int c = 0; c < CPL; c += 4) {
                const __nv_bfloat162 a = __floats2bfloat162_rn(v[c], v[c + 1]);
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[c + 2], v[c + 3]);
                uint2 u;
                u.x = *reinterpret_cast<const uint32_t*>(&a);
                u.y = *reinterpret_cast<const uint32_t*>(&b2);
                *reinterpret_cast<uint2*>(pb + c) = u;
            }
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) pb[c] = __float2bfloat16_rn(v[c]);
        }
    } else {
        store_row_g<CPL>(reinterpret_cast<float*>(y) + elem, v);
    }
}

constexpr int kScanWarps = 16;
constexpr int kFinWarps = 8;
constexpr int kFinGroups = 2;
constexpr int kScanThreads = (kScanWarps + kFinWarps + 1) * 32;
constexpr int kSmemBudget = 220 * 1024;

template <int CPL, bool BF>
__global__ void __launch_bounds__(kScanThreads, 1) k_scan(ScanParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int kZMax = CPL <= 4 ? 16 : 8;  // z values a finisher lane prefetches per chunk
    constexpr int kBatch = CPL >= 8 ? 4 : 8;  // events per TMEM round trip of a scan warp
    const int C = p.chunk, dv = p.d_v, ncta = p.ncta, M = p.M, K = p.K, NW = p.nw, F = p.nfin;
    const int S = p.stages, P = p.lslots, X = p.xslots;
    const int LW = (CPL > 1 || dv >= 32) ? 32 : dv;  // lanes holding channels (32 unless d_v = 16)
    const int es = BF ? 2 : 4;
    const int rank = static_cast<int>(cluster_ctarank());
    const int bh = static_cast<int>(blockIdx.x) / ncta;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Ml = (M - rank + ncta - 1) / ncta;
    const int nch = p.nch;
    const int cap = 2 * C * K;  // event capacity of a stage
    const Layout L = scan_layout((M + ncta - 1) / ncta, C, K, dv, es, S, P, X, ncta, p.hdr_words);
    const Bars BI = bar_index(S, P, X, ncta);
    const uint32_t bars = smem_addr(smem + L.bars);
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    uint64_t* bar_ptr = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
    float* m_s = reinterpret_cast<float*>(smem + L.m);
    unsigned char* nloc_s = smem + L.nloc;
    auto stage = [&](int c) { return smem + L.stage + static_cast<size_t>(c % S) * L.stage_bytes; };
    float* lring = reinterpret_cast<float*>(smem + L.lring);
    const size_t lslot_floats = L.lring_bytes / sizeof(float);
    float* xbuf = reinterpret_cast<float*>(smem + L.xbuf);
    const size_t xslot_floats = L.xbuf_bytes / sizeof(float);

    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < S; ++i) {
            mbar_init(bar_ptr + BI.sfull + i, 1);
            mbar_init(bar_ptr + BI.sfree + i, NW);
        }
        for (int i = 0; i < P; ++i) {
            mbar_init(bar_ptr + BI.ldone + i, NW);
            mbar_init(bar_ptr + BI.lfree + i, F / kFinGroups);
        }
        for (int i = 0; i < X; ++i) mbar_init(bar_ptr + BI.xfull + i, ncta > 1 ? (ncta - 1) * (F / kFinGroups) : 1);
        for (int i = 0; i < ncta * X; ++i) mbar_init(bar_ptr + BI.xfree + i, F / kFinGroups);
        fence_mbar_init_cluster();
    }
    if (warp == 0) tmem_alloc(holder, p.tmem_cols);
    for (int s = tid; s < Ml; s += blockDim.x)
        m_s[s] = p.m_in != nullptr ? p.m_in[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] : 0.0f;
    tmem_fence_before_sync();
    cluster_sync_all();  // barriers initialised cluster-wide before any peer arrives on them
    tmem_fence_after_sync();
    const uint32_t tbase = *holder;

    if (warp < NW) {
        // ============================================================ scan warps
        const int q4 = warp & 3;
        const uint32_t tq = tbase + (static_cast<uint32_t>(32 * q4) << 16);
        const int lch = (lane < LW ? lane : 0) * CPL;  // this lane's first channel
        for (int s = warp; s < Ml; s += NW) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) r[c] = (p.S_in != nullptr && lane < LW) ? p.S_in[row + lch + c] : 0.0f;
            tmem_st<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
        }
        tmem_wait_st();
        const unsigned lt_mask = (1u << lane) - 1u;
        for (int c = 0; c < nch; ++c) {
            wait_bounded<false>(bar(BI.sfull + c % S), (c / S) & 1, p.status, abort_flag, p.wait_ns);
            const int ls = c % P, kl = c / P;
            if (kl >= 1) wait_bounded<false>(bar(BI.lfree + ls), (kl - 1) & 1, p.status, abort_flag, p.wait_ns);
            const unsigned char* st = stage(c);
            const uint32_t* hd = reinterpret_cast<const uint32_t*>(st);
            if (!*abort_flag) {
                const int nt = min(static_cast<int>(hd[2]), C);
                const int beg = min(static_cast<int>(hd[4 + warp]), cap);
                const int end = max(beg, min(static_cast<int>(hd[5 + warp]), cap));
                if (warp == 0) {
                    const unsigned char* nb = st + (4 + NW + 1) * 4;
                    for (int i = lane; i < C; i += 32) nloc_s[ls * C + i] = nb[i];
                }
                const uint4* evs = reinterpret_cast<const uint4*>(st + L.ev_off);
                const unsigned char* vb = st + L.v_off;
                float* lr = lring + static_cast<size_t>(ls) * lslot_floats + lch;
                int e = beg;
                while (e < end) {
                    // The longest run of up to kBatch events on distinct slots.  Lane k < nb
                    // decodes event e + k once for the whole warp: its slot's tensor-memory
                    // address, the row it touches in shared memory and, for a write, GSU steps
                    // 1-3 (m = alpha*m + w, lambda = w / (m + eps)); the per-event loops below
                    // only fetch those values with shuffles.
                    const int navail = end - e;
                    const bool act = lane < kBatch && lane < navail;
                    uint4 r = make_uint4(0u, 0u, 0u, 0u);
                    if (act) r = evs[e + lane];
                    const uint32_t sl = act ? (r.x & 0xFFFFu) : 0x10000u + static_cast<uint32_t>(lane);
                    const uint32_t peers = __match_any_sync(0xffffffffu, sl);
                    const uint32_t dup = __ballot_sync(0xffffffffu, (peers & lt_mask) != 0u);
                    int nb = min(navail, kBatch);
                    if (dup != 0u) nb = min(nb, __ffs(dup) - 1);
                    // fields are clamped into range, so even a corrupt workspace cannot address
                    // outside tensor memory, the stage or the ring; the debug build also records
                    // the corruption
                    const int es_ = min(static_cast<int>(r.x & 0xFFFFu), Ml - 1);
                    const bool rd = (r.x >> 31) != 0u;
                    const int etl = min(static_cast<int>((r.x >> 16) & 0xFFu), nt - 1);
                    const int eq = min(static_cast<int>((r.x >> 24) & 0x3Fu), K - 1);
                    dcheck(lane >= nb || (static_cast<int>(r.x & 0xFFFFu) < Ml && (es_ & (NW - 1)) == warp &&
                                          static_cast<int>((r.x >> 16) & 0xFFu) < nt &&
                                          (!rd || static_cast<int>((r.x >> 24) & 0x3Fu) < K)),
                           p.status);
                    float eck = __uint_as_float(r.y);
                    if (lane < nb && !rd) {
                        const float mn = fmaf(__uint_as_float(r.z), m_s[es_], eck);
                        m_s[es_] = mn;
                        eck = __fdividef(eck, mn + p.eps_gsu);
                    }
                    const uint32_t eta = tq + static_cast<uint32_t>((es_ >> 2) * CPL);
                    // row offset in elements (value row of the stage, or read-partial row of the
                    // ring) with the read flag in bit 31
                    const uint32_t erow = rd ? (0x80000000u | static_cast<uint32_t>((etl * K + eq) * dv))
                                             : static_cast<uint32_t>(etl * dv);
                    uint32_t ta[kBatch];
                    float Sv[kBatch][CPL];
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        ta[k] = __shfl_sync(0xffffffffu, eta, k);
                        if (k < nb) tmem_ld<CPL>(ta[k], Sv[k]);
                    }
                    tmem_wait_ld();
                    bool wrote = false;
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        const float ck = __shfl_sync(0xffffffffu, eck, k);
                        const uint32_t row = __shfl_sync(0xffffffffu, erow, k);
                        if (k < nb) {
                            if ((row >> 31) == 0u) {
                                // GSU step 4 on the row
                                float vv[CPL];
                                load_row<CPL>(vb, static_cast<int>(row) + lch, BF, vv);
#pragma unroll
                                for (int cc = 0; cc < CPL; ++cc) Sv[k][cc] = fmaf(ck, vv[cc] - Sv[k][cc], Sv[k][cc]);
                                tmem_st<CPL>(ta[k], Sv[k]);
                                wrote = true;
                            } else {
                                // read: r * S into the partial ring at (token, q)
#pragma unroll
                                for (int cc = 0; cc < CPL; ++cc) Sv[k][cc] *= ck;
                                if (lane < LW) sts_row<CPL>(lr + (row & 0x7FFFFFFFu), Sv[k]);
                            }
                        }
                    }
                    if (wrote) tmem_wait_st();
                    e += nb;
                }
            }
            __syncwarp();
            if (lane == 0) {
                arrive_local(bar(BI.sfree + c % S));
                arrive_local(bar(BI.ldone + ls));
            }
        }
        // final state of the owned slots
        for (int s = warp; s < Ml; s += NW) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
            tmem_ld<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
            tmem_wait_ld();
            if (lane < LW) {
#pragma unroll
                for (int c = 0; c < CPL; ++c) p.S_out[row + lch + c] = r[c];
            }
            if (lane == 0) p.m_out[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] = m_s[s];
        }
    } else if (warp < NW + F) {
        // ============================================================ finisher warps
        // kFinGroups groups of finisher warps take alternate chunks, so one group's wait for
        // a peer CTA does not hold up the next chunk; chunk c goes to group c mod kFinGroups,
        // which divides ncta (or ncta is 1), so every chunk that one CTA finishes, and so
        // every use of one exchange slot, stays with one group, in chunk order
        const int fw = warp - NW;
        const int FG = F / kFinGroups, grp = fw / FG, gw = fw - grp * FG;
        const int lch = (lane < LW ? lane : 0) * CPL;
        float nwv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) nwv[c] = p.norm_w != nullptr ? p.norm_w[lch + c] : 1.0f;
        const int ft = (C + FG - 1) / FG;  // tokens per finisher warp per chunk (ft * CPL <= kZMax)
        for (int c = grp; c < nch; c += kFinGroups) {
            const int ls = c % P, kl = c / P;
            const int f = c % ncta;
            const int xs = (c / ncta) % X, kx = c / (ncta * X);
            const int nt = min(C, p.T - c * C);
            const bool own = f == rank;
            const int t0 = c * C;
            float zr[kZMax];
#pragma unroll
            for (int i = 0; i < kZMax; ++i) zr[i] = 0.0f;
            if (own) {
#pragma unroll
                for (int i = 0; i < kZMax / CPL; ++i) {
                    const int tl = gw + i * FG;
                    if (i < ft && tl < nt && lane < LW) {
                        float zz[CPL];
                        load_row_in<CPL>(p.z, ((static_cast<size_t>(b) * p.T + t0 + tl) * p.H + h) * dv + lch, BF,
                                         zz);
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) zr[i * CPL + cc] = zz[cc];
                    }
                }
            }
            wait_bounded<false>(bar(BI.ldone + ls), kl & 1, p.status, abort_flag, p.wait_ns);
            // this CTA's sum of each token's read partials, in q order
            const float* lr = lring + static_cast<size_t>(ls) * lslot_floats + lch;
            float o[kZMax];
#pragma unroll
            for (int i = 0; i < kZMax / CPL; ++i) {
                const int tl = gw + i * FG;
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) o[i * CPL + cc] = 0.0f;
                if (i < ft && tl < nt) {
                    const int n = min(static_cast<int>(nloc_s[ls * C + tl]), K);
                    for (int q = 0; q < n; ++q) {
                        float pr[CPL];
                        lds_row<CPL>(lr + static_cast<size_t>(tl * K + q) * dv, pr);
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) o[i * CPL + cc] += pr[cc];
                    }
                }
            }
            // the partial-ring slot is free again once every finisher warp has read it; the
            // scan warps move on without waiting for the exchange between CTAs
            __syncwarp();
            if (lane == 0) arrive_local(bar(BI.lfree + ls));
            if (ncta > 1) {
                if (own) wait_bounded<true>(bar(BI.xfull + xs), kx & 1, p.status, abort_flag, p.wait_ns);
                else if (kx >= 1) wait_bounded<true>(bar(BI.xfree + f * X + xs), (kx - 1) & 1, p.status, abort_flag, p.wait_ns);
            }
            const int xi = rank < f ? rank : rank - 1;  // this CTA's entry in f's exchange slot
            const uint32_t xdst = ncta > 1 && !own
                                      ? map_to_rank(smem_addr(xbuf + static_cast<size_t>(xs) * xslot_floats +
                                                              static_cast<size_t>(xi) * C * dv + lch),
                                                    static_cast<uint32_t>(f))
                                      : 0u;
#pragma unroll
            for (int i = 0; i < kZMax / CPL; ++i) {
                const int tl = gw + i * FG;
                if (i < ft && tl < nt) {
                    if (own) {
                        // rank order: peers below this CTA, this CTA, peers above
                        float tot[CPL];
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) tot[cc] = 0.0f;
                        for (int r2 = 0; r2 < ncta; ++r2) {
                            if (r2 == rank) {
#pragma unroll
                                for (int cc = 0; cc < CPL; ++cc) tot[cc] += o[i * CPL + cc];
                            } else {
                                const int xi2 = r2 < rank ? r2 : r2 - 1;
                                float pr[CPL];
                                lds_row<CPL>(xbuf + static_cast<size_t>(xs) * xslot_floats +
                                                 (static_cast<size_t>(xi2) * C + tl) * dv + lch,
                                             pr);
#pragma unroll
                                for (int cc = 0; cc < CPL; ++cc) tot[cc] += pr[cc];
                            }
                        }
                        float ss = 0.0f;
                        if (lane < LW) {
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) ss = fmaf(tot[cc], tot[cc], ss);
                        }
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                        const float inv = 1.0f / sqrtf(ss / dv + p.eps_norm);
                        if (lane < LW && !*abort_flag) {
                            float yv[CPL];
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) yv[cc] = tot[cc] * inv * nwv[cc] * zr[i * CPL + cc];
                            store_y<CPL>(p.y, ((static_cast<size_t>(b) * p.T + t0 + tl) * p.H + h) * dv + lch, yv,
                                         p.out_bf16);
                        }
                    } else if (lane < LW) {
                        float ov[CPL];
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) ov[cc] = o[i * CPL + cc];
                        st_cluster_row<CPL>(xdst + static_cast<uint32_t>(tl * dv * 4), ov);
                    }
                }
            }
            // each finisher warp signals its own rows (stores and reads of the warp ordered
            // before lane 0's release by the warp barrier)
            __syncwarp();
            if (ncta > 1 && lane == 0) {
                if (own) {
                    for (int r2 = 0; r2 < ncta; ++r2)
                        if (r2 != rank)
                            mbar_arrive_cluster(map_to_rank(bar(BI.xfree + rank * X + xs), static_cast<uint32_t>(r2)));
                } else {
                    mbar_arrive_cluster(map_to_rank(bar(BI.xfull + xs), static_cast<uint32_t>(f)));
                }
            }
        }
    } else {
        // ============================================================ loader warp
        const uint32_t vrow = static_cast<uint32_t>(dv * es);
        const uint32_t hdr_bytes = static_cast<uint32_t>(p.hdr_words * 4);
        uint32_t pf_start = 0, pf_n = 0;  // (first event, count) of chunk (c & ~31) + lane
        int issued = 0;                    // chunks whose copies were issued (0..issued-1)
        for (int c = 0; c < nch; ++c) {
            if ((c & 31) == 0) {
                const int cc = c + lane;
                if (cc < nch) {
                    const uint32_t* hp = p.hdr + ((static_cast<size_t>(bh) * nch + cc) * ncta + rank) * p.hdr_words;
                    pf_start = hp[0];
                    pf_n = hp[1];
                }
            }
            const uint32_t start = __shfl_sync(0xffffffffu, pf_start, c & 31);
            const uint32_t n = min(__shfl_sync(0xffffffffu, pf_n, c & 31), static_cast<uint32_t>(cap));
            const uint32_t first = min(start, static_cast<uint32_t>(cap) - n);
            const int nt = min(C, p.T - c * C);
            if (c >= S) {
                wait_bounded<false>(bar(BI.sfree + c % S), (c / S - 1) & 1, p.status, abort_flag, p.wait_ns);
                fence_proxy_async();
            }
            if (*abort_flag) continue;
            unsigned char* st = stage(c);
            const uint32_t sb = bar(BI.sfull + c % S);
            const uint32_t evb = n * static_cast<uint32_t>(sizeof(uint4));
            if (lane == 0) arrive_expect_tx(sb, hdr_bytes + evb + static_cast<uint32_t>(nt) * vrow);
            __syncwarp();
            if (lane == 0) {
                bulk_g2s(smem_addr(st), p.hdr + ((static_cast<size_t>(bh) * nch + c) * ncta + rank) * p.hdr_words,
                         hdr_bytes, sb);
                if (evb > 0)
                    bulk_g2s(smem_addr(st + L.ev_off),
                             p.events + (static_cast<size_t>(bh) * nch + c) * static_cast<size_t>(cap) + first, evb, sb);
            }
            for (int t = lane; t < nt; t += 32) {
                const size_t th = (static_cast<size_t>(b) * p.T + static_cast<size_t>(c) * C + t) * p.H + h;
                bulk_g2s(smem_addr(st + L.v_off + static_cast<size_t>(t) * vrow),
                         static_cast<const unsigned char*>(p.v) + th * vrow, vrow, sb);
            }
            issued = c + 1;
        }
        for (int c = max(0, issued - S); c < issued; ++c) drain_copies(bar(BI.sfull + c % S), (c / S) & 1);
    }

    tmem_fence_before_sync();
    cluster_sync_all();  // no CTA leaves while a peer may still store into its shared memory
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, p.tmem_cols);
}

// Failure-detection self-test: one thread waits, through wait_bounded, on a barrier that
// nothing ever signals; the wait gives up after limit_ns and records kDevTimeout.
__global__ void k_wait_selftest(uint32_t* status, uint64_t limit_ns)
{
    __shared__ uint64_t never;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&never, 1);
        fence_mbar_init_cluster();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bounded<false>(smem_addr(&never), 0, status, &abort_flag, limit_ns);
}

}  // namespace

bool scan_plan(int M, int d_v, int K, int in_bytes, ScanPlan* out)
{
    const int cpl = d_v < 32 ? 1 : d_v / 32;
    int n = 0;
    for (int c : {1, 2, 4, 8}) {
        const int Ml = (M + c - 1) / c;
        const int cols = ((Ml + 3) / 4) * cpl;
        if (cols <= 512) {
            n = c;
            break;
        }
    }
    if (n == 0) return false;
    const int Ml = (M + n - 1) / n;
    const int cols = ((Ml + 3) / 4) * cpl;
    uint32_t alloc = 32;
    while (alloc < static_cast<uint32_t>(cols)) alloc <<= 1;
    const int S = 6, X = 2;
    int C = 64, P = 2;
    for (; C >= 1; C >>= 1) {
        const int ft = (C + kFinWarps / kFinGroups - 1) / (kFinWarps / kFinGroups);
        if (ft * cpl > (cpl <= 4 ? 16 : 8)) continue;  // z values a finisher lane holds per chunk
        const size_t t = scan_layout(Ml, C, K, d_v, in_bytes, S, P, X, n, hdr_words_of(kScanWarps, C)).total;
        if (t <= static_cast<size_t>(kSmemBudget)) break;
    }
    if (C < 1) return false;
    // a deeper read-partial ring, where it fits, lets the scan warps run further ahead of the
    // finishers; the depth stays a multiple of kFinGroups, so every ring slot serves one
    // finisher group and its barrier phases are consumed in order
    if (scan_layout(Ml, C, K, d_v, in_bytes, S, 2 * P, X, n, hdr_words_of(kScanWarps, C)).total <=
        static_cast<size_t>(kSmemBudget))
        P *= 2;
    out->ncta = n;
    out->nw = kScanWarps;
    out->nfin = kFinWarps;
    out->chunk = C;
    out->stages = S;
    out->lslots = P;
    out->xslots = X;
    out->cpl = cpl;
    out->hdr_words = hdr_words_of(kScanWarps, C);
    out->tmem_cols = alloc;
    // more than half of the SM's shared memory: exactly one CTA (and one TMEM owner) per SM
    const size_t t = scan_layout(Ml, C, K, d_v, in_bytes, S, P, X, n, out->hdr_words).total;
    if (out->ncta * out->nw > 128) return false;
    out->smem_bytes = t < 116 * 1024 ? 116 * 1024 : t;
    return true;
}

ScanWorkspace scan_workspace(int B, int T, int H, int K, const ScanPlan& plan)
{
    ScanWorkspace w;
    const size_t nch = (static_cast<size_t>(T) + plan.chunk - 1) / plan.chunk;
    w.events_bytes = static_cast<size_t>(B) * H * nch * 2 * plan.chunk * K * sizeof(uint4);
    w.hdr_off = (w.events_bytes + 255) & ~static_cast<size_t>(255);
    w.hdr_bytes = static_cast<size_t>(B) * H * nch * plan.ncta * plan.hdr_words * sizeof(uint32_t);
    w.total = w.hdr_off + w.hdr_bytes;
    return w;
}

cudaError_t launch_scan(const ScanParams& p, size_t smem_bytes, cudaStream_t stream)
{
    void (*kern)(ScanParams) = nullptr;
    const bool bf = p.in_bf16 != 0;
    switch (p.d_v < 32 ? 1 : p.d_v / 32) {
        case 1: kern = bf ? k_scan<1, true> : k_scan<1, false>; break;
        case 2: kern = bf ? k_scan<2, true> : k_scan<2, false>; break;
        case 4: kern = bf ? k_scan<4, true> : k_scan<4, false>; break;
        case 8: kern = bf ? k_scan<8, true> : k_scan<8, false>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.B * p.H * p.ncta), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>((p.nw + p.nfin + 1) * 32), 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(p.ncta);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream)
{
    k_wait_selftest<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace ramnet
