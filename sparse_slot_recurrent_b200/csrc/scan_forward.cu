// scan_forward.cu -- K2: the prefill recurrence of the RAM-Net layer core.
//
// RAM-Net project page: the three-stage paragraph (decode, CAPE, GSU, then read,
// normalise, gate), the Gated Sparse Update paragraphs (four steps; unselected slots
// unchanged) and the GPU-execution paragraph (addresses for all tokens first, events
// grouped by slot, each slot's events in causal order, slots and channels in parallel).
//
// State layout.  One head's slot array S [M, d_v] fp32 lives in tensor memory (TMEM) for
// the whole sequence, spread over a cluster of `ncta` CTAs, one per SM.  Slot i belongs
// to CTA (i mod ncta) as local slot s = i / ncta, which sits in TMEM lane quadrant
// (s mod 4), columns [(s/4)*CPL, (s/4)*CPL + CPL); lane l of the quadrant holds channels
// [l*CPL, l*CPL + CPL).  One slot row is one tcgen05.ld/st of CPL columns by a warp of
// that quadrant.  Scan warp w (0..kScanWarps-1) owns the local slots with
// s mod kScanWarps == w, so each slot's events are applied by one warp, in token order.
//
// Work per chunk of C tokens (the decode kernel has already sorted the chunk's events
// into one token-ordered list per owner warp):
//   loader warp    bulk-copies the chunk block (owner offsets, event records, write
//                  retentions), the chunk's value rows and the output-gate rows of the
//                  tokens this CTA finishes into a ring of shared-memory stages;
//   mass warps     once a stage has landed, run GSU steps 1-3 (retention, mass, rate)
//                  for the writes of four owners each, 32 events per instruction, and
//                  write each rate into its event record;
//   scan warps     walk their own list one event at a time (one tcgen05.ld each): writes
//                  apply step 4 (content); reads are weighted and stored into row
//                  (token, r) of the read buffer, r = the read's rank within its token
//                  (K <= kScanWarps) or the scan warp (larger K: the warp's reads of one
//                  token are added up first), setting bit r of the token's mask.  After a
//                  barrier the scan warps add up each token's rows and send the sum to
//                  the CTA that finishes the token (token t: CTA t mod ncta), into slot
//                  (chunk mod kRecv) of its receive ring, by stores into its shared
//                  memory, then signal that CTA's receive barrier;
//   epilogue warps wait until every CTA has sent its sums of a chunk, add them up for
//                  the tokens of this CTA, apply RMSNorm over d_v, the norm weight and
//                  the output gate, store y and hand the receive slot back to all
//                  senders.
// Every hand-off is an mbarrier; every wait is bounded (about 2 s); a wait that gives up
// records RAMNET_ERR_TIMEOUT in the status word, raises the CTA's abort flag and the
// kernel carries on to the end without further waiting (all loops are bounded by the
// chunk's event capacity, so they end even on garbage).
#include "common.cuh"
#include "kernels.h"

namespace ramnet {

namespace {

constexpr int kScanWarps = 16;
constexpr int kLoadWarp = kScanWarps;
constexpr int kMassWarp0 = kScanWarps + 1;
constexpr int kMassWarps = 4;  // each takes kScanWarps / kMassWarps owners
constexpr int kEpiWarp0 = kMassWarp0 + kMassWarps;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int kStages = 6;  // staging ring depth
constexpr int kRecv = 4;    // receive ring depth
constexpr int kOwnPerMass = kScanWarps / kMassWarps;

// mbarrier indices
constexpr int kBarStage = 0;                          // [kStages] staged data landed (tx)
constexpr int kBarReady = kBarStage + kStages;        // [kStages] rates of the stage's writes computed
constexpr int kBarStageFree = kBarReady + kStages;    // [kStages] scan + epilogue warps done with a stage
constexpr int kBarRecv = kBarStageFree + kStages;     // [kRecv] every CTA sent its sums (remote arrivals)
constexpr int kBarRecvFree = kBarRecv + kRecv;        // [kRecv] every CTA finished a slot (remote arrivals)
constexpr int kBarFin = kBarRecvFree + kRecv;
constexpr int kNumBars = kBarFin + 1;

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

// Rows of the read buffer per token: one per read rank j when K <= kScanWarps, else one
// per scan warp (a warp's reads of one token are adjacent in its list and are summed in
// registers first).
__host__ __device__ inline int rows_per_token(int K) { return K <= kScanWarps ? K : kScanWarps; }

struct Layout {
    size_t bars, misc, m, stage, rows, flags, recv, total;
    size_t stage_bytes, blk_bytes, v_off, z_off, rows_bytes, flags_bytes, recv_bytes;
};

__host__ __device__ inline Layout scan_layout(int Ml, int C, int K, int dv, int ncta, int es, size_t chunk_bytes)
{
    Layout L;
    L.blk_bytes = align16(chunk_bytes);
    L.v_off = L.blk_bytes;
    L.z_off = L.v_off + align16(static_cast<size_t>(C) * dv * es);
    L.stage_bytes = L.z_off + align16(static_cast<size_t>(C) * dv * es);
    L.rows_bytes = align16(sizeof(float) * C * rows_per_token(K) * dv);
    L.flags_bytes = static_cast<size_t>(16) * C;  // one byte per read row, 16 per token
    L.recv_bytes = align16(sizeof(float) * ncta * ((C + ncta - 1) / ncta) * dv);  // [source CTA][own token][d_v]
    size_t o = 0;
    L.bars = o;
    o += align16(8 * kNumBars);
    L.misc = o;
    o += 16;
    L.m = o;
    o += align16(sizeof(float) * Ml);
    L.stage = o;
    o += kStages * L.stage_bytes;
    L.rows = o;
    o += L.rows_bytes;
    L.flags = o;
    o += L.flags_bytes;
    L.recv = o;
    o += kRecv * L.recv_bytes;
    L.total = o;
    return L;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// One try_wait on phase `parity`: the thread is suspended in hardware until the phase
// completes or about kSuspendNs have passed, so a waiting warp issues almost nothing.
constexpr uint32_t kSuspendNs = 100000;

__device__ __forceinline__ bool try_wait_cta(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool try_wait_clu(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of the mbarrier at shared address `bar`: at most
// kSpinLimit polls and `limit_ns` (2 s unless given).  On expiry the status word gets
// kDevTimeout and the CTA's abort flag is raised, after which every later wait of the CTA
// returns at once, so a kernel that lost a signal still ends within a few seconds.
template <bool kCluster>
__device__ __noinline__ void wait_bounded(uint32_t bar, uint32_t parity, uint32_t* status, volatile int* abort_flag,
                                          uint64_t limit_ns = 2000000000ull)
{
    if (*abort_flag) return;
    const uint64_t t_end = global_ns() + limit_ns;
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        if (kCluster ? try_wait_clu(bar, parity) : try_wait_cta(bar, parity)) return;
        if (global_ns() > t_end || *abort_flag) break;
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
        if (try_wait_cta(bar, parity)) return;
        if (global_ns() > t_end) return;
    }
}

__device__ __forceinline__ void arrive_cta(uint32_t bar)
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

// named barriers: 1 = the scan warps, 2 = the epilogue warps (0 is __syncthreads)
__device__ __forceinline__ void scan_barrier() { asm volatile("bar.sync 1, %0;" ::"n"(kScanWarps * 32) : "memory"); }
__device__ __forceinline__ void epi_barrier() { asm volatile("bar.sync 2, %0;" ::"n"(kEpiWarps * 32) : "memory"); }

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

template <int CPL>
__device__ __forceinline__ void store_row(float* dst, const float (&v)[CPL])
{
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int c = 0; c < CPL; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) dst[c] = v[c];
    }
}

// Push CPL values to shared::cluster address `caddr` (already mapped to the target CTA).
template <int CPL>
__device__ __forceinline__ void push_row(uint32_t caddr, const float (&v)[CPL])
{
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int c = 0; c < CPL; c += 4)
            asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(caddr + 4u * c), "f"(v[c]), "f"(v[c + 1]),
                         "f"(v[c + 2]), "f"(v[c + 3])
                         : "memory");
    } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(caddr + 4u * c), "f"(v[c]) : "memory");
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
        float* pf = reinterpret_cast<float*>(y) + elem;
        if constexpr (CPL % 4 == 0) {
#pragma unroll
            for (int c = 0; c < CPL; c += 4) *reinterpret_cast<float4*>(pf + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) pf[c] = v[c];
        }
    }
}

// Signal mbarrier `b` (a shared::cta address) in every CTA of the cluster.
__device__ __forceinline__ void arrive_all(uint32_t b, int ncta)
{
    if (ncta == 1) {
        arrive_cta(b);
    } else {
        for (int r = 0; r < ncta; ++r) mbar_arrive_cluster(map_to_rank(b, static_cast<uint32_t>(r)));
    }
}

template <int CPL>
__global__ void __launch_bounds__(kThreads, 1) k_scan(ScanParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = p.chunk, dv = p.d_v, ncta = p.ncta, M = p.M, K = p.K;
    const int LW = (CPL > 1 || dv >= 32) ? 32 : dv;  // lanes holding channels (32 unless d_v = 16)
    const int es = p.in_bf16 ? 2 : 4;
    const uint32_t rank = ncta > 1 ? cluster_ctarank() : 0u;
    const int bh = blockIdx.x / ncta;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Ml = (M - static_cast<int>(rank) + ncta - 1) / ncta;
    const int nch = (p.T + C - 1) / C;
    const int E = 2 * C * K;  // event capacity of a chunk; bounds every list walk
    const int Cown = (C + ncta - 1) / ncta;
    const Layout L = scan_layout((M + ncta - 1) / ncta, C, K, dv, ncta, es, p.chunk_bytes);
    const uint32_t bars = smem_addr(smem + L.bars);
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    uint64_t* bar_ptr = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
    float* m_s = reinterpret_cast<float*>(smem + L.m);
    float* rows = reinterpret_cast<float*>(smem + L.rows);
    unsigned char* flags = smem + L.flags;  // [C][16]: 1 where read row (t, r) was written
    auto stage = [&](int c) { return smem + L.stage + static_cast<size_t>(c % kStages) * L.stage_bytes; };
    auto recv_slot = [&](int c) { return reinterpret_cast<float*>(smem + L.recv + (c % kRecv) * L.recv_bytes); };
    const int NWc = kScanWarps;  // owners per CTA
    const int R = rows_per_token(K);
    const bool byw = K > kScanWarps;

    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar_ptr + kBarStage + i, 1);
            mbar_init(bar_ptr + kBarReady + i, kMassWarps * 32);
            mbar_init(bar_ptr + kBarStageFree + i, (kScanWarps + kEpiWarps) * 32);
        }
        for (int i = 0; i < kRecv; ++i) {
            mbar_init(bar_ptr + kBarRecv + i, static_cast<uint32_t>(ncta));
            mbar_init(bar_ptr + kBarRecvFree + i, static_cast<uint32_t>(ncta));
        }
        mbar_init(bar_ptr + kBarFin, static_cast<uint32_t>(ncta));
        fence_mbar_init_cluster();
    }
    if (warp == 0) tmem_alloc(holder, p.tmem_cols);
    for (int i = tid; i < 4 * C; i += kThreads) reinterpret_cast<uint32_t*>(flags)[i] = 0u;
    for (int s = tid; s < Ml; s += kThreads)
        m_s[s] = p.m_in != nullptr ? p.m_in[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] : 0.0f;
    tmem_fence_before_sync();
    __syncthreads();
    if (ncta > 1) cluster_sync_all();
    tmem_fence_after_sync();
    const uint32_t tbase = *holder;

    if (warp < kScanWarps) {
        // ============================================================ scan warps
        const int q = warp & 3;
        const uint32_t tq = tbase + (static_cast<uint32_t>(32 * q) << 16);
        const int lch = (lane < LW ? lane : 0) * CPL;  // this lane's first channel
        for (int s = warp; s < Ml; s += kScanWarps) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) r[c] = (p.S_in != nullptr && lane < LW) ? p.S_in[row + lch + c] : 0.0f;
            tmem_st<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
        }
        tmem_wait_st();
        for (int c = 0; c < nch; ++c) {
            const int n = min(C, p.T - c * C);
            wait_bounded<false>(bar(kBarReady + c % kStages), (c / kStages) & 1, p.status, abort_flag);
            const unsigned char* st = stage(c);
            const int* ofs = reinterpret_cast<const int*>(st);
            const uint2* recs = reinterpret_cast<const uint2*>(st + p.recs_off);
            const unsigned char* vb = st + L.v_off;
            const int o = static_cast<int>(rank) * NWc + warp;
            const int beg = min(max(ofs[o], 0), E);
            const int end = min(max(ofs[o + 1], beg), E);
            uint2 nxt = beg < end ? recs[beg] : make_uint2(0u, 0u);
            float vn[CPL];  // value row of event `nxt` (writes)
            load_row<CPL>(vb, static_cast<int>(nxt.x >> 24) * dv + lch, p.in_bf16, vn);
            int cur_t = -1, cur_r = 0;  // read row being summed
            float acc[CPL];
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) acc[cc] = 0.0f;
            for (int i = beg; i < end; ++i) {
                const uint2 rec = nxt;
                float vv[CPL];
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) vv[cc] = vn[cc];
                const uint32_t col = rec.x & 0x3FFu;
                const int t = static_cast<int>(rec.x >> 24);
                const float cf = __uint_as_float(rec.y);
                float S[CPL];
                tmem_ld<CPL>(tq + col, S);
                if (i + 1 < end) {
                    nxt = recs[i + 1];
                    load_row<CPL>(vb, static_cast<int>(nxt.x >> 24) * dv + lch, p.in_bf16, vn);
                }
                if (rec.x & 0x8000u) {
                    // Gated Sparse Update step 4: S += lambda * (v - S)
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) S[cc] = fmaf(cf, vv[cc] - S[cc], S[cc]);
                    tmem_st<CPL>(tq + col, S);
                    tmem_wait_st();
                } else if (!byw) {
                    // read j of token t: its weighted row goes straight to read row (t, j)
                    const int j = static_cast<int>((rec.x >> 16) & 0x3Fu);
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) S[cc] *= cf;
                    if (lane < LW) store_row<CPL>(rows + (t * R + j) * dv + lch, S);
                    flags[t * 16 + j] = 1;  // every lane stores the same byte
                } else {
                    // read, K > kScanWarps: summed into read row (t, warp) first
                    tmem_wait_ld();
                    if (t != cur_t) {
                        if (cur_t >= 0) {
                            if (lane < LW) store_row<CPL>(rows + (cur_t * R + cur_r) * dv + lch, acc);
                            flags[cur_t * 16 + cur_r] = 1;
                        }
                        cur_t = t;
                        cur_r = warp;
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) acc[cc] = 0.0f;
                    }
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) acc[cc] = fmaf(cf, S[cc], acc[cc]);
                }
            }
            if (cur_t >= 0) {
                if (lane < LW) store_row<CPL>(rows + (cur_t * R + cur_r) * dv + lch, acc);
                flags[cur_t * 16 + cur_r] = 1;
            }
            scan_barrier();  // every read row of the chunk is in
            // the receivers must have finished the chunk that last used this ring slot
            if (c >= kRecv)
                wait_bounded<true>(bar(kBarRecvFree + c % kRecv), ((c - kRecv) / kRecv) & 1, p.status, abort_flag);
            // this CTA's part of each token's read: sum its rows, send it to the token's CTA
            float* slot = recv_slot(c);
            for (int t = warp; t < n; t += kScanWarps) {
                const uint4 fb = *reinterpret_cast<const uint4*>(flags + t * 16);
                unsigned long long fm = 0ull;  // bit r: read row (t, r) present
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t wv = q4 == 0 ? fb.x : q4 == 1 ? fb.y : q4 == 2 ? fb.z : fb.w;
#pragma unroll
                    for (int by = 0; by < 4; ++by)
                        fm |= static_cast<unsigned long long>(((wv >> (8 * by)) & 0xFFu) != 0u) << (4 * q4 + by);
                }
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) acc[cc] = 0.0f;
                for (int guard = 0; fm != 0ull && guard < 64; ++guard) {
                    const int j = __ffsll(static_cast<long long>(fm)) - 1;
                    fm &= fm - 1ull;
                    float pr[CPL];
                    load_row<CPL>(reinterpret_cast<const unsigned char*>(rows), (t * R + j) * dv + lch, 0, pr);
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) acc[cc] += pr[cc];
                }
                __syncwarp();
                if (lane == 0) *reinterpret_cast<uint4*>(flags + t * 16) = make_uint4(0u, 0u, 0u, 0u);
                float* dst = slot + (static_cast<size_t>(rank) * Cown + t / ncta) * dv + lch;
                const uint32_t owner = static_cast<uint32_t>(t % ncta);
                if (lane < LW) {
                    if (owner == rank) store_row<CPL>(dst, acc);
                    else push_row<CPL>(map_to_rank(smem_addr(dst), owner), acc);
                }
            }
            arrive_cta(bar(kBarStageFree + c % kStages));
            scan_barrier();  // every sum of the chunk is sent; the read buffer is free
            if (warp == 0 && lane == 0) arrive_all(bar(kBarRecv + c % kRecv), ncta);
        }
        // final state of the owned slots
        for (int s = warp; s < Ml; s += kScanWarps) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
            tmem_ld<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
            tmem_wait_ld();
            if (lane < LW) {
#pragma unroll
                for (int c = 0; c < CPL; ++c) p.S_out[row + lch + c] = r[c];
            }
        }
    } else if (warp == kLoadWarp) {
        // ============================================================ loader warp
        const uint32_t vrow = static_cast<uint32_t>(dv * es);
        const uint32_t blk = static_cast<uint32_t>(p.chunk_bytes);
        for (int c = 0; c < nch; ++c) {
            const int n = min(C, p.T - c * C);
            if (c >= kStages) {
                wait_bounded<false>(bar(kBarStageFree + c % kStages), (c / kStages - 1) & 1, p.status, abort_flag);
                fence_proxy_async();
            }
            unsigned char* st = stage(c);
            const uint32_t sb = bar(kBarStage + c % kStages);
            const int nz = (n - static_cast<int>(rank) + ncta - 1) / ncta;  // tokens this CTA finishes
            if (lane == 0) arrive_expect_tx(sb, blk + static_cast<uint32_t>(n + nz) * vrow);
            __syncwarp();
            if (lane == 0)
                bulk_g2s(smem_addr(st), p.blocks + (static_cast<size_t>(bh) * nch + c) * p.chunk_bytes, blk, sb);
            for (int t = lane; t < n; t += 32) {
                const size_t th = (static_cast<size_t>(b) * p.T + c * C + t) * p.H + h;
                bulk_g2s(smem_addr(st + L.v_off + static_cast<size_t>(t) * vrow),
                         static_cast<const unsigned char*>(p.v) + th * vrow, vrow, sb);
                if (t % ncta == static_cast<int>(rank))
                    bulk_g2s(smem_addr(st + L.z_off + static_cast<size_t>(t) * vrow),
                             static_cast<const unsigned char*>(p.z) + th * vrow, vrow, sb);
            }
        }
        for (int c = max(0, nch - kStages); c < nch; ++c) drain_copies(bar(kBarStage + c % kStages), (c / kStages) & 1);
    } else if (warp < kEpiWarp0) {
        // ============================================================ mass warps
        // GSU steps 1-3 for the writes of owners [mi*kOwnPerMass, (mi+1)*kOwnPerMass):
        // m = alpha*m + w, lambda = w / (m + eps).  An owner's events are in token order,
        // so one slot's writes appear in token order; within a group of 32 events,
        // same-slot chains are resolved lane by lane.
        const int mi = warp - kMassWarp0;
        const int o0 = static_cast<int>(rank) * NWc + mi * kOwnPerMass;
        for (int c = 0; c < nch; ++c) {
            wait_bounded<false>(bar(kBarStage + c % kStages), (c / kStages) & 1, p.status, abort_flag);
            unsigned char* st = stage(c);
            const int* ofs = reinterpret_cast<const int*>(st);
            uint2* recs = reinterpret_cast<uint2*>(st + p.recs_off);
            const float* alph = reinterpret_cast<const float*>(st + p.alph_off);
            const int lo = min(max(ofs[o0], 0), E), hi = min(max(ofs[o0 + kOwnPerMass], lo), E);
            const int seg = lane < kOwnPerMass ? ofs[o0 + lane] : 0x7fffffff;  // owner segment starts
            for (int base = lo; base < hi; base += 32) {
                const int idx = base + lane;
                const uint2 rec = idx < hi ? recs[idx] : make_uint2(0u, 0u);
                const bool wr = idx < hi && (rec.x & 0x8000u);
                // owner warp of this event: its segment is the last one starting at or before idx
                int w = mi * kOwnPerMass;
#pragma unroll
                for (int j = 1; j < kOwnPerMass; ++j) w += idx >= __shfl_sync(0xffffffffu, seg, j) ? 1 : 0;
                const int sl = 4 * static_cast<int>((rec.x & 0x3FFu) / CPL) + (w & 3);
                const uint32_t peers = __match_any_sync(0xffffffffu, wr ? sl : -1 - lane);
                const uint32_t lt = (1u << lane) - 1u;
                const uint32_t before = peers & lt;
                const int pred = before ? 31 - __clz(before) : lane;
                const int depth = static_cast<int>(__reduce_max_sync(0xffffffffu, static_cast<unsigned>(__popc(before))));
                const float al = wr ? alph[idx] : 1.0f;
                const float wt = wr ? __uint_as_float(rec.y) : 0.0f;
                float mn = al * (wr ? m_s[sl] : 0.0f) + wt;
                for (int dd = 0; dd < depth; ++dd) {
                    const float mp = __shfl_sync(0xffffffffu, mn, pred);
                    if (before) mn = al * mp + wt;
                }
                __syncwarp();
                if (wr) {
                    if ((peers & ~lt & ~(1u << lane)) == 0u) m_s[sl] = mn;  // last write of this slot
                    recs[idx].y = __float_as_uint(__fdividef(wt, mn + p.eps_gsu));
                }
                __syncwarp();
            }
            // the rates were written through the generic proxy into memory that a later
            // bulk copy overwrites
            fence_proxy_async();
            arrive_cta(bar(kBarReady + c % kStages));
        }
        for (int s = lane; s < Ml; s += 32)
            if (((s & (kScanWarps - 1)) / kOwnPerMass) == mi)
                p.m_out[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] = m_s[s];
    } else {
        // ============================================================ epilogue warps
        const int e = warp - kEpiWarp0;
        const int lch = (lane < LW ? lane : 0) * CPL;
        float nw[CPL];
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) nw[cc] = p.norm_w != nullptr ? p.norm_w[lch + cc] : 1.0f;
        for (int d = 0; d < nch; ++d) {
            const int n = min(C, p.T - d * C);
            wait_bounded<true>(bar(kBarRecv + d % kRecv), (d / kRecv) & 1, p.status, abort_flag);
            const float* slot = recv_slot(d);
            const unsigned char* zb = stage(d) + L.z_off;
            for (int t = static_cast<int>(rank) + e * ncta; t < n; t += kEpiWarps * ncta) {
                float o[CPL];
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) o[cc] = 0.0f;
                if (lane < LW) {
                    for (int r = 0; r < ncta; ++r) {
                        float pr[CPL];
                        load_row<CPL>(reinterpret_cast<const unsigned char*>(slot), (r * Cown + t / ncta) * dv + lch, 0, pr);
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) o[cc] += pr[cc];
                    }
                }
                float sq = 0.0f;
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) sq = fmaf(o[cc], o[cc], sq);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
                const float inv = 1.0f / sqrtf(sq / dv + p.eps_norm);
                if (lane < LW) {
                    float zz[CPL];
                    load_row<CPL>(zb, t * dv + lch, p.in_bf16, zz);
                    const size_t base = ((static_cast<size_t>(b) * p.T + d * C + t) * p.H + h) * dv + lch;
                    float yv[CPL];
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) yv[cc] = o[cc] * inv * nw[cc] * zz[cc];
                    store_y<CPL>(p.y, base, yv, p.out_bf16);
                }
            }
            arrive_cta(bar(kBarStageFree + d % kStages));
            epi_barrier();  // all of this CTA's reads of the receive slot are done
            if (warp == kEpiWarp0 && lane == 0) arrive_all(bar(kBarRecvFree + d % kRecv), ncta);
        }
    }

    // no CTA leaves while a peer may still write into its shared memory or signal it
    __syncthreads();
    if (ncta > 1 && tid == 0) {
        for (int r = 0; r < ncta; ++r) mbar_arrive_cluster(map_to_rank(bar(kBarFin), static_cast<uint32_t>(r)));
        wait_bounded<true>(bar(kBarFin), 0, p.status, abort_flag);
    }
    tmem_fence_before_sync();
    __syncthreads();
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

cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream)
{
    k_wait_selftest<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

size_t chunk_block_bytes(int chunk, int K, int ncta, int nwarps, size_t* recs_off, size_t* alph_off)
{
    const size_t E = static_cast<size_t>(2) * chunk * K;
    const size_t ro = align16(sizeof(int) * (nwarps * ncta + 1));
    const size_t ao = ro + align16(sizeof(uint2) * E);
    if (recs_off) *recs_off = ro;
    if (alph_off) *alph_off = ao;
    return align16(ao + sizeof(float) * E);
}

bool scan_plan(int M, int d_v, int K, int in_bytes, ScanPlan* out)
{
    const int cpl = d_v < 32 ? 1 : d_v / 32;
    int n = 0;
    for (int c : {1, 2, 4, 8}) {
        const int Ml = (M + c - 1) / c;
        const int cols = ((Ml + 3) / 4) * cpl;
        if (cols <= 512 && d_v % c == 0) {
            n = c;
            break;
        }
    }
    if (n == 0) return false;
    const int Ml = (M + n - 1) / n;
    const int cols = ((Ml + 3) / 4) * cpl;
    uint32_t alloc = 32;
    while (alloc < static_cast<uint32_t>(cols)) alloc <<= 1;
    // output-gate columns of one CTA are copied per token with 16-byte bulk copies
    if (d_v / n < 8) return false;
    int C = 32;
    auto total = [&](int cc) {
        return scan_layout(Ml, cc, K, d_v, n, in_bytes, chunk_block_bytes(cc, K, n, kScanWarps, nullptr, nullptr)).total;
    };
    // the decode/route kernel's block for the largest number of chunks per block
    auto route = [&](int cc) { return route_smem_bytes(cc, route_chunks_per_block(cc, 1 << 30), K, n * kScanWarps); };
    const size_t budget = 220 * 1024;
    while (C > 2 && (total(C) > budget || route(C) > budget)) C >>= 1;
    if (total(C) > budget || route(C) > budget) return false;
    out->ncta = n;
    out->nwarps = kScanWarps;
    out->chunk = C;
    out->cpl = cpl;
    out->tmem_cols = alloc;
    // more than half of the SM's shared memory: exactly one CTA (and one TMEM owner) per SM
    const size_t t = total(C);
    out->smem_bytes = t < 116 * 1024 ? 116 * 1024 : t;
    out->nchunks = 0;
    return true;
}

cudaError_t launch_scan(const ScanParams& p, size_t smem_bytes, cudaStream_t stream)
{
    void (*kern)(ScanParams) = nullptr;
    switch (p.d_v < 32 ? 1 : p.d_v / 32) {
        case 1: kern = k_scan<1>; break;
        case 2: kern = k_scan<2>; break;
        case 4: kern = k_scan<4>; break;
        case 8: kern = k_scan<8>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.B * p.H * p.ncta));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(p.ncta);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ScanParams pc = p;
    return cudaLaunchKernelEx(&cfg, kern, pc);
}

}  // namespace ramnet
