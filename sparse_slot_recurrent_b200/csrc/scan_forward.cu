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
// that quadrant.  Scan warp w (0..7) owns the local slots with s mod 8 == w, and with
// them their write masses (shared memory).
//
// Work per chunk of C tokens (the decode kernel has already sorted the chunk's events
// into one token-ordered list per owner warp, cut into batches on distinct slots):
//   loader warp    bulk-copies the chunk block (owner offsets, event records, write
//                  retentions), the chunk's value rows and this CTA's output-gate
//                  columns into a ring of shared-memory stages;
//   scan warps     walk their own list one batch at a time: one tcgen05.ld per event and
//                  one wait per batch; writes update mass, rate and content; reads are
//                  summed in registers per token and stored once per (warp, token) as a
//                  partial row plus a flag byte;
//   epilogue warps (a) add up a chunk's partial rows and push the sum to every CTA of
//                  the cluster (stores into the peers' shared memory), (b) kLag chunks
//                  later add the pushed sums of all CTAs, apply RMSNorm over d_v and the
//                  output gate, and store y for this CTA's share of the channels.  The
//                  lag hides the latency of the cross-SM exchange.
// Every hand-off is an mbarrier; every wait is bounded (about 2 s); a wait that gives up
// records RAMNET_ERR_TIMEOUT in the status word, raises the CTA's abort flag and the
// kernel carries on to the end without further waiting.
#include "common.cuh"
#include "kernels.h"

namespace ramnet {

namespace {

constexpr int kScanWarps = 8;
constexpr int kLoadWarp = 8;
constexpr int kEpiWarp0 = 9;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kScanWarps + 1 + kEpiWarps) * 32;
constexpr int kStages = 6;  // staging ring depth
constexpr int kLag = 2;     // the epilogue finishes chunk c - kLag after pushing chunk c
// ring of pushed sums: a CTA may push chunk d + kRecv into a peer only after that peer has
// finished chunk d; with the push of chunk c issued before finishing chunk c - kLag this
// needs kRecv >= 2 * kLag + 2
constexpr int kRecv = 2 * kLag + 2;

// mbarrier indices
constexpr int kBarStage = 0;                           // [kStages] staged data landed (tx)
constexpr int kBarStageFree = kBarStage + kStages;     // [kStages] scan + epilogue done with a stage
constexpr int kBarRowsFull = kBarStageFree + kStages;  // [2] scan warps done with a chunk
constexpr int kBarRowsFree = kBarRowsFull + 2;         // [2] epilogue consumed the partial rows
constexpr int kBarRecv = kBarRowsFree + 2;             // [kRecv] every CTA pushed its sums
constexpr int kBarFin = kBarRecv + kRecv;
constexpr int kNumBars = kBarFin + 1;

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct Layout {
    size_t bars, misc, m, stage, rows, flags, recv, total;
    size_t stage_bytes, blk_bytes, v_off, z_off, rows_bytes, flags_bytes, recv_bytes;
};

__host__ __device__ inline Layout scan_layout(int Ml, int C, int dv, int ncta, int es, size_t chunk_bytes)
{
    Layout L;
    L.blk_bytes = align16(chunk_bytes);
    L.v_off = L.blk_bytes;
    L.z_off = L.v_off + align16(static_cast<size_t>(C) * dv * es);
    L.stage_bytes = L.z_off + align16(static_cast<size_t>(C) * (dv / ncta) * es);
    L.rows_bytes = align16(sizeof(float) * C * kScanWarps * dv);
    L.flags_bytes = align16(static_cast<size_t>(C) * kScanWarps);
    L.recv_bytes = align16(sizeof(float) * ncta * C * dv);
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
    o += 2 * L.rows_bytes;
    L.flags = o;
    o += 2 * L.flags_bytes;
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

__device__ __forceinline__ bool try_wait_cta(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool try_wait_clu(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of the mbarrier at shared address `bar`: at most
// kSpinLimit polls and about 2 s.  On expiry the status word gets kDevTimeout and the
// CTA's abort flag is raised, after which every later wait of the CTA returns at once,
// so a kernel that lost a signal still ends within a few seconds.
template <bool kCluster>
__device__ __noinline__ void wait_bounded(uint32_t bar, uint32_t parity, uint32_t* status, volatile int* abort_flag)
{
    if (*abort_flag) return;
    const uint64_t t_end = global_ns() + 2000000000ull;
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        if (kCluster ? try_wait_clu(bar, parity) : try_wait_cta(bar, parity)) return;
        if ((it & 1023u) == 1023u && (global_ns() > t_end || *abort_flag)) break;
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
        if ((it & 1023u) == 1023u && global_ns() > t_end) return;
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

__device__ __forceinline__ void epi_barrier() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); }

// 16-byte store into the shared memory of cluster CTA `rank` (same offset as `local`).
__device__ __forceinline__ void st_cluster_v4(const void* local, uint32_t rank, float4 v)
{
    const uint32_t a = map_to_rank(smem_addr(local), rank);
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_f32(const void* local, uint32_t rank, float v)
{
    const uint32_t a = map_to_rank(smem_addr(local), rank);
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

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

// Push CPL values to the same location in cluster CTA `rank`.
template <int CPL>
__device__ __forceinline__ void push_row(float* dst, uint32_t rank, const float (&v)[CPL])
{
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int c = 0; c < CPL; c += 4) st_cluster_v4(dst + c, rank, make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]));
    } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) st_cluster_f32(dst + c, rank, v[c]);
    }
}

template <int CPL>
__global__ void __launch_bounds__(kThreads, 1) k_scan(ScanParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = p.chunk, dv = p.d_v, ncta = p.ncta, M = p.M;
    const int LW = dv < 32 ? dv : 32;  // lanes holding channels
    const int es = p.in_bf16 ? 2 : 4;
    const int Dr = dv / ncta;          // output channels of this CTA
    const uint32_t rank = ncta > 1 ? cluster_ctarank() : 0u;
    const int bh = blockIdx.x / ncta;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Ml = (M - static_cast<int>(rank) + ncta - 1) / ncta;
    const int nch = (p.T + C - 1) / C;
    const Layout L = scan_layout((M + ncta - 1) / ncta, C, dv, ncta, es, p.chunk_bytes);
    const uint32_t bars = smem_addr(smem + L.bars);
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    uint64_t* bar_ptr = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
    float* m_s = reinterpret_cast<float*>(smem + L.m);
    auto stage = [&](int c) { return smem + L.stage + static_cast<size_t>(c % kStages) * L.stage_bytes; };

    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar_ptr + kBarStage + i, 1);
            mbar_init(bar_ptr + kBarStageFree + i, (kScanWarps + kEpiWarps) * 32);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_ptr + kBarRowsFull + i, kScanWarps * 32);
            mbar_init(bar_ptr + kBarRowsFree + i, kEpiWarps * 32);
        }
        for (int i = 0; i < kRecv; ++i) mbar_init(bar_ptr + kBarRecv + i, static_cast<uint32_t>(ncta));
        mbar_init(bar_ptr + kBarFin, static_cast<uint32_t>(ncta));
        fence_mbar_init_cluster();
    }
    if (warp == 0) tmem_alloc(holder, p.tmem_cols);
    {
        uint32_t* fl = reinterpret_cast<uint32_t*>(smem + L.flags);
        for (size_t i = tid; i < 2 * L.flags_bytes / 4; i += kThreads) fl[i] = 0u;
        for (int s = tid; s < Ml; s += kThreads)
            m_s[s] = p.m_in != nullptr ? p.m_in[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] : 0.0f;
    }
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
        for (int s = warp; s < Ml; s += 8) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) r[c] = (p.S_in != nullptr && lane < LW) ? p.S_in[row + lch + c] : 0.0f;
            tmem_st<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
        }
        tmem_wait_st();
        for (int c = 0; c < nch; ++c) {
            const int rb = c & 1;
            wait_bounded<false>(bar(kBarStage + c % kStages), (c / kStages) & 1, p.status, abort_flag);
            if (c >= 2) wait_bounded<false>(bar(kBarRowsFree + rb), ((c - 2) >> 1) & 1, p.status, abort_flag);
            const unsigned char* st = stage(c);
            const int* ofs = reinterpret_cast<const int*>(st);
            const uint2* recs = reinterpret_cast<const uint2*>(st + p.recs_off);
            const float* alph = reinterpret_cast<const float*>(st + p.alph_off);
            const unsigned char* vb = st + L.v_off;
            float* rows = reinterpret_cast<float*>(smem + L.rows + rb * L.rows_bytes);
            unsigned char* flags = smem + L.flags + rb * L.flags_bytes;
            const int o = static_cast<int>(rank) * 8 + warp;
            int i = ofs[o];
            const int end = ofs[o + 1];
            int cur_t = -1;  // token whose read sum is being accumulated
            float acc[CPL];
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) acc[cc] = 0.0f;
            while (i < end) {
                const int nb = static_cast<int>((recs[i].x >> 10) & 0xFu);
                uint2 r[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) r[k] = k < nb ? recs[i + k] : make_uint2(0u, 0u);
                float S[8][CPL];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < nb) tmem_ld<CPL>(tq + (r[k].x & 0x3FFu), S[k]);
                // masses and rates of the batch's writes while the loads are in flight
                float lam[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    lam[k] = 0.0f;
                    if (k < nb && (r[k].x & 0x8000u)) {
                        const int s = 4 * static_cast<int>((r[k].x & 0x3FFu) / CPL) + q;
                        const float w = __uint_as_float(r[k].y);
                        const float mn = alph[i + k] * m_s[s] + w;
                        lam[k] = w * __frcp_rn(mn + p.eps_gsu);
                        __syncwarp();
                        if (lane == 0) m_s[s] = mn;
                    }
                }
                __syncwarp();
                tmem_wait_ld();
                bool any_write = false;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (k < nb) {
                        const int t = static_cast<int>(r[k].x >> 16);
                        if (r[k].x & 0x8000u) {
                            float vv[CPL];
                            load_row<CPL>(vb, t * dv + lch, p.in_bf16, vv);
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) S[k][cc] = fmaf(lam[k], vv[cc] - S[k][cc], S[k][cc]);
                            tmem_st<CPL>(tq + (r[k].x & 0x3FFu), S[k]);
                            any_write = true;
                        } else {
                            if (t != cur_t) {
                                if (cur_t >= 0) {
                                    if (lane < LW) store_row<CPL>(rows + (cur_t * kScanWarps + warp) * dv + lch, acc);
                                    if (lane == 0) flags[cur_t * kScanWarps + warp] = 1;
                                }
                                cur_t = t;
#pragma unroll
                                for (int cc = 0; cc < CPL; ++cc) acc[cc] = 0.0f;
                            }
                            const float rw = __uint_as_float(r[k].y);
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) acc[cc] = fmaf(rw, S[k][cc], acc[cc]);
                        }
                    }
                }
                if (any_write) tmem_wait_st();
                i += nb;
            }
            if (cur_t >= 0) {
                if (lane < LW) store_row<CPL>(rows + (cur_t * kScanWarps + warp) * dv + lch, acc);
                if (lane == 0) flags[cur_t * kScanWarps + warp] = 1;
            }
            arrive_cta(bar(kBarRowsFull + rb));
            arrive_cta(bar(kBarStageFree + c % kStages));
        }
        // final state of the owned slots
        for (int s = warp; s < Ml; s += 8) {
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
    } else if (warp == kLoadWarp) {
        // ============================================================ loader warp
        const uint32_t vrow = static_cast<uint32_t>(dv * es);
        const uint32_t zrow = static_cast<uint32_t>(Dr * es);
        const uint32_t blk = static_cast<uint32_t>(p.chunk_bytes);
        for (int c = 0; c < nch; ++c) {
            const int n = min(C, p.T - c * C);
            if (c >= kStages) {
                wait_bounded<false>(bar(kBarStageFree + c % kStages), (c / kStages - 1) & 1, p.status, abort_flag);
                fence_proxy_async();
            }
            unsigned char* st = stage(c);
            const uint32_t sb = bar(kBarStage + c % kStages);
            if (lane == 0) arrive_expect_tx(sb, blk + static_cast<uint32_t>(n) * (vrow + zrow));
            __syncwarp();
            if (lane == 0)
                bulk_g2s(smem_addr(st), p.blocks + (static_cast<size_t>(bh) * nch + c) * p.chunk_bytes, blk, sb);
            for (int t = lane; t < n; t += 32) {
                const size_t th = (static_cast<size_t>(b) * p.T + c * C + t) * p.H + h;
                bulk_g2s(smem_addr(st + L.v_off + static_cast<size_t>(t) * vrow),
                         static_cast<const unsigned char*>(p.v) + th * vrow, vrow, sb);
                bulk_g2s(smem_addr(st + L.z_off + static_cast<size_t>(t) * zrow),
                         static_cast<const unsigned char*>(p.z) + (th * dv + static_cast<size_t>(rank) * Dr) * es, zrow, sb);
            }
        }
    } else {
        // ============================================================ epilogue warps
        const int e = warp - kEpiWarp0;
        const int lch = (lane < LW ? lane : 0) * CPL;
        const bool mine = lane < LW && lch >= static_cast<int>(rank) * Dr && lch < (static_cast<int>(rank) + 1) * Dr;
        float nw[CPL];
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) nw[cc] = p.norm_w != nullptr ? p.norm_w[lch + cc] : 1.0f;
        for (int c = 0; c < nch + kLag; ++c) {
            // (a) chunk c: sum this CTA's partial rows and push them to every CTA
            if (c < nch) {
                const int rb = c & 1;
                const int n = min(C, p.T - c * C);
                wait_bounded<false>(bar(kBarRowsFull + rb), (c >> 1) & 1, p.status, abort_flag);
                const float* rows = reinterpret_cast<const float*>(smem + L.rows + rb * L.rows_bytes);
                unsigned char* flags = smem + L.flags + rb * L.flags_bytes;
                float* recv = reinterpret_cast<float*>(smem + L.recv + (c % kRecv) * L.recv_bytes);
                for (int t = e; t < n; t += kEpiWarps) {
                    const uint2 fw = *reinterpret_cast<const uint2*>(flags + t * kScanWarps);
                    float o[CPL];
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) o[cc] = 0.0f;
#pragma unroll
                    for (int w = 0; w < kScanWarps; ++w) {
                        const uint32_t f = w < 4 ? (fw.x >> (8 * w)) & 0xFFu : (fw.y >> (8 * (w - 4))) & 0xFFu;
                        if (f) {
                            float pr[CPL];
                            load_row<CPL>(reinterpret_cast<const unsigned char*>(rows), (t * kScanWarps + w) * dv + lch, 0, pr);
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) o[cc] += pr[cc];
                        }
                    }
                    __syncwarp();
                    if (lane < 2) reinterpret_cast<uint32_t*>(flags + t * kScanWarps)[lane] = 0u;
                    // recv[r'][t][dv]: slot r' holds CTA r''s partial sums
                    float* dst = recv + (static_cast<size_t>(rank) * C + t) * dv + lch;
                    if (lane < LW) {
                        if (ncta == 1) {
                            store_row<CPL>(dst, o);
                        } else {
                            for (int r = 0; r < ncta; ++r) push_row<CPL>(dst, static_cast<uint32_t>(r), o);
                        }
                    }
                }
                arrive_cta(bar(kBarRowsFree + rb));
                epi_barrier();
                if (tid == kEpiWarp0 * 32) {
                    if (ncta == 1) {
                        arrive_cta(bar(kBarRecv + c % kRecv));
                    } else {
                        for (int r = 0; r < ncta; ++r)
                            mbar_arrive_cluster(map_to_rank(bar(kBarRecv + c % kRecv), static_cast<uint32_t>(r)));
                    }
                }
            }
            // (b) chunk d = c - kLag: all CTAs' sums are in; RMSNorm, gate, y
            if (c >= kLag) {
                const int d = c - kLag;
                const int n = min(C, p.T - d * C);
                wait_bounded<true>(bar(kBarRecv + d % kRecv), (d / kRecv) & 1, p.status, abort_flag);
                const float* recv = reinterpret_cast<const float*>(smem + L.recv + (d % kRecv) * L.recv_bytes);
                const unsigned char* zb = stage(d) + L.z_off;
                for (int t = e; t < n; t += kEpiWarps) {
                    float o[CPL];
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) o[cc] = 0.0f;
                    if (lane < LW) {
                        for (int r = 0; r < ncta; ++r) {
                            float pr[CPL];
                            load_row<CPL>(reinterpret_cast<const unsigned char*>(recv), (r * C + t) * dv + lch, 0, pr);
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
                    if (mine) {
                        float zz[CPL];
                        load_row<CPL>(zb, t * Dr + lch - static_cast<int>(rank) * Dr, p.in_bf16, zz);
                        const size_t base = ((static_cast<size_t>(b) * p.T + d * C + t) * p.H + h) * dv + lch;
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) store_out(p.y, base + cc, o[cc] * inv * nw[cc] * zz[cc], p.out_bf16);
                    }
                }
                arrive_cta(bar(kBarStageFree + d % kStages));
            }
        }
    }

    // copies still in flight after an abort must land before the CTA exits
    if (warp == kLoadWarp) {
        for (int c = max(0, nch - kStages); c < nch; ++c) drain_copies(bar(kBarStage + c % kStages), (c / kStages) & 1);
    }
    // no CTA leaves while a peer may still write into its shared memory
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

}  // namespace

size_t chunk_block_bytes(int chunk, int K, int ncta, size_t* recs_off, size_t* alph_off)
{
    const size_t E = static_cast<size_t>(2) * chunk * K;
    const size_t ro = align16(sizeof(int) * (8 * ncta + 1));
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
    int C = 16;
    auto total = [&](int cc) {
        return scan_layout(Ml, cc, d_v, n, in_bytes, chunk_block_bytes(cc, K, n, nullptr, nullptr)).total;
    };
    const size_t budget = 220 * 1024;
    while (C > 2 && total(C) > budget) C >>= 1;
    if (total(C) > budget) return false;
    out->ncta = n;
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
