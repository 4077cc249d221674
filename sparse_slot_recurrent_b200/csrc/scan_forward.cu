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
// into one token-ordered list per owner warp):
//   loader warp    bulk-copies this CTA's lists, the write retentions and the chunk's
//                  value rows into shared memory (2-deep ring);
//   scan warps     walk their own list in batches of up to 4 events on distinct slots:
//                  one tcgen05.ld per event, one wait, then writes (mass, rate, content)
//                  and reads (weighted row red-added into the chunk's o buffer);
//   epilogue warps add the partial o of all CTAs of the cluster through distributed
//                  shared memory, exchange the squared norms the same way, and write
//                  y = o / rms(o) * norm_w * z for this CTA's share of the channels.
// Every hand-off is an mbarrier; every wait is bounded (about 2 s); a wait that gives up
// records RAMNET_ERR_TIMEOUT in the status word and the kernel carries on to the end.
#include "common.cuh"
#include "kernels.h"

namespace ramnet {

namespace {

constexpr int kScanWarps = 8;
constexpr int kLoadWarp = 8;
constexpr int kEpiWarp0 = 9;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kScanWarps + 1 + kEpiWarps) * 32;

enum Bar { kStage = 0, kScan = 2, kOFree = 4, kZ = 6, kPeerO = 8, kPeerSS = 10, kFin = 12, kNumBars = 13 };

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct Layout {
    size_t bars, holder, m, offs, recs, alph, vbuf, zbuf, obuf, ss, total;
    size_t recs_bytes, alph_bytes, vbuf_bytes, zbuf_bytes, obuf_bytes;
};

__host__ __device__ inline Layout scan_layout(int Ml, int C, int K, int dv, int ncta, int es)
{
    Layout L;
    L.recs_bytes = align16(sizeof(uint2) * (2 * C * K + 4));
    L.alph_bytes = align16(sizeof(float) * (2 * C * K + 8));
    L.vbuf_bytes = align16(static_cast<size_t>(C) * dv * es);
    L.zbuf_bytes = align16(static_cast<size_t>(C) * (dv / ncta) * es);
    L.obuf_bytes = align16(sizeof(float) * C * dv);
    size_t o = 0;
    L.bars = o;
    o += align16(8 * kNumBars);
    L.holder = o;
    o += 16;
    L.offs = o;  // per buffer: 9 owner offsets + record base + alpha base
    o += align16(sizeof(int) * 2 * 12);
    L.m = o;
    o += align16(sizeof(float) * Ml);
    L.recs = o;
    o += 2 * L.recs_bytes;
    L.alph = o;
    o += 2 * L.alph_bytes;
    L.vbuf = o;
    o += 2 * L.vbuf_bytes;
    L.zbuf = o;
    o += 2 * L.zbuf_bytes;
    L.obuf = o;
    o += 2 * L.obuf_bytes;
    L.ss = o;
    o += align16(sizeof(float) * 2 * C);
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

// Cluster-wide signal: one thread arrives on the same mbarrier of every CTA.
__device__ __forceinline__ void signal_cluster(uint32_t bar, int ncta)
{
    for (int r = 0; r < ncta; ++r) mbar_arrive_cluster(map_to_rank(bar, static_cast<uint32_t>(r)));
}

// CPL consecutive input elements (fp32 or bf16) from shared memory, as fp32.
template <int CPL>
__device__ __forceinline__ void load_row(const unsigned char* base, int elem, int is_bf16, float (&v)[CPL])
{
    if (is_bf16) {
        const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(base) + elem;
#pragma unroll
        for (int c = 0; c < CPL; ++c) v[c] = __bfloat162float(pb[c]);
    } else {
        const float* pf = reinterpret_cast<const float*>(base) + elem;
#pragma unroll
        for (int c = 0; c < CPL; ++c) v[c] = pf[c];
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
    const Layout L = scan_layout((M + ncta - 1) / ncta, C, p.K, dv, ncta, es);
    const uint32_t bars = smem_addr(smem + L.bars);
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + L.holder);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.holder + 4);
    int* offs_s = reinterpret_cast<int*>(smem + L.offs);
    float* m_s = reinterpret_cast<float*>(smem + L.m);
    float* ss_s = reinterpret_cast<float*>(smem + L.ss);

    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kStage + i, 1);
            mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kScan + i, kScanWarps * 32);
            mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kOFree + i, kEpiWarps * 32);
            mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kZ + i, 1);
            mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kPeerO + i, static_cast<uint32_t>(ncta));
            mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kPeerSS + i, static_cast<uint32_t>(ncta));
        }
        mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars) + kFin, static_cast<uint32_t>(ncta));
        fence_mbar_init_cluster();
    }
    if (warp == 0) tmem_alloc(holder, p.tmem_cols);
    // zero both o buffers and the masses / initial state
    {
        float4* ob = reinterpret_cast<float4*>(smem + L.obuf);
        for (size_t i = tid; i < 2 * L.obuf_bytes / 16; i += kThreads) ob[i] = make_float4(0.f, 0.f, 0.f, 0.f);
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
        for (int s = warp; s < Ml; s += 8) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) r[c] = (p.S_in != nullptr && lane < LW) ? p.S_in[row + lane * CPL + c] : 0.0f;
            tmem_st<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
        }
        tmem_wait_st();
        for (int c = 0; c < nch; ++c) {
            const int bf = c & 1;
            wait_bounded<false>(bar(kStage + bf), (c >> 1) & 1, p.status, abort_flag);
            if (c >= 2) wait_bounded<false>(bar(kOFree + bf), ((c - 2) >> 1) & 1, p.status, abort_flag);
            const uint2* recs = reinterpret_cast<const uint2*>(smem + L.recs + bf * L.recs_bytes);
            const float* alph = reinterpret_cast<const float*>(smem + L.alph + bf * L.alph_bytes);
            const unsigned char* vb = smem + L.vbuf + bf * L.vbuf_bytes;
            float* ob = reinterpret_cast<float*>(smem + L.obuf + bf * L.obuf_bytes);
            const int* ofs = offs_s + bf * 12;
            const int rbase = ofs[9], abase = ofs[10];
            const int end = ofs[warp + 1] - rbase;
            const int ashift = rbase - abase;
            for (int i = ofs[warp] - rbase; i < end;) {
                // a batch of up to 4 events on distinct slots (columns)
                uint2 r[4];
                r[0] = recs[i];
                int nb = 1;
                if (i + 1 < end) {
                    r[1] = recs[i + 1];
                    const uint32_t c0 = r[0].x & 0x7FFFu, c1 = r[1].x & 0x7FFFu;
                    if (c1 != c0) {
                        nb = 2;
                        if (i + 2 < end) {
                            r[2] = recs[i + 2];
                            const uint32_t c2 = r[2].x & 0x7FFFu;
                            if (c2 != c0 && c2 != c1) {
                                nb = 3;
                                if (i + 3 < end) {
                                    r[3] = recs[i + 3];
                                    const uint32_t c3 = r[3].x & 0x7FFFu;
                                    if (c3 != c0 && c3 != c1 && c3 != c2) nb = 4;
                                }
                            }
                        }
                    }
                }
                float S[4][CPL];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (k < nb) tmem_ld<CPL>(tq + (r[k].x & 0x7FFFu), S[k]);
                // masses and rates of the batch's writes while the loads are in flight
                float lam[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    lam[k] = 0.0f;
                    if (k < nb && (r[k].x & 0x8000u)) {
                        const int s = 4 * static_cast<int>((r[k].x & 0x7FFFu) / CPL) + q;
                        const float w = __uint_as_float(r[k].y);
                        const float mn = alph[i + k + ashift] * m_s[s] + w;
                        lam[k] = w * __frcp_rn(mn + p.eps_gsu);
                        __syncwarp();
                        if (lane == 0) m_s[s] = mn;
                    }
                }
                __syncwarp();
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (k < nb) {
                        const int t = static_cast<int>(r[k].x >> 16);
                        if (r[k].x & 0x8000u) {
                            float vv[CPL];
                            load_row<CPL>(vb, t * dv + (lane < LW ? lane : 0) * CPL, p.in_bf16, vv);
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) S[k][cc] = fmaf(lam[k], vv[cc] - S[k][cc], S[k][cc]);
                            tmem_st<CPL>(tq + (r[k].x & 0x7FFFu), S[k]);
                        } else if (lane < LW) {
                            const float rw = __uint_as_float(r[k].y);
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) atomicAdd(&ob[t * dv + cc * LW + lane], rw * S[k][cc]);
                        }
                    }
                }
                tmem_wait_st();
                i += nb;
            }
            arrive_cta(bar(kScan + bf));
        }
        // final state of the owned slots
        for (int s = warp; s < Ml; s += 8) {
            const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
            float r[CPL];
            tmem_ld<CPL>(tq + static_cast<uint32_t>((s >> 2) * CPL), r);
            tmem_wait_ld();
            if (lane < LW) {
#pragma unroll
                for (int c = 0; c < CPL; ++c) p.S_out[row + lane * CPL + c] = r[c];
            }
            if (lane == 0) p.m_out[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] = m_s[s];
        }
    } else if (warp == kLoadWarp) {
        // ============================================================ loader warp
        for (int c = 0; c < nch; ++c) {
            const int bf = c & 1;
            const int n = min(C, p.T - c * C);
            if (c >= 2) {
                wait_bounded<false>(bar(kScan + bf), ((c - 2) >> 1) & 1, p.status, abort_flag);
                fence_proxy_async();
            }
            const long long chunk = static_cast<long long>(bh) * nch + c;
            const int* og = p.offs + chunk * p.offs_stride + 8 * rank;
            const int o = lane < 9 ? og[lane] : 0;
            const int lo = __shfl_sync(0xffffffffu, o, 0), hi = __shfl_sync(0xffffffffu, o, 8);
            const int lo_r = lo & ~1, lo_a = lo & ~3;
            const uint32_t rb = hi > lo ? static_cast<uint32_t>(align16(static_cast<size_t>(hi - lo_r) * 8)) : 0u;
            const uint32_t ab = hi > lo ? static_cast<uint32_t>(align16(static_cast<size_t>(hi - lo_a) * 4)) : 0u;
            const uint32_t vrow = static_cast<uint32_t>(dv * es);
            int* ofs = offs_s + bf * 12;
            if (lane < 9) ofs[lane] = o;
            if (lane == 9) ofs[9] = lo_r;
            if (lane == 10) ofs[10] = lo_a;
            __syncwarp();
            if (lane == 0) arrive_expect_tx(bar(kStage + bf), rb + ab + static_cast<uint32_t>(n) * vrow);
            __syncwarp();
            if (lane == 0 && rb) bulk_g2s(smem_addr(smem + L.recs + bf * L.recs_bytes), p.recs + chunk * p.recs_stride + lo_r, rb, bar(kStage + bf));
            if (lane == 1 && ab) bulk_g2s(smem_addr(smem + L.alph + bf * L.alph_bytes), p.alphas + chunk * p.recs_stride + lo_a, ab, bar(kStage + bf));
            for (int t = lane; t < n; t += 32) {
                const size_t th = (static_cast<size_t>(b) * p.T + c * C + t) * p.H + h;
                bulk_g2s(smem_addr(smem + L.vbuf + bf * L.vbuf_bytes + static_cast<size_t>(t) * vrow),
                         static_cast<const unsigned char*>(p.v) + th * vrow, vrow, bar(kStage + bf));
            }
        }
    } else {
        // ============================================================ epilogue warps
        const int e = warp - kEpiWarp0;
        const int etid = tid - kEpiWarp0 * 32;
        const int cpl_lane = Dr >= 32 ? Dr / 32 : 1;  // output channels per lane
        const bool lane_on = lane * cpl_lane < Dr;
        const int ch0 = static_cast<int>(rank) * Dr + lane * cpl_lane;
        const uint32_t zrow = static_cast<uint32_t>(Dr * es);
        for (int c = 0; c < nch; ++c) {
            const int bf = c & 1;
            const int n = min(C, p.T - c * C);
            const int t0 = c * C;
            // stage z (this CTA's channels) for the chunk
            if (e == 0) {
                fence_proxy_async();
                if (lane == 0) arrive_expect_tx(bar(kZ + bf), static_cast<uint32_t>(n) * zrow);
                __syncwarp();
                for (int t = lane; t < n; t += 32) {
                    const size_t th = (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h;
                    bulk_g2s(smem_addr(smem + L.zbuf + bf * L.zbuf_bytes + static_cast<size_t>(t) * zrow),
                             static_cast<const unsigned char*>(p.z) + (th * dv + static_cast<size_t>(rank) * Dr) * es,
                             zrow, bar(kZ + bf));
                }
            }
            wait_bounded<false>(bar(kScan + bf), (c >> 1) & 1, p.status, abort_flag);
            float* ob = reinterpret_cast<float*>(smem + L.obuf + bf * L.obuf_bytes);
            float* ss = ss_s + bf * C;
            // all CTAs' partial sums of this chunk are complete
            if (etid == 0) {
                if (ncta == 1) arrive_cta(bar(kPeerO + bf));
                else signal_cluster(bar(kPeerO + bf), ncta);
            }
            wait_bounded<true>(bar(kPeerO + bf), (c >> 1) & 1, p.status, abort_flag);
            for (int t = e; t < n; t += kEpiWarps) {
                float sq = 0.0f;
                if (lane_on) {
                    for (int k = 0; k < cpl_lane; ++k) {
                        const int ch = ch0 + k;
                        const int pos = t * dv + (ch % CPL) * LW + ch / CPL;
                        float o = 0.0f;
                        if (ncta == 1) {
                            o = ob[pos];
                        } else {
                            const uint32_t a = smem_addr(&ob[pos]);
                            for (int r = 0; r < ncta; ++r) o += ld_cluster_f32(map_to_rank(a, static_cast<uint32_t>(r)));
                            ob[pos] = o;
                        }
                        sq += o * o;
                    }
                }
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, d);
                if (lane == 0) ss[t] = sq;
            }
            epi_barrier();
            if (etid == 0) {
                if (ncta == 1) arrive_cta(bar(kPeerSS + bf));
                else signal_cluster(bar(kPeerSS + bf), ncta);
            }
            wait_bounded<true>(bar(kPeerSS + bf), (c >> 1) & 1, p.status, abort_flag);
            wait_bounded<false>(bar(kZ + bf), (c >> 1) & 1, p.status, abort_flag);
            const unsigned char* zb = smem + L.zbuf + bf * L.zbuf_bytes;
            for (int t = e; t < n; t += kEpiWarps) {
                float tot = 0.0f;
                if (ncta == 1) {
                    tot = ss[t];
                } else {
                    const uint32_t a = smem_addr(&ss[t]);
                    for (int r = 0; r < ncta; ++r) tot += ld_cluster_f32(map_to_rank(a, static_cast<uint32_t>(r)));
                }
                const float inv = 1.0f / sqrtf(tot / dv + p.eps_norm);
                if (lane_on) {
                    const size_t th = (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h;
                    for (int k = 0; k < cpl_lane; ++k) {
                        const int ch = ch0 + k;
                        const int pos = t * dv + (ch % CPL) * LW + ch / CPL;
                        const float zz = p.in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(zb)[t * Dr + ch - static_cast<int>(rank) * Dr])
                                                   : reinterpret_cast<const float*>(zb)[t * Dr + ch - static_cast<int>(rank) * Dr];
                        const float nw = p.norm_w != nullptr ? p.norm_w[ch] : 1.0f;
                        store_out(p.y, th * dv + ch, ob[pos] * inv * nw * zz, p.out_bf16);
                    }
                }
            }
            // every CTA has read this chunk's partial sums and every epilogue warp has
            // written its y: clear them for chunk c + 2
            epi_barrier();
            float4* ob4 = reinterpret_cast<float4*>(ob);
            for (size_t i = etid; i < L.obuf_bytes / 16; i += kEpiWarps * 32) ob4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            arrive_cta(bar(kOFree + bf));
        }
    }

    // copies still in flight after an abort must land before the CTA exits
    if (warp == kLoadWarp || warp == kEpiWarp0) {
        const int base = warp == kLoadWarp ? kStage : kZ;
        for (int c = max(0, nch - 2); c < nch; ++c) drain_copies(bar(base + (c & 1)), (c >> 1) & 1);
    }
    // no CTA leaves while a peer may still read its shared memory
    __syncthreads();
    if (ncta > 1 && tid == 0) {
        signal_cluster(bar(kFin), ncta);
        wait_bounded<true>(bar(kFin), 0, p.status, abort_flag);
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, p.tmem_cols);
}

}  // namespace

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
    int C = 64;
    while (C > 8 && (2 * C * K > 2048 || scan_layout(Ml, C, K, d_v, n, in_bytes).total > 200 * 1024)) C >>= 1;
    const size_t total = scan_layout(Ml, C, K, d_v, n, in_bytes).total;
    if (total > 200 * 1024) return false;
    out->ncta = n;
    out->chunk = C;
    out->cpl = cpl;
    out->tmem_cols = alloc;
    // more than half of the SM's shared memory: exactly one CTA (and one TMEM owner) per SM
    out->smem_bytes = total < 116 * 1024 ? 116 * 1024 : total;
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
