// scan_forward.cu -- K2: the prefill recurrence of the RAM-Net layer core.
//
// RAM-Net project page: the three-stage paragraph (decode, CAPE, GSU, then read,
// normalise, gate), the Gated Sparse Update paragraphs (four steps; unselected slots
// unchanged) and the GPU-execution paragraph (addresses for all tokens first, then the
// recurrence over slots whose channels run in parallel).
//
// Layout.  One head's slot array S [M, d_v] fp32 lives in tensor memory (TMEM) for the
// whole sequence, spread over a cluster of `ncta` CTAs, one per SM.  Slot i belongs to
// CTA (i mod ncta) as local slot s = i / ncta; local slot s sits in TMEM lane quadrant
// (s mod 4), columns [(s/4)*CPL, (s/4)*CPL + CPL), lane l of the quadrant holding
// channels c*32 + l (c < CPL).  A row access is then one tcgen05.ld/st of CPL columns by
// the quadrant's warp.  The write mass m of local slots is in shared memory.
// Warp w serves quadrant w%4 and local slots with ((s/4) mod 2) == w/4, so every slot has
// exactly one owner warp and the owner applies all events of its slots in token order.
//
// Per chunk of C tokens: stage addresses, gates and values in shared memory; every warp
// walks the chunk's events in order and applies those it owns (writes: mass, rate,
// content; reads: weighted row added into the chunk's o buffer); then the CTAs of the
// cluster exchange partial read sums and squared norms through distributed shared
// memory and write y for their share of the channels.
#include "common.cuh"
#include "kernels.h"

namespace ramnet {

namespace {

constexpr int kScanThreads = 256;

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct ScanLayout {
    size_t bar, holder, ok, m, widx, wwt, ridx, rwt, g, ss, vbuf, obuf, total;
};

__host__ __device__ inline ScanLayout scan_layout(int Ml, int C, int K, int dv)
{
    ScanLayout L;
    size_t o = 0;
    L.bar = o;
    o += 8;
    L.holder = o;
    o += 4;
    L.ok = o;
    o += 4;
    L.m = o;
    o += align16(sizeof(float) * Ml);
    L.widx = o;
    o += align16(sizeof(int32_t) * C * K);
    L.wwt = o;
    o += align16(sizeof(float) * C * K);
    L.ridx = o;
    o += align16(sizeof(int32_t) * C * K);
    L.rwt = o;
    o += align16(sizeof(float) * C * K);
    L.g = o;
    o += align16(sizeof(float) * C);
    L.ss = o;
    o += align16(sizeof(float) * 2 * C);
    L.vbuf = o;
    o += align16(sizeof(float) * C * dv);
    L.obuf = o;
    o += align16(sizeof(float) * C * dv);
    L.total = o;
    return L;
}

// Gated Sparse Update, step 1 (retention): (1 - w)^(g/(1-g)), g clamped to [0,1].
__device__ __forceinline__ float gsu_alpha(float w, float g)
{
    g = fminf(fmaxf(g, 0.0f), 1.0f);
    const float c = g / (1.0f - g);
    if (w <= 0.0f || c <= 0.0f) return 1.0f;
    if (w >= 1.0f) return 0.0f;
    return expf(c * log1pf(-w));
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Cluster-wide rendezvous on this CTA's mbarrier with a bounded wait (about 2 s).
// Thread 0 arrives on every CTA's barrier and waits; the verdict is broadcast to the CTA.
__device__ bool cluster_point(uint64_t* bar, uint32_t& phase, int ncta, int* ok_s, uint32_t* status)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = *ok_s;
        if (ok) {
            const uint32_t a = smem_addr(bar);
            for (int r = 0; r < ncta; ++r) mbar_arrive_cluster(map_to_rank(a, static_cast<uint32_t>(r)));
            ok = 0;
            const uint64_t t_end = global_ns() + 2000000000ull;
            for (uint32_t it = 0; it < kSpinLimit; ++it) {
                if (mbar_try_wait_cluster(bar, phase & 1u)) {
                    ok = 1;
                    break;
                }
                if ((it & 255u) == 255u && global_ns() > t_end) break;
            }
            if (!ok) set_status(status, kDevTimeout);
        }
        *ok_s = ok;
    }
    ++phase;
    __syncthreads();
    return *ok_s != 0;
}

template <int CPL>
__global__ void __launch_bounds__(kScanThreads, 1) k_scan_tmem(ScanParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = p.chunk, K = p.K, dv = p.d_v, ncta = p.ncta, M = p.M;
    const int LW = dv < 32 ? dv : 32;  // active lanes per row
    const uint32_t rank = ncta > 1 ? cluster_ctarank() : 0u;
    const int bh = blockIdx.x / ncta;
    const int b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int q = warp & 3, sub = warp >> 2;
    const int Ml = (M - static_cast<int>(rank) + ncta - 1) / ncta;
    const ScanLayout L = scan_layout((M + ncta - 1) / ncta, C, K, dv);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + L.holder);
    int* ok_s = reinterpret_cast<int*>(smem + L.ok);
    float* m_s = reinterpret_cast<float*>(smem + L.m);
    int32_t* widx_s = reinterpret_cast<int32_t*>(smem + L.widx);
    float* wwt_s = reinterpret_cast<float*>(smem + L.wwt);
    int32_t* ridx_s = reinterpret_cast<int32_t*>(smem + L.ridx);
    float* rwt_s = reinterpret_cast<float*>(smem + L.rwt);
    float* g_s = reinterpret_cast<float*>(smem + L.g);
    float* ss_s = reinterpret_cast<float*>(smem + L.ss);
    float* vbuf = reinterpret_cast<float*>(smem + L.vbuf);
    float* obuf = reinterpret_cast<float*>(smem + L.obuf);

    if (tid == 0) {
        *ok_s = 1;
        if (ncta > 1) {
            mbar_init(bar, static_cast<uint32_t>(ncta));
            fence_mbar_init_cluster();
        }
    }
    if (warp == 0) tmem_alloc(holder, p.tmem_cols);
    tmem_fence_before_sync();
    __syncthreads();
    if (ncta > 1) cluster_sync_all();
    tmem_fence_after_sync();
    const uint32_t tbase = *holder;
    const uint32_t tq = static_cast<uint32_t>(32 * q) << 16;

    // ---- initial state: owned rows into TMEM, masses into shared memory
    for (int s = 4 * sub + q; s < Ml; s += 8) {
        const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
        float r[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) r[c] = (p.S_in != nullptr && lane < LW) ? p.S_in[row + c * LW + lane] : 0.0f;
        tmem_st<CPL>(tbase + tq + static_cast<uint32_t>((s >> 2) * CPL), r);
    }
    tmem_wait_st();
    for (int s = tid; s < Ml; s += kScanThreads)
        m_s[s] = p.m_in != nullptr ? p.m_in[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] : 0.0f;
    __syncthreads();

    uint32_t phase = 0;
    bool ok = true;
    for (int t0 = 0; t0 < p.T && ok; t0 += C) {
        const int n = min(C, p.T - t0);
        float* ss = ss_s + ((t0 / C) & 1) * C;
        // ---- stage the chunk
        for (int e = tid; e < n * K; e += kScanThreads) {
            const int t = e / K, j = e - (e / K) * K;
            const size_t th = (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h;
            widx_s[e] = p.widx[th * K + j];
            wwt_s[e] = p.wwt[th * K + j];
            ridx_s[e] = p.ridx[th * K + j];
            rwt_s[e] = p.rwt[th * K + j];
        }
        for (int t = tid; t < n; t += kScanThreads) {
            const size_t th = (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h;
            g_s[t] = load_in(p.g, th, p.in_bf16);
            ss[t] = 0.0f;
        }
        for (int e = tid; e < n * dv; e += kScanThreads) {
            const int t = e / dv, ch = e - (e / dv) * dv;
            const size_t th = (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h;
            vbuf[t * dv + (ch % LW) * CPL + ch / LW] = load_in(p.v, th * dv + ch, p.in_bf16);
            obuf[e] = 0.0f;
        }
        __syncthreads();

        // ---- events of the chunk, in token order; writes of a token before its reads
        for (int t = 0; t < n; ++t) {
            const float g = g_s[t];
            for (int grp = 0; grp < 2 * K; grp += 32) {
                const int e = grp + lane;
                const bool valid = e < 2 * K;
                const bool is_w = e < K;
                const int j = is_w ? e : e - K;
                int slot = 0;
                float coef = 0.0f;
                if (valid) {
                    slot = is_w ? widx_s[t * K + j] : ridx_s[t * K + j];
                    coef = is_w ? wwt_s[t * K + j] : rwt_s[t * K + j];
                }
                const int s_loc = slot / ncta;
                const bool own = valid && (slot - s_loc * ncta) == static_cast<int>(rank) && (s_loc & 3) == q &&
                                 ((s_loc >> 2) & 1) == sub;
                uint32_t mask = __ballot_sync(0xffffffffu, own);
                while (mask) {
                    const int src = __ffs(mask) - 1;
                    mask &= mask - 1;
                    const int sl = __shfl_sync(0xffffffffu, s_loc, src);
                    const float cf = __shfl_sync(0xffffffffu, coef, src);
                    const uint32_t taddr = tbase + tq + static_cast<uint32_t>((sl >> 2) * CPL);
                    float S[CPL];
                    tmem_ld<CPL>(taddr, S);
                    tmem_wait_ld();
                    if (grp + src < K) {
                        // Gated Sparse Update steps 1-4 for this slot
                        const float mo = m_s[sl];
                        const float a = gsu_alpha(cf, g);
                        const float mn = a * mo + cf;
                        const float lam = cf / (mn + p.eps_gsu);
                        __syncwarp();
                        if (lane == 0) m_s[sl] = mn;
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < CPL; ++c) {
                            const float vv = lane < LW ? vbuf[t * dv + lane * CPL + c] : 0.0f;
                            S[c] = fmaf(lam, vv - S[c], S[c]);
                        }
                        tmem_st<CPL>(taddr, S);
                        tmem_wait_st();
                    } else if (lane < LW) {
#pragma unroll
                        for (int c = 0; c < CPL; ++c) atomicAdd(&obuf[t * dv + lane * CPL + c], cf * S[c]);
                    }
                }
            }
        }
        __syncthreads();

        // ---- read sums across the cluster, RMSNorm, gate, y
        if (ncta == 1) {
            for (int e = tid; e < n * dv; e += kScanThreads) {
                const int t = e / dv, ch = e - (e / dv) * dv;
                const float o = obuf[t * dv + (ch % LW) * CPL + ch / LW];
                atomicAdd(&ss[t], o * o);
            }
            __syncthreads();
        } else {
            ok = cluster_point(bar, phase, ncta, ok_s, p.status);
            if (!ok) break;
            const int Dr = dv / ncta;
            for (int e = tid; e < n * Dr; e += kScanThreads) {
                const int t = e / Dr, ch = static_cast<int>(rank) * Dr + (e - (e / Dr) * Dr);
                const int pos = t * dv + (ch % LW) * CPL + ch / LW;
                const uint32_t a = smem_addr(&obuf[pos]);
                float o = 0.0f;
                for (int r = 0; r < ncta; ++r) o += ld_cluster_f32(map_to_rank(a, static_cast<uint32_t>(r)));
                obuf[pos] = o;
                atomicAdd(&ss[t], o * o);
            }
            ok = cluster_point(bar, phase, ncta, ok_s, p.status);
            if (!ok) break;
        }
        {
            const int Dr = dv / ncta;
            for (int e = tid; e < n * Dr; e += kScanThreads) {
                const int t = e / Dr, ch = static_cast<int>(rank) * Dr + (e - (e / Dr) * Dr);
                const int pos = t * dv + (ch % LW) * CPL + ch / LW;
                float tot;
                if (ncta == 1) {
                    tot = ss[t];
                } else {
                    tot = 0.0f;
                    const uint32_t a = smem_addr(&ss[t]);
                    for (int r = 0; r < ncta; ++r) tot += ld_cluster_f32(map_to_rank(a, static_cast<uint32_t>(r)));
                }
                const float inv = 1.0f / sqrtf(tot / dv + p.eps_norm);
                const size_t th = (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h;
                const float nw = p.norm_w != nullptr ? p.norm_w[ch] : 1.0f;
                const float y = obuf[pos] * inv * nw * load_in(p.z, th * dv + ch, p.in_bf16);
                store_out(p.y, th * dv + ch, y, p.out_bf16);
            }
        }
        __syncthreads();
    }

    // ---- final state out
    for (int s = 4 * sub + q; s < Ml; s += 8) {
        const size_t row = (static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank) * dv;
        float r[CPL];
        tmem_ld<CPL>(tbase + tq + static_cast<uint32_t>((s >> 2) * CPL), r);
        tmem_wait_ld();
        if (lane < LW) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) p.S_out[row + c * LW + lane] = r[c];
        }
    }
    for (int s = tid; s < Ml; s += kScanThreads)
        p.m_out[static_cast<size_t>(bh) * M + static_cast<size_t>(s) * ncta + rank] = m_s[s];

    // no CTA leaves while a peer may still read its shared memory
    if (ncta > 1 && ok) cluster_point(bar, phase, ncta, ok_s, p.status);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, p.tmem_cols);
}

}  // namespace

bool scan_plan(int M, int d_v, int K, int* ncta, int* chunk, uint32_t* tmem_cols, size_t* smem_bytes)
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
    while (C > 8 && scan_layout(Ml, C, K, d_v).total > 200 * 1024) C >>= 1;
    const size_t total = scan_layout(Ml, C, K, d_v).total;
    if (total > 200 * 1024) return false;
    *ncta = n;
    *chunk = C;
    *tmem_cols = alloc;
    // more than half of the SM's shared memory: exactly one CTA (and one TMEM owner) per SM
    *smem_bytes = total < 116 * 1024 ? 116 * 1024 : total;
    return true;
}

cudaError_t launch_scan(const ScanParams& p, size_t smem_bytes, cudaStream_t stream)
{
    void (*kern)(ScanParams) = nullptr;
    switch (p.d_v < 32 ? 1 : p.d_v / 32) {
        case 1: kern = k_scan_tmem<1>; break;
        case 2: kern = k_scan_tmem<2>; break;
        case 4: kern = k_scan_tmem<4>; break;
        case 8: kern = k_scan_tmem<8>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.B * p.H * p.ncta));
    cfg.blockDim = dim3(kScanThreads);
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
