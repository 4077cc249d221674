// route.cu -- first launch of the prefill scan: the Address Decoder and CAPE for every token
// of every head, written as read and write events grouped by the scan warp that owns their
// slot.
//
// RAM-Net project page, GPU-execution paragraph: Top-K addresses for all tokens are
// computed in parallel first, and the read and write events are then grouped by slot so
// that each slot's events can be walked in causal order and slots without events cost
// nothing.  Here the grouping unit is the owner of a slot (one scan warp of one CTA of the
// head's cluster, see kernels.h), and within one owner the events stay in (token, stream)
// order, which is each slot's causal order: a token's writes before its reads.
//
// One CTA of 128 threads covers 64 tokens of one head: thread i < 64 decodes token i's key
// (its K events are writes; it also computes the retention alpha of GSU step 1), thread
// 64 + i its query (reads), so no warp runs both paths.  The events of each chunk are then
// placed by a stable counting sort on the owner, rows ordered by (token, stream): per
// (row, owner) counts in shared memory, an exclusive prefix over the chunk's rows per owner,
// and an exclusive prefix over owners per chunk.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

constexpr int kRouteThreads = 128;
constexpr int kRouteTokens = kRouteThreads / 2;

// Byte offset of the shared-memory kept lists (K > 32) after the count tables.
__host__ __device__ inline size_t route_kept_offset(int O, int nchb)
{
    return (sizeof(uint32_t) * (static_cast<size_t>(kRouteThreads) * O + static_cast<size_t>(nchb) * (O + 1)) + 15) &
           ~static_cast<size_t>(15);
}

// At K = 32 the search's kept list and merge buffers want ~200 registers; capping them for 3
// CTAs per SM (a little spilling) is faster than 2 CTAs per SM.  At K = 16 the cap keeps 4
// CTAs per SM (128 registers).
template <int KMAX, int DPMAX>
__global__ void __launch_bounds__(kRouteThreads, KMAX == 32 ? 3 : (KMAX == 16 ? 4 : 1)) k_route(RouteParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int O = p.ncta * p.nw;
    const int C = p.chunk, nchb = kRouteTokens / C;
    uint32_t* tc = reinterpret_cast<uint32_t*>(smem);  // [128][O] per-thread owner counts, then prefixes
    uint32_t* coff = tc + kRouteThreads * O;            // [nchb][O + 1] per-chunk owner offsets
    uint64_t* kept_s = reinterpret_cast<uint64_t*>(smem + route_kept_offset(O, nchb));  // K > 32 only
    const int lg_ncta = __ffs(p.ncta) - 1, lg_nw = __ffs(p.nw) - 1;

    const int tid = threadIdx.x;
    const int nblk_t = (p.T + kRouteTokens - 1) / kRouteTokens;
    const int bh = blockIdx.x / nblk_t, tb = blockIdx.x - (blockIdx.x / nblk_t) * nblk_t;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int tl_blk = tid & (kRouteTokens - 1), stream = tid / kRouteTokens;
    const int row_id = tl_blk * 2 + stream;  // (token, stream) order of the counting sort
    const int t = tb * kRouteTokens + tl_blk;
    const bool valid = t < p.T;
    const int ch = tl_blk / C, tl = tl_blk & (C - 1);
    const int c = tb * nchb + ch;
    const int K = p.K;

    for (int i = tid; i < kRouteThreads * O; i += kRouteThreads) tc[i] = 0u;
    __syncthreads();

    // ---- decode: Top-K, weights, CAPE, retention
    uint64_t out[KMAX];
    float w[KMAX];
    int32_t slot[KMAX];
    float al[KMAX];
    if (valid) {
        const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;  // [B,T,H] index
        const int L = p.U * p.d_p;
        const void* lg = stream == 0 ? p.k_logits : p.q_logits;
        if constexpr (KMAX <= 32)
            topk_search_net<KMAX, DPMAX>(lg, th * L, p.in_bf16, p.d_p, p.U, K, out);  // kept list in registers
        else
            topk_search<KMAX, DPMAX>(lg, th * L, p.in_bf16, p.d_p, p.U, K, kept_s + tid, kRouteThreads, out);
        topk_weights<KMAX>(out, K, p.renorm, lg, th * L, p.in_bf16, p.d_p, p.U, w);
        const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
        int32_t pm = 0;
        if (cape) {
            const int64_t pos = static_cast<int64_t>(p.pos0 != nullptr ? p.pos0[b] : 0) + p.t_offset + t;
            int64_t r = pos % p.M;
            pm = static_cast<int32_t>(r < 0 ? r + p.M : r);
        }
        const float gg = stream == 0 ? load_in(p.g, th, p.in_bf16) : 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            int32_t s = packed_index(out[j], p.M) + pm;
            slot[j] = s >= p.M ? s - p.M : s;
            al[j] = (stream == 0 && j < K) ? gsu_alpha(w[j], gg) : 0.0f;
        }
    }

    // ---- owners, rank within (thread, owner), and each read's rank among the token's reads
    //      held by the same CTA
    uint32_t meta[KMAX];  // owner | rank << 16
    uint32_t qv[KMAX];
    if (valid) {
        uint64_t cnt = 0;  // 8-bit read counters per CTA rank (ncta <= 8, K <= 64)
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < K && dcheck(slot[j] >= 0 && slot[j] < p.M, p.status)) {
                const int rk = slot[j] & (p.ncta - 1);
                const int o = (rk << lg_nw) + ((slot[j] >> lg_ncta) & (p.nw - 1));
                const uint32_t r = atomicAdd(&tc[row_id * O + o], 1u);
                meta[j] = static_cast<uint32_t>(o) | (r << 16);
                qv[j] = static_cast<uint32_t>((cnt >> (8 * rk)) & 0xFFull);
                cnt += 1ull << (8 * rk);
            }
        }
        if (stream == 1) {
            unsigned char* nb = reinterpret_cast<unsigned char*>(p.hdr);
            for (int rk = 0; rk < p.ncta; ++rk) {
                const size_t hw = ((static_cast<size_t>(bh) * p.nch + c) * p.ncta + rk) * p.hdr_words;
                nb[(hw + 4 + p.nw + 1) * 4 + tl] = static_cast<unsigned char>((cnt >> (8 * rk)) & 0xFFull);
            }
        }
    }
    __syncthreads();

    // ---- per chunk and owner: exclusive prefix of the counts over the chunk's threads
    if (tid < O) {
        for (int cc = 0; cc < nchb; ++cc) {
            uint32_t run = 0;
            for (int i = cc * 2 * C; i < (cc + 1) * 2 * C; ++i) {
                const uint32_t v = tc[i * O + tid];
                tc[i * O + tid] = run;
                run += v;
            }
            coff[cc * (O + 1) + tid] = run;
        }
    }
    __syncthreads();

    // ---- per chunk: exclusive prefix over owners (owner order = rank, then scan warp)
    {
        const int warp = tid >> 5, lane = tid & 31;
        const int opl = (O + 31) / 32;
        for (int cc = warp; cc < nchb; cc += kRouteThreads / 32) {
            uint32_t* row = coff + cc * (O + 1);
            uint32_t loc[4];
            uint32_t sum = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int o = lane * opl + i;
                loc[i] = (i < opl && o < O) ? row[o] : 0u;
                sum += loc[i];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t n = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += n;
            }
            uint32_t run = incl - sum;
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int o = lane * opl + i;
                if (i < opl && o < O) row[o] = run;
                run += loc[i];
            }
            if (lane == 31) row[O] = incl;
        }
    }
    __syncthreads();

    // ---- headers of this CTA's chunks: per rank the event range and the scan warps' ranges
    {
        const int hw_used = 5 + p.nw;
        for (int i = tid; i < nchb * p.ncta * hw_used; i += kRouteThreads) {
            const int cc = i / (p.ncta * hw_used);
            const int rem = i - cc * p.ncta * hw_used;
            const int rk = rem / hw_used, wd = rem - rk * hw_used;
            const int cg = tb * nchb + cc;
            if (cg * C >= p.T) continue;
            const uint32_t* row = coff + cc * (O + 1);
            const uint32_t start = row[rk * p.nw];
            uint32_t val;
            if (wd == 0) val = start;
            else if (wd == 1) val = row[(rk + 1) * p.nw] - start;
            else if (wd == 2) val = static_cast<uint32_t>(min(C, p.T - cg * C));
            else if (wd == 3) val = 0u;
            else val = row[rk * p.nw + (wd - 4)] - start;
            p.hdr[((static_cast<size_t>(bh) * p.nch + cg) * p.ncta + rk) * p.hdr_words + wd] = val;
        }
    }

    // ---- events at their sorted positions
    if (valid) {
        const uint32_t* row = coff + ch * (O + 1);
        uint4* ev = p.events + (static_cast<size_t>(bh) * p.nch + c) * (2 * static_cast<size_t>(C) * K);
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < K && dcheck(slot[j] >= 0 && slot[j] < p.M && static_cast<int>(meta[j] & 0xFFFFu) < O, p.status)) {
                const uint32_t o = meta[j] & 0xFFFFu;
                const uint32_t pos = row[o] + tc[row_id * O + o] + (meta[j] >> 16);
                if (!dcheck(pos < static_cast<uint32_t>(2 * C * K), p.status)) continue;
                const uint32_t s = static_cast<uint32_t>(slot[j]) >> lg_ncta;
                const uint32_t x = s | (static_cast<uint32_t>(tl) << 16) | ((stream ? qv[j] : 0u) << 24) |
                                   (static_cast<uint32_t>(stream) << 31);
                ev[pos] = make_uint4(x, __float_as_uint(w[j]), __float_as_uint(al[j]), static_cast<uint32_t>(slot[j]));
            }
        }
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_route_k(const RouteParams& p, cudaStream_t s)
{
    const int O = p.ncta * p.nw;
    const int nchb = kRouteTokens / p.chunk;
    const int nblk_t = (p.T + kRouteTokens - 1) / kRouteTokens;
    size_t smem = route_kept_offset(O, nchb);
    if (KMAX > 32) smem += sizeof(uint64_t) * KMAX * kRouteThreads;
    auto kern = k_route<KMAX, DPMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(p.B * p.H * nblk_t), kRouteThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int DPMAX>
cudaError_t route_k(const RouteParams& p, cudaStream_t s)
{
    if (p.K <= 8) return launch_route_k<8, DPMAX>(p, s);
    if (p.K <= 16) return launch_route_k<16, DPMAX>(p, s);
    if (p.K <= 32) return launch_route_k<32, DPMAX>(p, s);
    return launch_route_k<64, DPMAX>(p, s);
}

}  // namespace

cudaError_t launch_route(const RouteParams& p, cudaStream_t stream)
{
    const bool pow2 = (p.ncta & (p.ncta - 1)) == 0 && (p.nw & (p.nw - 1)) == 0 && (p.chunk & (p.chunk - 1)) == 0;
    if (p.T >= (1 << 30) || !pow2 || p.ncta * p.nw > kRouteThreads || kRouteTokens % p.chunk != 0 || p.K > 64)
        return cudaErrorInvalidValue;
    if (p.d_p <= 4) return route_k<4>(p, stream);
    if (p.d_p <= 8) return route_k<8>(p, stream);
    return route_k<16>(p, stream);
}

}  // namespace ramnet
