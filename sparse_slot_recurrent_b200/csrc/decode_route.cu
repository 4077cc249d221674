// decode_route.cu -- K1 of the prefill scan: Address Decoder + CAPE for one chunk of one
// head, then the chunk's write and read events sorted into per-owner event lists.
//
// RAM-Net project page, GPU-execution paragraph: Top-K addresses for all tokens are
// computed in parallel first, and the read/write events are grouped by slot so that
// each slot sees its own causal sequence.  Here the grouping is by owner warp of the
// scan kernel (a fixed set of slots per warp), keeping token order within each list:
//   owner o = (slot mod ncta) * 8 + ((slot / ncta) mod 8)
// and, within one token, the K writes come before the K reads (the read sees the
// token's own write).  Owners of one scan CTA are contiguous (o / 8 = CTA rank).
//
// Block = (b, h, chunk of C tokens); thread = (token, stream).  Each thread decodes one
// address (stream 0: key -> writes, stream 1: query -> reads), then a stable counting
// sort by owner places its K events: the owner-major table of per-thread counts is
// exclusive-scanned once, which yields every event's position.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int total = 0;
    for (int w = 0; w < nw; ++w) total += warp_tot[w];
    __syncthreads();
    warp_tot[nw] = total;  // grand total (read after the caller's next barrier)
    return base + x - v;
}

template <int KMAX, int DPMAX>
__global__ void __launch_bounds__(128) k_decode_route(RouteParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = p.chunk, nt = 2 * C;  // threads: stream-major (tid < C: key stream)
    const int NO = 8 * p.ncta;
    uint64_t* kept = reinterpret_cast<uint64_t*>(smem);                    // [KMAX][nt]
    int* table = reinterpret_cast<int*>(smem + sizeof(uint64_t) * KMAX * nt);  // [NO][nt] counts -> positions
    int* warp_tot = table + NO * nt;                                       // [nt/32 + 1]

    const int bh = blockIdx.x / p.nchunks, c = blockIdx.x - bh * p.nchunks;
    const int b = bh / p.H, h = bh - b * p.H;
    const int tid = threadIdx.x;
    const int stream = tid >= C ? 1 : 0, tl = tid - stream * C;
    const int t0 = c * C, n = min(C, p.T - t0);
    const bool valid = tl < n;
    const int so = 2 * tl + stream;  // position of this thread's events in token order
    const int L = p.U * p.d_p;

    int owner[KMAX];
    uint32_t meta[KMAX];
    float coef[KMAX], alpha[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) owner[j] = -1;
    if (valid) {
        const int t = t0 + tl;
        const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;
        const void* lg = stream == 0 ? p.k_logits : p.q_logits;
        uint64_t out[KMAX];
        topk_search<KMAX, DPMAX>(lg, th * L, p.in_bf16, p.d_p, p.U, p.K, kept + tid, nt, out);
        float w[KMAX];
        topk_weights<KMAX>(out, p.K, p.renorm, lg, th * L, p.in_bf16, p.d_p, p.U, w);
        const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
        const int64_t pos = static_cast<int64_t>(p.pos0 != nullptr ? p.pos0[b] : 0) + t;
        const float g = stream == 0 ? load_in(p.g, th, p.in_bf16) : 0.0f;
        const int lg_ncta = __ffs(p.ncta) - 1;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < p.K) {
                int32_t slot = packed_index(out[j], p.M);
                if (cape) slot = cape_shift(slot, pos, p.M);
                const int s = slot >> lg_ncta;
                owner[j] = (slot & (p.ncta - 1)) * 8 + (s & 7);
                meta[j] = (static_cast<uint32_t>(tl) << 16) | (stream == 0 ? 0x8000u : 0u) |
                          static_cast<uint32_t>((s >> 2) * p.cpl);
                coef[j] = w[j];
                alpha[j] = stream == 0 ? gsu_alpha(w[j], g) : 0.0f;
            }
        }
    }

    // per-thread owner counts, owner-major: table[o * nt + so]
    for (int i = tid; i < NO * nt; i += nt) table[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (owner[j] >= 0) table[owner[j] * nt + so] += 1;
    __syncthreads();
    // exclusive scan of the flattened table: thread i owns entries [i*NO, (i+1)*NO)
    {
        int loc[64];
        int sum = 0;
        for (int k = 0; k < NO; ++k) {
            loc[k] = table[tid * NO + k];
            sum += loc[k];
        }
        int run = block_exclusive_scan(sum, warp_tot);
        for (int k = 0; k < NO; ++k) {
            table[tid * NO + k] = run;
            run += loc[k];
        }
    }
    __syncthreads();
    // owner offsets of this chunk: start of each owner's segment, then the total
    const long long chunk = static_cast<long long>(bh) * p.nchunks + c;
    int* offs = p.offs + chunk * p.offs_stride;
    for (int o = tid; o <= NO; o += nt) offs[o] = o < NO ? table[o * nt] : warp_tot[(nt + 31) / 32];
    __syncthreads();
    // scatter: events of one owner keep token order (and writes before reads)
    uint2* recs = p.recs + chunk * p.recs_stride;
    float* alph = p.alphas + chunk * p.recs_stride;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (owner[j] >= 0) {
            const int posn = table[owner[j] * nt + so];
            table[owner[j] * nt + so] = posn + 1;
            recs[posn] = make_uint2(meta[j], __float_as_uint(coef[j]));
            alph[posn] = alpha[j];
        }
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_route(const RouteParams& p, cudaStream_t s)
{
    const int nt = 2 * p.chunk;
    const int NO = 8 * p.ncta;
    const size_t smem = sizeof(uint64_t) * KMAX * nt + sizeof(int) * (NO * nt + nt / 32 + 2);
    auto kern = k_decode_route<KMAX, DPMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(p.B * p.H * p.nchunks), nt, smem, s>>>(p);
    return cudaGetLastError();
}

template <int DPMAX>
cudaError_t route_k(const RouteParams& p, cudaStream_t s)
{
    if (p.K <= 8) return launch_route<8, DPMAX>(p, s);
    if (p.K <= 16) return launch_route<16, DPMAX>(p, s);
    if (p.K <= 32) return launch_route<32, DPMAX>(p, s);
    return launch_route<64, DPMAX>(p, s);
}

}  // namespace

cudaError_t launch_decode_route(const RouteParams& p, cudaStream_t stream)
{
    if (2 * p.chunk > 128 || 8 * p.ncta > 64) return cudaErrorInvalidValue;
    if (p.d_p <= 4) return route_k<4>(p, stream);
    if (p.d_p <= 8) return route_k<8>(p, stream);
    return route_k<16>(p, stream);
}

}  // namespace ramnet
