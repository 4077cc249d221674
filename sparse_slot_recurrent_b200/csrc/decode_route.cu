// decode_route.cu -- K1 of the prefill scan: Address Decoder + CAPE for one chunk of one
// head, then the chunk's write and read events sorted into per-owner event lists.
//
// RAM-Net project page, GPU-execution paragraph: Top-K addresses for all tokens are
// computed in parallel first, and the read/write events are grouped by slot so that
// each slot sees its own causal sequence.  Here the grouping is by owner warp of the
// scan kernel (a fixed set of slots per warp), keeping token order within each list:
//   owner o = (slot mod ncta) * NW + ((slot / ncta) mod NW),  NW = scan warps per CTA
// and, within one token, the K writes come before the K reads (the read sees the
// token's own write).  Owners of one scan CTA are contiguous (o / NW = CTA rank).
//
// Output per (b, h, chunk), one contiguous block of `chunk_bytes` (chunk_block_bytes()):
//   offs[NO + 1]   start of each owner's segment, then the total event count
//   recs[2*C*K]    {meta, weight}: meta = t << 24 | j << 16 | write << 15 | column, with
//                  t the token within the chunk, j the event's rank within its token's
//                  read (or write) set and column the slot's first TMEM column
//   alph[2*C*K]    GSU retention of write events (0 for reads)
//
// Block = (b, h, G consecutive chunks of C tokens); thread = (chunk, stream, token).  Each
// thread decodes one address (stream 0: key -> writes, stream 1: query -> reads); a
// stable counting sort by owner (one exclusive scan of the chunk-major, owner-major count
// table) places its K events within its chunk.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total_out)
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
    int base = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
        if (w < warp) base += warp_tot[w];
        total += warp_tot[w];
    }
    *total_out = total;
    return base + x - v;
}

template <int KMAX, int DPMAX>
__global__ void __launch_bounds__(128) k_decode_route(RouteParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = p.chunk, G = p.chunks_per_block;
    const int nt = blockDim.x;         // whole warps; threads >= 2*C*G carry no token
    const int nact = 2 * C * G;        // threads: (chunk g, stream, token)
    const int NW = p.nwarps;           // scan warps (owners) per CTA
    const int NO = NW * p.ncta;
    const int E = 2 * C * p.K;         // event capacity of one chunk
    const int TS = NO * 2 * C;         // table entries of one chunk
    uint64_t* kept = reinterpret_cast<uint64_t*>(smem);                          // [KMAX][nt]
    int* table = reinterpret_cast<int*>(smem + sizeof(uint64_t) * KMAX * nt);    // [G][NO][2C]
    int* warp_tot = table + G * TS;                                              // [4]
    uint2* srec = reinterpret_cast<uint2*>(warp_tot + 8);                        // [G][E]
    float* salp = reinterpret_cast<float*>(srec + G * E);                        // [G][E]
    int* soff = reinterpret_cast<int*>(salp + G * E);                            // [G][NO + 1]

    const int nblk = (p.nchunks + G - 1) / G;
    const int bh = blockIdx.x / nblk, c0 = (blockIdx.x - bh * nblk) * G;
    const int b = bh / p.H, h = bh - b * p.H;
    const int tid = threadIdx.x;
    const bool active = tid < nact;
    const int g = active ? tid / (2 * C) : 0, r2 = active ? tid - g * 2 * C : 0;
    const int stream = r2 >= C ? 1 : 0, tl = r2 - stream * C;
    const int c = c0 + g;
    const int t0 = c * C, n = c < p.nchunks ? min(C, p.T - t0) : 0;
    const bool valid = active && tl < n;
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
        const float gg = stream == 0 ? load_in(p.g, th, p.in_bf16) : 0.0f;
        if (stream == 0) {
            // the read accumulator of this token-head starts at zero
            float4* orow = reinterpret_cast<float4*>(p.o + th * p.d_v);
            for (int i = 0; i < p.d_v / 4; ++i) orow[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        const int lg_ncta = __ffs(p.ncta) - 1;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < p.K) {
                int32_t slot = packed_index(out[j], p.M);
                if (cape) slot = cape_shift(slot, pos, p.M);
                const int s = slot >> lg_ncta;
                owner[j] = (slot & (p.ncta - 1)) * NW + (s & (NW - 1));
                meta[j] = (static_cast<uint32_t>(tl) << 24) | (static_cast<uint32_t>(j) << 16) |
                          (stream == 0 ? 0x8000u : 0u) | static_cast<uint32_t>((s >> 2) * p.cpl);
                coef[j] = w[j];
                alpha[j] = stream == 0 ? gsu_alpha(w[j], gg) : 0.0f;
            }
        }
    }

    // per-thread owner counts: table[g][o][so]
    int* tg = table + g * TS;
    for (int i = tid; i < G * TS; i += nt) table[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (owner[j] >= 0) tg[owner[j] * 2 * C + so] += 1;
    __syncthreads();
    // exclusive scan of the flattened table (chunk-major, then owner, then token order);
    // thread i owns entries [i*W, min((i+1)*W, G*TS)), W = ceil(G*TS / nt) <= NO
    int total = 0;
    {
        const int W = (G * TS + nt - 1) / nt;
        const int lo = min(tid * W, G * TS), hi = min(lo + W, G * TS);
        int sum = 0;
        for (int k = lo; k < hi; ++k) sum += table[k];
        int run = block_exclusive_scan(sum, warp_tot, &total);
        for (int k = lo; k < hi; ++k) {
            const int v = table[k];
            table[k] = run;
            run += v;
        }
    }
    __syncthreads();
    const int chunk_base = table[g * TS];  // read before the scatter below modifies the table
    // per chunk: owner segment starts (relative to the chunk) and the chunk's total
    for (int i = tid; i < G * (NO + 1); i += nt) {
        const int gg = i / (NO + 1), o = i - gg * (NO + 1);
        const int base = table[gg * TS];
        const int next = gg + 1 < G ? table[(gg + 1) * TS] : total;
        soff[i] = (o < NO ? table[gg * TS + o * 2 * C] : next) - base;
    }
    __syncthreads();
    // scatter into shared memory: events of one owner keep token order, writes first
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (owner[j] >= 0) {
            const int posn = tg[owner[j] * 2 * C + so];
            tg[owner[j] * 2 * C + so] = posn + 1;
            srec[g * E + posn - chunk_base] = make_uint2(meta[j], __float_as_uint(coef[j]));
            salp[g * E + posn - chunk_base] = alpha[j];
        }
    }
    __syncthreads();
    // the chunk blocks: offsets, records, retentions
    for (int gg = 0; gg < G; ++gg) {
        const int cc = c0 + gg;
        if (cc >= p.nchunks) break;
        unsigned char* blk = p.blocks + (static_cast<size_t>(bh) * p.nchunks + cc) * p.chunk_bytes;
        int* goff = reinterpret_cast<int*>(blk);
        uint2* grec = reinterpret_cast<uint2*>(blk + p.recs_off);
        float* galp = reinterpret_cast<float*>(blk + p.alph_off);
        const int cnt = soff[gg * (NO + 1) + NO];
        for (int o = tid; o <= NO; o += nt) goff[o] = soff[gg * (NO + 1) + o];
        for (int i = tid; i < cnt; i += nt) {
            grec[i] = srec[gg * E + i];
            galp[i] = salp[gg * E + i];
        }
    }
}

int kmax_of(int K) { return K <= 8 ? 8 : K <= 16 ? 16 : K <= 32 ? 32 : 64; }

template <int KMAX, int DPMAX>
cudaError_t launch_route(const RouteParams& p, cudaStream_t s)
{
    const int G = p.chunks_per_block;
    const int nt = 2 * p.chunk * G;
    const size_t smem = route_smem_bytes(p.chunk, G, p.K, p.nwarps * p.ncta);
    auto kern = k_decode_route<KMAX, DPMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int nblk = (p.nchunks + G - 1) / G;
    const int threads = (nt + 31) / 32 * 32;  // whole warps (the block scan uses full-warp shuffles)
    kern<<<static_cast<unsigned>(p.B * p.H * nblk), threads, smem, s>>>(p);
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

size_t route_smem_bytes(int chunk, int G, int K, int n_owners)
{
    const int nt = (2 * chunk * G + 31) / 32 * 32;
    const size_t E = static_cast<size_t>(2) * chunk * K;
    return sizeof(uint64_t) * kmax_of(K) * nt + sizeof(int) * (static_cast<size_t>(G) * n_owners * 2 * chunk + 8) +
           (sizeof(uint2) + sizeof(float)) * G * E + sizeof(int) * G * (n_owners + 1);
}

// as many chunks per block as fit 128 threads (a power of two)
int route_chunks_per_block(int chunk, int nchunks)
{
    int G = 1;
    while (2 * chunk * G * 2 <= 128 && G * 2 <= nchunks) G *= 2;
    return G;
}

cudaError_t launch_decode_route(const RouteParams& p_in, cudaStream_t stream)
{
    RouteParams p = p_in;
    if (2 * p.chunk > 128 || p.nwarps * p.ncta > 128) return cudaErrorInvalidValue;
    p.chunks_per_block = route_chunks_per_block(p.chunk, p.nchunks);
    if (p.d_p <= 4) return route_k<4>(p, stream);
    if (p.d_p <= 8) return route_k<8>(p, stream);
    return route_k<16>(p, stream);
}

}  // namespace ramnet
