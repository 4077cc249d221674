// decode_events.cu -- K1 of the prefill scan: the Address Decoder and CAPE for every token
// of every head, written as read and write events in token order.
//
// RAM-Net project page, GPU-execution paragraph: Top-K addresses for all tokens are
// computed in parallel first; the scan then walks each slot's events in causal order.  One
// thread decodes one (token, head, stream): stream 0 the key (its K events are writes),
// stream 1 the query (reads).  Per event it also computes the retention alpha of GSU step
// 1 for writes.  Output, per (b, h), token-major:
//   events[b][h][t][stream][j] = {slot, weight (f32 bits), alpha (f32 bits, writes),
//                                 t << 1 | stream}
// so within one head the events are in token order, a token's writes before its reads;
// the scan kernel's warps pick their own slots' events out of this order.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

constexpr int kEventThreads = 128;

template <int KMAX, int DPMAX>
__global__ void __launch_bounds__(kEventThreads) k_decode_events(EventParams p)
{
    extern __shared__ uint64_t kept_s[];  // [KMAX][kEventThreads], K > 16 only
    const long long n = static_cast<long long>(p.B) * p.H * p.T * 2;
    const long long i = static_cast<long long>(blockIdx.x) * kEventThreads + threadIdx.x;
    if (i >= n) return;
    const int stream = static_cast<int>(i & 1);
    const long long hti = i >> 1;  // (b*H + h)*T + t
    const int t = static_cast<int>(hti % p.T);
    const int bh = static_cast<int>(hti / p.T);
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;  // [B,T,H] index
    const int L = p.U * p.d_p;
    const void* lg = stream == 0 ? p.k_logits : p.q_logits;
    uint64_t out[KMAX];
    if constexpr (KMAX <= 16)
        topk_search_net<KMAX, DPMAX>(lg, th * L, p.in_bf16, p.d_p, p.U, p.K, out);  // kept list in registers
    else
        topk_search<KMAX, DPMAX>(lg, th * L, p.in_bf16, p.d_p, p.U, p.K, kept_s + threadIdx.x, kEventThreads, out);
    float w[KMAX];
    topk_weights<KMAX>(out, p.K, p.renorm, lg, th * L, p.in_bf16, p.d_p, p.U, w);
    const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
    const int64_t pos = static_cast<int64_t>(p.pos0 != nullptr ? p.pos0[b] : 0) + t;
    const float gg = stream == 0 ? load_in(p.g, th, p.in_bf16) : 0.0f;
    uint4* ev = p.events + static_cast<size_t>(i) * p.K;
    const uint32_t tag = (static_cast<uint32_t>(t) << 1) | static_cast<uint32_t>(stream);
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < p.K) {
            int32_t slot = packed_index(out[j], p.M);
            if (cape) slot = cape_shift(slot, pos, p.M);
            const float al = stream == 0 ? gsu_alpha(w[j], gg) : 0.0f;
            ev[j] = make_uint4(static_cast<uint32_t>(slot), __float_as_uint(w[j]), __float_as_uint(al), tag);
        }
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_events(const EventParams& p, cudaStream_t s)
{
    const long long n = static_cast<long long>(p.B) * p.H * p.T * 2;
    const unsigned blocks = static_cast<unsigned>((n + kEventThreads - 1) / kEventThreads);
    const size_t smem = KMAX <= 16 ? 0 : sizeof(uint64_t) * KMAX * kEventThreads;
    auto kern = k_decode_events<KMAX, DPMAX>;
    if (smem > 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    kern<<<blocks, kEventThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int DPMAX>
cudaError_t events_k(const EventParams& p, cudaStream_t s)
{
    if (p.K <= 8) return launch_events<8, DPMAX>(p, s);
    if (p.K <= 16) return launch_events<16, DPMAX>(p, s);
    if (p.K <= 32) return launch_events<32, DPMAX>(p, s);
    return launch_events<64, DPMAX>(p, s);
}

}  // namespace

cudaError_t launch_decode_events(const EventParams& p, cudaStream_t stream)
{
    if (p.T >= (1 << 30)) return cudaErrorInvalidValue;
    if (p.d_p <= 4) return events_k<4>(p, stream);
    if (p.d_p <= 8) return events_k<8>(p, stream);
    return events_k<16>(p, stream);
}

}  // namespace ramnet
