// decode_addresses.cu -- K1: Address Decoder + CAPE for every token of every head.
//
// RAM-Net project page: Product Softmax paragraph (M = d_p^U slots from U*d_p scores),
// the exact Top-K search described after the five views, and the CAPE paragraphs.
// One thread decodes one (token, head): the decode is independent per token, so the grid
// simply covers B*T*H threads (GPU-execution paragraph: addresses for all tokens first).
// The search is the one the prefill route kernel and the decode step run: the kept list in
// registers (topk_search_net) for K <= 32, in shared memory (topk_search) above.
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

template <int KMAX, int DPMAX>
__global__ void __launch_bounds__(128) k_decode_addresses(DecodeParams p)
{
    extern __shared__ uint64_t kept_s[];  // [KMAX][blockDim.x], K > 32 only
    const long long n = static_cast<long long>(p.B) * p.T * p.H;
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int h = static_cast<int>(i % p.H);
    const long long bt = i / p.H;
    const int t = static_cast<int>(bt % p.T);
    const int b = static_cast<int>(bt / p.T);
    const size_t off = static_cast<size_t>(b * p.sb + t * p.st + h * p.sh);
    uint64_t out[KMAX];
    if constexpr (KMAX <= 32)
        topk_search_net<KMAX, DPMAX>(p.logits, off, p.in_bf16, p.d_p, p.U, p.K, out);
    else
        topk_search<KMAX, DPMAX>(p.logits, off, p.in_bf16, p.d_p, p.U, p.K, kept_s + threadIdx.x, blockDim.x, out);
    float w[KMAX];
    topk_weights<KMAX>(out, p.K, p.renorm, p.logits, off, p.in_bf16, p.d_p, p.U, w);
    const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
    const int64_t pos = static_cast<int64_t>(p.pos0 ? p.pos0[b] : 0) + t;
    const int32_t pm = cape ? cape_shift(0, pos, p.M) : 0;  // pos mod M, once per token
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < p.K) {
            int32_t idx = packed_index(out[j], p.M) + pm;
            if (idx >= p.M) idx -= p.M;
            if (!dcheck(idx >= 0 && idx < p.M, p.status)) idx = 0;
            p.idx_out[i * p.K + j] = idx;
            p.w_out[i * p.K + j] = w[j];
        }
    }
}

template <int KMAX, int DPMAX>
static cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream)
{
    const int threads = 128;
    const long long n = static_cast<long long>(p.B) * p.T * p.H;
    const long long blocks = (n + threads - 1) / threads;
    const size_t smem = KMAX <= 32 ? 0 : sizeof(uint64_t) * KMAX * threads;
    auto kern = k_decode_addresses<KMAX, DPMAX>;
    if (smem > 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    kern<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int DPMAX>
static cudaError_t dispatch_k(const DecodeParams& p, cudaStream_t s)
{
    if (p.K <= 8) return launch_decode<8, DPMAX>(p, s);
    if (p.K <= 16) return launch_decode<16, DPMAX>(p, s);
    if (p.K <= 32) return launch_decode<32, DPMAX>(p, s);
    return launch_decode<64, DPMAX>(p, s);
}

cudaError_t launch_decode_addresses(const DecodeParams& p, cudaStream_t stream)
{
    if (p.d_p <= 4) return dispatch_k<4>(p, stream);
    if (p.d_p <= 8) return dispatch_k<8>(p, stream);
    return dispatch_k<16>(p, stream);
}

}  // namespace ramnet
