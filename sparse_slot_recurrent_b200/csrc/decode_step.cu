// decode_step.cu -- K3: one autoregressive token per (b,h) against an HBM-resident state.
//
// RAM-Net project page, GPU-execution paragraph on decoding: the step touches only the
// slots its token selects and never scans the whole state.  Per (b,h): decode the key and
// query addresses (Product Softmax Top-K + CAPE), apply the Gated Sparse Update to the K
// write rows of S and their masses, read the K read rows (after the write), RMSNorm,
// gate, store y.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

constexpr int kStepThreads = 128;

template <int KMAX, int DPMAX>
__global__ void __launch_bounds__(kStepThreads) k_decode_step(StepParams p)
{
    __shared__ uint64_t kept_s[KMAX * 2];
    __shared__ int32_t wi_s[KMAX], ri_s[KMAX];
    __shared__ float ww_s[KMAX], rw_s[KMAX], lam_s[KMAX];
    __shared__ float red_s[kStepThreads / 32];
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x;
    const int L = p.U * p.d_p;
    const int K = p.K, dv = p.d_v, M = p.M;

    // ---- address decode: lane 0 the key (write set), lane 1 the query (read set)
    if (tid < 2) {
        const void* lg = tid == 0 ? p.k_logits : p.q_logits;
        const size_t off = static_cast<size_t>(bh) * L;
        uint64_t out[KMAX];
        topk_search<KMAX, DPMAX>(lg, off, p.in_bf16, p.d_p, p.U, K, kept_s + tid, 2, out);
        float w[KMAX];
        topk_weights<KMAX>(out, K, p.renorm, lg, off, p.in_bf16, p.d_p, p.U, w);
        const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
        const int64_t pos = p.pos != nullptr ? p.pos[b] : 0;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < K) {
                int32_t idx = packed_index(out[j], M);
                if (cape) idx = cape_shift(idx, pos, M);
                if (tid == 0) {
                    wi_s[j] = idx;
                    ww_s[j] = w[j];
                } else {
                    ri_s[j] = idx;
                    rw_s[j] = w[j];
                }
            }
        }
    }
    __syncthreads();

    // ---- GSU steps 1-3: mass and rate of each (distinct) write slot
    float* mrow = p.m + static_cast<size_t>(bh) * M;
    if (tid < K) {
        const float g = load_in(p.g, bh, p.in_bf16);
        const int i = wi_s[tid];
        const float w = ww_s[tid];
        const float mn = gsu_alpha(w, g) * mrow[i] + w;
        mrow[i] = mn;
        lam_s[tid] = w / (mn + p.eps_gsu);
    }
    __syncthreads();

    // ---- step 4 on the write rows, then the read (same thread owns a channel throughout)
    float* S = p.S + static_cast<size_t>(bh) * M * dv;
    float ss = 0.0f;
    float o_keep[2] = {0.0f, 0.0f};
    int slot = 0;
    for (int ch = tid; ch < dv; ch += kStepThreads, ++slot) {
        const float vv = load_in(p.v, static_cast<size_t>(bh) * dv + ch, p.in_bf16);
        for (int j = 0; j < K; ++j) {
            float* sp = S + static_cast<size_t>(wi_s[j]) * dv + ch;
            const float s0 = *sp;
            *sp = fmaf(lam_s[j], vv - s0, s0);
        }
        float o = 0.0f;
        for (int j = 0; j < K; ++j) o += rw_s[j] * S[static_cast<size_t>(ri_s[j]) * dv + ch];
        ss += o * o;
        o_keep[slot] = o;
    }
    // ---- RMSNorm over d_v and the output gate
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((tid & 31) == 0) red_s[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
    for (int w = 0; w < kStepThreads / 32; ++w) tot += red_s[w];
    const float inv = 1.0f / sqrtf(tot / dv + p.eps_norm);
    slot = 0;
    for (int ch = tid; ch < dv; ch += kStepThreads, ++slot) {
        const float nw = p.norm_w != nullptr ? p.norm_w[ch] : 1.0f;
        const float y = o_keep[slot] * inv * nw * load_in(p.z, static_cast<size_t>(bh) * dv + ch, p.in_bf16);
        store_out(p.y, static_cast<size_t>(bh) * dv + ch, y, p.out_bf16);
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_step(const StepParams& p, cudaStream_t s)
{
    k_decode_step<KMAX, DPMAX><<<static_cast<unsigned>(p.B * p.H), kStepThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <int DPMAX>
cudaError_t step_k(const StepParams& p, cudaStream_t s)
{
    if (p.K <= 8) return launch_step<8, DPMAX>(p, s);
    if (p.K <= 16) return launch_step<16, DPMAX>(p, s);
    if (p.K <= 32) return launch_step<32, DPMAX>(p, s);
    return launch_step<64, DPMAX>(p, s);
}

}  // namespace

cudaError_t launch_decode_step(const StepParams& p, cudaStream_t stream)
{
    if (p.d_v > 2 * kStepThreads) return cudaErrorInvalidValue;
    if (p.d_p <= 4) return step_k<4>(p, stream);
    if (p.d_p <= 8) return step_k<8>(p, stream);
    return step_k<16>(p, stream);
}

}  // namespace ramnet
