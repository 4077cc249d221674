// decode_step.cu -- K3: one autoregressive token per (b,h) against an HBM-resident state.
//
// RAM-Net project page, GPU-execution paragraph on decoding: the step touches only the
// slots its token selects and never scans the whole state.  Per (b,h): decode the key and
// query addresses (Product Softmax Top-K + CAPE), apply the Gated Sparse Update to the K
// write rows of S and their masses, read the K read rows (after the write), RMSNorm,
// gate, store y.
//
// The step is bound by HBM latency and bandwidth on scattered 4*d_v-byte rows, so the
// kernel keeps many row accesses in flight: one 64-thread CTA per (b,h) (up to 32 CTAs per
// SM), the key and the query decoded by lane 0 of warp 0 and warp 1 (no divergence between
// them), and each thread loading all rows of a batch of kRowBatch slots before using any.
// Write rows are distinct slots (Top-K without repeats, CAPE a bijection).  A read row
// loaded by the same thread after its own store of that row sees the stored value (same
// address, program order), so the read loads follow the write stores without a barrier.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

constexpr int kStepThreads = 64;
constexpr int kRowBatch = 16;  // rows per thread in flight

template <int KMAX, int DPMAX, int CPT>
__global__ void __launch_bounds__(kStepThreads) k_decode_step(StepParams p)
{
    __shared__ uint64_t kept_s[2][KMAX];
    __shared__ int32_t wi_s[KMAX], ri_s[KMAX];
    __shared__ float ww_s[KMAX], rw_s[KMAX], lam_s[KMAX];
    __shared__ float red_s[kStepThreads / 32];
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = p.U * p.d_p;
    const int K = p.K, dv = p.d_v, M = p.M;

    // ---- address decode: warp 0 lane 0 the key (write set), warp 1 lane 0 the query
    if (lane == 0) {
        const void* lg = warp == 0 ? p.k_logits : p.q_logits;
        const size_t off = static_cast<size_t>(bh) * L;
        uint64_t out[KMAX];
        topk_search<KMAX, DPMAX>(lg, off, p.in_bf16, p.d_p, p.U, K, kept_s[warp], 1, out);
        float w[KMAX];
        topk_weights<KMAX>(out, K, p.renorm, lg, off, p.in_bf16, p.d_p, p.U, w);
        const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
        const int64_t pos = p.pos != nullptr ? p.pos[b] : 0;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < K) {
                int32_t idx = packed_index(out[j], M);
                if (cape) idx = cape_shift(idx, pos, M);
                if (warp == 0) {
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
    for (int j = tid; j < K; j += kStepThreads) {
        const float g = load_in(p.g, bh, p.in_bf16);
        const int i = wi_s[j];
        const float w = ww_s[j];
        const float mn = gsu_alpha(w, g) * mrow[i] + w;
        mrow[i] = mn;
        lam_s[j] = w / (mn + p.eps_gsu);
    }
    __syncthreads();

    // ---- step 4 on the write rows, then the reads; thread owns channels tid + 64*c
    float* S = p.S + static_cast<size_t>(bh) * M * dv;
    float vv[CPT], o[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int ch = tid + kStepThreads * c;
        vv[c] = ch < dv ? load_in(p.v, static_cast<size_t>(bh) * dv + ch, p.in_bf16) : 0.0f;
        o[c] = 0.0f;
    }
    for (int j0 = 0; j0 < K; j0 += kRowBatch) {
        float s[kRowBatch][CPT];
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const int ch = tid + kStepThreads * c;
                s[k][c] = (j0 + k < K && ch < dv) ? S[static_cast<size_t>(wi_s[j0 + k]) * dv + ch] : 0.0f;
            }
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) {
            if (j0 + k < K) {
                const float lam = lam_s[j0 + k];
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    const int ch = tid + kStepThreads * c;
                    if (ch < dv) S[static_cast<size_t>(wi_s[j0 + k]) * dv + ch] = fmaf(lam, vv[c] - s[k][c], s[k][c]);
                }
            }
        }
    }
    for (int j0 = 0; j0 < K; j0 += kRowBatch) {
        float s[kRowBatch][CPT];
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const int ch = tid + kStepThreads * c;
                s[k][c] = (j0 + k < K && ch < dv) ? S[static_cast<size_t>(ri_s[j0 + k]) * dv + ch] : 0.0f;
            }
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) {
            if (j0 + k < K) {
                const float r = rw_s[j0 + k];
#pragma unroll
                for (int c = 0; c < CPT; ++c) o[c] = fmaf(r, s[k][c], o[c]);
            }
        }
    }
    // ---- RMSNorm over d_v and the output gate
    float ss = 0.0f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) ss = fmaf(o[c], o[c], ss);
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) red_s[warp] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kStepThreads / 32; ++w) tot += red_s[w];
    const float inv = 1.0f / sqrtf(tot / dv + p.eps_norm);
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int ch = tid + kStepThreads * c;
        if (ch < dv) {
            const float nw = p.norm_w != nullptr ? p.norm_w[ch] : 1.0f;
            const float y = o[c] * inv * nw * load_in(p.z, static_cast<size_t>(bh) * dv + ch, p.in_bf16);
            store_out(p.y, static_cast<size_t>(bh) * dv + ch, y, p.out_bf16);
        }
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_step(const StepParams& p, cudaStream_t s)
{
    const unsigned grid = static_cast<unsigned>(p.B * p.H);
    if (p.d_v <= 64) {
        k_decode_step<KMAX, DPMAX, 1><<<grid, kStepThreads, 0, s>>>(p);
    } else if (p.d_v <= 128) {
        k_decode_step<KMAX, DPMAX, 2><<<grid, kStepThreads, 0, s>>>(p);
    } else {
        k_decode_step<KMAX, DPMAX, 4><<<grid, kStepThreads, 0, s>>>(p);
    }
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
    if (p.d_v > 4 * kStepThreads) return cudaErrorInvalidValue;
    if (p.d_p <= 4) return step_k<4>(p, stream);
    if (p.d_p <= 8) return step_k<8>(p, stream);
    return step_k<16>(p, stream);
}

}  // namespace ramnet
