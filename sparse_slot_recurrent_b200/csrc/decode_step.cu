// decode_step.cu -- K3: one autoregressive token per (b,h) against an HBM-resident state.
//
// RAM-Net project page, GPU-execution paragraph on decoding: the step touches only the
// slots its token selects and never scans the whole state.  Per (b,h): decode the key and
// query addresses (Product Softmax Top-K + CAPE), apply the Gated Sparse Update to the K
// write rows of S and their masses, read the K read rows (after the write), RMSNorm,
// gate, store y.
//
// One CTA of 128 threads handles kUnits (b,h) units:
//   1. warp 0 decodes the kUnits keys (lanes 0..15) and queries (lanes 16..31) at once,
//      one address per lane, so the integer Top-K search runs on every lane;
//   2. all threads apply GSU steps 1-3 (retention, mass, rate) to the K write slots of
//      every unit;
//   3. warp w takes units w, w+4, ...: lane l owns channels [l*CPL, l*CPL + CPL) of a row,
//      so a slot row is one coalesced warp access; the K write rows of a unit are loaded
//      together (16 in flight per lane, 8 at d_v = 256), updated and stored, then its K read rows
//      are loaded together and summed; RMSNorm by a warp reduction, gate, store y.
// Write rows of one unit are distinct slots (Top-K without repeats, CAPE a bijection).  A
// read row loaded by the same lane after its own store of that row sees the stored value
// (same address, program order), so the read loads follow the write stores directly.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace ramnet {

namespace {

constexpr int kStepThreads = 128;
constexpr int kUnits = 16;     // (b,h) units per CTA

template <int KMAX, int DPMAX, int CPL>
__global__ void __launch_bounds__(kStepThreads) k_decode_step(StepParams p)
{
    __shared__ uint64_t kept_s[KMAX][32];
    __shared__ int32_t wi_s[kUnits][KMAX], ri_s[kUnits][KMAX];
    __shared__ float ww_s[kUnits][KMAX], rw_s[kUnits][KMAX], lam_s[kUnits][KMAX];
    constexpr int kRowBatch = CPL >= 8 ? 8 : 16;  // rows per lane in flight
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = p.U * p.d_p;
    const int K = p.K, dv = p.d_v, M = p.M;
    const int units = p.B * p.H;
    const int u0 = blockIdx.x * kUnits;

    // ---- 1. address decode: lane l of warp 0 decodes stream l / 16 of unit u0 + l % 16
    if (warp == 0) {
        const int ul = lane & (kUnits - 1), stream = lane / kUnits;
        const int bh = u0 + ul;
        if (bh < units) {
            const void* lg = stream == 0 ? p.k_logits : p.q_logits;
            const size_t off = static_cast<size_t>(bh) * L;
            uint64_t out[KMAX];
            if constexpr (KMAX <= 32)
                topk_search_net<KMAX, DPMAX>(lg, off, p.in_bf16, p.d_p, p.U, K, out);  // kept list in registers
            else
                topk_search<KMAX, DPMAX>(lg, off, p.in_bf16, p.d_p, p.U, K, &kept_s[0][lane], 32, out);
            float w[KMAX];
            topk_weights<KMAX>(out, K, p.renorm, lg, off, p.in_bf16, p.d_p, p.U, w);
            const int h = bh % p.H, b = bh / p.H;
            const bool cape = p.cape_mask != nullptr && p.cape_mask[h] != 0;
            const int64_t pos = p.pos != nullptr ? p.pos[b] : 0;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < K) {
                    int32_t idx = packed_index(out[j], M);
                    if (cape) idx = cape_shift(idx, pos, M);
                    if (!dcheck(idx >= 0 && idx < M, p.status)) idx = 0;
                    if (stream == 0) {
                        wi_s[ul][j] = idx;
                        ww_s[ul][j] = w[j];
                    } else {
                        ri_s[ul][j] = idx;
                        rw_s[ul][j] = w[j];
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---- 2. GSU steps 1-3: mass and rate of each (distinct) write slot of each unit
    for (int i = tid; i < kUnits * K; i += kStepThreads) {
        const int ul = i / K, j = i - ul * K;
        const int bh = u0 + ul;
        if (bh < units) {
            float* mrow = p.m + static_cast<size_t>(bh) * M;
            const float g = load_in(p.g, bh, p.in_bf16);
            const int s = wi_s[ul][j];
            const float w = ww_s[ul][j];
            const float mn = gsu_alpha(w, g) * mrow[s] + w;
            mrow[s] = mn;
            lam_s[ul][j] = w / (mn + p.eps_gsu);
        }
    }
    __syncthreads();

    // ---- 3. content update, read, RMSNorm and gate; one warp per unit at a time
    const int LW = (CPL > 1 || dv >= 32) ? 32 : dv;  // lanes holding channels
    const bool act = lane < LW;
    const int ch0 = (act ? lane : 0) * CPL;
    float nw[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) nw[c] = p.norm_w != nullptr ? p.norm_w[ch0 + c] : 1.0f;
    for (int ul = warp; ul < kUnits; ul += kStepThreads / 32) {
        const int bh = u0 + ul;
        if (bh >= units) break;
        float* S = p.S + static_cast<size_t>(bh) * M * dv;
        float vv[CPL], o[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            vv[c] = load_in(p.v, static_cast<size_t>(bh) * dv + ch0 + c, p.in_bf16);
            o[c] = 0.0f;
        }
        for (int j0 = 0; j0 < K; j0 += kRowBatch) {
            float s[kRowBatch][CPL];
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k)
                if (j0 + k < K && act) load_row_g<CPL>(S + static_cast<size_t>(wi_s[ul][j0 + k]) * dv + ch0, s[k]);
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k) {
                if (j0 + k < K && act) {
                    const float lam = lam_s[ul][j0 + k];
#pragma unroll
                    for (int c = 0; c < CPL; ++c) s[k][c] = fmaf(lam, vv[c] - s[k][c], s[k][c]);
                    store_row_g<CPL>(S + static_cast<size_t>(wi_s[ul][j0 + k]) * dv + ch0, s[k]);
                }
            }
        }
        for (int j0 = 0; j0 < K; j0 += kRowBatch) {
            float s[kRowBatch][CPL];
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k)
                if (j0 + k < K && act) load_row_g<CPL>(S + static_cast<size_t>(ri_s[ul][j0 + k]) * dv + ch0, s[k]);
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k) {
                if (j0 + k < K && act) {
                    const float r = rw_s[ul][j0 + k];
#pragma unroll
                    for (int c = 0; c < CPL; ++c) o[c] = fmaf(r, s[k][c], o[c]);
                }
            }
        }
        float ss = 0.0f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) ss = fmaf(o[c], o[c], ss);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = 1.0f / sqrtf(ss / dv + p.eps_norm);
        if (act) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const size_t e = static_cast<size_t>(bh) * dv + ch0 + c;
                store_out(p.y, e, o[c] * inv * nw[c] * load_in(p.z, e, p.in_bf16), p.out_bf16);
            }
        }
    }
}

template <int KMAX, int DPMAX>
cudaError_t launch_step(const StepParams& p, cudaStream_t s)
{
    const unsigned grid = static_cast<unsigned>((p.B * p.H + kUnits - 1) / kUnits);
    switch (p.d_v < 32 ? 1 : p.d_v / 32) {
        case 1: k_decode_step<KMAX, DPMAX, 1><<<grid, kStepThreads, 0, s>>>(p); break;
        case 2: k_decode_step<KMAX, DPMAX, 2><<<grid, kStepThreads, 0, s>>>(p); break;
        case 4: k_decode_step<KMAX, DPMAX, 4><<<grid, kStepThreads, 0, s>>>(p); break;
        case 8: k_decode_step<KMAX, DPMAX, 8><<<grid, kStepThreads, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
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
    if (p.d_v > 256) return cudaErrorInvalidValue;
    if (p.d_p <= 4) return step_k<4>(p, stream);
    if (p.d_p <= 8) return step_k<8>(p, stream);
    return step_k<16>(p, stream);
}

}  // namespace ramnet
