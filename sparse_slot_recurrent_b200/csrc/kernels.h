// kernels.h -- launch parameters and launchers of the RAM-Net kernels (host side).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace ramnet {

// Status bits written by kernels into the library's device status word.
enum : uint32_t { kDevTimeout = 1u, kDevCheck = 2u };

struct DecodeParams {
    const void* logits;  // [B,T,H,U*d_p], element (b,t,h,l) at b*sb + t*st + h*sh + l
    int64_t sb, st, sh;
    int in_bf16;
    int d_p, U, K, M, renorm;
    int B, T, H;
    const int32_t* pos0;       // [B] or null
    const uint8_t* cape_mask;  // [H] or null
    int32_t* idx_out;          // [B,T,H,K]
    float* w_out;              // [B,T,H,K]
    uint32_t* status;          // device status word (range checks of the debug build)
};

// ---------------------------------------------------------------- prefill scan plan
//
// One head's slot array S [M, d_v] is split over `ncta` CTAs (a thread-block cluster):
// slot i belongs to CTA rank (i mod ncta) as local slot s = i / ncta, and inside that CTA
// to scan warp (s mod nw).  An "owner" is one (rank, scan warp) pair, numbered
// rank * nw + warp.  Tokens are processed in chunks of `chunk` tokens.
//
// Workspace written by the route kernel and read by the scan kernel:
//   events  [B*H][nch][2*chunk*K] uint4, per (head, chunk) sorted by owner and, within one
//           owner, by (token, stream) (a token's writes before its reads):
//             x = s | tl << 16 | q << 24 | stream << 31
//                 s  local slot index, tl token within the chunk, stream 0 = write / 1 = read,
//                 q  (reads) rank of this read among the token's reads held by the same CTA,
//                    in rank (j) order; 0 for writes
//             y = weight (f32 bits), z = retention alpha (f32 bits, writes; 0 for reads),
//             w = slot index (after CAPE)
//   hdr     [B*H][nch][ncta][hdr_words] uint32, per (head, chunk, rank):
//             [0] first event of the rank in the chunk's sorted events, [1] its event count,
//             [2] tokens in the chunk, [3] 0, [4 + w] (w = 0..nw) start of scan warp w's
//             events relative to [0] ([4 + nw] = count), then chunk bytes: the number of
//             the token's reads held by this rank, token tl at byte tl.
struct ScanPlan {
    int ncta;        // CTAs per head (cluster size)
    int nw;          // scan warps per CTA
    int nfin;        // finisher warps per CTA
    int chunk;       // tokens per chunk
    int stages;      // staging ring depth (chunks of events and value rows)
    int lslots;      // read-partial ring depth (chunks)
    int xslots;      // exchange ring depth (chunks finished by this CTA)
    int cpl;         // channels per lane (d_v / 32, 1 for d_v = 16)
    int hdr_words;   // words per (head, chunk, rank) header
    uint32_t tmem_cols;
    size_t smem_bytes;
};

// Route kernel (first launch of the prefill): Top-K addresses, weights, CAPE and write
// retentions for every (token, stream), bucketed per owner.
struct RouteParams {
    const void* k_logits;  // [B,T,H,U*d_p]
    const void* q_logits;
    const void* g;  // [B,T,H]
    int in_bf16;
    int d_p, U, K, M, renorm;
    int B, T, H;
    const int32_t* pos0;       // [B] or null
    int64_t t_offset;          // position of token 0 relative to pos0 (pieces of a longer sequence)
    const uint8_t* cape_mask;  // [H] or null
    int ncta, nw, chunk, nch, hdr_words;
    uint4* events;
    uint32_t* hdr;
    uint32_t* status;
};

struct ScanParams {
    const uint4* events;
    const uint32_t* hdr;
    const void* v;  // [B,T,H,d_v]
    const void* z;  // [B,T,H,d_v]
    int in_bf16;
    const float* norm_w;  // [d_v] or null
    const float* S_in;    // [B,H,M,d_v] or null
    const float* m_in;    // [B,H,M] or null
    void* y;              // [B,T,H,d_v]
    int out_bf16;
    float* S_out;  // [B,H,M,d_v]
    float* m_out;  // [B,H,M]
    int B, T, H, K, M, d_v;
    int ncta, nw, nfin, chunk, nch, stages, lslots, xslots, hdr_words;
    float eps_gsu, eps_norm;
    uint32_t tmem_cols;
    uint64_t wait_ns;  // limit of every bounded wait of the kernel
    uint32_t* status;
};

struct StepParams {
    const void* k_logits;  // [B,H,L]
    const void* q_logits;
    const void* v;  // [B,H,d_v]
    const void* g;  // [B,H]
    const void* z;  // [B,H,d_v]
    int in_bf16;
    const float* norm_w;
    const uint8_t* cape_mask;
    const int32_t* pos;  // [B] or null
    float* S;            // [B,H,M,d_v]
    float* m;            // [B,H,M]
    void* y;             // [B,H,d_v]
    int out_bf16;
    int B, H, d_p, U, K, M, d_v, renorm;
    float eps_gsu, eps_norm;
    uint32_t* status;
};

// Plan of the prefill scan for these sizes and input element size; false if one head's
// slot array does not fit the tensor memory of 8 SMs or the shared memory budget.
bool scan_plan(int M, int d_v, int K, int in_bytes, ScanPlan* plan);

// Workspace of the prefill: events then headers (each at a 256-byte boundary).
struct ScanWorkspace {
    size_t events_bytes, hdr_off, hdr_bytes, total;
};
ScanWorkspace scan_workspace(int B, int T, int H, int K, const ScanPlan& plan);

cudaError_t launch_decode_addresses(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_route(const RouteParams& p, cudaStream_t stream);
cudaError_t launch_scan(const ScanParams& p, size_t smem_bytes, cudaStream_t stream);
// One block whose bounded wait on a never-signalled barrier runs out after limit_ns.
cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_decode_step(const StepParams& p, cudaStream_t stream);

}  // namespace ramnet
