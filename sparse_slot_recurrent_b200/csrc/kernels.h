// kernels.h -- launch parameters and launchers of the RAM-Net kernels (host side).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace ramnet {

// Status bits written by kernels into the library's device status word.
enum : uint32_t { kDevTimeout = 1u, kDevCheck = 2u };

struct DecodeParams {
    const void* logits;  // [B,T,H,U*d_p]
    int in_bf16;
    int d_p, U, K, M, renorm;
    int B, T, H;
    const int32_t* pos0;       // [B] or null
    const uint8_t* cape_mask;  // [H] or null
    int32_t* idx_out;          // [B,T,H,K]
    float* w_out;              // [B,T,H,K]
};

// Event decode (first kernel of the prefill scan): every token's K write and K read events,
// events[b][h][t][stream][j] = {slot, weight bits, alpha bits, t << 1 | stream}.
struct EventParams {
    const void* k_logits;  // [B,T,H,U*d_p]
    const void* q_logits;
    const void* g;  // [B,T,H]
    int in_bf16;
    int d_p, U, K, M, renorm;
    int B, T, H;
    const int32_t* pos0;       // [B] or null
    const uint8_t* cape_mask;  // [H] or null
    uint4* events;             // [B,H,T,2,K]
};

struct ScanParams {
    const uint4* events;  // [B,H,T,2,K] written by the event decode
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
    int ncta;   // CTAs per (b,h); CTA r holds the slots i with i mod ncta == r
    int chunk;  // tokens per chunk
    float eps_gsu, eps_norm;
    uint32_t tmem_cols;
    uint32_t* status;
    float* o;  // [B,T,H,d_v] read accumulator (reset to zero by ramnet_scan_route)
};

struct ScanPlan {
    int ncta, chunk, cpl;
    uint32_t tmem_cols;
    size_t smem_bytes;
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
};

// Tensor-memory plan of the prefill scan: how many CTAs share one head's slot array, the
// chunk length, and the TMEM columns and shared memory of each CTA.  Returns false if the
// slot array does not fit.
bool scan_plan(int M, int d_v, int K, int in_bytes, ScanPlan* plan);


cudaError_t launch_decode_addresses(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_decode_events(const EventParams& p, cudaStream_t stream);
cudaError_t launch_scan(const ScanParams& p, size_t smem_bytes, cudaStream_t stream);
// One block whose bounded wait on a never-signalled barrier runs out after limit_ns.
cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_decode_step(const StepParams& p, cudaStream_t stream);

}  // namespace ramnet
