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

// Decode + route (first kernel of the prefill scan): per (b, h, chunk) the token-ordered
// event list of every owner warp of the scan kernel.
// Decode + route (first kernel of the prefill scan): per (b, h, chunk) one block of
// `chunk_bytes` holding the owner offsets, the owner-sorted event records and the write
// retentions (layout: chunk_block_bytes()).
struct RouteParams {
    const void* k_logits;  // [B,T,H,U*d_p]
    const void* q_logits;
    const void* g;  // [B,T,H]
    int in_bf16;
    int d_p, U, K, M, renorm;
    int B, T, H;
    const int32_t* pos0;       // [B] or null
    const uint8_t* cape_mask;  // [H] or null
    int ncta, cpl, chunk, nchunks;
    int nwarps;             // scan warps per CTA (owners per CTA)
    int chunks_per_block;   // set by the launcher
    unsigned char* blocks;  // [B*H*nchunks][chunk_bytes]
    size_t chunk_bytes, recs_off, alph_off;
    float* o;               // [B,T,H,d_v] read accumulator, zeroed here
    int d_v;
};

struct ScanParams {
    const unsigned char* blocks;  // chunk blocks written by the route kernel
    size_t chunk_bytes, recs_off, alph_off;
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
    int ncta;   // CTAs per (b,h) = cluster size
    int chunk;  // tokens per chunk
    float eps_gsu, eps_norm;
    uint32_t tmem_cols;
    uint32_t* status;
    float* o;  // [B,T,H,d_v] read accumulator (zeroed by the route kernel)
};

struct ScanPlan {
    int ncta, chunk, cpl, nchunks, nwarps;
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

// Tensor-memory plan of the prefill scan: how many CTAs (cluster size) share one head's
// slot array, the chunk length, and the TMEM columns and shared memory of each CTA.
// Returns false if the slot array does not fit.
bool scan_plan(int M, int d_v, int K, int in_bytes, ScanPlan* plan);
// Bytes of one chunk block (offsets, records, retentions) and the offsets of its parts.
size_t chunk_block_bytes(int chunk, int K, int ncta, int nwarps, size_t* recs_off, size_t* alph_off);

cudaError_t launch_decode_addresses(const DecodeParams& p, cudaStream_t stream);
// Shared memory of one decode/route block of G chunks (largest G: 64 / chunk).
size_t route_smem_bytes(int chunk, int G, int K, int n_owners);
int route_chunks_per_block(int chunk, int nchunks);
cudaError_t launch_decode_route(const RouteParams& p, cudaStream_t stream);
cudaError_t launch_scan(const ScanParams& p, size_t smem_bytes, cudaStream_t stream);
// One block whose bounded wait on a never-signalled barrier runs out after limit_ns.
cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_decode_step(const StepParams& p, cudaStream_t stream);

}  // namespace ramnet
