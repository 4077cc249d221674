/*
 * ramnet.h -- C ABI of the B200 (sm_100a) RAM-Net layer core.
 *
 * The layer follows the RAM-Net project page ("RAM-Net: Linear-Time Sequence Modeling
 * with Sparsely Addressable State", muoncat.github.io/ramnet_web).  Each token of each
 * head brings an address logit vector for its key (write) and its query (read), a value
 * v, a write gate g and an output gate z.  The layer:
 *   1. Address Decoder / Product Softmax: splits each logit vector into U groups of d_p
 *      scores, and finds the exact Top-K of the M = d_p^U slot weights
 *      prod_u softmax(x_u)[d_u] by a level-by-level prefix-tree search;
 *   2. CAPE: shifts the selected slot indices cyclically by the token position on heads
 *      whose CAPE flag is set;
 *   3. Gated Sparse Update: updates content and write mass of the K write slots only;
 *   4. reads the K read slots combined by their weights, applies RMSNorm over d_v and
 *      multiplies by the output gate.
 *
 * Numerical definitions (identical on every entry point):
 *   - Ranking score of one digit logit x: q(x) = round_half_even(clamp(x, -4095, 4095)
 *     * 2^32) as a 64-bit integer (NaN ranks lowest); a slot's score is the integer sum
 *     of its U digit scores.  Higher score wins; equal scores go to the lower slot index
 *     (taken before the CAPE shift).  Slot index i = sum_u d_u * d_p^(U-1-u): group 0 of
 *     the logits is the most significant digit.
 *   - Weights of the K selected slots (rank order): renorm != 0: w_j = exp(s_j - s_0) /
 *     sum_k exp(s_k - s_0) with s the slot's digit-logit sum; renorm == 0: w_j =
 *     prod_u softmax(x_u)[d_u].  Logits are expected within +-4095 (the clamp also
 *     enters the weights).
 *   - CAPE: slot -> (slot + pos) mod M with pos = pos0[b] + t.
 *   - Gated Sparse Update of write slot i with weight w, gate g in [0,1] (clamped):
 *     alpha = (1 - w)^(g/(1-g)) [alpha = 1 when w == 0 or g == 0; 0 when g == 1 or
 *     w == 1], m_i <- alpha*m_i + w, lambda = w/(m_i + eps_gsu), S_i <- S_i +
 *     lambda*(v - S_i).  Slots not written keep content and mass bit for bit.
 *   - Read after the token's own write: o = sum_j r_j S_{read_j};
 *     y = o / sqrt(mean(o^2) + eps_norm) * norm_w * z.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE memory owned by the caller, unless stated otherwise; the
 *     library never frees or keeps them.  Arrays are dense row-major (C order) with the
 *     stated shapes; every base pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls
 *     are asynchronous on that stream: outputs are valid once the stream has reached
 *     the call.  The caller keeps inputs alive until then.
 *   - Argument checks happen on the host before anything is launched; a failing check
 *     returns RAMNET_ERR_INVALID_ARG or RAMNET_ERR_UNSUPPORTED and launches nothing.
 *     A launch error returns RAMNET_ERR_CUDA.  ramnet_last_error() describes the last
 *     failure of the calling thread.
 *   - Where warps of a kernel wait for one another (the prefill scan's staging ring) every
 *     wait is bounded (about 2 s); when a wait gives up the kernel records it in a device
 *     status word and finishes early.  ramnet_sync_status() reads (and clears) that word.
 *   - No call allocates device memory.  Scratch space comes from the caller
 *     (ramnet_scan_forward's workspace) or, for ramnet_scan_forward_noalloc, from a
 *     fixed array inside the library's device image.
 *   - Limits: 2 <= d_p <= 16, 1 <= U <= 8, M = d_p^U <= 65536, 1 <= K <= min(M, 64),
 *     d_v in {16, 32, 64, 128, 256}.  ramnet_scan_forward additionally needs the slot
 *     array of one head to fit the tensor memory of at most 8 SMs (M * max(d_v,32) *
 *     4 bytes <= 8 * 256 KiB); larger shapes return RAMNET_ERR_UNSUPPORTED.
 */
#ifndef RAMNET_H
#define RAMNET_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RAMNET_OK = 0,
    RAMNET_ERR_INVALID_ARG = 1,   /* bad pointer, shape, alignment or value */
    RAMNET_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels implement */
    RAMNET_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    RAMNET_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up */
    RAMNET_ERR_DEVICE_CHECK = 5   /* a device-side consistency check failed */
} ramnet_status;

typedef enum {
    RAMNET_F32 = 0,
    RAMNET_BF16 = 1
} ramnet_dtype;

/* Layer hyper-parameters.  M = d_p^U slots per head. */
typedef struct {
    int32_t d_p;      /* values per digit (softmax group size)            */
    int32_t U;        /* digits per address (number of softmax groups)     */
    int32_t K;        /* slots selected per read and per write             */
    int32_t d_v;      /* value / slot width                                */
    float eps_gsu;    /* epsilon of the GSU update rate (e.g. 1e-6)        */
    float eps_norm;   /* epsilon inside the output RMSNorm (e.g. 1e-6)     */
    int32_t renorm;   /* 1: weights renormalised over the K selected slots */
} ramnet_config;

/* Element strides of a [B,T,H,L] logits array whose last dimension is contiguous: element
 * (b, t, h, l) sits at b*b_stride + t*t_stride + h*h_stride + l.  Strides are >= 0 and may
 * describe a permuted or sliced view (for example a [B,H,T,L] array read as [B,T,H,L]). */
typedef struct {
    int64_t b, t, h;
} ramnet_strides;

/*
 * ramnet_decode_addresses -- Address Decoder and CAPE for a batch of tokens.
 * Project page: Product Softmax paragraph, the five views (exact Top-K search in the
 * Multilevel Decision Tree view and the exactness paragraph after them), CAPE paragraphs.
 *
 *   logits    [B,T,H,U*d_p]  dtype `dt` (RAMNET_F32 or RAMNET_BF16), laid out as `strides`
 *             says (NULL: dense, strides (T*H*L, H*L, L)); only element alignment is needed
 *   pos0      [B] int32 start position of each sequence, or NULL (all 0)
 *   cape_mask [H] uint8, nonzero = CAPE on for that head, or NULL (CAPE off)
 *   idx_out   [B,T,H,K] int32 (dense): selected slot indices, best first, after CAPE
 *   w_out     [B,T,H,K] fp32 (dense): their weights (same order)
 * Errors: INVALID_ARG for null logits/outputs, non-positive sizes, a negative stride,
 * misalignment or a config outside the limits.
 */
ramnet_status ramnet_decode_addresses(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                      const void* logits, ramnet_dtype dt, const ramnet_strides* strides,
                                      const int32_t* pos0, const uint8_t* cape_mask, int32_t* idx_out,
                                      float* w_out, void* stream);

/*
 * ramnet_scan_workspace_bytes -- scratch bytes ramnet_scan_forward needs for these sizes
 * (the larger of the fp32- and bf16-input plans): the decoded read and write events
 * (16 bytes each, 2*K per token, grouped per chunk of tokens) and a small header per
 * (head, chunk, CTA rank); see ramnet_scan_layout.  Returns 0 for invalid arguments.
 */
size_t ramnet_scan_workspace_bytes(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H);

/*
 * ramnet_scan_layout -- how ramnet_scan_forward splits the work for this config and input
 * dtype, which fixes the workspace contents after ramnet_scan_route.  The pages have no
 * counterpart: it serves tools and tests that read the workspace.
 *
 *   *chunk       tokens per chunk C (nch = ceil(T / C) chunks per head)
 *   *ncta        CTAs per head (one thread-block cluster); slot i belongs to rank i mod ncta
 *                as local slot s = i / ncta
 *   *scan_warps  scan warps per CTA (nw); local slot s belongs to scan warp s mod nw
 *   *hdr_words   32-bit words per (head, chunk, rank) header
 *
 * Workspace contents after ramnet_scan_route (head = b*H + h):
 *   events at offset 0: [B*H][nch][2*C*K] records of 4 uint32 {x, weight, alpha, slot}; a
 *     chunk's records are sorted by owner (rank * nw + scan warp) and, within one owner, by
 *     (token, stream).  x = s | tl << 16 | q << 24 | stream << 31 with s the local slot, tl
 *     the token within the chunk, stream 0 for a write (key) and 1 for a read (query), q
 *     the read's rank among the token's reads held by the same rank; weight and alpha are
 *     f32 bits (alpha = the write's retention, 0 for reads); slot is the index after CAPE.
 *   headers at offset round_up(B*H*nch*2*C*K*16, 256): [B*H][nch][ncta][hdr_words] uint32:
 *     [0] first record of the rank in the chunk, [1] the rank's record count, [2] tokens
 *     in the chunk, [3] 0, [4 + w] (w = 0..nw) start of scan warp w's records relative to
 *     [0], then one byte per token: how many of its reads the rank holds.
 * Errors: INVALID_ARG (config, dtype, NULL outputs), UNSUPPORTED as ramnet_scan_forward.
 */
ramnet_status ramnet_scan_layout(const ramnet_config* cfg, ramnet_dtype in_dt, int32_t* chunk, int32_t* ncta,
                                 int32_t* scan_warps, int32_t* hdr_words);

/*
 * ramnet_scan_forward -- prefill: the whole layer core over T tokens, per (b,h) in token
 * order.  Project page: the three-stage processing paragraph, Gated Sparse Update (four
 * steps and the unselected-slot rule), and the GPU-execution paragraph (Top-K for all
 * tokens in parallel first, then the recurrence).
 *
 *   k_logits, q_logits [B,T,H,U*d_p]  in_dt   key (write) / query (read) address logits
 *   v, z               [B,T,H,d_v]    in_dt   value, output gate (multiplied as given)
 *   g                  [B,T,H]        in_dt   write gate in [0,1] (activated gamma)
 *   norm_w             [d_v] fp32 or NULL (ones)
 *   cape_mask          [H] uint8 or NULL (off);  pos0 [B] int32 or NULL (0)
 *   S_in               [B,H,M,d_v] fp32 initial slot contents, or NULL (zeros)
 *   m_in               [B,H,M] fp32 initial write mass, or NULL (zeros)
 *   y                  [B,T,H,d_v] out_dt output
 *   S_out, m_out       final state, same shapes as S_in, m_in (may alias them)
 *   workspace          device scratch of at least ramnet_scan_workspace_bytes() bytes,
 *                      16-byte aligned; contents on entry are ignored
 * Errors: INVALID_ARG (null required pointer, sizes, alignment, too small workspace),
 * UNSUPPORTED (slot array too large for tensor memory, see limits).
 */
ramnet_status ramnet_scan_forward(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                  ramnet_dtype in_dt, const void* k_logits, const void* q_logits,
                                  const void* v, const void* g, const void* z,
                                  const float* norm_w, const uint8_t* cape_mask,
                                  const int32_t* pos0, const float* S_in, const float* m_in,
                                  void* y, ramnet_dtype out_dt, float* S_out, float* m_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * ramnet_scan_route, ramnet_scan_recur -- ramnet_scan_forward in its two launches, for
 * callers that time or schedule them apart.  ramnet_scan_forward(...) is exactly
 * ramnet_scan_route(...) followed on the same stream by ramnet_scan_recur(...) with the
 * same cfg, B, T, H, in_dt and workspace.
 *
 * ramnet_scan_route: the address decoder for every token and stream (Product-Softmax
 *   Top-K, weights, CAPE; project page, Product Softmax and CAPE paragraphs), the write
 *   retentions of GSU step 1, and the grouping of all read and write events by the scan
 *   warp that owns their slot (GPU-execution paragraph: addresses for all tokens first,
 *   events grouped by slot).  Reads k_logits, q_logits, g, cape_mask, pos0 as in
 *   ramnet_scan_forward; writes the workspace (contents on entry ignored; layout in
 *   ramnet_scan_layout).
 * ramnet_scan_recur: the recurrence (GSU steps 1-4, sparse read after the token's write,
 *   RMSNorm, norm weight, output gate) over the events in the workspace, which must hold
 *   what ramnet_scan_route wrote for the same arguments.  It only reads the workspace, so
 *   it may run more than once after one ramnet_scan_route (same results each time: every
 *   sum on the path has a fixed order).
 *   v, z, norm_w, S_in, m_in, y, S_out, m_out as in ramnet_scan_forward.
 * Errors: as ramnet_scan_forward.
 */
ramnet_status ramnet_scan_route(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                ramnet_dtype in_dt, const void* k_logits, const void* q_logits,
                                const void* g, const uint8_t* cape_mask, const int32_t* pos0,
                                void* workspace, size_t workspace_bytes, void* stream);
ramnet_status ramnet_scan_recur(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                ramnet_dtype in_dt, const void* v, const void* z,
                                const float* norm_w, const float* S_in, const float* m_in, void* y,
                                ramnet_dtype out_dt, float* S_out, float* m_out,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * ramnet_scan_forward_host -- the prefill scan with the per-token tensors in HOST memory:
 * k_logits, q_logits, v, g, z ([B,T,H,.], last dim contiguous, as ramnet_scan_forward) are
 * read from the host and y is written to the host; norm_w, cape_mask, pos0, S_in, m_in,
 * S_out and m_out are device pointers as in ramnet_scan_forward.  Same results as
 * ramnet_scan_forward, bit for bit.
 *
 * The sequence is cut into `pieces` runs of ceil(T / pieces) tokens.  The scan is causal
 * and its state (S, m) is the whole carry, so run i starts from the state run i-1 left in
 * S_out / m_out (run 0 from S_in / m_in) and its CAPE positions continue at
 * pos0[b] + (first token of the run); this is the RAM-Net project page's recurrence taken
 * piece by piece.  Copies of run i+1 into the device and of run i-1's y out of it overlap
 * run i's kernels (two copy streams created for the call; page-locked host memory lets the
 * copies run asynchronously).  Work is ordered after earlier work on `stream`, and
 * `stream` waits for the whole call, the last copy out included.
 *
 *   scratch: device memory of ramnet_scan_forward_host_scratch_bytes() bytes (two
 *            staging buffers for the inputs and y of a run, and one workspace), 16-byte
 *            aligned, owned by the caller and not used by other work during the call.
 *   Errors:  INVALID_ARG (NULL host tensor, pieces < 1, scratch too small, and the checks
 *            of ramnet_scan_forward), UNSUPPORTED, CUDA.
 */
size_t ramnet_scan_forward_host_scratch_bytes(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                              ramnet_dtype in_dt, ramnet_dtype out_dt, int32_t pieces);
ramnet_status ramnet_scan_forward_host(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                       ramnet_dtype in_dt, const void* k_logits, const void* q_logits,
                                       const void* v, const void* g, const void* z,
                                       const float* norm_w, const uint8_t* cape_mask,
                                       const int32_t* pos0, const float* S_in, const float* m_in,
                                       void* y, ramnet_dtype out_dt, float* S_out, float* m_out,
                                       int32_t pieces, void* scratch, size_t scratch_bytes,
                                       void* stream);

/* Size of the scratch array built into the library for ramnet_scan_forward_noalloc. */
#define RAMNET_NOALLOC_SCRATCH_BYTES ((size_t)32 * 1024 * 1024)

/*
 * ramnet_scan_forward_noalloc -- ramnet_scan_forward without a caller-provided workspace.
 * The RAM-Net pages describe no such call: it exists for callers that cannot pass device
 * memory of their own (host code without a device allocator, or a hot path on which an
 * allocation could block or fail).  Same arguments, results and errors as
 * ramnet_scan_forward, minus workspace and workspace_bytes.
 *
 *   Scratch:   a static, 256-byte aligned device array of RAMNET_NOALLOC_SCRATCH_BYTES
 *              (32 MiB) per device, part of the library's device image.  Sizes for which
 *              ramnet_scan_workspace_bytes() exceeds that return RAMNET_ERR_UNSUPPORTED
 *              with a message giving both numbers.  Nothing in the array has to start at
 *              zero: each call writes all the scratch it later reads.
 *   Set-up:    the first call on a device (with that device current) looks up the
 *              array's device address once and keeps it for the current CUDA context; a
 *              call made in a new context (after cudaDeviceReset, or after the primary
 *              context was released and created again) looks it up again.  Make the first
 *              call in a context before beginning any stream capture.
 *   Sharing:   all calls on a device use the same array.  Calls whose work can overlap
 *              on the device (other streams, other host threads) race on it; issue them
 *              on one stream, or use ramnet_scan_forward with separate workspaces.
 *   Allocation: none, host or device.
 */
ramnet_status ramnet_scan_forward_noalloc(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                          ramnet_dtype in_dt, const void* k_logits,
                                          const void* q_logits, const void* v, const void* g,
                                          const void* z, const float* norm_w,
                                          const uint8_t* cape_mask, const int32_t* pos0,
                                          const float* S_in, const float* m_in, void* y,
                                          ramnet_dtype out_dt, float* S_out, float* m_out,
                                          void* stream);

/*
 * ramnet_decode_step -- one autoregressive token per (b,h) against an HBM-resident state,
 * touching only the slots the token selects.  Project page: GPU-execution paragraph on
 * autoregressive decoding (no scan over the full state), plus the same three stages.
 *
 *   k_logits, q_logits [B,H,U*d_p] in_dt;  v, z [B,H,d_v] in_dt;  g [B,H] in_dt
 *   norm_w [d_v] fp32 or NULL;  cape_mask [H] uint8 or NULL
 *   pos    [B] int32 position of this token in its sequence, or NULL (0)
 *   S      [B,H,M,d_v] fp32, m [B,H,M] fp32: state, updated in place
 *   y      [B,H,d_v] out_dt
 * Errors: INVALID_ARG as above.
 */
ramnet_status ramnet_decode_step(const ramnet_config* cfg, int32_t B, int32_t H, ramnet_dtype in_dt,
                                 const void* k_logits, const void* q_logits, const void* v,
                                 const void* g, const void* z, const float* norm_w,
                                 const uint8_t* cape_mask, const int32_t* pos, float* S, float* m,
                                 void* y, ramnet_dtype out_dt, void* stream);

/*
 * ramnet_selftest_wait_timeout -- failure-detection self-test.  The pages have no
 * counterpart: it checks this library's own guard against lost signals.  Launches one
 * block on `stream` whose bounded wait (the same routine every wait of the prefill scan
 * uses) is on a barrier that nothing signals, so it gives up after limit_us microseconds
 * and records RAMNET_ERR_TIMEOUT in the device status word; the next
 * ramnet_sync_status(stream) returns RAMNET_ERR_TIMEOUT and clears it.  No fault, trap
 * or hang is involved and the context stays usable.
 * Errors: INVALID_ARG unless 1 <= limit_us <= 2000000.
 */
ramnet_status ramnet_selftest_wait_timeout(uint32_t limit_us, void* stream);

/*
 * ramnet_set_scan_wait_limit -- failure-detection hook, no counterpart in the pages.  Sets
 * the limit of every bounded wait inside the prefill recurrence (ramnet_scan_recur,
 * ramnet_scan_forward, ramnet_scan_forward_noalloc) launched after the call, for the whole
 * process: limit_us microseconds, or 0 for the default of 2 s.  A wait that runs out records
 * RAMNET_ERR_TIMEOUT in the device status word and the kernel winds down: its remaining
 * work is skipped, so y, S_out and m_out are then incomplete.  A limit far below the
 * kernel's own hand-over times makes the recurrence time out on purpose, which is how its
 * abort path is tested.
 * Errors: INVALID_ARG if limit_us > 2000000.
 */
ramnet_status ramnet_set_scan_wait_limit(uint32_t limit_us);

/*
 * ramnet_sync_status -- waits for `stream`, then returns RAMNET_ERR_TIMEOUT or
 * RAMNET_ERR_DEVICE_CHECK if a kernel of this library on the current device recorded a
 * gave-up wait or a failed check since the last call (and clears the record), or
 * RAMNET_ERR_CUDA if the stream reports an error; RAMNET_OK otherwise.
 */
ramnet_status ramnet_sync_status(void* stream);

/* Message describing the calling thread's last failure ("" if none).  Owned by the
 * library; valid until the next call from the same thread. */
const char* ramnet_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RAMNET_H */
