// ramnet_api.cu -- the C ABI declared in include/ramnet.h: argument checks, launches,
// status reporting.  Nothing here allocates device memory.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/ramnet.h"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;
// limit of every bounded wait of the prefill recurrence (process-wide; ramnet_set_scan_wait_limit)
std::atomic<uint64_t> g_scan_wait_ns{2000000000ull};

// Device-side status word of this library (one per device that loads the library).
__device__ uint32_t g_device_status;

ramnet_status fail(ramnet_status s, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

ramnet_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(RAMNET_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(ramnet_dtype d) { return d == RAMNET_F32 || d == RAMNET_BF16; }

// Shared config checks; on success writes M.
ramnet_status check_config(const ramnet_config* cfg, int* M_out)
{
    if (cfg == nullptr) return fail(RAMNET_ERR_INVALID_ARG, "cfg is NULL");
    if (cfg->d_p < 2 || cfg->d_p > 16) return fail(RAMNET_ERR_INVALID_ARG, "d_p=%d outside [2,16]", cfg->d_p);
    if (cfg->U < 1 || cfg->U > 8) return fail(RAMNET_ERR_INVALID_ARG, "U=%d outside [1,8]", cfg->U);
    long long M = 1;
    for (int u = 0; u < cfg->U; ++u) {
        M *= cfg->d_p;
        if (M > 65536) return fail(RAMNET_ERR_INVALID_ARG, "M = d_p^U exceeds 65536");
    }
    if (cfg->K < 1 || cfg->K > 64 || cfg->K > M)
        return fail(RAMNET_ERR_INVALID_ARG, "K=%d outside [1, min(M=%lld, 64)]", cfg->K, M);
    if (!(cfg->d_v == 16 || cfg->d_v == 32 || cfg->d_v == 64 || cfg->d_v == 128 || cfg->d_v == 256))
        return fail(RAMNET_ERR_INVALID_ARG, "d_v=%d not in {16,32,64,128,256}", cfg->d_v);
    if (!(cfg->eps_gsu >= 0.0f) || !(cfg->eps_norm >= 0.0f))
        return fail(RAMNET_ERR_INVALID_ARG, "epsilons must be >= 0");
    *M_out = static_cast<int>(M);
    return RAMNET_OK;
}

ramnet_status check_sizes(long long B, long long T, long long H)
{
    if (B < 1 || T < 1 || H < 1) return fail(RAMNET_ERR_INVALID_ARG, "B, T, H must be >= 1");
    if (B * T * H > (1ll << 31) - 1) return fail(RAMNET_ERR_INVALID_ARG, "B*T*H too large");
    return RAMNET_OK;
}

#define REQUIRE_PTR(p)                                                                          \
    do {                                                                                        \
        if ((p) == nullptr) return fail(RAMNET_ERR_INVALID_ARG, "%s is NULL", #p);              \
        if (!aligned16(p)) return fail(RAMNET_ERR_INVALID_ARG, "%s not 16-byte aligned", #p); \
    } while (0)
#define OPTIONAL_PTR(p)                                                                         \
    do {                                                                                        \
        if ((p) != nullptr && !aligned16(p))                                                    \
            return fail(RAMNET_ERR_INVALID_ARG, "%s not 16-byte aligned", #p);                  \
    } while (0)

uint32_t* device_status_ptr()
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    return static_cast<uint32_t*>(p);
}

}  // namespace

namespace ramnet {

// Sets the text ramnet_last_error returns on this thread (for entry points in other files).
ramnet_status set_last_error(ramnet_status s, const char* msg)
{
    g_last_error = msg;
    return s;
}

}  // namespace ramnet

extern "C" {

const char* ramnet_last_error(void) { return g_last_error.c_str(); }

ramnet_status ramnet_decode_addresses(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, const void* logits,
                                      ramnet_dtype dt, const ramnet_strides* strides, const int32_t* pos0,
                                      const uint8_t* cape_mask, int32_t* idx_out, float* w_out, void* stream)
{
    g_last_error.clear();
    int M = 0;
    ramnet_status st = check_config(cfg, &M);
    if (st != RAMNET_OK) return st;
    if ((st = check_sizes(B, T, H)) != RAMNET_OK) return st;
    if (!valid_dtype(dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype %d", static_cast<int>(dt));
    if (logits == nullptr) return fail(RAMNET_ERR_INVALID_ARG, "logits is NULL");
    const size_t es = dt == RAMNET_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(logits) & (es - 1)) != 0)
        return fail(RAMNET_ERR_INVALID_ARG, "logits not aligned to its element size");
    const int64_t L = static_cast<int64_t>(cfg->U) * cfg->d_p;
    int64_t sb = static_cast<int64_t>(T) * H * L, stt = static_cast<int64_t>(H) * L, sh = L;
    if (strides != nullptr) {
        sb = strides->b;
        stt = strides->t;
        sh = strides->h;
        if (sb < 0 || stt < 0 || sh < 0) return fail(RAMNET_ERR_INVALID_ARG, "negative logits stride");
        const double span = static_cast<double>(B - 1) * sb + static_cast<double>(T - 1) * stt +
                            static_cast<double>(H - 1) * sh + static_cast<double>(L);
        if (span > 9.0e18) return fail(RAMNET_ERR_INVALID_ARG, "logits strides overflow");
    }
    REQUIRE_PTR(idx_out);
    REQUIRE_PTR(w_out);
    OPTIONAL_PTR(pos0);
    OPTIONAL_PTR(cape_mask);
    uint32_t* status = device_status_ptr();
    if (status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
    ramnet::DecodeParams p{logits, sb, stt, sh, dt == RAMNET_BF16, cfg->d_p, cfg->U, cfg->K, M, cfg->renorm != 0,
                           B, T, H, pos0, cape_mask, idx_out, w_out, status};
    cudaError_t e = ramnet::launch_decode_addresses(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode_addresses launch");
    return RAMNET_OK;
}

size_t ramnet_scan_workspace_bytes(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H)
{
    int M = 0;
    if (check_config(cfg, &M) != RAMNET_OK || check_sizes(B, T, H) != RAMNET_OK) return 0;
    // the chunk length depends on the input element size: the larger of the two
    size_t total = 0;
    for (int in_bytes : {2, 4}) {
        ramnet::ScanPlan plan;
        if (!ramnet::scan_plan(M, cfg->d_v, cfg->K, in_bytes, &plan)) return 0;
        const size_t t = ramnet::scan_workspace(B, T, H, cfg->K, plan).total;
        total = t > total ? t : total;
    }
    return total;
}

ramnet_status ramnet_scan_layout(const ramnet_config* cfg, ramnet_dtype in_dt, int32_t* chunk, int32_t* ncta,
                                 int32_t* scan_warps, int32_t* hdr_words)
{
    g_last_error.clear();
    int M = 0;
    ramnet_status st = check_config(cfg, &M);
    if (st != RAMNET_OK) return st;
    if (!valid_dtype(in_dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype %d", static_cast<int>(in_dt));
    if (chunk == nullptr || ncta == nullptr || scan_warps == nullptr || hdr_words == nullptr)
        return fail(RAMNET_ERR_INVALID_ARG, "output pointer is NULL");
    ramnet::ScanPlan plan;
    if (!ramnet::scan_plan(M, cfg->d_v, cfg->K, in_dt == RAMNET_BF16 ? 2 : 4, &plan))
        return fail(RAMNET_ERR_UNSUPPORTED, "slot array M=%d x d_v=%d does not fit the tensor memory of 8 SMs", M,
                    cfg->d_v);
    *chunk = plan.chunk;
    *ncta = plan.ncta;
    *scan_warps = plan.nw;
    *hdr_words = plan.hdr_words;
    return RAMNET_OK;
}

}  // extern "C"

namespace {

// Checks shared by the three prefill entry points; on success fills M, the plan and the
// workspace layout.
ramnet_status check_scan(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt,
                         const void* workspace, size_t workspace_bytes, int* M, ramnet::ScanPlan* plan,
                         ramnet::ScanWorkspace* wl)
{
    ramnet_status st = check_config(cfg, M);
    if (st != RAMNET_OK) return st;
    if ((st = check_sizes(B, T, H)) != RAMNET_OK) return st;
    if (!valid_dtype(in_dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype");
    REQUIRE_PTR(workspace);
    if (!ramnet::scan_plan(*M, cfg->d_v, cfg->K, in_dt == RAMNET_BF16 ? 2 : 4, plan))
        return fail(RAMNET_ERR_UNSUPPORTED, "slot array M=%d x d_v=%d does not fit the tensor memory of 8 SMs", *M,
                    cfg->d_v);
    *wl = ramnet::scan_workspace(B, T, H, cfg->K, *plan);
    if (workspace_bytes < wl->total)
        return fail(RAMNET_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, wl->total);
    return RAMNET_OK;
}

ramnet_status route_part(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt, int M,
                         const ramnet::ScanPlan& plan, const ramnet::ScanWorkspace& wl, const void* k_logits,
                         const void* q_logits, const void* g, const uint8_t* cape_mask, const int32_t* pos0,
                         void* workspace, cudaStream_t s, int64_t t_offset = 0)
{
    ramnet::RouteParams rp{};
    rp.t_offset = t_offset;
    rp.k_logits = k_logits;
    rp.q_logits = q_logits;
    rp.g = g;
    rp.in_bf16 = in_dt == RAMNET_BF16;
    rp.d_p = cfg->d_p;
    rp.U = cfg->U;
    rp.K = cfg->K;
    rp.M = M;
    rp.renorm = cfg->renorm != 0;
    rp.B = B;
    rp.T = T;
    rp.H = H;
    rp.pos0 = pos0;
    rp.cape_mask = cape_mask;
    rp.ncta = plan.ncta;
    rp.nw = plan.nw;
    rp.chunk = plan.chunk;
    rp.nch = (T + plan.chunk - 1) / plan.chunk;
    rp.hdr_words = plan.hdr_words;
    rp.events = static_cast<uint4*>(workspace);
    rp.hdr = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(workspace) + wl.hdr_off);
    rp.status = device_status_ptr();
    if (rp.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
    cudaError_t e = ramnet::launch_route(rp, s);
    if (e != cudaSuccess) return cuda_fail(e, "scan: route launch");
    return RAMNET_OK;
}

ramnet_status recur_part(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt, int M,
                         const ramnet::ScanPlan& plan, const ramnet::ScanWorkspace& wl, const void* v, const void* z,
                         const float* norm_w, const float* S_in, const float* m_in, void* y, ramnet_dtype out_dt,
                         float* S_out, float* m_out, void* workspace, cudaStream_t s)
{
    uint32_t* status = device_status_ptr();
    if (status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
    ramnet::ScanParams sp{};
    sp.events = static_cast<const uint4*>(workspace);
    sp.hdr = reinterpret_cast<const uint32_t*>(static_cast<const unsigned char*>(workspace) + wl.hdr_off);
    sp.v = v;
    sp.z = z;
    sp.in_bf16 = in_dt == RAMNET_BF16;
    sp.norm_w = norm_w;
    sp.S_in = S_in;
    sp.m_in = m_in;
    sp.y = y;
    sp.out_bf16 = out_dt == RAMNET_BF16;
    sp.S_out = S_out;
    sp.m_out = m_out;
    sp.B = B;
    sp.T = T;
    sp.H = H;
    sp.K = cfg->K;
    sp.M = M;
    sp.d_v = cfg->d_v;
    sp.ncta = plan.ncta;
    sp.nw = plan.nw;
    sp.nfin = plan.nfin;
    sp.chunk = plan.chunk;
    sp.nch = (T + plan.chunk - 1) / plan.chunk;
    sp.stages = plan.stages;
    sp.lslots = plan.lslots;
    sp.xslots = plan.xslots;
    sp.hdr_words = plan.hdr_words;
    sp.eps_gsu = cfg->eps_gsu;
    sp.eps_norm = cfg->eps_norm;
    sp.tmem_cols = plan.tmem_cols;
    sp.wait_ns = g_scan_wait_ns.load(std::memory_order_relaxed);
    sp.status = status;
    cudaError_t e = ramnet::launch_scan(sp, plan.smem_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    return RAMNET_OK;
}

}  // namespace

extern "C" {

ramnet_status ramnet_scan_forward(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt,
                                  const void* k_logits, const void* q_logits, const void* v, const void* g,
                                  const void* z, const float* norm_w, const uint8_t* cape_mask, const int32_t* pos0,
                                  const float* S_in, const float* m_in, void* y, ramnet_dtype out_dt, float* S_out,
                                  float* m_out, void* workspace, size_t workspace_bytes, void* stream)
{
    g_last_error.clear();
    int M = 0;
    ramnet::ScanPlan plan;
    ramnet::ScanWorkspace wl;
    ramnet_status st = check_scan(cfg, B, T, H, in_dt, workspace, workspace_bytes, &M, &plan, &wl);
    if (st != RAMNET_OK) return st;
    if (!valid_dtype(out_dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype");
    REQUIRE_PTR(k_logits);
    REQUIRE_PTR(q_logits);
    REQUIRE_PTR(v);
    REQUIRE_PTR(g);
    REQUIRE_PTR(z);
    REQUIRE_PTR(y);
    REQUIRE_PTR(S_out);
    REQUIRE_PTR(m_out);
    OPTIONAL_PTR(norm_w);
    OPTIONAL_PTR(cape_mask);
    OPTIONAL_PTR(pos0);
    OPTIONAL_PTR(S_in);
    OPTIONAL_PTR(m_in);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = route_part(cfg, B, T, H, in_dt, M, plan, wl, k_logits, q_logits, g, cape_mask, pos0, workspace, s);
    if (st != RAMNET_OK) return st;
    return recur_part(cfg, B, T, H, in_dt, M, plan, wl, v, z, norm_w, S_in, m_in, y, out_dt, S_out, m_out, workspace,
                      s);
}

ramnet_status ramnet_scan_route(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt,
                                const void* k_logits, const void* q_logits, const void* g, const uint8_t* cape_mask,
                                const int32_t* pos0, void* workspace, size_t workspace_bytes, void* stream)
{
    g_last_error.clear();
    int M = 0;
    ramnet::ScanPlan plan;
    ramnet::ScanWorkspace wl;
    ramnet_status st = check_scan(cfg, B, T, H, in_dt, workspace, workspace_bytes, &M, &plan, &wl);
    if (st != RAMNET_OK) return st;
    REQUIRE_PTR(k_logits);
    REQUIRE_PTR(q_logits);
    REQUIRE_PTR(g);
    OPTIONAL_PTR(cape_mask);
    OPTIONAL_PTR(pos0);
    return route_part(cfg, B, T, H, in_dt, M, plan, wl, k_logits, q_logits, g, cape_mask, pos0, workspace,
                      static_cast<cudaStream_t>(stream));
}

ramnet_status ramnet_scan_recur(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt,
                                const void* v, const void* z, const float* norm_w, const float* S_in,
                                const float* m_in, void* y, ramnet_dtype out_dt, float* S_out, float* m_out,
                                void* workspace, size_t workspace_bytes, void* stream)
{
    g_last_error.clear();
    int M = 0;
    ramnet::ScanPlan plan;
    ramnet::ScanWorkspace wl;
    ramnet_status st = check_scan(cfg, B, T, H, in_dt, workspace, workspace_bytes, &M, &plan, &wl);
    if (st != RAMNET_OK) return st;
    if (!valid_dtype(out_dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype");
    REQUIRE_PTR(v);
    REQUIRE_PTR(z);
    REQUIRE_PTR(y);
    REQUIRE_PTR(S_out);
    REQUIRE_PTR(m_out);
    OPTIONAL_PTR(norm_w);
    OPTIONAL_PTR(S_in);
    OPTIONAL_PTR(m_in);
    return recur_part(cfg, B, T, H, in_dt, M, plan, wl, v, z, norm_w, S_in, m_in, y, out_dt, S_out, m_out,
                      workspace, static_cast<cudaStream_t>(stream));
}

ramnet_status ramnet_selftest_wait_timeout(uint32_t limit_us, void* stream)
{
    g_last_error.clear();
    if (limit_us < 1 || limit_us > 2000000) return fail(RAMNET_ERR_INVALID_ARG, "limit_us=%u outside [1, 2000000]", limit_us);
    uint32_t* status = device_status_ptr();
    if (status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
    cudaError_t e = ramnet::launch_wait_selftest(status, static_cast<uint64_t>(limit_us) * 1000ull,
                                                 static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
    return RAMNET_OK;
}

ramnet_status ramnet_set_scan_wait_limit(uint32_t limit_us)
{
    g_last_error.clear();
    if (limit_us > 2000000) return fail(RAMNET_ERR_INVALID_ARG, "limit_us=%u above 2000000", limit_us);
    g_scan_wait_ns.store(limit_us == 0 ? 2000000000ull : static_cast<uint64_t>(limit_us) * 1000ull,
                         std::memory_order_relaxed);
    return RAMNET_OK;
}

ramnet_status ramnet_decode_step(const ramnet_config* cfg, int32_t B, int32_t H, ramnet_dtype in_dt,
                                 const void* k_logits, const void* q_logits, const void* v, const void* g,
                                 const void* z, const float* norm_w, const uint8_t* cape_mask, const int32_t* pos,
                                 float* S, float* m, void* y, ramnet_dtype out_dt, void* stream)
{
    g_last_error.clear();
    int M = 0;
    ramnet_status st = check_config(cfg, &M);
    if (st != RAMNET_OK) return st;
    if ((st = check_sizes(B, 1, H)) != RAMNET_OK) return st;
    if (!valid_dtype(in_dt) || !valid_dtype(out_dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype");
    REQUIRE_PTR(k_logits);
    REQUIRE_PTR(q_logits);
    REQUIRE_PTR(v);
    REQUIRE_PTR(g);
    REQUIRE_PTR(z);
    REQUIRE_PTR(S);
    REQUIRE_PTR(m);
    REQUIRE_PTR(y);
    OPTIONAL_PTR(norm_w);
    OPTIONAL_PTR(cape_mask);
    OPTIONAL_PTR(pos);
    ramnet::StepParams p{};
    p.k_logits = k_logits;
    p.q_logits = q_logits;
    p.v = v;
    p.g = g;
    p.z = z;
    p.in_bf16 = in_dt == RAMNET_BF16;
    p.norm_w = norm_w;
    p.cape_mask = cape_mask;
    p.pos = pos;
    p.S = S;
    p.m = m;
    p.y = y;
    p.out_bf16 = out_dt == RAMNET_BF16;
    p.B = B;
    p.H = H;
    p.d_p = cfg->d_p;
    p.U = cfg->U;
    p.K = cfg->K;
    p.M = M;
    p.d_v = cfg->d_v;
    p.renorm = cfg->renorm != 0;
    p.eps_gsu = cfg->eps_gsu;
    p.eps_norm = cfg->eps_norm;
    p.status = device_status_ptr();
    if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
    cudaError_t e = ramnet::launch_decode_step(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode_step launch");
    return RAMNET_OK;
}

ramnet_status ramnet_sync_status(void* stream)
{
    g_last_error.clear();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    uint32_t word = 0;
    e = cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "read status word");
    if (word != 0) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clear status word");
        if (word & ramnet::kDevTimeout) return fail(RAMNET_ERR_TIMEOUT, "a device-side wait gave up (status 0x%x)", word);
        return fail(RAMNET_ERR_DEVICE_CHECK, "a device-side check failed (status 0x%x)", word);
    }
    return RAMNET_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ prefill from host memory
namespace {

struct HostPieces {
    int n;          // pieces
    int tp;         // tokens per piece (the last may be shorter)
    size_t in_piece[5];  // bytes of one piece of k, q, v, g, z
    size_t y_piece;
    size_t in_off[2][5], y_off[2], ws_off, total;
    ramnet::ScanWorkspace wl;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

HostPieces host_pieces(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt,
                       ramnet_dtype out_dt, int32_t pieces, const ramnet::ScanPlan& plan)
{
    HostPieces hp{};
    hp.n = pieces < 1 ? 1 : (pieces > T ? T : pieces);
    hp.tp = (T + hp.n - 1) / hp.n;
    hp.n = (T + hp.tp - 1) / hp.tp;
    const size_t es = in_dt == RAMNET_BF16 ? 2 : 4, eo = out_dt == RAMNET_BF16 ? 2 : 4;
    const size_t th = static_cast<size_t>(B) * hp.tp * H;
    const size_t L = static_cast<size_t>(cfg->U) * cfg->d_p;
    hp.in_piece[0] = hp.in_piece[1] = th * L * es;
    hp.in_piece[2] = hp.in_piece[4] = th * cfg->d_v * es;
    hp.in_piece[3] = th * es;
    hp.y_piece = th * cfg->d_v * eo;
    size_t o = 0;
    for (int buf = 0; buf < 2; ++buf) {
        for (int i = 0; i < 5; ++i) {
            hp.in_off[buf][i] = o;
            o += align256(hp.in_piece[i]);
        }
        hp.y_off[buf] = o;
        o += align256(hp.y_piece);
    }
    hp.wl = ramnet::scan_workspace(B, hp.tp, H, cfg->K, plan);
    hp.ws_off = o;
    o += align256(hp.wl.total);
    hp.total = o;
    return hp;
}

}  // namespace

extern "C" {

size_t ramnet_scan_forward_host_scratch_bytes(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                              ramnet_dtype in_dt, ramnet_dtype out_dt, int32_t pieces)
{
    g_last_error.clear();
    int M = 0;
    if (check_config(cfg, &M) != RAMNET_OK || check_sizes(B, T, H) != RAMNET_OK || !valid_dtype(in_dt) ||
        !valid_dtype(out_dt))
        return 0;
    ramnet::ScanPlan plan;
    if (!ramnet::scan_plan(M, cfg->d_v, cfg->K, in_dt == RAMNET_BF16 ? 2 : 4, &plan)) return 0;
    return host_pieces(cfg, B, T, H, in_dt, out_dt, pieces, plan).total;
}

ramnet_status ramnet_scan_forward_host(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H, ramnet_dtype in_dt,
                                       const void* k_logits, const void* q_logits, const void* v, const void* g,
                                       const void* z, const float* norm_w, const uint8_t* cape_mask,
                                       const int32_t* pos0, const float* S_in, const float* m_in, void* y,
                                       ramnet_dtype out_dt, float* S_out, float* m_out, int32_t pieces,
                                       void* scratch, size_t scratch_bytes, void* stream)
{
    g_last_error.clear();
    int M = 0;
    ramnet_status st = check_config(cfg, &M);
    if (st != RAMNET_OK) return st;
    if ((st = check_sizes(B, T, H)) != RAMNET_OK) return st;
    if (!valid_dtype(in_dt) || !valid_dtype(out_dt)) return fail(RAMNET_ERR_INVALID_ARG, "bad dtype");
    if (pieces < 1) return fail(RAMNET_ERR_INVALID_ARG, "pieces=%d < 1", pieces);
    if (k_logits == nullptr || q_logits == nullptr || v == nullptr || g == nullptr || z == nullptr || y == nullptr)
        return fail(RAMNET_ERR_INVALID_ARG, "a host input or y is NULL");
    REQUIRE_PTR(S_out);
    REQUIRE_PTR(m_out);
    REQUIRE_PTR(scratch);
    OPTIONAL_PTR(norm_w);
    OPTIONAL_PTR(cape_mask);
    OPTIONAL_PTR(pos0);
    OPTIONAL_PTR(S_in);
    OPTIONAL_PTR(m_in);
    ramnet::ScanPlan plan;
    if (!ramnet::scan_plan(M, cfg->d_v, cfg->K, in_dt == RAMNET_BF16 ? 2 : 4, &plan))
        return fail(RAMNET_ERR_UNSUPPORTED, "slot array M=%d x d_v=%d does not fit the tensor memory of 8 SMs", M,
                    cfg->d_v);
    const HostPieces hp = host_pieces(cfg, B, T, H, in_dt, out_dt, pieces, plan);
    if (scratch_bytes < hp.total)
        return fail(RAMNET_ERR_INVALID_ARG, "scratch of %zu bytes, %zu needed", scratch_bytes, hp.total);

    const size_t es = in_dt == RAMNET_BF16 ? 2 : 4, eo = out_dt == RAMNET_BF16 ? 2 : 4;
    const size_t L = static_cast<size_t>(cfg->U) * cfg->d_p;
    const size_t row_bytes[5] = {L * es, L * es, static_cast<size_t>(cfg->d_v) * es, es,
                                 static_cast<size_t>(cfg->d_v) * es};  // per token-head
    const void* src[5] = {k_logits, q_logits, v, g, z};
    unsigned char* base = static_cast<unsigned char*>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // copy-in and copy-out streams; events order them against the compute stream `s`
    cudaStream_t sin = nullptr, sout = nullptr;
    cudaEvent_t ev_start = nullptr, ev_in[2] = {nullptr, nullptr}, ev_done[2] = {nullptr, nullptr},
                ev_out[2] = {nullptr, nullptr};
    cudaError_t e = cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_done[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming);
    }
    // the staging buffers may still be in use by earlier work on `s`
    if (e == cudaSuccess) e = cudaEventRecord(ev_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sin, ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, ev_start, 0);
    for (int i = 0; i < hp.n && e == cudaSuccess && st == RAMNET_OK; ++i) {
        const int buf = i & 1;
        const int t0 = i * hp.tp, tn = (T - t0) < hp.tp ? (T - t0) : hp.tp;
        // inputs of piece i: B rows of tn*H token-heads each, strided by T*H in the host arrays
        if (i >= 2) e = cudaStreamWaitEvent(sin, ev_done[buf], 0);  // piece i-2 consumed its inputs
        for (int a = 0; a < 5 && e == cudaSuccess; ++a) {
            const size_t w = static_cast<size_t>(tn) * H * row_bytes[a];
            e = cudaMemcpy2DAsync(base + hp.in_off[buf][a], w, static_cast<const unsigned char*>(src[a]) +
                                  static_cast<size_t>(t0) * H * row_bytes[a],
                                  static_cast<size_t>(T) * H * row_bytes[a], w, static_cast<size_t>(B),
                                  cudaMemcpyHostToDevice, sin);
        }
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[buf], sin);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_in[buf], 0);
        if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(s, ev_out[buf], 0);  // y staging of piece i-2 read
        if (e != cudaSuccess) break;
        // piece i on the compute stream; the state is carried in S_out / m_out
        void* ws = base + hp.ws_off;
        const float* Si = i == 0 ? S_in : S_out;
        const float* mi = i == 0 ? m_in : m_out;
        const ramnet::ScanWorkspace wl = ramnet::scan_workspace(B, tn, H, cfg->K, plan);
        st = route_part(cfg, B, tn, H, in_dt, M, plan, wl, base + hp.in_off[buf][0], base + hp.in_off[buf][1],
                        base + hp.in_off[buf][3], cape_mask, pos0, ws, s, t0);
        if (st == RAMNET_OK)
            st = recur_part(cfg, B, tn, H, in_dt, M, plan, wl, base + hp.in_off[buf][2], base + hp.in_off[buf][4],
                            norm_w, Si, mi, base + hp.y_off[buf], out_dt, S_out, m_out, ws, s);
        if (st != RAMNET_OK) break;
        e = cudaEventRecord(ev_done[buf], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, ev_done[buf], 0);
        if (e == cudaSuccess) {
            const size_t w = static_cast<size_t>(tn) * H * cfg->d_v * eo;
            e = cudaMemcpy2DAsync(static_cast<unsigned char*>(y) + static_cast<size_t>(t0) * H * cfg->d_v * eo,
                                  static_cast<size_t>(T) * H * cfg->d_v * eo, base + hp.y_off[buf], w, w,
                                  static_cast<size_t>(B), cudaMemcpyDeviceToHost, sout);
        }
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[buf], sout);
    }
    // the caller's stream ends after the last copy out
    if (e == cudaSuccess && st == RAMNET_OK) {
        for (int b2 = 0; b2 < 2 && e == cudaSuccess; ++b2) e = cudaStreamWaitEvent(s, ev_out[b2], 0);
        for (int b2 = 0; b2 < 2 && e == cudaSuccess; ++b2) e = cudaStreamWaitEvent(s, ev_in[b2], 0);
    }
    // streams and events are released once their work is done
    if (sin) cudaStreamDestroy(sin);
    if (sout) cudaStreamDestroy(sout);
    if (ev_start) cudaEventDestroy(ev_start);
    for (int i = 0; i < 2; ++i) {
        if (ev_in[i]) cudaEventDestroy(ev_in[i]);
        if (ev_done[i]) cudaEventDestroy(ev_done[i]);
        if (ev_out[i]) cudaEventDestroy(ev_out[i]);
    }
    if (st != RAMNET_OK) return st;
    if (e != cudaSuccess) return cuda_fail(e, "scan from host: copies and ordering");
    return RAMNET_OK;
}

}  // extern "C"
