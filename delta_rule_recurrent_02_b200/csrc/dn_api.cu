// dn_api.cu -- the C ABI: argument validation, kernel choice, launch, status.
#include <cuda_runtime.h>
#include <atomic>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "../../include/dn.h"
#include "dn_kernels.h"

namespace {

thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_last_error[0] = '\0';
    return DN_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(DN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Device status word: kernels with bounded waits OR a code into it when they
// give up.  One per device (a module-scope __device__ variable exists once per
// device context).
__device__ unsigned int g_device_status;

unsigned int* status_word(cudaError_t* err) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_device_status);
    return static_cast<unsigned int*>(p);
}

struct Range {
    uintptr_t lo, hi;   // [lo, hi)
    bool valid() const { return lo != 0 && hi > lo; }
};

Range rng(const void* p, int64_t bytes) {
    Range r;
    r.lo = reinterpret_cast<uintptr_t>(p);
    r.hi = r.lo + (uintptr_t)(bytes > 0 ? bytes : 0);
    return r;
}

bool overlap(Range a, Range b) {
    if (!a.valid() || !b.valid()) return false;
    return a.lo < b.hi && b.lo < a.hi;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool supported_d(int d) { return d == 64 || d == 128; }

// Size / enum / path checks shared by dn_chunk_fwd_ex and dn_chunk_fwd_workspace_size.
// Fills the non-pointer fields of *a and the kernel choice.
int plan_chunk(int B, int T, int H, int d_k, int d_v, int chunk, dn_dtype dtype, dn_gate gate, dn_path path,
               dn::ChunkArgs* a, bool* use_tc, const int* cu_seqlens = nullptr, int N = 0) {
    if (B < 0 || T < 0 || H < 0) return fail(DN_ERR_INVALID, "B, T, H must be >= 0 (got %d, %d, %d)", B, T, H);
    if (dtype != DN_F32 && dtype != DN_BF16) return fail(DN_ERR_INVALID, "unknown dtype %d", (int)dtype);
    if (gate != DN_GATE_NONE && gate != DN_GATE_SCALAR && gate != DN_GATE_PER_KEY)
        return fail(DN_ERR_INVALID, "unknown gate %d", (int)gate);
    if (path != DN_PATH_AUTO && path != DN_PATH_SIMT && path != DN_PATH_TC && path != DN_PATH_TC_STALL_TEST)
        return fail(DN_ERR_INVALID, "unknown path %d", (int)path);
    if (d_k <= 0 || d_v <= 0) return fail(DN_ERR_INVALID, "d_k, d_v must be > 0");
    if (chunk <= 0) return fail(DN_ERR_INVALID, "chunk must be > 0 (got %d)", chunk);
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(DN_ERR_UNSUPPORTED, "d_k, d_v must be 64 or 128 (got %d, %d)", d_k, d_v);
    *a = dn::ChunkArgs{};
    a->B = B; a->T = T; a->H = H; a->dk = d_k; a->dv = d_v; a->chunk = chunk;
    a->bf16 = dtype == DN_BF16; a->gate = (int)gate;
    a->test_flags = path == DN_PATH_TC_STALL_TEST ? 1 : 0;
    if (cu_seqlens) {
        // a packed batch: the tensor-core kernels, no gate or the scalar gate
        if (B != 1) return fail(DN_ERR_INVALID, "a packed batch has B = 1 (got %d)", B);
        if (N < 1) return fail(DN_ERR_INVALID, "a packed batch needs N >= 1 sequences (got %d)", N);
        if (path == DN_PATH_SIMT) return fail(DN_ERR_UNSUPPORTED, "packed batches run on the tensor-core path");
        if (gate == DN_GATE_PER_KEY) return fail(DN_ERR_UNSUPPORTED, "packed batches take no gate or the scalar gate");
        a->cu_seqlens = cu_seqlens;
        a->N = N;
        if (!dn::tc_supports(*a))
            return fail(DN_ERR_UNSUPPORTED, "packed batches need bf16, chunk 64 and d_k = d_v = 128");
        *use_tc = true;
        return DN_OK;
    }
    // kernel choice before any CUDA call: an unsupported request touches no device state
    *use_tc = false;
    if (path == DN_PATH_TC || path == DN_PATH_TC_STALL_TEST) {
        if (!dn::tc_supports(*a))
            return fail(DN_ERR_UNSUPPORTED, "tensor-core path needs bf16, chunk 64 and d_k = d_v = 128");
        *use_tc = true;
    } else if (path == DN_PATH_AUTO) {
        *use_tc = dn::tc_supports(*a);
    }
    if (!*use_tc && chunk > 64) return fail(DN_ERR_UNSUPPORTED, "chunk must be <= 64 (got %d)", chunk);
    return DN_OK;
}

size_t workspace_needed(const dn::ChunkArgs& a, bool use_tc) {
    return use_tc && (int64_t)a.B * a.H * a.T > 0 ? dn::tc_workspace_bytes(a) : 0;
}

}  // namespace

namespace dn {
int report_error(int code, const char* msg) { return fail(code, "%s", msg); }

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace dn

extern "C" {

int dn_version(void) { return (2 << 16) | 8; }

unsigned long long dn_kernel_launches(void) { return dn::g_launches.load(std::memory_order_relaxed); }

const char* dn_status_str(int status) {
    switch (status) {
        case DN_OK: return "DN_OK";
        case DN_ERR_INVALID: return "DN_ERR_INVALID: invalid argument";
        case DN_ERR_UNSUPPORTED: return "DN_ERR_UNSUPPORTED: request outside the supported set";
        case DN_ERR_CUDA: return "DN_ERR_CUDA: CUDA call or kernel launch failed";
        case DN_ERR_TIMEOUT: return "DN_ERR_TIMEOUT: a bounded device wait gave up";
        default: return "unknown dn_status";
    }
}

const char* dn_last_error(void) { return g_last_error; }

int dn_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int chunk, dn_dtype dtype, dn_gate gate,
                                dn_path path, size_t* bytes) {
    if (!bytes) return fail(DN_ERR_INVALID, "bytes must not be NULL");
    dn::ChunkArgs a;
    bool use_tc;
    const int st = plan_chunk(B, T, H, d_k, d_v, chunk, dtype, gate, path, &a, &use_tc);
    if (st != DN_OK) return st;
    *bytes = workspace_needed(a, use_tc);
    return ok();
}

static int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* beta,
                    const float* g, const float* S0, void* o, float* S_T,
                    int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                    dn_dtype dtype, dn_gate gate, dn_path path, void* workspace, size_t workspace_bytes,
                    void* cuda_stream, float* snaps, int every, const float* A_log = nullptr,
                    const float* dt_bias = nullptr, int rep = 1, int pro_mul = 1,
                    const int* cu_seqlens = nullptr, int N = 0, int norm = 0, const void* z = nullptr,
                    const float* norm_w = nullptr, float eps = 0.f) {
    dn::ChunkArgs a;
    bool use_tc;
    const int pst = plan_chunk(B, T, H, d_k, d_v, chunk, dtype, gate, path, &a, &use_tc, cu_seqlens, N);
    if (pst != DN_OK) return pst;
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return fail(DN_ERR_INVALID, "scale is not finite");
    const int64_t ntok = (int64_t)B * H * T;
    const int64_t esz = dtype == DN_BF16 ? 2 : 4;
    const bool empty_tokens = ntok == 0;
    if (!empty_tokens && (!q || !k || !v || !beta || !o))
        return fail(DN_ERR_INVALID, "q, k, v, beta and o are required");
    if (gate == DN_GATE_NONE && g) return fail(DN_ERR_INVALID, "g must be NULL when gate is DN_GATE_NONE");
    if (gate != DN_GATE_NONE && !g && !empty_tokens) return fail(DN_ERR_INVALID, "g is required for this gate");
    const void* p16[] = {q, k, v, o, S0, S_T};
    const char* n16[] = {"q", "k", "v", "o", "S0", "S_T"};
    for (int i = 0; i < 6; ++i)
        if (p16[i] && !aligned(p16[i], 16)) return fail(DN_ERR_INVALID, "%s is not 16-byte aligned", n16[i]);
    if ((beta && !aligned(beta, 4)) || (g && !aligned(g, 4)))
        return fail(DN_ERR_INVALID, "beta and g must be 4-byte aligned");
    if (gate == DN_GATE_PER_KEY && g && !aligned(g, 16))
        return fail(DN_ERR_INVALID, "a per-key g must be 16-byte aligned");
    const int64_t gcount = gate == DN_GATE_PER_KEY ? ntok * d_k : ntok;
    // states: per (b, h), or per (sequence, head) of a packed batch
    const int64_t sbytes = (int64_t)(cu_seqlens ? N : B) * H * d_k * d_v * 4;
    if (rep < 1 || H % rep != 0) return fail(DN_ERR_INVALID, "H (%d) must be a multiple of the key heads", H);
    if (rep > 1 && (!use_tc || gate == DN_GATE_PER_KEY))
        return fail(DN_ERR_UNSUPPORTED, "grouped value heads need the tensor-core path and no per-key gate");
    Range rq = rng(q, ntok / rep * d_k * esz), rk = rng(k, ntok / rep * d_k * esz), rv = rng(v, ntok * d_v * esz);
    Range rb = rng(beta, ntok * 4), rg = rng(g, gcount * 4), rs0 = rng(S0, sbytes);
    Range ro = rng(o, ntok * d_v * esz), rst = rng(S_T, sbytes);
    Range ins[] = {rq, rk, rv, rb, rg, rs0};
    for (Range r : ins)
        if (overlap(ro, r) || overlap(ro, rst)) return fail(DN_ERR_INVALID, "o overlaps another argument");
    Range ins2[] = {rq, rk, rv, rb, rg};
    for (Range r : ins2)
        if (overlap(rst, r)) return fail(DN_ERR_INVALID, "S_T overlaps an input other than S0");
    if (S_T && S0 && (void*)S_T != (const void*)S0 && overlap(rst, rs0))
        return fail(DN_ERR_INVALID, "S_T partly overlaps S0");
    if (cu_seqlens) {
        if (snaps || A_log || dt_bias || rep != 1)
            return fail(DN_ERR_UNSUPPORTED, "packed batches take no snapshots, prologue or grouped heads");
        if (!aligned(cu_seqlens, 4)) return fail(DN_ERR_INVALID, "cu_seqlens must be 4-byte aligned");
        Range rcu = rng(cu_seqlens, (int64_t)(N + 1) * 4);
        if (overlap(ro, rcu) || overlap(rst, rcu)) return fail(DN_ERR_INVALID, "o or S_T overlaps cu_seqlens");
    }
    // the layer prologue (dn_chunk_fwd_gdn): beta and g hold the raw b and a
    const bool pro = A_log != nullptr || dt_bias != nullptr;
    Range rpa = rng(A_log, (int64_t)H * 4), rpd = rng(dt_bias, (int64_t)H * 4);
    if (pro) {
        if (!A_log || !dt_bias) return fail(DN_ERR_INVALID, "A_log and dt_bias are both required");
        if (!aligned(A_log, 4) || !aligned(dt_bias, 4)) return fail(DN_ERR_INVALID, "A_log and dt_bias must be 4-byte aligned");
        if (overlap(ro, rpa) || overlap(ro, rpd) || overlap(rst, rpa) || overlap(rst, rpd))
            return fail(DN_ERR_INVALID, "o or S_T overlaps A_log or dt_bias");
    }
    if (norm) {
        // the gated RMSNorm on the output rows: tensor-core path, with the prologue
        if (!pro) return fail(DN_ERR_INVALID, "the gated norm comes with the layer prologue");
        if (!use_tc) return fail(DN_ERR_UNSUPPORTED, "the fused gated norm runs on the tensor-core path");
        if (!z || !norm_w) return fail(DN_ERR_INVALID, "z and norm_weight are both required for the norm");
        if (!(eps > 0.f) || eps > 1.f) return fail(DN_ERR_INVALID, "eps must be in (0, 1]");
        if (!aligned(z, 16) || !aligned(norm_w, 16)) return fail(DN_ERR_INVALID, "z and norm_weight must be 16-byte aligned");
        Range rz = rng(z, ntok * d_v * esz), rw = rng(norm_w, (int64_t)d_v * 4);
        if (overlap(ro, rz) || overlap(ro, rw) || overlap(rst, rz) || overlap(rst, rw))
            return fail(DN_ERR_INVALID, "o or S_T overlaps z or norm_weight");
    }
    // snapshots: the state after every `every` chunks, at full chunk boundaries only
    if (snaps && every < 1) return fail(DN_ERR_INVALID, "every must be >= 1 (got %d)", every);
    const int n_snap = snaps ? (int)(T / ((int64_t)every * chunk)) : 0;
    Range rsn = rng(n_snap > 0 ? snaps : nullptr, (int64_t)B * H * n_snap * d_k * d_v * 4);
    if (n_snap > 0) {
        if (!aligned(snaps, 16)) return fail(DN_ERR_INVALID, "snaps is not 16-byte aligned");
        Range all[] = {rq, rk, rv, rb, rg, rs0, ro, rst};
        for (Range r : all)
            if (overlap(rsn, r)) return fail(DN_ERR_INVALID, "snaps overlaps another argument");
    }
    const size_t need = workspace_needed(a, use_tc);
    if (workspace && need > 0) {
        if (workspace_bytes < need)
            return fail(DN_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes, need);
        if (!aligned(workspace, 256)) return fail(DN_ERR_INVALID, "workspace is not 256-byte aligned");
        Range rw = rng(workspace, (int64_t)need);
        Range rcu = rng(cu_seqlens, (int64_t)(N + 1) * 4);
        Range all[] = {rq, rk, rv, rb, rg, rs0, ro, rst, rsn, rpa, rpd, rcu};
        for (Range r : all)
            if (overlap(rw, r)) return fail(DN_ERR_INVALID, "workspace overlaps another argument");
    }

    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if ((int64_t)B * H == 0) return ok();

    a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.S0 = S0; a.o = o; a.S_T = S_T;
    a.scale = scale;
    a.snaps = n_snap > 0 ? snaps : nullptr;
    a.snap_every = every;
    a.n_snap = n_snap;
    a.rep = rep;
    a.prologue = pro ? pro_mul : 0;
    a.norm = norm; a.z = z; a.norm_weight = norm_w; a.eps = eps;
    a.A_log = A_log;
    a.dt_bias = dt_bias;

    cudaError_t e;
    a.status = status_word(&e);
    if (e != cudaSuccess) return cuda_fail(e, "status word");

    if (T == 0) {   // nothing to read: the final state is the initial one
        if (!S_T) return ok();
        if (S0 && (const void*)S0 != (void*)S_T) e = cudaMemcpyAsync(S_T, S0, sbytes, cudaMemcpyDeviceToDevice, st);
        else if (!S0) e = cudaMemsetAsync(S_T, 0, sbytes, st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "T = 0 state copy");
    }

    if (!use_tc) {
        e = dn::launch_chunk_simt(a, st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "SIMT chunk kernel");
    }
    // the tensor-core path keeps W^T and u^T of every chunk in a workspace: the
    // caller's, else a stream-ordered allocation released on the same stream
    void* own = nullptr;
    if (!workspace) {
        e = cudaMallocAsync(&own, need, st);
        if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    }
    a.ws = workspace ? workspace : own;
    e = dn::launch_chunk_tc(a, st);
    if (own) {
        const cudaError_t ef = cudaFreeAsync(own, st);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? ok() : cuda_fail(e, "tensor-core chunk kernels");
}

int dn_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* beta,
                    const float* g, const float* S0, void* o, float* S_T,
                    int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                    dn_dtype dtype, dn_gate gate, dn_path path, void* workspace, size_t workspace_bytes,
                    void* cuda_stream) {
    return chunk_fwd_impl(q, k, v, beta, g, S0, o, S_T, B, T, H, d_k, d_v, chunk, scale, dtype, gate, path,
                          workspace, workspace_bytes, cuda_stream, nullptr, 0);
}

int dn_chunk_fwd_snapshots(const void* q, const void* k, const void* v, const float* beta,
                           const float* g, const float* S0, void* o, float* S_T, float* snaps, int every,
                           int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                           dn_dtype dtype, dn_gate gate, dn_path path, void* workspace, size_t workspace_bytes,
                           void* cuda_stream) {
    return chunk_fwd_impl(q, k, v, beta, g, S0, o, S_T, B, T, H, d_k, d_v, chunk, scale, dtype, gate, path,
                          workspace, workspace_bytes, cuda_stream, snaps, every);
}

int dn_chunk_fwd_gdn(const void* q, const void* k, const void* v, const float* b, const float* a,
                     const float* A_log, const float* dt_bias, const float* S0, void* o, float* S_T,
                     int B, int T, int H, int d_k, int d_v, float scale,
                     void* workspace, size_t workspace_bytes, void* cuda_stream) {
    if (!A_log || !dt_bias) return fail(DN_ERR_INVALID, "A_log and dt_bias are required");
    return chunk_fwd_impl(q, k, v, b, a, S0, o, S_T, B, T, H, d_k, d_v, 64, scale, DN_BF16, DN_GATE_SCALAR,
                          DN_PATH_TC, workspace, workspace_bytes, cuda_stream, nullptr, 0, A_log, dt_bias);
}

int dn_chunk_fwd_gdn_ex(const void* q, const void* k, const void* v, const float* b, const float* a,
                        const float* A_log, const float* dt_bias, const float* S0, void* o, float* S_T, int B, int T,
                        int H, int d_k, int d_v, int chunk, float scale, dn_dtype dtype, dn_path path, int flags,
                        const void* z, const float* norm_weight, float eps, void* workspace,
                        size_t workspace_bytes, void* cuda_stream) {
    if (!A_log || !dt_bias) return fail(DN_ERR_INVALID, "A_log and dt_bias are required");
    if (flags & ~(DN_GDN_BETA_2SIGMOID | DN_GDN_NORM_SIGMOID))
        return fail(DN_ERR_INVALID, "unknown flags 0x%x", flags);
    if ((flags & DN_GDN_NORM_SIGMOID) && !z) return fail(DN_ERR_INVALID, "DN_GDN_NORM_SIGMOID needs z");
    const int norm = z ? ((flags & DN_GDN_NORM_SIGMOID) ? 2 : 1) : 0;
    return chunk_fwd_impl(q, k, v, b, a, S0, o, S_T, B, T, H, d_k, d_v, chunk, scale, dtype, DN_GATE_SCALAR,
                          path, workspace, workspace_bytes, cuda_stream, nullptr, 0, A_log, dt_bias, 1,
                          flags & DN_GDN_BETA_2SIGMOID ? 2 : 1, nullptr, 0, norm, z, norm_weight, eps);
}

int dn_chunk_fwd(const void* q, const void* k, const void* v, const float* beta,
                 const float* g, const float* S0, void* o, float* S_T,
                 int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                 dn_dtype dtype, dn_gate gate, void* cuda_stream) {
    return dn_chunk_fwd_ex(q, k, v, beta, g, S0, o, S_T, B, T, H, d_k, d_v, chunk, scale,
                           dtype, gate, DN_PATH_AUTO, nullptr, 0, cuda_stream);
}

static int decode_impl(const void* q, const void* k, const void* v, const float* beta,
                       const float* g, float* S, void* o, int B, int H, int d_k, int d_v,
                       float scale, dn_dtype dtype, dn_gate gate, void* cuda_stream,
                       const float* A_log = nullptr, const float* dt_bias = nullptr, int rep = 1,
                       int pro_mul = 1, int norm = 0, const void* z = nullptr, const float* norm_w = nullptr,
                       float eps = 0.f) {
    if (B < 0 || H < 0) return fail(DN_ERR_INVALID, "B, H must be >= 0 (got %d, %d)", B, H);
    if (rep < 1 || H % rep != 0) return fail(DN_ERR_INVALID, "H (%d) must be a multiple of the key heads", H);
    if (dtype != DN_F32 && dtype != DN_BF16) return fail(DN_ERR_INVALID, "unknown dtype %d", (int)dtype);
    if (gate != DN_GATE_NONE && gate != DN_GATE_SCALAR && gate != DN_GATE_PER_KEY)
        return fail(DN_ERR_INVALID, "unknown gate %d", (int)gate);
    if (d_k <= 0 || d_v <= 0) return fail(DN_ERR_INVALID, "d_k, d_v must be > 0");
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return fail(DN_ERR_INVALID, "scale is not finite");
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(DN_ERR_UNSUPPORTED, "d_k, d_v must be 64 or 128 (got %d, %d)", d_k, d_v);
    const int64_t nh = (int64_t)B * H;
    if (nh == 0) return ok();
    if (!q || !k || !v || !beta || !S || !o) return fail(DN_ERR_INVALID, "q, k, v, beta, S and o are required");
    if (gate == DN_GATE_NONE && g) return fail(DN_ERR_INVALID, "g must be NULL when gate is DN_GATE_NONE");
    if (gate != DN_GATE_NONE && !g) return fail(DN_ERR_INVALID, "g is required for this gate");
    const void* p16[] = {q, k, v, o, S};
    const char* n16[] = {"q", "k", "v", "o", "S"};
    for (int i = 0; i < 5; ++i)
        if (!aligned(p16[i], 16)) return fail(DN_ERR_INVALID, "%s is not 16-byte aligned", n16[i]);
    if (!aligned(beta, 4) || (g && !aligned(g, 4))) return fail(DN_ERR_INVALID, "beta and g must be 4-byte aligned");
    if (gate == DN_GATE_PER_KEY && !aligned(g, 16)) return fail(DN_ERR_INVALID, "a per-key g must be 16-byte aligned");
    const int64_t esz = dtype == DN_BF16 ? 2 : 4;
    Range rq = rng(q, nh / rep * d_k * esz), rk = rng(k, nh / rep * d_k * esz), rv = rng(v, nh * d_v * esz);
    Range rb = rng(beta, nh * 4), rg = rng(g, (gate == DN_GATE_PER_KEY ? nh * d_k : nh) * 4);
    Range rs = rng(S, nh * d_k * d_v * 4), ro = rng(o, nh * d_v * esz);
    Range others[] = {rq, rk, rv, rb, rg, rs};
    for (Range r : others)
        if (overlap(ro, r)) return fail(DN_ERR_INVALID, "o overlaps another argument");
    Range ins[] = {rq, rk, rv, rb, rg};
    for (Range r : ins)
        if (overlap(rs, r)) return fail(DN_ERR_INVALID, "S overlaps an input");
    const bool pro = A_log != nullptr;
    if (pro) {
        if (!aligned(A_log, 4) || !aligned(dt_bias, 4)) return fail(DN_ERR_INVALID, "A_log and dt_bias must be 4-byte aligned");
        Range rpa = rng(A_log, (int64_t)H * 4), rpd = rng(dt_bias, (int64_t)H * 4);
        if (overlap(ro, rpa) || overlap(ro, rpd) || overlap(rs, rpa) || overlap(rs, rpd))
            return fail(DN_ERR_INVALID, "o or S overlaps A_log or dt_bias");
    }
    if (norm) {
        // the gated RMSNorm on the output row: z [B, H, d_v] dtype, weight [d_v] fp32
        if (!z || !norm_w) return fail(DN_ERR_INVALID, "z and norm_weight are both required for the norm");
        if (!(eps > 0.f) || eps > 1.f) return fail(DN_ERR_INVALID, "eps must be in (0, 1]");
        if (!aligned(z, 16) || !aligned(norm_w, 16)) return fail(DN_ERR_INVALID, "z and norm_weight must be 16-byte aligned");
        Range rz = rng(z, nh * d_v * esz), rw = rng(norm_w, (int64_t)d_v * 4);
        if (overlap(ro, rz) || overlap(ro, rw) || overlap(rs, rz) || overlap(rs, rw))
            return fail(DN_ERR_INVALID, "o or S overlaps z or norm_weight");
    }

    dn::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.S = S; a.o = o;
    a.B = B; a.H = H; a.dk = d_k; a.dv = d_v; a.scale = scale;
    a.bf16 = dtype == DN_BF16; a.gate = (int)gate;
    a.prologue = pro ? pro_mul : 0; a.A_log = A_log; a.dt_bias = dt_bias;
    a.rep = rep;
    a.norm = norm; a.z = z; a.norm_weight = norm_w; a.eps = eps;
    cudaError_t e = dn::launch_decode_step(a, static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel");
    return ok();
}

int dn_decode_step_gva(const void* q, const void* k, const void* v, const float* beta, const float* g, float* S,
                       void* o, int B, int H_k, int H, int d_k, int d_v, float scale, dn_dtype dtype, dn_gate gate,
                       void* cuda_stream) {
    if (H_k < 1 || H % H_k != 0) return fail(DN_ERR_INVALID, "H (%d) must be a multiple of H_k (%d)", H, H_k);
    return decode_impl(q, k, v, beta, g, S, o, B, H, d_k, d_v, scale, dtype, gate, cuda_stream, nullptr, nullptr,
                       H / H_k);
}

int dn_decode_step(const void* q, const void* k, const void* v, const float* beta,
                   const float* g, float* S, void* o, int B, int H, int d_k, int d_v,
                   float scale, dn_dtype dtype, dn_gate gate, void* cuda_stream) {
    return decode_impl(q, k, v, beta, g, S, o, B, H, d_k, d_v, scale, dtype, gate, cuda_stream);
}

int dn_decode_step_gdn(const void* q, const void* k, const void* v, const float* b, const float* a,
                       const float* A_log, const float* dt_bias, float* S, void* o, int B, int H, int d_k,
                       int d_v, float scale, dn_dtype dtype, void* cuda_stream) {
    if ((int64_t)B * H > 0 && (!A_log || !dt_bias)) return fail(DN_ERR_INVALID, "A_log and dt_bias are required");
    return decode_impl(q, k, v, b, a, S, o, B, H, d_k, d_v, scale, dtype, DN_GATE_SCALAR, cuda_stream, A_log,
                       dt_bias);
}

int dn_decode_step_gdn_ex(const void* q, const void* k, const void* v, const float* b, const float* a,
                          const float* A_log, const float* dt_bias, float* S, void* o, int B, int H, int d_k,
                          int d_v, float scale, dn_dtype dtype, int flags, const void* z, const float* norm_weight,
                          float eps, void* cuda_stream) {
    if ((int64_t)B * H > 0 && (!A_log || !dt_bias)) return fail(DN_ERR_INVALID, "A_log and dt_bias are required");
    if (flags & ~(DN_GDN_BETA_2SIGMOID | DN_GDN_NORM_SIGMOID))
        return fail(DN_ERR_INVALID, "unknown flags 0x%x", flags);
    if ((flags & DN_GDN_NORM_SIGMOID) && !z) return fail(DN_ERR_INVALID, "DN_GDN_NORM_SIGMOID needs z");
    const int norm = z ? ((flags & DN_GDN_NORM_SIGMOID) ? 2 : 1) : 0;
    return decode_impl(q, k, v, b, a, S, o, B, H, d_k, d_v, scale, dtype, DN_GATE_SCALAR, cuda_stream, A_log,
                       dt_bias, 1, flags & DN_GDN_BETA_2SIGMOID ? 2 : 1, norm, z, norm_weight, eps);
}

int dn_causal_conv1d(const void* x, int ld_x, const float* weight, const void* state_in, void* y,
                     void* state_out, int B, int T, int C, int K, int head_dim, int activation, dn_dtype dtype,
                     void* cuda_stream) {
    if (B < 0 || T < 0 || C < 0) return fail(DN_ERR_INVALID, "B, T, C must be >= 0 (got %d, %d, %d)", B, T, C);
    if (dtype != DN_F32 && dtype != DN_BF16) return fail(DN_ERR_INVALID, "unknown dtype %d", (int)dtype);
    if (K < 1 || K > 4) return fail(DN_ERR_UNSUPPORTED, "K must be 1..4 (got %d)", K);
    if (activation != 0 && activation != 1) return fail(DN_ERR_INVALID, "activation must be 0 or 1");
    if (B == 0 || C == 0) return ok();
    if (ld_x < C) return fail(DN_ERR_INVALID, "ld_x (%d) must be >= C (%d)", ld_x, C);
    if (head_dim <= 0 || C % head_dim != 0) return fail(DN_ERR_INVALID, "head_dim (%d) must divide C (%d)", head_dim, C);
    if (B > 65535 || T > 16 * 65535) return fail(DN_ERR_UNSUPPORTED, "B <= 65535 and T <= 1048560 (got %d, %d)", B, T);
    if (!weight || (T > 0 && (!x || !y))) return fail(DN_ERR_INVALID, "x, weight and y are required");
    const int64_t esz = dtype == DN_BF16 ? 2 : 4;
    const void* pe[] = {x, y, state_in, state_out};
    for (const void* p : pe)
        if (p && !aligned(p, (uintptr_t)esz)) return fail(DN_ERR_INVALID, "x, y and the states must be %d-byte aligned", (int)esz);
    if (!aligned(weight, 4)) return fail(DN_ERR_INVALID, "weight must be 4-byte aligned");
    const int64_t nst = (int64_t)B * (K - 1) * C * esz;
    Range rx = rng(x, T > 0 ? ((int64_t)B * T - 1) * ld_x * esz + (int64_t)C * esz : 0);
    Range rw = rng(weight, (int64_t)C * K * 4), ry = rng(y, (int64_t)B * T * C * esz);
    Range rsi = rng(state_in, K > 1 ? nst : 0), rso = rng(state_out, K > 1 ? nst : 0);
    if (overlap(ry, rx) || overlap(ry, rw) || overlap(ry, rsi) || overlap(ry, rso))
        return fail(DN_ERR_INVALID, "y overlaps another argument");
    if (overlap(rso, rx) || overlap(rso, rw)) return fail(DN_ERR_INVALID, "state_out overlaps x or weight");
    if (overlap(rso, rsi) && !(state_out == state_in && T <= 16))
        return fail(DN_ERR_INVALID, "state_out may be state_in itself only when T <= 16; otherwise it must not overlap it");
    const int V = (int)(8 / esz);     // channels per 8-byte access
    bool vec = C % V == 0 && ld_x % V == 0 && head_dim % V == 0;
    bool vec16 = C % (2 * V) == 0 && ld_x % (2 * V) == 0 && head_dim % (2 * V) == 0;
    for (const void* p : pe) {
        if (p && !aligned(p, 8)) vec = false;
        if (p && !aligned(p, 16)) vec16 = false;
    }
    if (!aligned(weight, 16)) vec16 = false;
    dn::ConvArgs a;
    a.x = x; a.ld_x = ld_x; a.weight = weight; a.state_in = state_in; a.y = y; a.state_out = state_out;
    a.B = B; a.T = T; a.C = C; a.K = K; a.head_dim = head_dim;
    a.activation = activation == 1; a.bf16 = dtype == DN_BF16; a.vec = vec; a.vec16 = vec16;
    if (T == 0 && (!state_out || K == 1)) return ok();
    cudaError_t e = dn::launch_causal_conv1d(a, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "causal conv kernel");
}

int dn_rms_norm_gated(const void* x, const void* z, const float* weight, void* y, int B, int T, int H, int D,
                      float eps, int x_head_major, int activation, dn_dtype dtype, void* cuda_stream) {
    if (B < 0 || T < 0 || H < 0) return fail(DN_ERR_INVALID, "B, T, H must be >= 0 (got %d, %d, %d)", B, T, H);
    if (dtype != DN_F32 && dtype != DN_BF16) return fail(DN_ERR_INVALID, "unknown dtype %d", (int)dtype);
    if (D != 64 && D != 128 && D != 256) return fail(DN_ERR_UNSUPPORTED, "D must be 64, 128 or 256 (got %d)", D);
    if (!(eps >= 0.f) || eps > 3.0e38f) return fail(DN_ERR_INVALID, "eps must be finite and >= 0");
    if (activation != 0 && activation != 1) return fail(DN_ERR_INVALID, "activation must be 0 or 1");
    if (x_head_major != 0 && x_head_major != 1) return fail(DN_ERR_INVALID, "x_head_major must be 0 or 1");
    const int64_t rows = (int64_t)B * T * H;
    if (rows == 0) return ok();
    if (!x || !z || !weight || !y) return fail(DN_ERR_INVALID, "x, z, weight and y are required");
    if (!aligned(x, 16) || !aligned(z, 16) || !aligned(y, 16)) return fail(DN_ERR_INVALID, "x, z and y must be 16-byte aligned");
    if (!aligned(weight, 4)) return fail(DN_ERR_INVALID, "weight must be 4-byte aligned");
    const int64_t esz = dtype == DN_BF16 ? 2 : 4;
    Range rx = rng(x, rows * D * esz), rz = rng(z, rows * D * esz), ry = rng(y, rows * D * esz);
    Range rw = rng(weight, (int64_t)D * 4);
    if (overlap(ry, rx) || overlap(ry, rz) || overlap(ry, rw)) return fail(DN_ERR_INVALID, "y overlaps another argument");
    dn::NormArgs a;
    a.x = x; a.z = z; a.weight = weight; a.y = y; a.B = B; a.T = T; a.H = H; a.D = D; a.eps = eps;
    a.silu = activation == 1; a.x_head_major = x_head_major == 1; a.bf16 = dtype == DN_BF16;
    cudaError_t e = dn::launch_rms_norm_gated(a, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "gated RMSNorm kernel");
}

int dn_chunk_fwd_gva(const void* q, const void* k, const void* v, const float* beta, const float* g,
                     const float* S0, void* o, float* S_T, int B, int T, int H_k, int H, int d_k, int d_v,
                     float scale, dn_dtype dtype, dn_gate gate, void* workspace, size_t workspace_bytes,
                     void* cuda_stream) {
    if (H_k < 1 || H % H_k != 0) return fail(DN_ERR_INVALID, "H (%d) must be a multiple of H_k (%d)", H, H_k);
    return chunk_fwd_impl(q, k, v, beta, g, S0, o, S_T, B, T, H, d_k, d_v, 64, scale, dtype, gate, DN_PATH_TC,
                          workspace, workspace_bytes, cuda_stream, nullptr, 1, nullptr, nullptr, H / H_k);
}

int dn_chunk_fwd_varlen_workspace_size(int N, int T, int H, int d_k, int d_v, dn_dtype dtype, dn_gate gate,
                                       size_t* bytes) {
    if (!bytes) return fail(DN_ERR_INVALID, "bytes must not be NULL");
    dn::ChunkArgs a;
    bool use_tc;
    static const int kAnyCu = 0;   // stands for the device array: only its presence matters here
    const int st = plan_chunk(1, T, H, d_k, d_v, 64, dtype, gate, DN_PATH_AUTO, &a, &use_tc, &kAnyCu, N);
    if (st != DN_OK) return st;
    *bytes = workspace_needed(a, use_tc);
    return ok();
}

int dn_chunk_fwd_varlen(const void* q, const void* k, const void* v, const float* beta, const float* g,
                        const float* S0, void* o, float* S_T, const int* cu_seqlens, int N, int T, int H,
                        int d_k, int d_v, float scale, dn_dtype dtype, dn_gate gate, void* workspace,
                        size_t workspace_bytes, void* cuda_stream) {
    if (!cu_seqlens) return fail(DN_ERR_INVALID, "cu_seqlens is required");
    return chunk_fwd_impl(q, k, v, beta, g, S0, o, S_T, 1, T, H, d_k, d_v, 64, scale, dtype, gate, DN_PATH_AUTO,
                          workspace, workspace_bytes, cuda_stream, nullptr, 0, nullptr, nullptr, 1, 1, cu_seqlens,
                          N);
}

int dn_chunk_fwd_general(const void* q, const float* w_log, const void* kappa, const float* a, const void* k,
                         const void* v, const float* S0, void* o, float* S_T, int B, int T, int H, int d_k, int d_v,
                         int chunk, float scale, dn_dtype dtype, void* cuda_stream) {
    if (B < 0 || T < 0 || H < 0) return fail(DN_ERR_INVALID, "B, T, H must be >= 0 (got %d, %d, %d)", B, T, H);
    if (dtype != DN_F32 && dtype != DN_BF16) return fail(DN_ERR_INVALID, "unknown dtype %d", (int)dtype);
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return fail(DN_ERR_INVALID, "scale is not finite");
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(DN_ERR_UNSUPPORTED, "d_k, d_v must be 64 or 128 (got %d, %d)", d_k, d_v);
    if (chunk < 1 || chunk > dn::general_max_chunk())
        return fail(DN_ERR_UNSUPPORTED, "chunk must be 1..%d (got %d)", dn::general_max_chunk(), chunk);
    const int64_t ntok = (int64_t)B * H * T;
    if (ntok > 0 && (!q || !w_log || !kappa || !a || !k || !v || !o))
        return fail(DN_ERR_INVALID, "q, w_log, kappa, a, k, v and o are required");
    const int64_t esz = dtype == DN_BF16 ? 2 : 4;
    const void* p16[] = {q, kappa, k, v, o, S0, S_T};
    const char* n16[] = {"q", "kappa", "k", "v", "o", "S0", "S_T"};
    for (int i = 0; i < 7; ++i)
        if (p16[i] && !aligned(p16[i], 16)) return fail(DN_ERR_INVALID, "%s is not 16-byte aligned", n16[i]);
    if ((w_log && !aligned(w_log, 4)) || (a && !aligned(a, 4)))
        return fail(DN_ERR_INVALID, "w_log and a must be 4-byte aligned");
    const int64_t sbytes = (int64_t)B * H * d_k * d_v * 4;
    Range rq = rng(q, ntok * d_k * esz), rw = rng(w_log, ntok * d_k * 4), rkp = rng(kappa, ntok * d_k * esz);
    Range ra = rng(a, ntok * d_k * 4), rk = rng(k, ntok * d_k * esz), rv = rng(v, ntok * d_v * esz);
    Range rs0 = rng(S0, sbytes), ro = rng(o, ntok * d_v * esz), rst = rng(S_T, sbytes);
    Range ins[] = {rq, rw, rkp, ra, rk, rv, rs0};
    for (Range r : ins)
        if (overlap(ro, r) || overlap(ro, rst)) return fail(DN_ERR_INVALID, "o overlaps another argument");
    Range ins2[] = {rq, rw, rkp, ra, rk, rv};
    for (Range r : ins2)
        if (overlap(rst, r)) return fail(DN_ERR_INVALID, "S_T overlaps an input other than S0");
    if (S_T && S0 && (void*)S_T != (const void*)S0 && overlap(rst, rs0))
        return fail(DN_ERR_INVALID, "S_T partly overlaps S0");
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if ((int64_t)B * H == 0) return ok();
    cudaError_t e;
    if (T == 0) {
        if (!S_T) return ok();
        if (S0 && (const void*)S0 != (void*)S_T) e = cudaMemcpyAsync(S_T, S0, sbytes, cudaMemcpyDeviceToDevice, st);
        else if (!S0) e = cudaMemsetAsync(S_T, 0, sbytes, st);
        else e = cudaSuccess;
        return e == cudaSuccess ? ok() : cuda_fail(e, "T = 0 state copy");
    }
    dn::GeneralArgs ga{q, w_log, kappa, a, k, v, S0, o, S_T, B, T, H, d_k, d_v, chunk, scale, dtype == DN_BF16};
    e = dn::launch_chunk_general(ga, st);
    return e == cudaSuccess ? ok() : cuda_fail(e, "generalised-rule chunk kernel");
}

int dn_device_status(void* cuda_stream) {
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int word = 0;
    e = cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "read status word");
    if (word != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clear status word");
        if (word & 2u)
            return fail(DN_ERR_INVALID, "cu_seqlens did not rise from 0 to T: nothing was computed (status 0x%x)",
                        word);
        return fail(DN_ERR_TIMEOUT, "a kernel gave up on a bounded wait (status 0x%x)", word);
    }
    return ok();
}

}  // extern "C"
