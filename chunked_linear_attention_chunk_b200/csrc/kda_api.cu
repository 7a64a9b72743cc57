// kda_api.cu -- the extern "C" boundary of libkda: argument validation, aliasing
// checks, workspace sizing and dispatch to the kernels.  See include/kda.h for the
// contract of every entry point.
#include <cmath>
#include <cstring>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

__device__ unsigned int g_device_status = 0;

int num_sms()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return 148;
    if (dev < 64 && cache[dev] > 0)
        return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64)
        cache[dev] = n;
    return n;
}

// Looked up on every launch (it allocates nothing): a cached address could outlive the
// context it belongs to (cudaDeviceReset, another context made current on the device).
unsigned int *device_status_ptr()
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess)
        return nullptr;
    return static_cast<unsigned int *>(p);
}

namespace {

constexpr int64_t kMaxElems = (int64_t)1 << 40;
constexpr int kMaxPackedTokens = 0x7fffffff - 64;  // packed axis; cu_seqlens are int32

struct Range {
    uintptr_t lo = 0, hi = 0;  // [lo, hi)
    Range() = default;
    Range(const void *p, int64_t bytes) : lo((uintptr_t)p), hi((uintptr_t)p + (uintptr_t)(bytes > 0 ? bytes : 0)) {}
    bool empty() const { return lo == 0 || hi <= lo; }
};

bool overlaps(const Range &x, const Range &y)
{
    if (x.empty() || y.empty())
        return false;
    return x.lo < y.hi && y.lo < x.hi;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// beta is read one element at a time: its natural alignment is enough.
bool beta_aligned(const void *beta, int es) { return ((uintptr_t)beta % (uintptr_t)es) == 0; }

int elem_size(kda_dtype dt) { return dt == KDA_BF16 ? 2 : 4; }

bool dtype_ok(kda_dtype dt) { return dt == KDA_BF16 || dt == KDA_F32; }

kda_status check_gmin(float g_min)
{
    if (!std::isfinite(g_min) || !(g_min < 0.0f))
        return KDA_ERR_INVALID_ARG;
    if (g_min < KDA_G_MIN_LOWEST)
        return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Product of non-negative ints with an overflow bound; -1 when it exceeds kMaxElems.
int64_t safe_prod(std::initializer_list<int64_t> xs)
{
    int64_t p = 1;
    for (int64_t x : xs) {
        if (x < 0)
            return -1;
        if (x != 0 && p > kMaxElems / x)
            return -1;
        p *= x;
    }
    return p;
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

int kda_version(void) { return 100; }

const char *kda_status_string(kda_status s)
{
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT";
    case KDA_ERR_ALIAS: return "KDA_ERR_ALIAS";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
    case KDA_ERR_DEVICE_BOUNDS: return "KDA_ERR_DEVICE_BOUNDS";
    }
    return "KDA_ERR_UNKNOWN";
}

kda_status kda_gate_fwd(const void *a, kda_dtype a_dtype, float g_min, float *g, int64_t n, kda_stream_t stream)
{
    if (!dtype_ok(a_dtype) || n < 0 || n > kMaxElems)
        return KDA_ERR_INVALID_ARG;
    kda_status st = check_gmin(g_min);
    if (st != KDA_OK)
        return st;
    if (n == 0)
        return KDA_OK;
    if (!a || !g)
        return KDA_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(g))
        return KDA_ERR_ALIGNMENT;
    if (overlaps(Range(a, n * elem_size(a_dtype)), Range(g, n * 4)))
        return KDA_ERR_ALIAS;
    return from_cuda(launch_gate(a, a_dtype, (double)g_min, g, n, (cudaStream_t)stream));
}

kda_status kda_gate_fwd_heads(const void *a, kda_dtype a_dtype, float g_min, const float *A_log, int64_t n_tok,
                              int H, int dk, float *g, kda_stream_t stream)
{
    if (!dtype_ok(a_dtype) || n_tok < 0 || H < 1 || dk < 1)
        return KDA_ERR_INVALID_ARG;
    kda_status st = check_gmin(g_min);
    if (st != KDA_OK)
        return st;
    if (dk % 8 != 0)
        return KDA_ERR_UNSUPPORTED;
    const int64_t n = safe_prod({n_tok, H, dk});
    if (n < 0)
        return KDA_ERR_INVALID_ARG;
    if (n == 0)
        return KDA_OK;
    if (!a || !g || !A_log)
        return KDA_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(g) || ((uintptr_t)A_log & 3u))
        return KDA_ERR_ALIGNMENT;
    const Range rg(g, n * 4);
    if (overlaps(rg, Range(a, n * elem_size(a_dtype))) || overlaps(rg, Range(A_log, (int64_t)H * 4)))
        return KDA_ERR_ALIAS;
    return from_cuda(launch_gate_heads(a, a_dtype, (double)g_min, A_log, n_tok, H, dk, g, (cudaStream_t)stream));
}

size_t kda_chunk_fwd_workspace(int B, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (B < 1 || H < 1 || T < 0 || dk != dv || (dk != 64 && dk != 128) || !dtype_ok(dtype))
        return 0;
    if (dtype != KDA_BF16 || T == 0)
        return 0;
    return chunk_bf16_workspace(B, T, H, dk);
}

}  // extern "C"

namespace {

// Sizes of one chunk-forward call, checked once.
struct ChunkShape {
    int B = 0, T = 0, H = 0, D = 0;
    kda_dtype dtype = KDA_BF16;
    int64_t ntok = 0, nk = 0, nv = 0, ns = 0;
    size_t ws = 0;  // workspace bytes kda_chunk_fwd_workspace reports
    int es = 2;     // element size of the token tensors
};

kda_status check_shape(int B, int T, int H, int dk, int dv, kda_dtype dtype, ChunkShape &sh)
{
    if (!dtype_ok(dtype) || B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1)
        return KDA_ERR_INVALID_ARG;
    if (dk != dv || (dk != 64 && dk != 128))
        return KDA_ERR_UNSUPPORTED;
    sh.ntok = safe_prod({B, T, H});
    sh.nk = safe_prod({B, T, H, dk});
    sh.nv = safe_prod({B, T, H, dv});
    sh.ns = safe_prod({B, H, dk, dv});
    if (sh.ntok < 0 || sh.nk < 0 || sh.nv < 0 || sh.ns < 0)
        return KDA_ERR_INVALID_ARG;
    if (dtype == KDA_BF16 && (int64_t)B * H > 65535)
        return KDA_ERR_UNSUPPORTED;
    sh.B = B, sh.T = T, sh.H = H, sh.D = dk, sh.dtype = dtype;
    sh.ws = kda_chunk_fwd_workspace(B, T, H, dk, dv, dtype);
    sh.es = elem_size(dtype);
    return KDA_OK;
}

kda_status check_gate(kda_gate gate, float g_min, kda_dtype dtype)
{
    if (gate == KDA_GATE_BOUNDED)
        return check_gmin(g_min);
    if (gate == KDA_GATE_LOGSIGMOID)
        return dtype == KDA_BF16 ? KDA_OK : KDA_ERR_UNSUPPORTED;
    return KDA_ERR_INVALID_ARG;
}

bool all_aligned(std::initializer_list<const void *> ps)
{
    for (const void *p : ps)
        if (p && !aligned16(p))
            return false;
    return true;
}

kda_status check_workspace(const ChunkShape &sh, const void *workspace, size_t ws_bytes)
{
    if (sh.ws > 0 && (!workspace || ws_bytes < sh.ws))
        return KDA_ERR_WORKSPACE;
    return KDA_OK;
}

// The inputs of the prep: q, k, v, a, beta present (T > 0), aligned, and not overlapped by
// the workspace it writes.
kda_status check_prep_args(const ChunkShape &sh, const void *q, const void *k, const void *v, const void *a,
                           const void *beta, const void *workspace, size_t ws_bytes)
{
    if (sh.T > 0 && (!q || !k || !v || !a || !beta))
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, a, workspace}) || !beta_aligned(beta, sh.es))
        return KDA_ERR_ALIGNMENT;
    kda_status st = check_workspace(sh, workspace, ws_bytes);
    if (st != KDA_OK)
        return st;
    const Range rws(sh.ws > 0 ? workspace : nullptr, (int64_t)sh.ws);
    const int es = sh.es;
    for (const Range &in : {Range(q, sh.nk * es), Range(k, sh.nk * es), Range(v, sh.nv * es), Range(a, sh.nk * es),
                            Range(beta, sh.ntok * es)})
        if (overlaps(rws, in))
            return KDA_ERR_ALIAS;
    return KDA_OK;
}

// The outputs of the scan: o present (T > 0) and overlapping nothing else; S_T either S0
// itself or disjoint from it, and disjoint from the workspace; S0 disjoint from the
// workspace.
kda_status check_scan_args(const ChunkShape &sh, const void *workspace, size_t ws_bytes, const float *S0, void *o,
                           float *S_T)
{
    if (sh.T > 0 && !o)
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({workspace, S0, o, S_T}))
        return KDA_ERR_ALIGNMENT;
    kda_status st = check_workspace(sh, workspace, ws_bytes);
    if (st != KDA_OK)
        return st;
    const Range rws(sh.ws > 0 ? workspace : nullptr, (int64_t)sh.ws);
    const Range rS0(S0, sh.ns * 4), ro(sh.T > 0 ? o : nullptr, sh.nv * sh.es), rST(S_T, sh.ns * 4);
    for (const Range &r : {rS0, rST, rws})
        if (overlaps(ro, r))
            return KDA_ERR_ALIAS;
    if (overlaps(rST, rws) || overlaps(rS0, rws))
        return KDA_ERR_ALIAS;
    if (overlaps(rST, rS0) && S_T != S0)
        return KDA_ERR_ALIAS;
    return KDA_OK;
}

// T == 0: the final state is the initial one.
kda_status copy_state(const ChunkShape &sh, const float *S0, float *S_T, cudaStream_t s)
{
    if (!S_T || S_T == S0)
        return KDA_OK;
    if (S0)
        return from_cuda(cudaMemcpyAsync(S_T, S0, (size_t)sh.ns * 4, cudaMemcpyDeviceToDevice, s));
    return from_cuda(cudaMemsetAsync(S_T, 0, (size_t)sh.ns * 4, s));
}

}  // namespace

namespace kda {

// Every check of one chunk-forward problem (shape, gate, alignment, aliasing and, when
// `check_ws` is set, the workspace size), done once on the whole problem before anything is
// launched.  Shared by kda_chunk_fwd, kda_chunk_fwd_logsigmoid and kda_chunk_fwd_noalloc.
kda_status validate_chunk_fwd(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                              const void *v, const void *a, const void *beta, float g_min, kda_gate gate,
                              const float *S0, const void *o, const float *S_T, const void *workspace,
                              size_t ws_bytes, bool check_ws)
{
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, dtype, sh);
    if (st == KDA_OK)
        st = check_gate(gate, g_min, dtype);
    if (st != KDA_OK)
        return st;
    if (!check_ws) {  // the caller supplies its own scratch; only the overlap checks use the range
        sh.ws = workspace ? ws_bytes : 0;
        ws_bytes = sh.ws;
    }
    st = check_prep_args(sh, q, k, v, a, beta, workspace, ws_bytes);
    if (st == KDA_OK)
        st = check_scan_args(sh, workspace, ws_bytes, S0, const_cast<void *>(o), const_cast<float *>(S_T));
    if (st != KDA_OK)
        return st;
    // the outputs must not overlap the inputs either
    const int es = sh.es;
    const Range ro(T > 0 ? o : nullptr, sh.nv * es), rST(S_T, sh.ns * 4);
    for (const Range &in : {Range(q, sh.nk * es), Range(k, sh.nk * es), Range(v, sh.nv * es), Range(a, sh.nk * es),
                            Range(beta, sh.ntok * es)})
        if (overlaps(ro, in) || overlaps(rST, in))
            return KDA_ERR_ALIAS;
    return KDA_OK;
}

// The launches of one validated chunk-forward problem.
kda_status dispatch_chunk_fwd(int B, int T, int H, int dk, kda_dtype dtype, const void *q, const void *k,
                              const void *v, const void *a, const void *beta, float g_min, kda_gate gate,
                              const float *S0, void *o, float *S_T, void *workspace, cudaStream_t s)
{
    if (T == 0) {
        ChunkShape sh;
        sh.ns = (int64_t)B * H * dk * dk;
        return copy_state(sh, S0, S_T, s);
    }
    if (dtype == KDA_F32)
        return from_cuda(launch_chunk_f32(B, T, H, dk, static_cast<const float *>(q), static_cast<const float *>(k),
                                          static_cast<const float *>(v), static_cast<const float *>(a),
                                          static_cast<const float *>(beta), g_min, S0, static_cast<float *>(o), S_T,
                                          s));
    kda_status st = from_cuda(
        launch_prep_bf16(B, T, H, dk, q, k, v, a, beta, g_min, gate == KDA_GATE_LOGSIGMOID, nullptr, workspace, s));
    if (st != KDA_OK)
        return st;
    return from_cuda(launch_scan_bf16(B, T, H, dk, workspace, S0, o, S_T, s));
}

}  // namespace kda

namespace {

// Validation and dispatch shared by kda_chunk_fwd and kda_chunk_fwd_logsigmoid.
kda_status chunk_fwd_impl(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                          const void *v, const void *a, const void *beta, float g_min, kda_gate gate,
                          const float *S0, void *o, float *S_T, void *workspace, size_t ws_bytes,
                          kda_stream_t stream)
{
    const kda_status st = validate_chunk_fwd(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, gate, S0, o, S_T,
                                             workspace, ws_bytes, true);
    if (st != KDA_OK)
        return st;
    return dispatch_chunk_fwd(B, T, H, dk, dtype, q, k, v, a, beta, g_min, gate, S0, o, S_T, workspace,
                              (cudaStream_t)stream);
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                         const void *v, const void *a, const void *beta, float g_min, const float *S0, void *o,
                         float *S_T, void *workspace, size_t ws_bytes, kda_stream_t stream)
{
    return chunk_fwd_impl(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, KDA_GATE_BOUNDED, S0, o, S_T, workspace,
                          ws_bytes, stream);
}

kda_status kda_chunk_fwd_logsigmoid(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q,
                                    const void *k, const void *v, const void *a, const void *beta, const float *S0,
                                    void *o, float *S_T, void *workspace, size_t ws_bytes, kda_stream_t stream)
{
    return chunk_fwd_impl(B, T, H, dk, dv, dtype, q, k, v, a, beta, 0.0f, KDA_GATE_LOGSIGMOID, S0, o, S_T,
                          workspace, ws_bytes, stream);
}

size_t kda_chunk_fwd_varlen_workspace(int N, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (N < 1 || T < 0 || T > kMaxPackedTokens || H < 1 || dk != dv || (dk != 64 && dk != 128) || dtype != KDA_BF16)
        return 0;
    return chunk_bf16_varlen_workspace(N, T, H, dk);
}

kda_status kda_chunk_fwd_varlen(int N, const int32_t *cu_seqlens, int T, int H, int dk, int dv, kda_dtype dtype,
                                kda_gate gate, float g_min, const float *A_log, const void *q, const void *k,
                                const void *v, const void *a, const void *beta, const float *S0, void *o,
                                float *S_T, void *workspace, size_t ws_bytes, kda_stream_t stream)
{
    if (!dtype_ok(dtype) || N < 1 || H < 1 || T < 0 || dk < 1 || dv < 1)
        return KDA_ERR_INVALID_ARG;
    kda_status st = check_gate(gate, g_min, KDA_BF16);
    if (st != KDA_OK)
        return st;
    if (dk != dv || (dk != 64 && dk != 128) || dtype != KDA_BF16 || T > kMaxPackedTokens || (int64_t)N * H > 65535)
        return KDA_ERR_UNSUPPORTED;
    const int64_t nk = (int64_t)T * H * dk, ntok = (int64_t)T * H, ns = (int64_t)N * H * dk * dv;
    if (!cu_seqlens || (T > 0 && (!q || !k || !v || !a || !beta || !o)))
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, a, S0, o, S_T, workspace}) || !beta_aligned(beta, 2) || ((uintptr_t)cu_seqlens & 3u) ||
        ((uintptr_t)A_log & 3u))
        return KDA_ERR_ALIGNMENT;
    const size_t need = kda_chunk_fwd_varlen_workspace(N, T, H, dk, dv, dtype);
    if (!workspace || ws_bytes < need)
        return KDA_ERR_WORKSPACE;
    const Range rq(q, nk * 2), rk(k, nk * 2), rv(v, nk * 2), ra(a, nk * 2), rb(beta, ntok * 2),
        rcu(cu_seqlens, (int64_t)(N + 1) * 4), rS0(S0, ns * 4), ro(T > 0 ? o : nullptr, nk * 2), rST(S_T, ns * 4),
        rws(workspace, (int64_t)need), rA(A_log, (int64_t)H * 4);
    for (const Range &in : {rq, rk, rv, ra, rb, rcu, rA, rS0, rST, rws})
        if (overlaps(ro, in))
            return KDA_ERR_ALIAS;
    for (const Range &in : {rq, rk, rv, ra, rb, rcu, rA, rws})
        if (overlaps(rST, in))
            return KDA_ERR_ALIAS;
    if (overlaps(rST, rS0) && S_T != S0)
        return KDA_ERR_ALIAS;
    for (const Range &in : {rq, rk, rv, ra, rb, rcu, rA, rS0})
        if (overlaps(rws, in))
            return KDA_ERR_ALIAS;
    return from_cuda(launch_chunk_bf16_varlen(N, cu_seqlens, T, H, dk, q, k, v, a, beta, g_min,
                                              gate == KDA_GATE_LOGSIGMOID, A_log, S0, o, S_T, workspace,
                                              (cudaStream_t)stream));
}

kda_status kda_chunk_fwd_scan_affine(int B, int T, int H, int dk, int dv, const void *workspace, size_t ws_bytes,
                                     float *S_zero, float *M, kda_stream_t stream)
{
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, KDA_BF16, sh);
    if (st != KDA_OK)
        return st;
    if (!S_zero || !M)
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({workspace, S_zero, M}))
        return KDA_ERR_ALIGNMENT;
    if ((st = check_workspace(sh, workspace, ws_bytes)) != KDA_OK)
        return st;
    const Range rws(sh.ws > 0 ? workspace : nullptr, (int64_t)sh.ws), rz(S_zero, sh.ns * 4), rm(M, sh.ns * 4);
    if (overlaps(rz, rm) || overlaps(rz, rws) || overlaps(rm, rws))
        return KDA_ERR_ALIAS;
    return from_cuda(launch_scan_affine_bf16(B, T, H, dk, workspace, S_zero, M, (cudaStream_t)stream));
}

kda_status kda_state_combine(int R, int B, int H, int dk, int dv, const float *M, const float *S_zero,
                             const float *S0, float *S_in, kda_stream_t stream)
{
    if (R < 0 || B < 1 || H < 1 || dk < 1 || dv < 1)
        return KDA_ERR_INVALID_ARG;
    if (dk != dv || (dk != 64 && dk != 128) || (int64_t)B * H > 65535)
        return KDA_ERR_UNSUPPORTED;
    const int64_t per = safe_prod({B, H, dk, dv});
    if (per < 0 || safe_prod({R + 1, per}) < 0)
        return KDA_ERR_INVALID_ARG;
    if (!S_in || (R > 0 && (!M || !S_zero)))
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({M, S_zero, S0, S_in}))
        return KDA_ERR_ALIGNMENT;
    const Range rin(S_in, (R + 1) * per * 4);
    for (const Range &x : {Range(M, R * per * 4), Range(S_zero, R * per * 4), Range(S0, per * 4)})
        if (overlaps(rin, x))
            return KDA_ERR_ALIAS;
    return from_cuda(launch_combine(R, B * H, dk, M, S_zero, S0, S_in, (cudaStream_t)stream));
}

kda_status kda_chunk_fwd_prep(int B, int T, int H, int dk, int dv, kda_gate gate, float g_min, const float *A_log,
                              const void *q, const void *k, const void *v, const void *a, const void *beta,
                              void *workspace, size_t ws_bytes, kda_stream_t stream)
{
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, KDA_BF16, sh);
    if (st == KDA_OK)
        st = check_gate(gate, g_min, KDA_BF16);
    if (st == KDA_OK)
        st = check_prep_args(sh, q, k, v, a, beta, workspace, ws_bytes);
    if (st == KDA_OK && ((uintptr_t)A_log & 3u))
        st = KDA_ERR_ALIGNMENT;
    if (st == KDA_OK && sh.ws > 0 && overlaps(Range(workspace, (int64_t)sh.ws), Range(A_log, (int64_t)H * 4)))
        st = KDA_ERR_ALIAS;
    if (st != KDA_OK || T == 0)
        return st;
    return from_cuda(launch_prep_bf16(B, T, H, dk, q, k, v, a, beta, g_min, gate == KDA_GATE_LOGSIGMOID, A_log,
                                      workspace, (cudaStream_t)stream));
}

kda_status kda_chunk_fwd_scan(int B, int T, int H, int dk, int dv, const void *workspace, size_t ws_bytes,
                              const float *S0, void *o, float *S_T, kda_stream_t stream)
{
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, KDA_BF16, sh);
    if (st == KDA_OK)
        st = check_scan_args(sh, workspace, ws_bytes, S0, o, S_T);
    if (st != KDA_OK)
        return st;
    if (T == 0)
        return copy_state(sh, S0, S_T, (cudaStream_t)stream);
    return from_cuda(launch_scan_bf16(B, T, H, dk, workspace, S0, o, S_T, (cudaStream_t)stream));
}

// Two stretches' records, each slot rounded up to 256 bytes.
size_t kda_chunk_fwd_segmented_workspace(int B, int T, int H, int dk, int dv, int seg_T)
{
    if (seg_T < KDA_CHUNK || seg_T % KDA_CHUNK != 0 || T < 0)
        return 0;
    const size_t slot = kda_chunk_fwd_workspace(1, T < seg_T ? T : seg_T, H, dk, dv, KDA_BF16);
    if (B < 1 || slot == 0)
        return 0;
    return 2 * ((slot + 255) / 256 * 256);
}

kda_status kda_chunk_fwd_segmented(int B, int T, int H, int dk, int dv, kda_dtype dtype, int seg_T, const void *q,
                                   const void *k, const void *v, const void *a, const void *beta, float g_min,
                                   const float *S0, void *o, float *S_T, void *workspace, size_t ws_bytes,
                                   kda_stream_t stream)
{
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, dtype, sh);
    if (st != KDA_OK)
        return st;
    if (dtype != KDA_BF16)
        return KDA_ERR_UNSUPPORTED;
    if (seg_T < KDA_CHUNK || seg_T % KDA_CHUNK != 0 || !S_T)
        return KDA_ERR_INVALID_ARG;
    // every check of kda_chunk_fwd on the whole problem, the workspace range included
    st = validate_chunk_fwd(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, KDA_GATE_BOUNDED, S0, o, S_T,
                            workspace, ws_bytes, false);
    if (st != KDA_OK)
        return st;
    const cudaStream_t s = (cudaStream_t)stream;
    if (T == 0)
        return copy_state(sh, S0, S_T, s);
    const size_t need = kda_chunk_fwd_segmented_workspace(B, T, H, dk, dv, seg_T);
    if (!workspace || ws_bytes < need)
        return KDA_ERR_WORKSPACE;
    const int64_t nseg = ((int64_t)T + seg_T - 1) / seg_T, units = (int64_t)B * nseg;
    const size_t slot = need / 2;
    unsigned char *ws[2] = {static_cast<unsigned char *>(workspace), static_cast<unsigned char *>(workspace) + slot};
    const int64_t tok = (int64_t)H * dk * 2, st_elems = (int64_t)H * dk * dv;  // bytes per token row; state floats
    auto at = [](const void *p, int64_t off) { return static_cast<const unsigned char *>(p) + off; };

    // two streams of this call (released once their work is done): the preps at the lowest
    // priority, the scans at the highest, so that a scan's CTAs are placed ahead of the next
    // prep's; both start after the work already on `stream`, which waits for the last scan
    int lo = 0, hi = 0;
    cudaStream_t sp = nullptr, sc = nullptr;
    cudaEvent_t ev_start = nullptr, ev_prep = nullptr, ev_scan[2] = {nullptr, nullptr};
    cudaError_t e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
    if (e == cudaSuccess)
        e = cudaStreamCreateWithPriority(&sp, cudaStreamNonBlocking, lo);
    if (e == cudaSuccess)
        e = cudaStreamCreateWithPriority(&sc, cudaStreamNonBlocking, hi);
    for (cudaEvent_t *ev : {&ev_start, &ev_prep, &ev_scan[0], &ev_scan[1]})
        if (e == cudaSuccess)
            e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e == cudaSuccess)
        e = cudaEventRecord(ev_start, s);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(sp, ev_start, 0);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(sc, ev_start, 0);
    // unit u = (batch element b, stretch i): the prep on `sp` (after the scan that last read its
    // slot), the scan on `sc` after that prep, the state carried in S_T
    int64_t last = -1;  // the last unit whose scan is recorded
    for (int64_t u = 0; u < units && e == cudaSuccess; ++u) {
        const int64_t b = u / nseg, i = u % nseg, t0 = i * seg_T;
        const int len = (int)(T - t0 < seg_T ? T - t0 : seg_T);
        const int64_t row = b * T + t0;  // first token row of the stretch
        if (u >= 2)
            e = cudaStreamWaitEvent(sp, ev_scan[u & 1], 0);
        if (e == cudaSuccess)
            e = launch_prep_bf16(1, len, H, dk, at(q, row * tok), at(k, row * tok), at(v, row * tok),
                                 at(a, row * tok), at(beta, row * H * 2), g_min, false, nullptr, ws[u & 1], sp);
        if (e == cudaSuccess)
            e = cudaEventRecord(ev_prep, sp);
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(sc, ev_prep, 0);
        if (e == cudaSuccess) {
            float *Sb = S_T + b * st_elems;
            const float *Sin = i > 0 ? Sb : (S0 ? S0 + b * st_elems : nullptr);
            e = launch_scan_bf16(1, len, H, dk, ws[u & 1], Sin, static_cast<unsigned char *>(o) + row * (int64_t)H * dv * 2,
                                 Sb, sc);
        }
        if (e == cudaSuccess && (e = cudaEventRecord(ev_scan[u & 1], sc)) == cudaSuccess)
            last = u;
    }
    if (last >= 0) {  // later work on `stream` follows the last scan, which follows every prep
        const cudaError_t ej = cudaStreamWaitEvent(s, ev_scan[last & 1], 0);
        if (e == cudaSuccess)
            e = ej;
    }
    // (destroying an event or a stream whose work is pending releases it once that work is done)
    for (cudaEvent_t ev : {ev_start, ev_prep, ev_scan[0], ev_scan[1]})
        if (ev)
            cudaEventDestroy(ev);
    for (cudaStream_t st2 : {sp, sc})
        if (st2)
            cudaStreamDestroy(st2);
    return from_cuda(e);
}

kda_status kda_decode_step(int N, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k, const void *v,
                           const void *a, const void *beta, float g_min, float *S, void *o, kda_stream_t stream)
{
    if (!dtype_ok(dtype) || N < 1 || H < 1 || dk < 1 || dv < 1)
        return KDA_ERR_INVALID_ARG;
    kda_status st = check_gmin(g_min);
    if (st != KDA_OK)
        return st;
    if (dk != dv || (dk != 64 && dk != 128))
        return KDA_ERR_UNSUPPORTED;
    const int64_t nh = safe_prod({N, H});
    const int64_t ns = safe_prod({N, H, dk, dv});
    if (nh < 0 || ns < 0 || nh > 0x7fffffff)
        return KDA_ERR_INVALID_ARG;
    if (!q || !k || !v || !a || !beta || !S || !o)
        return KDA_ERR_INVALID_ARG;
    const int es = elem_size(dtype);
    const void *ptrs[] = {q, k, v, a, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p))
            return KDA_ERR_ALIGNMENT;
    if (!beta_aligned(beta, es))
        return KDA_ERR_ALIGNMENT;
    const Range rq(q, nh * dk * es), rk(k, nh * dk * es), rv(v, nh * dv * es), ra(a, nh * dk * es),
        rb(beta, nh * es), rS(S, ns * 4), ro(o, nh * dv * es);
    for (const Range &in : {rq, rk, rv, ra, rb, rS})
        if (overlaps(ro, in))
            return KDA_ERR_ALIAS;
    for (const Range &in : {rq, rk, rv, ra, rb})
        if (overlaps(rS, in))
            return KDA_ERR_ALIAS;
    return from_cuda(launch_decode(N, H, dk, dtype, q, k, v, a, beta, g_min, S, o, (cudaStream_t)stream));
}

size_t kda_chunk_bwd_workspace(int B, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (B < 1 || H < 1 || T <= 0 || dk != dv || (dk != 64 && dk != 128) || dtype != KDA_BF16)
        return 0;
    return chunk_bf16_bwd_workspace(B, T, H, dk);
}

kda_status kda_chunk_bwd_offsets(int B, int T, int H, int dk, int dv, size_t *states_offset,
                                 size_t *dstates_offset)
{
    if (!states_offset || !dstates_offset)
        return KDA_ERR_INVALID_ARG;
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, KDA_BF16, sh);
    if (st != KDA_OK)
        return st;
    if (T == 0) {
        *states_offset = *dstates_offset = 0;
        return KDA_OK;
    }
    chunk_bf16_bwd_offsets(B, T, H, dk, states_offset, dstates_offset);
    return KDA_OK;
}

}  // extern "C"

namespace {

// Validation and dispatch of kda_chunk_bwd and kda_chunk_bwd_recorded (have_records: the
// workspace holds the forward's records; the prep is not launched).
kda_status chunk_bwd_impl(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                          const void *v, const void *a, const void *beta, float g_min, const float *A_log,
                          const float *S0, const void *dO, const float *dS_T, float *dq, float *dk_, float *dv_,
                          float *da, float *dbeta, float *dS0, float *dA_log, void *workspace, size_t ws_bytes,
                          kda_stream_t stream, bool have_records)
{
    ChunkShape sh;
    kda_status st = check_shape(B, T, H, dk, dv, dtype, sh);
    if (st != KDA_OK)
        return st;
    // the saved state arrays are addressed as (records x dk) rows with 32-bit coordinates
    if (dtype != KDA_BF16 || (int64_t)B * H * (((int64_t)T + 63) / 64) * dk > 0x7fffffff)
        return KDA_ERR_UNSUPPORTED;
    st = check_gmin(g_min);
    if (st != KDA_OK)
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (dA_log && !A_log)
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({S0, dS_T, dS0}) || ((uintptr_t)A_log & 3u) || ((uintptr_t)dA_log & 3u))
        return KDA_ERR_ALIGNMENT;
    const Range rS0(S0, sh.ns * 4), rdST(dS_T, sh.ns * 4), rdS0(dS0, sh.ns * 4), rA(A_log, (int64_t)H * 4),
        rdA(dA_log, (int64_t)H * 4);
    if (overlaps(rdS0, rS0) || overlaps(rdS0, rdST) || overlaps(rdS0, rA) || overlaps(rdA, rA) ||
        overlaps(rdA, rS0) || overlaps(rdA, rdST) || overlaps(rdA, rdS0))
        return KDA_ERR_ALIAS;
    if (T == 0) {
        if (dA_log) {
            const kda_status z = from_cuda(cudaMemsetAsync(dA_log, 0, (size_t)H * 4, s));
            if (z != KDA_OK)
                return z;
        }
        if (!dS0)
            return KDA_OK;
        if (dS_T)
            return from_cuda(cudaMemcpyAsync(dS0, dS_T, (size_t)sh.ns * 4, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(dS0, 0, (size_t)sh.ns * 4, s));
    }
    if (!q || !k || !v || !a || !beta || !dO || !dq || !dk_ || !dv_ || !da || !dbeta)
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, a, dO, dq, dk_, dv_, da, dbeta, workspace}) || !beta_aligned(beta, 2))
        return KDA_ERR_ALIGNMENT;
    const size_t need = chunk_bf16_bwd_workspace(B, T, H, dk);
    if (!workspace || ws_bytes < need)
        return KDA_ERR_WORKSPACE;
    const int64_t es = 2;
    const Range ins[] = {Range(q, sh.nk * es), Range(k, sh.nk * es), Range(v, sh.nv * es), Range(a, sh.nk * es),
                         Range(beta, sh.ntok * es), Range(dO, sh.nv * es), rS0, rdST, rA};
    const Range outs[] = {Range(dq, sh.nk * 4), Range(dk_, sh.nk * 4), Range(dv_, sh.nv * 4), Range(da, sh.nk * 4),
                          Range(dbeta, sh.ntok * 4), rdS0, rdA, Range(workspace, (int64_t)need)};
    for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
        for (const Range &in : ins)
            if (overlaps(outs[i], in))
                return KDA_ERR_ALIAS;
        for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
            if (overlaps(outs[i], outs[j]))
                return KDA_ERR_ALIAS;
    }
    return from_cuda(launch_chunk_bwd_bf16(B, T, H, dk, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk_, dv_,
                                           da, dbeta, dS0, dA_log, workspace, s, have_records));
}

}  // namespace

extern "C" {

kda_status kda_chunk_bwd(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                         const void *v, const void *a, const void *beta, float g_min, const float *A_log,
                         const float *S0, const void *dO, const float *dS_T, float *dq, float *dk_, float *dv_,
                         float *da, float *dbeta, float *dS0, float *dA_log, void *workspace, size_t ws_bytes,
                         kda_stream_t stream)
{
    return chunk_bwd_impl(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk_, dv_, da,
                          dbeta, dS0, dA_log, workspace, ws_bytes, stream, false);
}

kda_status kda_chunk_bwd_recorded(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                                  const void *v, const void *a, const void *beta, float g_min, const float *A_log,
                                  const float *S0, const void *dO, const float *dS_T, float *dq, float *dk_,
                                  float *dv_, float *da, float *dbeta, float *dS0, float *dA_log, void *workspace,
                                  size_t ws_bytes, kda_stream_t stream)
{
    return chunk_bwd_impl(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk_, dv_, da,
                          dbeta, dS0, dA_log, workspace, ws_bytes, stream, true);
}

size_t kda_chunk_bwd_varlen_workspace(int N, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (N < 1 || T < 1 || T > kMaxPackedTokens || H < 1 || dk != dv || (dk != 64 && dk != 128) || dtype != KDA_BF16)
        return 0;
    return chunk_bf16_bwd_varlen_workspace(N, T, H, dk);
}

kda_status kda_chunk_bwd_varlen(int N, const int32_t *cu_seqlens, int T, int H, int dk, int dv, kda_dtype dtype,
                                float g_min, const float *A_log, const void *q, const void *k, const void *v,
                                const void *a, const void *beta, const float *S0, const void *dO, const float *dS_T,
                                float *dq, float *dk_, float *dv_, float *da, float *dbeta, float *dS0,
                                float *dA_log, void *workspace, size_t ws_bytes, kda_stream_t stream)
{
    if (!dtype_ok(dtype) || N < 1 || H < 1 || T < 0 || dk < 1 || dv < 1)
        return KDA_ERR_INVALID_ARG;
    kda_status st = check_gmin(g_min);
    if (st != KDA_OK)
        return st;
    if (dk != dv || (dk != 64 && dk != 128) || dtype != KDA_BF16 || T > kMaxPackedTokens || (int64_t)N * H > 65535 ||
        (int64_t)H * (((int64_t)T + 63) / 64 + N) * dk > 0x7fffffff)
        return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens || (dA_log && !A_log))
        return KDA_ERR_INVALID_ARG;
    const int64_t nk = (int64_t)T * H * dk, ntok = (int64_t)T * H, ns = (int64_t)N * H * dk * dv;
    if (!all_aligned({S0, dS_T, dS0}) || ((uintptr_t)cu_seqlens & 3u) || ((uintptr_t)A_log & 3u) ||
        ((uintptr_t)dA_log & 3u))
        return KDA_ERR_ALIGNMENT;
    const Range rcu(cu_seqlens, (int64_t)(N + 1) * 4), rS0(S0, ns * 4), rdST(dS_T, ns * 4), rdS0(dS0, ns * 4),
        rA(A_log, (int64_t)H * 4), rdA(dA_log, (int64_t)H * 4);
    if (T == 0) {
        // nothing to differentiate through; the state gradient passes unchanged (cu is not read)
        if (overlaps(rdS0, rS0) || overlaps(rdS0, rdST) || overlaps(rdS0, rA) || overlaps(rdA, rA) ||
            overlaps(rdA, rdS0) || overlaps(rdA, rdST) || overlaps(rdA, rS0) || overlaps(rdS0, rcu) ||
            overlaps(rdA, rcu))
            return KDA_ERR_ALIAS;
        cudaStream_t s = (cudaStream_t)stream;
        if (dA_log && (st = from_cuda(cudaMemsetAsync(dA_log, 0, (size_t)H * 4, s))) != KDA_OK)
            return st;
        if (!dS0)
            return KDA_OK;
        if (dS_T)
            return from_cuda(cudaMemcpyAsync(dS0, dS_T, (size_t)ns * 4, cudaMemcpyDeviceToDevice, s));
        return from_cuda(cudaMemsetAsync(dS0, 0, (size_t)ns * 4, s));
    }
    if (!q || !k || !v || !a || !beta || !dO || !dq || !dk_ || !dv_ || !da || !dbeta)
        return KDA_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, a, dO, dq, dk_, dv_, da, dbeta, workspace}) || !beta_aligned(beta, 2))
        return KDA_ERR_ALIGNMENT;
    const size_t need = chunk_bf16_bwd_varlen_workspace(N, T, H, dk);
    if (!workspace || ws_bytes < need)
        return KDA_ERR_WORKSPACE;
    const Range ins[] = {Range(q, nk * 2), Range(k, nk * 2), Range(v, nk * 2), Range(a, nk * 2), Range(beta, ntok * 2),
                         Range(dO, nk * 2), rS0, rdST, rA, rcu};
    const Range outs[] = {Range(dq, nk * 4), Range(dk_, nk * 4), Range(dv_, nk * 4), Range(da, nk * 4),
                          Range(dbeta, ntok * 4), rdS0, rdA, Range(workspace, (int64_t)need)};
    for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
        for (const Range &in : ins)
            if (overlaps(outs[i], in))
                return KDA_ERR_ALIAS;
        for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
            if (overlaps(outs[i], outs[j]))
                return KDA_ERR_ALIAS;
    }
    return from_cuda(launch_chunk_bwd_bf16_varlen(N, cu_seqlens, T, H, dk, q, k, v, a, beta, g_min, A_log, S0, dO,
                                                  dS_T, dq, dk_, dv_, da, dbeta, dS0, dA_log, workspace,
                                                  (cudaStream_t)stream));
}

kda_status kda_device_status(kda_stream_t stream)
{
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
            return KDA_ERR_CUDA;
        return (kda_status)v;
    }
    return KDA_OK;
}

}  // extern "C"
