// noalloc.cu -- kda_chunk_fwd_noalloc: the chunked forward without caller-provided
// scratch, for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: code that runs while a CUDA graph
// is being captured (allocation calls are not allowed inside a capture), serving loops
// that must never call cudaMalloc (it can synchronise the device and stall every stream),
// and hosts whose device memory is owned by another allocator with nothing left over.
// For them this entry point uses a fixed scratch array that lives in the library itself:
// a file-scope device array of kScratchBytes, which every GPU that loads the library
// keeps until the process exits.  Nothing here allocates.
//
// The scratch holds the per-chunk records of kda_chunk_fwd for one stretch of whole
// 64-token chunks of one batch element at a time and the gate table after them, plus a
// carry slot for the state when the caller passes no S_T.  Longer inputs are processed stretch by stretch with the
// float32 state carried between calls, which gives exactly the same result as one call.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr size_t kScratchBytes = (size_t)64 << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array in the current device's context.  Host code only
// holds a stand-in for the array's name, so the address is looked up on every call (this
// allocates nothing); a cached address could outlive its context (cudaDeviceReset, another
// context made current on the same device).  The first lookup on a device may load the
// module, which is why the first call should come before any stream capture.
cudaError_t scratch_ptr(void **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
        return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" size_t kda_chunk_fwd_noalloc_max_scratch(void) { return kScratchBytes; }

extern "C" kda_status kda_chunk_fwd_noalloc(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q,
                                            const void *k, const void *v, const void *a, const void *beta,
                                            float g_min, const float *S0, void *o, float *S_T,
                                            kda_stream_t stream)
{
    // Every check runs once on the whole (B, T) problem -- shapes, gate bound, alignment, and
    // overlaps between any two tensors, across batch elements too -- before anything is
    // launched.  The scratch is library memory no caller pointer can reach, so it takes no
    // part in the overlap checks.
    kda_status st = validate_chunk_fwd(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, KDA_GATE_BOUNDED, S0, o,
                                       S_T, nullptr, 0, false);
    if (st != KDA_OK)
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    // The float32 path and T = 0 need no scratch.
    if (dtype == KDA_F32 || T == 0)
        return dispatch_chunk_fwd(B, T, H, dk, dtype, q, k, v, a, beta, g_min, KDA_GATE_BOUNDED, S0, o, S_T,
                                  nullptr, s);

    const size_t rec = chunk_bf16_records(1, KDA_CHUNK, H, dk);  // one chunk of every head
    const size_t state_bytes = ((size_t)H * dk * dv * 4 + 255) / 256 * 256;  // carry slot, one batch element
    const size_t table = kGateTableEntries * 4;  // the gate table after the records (no per-head scale here)
    if (state_bytes + table + rec > kScratchBytes)
        return KDA_ERR_WORKSPACE;  // not even one chunk of all heads fits the fixed scratch
    const int64_t chunks = (int64_t)((kScratchBytes - state_bytes - table) / rec);
    const int64_t stretch = chunks * KDA_CHUNK;  // tokens per launch pair

    void *scratch = nullptr;
    if (scratch_ptr(&scratch) != cudaSuccess)
        return KDA_ERR_CUDA;
    float *carry_slot = static_cast<float *>(scratch);
    void *ws = static_cast<unsigned char *>(scratch) + state_bytes;

    const size_t es = 2;  // bf16
    const unsigned char *qb = static_cast<const unsigned char *>(q);
    const unsigned char *kb = static_cast<const unsigned char *>(k);
    const unsigned char *vb = static_cast<const unsigned char *>(v);
    const unsigned char *ab = static_cast<const unsigned char *>(a);
    const unsigned char *bb = static_cast<const unsigned char *>(beta);
    unsigned char *ob = static_cast<unsigned char *>(o);
    const size_t state_elems = (size_t)H * dk * dv;
    for (int b = 0; b < B; ++b) {
        const float *s_in = S0 ? S0 + (size_t)b * state_elems : nullptr;
        // without S_T the state between stretches lives in the carry slot, reused by every
        // batch element (each one's first stretch starts from its own S0, never the slot)
        float *carry = S_T ? S_T + (size_t)b * state_elems : carry_slot;
        for (int64_t t0 = 0; t0 < T; t0 += stretch) {
            const int len = (int)(T - t0 < stretch ? T - t0 : stretch);
            const size_t tok = (size_t)b * T + (size_t)t0;  // first token row of this stretch
            st = dispatch_chunk_fwd(1, len, H, dk, dtype, qb + tok * H * dk * es, kb + tok * H * dk * es,
                                    vb + tok * H * dv * es, ab + tok * H * dk * es, bb + tok * H * es, g_min,
                                    KDA_GATE_BOUNDED, t0 == 0 ? s_in : carry, ob + tok * H * dv * es, carry, ws, s);
            if (st != KDA_OK)
                return st;
        }
    }
    return KDA_OK;
}
