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
// 64-token chunks of one batch element at a time, plus a carry slot for the state when
// the caller passes no S_T.  Longer inputs are processed stretch by stretch with the
// float32 state carried between calls, which gives exactly the same result as one call.
#include <mutex>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr size_t kScratchBytes = (size_t)64 << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device, looked up once per device.
cudaError_t scratch_ptr(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
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
    if ((dtype != KDA_BF16 && dtype != KDA_F32) || B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1)
        return KDA_ERR_INVALID_ARG;
    // The float32 path needs no scratch: the regular entry point allocates nothing either.
    if (dtype == KDA_F32 || T == 0)
        return kda_chunk_fwd(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, S0, o, S_T, nullptr, 0, stream);

    const size_t rec = kda_chunk_fwd_workspace(1, KDA_CHUNK, H, dk, dv, dtype);  // one chunk, all heads
    if (rec == 0)  // unsupported head dims: let the regular checks name the reason
        return kda_chunk_fwd(B, T, H, dk, dv, dtype, q, k, v, a, beta, g_min, S0, o, S_T, nullptr, 0, stream);
    const size_t state_bytes = ((size_t)H * dk * dv * 4 + 255) / 256 * 256;  // carry slot, one batch element
    if (state_bytes + rec > kScratchBytes)
        return KDA_ERR_WORKSPACE;  // not even one chunk of all heads fits the fixed scratch
    const int64_t chunks = (int64_t)((kScratchBytes - state_bytes) / rec);
    const int64_t stretch = chunks * KDA_CHUNK;  // tokens per call

    void *scratch = nullptr;
    if (scratch_ptr(&scratch) != cudaSuccess)
        return KDA_ERR_CUDA;
    float *carry_slot = static_cast<float *>(scratch);
    void *ws = static_cast<unsigned char *>(scratch) + state_bytes;
    const size_t ws_bytes = kScratchBytes - state_bytes;

    const size_t es = 2;  // bf16
    const unsigned char *qb = static_cast<const unsigned char *>(q);
    const unsigned char *kb = static_cast<const unsigned char *>(k);
    const unsigned char *vb = static_cast<const unsigned char *>(v);
    const unsigned char *ab = static_cast<const unsigned char *>(a);
    const unsigned char *bb = static_cast<const unsigned char *>(beta);
    unsigned char *ob = static_cast<unsigned char *>(o);
    if (!qb || !kb || !vb || !ab || !bb || !ob)
        return KDA_ERR_INVALID_ARG;
    const size_t state_elems = (size_t)H * dk * dv;
    for (int b = 0; b < B; ++b) {
        const float *s_in = S0 ? S0 + (size_t)b * state_elems : nullptr;
        float *carry = S_T ? S_T + (size_t)b * state_elems : carry_slot;
        for (int64_t t0 = 0; t0 < T; t0 += stretch) {
            const int len = (int)(T - t0 < stretch ? T - t0 : stretch);
            const size_t tok = (size_t)b * T + (size_t)t0;  // first token row of this stretch
            const kda_status st = kda_chunk_fwd(
                1, len, H, dk, dv, dtype, qb + tok * H * dk * es, kb + tok * H * dk * es, vb + tok * H * dv * es,
                ab + tok * H * dk * es, bb + tok * H * es, g_min, t0 == 0 ? s_in : carry, ob + tok * H * dv * es,
                carry, ws, ws_bytes, stream);
            if (st != KDA_OK)
                return st;
        }
    }
    return KDA_OK;
}
