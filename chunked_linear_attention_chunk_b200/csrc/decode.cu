// decode.cu -- K4: one decode token for N independent sequences, state in place.
//
// The constant-size incremental state of "Trillion-Parameter MoE Multimodal Models:
// Engineering ..." section 3.2, advanced by one token of the gated delta rule:
//   S_dec = Diag(e^{g}) S,  g = g_min * sigmoid(a);   w = S_dec^T k;  y = S_dec^T q
//   u = beta (v - w);   S' = S_dec + k u^T;   o = S'^T q = y + (k . q) u
// Memory-bound: every (n, h) state (dk x dv float32) is read once and written once.
// One CTA per (n, h); each warp streams whole 512-byte state rows with 16-byte
// accesses and keeps its rows in registers between the read and the write.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

template <typename Tin>
__device__ __forceinline__ float ld_scalar(const Tin *p);
template <>
__device__ __forceinline__ float ld_scalar<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_scalar<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <typename Tin>
__device__ __forceinline__ void st_scalar(Tin *p, float x);
template <>
__device__ __forceinline__ void st_scalar<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st_scalar<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = __float2bfloat16(x); }

template <int D, typename Tin>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const Tin *__restrict__ a, const Tin *__restrict__ beta, double g_min, float *__restrict__ S,
                  Tin *__restrict__ o)
{
    constexpr int CPT = D / 32;           // columns per lane (4 for D = 128: one float4)
    constexpr int RPW = D / kDecWarps;    // rows per warp
    static_assert(CPT == 4 || CPT == 2, "D must be 64 or 128");
    __shared__ float sq[D], sk[D], sdec[D];
    __shared__ float red_w[kDecWarps][D], red_y[kDecWarps][D];
    __shared__ float s_kq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t nh = blockIdx.x;
    const int64_t tok = nh * D;
    float *Sp = S + nh * (int64_t)D * D;

    // issue the state loads first: they are the bulk of the traffic
    float s[RPW][CPT];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp + i * kDecWarps;
        if constexpr (CPT == 4) {
            const float4 x = __ldcs(reinterpret_cast<const float4 *>(Sp + (int64_t)r * D) + lane);
            s[i][0] = x.x;
            s[i][1] = x.y;
            s[i][2] = x.z;
            s[i][3] = x.w;
        } else {
            const float2 x = __ldcs(reinterpret_cast<const float2 *>(Sp + (int64_t)r * D) + lane);
            s[i][0] = x.x;
            s[i][1] = x.y;
        }
    }
    for (int i = tid; i < D; i += kDecThreads) {
        sq[i] = ld_scalar(q + tok + i);
        sk[i] = ld_scalar(k + tok + i);
        sdec[i] = expf(gate_bounded_exact(ld_scalar(a + tok + i), g_min));
    }
    __syncthreads();
    if (warp == 0) {
        float kq = 0.0f;
        for (int i = lane; i < D; i += 32)
            kq += sk[i] * sq[i];
        kq = warp_sum(kq);
        if (lane == 0)
            s_kq = kq;
    }
    // decay, then partial column sums w = S_dec^T k and y = S_dec^T q over this warp's rows
    float pw[CPT] = {}, py[CPT] = {};
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp + i * kDecWarps;
        const float d = sdec[r], kr = sk[r], qr = sq[r];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            s[i][c] *= d;
            pw[c] += s[i][c] * kr;
            py[c] += s[i][c] * qr;
        }
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        red_w[warp][lane * CPT + c] = pw[c];
        red_y[warp][lane * CPT + c] = py[c];
    }
    __syncthreads();
    // every thread needs u for its CPT columns: reduce over warps redundantly per warp
    const float bt = ld_scalar(beta + nh);
    const float kq = s_kq;
    float u[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int j = lane * CPT + c;
        float w = 0.0f, y = 0.0f;
#pragma unroll
        for (int x = 0; x < kDecWarps; ++x) {
            w += red_w[x][j];
            y += red_y[x][j];
        }
        u[c] = bt * (ld_scalar(v + tok + j) - w);
        if (warp == 0)
            st_scalar(o + tok + j, y + kq * u[c]);
    }
    // S' = S_dec + k u^T
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp + i * kDecWarps;
        const float kr = sk[r];
        if constexpr (CPT == 4) {
            float4 x = make_float4(s[i][0] + kr * u[0], s[i][1] + kr * u[1], s[i][2] + kr * u[2],
                                   s[i][3] + kr * u[3]);
            __stcs(reinterpret_cast<float4 *>(Sp + (int64_t)r * D) + lane, x);
        } else {
            float2 x = make_float2(s[i][0] + kr * u[0], s[i][1] + kr * u[1]);
            __stcs(reinterpret_cast<float2 *>(Sp + (int64_t)r * D) + lane, x);
        }
    }
}

template <int D, typename Tin>
cudaError_t launch_dec(int N, int H, const void *q, const void *k, const void *v, const void *a, const void *beta,
                       float g_min, float *S, void *o, cudaStream_t s)
{
    const int64_t units = (int64_t)N * H;
    decode_kernel<D, Tin><<<(unsigned)units, kDecThreads, 0, s>>>(
        static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v),
        static_cast<const Tin *>(a), static_cast<const Tin *>(beta), (double)g_min, S, static_cast<Tin *>(o));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int N, int H, int D, kda_dtype dt, const void *q, const void *k, const void *v,
                          const void *a, const void *beta, float g_min, float *S, void *o, cudaStream_t s)
{
    if (dt == KDA_BF16)
        return D == 64 ? launch_dec<64, __nv_bfloat16>(N, H, q, k, v, a, beta, g_min, S, o, s)
                       : launch_dec<128, __nv_bfloat16>(N, H, q, k, v, a, beta, g_min, S, o, s);
    return D == 64 ? launch_dec<64, float>(N, H, q, k, v, a, beta, g_min, S, o, s)
                   : launch_dec<128, float>(N, H, q, k, v, a, beta, g_min, S, o, s);
}

}  // namespace kda
