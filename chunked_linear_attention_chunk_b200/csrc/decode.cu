// decode.cu -- K4: one decode token for N independent sequences, state in place.
//
// The constant-size incremental state of "Trillion-Parameter MoE Multimodal Models:
// Engineering ..." section 3.2, advanced by one token of the gated delta rule:
//   S_dec = Diag(e^{g}) S,  g = g_min * sigmoid(a);   w = S_dec^T k;  y = S_dec^T q
//   u = beta (v - w);   S' = S_dec + k u^T;   o = S'^T q = y + (k . q) u
// Memory-bound: every (n, h) state (dk x dv float32) is read once and written once.
//
// A persistent CTA per SM walks the (n, h) units with a 3-stage shared-memory pipeline:
// bulk copies bring a unit's state and token vectors in two units ahead, the threads
// update the state in place in shared memory, and a bulk store writes it back while
// the next units are computed, so HBM sees a steady stream of reads and writes.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecStages = 3;

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

// One pipeline stage: the unit's state, then its q, k, v, a vectors.
template <int D, typename Tin>
struct DecStage {
    static constexpr uint32_t kState = (uint32_t)D * D * 4;
    static constexpr uint32_t kVec = (uint32_t)D * sizeof(Tin);
    static constexpr uint32_t kBytes = kState + 4 * kVec;
    static_assert(kVec % 16 == 0 && kBytes % 16 == 0, "bulk copy sizes are multiples of 16 bytes");
};

template <int D, typename Tin>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(int64_t units, const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const Tin *__restrict__ a, const Tin *__restrict__ beta, double g_min, float *__restrict__ S,
                  Tin *__restrict__ o, unsigned int *status)
{
    using St = DecStage<D, Tin>;
    constexpr int CPT = D / 32;         // columns per lane (4 for D = 128: one float4)
    constexpr int RPW = D / kDecWarps;  // rows per warp
    static_assert(CPT == 4 || CPT == 2, "D must be 64 or 128");
    extern __shared__ __align__(128) unsigned char dec_smem[];
    __shared__ __align__(8) uint64_t full[kDecStages];
    __shared__ float sdec[D];
    __shared__ float red_w[kDecWarps][D], red_y[kDecWarps][D];
    __shared__ float s_kq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t first = blockIdx.x, stride = gridDim.x;

    auto issue = [&](int64_t u, int s) {  // one thread: bring unit u into stage s
        unsigned char *b = dec_smem + (size_t)s * St::kBytes;
        mbar_arrive_expect_tx(&full[s], St::kBytes);
        bulk_g2s(b, S + u * D * D, St::kState, &full[s]);
        bulk_g2s(b + St::kState, q + u * D, St::kVec, &full[s]);
        bulk_g2s(b + St::kState + St::kVec, k + u * D, St::kVec, &full[s]);
        bulk_g2s(b + St::kState + 2 * St::kVec, v + u * D, St::kVec, &full[s]);
        bulk_g2s(b + St::kState + 3 * St::kVec, a + u * D, St::kVec, &full[s]);
    };
    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s)
            mbar_init(&full[s], 1);
        fence_mbar_init_cluster();
        for (int s = 0; s < kDecStages - 1; ++s)
            if (first + s * stride < units)
                issue(first + s * stride, s);
    }
    __syncthreads();

    float bt_next = first < units ? ld_scalar(beta + first) : 0.0f;  // beta one unit ahead
    int it = 0;
    for (int64_t u = first; u < units; u += stride, ++it) {
        const int s = it % kDecStages;
        const float bt = bt_next;
        if (u + stride < units)
            bt_next = ld_scalar(beta + u + stride);
        mbar_wait_bounded(&full[s], (uint32_t)(it / kDecStages) & 1u, status);
        float *Ss = reinterpret_cast<float *>(dec_smem + (size_t)s * St::kBytes);
        const Tin *sq = reinterpret_cast<const Tin *>(dec_smem + (size_t)s * St::kBytes + St::kState);
        const Tin *sk = sq + D, *sv = sq + 2 * D, *sa = sq + 3 * D;

        for (int i = tid; i < D; i += kDecThreads)
            sdec[i] = expf(gate_bounded_exact(ld_scalar(sa + i), g_min));
        if (warp == kDecWarps - 1) {
            float kq = 0.0f;
            for (int i = lane; i < D; i += 32)
                kq += ld_scalar(sk + i) * ld_scalar(sq + i);
            kq = warp_sum(kq);
            if (lane == 0)
                s_kq = kq;
        }
        __syncthreads();
        // decay this warp's rows, partial column sums w = S_dec^T k and y = S_dec^T q
        float st[RPW][CPT];
        float pw[CPT] = {}, py[CPT] = {};
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int r = warp + i * kDecWarps;
            const float d = sdec[r], kr = ld_scalar(sk + r), qr = ld_scalar(sq + r);
            if constexpr (CPT == 4) {
                const float4 x = reinterpret_cast<const float4 *>(Ss + r * D)[lane];
                st[i][0] = x.x * d;
                st[i][1] = x.y * d;
                st[i][2] = x.z * d;
                st[i][3] = x.w * d;
            } else {
                const float2 x = reinterpret_cast<const float2 *>(Ss + r * D)[lane];
                st[i][0] = x.x * d;
                st[i][1] = x.y * d;
            }
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                pw[c] += st[i][c] * kr;
                py[c] += st[i][c] * qr;
            }
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            red_w[warp][lane * CPT + c] = pw[c];
            red_y[warp][lane * CPT + c] = py[c];
        }
        __syncthreads();
        // every warp reduces the partial sums of its lane's columns (redundantly per warp)
        const float kq = s_kq;
        float uu[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int j = lane * CPT + c;
            float w = 0.0f, y = 0.0f;
#pragma unroll
            for (int x = 0; x < kDecWarps; ++x) {
                w += red_w[x][j];
                y += red_y[x][j];
            }
            uu[c] = bt * (ld_scalar(sv + j) - w);
            if (warp == 0)
                st_scalar(o + u * D + j, y + kq * uu[c]);
        }
        // S' = S_dec + k u^T, in place in the stage
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int r = warp + i * kDecWarps;
            const float kr = ld_scalar(sk + r);
            if constexpr (CPT == 4)
                reinterpret_cast<float4 *>(Ss + r * D)[lane] = make_float4(
                    st[i][0] + kr * uu[0], st[i][1] + kr * uu[1], st[i][2] + kr * uu[2], st[i][3] + kr * uu[3]);
            else
                reinterpret_cast<float2 *>(Ss + r * D)[lane] = make_float2(st[i][0] + kr * uu[0], st[i][1] + kr * uu[1]);
        }
        fence_proxy_async_smem();
        __syncthreads();  // also: every thread is done with sdec / red_* / s_kq of this unit
        if (tid == 0) {
            bulk_s2g(S + u * D * D, Ss, St::kState);
            bulk_commit();
            // the stage of unit u + 2 stride held unit u - stride: its store must have read it
            if (u + (kDecStages - 1) * stride < units) {
                bulk_wait_read_1();
                issue(u + (kDecStages - 1) * stride, (it + kDecStages - 1) % kDecStages);
            }
        }
    }
    if (tid == 0)
        bulk_wait_all();
}

template <int D, typename Tin>
cudaError_t launch_dec(int N, int H, const void *q, const void *k, const void *v, const void *a, const void *beta,
                       float g_min, float *S, void *o, cudaStream_t s)
{
    using St = DecStage<D, Tin>;
    unsigned int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidDevice;
    const int64_t units = (int64_t)N * H;
    const size_t smem = (size_t)kDecStages * St::kBytes;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<D, Tin>, kDecThreads, smem);
    if (e != cudaSuccess)
        return e;
    const int64_t resident = (int64_t)num_sms() * (per_sm > 0 ? per_sm : 1);
    const unsigned grid = (unsigned)(units < resident ? units : resident);
    decode_kernel<D, Tin><<<grid, kDecThreads, smem, s>>>(
        units, static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v),
        static_cast<const Tin *>(a), static_cast<const Tin *>(beta), (double)g_min, S, static_cast<Tin *>(o), status);
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
