// chunk_f32.cu -- K5: float32 CUDA-core chunked forward (the debug path).
//
// Same chunked algebra as the tensor-core path, in float32 on CUDA cores, with the
// state carried every 16 tokens (one decay tile per chunk, so one reference point):
//   G_r   = sum_{s<=r} g_s inside the chunk, reference G_m at the tile's middle token;
//   A_rj  = beta_r (k_r e^{G_r-G_m}) . (k_j e^{G_m-G_j})        j <  r
//   P_rj  =        (q_r e^{G_r-G_m}) . (k_j e^{G_m-G_j})        j <= r
//   (I + A) U = diag(beta) (V - Kbar S),  Kbar = k e^{G}          (forward substitution)
//   O = Qbar S + P U,  Qbar = q e^{G}
//   S <- Diag(e^{G_last}) S + Khat^T U,  Khat = k e^{G_last - G}
// The pairwise decay inside the tile is factored through the reference (the pages'
// 1/Gamma, "Trillion-Scale MoE Multimodal Models ..." section 3.1), which the lower
// bound on g keeps in range ("... section 3.2"; "Breaking Through ..." section 2.1).
// One CTA per (batch, head); the whole state lives in shared memory.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kC = 16;        // tokens per chunk (= one decay tile)
constexpr int kRef = 7;       // reference token inside the tile (its middle)
constexpr int kThreads = 256;

template <int D>
struct F32Smem {
    static constexpr int LD = D + 1;  // padded rows: column walks hit distinct banks
    float S[D * D];
    float Kr[kC * LD], Qr[kC * LD], Kc[kC * LD];  // tile-referenced factors
    float Kb[kC * LD], Qb[kC * LD], Kh[kC * LD];  // chunk-start / chunk-end factors
    float G[kC * D];
    float V[kC * D];
    float U[kC * D];
    float A[kC * kC], P[kC * kC];
    float beta[kC];
    float gam[D];
};

template <int D>
__global__ void __launch_bounds__(kThreads) chunk_f32_kernel(int T, int H, const float *__restrict__ q,
                                                             const float *__restrict__ k,
                                                             const float *__restrict__ v,
                                                             const float *__restrict__ a,
                                                             const float *__restrict__ beta, double g_min,
                                                             const float *__restrict__ S0,
                                                             float *__restrict__ o, float *__restrict__ S_T)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    F32Smem<D> &sm = *reinterpret_cast<F32Smem<D> *>(smem_raw);
    constexpr int LD = F32Smem<D>::LD;
    constexpr int RG = kThreads / D;  // row groups when threads map to (column, row group)
    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int64_t sbase = (int64_t)bh * D * D;

    for (int i = tid; i < D * D; i += kThreads)
        sm.S[i] = S0 ? S0[sbase + i] : 0.0f;

    const int j = tid % D;   // value column handled by this thread
    const int rg = tid / D;  // row group
    for (int t0 = 0; t0 < T; t0 += kC) {
        const int n = min(kC, T - t0);
        __syncthreads();
        // -- load the chunk: gate + inclusive cumulative log-decay, one thread per channel
        if (tid < D) {
            float acc = 0.0f;
            for (int r = 0; r < kC; ++r) {
                float g = 0.0f;
                if (r < n) {
                    const int64_t off = (((int64_t)b * T + t0 + r) * H + h) * D + tid;
                    g = gate_bounded_exact(a[off], g_min);
                }
                acc += g;
                sm.G[r * D + tid] = acc;
            }
        }
        for (int i = tid; i < kC * D; i += kThreads) {
            const int r = i / D, c = i % D;
            const int64_t off = (((int64_t)b * T + t0 + r) * H + h) * D + c;
            sm.V[i] = r < n ? v[off] : 0.0f;
        }
        if (tid < kC)
            sm.beta[tid] = tid < n ? beta[((int64_t)b * T + t0 + tid) * H + h] : 0.0f;
        __syncthreads();
        // -- decay factors
        for (int i = tid; i < kC * D; i += kThreads) {
            const int r = i / D, c = i % D;
            const int64_t off = (((int64_t)b * T + t0 + r) * H + h) * D + c;
            const float kv = r < n ? k[off] : 0.0f;
            const float qv = r < n ? q[off] : 0.0f;
            const float Gr = sm.G[r * D + c], Gm = sm.G[kRef * D + c], Gl = sm.G[(kC - 1) * D + c];
            const float up = expf(Gr - Gm), down = expf(Gm - Gr);
            sm.Kr[r * LD + c] = kv * up;
            sm.Qr[r * LD + c] = qv * up;
            sm.Kc[r * LD + c] = kv * down;
            const float e = expf(Gr);
            sm.Kb[r * LD + c] = kv * e;
            sm.Qb[r * LD + c] = qv * e;
            sm.Kh[r * LD + c] = kv * expf(Gl - Gr);
        }
        if (tid < D)
            sm.gam[tid] = expf(sm.G[(kC - 1) * D + tid]);
        __syncthreads();
        // -- tile products A (strictly lower, beta-scaled) and P (lower incl.)
        {
            const int r = tid / kC, c = tid % kC;  // kThreads == kC*kC
            float sa = 0.0f, sp = 0.0f;
            for (int x = 0; x < D; ++x) {
                const float kc = sm.Kc[c * LD + x];
                sa += sm.Kr[r * LD + x] * kc;
                sp += sm.Qr[r * LD + x] * kc;
            }
            sm.A[r * kC + c] = c < r ? sm.beta[r] * sa : 0.0f;
            sm.P[r * kC + c] = c <= r ? sp : 0.0f;
        }
        // -- right-hand side R = diag(beta)(V - Kbar S) and Y = Qbar S
        float y[kC / RG];
        {
            float ks[kC / RG];
#pragma unroll
            for (int i = 0; i < kC / RG; ++i)
                ks[i] = y[i] = 0.0f;
            for (int x = 0; x < D; ++x) {
                const float s = sm.S[x * D + j];
#pragma unroll
                for (int i = 0; i < kC / RG; ++i) {
                    const int r = rg + i * RG;
                    ks[i] += sm.Kb[r * LD + x] * s;
                    y[i] += sm.Qb[r * LD + x] * s;
                }
            }
#pragma unroll
            for (int i = 0; i < kC / RG; ++i) {
                const int r = rg + i * RG;
                sm.U[r * D + j] = sm.beta[r] * (sm.V[r * D + j] - ks[i]);
            }
        }
        __syncthreads();
        // -- forward substitution (I + A) U = R, one thread per value column
        if (tid < D) {
            float u[kC];
#pragma unroll
            for (int r = 0; r < kC; ++r) {
                float s = sm.U[r * D + tid];
#pragma unroll
                for (int x = 0; x < r; ++x)
                    s -= sm.A[r * kC + x] * u[x];
                u[r] = s;
            }
#pragma unroll
            for (int r = 0; r < kC; ++r)
                sm.U[r * D + tid] = u[r];
        }
        __syncthreads();
        // -- outputs O = Qbar S + P U
#pragma unroll
        for (int i = 0; i < kC / RG; ++i) {
            const int r = rg + i * RG;
            float acc = y[i];
            for (int x = 0; x <= r; ++x)
                acc += sm.P[r * kC + x] * sm.U[x * D + j];
            if (r < n)
                o[(((int64_t)b * T + t0 + r) * H + h) * D + j] = acc;
        }
        // -- state update S <- Diag(gamma) S + Khat^T U (each thread owns column j)
        for (int x = rg; x < D; x += RG) {
            float acc = sm.gam[x] * sm.S[x * D + j];
#pragma unroll
            for (int r = 0; r < kC; ++r)
                acc += sm.Kh[r * LD + x] * sm.U[r * D + j];
            sm.S[x * D + j] = acc;
        }
    }
    __syncthreads();
    if (S_T)
        for (int i = tid; i < D * D; i += kThreads)
            S_T[sbase + i] = sm.S[i];
}

template <int D>
cudaError_t launch_f32_d(int B, int T, int H, const float *q, const float *k, const float *v, const float *a,
                         const float *beta, float g_min, const float *S0, float *o, float *S_T, cudaStream_t s)
{
    const size_t smem = sizeof(F32Smem<D>);
    cudaError_t e = cudaFuncSetAttribute(chunk_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    chunk_f32_kernel<D><<<B * H, kThreads, smem, s>>>(T, H, q, k, v, a, beta, (double)g_min, S0, o, S_T);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_f32(int B, int T, int H, int D, const float *q, const float *k, const float *v,
                             const float *a, const float *beta, float g_min, const float *S0, float *o,
                             float *S_T, cudaStream_t s)
{
    if (D == 64)
        return launch_f32_d<64>(B, T, H, q, k, v, a, beta, g_min, S0, o, S_T, s);
    return launch_f32_d<128>(B, T, H, q, k, v, a, beta, g_min, S0, o, S_T, s);
}

}  // namespace kda
