// gate.cu -- K1: the lower-bounded log-decay gate, g = g_min * sigmoid(a).
//
// "Trillion-Scale MoE Multimodal Models ..." section 3.2 replaces the unbounded
// negative-softplus log-decay with g = g_min * Sigmoid(...), g_min = -5;
// "Breaking Through Trillion-Parameter Multimodal MoE ..." section 2.1 states the range
// [g_min, 0).  This stand-alone kernel evaluates the gate in float64 and rounds once to
// float32, so its output is bit-exact against an fp64 evaluation.  It is HBM-bound:
// 16-byte vector loads and stores, grid sized to a multiple of the SM count.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

template <typename Tin>
struct GateVec;

template <>
struct GateVec<__nv_bfloat16> {
    static constexpr int kPerVec = 8;  // 8 x bf16 = 16 bytes
    __device__ static void load(const __nv_bfloat16 *p, float (&x)[8])
    {
        uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = unpack_bf16x2(w[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    }
    __device__ static float scalar(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
};

template <>
struct GateVec<float> {
    static constexpr int kPerVec = 4;  // 4 x f32 = 16 bytes
    __device__ static void load(const float *p, float (&x)[4])
    {
        float4 u = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = u.x;
        x[1] = u.y;
        x[2] = u.z;
        x[3] = u.w;
    }
    __device__ static float scalar(const float *p) { return *p; }
};

template <typename Tin>
__global__ void __launch_bounds__(256) gate_kernel(const Tin *__restrict__ a, int64_t n, double g_min,
                                                   float *__restrict__ g)
{
    constexpr int V = GateVec<Tin>::kPerVec;
    const int64_t nvec = n / V;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        float x[V];
        GateVec<Tin>::load(a + i * V, x);
        float y[V];
#pragma unroll
        for (int j = 0; j < V; ++j)
            y[j] = gate_bounded_exact(x[j], g_min);
        float4 *out = reinterpret_cast<float4 *>(g + i * V);
#pragma unroll
        for (int j = 0; j < V / 4; ++j)
            __stcs(out + j, make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]));
    }
    // ragged tail (fewer than V elements)
    const int64_t tail = nvec * V;
    if (blockIdx.x == 0 && threadIdx.x < n - tail) {
        const int64_t i = tail + threadIdx.x;
        g[i] = gate_bounded_exact(GateVec<Tin>::scalar(a + i), g_min);
    }
}

// Per-head scaled form g = g_min * sigmoid(e^{A_h} a) on a [n_tok, H, dk] layout: the
// argument a * e^{A_h} is formed in float64 too, so the result is still one rounding from
// the fp64 value.  dk is a multiple of the vector width, so a vector never spans two heads.
template <typename Tin>
__global__ void __launch_bounds__(256) gate_heads_kernel(const Tin *__restrict__ a, int64_t nvec, int H, int dk,
                                                         const float *__restrict__ A_log, double g_min,
                                                         float *__restrict__ g)
{
    constexpr int V = GateVec<Tin>::kPerVec;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        const int head = (int)(((i * V) / dk) % H);
        const double scale = exp((double)A_log[head]);
        float x[V];
        GateVec<Tin>::load(a + i * V, x);
        float y[V];
#pragma unroll
        for (int j = 0; j < V; ++j)
            y[j] = gate_heads_exact(x[j], scale, g_min);
        float4 *out = reinterpret_cast<float4 *>(g + i * V);
#pragma unroll
        for (int j = 0; j < V / 4; ++j)
            __stcs(out + j, make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]));
    }
}

// The gate of every bfloat16 bit pattern of the pre-activation: tab[bits], or with a per-head
// scale tab[h * 65536 + bits].  The entries come from the same fp64 functions as the
// stand-alone gate kernels, so a lookup gives exactly what kda_gate_fwd (kda_gate_fwd_heads)
// returns for that input.  The chunk kernels read g this way, one table per call.
__global__ void __launch_bounds__(256) gate_table_kernel(int logsigmoid, double g_min, const float *__restrict__ A_log,
                                                         int nh, float *__restrict__ tab)
{
    const int64_t n = (int64_t)nh << 16;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float a = bf16_bits_to_float((uint16_t)(i & 0xffff));
        float g;
        if (logsigmoid)
            g = gate_logsigmoid_exact(a);
        else if (A_log)
            g = gate_heads_exact(a, exp((double)A_log[i >> 16]), g_min);
        else
            g = gate_bounded_exact(a, g_min);
        tab[i] = g;
    }
}

cudaError_t launch_gate_table(bool logsigmoid, double g_min, const float *A_log, int H, float *tab, cudaStream_t s)
{
    const int nh = (A_log && !logsigmoid) ? H : 1;
    int64_t blocks = (((int64_t)nh << 16) + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    blocks = blocks > cap ? cap : blocks;
    gate_table_kernel<<<(unsigned)blocks, 256, 0, s>>>(logsigmoid ? 1 : 0, g_min, logsigmoid ? nullptr : A_log, nh,
                                                        tab);
    return cudaGetLastError();
}

cudaError_t launch_gate_heads(const void *a, kda_dtype dt, double g_min, const float *A_log, int64_t n_tok, int H,
                              int dk, float *g, cudaStream_t s)
{
    const int per = dt == KDA_BF16 ? 8 : 4;
    const int64_t nvec = n_tok * H * dk / per;
    int64_t blocks = (nvec + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    blocks = blocks > cap ? cap : (blocks < 1 ? 1 : blocks);
    if (dt == KDA_BF16)
        gate_heads_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(a), nvec, H, dk, A_log, g_min, g);
    else
        gate_heads_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const float *>(a), nvec, H, dk,
                                                                   A_log, g_min, g);
    return cudaGetLastError();
}

cudaError_t launch_gate(const void *a, kda_dtype dt, double g_min, float *g, int64_t n, cudaStream_t s)
{
    const int per = dt == KDA_BF16 ? 8 : 4;
    const int64_t nvec = n / per;
    const int threads = 256;
    int64_t blocks = (nvec + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    if (dt == KDA_BF16)
        gate_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(a), n, g_min, g);
    else
        gate_kernel<float><<<(unsigned)blocks, threads, 0, s>>>(static_cast<const float *>(a), n, g_min, g);
    return cudaGetLastError();
}

}  // namespace kda
