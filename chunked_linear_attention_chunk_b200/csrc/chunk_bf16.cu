// chunk_bf16.cu -- K2 (intra-chunk prep) and K3 (inter-chunk scan): the bfloat16
// tensor-core chunked forward of the bounded-decay gated delta rule.
//
// Chunked form (derived from the recurrence S_t = (I - b k k^T) Diag(e^{g_t}) S_{t-1}
// + b k v^T, o_t = S_t^T q_t).  Inside a chunk of C = 64 tokens with entering state S,
// G_r = sum_{s<=r} g_s (inclusive, per key channel):
//   A_rj = beta_r sum_c k_rc k_jc e^{G_rc - G_jc}   (j < r),  T = (I + A)^{-1}
//   P_rj =        sum_c q_rc k_jc e^{G_rc - G_jc}   (j <= r)
//   W = T diag(beta) Kbar,  Utilde = T diag(beta) V,   Kbar = k e^{G}
//   U = Utilde - W S;  O = Qbar S + P U;  S <- Diag(e^{G_last}) S + Khat^T U
//   with Qbar = q e^{G} and Khat = k e^{G_last - G} (every factor <= 1).
//
// The only unbounded factor is the inverse decay 1/Gamma inside A and P ("Trillion-
// Scale MoE Multimodal Models ..." section 3.1).  With g >= g_min = -5 ("... section
// 3.2"; "Breaking Through ..." section 2.1) it is factored per 16-token column tile J
// through the tile's middle token m_J:
//   e^{G_r - G_j} = e^{G_r - G_{m_J}} * e^{G_{m_J} - G_j},  j in tile J, r in tiles >= J,
// so every operand stays below e^{40} and ALL tiles, diagonal ones included, are dense
// tensor-core products ("... section 3.3": no element-wise diagonal path).
//
// K2 runs one CTA per (chunk, batch*head), fully parallel, and writes per chunk
// W, Utilde, Qbar, Khat (bf16, C x D), P (bf16, C x C) and Gamma_C = e^{G_last} (f32)
// to the caller's workspace.  K3 runs one CTA per (value-column block, batch*head) and
// walks the chunks in order with the fp32 state block in registers.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kC = KDA_CHUNK;  // tokens per chunk (state carried every kC tokens)
constexpr int kTile = KDA_TILE;
constexpr int kTiles = kC / kTile;
constexpr int kRef = 7;        // reference token inside each 16-token tile (its middle)

// ------------------------------------------------------------------ workspace record
template <int D>
struct Rec {
    static constexpr size_t kMat = (size_t)kC * D * 2;  // one C x D bf16 matrix
    static constexpr size_t W = 0;
    static constexpr size_t U = kMat;
    static constexpr size_t Qb = 2 * kMat;
    static constexpr size_t Kh = 3 * kMat;
    static constexpr size_t P = 4 * kMat;                // C x C bf16
    static constexpr size_t Gam = P + (size_t)kC * kC * 2;  // D x f32
    static constexpr size_t Bytes = Gam + (size_t)D * 4;
    static_assert(Bytes % 128 == 0, "records stay 128-byte aligned");
};

// ------------------------------------------------------------------ K2: prep
constexpr int kPrepThreads = 256;

template <int D>
struct PrepSmem {
    static constexpr int LDB = D + 8;   // bf16 row stride (16-byte pad: conflict-free ldmatrix)
    static constexpr int LDG = D + 8;   // f32 row stride (conflict-free float2 fragment reads)
    static constexpr int LDA = kC + 1;  // f32 C x C matrices
    static constexpr int LDT = kC + 8;  // bf16 C x C matrices
    __nv_bfloat16 k[kC * LDB];
    __nv_bfloat16 q[kC * LDB];   // later: W staging
    __nv_bfloat16 v[kC * LDB];
    __nv_bfloat16 ec[kC * LDB];  // k_j e^{G_{m(j)} - G_j}; later: Utilde staging
    __nv_bfloat16 kb[kC * LDB];  // Kbar = k e^{G}
    float G[kC * LDG];
    float A[kC * LDA];
    float Tm[kC * LDA];
    __nv_bfloat16 tb[kC * LDT];  // bf16(T diag(beta))
    __nv_bfloat16 pst[kC * LDT]; // P staging
    float beta[kC];
    float X[4][kTile][kTile + 1];  // triangular-solve scratch, one per warp
};

// One 16x16 output block of the level-L block substitution, done by one warp:
//   T_IJ = -T_II * sum_{K=J}^{I-1} A_IK T_KJ
__device__ __forceinline__ void solve_offdiag_block(float *A, float *Tm, float (*X)[kTile + 1], int I, int J,
                                                    int lane)
{
    constexpr int LDA = kC + 1;
    const int cc = lane % kTile;
    const int r0 = (lane / kTile) * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rr = r0 + i;
        float s = 0.0f;
        for (int K = J; K < I; ++K) {
#pragma unroll
            for (int x = 0; x < kTile; ++x)
                s += A[(kTile * I + rr) * LDA + kTile * K + x] * Tm[(kTile * K + x) * LDA + kTile * J + cc];
        }
        X[rr][cc] = s;
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rr = r0 + i;
        float s = 0.0f;
#pragma unroll
        for (int x = 0; x < kTile; ++x)
            s += Tm[(kTile * I + rr) * LDA + kTile * I + x] * X[x][cc];
        Tm[(kTile * I + rr) * LDA + kTile * J + cc] = -s;
    }
    __syncwarp();
}

template <int D>
__global__ void __launch_bounds__(kPrepThreads, 1)
    prep_kernel(int T, int H, int NT, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ a,
                const __nv_bfloat16 *__restrict__ beta, float g_min, unsigned char *__restrict__ ws)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    using SM = PrepSmem<D>;
    SM &sm = *reinterpret_cast<SM *>(smem_raw);
    constexpr int LDB = SM::LDB, LDG = SM::LDG, LDA = SM::LDA, LDT = SM::LDT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int t0 = chunk * kC;
    const int n = min(kC, T - t0);
    unsigned char *rec = ws + ((size_t)bh * NT + chunk) * Rec<D>::Bytes;
    const int64_t rowstride = (int64_t)H * D;  // elements between consecutive tokens
    const int64_t base = (((int64_t)b * T + t0) * H + h) * D;

    // -- 1. async loads of k, q, v (zero-filled past the end of the sequence)
    for (int i = tid; i < kC * (D / 8); i += kPrepThreads) {
        const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
        const bool ok = r < n;
        const int64_t off = base + (ok ? (int64_t)r * rowstride : 0) + c8;
        cp_async_16_zfill(&sm.k[r * LDB + c8], k + off, ok);
        cp_async_16_zfill(&sm.q[r * LDB + c8], q + off, ok);
        cp_async_16_zfill(&sm.v[r * LDB + c8], v + off, ok);
    }
    cp_async_commit();
    if (tid < kC)
        sm.beta[tid] = tid < n ? __bfloat162float(beta[((int64_t)b * T + t0 + tid) * H + h]) : 0.0f;

    // -- 2. gate and inclusive cumulative log-decay; kPrepThreads/D threads per channel
    {
        constexpr int TPC = kPrepThreads / D;
        constexpr int L = kC / TPC;
        const int c = tid % D, part = tid / D;
        float acc = 0.0f;
        for (int r = part * L; r < part * L + L; ++r) {
            float g = 0.0f;
            if (r < n)
                g = gate_bounded_fast(__bfloat162float(a[base + (int64_t)r * rowstride + c]), g_min);
            acc += g;
            sm.G[r * LDG + c] = acc;
        }
        __syncthreads();
        float off = 0.0f;
        for (int p = 0; p < part; ++p)
            off += sm.G[(p * L + L - 1) * LDG + c];
        __syncthreads();
        if (part > 0)
            for (int r = part * L; r < part * L + L; ++r)
                sm.G[r * LDG + c] += off;
    }
    cp_async_wait<0>();
    __syncthreads();

    // -- 3. elementwise decay factors; Qbar, Khat, Gamma_C go straight to the workspace
    {
        __nv_bfloat16 *gQb = reinterpret_cast<__nv_bfloat16 *>(rec + Rec<D>::Qb);
        __nv_bfloat16 *gKh = reinterpret_cast<__nv_bfloat16 *>(rec + Rec<D>::Kh);
        for (int i = tid; i < kC * (D / 8); i += kPrepThreads) {
            const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
            const int m = (r / kTile) * kTile + kRef;
            const uint4 ku = *reinterpret_cast<const uint4 *>(&sm.k[r * LDB + c8]);
            const uint4 qu = *reinterpret_cast<const uint4 *>(&sm.q[r * LDB + c8]);
            const uint32_t kw[4] = {ku.x, ku.y, ku.z, ku.w};
            const uint32_t qw[4] = {qu.x, qu.y, qu.z, qu.w};
            uint32_t ec[4], kb[4], qb[4], kh[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int c = c8 + 2 * p;
                const float2 kk = unpack_bf16x2(kw[p]), qq = unpack_bf16x2(qw[p]);
                const float G0 = sm.G[r * LDG + c], G1 = sm.G[r * LDG + c + 1];
                const float M0 = sm.G[m * LDG + c], M1 = sm.G[m * LDG + c + 1];
                const float L0 = sm.G[(kC - 1) * LDG + c], L1 = sm.G[(kC - 1) * LDG + c + 1];
                const float e0 = __expf(G0), e1 = __expf(G1);
                ec[p] = pack_bf16x2(kk.x * __expf(M0 - G0), kk.y * __expf(M1 - G1));
                kb[p] = pack_bf16x2(kk.x * e0, kk.y * e1);
                qb[p] = pack_bf16x2(qq.x * e0, qq.y * e1);
                kh[p] = pack_bf16x2(kk.x * __expf(L0 - G0), kk.y * __expf(L1 - G1));
            }
            *reinterpret_cast<uint4 *>(&sm.ec[r * LDB + c8]) = make_uint4(ec[0], ec[1], ec[2], ec[3]);
            *reinterpret_cast<uint4 *>(&sm.kb[r * LDB + c8]) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
            *reinterpret_cast<uint4 *>(&gQb[r * D + c8]) = make_uint4(qb[0], qb[1], qb[2], qb[3]);
            *reinterpret_cast<uint4 *>(&gKh[r * D + c8]) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
        }
        float *gGam = reinterpret_cast<float *>(rec + Rec<D>::Gam);
        for (int c = tid; c < D; c += kPrepThreads)
            gGam[c] = __expf(sm.G[(kC - 1) * LDG + c]);
        for (int i = tid; i < kC * kC; i += kPrepThreads)
            sm.pst[(i / kC) * LDT + (i % kC)] = __float2bfloat16(0.0f);
    }
    __syncthreads();

    // -- 4. dense tile products A and P: one warp per (row tile I, column tile J <= I).
    //       Row operands k_r e^{G_r - G_{m_J}} and q_r e^{G_r - G_{m_J}} are built in
    //       registers from G; the column operand is ec (tile J, referenced at m_J).
    {
        const int grp = lane >> 2, tq = lane & 3;
        for (int pidx = warp; pidx < kTiles * (kTiles + 1) / 2; pidx += kPrepThreads / 32) {
            int I = 0, J = pidx;
            while (J > I) {  // pidx -> (I, J): 0:(0,0) 1:(1,0) 2:(1,1) 3:(2,0) ...
                J -= I + 1;
                ++I;
            }
            const int m = J * kTile + kRef;
            float accA[2][4] = {}, accP[2][4] = {};
#pragma unroll 2
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t ak[4], aq[4];
#pragma unroll
                for (int reg = 0; reg < 4; ++reg) {
                    const int r = I * kTile + grp + 8 * (reg & 1);
                    const int c = ks * 16 + 2 * tq + 8 * (reg >> 1);
                    const float2 Gr = *reinterpret_cast<const float2 *>(&sm.G[r * LDG + c]);
                    const float2 Gm = *reinterpret_cast<const float2 *>(&sm.G[m * LDG + c]);
                    const float e0 = __expf(Gr.x - Gm.x), e1 = __expf(Gr.y - Gm.y);
                    const float2 kk = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(&sm.k[r * LDB + c]));
                    const float2 qq = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(&sm.q[r * LDB + c]));
                    ak[reg] = pack_bf16x2(kk.x * e0, kk.y * e1);
                    aq[reg] = pack_bf16x2(qq.x * e0, qq.y * e1);
                }
                uint32_t bf[4];
                {
                    const int mi = lane >> 3;
                    const int row = J * kTile + (lane & 7) + 8 * (mi >> 1);
                    const int col = ks * 16 + 8 * (mi & 1);
                    ldmatrix_x4(bf, &sm.ec[row * LDB + col]);
                }
                const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
                mma_bf16_16816(accA[0], ak, b0);
                mma_bf16_16816(accA[1], ak, b1);
                mma_bf16_16816(accP[0], aq, b0);
                mma_bf16_16816(accP[1], aq, b1);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = I * kTile + grp + 8 * (e >> 1);
                    const int j = J * kTile + nt * 8 + 2 * tq + (e & 1);
                    const bool lowA = I > J || j < r, lowP = I > J || j <= r;
                    sm.A[r * LDA + j] = lowA ? sm.beta[r] * accA[nt][e] : 0.0f;
                    sm.pst[r * LDT + j] = __float2bfloat16(lowP ? accP[nt][e] : 0.0f);
                }
        }
    }
    __syncthreads();

    // -- 5. T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution, then block
    //       substitution level by level.
    if (warp < kTiles && lane < kTile) {
        const int I = warp, c = lane;
        float x[kTile];
#pragma unroll
        for (int r = 0; r < kTile; ++r)
            x[r] = r == c ? 1.0f : 0.0f;
#pragma unroll
        for (int r = 1; r < kTile; ++r) {
            float s = 0.0f;
#pragma unroll
            for (int y = 0; y < r; ++y)
                s += sm.A[(I * kTile + r) * LDA + I * kTile + y] * x[y];
            if (r > c)
                x[r] = -s;
        }
#pragma unroll
        for (int r = 0; r < kTile; ++r)
            sm.Tm[(I * kTile + r) * LDA + I * kTile + c] = x[r];
    }
    // upper blocks of T are zero
    for (int i = tid; i < kC * kC; i += kPrepThreads) {
        const int r = i / kC, j = i % kC;
        if (j / kTile > r / kTile)
            sm.Tm[r * LDA + j] = 0.0f;
    }
    __syncthreads();
    for (int lvl = 1; lvl < kTiles; ++lvl) {
        if (warp < kTiles - lvl)
            solve_offdiag_block(sm.A, sm.Tm, sm.X[warp], warp + lvl, warp, lane);
        __syncthreads();
    }
    // bf16(T diag(beta)); P staging -> workspace
    for (int i = tid; i < kC * kC; i += kPrepThreads) {
        const int r = i / kC, j = i % kC;
        sm.tb[r * LDT + j] = __float2bfloat16(sm.Tm[r * LDA + j] * sm.beta[j]);
    }
    {
        __nv_bfloat16 *gP = reinterpret_cast<__nv_bfloat16 *>(rec + Rec<D>::P);
        for (int i = tid; i < kC * (kC / 8); i += kPrepThreads) {
            const int r = i / (kC / 8), c8 = (i % (kC / 8)) * 8;
            *reinterpret_cast<uint4 *>(&gP[r * kC + c8]) = *reinterpret_cast<const uint4 *>(&sm.pst[r * LDT + c8]);
        }
    }
    __syncthreads();

    // -- 6. W = (T beta) Kbar, Utilde = (T beta) V: warp -> (row tile I, half of D)
    {
        const int grp = lane >> 2, tq = lane & 3;
        const int I = warp % kTiles, nh = warp / kTiles;
        constexpr int NTL = D / 16;  // n8 tiles per warp (half of D)
        float accW[NTL][4] = {}, accU[NTL][4] = {};
        for (int ks = 0; ks <= I; ++ks) {
            uint32_t af[4];
            {
                const int mi = lane >> 3;
                const int row = I * kTile + (lane & 7) + 8 * (mi & 1);
                const int col = ks * 16 + 8 * (mi >> 1);
                ldmatrix_x4(af, &sm.tb[row * LDT + col]);
            }
#pragma unroll
            for (int np = 0; np < NTL / 2; ++np) {
                const int mi = lane >> 3;
                const int row = ks * 16 + (lane & 7) + 8 * (mi & 1);
                const int col = nh * (D / 2) + np * 16 + 8 * (mi >> 1);
                uint32_t bk[4], bv[4];
                ldmatrix_x4_trans(bk, &sm.kb[row * LDB + col]);
                ldmatrix_x4_trans(bv, &sm.v[row * LDB + col]);
                const uint32_t k0[2] = {bk[0], bk[1]}, k1[2] = {bk[2], bk[3]};
                const uint32_t v0[2] = {bv[0], bv[1]}, v1[2] = {bv[2], bv[3]};
                mma_bf16_16816(accW[2 * np], af, k0);
                mma_bf16_16816(accW[2 * np + 1], af, k1);
                mma_bf16_16816(accU[2 * np], af, v0);
                mma_bf16_16816(accU[2 * np + 1], af, v1);
            }
        }
        // stage in shared memory (q and ec are free now), then coalesced copies out
#pragma unroll
        for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = I * kTile + grp + 8 * hh;
                const int c = nh * (D / 2) + nt * 8 + 2 * tq;
                *reinterpret_cast<uint32_t *>(&sm.q[r * LDB + c]) =
                    pack_bf16x2(accW[nt][2 * hh], accW[nt][2 * hh + 1]);
                *reinterpret_cast<uint32_t *>(&sm.ec[r * LDB + c]) =
                    pack_bf16x2(accU[nt][2 * hh], accU[nt][2 * hh + 1]);
            }
    }
    __syncthreads();
    {
        __nv_bfloat16 *gW = reinterpret_cast<__nv_bfloat16 *>(rec + Rec<D>::W);
        __nv_bfloat16 *gU = reinterpret_cast<__nv_bfloat16 *>(rec + Rec<D>::U);
        for (int i = tid; i < kC * (D / 8); i += kPrepThreads) {
            const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
            *reinterpret_cast<uint4 *>(&gW[r * D + c8]) = *reinterpret_cast<const uint4 *>(&sm.q[r * LDB + c8]);
            *reinterpret_cast<uint4 *>(&gU[r * D + c8]) = *reinterpret_cast<const uint4 *>(&sm.ec[r * LDB + c8]);
        }
    }
}

// ------------------------------------------------------------------ K3: scan
constexpr int kScanThreads = 128;  // 4 warps: warp w owns chunk rows [16w, 16w+16)

template <int D, int BV>
struct ScanStage {
    static constexpr int LDB = D + 8;
    static constexpr int LDP = kC + 8;
    static constexpr int LDU = BV + 8;
    __nv_bfloat16 W[kC * LDB];
    __nv_bfloat16 Qb[kC * LDB];
    __nv_bfloat16 Kh[kC * LDB];
    __nv_bfloat16 P[kC * LDP];
    __nv_bfloat16 U[kC * LDU];
    float gam[D];
};

template <int D, int BV>
struct ScanSmem {
    static constexpr int LDU = BV + 8;
    ScanStage<D, BV> st[2];
    __nv_bfloat16 Sb[D * LDU];  // current state block, bf16 (B operand)
    __nv_bfloat16 Uc[kC * LDU]; // corrected U = Utilde - W S, bf16 (B operand)
};

template <int D, int BV>
__device__ __forceinline__ void scan_load_stage(ScanStage<D, BV> &st, const unsigned char *rec, int col0, int tid)
{
    constexpr int LDB = ScanStage<D, BV>::LDB, LDP = ScanStage<D, BV>::LDP, LDU = ScanStage<D, BV>::LDU;
    const __nv_bfloat16 *gW = reinterpret_cast<const __nv_bfloat16 *>(rec + Rec<D>::W);
    const __nv_bfloat16 *gQ = reinterpret_cast<const __nv_bfloat16 *>(rec + Rec<D>::Qb);
    const __nv_bfloat16 *gK = reinterpret_cast<const __nv_bfloat16 *>(rec + Rec<D>::Kh);
    const __nv_bfloat16 *gP = reinterpret_cast<const __nv_bfloat16 *>(rec + Rec<D>::P);
    const __nv_bfloat16 *gU = reinterpret_cast<const __nv_bfloat16 *>(rec + Rec<D>::U);
    const float *gG = reinterpret_cast<const float *>(rec + Rec<D>::Gam);
    for (int i = tid; i < kC * (D / 8); i += kScanThreads) {
        const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
        cp_async_16(&st.W[r * LDB + c8], gW + r * D + c8);
        cp_async_16(&st.Qb[r * LDB + c8], gQ + r * D + c8);
        cp_async_16(&st.Kh[r * LDB + c8], gK + r * D + c8);
    }
    for (int i = tid; i < kC * (kC / 8); i += kScanThreads) {
        const int r = i / (kC / 8), c8 = (i % (kC / 8)) * 8;
        cp_async_16(&st.P[r * LDP + c8], gP + r * kC + c8);
    }
    for (int i = tid; i < kC * (BV / 8); i += kScanThreads) {
        const int r = i / (BV / 8), c8 = (i % (BV / 8)) * 8;
        cp_async_16(&st.U[r * LDU + c8], gU + r * D + col0 + c8);
    }
    for (int i = tid; i < D / 4; i += kScanThreads)
        cp_async_16(&st.gam[4 * i], gG + 4 * i);
}

template <int D, int BV>
__global__ void __launch_bounds__(kScanThreads, 1)
    scan_kernel(int T, int H, int NT, const unsigned char *__restrict__ ws, const float *__restrict__ S0,
                __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    using SM = ScanSmem<D, BV>;
    SM &sm = *reinterpret_cast<SM *>(smem_raw);
    constexpr int LDB = ScanStage<D, BV>::LDB, LDP = ScanStage<D, BV>::LDP, LDU = SM::LDU;
    constexpr int MT = D / 64;   // 16-row state tiles per warp (warp owns D/4 state rows)
    constexpr int NTL = BV / 8;  // n8 tiles across the value block
    constexpr int KS = D / 16;   // k16 steps over the key dim
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = lane >> 2, tq = lane & 3;
    const int col0 = blockIdx.x * BV, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const unsigned char *recs = ws + (size_t)bh * NT * Rec<D>::Bytes;
    const int srow0 = warp * (D / 4);

    // state block in registers (C-fragment layout): rows srow0 + 16 mt + grp (+8)
    float S[MT][NTL][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = srow0 + 16 * mt + grp + 8 * hh;
                const int c = col0 + nt * 8 + 2 * tq;
                float2 s = make_float2(0.0f, 0.0f);
                if (S0)
                    s = *reinterpret_cast<const float2 *>(&S0[((size_t)bh * D + r) * D + c]);
                S[mt][nt][2 * hh] = s.x;
                S[mt][nt][2 * hh + 1] = s.y;
                *reinterpret_cast<uint32_t *>(&sm.Sb[r * LDU + nt * 8 + 2 * tq]) = pack_bf16x2(s.x, s.y);
            }

    scan_load_stage<D, BV>(sm.st[0], recs, col0, tid);
    cp_async_commit();

    for (int c = 0; c < NT; ++c) {
        if (c + 1 < NT) {
            scan_load_stage<D, BV>(sm.st[(c + 1) & 1], recs + (size_t)(c + 1) * Rec<D>::Bytes, col0, tid);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        ScanStage<D, BV> &st = sm.st[c & 1];

        // (1) X = W S and Y = Qbar S for chunk rows [16 warp, +16)
        float X[NTL][4] = {}, Y[NTL][4] = {};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t aw[4], aq[4];
            {
                const int mi = lane >> 3;
                const int row = warp * 16 + (lane & 7) + 8 * (mi & 1);
                const int col = ks * 16 + 8 * (mi >> 1);
                ldmatrix_x4(aw, &st.W[row * LDB + col]);
                ldmatrix_x4(aq, &st.Qb[row * LDB + col]);
            }
#pragma unroll
            for (int np = 0; np < NTL / 2; ++np) {
                const int mi = lane >> 3;
                const int row = ks * 16 + (lane & 7) + 8 * (mi & 1);
                const int col = np * 16 + 8 * (mi >> 1);
                uint32_t bs[4];
                ldmatrix_x4_trans(bs, &sm.Sb[row * LDU + col]);
                const uint32_t s0[2] = {bs[0], bs[1]}, s1[2] = {bs[2], bs[3]};
                mma_bf16_16816(X[2 * np], aw, s0);
                mma_bf16_16816(X[2 * np + 1], aw, s1);
                mma_bf16_16816(Y[2 * np], aq, s0);
                mma_bf16_16816(Y[2 * np + 1], aq, s1);
            }
        }
        // (2) U = Utilde - X -> Uc (bf16)
#pragma unroll
        for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 16 + grp + 8 * hh;
                const int cc = nt * 8 + 2 * tq;
                const float2 ut = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(&st.U[r * LDU + cc]));
                *reinterpret_cast<uint32_t *>(&sm.Uc[r * LDU + cc]) =
                    pack_bf16x2(ut.x - X[nt][2 * hh], ut.y - X[nt][2 * hh + 1]);
            }
        __syncthreads();

        // (3) B fragments of U (tokens x value block), shared by P U and Khat^T U
        uint32_t bu[kC / 16][NTL][2];
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
#pragma unroll
            for (int np = 0; np < NTL / 2; ++np) {
                const int mi = lane >> 3;
                const int row = ks * 16 + (lane & 7) + 8 * (mi & 1);
                const int col = np * 16 + 8 * (mi >> 1);
                uint32_t r4[4];
                ldmatrix_x4_trans(r4, &sm.Uc[row * LDU + col]);
                bu[ks][2 * np][0] = r4[0];
                bu[ks][2 * np][1] = r4[1];
                bu[ks][2 * np + 1][0] = r4[2];
                bu[ks][2 * np + 1][1] = r4[3];
            }
        // O = Y + P U (P is lower triangular: k-steps 0..warp)
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
            if (ks > warp)
                break;
            uint32_t ap[4];
            const int mi = lane >> 3;
            const int row = warp * 16 + (lane & 7) + 8 * (mi & 1);
            const int col = ks * 16 + 8 * (mi >> 1);
            ldmatrix_x4(ap, &st.P[row * LDP + col]);
#pragma unroll
            for (int nt = 0; nt < NTL; ++nt)
                mma_bf16_16816(Y[nt], ap, bu[ks][nt]);
        }
        {
            const int tbase = c * kC + warp * 16;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int t = tbase + grp + 8 * hh;
                if (t < T) {
                    __nv_bfloat16 *orow = o + (((int64_t)b * T + t) * H + h) * D + col0;
#pragma unroll
                    for (int nt = 0; nt < NTL; ++nt)
                        *reinterpret_cast<uint32_t *>(&orow[nt * 8 + 2 * tq]) =
                            pack_bf16x2(Y[nt][2 * hh], Y[nt][2 * hh + 1]);
                }
            }
        }
        // (4) S <- Diag(Gamma_C) S + Khat^T U
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const float g0 = st.gam[srow0 + 16 * mt + grp], g1 = st.gam[srow0 + 16 * mt + grp + 8];
#pragma unroll
            for (int nt = 0; nt < NTL; ++nt) {
                S[mt][nt][0] *= g0;
                S[mt][nt][1] *= g0;
                S[mt][nt][2] *= g1;
                S[mt][nt][3] *= g1;
            }
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks) {
                uint32_t ak[4];
                const int mi = lane >> 3;
                const int row = ks * 16 + (lane & 7) + 8 * (mi >> 1);   // token
                const int col = srow0 + 16 * mt + 8 * (mi & 1);        // key channel
                ldmatrix_x4_trans(ak, &st.Kh[row * LDB + col]);
#pragma unroll
                for (int nt = 0; nt < NTL; ++nt)
                    mma_bf16_16816(S[mt][nt], ak, bu[ks][nt]);
            }
        }
        // (5) bf16 copy of the new state for the next chunk
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = srow0 + 16 * mt + grp + 8 * hh;
                    *reinterpret_cast<uint32_t *>(&sm.Sb[r * LDU + nt * 8 + 2 * tq]) =
                        pack_bf16x2(S[mt][nt][2 * hh], S[mt][nt][2 * hh + 1]);
                }
        __syncthreads();
    }

    if (S_T) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NTL; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = srow0 + 16 * mt + grp + 8 * hh;
                    const int cc = col0 + nt * 8 + 2 * tq;
                    *reinterpret_cast<float2 *>(&S_T[((size_t)bh * D + r) * D + cc]) =
                        make_float2(S[mt][nt][2 * hh], S[mt][nt][2 * hh + 1]);
                }
    }
}

template <int D>
cudaError_t launch_bf16_d(int B, int T, int H, const void *q, const void *k, const void *v, const void *a,
                          const void *beta, float g_min, const float *S0, void *o, float *S_T, void *ws,
                          cudaStream_t s)
{
    constexpr int BV = 32;
    const int NT = (T + kC - 1) / kC;
    const int BH = B * H;
    unsigned char *w = static_cast<unsigned char *>(ws);
    {
        const size_t smem = sizeof(PrepSmem<D>);
        cudaError_t e = cudaFuncSetAttribute(prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        prep_kernel<D><<<dim3(NT, BH), kPrepThreads, smem, s>>>(
            T, H, NT, static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
            static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(a),
            static_cast<const __nv_bfloat16 *>(beta), g_min, w);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    {
        const size_t smem = sizeof(ScanSmem<D, BV>);
        cudaError_t e =
            cudaFuncSetAttribute(scan_kernel<D, BV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        scan_kernel<D, BV><<<dim3(D / BV, BH), kScanThreads, smem, s>>>(
            T, H, NT, w, S0, static_cast<__nv_bfloat16 *>(o), S_T);
        return cudaGetLastError();
    }
}

}  // namespace

size_t chunk_bf16_workspace(int B, int T, int H, int D)
{
    const size_t NT = ((size_t)T + kC - 1) / kC;
    const size_t rec = D == 64 ? Rec<64>::Bytes : Rec<128>::Bytes;
    return (size_t)B * H * NT * rec;
}

cudaError_t launch_chunk_bf16(int B, int T, int H, int D, const void *q, const void *k, const void *v,
                              const void *a, const void *beta, float g_min, const float *S0, void *o,
                              float *S_T, void *workspace, cudaStream_t s)
{
    if (D == 64)
        return launch_bf16_d<64>(B, T, H, q, k, v, a, beta, g_min, S0, o, S_T, workspace, s);
    return launch_bf16_d<128>(B, T, H, q, k, v, a, beta, g_min, S0, o, S_T, workspace, s);
}

}  // namespace kda
