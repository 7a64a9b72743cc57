// chunk_bf16.cu -- K2 (intra-chunk prep) and K3 (inter-chunk scan): the bfloat16
// tensor-core chunked forward of the bounded-decay gated delta rule.
//
// Chunked form (derived from the recurrence S_t = (I - b k k^T) Diag(e^{g_t}) S_{t-1}
// + b k v^T, o_t = S_t^T q_t).  Inside a chunk of C = 64 tokens with entering state S,
// G_r = sum_{s<=r} g_s (inclusive, per key channel):
//   A_rj = beta_r sum_c k_rc k_jc e^{G_rc - G_jc}   (j < r),  T = (I + A)^{-1}
//   P_rj =        sum_c q_rc k_jc e^{G_rc - G_jc}   (j <= r)
//   W = T diag(beta) Kbar,  Utilde = T diag(beta) V,   Kbar = k e^{G}
//   U = Utilde - W S;  O = Qbar S + P U;  S' = Diag(e^{G_last}) S + Khat^T U
//   with Qbar = q e^{G} and Khat = k e^{G_last - G} (every factor <= 1).
// Substituting U once, per chunk, gives the form the scan walks with a single tensor-core
// round per chunk:
//   S' = Diag(Gamma) S - N S + Bm,   O = Q' S + O',
//   N = Khat^T W (D x D),  Bm = Khat^T Utilde (D x D),  Q' = Qbar - P W,  O' = P Utilde.
//
// The only unbounded factor is the inverse decay 1/Gamma inside A and P ("Trillion-
// Scale MoE Multimodal Models ..." section 3.1).  With g >= g_min = -5 ("... section
// 3.2"; "Breaking Through ..." section 2.1) it is factored per 16-token column tile J
// through the tile's middle token m_J:
//   e^{G_r - G_j} = e^{G_r - G_{m_J}} * e^{G_{m_J} - G_j},  j in tile J, r in tiles >= J,
// so every operand stays below e^{40} and ALL tiles, diagonal ones included, are dense
// tensor-core products ("... section 3.3": no element-wise diagonal path).
//
// K2 (prep) runs one CTA per (chunk, batch*head), two CTAs per SM.  The 16-token tile
// products A and P are warp-level MMAs; the dense contractions W | Utilde = (T beta)
// [Kbar | V], then Khat^T [W | Utilde] and P [W | Utilde], are 5th-generation tensor
// core MMAs (tcgen05) with fp32 accumulators in tensor memory.  It writes one record per
// chunk (N, Q', Gamma, Bm, O') to the caller's workspace in the swizzled layouts the
// tensor core reads, so a linear bulk copy is directly an MMA operand.
// K3 (scan) runs one CTA per (32-column block of the value dim, batch*head); a producer
// warp streams the records through a 3-stage mbarrier pipeline with bulk copies, and per
// chunk one tcgen05 round computes [N S, Q' S] while four consumer warps, one TMEM lane
// (= one state row or chunk row) per thread, keep the fp32 state block in registers.  With
// more such chains than SMs, one CTA takes two blocks (eight consumer warps, an N = 64
// round, two stages) so that all chains run in one wave.
#include <cudaTypedefs.h>

#include <algorithm>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "tcgen05.cuh"

namespace kda {

namespace {

constexpr int kC = KDA_CHUNK;  // tokens per chunk (state carried every kC tokens)
constexpr int kTile = KDA_TILE;
constexpr int kTiles = kC / kTile;
constexpr int kRef = 7;   // reference token inside each 16-token tile (its middle)
constexpr int kBV = 32;   // value columns per scan CTA

// ------------------------------------------------------------------ workspace record
// One record per (batch*head, chunk):
//   Nm   N = Khat^T W, D x D, K-major 128-byte swizzle (row = key channel)
//   Qp   Q' = Qbar - P W, 64 x D, K-major 128-byte swizzle (row = token)
//   Gam  Gamma = e^{G_last}, D floats
//   then, per 32-column value block b: Bm[:, block b] (D x 32) and O'[:, block b]
//   (64 x 32), both MN-major 64-byte swizzle.
// An M = 128 MMA over Nm (D = 64) or Qp reads 64 rows past the operand: those rows fall on
// the following fields of the same record and only feed accumulator lanes never read.
template <int D>
struct Rec {
    static constexpr uint32_t Nm = 0;
    static constexpr uint32_t Qp = (uint32_t)D * D * 2;
    static constexpr uint32_t Gam = Qp + (uint32_t)kC * D * 2;
    static constexpr uint32_t Shared = Gam + (uint32_t)D * 4;  // bytes every scan CTA needs
    static constexpr uint32_t BmBlk = (uint32_t)D * kBV * 2;
    static constexpr uint32_t OpBlk = (uint32_t)kC * kBV * 2;
    static constexpr uint32_t Blk = BmBlk + OpBlk;             // per value block
    static constexpr uint32_t Bytes = Shared + (uint32_t)(D / kBV) * Blk;
    static_assert(Bytes % 128 == 0 && Shared % 16 == 0 && Blk % 16 == 0, "record alignment");
    static_assert(Qp % 1024 == 0, "swizzle atoms are 1024-byte aligned");
    // the padded rows of the scan's M = 128 reads stay inside a stage
    static_assert(Qp + (D / 64 - 1) * kC * 128 + 2 * kC * 128 <= Shared + Blk, "padded rows in bounds");
};

// ------------------------------------------------------------------ where chunks live
// Regular batch: B sequences of T tokens, record row (b*H + h) of NT = ceil(T/64) records.
// Packed variable-length batch: N sequences back to back on one token axis of T tokens,
// sequence s spanning [cu[s], cu[s+1]); its chunks (ceil(len/64), none crossing into the
// next sequence) are records choff[s] .. choff[s+1]-1 of head h's row of NT records.
struct SeqMap {
    const int32_t *cu = nullptr;     // packed batch: N + 1 token offsets; null for a regular batch
    const int32_t *choff = nullptr;  // packed batch: N + 1 chunk offsets (prefix sums of ceil(len/64))
    int nseq = 0;                    // B or N
    int T = 0;                       // tokens per sequence (regular) or on the packed axis
    int NT = 0;                      // records per row
    int64_t nrec = 0;                // records the workspace holds
    int64_t ntok = 0;                // tokens on the flattened token axis (B * T, or T packed)
};

struct ChunkLoc {
    int64_t tok0;  // first token of the chunk on the flattened token axis (b*T + t)
    int n;         // tokens of the chunk that exist (1..64)
    size_t rec;    // record index
    int h;
    bool live;
};

// The chunk of prep CTA (x, y): regular grid (NT, B*H), packed (NT, H).
__device__ __forceinline__ ChunkLoc locate_chunk(const SeqMap &m, int H, int x, int y)
{
    ChunkLoc L;
    if (!m.cu) {
        const int chunk = x, bh = y;
        const int b = bh / H, t0 = chunk * kC;
        L.tok0 = (int64_t)b * m.T + t0;
        L.n = min(kC, m.T - t0);
        L.rec = (size_t)bh * m.NT + chunk;
        L.h = bh % H;
        L.live = true;
        return L;
    }
    const int g = x;
    L.h = y;
    L.live = g < m.choff[m.nseq];
    if (!L.live)
        return L;
    int lo = 0, hi = m.nseq;  // the sequence s with choff[s] <= g < choff[s+1]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (m.choff[mid] <= g)
            lo = mid;
        else
            hi = mid;
    }
    const int c = g - m.choff[lo];
    L.tok0 = (int64_t)m.cu[lo] + (int64_t)c * kC;
    L.n = (int)min((int64_t)kC, (int64_t)m.cu[lo + 1] - L.tok0);
    L.rec = (size_t)L.h * m.NT + g;
    return L;
}

struct SeqLoc {
    int64_t tok0;  // first token of the sequence on the flattened token axis
    int len;       // its tokens
    int nchunks;
    size_t rec0;   // its first record
    int sh;        // state index (sequence * H + h)
    int h;
};

// The sequence of scan CTA row blockIdx.y = sequence * H + h (both layouts).
__device__ __forceinline__ SeqLoc locate_seq(const SeqMap &m, int H)
{
    SeqLoc L;
    L.sh = blockIdx.y;
    const int sq = L.sh / H;
    L.h = L.sh % H;
    if (!m.cu) {
        L.tok0 = (int64_t)sq * m.T;
        L.len = m.T;
        L.nchunks = m.NT;
        L.rec0 = (size_t)L.sh * m.NT;
    } else {
        L.tok0 = m.cu[sq];
        L.len = m.cu[sq + 1] - m.cu[sq];
        L.nchunks = m.choff[sq + 1] - m.choff[sq];
        L.rec0 = (size_t)L.h * m.NT + m.choff[sq];
    }
    return L;
}

// ------------------------------------------------------------------ K2: prep
constexpr int kPrepWarps = 10;  // one per 16x16 tile pair of the chunk
constexpr int kPrepThreads = kPrepWarps * 32;
// The first eight warps take the roles tied to the layout: two TMEM lane quarters x two
// column halves in the epilogues, two threads per key channel in the cumulative sum.
constexpr int kCoreThreads = 256;
static_assert(kPrepWarps >= 8 && kPrepWarps >= kTiles * (kTiles + 1) / 2, "prep warp roles");

template <int D>
struct PrepLayout {
    static constexpr uint32_t kMat = (uint32_t)kC * D * 2;  // one 64 x D bf16 operand
    // token-major operands (row = token, MN-major 128-byte swizzle by 64-channel block)
    static constexpr uint32_t RQ = 0;          // q -> Qr = q E -> Qbar
    static constexpr uint32_t RK = RQ + kMat;  // k -> Kr = k E -> Kbar   } adjacent: the B
    static constexpr uint32_t RV = RK + kMat;  // v                       } operand [Kbar | V]
    static constexpr uint32_t RX = RV + kMat;  // a -> Ec = k / E -> Khat
    static constexpr uint32_t RP = RX + kMat;  // P, K-major 128-byte swizzle (64 x 64)
    // G: fp32 [64][D] -> A [64][65] | T [64][65] | solve scratch -> T beta -> [W | Utilde]
    static constexpr uint32_t RG = RP + (uint32_t)kC * kC * 2;
    static constexpr uint32_t kGBytes = 2u * kC * D * 2 > (uint32_t)kC * D * 4 ? 2u * kC * D * 2 : (uint32_t)kC * D * 4;
    static constexpr uint32_t kSolveBytes = 2u * kC * (kC + 1) * 4;
    static constexpr uint32_t kRGBytes = ((kGBytes > kSolveBytes ? kGBytes : kSolveBytes) + 1023) / 1024 * 1024;
    static constexpr uint32_t RA = RG;                                // f32 [64][65]; its upper
    static constexpr uint32_t RT = RG + (uint32_t)kC * (kC + 1) * 4;  // blocks hold the solve scratch
    // small tables
    static constexpr uint32_t RBeta = RG + kRGBytes;       // f32 [64]
    // scale tables as bf16 hi / lo pairs (hi [4][D], then lo [4][D]): x * (hi + lo) in two
    // packed bf16 operations with one effective rounding
    static constexpr uint32_t REm = RBeta + kC * 4;        // e^{G_{m_I}}
    static constexpr uint32_t REl = REm + kTiles * D * 4;  // e^{G_last - G_{m_I}}
    static constexpr uint32_t RDd = REl + kTiles * D * 4;  // bf16 [6][D]  e^{G_{m_I} - G_{m_J}}
    static constexpr uint32_t RBar = RDd + 6 * D * 2;      // mbarriers: round 1, U1..U4, a, q|k|v
    static constexpr uint32_t RTmem = RBar + 7 * 8;
    static constexpr uint32_t Bytes = RTmem + 8;
    static_assert(RG % 1024 == 0 && RP % 1024 == 0, "operand alignment");
    // two CTAs per SM: 228 KB of shared memory per SM, 1 KB of it reserved per CTA
    static_assert(2 * (Bytes + 1024) <= 233472, "two prep CTAs fit one SM");
};

// 16-byte chunk address of (token r, channels c8..c8+7) in a token-major operand.
__device__ __forceinline__ uint32_t tok_off(int r, int c8) { return tc::mnmaj_sw128(r, c8, kC); }

// One 16x16 output block of the block substitution, by one warp with tf32 tensor-core
// MMAs:  X = diag(rs_I) sum_{K=J}^{I-1} A_IK T_KJ,  T_IJ = -T_II X  (rs = the row scale, or 1
// without it).  A and T are fp32 [64][LD]; X goes through a 16x16 scratch (row stride LD) to
// turn the accumulator layout into an operand layout.
template <int LD>
__device__ __forceinline__ void solve_block_tf32(const float *A, float *Tm, float *X, int I, int J, int lane,
                                                 const float *rs = nullptr)
{
    const int g = lane >> 2, t = lane & 3;
    float acc[2][4] = {};
    auto product = [&](const float *Am, int arow, int acol, const float *Bm, int brow, int bcol, int bld) {
#pragma unroll
        for (int kk = 0; kk < kTile; kk += 8) {
            uint32_t af[4];
            af[0] = to_tf32(Am[(arow + g) * LD + acol + kk + t]);
            af[1] = to_tf32(Am[(arow + g + 8) * LD + acol + kk + t]);
            af[2] = to_tf32(Am[(arow + g) * LD + acol + kk + t + 4]);
            af[3] = to_tf32(Am[(arow + g + 8) * LD + acol + kk + t + 4]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bf[2];
                bf[0] = to_tf32(Bm[(brow + kk + t) * bld + bcol + nt * 8 + g]);
                bf[1] = to_tf32(Bm[(brow + kk + t + 4) * bld + bcol + nt * 8 + g]);
                mma_tf32_1688(acc[nt], af, bf);
            }
        }
    };
    for (int K = J; K < I; ++K)
        product(A, I * kTile, K * kTile, Tm, K * kTile, J * kTile, LD);
    const float s0 = rs ? rs[I * kTile + g] : 1.0f, s1 = rs ? rs[I * kTile + g + 8] : 1.0f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        X[g * LD + nt * 8 + 2 * t] = s0 * acc[nt][0];
        X[g * LD + nt * 8 + 2 * t + 1] = s0 * acc[nt][1];
        X[(g + 8) * LD + nt * 8 + 2 * t] = s1 * acc[nt][2];
        X[(g + 8) * LD + nt * 8 + 2 * t + 1] = s1 * acc[nt][3];
        acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
    }
    __syncwarp();
    product(Tm, I * kTile, I * kTile, X, 0, 0, LD);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        float *o = Tm + (I * kTile + g) * LD + J * kTile + nt * 8 + 2 * t;
        o[0] = -acc[nt][0];
        o[1] = -acc[nt][1];
        o[8 * LD] = -acc[nt][2];
        o[8 * LD + 1] = -acc[nt][3];
    }
}

// Multiply 8 packed bf16 x by scalars given as bf16 hi + lo: rn(x hi + rn(x lo)), which is x (hi
// + lo) rounded once up to a 2^-17 relative term (a fused packed multiply-add after a packed
// multiply).
__device__ __forceinline__ uint4 mul8_hilo(uint4 x, uint4 hi, uint4 lo)
{
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, hs[4] = {hi.x, hi.y, hi.z, hi.w}, ls[4] = {lo.x, lo.y, lo.z, lo.w};
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 xv = *reinterpret_cast<const __nv_bfloat162 *>(&xs[i]);
        const __nv_bfloat162 t = __hmul2(xv, *reinterpret_cast<const __nv_bfloat162 *>(&ls[i]));
        const __nv_bfloat162 y = __hfma2(xv, *reinterpret_cast<const __nv_bfloat162 *>(&hs[i]), t);
        r[i] = *reinterpret_cast<const uint32_t *>(&y);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// 8 floats (as bits) -> bf16 hi = rn(x) and lo = rn(x - hi), so hi + lo carries x to about
// 2^-16 relative.
__device__ __forceinline__ void pack8_hilo(const uint32_t *x, uint4 &hi, uint4 &lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float a = __uint_as_float(x[2 * p]), b = __uint_as_float(x[2 * p + 1]);
        h[p] = pack_bf16x2(a, b);
        const float2 hf = unpack_bf16x2(h[p]);
        l[p] = pack_bf16x2(a - hf.x, b - hf.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ uint4 pack8(const uint32_t *x)
{
    return make_uint4(pack_bf16x2(__uint_as_float(x[0]), __uint_as_float(x[1])),
                      pack_bf16x2(__uint_as_float(x[2]), __uint_as_float(x[3])),
                      pack_bf16x2(__uint_as_float(x[4]), __uint_as_float(x[5])),
                      pack_bf16x2(__uint_as_float(x[6]), __uint_as_float(x[7])));
}

// Diagonal 16x16 tiles of the ablation path (unbounded gate), computed element by
// element: 4 tiles x 136 lower (r, j) pairs, one exponential per (r, j, channel).  Thread
// `tid` owns pairs p = (tid % 64) + 64 s, s < 3, of tile tid / 64; pair p <-> (r, j) with
// r (r + 1) / 2 <= p < (r + 1) (r + 2) / 2, j = p - r (r + 1) / 2 <= r.
constexpr int kDiagPairs = kTile * (kTile + 1) / 2;
constexpr int kDiagSlots = 3;
static_assert(kTiles * 64 == 256 && 64 * kDiagSlots >= kDiagPairs, "diagonal pair mapping");

__device__ __forceinline__ void diag_pair(int p, int &r, int &j)
{
    r = 0;
    while ((r + 1) * (r + 2) / 2 <= p)
        ++r;
    j = p - r * (r + 1) / 2;
}

// The token tensors as TMA tensor maps over this GPU's memory: dims (innermost first)
// {D, H, T, B} for a regular batch, {D, H, T} for a packed one; boxes of 64 channels x one
// head x 64 tokens land with the 128-byte swizzle, which is the token-major operand layout
// (one 128-byte row per token, a 64-channel block per 8 KB).
struct TokenMaps {
    CUtensorMap q, k, v, a;
};

// Warps of the fused gate / cumulative-sum / decay-factor pass: one per (16-token tile,
// 64-channel half), a lane per channel pair.
template <int D>
constexpr int kFusedWarps = kTiles * (D / 64);

template <int D, bool kLogSig>
__global__ void __launch_bounds__(kPrepThreads, 2)
    prep_kernel(const __grid_constant__ TokenMaps tm, SeqMap map, int H, const __nv_bfloat16 *__restrict__ beta,
                const float *__restrict__ gtab, bool per_head_tab, unsigned char *__restrict__ ws,
                unsigned int *status)
{
    extern __shared__ __align__(1024) unsigned char prep_smem[];
    using L = PrepLayout<D>;
    using R = Rec<D>;
    // Two CTAs share an SM only without alignment slack: the swizzled operands need a
    // 1024-byte aligned base, which the dynamic shared window provides; refuse otherwise.
    if (smem_u32(prep_smem) & 1023u) {
        if (threadIdx.x == 0)
            report_device_error(status, KDA_ERR_UNSUPPORTED);
        return;
    }
    unsigned char *sm = prep_smem;
    constexpr int LDA = kC + 1;
    constexpr int CPR = D / 8;  // 16-byte chunks per token row
    constexpr int NFW = kFusedWarps<D>;
    float *sG = reinterpret_cast<float *>(sm + L::RG);   // [64][D] (ablation only)
    float *sA = reinterpret_cast<float *>(sm + L::RA);   // [64][65]
    float *sT = reinterpret_cast<float *>(sm + L::RT);   // [64][65]
    float *sBeta = reinterpret_cast<float *>(sm + L::RBeta);
    __nv_bfloat16 *sEm = reinterpret_cast<__nv_bfloat16 *>(sm + L::REm);  // hi [4][D] | lo [4][D]
    __nv_bfloat16 *sEl = reinterpret_cast<__nv_bfloat16 *>(sm + L::REl);
    __nv_bfloat16 *sDd = reinterpret_cast<__nv_bfloat16 *>(sm + L::RDd);
    // per-(tile, channel) totals and local mid-tile values of the cumulative sum, in P's slot
    // (P is written from step 4 on)
    float *sTot = reinterpret_cast<float *>(sm + L::RP);
    float *sMid = sTot + kTiles * D;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::RBar);  // round 1, U1..U4, a, q|k|v
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::RTmem);
    static_assert(2 * kTiles * D * 4 <= kC * kC * 2, "cumulative-sum tables fit P's slot");

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = lane >> 2, tq = lane & 3;
    const ChunkLoc loc = locate_chunk(map, H, blockIdx.x, blockIdx.y);
    if (!loc.live)  // packed batch: grid slots past the last chunk
        return;
    if constexpr (kDebugChecks) {
        if ((int64_t)loc.rec >= map.nrec || loc.n < 1 || loc.tok0 < 0 || loc.tok0 + loc.n > map.ntok ||
            loc.h < 0 || loc.h >= H) {
            if (threadIdx.x == 0)
                report_device_error(status, KDA_ERR_DEVICE_BOUNDS);
            return;
        }
    }
    const int n = loc.n, h = loc.h;
    unsigned char *rec = ws + loc.rec * R::Bytes;
    const float *tab = gtab + (per_head_tab ? (size_t)h * kGateTableEntries : 0);

    // -- 0. one thread issues the tensor copies of the chunk's a, then q, k, v (64 tokens x 64
    //       channels per box; a regular batch reads zeros past its sequence, a packed one
    //       reads the next sequence's tokens there, which step 1 masks); the other warps load
    //       beta and allocate tensor memory meanwhile
    uint64_t *bar_a = bar + 5, *bar_qkv = bar + 6;
    if (tid == 0) {
        for (int i = 0; i < 7; ++i)
            mbar_init(bar + i, 1);
        fence_mbar_init_cluster();
        constexpr uint32_t kBox = (uint32_t)kC * 64 * 2;
        const int b = map.cu ? 0 : (int)(blockIdx.y / H), t0 = map.cu ? 0 : (int)blockIdx.x * kC;
        auto load = [&](const CUtensorMap *m, uint32_t dst, uint64_t *bb) {
            for (int cb = 0; cb < D / 64; ++cb) {
                if (map.cu)
                    tma_load_3d(sm + dst + cb * kBox, m, cb * 64, h, (int)loc.tok0, bb);
                else
                    tma_load_4d(sm + dst + cb * kBox, m, cb * 64, h, t0, b, bb);
            }
        };
        mbar_arrive_expect_tx(bar_a, (D / 64) * kBox);
        load(&tm.a, L::RX, bar_a);
        mbar_arrive_expect_tx(bar_qkv, 3 * (D / 64) * kBox);
        load(&tm.q, L::RQ, bar_qkv);
        load(&tm.k, L::RK, bar_qkv);
        load(&tm.v, L::RV, bar_qkv);
    }
    if (warp == 0)
        tc::tmem_alloc(tslot, 2 * D);
    if (tid >= kPrepThreads - kC) {
        const int r = tid - (kPrepThreads - kC);
        sBeta[r] = r < n ? __bfloat162float(beta[(loc.tok0 + r) * H + h]) : 0.0f;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;

    // -- 1. fused pass, warp (tile I, channel half), lane = channel pair c0, c0 + 1:
    //       g from the table (0 past the sequence), its inclusive cumulative sum G over the
    //       tile in registers, the tiles' totals exchanged through shared memory; then the
    //       per-(tile, channel) scalars and Gamma_C = e^{G_last}.
    //       Bounded gate: one reference per tile, its middle token m_I (row and column role
    //       alike).  Unbounded gate: the row role of tile I takes G just before the tile (b_I;
    //       0 for I = 0), the column role of tile J the tile's last token (e_J), so every
    //       off-diagonal factor is at most 1 whatever g is.
    float dA[kDiagSlots] = {}, dP[kDiagSlots] = {};
    {
        const bool fw = warp < NFW;
        const int I = warp % kTiles, c0 = (warp / kTiles) * 64 + 2 * lane;
        float G0[kTile], G1[kTile];  // G of tokens 16 I + s, channels c0 and c0 + 1
        float rr0 = 0.f, rr1 = 0.f, cr0 = 0.f, cr1 = 0.f, gl0 = 0.f, gl1 = 0.f;
        if (fw) {
            mbar_wait_bounded(bar_a, 0, status);
            uint32_t ab[kTile];
#pragma unroll
            for (int s2 = 0; s2 < kTile; ++s2)
                ab[s2] = *reinterpret_cast<const uint32_t *>(sm + L::RX + tok_off(I * kTile + s2, c0));
            float x0 = 0.f, x1 = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < kTile; ++s2) {
                const bool ok = I * kTile + s2 < n;
                const float g0 = __ldg(tab + (ab[s2] & 0xffffu)), g1 = __ldg(tab + (ab[s2] >> 16));
                x0 += ok ? g0 : 0.f;
                x1 += ok ? g1 : 0.f;
                G0[s2] = x0;
                G1[s2] = x1;
            }
            *reinterpret_cast<float2 *>(&sTot[I * D + c0]) = make_float2(x0, x1);
            *reinterpret_cast<float2 *>(&sMid[I * D + c0]) = make_float2(G0[kRef], G1[kRef]);
            asm volatile("bar.sync 1, %0;" ::"n"(NFW * 32) : "memory");
            // offsets of every tile (sums in tile order), this tile's references; every tile's total
            // and local reference value read here, before this warp's stores below
            float off0[kTiles], off1[kTiles], ref0[kTiles], ref1[kTiles];
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int J = 0; J < kTiles; ++J) {
                off0[J] = a0;
                off1[J] = a1;
                const float2 t = *reinterpret_cast<const float2 *>(&sTot[J * D + c0]);
                const float2 m = kLogSig ? t : *reinterpret_cast<const float2 *>(&sMid[J * D + c0]);
                ref0[J] = m.x;
                ref1[J] = m.y;
                a0 += t.x;
                a1 += t.y;
            }
            gl0 = a0, gl1 = a1;
            float o0 = 0.f, o1 = 0.f, ti0 = 0.f, ti1 = 0.f;
#pragma unroll
            for (int J = 0; J < kTiles; ++J)
                if (J == I)
                    o0 = off0[J], o1 = off1[J], ti0 = ref0[J], ti1 = ref1[J];
            // the tables in P's slot are read: the warps the front end leaves idle may zero P
            asm volatile("bar.arrive 2, %0;" ::"n"(kPrepThreads) : "memory");
#pragma unroll
            for (int s2 = 0; s2 < kTile; ++s2) {
                G0[s2] += o0;
                G1[s2] += o1;
            }
            // column reference of tile J (a G value; J is a compile-time index wherever used)
            auto col_ref = [&](int J, int ch) -> float { return ch ? off1[J] + ref1[J] : off0[J] + ref0[J]; };
            // this tile's row and column references
            if constexpr (kLogSig) {
                rr0 = o0, rr1 = o1;
                cr0 = o0 + ti0, cr1 = o1 + ti1;  // the tile's total (ref is the total here)
            } else {
                rr0 = cr0 = G0[kRef];
                rr1 = cr1 = G1[kRef];
            }
            {  // e^{row ref} and e^{G_last - col ref} as bf16 hi / lo pairs
                const float em0 = __expf(rr0), em1 = __expf(rr1);
                const float el0 = __expf(gl0 - cr0), el1 = __expf(gl1 - cr1);
                const uint32_t emh = pack_bf16x2(em0, em1), elh = pack_bf16x2(el0, el1);
                const float2 emf = unpack_bf16x2(emh), elf = unpack_bf16x2(elh);
                *reinterpret_cast<uint32_t *>(&sEm[I * D + c0]) = emh;
                *reinterpret_cast<uint32_t *>(&sEm[(kTiles + I) * D + c0]) = pack_bf16x2(em0 - emf.x, em1 - emf.y);
                *reinterpret_cast<uint32_t *>(&sEl[I * D + c0]) = elh;
                *reinterpret_cast<uint32_t *>(&sEl[(kTiles + I) * D + c0]) = pack_bf16x2(el0 - elf.x, el1 - elf.y);
            }
#pragma unroll
            for (int J = 0; J < kTiles - 1; ++J)  // e^{row ref I - col ref J}, J < I
                if (J < I)
                    *reinterpret_cast<uint32_t *>(&sDd[(I * (I - 1) / 2 + J) * D + c0]) =
                        pack_bf16x2(__expf(rr0 - col_ref(J, 0)), __expf(rr1 - col_ref(J, 1)));
            if (I == kTiles - 1)
                *reinterpret_cast<float2 *>(rec + R::Gam + c0 * 4) = make_float2(__expf(gl0), __expf(gl1));
            if constexpr (kLogSig) {  // the element-wise diagonal tiles read G
#pragma unroll
                for (int s2 = 0; s2 < kTile; ++s2)
                    *reinterpret_cast<float2 *>(&sG[(I * kTile + s2) * D + c0]) = make_float2(G0[s2], G1[s2]);
            }
        } else {
            // upper blocks of P are zero (its slot holds the cumulative-sum tables until every
            // front-end warp has read them)
            asm volatile("bar.sync 2, %0;" ::"n"(kPrepThreads) : "memory");
            for (int i = tid - NFW * 32; i < kC * (kC / 2); i += kPrepThreads - NFW * 32) {
                const int r = i / (kC / 2), j = (i % (kC / 2)) * 2;
                if (j / kTile > r / kTile)
                    *reinterpret_cast<uint32_t *>(sm + L::RP + tc::kmaj_sw128(r, j, kC)) = 0u;
            }
        }

        if constexpr (kLogSig) {
            // -- 1a. unbounded gate only: the diagonal tiles element by element from the raw
            //        q, k and G (their decay cannot be factored), held in registers until step 4
            __syncthreads();
            mbar_wait_bounded(bar_qkv, 0, status);
            const int It = tid >> 6;
#pragma unroll
            for (int s = 0; s < kDiagSlots; ++s) {
                const int p = (tid & 63) + 64 * s;
                if (tid < kCoreThreads && p < kDiagPairs) {
                    int r, j;
                    diag_pair(p, r, j);
                    const int tr = It * kTile + r, tj = It * kTile + j;
                    float sa = 0.0f, sp = 0.0f;
                    if (tr < n) {
                        for (int c8 = 0; c8 < D; c8 += 8) {
                            const uint4 ku = *reinterpret_cast<const uint4 *>(sm + L::RK + tok_off(tr, c8));
                            const uint4 qu = *reinterpret_cast<const uint4 *>(sm + L::RQ + tok_off(tr, c8));
                            const uint4 ju = *reinterpret_cast<const uint4 *>(sm + L::RK + tok_off(tj, c8));
                            const uint32_t kw[4] = {ku.x, ku.y, ku.z, ku.w}, qw[4] = {qu.x, qu.y, qu.z, qu.w},
                                           jw[4] = {ju.x, ju.y, ju.z, ju.w};
#pragma unroll
                            for (int w = 0; w < 4; ++w) {
                                const float2 kr = unpack_bf16x2(kw[w]), qr = unpack_bf16x2(qw[w]),
                                             kj = unpack_bf16x2(jw[w]);
                                const float2 gr = *reinterpret_cast<const float2 *>(&sG[tr * D + c8 + 2 * w]);
                                const float2 gj = *reinterpret_cast<const float2 *>(&sG[tj * D + c8 + 2 * w]);
                                const float e0 = __expf(gr.x - gj.x), e1 = __expf(gr.y - gj.y);
                                sa = fmaf(kr.x * kj.x, e0, sa);
                                sa = fmaf(kr.y * kj.y, e1, sa);
                                sp = fmaf(qr.x * kj.x, e0, sp);
                                sp = fmaf(qr.y * kj.y, e1, sp);
                            }
                        }
                    }
                    dA[s] = j < r ? sBeta[tr] * sa : 0.0f;
                    dP[s] = sp;
                }
            }
            __syncthreads();  // raw q, k are overwritten next
        }

        // -- 2. decay factors, in place: Kr = k e^{G - row ref}, Qr = q e^{G - row ref}
        //       (over k, q) and Ec = k e^{col ref - G} (over a); rows past the sequence are
        //       zero in all three and in v (a packed batch loaded the next sequence there)
        if (fw) {
            mbar_wait_bounded(bar_qkv, 0, status);
            // the tile's k and q first: the stores below go to the same arrays, so loads placed
            // after them could not be moved ahead
            uint32_t kw[kTile], qw[kTile];
#pragma unroll
            for (int s2 = 0; s2 < kTile; ++s2) {
                const uint32_t d = tok_off(I * kTile + s2, c0);
                kw[s2] = *reinterpret_cast<const uint32_t *>(sm + L::RK + d);
                qw[s2] = *reinterpret_cast<const uint32_t *>(sm + L::RQ + d);
            }
#pragma unroll
            for (int s2 = 0; s2 < kTile; ++s2) {
                const int r = I * kTile + s2;
                const uint32_t d = tok_off(r, c0);
                const float x0 = G0[s2] - rr0, x1 = G1[s2] - rr1;
                const float y0 = cr0 - G0[s2], y1 = cr1 - G1[s2];
                uint32_t kr = 0u, qr = 0u, ec = 0u;
                if (r < n) {
                    const float2 kk = unpack_bf16x2(kw[s2]);
                    const float2 qq = unpack_bf16x2(qw[s2]);
                    const float e0 = __expf(x0), e1 = __expf(x1), i0 = __expf(y0), i1 = __expf(y1);
                    kr = pack_bf16x2(kk.x * e0, kk.y * e1);
                    qr = pack_bf16x2(qq.x * e0, qq.y * e1);
                    ec = pack_bf16x2(kk.x * i0, kk.y * i1);
                } else {
                    *reinterpret_cast<uint32_t *>(sm + L::RV + d) = 0u;
                }
                *reinterpret_cast<uint32_t *>(sm + L::RK + d) = kr;
                *reinterpret_cast<uint32_t *>(sm + L::RQ + d) = qr;
                *reinterpret_cast<uint32_t *>(sm + L::RX + d) = ec;
            }
        }
    }
    __syncthreads();


    // -- 4. dense 16-token tile products A and P, one warp per (row tile I, column tile
    //       J <= I): row operands Kr, Qr of tile I (scaled by e^{G_{m_I} - G_{m_J}} when
    //       I > J), column operand Ec of tile J.  A (fp32, beta-scaled, strictly lower)
    //       goes over G, which is no longer needed; P (bf16, lower) to its operand slot.
    //       Unbounded gate: off-diagonal tiles only (the diagonal ones come from step 3a).
    constexpr int kTilePairs = kLogSig ? kTiles * (kTiles - 1) / 2 : kTiles * (kTiles + 1) / 2;
    for (int pidx = warp; pidx < kTilePairs; pidx += kPrepWarps) {
        int I = kLogSig ? 1 : 0, J = pidx;
        while (kLogSig ? J >= I : J > I) {  // pidx -> (I, J): 0:(0,0) 1:(1,0) 2:(1,1) 3:(2,0) ...
            J -= kLogSig ? I : I + 1;       //   or, off-diagonal only: 0:(1,0) 1:(2,0) 2:(2,1) ...
            ++I;
        }
        const __nv_bfloat16 *dsc = I > J ? &sDd[(I * (I - 1) / 2 + J) * D] : nullptr;
        float accA[2][4] = {}, accP[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t ak[4], aq[4], bf[4];
            const int mi = lane >> 3;
            {
                const int row = I * kTile + (lane & 7) + 8 * (mi & 1);
                const int col = ks * 16 + 8 * (mi >> 1);
                ldmatrix_x4(ak, sm + L::RK + tok_off(row, col));
                ldmatrix_x4(aq, sm + L::RQ + tok_off(row, col));
            }
            if (dsc) {
#pragma unroll
                for (int reg = 0; reg < 4; ++reg) {
                    const int c = ks * 16 + 2 * tq + 8 * (reg >> 1);
                    const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162 *>(&dsc[c]);
                    __nv_bfloat162 kk = *reinterpret_cast<__nv_bfloat162 *>(&ak[reg]);
                    __nv_bfloat162 qq = *reinterpret_cast<__nv_bfloat162 *>(&aq[reg]);
                    kk = __hmul2(kk, s2);
                    qq = __hmul2(qq, s2);
                    ak[reg] = *reinterpret_cast<uint32_t *>(&kk);
                    aq[reg] = *reinterpret_cast<uint32_t *>(&qq);
                }
            }
            {
                const int row = J * kTile + (lane & 7) + 8 * (mi >> 1);
                const int col = ks * 16 + 8 * (mi & 1);
                ldmatrix_x4(bf, sm + L::RX + tok_off(row, col));
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
            for (int hh = 0; hh < 2; ++hh) {
                const int r = I * kTile + grp + 8 * hh;
                const int j = J * kTile + nt * 8 + 2 * tq;
                const bool lo0 = I > J || j < r, lo1 = I > J || j + 1 < r;
                const bool lp0 = I > J || j <= r, lp1 = I > J || j + 1 <= r;
                sA[r * LDA + j] = lo0 ? sBeta[r] * accA[nt][2 * hh] : 0.0f;
                sA[r * LDA + j + 1] = lo1 ? sBeta[r] * accA[nt][2 * hh + 1] : 0.0f;
                *reinterpret_cast<uint32_t *>(sm + L::RP + tc::kmaj_sw128(r, j, kC)) =
                    pack_bf16x2(lp0 ? accP[nt][2 * hh] : 0.0f, lp1 ? accP[nt][2 * hh + 1] : 0.0f);
            }
    }
    if constexpr (kLogSig) {  // the element-wise diagonal tiles (G, now overwritten, is no longer read)
        const int I = tid >> 6;
#pragma unroll
        for (int s = 0; s < kDiagSlots; ++s) {
            const int p = (tid & 63) + 64 * s;
            if (tid < kCoreThreads && p < kDiagPairs) {
                int r, j;
                diag_pair(p, r, j);
                const int tr = I * kTile + r, tj = I * kTile + j;
                sA[tr * LDA + tj] = dA[s];
                *reinterpret_cast<__nv_bfloat16 *>(sm + L::RP + tc::kmaj_sw128(tr, tj, kC)) = __float2bfloat16(dP[s]);
            }
        }
        for (int i = tid; i < kTiles * kTile * kTile; i += kPrepThreads) {  // P above the diagonal
            const int I = i / (kTile * kTile), r = (i / kTile) % kTile, j = i % kTile;
            if (j > r)
                *reinterpret_cast<__nv_bfloat16 *>(sm + L::RP + tc::kmaj_sw128(I * kTile + r, I * kTile + j, kC)) =
                    __float2bfloat16(0.0f);
        }
    }
    __syncthreads();

    // -- 4b/5. warps 4 and up: chunk-referenced operands in place (Kbar = Kr e^{G_m},
    //         Qbar = Qr e^{G_m}, Khat = Ec e^{G_last - G_m}); at the same time warps 0..3
    //         start T = (I + A)^{-1} with the 16x16 diagonal blocks (forward substitution,
    //         one lane per column).  Then block substitution, one warp per block column.
    if (warp >= kTiles) {
        // each item's loads before its stores (they write the arrays they read)
        for (int i = tid - kTiles * 32; i < kC * CPR; i += kPrepThreads - kTiles * 32) {
            const int r = i / CPR, c8 = (i % CPR) * 8;
            const int tile = r / kTile;
            const uint32_t d = tok_off(r, c8);
            const uint4 emh = *reinterpret_cast<const uint4 *>(&sEm[tile * D + c8]);
            const uint4 eml = *reinterpret_cast<const uint4 *>(&sEm[(kTiles + tile) * D + c8]);
            const uint4 elh = *reinterpret_cast<const uint4 *>(&sEl[tile * D + c8]);
            const uint4 ell = *reinterpret_cast<const uint4 *>(&sEl[(kTiles + tile) * D + c8]);
            const uint4 vk = *reinterpret_cast<const uint4 *>(sm + L::RK + d);
            const uint4 vq = *reinterpret_cast<const uint4 *>(sm + L::RQ + d);
            const uint4 vx = *reinterpret_cast<const uint4 *>(sm + L::RX + d);
            *reinterpret_cast<uint4 *>(sm + L::RK + d) = mul8_hilo(vk, emh, eml);
            *reinterpret_cast<uint4 *>(sm + L::RQ + d) = mul8_hilo(vq, emh, eml);
            *reinterpret_cast<uint4 *>(sm + L::RX + d) = mul8_hilo(vx, elh, ell);
        }
    } else if (lane < kTile) {
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
                s = fmaf(sA[(I * kTile + r) * LDA + I * kTile + y], x[y], s);
            if (r > c)
                x[r] = -s;
        }
#pragma unroll
        for (int r = 0; r < kTile; ++r)
            sT[(I * kTile + r) * LDA + I * kTile + c] = x[r];
    }
    __syncthreads();
    // block column J on warp J, top to bottom: block (I, J) needs only T_KJ (J <= K < I, this
    // warp's own earlier blocks) and the diagonal T_II, so the warps need no CTA barrier between
    if (warp < kTiles - 1) {
        for (int I = warp + 1; I < kTiles; ++I) {
            solve_block_tf32<kC + 1>(sA, sT, sA + (warp + 1) * kTile /* upper block (0, warp+1) of A */, I, warp,
                                     lane);
            __syncwarp();
        }
    }
    __syncthreads();
    // T diag(beta) as the K-major A operand (over A's place), written twice: as rows 0..63
    // and again as rows 64..127 of the M = 128 MMA, so TMEM lanes 64..127 hold a second copy
    // of the result and all four lane quarters can drain it
    {  // every load first (T's region is not the one written, but the compiler cannot tell)
        constexpr int NIT = (kC * (kC / 2) + kPrepThreads - 1) / kPrepThreads;
        float t0[NIT], t1[NIT], b0[NIT], b1[NIT];
#pragma unroll
        for (int it = 0; it < NIT; ++it) {
            const int i = tid + it * kPrepThreads, r = i / (kC / 2), j = (i % (kC / 2)) * 2;
            const bool live = i < kC * (kC / 2) && j / kTile <= r / kTile;  // blocks above: zero
            t0[it] = live ? sT[r * LDA + j] : 0.f;
            t1[it] = live ? sT[r * LDA + j + 1] : 0.f;
            b0[it] = live ? sBeta[j] : 0.f;
            b1[it] = live ? sBeta[j + 1] : 0.f;
        }
#pragma unroll
        for (int it = 0; it < NIT; ++it) {
            const int i = tid + it * kPrepThreads, r = i / (kC / 2), j = (i % (kC / 2)) * 2;
            if (i < kC * (kC / 2)) {
                const uint32_t tb = pack_bf16x2(t0[it] * b0[it], t1[it] * b1[it]);
                *reinterpret_cast<uint32_t *>(sm + L::RG + tc::kmaj_sw128(r, j, kC)) = tb;
                *reinterpret_cast<uint32_t *>(sm + L::RG + tc::kmaj_sw128(kC + r, j, kC)) = tb;
            }
        }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    // -- 6. tensor core round 1: [W | Utilde] = (T beta) [Kbar | V]  (64 x 2D, TMEM cols 0..2D)
    uint32_t phase = 0;
    if (tid == 0) {
        const uint32_t id = tc::idesc_bf16(128, 2 * D, false, true);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
            const uint64_t ad = tc::smem_desc(smem_u32(sm + L::RG) + ks * 32, 16, 1024, tc::kSw128);
            const uint64_t bd = tc::smem_desc(smem_u32(sm + L::RK) + ks * 2048, kC * 128, 1024, tc::kSw128);
            tc::mma_bf16(tmem, ad, bd, id, ks > 0 ? 1u : 0u);
        }
        tc::commit(bar);
    }
    mbar_wait_bounded(bar, phase, status);
    phase ^= 1;
    tc::fence_after_sync();
    // [W | Utilde] (chunk rows 0..63 = TMEM lanes 0..63) -> bf16 token-major operands over G,
    // and the remainder Utilde - rn(Utilde) over V (no longer an operand): Bm = Khat^T Utilde
    // takes both halves, so the term that dominates the next state is not rounded on its way.
    // Warps 0..3 drain W, warps 4..7 Utilde (hi and lo); lane quarters 0, 1 (chunk rows
    // 0..63) take the first D / 2 columns, quarters 2, 3 (the same rows, copied) the rest.
    if (warp < 8) {
        const int r = (warp & 1) * 32 + lane;
        const bool ut = warp >= 4;
        const int cbase = ut ? D : 0;
        const int cbeg = (warp & 2) ? D / 2 : 0;
#pragma unroll
        for (int c0 = cbeg; c0 < cbeg + D / 2; c0 += 32) {
            uint32_t x[32];
            tc::ld_32x32b_x32(tc::taddr(tmem, (warp & 3) * 32, cbase + c0), x);
            tc::wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 8) {  // [W | Utilde] column; 64-column blocks 8 KB apart
                if (ut) {  // Utilde_lo, at the offsets Utilde has relative to G, over V
                    uint4 hi, lo;
                    pack8_hilo(&x[j], hi, lo);
                    *reinterpret_cast<uint4 *>(sm + L::RG + tok_off(r, cbase + c0 + j)) = hi;
                    *reinterpret_cast<uint4 *>(sm + L::RK + tok_off(r, cbase + c0 + j)) = lo;
                } else {
                    *reinterpret_cast<uint4 *>(sm + L::RG + tok_off(r, c0 + j)) = pack8(&x[j]);
                }
            }
        }
        tc::fence_smem_to_async();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    // -- 7. four tensor-core units on the operands in place, each completing on its own
    //       mbarrier, so the tensor core runs one unit while the warps drain another:
    //         U1  N = Khat^T W                TMEM cols 0..D    staged over Kbar | W
    //         U2  P W                         cols D..2D        Q' = Qbar - P W in place of Qbar
    //         U3  Bm = Khat^T (Ut_hi + Ut_lo) cols 0..D         staged over Khat | Ut_lo
    //         U4  O' = P Ut_hi                cols D..2D        staged over Ut_hi
    //       U3 is issued once U1's columns are read, U4 once U2's are.  Every staging area
    //       is free when written (Kbar after round 1, W once U1 and U2 are done; Qbar is Q'
    //       itself; Khat and Ut_lo once U3 is done, U4 reading only P and Ut_hi; Ut_hi once
    //       U4 is done), so no store waits for another to finish reading shared memory.
    //       O' takes Utilde at bf16 (hi): it only feeds the output.
    constexpr int NB = D / kBV;  // value blocks of the record
    static_assert((NB / 2) * R::BmBlk <= L::kMat && NB * R::OpBlk <= L::kMat, "Bm / O' staging fits");
    static_assert((uint32_t)D * 64 * 2 <= L::kMat, "a 64-column block of N fits one operand slot");
    uint64_t *bar_u = bar + 1;
    const uint32_t xw = smem_u32(sm + L::RG), xu = xw + L::kMat;      // W_hi, Ut_hi
    const uint32_t xu_lo = smem_u32(sm + L::RK) + L::kMat;              // Ut_lo (over V)
    auto issue_kt = [&](uint32_t xb, uint32_t col, uint32_t acc0) {  // Khat^T X
        const uint32_t id = tc::idesc_bf16(128, D, true, true);       // A = Khat^T (MN-major)
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
            const uint64_t ad = tc::smem_desc(smem_u32(sm + L::RX) + ks * 2048, kC * 128, 1024, tc::kSw128);
            const uint64_t bd = tc::smem_desc(xb + ks * 2048, kC * 128, 1024, tc::kSw128);
            tc::mma_bf16(tmem + col, ad, bd, id, ks > 0 ? 1u : acc0);
        }
    };
    // N's 64-column blocks: block 0 over Kbar, block 1 (D = 128) over W
    auto n_stage = [&](int blk64) -> unsigned char * { return sm + (blk64 == 0 ? L::RK : L::RG); };
    auto issue_p = [&](uint32_t xb, uint32_t col) {                   // P X
        const uint32_t id = tc::idesc_bf16(128, D, false, true);      // A = P (K-major)
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
            const uint64_t ad = tc::smem_desc(smem_u32(sm + L::RP) + ks * 32, 16, 1024, tc::kSw128);
            const uint64_t bd = tc::smem_desc(xb + ks * 2048, kC * 128, 1024, tc::kSw128);
            tc::mma_bf16(tmem + col, ad, bd, id, ks > 0 ? 1u : 0u);
        }
    };
    auto bm_stage = [&](int blk) -> unsigned char * {  // Bm block blk: over Khat, then Ut_lo
        return blk < NB / 2 ? sm + L::RX + blk * R::BmBlk : sm + L::RK + L::kMat + (blk - NB / 2) * R::BmBlk;
    };
    auto sync_all = [&]() {
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    if (tid == 0) {
        issue_kt(xw, 0, 0u);
        tc::commit(&bar_u[0]);
        issue_p(xw, D);
        tc::commit(&bar_u[1]);
    }
    // Khat^T X epilogues: row i (key channel) = TMEM lane i; warp w reads the lanes of
    // quarter w % 4 and half w / 4 of the columns.  P X epilogues: chunk row r = lane r < 64.
    const bool kt_rows = warp < 8 && (warp & 3) * 32 < D, p_rows = warp < 8 && (warp & 3) < 2;
    const int lrow = (warp & 3) * 32 + lane, chalf = (warp >> 2) * (D / 2);

    // U1 -> N over Kbar | W (W is read by U1 and U2, so wait for U2 as well)
    mbar_wait_bounded(&bar_u[0], 0, status);
    mbar_wait_bounded(&bar_u[1], 0, status);
    tc::fence_after_sync();
    if (kt_rows) {
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
            uint32_t x[32];
            tc::ld_32x32b_x32(tc::taddr(tmem, (warp & 3) * 32, chalf + c0), x);
            tc::wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                const int col = chalf + c0 + j;
                *reinterpret_cast<uint4 *>(n_stage(col >> 6) + tc::kmaj_sw128(lrow, col & 63, D)) = pack8(&x[j]);
            }
        }
    }
    sync_all();
    if (tid == 0) {
        issue_kt(xu, 0, 0u);
        issue_kt(xu_lo, 0, 1u);
        tc::commit(&bar_u[2]);
    }
    // U2 -> Q' = Qbar - P W, in place (same layout as the record)
    if (p_rows) {
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
            uint32_t x[32];
            tc::ld_32x32b_x32(tc::taddr(tmem, (warp & 3) * 32, D + chalf + c0), x);
            uint4 qbs[4];  // Qbar's four 8-column chunks, loaded before any of them is written back
#pragma unroll
            for (int j = 0; j < 32; j += 8)
                qbs[j / 8] = *reinterpret_cast<const uint4 *>(sm + L::RQ + tok_off(lrow, chalf + c0 + j));
            tc::wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                uint4 *pq = reinterpret_cast<uint4 *>(sm + L::RQ + tok_off(lrow, chalf + c0 + j));
                const uint4 qb = qbs[j / 8];
                const uint32_t qw[4] = {qb.x, qb.y, qb.z, qb.w};
                uint32_t o4[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 f = unpack_bf16x2(qw[p]);
                    o4[p] = pack_bf16x2(f.x - __uint_as_float(x[j + 2 * p]), f.y - __uint_as_float(x[j + 2 * p + 1]));
                }
                *pq = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
    }
    tc::fence_smem_to_async();
    sync_all();
    if (tid == 0) {
        issue_p(xu, D);
        tc::commit(&bar_u[3]);
        for (int b64 = 0; b64 < D / 64; ++b64)
            bulk_s2g(rec + R::Nm + b64 * (D * 128), n_stage(b64), D * 128);
        bulk_s2g(rec + R::Qp, sm + L::RQ, kC * D * 2);
        bulk_commit();
    }
    // U3 -> Bm blocks over Khat and W
    mbar_wait_bounded(&bar_u[2], 0, status);
    tc::fence_after_sync();
    if (kt_rows) {
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
            uint32_t x[32];
            tc::ld_32x32b_x32(tc::taddr(tmem, (warp & 3) * 32, chalf + c0), x);
            tc::wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                const int col = chalf + c0 + j;
                *reinterpret_cast<uint4 *>(bm_stage(col / kBV) + tc::mnmaj_sw64(lrow, col % kBV)) = pack8(&x[j]);
            }
        }
    }
    tc::fence_smem_to_async();
    sync_all();
    if (tid == 0) {
        for (int blk = 0; blk < NB; ++blk)
            bulk_s2g(rec + R::Shared + blk * R::Blk, bm_stage(blk), R::BmBlk);
        bulk_commit();
    }
    // U4 -> O' blocks over Utilde
    mbar_wait_bounded(&bar_u[3], 0, status);
    tc::fence_after_sync();
    if (p_rows) {
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
            uint32_t x[32];
            tc::ld_32x32b_x32(tc::taddr(tmem, (warp & 3) * 32, D + chalf + c0), x);
            tc::wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                const int col = chalf + c0 + j;
                *reinterpret_cast<uint4 *>(sm + L::RG + L::kMat + (col / kBV) * R::OpBlk +
                                           tc::mnmaj_sw64(lrow, col % kBV)) = pack8(&x[j]);
            }
        }
    }
    tc::fence_smem_to_async();
    sync_all();
    if (tid == 0) {
        for (int blk = 0; blk < NB; ++blk)
            bulk_s2g(rec + R::Shared + blk * R::Blk + R::BmBlk, sm + L::RG + L::kMat + blk * R::OpBlk, R::OpBlk);
        bulk_commit();
        bulk_wait_read_all();  // staging must stay valid until the stores have read it
    }
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, 2 * D);
}

// ------------------------------------------------------------------ K3: scan
constexpr int kScanWarps = 4;                        // consumer warps (one TMEM lane quarter each)
constexpr int kScanThreads = (kScanWarps + 1) * 32;  // + one producer warp
constexpr int kStages = 3;

// Threads of a forward scan CTA over kW value blocks: four consumer warps per block (warp w
// reads TMEM lane quarter w % 4 and block w / 4), one producer warp.
template <int kW>
constexpr int scan_threads() { return (kScanWarps * kW + 1) * 32; }

// kW value blocks per CTA: 1, or 2 where one block per CTA would take more than one wave of
// the GPU's SMs (the two blocks then share the stage's N and Q'; at D = 128 two stages fit
// the shared memory, not three).
template <int D, bool kSave, int kW = 1>
struct ScanSmem {
    static constexpr uint32_t kStageBytes = Rec<D>::Shared + kW * Rec<D>::Blk;  // shared part + own value blocks
    static constexpr uint32_t kStageStride = (kStageBytes + 1023) / 1024 * 1024;
    static constexpr int kSt =
        kW == 1 || kStages * kStageStride + (uint32_t)D * kBV * kW * 2 + 2048 <= 232448 - 1024 ? kStages : 2;
    alignas(1024) unsigned char stage[kSt][kStageStride];
    // S block, bf16, MN-major (row = key channel): the 64-byte swizzle over 32 columns (kW = 1),
    // the 128-byte swizzle over 64 (kW = 2)
    alignas(1024) unsigned char sbuf[D * kBV * kW * 2];
    // kSave: the float32 block entering a chunk, double-buffered, for the tensor store
    alignas(1024) unsigned char hbuf[2][kSave ? D * kBV * 4 : 16];
    uint64_t full[kSt];                             // stage filled (arrive + bytes)
    uint64_t empty[kSt];                            // stage released by the consumers
    uint64_t mma_bar;                               // tcgen05 MMA batch completed
    uint32_t tmem_slot;
};

// Byte offset of (row, column j < kBV) in a saved float32 state block as the tensor store
// reads it: rows of kBV floats (128 B), 16-byte chunks XOR (row & 7) (the 128-byte swizzle).
__device__ __forceinline__ uint32_t hblk_off(int row, int j)
{
    return (uint32_t)row * 128u + ((uint32_t)((j >> 2) ^ (row & 7)) << 4) + (uint32_t)(j & 3) * 4u;
}

// One thread row's kBV floats into a saved-block buffer.
__device__ __forceinline__ void stage_state_f32(unsigned char *buf, int row, const float (&S)[kBV])
{
#pragma unroll
    for (int j = 0; j < kBV; j += 4)
        *reinterpret_cast<float4 *>(buf + hblk_off(row, j)) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
}

template <int kW = 1>
__device__ __forceinline__ void consumer_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kScanWarps * kW * 32) : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Row `row` of the state block as the bf16 MMA operand (MN-major, 64-byte swizzle).
__device__ __forceinline__ void store_state(unsigned char *sbuf, int row, const float (&S)[kBV])
{
#pragma unroll
    for (int j = 0; j < kBV; j += 8)
        *reinterpret_cast<uint4 *>(sbuf + tc::mnmaj_sw64(row, j)) =
            make_uint4(pack_bf16x2(S[j], S[j + 1]), pack_bf16x2(S[j + 2], S[j + 3]),
                       pack_bf16x2(S[j + 4], S[j + 5]), pack_bf16x2(S[j + 6], S[j + 7]));
}

// Columns [c0, c0 + kBV) of row `row` of a 64-column state block as the bf16 MMA operand
// (MN-major, 128-byte swizzle).
__device__ __forceinline__ void store_state_w(unsigned char *sbuf, int row, int c0, const float (&S)[kBV])
{
#pragma unroll
    for (int j = 0; j < kBV; j += 8)
        *reinterpret_cast<uint4 *>(sbuf + tc::mnmaj_sw128(row, c0 + j, 128)) =
            make_uint4(pack_bf16x2(S[j], S[j + 1]), pack_bf16x2(S[j + 2], S[j + 3]),
                       pack_bf16x2(S[j + 4], S[j + 5]), pack_bf16x2(S[j + 6], S[j + 7]));
}

// kSave: also write the fp32 state entering every chunk to the state array of hs_map (one
// D x D block per record, indexed like the records), for the backward: the rows stage their
// block in shared memory and one thread stores it with a 2-D tensor store per chunk.
template <int D, bool kAffine, bool kSave, int kW = 1>
__global__ void __launch_bounds__(scan_threads<kW>(), 1)
    scan_kernel(SeqMap map, int H, const unsigned char *__restrict__ ws, const float *__restrict__ S0,
                __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T, float *__restrict__ M_out,
                const __grid_constant__ CUtensorMap hs_map, unsigned int *status)
{
    extern __shared__ __align__(1024) unsigned char scan_smem[];
    using SM = ScanSmem<D, kSave, kW>;
    using R = Rec<D>;
    static_assert(kW == 1 || (kW == 2 && !kAffine && !kSave && D / kBV % 2 == 0), "wide scan: plain forward only");
    SM &sm = *reinterpret_cast<SM *>(scan_smem + ((1024u - (smem_u32(scan_smem) & 1023u)) & 1023u));
    constexpr uint32_t kTmemCols = 2 * kBV * kW;  // [0, kW kBV): N S; [kW kBV, 2 kW kBV): Q' S
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Column blocks past D / kBV (affine mode only) carry the transfer map instead of the
    // state: they start from the identity, add no Bm and write M_out.
    constexpr int NB = D / kBV;
    const bool xfer = kAffine && blockIdx.x >= NB;
    const int blk = xfer ? blockIdx.x - NB : blockIdx.x, col0 = blk * kBV * kW;
    const SeqLoc seq = locate_seq(map, H);
    if constexpr (kDebugChecks) {
        // the records this CTA reads and the token rows it can write (an invalid packed-batch
        // table leaves nchunks = 0: nothing read or written, S_T still set)
        const int64_t span = min((int64_t)seq.len, (int64_t)seq.nchunks * kC);
        if (seq.nchunks < 0 || (int64_t)seq.rec0 + seq.nchunks > map.nrec || seq.sh >= map.nseq * H ||
            (span > 0 && (seq.tok0 < 0 || seq.tok0 + span > map.ntok))) {
            if (threadIdx.x == 0)
                report_device_error(status, KDA_ERR_DEVICE_BOUNDS);
            return;
        }
    }
    const int h = seq.h, NT = seq.nchunks, bh = seq.sh;
    const unsigned char *recs = ws + seq.rec0 * R::Bytes;

    if (tid == 0) {
        for (int s = 0; s < SM::kSt; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.mma_bar, 1);
        fence_mbar_init_cluster();
    }
    if (warp == 0)
        tc::tmem_alloc(&sm.tmem_slot, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_slot;

    if (warp == kScanWarps * kW) {
        // ---------------- producer: one lane issues the bulk copies
        if (lane == 0) {
            for (int c = 0; c < NT; ++c) {
                const int s = c % SM::kSt;
                if (c >= SM::kSt)
                    mbar_wait_bounded(&sm.empty[s], ((c / SM::kSt) - 1) & 1, status);
                mbar_arrive_expect_tx(&sm.full[s], SM::kStageBytes);
                const unsigned char *rec = recs + (size_t)c * R::Bytes;
                bulk_g2s(sm.stage[s], rec, R::Shared, &sm.full[s]);
                bulk_g2s(sm.stage[s] + R::Shared, rec + R::Shared + blk * kW * R::Blk, kW * R::Blk, &sm.full[s]);
            }
        }
        __syncwarp();
    } else {
        // ---------------- consumers: thread `row` owns TMEM lane `row`; warp w takes lane
        // quarter w % 4 of value block w / 4 (the columns from ccol on)
        const int q4 = kW == 1 ? warp : (warp & 3), wc = kW == 1 ? 0 : (warp >> 2);
        const int row = q4 * 32 + lane, ccol = col0 + wc * kBV;
        const bool srow = row < D;  // owns state row `row` (key channel)
        const uint32_t lane_addr = tc::taddr(tmem, (uint32_t)q4 * 32, (uint32_t)(wc * kBV));
        float S[kBV];
        if (srow) {
#pragma unroll
            for (int j = 0; j < kBV; j += 4) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (xfer) {  // identity columns col0 .. col0 + kBV of the transfer map
                    v.x = row == col0 + j ? 1.f : 0.f;
                    v.y = row == col0 + j + 1 ? 1.f : 0.f;
                    v.z = row == col0 + j + 2 ? 1.f : 0.f;
                    v.w = row == col0 + j + 3 ? 1.f : 0.f;
                } else if (S0) {
                    v = *reinterpret_cast<const float4 *>(&S0[((size_t)bh * D + row) * D + ccol + j]);
                }
                S[j] = v.x;
                S[j + 1] = v.y;
                S[j + 2] = v.z;
                S[j + 3] = v.w;
            }
            if constexpr (kW == 1)
                store_state(sm.sbuf, row, S);
            else
                store_state_w(sm.sbuf, row, wc * kBV, S);
            if constexpr (kSave)
                stage_state_f32(sm.hbuf[0], row, S);
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        consumer_sync<kW>();
        tc::fence_after_sync();

        const uint32_t id_k = tc::idesc_bf16(128, kBV * kW, false, true);  // A K-major, B MN-major
        // The MMA round is issued from warp 2 so that warps 0 and 1 (TMEM lanes 0..63, the chunk's
        // rows) can finish a chunk's output after the closing barrier while the next round runs.
        constexpr int kIssuer = 64;
        const uint32_t sbuf_a = smem_u32(sm.sbuf);
        uint32_t mma_phase = 0;
        for (int c = 0; c < NT; ++c) {
            const int s = c % SM::kSt;
            mbar_wait_bounded(&sm.full[s], (c / SM::kSt) & 1, status);
            const unsigned char *st = sm.stage[s];
            const uint32_t st_a = smem_u32(st);

            // [N S | Q' S] in one round (rows past N (D = 64) and past Q' are don't-cares)
            if (tid == kIssuer) {
                tc::fence_after_sync();
                if constexpr (kSave) {
                    // the block entering chunk c, staged by every row thread before the last
                    // consumer barrier; wait until the store of chunk c - 1 has read its buffer,
                    // which the rows refill (for chunk c + 1) only after this round's MMAs
                    tma_store_2d(&hs_map, col0, (int)((seq.rec0 + c) * D), sm.hbuf[c & 1]);
                    bulk_commit();
                    bulk_wait_read_1();
                }
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t bd = kW == 1 ? tc::smem_desc(sbuf_a + ks * 1024, 0, 512, tc::kSw64)
                                                : tc::smem_desc(sbuf_a + ks * 2048, D * 128, 1024, tc::kSw128);
                    const uint64_t an =
                        tc::smem_desc(st_a + R::Nm + (ks >> 2) * (D * 128) + (ks & 3) * 32, 16, 1024, tc::kSw128);
                    const uint64_t aq =
                        tc::smem_desc(st_a + R::Qp + (ks >> 2) * (kC * 128) + (ks & 3) * 32, 16, 1024, tc::kSw128);
                    tc::mma_bf16(tmem, an, bd, id_k, ks > 0 ? 1u : 0u);
                    if constexpr (!kSave)  // the state-saving scan forms no output
                        tc::mma_bf16(tmem + kBV * kW, aq, bd, id_k, ks > 0 ? 1u : 0u);
                }
                tc::commit(&sm.mma_bar);
            }
            // Diag(Gamma) S + Bm while the tensor core runs (stage data is in since `full`)
            if (srow) {
                const float g = reinterpret_cast<const float *>(st + R::Gam)[row];
                const unsigned char *bmp = st + R::Shared + wc * R::Blk;
#pragma unroll
                for (int j = 0; j < kBV; j += 8) {
                    const uint4 bu = *reinterpret_cast<const uint4 *>(bmp + tc::mnmaj_sw64(row, j));
                    const uint32_t bw[4] = {bu.x, bu.y, bu.z, bu.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 bf = xfer ? make_float2(0.f, 0.f) : unpack_bf16x2(bw[q]);
                        S[j + 2 * q] = fmaf(g, S[j + 2 * q], bf.x);
                        S[j + 2 * q + 1] = fmaf(g, S[j + 2 * q + 1], bf.y);
                    }
                }
            }
            mbar_wait_bounded(&sm.mma_bar, mma_phase, status);
            mma_phase ^= 1;
            tc::fence_after_sync();

            const unsigned char *blkp = st + R::Shared + wc * R::Blk;
            const bool orow_w = !kSave && o && q4 < 2;  // O = Q' S + O' for chunk rows 0..63 (quarters 0, 1)
            uint32_t y[kBV];
            uint4 ou[kBV / 8];
            // S <- (Diag(Gamma) S + Bm) - N S; bf16 copy for the next chunk
            if (srow) {
                uint32_t d[kBV];
                tc::ld_32x32b_x32(lane_addr, d);
                if (orow_w)
                    tc::ld_32x32b_x32(lane_addr + kBV * kW, y);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < kBV; ++j)
                    S[j] -= __uint_as_float(d[j]);
                if constexpr (kW == 1)
                    store_state(sm.sbuf, row, S);
                else
                    store_state_w(sm.sbuf, row, wc * kBV, S);
                if constexpr (kSave) {
                    if (c + 1 < NT)
                        stage_state_f32(sm.hbuf[(c + 1) & 1], row, S);
                }
                tc::fence_smem_to_async();
            }
            // the O' rows too before the barrier (the stage is released after it)
            if (orow_w) {
#pragma unroll
                for (int j = 0; j < kBV; j += 8)
                    ou[j / 8] = *reinterpret_cast<const uint4 *>(blkp + R::BmBlk + tc::mnmaj_sw64(row, j));
            }
            tc::fence_before_sync();
            consumer_sync<kW>();
            tc::fence_after_sync();
            if (tid == kIssuer)
                mbar_arrive_local(&sm.empty[s]);
            if (orow_w) {  // the output while the next chunk's round runs
                const int t = c * kC + row;
                if (t < seq.len) {
                    uint4 *orow = reinterpret_cast<uint4 *>(o + ((seq.tok0 + t) * H + h) * D + ccol);
#pragma unroll
                    for (int j = 0; j < kBV; j += 8) {
                        const uint32_t ow[4] = {ou[j / 8].x, ou[j / 8].y, ou[j / 8].z, ou[j / 8].w};
                        uint32_t r4[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const float2 of = unpack_bf16x2(ow[p]);
                            r4[p] = pack_bf16x2(of.x + __uint_as_float(y[j + 2 * p]),
                                                of.y + __uint_as_float(y[j + 2 * p + 1]));
                        }
                        orow[j / 8] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
                    }
                }
            }
        }

        if constexpr (kSave) {
            if (tid == kIssuer)
                bulk_wait_all();  // the last blocks are written before the CTA leaves
        }
        float *Sout = xfer ? M_out : S_T;
        if (Sout && srow)
#pragma unroll
            for (int j = 0; j < kBV; j += 4)
                *reinterpret_cast<float4 *>(&Sout[((size_t)bh * D + row) * D + ccol + j]) =
                    make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0)
        tc::tmem_dealloc(tmem, kTmemCols);
}

// ================================================================== backward
// The chunked backward, derived from the chunked form above.  With dS' = dL/d(state after
// the chunk) and dO = dL/dO (per chunk, entering state S):
//   dU = Khat dS' + P^T dO,   dKhat = U dS'^T,   dQbar = dO S^T,   dP = lower_incl(dO U^T)
//   dW = -dU S^T,   dGamma = rowsum(dS' * S),   dS = Diag(Gamma) dS' + Qbar^T dO - W^T dU
// and, substituting dU, the state gradient walks the chunks backwards with the records the
// forward wrote:
//   dS = (Diag(Gamma) - N)^T dS' + Q'^T dO.
// Through the WY form (W = T Bk, Utilde = T Bv, Bk = diag(beta) Kbar, Bv = diag(beta) V,
// T = (I + A)^{-1}):  dBk = T^T dW,  dBv = T^T dU,  dT = dW Bk^T + dU Bv^T,
// dA = -strict_lower(T^T dT T^T); then the pairwise decay products A and P hand their
// gradients to q, k and the cumulative log-decay G, and dg is the reverse cumulative sum
// of dG inside the chunk.
//
// Three launches after the forward prep: the scan again with the entering state of every
// chunk saved (scan_kernel<.., kSave>), the reverse state-gradient scan (dscan_kernel,
// tcgen05), and the per-chunk gradients (bwd_chunk_kernel).

// ------------------------------------------------------------------ reverse state-gradient scan
// One CTA per (32-column block of dv, sequence*head), chunks in reverse order.  Per chunk one
// tcgen05 round computes [N^T dS' | Q'^T dO]: N and Q' are the record's K-major operands,
// read here as MN-major (transposed) A operands; dS' (bf16 copy) and the chunk's dO block
// are MN-major B operands.  The fp32 gradient block stays in registers, one row per thread;
// every chunk's block (the gradient of the state after it) leaves by a 2-D tensor store.
template <int D>
struct DScanSmem {
    // An M = 128 MN-major read of Q' (and of N when D = 64) covers two 64-row MN blocks; past
    // the operand those bytes only feed accumulator lanes that are never read.
    static constexpr uint32_t kRead = Rec<D>::Qp + 2u * kC * 128u > Rec<D>::Shared ? Rec<D>::Qp + 2u * kC * 128u
                                                                                   : Rec<D>::Shared;
    static constexpr uint32_t kStageStride = (kRead + 1023) / 1024 * 1024;
    alignas(1024) unsigned char stage[kStages][kStageStride];
    alignas(1024) unsigned char sbuf[D * kBV * 2];   // dS' block, bf16, MN-major 64-byte swizzle
    alignas(1024) unsigned char obuf[kC * kBV * 2];  // dO block of the chunk, same layout (row = token)
    alignas(1024) unsigned char hbuf[2][D * kBV * 4];  // float32 block for the tensor store, double-buffered
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t mma_bar;
    uint32_t tmem_slot;
};

template <int D>
__global__ void __launch_bounds__(kScanThreads, 1)
    dscan_kernel(SeqMap map, int H, const unsigned char *__restrict__ ws, const __nv_bfloat16 *__restrict__ dO,
                 const float *__restrict__ dS_T, const __grid_constant__ CUtensorMap dhs_map,
                 float *__restrict__ dS0, unsigned int *status)
{
    extern __shared__ __align__(1024) unsigned char dscan_smem[];
    using SM = DScanSmem<D>;
    using R = Rec<D>;
    SM &sm = *reinterpret_cast<SM *>(dscan_smem + ((1024u - (smem_u32(dscan_smem) & 1023u)) & 1023u));
    constexpr uint32_t kTmemCols = 2 * kBV;  // [0, kBV): N^T dS'; [kBV, 2 kBV): Q'^T dO
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int blk = blockIdx.x, col0 = blk * kBV;
    const SeqLoc seq = locate_seq(map, H);
    if constexpr (kDebugChecks) {
        const int64_t span = min((int64_t)seq.len, (int64_t)seq.nchunks * kC);
        if (seq.nchunks < 0 || (int64_t)seq.rec0 + seq.nchunks > map.nrec || seq.sh >= map.nseq * H ||
            (span > 0 && (seq.tok0 < 0 || seq.tok0 + span > map.ntok))) {
            if (threadIdx.x == 0)
                report_device_error(status, KDA_ERR_DEVICE_BOUNDS);
            return;
        }
    }
    const int h = seq.h, NT = seq.nchunks, bh = seq.sh;
    const unsigned char *recs = ws + seq.rec0 * R::Bytes;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.mma_bar, 1);
        fence_mbar_init_cluster();
    }
    if (warp == 0)
        tc::tmem_alloc(&sm.tmem_slot, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_slot;

    if (warp == kScanWarps) {
        // ---------------- producer: the records' shared part, last chunk first
        if (lane == 0) {
            for (int i = 0; i < NT; ++i) {
                const int c = NT - 1 - i, s = i % kStages;
                if (i >= kStages)
                    mbar_wait_bounded(&sm.empty[s], ((i / kStages) - 1) & 1, status);
                mbar_arrive_expect_tx(&sm.full[s], R::Shared);
                bulk_g2s(sm.stage[s], recs + (size_t)c * R::Bytes, R::Shared, &sm.full[s]);
            }
        }
        __syncwarp();
    } else {
        const int row = warp * 32 + lane;
        const bool srow = row < D;    // owns gradient row `row` (key channel)
        const bool trow = row < kC;   // loads token row `row` of the chunk's dO block
        const uint32_t lane_addr = tc::taddr(tmem, (uint32_t)warp * 32, 0);
        float S[kBV];
#pragma unroll
        for (int j = 0; j < kBV; ++j)
            S[j] = 0.f;
        if (srow && dS_T) {
#pragma unroll
            for (int j = 0; j < kBV; j += 4) {
                const float4 v = *reinterpret_cast<const float4 *>(&dS_T[((size_t)bh * D + row) * D + col0 + j]);
                S[j] = v.x;
                S[j + 1] = v.y;
                S[j + 2] = v.z;
                S[j + 3] = v.w;
            }
        }
        // dO row of chunk c (zero past the sequence)
        auto load_do = [&](int c, uint4 (&r)[4]) {
            const int t = c * kC + row;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                r[q] = make_uint4(0u, 0u, 0u, 0u);
            if (trow && t < seq.len) {
                const uint4 *p = reinterpret_cast<const uint4 *>(dO + ((seq.tok0 + t) * H + h) * D + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    r[q] = p[q];
            }
        };
        uint4 cur[4];
        if (NT > 0)
            load_do(NT - 1, cur);

        const uint32_t id_t = tc::idesc_bf16(128, kBV, true, true);  // A MN-major, B MN-major
        const uint32_t sbuf_a = smem_u32(sm.sbuf), obuf_a = smem_u32(sm.obuf);
        uint32_t mma_phase = 0;
        for (int i = 0; i < NT; ++i) {
            const int c = NT - 1 - i, s = i % kStages;
            // dS' of chunk c (the gradient of the state after it) is what the rows hold now; its
            // float32 block goes out by a tensor store (buffer i & 1: the store of iteration i - 2
            // has read it, thread 0 waited for that before the last barrier of iteration i - 1)
            if (srow) {
                stage_state_f32(sm.hbuf[i & 1], row, S);
                store_state(sm.sbuf, row, S);
            }
            if (trow) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(sm.obuf + tc::mnmaj_sw64(row, q * 8)) = cur[q];
                if (c > 0)
                    load_do(c - 1, cur);
            }
            tc::fence_smem_to_async();
            tc::fence_before_sync();
            consumer_sync();
            tc::fence_after_sync();
            mbar_wait_bounded(&sm.full[s], (i / kStages) & 1, status);
            const unsigned char *st = sm.stage[s];
            const uint32_t st_a = smem_u32(st);
            if (tid == 0) {
                tc::fence_after_sync();
                tma_store_2d(&dhs_map, col0, (int)((seq.rec0 + c) * D), sm.hbuf[i & 1]);
                bulk_commit();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t an = tc::smem_desc(st_a + R::Nm + ks * 2048, D * 128, 1024, tc::kSw128);
                    const uint64_t bd = tc::smem_desc(sbuf_a + ks * 1024, 0, 512, tc::kSw64);
                    tc::mma_bf16(tmem, an, bd, id_t, ks > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks) {
                    const uint64_t aq = tc::smem_desc(st_a + R::Qp + ks * 2048, kC * 128, 1024, tc::kSw128);
                    const uint64_t bo = tc::smem_desc(obuf_a + ks * 1024, 0, 512, tc::kSw64);
                    tc::mma_bf16(tmem + kBV, aq, bo, id_t, ks > 0 ? 1u : 0u);
                }
                tc::commit(&sm.mma_bar);
            }
            if (srow) {
                const float g = reinterpret_cast<const float *>(st + R::Gam)[row];
#pragma unroll
                for (int j = 0; j < kBV; ++j)
                    S[j] *= g;
            }
            mbar_wait_bounded(&sm.mma_bar, mma_phase, status);
            mma_phase ^= 1;
            tc::fence_after_sync();
            if (srow) {
                uint32_t d[kBV], y[kBV];
                tc::ld_32x32b_x32(lane_addr, d);
                tc::ld_32x32b_x32(lane_addr + kBV, y);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < kBV; ++j)
                    S[j] += __uint_as_float(y[j]) - __uint_as_float(d[j]);
            }
            if (tid == 0)
                bulk_wait_read_1();  // the store of iteration i - 1 has read buffer (i + 1) & 1
            tc::fence_before_sync();
            consumer_sync();
            tc::fence_after_sync();
            if (tid == 0)
                mbar_arrive_local(&sm.empty[s]);
        }
        if (tid == 0)
            bulk_wait_all();  // the last blocks are written before the CTA leaves
        if (dS0 && srow)
#pragma unroll
            for (int j = 0; j < kBV; j += 4)
                *reinterpret_cast<float4 *>(&dS0[((size_t)bh * D + row) * D + col0 + j]) =
                    make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0)
        tc::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ per-chunk gradients
// Persistent: kBwdSlots CTAs of 512 threads walk the chunks.  q, k, G and the chunk's 64 x 64
// matrices A', T, dT and dA stay in shared memory; P and the 64 x D intermediates live in a
// float32 scratch slot of the workspace per CTA (written and read back by the same CTA; L2
// holds part of it).  Dense contractions go through cta_gemm (TF32 mma.sync, fp32
// accumulation).  The pairwise decay
// products are 16 x 16 tile pairs on the same mma, with the decay factored through a
// reference token of the ROW tile (the forward's prep uses the column tile's middle token;
// either factoring is exact): the row tile's first token for tiles below the diagonal (both
// factors <= 1), its middle token on the diagonal (factors <= e^{8 |g_min|}).
constexpr int kBwdThreads = 512;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdSlots = 148;  // one CTA per SM of a 148-SM part

template <int D>
struct BwdSlot {  // float offsets inside one scratch slot, 64 x D row-major blocks
    static constexpr int CD = kC * D;
    static constexpr int Kb = 0, Kh = Kb + CD;
    static constexpr int Bk = Kh + CD;   // diag(beta) Kbar, later dBk
    static constexpr int Bv = Bk + CD;   // diag(beta) V, later dBv
    static constexpr int W = Bv + CD;    // Bv - Bk S, then dW, then the pairwise dq
    static constexpr int U = W + CD;     // U, then dk
    static constexpr int dO = U + CD;    // dO, then the pairwise dG
    static constexpr int dU = dO + CD;
    static constexpr int dKh = dU + CD;
    static constexpr int dQb = dKh + CD;
    static constexpr int Gp = dQb + CD;  // dg/da = g_min sigma(a) (1 - sigma(a))
    static constexpr int X = Gp + CD;    // dT T^T, 64 x 64
    static constexpr int P = X + kC * kC;  // the pairwise products P, 64 x 64
    static constexpr int floats = P + kC * kC;
};

// Operand sources of cta_gemm.  "K" = consecutive along the contraction index, "M" / "N" =
// consecutive along the output row / column index.  Global ones (the scratch slot, the saved
// states) are staged into shared memory by 16-byte cp.async copies; shared ones are read in
// place.
enum GemmSrc : int {
    kGlobK,  // A(i, k) = p[i * ld + k]  or  B(k, j) = p[j * ld + k]
    kGlobMN, // A(i, k) = p[k * ld + i]  or  B(k, j) = p[k * ld + j]
    kSmemK,  // as kGlobK, in shared memory
    kSmemM,  // A only: as kGlobMN, in shared memory
};

constexpr int kGKS = 32;    // contraction step per pipeline stage
constexpr int kGStages = 2; // cp.async stages (double buffer)
// one stage: A 64 x 32 (K-consecutive rows padded to 36, or 32 x 64 padded to 72), B 32 x TN
// (N-consecutive rows padded to TN + 8) or TN x 32 (K-consecutive, 16-byte chunks XOR-swizzled)
constexpr int kGStageA = kC * (kGKS + 4);
constexpr int kGStageB = kGKS * (128 + 8);
constexpr int kGStageFloats = kGStageA + kGStageB;
constexpr int kGStage = kGStages * kGStageFloats;
static_assert(kGKS * 72 <= kGStageA && 128 * kGKS <= kGStageB, "stage layouts fit");
static_assert(2 * 16 * 256 <= kGStage, "the partial-sum exchange fits the ring");

template <int D>
struct BwdSmem {  // float offsets in shared memory
    static constexpr int LDD = D + 4;    // conflict-free mma fragment reads
    static constexpr int LDC = kC + 4;
    static constexpr int q = 0, k = q + kC * LDD, G = k + kC * LDD;  // q later holds dG
    static constexpr int Ap = G + kC * LDD, T = Ap + kC * LDC;
    static constexpr int dT = T + kC * LDC;  // scratch of the block solve, then dT, then dP
    static constexpr int dA = dT + kC * LDC;
    static constexpr int stage = dA + kC * LDC;  // cta_gemm's ring (16-byte aligned)
    static constexpr int seg = stage;  // after the contractions: row-segment sums of dG, then of dKhat * Khat
    static constexpr int beta = stage + kGStage;
    static constexpr int dGam = beta + kC;
    static constexpr int red = dGam + D;  // per-warp partial sums of dA_log
    static constexpr int floats = red + kBwdWarps;
    static constexpr size_t bytes = (size_t)floats * 4;
    static_assert(stage % 4 == 0, "cp.async destinations are 16-byte aligned");
    static_assert(2 * kBwdThreads <= kGStage, "segment sums fit the ring");
    static_assert(bytes <= 232448, "shared memory per block");
};

template <int TN>
__device__ __forceinline__ int gemm_bk_off(int j, int k)  // (k, j) of a staged K-consecutive B
{
    return j * kGKS + ((((k >> 2) ^ j) & 7) << 2) + (k & 3);
}

// ldmatrix of four 8 x 4 fp32 blocks (each row 16 bytes): thread T receives element
// (T / 4, T % 4) of block q in r[q]; lane l gives the address of row l % 8 of block l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const float *row_ptr)
{
    ldmatrix_x4(r, row_ptr);
}

// Where cta_gemm puts its result: dst[i, j] = sign * C[i, j] (+ acc_in[i, j]), rows of ld floats
// (global or shared memory); with mask 1 only j < i is kept (0 elsewhere), with mask 2 j <= i.
struct GemmOut {
    float *dst;
    int ld;
    float sign;
    const float *acc_in;
    int ld_in;
    int mask;
};

// C[64 x TN] = A[64 x K] B[K x TN] (+ A2[64 x K2] B2[K2 x TN], operands of the same kinds) on the
// whole CTA (K, K2 multiples of 32), written as the GemmOut says, each output pair (j even) once
// (a thread loads all its acc_in values before its first store, so a read-modify-write of one
// array costs one memory round trip, not one per element).  TF32 mma.sync with fp32
// accumulation; operands enter the tensor cores as their fp32 bit patterns (the hardware
// uses the TF32 part).  The contraction is split between two groups of eight warps: per
// 32-wide step, group 0 takes its first 16 indices and group 1 the rest, each warp a 32 x TN/4
// tile, and the two partial sums meet in shared memory at the end.  The global operands move
// through two shared-memory stages (double buffer), one CTA barrier per step.  Starts and
// ends with every thread past a barrier.
// One copy of the code per operand-kind combination (not per call site), so the gradient
// kernel's instruction footprint stays small.
template <int TN, int SA, int SB>
__device__ __noinline__ void cta_gemm(int K, const float *A, int lda, const float *B, int ldb, float *stage, GemmOut out,
                                      int K2 = 0, const float *A2 = nullptr, int lda2 = 0, const float *B2 = nullptr,
                                      int ldb2 = 0)
{
    const float *const acc_in = out.acc_in;
    const int ld_in = out.ld_in;
    const float sign = out.sign;
    auto epi = [&](int i, int j, float x0, float x1) {
        if (out.mask == 1) {
            x0 = j < i ? x0 : 0.f;
            x1 = j + 1 < i ? x1 : 0.f;
        } else if (out.mask == 2) {
            x0 = j <= i ? x0 : 0.f;
            x1 = j + 1 <= i ? x1 : 0.f;
        }
        *reinterpret_cast<float2 *>(out.dst + i * out.ld + j) = make_float2(x0, x1);
    };
    static_assert(TN == 64 || TN == 128, "output tile width");
    static_assert(SB != kSmemM, "B in place is K-consecutive");
    constexpr int NF = TN / 32, LDBN = TN + 8;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int grp = warp >> 3, wl = warp & 7;
    const int wm = (wl >> 2) * 32, wn = (wl & 3) * (TN / 4);
    const int lr = lane & 7, lq = lane >> 3;  // ldmatrix: row within a block, block
    const int nk1 = K / kGKS, nk = nk1 + K2 / kGKS;
    // step s of the contraction: its operands and its offset inside them
    auto seg = [&](int s, const float *&Ap, int &la, const float *&Bp, int &lb) -> int {
        const bool second = s >= nk1;
        Ap = second ? A2 : A, la = second ? lda2 : lda, Bp = second ? B2 : B, lb = second ? ldb2 : ldb;
        return (second ? s - nk1 : s) * kGKS;
    };
    auto issue = [&](int s, int slot) {
        float *sA = stage + slot * kGStageFloats, *sB = sA + kGStageA;
        const float *A, *B;
        int lda, ldb;
        const int k0 = seg(s, A, lda, B, ldb);
        constexpr int CPR = kGKS / 4;  // 16-byte chunks per K-consecutive row
        static_assert(kC * CPR == kBwdThreads && kGKS * (kC / 4) == kBwdThreads, "one A chunk per thread");
        if constexpr (SA == kGlobK) {
            const int i = tid / CPR, c = tid % CPR;
            cp_async_16(sA + i * (kGKS + 4) + 4 * c, A + (size_t)i * lda + k0 + 4 * c);
        } else if constexpr (SA == kGlobMN) {
            const int k = tid / (kC / 4), c = tid % (kC / 4);
            cp_async_16(sA + k * 72 + 4 * c, A + (size_t)(k0 + k) * lda + 4 * c);
        }
#pragma unroll
        for (int e = tid; e < kGKS * TN / 4; e += kBwdThreads) {
            if constexpr (SB == kGlobMN) {
                const int k = e / (TN / 4), c = e % (TN / 4);
                cp_async_16(sB + k * LDBN + 4 * c, B + (size_t)(k0 + k) * ldb + 4 * c);
            } else if constexpr (SB == kGlobK) {
                const int j = e / CPR, c = e % CPR;
                cp_async_16(sB + gemm_bk_off<TN>(j, 4 * c), B + (size_t)j * ldb + k0 + 4 * c);
            }
        }
    };
    // A fragments of the warp's two 16-row blocks at contraction offset kk of step k0
    auto load_a = [&](const float *sA, const float *A, int lda, int k0, int kk, uint32_t (&af)[2][4]) {
#pragma unroll
        for (int mf = 0; mf < 2; ++mf) {
            const int r0 = wm + mf * 16;
            if constexpr (SA == kGlobK || SA == kSmemK) {
                const int row = r0 + (lq & 1) * 8 + lr, col = kk + (lq >> 1) * 4;
                ldsm_x4(af[mf], SA == kGlobK ? sA + row * (kGKS + 4) + col : A + row * lda + k0 + col);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = r0 + g + (q & 1) * 8, k = kk + t + (q >> 1) * 4;
                    af[mf][q] = __float_as_uint(SA == kGlobMN ? sA[k * 72 + i] : A[(k0 + k) * lda + i]);
                }
            }
        }
    };
    auto load_b = [&](const float *sB, const float *B, int ldb, int k0, int kk, uint32_t (&bf)[NF][2]) {
        if constexpr (SB == kGlobMN) {
#pragma unroll
            for (int nf = 0; nf < NF; ++nf) {
                const int j = wn + nf * 8 + g;
                bf[nf][0] = __float_as_uint(sB[(kk + t) * LDBN + j]);
                bf[nf][1] = __float_as_uint(sB[(kk + t + 4) * LDBN + j]);
            }
        } else {
            // rows j (K-consecutive): block q of an x4 = (column block, k half)
            auto addr = [&](int j, int k) -> const float * {
                return SB == kGlobK ? sB + gemm_bk_off<TN>(j, k) : B + j * ldb + k0 + k;
            };
            if constexpr (NF == 4) {
#pragma unroll
                for (int hk = 0; hk < 2; ++hk) {
                    uint32_t r[4];
                    ldsm_x4(r, addr(wn + lq * 8 + lr, kk + hk * 4));
#pragma unroll
                    for (int nf = 0; nf < 4; ++nf)
                        bf[nf][hk] = r[nf];
                }
            } else {
                uint32_t r[4];
                ldsm_x4(r, addr(wn + (lq & 1) * 8 + lr, kk + (lq >> 1) * 4));
                bf[0][0] = r[0], bf[1][0] = r[1], bf[0][1] = r[2], bf[1][1] = r[3];
            }
        }
    };
#pragma unroll
    for (int s = 0; s < kGStages - 1; ++s) {
        if (s < nk)
            issue(s, s);
        cp_async_commit();
    }
    float acc[2][NF][4] = {};
    for (int s = 0; s < nk; ++s) {
        cp_async_wait<kGStages - 2>();
        __syncthreads();  // stage s is in for every thread; stage s - 1 is no longer read
        if (s + kGStages - 1 < nk)
            issue(s + kGStages - 1, (s + kGStages - 1) % kGStages);
        cp_async_commit();
        const float *sA = stage + (s % kGStages) * kGStageFloats, *sB = sA + kGStageA;
        const float *Ap, *Bp;
        int la, lb;
        const int k0 = seg(s, Ap, la, Bp, lb);
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // this group's two 8-wide slices of the step
            const int kk = grp * 16 + h * 8;
            uint32_t af[2][4], bf[NF][2];
            load_a(sA, Ap, la, k0, kk, af);
            load_b(sB, Bp, lb, k0, kk, bf);
#pragma unroll
            for (int mf = 0; mf < 2; ++mf)
#pragma unroll
                for (int nf = 0; nf < NF; ++nf)
                    mma_tf32_1688(acc[mf][nf], af[mf], bf[nf]);
        }
    }
    float2 prev[NF][2];
    if (acc_in) {
#pragma unroll
        for (int nf = 0; nf < NF; ++nf)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                prev[nf][hh] = *reinterpret_cast<const float2 *>(acc_in + (wm + grp * 16 + g + 8 * hh) * ld_in +
                                                                 wn + nf * 8 + 2 * t);
    }
    // partial sums: group g finishes row block mf = g of its tile and hands the other over
    cp_async_wait<0>();
    __syncthreads();  // the ring is free
    float *xch = stage;  // [2][NF * 4][256]: row block, value, thread of the group
    const int gt = wl * 32 + lane;
#pragma unroll
    for (int nf = 0; nf < NF; ++nf)
#pragma unroll
        for (int v = 0; v < 4; ++v)
            xch[((1 - grp) * NF * 4 + nf * 4 + v) * 256 + gt] = grp ? acc[0][nf][v] : acc[1][nf][v];
    __syncthreads();
#pragma unroll
    for (int nf = 0; nf < NF; ++nf) {
        float c[4];
#pragma unroll
        for (int v = 0; v < 4; ++v)
            c[v] = (grp ? acc[1][nf][v] : acc[0][nf][v]) + xch[(grp * NF * 4 + nf * 4 + v) * 256 + gt];
        const int i = wm + grp * 16 + g, j = wn + nf * 8 + 2 * t;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            c[2 * hh] = acc_in ? fmaf(sign, c[2 * hh], prev[nf][hh].x) : sign * c[2 * hh];
            c[2 * hh + 1] = acc_in ? fmaf(sign, c[2 * hh + 1], prev[nf][hh].y) : sign * c[2 * hh + 1];
        }
        epi(i, j, c[0], c[1]);
        epi(i + 8, j, c[2], c[3]);
    }
    __syncthreads();
}

// One tile pair (I, J), J <= I, of the forward pairwise products on one warp:
//   A'_rs = sum_c k_rc k_sc e^{G_rc - G_sc} (s < r),  P_rs = sum_c q_rc k_sc e^{..} (s <= r)
// with e^{G_r - G_s} = e^{G_r - G_m} e^{G_m - G_s}, m the reference token of tile I.
template <int D>
__device__ void pair_fwd_tile(const float *sq, const float *sk, const float *sG, float *Ap, float *P, int I, int J,
                              int lane)
{
    using SL = BwdSmem<D>;
    constexpr int LDD = SL::LDD, LDC = SL::LDC;
    const int g = lane >> 2, t = lane & 3;
    const int m = J < I ? I * kTile : I * kTile + kRef;
    const int r0 = I * kTile, s0 = J * kTile;
    float aA[2][4] = {}, aP[2][4] = {};
#pragma unroll 2
    for (int kk = 0; kk < D; kk += 8) {
        uint32_t fk[4], fq[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int r = r0 + g + (x & 1) * 8, c = kk + t + (x >> 1) * 4;
            const float f = __expf(sG[r * LDD + c] - sG[m * LDD + c]);
            fk[x] = to_tf32(sk[r * LDD + c] * f);
            fq[x] = to_tf32(sq[r * LDD + c] * f);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t b[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int c = kk + t + x * 4, s = s0 + nt * 8 + g;
                b[x] = to_tf32(sk[s * LDD + c] * __expf(sG[m * LDD + c] - sG[s * LDD + c]));
            }
            mma_tf32_1688(aA[nt], fk, b);
            mma_tf32_1688(aP[nt], fq, b);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int r = r0 + g + (x >> 1) * 8, s = s0 + nt * 8 + 2 * t + (x & 1);
            Ap[r * LDC + s] = s < r ? aA[nt][x] : 0.f;
            P[r * kC + s] = s <= r ? aP[nt][x] : 0.f;  // P: row stride kC (the scratch slot)
        }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_chunk_kernel(SeqMap map, int H, int nunits, const __nv_bfloat16 *__restrict__ qg,
                     const __nv_bfloat16 *__restrict__ kg, const __nv_bfloat16 *__restrict__ vg,
                     const __nv_bfloat16 *__restrict__ ag, const __nv_bfloat16 *__restrict__ betag, float g_min,
                     const float *__restrict__ A_log, const float *__restrict__ gtab,
                     const __nv_bfloat16 *__restrict__ dOg,
                     const float *__restrict__ Hs, const float *__restrict__ dHs, float *scratch,
                     float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ da,
                     float *__restrict__ dbeta, float *__restrict__ dA_part, unsigned int *status)
{
    using L = BwdSlot<D>;
    using SL = BwdSmem<D>;
    constexpr int CD = kC * D, LDD = SL::LDD, LDC = SL::LDC;
    constexpr int NQ = D / 32;  // 32-channel quarters (per warp) of the pairwise backward
    extern __shared__ __align__(16) float bsm[];
    float *const sq = bsm + SL::q, *const sk = bsm + SL::k, *const sG = bsm + SL::G;
    float *const sAp = bsm + SL::Ap, *const sT = bsm + SL::T;
    float *const sdT = bsm + SL::dT, *const sdA = bsm + SL::dA;
    float *const stage = bsm + SL::stage;
    float *const sbeta = bsm + SL::beta, *const sdGam = bsm + SL::dGam;
    float *const sseg = bsm + SL::seg, *const sred = bsm + SL::red;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *sl = scratch + (size_t)blockIdx.x * L::floats;
    float *const Kb = sl + L::Kb, *const Kh = sl + L::Kh, *const Bk = sl + L::Bk;
    float *const Bv = sl + L::Bv, *const W = sl + L::W, *const U = sl + L::U, *const dOs = sl + L::dO;
    float *const dU = sl + L::dU, *const dKh = sl + L::dKh, *const dQb = sl + L::dQb, *const Gp = sl + L::Gp;
    float *const Xg = sl + L::X, *const Pg = sl + L::P;  // P: 64 x 64, row stride kC

    for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
        // regular batch: unit = (b*H + h) * NT + chunk; packed batch: unit = h * NT + chunk slot
        const ChunkLoc loc = locate_chunk(map, H, unit % map.NT, unit / map.NT);
        if (!loc.live)
            continue;
        if constexpr (kDebugChecks) {
            if (loc.n < 1 || loc.n > kC || (int64_t)loc.rec >= map.nrec || loc.tok0 < 0 ||
                loc.tok0 + loc.n > map.ntok) {
                if (tid == 0)
                    report_device_error(status, KDA_ERR_DEVICE_BOUNDS);
                return;
            }
        }
        const int n = loc.n, h = loc.h;
        const int64_t tok0 = loc.tok0;
        const float *S = Hs + loc.rec * (size_t)D * D;
        const float *dSn = dHs + loc.rec * (size_t)D * D;
        auto tix = [&](int r) { return (tok0 + r) * H + h; };  // token-head row index
        // the gate's argument is scale * a (scale = e^{A_log[h]}, or 1); g itself comes from the
        // gate table the forward prep used (per head with the scale)
        const float scale = A_log ? __expf(A_log[h]) : 1.0f;
        const float *tab = gtab + (A_log ? (size_t)h * kGateTableEntries : 0);
        // 1. inputs (rows past the chunk's tokens are zero, with g = 0), and dg/da; eight channels
        //    per item (16-byte loads)
        static_assert(CD % (8 * kBwdThreads) == 0, "whole passes over the chunk");
#pragma unroll
        for (int pass8 = 0; pass8 < CD / 8 / kBwdThreads; ++pass8) {
            const int it = tid + pass8 * kBwdThreads;
            const int r = it / (D / 8), c = (it % (D / 8)) * 8, e = r * D + c;
            const bool ok = r < n;
            const size_t gi = (size_t)tix(ok ? r : 0) * D + c;
            const uint4 au = __ldg(reinterpret_cast<const uint4 *>(ag + gi));
            uint4 qu = __ldg(reinterpret_cast<const uint4 *>(qg + gi)), ku = __ldg(reinterpret_cast<const uint4 *>(kg + gi));
            uint4 vu = __ldg(reinterpret_cast<const uint4 *>(vg + gi)), du = __ldg(reinterpret_cast<const uint4 *>(dOg + gi));
            if (!ok)
                qu = ku = vu = du = make_uint4(0u, 0u, 0u, 0u);
            const float bt = ok ? __bfloat162float(betag[tix(r)]) : 0.f;  // Bv = beta v
            const uint32_t aw[4] = {au.x, au.y, au.z, au.w}, qw[4] = {qu.x, qu.y, qu.z, qu.w},
                           kw[4] = {ku.x, ku.y, ku.z, ku.w}, vw[4] = {vu.x, vu.y, vu.z, vu.w},
                           dw[4] = {du.x, du.y, du.z, du.w};
            float fq[8], fk[8], fg[8], fp[8], fv[8], fd[8];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float2 q2 = unpack_bf16x2(qw[w]), k2 = unpack_bf16x2(kw[w]), v2 = unpack_bf16x2(vw[w]),
                             d2 = unpack_bf16x2(dw[w]), a2 = unpack_bf16x2(aw[w]);
                fq[2 * w] = q2.x, fq[2 * w + 1] = q2.y;
                fk[2 * w] = k2.x, fk[2 * w + 1] = k2.y;
                fv[2 * w] = bt * v2.x, fv[2 * w + 1] = bt * v2.y;
                fd[2 * w] = d2.x, fd[2 * w + 1] = d2.y;
                fg[2 * w] = ok ? __ldg(tab + (aw[w] & 0xffffu)) : 0.f;
                fg[2 * w + 1] = ok ? __ldg(tab + (aw[w] >> 16)) : 0.f;
                const float s0 = __fdividef(1.f, 1.f + __expf(-scale * a2.x)), s1 = __fdividef(1.f, 1.f + __expf(-scale * a2.y));
                fp[2 * w] = g_min * s0 * (1.f - s0) * scale;
                fp[2 * w + 1] = g_min * s1 * (1.f - s1) * scale;
            }
#pragma unroll
            for (int h4 = 0; h4 < 8; h4 += 4) {
                *reinterpret_cast<float4 *>(sq + r * LDD + c + h4) = make_float4(fq[h4], fq[h4 + 1], fq[h4 + 2], fq[h4 + 3]);
                *reinterpret_cast<float4 *>(sk + r * LDD + c + h4) = make_float4(fk[h4], fk[h4 + 1], fk[h4 + 2], fk[h4 + 3]);
                *reinterpret_cast<float4 *>(sG + r * LDD + c + h4) = make_float4(fg[h4], fg[h4 + 1], fg[h4 + 2], fg[h4 + 3]);
                *reinterpret_cast<float4 *>(Gp + e + h4) = make_float4(fp[h4], fp[h4 + 1], fp[h4 + 2], fp[h4 + 3]);
                *reinterpret_cast<float4 *>(Bv + e + h4) = make_float4(fv[h4], fv[h4 + 1], fv[h4 + 2], fv[h4 + 3]);
                *reinterpret_cast<float4 *>(dOs + e + h4) = make_float4(fd[h4], fd[h4 + 1], fd[h4 + 2], fd[h4 + 3]);
            }
        }
        for (int r = tid; r < kC; r += kBwdThreads)
            sbeta[r] = r < n ? __bfloat162float(betag[tix(r)]) : 0.f;
        __syncthreads();
        // 2. G = inclusive cumulative sum over the chunk, per channel
        for (int c = tid; c < D; c += kBwdThreads) {
            float acc = 0.f;
            for (int r = 0; r < kC; ++r) {
                acc += sG[r * LDD + c];
                sG[r * LDD + c] = acc;
            }
        }
        __syncthreads();
        // 3. decay-scaled operands (scratch) and 4. the pairwise products A', P (warps 0..9)
        for (int e = tid; e < CD; e += kBwdThreads) {
            const int r = e / D, c = e % D;
            const float Gv = sG[r * LDD + c], e1 = __expf(Gv), eh = __expf(sG[(kC - 1) * LDD + c] - Gv);
            const float kv = sk[r * LDD + c];
            Kb[e] = kv * e1;
            Kh[e] = kv * eh;
            Bk[e] = sbeta[r] * kv * e1;
        }
        if (warp < kTiles * (kTiles + 1) / 2) {
            int I = 0, J = warp;  // warp -> (I, J), J <= I, row by row
            while (J > I) {
                J -= I + 1;
                ++I;
            }
            pair_fwd_tile<D>(sq, sk, sG, sAp, Pg, I, J, lane);
        }
        for (int e = tid; e < kC * kC; e += kBwdThreads) {
            const int r = e / kC, s = e % kC;
            sT[r * LDC + s] = r == s ? 1.f : 0.f;
            if (s / kTile > r / kTile)  // tiles above the diagonal (the pairwise tiles write the rest)
                sAp[r * LDC + s] = Pg[r * kC + s] = 0.f;
        }
        __syncthreads();
        // 5. T = (I + A)^{-1}, A = diag(beta) A', unit lower triangular, by 16 x 16 blocks: the
        //    diagonal blocks by forward substitution (one lane per column, the column in registers),
        //    then the blocks below, T_IJ = -T_II diag(beta_I) sum_{K=J}^{I-1} A'_IK T_KJ, one warp per
        //    block column with tf32 tensor-core products.
        if (warp < kTiles && lane < kTile) {
            const int I = warp, c = lane;
            float x[kTile];
#pragma unroll
            for (int r = 0; r < kTile; ++r)
                x[r] = r == c ? 1.0f : 0.0f;
#pragma unroll
            for (int r = 1; r < kTile; ++r) {
                float acc = 0.0f;
#pragma unroll
                for (int y = 0; y < r; ++y)
                    acc = fmaf(sAp[(I * kTile + r) * LDC + I * kTile + y], x[y], acc);
                if (r > c)
                    x[r] = -sbeta[I * kTile + r] * acc;
            }
#pragma unroll
            for (int r = 0; r < kTile; ++r)
                sT[(I * kTile + r) * LDC + I * kTile + c] = x[r];
        }
        __syncthreads();
        if (warp < kTiles - 1) {  // block column J on warp J, top to bottom (no CTA barrier between)
            for (int I = warp + 1; I < kTiles; ++I) {
                // scratch: a 16 x 16 block of sdT per warp (free until step 6)
                solve_block_tf32<LDC>(sAp, sT, sdT + warp * kTile * LDC, I, warp, lane, sbeta);
                __syncwarp();
            }
        }
        __syncthreads();
        // 6. dense contractions
        // A operand T: kSmemK over sT; T^T: kSmemM over sT.  Row-major 64 x D blocks of the slot
        // are kGlobK as A, kGlobMN as B; S and dS' (row-major D x D) are kGlobMN as B, and their
        // transposes kGlobK.
        // U = T (Bv - Bk S) = Utilde - W S: X = Bv - Bk S over W's slot, then U = T X
        cta_gemm<D, kGlobK, kGlobMN>(D, Bk, D, S, D, stage, GemmOut{W, D, -1.f, Bv, D, 0});
        cta_gemm<D, kSmemK, kGlobMN>(kC, sT, LDC, W, D, stage, GemmOut{U, D, 1.f, nullptr, 0, 0});
        cta_gemm<D, kGlobK, kGlobMN>(D, Kh, D, dSn, D, stage, GemmOut{dU, D, 1.f, nullptr, 0, 0});
        cta_gemm<D, kGlobMN, kGlobMN>(kC, Pg, kC, dOs, D, stage, GemmOut{dU, D, 1.f, dU, D, 0});
        cta_gemm<D, kGlobK, kGlobK>(D, U, D, dSn, D, stage, GemmOut{dKh, D, 1.f, nullptr, 0, 0});
        cta_gemm<D, kGlobK, kGlobK>(D, dOs, D, S, D, stage, GemmOut{dQb, D, 1.f, nullptr, 0, 0});
        cta_gemm<D, kGlobK, kGlobK>(D, dU, D, S, D, stage, GemmOut{W, D, -1.f, nullptr, 0, 0});
        float *const dW = W;
        // dGamma_i = sum_j dS'_ij S_ij, warp per row
#pragma unroll
        for (int ii = 0; ii < D / kBwdWarps; ++ii) {
            const int i = warp + ii * kBwdWarps;
            float acc = 0.f;
#pragma unroll
            for (int jj = 0; jj < D / 32; ++jj)
                acc = fmaf(dSn[(size_t)i * D + lane + 32 * jj], S[(size_t)i * D + lane + 32 * jj], acc);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0)
                sdGam[i] = acc;
        }
        // dT = dW Bk^T + dU Bv^T, one contraction over both
        cta_gemm<64, kGlobK, kGlobK>(D, dW, D, Bk, D, stage, GemmOut{sdT, LDC, 1.f, nullptr, 0, 0}, D, dU, D, Bv, D);
        cta_gemm<D, kSmemM, kGlobMN>(kC, sT, LDC, dW, D, stage, GemmOut{Bk, D, 1.f, nullptr, 0, 0});
        cta_gemm<D, kSmemM, kGlobMN>(kC, sT, LDC, dU, D, stage, GemmOut{Bv, D, 1.f, nullptr, 0, 0});
        cta_gemm<64, kSmemK, kSmemK>(kC, sdT, LDC, sT, LDC, stage, GemmOut{Xg, kC, 1.f, nullptr, 0, 0});
        cta_gemm<64, kSmemM, kGlobMN>(kC, sT, LDC, Xg, kC, stage, GemmOut{sdA, LDC, -1.f, nullptr, 0, 1});
        cta_gemm<64, kGlobK, kGlobK>(D, dOs, D, U, D, stage, GemmOut{sdT, LDC, 1.f, nullptr, 0, 2});
        float *const dBk = Bk, *const dBv = Bv, *const sdP = sdT;  // dA' = diag(beta) dA
        // 7. pairwise products backward, one warp per (tile I, 32-channel quarter); E_rs = e^{G_r - G_s}
        //    per channel.  Rows of tile I:
        //      dq_r = sum_{s<=r} dP_rs k_s E_rs,  dk_r = sum_{s<r} dA'_rs k_s E_rs,  dG_r = q_r dq_r + k_r dk_r;
        //    columns of tile J = I (each row tile I' >= J with its own reference):
        //      dk_s += sum_{r>=s} (dP_rs q_r + dA'_rs k_r) E_rs,  dG_s -= k_s (that sum).
        //    The row tile I has I + 1 tile pairs and the column tile 4 - I, five per warp.  Both
        //    passes give a thread the same (token, channel) elements, so it sums them in registers
        //    and stores dq -> W, dk -> U and dG -> dO once.
        if (warp < kTiles * NQ) {
            const int I = warp / NQ, c0 = (warp % NQ) * 32, g = lane >> 2, t = lane & 3;
            float vq[4][4] = {}, vk[4][4] = {};
            for (int pass = 0; pass < 2; ++pass) {  // 0: tiles J < I (reference 16 I), 1: J = I (middle)
                const int m = pass == 0 ? I * kTile : I * kTile + kRef;
                float aq[4][4] = {}, ak[4][4] = {};
                const int J0 = pass == 0 ? 0 : I, J1 = pass == 0 ? I : I + 1;
                for (int J = J0; J < J1; ++J) {
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        uint32_t fp[4], fa[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const int r = I * kTile + g + (x & 1) * 8, s = J * kTile + ks * 8 + t + (x >> 1) * 4;
                            fp[x] = to_tf32(sdP[r * LDC + s]);
                            fa[x] = to_tf32(sbeta[r] * sdA[r * LDC + s]);
                        }
#pragma unroll
                        for (int nf = 0; nf < 4; ++nf) {
                            uint32_t b[2];
#pragma unroll
                            for (int x = 0; x < 2; ++x) {
                                const int s = J * kTile + ks * 8 + t + x * 4, c = c0 + nf * 8 + g;
                                b[x] = to_tf32(sk[s * LDD + c] * __expf(sG[m * LDD + c] - sG[s * LDD + c]));
                            }
                            mma_tf32_1688(aq[nf], fp, b);
                            mma_tf32_1688(ak[nf], fa, b);
                        }
                    }
                }
#pragma unroll
                for (int nf = 0; nf < 4; ++nf)
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int r = I * kTile + g + (x >> 1) * 8, c = c0 + nf * 8 + 2 * t + (x & 1);
                        const float f = __expf(sG[r * LDD + c] - sG[m * LDD + c]);
                        vq[nf][x] = fmaf(aq[nf][x], f, vq[nf][x]);
                        vk[nf][x] = fmaf(ak[nf][x], f, vk[nf][x]);
                    }
            }
            const int J = I;
            float tot[4][4] = {};
            for (int Ir = J; Ir < kTiles; ++Ir) {
                const int m = Ir > J ? Ir * kTile : Ir * kTile + kRef;
                float acc[4][4] = {};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    uint32_t fp[4], fa[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {  // A(s, r) = dP_rs: s = row of the product
                        const int s = J * kTile + g + (x & 1) * 8, r = Ir * kTile + ks * 8 + t + (x >> 1) * 4;
                        fp[x] = to_tf32(sdP[r * LDC + s]);
                        fa[x] = to_tf32(sbeta[r] * sdA[r * LDC + s]);
                    }
#pragma unroll
                    for (int nf = 0; nf < 4; ++nf) {
                        uint32_t bq[2], bk[2];
#pragma unroll
                        for (int x = 0; x < 2; ++x) {
                            const int r = Ir * kTile + ks * 8 + t + x * 4, c = c0 + nf * 8 + g;
                            const float f = __expf(sG[r * LDD + c] - sG[m * LDD + c]);
                            bq[x] = to_tf32(sq[r * LDD + c] * f);
                            bk[x] = to_tf32(sk[r * LDD + c] * f);
                        }
                        mma_tf32_1688(acc[nf], fp, bq);
                        mma_tf32_1688(acc[nf], fa, bk);
                    }
                }
#pragma unroll
                for (int nf = 0; nf < 4; ++nf)
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int s = J * kTile + g + (x >> 1) * 8, c = c0 + nf * 8 + 2 * t + (x & 1);
                        tot[nf][x] = fmaf(acc[nf][x], __expf(sG[m * LDD + c] - sG[s * LDD + c]), tot[nf][x]);
                    }
            }
#pragma unroll
            for (int nf = 0; nf < 4; ++nf)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // element pairs (x = 2 hh, 2 hh + 1): channels c, c + 1
                    const int r = I * kTile + g + hh * 8, c = c0 + nf * 8 + 2 * t;
                    const float2 q2 = *reinterpret_cast<const float2 *>(sq + r * LDD + c);
                    const float2 k2 = *reinterpret_cast<const float2 *>(sk + r * LDD + c);
                    const float q0 = vq[nf][2 * hh], q1 = vq[nf][2 * hh + 1];
                    const float k0 = vk[nf][2 * hh], k1 = vk[nf][2 * hh + 1];
                    const float t0 = tot[nf][2 * hh], t1 = tot[nf][2 * hh + 1];
                    *reinterpret_cast<float2 *>(W + r * D + c) = make_float2(q0, q1);
                    *reinterpret_cast<float2 *>(U + r * D + c) = make_float2(k0 + t0, k1 + t1);
                    *reinterpret_cast<float2 *>(dOs + r * D + c) =
                        make_float2(q2.x * q0 + k2.x * (k0 - t0), q2.y * q1 + k2.y * (k1 - t1));
                }
        }
        __syncthreads();
        // 8. the decay-scaled operands' gradients; outputs dq, dk, dv; dG -> sq.  Four channels per
        //    item (16-byte accesses).
        for (int it = tid; it < CD / 4; it += kBwdThreads) {
            const int r = it / (D / 4), c = (it % (D / 4)) * 4, e = r * D + c;
            const float4 G4 = *reinterpret_cast<const float4 *>(sG + r * LDD + c);
            const float4 Gl = *reinterpret_cast<const float4 *>(sG + (kC - 1) * LDD + c);
            const float4 k4 = *reinterpret_cast<const float4 *>(sk + r * LDD + c);
            const float4 q4 = *reinterpret_cast<const float4 *>(sq + r * LDD + c);
            // explicit global loads: they may run ahead of this thread's shared-memory stores
            const float4 w4 = __ldcg(reinterpret_cast<const float4 *>(W + e)), dq4 = __ldcg(reinterpret_cast<const float4 *>(dQb + e));
            const float4 u4 = __ldcg(reinterpret_cast<const float4 *>(U + e)), bk4 = __ldcg(reinterpret_cast<const float4 *>(dBk + e));
            const float4 kh4 = __ldcg(reinterpret_cast<const float4 *>(dKh + e)), o4 = __ldcg(reinterpret_cast<const float4 *>(dOs + e));
            const float4 bv4 = __ldcg(reinterpret_cast<const float4 *>(dBv + e));
            const float br = sbeta[r];
            const float Gv[4] = {G4.x, G4.y, G4.z, G4.w}, Gt[4] = {Gl.x, Gl.y, Gl.z, Gl.w};
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w}, qv[4] = {q4.x, q4.y, q4.z, q4.w};
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, dqb[4] = {dq4.x, dq4.y, dq4.z, dq4.w};
            const float uv[4] = {u4.x, u4.y, u4.z, u4.w}, bkv[4] = {bk4.x, bk4.y, bk4.z, bk4.w};
            const float khv[4] = {kh4.x, kh4.y, kh4.z, kh4.w}, ov[4] = {o4.x, o4.y, o4.z, o4.w};
            const float bvv[4] = {bv4.x, bv4.y, bv4.z, bv4.w};
            float oq[4], ok4[4], ov4[4], og[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float e1 = __expf(Gv[u]), eh = __expf(Gt[u] - Gv[u]);
                const float dkb = br * bkv[u];
                oq[u] = wv[u] + dqb[u] * e1;
                ok4[u] = uv[u] + dkb * e1 + khv[u] * eh;
                og[u] = ov[u] + (dqb[u] * qv[u] + dkb * kv[u]) * e1 - khv[u] * kv[u] * eh;
                ov4[u] = br * bvv[u];
            }
            *reinterpret_cast<float4 *>(sq + r * LDD + c) = make_float4(og[0], og[1], og[2], og[3]);
            if (r < n) {
                const size_t gi = (size_t)tix(r) * D + c;
                *reinterpret_cast<float4 *>(dq + gi) = make_float4(oq[0], oq[1], oq[2], oq[3]);
                *reinterpret_cast<float4 *>(dk + gi) = make_float4(ok4[0], ok4[1], ok4[2], ok4[3]);
                *reinterpret_cast<float4 *>(dv + gi) = make_float4(ov4[0], ov4[1], ov4[2], ov4[3]);
            }
        }
        __syncthreads();
        // 9. dg = reverse cumulative sum of dG (G_last also carries Gamma and Khat); da = dg g'(a).
        //    Thread (segment, channel): sums of row segments first, then each segment's scan.
        constexpr int NSEG = kBwdThreads / D, SR = kC / NSEG;
        {
            const int c = tid % D, sgi = tid / D, r0 = sgi * SR;
            const float Gl = sG[(kC - 1) * LDD + c];
            float loc = 0.f, lkh = 0.f;  // dG, and dKhat * Khat (G_last's share), over the segment
#pragma unroll
            for (int u = 0; u < SR; ++u) {
                const int r = r0 + u;
                loc += sq[r * LDD + c];
                lkh = fmaf(__ldcg(dKh + r * D + c) * sk[r * LDD + c], __expf(Gl - sG[r * LDD + c]), lkh);
            }
            sseg[sgi * D + c] = loc;
            sseg[kBwdThreads + sgi * D + c] = lkh;
        }
        __syncthreads();
        {
            const int c = tid % D, sgi = tid / D, r0 = sgi * SR;
            float gp[SR];
#pragma unroll
            for (int u = 0; u < SR; ++u)
                gp[u] = __ldcg(Gp + (r0 + u) * D + c);
            float acc = sdGam[c] * __expf(sG[(kC - 1) * LDD + c]);
            for (int s2 = 0; s2 < NSEG; ++s2)
                acc += sseg[kBwdThreads + s2 * D + c];
            for (int s2 = sgi + 1; s2 < NSEG; ++s2)
                acc += sseg[s2 * D + c];
            float dal = 0.f;  // sum of da * a over the segment: this chunk's share of dL/dA_log
#pragma unroll
            for (int u = SR - 1; u >= 0; --u) {
                const int r = r0 + u;
                acc += sq[r * LDD + c];
                if (r < n) {
                    const size_t gi = (size_t)tix(r) * D + c;
                    const float dav = acc * gp[u];
                    da[gi] = dav;
                    if (dA_part)
                        dal = fmaf(dav, __bfloat162float(ag[gi]), dal);
                }
            }
            if (dA_part) {  // dL/dA_log = sum over the head's tokens and channels of da * a
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    dal += __shfl_xor_sync(0xffffffffu, dal, o);
                if (lane == 0)
                    sred[warp] = dal;
            }
        }
        // 10. dbeta_r = sum_c dBk_rc Kbar_rc + sum_c dBv_rc v_rc + sum_s dA_rs A'_rs; warp per row,
        //     the warp's rows summed together (rows past the chunk read row 0 and store nothing)
        {
            constexpr int RPW = kC / kBwdWarps;
            float acc[RPW];
#pragma unroll
            for (int rr = 0; rr < RPW; ++rr) {
                const int r = warp + rr * kBwdWarps, rv = r < n ? r : 0;
                float a = 0.f;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    const int c = lane + 32 * cc;
                    a += __ldcg(dBk + r * D + c) * __ldcg(Kb + r * D + c) +
                         __ldcg(dBv + r * D + c) * __bfloat162float(vg[(size_t)tix(rv) * D + c]);
                }
#pragma unroll
                for (int ss = 0; ss < kC / 32; ++ss)
                    a += sdA[r * LDC + lane + 32 * ss] * sAp[r * LDC + lane + 32 * ss];
                acc[rr] = a;
            }
#pragma unroll
            for (int rr = 0; rr < RPW; ++rr) {
                float a = acc[rr];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    a += __shfl_xor_sync(0xffffffffu, a, o);
                const int r = warp + rr * kBwdWarps;
                if (lane == 0 && r < n)
                    dbeta[tix(r)] = a;
            }
        }
        __syncthreads();  // shared memory and the slot are reused by the next chunk
        if (dA_part && tid == 0) {
            float sum = 0.f;
            for (int w = 0; w < kBwdWarps; ++w)
                sum += sred[w];
            dA_part[loc.rec] = sum;
        }
    }
}

// dL/dA_log[h]: the sum of the per-chunk partials of head h, in a fixed order.  One CTA per
// head; regular batch: records (b H + h) NT + n; packed batch: records h NT + g, g < chunks.
constexpr int kRedThreads = 256;

__global__ void __launch_bounds__(kRedThreads)
    dalog_reduce_kernel(SeqMap map, int H, const float *__restrict__ part, float *__restrict__ dA_log)
{
    __shared__ float buf[kRedThreads];
    const int h = blockIdx.x, tid = threadIdx.x;
    const int64_t per = map.cu ? (int64_t)map.choff[map.nseq] : (int64_t)map.nseq * map.NT;
    float acc = 0.f;
    for (int64_t i = tid; i < per; i += kRedThreads) {
        const int64_t rec = map.cu ? (int64_t)h * map.NT + i
                                   : ((i / map.NT) * H + h) * (int64_t)map.NT + i % map.NT;
        acc += part[rec];
    }
    buf[tid] = acc;
    __syncthreads();
    for (int s2 = kRedThreads / 2; s2 > 0; s2 >>= 1) {
        if (tid < s2)
            buf[tid] += buf[tid + s2];
        __syncthreads();
    }
    if (tid == 0)
        dA_log[h] = buf[0];
}

// cuTensorMapEncodeTiled, reached through the runtime (the library does not link the driver).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// One token tensor [B, T, H, D] (B = 0: a packed [T, H, D]) of bf16 as a tensor map with boxes
// of 64 channels x 1 head x 64 tokens, 128-byte swizzle, zeros outside the tensor.
cudaError_t make_token_map(CUtensorMap *m, const void *base, int D, int H, int64_t T, int B)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)(B > 0 ? B : 1)};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B > 0 ? 4 : 3, const_cast<void *>(base), dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// A float32 array of D x D state blocks (one per record) as a tensor map of nrec * D rows of D
// floats, boxes of 32 columns x D rows with the 128-byte swizzle (the scans' saved blocks).
cudaError_t make_state_map(CUtensorMap *m, float *base, int64_t nrec, int D)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    if (nrec * D >= ((int64_t)1 << 31))  // row coordinates are 32-bit
        return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(nrec * D)};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 4};
    const cuuint32_t box[2] = {(cuuint32_t)kBV, (cuuint32_t)D};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The gate table (launch_gate_table) lives in the workspace at `gtab`; the prep looks g up in it.
template <int D, bool kLogSig>
cudaError_t launch_prep_d(const SeqMap &m, int H, dim3 grid, const void *q, const void *k, const void *v,
                          const void *a, const void *beta, float g_min, const float *A_log, void *ws, float *gtab,
                          cudaStream_t s)
{
    unsigned int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidDevice;
    TokenMaps tm;
    const int B = m.cu ? 0 : m.nseq;
    cudaError_t e = make_token_map(&tm.q, q, D, H, m.T, B);
    if (e == cudaSuccess)
        e = make_token_map(&tm.k, k, D, H, m.T, B);
    if (e == cudaSuccess)
        e = make_token_map(&tm.v, v, D, H, m.T, B);
    if (e == cudaSuccess)
        e = make_token_map(&tm.a, a, D, H, m.T, B);
    if (e == cudaSuccess)
        e = launch_gate_table(kLogSig, (double)g_min, A_log, H, gtab, s);
    if (e != cudaSuccess)
        return e;
    const size_t smem = PrepLayout<D>::Bytes;
    e = cudaFuncSetAttribute(prep_kernel<D, kLogSig>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    prep_kernel<D, kLogSig><<<grid, kPrepThreads, smem, s>>>(tm, m, H, static_cast<const __nv_bfloat16 *>(beta), gtab,
                                                             A_log != nullptr && !kLogSig,
                                                             static_cast<unsigned char *>(ws), status);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_scan_d(const SeqMap &m, int H, const void *ws, const float *S0, void *o, float *S_T,
                          float *M_out, cudaStream_t s, float *Hs = nullptr)
{
    unsigned int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidDevice;
    cudaError_t e;
    if (!Hs && !M_out) {
        // the plain forward: two value blocks per CTA where one per CTA would need more CTAs
        // than the GPU has SMs (one scan CTA fits an SM), so the chains run in one wave
        int dev = 0, nsm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        if ((int64_t)m.nseq * H * (D / kBV) > nsm) {
            const size_t smem2 = sizeof(ScanSmem<D, false, 2>) + 1024;
            e = cudaFuncSetAttribute(scan_kernel<D, false, false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem2);
            if (e != cudaSuccess)
                return e;
            scan_kernel<D, false, false, 2><<<dim3(D / kBV / 2, m.nseq * H), scan_threads<2>(), smem2, s>>>(
                m, H, static_cast<const unsigned char *>(ws), S0, static_cast<__nv_bfloat16 *>(o), S_T, nullptr,
                CUtensorMap{}, status);
            return cudaGetLastError();
        }
    }
    // + alignment slack; the state-saving variant holds two more float32 blocks
    const size_t smem = (Hs ? sizeof(ScanSmem<D, true>) : sizeof(ScanSmem<D, false>)) + 1024;
    // with M_out: the state blocks and, after them, as many transfer-map blocks
    auto kernel = Hs ? scan_kernel<D, false, true> : M_out ? scan_kernel<D, true, false> : scan_kernel<D, false, false>;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    CUtensorMap hs_map{};
    if (Hs && (e = make_state_map(&hs_map, Hs, m.nrec, D)) != cudaSuccess)
        return e;
    kernel<<<dim3((M_out ? 2 : 1) * (D / kBV), m.nseq * H), kScanThreads, smem, s>>>(
        m, H, static_cast<const unsigned char *>(ws), S0, static_cast<__nv_bfloat16 *>(o), S_T, M_out, hs_map, status);
    return cudaGetLastError();
}

cudaError_t launch_prep(const SeqMap &m, int H, int D, dim3 grid, const void *q, const void *k, const void *v,
                        const void *a, const void *beta, float g_min, bool logsigmoid, const float *A_log, void *ws,
                        float *gtab, cudaStream_t s)
{
    if (logsigmoid)
        return D == 64 ? launch_prep_d<64, true>(m, H, grid, q, k, v, a, beta, g_min, A_log, ws, gtab, s)
                       : launch_prep_d<128, true>(m, H, grid, q, k, v, a, beta, g_min, A_log, ws, gtab, s);
    return D == 64 ? launch_prep_d<64, false>(m, H, grid, q, k, v, a, beta, g_min, A_log, ws, gtab, s)
                   : launch_prep_d<128, false>(m, H, grid, q, k, v, a, beta, g_min, A_log, ws, gtab, s);
}

// Bytes of the gate tables a workspace reserves: one per head (the per-head scale needs them).
size_t gate_table_bytes(int H) { return (size_t)H * kGateTableEntries * 4; }

cudaError_t launch_scan(const SeqMap &m, int H, int D, const void *ws, const float *S0, void *o, float *S_T,
                        cudaStream_t s, float *M_out = nullptr)
{
    return D == 64 ? launch_scan_d<64>(m, H, ws, S0, o, S_T, M_out, s)
                   : launch_scan_d<128>(m, H, ws, S0, o, S_T, M_out, s);
}

// Backward workspace: the forward records (and, for a packed batch, the chunk table), then the
// entering state of every chunk and the gradient of the state after it (fp32, D x D per
// record, in record order), the per-chunk partials of dL/dA_log, and the per-CTA scratch slots
// of bwd_chunk_kernel.
struct BwdLayout {
    size_t table, gtab, states, dstates, parts, scratch, total;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }
// A regular batch's backward workspace starts like the forward's: the records, then the gate
// table right after them (no padding), so the forward's prep output can be used in place.
static_assert(Rec<64>::Bytes % 256 == 0 && Rec<128>::Bytes % 256 == 0, "gate table at the forward's offset");

BwdLayout bwd_layout(int64_t nrec, int64_t nunits, int D, int H, int nseq_packed = 0)
{
    const size_t rec = D == 64 ? Rec<64>::Bytes : Rec<128>::Bytes;
    const size_t blk = (size_t)D * D * 4;
    const size_t slot = (size_t)(D == 64 ? BwdSlot<64>::floats : BwdSlot<128>::floats) * 4;
    BwdLayout l;
    l.table = (size_t)nrec * rec;
    l.gtab = round256(l.table + (nseq_packed ? (size_t)(nseq_packed + 1) * 4 : 0));
    l.states = round256(l.gtab + gate_table_bytes(H));
    l.dstates = l.states + (size_t)nrec * blk;
    l.parts = l.dstates + (size_t)nrec * blk;
    l.scratch = round256(l.parts + (size_t)nrec * 4);
    l.total = l.scratch + (size_t)std::min<int64_t>(nunits, kBwdSlots) * slot;
    return l;
}

template <int D>
cudaError_t launch_bwd_d(const SeqMap &m, int H, dim3 prep_grid, int64_t nunits, const BwdLayout &l,
                         const void *q, const void *k, const void *v, const void *a, const void *beta, float g_min,
                         const float *A_log, const float *S0, const void *dO, const float *dS_T, float *dq, float *dk,
                         float *dv, float *da, float *dbeta, float *dS0, float *dA_log, void *ws, cudaStream_t s,
                         bool have_records = false)
{
    unsigned int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidDevice;
    unsigned char *base = static_cast<unsigned char *>(ws);
    float *Hs = reinterpret_cast<float *>(base + l.states), *dHs = reinterpret_cast<float *>(base + l.dstates);
    float *parts = dA_log ? reinterpret_cast<float *>(base + l.parts) : nullptr;
    float *scratch = reinterpret_cast<float *>(base + l.scratch);
    float *gtab = reinterpret_cast<float *>(base + l.gtab);
    // the records and the gate table (same offsets as the forward's workspace) unless the
    // forward's prep already wrote them there
    cudaError_t e = have_records ? cudaSuccess
                                 : launch_prep_d<D, false>(m, H, prep_grid, q, k, v, a, beta, g_min, A_log, ws, gtab, s);
    if (e == cudaSuccess)
        e = launch_scan_d<D>(m, H, ws, S0, nullptr, nullptr, nullptr, s, Hs);
    if (e != cudaSuccess)
        return e;
    const size_t smem = sizeof(DScanSmem<D>) + 1024;
    e = cudaFuncSetAttribute(dscan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    CUtensorMap dhs_map{};
    if ((e = make_state_map(&dhs_map, dHs, m.nrec, D)) != cudaSuccess)
        return e;
    dscan_kernel<D><<<dim3(D / kBV, m.nseq * H), kScanThreads, smem, s>>>(
        m, H, static_cast<const unsigned char *>(ws), static_cast<const __nv_bfloat16 *>(dO), dS_T, dhs_map, dS0,
        status);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int grid = (int)std::min<int64_t>(nunits, kBwdSlots);
    e = cudaFuncSetAttribute(bwd_chunk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BwdSmem<D>::bytes);
    if (e != cudaSuccess)
        return e;
    bwd_chunk_kernel<D><<<grid, kBwdThreads, BwdSmem<D>::bytes, s>>>(
        m, H, (int)nunits, static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(a),
        static_cast<const __nv_bfloat16 *>(beta), g_min, A_log, gtab, static_cast<const __nv_bfloat16 *>(dO), Hs,
        dHs, scratch, dq, dk, dv, da, dbeta, parts, status);
    e = cudaGetLastError();
    if (e != cudaSuccess || !dA_log)
        return e;
    dalog_reduce_kernel<<<H, kRedThreads, 0, s>>>(m, H, parts, dA_log);
    return cudaGetLastError();
}

SeqMap regular_map(int B, int T, int H)
{
    SeqMap m;
    m.nseq = B;
    m.T = T;
    m.NT = (T + kC - 1) / kC;
    m.nrec = (int64_t)B * H * m.NT;
    m.ntok = (int64_t)B * T;
    return m;
}

// ------------------------------------------------------------------ packed-batch chunk table
// One CTA: checks cu (cu[0] = 0, non-decreasing, cu[N] = T) and writes choff[s] = sum over
// earlier sequences of ceil(len/64).  An invalid cu records KDA_ERR_INVALID_ARG and leaves an
// all-zero table, so the prep and scan that follow touch nothing but S_T (= S0).
constexpr int kTableThreads = 1024;

__global__ void __launch_bounds__(kTableThreads)
    seq_table_kernel(const int32_t *__restrict__ cu, int N, int T, int32_t *__restrict__ choff, unsigned int *status)
{
    __shared__ int32_t part[kTableThreads];
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0)
        bad = (cu[0] != 0 || cu[N] != T) ? 1 : 0;
    __syncthreads();
    for (int s0 = 0; s0 < N; s0 += kTableThreads) {
        const int s = s0 + tid;
        if (s < N && cu[s + 1] < cu[s])
            bad = 1;
    }
    __syncthreads();
    const bool ok = bad == 0;
    int carry = 0;
    if (tid == 0)
        choff[0] = 0;
    for (int s0 = 0; s0 < N; s0 += kTableThreads) {
        const int s = s0 + tid;
        const int len = (ok && s < N) ? cu[s + 1] - cu[s] : 0;
        part[tid] = (len + kC - 1) / kC;
        __syncthreads();
        for (int d = 1; d < kTableThreads; d <<= 1) {  // inclusive scan (Hillis-Steele)
            const int x = tid >= d ? part[tid - d] : 0;
            __syncthreads();
            part[tid] += x;
            __syncthreads();
        }
        if (s < N)
            choff[s + 1] = carry + part[tid];
        carry += part[kTableThreads - 1];
        __syncthreads();
    }
    if (!ok && tid == 0)
        report_device_error(status, KDA_ERR_INVALID_ARG);
}

size_t varlen_records(int N, int T) { return ((size_t)T + kC - 1) / kC + (size_t)N; }

}  // namespace

size_t chunk_bf16_records(int B, int T, int H, int D)
{
    const size_t NT = ((size_t)T + kC - 1) / kC;
    const size_t rec = D == 64 ? Rec<64>::Bytes : Rec<128>::Bytes;
    return (size_t)B * H * NT * rec;
}

size_t chunk_bf16_workspace(int B, int T, int H, int D) { return chunk_bf16_records(B, T, H, D) + gate_table_bytes(H); }

cudaError_t launch_prep_bf16(int B, int T, int H, int D, const void *q, const void *k, const void *v,
                             const void *a, const void *beta, float g_min, bool logsigmoid, const float *A_log,
                             void *workspace, cudaStream_t s)
{
    const SeqMap m = regular_map(B, T, H);
    float *gtab = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + chunk_bf16_records(B, T, H, D));
    return launch_prep(m, H, D, dim3(m.NT, B * H), q, k, v, a, beta, g_min, logsigmoid, A_log, workspace, gtab, s);
}

cudaError_t launch_scan_bf16(int B, int T, int H, int D, const void *workspace, const float *S0, void *o,
                             float *S_T, cudaStream_t s)
{
    return launch_scan(regular_map(B, T, H), H, D, workspace, S0, o, S_T, s);
}

cudaError_t launch_scan_affine_bf16(int B, int T, int H, int D, const void *workspace, float *S_zero, float *M,
                                    cudaStream_t s)
{
    return launch_scan(regular_map(B, T, H), H, D, workspace, nullptr, nullptr, S_zero, s, M);
}

size_t chunk_bf16_bwd_workspace(int B, int T, int H, int D)
{
    const SeqMap m = regular_map(B, T, H);
    return bwd_layout(m.nrec, m.nrec, D, H).total;
}

void chunk_bf16_bwd_offsets(int B, int T, int H, int D, size_t *states, size_t *dstates)
{
    const SeqMap m = regular_map(B, T, H);
    const BwdLayout l = bwd_layout(m.nrec, m.nrec, D, H);
    *states = l.states;
    *dstates = l.dstates;
}

cudaError_t launch_chunk_bwd_bf16(int B, int T, int H, int D, const void *q, const void *k, const void *v,
                                  const void *a, const void *beta, float g_min, const float *A_log, const float *S0,
                                  const void *dO, const float *dS_T, float *dq, float *dk, float *dv, float *da,
                                  float *dbeta, float *dS0, float *dA_log, void *workspace, cudaStream_t s,
                                  bool have_records)
{
    const SeqMap m = regular_map(B, T, H);
    const dim3 grid(m.NT, B * H);
    const BwdLayout l = bwd_layout(m.nrec, m.nrec, D, H);
    return D == 64 ? launch_bwd_d<64>(m, H, grid, m.nrec, l, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk, dv,
                                      da, dbeta, dS0, dA_log, workspace, s, have_records)
                   : launch_bwd_d<128>(m, H, grid, m.nrec, l, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk,
                                       dv, da, dbeta, dS0, dA_log, workspace, s, have_records);
}

size_t chunk_bf16_bwd_varlen_workspace(int N, int T, int H, int D)
{
    const int64_t nrec = (int64_t)H * (int64_t)varlen_records(N, T);
    return bwd_layout(nrec, nrec, D, H, N).total;
}

cudaError_t launch_chunk_bwd_bf16_varlen(int N, const int32_t *cu, int T, int H, int D, const void *q, const void *k,
                                         const void *v, const void *a, const void *beta, float g_min,
                                         const float *A_log, const float *S0, const void *dO, const float *dS_T,
                                         float *dq, float *dk, float *dv, float *da, float *dbeta, float *dS0,
                                         float *dA_log, void *workspace, cudaStream_t s)
{
    unsigned int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidDevice;
    SeqMap m;
    m.cu = cu;
    m.nseq = N;
    m.T = T;
    m.NT = (int)varlen_records(N, T);
    m.nrec = (int64_t)H * m.NT;
    m.ntok = T;
    const BwdLayout l = bwd_layout(m.nrec, m.nrec, D, H, N);
    int32_t *choff = reinterpret_cast<int32_t *>(static_cast<unsigned char *>(workspace) + l.table);
    m.choff = choff;
    seq_table_kernel<<<1, kTableThreads, 0, s>>>(cu, N, T, choff, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const dim3 grid(m.NT, H);
    return D == 64 ? launch_bwd_d<64>(m, H, grid, m.nrec, l, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk, dv,
                                      da, dbeta, dS0, dA_log, workspace, s)
                   : launch_bwd_d<128>(m, H, grid, m.nrec, l, q, k, v, a, beta, g_min, A_log, S0, dO, dS_T, dq, dk,
                                       dv, da, dbeta, dS0, dA_log, workspace, s);
}

// ------------------------------------------------------------------ segment combine
// S_in[0] = S0 (or 0); S_in[r + 1] = M[r] S_in[r] + S_zero[r], r < R.  One CTA per
// (32-column block, b*h) keeps its block of the running state in shared memory; thread t
// computes row t / 2, columns (t % 2) * 16 .. + 16 of the next one.  Float32 FMAs.
constexpr int kCombThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombThreads)
    combine_kernel(int R, int BH, const float *__restrict__ M, const float *__restrict__ S_zero,
                   const float *__restrict__ S0, float *__restrict__ S_in)
{
    __shared__ float Sb[D][kBV + 1];
    const int tid = threadIdx.x, col0 = blockIdx.x * kBV, bh = blockIdx.y;
    const size_t mstride = (size_t)BH * D * D;  // one segment's maps (and states: dk == dv)
    for (int i = tid; i < D * kBV; i += kCombThreads) {
        const int r = i / kBV, c = i % kBV;
        const float v = S0 ? S0[((size_t)bh * D + r) * D + col0 + c] : 0.0f;
        Sb[r][c] = v;
        S_in[((size_t)bh * D + r) * D + col0 + c] = v;
    }
    __syncthreads();
    static_assert(2 * D <= 2 * kCombThreads && kBV == 32, "two threads per row, 16 columns each");
    for (int seg = 0; seg < R; ++seg) {
        const float *Mr = M + seg * mstride + (size_t)bh * D * D;
        const float *Zr = S_zero + seg * mstride + (size_t)bh * D * D;
        float acc[16];
        const int row = tid / 2, cb = (tid % 2) * 16;
        const bool live = row < D;
        if (live) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                acc[j] = Zr[(size_t)row * D + col0 + cb + j];
            for (int k4 = 0; k4 < D; k4 += 4) {
                const float4 m = *reinterpret_cast<const float4 *>(&Mr[(size_t)row * D + k4]);
                const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        acc[j] = fmaf(mk[kk], Sb[k4 + kk][cb + j], acc[j]);
            }
        }
        __syncthreads();
        if (live)
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                Sb[row][cb + j] = acc[j];
                S_in[(seg + 1) * mstride + ((size_t)bh * D + row) * D + col0 + cb + j] = acc[j];
            }
        __syncthreads();
    }
}

cudaError_t launch_combine(int R, int BH, int D, const float *M, const float *S_zero, const float *S0, float *S_in,
                           cudaStream_t s)
{
    const dim3 grid(D / kBV, BH);
    if (D == 64)
        combine_kernel<64><<<grid, kCombThreads, 0, s>>>(R, BH, M, S_zero, S0, S_in);
    else
        combine_kernel<128><<<grid, kCombThreads, 0, s>>>(R, BH, M, S_zero, S0, S_in);
    return cudaGetLastError();
}

size_t chunk_bf16_varlen_workspace(int N, int T, int H, int D)
{
    const size_t rec = D == 64 ? Rec<64>::Bytes : Rec<128>::Bytes;
    const size_t table = ((size_t)(N + 1) * 4 + 255) / 256 * 256;
    return (size_t)H * varlen_records(N, T) * rec + table + gate_table_bytes(H);
}

cudaError_t launch_chunk_bf16_varlen(int N, const int32_t *cu, int T, int H, int D, const void *q, const void *k,
                                     const void *v, const void *a, const void *beta, float g_min, bool logsigmoid,
                                     const float *A_log, const float *S0, void *o, float *S_T, void *workspace,
                                     cudaStream_t s)
{
    unsigned int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidDevice;
    const size_t rec = D == 64 ? Rec<64>::Bytes : Rec<128>::Bytes;
    SeqMap m;
    m.cu = cu;
    m.nseq = N;
    m.T = T;
    m.NT = (int)varlen_records(N, T);
    m.nrec = (int64_t)H * m.NT;
    m.ntok = T;
    int32_t *choff = reinterpret_cast<int32_t *>(static_cast<unsigned char *>(workspace) + (size_t)H * m.NT * rec);
    m.choff = choff;
    seq_table_kernel<<<1, kTableThreads, 0, s>>>(cu, N, T, choff, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    float *gtab = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(choff) +
                                            ((size_t)(N + 1) * 4 + 255) / 256 * 256);
    e = launch_prep(m, H, D, dim3(m.NT, H), q, k, v, a, beta, g_min, logsigmoid, A_log, workspace, gtab, s);
    if (e != cudaSuccess)
        return e;
    return launch_scan(m, H, D, workspace, S0, o, S_T, s);
}

}  // namespace kda
