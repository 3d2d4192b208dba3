// oal_tc.cu -- tcgen05 / TMA kernels of the bf16 chunked prefill on B200 (sm_100a).
//
// Equations: "OAL: 按 QK 离群贡献分组的正二次注意力核" (reproduction note of arXiv 2610.13674),
// section 核心公式, numbered in order of appearance: (2) grouped score, (3) kernel kappa,
// (4) prefix states, (5) readout.  With the packed feature map of oal_common.cuh, the state
// of a (b, kv) head after token i is S_i = sum_{j<=i} psi(k_j) [v_j; 1] (2176 x 65) and
// u_i = phi(q_i)^T S_i.  Chunked with C = 128 tokens, the prefill runs as three kernels:
//
//   chunk deltas (b, kv, chunk c, slab of 128 packed rows; every unit independent):
//     producer warps build psi(K_c)^T (MN-major, bf16) in shared memory, split exactly into
//     hi = bf16(psi) and lo = psi - hi; N=80 MMAs accumulate dS_c = psi(K_c)^T [V_c; 1] in
//     TMEM (the [.; 1] column comes from a constant "ones" atom addressed through the B
//     descriptor's leading byte offset) and epilogue warps store it in fp32.
//   prefix scan (SIMT, memory bound): S_c = sum_{c' < c} dS_c' for every chunk, written as
//     bf16 K-major B-operand images, and the final state S_NC in fp32 (eq. 4 in chunk form).
//   readout (b, h, chunk c): 128 query rows of one head.  The intra-chunk kernel runs first
//     on tensor cores in the factored form of eq. (3),
//       kappa = eps + sum_m (L_0m + (q o w_m) . k)^2,   w_m[r] = L_{g(r),m} / sqrt(d)
//     (= ||L^T sbar||^2): score tiles S_m = (Q o w_m) K^T in TMEM, kappa accumulated in
//     registers, masked causally and multiplied into [V_c; 1].  Then phi(Q_c) is written
//     straight into tensor memory (tcgen05.st) slice by slice and multiplied with the image
//     of S_c by N=80 MMAs reading A from TMEM, into the same accumulator; finally
//     yhat = u[:64] / u[64] (eq. 5).
//
// Every wait is bounded (1 s); one that runs out sets OAL_ERR_TIMEOUT and the CTA leaves its
// loops in order (copies drained, MMAs committed, TMEM freed) instead of hanging.
#include <algorithm>
#include <mutex>
#include <utility>

#include <cuda.h>

#include "oal_common.cuh"
#include "oal_kernels.cuh"
#include "oal_tc_util.cuh"

namespace oal {
namespace tc {

constexpr int kC = 128;                                    // chunk = tile rows
constexpr int kSlabRows = 128;                             // packed rows per builder item
constexpr int kNumSlabs = kFP / kSlabRows;                 // 17
constexpr int kSlices = kFP / 64;                          // 34 readout K-slices
constexpr int kOffDiagSlices = kOffDiagRows / 64;          // 28
constexpr uint32_t kImgSliceBytes = 80 * 64 * 2;           // K-major [80 n][64 rows]
constexpr uint32_t kImgLoadBytes = 65 * 128;               // rows 0..64 (65..79 are zero)
constexpr size_t kImgChunkBytes = size_t(kSlices) * kImgSliceBytes;
constexpr uint32_t kTileBytes = kC * 64 * 2;               // 16384: one 128 x 64 bf16 tile
constexpr uint32_t kOnesAtomBytes = kC * 128;              // 16384: 128 rows x 128 B
constexpr uint16_t kBf16One = 0x3F80;

constexpr int kWarps = 18;
constexpr int kThreads = kWarps * 32;
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;
constexpr uint32_t kTmemCols = 512;

static_assert(kFP % kSlabRows == 0 && kFP % 64 == 0, "feature padding");

// ---- shared memory (offsets from a 1024-aligned base) ---------------------------------------
// reader
constexpr uint32_t kRdOffK = 0;           // K tile (score B operand, K-major)
constexpr uint32_t kRdOffV = 16384;       // V tile (PV B operand, MN-major)
constexpr uint32_t kRdOffQ = 32768;       // Q tile (bf16, K-major): phi and Aq read it
constexpr uint32_t kRdOffAq = 49152;      // Aq0 | Aq1 (score A operands); the P tile aliases
constexpr uint32_t kRdOffA = 81920;       // 4 x 16 KB phi stages (readout A operand, K-major)
constexpr uint32_t kRdOffB = 147456;      // 2 x 20 KB state-image stages of 2 slices (B operand)
constexpr uint32_t kRdOffCoef = 188416;   // 2176 fp32 coefficients
constexpr uint32_t kRdOffCoefH = 197120;  // 1792 bf16 coefficients of the off-diagonal rows
constexpr uint32_t kRdOffW = 200704;      // 9 x 64 fp32
constexpr uint32_t kRdOffC0 = 203008;     // 9 fp32
constexpr uint32_t kRdOffOnes = 203776;   // 16 KB ones atom; then image stage 2 (20 KB) reuses it
// chunk-delta builder
constexpr uint32_t kStOffKV = 0;          // 3 x (K 16 KB + V 16 KB)
constexpr uint32_t kStOffA = 98304;       // 3 x (hi 16 KB + lo 16 KB) psi stages
constexpr uint32_t kOffOnes = 196608;     // 16 KB ones atom
// both
constexpr uint32_t kOffCtl = 224256;      // barriers and control words
constexpr uint32_t kSmemBytes = kOffCtl + 1024 + 1024;

constexpr int kPhiSets = 4;                                // reader warps (w >> 2) per slice
// phi stages (SMEM, 1 slice): two per warp set (stages kq and kq + 4), so that every wait on
// a stage barrier is for the phase right after the one the waiter last saw complete (parity
// waits cannot tell phases two apart).  Stages 0..3 have their own region; stages 4..7 reuse
// the K, V and Aq | P tiles once the intra-chunk MMAs that read them have completed.
constexpr int kRdStages = 2 * kPhiSets;
// image stages (SMEM, 2 slices each): stages 0, 1 have their own region, stage 2 reuses the
// ones atom once the intra-chunk P [V | 1] MMAs have completed
constexpr int kBStages = 3;
constexpr uint32_t kImgPairBytes = 2 * kImgSliceBytes;     // one tensor copy: 160 rows
constexpr uint32_t kPhiTileBytes = kC * 64 * 2;            // 128 rows x 64 packed rows, bf16
constexpr int kKVStages = 3;
constexpr int kDAStages = 3;  // psi stages (hi + lo tiles of one half chunk)
constexpr int kDAcc = 4;      // TMEM accumulators of the delta builder (128 columns each)
constexpr uint32_t kStATile = 64 * kSlabRows * 2;          // 64 tokens x 128 rows = 16 KB
// reader TMEM map: U in [0, 80); score tiles S0 | S1 in [128, 384).  phi stays in shared
// memory: warp stores into tensor memory stall concurrent MMAs, shared-memory stores do not.
constexpr uint32_t kColU = 0, kColS0 = 128;
static_assert(kStOffKV + kKVStages * 2 * kTileBytes <= kStOffA &&
                  kStOffA + kDAStages * 2 * kStATile <= kOffOnes &&
                  kOffOnes + kOnesAtomBytes <= kOffCtl && kDAcc * 128 <= int(kTmemCols),
              "delta builder shared-memory and TMEM map");
__host__ __device__ constexpr uint32_t rd_stage_off(int st)
{
    return st < kPhiSets ? kRdOffA + uint32_t(st) * kPhiTileBytes
                         : (st == 4 ? kRdOffK : st == 5 ? kRdOffV : kRdOffAq + (st - 6) * kTileBytes);
}
static_assert(kRdOffK + kTileBytes <= kRdOffV && kRdOffV + kTileBytes <= kRdOffQ &&
                  kRdOffAq + 2 * kTileBytes <= kRdOffA && kTileBytes == kPhiTileBytes,
              "reused phi stages");
__host__ __device__ constexpr uint32_t rd_bstage_off(int bs)
{
    return bs < 2 ? kRdOffB + uint32_t(bs) * kImgPairBytes : kRdOffOnes;
}
static_assert(kRdOffA + kPhiSets * kPhiTileBytes <= kRdOffB &&
                  kRdOffB + 2 * kImgPairBytes <= kRdOffCoef && kRdOffC0 + 64 <= kRdOffOnes &&
                  kRdOffOnes % 1024 == 0 && kRdOffOnes + kImgPairBytes <= kOffCtl &&
                  kOnesAtomBytes <= kImgPairBytes,
              "reader shared-memory map");

struct RdBars {
    uint64_t qkv_full, aq_full[2], s_full[2], s_empty[2], p_full, pv_done;
    uint64_t a_full[kRdStages], a_empty[kRdStages], b_full[kBStages], b_empty[kBStages];
    uint64_t u_full, done;
};
struct StBars {
    uint64_t kv_full[kKVStages], kv_empty[kKVStages], a_full[kDAStages], a_empty[kDAStages];
    uint64_t acc_full[kDAcc], acc_empty[kDAcc], done;
};
struct Ctl {
    union {
        RdBars rd;
        StBars st;
        uint64_t raw[64];
    } bar;
    uint32_t tmem_base;
    int abort_flag;
    int G;
};
static_assert(sizeof(Ctl) <= 1024, "control block");
static_assert(sizeof(RdBars) <= sizeof(uint64_t) * 64 && sizeof(StBars) <= sizeof(uint64_t) * 64,
              "barrier block");

struct Params {
    const CUtensorMap* tm_q;
    const CUtensorMap* tm_k;
    const CUtensorMap* tm_v;
    const CUtensorMap* tm_img;  // chunk-state images as {64 f, slices * 80 rows}, box {64, 160}
    const int32_t* gid;
    const float* L;
    const int32_t* G;
    float eps;
    const float* coef_all;   // state header coefficient table [Hq][kFP]
    unsigned char* img;      // chunk-state images [B*Hkv][NC][34 slices][80 n][64 f] bf16
    float* dS;               // chunk deltas [B*Hkv][NC][65][kFP] fp32
    float* out;
    int B, Hq, Hkv, T, NC;
    int cont;                // 1: the state already holds a prefix; these tokens continue it
};

// ------------------------------------------------------------------------------------------
// helpers
// ------------------------------------------------------------------------------------------
template <typename F, int... I>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, I...>)
{
    (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F&& f)
{
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void bounded_spin_done(uint64_t* bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kWaitLimitNs) {
    }
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16x2(v.x, v.y); }





// MN-major SW128 atom whose N-element 0 is 1 for every K row (the [.; 1] column of [V; 1])
__device__ __forceinline__ void init_ones_atom(unsigned char* atom)
{
    for (int e = threadIdx.x; e < int(kOnesAtomBytes / 4); e += blockDim.x)
        reinterpret_cast<uint32_t*>(atom)[e] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < kC; j += blockDim.x)
        *reinterpret_cast<uint16_t*>(atom + (j >> 3) * 1024 + (j & 7) * 128 + (j & 7) * 16) =
            kBf16One;
}

// (R, T) of the 28 off-diagonal 8 x 8 blocks (R < T, lexicographic), as 8 R + T
#define OAL_BLOCK_RT                                                                       \
    1, 2, 3, 4, 5, 6, 7, 10, 11, 12, 13, 14, 15, 19, 20, 21, 22, 23, 28, 29, 30, 31, 37, 38, \
        39, 46, 47, 55
constexpr uint8_t kBlockRT[kOffDiagSlices] = {OAL_BLOCK_RT};
__constant__ uint8_t c_block_rt[kOffDiagSlices] = {OAL_BLOCK_RT};
#undef OAL_BLOCK_RT
constexpr bool block_rt_table_ok()
{
    for (int s = 0; s < kOffDiagSlices; ++s) {
        const RT rt = feature_rt(64 * s);
        if (rt.r != 8 * (kBlockRT[s] >> 3) || rt.t != 8 * (kBlockRT[s] & 7)) return false;
    }
    return true;
}
static_assert(block_rt_table_ok(), "off-diagonal block table");

// ------------------------------------------------------------------------------------------
// chunk-delta builder: psi producers (thread = token j of a half chunk, quarter qf of the
// slab's 128 rows).  psi = k_r k_t of two bf16 values has at most 16 significant bits, so it
// splits exactly into hi = bf16(psi) and lo = psi - hi (also a bf16 value); both are written
// as MN-major A tiles and the MMA accumulates hi^T [V; 1] + lo^T [V; 1] in fp32.
// ------------------------------------------------------------------------------------------
// MN-major A tile (128 rows x 64 tokens): the 8-row chunk starting at row m for token j
__device__ __forceinline__ uint32_t st_a_off(int m, int j)
{
    return uint32_t((m >> 6) * 8192 + (j >> 3) * 1024 + (j & 7) * 128 +
                    ((((m & 63) >> 3) ^ (j & 7)) << 4));
}

// a * b + c on packed bf16 pairs, one rounding
__device__ __forceinline__ uint32_t bfma2(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// off-diagonal slabs: 32 rows = 4 dims a of block R times the 8 dims of block T.  They never
// involve the constant slot, and K rows past T are zero-filled by the copy.
__device__ __forceinline__ void psi_offdiag(const unsigned char* ktile, int trow, uint32_t abase,
                                            int j, int slab, int qf)
{
    const int rt = c_block_rt[2 * slab + (qf >> 1)];
    const uint2 wa =
        *reinterpret_cast<const uint2*>(ktile + kmajor_chunk(trow, rt >> 3) + 8 * (qf & 1));
    const uint4 wt = *reinterpret_cast<const uint4*>(ktile + kmajor_chunk(trow, rt & 7));
    const uint32_t xs[4] = {dup_lo(wa.x), dup_hi(wa.x), dup_lo(wa.y), dup_hi(wa.y)};
    const int m0 = 64 * (qf >> 1) + 32 * (qf & 1);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const uint32_t h0 = bmul2(xs[a], wt.x), h1 = bmul2(xs[a], wt.y);
        const uint32_t h2 = bmul2(xs[a], wt.z), h3 = bmul2(xs[a], wt.w);
        const uint32_t off = st_a_off(m0 + 8 * a, j);
        sts128(abase + off, h0, h1, h2, h3);
        sts128(abase + kStATile + off, bfma2(xs[a], wt.x, h0 ^ 0x80008000u),
               bfma2(xs[a], wt.y, h1 ^ 0x80008000u), bfma2(xs[a], wt.z, h2 ^ 0x80008000u),
               bfma2(xs[a], wt.w, h3 ^ 0x80008000u));
    }
}

template <int F0>
constexpr bool psi_chunk_needed(int ch)
{
    for (int i = 0; i < 32; ++i) {
        const RT rt = feature_rt(F0 + i);
        if ((rt.r < 64 && rt.r / 8 == ch) || (rt.t < 64 && rt.t / 8 == ch)) return true;
    }
    return false;
}

// diagonal / linear / constant slabs: 32 rows with compile-time (r, t); fp32 products (exact)
// split into hi and lo
template <int F0>
__device__ __forceinline__ void psi_static(const unsigned char* ktile, int trow, float one,
                                           uint32_t abase, int j)
{
    float k[66];
    static_for<8>([&](auto CH) {
        constexpr int ch = decltype(CH)::value;
        if constexpr (psi_chunk_needed<F0>(ch)) {
            const uint4 w = *reinterpret_cast<const uint4*>(ktile + kmajor_chunk(trow, ch));
            k[ch * 8 + 0] = bf16lo_to_f32(w.x);
            k[ch * 8 + 1] = bf16hi_to_f32(w.x);
            k[ch * 8 + 2] = bf16lo_to_f32(w.y);
            k[ch * 8 + 3] = bf16hi_to_f32(w.y);
            k[ch * 8 + 4] = bf16lo_to_f32(w.z);
            k[ch * 8 + 5] = bf16hi_to_f32(w.z);
            k[ch * 8 + 6] = bf16lo_to_f32(w.w);
            k[ch * 8 + 7] = bf16hi_to_f32(w.w);
        }
    });
    k[64] = one;
    k[65] = 0.f;
    constexpr int m0 = F0 % kSlabRows;
    static_for<4>([&](auto CH) {
        constexpr int ch = decltype(CH)::value;
        uint32_t h[4], l[4];
        static_for<4>([&](auto E) {
            constexpr int e = decltype(E)::value;
            constexpr RT a = feature_rt(F0 + ch * 8 + 2 * e);
            constexpr RT b = feature_rt(F0 + ch * 8 + 2 * e + 1);
            const float pa = k[a.r] * k[a.t], pb = k[b.r] * k[b.t];
            h[e] = pack_bf16x2(pa, pb);
            l[e] = pack_bf16x2(pa - bf16lo_to_f32(h[e]), pb - bf16hi_to_f32(h[e]));
        });
        sts128(abase + st_a_off(m0 + 8 * ch, j), h[0], h[1], h[2], h[3]);
        sts128(abase + kStATile + st_a_off(m0 + 8 * ch, j), l[0], l[1], l[2], l[3]);
    });
}

__device__ __forceinline__ void psi_tile(int slab, int qf, const unsigned char* ktile, int trow,
                                         float one, uint32_t abase, int j)
{
    if (slab < kOffDiagSlices / 2) {
        psi_offdiag(ktile, trow, abase, j, slab, qf);
        return;
    }
    const int sel = (slab - kOffDiagSlices / 2) * 4 + qf;
    static_for<(kNumSlabs - kOffDiagSlices / 2) * 4>([&](auto I) {
        constexpr int i = decltype(I)::value;
        if (sel == i) psi_static<kOffDiagRows + i * 32>(ktile, trow, one, abase, j);
    });
}

// unit u -> (bkv, chunk c, slab); slabs of one chunk are consecutive
struct DeltaUnit {
    int bkv, c, slab;
};
__device__ __forceinline__ DeltaUnit delta_unit(int u, int NC)
{
    const int rest = u / kNumSlabs;
    return DeltaUnit{rest / NC, rest % NC, u % kNumSlabs};
}

// ------------------------------------------------------------------------------------------
// chunk-delta item: units [u0, u1), each dS_c = psi(K_c)^T [V_c; 1] for the 128 packed rows
// of one slab, stored in fp32 as dS[bkv][c][n][f] (n = column of [v; 1]).
// Warps 0-7 psi producers, 8-15 epilogue, 16 TMA, 17 MMA.
// ------------------------------------------------------------------------------------------
__device__ void delta_item(unsigned char* sm, Ctl& ctl, uint32_t tmem, const Params& P, int u0,
                           int u1)
{
    StBars& bar = ctl.bar.st;
    volatile int* abort_flag = &ctl.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NC = P.NC, T = P.T, nu = u1 - u0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKVStages; ++i) {
            mbar_init(&bar.kv_full[i], 1);
            mbar_init(&bar.kv_empty[i], 8 + 1);
        }
        for (int i = 0; i < kDAStages; ++i) {
            mbar_init(&bar.a_full[i], 8);
            mbar_init(&bar.a_empty[i], 1);
        }
        for (int i = 0; i < kDAcc; ++i) {
            mbar_init(&bar.acc_full[i], 1);
            mbar_init(&bar.acc_empty[i], 8);
        }
        mbar_init(&bar.done, 1);
        ctl.abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == kTmaWarp) {
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < nu; ++i) {
                const DeltaUnit du = delta_unit(u0 + i, NC);
                const int s = i % kKVStages;
                if (i >= kKVStages &&
                    !mbar_wait(&bar.kv_empty[s], ((i / kKVStages) - 1) & 1, abort_flag))
                    break;
                unsigned char* kvs = sm + kStOffKV + s * 2 * kTileBytes;
                mbar_expect_tx(&bar.kv_full[s], 2 * kTileBytes);
                tma_load_3d(kvs, P.tm_k, &bar.kv_full[s], 0, du.c * kC, du.bkv);
                tma_load_3d(kvs + kTileBytes, P.tm_v, &bar.kv_full[s], 0, du.c * kC, du.bkv);
                ++issued;
            }
            for (int i = max(0, issued - kKVStages); i < issued; ++i)
                bounded_spin_done(&bar.kv_full[i % kKVStages], (i / kKVStages) & 1);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // the whole warp runs the issue loop; one elected lane issues
        constexpr uint32_t id = idesc_bf16(128, 80, true, true);
        const uint32_t a0 = smem_u32(sm + kStOffA), kv0 = smem_u32(sm + kStOffKV);
        const uint32_t ones = smem_u32(sm + kOffOnes);
        bool ok = true;
        for (int i = 0; i < nu && ok; ++i) {
            const int s = i % kDAcc, st = i % kKVStages;
            if (i >= kDAcc) ok = mbar_wait(&bar.acc_empty[s], ((i / kDAcc) - 1) & 1, abort_flag);
            if (ok) ok = mbar_wait(&bar.kv_full[st], (i / kKVStages) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const uint32_t d = tmem + s * 128;
            const uint32_t vt = kv0 + st * 2 * kTileBytes + kTileBytes;
            const uint32_t lbo = ones - vt;  // V atom -> ones atom (N elements 64..)
            for (int hc = 0; hc < 2; ++hc) {
                const int w = 2 * i + hc, as = w % kDAStages;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bar.a_full[as], (w / kDAStages) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t ab = a0 + as * 2 * kStATile;
#pragma unroll
                    for (int x = 0; x < 8; ++x) {  // hi (x < 4), lo (x >= 4) over 4 K-steps
                        const int ks = x & 3;
                        mma_bf16(d, sdesc_sw128(ab + (x >> 2) * kStATile + ks * 2048, 8192, 1024),
                                 sdesc_sw128(vt + hc * 8192 + ks * 2048, lbo, 1024), id,
                                 (hc | x) ? 1u : 0u);
                    }
                    mma_commit(&bar.a_empty[as]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) {
                mma_commit(&bar.acc_full[s]);
                mma_commit(&bar.kv_empty[st]);
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(&bar.done);
        __syncwarp();
        if (lane == 0) bounded_spin_done(&bar.done, 0);
        __syncwarp();
    } else if (warp < 8) {
        const int t = threadIdx.x, j = t & 63, qf = t >> 6;
        const uint32_t a0 = smem_u32(sm + kStOffA);
        for (int i = 0; i < nu; ++i) {
            const DeltaUnit du = delta_unit(u0 + i, NC);
            const int st = i % kKVStages;
            if (!mbar_wait(&bar.kv_full[st], (i / kKVStages) & 1, abort_flag)) break;
            const unsigned char* kt = sm + kStOffKV + st * 2 * kTileBytes;
            bool ok = true;
            for (int hc = 0; hc < 2; ++hc) {
                const int w = 2 * i + hc, as = w % kDAStages;
                if (w >= kDAStages &&
                    !mbar_wait(&bar.a_empty[as], ((w / kDAStages) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int trow = hc * 64 + j;
                const float one = (du.c * kC + trow < T) ? 1.f : 0.f;
                psi_tile(du.slab, qf, kt, trow, one, a0 + as * 2 * kStATile, j);
                fence_proxy_async();
                warp_arrive(&bar.a_full[as]);
            }
            if (!ok) break;
            warp_arrive(&bar.kv_empty[st]);
        }
    } else {
        // epilogue: thread = (packed row of the slab, column half)
        const int q4 = warp & 3, hfe = (warp - 8) >> 2;
        const int fl = q4 * 32 + lane;
        for (int i = 0; i < nu; ++i) {
            const DeltaUnit du = delta_unit(u0 + i, NC);
            const int s = i % kDAcc;
            // all epilogue threads leave together, so no named barrier is left half-joined
            const bool got = mbar_wait(&bar.acc_full[s], (i / kDAcc) & 1, abort_flag);
            if (!named_bar_and(2, 256, got)) break;
            tc_fence_after();
            const uint32_t lanebase = tmem + (uint32_t(q4 * 32) << 16) + s * 128;
            float v0[16], v1[16], vz[16];
            tmem_ld16(lanebase + hfe * 32, v0);
            tmem_ld16(lanebase + hfe * 32 + 16, v1);
            if (hfe == 1) tmem_ld16(lanebase + 64, vz);
            tmem_ld_wait();
            tc_fence_before();
            warp_arrive(&bar.acc_empty[s]);
            float* dst = P.dS + (size_t(du.bkv) * NC + du.c) * kW * kFP + du.slab * kSlabRows + fl;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                dst[size_t(hfe * 32 + x) * kFP] = v0[x];
                dst[size_t(hfe * 32 + 16 + x) * kFP] = v1[x];
            }
            if (hfe == 1) dst[size_t(64) * kFP] = vz[0];
        }
    }
}

// ------------------------------------------------------------------------------------------
// reader: phi producers (thread = query row; one slice = 64 packed rows = 32 TMEM columns)
// ------------------------------------------------------------------------------------------

// off-diagonal slice s = block (R, T): rows (8R + a, 8T + b), a, b = 0..7.  Packed bf16
// arithmetic: phi = bf16(bf16(q_r q_t) c) with c rounded to bf16 -- three roundings of 2^-9,
// the same order as the bf16 operand rounding the tensor core sees anyway, and no fp32 ->
// bf16 conversions (which issue at a quarter of the FMA rate).
__device__ __forceinline__ void phi_offdiag(const unsigned char* qt, const uint32_t* coefh, int s,
                                            int row, uint32_t (&w)[32])
{
    const int rt = c_block_rt[s];
    const uint4 qr = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, rt >> 3));
    const uint4 qc = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, rt & 7));
    const uint32_t rr[4] = {qr.x, qr.y, qr.z, qr.w};
    const uint32_t* cf = coefh + 32 * s;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const uint32_t xa = (a & 1) ? dup_hi(rr[a >> 1]) : dup_lo(rr[a >> 1]);
        const uint4 c = *reinterpret_cast<const uint4*>(cf + 4 * a);
        w[4 * a + 0] = bmul2(bmul2(xa, qc.x), c.x);
        w[4 * a + 1] = bmul2(bmul2(xa, qc.y), c.y);
        w[4 * a + 2] = bmul2(bmul2(xa, qc.z), c.z);
        w[4 * a + 3] = bmul2(bmul2(xa, qc.w), c.w);
    }
}

template <int F0>
constexpr bool phi_chunk_needed(int ch)  // 8-dim chunk of the q row
{
    for (int i = 0; i < 64; ++i) {
        const RT rt = feature_rt(F0 + i);
        if ((rt.r < 64 && rt.r / 8 == ch) || (rt.t < 64 && rt.t / 8 == ch)) return true;
    }
    return false;
}

// diagonal / linear / constant slices: 64 rows with compile-time (r, t); fp32 products,
// one rounding
template <int F0>
__device__ __forceinline__ void phi_static(const unsigned char* qt, const float* coef, int row,
                                           uint32_t (&w)[32])
{
    float q[66];
    static_for<8>([&](auto CH) {
        constexpr int ch = decltype(CH)::value;
        if constexpr (phi_chunk_needed<F0>(ch)) {
            const uint4 v = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, ch));
            q[8 * ch + 0] = bf16lo_to_f32(v.x);
            q[8 * ch + 1] = bf16hi_to_f32(v.x);
            q[8 * ch + 2] = bf16lo_to_f32(v.y);
            q[8 * ch + 3] = bf16hi_to_f32(v.y);
            q[8 * ch + 4] = bf16lo_to_f32(v.z);
            q[8 * ch + 5] = bf16hi_to_f32(v.z);
            q[8 * ch + 6] = bf16lo_to_f32(v.w);
            q[8 * ch + 7] = bf16hi_to_f32(v.w);
        }
    });
    q[64] = 1.f;
    q[65] = 0.f;
    static_for<8>([&](auto X) {
        constexpr int x = decltype(X)::value;
        const float4 c0 = *reinterpret_cast<const float4*>(coef + F0 + 8 * x);
        const float4 c1 = *reinterpret_cast<const float4*>(coef + F0 + 8 * x + 4);
        const float cf[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        static_for<4>([&](auto E) {
            constexpr int e = decltype(E)::value;
            constexpr RT a = feature_rt(F0 + 8 * x + 2 * e);
            constexpr RT b = feature_rt(F0 + 8 * x + 2 * e + 1);
            w[4 * x + e] =
                pack_bf16x2(cf[2 * e] * (q[a.r] * q[a.t]), cf[2 * e + 1] * (q[b.r] * q[b.t]));
        });
    });
}

__device__ __forceinline__ void phi_diag(const unsigned char* qt, const float* coef, int s,
                                         int row, uint32_t (&w)[32])
{
    const int sel = s - kOffDiagSlices;
    static_for<kSlices - kOffDiagSlices>([&](auto I) {
        constexpr int i = decltype(I)::value;
        if (sel == i) phi_static<kOffDiagRows + i * 64>(qt, coef, row, w);
    });
}

// ------------------------------------------------------------------------------------------
// reader item: (bh, chunk c).  Warps 0-15 (row quarter qw = w & 3, set kq = w >> 2):
//   intra-chunk phase: Aq tiles (dims [16 kq, 16 kq + 16)), kappa over keys
//   [32 kq, 32 kq + 32) of score tiles S_0..S_G, P tile;
//   inter-chunk phase: phi of slices s = kq (mod 4) into TMEM stages;
//   epilogue: yhat columns [16 kq, 16 kq + 16).
// Warp 16: TMA, warp 17: MMA (S_0..S_G, then P [V; 1], then the 34 readout slices).
// ------------------------------------------------------------------------------------------
__device__ void reader_item(unsigned char* sm, Ctl& ctl, uint32_t tmem, const Params& P, int bh,
                            int c)
{
    RdBars& bar = ctl.bar.rd;
    volatile int* abort_flag = &ctl.abort_flag;
    const int Hq = P.Hq, Hkv = P.Hkv, T = P.T, NC = P.NC;
    const int b = bh / Hq, h = bh % Hq, kv = h / (Hq / Hkv), bkv = b * Hkv + kv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* coef = reinterpret_cast<float*>(sm + kRdOffCoef);
    uint32_t* coefh = reinterpret_cast<uint32_t*>(sm + kRdOffCoefH);
    float* wch = reinterpret_cast<float*>(sm + kRdOffW);
    float* c0 = reinterpret_cast<float*>(sm + kRdOffC0);
    const bool has_inter = c > 0 || P.cont;

    if (threadIdx.x == 0) {
        mbar_init(&bar.qkv_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar.aq_full[i], 16);
            mbar_init(&bar.s_full[i], 1);
            mbar_init(&bar.s_empty[i], 16);
        }
        mbar_init(&bar.p_full, 16);
        mbar_init(&bar.pv_done, 1);
        for (int i = 0; i < kRdStages; ++i) {
            mbar_init(&bar.a_full[i], 4);
            mbar_init(&bar.a_empty[i], 1);
        }
        for (int i = 0; i < kBStages; ++i) {
            mbar_init(&bar.b_full[i], 1);
            mbar_init(&bar.b_empty[i], 1);
        }
        mbar_init(&bar.u_full, 1);
        mbar_init(&bar.done, 1);
        ctl.abort_flag = 0;
        int Gh = P.G[h];
        if (Gh < 1 || Gh > kGMax) {
            raise_error(OAL_ERR_GROUPS);
            Gh = Gh < 1 ? 1 : kGMax;
        }
        ctl.G = Gh;
        fence_mbar_init();
    }
    __syncthreads();
    const int G = ctl.G;
    if (warp == kTmaWarp && lane == 0) {
        // tiles and the coefficient table first: they do not depend on the setup below
        mbar_expect_tx(&bar.qkv_full, 3 * kTileBytes + kFP * 4);
        tma_load_3d(sm + kRdOffQ, P.tm_q, &bar.qkv_full, 0, c * kC, bh);
        tma_load_3d(sm + kRdOffK, P.tm_k, &bar.qkv_full, 0, c * kC, bkv);
        tma_load_3d(sm + kRdOffV, P.tm_v, &bar.qkv_full, 0, c * kC, bkv);
        bulk_g2s(coef, P.coef_all + size_t(h) * kFP, kFP * 4, &bar.qkv_full);
    }
    for (int e = threadIdx.x; e < kGM1 * 64; e += blockDim.x) {
        const int m = e >> 6, r = e & 63;
        int g = P.gid[h * kD + r];
        if (g < 1 || g > G) {
            raise_error(OAL_ERR_GROUPS);
            g = g < 1 ? 1 : G;
        }
        wch[e] = (m <= G) ? P.L[size_t(h) * kGM1 * kGM1 + g * kGM1 + m] * 0.125f : 0.f;
    }
    if (threadIdx.x < kGM1) c0[threadIdx.x] = P.L[size_t(h) * kGM1 * kGM1 + threadIdx.x];
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == kTmaWarp) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            if (has_inter && ok) {
                // slices 2u, 2u + 1 of image (bkv, c) in one copy of 160 rows
                const int row0 = (bkv * NC + c) * kSlices * 80;
                for (int u = 0; u < kSlices / 2; ++u) {
                    const int bs = u % kBStages;
                    if (u >= kBStages &&
                        !mbar_wait(&bar.b_empty[bs], ((u / kBStages) - 1) & 1, abort_flag))
                        break;
                    // stage 2 is the ones atom until the P [V | 1] MMAs are done
                    if (u == 2 && !mbar_wait(&bar.pv_done, 0, abort_flag)) break;
                    mbar_expect_tx(&bar.b_full[bs], kImgPairBytes);
                    tma_load_2d(sm + rd_bstage_off(bs), P.tm_img, &bar.b_full[bs], 0,
                                row0 + 160 * u);
                    ++issued;
                }
            }
            bounded_spin_done(&bar.qkv_full, 0);
            for (int u = max(0, issued - kBStages); u < issued; ++u)
                bounded_spin_done(&bar.b_full[u % kBStages], (u / kBStages) & 1);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // the whole warp runs the issue loop (waits by every lane); one elected lane issues
        constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_u = idesc_bf16(128, 80, false, false);   // A, B K-major
        constexpr uint32_t id_pv = idesc_bf16(128, 80, false, true);   // B = [V | ones] MN
        const uint32_t aq0 = smem_u32(sm + kRdOffAq), kt = smem_u32(sm + kRdOffK);
        const uint32_t vt = smem_u32(sm + kRdOffV), ones = smem_u32(sm + kRdOffOnes);
        const uint32_t sm0 = smem_u32(sm);
        bool ok = mbar_wait(&bar.qkv_full, 0, abort_flag);
        // grouped score tiles S_m = (Q o w_m) K^T, double-buffered in TMEM
        for (int m = 0; m <= G && ok; ++m) {
            const int sb = m & 1;
            ok = mbar_wait(&bar.aq_full[sb], (m >> 1) & 1, abort_flag);
            if (ok && m >= 2) ok = mbar_wait(&bar.s_empty[sb], ((m >> 1) - 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + kColS0 + sb * 128,
                             sdesc_sw128(aq0 + sb * kTileBytes + ks * 32, 16, 1024),
                             sdesc_sw128(kt + ks * 32, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                mma_commit(&bar.s_full[sb]);
            }
            __syncwarp();
        }
        // intra-chunk term: U = P [V | 1]
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.p_full, 0, abort_flag));
        if (ok) {
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + kColU,
                             sdesc_sw128(aq0 + (ks >> 2) * kTileBytes + (ks & 3) * 32, 16, 1024),
                             sdesc_sw128(vt + ks * 2048, ones - vt, 1024), id_pv,
                             ks > 0 ? 1u : 0u);
                mma_commit(&bar.pv_done);  // K, V, Aq | P are free for phi stages 4..7
            }
            __syncwarp();
        }
        // inter-chunk readout U += phi(Q_c) S_c, two slices (one image stage) per round:
        // A = phi slices 2u, 2u + 1 (stages (2u) % 8, (2u + 1) % 8), B = image pair u
        for (int u = 0; u < kSlices / 2 && ok && has_inter; ++u) {
            const int s0 = 2 * u, bs = u % kBStages;
            ok = mbar_wait(&bar.a_full[s0 % kRdStages], (s0 / kRdStages) & 1, abort_flag) &&
                 mbar_wait(&bar.a_full[(s0 + 1) % kRdStages], ((s0 + 1) / kRdStages) & 1,
                           abort_flag) &&
                 mbar_wait(&bar.b_full[bs], (u / kBStages) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int st = (s0 + x) % kRdStages;
                    const uint32_t bsl = sm0 + rd_bstage_off(bs) + x * kImgSliceBytes;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + kColU,
                                 sdesc_sw128(sm0 + rd_stage_off(st) + ks * 32, 16, 1024),
                                 sdesc_sw128(bsl + ks * 32, 16, 1024), id_u, 1u);
                    mma_commit(&bar.a_empty[st]);
                }
                mma_commit(&bar.b_empty[bs]);
            }
            __syncwarp();
        }
        if (elect_one()) {
            if (ok) mma_commit(&bar.u_full);
            mma_commit(&bar.done);
        }
        __syncwarp();
        if (lane == 0) bounded_spin_done(&bar.done, 0);
        __syncwarp();
    } else {
        const int qw = warp & 3, kq = warp >> 2, row = qw * 32 + lane;
        const unsigned char* qt = sm + kRdOffQ;
        const uint32_t aq0 = smem_u32(sm + kRdOffAq);
        const uint32_t lanebase = tmem + (uint32_t(qw * 32) << 16);
        bool ok = mbar_wait(&bar.qkv_full, 0, abort_flag);


        // ---- intra-chunk phase ----
        // Aq_m = Q o w_m (bf16, K-major); this warp writes dims [16 kq, 16 kq + 16)
        auto produce_aq = [&](int m) {
            const uint32_t base = aq0 + (m & 1) * kTileBytes;
            const float* w = wch + m * 64;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int ch = 2 * kq + x;
                const uint4 qv = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, ch));
                const float4 wa = *reinterpret_cast<const float4*>(w + 8 * ch);
                const float4 wb = *reinterpret_cast<const float4*>(w + 8 * ch + 4);
                sts128(base + kmajor_chunk(row, ch),
                       pack2(__fmul2_rn(f2(bf16lo_to_f32(qv.x), bf16hi_to_f32(qv.x)), f2(wa.x, wa.y))),
                       pack2(__fmul2_rn(f2(bf16lo_to_f32(qv.y), bf16hi_to_f32(qv.y)), f2(wa.z, wa.w))),
                       pack2(__fmul2_rn(f2(bf16lo_to_f32(qv.z), bf16hi_to_f32(qv.z)), f2(wb.x, wb.y))),
                       pack2(__fmul2_rn(f2(bf16lo_to_f32(qv.w), bf16hi_to_f32(qv.w)), f2(wb.z, wb.w))));
            }
            fence_proxy_async();
            warp_arrive(&bar.aq_full[m & 1]);
        };
        // phi slice s of this row -> shared stage s % 8 (kq or kq + 4; K-major, 128B-swizzled
        // rows)
        const uint32_t sm0 = smem_u32(sm);
        auto produce_phi = [&](int s) -> bool {
            const int st = s % kRdStages;
            uint32_t w[32];
            if (s < kOffDiagSlices) phi_offdiag(qt, coefh, s, row, w);
            else phi_diag(qt, coef, s, row, w);
            if (s >= kRdStages &&
                !mbar_wait(&bar.a_empty[st], ((s / kRdStages) - 1) & 1, abort_flag))
                return false;
            // first use of a reused stage: the intra-chunk MMAs must be done with it
            if (s >= kPhiSets && s < kRdStages && !mbar_wait(&bar.pv_done, 0, abort_flag))
                return false;
            const uint32_t base = sm0 + rd_stage_off(st);
#pragma unroll
            for (int x = 0; x < 8; ++x)
                sts128(base + kmajor_chunk(row, x), w[4 * x], w[4 * x + 1], w[4 * x + 2],
                       w[4 * x + 3]);
            fence_proxy_async();
            warp_arrive(&bar.a_full[st]);
            return true;
        };
        if (ok) {
            // bf16 copy of the off-diagonal coefficients (read by phi)
            for (int i = threadIdx.x; i < kOffDiagRows / 2; i += 16 * 32)
                coefh[i] = pack_bf16x2(coef[2 * i], coef[2 * i + 1]);
        }
        named_bar_sync(1, 16 * 32);
        if (ok) {
            // the first phi slice of this set is staged before the intra-chunk phase, so the
            // readout MMAs can start as soon as the intra-chunk ones are issued
            if (has_inter) ok = produce_phi(kq);
            produce_aq(0);
            if (G >= 1) produce_aq(1);
        }
        const bool live = kq <= qw;  // keys [32 kq, 32 kq + 32) vs rows [32 qw, 32 qw + 32)
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
        for (int m = 0; m <= G && ok; ++m) {
            const int sb = m & 1;
            if (!mbar_wait(&bar.s_full[sb], (m >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (live) {
                const float cm = c0[m];
                const uint32_t taddr = lanebase + kColS0 + sb * 128 + 32 * kq;
                float v[32];
                tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float2 t = __fadd2_rn(f2(cm, cm), f2(v[i], v[i + 1]));
                    const float2 a = __ffma2_rn(t, t, f2(acc[i], acc[i + 1]));
                    acc[i] = a.x;
                    acc[i + 1] = a.y;
                }
            }
            tc_fence_before();
            warp_arrive(&bar.s_empty[sb]);
            if (m + 2 <= G) produce_aq(m + 2);
        }
        if (ok) {
            // P tile (K-major, 2 K-atoms over the 128 keys; aliases Aq0 | Aq1): keys
            // [32 kq, 32 kq + 32) are chunks 4 (kq & 1) .. + 3 of atom kq >> 1
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                uint32_t wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j0 = 32 * kq + 8 * x + 2 * e;
                    const float k0 = (j0 <= row) ? P.eps + acc[8 * x + 2 * e] : 0.f;
                    const float k1 = (j0 + 1 <= row) ? P.eps + acc[8 * x + 2 * e + 1] : 0.f;
                    wv[e] = pack_bf16x2(k0, k1);
                }
                sts128(aq0 + (kq >> 1) * kTileBytes + kmajor_chunk(row, 4 * (kq & 1) + x),
                       wv[0], wv[1], wv[2], wv[3]);
            }
            fence_proxy_async();
            warp_arrive(&bar.p_full);
        }
        // ---- inter-chunk phase: phi(Q_c) slices kq + 4, kq + 8, ... ----
        for (int s = kq + kPhiSets; s < kSlices && ok && has_inter; s += kPhiSets)
            ok = produce_phi(s);

        // ---- epilogue: yhat = u[:64] / u[64], columns [16 kq, 16 kq + 16) of this row ----
        if (ok) ok = mbar_wait(&bar.u_full, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            float u[16], dz[16];
            tmem_ld16(lanebase + kColU + 16 * kq, u);
            tmem_ld16(lanebase + kColU + 64, dz);
            tmem_ld_wait();
            const int irow = c * kC + row;
            if (irow < T) {
                const float inv = 1.f / dz[0];
                float4* o = reinterpret_cast<float4*>(P.out + (size_t(bh) * T + irow) * kDV +
                                                      16 * kq);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[i] = make_float4(u[4 * i] * inv, u[4 * i + 1] * inv, u[4 * i + 2] * inv,
                                       u[4 * i + 3] * inv);
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// kernels: 0 = chunk deltas (persistent: CTA i takes a contiguous range of units),
// 1 = readers (one CTA per (b*h, chunk), B*Hq*NC in all).  Both may be launched as programmatic dependents of the
// preceding kernel in the stream: griddepcontrol.wait orders every read of its outputs.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_img, Params P)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl& ctl = *reinterpret_cast<Ctl*>(sm + kOffCtl);
    const int warp = threadIdx.x >> 5;
    P.tm_q = &tm_q;
    P.tm_k = &tm_k;
    P.tm_v = &tm_v;
    P.tm_img = &tm_img;

    if (warp == kMmaWarp) {
        tmem_alloc(&ctl.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    init_ones_atom(sm + (kMode == 0 ? kOffOnes : kRdOffOnes));
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    grid_dep_launch();  // the next kernel may start its prologue
    grid_dep_wait();    // outputs of the previous kernel are visible from here on

    if (kMode == 0) {
        const int units = P.B * P.Hkv * P.NC * kNumSlabs;
        const int u0 = int((long long)units * blockIdx.x / gridDim.x);
        const int u1 = int((long long)units * (blockIdx.x + 1) / gridDim.x);
        if (u1 > u0) delta_item(sm, ctl, tmem, P, u0, u1);
    } else {
        // items with an inter-chunk part first, chunk-major with the heads of a chunk adjacent
        // (they share the chunk's image in L2); the chunk-0 items last, so that the final
        // partial wave holds short items (chunk 0 has no inter-chunk part unless the call
        // continues a prefix)
        const int nbh = P.B * P.Hq, heavy = nbh * (P.NC - 1), idx = blockIdx.x;
        if (idx < heavy) reader_item(sm, ctl, tmem, P, idx % nbh, 1 + idx / nbh);
        else reader_item(sm, ctl, tmem, P, idx - heavy, 0);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Exclusive prefix over chunks of one (bkv, 64-row slice, 8 columns): image_c =
// bf16(sum_{c' < c} dS_c') for c >= 1, stored row-major as [80 n][64 f] per slice (the
// readout's tensor copy swizzles it into the K-major B-operand layout; rows 65.. are never
// read), final state = sum over all chunks.  Thread = (n, row pair).
// The last z-plane of the grid instead builds the coefficient tables and the state header
// (one block per query head), which the readout reads after this kernel.
constexpr int kScanCols = 8;
constexpr int kImgRows = 80;
__global__ void __launch_bounds__(256) scan_kernel(const float* __restrict__ dS,
                                                   unsigned char* __restrict__ img,
                                                   float* __restrict__ body, int NC,
                                                   const int32_t* __restrict__ gid,
                                                   const float* __restrict__ L,
                                                   const int32_t* __restrict__ G, float eps,
                                                   unsigned char* __restrict__ state, int B,
                                                   int Hq, int Hkv, long long tokens, int cont)
{
    grid_dep_launch();
    if (blockIdx.z == gridDim.z - 1) {  // independent of the deltas: no wait
        const int h = blockIdx.y * gridDim.x + blockIdx.x;
        if (h < Hq) prep_head(h, gid, L, G, eps, state, B, Hq, Hkv, tokens, cont != 0);
        return;
    }
    grid_dep_wait();
    const int sl = blockIdx.x, bkv = blockIdx.z;
    const int nl = threadIdx.x >> 5, p = threadIdx.x & 31;
    const int n = blockIdx.y * kScanCols + nl;
    __shared__ float fin[kScanCols][64 + 1];
    float* unit = body + size_t(bkv) * kFP * kW;
    // the prefix before this call: zero, or (continuation) the state's current contents
    float a0 = 0.f, a1 = 0.f;
    const int f = sl * 64 + 2 * p, c_first = cont ? 0 : 1;
    if (cont && n < kDV) {
        a0 = unit[size_t(f) * kDV + n];
        a1 = unit[size_t(f + 1) * kDV + n];
    } else if (cont && n == kDV) {
        a0 = unit[size_t(kFP) * kDV + f];
        a1 = unit[size_t(kFP) * kDV + f + 1];
    }
    if (n >= kW && n < kImgRows) {
        // rows 65..79 of every image: zero (the readout's N = 80 MMA reads them)
        unsigned char* dst = img + (size_t(bkv) * NC * kSlices + sl) * kImgSliceBytes + n * 128 + 4 * p;
        for (int c = c_first; c < NC; ++c)
            *reinterpret_cast<uint32_t*>(dst + size_t(c) * kSlices * kImgSliceBytes) = 0u;
    }
    if (n < kW) {
        const float* src = dS + (size_t(bkv) * NC * kW + n) * kFP + sl * 64 + 2 * p;
        unsigned char* dst = img + (size_t(bkv) * NC * kSlices + sl) * kImgSliceBytes +
                             n * 128 + 4 * p;
        const size_t sstride = size_t(kW) * kFP, dstride = size_t(kSlices) * kImgSliceBytes;
        int c = 0;
        for (; c + 4 <= NC; c += 4) {
            float2 d[4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
                d[x] = __ldcs(reinterpret_cast<const float2*>(src + (c + x) * sstride));
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                if (c + x >= c_first)
                    *reinterpret_cast<uint32_t*>(dst + (c + x) * dstride) = pack_bf16x2(a0, a1);
                a0 += d[x].x;
                a1 += d[x].y;
            }
        }
        for (; c < NC; ++c) {
            const float2 d = __ldcs(reinterpret_cast<const float2*>(src + c * sstride));
            if (c >= c_first)
                *reinterpret_cast<uint32_t*>(dst + c * dstride) = pack_bf16x2(a0, a1);
            a0 += d.x;
            a1 += d.y;
        }
    }
    fin[nl][2 * p] = a0;
    fin[nl][2 * p + 1] = a1;
    __syncthreads();  // every read of the old state in this block precedes the writes below
    // final state of unit bkv: Hv[f][n] (n < 64), z[f] (n == 64)
    const int fl = threadIdx.x >> 2, cq = threadIdx.x & 3;
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const int nn = blockIdx.y * kScanCols + 2 * cq + x;
        if (nn < kDV) unit[size_t(sl * 64 + fl) * kDV + nn] = fin[2 * cq + x][fl];
        else if (nn == kDV) unit[size_t(kFP) * kDV + sl * 64 + fl] = fin[2 * cq + x][fl];
    }
}

}  // namespace tc

// ------------------------------------------------------------------------------------------
// host side: tensor maps and launch
// ------------------------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [heads][T][64] bf16 viewed as 3D {64, T, heads}; box {64, 128, 1}; 128B swizzle; rows past
// T read as zero.
bool make_map(CUtensorMap* m, const void* base, int T, int heads)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, cuuint64_t(T), cuuint64_t(heads)};
    const cuuint64_t strides[2] = {64 * 2, cuuint64_t(T) * 64 * 2};
    const cuuint32_t box[3] = {64, tc::kC, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// chunk-state images [slices][80 rows][64] bf16 viewed as 2D {64, slices * 80}; box {64, 160}
// = two consecutive slices per copy (copies from L2 cost about the same per copy from 8 to
// 20 KB, so fewer and larger ones); 128B swizzle on the way in.
bool make_img_map(CUtensorMap* m, const void* base, size_t slices)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {64, cuuint64_t(slices) * 80};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {64, 160};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace

size_t tc_image_bytes(int B, int Hkv, int T)
{
    const size_t NC = size_t((T + tc::kC - 1) / tc::kC);
    return size_t(B) * Hkv * NC * tc::kImgChunkBytes;
}

size_t tc_workspace_bytes(int B, int Hkv, int T)
{
    const size_t NC = size_t((T + tc::kC - 1) / tc::kC);
    return tc_image_bytes(B, Hkv, T) + size_t(B) * Hkv * NC * kW * kFP * 4;
}

namespace {

// Launch with the programmatic-dependent attribute: the kernel may be scheduled while its
// predecessor in the stream is still running, and waits for it in griddepcontrol.wait.
template <typename... Args>
cudaError_t launch_ex(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      bool dependent, Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

int launch_prefill_tc(const void* q, const void* k, const void* v, const int32_t* gid,
                      const float* L, const int32_t* G, float eps, float* out, void* state,
                      void* ws, int B, int T, int Hq, int Hkv, bool overlap, bool cont,
                      cudaStream_t st)
{
    if (B == 0) return OAL_OK;
    const int NC = (T + tc::kC - 1) / tc::kC;
    unsigned char* sb = static_cast<unsigned char*>(state);
    float* body = reinterpret_cast<float*>(sb + kHeaderBytes + coef_bytes(Hq));
    if (T == 0) {
        if (!cont) OAL_CUDA_TRY(cudaMemsetAsync(body, 0, size_t(B) * Hkv * state_unit_bytes(), st));
        return OAL_OK;
    }
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    CUtensorMap mq, mk, mv, mi;
    // without out (state only) q is not read: its map then describes k and is never used
    if (!(out ? make_map(&mq, q, T, B * Hq) : make_map(&mq, k, T, B * Hkv)) ||
        !make_map(&mk, k, T, B * Hkv) ||
        !make_map(&mv, v, T, B * Hkv) ||
        !make_img_map(&mi, wsb, size_t(B) * Hkv * NC * tc::kSlices))
        return OAL_ERR_CUDA;
    tc::Params P{};
    P.gid = gid;
    P.L = L;
    P.G = G;
    P.eps = eps;
    P.coef_all = reinterpret_cast<const float*>(sb + kHeaderBytes);
    P.img = wsb;
    P.dS = reinterpret_cast<float*>(wsb + tc_image_bytes(B, Hkv, T));
    P.out = out;
    P.B = B;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.T = T;
    P.NC = NC;
    P.cont = cont ? 1 : 0;
    const int units = B * Hkv * NC * tc::kNumSlabs;
    const int grid0 = std::max(1, std::min(sm_count(), units));
    OAL_CUDA_TRY(cudaFuncSetAttribute(tc::prefill_tc_kernel<0>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(tc::kSmemBytes)));
    OAL_CUDA_TRY(cudaFuncSetAttribute(tc::prefill_tc_kernel<1>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(tc::kSmemBytes)));
    {
        LaunchScope ls("delta_tc", st);
        OAL_CUDA_TRY(launch_ex(tc::prefill_tc_kernel<0>, dim3(grid0), dim3(tc::kThreads),
                               tc::kSmemBytes, st, false, mq, mk, mv, mi, P));
    }
    {
        LaunchScope ls("scan", st);
        OAL_CUDA_TRY(launch_ex(tc::scan_kernel,
                               dim3(tc::kSlices, tc::kImgRows / tc::kScanCols, B * Hkv + 1),
                               dim3(256), 0, st, overlap, (const float*)P.dS, P.img, body, NC,
                               gid, L, G, eps, sb, B, Hq, Hkv, (long long)T, P.cont));
    }
    if (out == nullptr) return OAL_OK;  // no out: the state alone is wanted
    {
        LaunchScope ls("readout_tc", st);
        OAL_CUDA_TRY(launch_ex(tc::prefill_tc_kernel<1>, dim3(NC * B * Hq), dim3(tc::kThreads),
                               tc::kSmemBytes, st, overlap, mq, mk, mv, mi, P));
    }
    return OAL_OK;
}

}  // namespace oal
