// oal_tc.cu -- tcgen05 / TMA kernels of the bf16 chunked prefill on B200 (sm_100a).
//
// Equations: "OAL: 按 QK 离群贡献分组的正二次注意力核" (reproduction note of arXiv 2610.13674),
// section 核心公式, numbered in order of appearance: (2) grouped score, (3) kernel kappa,
// (4) prefix states, (5) readout.  With the packed feature map of oal_common.cuh, the state
// of a (b, kv) head after token i is S_i = sum_{j<=i} psi(k_j) [v_j; 1] (2176 x 65) and
// u_i = phi(q_i)^T S_i.  Chunked with C = 128 tokens, the prefill runs as four kernels:
//
//   chunk deltas (b, kv, chunk c, slab of 128 packed rows; every unit independent):
//     producer warps build psi(K_c)^T (MN-major, bf16) in shared memory, split exactly into
//     hi = bf16(psi) and lo = psi - hi; N=80 MMAs, issued by two warps (even and odd units),
//     accumulate dS_c = psi(K_c)^T [V_c; 1] in TMEM (the [.; 1] column comes from a constant
//     "ones" atom addressed through the B descriptor's leading byte offset) and epilogue
//     warps store it in fp32.
//   intra-chunk part (oal_tc_intra.cuh; b, h, chunk c), launched after the scan as its
//     programmatic dependent (it needs only q, k, v, so its CTAs fill SMs as the scan's
//     blocks retire): the factored form of eq. (3),
//       kappa = eps + sum_m (L_0m + (q o w_m) . k)^2,   w_m[r] = L_{g(r),m} / sqrt(d)
//     (= ||L^T sbar||^2): score tiles S_m = (Q o w_m) K^T in TMEM, kappa accumulated in
//     registers, masked causally and multiplied into [V_c; 1].
//   prefix scan (SIMT, memory bound): S_c = sum_{c' < c} dS_c' for every chunk, written as
//     bf16 images of the B operand, and the final state S_NC in fp32 (eq. 4 in chunk form).
//     (Launch order: deltas, scan, intra-chunk part, readout, each a programmatic dependent of
//     the one before on the caller's stream.)
//   inter-chunk readout (oal_tc_readout.cuh; persistent over items b, h, chunk c): phi(Q_c)
//     is written into tensor memory slice pair by slice pair and multiplied with the image of
//     S_c by N=80 MMAs reading A from TMEM; the epilogue adds the intra-chunk sum and writes
//     yhat = u[:64] / u[64] (eq. 5).
//
// Every wait is bounded (1 s); one that runs out sets OAL_ERR_TIMEOUT and the CTA leaves its
// loops in order (copies drained, MMAs committed, TMEM freed) instead of hanging.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

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

constexpr int kWarps = 19;
constexpr int kThreads = kWarps * 32;
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;   // MMA issuer of the even units (and tensor-memory owner)
constexpr int kMmaWarpB = 18;  // MMA issuer of the odd units
constexpr uint32_t kTmemCols = 512;

static_assert(kFP % kSlabRows == 0 && kFP % 64 == 0, "feature padding");

// ---- shared memory (offsets from a 1024-aligned base) ---------------------------------------
// chunk-delta builder
constexpr uint32_t kStOffKV = 0;          // 3 x (K 16 KB + V 16 KB)
constexpr uint32_t kStOffA = 98304;       // 3 x (hi 16 KB + lo 16 KB) psi stages
constexpr uint32_t kOffOnes = 196608;     // 16 KB ones atom
// both
constexpr uint32_t kOffCtl = 224256;      // barriers and control words
constexpr uint32_t kSmemBytes = kOffCtl + 1024 + 1024;

constexpr uint32_t kImgPairBytes = 2 * kImgSliceBytes;     // one tensor copy: 160 rows
constexpr int kKVStages = 3;
constexpr int kDAStages = 3;  // psi stages (hi + lo tiles of one half chunk)
constexpr int kDAcc = 4;      // TMEM accumulators of the delta builder (128 columns each)
constexpr uint32_t kStATile = 64 * kSlabRows * 2;          // 64 tokens x 128 rows = 16 KB
static_assert(kStOffKV + kKVStages * 2 * kTileBytes <= kStOffA &&
                  kStOffA + kDAStages * 2 * kStATile <= kOffOnes &&
                  kOffOnes + kOnesAtomBytes <= kOffCtl && kDAcc * 128 <= int(kTmemCols),
              "delta builder shared-memory and TMEM map");
struct StBars {
    uint64_t kv_full[kKVStages], kv_empty[kKVStages], a_full[kDAStages], a_empty[kDAStages];
    uint64_t acc_full[kDAcc], acc_empty[kDAcc], done, done_b;
};
struct Ctl {
    union {
        StBars st;
        uint64_t raw[64];
    } bar;
    uint32_t tmem_base;
    int abort_flag;
    int G;
};
static_assert(sizeof(Ctl) <= 1024, "control block");
static_assert(sizeof(StBars) <= sizeof(uint64_t) * 64, "barrier block");

// One sequence of a packed variable-length batch (all counts are sums over the sequences
// before it, so that a flat unit or item index finds its sequence by binary search).
struct SeqDesc {
    int T, NC;    // tokens and chunks of the sequence
    int tok;      // tokens before it: its q block starts at row tok * Hq of [rows][64]
    int chunk0;   // its first chunk-state index (images, deltas): sum of Hkv * NC
    int unit0;    // its first chunk-delta unit: sum of Hkv * NC * 17
    int intra0;   // its first intra-chunk item: sum of Hq * NC
    int read0;    // its first readout item: sum of Hq * max(NC - 1, 0)
    int pad;
};
static_assert(sizeof(SeqDesc) == 32, "descriptor layout");
constexpr int kSdUnit0 = 4, kSdIntra0 = 5, kSdRead0 = 6;  // int offsets in SeqDesc

struct Params {
    const CUtensorMap* tm_q;
    const CUtensorMap* tm_k;
    const CUtensorMap* tm_v;
    const CUtensorMap* tm_img;  // chunk-state images as {64 f, slices * 80 rows}, box {64, 65}
    const int32_t* gid;
    const float* L;
    const int32_t* G;
    float eps;
    const unsigned char* rtab;  // per-head readout tables [Hq][kTabBytes] (workspace)
    unsigned char* img;      // chunk-state images [B*Hkv][NC][34 slices][80 n][64 f] bf16
    float* dS;               // chunk deltas [B*Hkv][NC][65][kFP] fp32
    float* out;
    int B, Hq, Hkv, T, NC;
    int cont;                // 1: the state already holds a prefix; these tokens continue it
    int skip_copies;         // test hook: the readout issues no copies, so its waits run out
    int n_units, n_intra, n_read;  // chunk-delta units, intra-chunk items, readout items
    // packed variable-length batch (nseq > 0): B, T and NC above are unused; sequence i has
    // descriptor seqs[i] and tensor maps maps[3 i + {0, 1, 2}] (q, k, v) in global memory
    int nseq;
    const SeqDesc* seqs;
    const CUtensorMap* maps;
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

// diagonal / linear / constant slabs: 32 rows with compile-time (r, t), split exactly into hi
// and lo like the off-diagonal ones: each pair of rows gathers its two k_r and its two k_t
// into one bf16x2 register each with one byte permute (k_64 = `one`, k_65 = 0 from a constant
// word), then hi = bf16(k_r k_t) and lo = the exact remainder.
template <int F0>
__device__ __forceinline__ void psi_static(const unsigned char* ktile, int trow, float one,
                                           uint32_t abase, int j)
{
    uint32_t kw[32];  // packed bf16 pairs of the k chunks these rows read
    static_for<8>([&](auto CH) {
        constexpr int ch = decltype(CH)::value;
        if constexpr (psi_chunk_needed<F0>(ch)) {
            const uint4 w = *reinterpret_cast<const uint4*>(ktile + kmajor_chunk(trow, ch));
            kw[ch * 4 + 0] = w.x;
            kw[ch * 4 + 1] = w.y;
            kw[ch * 4 + 2] = w.z;
            kw[ch * 4 + 3] = w.w;
        }
    });
    const uint32_t onez = pack_bf16x2(one, 0.f);  // bf16 halves (k_64, k_65) = (one, 0)
    auto word = [&](auto R) -> uint32_t {
        constexpr int r = decltype(R)::value;
        if constexpr (r >= 64) return onez;
        else return kw[r >> 1];
    };
    auto half = [](int r) constexpr -> int { return r >= 64 ? r - 64 : (r & 1); };
    constexpr int m0 = F0 % kSlabRows;
    static_for<4>([&](auto CH) {
        constexpr int ch = decltype(CH)::value;
        uint32_t h[4], l[4];
        static_for<4>([&](auto E) {
            constexpr int e = decltype(E)::value;
            constexpr RT a = feature_rt(F0 + ch * 8 + 2 * e);
            constexpr RT b = feature_rt(F0 + ch * 8 + 2 * e + 1);
            // low half from the first word, high half from the second (bytes 4..7)
            constexpr uint32_t sr = (half(a.r) ? 0x32u : 0x10u) | ((half(b.r) ? 0x76u : 0x54u) << 8);
            constexpr uint32_t st = (half(a.t) ? 0x32u : 0x10u) | ((half(b.t) ? 0x76u : 0x54u) << 8);
            const uint32_t xr = __byte_perm(word(std::integral_constant<int, a.r>{}),
                                            word(std::integral_constant<int, b.r>{}), sr);
            const uint32_t xt = __byte_perm(word(std::integral_constant<int, a.t>{}),
                                            word(std::integral_constant<int, b.t>{}), st);
            h[e] = bmul2(xr, xt);
            l[e] = bfma2(xr, xt, h[e] ^ 0x80008000u);
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

// The sequence of a packed batch whose run of indices (field f of the descriptors: first
// unit or item) contains idx; sequences with an empty run are skipped.
__device__ __forceinline__ int seq_of(const SeqDesc* sd, int n, int idx, int f)
{
    const int* p = reinterpret_cast<const int*>(sd) + f;
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p + 8 * mid) <= idx) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Order this thread's later tensor copies after the host's write of a tensor map that lives
// in global memory (the maps of a packed batch).
__device__ __forceinline__ void tmap_acquire(const CUtensorMap* m)
{
    asm volatile("fence.proxy.tensormap::generic.acquire.sys [%0], 128;" ::"l"(m) : "memory");
}

// unit u -> (kv head, chunk c, slab); slabs of one chunk are consecutive.  mk / mv and kvz:
// the tensor maps and z coordinate of the unit's K and V tiles; T: the sequence's tokens;
// chunk: its chunk-state index (deltas, images).
struct DeltaUnit {
    int c, slab, T, kvz;
    size_t chunk;
    const CUtensorMap *mk, *mv;
};
__device__ __forceinline__ DeltaUnit delta_unit(int u, const Params& P)
{
    if (P.nseq == 0) {
        const int rest = u / kNumSlabs, bkv = rest / P.NC, c = rest % P.NC;
        return DeltaUnit{c, u % kNumSlabs, P.T, bkv, size_t(bkv) * P.NC + c, P.tm_k, P.tm_v};
    }
    const int i = seq_of(P.seqs, P.nseq, u, kSdUnit0);
    const SeqDesc sd = P.seqs[i];
    const int lu = u - sd.unit0, rest = lu / kNumSlabs, kv = rest / sd.NC, c = rest % sd.NC;
    return DeltaUnit{c, lu % kNumSlabs, sd.T, kv, size_t(sd.chunk0) + size_t(kv) * sd.NC + c,
                     P.maps + 3 * i + 1, P.maps + 3 * i + 2};
}

// An item (query head h of one sequence, chunk c) of the intra-chunk kernels (intra = true)
// or of the inter-chunk readout.  mq / mk / mv and qz / kvz: tensor maps and z coordinates of
// its Q, K, V tiles; orow: row of the sequence's token 0 of head h in out [rows][64] and in
// the normalisers; chunk: chunk-state index of (sequence, kv head, c).
struct ItemRef {
    const CUtensorMap *mq, *mk, *mv;
    int qz, kvz, c, T, h;
    size_t orow, chunk;
};
__device__ __forceinline__ ItemRef item_ref(int idx, const Params& P, bool intra)
{
    ItemRef r;
    if (P.nseq == 0) {
        const int nbh = P.B * P.Hq;
        int bh, c;
        if (P.cont || !intra) {
            bh = idx % nbh;
            c = idx / nbh + (P.cont || intra ? 0 : 1);
        } else if (idx < nbh * (P.NC - 1)) {  // chunks with an inter-chunk part first
            bh = idx % nbh;
            c = 1 + idx / nbh;
        } else {
            bh = idx - nbh * (P.NC - 1);
            c = 0;
        }
        const int b = bh / P.Hq, h = bh % P.Hq, bkv = b * P.Hkv + h / (P.Hq / P.Hkv);
        r.mq = P.tm_q;
        r.mk = P.tm_k;
        r.mv = P.tm_v;
        r.qz = bh;
        r.kvz = bkv;
        r.c = c;
        r.T = P.T;
        r.h = h;
        r.orow = size_t(bh) * P.T;
        r.chunk = size_t(bkv) * P.NC + c;
        return r;
    }
    const int i = seq_of(P.seqs, P.nseq, idx, intra ? kSdIntra0 : kSdRead0);
    const SeqDesc sd = P.seqs[i];
    const int l = idx - (intra ? sd.intra0 : sd.read0);
    const int h = l % P.Hq, c = l / P.Hq + (intra ? 0 : 1), kv = h / (P.Hq / P.Hkv);
    r.mq = P.maps + 3 * i;
    r.mk = P.maps + 3 * i + 1;
    r.mv = P.maps + 3 * i + 2;
    r.qz = h;
    r.kvz = kv;
    r.c = c;
    r.T = sd.T;
    r.h = h;
    r.orow = size_t(sd.tok) * P.Hq + size_t(h) * sd.T;
    r.chunk = size_t(sd.chunk0) + size_t(kv) * sd.NC + c;
    return r;
}

// ------------------------------------------------------------------------------------------
// chunk-delta item: units [u0, u1), each dS_c = psi(K_c)^T [V_c; 1] for the 128 packed rows
// of one slab, stored in fp32 as dS[bkv][c][n][f] (n = column of [v; 1]).
// Warps 0-7 psi producers, 8-15 epilogue, 16 TMA, 17 and 18 MMA (even and odd units).
// ------------------------------------------------------------------------------------------
__device__ void delta_item(unsigned char* sm, Ctl& ctl, uint32_t tmem, const Params& P, int u0,
                           int u1)
{
    StBars& bar = ctl.bar.st;
    volatile int* abort_flag = &ctl.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nu = u1 - u0;

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
        mbar_init(&bar.done_b, 1);
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
                const DeltaUnit du = delta_unit(u0 + i, P);
                const int s = i % kKVStages;
                if (i >= kKVStages &&
                    !mbar_wait(&bar.kv_empty[s], ((i / kKVStages) - 1) & 1, abort_flag))
                    break;
                unsigned char* kvs = sm + kStOffKV + s * 2 * kTileBytes;
                if (P.nseq) {
                    tmap_acquire(du.mk);
                    tmap_acquire(du.mv);
                }
                mbar_expect_tx(&bar.kv_full[s], 2 * kTileBytes);
                tma_load_3d(kvs, du.mk, &bar.kv_full[s], 0, du.c * kC, du.kvz);
                tma_load_3d(kvs + kTileBytes, du.mv, &bar.kv_full[s], 0, du.c * kC, du.kvz);
                ++issued;
            }
            for (int i = max(0, issued - kKVStages); i < issued; ++i)
                bounded_spin_done(&bar.kv_full[i % kKVStages], (i / kKVStages) & 1);
        }
        __syncwarp();
    } else if (warp == kMmaWarp || warp == kMmaWarpB) {
        // two issuers, even and odd units (each unit has its own accumulator): a barrier wait
        // or commit stalls the issuing thread while the tensor pipe drains its short queue,
        // and the other issuer's MMAs fill that gap.  The whole warp runs the issue loop; one
        // elected lane issues.
        constexpr uint32_t id = idesc_bf16(128, 80, true, true);
        const uint32_t a0 = smem_u32(sm + kStOffA), kv0 = smem_u32(sm + kStOffKV);
        const uint32_t ones = smem_u32(sm + kOffOnes);
        uint64_t* done = warp == kMmaWarp ? &bar.done : &bar.done_b;
        bool ok = true;
        for (int i = warp == kMmaWarp ? 0 : 1; i < nu && ok; i += 2) {
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
        if (elect_one()) mma_commit(done);
        __syncwarp();
        if (lane == 0) bounded_spin_done(done, 0);
        __syncwarp();
    } else if (warp < 8) {
        const int t = threadIdx.x, j = t & 63, qf = t >> 6;
        const uint32_t a0 = smem_u32(sm + kStOffA);
        for (int i = 0; i < nu; ++i) {
            const DeltaUnit du = delta_unit(u0 + i, P);
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
                const float one = (du.c * kC + trow < du.T) ? 1.f : 0.f;
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
            const DeltaUnit du = delta_unit(u0 + i, P);
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
            float* dst = P.dS + du.chunk * kW * kFP + du.slab * kSlabRows + fl;
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
// The same slice when the 8 dims of block R share one group: the weight of (a, b) is then
// c_b for every a, so phi = bf16(q_a bf16(c_b q_b)) -- one packed product per pair of rows
// after the 4 that form c o q over block T (two roundings, as above).
__device__ __forceinline__ void phi_offdiag_pure(const unsigned char* qt, const uint32_t* coefh,
                                                 int s, int row, uint32_t (&w)[32])
{
    const int rt = c_block_rt[s];
    const uint4 qr = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, rt >> 3));
    const uint4 qc = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, rt & 7));
    const uint4 c = *reinterpret_cast<const uint4*>(coefh + 32 * s);  // row a = 0 of the slice
    const uint32_t y[4] = {bmul2(c.x, qc.x), bmul2(c.y, qc.y), bmul2(c.z, qc.z), bmul2(c.w, qc.w)};
    const uint32_t rr[4] = {qr.x, qr.y, qr.z, qr.w};
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const uint32_t xa = (a & 1) ? dup_hi(rr[a >> 1]) : dup_lo(rr[a >> 1]);
        w[4 * a + 0] = bmul2(xa, y[0]);
        w[4 * a + 1] = bmul2(xa, y[1]);
        w[4 * a + 2] = bmul2(xa, y[2]);
        w[4 * a + 3] = bmul2(xa, y[3]);
    }
}

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

// ------------------------------------------------------------------------------------------
// Kernels.  Chunk deltas: persistent, CTA i takes a contiguous range of units.  The scan and
// the readout may be launched as programmatic dependents of the preceding kernel in the
// stream: griddepcontrol.wait orders every read of its outputs.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    delta_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 Params P)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl& ctl = *reinterpret_cast<Ctl*>(sm + kOffCtl);
    const int warp = threadIdx.x >> 5;
    P.tm_k = &tm_k;
    P.tm_v = &tm_v;

    if (warp == kMmaWarp) {
        tmem_alloc(&ctl.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    init_ones_atom(sm + kOffOnes);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    grid_dep_launch();  // the next kernel may start its prologue
    grid_dep_wait();    // outputs of the previous kernel are visible from here on

    const int units = P.n_units;
    const int u0 = int((long long)units * blockIdx.x / gridDim.x);
    const int u1 = int((long long)units * (blockIdx.x + 1) / gridDim.x);
    if (u1 > u0) delta_item(sm, ctl, tmem, P, u0, u1);

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// A barrier wait by a whole warp (every lane waits; true only if the phase completed for all).
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

// The same for warps whose waits are long or off the critical path: suspended while waiting.
__device__ __forceinline__ bool wait_all_sleep(uint64_t* bar, uint32_t parity,
                                               volatile int* abort_flag)
{
    return __all_sync(0xffffffffu, mbar_wait_sleep(bar, parity, abort_flag));
}

#include "oal_tc_intra.cuh"
#include "oal_tc_readout.cuh"
#include "oal_tc_intra_fm.cuh"

// Exclusive prefix over chunks of one (bkv, 64-row slice, 16 columns): image_c =
// bf16(sum_{c' < c} dS_c') for c >= 1, stored row-major as [80 n][64 f] per slice (the
// readout's tensor copy swizzles rows 0..64 into the K-major B-operand layout; rows 65..79
// are never written or read -- the readout keeps them zero in shared memory), final state =
// sum over all chunks.  Thread = (column n, 4 consecutive rows): 16-byte loads, 8 chunks in
// flight, 8-byte image stores.
// With `prep`, the last z-plane of the grid instead builds the coefficient tables and the
// state header (one block per query head), which the readout reads after this kernel; without
// it (free coefficients) the caller has written them before the prefill.
constexpr int kScanCols = 16;
constexpr int kImgRows = 80;
constexpr int kScanColGroups = (kW + kScanCols - 1) / kScanCols;  // 5
__global__ void __launch_bounds__(256) scan_kernel(const float* __restrict__ dS,
                                                   unsigned char* __restrict__ img,
                                                   float* __restrict__ body, int NC,
                                                   const int32_t* __restrict__ gid,
                                                   const float* __restrict__ L,
                                                   const int32_t* __restrict__ G, float eps,
                                                   unsigned char* __restrict__ state, int B,
                                                   int Hq, int Hkv, long long tokens, int cont,
                                                   unsigned char* __restrict__ rtab, int prep,
                                                   const SeqDesc* __restrict__ seqs, int nseq,
                                                   size_t state_stride)
{
    grid_dep_launch();
    if (prep && blockIdx.z == gridDim.z - 1) {  // independent of the deltas: no wait
        const int nb = gridDim.x * gridDim.y, e0 = blockIdx.y * gridDim.x + blockIdx.x;
        // prep_head keeps its group table in shared memory: every pass of a block's loop ends
        // with a barrier before the next pass overwrites it
        if (nseq == 0) {
            for (int e = e0; e < Hq; e += nb) {
                prep_head(e, gid, L, G, eps, state, B, Hq, Hkv, tokens, cont != 0, rtab);
                __syncthreads();
            }
        } else {  // a packed batch: every sequence's state (B = 1) gets a header and the tables
            for (int e = e0; e < Hq * nseq; e += nb) {
                const int i = e / Hq;
                prep_head(e % Hq, gid, L, G, eps, state + size_t(i) * state_stride, 1, Hq, Hkv,
                          seqs[i].T, false, i == 0 ? rtab : nullptr);
                __syncthreads();
            }
        }
        return;
    }
    grid_dep_wait();
    const int sl = blockIdx.x;
    const int nl = threadIdx.x >> 4, rq = threadIdx.x & 15;
    const int n = blockIdx.y * kScanCols + nl;
    __shared__ float fin[kScanCols][64 + 4];
    // this block's (b, kv) unit: its chunk-state index base and its part of the final state
    size_t chunk0;
    float* unit;
    if (nseq == 0) {
        const int bkv = blockIdx.z;
        chunk0 = size_t(bkv) * NC;
        unit = body + size_t(bkv) * kFP * kW;
    } else {
        const int i = blockIdx.z / Hkv, kv = blockIdx.z % Hkv;
        const SeqDesc sd = seqs[i];
        NC = sd.NC;
        chunk0 = size_t(sd.chunk0) + size_t(kv) * sd.NC;
        unit = reinterpret_cast<float*>(state + size_t(i) * state_stride + kHeaderBytes +
                                        coef_bytes(Hq)) + size_t(kv) * kFP * kW;
    }
    // the prefix before this call: zero, or (continuation) the state's current contents
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    const int f = sl * 64 + 4 * rq, c_first = cont ? 0 : 1;
    if (cont && n < kDV) {
#pragma unroll
        for (int e = 0; e < 4; ++e) a[e] = unit[size_t(f + e) * kDV + n];
    } else if (cont && n == kDV) {
        const float4 z4 = *reinterpret_cast<const float4*>(unit + size_t(kFP) * kDV + f);
        a[0] = z4.x; a[1] = z4.y; a[2] = z4.z; a[3] = z4.w;
    }
    if (n < kW) {
        const float* src = dS + (chunk0 * kW + n) * kFP + f;
        unsigned char* dst = img + (chunk0 * kSlices + sl) * kImgSliceBytes + n * 128 + 8 * rq;
        const size_t sstride = size_t(kW) * kFP, dstride = size_t(kSlices) * kImgSliceBytes;
        constexpr int kDepth = 8;
        for (int c0 = 0; c0 < NC; c0 += kDepth) {
            float4 d[kDepth];
#pragma unroll
            for (int x = 0; x < kDepth; ++x)
                if (c0 + x < NC)
                    d[x] = __ldcs(reinterpret_cast<const float4*>(src + (c0 + x) * sstride));
#pragma unroll
            for (int x = 0; x < kDepth; ++x) {
                const int c = c0 + x;
                if (c < NC) {
                    if (c >= c_first)
                        *reinterpret_cast<uint2*>(dst + c * dstride) =
                            make_uint2(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]));
                    a[0] += d[x].x;
                    a[1] += d[x].y;
                    a[2] += d[x].z;
                    a[3] += d[x].w;
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) fin[nl][4 * rq + e] = a[e];
    __syncthreads();  // every read of the old state in this block precedes the writes below
    // final state of unit bkv: Hv[f][n] (n < 64), z[f] (n == 64); thread = (row, 4 columns)
    const int fl = threadIdx.x >> 2, cq = threadIdx.x & 3;
    const int nn0 = blockIdx.y * kScanCols + 4 * cq;
    if (nn0 + 3 < kDV) {
        *reinterpret_cast<float4*>(unit + size_t(sl * 64 + fl) * kDV + nn0) =
            make_float4(fin[4 * cq][fl], fin[4 * cq + 1][fl], fin[4 * cq + 2][fl],
                        fin[4 * cq + 3][fl]);
    } else if (nn0 == kDV) {
        unit[size_t(kFP) * kDV + sl * 64 + fl] = fin[4 * cq][fl];
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
bool make_map_uncached(CUtensorMap* m, const void* base, int T, int heads);
bool make_img_map_uncached(CUtensorMap* m, const void* base, size_t slices);

// Tensor maps are pure functions of (base address, sizes): the last few of each host thread
// are kept, so repeated calls on the same buffers skip the encoding.
struct MapCacheEntry {
    const void* base;
    unsigned long long a, b;
    int kind;
    CUtensorMap map;
};
bool map_cache_get(int kind, const void* base, unsigned long long a, unsigned long long b,
                   CUtensorMap* m, MapCacheEntry** slot)
{
    constexpr int kEntries = 16;
    thread_local MapCacheEntry cache[kEntries] = {};
    thread_local int next = 0;
    int dev = -1;
    cudaGetDevice(&dev);
    const unsigned long long bk = b ^ (static_cast<unsigned long long>(dev + 1) << 48);
    for (auto& e : cache)
        if (e.kind == kind + 1 && e.base == base && e.a == a && e.b == bk) {
            *m = e.map;
            return true;
        }
    MapCacheEntry& e = cache[next];
    next = (next + 1) % kEntries;
    e.kind = 0;  // filled by the caller once the encoding succeeded
    e.base = base;
    e.a = a;
    e.b = bk;
    *slot = &e;
    return false;
}

bool make_map(CUtensorMap* m, const void* base, int T, int heads)
{
    MapCacheEntry* slot = nullptr;
    if (map_cache_get(0, base, (unsigned long long)T, (unsigned long long)heads, m, &slot))
        return true;
    if (!make_map_uncached(m, base, T, heads)) return false;
    slot->map = *m;
    slot->kind = 1;
    return true;
}

bool make_map_uncached(CUtensorMap* m, const void* base, int T, int heads)
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

// chunk-state images [slices][80 rows][64] bf16 viewed as 2D {64, slices * 80}; box {64, 65}
// = rows 0..64 of one slice per copy (rows 65..79 are kept zero in shared memory by the
// readout and never written by the scan); 128B swizzle on the way in.
bool make_img_map(CUtensorMap* m, const void* base, size_t slices)
{
    MapCacheEntry* slot = nullptr;
    if (map_cache_get(1, base, (unsigned long long)slices, 0ull, m, &slot)) return true;
    if (!make_img_map_uncached(m, base, slices)) return false;
    slot->map = *m;
    slot->kind = 2;
    return true;
}

bool make_img_map_uncached(CUtensorMap* m, const void* base, size_t slices)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {64, cuuint64_t(slices) * 80};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {64, kW};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Test hook of oal_set_debug_skip_copies (process-wide).
std::atomic<int> g_skip_copies{0};

namespace {

int sm_count()
{
    constexpr int kMaxDev = 64;
    static std::atomic<int> cached[kMaxDev] = {};
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < kMaxDev && (n = cached[dev].load(std::memory_order_relaxed)) > 0)
        return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < kMaxDev) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// The kernel attributes of the tensor-core prefill, set once per device (they are properties
// of the kernels in the current device's context).
cudaError_t set_tc_attributes_once();


}  // namespace

size_t tc_image_bytes(int B, int Hkv, int T)
{
    const size_t NC = size_t((T + tc::kC - 1) / tc::kC);
    return size_t(B) * Hkv * NC * tc::kImgChunkBytes;
}

static size_t tc_delta_bytes(int B, int Hkv, int T)
{
    const size_t NC = size_t((T + tc::kC - 1) / tc::kC);
    return size_t(B) * Hkv * NC * kW * kFP * 4;
}

// normalisers of the intra-chunk sums, [B*Hq][T] fp32
static size_t tc_zin_bytes(int B, int Hq, int T) { return align256(size_t(B) * Hq * T * 4); }

size_t tc_workspace_bytes(int B, int Hq, int Hkv, int T)
{
    return tc_image_bytes(B, Hkv, T) + tc_delta_bytes(B, Hkv, T) + size_t(Hq) * kTabBytes +
           tc_zin_bytes(B, Hq, T);
}

unsigned char* tc_rtab(void* ws, int B, int Hkv, int T)
{
    return static_cast<unsigned char*>(ws) + tc_image_bytes(B, Hkv, T) + tc_delta_bytes(B, Hkv, T);
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

namespace {

cudaError_t set_tc_attributes_once()
{
    constexpr int kMaxDev = 64;
    static std::atomic<int> done[kMaxDev] = {};
    static std::mutex mu;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDev && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> g(mu);
    const std::pair<const void*, int> smem[] = {
        {reinterpret_cast<const void*>(tc::delta_kernel), int(tc::kSmemBytes)},
        {reinterpret_cast<const void*>(tc::intra::intra_kernel), int(tc::intra::kSmemBytes)},
        {reinterpret_cast<const void*>(tc::fm::intra_fm_kernel), int(tc::fm::kSmemBytes)},
        {reinterpret_cast<const void*>(tc::rd::readout_kernel), int(tc::rd::kSmemBytes)}};
    for (const auto& k : smem)
        if ((e = cudaFuncSetAttribute(k.first, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      k.second)) != cudaSuccess)
            return e;
    // two intra-chunk CTAs per SM need the whole shared-memory carve-out
    if ((e = cudaFuncSetAttribute(reinterpret_cast<const void*>(tc::intra::intra_kernel),
                                  cudaFuncAttributePreferredSharedMemoryCarveout, 100)) != cudaSuccess)
        return e;
    if (dev >= 0 && dev < kMaxDev) done[dev].store(1, std::memory_order_release);
    return cudaSuccess;
}

// What the scan kernel needs besides Params: the state (or, for a packed batch, the first of
// the per-sequence states and their stride) and the prep plane's inputs.
struct ScanArgs {
    float* body;
    unsigned char* state;
    size_t stride;
    const int32_t* gid;
    const float* L;
    const int32_t* G;
    float eps;
    long long tokens;
    int prep;
};

// The kernel sequence shared by a uniform batch and a packed one: chunk deltas -> (helper
// stream: intra-chunk sums) -> scan -> join -> inter-chunk readout.  P carries the unit and
// item counts; grids follow from them.
int run_prefill_tc(tc::Params& P, const CUtensorMap& mq, const CUtensorMap& mk,
                   const CUtensorMap& mv, const CUtensorMap& mi, float* zin, const ScanArgs& sa,
                   int scan_planes, bool fm_intra, bool overlap, cudaStream_t st)
{
    const bool with_out = P.out != nullptr;
    const int nsm = sm_count();
    OAL_CUDA_TRY(set_tc_attributes_once());
    // One stream, each kernel a programmatic dependent of the one before: chunk deltas ->
    // scan -> intra-chunk sums -> readout.  The intra-chunk kernel needs only q, k, v, so its
    // CTAs fill SMs as the memory-bound scan's blocks retire instead of waiting for the scan;
    // it waits for the scan only at its very end, so that its completion (what the readout
    // waits for) implies the scan's.
    if (P.n_units > 0) {
        const int grid0 = std::max(1, std::min(nsm, P.n_units));
        LaunchScope ls("delta_tc", st);
        OAL_CUDA_TRY(launch_ex(tc::delta_kernel, dim3(grid0), dim3(tc::kThreads), tc::kSmemBytes,
                               st, false, mk, mv, P));
    }
    {
        LaunchScope ls("scan", st);
        OAL_CUDA_TRY(launch_ex(tc::scan_kernel,
                               dim3(tc::kSlices, tc::kScanColGroups, scan_planes + sa.prep),
                               dim3(256), 0, st, overlap && P.n_units > 0, (const float*)P.dS,
                               P.img, sa.body, P.NC, sa.gid, sa.L, sa.G, sa.eps, sa.state, P.B,
                               P.Hq, P.Hkv, sa.tokens, P.cont, const_cast<unsigned char*>(P.rtab), sa.prep,
                               (const tc::SeqDesc*)P.seqs, P.nseq, sa.stride));
    }
    if (!with_out) return OAL_OK;  // no out: the state alone is wanted
    if (P.n_intra > 0) {
        // chunk 0 of a fresh prefill is final here
        if (fm_intra) {  // free coefficients: Phi(Q_c) Psi(K_c)^T through the feature map
            LaunchScope ls("intra_fm_tc", st);
            OAL_CUDA_TRY(launch_ex(tc::fm::intra_fm_kernel, dim3(P.n_intra),
                                   dim3(tc::fm::kThreads), tc::fm::kSmemBytes, st, overlap, mq,
                                   mk, mv, P, zin));
        } else {
            // persistent: two CTAs per SM walk the items (b*h, chunk)
            const int grid1 = std::max(1, std::min(tc::intra::kCtasPerSm * nsm, P.n_intra));
            LaunchScope ls("intra_tc", st);
            OAL_CUDA_TRY(launch_ex(tc::intra::intra_kernel, dim3(grid1),
                                   dim3(tc::intra::kThreads), tc::intra::kSmemBytes, st, overlap,
                                   mq, mk, mv, P, zin));
        }
    }
    if (P.n_read > 0) {
        // persistent: one CTA per SM walks the items (b*h, chunk) with an inter-chunk part
        const int grid2 = std::max(1, std::min(nsm, P.n_read));
        LaunchScope ls("readout_tc", st);
        OAL_CUDA_TRY(launch_ex(tc::rd::readout_kernel, dim3(grid2), dim3(tc::rd::kThreads),
                               tc::rd::kSmemBytes, st, overlap, mq, mi, P, (const float*)zin));
    }
    return OAL_OK;
}

}  // namespace

int launch_prefill_tc(const void* q, const void* k, const void* v, const int32_t* gid,
                      const float* L, const int32_t* G, float eps, float* out, void* state,
                      void* ws, int B, int T, int Hq, int Hkv, bool overlap, bool cont,
                      cudaStream_t st, bool fm_intra)
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
    P.img = wsb;
    P.dS = reinterpret_cast<float*>(wsb + tc_image_bytes(B, Hkv, T));
    unsigned char* rtab = tc_rtab(ws, B, Hkv, T);
    P.rtab = rtab;
    float* zin = reinterpret_cast<float*>(rtab + size_t(Hq) * kTabBytes);
    P.out = out;
    P.B = B;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.T = T;
    P.NC = NC;
    P.cont = cont ? 1 : 0;
    P.skip_copies = g_skip_copies.load() ? 1 : 0;
    P.n_units = B * Hkv * NC * tc::kNumSlabs;
    P.n_intra = NC * B * Hq;
    P.n_read = B * Hq * (cont ? NC : NC - 1);
    P.nseq = 0;
    ScanArgs sa{body, sb, 0, gid, L, G, eps, (long long)T, fm_intra ? 0 : 1};
    return run_prefill_tc(P, mq, mk, mv, mi, zin, sa, B * Hkv, fm_intra, overlap, st);
}

// ---- packed variable-length batch ----------------------------------------------------------

TcPackedLayout tc_packed_layout(int Hq, int Hkv, const int32_t* lens, int n)
{
    TcPackedLayout l{};
    long long chunks = 0, tokens = 0;
    for (int i = 0; i < n; ++i) {
        chunks += (lens[i] + tc::kC - 1) / tc::kC;
        tokens += lens[i];
    }
    l.chunks = chunks;
    l.tokens = tokens;
    l.img = 0;
    l.dS = l.img + size_t(chunks) * Hkv * tc::kImgChunkBytes;
    l.rtab = l.dS + size_t(chunks) * Hkv * kW * kFP * 4;
    l.zin = l.rtab + size_t(Hq) * kTabBytes;
    l.seqs = l.zin + align256(size_t(tokens) * Hq * 4);
    l.maps = l.seqs + align256(size_t(n) * sizeof(tc::SeqDesc));
    l.total = std::max<size_t>(256, l.maps + align256(size_t(n) * 3 * sizeof(CUtensorMap)));
    return l;
}

int launch_prefill_tc_packed(const void* q, const void* k, const void* v, const int32_t* gid,
                             const float* L, const int32_t* G, float eps, float* out,
                             unsigned char* states, size_t stride, void* ws, const int32_t* lens,
                             int n, int Hq, int Hkv, bool overlap, cudaStream_t st)
{
    if (n == 0) return OAL_OK;
    const TcPackedLayout lay = tc_packed_layout(Hq, Hkv, lens, n);
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    std::vector<tc::SeqDesc> sd(static_cast<size_t>(n));
    std::vector<CUtensorMap> maps(size_t(n) * 3);
    std::memset(maps.data(), 0, maps.size() * sizeof(CUtensorMap));
    const size_t rq = size_t(Hq) * OAL_HEAD_DIM * 2, rkv = size_t(Hkv) * OAL_HEAD_DIM * 2;
    int tok = 0, chunk0 = 0, unit0 = 0, intra0 = 0, read0 = 0;
    for (int i = 0; i < n; ++i) {
        const int T = lens[i], NC = (T + tc::kC - 1) / tc::kC;
        sd[size_t(i)] = tc::SeqDesc{T, NC, tok, chunk0, unit0, intra0, read0, 0};
        if (T > 0) {  // a sequence without tokens has no units or items: its maps stay unused
            const unsigned char* qi = static_cast<const unsigned char*>(q) + size_t(tok) * rq;
            const unsigned char* ki = static_cast<const unsigned char*>(k) + size_t(tok) * rkv;
            const unsigned char* vi = static_cast<const unsigned char*>(v) + size_t(tok) * rkv;
            if (!make_map(&maps[3 * size_t(i)], qi, T, Hq) ||
                !make_map(&maps[3 * size_t(i) + 1], ki, T, Hkv) ||
                !make_map(&maps[3 * size_t(i) + 2], vi, T, Hkv))
                return OAL_ERR_CUDA;
        }
        tok += T;
        chunk0 += Hkv * NC;
        unit0 += Hkv * NC * tc::kNumSlabs;
        intra0 += Hq * NC;
        read0 += Hq * std::max(NC - 1, 0);
    }
    CUtensorMap mi, none;
    std::memset(&none, 0, sizeof(none));
    if (lay.chunks > 0 && !make_img_map(&mi, wsb, size_t(lay.chunks) * Hkv * tc::kSlices))
        return OAL_ERR_CUDA;
    if (lay.chunks == 0) mi = none;
    // descriptors and tensor maps into the workspace, ahead of the kernels on the same stream
    OAL_CUDA_TRY(cudaMemcpyAsync(wsb + lay.seqs, sd.data(), sd.size() * sizeof(tc::SeqDesc),
                                 cudaMemcpyHostToDevice, st));
    OAL_CUDA_TRY(cudaMemcpyAsync(wsb + lay.maps, maps.data(), maps.size() * sizeof(CUtensorMap),
                                 cudaMemcpyHostToDevice, st));
    tc::Params P{};
    P.gid = gid;
    P.L = L;
    P.G = G;
    P.eps = eps;
    P.img = wsb + lay.img;
    P.dS = reinterpret_cast<float*>(wsb + lay.dS);
    P.rtab = wsb + lay.rtab;
    float* zin = reinterpret_cast<float*>(wsb + lay.zin);
    P.out = out;
    P.B = n;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.T = 0;
    P.NC = 0;
    P.cont = 0;
    P.skip_copies = g_skip_copies.load() ? 1 : 0;
    P.n_units = unit0;
    P.n_intra = intra0;
    P.n_read = read0;
    P.nseq = n;
    P.seqs = reinterpret_cast<const tc::SeqDesc*>(wsb + lay.seqs);
    P.maps = reinterpret_cast<const CUtensorMap*>(wsb + lay.maps);
    ScanArgs sa{nullptr, states, stride, gid, L, G, eps, 0, 1};
    return run_prefill_tc(P, none, none, none, mi, zin, sa, n * Hkv, false, overlap, st);
}

}  // namespace oal
