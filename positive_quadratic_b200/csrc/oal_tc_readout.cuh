// oal_tc_readout.cuh -- the inter-chunk readout of the chunked bf16 prefill on tensor cores
// (included by oal_tc.cu inside namespace oal::tc).
//
// "OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式: for query row i of chunk c,
//   u_i = phi(q_i)^T S_c + U_intra_i,    yhat_i = u_i[0:64] / u_i[64]            (eq. (5))
// where S_c is the chunk's exclusive prefix state (eq. (4), stored as a bf16 image by the
// scan kernel) and U_intra_i the intra-chunk sum of eqs. (2)-(3) left by the intra kernel
// (U_intra[:64] in `out`, U_intra[64] in the workspace).
//
// One CTA per SM walks a static list of items (b*h, chunk c >= 1, or every chunk when the call
// continues a prefix).  Work moves in slice pairs: a pair is 2 x 64 packed rows, its phi in
// tensor-memory slot g % 4 (64 columns) and its state image in 20 KB shared-memory stage g % 6
// (g counts pairs over all items of the CTA), so the image copies run two pairs ahead of the
// phi slots.
// Roles (24 warps):
//   warps 0-15   phi producers: set = warp >> 2 produces the pairs g = set (mod 4) into slot
//                `set`, row quarter = warp & 3; phi of both slices, then (after the slot and
//                the image stage are free / loaded) tcgen05.st into the slot.  A pair is
//                published only once its image has landed, so an MMA issuer waits on one
//                barrier per pair.  Sixteen producers: one packed-bf16 phi slice costs a warp
//                about 500 cycles, so four warps per scheduler are needed to keep up.
//   warps 16-19  epilogue (row quarter = warp - 16): U_A + U_B + U_intra, normalised.  The
//                item's U_intra rows are copied into shared memory while the item runs, so
//                the accumulators are released as soon as they have been read.
//   warps 20, 21 MMA issuers A (even pairs, accumulator U_A) and B (odd pairs, U_B).  Each
//                barrier wait, fence or commit stalls the issuing thread for a few hundred
//                cycles while the tensor pipe drains its short queue; with two issuers one
//                issues while the other waits.  U_A + U_B is summed in a fixed order.
//   warps 22, 23 state-image copies, one slice of each pair each: one tiled tensor copy of
//                the slice's 65 live rows (the 15 padding rows of the N = 80 operand stay zero
//                from the CTA's start).  Warp 22 also loads the Q tile and per-head
//                coefficient table one item ahead (double-buffered).
// Tensor memory (512 columns): U_A [0, 80), U_B [96, 176), phi slots [192, 448).
// Every wait is bounded; one that runs out sets OAL_ERR_TIMEOUT and every role leaves its loop
// in order (copies drained, MMAs committed, tensor memory freed by the allocating warp).

namespace rd {

constexpr int kPhiWarps = 16, kEpiWarp0 = 16, kMmaA = 20, kMmaB = 21, kImgWarp0 = 22;
constexpr int kWarps = 24;
constexpr int kThreads = kWarps * 32;
constexpr int kSlots = 4;            // pair slots of phi in tensor memory
// image stages (pair g in stage g % kStages).  Even and at least kSlots: the next use of the
// stage holding pair g - 4 is then pair g - 4 + kStages, issued by pair g's MMA issuer after
// pair g, so a barrier of that stage is never two phases ahead of a waiter (see below).
constexpr int kStages = 6;
constexpr int kPairs = kSlices / 2;  // 17

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0;                                     // 2 x 16 KB Q tiles
constexpr uint32_t kOffB = 32768;                                 // 6 x 20 KB image stages
constexpr uint32_t kOffTab = kOffB + kStages * kImgPairBytes;     // 2 x per-head tables
constexpr uint32_t kOffCtl = kOffTab + 2 * kTabBytes;
constexpr uint32_t kOffUI = kOffCtl + 1024;                       // U_intra rows [128][64] fp32
constexpr uint32_t kSmemBytes = kOffUI + kC * kDV * 4 + 1024;
static_assert(kOffB % 1024 == 0 && kOffTab % 16 == 0 && kOffCtl % 8 == 0, "alignment");
static_assert(kSmemBytes <= 232448, "shared memory");

// tensor memory columns
constexpr uint32_t kColUA = 0, kColUB = 96, kColPhi = 192;
static_assert(kColPhi + kSlots * 64 <= kTmemCols && kColUB + 80 <= kColPhi, "tensor memory map");

struct Bars {
    uint64_t q_full[2], q_empty[2];
    uint64_t f_full[kSlots];                    // phi of the slot's pair published
    uint64_t b_full[kStages], done_mma[kStages];  // image landed; the stage's pair multiplied
    uint64_t u_full, u_empty, done_a, done_b, ui_full;
};
struct Ctl {
    Bars bar;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Ctl) <= 1024, "control block");

// Items of the inter-chunk readout (item_ref): chunk-major within a sequence, the query heads
// of a chunk adjacent (they read the same state image, which then stays in L2).

// 8-dim chunks of the q row that the packed rows [F, F + n) read
template <int F, int n>
constexpr bool rows_need_chunk(int ch)
{
    for (int i = 0; i < n; ++i) {
        const RT rt = feature_rt(F + i);
        if ((rt.r < 64 && rt.r / 8 == ch) || (rt.t < 64 && rt.t / 8 == ch)) return true;
    }
    return false;
}

// phi of the diagonal / linear / constant slices (64 rows with compile-time (r, t)), in
// packed bf16 like the off-diagonal slices: phi = bf16(bf16(q_r q_t) * bf16(c)).  coef_t holds
// the (fp32) coefficients of rows 1792.. .  The q values are loaded per group of 8 rows, so
// that only the chunks a group reads are live at a time; each pair of rows takes its two q_r
// and its two q_t into one bf16x2 register each with one byte permute (q_64 = 1 and q_65 = 0
// come from a constant word).
template <int F0>
__device__ __forceinline__ void phi_tail_static(const unsigned char* qt, const float* coef_t,
                                                int row, uint32_t (&w)[32])
{
    constexpr uint32_t kOneZero = 0x00003F80u;  // bf16 halves (1, 0)
    static_for<8>([&](auto X) {
        constexpr int x = decltype(X)::value;
        constexpr int F = F0 + 8 * x;
        uint32_t qp[32];  // packed bf16 pairs of the chunks this group reads
        static_for<8>([&](auto CH) {
            constexpr int ch = decltype(CH)::value;
            if constexpr (rows_need_chunk<F, 8>(ch)) {
                const uint4 v = *reinterpret_cast<const uint4*>(qt + kmajor_chunk(row, ch));
                qp[4 * ch + 0] = v.x;
                qp[4 * ch + 1] = v.y;
                qp[4 * ch + 2] = v.z;
                qp[4 * ch + 3] = v.w;
            }
        });
        // the 32-bit word holding q_r, and the half of it (r = 64, 65: the constant word)
        auto word = [&](auto R) -> uint32_t {
            constexpr int r = decltype(R)::value;
            if constexpr (r >= 64) return kOneZero;
            else return qp[r >> 1];
        };
        auto half = [](int r) constexpr -> int { return r >= 64 ? r - 64 : (r & 1); };
        const float* cp = coef_t + (F - kOffDiagRows);
        const float4 c0 = *reinterpret_cast<const float4*>(cp);
        const float4 c1 = *reinterpret_cast<const float4*>(cp + 4);
        const uint32_t cw[4] = {pack_bf16x2(c0.x, c0.y), pack_bf16x2(c0.z, c0.w),
                                pack_bf16x2(c1.x, c1.y), pack_bf16x2(c1.z, c1.w)};
        static_for<4>([&](auto E) {
            constexpr int e = decltype(E)::value;
            constexpr RT a = feature_rt(F + 2 * e);
            constexpr RT b = feature_rt(F + 2 * e + 1);
            // low half from the first word, high half from the second (bytes 4..7)
            constexpr uint32_t sr = (half(a.r) ? 0x32u : 0x10u) | ((half(b.r) ? 0x76u : 0x54u) << 8);
            constexpr uint32_t st = (half(a.t) ? 0x32u : 0x10u) | ((half(b.t) ? 0x76u : 0x54u) << 8);
            const uint32_t xr = __byte_perm(word(std::integral_constant<int, a.r>{}),
                                            word(std::integral_constant<int, b.r>{}), sr);
            const uint32_t xt = __byte_perm(word(std::integral_constant<int, a.t>{}),
                                            word(std::integral_constant<int, b.t>{}), st);
            w[4 * x + e] = bmul2(bmul2(xr, xt), cw[e]);
        });
    });
}

__device__ __forceinline__ void phi_slice(const unsigned char* qt, const unsigned char* tab, int s,
                                          int row, uint32_t (&w)[32])
{
    if (s < kOffDiagSlices) {
        const uint32_t* ch = reinterpret_cast<const uint32_t*>(tab + kTabCoefH);
        if (tab[kTabPure + (c_block_rt[s] >> 3)])  // the same for the whole item
            phi_offdiag_pure(qt, ch, s, row, w);
        else
            phi_offdiag(qt, ch, s, row, w);
        return;
    }
    const float* ct = reinterpret_cast<const float*>(tab + kTabCoefT);
    const int sel = s - kOffDiagSlices;
    static_for<kSlices - kOffDiagSlices>([&](auto I) {
        constexpr int i = decltype(I)::value;
        if (sel == i) phi_tail_static<kOffDiagRows + i * 64>(qt, ct, row, w);
    });
}

__global__ void __launch_bounds__(kThreads, 1)
    readout_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_img, Params P,
                   const float* __restrict__ zin)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl& ctl = *reinterpret_cast<Ctl*>(sm + kOffCtl);
    Bars& bar = ctl.bar;
    volatile int* abort_flag = &ctl.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = P.n_read;
    P.tm_q = &tm_q;
    P.tm_img = &tm_img;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar.q_full[i], 1);
            mbar_init(&bar.q_empty[i], kPhiWarps);
        }
        for (int i = 0; i < kSlots; ++i) mbar_init(&bar.f_full[i], 4);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bar.b_full[i], 2);
            mbar_init(&bar.done_mma[i], 1);
        }
        mbar_init(&bar.u_full, 2);
        mbar_init(&bar.u_empty, 4);
        mbar_init(&bar.done_a, 1);
        mbar_init(&bar.done_b, 1);
        mbar_init(&bar.ui_full, 1);
        ctl.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaA) {
        tmem_alloc(&ctl.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // image stages: copies fill rows 0..64 of each slice; rows 65..79 (the N = 80 padding of
    // the MMA) stay zero from here on
    for (int i = threadIdx.x; i < int(kStages * kImgPairBytes / 16); i += blockDim.x)
        reinterpret_cast<uint4*>(sm + kOffB)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    grid_dep_launch();
    grid_dep_wait();  // images, tables and the intra-chunk sums are complete from here

    if (warp < kPhiWarps) {
        // ---- phi producers -------------------------------------------------------------------
        const int qw = warp & 3, set = warp >> 2, row = qw * 32 + lane;
        const uint32_t lanebase = tmem + (uint32_t(qw * 32) << 16);
        const uint32_t slotcol = lanebase + kColPhi + set * 64;
        bool ok = true;
        for (int j = 0, idx = blockIdx.x; idx < n_items && ok; ++j, idx += gridDim.x) {
            const int qb = j & 1, gp0 = j * kPairs;
            ok = wait_all_sleep(&bar.q_full[qb], (j >> 1) & 1, abort_flag);
            if (!ok) break;
            const unsigned char* qt = sm + kOffQ + qb * kTileBytes;
            const unsigned char* tab = sm + kOffTab + qb * kTabBytes;
            // this set's pairs of the item: g = gp0 + p with g % 4 == set
            for (int p = (set - gp0 % kSlots + kSlots) % kSlots; p < kPairs && ok; p += kSlots) {
                const int g = gp0 + p;
                uint32_t w[32];
                phi_slice(qt, tab, 2 * p, row, w);
                // the slot is free once pair g - 4 has been multiplied (the next completion of
                // that stage's barrier is pair g - 4 + kStages, after pair g on the same issuer)
                ok = g < kSlots || wait_all(&bar.done_mma[(g - kSlots) % kStages],
                                            ((g - kSlots) / kStages) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                tmem_st32(slotcol, w);
                phi_slice(qt, tab, 2 * p + 1, row, w);
                tmem_st32(slotcol + 32, w);
                ok = wait_all(&bar.b_full[g % kStages], (g / kStages) & 1, abort_flag);
                if (!ok) break;
                tmem_st_wait();
                tc_fence_before();
                warp_arrive(&bar.f_full[set]);
            }
            if (ok) warp_arrive(&bar.q_empty[qb]);
        }
    } else if (warp < kEpiWarp0 + 4) {
        // ---- epilogue: yhat = (U_A + U_B + U_intra)[:64] / (U_A + U_B + U_intra)[64] ---------
        const int qw = warp - kEpiWarp0, row = qw * 32 + lane;
        const uint32_t lanebase = tmem + (uint32_t(qw * 32) << 16);
        const float* ui = reinterpret_cast<const float*>(sm + kOffUI) + row * kDV;
        // the U_intra rows of item jj (one bulk copy of up to 32 KB, rows 256 B apart)
        auto prefetch = [&](int idx) {
            const ItemRef it = item_ref(idx, P, false);
            const int nrows = min(kC, it.T - it.c * kC);
            mbar_expect_tx(&bar.ui_full, uint32_t(nrows) * kDV * 4);
            bulk_g2s(sm + kOffUI, P.out + (it.orow + size_t(it.c) * kC) * kDV,
                     uint32_t(nrows) * kDV * 4, &bar.ui_full);
        };
        int last_pf = -1;  // item index j of the last U_intra copy issued, if not waited for
        if (qw == 0 && lane == 0 && int(blockIdx.x) < n_items && !P.skip_copies) {
            prefetch(blockIdx.x);
            last_pf = 0;
        }
        // all four warps run the same iterations and leave together (named barrier below)
        for (int j = 0, idx = blockIdx.x; idx < n_items; ++j, idx += gridDim.x) {
            const ItemRef it = item_ref(idx, P, false);
            const int irow = it.c * kC + row;
            const bool valid = irow < it.T;
            const size_t ro = it.orow + irow;
            const float zi = valid ? zin[ro] : 0.f;  // in flight while the item runs
            const bool got = wait_all_sleep(&bar.ui_full, j & 1, abort_flag) &&
                             wait_all_sleep(&bar.u_full, j & 1, abort_flag);
            if (got) {
                last_pf = -1;
                tc_fence_after();
                float z = tmem_ld1(lanebase + kColUA + 64);
                const float zb = tmem_ld1(lanebase + kColUB + 64);
                tmem_ld_wait();
                const float inv = 1.f / ((z + zb) + zi);
                float4* o = reinterpret_cast<float4*>(P.out + ro * kDV);
#pragma unroll 1
                for (int x = 0; x < 4; ++x) {
                    float ua[16], ub[16];
                    tmem_ld16(lanebase + kColUA + 16 * x, ua);
                    tmem_ld16(lanebase + kColUB + 16 * x, ub);
                    tmem_ld_wait();
                    if (x == 3) {  // every read of the accumulators is done
                        tc_fence_before();
                        warp_arrive(&bar.u_empty);
                    }
                    if (valid) {
#pragma unroll
                        for (int i0 = 0; i0 < 4; ++i0) {
                            const int i = (i0 + lane) & 3;  // staggered: fewer bank conflicts
                            const float4 u4 =
                                *reinterpret_cast<const float4*>(ui + 16 * x + 4 * i);
                            float a[4], bb[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                // ua/ub[4 i + e] without dynamic register indexing
                                float va = ua[e], vb = ub[e];
#pragma unroll
                                for (int k = 1; k < 4; ++k)
                                    if (i == k) {
                                        va = ua[4 * k + e];
                                        vb = ub[4 * k + e];
                                    }
                                a[e] = va;
                                bb[e] = vb;
                            }
                            o[4 * x + i] = make_float4(((a[0] + bb[0]) + u4.x) * inv,
                                                       ((a[1] + bb[1]) + u4.y) * inv,
                                                       ((a[2] + bb[2]) + u4.z) * inv,
                                                       ((a[3] + bb[3]) + u4.w) * inv);
                        }
                    }
                }
            }
            // the staged rows are free for the next copy once all four warps are done
            if (!named_bar_and(1, 128, got)) break;
            const int nidx = idx + gridDim.x;
            if (qw == 0 && lane == 0 && nidx < n_items && !P.skip_copies) {
                prefetch(nidx);
                last_pf = j + 1;
            }
        }
        // no copy may still be in flight when the CTA exits
        if (qw == 0 && lane == 0 && last_pf >= 0) bounded_spin_done(&bar.ui_full, last_pf & 1);
        __syncwarp();
    } else if (warp == kMmaA || warp == kMmaB) {
        // ---- MMA issuers: U += phi(pair) image(pair), 8 MMAs M=128 N=80 K=16 per pair ---------
        const bool isA = warp == kMmaA;
        constexpr uint32_t id_u = idesc_bf16(128, 80, false, false);  // A (TMEM), B K-major
        const uint32_t sm0 = smem_u32(sm);
        const uint32_t ucol = tmem + (isA ? kColUA : kColUB);
        bool ok = true;
        for (int j = 0, idx = blockIdx.x; idx < n_items && ok; ++j, idx += gridDim.x) {
            const int gp0 = j * kPairs;
            // the previous item's epilogue has read this accumulator
            if (j >= 1) ok = wait_all(&bar.u_empty, (j - 1) & 1, abort_flag);
            for (int p = isA ? 0 : 1; p < kPairs && ok; p += 2) {
                const int g = gp0 + p, slot = g % kSlots;
                ok = wait_all(&bar.f_full[slot], (g / kSlots) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t bst = sm0 + kOffB + (g % kStages) * kImgPairBytes;
#pragma unroll
                    for (int x = 0; x < 2; ++x)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16_ts(ucol, tmem + kColPhi + slot * 64 + x * 32 + ks * 8,
                                        sdesc_sw128(bst + x * kImgSliceBytes + ks * 32, 16, 1024),
                                        id_u, (p > 1 || x > 0 || ks > 0) ? 1u : 0u);
                    mma_commit(&bar.done_mma[g % kStages]);
                }
                __syncwarp();
            }
            if (ok) {
                if (elect_one()) mma_commit(&bar.u_full);
                __syncwarp();
            }
        }
        uint64_t* done = isA ? &bar.done_a : &bar.done_b;
        if (elect_one()) mma_commit(done);
        __syncwarp();
        if (lane == 0) bounded_spin_done(done, 0);
        __syncwarp();
    } else if (warp < kImgWarp0 + 2) {
        // ---- state-image copies: slice x = warp - kImgWarp0 of every pair (65 of its 80 rows);
        // warp x = 0 also loads Q tile + table of item j + 1 while item j's images stream ----
        const int x = warp - kImgWarp0;
        if (lane == 0) {
            int issued = 0, lq = -1;
            bool ok = true;
            auto load_q = [&](int jj, int qidx) {
                if (P.skip_copies) return;
                const ItemRef it = item_ref(qidx, P, false);
                const int qb = jj & 1;
                if (P.nseq) tmap_acquire(it.mq);
                mbar_expect_tx(&bar.q_full[qb], kTileBytes + kTabBytes);
                tma_load_3d(sm + kOffQ + qb * kTileBytes, it.mq, &bar.q_full[qb], 0, it.c * kC,
                            it.qz);
                bulk_g2s(sm + kOffTab + qb * kTabBytes, P.rtab + size_t(it.h) * kTabBytes,
                         kTabBytes, &bar.q_full[qb]);
                lq = jj;
            };
            if (x == 0) {
                if (int(blockIdx.x) < n_items) load_q(0, blockIdx.x);
                if (int(blockIdx.x + gridDim.x) < n_items) load_q(1, blockIdx.x + gridDim.x);
            }
            for (int j = 0, idx = blockIdx.x; idx < n_items && ok; ++j, idx += gridDim.x) {
                const int nidx = idx + gridDim.x;
                const int row0 = int(item_ref(idx, P, false).chunk) * kSlices * 80;
                for (int p = 0; p < kPairs; ++p) {
                    // stage st is free once pair g - kStages has been multiplied; the next
                    // completion of its barrier is pair g's, which needs this copy
                    const int g = j * kPairs + p, st = g % kStages, use = g / kStages;
                    if (use >= 1 &&
                        !mbar_wait_sleep(&bar.done_mma[st], (use - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!P.skip_copies) {
                        mbar_expect_tx(&bar.b_full[st], kImgLoadBytes);
                        tma_load_2d(sm + kOffB + st * kImgPairBytes + x * kImgSliceBytes,
                                    P.tm_img, &bar.b_full[st], 0, row0 + 160 * p + 80 * x);
                        issued = g + 1;
                    }
                    if (x == 0 && p == kSlots && j >= 1 && nidx < n_items) {
                        // buffer (j + 1) & 1 is free once the producers finished item j - 1,
                        // which they have by the time this item's first slot is reused
                        if (!mbar_wait_sleep(&bar.q_empty[(j + 1) & 1], ((j - 1) >> 1) & 1,
                                             abort_flag)) {
                            ok = false;
                            break;
                        }
                        load_q(j + 1, nidx);
                    }
                }
            }
            // no copy may still be in flight when the CTA exits
            for (int g = max(0, issued - kStages); g < issued; ++g)
                bounded_spin_done(&bar.b_full[g % kStages], (g / kStages) & 1);
            for (int i = max(0, lq - 1); i <= lq; ++i)
                bounded_spin_done(&bar.q_full[i & 1], (i >> 1) & 1);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace rd
