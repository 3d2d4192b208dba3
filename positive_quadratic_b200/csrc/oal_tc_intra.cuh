// oal_tc_intra.cuh -- the intra-chunk part of the chunked bf16 prefill on tensor cores
// (included by oal_tc.cu inside namespace oal::tc).
//
// "OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式: for query row i of chunk c,
//   U_intra_i = sum_{j in chunk c, j <= i} kappa(q_i, k_j) [v_j; 1]          (eqs. (2)-(3))
// with kappa in the factored form kappa = eps + sum_m (L_0m + (q o w_m) . k)^2,
// w_m[r] = L_{g(r),m} / sqrt(d_h), which equals eps + ||L^T sbar||^2 = eq. (3).
//
// Persistent: two CTAs per SM, each walking the items (b*h, chunk c) blockIdx.x,
// blockIdx.x + gridDim.x, ...  so that one CTA's tensor work fills the other's latency chain
// and the set-up (barriers, tensor memory, the ones atom) is paid once per CTA.
// Warps 0-7 (row quarter qw = warp & 3, key half kh = warp >> 2): Aq_m = Q o w_m tiles (dims
// [32 kh, 32 kh + 32)), kappa over keys [64 kh, 64 kh + 64) of each score tile S_m = Aq_m K^T
// (tensor memory, two buffers: tile t + 1 is computed while tile t is read; t counts tiles over
// the CTA's items), the causal P tile, and the epilogue.  Warp 8 issues the MMAs (S_m, then
// U = P [V | 1]).  Warp 9 forms the next item's score weights and loads its Q and K as soon
// as every score MMA of the current item has completed (both are then free) and its V as
// soon as U has (the next item's first tiles then start without waiting for memory).
// Output: a chunk without an inter-chunk part (chunk 0 of a fresh prefill) is complete, so
// yhat = U[:64] / U[64] goes to `out`; otherwise U[:64] goes to `out` and U[64] to `zin`, and
// the inter-chunk readout adds phi(q) S_c before normalising.

namespace intra {

constexpr int kWarps = 10;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp = 8, kLdWarp = 9;
constexpr int kCtasPerSm = 2;
constexpr uint32_t kTmemCols = 256;
// score tiles alternate between [0, 128) and [128, 256) (tile t in buffer t & 1); U = P [V | 1]
// reuses [0, 80) once every tile of the item has been read, and the next item's first score
// MMAs wait for Aq tiles that the kappa warps write only after they have read U
constexpr uint32_t kColS = 0, kColU = 0;

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kOffK = 0, kOffV = 16384, kOffQ = 32768, kOffAq = 49152, kOffOnes = 81920;
constexpr uint32_t kOffW = 98304;                        // fp32 [2][9][64] score weights
constexpr uint32_t kOffC0 = kOffW + 2 * kGM1 * 64 * 4;   // fp32 [2][16] L_0m
constexpr uint32_t kOffLs = kOffC0 + 2 * 16 * 4;         // fp32 [96] L of the next item's head
constexpr uint32_t kOffCtl = kOffLs + 96 * 4;
constexpr uint32_t kSmemBytes = kOffCtl + 512 + 1024;
static_assert(kOffCtl % 8 == 0 && kCtasPerSm * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");

struct Ctl {
    uint64_t qk_full, v_full, w_full[2], aq_full[2], s_full[2], s_empty[2], p_full, u_full, done;
    uint64_t k_free;  // the item's score MMAs (the last readers of Q and K) have completed
    uint32_t tmem_base;
    int abort_flag;
    int G[2];  // groups of the items with parity 0 / 1
};
static_assert(sizeof(Ctl) <= 512, "control block");

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, Params P, float* __restrict__ zin)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl& ctl = *reinterpret_cast<Ctl*>(sm + kOffCtl);
    volatile int* abort_flag = &ctl.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* wch = reinterpret_cast<float*>(sm + kOffW);
    float* c0 = reinterpret_cast<float*>(sm + kOffC0);
    const int n_items = P.n_intra;

    P.tm_q = &tm_q;
    P.tm_k = &tm_k;
    P.tm_v = &tm_v;

    if (threadIdx.x == 0) {
        mbar_init(&ctl.qk_full, 1);
        mbar_init(&ctl.v_full, 1);
        mbar_init(&ctl.w_full[0], 1);
        mbar_init(&ctl.w_full[1], 1);
        mbar_init(&ctl.aq_full[0], 8);
        mbar_init(&ctl.aq_full[1], 8);
        mbar_init(&ctl.s_full[0], 1);
        mbar_init(&ctl.s_full[1], 1);
        mbar_init(&ctl.s_empty[0], 8);
        mbar_init(&ctl.s_empty[1], 8);
        mbar_init(&ctl.p_full, 8);
        mbar_init(&ctl.u_full, 1);
        mbar_init(&ctl.done, 1);
        mbar_init(&ctl.k_free, 1);
        ctl.abort_flag = 0;
        fence_mbar_init();
    }
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
    grid_dep_launch();  // the next kernel of the prefill may start its prologue

    if (warp < 8) {
        const int qw = warp & 3, kh = warp >> 2, row = qw * 32 + lane;
        const uint32_t lanebase = tmem + (uint32_t(qw * 32) << 16);
        const uint32_t aq0 = smem_u32(sm + kOffAq);
        const unsigned char* qt = sm + kOffQ;
        const bool live = 64 * kh <= 32 * qw + 31;  // some key of this half <= some row
        // Aq of tile t = Q o w_m into buffer t & 1 (bf16, K-major); this warp writes dims
        // [32 kh, 32 kh + 32)
        auto produce_aq = [&](int t, const float* w) {
            const uint32_t base = aq0 + (t & 1) * kTileBytes;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int ch = 4 * kh + x;
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
            warp_arrive(&ctl.aq_full[t & 1]);
        };
        bool ok = true;
        for (int j = 0, tb = 0; int(blockIdx.x + j * gridDim.x) < n_items && ok; ++j) {
            ok = wait_all_sleep(&ctl.w_full[j & 1], (j >> 1) & 1, abort_flag) &&
                 wait_all_sleep(&ctl.qk_full, j & 1, abort_flag);
            if (!ok) break;
            const int G = ctl.G[j & 1];
            const float* wj = wch + (j & 1) * kGM1 * 64;
            // the previous item's P tile (over both Aq buffers) has been multiplied and its U
            // read: both buffers are free
            produce_aq(tb, wj);
            if (G >= 1) produce_aq(tb + 1, wj + 64);
            float acc[64];
#pragma unroll
            for (int x = 0; x < 64; ++x) acc[x] = 0.f;
            for (int m = 0; m <= G; ++m) {
                const int t = tb + m;
                ok = wait_all_sleep(&ctl.s_full[t & 1], (t >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (live) {
                    const float cm = c0[(j & 1) * 16 + m];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        float v[16];
                        tmem_ld16(lanebase + kColS + (t & 1) * 128 + 64 * kh + 16 * x, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const float2 tv = __fadd2_rn(f2(cm, cm), f2(v[i], v[i + 1]));
                            const float2 a =
                                __ffma2_rn(tv, tv, f2(acc[16 * x + i], acc[16 * x + i + 1]));
                            acc[16 * x + i] = a.x;
                            acc[16 * x + i + 1] = a.y;
                        }
                    }
                }
                tc_fence_before();
                warp_arrive(&ctl.s_empty[t & 1]);
                // S_t completed: its Aq buffer is free
                if (m + 2 <= G) produce_aq(t + 2, wj + 64 * (m + 2));
            }
            if (!ok) break;
            // P tile (K-major, atom kh = keys [64 kh, 64 kh + 64); aliases Aq0 | Aq1, free once
            // the last score tile completed)
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                uint32_t wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j0 = 64 * kh + 8 * x + 2 * e;
                    const float k0 = (j0 <= row) ? P.eps + acc[8 * x + 2 * e] : 0.f;
                    const float k1 = (j0 + 1 <= row) ? P.eps + acc[8 * x + 2 * e + 1] : 0.f;
                    wv[e] = pack_bf16x2(k0, k1);
                }
                sts128(aq0 + kh * kTileBytes + kmajor_chunk(row, x), wv[0], wv[1], wv[2], wv[3]);
            }
            fence_proxy_async();
            warp_arrive(&ctl.p_full);
            ok = wait_all_sleep(&ctl.u_full, j & 1, abort_flag);
            if (!ok) break;
            // epilogue: columns [32 kh, 32 kh + 32) of U (and the normaliser U[64])
            const ItemRef it = item_ref(blockIdx.x + j * gridDim.x, P, true);
            const int c = it.c;
            const bool final_out = (c == 0) && !P.cont;
            tc_fence_after();
            float u[32];
            tmem_ld16(lanebase + kColU + 32 * kh, *reinterpret_cast<float(*)[16]>(&u[0]));
            tmem_ld16(lanebase + kColU + 32 * kh + 16, *reinterpret_cast<float(*)[16]>(&u[16]));
            const float z = tmem_ld1(lanebase + kColU + 64);
            tmem_ld_wait();
            tc_fence_before();  // U is read before this warp's next Aq arrival
            const int irow = c * kC + row;
            if (irow < it.T) {
                float4* o = reinterpret_cast<float4*>(P.out + (it.orow + irow) * kDV + 32 * kh);
                const float inv = final_out ? 1.f / z : 1.f;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    o[i] = make_float4(u[4 * i] * inv, u[4 * i + 1] * inv, u[4 * i + 2] * inv,
                                       u[4 * i + 3] * inv);
                if (!final_out && kh == 0) zin[it.orow + irow] = z;
            }
            tb += G + 1;
        }
    } else if (warp == kMmaWarp) {
        constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_pv = idesc_bf16(128, 80, false, true);  // B = [V | ones] MN
        const uint32_t aq0 = smem_u32(sm + kOffAq), kt = smem_u32(sm + kOffK);
        const uint32_t vt = smem_u32(sm + kOffV), ones = smem_u32(sm + kOffOnes);
        bool ok = true;
        for (int j = 0, idx = blockIdx.x, tb = 0; idx < n_items && ok; ++j, idx += gridDim.x) {
            ok = wait_all(&ctl.w_full[j & 1], (j >> 1) & 1, abort_flag) &&
                 wait_all(&ctl.qk_full, j & 1, abort_flag);
            if (!ok) break;
            const int G = ctl.G[j & 1];
            for (int m = 0; m <= G && ok; ++m) {
                // buffer t & 1 is free once tile t - 2 has been read (the next completion of
                // that barrier is tile t's read, after this MMA)
                const int t = tb + m;
                ok = wait_all(&ctl.aq_full[t & 1], (t >> 1) & 1, abort_flag);
                if (ok && t >= 2) ok = wait_all(&ctl.s_empty[t & 1], ((t - 2) >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + kColS + (t & 1) * 128,
                                 sdesc_sw128(aq0 + (t & 1) * kTileBytes + ks * 32, 16, 1024),
                                 sdesc_sw128(kt + ks * 32, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                    mma_commit(&ctl.s_full[t & 1]);
                }
                __syncwarp();
            }
            if (!ok) break;
            // one completion per item, after every score MMA of it (and so after every read of
            // its Q and K): the loader may then overwrite them
            if (elect_one()) mma_commit(&ctl.k_free);
            __syncwarp();
            ok = wait_all(&ctl.p_full, j & 1, abort_flag) &&
                         wait_all(&ctl.v_full, j & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + kColU,
                             sdesc_sw128(aq0 + (ks >> 2) * kTileBytes + (ks & 3) * 32, 16, 1024),
                             sdesc_sw128(vt + ks * 2048, ones - vt, 1024), id_pv, ks > 0 ? 1u : 0u);
                mma_commit(&ctl.u_full);
            }
            __syncwarp();
            tb += G + 1;
        }
        // every MMA of this CTA has completed before tensor memory is freed
        if (elect_one()) mma_commit(&ctl.done);
        __syncwarp();
        if (lane == 0) bounded_spin_done(&ctl.done, 0);
        __syncwarp();
    } else if (warp == kLdWarp) {
        float* Ls = reinterpret_cast<float*>(sm + kOffLs);
        // score weights of item j (buffer j & 1): w_m[r] = L_{g(r),m} / sqrt(d_h) (0 for m > G)
        // and L_0m, formed by the whole warp; lane 0 then publishes them
        auto weights = [&](int j, const ItemRef& x) {
            const int h = x.h;
            int Gh = P.G[h];
            const int g0 = P.gid[h * kD + lane], g1 = P.gid[h * kD + 32 + lane];
            const float* Lh = P.L + size_t(h) * kGM1 * kGM1;
            const float l0 = Lh[lane], l1 = Lh[32 + lane], l2 = lane < 17 ? Lh[64 + lane] : 0.f;
            if (Gh < 1 || Gh > kGMax) {
                if (lane == 0) raise_error(OAL_ERR_GROUPS);
                Gh = Gh < 1 ? 1 : kGMax;
            }
            Ls[lane] = l0;
            Ls[32 + lane] = l1;
            if (lane < 17) Ls[64 + lane] = l2;
            __syncwarp();
            float* w = wch + (j & 1) * kGM1 * 64;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                int g = half ? g1 : g0;
                if (g < 1 || g > Gh) {
                    raise_error(OAL_ERR_GROUPS);
                    g = g < 1 ? 1 : Gh;
                }
#pragma unroll
                for (int m = 0; m < kGM1; ++m)
                    w[m * 64 + 32 * half + lane] = m <= Gh ? Ls[g * kGM1 + m] * 0.125f : 0.f;
            }
            if (lane < 16) c0[(j & 1) * 16 + lane] = lane <= Gh ? Ls[lane] : 0.f;
            if (lane == 0) ctl.G[j & 1] = Gh;
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.w_full[j & 1]);
            __syncwarp();
        };
        auto load_qk = [&](const ItemRef& x) {
            mbar_expect_tx(&ctl.qk_full, 2 * kTileBytes);
            if (P.nseq) {
                tmap_acquire(x.mq);
                tmap_acquire(x.mk);
            }
            tma_load_3d(sm + kOffQ, x.mq, &ctl.qk_full, 0, x.c * kC, x.qz);
            tma_load_3d(sm + kOffK, x.mk, &ctl.qk_full, 0, x.c * kC, x.kvz);
        };
        auto load_v = [&](const ItemRef& x) {
            mbar_expect_tx(&ctl.v_full, kTileBytes);
            if (P.nseq) tmap_acquire(x.mv);
            tma_load_3d(sm + kOffV, x.mv, &ctl.v_full, 0, x.c * kC, x.kvz);
        };
        int n_qk = 0, n_v = 0;  // loads issued (counted by lane 0, which issues them)
        bool ok = true;
        if (int(blockIdx.x) < n_items) {
            const ItemRef x = item_ref(blockIdx.x, P, true);
            if (lane == 0) {
                load_qk(x);
                load_v(x);
            }
            n_qk = n_v = 1;
            weights(0, x);
        }
        for (int j = 0, idx = blockIdx.x; idx < n_items && ok; ++j, idx += gridDim.x) {
            const int nidx = idx + gridDim.x;
            if (nidx < n_items) {
                const ItemRef x = item_ref(nidx, P, true);
                // buffer (j + 1) & 1 was item j - 1's, whose U (after its last use of the
                // weights) this warp waited for in the previous iteration
                weights(j + 1, x);
                if (lane == 0) {
                    // one completion of each barrier per item, waited in order, so a parity
                    // wait here is never two phases behind
                    ok = mbar_wait_sleep(&ctl.k_free, j & 1, abort_flag);
                    if (ok) {
                        load_qk(x);
                        ++n_qk;
                        ok = mbar_wait_sleep(&ctl.u_full, j & 1, abort_flag);  // V is free
                    }
                    if (ok) {
                        load_v(x);
                        ++n_v;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            }
        }
        // no copy may still be in flight at exit (every issued load completes its barrier)
        if (lane == 0) {
            if (n_qk) bounded_spin_done(&ctl.qk_full, (n_qk - 1) & 1);
            if (n_v) bounded_spin_done(&ctl.v_full, (n_v - 1) & 1);
        }
        __syncwarp();
    }

    // launched as a dependent of the scan without reading its outputs: complete only after it
    grid_dep_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace intra
