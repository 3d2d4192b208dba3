// oal_tc_intra_fm.cuh -- the intra-chunk part of the chunked bf16 prefill through the packed
// feature map, for kernels with free coefficients (included by oal_tc.cu inside namespace
// oal::tc).
//
// The ungrouped Hadamard form (abstract of arXiv 2610.13674; eq. (5) of "OAL: 按 QK 离群贡献
// 分组的正二次注意力核", section 核心公式, with free a, b_r, C_rt) has no factored form of few
// score tiles: C may have full rank.  Its kernel is still the packed inner product
//   kappa(q_i, k_j) = sum_f phi_f(q_i) psi_f(k_j),   phi_f = C'_f qhat_r qhat_t,
//   psi_f = khat_r khat_t,
// so for query row i of chunk c
//   U_intra_i = sum_{j in chunk c, j <= i} kappa(q_i, k_j) [v_j; 1]
// is P = Phi(Q_c) Psi(K_c)^T (128 x 128 over the 2176 packed rows), masked causally, then
// P [V_c | 1] -- the readout's phi slices against key-side slices instead of state images.
//
// One CTA per item (b*h, chunk c).  Warps 0-15 (set = warp >> 2, row quarter = warp & 3)
// produce slice s = set (mod 4): phi(Q_c) of the slice into tensor-memory slot `set` and
// psi(K_c) of the slice (bf16 of k_r k_t, one rounding) into shared-memory stage `set`, as
// the K-major B operand.  Warps 16 and 17 issue the even and odd slices' MMAs (A from tensor
// memory) into two accumulators P_A and P_B, so one issues while the other waits.  Warps 0-7
// then form the causal bf16 P tile from P_A + P_B (fixed order) and write the output; warp 16
// issues U = P [V | 1]; warp 18 loads Q, K, V and the head's coefficient table.
// Output as the factored intra-chunk kernel: chunk 0 of a fresh prefill gets yhat, other
// chunks U[:64] in `out` and U[64] in `zin` for the inter-chunk readout to complete.

namespace fm {

constexpr int kMmaA = 16, kMmaB = 17, kLdWarp = 18;
constexpr int kWarps = 19;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0, kOffK = 16384, kOffV = 32768, kOffOnes = 49152;
constexpr uint32_t kOffPsi = 65536;                           // 4 x 16 KB psi stages
constexpr uint32_t kOffPt = kOffPsi;                          // P tile (2 x 16 KB), after all MMAs
constexpr uint32_t kOffTab = kOffPsi + kStages * kTileBytes;  // the head's coefficient table
constexpr uint32_t kOffUnit = kOffTab + kTabBytes;            // unit table: psi = phi with C' = 1
constexpr uint32_t kOffCtl = kOffUnit + kTabBytes;
constexpr uint32_t kSmemBytes = kOffCtl + 1024 + 1024;
static_assert(kOffTab % 1024 == 0 && kOffCtl % 16 == 0 && kSmemBytes <= 232448, "shared memory");

// tensor memory: P_A [0, 128), P_B [128, 256), phi slots [256, 384); U reuses [0, 80) once
// P_A has been read
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColPA = 0, kColPB = 128, kColPhi = 256, kColU = 0;

struct Ctl {
    uint64_t qkv_full, f_full[kStages], e[kStages], p_full, pt_full, u_full, done_a, done_b;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Ctl) <= 1024, "control block");

__global__ void __launch_bounds__(kThreads, 1)
    intra_fm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, Params P, float* __restrict__ zin)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl& ctl = *reinterpret_cast<Ctl*>(sm + kOffCtl);
    volatile int* abort_flag = &ctl.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    P.tm_q = &tm_q;
    P.tm_k = &tm_k;
    P.tm_v = &tm_v;
    const ItemRef it = item_ref(blockIdx.x, P, true);
    const int c = it.c, h = it.h;
    const bool final_out = (c == 0) && !P.cont;

    if (threadIdx.x == 0) {
        mbar_init(&ctl.qkv_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&ctl.f_full[i], 4);
            mbar_init(&ctl.e[i], 1);
        }
        mbar_init(&ctl.p_full, 2);
        mbar_init(&ctl.pt_full, 8);
        mbar_init(&ctl.u_full, 1);
        mbar_init(&ctl.done_a, 1);
        mbar_init(&ctl.done_b, 1);
        ctl.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaA) {
        tmem_alloc(&ctl.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // unit table: bf16 / fp32 ones for every packed row and every block "pure", so that
    // phi_slice of a key row gives psi = bf16(khat_r khat_t)
    for (int i = threadIdx.x; i < int(kTabBytes / 4); i += blockDim.x) {
        const uint32_t off = uint32_t(i) * 4;
        uint32_t w = 0u;
        if (off < kTabCoefT) w = 0x3F803F80u;
        else if (off < kTabCoefT + 384 * 4) w = 0x3F800000u;
        else if (off >= kTabPure && off < kTabPure + 8) w = 0x01010101u;
        reinterpret_cast<uint32_t*>(sm + kOffUnit)[i] = w;
    }
    init_ones_atom(sm + kOffOnes);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    grid_dep_launch();
    if (warp == kLdWarp && lane == 0) {
        mbar_expect_tx(&ctl.qkv_full, 3 * kTileBytes + kTabBytes);
        if (P.nseq) {
            tmap_acquire(it.mq);
            tmap_acquire(it.mk);
            tmap_acquire(it.mv);
        }
        tma_load_3d(sm + kOffQ, it.mq, &ctl.qkv_full, 0, c * kC, it.qz);
        tma_load_3d(sm + kOffK, it.mk, &ctl.qkv_full, 0, c * kC, it.kvz);
        tma_load_3d(sm + kOffV, it.mv, &ctl.qkv_full, 0, c * kC, it.kvz);
        bulk_g2s(sm + kOffTab, P.rtab + size_t(h) * kTabBytes, kTabBytes, &ctl.qkv_full);
    }

    if (warp < kMmaA) {
        // ---- producers: phi(Q_c) slice -> tensor memory, psi(K_c) slice -> shared memory ----
        const int qw = warp & 3, set = warp >> 2, row = qw * 32 + lane;
        const uint32_t lanebase = tmem + (uint32_t(qw * 32) << 16);
        const uint32_t stage = smem_u32(sm + kOffPsi) + set * kTileBytes;
        const unsigned char* qt = sm + kOffQ;
        const unsigned char* kt = sm + kOffK;
        const unsigned char* tab = sm + kOffTab;
        const unsigned char* unit = sm + kOffUnit;
        bool ok = wait_all_sleep(&ctl.qkv_full, 0, abort_flag);
        for (int s = set, use = 0; s < kSlices && ok; s += kStages, ++use) {
            uint32_t w[32];
            rd::phi_slice(qt, tab, s, row, w);
            ok = use == 0 || wait_all(&ctl.e[set], (use - 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            tmem_st32(lanebase + kColPhi + 32 * set, w);
            rd::phi_slice(kt, unit, s, row, w);  // psi of key row `row`
#pragma unroll
            for (int x = 0; x < 8; ++x)
                sts128(stage + kmajor_chunk(row, x), w[4 * x], w[4 * x + 1], w[4 * x + 2],
                       w[4 * x + 3]);
            tmem_st_wait();
            fence_proxy_async();
            tc_fence_before();
            warp_arrive(&ctl.f_full[set]);
        }
        if (warp < 8) {
            // ---- P tile: P_A + P_B over keys [64 kh, 64 kh + 64), masked j <= i, bf16 ------
            const int kh = warp >> 2;
            if (ok) ok = wait_all_sleep(&ctl.p_full, 0, abort_flag);
            if (ok) {
                tc_fence_after();
                const uint32_t pt = smem_u32(sm + kOffPt) + kh * kTileBytes;
#pragma unroll 1
                for (int x = 0; x < 4; ++x) {
                    float pa[16], pb[16];
                    tmem_ld16(lanebase + kColPA + 64 * kh + 16 * x, pa);
                    tmem_ld16(lanebase + kColPB + 64 * kh + 16 * x, pb);
                    tmem_ld_wait();
#pragma unroll
                    for (int hc = 0; hc < 2; ++hc) {
                        uint32_t wv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i0 = 8 * hc + 2 * e, j0 = 64 * kh + 16 * x + i0;
                            const float k0 = (j0 <= row) ? pa[i0] + pb[i0] : 0.f;
                            const float k1 = (j0 + 1 <= row) ? pa[i0 + 1] + pb[i0 + 1] : 0.f;
                            wv[e] = pack_bf16x2(k0, k1);
                        }
                        sts128(pt + kmajor_chunk(row, 2 * x + hc), wv[0], wv[1], wv[2], wv[3]);
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                warp_arrive(&ctl.pt_full);
                ok = wait_all_sleep(&ctl.u_full, 0, abort_flag);
            }
            if (ok) {
                // epilogue: columns [32 kh, 32 kh + 32) of U (and the normaliser U[64])
                tc_fence_after();
                float u[32];
                tmem_ld16(lanebase + kColU + 32 * kh, *reinterpret_cast<float(*)[16]>(&u[0]));
                tmem_ld16(lanebase + kColU + 32 * kh + 16, *reinterpret_cast<float(*)[16]>(&u[16]));
                const float z = tmem_ld1(lanebase + kColU + 64);
                tmem_ld_wait();
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
            }
        }
    } else if (warp == kMmaA || warp == kMmaB) {
        // ---- MMA issuers: P_A (even slices) / P_B (odd slices) += phi_s psi_s^T ------------
        const bool isA = warp == kMmaA;
        constexpr uint32_t id_p = idesc_bf16(128, 128, false, false);  // A (TMEM), B K-major
        constexpr uint32_t id_pv = idesc_bf16(128, 80, false, true);   // B = [V | ones] MN
        const uint32_t psi0 = smem_u32(sm + kOffPsi);
        const uint32_t pcol = tmem + (isA ? kColPA : kColPB);
        bool ok = true;
        for (int s = isA ? 0 : 1; s < kSlices && ok; s += 2) {
            const int slot = s % kStages, use = s / kStages;
            ok = wait_all(&ctl.f_full[slot], use & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(pcol, tmem + kColPhi + 32 * slot + 8 * ks,
                                sdesc_sw128(psi0 + slot * kTileBytes + 32 * ks, 16, 1024), id_p,
                                (s > 1 || ks > 0) ? 1u : 0u);
                mma_commit(&ctl.e[slot]);
            }
            __syncwarp();
        }
        if (ok) {
            if (elect_one()) mma_commit(&ctl.p_full);
            __syncwarp();
        }
        if (isA && ok) {
            ok = wait_all(&ctl.pt_full, 0, abort_flag);
            if (ok) {
                tc_fence_after();
                const uint32_t pt = smem_u32(sm + kOffPt), vt = smem_u32(sm + kOffV);
                const uint32_t ones = smem_u32(sm + kOffOnes);
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tmem + kColU,
                                 sdesc_sw128(pt + (ks >> 2) * kTileBytes + (ks & 3) * 32, 16, 1024),
                                 sdesc_sw128(vt + ks * 2048, ones - vt, 1024), id_pv,
                                 ks > 0 ? 1u : 0u);
                    mma_commit(&ctl.u_full);
                }
                __syncwarp();
            }
        }
        // every MMA of this issuer has completed before tensor memory is freed
        uint64_t* done = isA ? &ctl.done_a : &ctl.done_b;
        if (elect_one()) mma_commit(done);
        __syncwarp();
        if (lane == 0) bounded_spin_done(done, 0);
        __syncwarp();
    } else if (warp == kLdWarp && lane == 0) {
        bounded_spin_done(&ctl.qkv_full, 0);  // no copy in flight at exit
    }

    // launched as a dependent of the scan without reading its outputs: complete only after it
    grid_dep_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace fm
