// oal_tc_intra.cuh -- the intra-chunk part of the chunked bf16 prefill on tensor cores
// (included by oal_tc.cu inside namespace oal::tc).
//
// "OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式: for query row i of chunk c,
//   U_intra_i = sum_{j in chunk c, j <= i} kappa(q_i, k_j) [v_j; 1]          (eqs. (2)-(3))
// with kappa in the factored form kappa = eps + sum_m (L_0m + (q o w_m) . k)^2,
// w_m[r] = L_{g(r),m} / sqrt(d_h), which equals eps + ||L^T sbar||^2 = eq. (3).
//
// One CTA per item (b*h, chunk c), two CTAs per SM so that one CTA's tensor work fills the
// other's latency chain.  Warps 0-7 (row quarter qw = warp & 3, key half kh = warp >> 2):
// Aq_m = Q o w_m tiles (dims [32 kh, 32 kh + 32)), kappa over keys [64 kh, 64 kh + 64) of each
// score tile S_m = Aq_m K^T (tensor memory, two buffers: tile m + 1 is computed while tile m is
// read), the causal P tile, and the epilogue.  Warp 8 issues the MMAs (S_m, then
// U = P [V | 1]); warp 9 loads Q, K, V.
// Output: a chunk without an inter-chunk part (chunk 0 of a fresh prefill) is complete, so
// yhat = U[:64] / U[64] goes to `out`; otherwise U[:64] goes to `out` and U[64] to `zin`, and
// the inter-chunk readout adds phi(q) S_c before normalising.

namespace intra {

constexpr int kWarps = 10;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp = 8, kLdWarp = 9;
constexpr uint32_t kTmemCols = 256;
// score tiles S_m alternate between [0, 128) and [128, 256), so tile m + 1 is computed while
// tile m is read; U = P [V | 1] reuses [0, 80) once every tile has been read
constexpr uint32_t kColS = 0, kColU = 0;

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kOffK = 0, kOffV = 16384, kOffQ = 32768, kOffAq = 49152, kOffOnes = 81920;
constexpr uint32_t kOffW = 98304;                   // fp32 [9][64] score weights
constexpr uint32_t kOffC0 = kOffW + kGM1 * 64 * 4;  // fp32 [9] L_0m
constexpr uint32_t kOffCtl = kOffC0 + 64;
constexpr uint32_t kSmemBytes = kOffCtl + 512 + 1024;
static_assert(kOffCtl % 8 == 0 && 2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");

struct Ctl {
    uint64_t qkv_full, aq_full[2], s_full[2], s_empty[2], p_full, u_full, done;
    uint32_t tmem_base;
    int abort_flag;
    int G;
};

__global__ void __launch_bounds__(kThreads, 2)
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

    P.tm_q = &tm_q;
    P.tm_k = &tm_k;
    P.tm_v = &tm_v;
    const ItemRef it = item_ref(blockIdx.x, P, true);
    const int c = it.c, h = it.h;
    const bool final_out = (c == 0) && !P.cont;

    if (threadIdx.x == 0) {
        mbar_init(&ctl.qkv_full, 1);
        mbar_init(&ctl.aq_full[0], 8);
        mbar_init(&ctl.aq_full[1], 8);
        mbar_init(&ctl.s_full[0], 1);
        mbar_init(&ctl.s_full[1], 1);
        mbar_init(&ctl.s_empty[0], 8);
        mbar_init(&ctl.s_empty[1], 8);
        mbar_init(&ctl.p_full, 8);
        mbar_init(&ctl.u_full, 1);
        mbar_init(&ctl.done, 1);
        ctl.abort_flag = 0;
        int Gh = P.G[h];
        if (Gh < 1 || Gh > kGMax) {
            raise_error(OAL_ERR_GROUPS);
            Gh = Gh < 1 ? 1 : kGMax;
        }
        ctl.G = Gh;
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
    const int G = ctl.G;
    grid_dep_launch();  // the next kernel of the prefill may start its prologue
    if (warp == kLdWarp && lane == 0) {
        mbar_expect_tx(&ctl.qkv_full, 3 * kTileBytes);
        if (P.nseq) {
            tmap_acquire(it.mq);
            tmap_acquire(it.mk);
            tmap_acquire(it.mv);
        }
        tma_load_3d(sm + kOffQ, it.mq, &ctl.qkv_full, 0, c * kC, it.qz);
        tma_load_3d(sm + kOffK, it.mk, &ctl.qkv_full, 0, c * kC, it.kvz);
        tma_load_3d(sm + kOffV, it.mv, &ctl.qkv_full, 0, c * kC, it.kvz);
    }
    // score weights w_m[r] = L_{g(r),m} / sqrt(d_h) (0 for m > G) and L_0m
    for (int e = threadIdx.x; e < kGM1 * 64; e += blockDim.x) {
        const int m = e >> 6, r = e & 63;
        int g = P.gid[h * kD + r];
        if (g < 1 || g > G) {
            raise_error(OAL_ERR_GROUPS);
            g = g < 1 ? 1 : G;
        }
        wch[e] = (m <= G) ? P.L[size_t(h) * kGM1 * kGM1 + g * kGM1 + m] * 0.125f : 0.f;
    }
    if (threadIdx.x < kGM1)
        c0[threadIdx.x] = threadIdx.x <= G ? P.L[size_t(h) * kGM1 * kGM1 + threadIdx.x] : 0.f;
    __syncthreads();

    if (warp < 8) {
        const int qw = warp & 3, kh = warp >> 2, row = qw * 32 + lane;
        const uint32_t lanebase = tmem + (uint32_t(qw * 32) << 16);
        const uint32_t aq0 = smem_u32(sm + kOffAq);
        const unsigned char* qt = sm + kOffQ;
        bool ok = wait_all_sleep(&ctl.qkv_full, 0, abort_flag);
        // Aq_m = Q o w_m (bf16, K-major); this warp writes dims [32 kh, 32 kh + 32)
        auto produce_aq = [&](int m) {
            const uint32_t base = aq0 + (m & 1) * kTileBytes;
            const float* w = wch + m * 64;
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
            warp_arrive(&ctl.aq_full[m & 1]);
        };
        if (ok) {
            produce_aq(0);
            if (G >= 1) produce_aq(1);
        }
        const bool live = 64 * kh <= 32 * qw + 31;  // some key of this half <= some row
        float acc[64];
#pragma unroll
        for (int x = 0; x < 64; ++x) acc[x] = 0.f;
        for (int m = 0; m <= G && ok; ++m) {
            ok = wait_all_sleep(&ctl.s_full[m & 1], (m >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            if (live) {
                const float cm = c0[m];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    float v[16];
                    tmem_ld16(lanebase + kColS + (m & 1) * 128 + 64 * kh + 16 * x, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const float2 t = __fadd2_rn(f2(cm, cm), f2(v[i], v[i + 1]));
                        const float2 a = __ffma2_rn(t, t, f2(acc[16 * x + i], acc[16 * x + i + 1]));
                        acc[16 * x + i] = a.x;
                        acc[16 * x + i + 1] = a.y;
                    }
                }
            }
            tc_fence_before();
            warp_arrive(&ctl.s_empty[m & 1]);
            if (m + 2 <= G) produce_aq(m + 2);  // S_m completed: its Aq buffer is free
        }
        if (ok) {
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
    } else if (warp == kMmaWarp) {
        constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_pv = idesc_bf16(128, 80, false, true);  // B = [V | ones] MN
        const uint32_t aq0 = smem_u32(sm + kOffAq), kt = smem_u32(sm + kOffK);
        const uint32_t vt = smem_u32(sm + kOffV), ones = smem_u32(sm + kOffOnes);
        bool ok = wait_all(&ctl.qkv_full, 0, abort_flag);
        for (int m = 0; m <= G && ok; ++m) {
            // tile buffer m & 1 is free once tile m - 2 has been read (the next completion of
            // that barrier is tile m's read, after this MMA)
            ok = wait_all(&ctl.aq_full[m & 1], (m >> 1) & 1, abort_flag);
            if (ok && m >= 2) ok = wait_all(&ctl.s_empty[m & 1], ((m - 2) >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + kColS + (m & 1) * 128,
                             sdesc_sw128(aq0 + (m & 1) * kTileBytes + ks * 32, 16, 1024),
                             sdesc_sw128(kt + ks * 32, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                mma_commit(&ctl.s_full[m & 1]);
            }
            __syncwarp();
        }
        if (ok) ok = wait_all(&ctl.p_full, 0, abort_flag);
        if (ok) {
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
        }
        // every MMA of this CTA has completed before tensor memory is freed
        if (elect_one()) mma_commit(&ctl.done);
        __syncwarp();
        if (lane == 0) bounded_spin_done(&ctl.done, 0);
        __syncwarp();
    } else if (warp == kLdWarp && lane == 0) {
        bounded_spin_done(&ctl.qkv_full, 0);  // no copy in flight at exit
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
