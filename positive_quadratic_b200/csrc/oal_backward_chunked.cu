// oal_backward_chunked.cu -- training-scale gradients: the chunked reverse of the prefill, on
// CUDA cores in fp32.
//
// "OAL: 按 QK 离群贡献分组的正二次注意力核" trains the kernel coefficients jointly with the
// model (its pipeline figure); the pages print no gradient.  With the packed feature map of
// section 核心公式 (phi_f(q) = C'_f qhat_r qhat_t, psi_f(k) = khat_r khat_t, kappa_ij =
// phi(q_i) . psi(k_j), eqs. (3)-(5)), u_i = sum_{j<=i} kappa_ij w_j with w_j = [v_j; 1] and
// yhat_i = u_i[:64] / u_i[64] = u_i[:64] / D_i, the chain rule for dLoss/dyhat = dy gives
//   g_i := dLoss/du_i = [dy_i / D_i ; -(dy_i . yhat_i) / D_i],   dkappa_ij = g_i . w_j.
// Split at the chunk of 64 tokens that holds the row (key), every sum over pairs is a
// within-chunk part plus a part through chunk states:
//   dphi(q_i)  = sum_{j < c0} dkappa_ij psi_j = S_c g_i               S_c = sum_{j<c0} psi_j w_j^T
//   dpsi(k_j)  = sum_{i >= c1} dkappa_ij phi_i = R_c w_j              R_c = sum_{i>=c1} phi_i g_i^T
//   dw_j      += sum_{i >= c1} kappa_ij g_i = R_c^T psi_j
//   dC'_f      = sum_i dphi_f(q_i) qhat_r qhat_t
// (c0 / c1: first token of the row's / one past the key's chunk; R_c sums the query heads of
// the kv group).  dq, dk follow from dphi, dpsi through the products qhat_r qhat_t and
// khat_r khat_t; dC' goes to dM (C'_f = (2 - [r = t]) M_{g(r)g(t)} s_r s_t, plus eps on the
// constant row) and dL = (dM + dM^T) L as in the dense form.  The within-chunk parts are the
// dense form's pair terms restricted to the chunk, with D_i and yhat_i of the whole sequence.
// Passes, each thread owning what it writes (deterministic):
//   forward  : coefficients, exclusive prefix states S_c (fp32), yhat and D for every row;
//   g        : the upstream gradient rows g_i;
//   intra    : rows (dq, the row's dM and deps) and keys (dk, dv) over within-chunk pairs;
//   suffix   : R_c for every chunk (each chunk's sum, chunk-parallel, then a reverse exclusive
//              scan over chunks);
//   inter    : rows add S_c g_i through phi to dq and leave per-(head, chunk) partial dC';
//              keys add R_c w_j through psi to dk and R_c^T psi_j to dv;
//   heads    : dM from the row partials and dC', dL, deps.
// Work is O(B Hq T (64 (d_h + G^2) + 2176 * 65)): linear in T.
#pragma once

#include <algorithm>

#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

constexpr int kCbC = 64;  // chunk (and tile) of the chunked backward

struct CbArgs {
    int B, T, Hq, Hkv, NC;
    float eps;
    const int32_t* gid;
    const float* L;
    const int32_t* G;
    const float* dy;      // [B][Hq][T][64]
    float* dq;            // [B][Hq][T][64]
    float* dk;            // [B][Hkv][T][64]
    float* dv;            // [B][Hkv][T][64]
    float* dL;            // [Hq][9][9]
    float* deps;          // [1]
    unsigned char* st;    // scratch state: header, coefficients C' [Hq][2176], final state
    float* Hc;            // [B*Hkv][NC][65][2176] exclusive prefix states S_c
    float* R;             // [B*Hkv][NC][65][2176] exclusive suffix states R_c
    float* rowD;          // [B][Hq][T]
    float* rowY;          // [B][Hq][T][64]
    float* Gr;            // [B][Hq][T][65]
    float* dcp;           // [B*Hq][NC][2176] partial dC'
    float* rowM;          // [B][Hq][T][81]
    float* rowE;          // [B][Hq][T]
    float* headE;         // [Hq]
};

__host__ __device__ __forceinline__ const float* cb_coef(const CbArgs& A)
{
    return reinterpret_cast<const float*>(A.st + kHeaderBytes);
}

// g_i = [dy_i / D_i ; -(dy_i . yhat_i) / D_i]; one warp per row
__global__ void __launch_bounds__(256) cb_g_kernel(CbArgs A)
{
    const size_t rows = size_t(A.B) * A.Hq * A.T;
    const size_t row = size_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* d = A.dy + row * kDV;
    const float* y = A.rowY + row * kDV;
    const float inv = 1.f / A.rowD[row];
    float s = d[lane] * y[lane] + d[lane + 32] * y[lane + 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    float* g = A.Gr + row * kW;
    g[lane] = d[lane] * inv;
    g[lane + 32] = d[lane + 32] * inv;
    if (lane == 0) g[kDV] = -s * inv;
}

// Within-chunk pairs, rows: thread = row i, keys j in [c0, i].  Writes dq (the inter pass adds
// to it), the row's dM and deps.
template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads) cb_intra_rows_kernel(const Tin* __restrict__ q,
                                                                    const Tin* __restrict__ k,
                                                                    const Tin* __restrict__ v,
                                                                    CbArgs A)
{
    const int bh = blockIdx.y, b = bh / A.Hq, h = bh % A.Hq, kv = h / (A.Hq / A.Hkv);
    const int i = blockIdx.x * kBwdThreads + threadIdx.x;
    __shared__ float m[kMM];
    __shared__ int g[kD];
    __shared__ int sG;
    if (threadIdx.x == 0) {
        BwdArgs B0{};
        B0.G = A.G;
        B0.gid = A.gid;
        B0.L = A.L;
        sG = bwd_head_setup(B0, h, m, g);
    }
    __syncthreads();
    if (i >= A.T) return;
    const int Gh = sG;
    const size_t row = size_t(bh) * A.T + i;
    const Tin* qi = q + row * kD;
    const Tin* kb = k + size_t(b * A.Hkv + kv) * A.T * kD;
    const Tin* vb = v + size_t(b * A.Hkv + kv) * A.T * kDV;
    const float* gi = A.Gr + row * kW;
    float sb[kGM1], ms[kGM1], dqr[kD], dM[kMM];
    for (int r = 0; r < kD; ++r) dqr[r] = 0.f;
    for (int e = 0; e < kMM; ++e) dM[e] = 0.f;
    float de = 0.f;
    for (int j = (i / kCbC) * kCbC; j <= i; ++j) {
        const Tin* kj = kb + size_t(j) * kD;
        bwd_kappa(qi, kj, g, m, Gh, A.eps, sb, ms);
        float dk_ = gi[kDV];
        for (int n = 0; n < kDV; ++n) dk_ = fmaf(gi[n], to_f32(vb[size_t(j) * kDV + n]), dk_);
        for (int r = 0; r < kD; ++r) dqr[r] = fmaf(dk_ * 2.f * ms[g[r]] * 0.125f, to_f32(kj[r]), dqr[r]);
        for (int c = 0; c <= Gh; ++c)
            for (int e = 0; e <= Gh; ++e) dM[c * kGM1 + e] = fmaf(dk_ * sb[c], sb[e], dM[c * kGM1 + e]);
        de += dk_;
    }
    for (int r = 0; r < kD; ++r) A.dq[row * kD + r] = dqr[r];
    for (int e = 0; e < kMM; ++e) A.rowM[row * kMM + e] = dM[e];
    A.rowE[row] = de;
}

// Within-chunk pairs, keys: thread = (key j, query head x of the group), rows i in [j, end of
// j's chunk); the eight lanes of a key (x = lane & 7, heads past the group's contribute zero)
// add their dk and dv with a fixed butterfly.  Writes dk and dv (the inter pass adds to them).
constexpr int kKeysPerBlock = 16;
template <typename Tin>
__global__ void __launch_bounds__(8 * kKeysPerBlock) cb_intra_keys_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v, CbArgs A)
{
    const int bkv = blockIdx.y, b = bkv / A.Hkv, kv = bkv % A.Hkv, grp = A.Hq / A.Hkv;
    const int x = threadIdx.x & 7, j = blockIdx.x * kKeysPerBlock + (threadIdx.x >> 3);
    __shared__ float m[kMaxGroup][kMM];
    __shared__ int g[kMaxGroup][kD];
    __shared__ int sG[kMaxGroup];
    if (threadIdx.x < grp) {
        BwdArgs B0{};
        B0.G = A.G;
        B0.gid = A.gid;
        B0.L = A.L;
        sG[threadIdx.x] = bwd_head_setup(B0, kv * grp + threadIdx.x, m[threadIdx.x],
                                         g[threadIdx.x]);
    }
    __syncthreads();
    float dkr[kD], dvr[kDV], sb[kGM1], ms[kGM1];
    for (int r = 0; r < kD; ++r) dkr[r] = 0.f;
    for (int n = 0; n < kDV; ++n) dvr[n] = 0.f;
    if (j < A.T && x < grp) {
        const Tin* kj = k + (size_t(bkv) * A.T + j) * kD;
        const Tin* vj = v + (size_t(bkv) * A.T + j) * kDV;
        const int iend = min(A.T, (j / kCbC + 1) * kCbC);
        const int h = kv * grp + x, bh = b * A.Hq + h;
        for (int i = j; i < iend; ++i) {
            const size_t row = size_t(bh) * A.T + i;
            const Tin* qi = q + row * kD;
            const float kap = bwd_kappa(qi, kj, g[x], m[x], sG[x], A.eps, sb, ms);
            const float* gi = A.Gr + row * kW;
            float dk_ = gi[kDV];
            for (int n = 0; n < kDV; ++n) {
                dk_ = fmaf(gi[n], to_f32(vj[n]), dk_);
                dvr[n] = fmaf(kap, gi[n], dvr[n]);
            }
            for (int r = 0; r < kD; ++r)
                dkr[r] = fmaf(dk_ * 2.f * ms[g[x][r]] * 0.125f, to_f32(qi[r]), dkr[r]);
        }
    }
    // sum over the group's heads: lanes x, x ^ 4, x ^ 2, x ^ 1 of the key, a fixed order
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
#pragma unroll
        for (int r = 0; r < kD; ++r) dkr[r] += __shfl_xor_sync(0xffffffffu, dkr[r], o);
#pragma unroll
        for (int n = 0; n < kDV; ++n) dvr[n] += __shfl_xor_sync(0xffffffffu, dvr[n], o);
    }
    if (j < A.T && x == 0) {
        for (int r = 0; r < kD; ++r) A.dk[(size_t(bkv) * A.T + j) * kD + r] = dkr[r];
        for (int n = 0; n < kDV; ++n) A.dv[(size_t(bkv) * A.T + j) * kDV + n] = dvr[n];
    }
}

// Suffix states R_c = sum over rows of later chunks and the group's query heads of
// phi_h(q_i) g_i^T, in two passes: cb_chunk_agg_kernel writes each chunk's own sum to R[c]
// (block = 64 packed rows x chunk x (b, kv); thread = (packed row, column group of 17 columns
// of [.; 1])), then chunk_scan_kernel (reverse) makes it the exclusive suffix in place.
// Layout [bkv][c][n][f] like S_c.
struct CbAggSmem {
    float qs[64][kDA + 1];  // qhat rows of the chunk for one query head (and 1, 0)
    float A[64][68];        // phi of the rows, [row][packed row of the slab]
    float B[64][68];        // g rows
};

template <typename Tin>
__global__ void __launch_bounds__(256) cb_chunk_agg_kernel(const Tin* __restrict__ q, CbArgs A)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CbAggSmem& sm = *reinterpret_cast<CbAggSmem*>(smem_raw);
    const int slab = blockIdx.x, bkv = blockIdx.z;
    const int b = bkv / A.Hkv, kv = bkv % A.Hkv;
    const int grp = A.Hq / A.Hkv;
    const int tid = threadIdx.x, fi = tid & 63, cg = tid >> 6;
    const int f = slab * 64 + fi;
    const RT rt = feature_rt(f);
    const float* coef = cb_coef(A);
    for (int c = blockIdx.y; c < A.NC; c += gridDim.y) {  // (gridDim.y < NC only past 65535)
        float t4[4][4], tn[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            tn[i] = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) t4[i][jj] = 0.f;
        }
        const int t0 = c * kCbC;
        for (int x = 0; x < grp; ++x) {
            const int h = kv * grp + x;
            const size_t r0 = (size_t(b) * A.Hq + h) * A.T + t0;
            const float cf = coef[size_t(h) * kFP + f];
            for (int e = tid; e < 64 * kD; e += 256) {
                const int j = e / kD, r = e % kD;
                sm.qs[j][r] = t0 + j < A.T ? to_f32(q[(r0 + j) * kD + r]) : 0.f;
            }
            for (int e = tid; e < 64 * kW; e += 256) {
                const int j = e / kW, n = e % kW;
                sm.B[j][n] = t0 + j < A.T ? A.Gr[(r0 + j) * kW + n] : 0.f;
            }
            if (tid < 64) {
                sm.qs[tid][kD] = 1.f;
                sm.qs[tid][kD + 1] = 0.f;
            }
            __syncthreads();
            for (int j = cg; j < 64; j += 4) sm.A[j][fi] = cf * sm.qs[j][rt.r] * sm.qs[j][rt.t];
            __syncthreads();
            tile_acc_simt(sm.A, sm.B, t4, tn);
            __syncthreads();
        }
        tile_store_simt(A.R + (size_t(bkv) * A.NC + c) * kW * kFP, slab * 64, t4, tn);
    }
}

struct CbRowSmem {
    float qs[64][kDA + 1];   // qhat rows (the tile's query rows, or the chunk's key rows)
    float gs[64][kW];        // g rows, or [v; 1] rows
    float gT[kW][68];        // gs transposed, rows 16-byte aligned
    float hs[kW][64];        // a 64-row slab of S_c or R_c, [n][f]
    float ps[64][65];        // dphi or dpsi of the slab, [row][f]
    float ds[64][kD + 1];    // dq or dk of the tile's rows
    float red[4][64];
};

// Inter-chunk rows: tile = chunk c >= 1 of (b, h).  dphi_i = S_c g_i slab by slab; dq_i +=
// sum_f dphi_f C'_f d(qhat_r qhat_t)/dq; partial dC'_f = sum_i dphi_f(q_i) qhat_r qhat_t.
template <typename Tin>
__global__ void __launch_bounds__(256) cb_inter_rows_kernel(const Tin* __restrict__ q, CbArgs A)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CbRowSmem& sm = *reinterpret_cast<CbRowSmem*>(smem_raw);
    const int c = blockIdx.x, bh = blockIdx.y, b = bh / A.Hq, h = bh % A.Hq;
    const int bkv = b * A.Hkv + h / (A.Hq / A.Hkv);
    const int tid = threadIdx.x, ri = tid & 63, cg = tid >> 6;
    const int i0 = c * kCbC;
    float* dcp = A.dcp + (size_t(bh) * A.NC + c) * kFP;
    if (c == 0) {  // S_0 = 0: no inter-chunk part
        for (int f = tid; f < kFP; f += 256) dcp[f] = 0.f;
        return;
    }
    const size_t r0 = size_t(bh) * A.T + i0;
    for (int e = tid; e < 64 * kD; e += 256) {
        const int j = e / kD, r = e % kD;
        sm.qs[j][r] = i0 + j < A.T ? to_f32(q[(r0 + j) * kD + r]) : 0.f;
        sm.ds[j][r] = 0.f;
    }
    for (int e = tid; e < 64 * kW; e += 256) {
        const int j = e / kW, n = e % kW;
        sm.gs[j][n] = i0 + j < A.T ? A.Gr[(r0 + j) * kW + n] : 0.f;
    }
    if (tid < 64) {
        sm.qs[tid][kD] = 1.f;
        sm.qs[tid][kD + 1] = 0.f;
    }
    for (int e = tid; e < 64 * kW; e += 256) {
        const int j = e / kW, n = e % kW;
        sm.gT[n][j] = i0 + j < A.T ? A.Gr[(r0 + j) * kW + n] : 0.f;
    }
    __syncthreads();
    const float* Hs = A.Hc + (size_t(bkv) * A.NC + c) * kW * kFP;
    const float* cf = cb_coef(A) + size_t(h) * kFP;
    // dphi tile: thread owns rows 4 (tid & 15) .. + 3 and packed rows 4 (tid >> 4) .. + 3 of
    // the slab, the sum over n in order
    const int rg = tid & 15, fq = tid >> 4;
    for (int slab = 0; slab < kFP / 64; ++slab) {
        for (int e = tid; e < kW * 64; e += 256) {
            const int n = e / 64, fl = e % 64;
            sm.hs[n][fl] = Hs[size_t(n) * kFP + slab * 64 + fl];
        }
        __syncthreads();
        {
            float t4[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) t4[i][jj] = 0.f;
#pragma unroll 5
            for (int n = 0; n < kW; ++n) {
                const float4 hv = *reinterpret_cast<const float4*>(&sm.hs[n][4 * fq]);
                const float4 gv = *reinterpret_cast<const float4*>(&sm.gT[n][4 * rg]);
                const float hf[4] = {hv.x, hv.y, hv.z, hv.w}, gr[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) t4[i][jj] = fmaf(hf[jj], gr[i], t4[i][jj]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) sm.ps[4 * rg + i][4 * fq + jj] = t4[i][jj];
        }
        __syncthreads();
        // dq: thread (row ri, cg) owns the dims d = cg (mod 4)
        for (int fl = 0; fl < 64; ++fl) {
            const int f = slab * 64 + fl;
            const RT rt = feature_rt_tab(f);
            const float w = sm.ps[ri][fl] * cf[f];
            if (rt.r < kD && (rt.r & 3) == cg)
                sm.ds[ri][rt.r] += rt.r == rt.t ? 2.f * w * sm.qs[ri][rt.r] : w * sm.qs[ri][rt.t];
            if (rt.t < kD && rt.t != rt.r && (rt.t & 3) == cg) sm.ds[ri][rt.t] += w * sm.qs[ri][rt.r];
        }
        // partial dC' of the slab's rows: thread (f, row group)
        {
            const RT rt = feature_rt_tab(slab * 64 + ri);
            float part = 0.f;
            for (int j = cg; j < 64; j += 4)
                part = fmaf(sm.ps[j][ri], sm.qs[j][rt.r] * sm.qs[j][rt.t], part);
            sm.red[cg][ri] = part;
        }
        __syncthreads();
        if (tid < 64)
            dcp[slab * 64 + tid] = ((sm.red[0][tid] + sm.red[1][tid]) + sm.red[2][tid]) + sm.red[3][tid];
        __syncthreads();
    }
    if (i0 + ri < A.T)
        for (int d = cg; d < kD; d += 4) A.dq[(r0 + ri) * kD + d] += sm.ds[ri][d];
}

// Inter-chunk keys: tile = chunk c < NC - 1 of (b, kv).  dpsi_j = R_c w_j slab by slab; dk_j +=
// sum_f dpsi_f d(khat_r khat_t)/dk; dw_j += R_c^T psi_j, dv_j = dw_j[:64].
template <typename Tin>
__global__ void __launch_bounds__(256) cb_inter_keys_kernel(const Tin* __restrict__ k,
                                                            const Tin* __restrict__ v, CbArgs A)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CbRowSmem& sm = *reinterpret_cast<CbRowSmem*>(smem_raw);
    const int c = blockIdx.x, bkv = blockIdx.y;
    if (c >= A.NC - 1) return;  // R of the last chunk is 0
    const int tid = threadIdx.x, rj = tid & 63, cg = tid >> 6;
    const int j0 = c * kCbC;
    const size_t r0 = size_t(bkv) * A.T + j0;
    for (int e = tid; e < 64 * kD; e += 256) {
        const int j = e / kD, r = e % kD;
        const bool ok = j0 + j < A.T;
        sm.qs[j][r] = ok ? to_f32(k[(r0 + j) * kD + r]) : 0.f;
        sm.gs[j][r] = ok ? to_f32(v[(r0 + j) * kDV + r]) : 0.f;
        sm.ds[j][r] = 0.f;
    }
    if (tid < 64) {
        sm.qs[tid][kD] = 1.f;
        sm.qs[tid][kD + 1] = 0.f;
        sm.gs[tid][kDV] = j0 + tid < A.T ? 1.f : 0.f;
    }
    __syncthreads();
    float dw[17];
#pragma unroll
    for (int u = 0; u < 17; ++u) dw[u] = 0.f;
    const float* Rs = A.R + (size_t(bkv) * A.NC + c) * kW * kFP;
    for (int slab = 0; slab < kFP / 64; ++slab) {
        for (int e = tid; e < kW * 64; e += 256) {
            const int n = e / 64, fl = e % 64;
            sm.hs[n][fl] = Rs[size_t(n) * kFP + slab * 64 + fl];
        }
        __syncthreads();
        for (int u = 0; u < 16; ++u) {
            const int fl = cg + 4 * u;
            float d = 0.f;
            for (int n = 0; n < kW; ++n) d = fmaf(sm.hs[n][fl], sm.gs[rj][n], d);
            sm.ps[rj][fl] = d;
        }
        for (int fl = 0; fl < 64; ++fl) {
            const RT rt = feature_rt_tab(slab * 64 + fl);
            const float psi = sm.qs[rj][rt.r] * sm.qs[rj][rt.t];
#pragma unroll
            for (int u = 0; u < 17; ++u) {
                const int n = cg + 4 * u;
                if (n < kW) dw[u] = fmaf(sm.hs[n][fl], psi, dw[u]);
            }
        }
        __syncthreads();
        for (int fl = 0; fl < 64; ++fl) {
            const RT rt = feature_rt_tab(slab * 64 + fl);
            const float w = sm.ps[rj][fl];
            if (rt.r < kD && (rt.r & 3) == cg)
                sm.ds[rj][rt.r] += rt.r == rt.t ? 2.f * w * sm.qs[rj][rt.r] : w * sm.qs[rj][rt.t];
            if (rt.t < kD && rt.t != rt.r && (rt.t & 3) == cg) sm.ds[rj][rt.t] += w * sm.qs[rj][rt.r];
        }
        __syncthreads();
    }
    if (j0 + rj < A.T) {
        for (int d = cg; d < kD; d += 4) A.dk[(r0 + rj) * kD + d] += sm.ds[rj][d];
#pragma unroll
        for (int u = 0; u < 17; ++u) {
            const int n = cg + 4 * u;
            if (n < kDV) A.dv[(r0 + rj) * kDV + n] += dw[u];
        }
    }
}

// Per (b*h, chunk): the chunk's rows' dM and deps partials, summed in row order into the
// chunk's first row (each thread owns one of the 81 dM entries, thread 81 deps).
__global__ void __launch_bounds__(96) cb_rowsum_kernel(CbArgs A)
{
    const int c = blockIdx.x, bh = blockIdx.y, e = threadIdx.x;
    const size_t r0 = size_t(bh) * A.T + size_t(c) * kCbC;
    const int n = min(kCbC, A.T - c * kCbC);
    if (e < kMM) {
        float s = 0.f;
        for (int i = 0; i < n; ++i) s += A.rowM[(r0 + i) * kMM + e];
        A.rowM[r0 * kMM + e] = s;
    } else if (e == kMM) {
        float s = 0.f;
        for (int i = 0; i < n; ++i) s += A.rowE[r0 + i];
        A.rowE[r0] = s;
    }
}

// Per (head, packed row f): the partial dC'_f of every (b, chunk), summed in that order into
// the (b = 0, chunk 0) slot.
__global__ void __launch_bounds__(256) cb_dcsum_kernel(CbArgs A)
{
    const int f = blockIdx.x * blockDim.x + threadIdx.x, h = blockIdx.y;
    if (f >= kF) return;
    float acc = 0.f;
    for (int b = 0; b < A.B; ++b)
        for (int c = 0; c < A.NC; ++c)
            acc += A.dcp[((size_t(b) * A.Hq + h) * A.NC + c) * kFP + f];
    A.dcp[size_t(h) * A.NC * kFP + f] = acc;
}

// dM_h = the rows' within-chunk partials plus dC'_h mapped through C'_f = (2 - [r = t])
// M_{g(r)g(t)} s_r s_t (each ordered pair (r, t) carries half of an off-diagonal row), summed in
// a fixed order; dL_h = (dM + dM^T) L; deps_h = within-chunk partials + dC' of the constant row.
__global__ void __launch_bounds__(kMM) cb_heads_kernel(CbArgs A)
{
    const int h = blockIdx.x, e = threadIdx.x;
    __shared__ float dM[kMM];
    __shared__ float dC[kFP];
    __shared__ int g[kDA];
    __shared__ int sG;
    if (e == 0) {
        int Gh = A.G[h];
        sG = Gh < 1 ? 1 : (Gh > kGMax ? kGMax : Gh);
    }
    __syncthreads();
    const int Gh = sG;
    if (e < kD) {
        int x = A.gid[h * kD + e];
        g[e] = x < 1 ? 1 : (x > Gh ? Gh : x);
    } else if (e < kDA) {
        g[e] = 0;  // the constant slot belongs to sbar_0
    }
    // dC'_h: cb_dcsum_kernel left the sum over every (b, chunk) in the (b = 0, chunk 0) slot
    const bool any = A.B > 0 && A.NC > 0;
    for (int f = e; f < kF; f += kMM) dC[f] = any ? A.dcp[size_t(h) * A.NC * kFP + f] : 0.f;
    // the rows' partials: cb_rowsum_kernel left each chunk's sum in the chunk's first row
    float s = 0.f, de = 0.f;
    for (int b = 0; b < A.B; ++b)
        for (int c = 0; c < A.NC; ++c) {
            const size_t row = (size_t(b) * A.Hq + h) * A.T + size_t(c) * kCbC;
            s += A.rowM[row * kMM + e];
            if (e == 0) de += A.rowE[row];
        }
    __syncthreads();
    const int a = e / kGM1, mm = e % kGM1;
    float sc = 0.f;  // dC' reaching M_{a mm}
    if (a <= Gh && mm <= Gh) {
        for (int f = 0; f < kF; ++f) {
            const RT rt = feature_rt_tab(f);
            const int ga = g[rt.r], gb = g[rt.t];
            float wgt = (ga == a && gb == mm) ? 1.f : 0.f;
            if (rt.r != rt.t && gb == a && ga == mm) wgt += 1.f;
            if (wgt != 0.f) {
                const float sr = rt.r < kD ? 0.125f : 1.f, st = rt.t < kD ? 0.125f : 1.f;
                sc = fmaf(dC[f] * wgt, sr * st, sc);
            }
        }
    }
    if (e == 0) de += dC[kConstRow];  // C'_const = M_00 + eps
    dM[e] = s + sc;
    __syncthreads();
    float val = 0.f;
    if (a <= Gh && mm <= Gh) {
        const float* Lh = A.L + size_t(h) * kMM;
        for (int c = 0; c <= Gh; ++c) val = fmaf(dM[a * kGM1 + c] + dM[c * kGM1 + a], Lh[c * kGM1 + mm], val);
    }
    A.dL[size_t(h) * kMM + e] = val;
    if (e == 0) A.headE[h] = de;
}

__global__ void cb_eps_kernel(CbArgs A)
{
    float s = 0.f;
    for (int h = 0; h < A.Hq; ++h) s += A.headE[h];
    *A.deps = s;
}

struct CbLayout {
    size_t st, Hc, R, rowD, rowY, Gr, dcp, rowM, rowE, headE, total;
};

CbLayout cb_layout(int B, int T, int Hq, int Hkv)
{
    CbLayout l{};
    const size_t NC = size_t((T + kCbC - 1) / kCbC), rows = size_t(B) * Hq * T;
    const size_t states = size_t(B) * Hkv * NC * kW * kFP * 4;
    size_t o = 0;
    auto take = [&](size_t n) {
        const size_t at = o;
        o += align256(n);
        return at;
    };
    l.st = take(kHeaderBytes + coef_bytes(Hq) + size_t(B) * Hkv * state_unit_bytes());
    l.Hc = take(states);
    l.R = take(states);
    l.rowD = take(rows * 4);
    l.rowY = take(rows * kDV * 4);
    l.Gr = take(rows * kW * 4);
    l.dcp = take(size_t(B) * Hq * NC * kFP * 4);
    l.rowM = take(rows * kMM * 4);
    l.rowE = take(rows * 4);
    l.headE = take(size_t(Hq) * 4);
    l.total = std::max<size_t>(o, 256);
    return l;
}

template <typename Tin>
static int launch_backward_chunked_t(const Tin* q, const Tin* k, const Tin* v, CbArgs A,
                                     cudaStream_t st)
{
    const int B = A.B, T = A.T, Hq = A.Hq, Hkv = A.Hkv, NC = A.NC;
    int rc = launch_prep(A.gid, A.L, A.G, A.eps, A.st, B, Hq, Hkv, T, st);
    if (rc) return rc;
    if (B > 0 && T > 0) {
        float* body = reinterpret_cast<float*>(A.st + kHeaderBytes + coef_bytes(Hq));
        {
            LaunchScope ls("backward_state", st);
            const int rc2 = launch_chunk_states_simt(k, v, T, kCbC, NC, A.Hc, body, B * Hkv, st);
            if (rc2) return rc2;
        }
        {
            const size_t smem = sizeof(ReadoutSmem);
            auto kern = readout_simt_kernel<Tin, false>;
            OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              int(smem)));
            LaunchScope ls("backward_forward", st);
            kern<<<dim3((T + 63) / 64, B * Hq), 256, smem, st>>>(
                q, k, v, A.gid, A.L, A.G, A.eps, cb_coef(A), A.Hc, A.rowY, Hq, Hkv, T, kCbC, NC,
                A.rowD);
            OAL_LAUNCH_CHECK();
        }
        {
            LaunchScope ls("backward_g", st);
            const size_t rows = size_t(B) * Hq * T;
            cb_g_kernel<<<unsigned((rows + 7) / 8), 256, 0, st>>>(A);
            OAL_LAUNCH_CHECK();
        }
        {
            LaunchScope ls("backward_intra_rows", st);
            cb_intra_rows_kernel<Tin><<<dim3((T + kBwdThreads - 1) / kBwdThreads, B * Hq),
                                        kBwdThreads, 0, st>>>(q, k, v, A);
            OAL_LAUNCH_CHECK();
        }
        {
            LaunchScope ls("backward_intra_keys", st);
            cb_intra_keys_kernel<Tin><<<dim3((T + kKeysPerBlock - 1) / kKeysPerBlock, B * Hkv),
                                        8 * kKeysPerBlock, 0, st>>>(q, k, v, A);
            OAL_LAUNCH_CHECK();
        }
        {
            LaunchScope ls("backward_suffix", st);
            OAL_CUDA_TRY(cudaFuncSetAttribute(cb_chunk_agg_kernel<Tin>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              int(sizeof(CbAggSmem))));
            cb_chunk_agg_kernel<Tin><<<dim3(kFP / 64, std::min(NC, 65535), B * Hkv), 256,
                                       sizeof(CbAggSmem), st>>>(q, A);
            OAL_LAUNCH_CHECK();
            chunk_scan_kernel<<<dim3((kW * kFP + 255) / 256, B * Hkv), 256, 0, st>>>(A.R, NC, 1,
                                                                                   nullptr);
            OAL_LAUNCH_CHECK();
        }
        const size_t smem = sizeof(CbRowSmem);
        {
            auto kern = cb_inter_rows_kernel<Tin>;
            OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              int(smem)));
            LaunchScope ls("backward_inter_rows", st);
            kern<<<dim3(NC, B * Hq), 256, smem, st>>>(q, A);
            OAL_LAUNCH_CHECK();
        }
        {
            auto kern = cb_inter_keys_kernel<Tin>;
            OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              int(smem)));
            LaunchScope ls("backward_inter_keys", st);
            kern<<<dim3(NC, B * Hkv), 256, smem, st>>>(k, v, A);
            OAL_LAUNCH_CHECK();
        }
    }
    {
        LaunchScope ls("backward_heads", st);
        if (B > 0 && T > 0) {
            cb_rowsum_kernel<<<dim3(NC, B * Hq), 96, 0, st>>>(A);
            OAL_LAUNCH_CHECK();
            cb_dcsum_kernel<<<dim3((kF + 255) / 256, Hq), 256, 0, st>>>(A);
            OAL_LAUNCH_CHECK();
        }
        cb_heads_kernel<<<Hq, kMM, 0, st>>>(A);
        OAL_LAUNCH_CHECK();
    }
    LaunchScope ls("backward_eps", st);
    cb_eps_kernel<<<1, 1, 0, st>>>(A);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

}  // namespace oal

extern "C" {

int oal_backward_workspace_bytes(const oal_shape* s, size_t* bytes)
{
    using namespace oal;
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hq))) return rc;
    if (!bytes) return OAL_ERR_NULL;
    *bytes = cb_layout(s->B, s->T, s->Hq, s->Hkv).total;
    return OAL_OK;
}

int oal_backward(const void* q, const void* k, const void* v, const int32_t* group_id,
                 const float* L, const int32_t* G, float eps, const float* dy, float* dq,
                 float* dk, float* dv, float* dL, float* deps, void* workspace,
                 size_t workspace_bytes, const oal_shape* s, void* stream)
{
    using namespace oal;
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hq))) return rc;
    if (!group_id || !L || !G || !dL || !deps) return OAL_ERR_NULL;
    if ((rc = check_io(s, q, k, v, dq))) return rc;
    if ((long long)s->B * s->T > 0 && (!dy || !dk || !dv)) return OAL_ERR_NULL;
    if (!aligned16(dL) || !aligned16(L) || !aligned16(G) || !aligned16(group_id))
        return OAL_ERR_ALIGN;
    if ((long long)s->B * s->T > 0 && (!aligned16(dy) || !aligned16(dk) || !aligned16(dv)))
        return OAL_ERR_ALIGN;
    const CbLayout lay = cb_layout(s->B, s->T, s->Hq, s->Hkv);
    if (!workspace || workspace_bytes < lay.total) return OAL_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return OAL_ERR_ALIGN;
    unsigned char* w = static_cast<unsigned char*>(workspace);
    CbArgs A;
    A.B = s->B;
    A.T = s->T;
    A.Hq = s->Hq;
    A.Hkv = s->Hkv;
    A.NC = (s->T + kCbC - 1) / kCbC;
    A.eps = eps;
    A.gid = group_id;
    A.L = L;
    A.G = G;
    A.dy = dy;
    A.dq = dq;
    A.dk = dk;
    A.dv = dv;
    A.dL = dL;
    A.deps = deps;
    A.st = w + lay.st;
    A.Hc = reinterpret_cast<float*>(w + lay.Hc);
    A.R = reinterpret_cast<float*>(w + lay.R);
    A.rowD = reinterpret_cast<float*>(w + lay.rowD);
    A.rowY = reinterpret_cast<float*>(w + lay.rowY);
    A.Gr = reinterpret_cast<float*>(w + lay.Gr);
    A.dcp = reinterpret_cast<float*>(w + lay.dcp);
    A.rowM = reinterpret_cast<float*>(w + lay.rowM);
    A.rowE = reinterpret_cast<float*>(w + lay.rowE);
    A.headE = reinterpret_cast<float*>(w + lay.headE);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (s->dtype == OAL_BF16)
        return launch_backward_chunked_t(static_cast<const __nv_bfloat16*>(q),
                                         static_cast<const __nv_bfloat16*>(k),
                                         static_cast<const __nv_bfloat16*>(v), A, st);
    return launch_backward_chunked_t(static_cast<const float*>(q), static_cast<const float*>(k),
                                     static_cast<const float*>(v), A, st);
}

}  // extern "C"
