// oal_simt.cu -- CUDA-core kernels of the OAL library: coefficient expansion, the fp32
// chunked prefill (state builder + readout with the intra-chunk dense kernel), the O(T^2)
// dense form, and the memory-bound decode step.
//
// Equations cited are those of "OAL: 按 QK 离群贡献分组的正二次注意力核" (reproduction note of
// arXiv 2610.13674), section 核心公式, numbered in order of appearance: (2) grouped score,
// (3) kernel kappa, (4) prefix states H0/H1/H2, (5) readout.  The packed feature map that
// merges H0/H1/H2 into one state is described in oal_common.cuh.
#include <type_traits>

#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

// (r, t) of every packed row as r | t << 8: a table for the loops that visit many rows, which
// would otherwise walk the block structure of feature_rt once per row.
struct RtTable {
    uint16_t v[kF];
};
constexpr RtTable make_rt_table()
{
    RtTable tab{};
    for (int f = 0; f < kF; ++f) {
        const RT rt = feature_rt(f);
        tab.v[f] = uint16_t(rt.r | (rt.t << 8));
    }
    return tab;
}
__device__ const RtTable c_rt_tab = make_rt_table();
__device__ __forceinline__ RT feature_rt_tab(int f)
{
    if (f >= kF) return RT{kD + 1, kD + 1};
    const uint32_t x = c_rt_tab.v[f];
    return RT{int(x & 255u), int(x >> 8)};
}

// ------------------------------------------------------------------------------------------
// a1: coefficient expansion.  M = L L^T (fp64), then the packed readout coefficients
// Cp_f (oal_common.cuh) per query head, written into the state buffer's coefficient table;
// block 0 also writes the state header.  Group ids and G are validated; out-of-range values
// raise OAL_ERR_GROUPS and are clamped so that nothing reads outside M.
// ------------------------------------------------------------------------------------------
// One block of 256 threads per query head h: M = L L^T in fp64, the packed coefficient table
// of that head, and (head 0) the state header.
__device__ __forceinline__ void prep_head(int h, const int32_t* __restrict__ gid,
                                          const float* __restrict__ L,
                                          const int32_t* __restrict__ G, float eps,
                                          unsigned char* __restrict__ state, int B, int Hq,
                                          int Hkv, long long tokens, bool add_tokens = false,
                                          unsigned char* __restrict__ rtab = nullptr)
{
    const int tid = threadIdx.x;
    __shared__ double M[kGM1][kGM1];
    __shared__ int g[kDA];
    __shared__ int sG;
    if (tid == 0) {
        int Gh = G[h];
        if (Gh < 1 || Gh > kGMax) {
            raise_error(OAL_ERR_GROUPS);
            Gh = Gh < 1 ? 1 : kGMax;
        }
        sG = Gh;
    }
    __syncthreads();
    const int Gh = sG;
    if (tid < kD) {
        int x = gid[h * kD + tid];
        if (x < 1 || x > Gh) {
            raise_error(OAL_ERR_GROUPS);
            x = x < 1 ? 1 : Gh;
        }
        g[tid] = x;
    } else if (tid < kDA) {
        g[tid] = 0;  // the constant slot (index 64) belongs to sbar_0; 65 is padding
    }
    if (tid < kGM1 * kGM1) {
        const int a = tid / kGM1, c = tid % kGM1;
        double acc = 0.0;
        if (a <= Gh && c <= Gh) {
            const float* Lh = L + size_t(h) * kGM1 * kGM1;
            for (int m = 0; m <= Gh; ++m) acc += double(Lh[a * kGM1 + m]) * double(Lh[c * kGM1 + m]);
        }
        M[a][c] = acc;
    }
    __syncthreads();
    float* coef = reinterpret_cast<float*>(state + kHeaderBytes) + size_t(h) * kFP;
    for (int f = tid; f < kFP; f += blockDim.x) {
        double val = 0.0;
        if (f < kF) {
            const RT rt = feature_rt(f);
            const double sr = rt.r < kD ? 0.125 : 1.0, st = rt.t < kD ? 0.125 : 1.0;
            val = (rt.r == rt.t ? 1.0 : 2.0) * M[g[rt.r]][g[rt.t]] * sr * st;
            if (f == kConstRow) val += double(eps);
        }
        coef[f] = float(val);
        if (rtab) {  // the readout table: bf16 off-diagonal coefficients, fp32 for the rest
            unsigned char* tb = rtab + size_t(h) * kTabBytes;
            if (f < kOffDiagRows)
                reinterpret_cast<__nv_bfloat16*>(tb + kTabCoefH)[f] = __float2bfloat16_rn(float(val));
            else
                reinterpret_cast<float*>(tb + kTabCoefT)[f - kOffDiagRows] = float(val);
        }
    }
    if (rtab) {
        // score-tile weights of the factored intra-chunk kernel, eq. (3) as
        // kappa = eps + sum_m (L_0m + sum_r q_r k_r L_{g(r),m} / sqrt(d_h))^2
        unsigned char* tb = rtab + size_t(h) * kTabBytes;
        const float* Lh = L + size_t(h) * kGM1 * kGM1;
        for (int e = tid; e < kGM1 * kD; e += blockDim.x) {
            const int m = e / kD, r = e % kD;
            reinterpret_cast<float*>(tb + kTabW)[e] = m <= Gh ? Lh[g[r] * kGM1 + m] * 0.125f : 0.f;
        }
        if (tid < kGM1) reinterpret_cast<float*>(tb + kTabC0)[tid] = tid <= Gh ? Lh[tid] : 0.f;
        if (tid == 0) *reinterpret_cast<int*>(tb + kTabG) = Gh;
        if (tid < 8) {  // block R of 8 dims in a single group: its phi weights depend on t only
            bool pure = true;
            for (int a = 1; a < 8; ++a) pure = pure && g[8 * tid + a] == g[8 * tid];
            tb[kTabPure + tid] = pure ? 1 : 0;
        }
        for (uint32_t b = kTabPure + 8 + tid; b < kTabBytes; b += blockDim.x) tb[b] = 0;
    }
    if (h == 0 && tid == 0) {
        StateHeader* hd = reinterpret_cast<StateHeader*>(state);
        hd->magic = kStateMagic;
        hd->abi = OAL_ABI_VERSION;
        hd->B = B;
        hd->Hq = Hq;
        hd->Hkv = Hkv;
        hd->dh = kD;
        hd->dv = kDV;
        hd->feat_pad = kFP;
        hd->tokens = add_tokens ? hd->tokens + tokens : tokens;
        hd->eps = eps;
        for (int i = 0; i < int(sizeof(hd->reserved) / sizeof(hd->reserved[0])); ++i)
            hd->reserved[i] = 0;  // every byte of the state is defined
    }
}

__global__ void __launch_bounds__(256) prep_kernel(const int32_t* __restrict__ gid,
                                                   const float* __restrict__ L,
                                                   const int32_t* __restrict__ G, float eps,
                                                   unsigned char* __restrict__ state, int B,
                                                   int Hq, int Hkv, long long tokens)
{
    prep_head(blockIdx.x, gid, L, G, eps, state, B, Hq, Hkv, tokens);
}

// ------------------------------------------------------------------------------------------
// a5-a7 (fp32 path): chunk states.  One block owns 64 packed rows of one (b, kv) state and
// walks the chunks in order.  Before adding chunk c it stores the exclusive prefix
// S_c = sum_{j < cC} psi(k_j) [v_j; 1] (eq. (4)) to Hc[(bkv*NC + c)][n][f] (fp32, column
// major); after the last chunk it writes the inclusive state into the state buffer.
// ------------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256) state_simt_kernel(const Tin* __restrict__ k,
                                                         const Tin* __restrict__ v, int T,
                                                         int C, int NC, float* __restrict__ Hc,
                                                         float* __restrict__ body)
{
    const int slab = blockIdx.x, bkv = blockIdx.y;
    const int tid = threadIdx.x, fi = tid & 63, cg = tid >> 6;
    const int f = slab * 64 + fi;
    const RT rt = feature_rt(f);
    __shared__ float ks[64][kDA + 1];
    __shared__ float vs[64][kW];
    const Tin* kb = k + size_t(bkv) * T * kD;
    const Tin* vb = v + size_t(bkv) * T * kDV;
    float run[17], acc[17];
#pragma unroll
    for (int u = 0; u < 17; ++u) run[u] = 0.f;
    for (int c = 0; c < NC; ++c) {
        if (Hc) {
            float* dst = Hc + (size_t(bkv) * NC + c) * kW * kFP;
#pragma unroll
            for (int u = 0; u < 17; ++u) {
                const int n = cg + 4 * u;
                if (n < kW) dst[size_t(n) * kFP + f] = run[u];
            }
        }
#pragma unroll
        for (int u = 0; u < 17; ++u) acc[u] = 0.f;
        const int t0 = c * C, t1 = min(t0 + C, T);
        for (int s0 = t0; s0 < t1; s0 += 64) {
            for (int e = tid; e < 64 * kD; e += 256) {
                const int j = e / kD, r = e % kD, tok = s0 + j;
                ks[j][r] = tok < t1 ? to_f32(kb[size_t(tok) * kD + r]) : 0.f;
                vs[j][r] = tok < t1 ? to_f32(vb[size_t(tok) * kDV + r]) : 0.f;
            }
            if (tid < 64) {
                const bool ok = s0 + tid < t1;
                ks[tid][kD] = ok ? 1.f : 0.f;
                ks[tid][kD + 1] = 0.f;
                vs[tid][kDV] = ok ? 1.f : 0.f;
            }
            __syncthreads();
            for (int j = 0; j < 64; ++j) {
                const float psi = ks[j][rt.r] * ks[j][rt.t];
#pragma unroll
                for (int u = 0; u < 17; ++u) {
                    const int n = cg + 4 * u;
                    if (n < kW) acc[u] = fmaf(psi, vs[j][n], acc[u]);
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int u = 0; u < 17; ++u) run[u] += acc[u];
    }
    float* unit = body + size_t(bkv) * kFP * kW;
#pragma unroll
    for (int u = 0; u < 17; ++u) {
        const int n = cg + 4 * u;
        if (n < kDV) unit[size_t(f) * kDV + n] = run[u];
        else if (n == kDV) unit[size_t(kFP) * kDV + f] = run[u];
    }
}

// ------------------------------------------------------------------------------------------
// a8-a10 (fp32 path) and a12: readout of 64 query rows of one (b, h).
// inter (prefill only): u_i += phi(q_i)^T S_c with phi_f(q) = Cp_f qhat_r qhat_t (eq. (5));
// intra: u_i += sum_j kappa(q_i, k_j) [v_j; 1] over j in [j0, i] with kappa from eqs.
// (2)-(3) (j0 = start of the chunk for prefill, 0 for the dense form); then
// yhat_i = u_i[0:64] / u_i[64] (and, when den_out is given, D_i = u_i[64]).
// ------------------------------------------------------------------------------------------
// The inter-chunk tile's operands, transposed: phi of the 64 rows and a 64-row slab of S_c,
// each [f][row or n] with rows 16-byte aligned (68 floats), so that a thread reads four
// consecutive rows or columns as one vector.
struct InterTiles {
    float psT[64][68];
    float hsT[64][68];
};

struct ReadoutSmem {
    float qs[64][kDA + 1];
    float ps[64][65];
    union {
        InterTiles t;
        struct {
            float ks[64][kD + 1];
            float vs[64][kW];
        } kv;
    } u;
    float Ms[kGM1][kGM1];
    int gperm[kD];
    int gstart[kGM1 + 1];
    int G;
};

// Inter-chunk part of a 64-row readout tile: res[row][n] = sum_f phi_f(q_row) S_c[n][f] with
// phi_f = cf_f qhat_r qhat_t (eq. (5)), the sum running over the 64-row slabs of S_c and the
// rows f of each slab in order.  256 threads; in the products, thread t owns rows
// 4 (t & 15) .. + 3 and columns 4 (t >> 4) .. + 3 (and column 64 for t < 16), reading four
// phi values and four S values per f as two vectors.  Ends with res complete and synchronised.
template <class Smem>
__device__ __forceinline__ void inter_tile_simt(Smem& sm, const float* __restrict__ Hs,
                                                const float* __restrict__ cf,
                                                float (*res)[65])
{
    const int tid = threadIdx.x, ri = tid & 63, cg = tid >> 6;
    const int rg = tid & 15, cq = tid >> 4;
    float t4[4][4], tn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        tn[i] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) t4[i][j] = 0.f;
    }
    for (int slab = 0; slab < kFP / 64; ++slab) {
        const int f = slab * 64 + ri;
        for (int n = cg; n < kW; n += 4) sm.u.t.hsT[ri][n] = Hs[size_t(n) * kFP + f];
        const RT rt = feature_rt_tab(f);
        const float cfv = cf[f];
        for (int row = cg; row < 64; row += 4)
            sm.u.t.psT[ri][row] = cfv * sm.qs[row][rt.r] * sm.qs[row][rt.t];
        __syncthreads();
#pragma unroll 4
        for (int ff = 0; ff < 64; ++ff) {
            const float4 a = *reinterpret_cast<const float4*>(&sm.u.t.psT[ff][4 * rg]);
            const float4 b = *reinterpret_cast<const float4*>(&sm.u.t.hsT[ff][4 * cq]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) t4[i][j] = fmaf(av[i], bv[j], t4[i][j]);
            if (cq == 0) {
                const float bn = sm.u.t.hsT[ff][kDV];
#pragma unroll
                for (int i = 0; i < 4; ++i) tn[i] = fmaf(av[i], bn, tn[i]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) res[4 * rg + i][4 * cq + j] = t4[i][j];
        if (cq == 0) res[4 * rg + i][kDV] = tn[i];
    }
    __syncthreads();
}

template <typename Tin, bool kDense>
__global__ void __launch_bounds__(256) readout_simt_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const int32_t* __restrict__ gid, const float* __restrict__ L, const int32_t* __restrict__ G,
    float eps, const float* __restrict__ coef, const float* __restrict__ Hc,
    float* __restrict__ out, int Hq, int Hkv, int T, int C, int NC,
    float* __restrict__ den_out)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ReadoutSmem& sm = *reinterpret_cast<ReadoutSmem*>(smem_raw);
    const int tile = blockIdx.x, bh = blockIdx.y;
    const int b = bh / Hq, h = bh % Hq, kv = h / (Hq / Hkv), bkv = b * Hkv + kv;
    const int i0 = tile * 64;
    const int tid = threadIdx.x, ri = tid & 63, cg = tid >> 6;
    const Tin* qb = q + size_t(bh) * T * kD;
    const Tin* kb = k + size_t(bkv) * T * kD;
    const Tin* vb = v + size_t(bkv) * T * kDV;

    for (int e = tid; e < 64 * kD; e += 256) {
        const int j = e / kD, r = e % kD;
        sm.qs[j][r] = i0 + j < T ? to_f32(qb[size_t(i0 + j) * kD + r]) : 0.f;
    }
    if (tid < 64) {
        sm.qs[tid][kD] = 1.f;
        sm.qs[tid][kD + 1] = 0.f;
    }
    if (tid == 0) {
        int Gh = G[h];
        if (Gh < 1 || Gh > kGMax) {
            raise_error(OAL_ERR_GROUPS);
            Gh = Gh < 1 ? 1 : kGMax;
        }
        sm.G = Gh;
        // dims sorted by group (counting sort), so each s_g is a contiguous run
        int cnt[kGM1 + 1];
        for (int g = 0; g <= kGM1; ++g) cnt[g] = 0;
        for (int r = 0; r < kD; ++r) {
            int x = gid[h * kD + r];
            if (x < 1 || x > Gh) {
                raise_error(OAL_ERR_GROUPS);
                x = x < 1 ? 1 : Gh;
            }
            cnt[x + 1]++;
        }
        for (int g = 1; g <= kGM1; ++g) cnt[g] += cnt[g - 1];
        for (int g = 0; g <= kGM1; ++g) sm.gstart[g] = cnt[g];
        for (int r = 0; r < kD; ++r) {
            int x = gid[h * kD + r];
            x = x < 1 ? 1 : (x > Gh ? Gh : x);
            sm.gperm[cnt[x]++] = r;
        }
    }
    __syncthreads();
    const int Gh = sm.G;
    if (tid < kGM1 * kGM1) {
        const int a = tid / kGM1, c = tid % kGM1;
        float acc = 0.f;
        if (a <= Gh && c <= Gh) {
            const float* Lh = L + size_t(h) * kGM1 * kGM1;
            for (int m = 0; m <= Gh; ++m) acc = fmaf(Lh[a * kGM1 + m], Lh[c * kGM1 + m], acc);
        }
        sm.Ms[a][c] = acc;
    }
    __syncthreads();

    float acc[17];
#pragma unroll
    for (int u = 0; u < 17; ++u) acc[u] = 0.f;

    const int c = i0 / C;
    if (!kDense && c > 0) {
        inter_tile_simt(sm, Hc + (size_t(bkv) * NC + c) * kW * kFP, coef + size_t(h) * kFP,
                        sm.ps);
#pragma unroll
        for (int u = 0; u < 17; ++u) {
            const int n = cg + 4 * u;
            if (n < kW) acc[u] = sm.ps[ri][n];
        }
        __syncthreads();  // ps is the intra-chunk weights' buffer from here on
    }

    const int j0 = kDense ? 0 : c * C;
    const int j1 = min(i0 + 64, T);
    for (int kb0 = j0; kb0 < j1; kb0 += 64) {
        for (int e = tid; e < 64 * kD; e += 256) {
            const int j = e / kD, r = e % kD, tok = kb0 + j;
            sm.u.kv.ks[j][r] = tok < T ? to_f32(kb[size_t(tok) * kD + r]) : 0.f;
            sm.u.kv.vs[j][r] = tok < T ? to_f32(vb[size_t(tok) * kDV + r]) : 0.f;
        }
        if (tid < 64) sm.u.kv.vs[tid][kDV] = 1.f;
        __syncthreads();
        const int i = i0 + ri;
        for (int key = cg; key < 64; key += 4) {
            const int j = kb0 + key;
            float kap = 0.f;
            if (j <= i && j < T && i < T) {
                float sb[kGM1];
                sb[0] = 1.f;
#pragma unroll
                for (int g = 1; g < kGM1; ++g) {
                    float s = 0.f;
                    if (g <= Gh) {
                        for (int e = sm.gstart[g]; e < sm.gstart[g + 1]; ++e) {
                            const int r = sm.gperm[e];
                            s = fmaf(sm.qs[ri][r], sm.u.kv.ks[key][r], s);
                        }
                    }
                    sb[g] = s * 0.125f;
                }
                float quad = 0.f;
#pragma unroll
                for (int a = 0; a < kGM1; ++a) {
                    float row = 0.f;
#pragma unroll
                    for (int bb = 0; bb < kGM1; ++bb) row = fmaf(sm.Ms[a][bb], sb[bb], row);
                    quad = fmaf(sb[a], row, quad);
                }
                kap = eps + quad;
            }
            sm.ps[ri][key] = kap;
        }
        __syncthreads();
        for (int key = 0; key < 64; ++key) {
            const float p = sm.ps[ri][key];
#pragma unroll
            for (int u = 0; u < 17; ++u) {
                const int n = cg + 4 * u;
                if (n < kW) acc[u] = fmaf(p, sm.u.kv.vs[key][n], acc[u]);
            }
        }
        __syncthreads();
    }

    // normalise: the denominator u[64] lives in the cg == 0 thread (u index 16)
#pragma unroll
    for (int u = 0; u < 17; ++u) {
        const int n = cg + 4 * u;
        if (n < kW) sm.ps[ri][n] = acc[u];
    }
    __syncthreads();
    const int i = i0 + ri;
    if (i < T) {
        const float den = sm.ps[ri][kDV];
        float* o = out + (size_t(bh) * T + i) * kDV;
        for (int n = cg; n < kDV; n += 4) o[n] = sm.ps[ri][n] / den;
        if (den_out && cg == 0) den_out[size_t(bh) * T + i] = den;  // the normaliser D_i
    }
}

// ------------------------------------------------------------------------------------------
// a11: decode step.  Block (slab, bkv) streams 240 packed rows of one (b, kv) state once:
// S_f += psi_f(k) [v; 1] (eq. (4) with one new token), then accumulates
// u_h += phi_{h,f}(q_h) S_f for the Hq/Hkv query heads of that kv head (eq. (5)).  Row data
// moves as 128-bit loads and stores (a half warp per 256-byte row), the first rows requested
// before the per-row weights are formed and every batch of rows prefetched while the previous
// one is computed.  Per-block partial u go to the workspace in a fixed order (warp partials
// summed in shared memory, no float atomics); decode_finish_kernel, launched as a
// programmatic dependent, sums the slab partials in slab order and writes yhat.  Every sum
// has a fixed order, so a step is bit-reproducible.
// ------------------------------------------------------------------------------------------
// 9 slabs of 240 packed rows per (b, kv) head: 256 threads with at most 64 registers, so four
// blocks share an SM (592 resident) and a batch-64 step (1152 blocks) takes 1.95 waves -- the
// block count is chosen against the resident slots, since a last wave of a few blocks costs a
// whole block time.
constexpr int kDecRows = 240;
constexpr int kDecThreads = 256;
constexpr int kDecBatch = 2;   // rows per thread per batch (a half warp per row); the next batch is in flight
constexpr int kDecWarps = kDecThreads / 32;

template <typename Tin, int kGrp>  // kGrp = Hq / Hkv query heads per kv head
__global__ void __launch_bounds__(kDecThreads, 4) decode_kernel(const Tin* __restrict__ q,
                                                              const Tin* __restrict__ k,
                                                              const Tin* __restrict__ v,
                                                              unsigned char* __restrict__ state,
                                                              float* __restrict__ out,
                                                              float* __restrict__ part,
                                                              int Hq, int Hkv)
{
    const int slab = blockIdx.x, bkv = blockIdx.y, nslab = gridDim.x;
    constexpr int grp = kGrp;
    const int b = bkv / Hkv, kv = bkv % Hkv, h0 = kv * grp;
    const int tid = threadIdx.x, lane4 = tid & 15, rsub = tid >> 4, warp = tid >> 5;
    const float* coef = reinterpret_cast<const float*>(state + kHeaderBytes);
    float* unit = reinterpret_cast<float*>(state + kHeaderBytes + coef_bytes(Hq)) +
                  size_t(bkv) * kFP * kW;
    float* Hv = unit;
    float* z = unit + size_t(kFP) * kDV;

    __shared__ __align__(16) float vh[kW + 3];
    __shared__ float kh[kDA];
    __shared__ float qh[kMaxGroup][kDA];
    // per row: phi of the query heads (columns 0..grp-1) and psi (column kPsi); one 32-byte
    // record up to 7 heads, 48 bytes for 8
    constexpr int kRec = kGrp <= 7 ? 8 : 12, kPsi = kGrp <= 7 ? 7 : 8;
    __shared__ __align__(16) float wrow[kDecRows][kRec];
    __shared__ float red[kDecWarps][kMaxGroup][kW];

    const int f0 = slab * kDecRows;
    const int nrows = max(0, min(kDecRows, kF - f0));
    constexpr int kRowStep = kDecThreads / 16;  // rows one pass of the block covers
    // the first batch of rows is requested before anything else
    float4 hv[kDecBatch];
#pragma unroll
    for (int x = 0; x < kDecBatch; ++x) {
        const int row = rsub + kRowStep * x;
        if (row < nrows)
            hv[x] = __ldcs(reinterpret_cast<const float4*>(Hv + size_t(f0 + row) * kDV) + lane4);
    }

    // this thread's row of the slab (kDecRows < kDecThreads: at most one): its readout
    // coefficients and z entry are requested now too, so that their latency overlaps the
    // loads of q, k, v below
    static_assert(kDecRows <= kDecThreads, "one prologue row per thread");
    const bool has_row = tid < nrows;
    float cpre[kGrp];
    float zpre = 0.f;
    if (has_row) {
#pragma unroll
        for (int g = 0; g < kGrp; ++g) cpre[g] = coef[size_t(h0 + g) * kFP + f0 + tid];
        zpre = z[f0 + tid];
    }
    if (tid < kD) {
        kh[tid] = to_f32(k[size_t(bkv) * kD + tid]);
        vh[tid] = to_f32(v[size_t(bkv) * kDV + tid]);
    } else if (tid == kD) {
        kh[kD] = 1.f;
        kh[kD + 1] = 0.f;
        vh[kDV] = 1.f;
    }
    for (int e = tid; e < grp * kDA; e += kDecThreads) {
        const int g = e / kDA, r = e % kDA;
        qh[g][r] = r < kD ? to_f32(q[(size_t(b) * Hq + h0 + g) * kD + r]) : (r == kD ? 1.f : 0.f);
    }
    __syncthreads();
    if (has_row) {
        const int row = tid;
        const RT rt = feature_rt(f0 + row);
        float w[kRec];
#pragma unroll
        for (int g = 0; g < kRec; ++g)
            w[g] = g < grp ? cpre[g < grp ? g : 0] * qh[g][rt.r] * qh[g][rt.t] : 0.f;
        w[kPsi] = kh[rt.r] * kh[rt.t];
#pragma unroll
        for (int x = 0; x < kRec; x += 4)
            *reinterpret_cast<float4*>(&wrow[row][x]) = make_float4(w[x], w[x + 1], w[x + 2], w[x + 3]);
    }
    __syncthreads();

    // eq. (4) rank-1 update of Hv and eq. (5) readout, one 64-float row per half-warp
    float acc[kGrp][4];
#pragma unroll
    for (int g = 0; g < kGrp; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
    const float4 v4 = *reinterpret_cast<const float4*>(&vh[lane4 * 4]);
#pragma unroll 1
    for (int base = rsub; base < nrows; base += kRowStep * kDecBatch) {
        // prefetch the next batch (all loads of a batch are issued before its stores)
        float4 nx[kDecBatch];
#pragma unroll
        for (int x = 0; x < kDecBatch; ++x) {
            const int row = base + kRowStep * (kDecBatch + x);
            if (row < nrows)
                nx[x] = __ldcs(reinterpret_cast<const float4*>(Hv + size_t(f0 + row) * kDV) + lane4);
        }
#pragma unroll
        for (int x = 0; x < kDecBatch; ++x) {
            const int row = base + kRowStep * x;
            if (row < nrows) {
                float ph[kRec];
#pragma unroll
                for (int y = 0; y < kRec; y += 4) {
                    const float4 w4 = *reinterpret_cast<const float4*>(&wrow[row][y]);
                    ph[y] = w4.x;
                    ph[y + 1] = w4.y;
                    ph[y + 2] = w4.z;
                    ph[y + 3] = w4.w;
                }
                const float psi = ph[kPsi];
                float4 h = hv[x];
                h.x = fmaf(psi, v4.x, h.x);
                h.y = fmaf(psi, v4.y, h.y);
                h.z = fmaf(psi, v4.z, h.z);
                h.w = fmaf(psi, v4.w, h.w);
                __stcs(reinterpret_cast<float4*>(Hv + size_t(f0 + row) * kDV) + lane4, h);
#pragma unroll
                for (int g = 0; g < kGrp; ++g) {
                    acc[g][0] = fmaf(ph[g], h.x, acc[g][0]);
                    acc[g][1] = fmaf(ph[g], h.y, acc[g][1]);
                    acc[g][2] = fmaf(ph[g], h.z, acc[g][2]);
                    acc[g][3] = fmaf(ph[g], h.w, acc[g][3]);
                }
            }
        }
#pragma unroll
        for (int x = 0; x < kDecBatch; ++x) hv[x] = nx[x];
    }
    float accz[kGrp];
#pragma unroll
    for (int g = 0; g < kGrp; ++g) accz[g] = 0.f;
    if (has_row) {
        const int row = tid;
        const float zz = zpre + wrow[row][kPsi];
        z[f0 + row] = zz;
        const float* ph = wrow[row];
#pragma unroll
        for (int g = 0; g < kGrp; ++g) accz[g] = fmaf(ph[g], zz, accz[g]);
    }
    // fixed-order reduction: the two half-warps of a warp hold the same columns; every warp
    // writes its partial, then one thread per (head, column) sums the warps in order
#pragma unroll
    for (int g = 0; g < kGrp; ++g) {
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[g][c] += __shfl_xor_sync(0xffffffffu, acc[g][c], 16);
        float zz = accz[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
        if ((tid & 31) < 16) {
#pragma unroll
            for (int c = 0; c < 4; ++c) red[warp][g][lane4 * 4 + c] = acc[g][c];
        }
        if ((tid & 31) == 0) red[warp][g][kDV] = zz;
    }
    __syncthreads();
    float* mypart = part + (size_t(bkv) * nslab + slab) * grp * kW;
    for (int e = tid; e < grp * kW; e += kDecThreads) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) sum += red[w][e / kW][e % kW];
        mypart[e] = sum;
    }
    // the finishing kernel (a programmatic dependent) may launch once every block is here; it
    // waits for this grid's completion before reading the partials
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The end of a decode step: per (b, kv) the slab partials summed in slab order, yhat =
// u[:64] / u[64] for the Hq/Hkv query heads, and the token count of the state header.
// One block per (b, kv); launched as a programmatic dependent of decode_kernel.
template <int kGrp>
__global__ void __launch_bounds__(256) decode_finish_kernel(const float* __restrict__ part,
                                                            float* __restrict__ out,
                                                            unsigned char* __restrict__ state,
                                                            int Hq, int Hkv, int nslab)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials are complete
    constexpr int grp = kGrp;
    const int bkv = blockIdx.x, b = bkv / Hkv, kv = bkv % Hkv, h0 = kv * grp;
    __shared__ float ufin[kMaxGroup][kW];
    const float* allpart = part + size_t(bkv) * nslab * grp * kW;
    constexpr int kSlabs = (kF + kDecRows - 1) / kDecRows;  // the grid's slab count
    for (int e = threadIdx.x; e < grp * kW; e += blockDim.x) {
        // every slab's partial requested at once, then summed in slab order
        float pv[kSlabs];
#pragma unroll
        for (int sl = 0; sl < kSlabs; ++sl)
            pv[sl] = sl < nslab ? allpart[size_t(sl) * grp * kW + e] : 0.f;
        float s = 0.f;
#pragma unroll
        for (int sl = 0; sl < kSlabs; ++sl)
            if (sl < nslab) s += pv[sl];
        ufin[e / kW][e % kW] = s;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < grp * kDV; e += blockDim.x) {
        const int g = e / kDV, n = e % kDV;
        out[(size_t(b) * Hq + h0 + g) * kDV + n] = ufin[g][n] / ufin[g][kDV];
    }
    if (threadIdx.x == 0 && bkv == 0) reinterpret_cast<StateHeader*>(state)->tokens += 1;
}

int launch_prep(const int32_t* gid, const float* L, const int32_t* G, float eps, void* state,
                int B, int Hq, int Hkv, long long tokens, cudaStream_t st)
{
    LaunchScope ls("prep", st);
    prep_kernel<<<Hq, 256, 0, st>>>(gid, L, G, eps, static_cast<unsigned char*>(state), B, Hq,
                                    Hkv, tokens);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

// ------------------------------------------------------------------------------------------
// The same chunk states, chunk-parallel: chunk_delta_simt_kernel writes each chunk's own sum
// psi(k_j) [v_j; 1] over its tokens to Hc[bkv][c] (block = 64 packed rows x chunk x (b, kv),
// the per-chunk arithmetic of state_simt_kernel), then chunk_scan_kernel turns Hc into the
// exclusive prefix in place, adding the chunks in order, and writes the inclusive state: the
// same sums in the same order as state_simt_kernel, so the same bits, with every chunk's
// products computed at once instead of one chunk after another.
// ------------------------------------------------------------------------------------------
// out[n][f] += sum over the 64 rows j of A[j][f] B[j][n], in row order, for one 64-row tile.
// 256 threads: thread t owns f = 4 (t & 15) .. + 3 and n = 4 (t >> 4) .. + 3 (and n = 64 for
// t < 16), reading four A and four B values per row as vectors.
__device__ __forceinline__ void tile_acc_simt(const float (*A)[68], const float (*B)[68],
                                              float (&t4)[4][4], float (&tn)[4])
{
    const int fg = threadIdx.x & 15, nq = threadIdx.x >> 4;
#pragma unroll 4
    for (int j = 0; j < 64; ++j) {
        const float4 a = *reinterpret_cast<const float4*>(&A[j][4 * fg]);
        const float4 b = *reinterpret_cast<const float4*>(&B[j][4 * nq]);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) t4[i][jj] = fmaf(av[i], bv[jj], t4[i][jj]);
        if (nq == 0) {
            const float bn = B[j][kDV];
#pragma unroll
            for (int i = 0; i < 4; ++i) tn[i] = fmaf(av[i], bn, tn[i]);
        }
    }
}

// The tile's sums to dst[n * kFP + f0 + f] (65 columns n, 64 packed rows f).
__device__ __forceinline__ void tile_store_simt(float* __restrict__ dst, int f0,
                                                const float (&t4)[4][4], const float (&tn)[4])
{
    const int fg = threadIdx.x & 15, nq = threadIdx.x >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) dst[size_t(4 * nq + jj) * kFP + f0 + 4 * fg + i] = t4[i][jj];
        if (nq == 0) dst[size_t(kDV) * kFP + f0 + 4 * fg + i] = tn[i];
    }
}

struct DeltaSmem {
    float ks[64][kDA + 1];  // k rows of the tile (and the constant 1, 0)
    float A[64][68];        // psi of the tile's rows, [token][packed row of the slab]
    float B[64][68];        // [v; 1] of the tile's rows
};

template <typename Tin>
__global__ void __launch_bounds__(256) chunk_delta_simt_kernel(const Tin* __restrict__ k,
                                                               const Tin* __restrict__ v, int T,
                                                               int C, int NC,
                                                               float* __restrict__ Hc)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DeltaSmem& sm = *reinterpret_cast<DeltaSmem*>(smem_raw);
    const int slab = blockIdx.x, bkv = blockIdx.z;
    const int tid = threadIdx.x, fi = tid & 63, cg = tid >> 6;
    const RT rt = feature_rt(slab * 64 + fi);
    const Tin* kb = k + size_t(bkv) * T * kD;
    const Tin* vb = v + size_t(bkv) * T * kDV;
    for (int c = blockIdx.y; c < NC; c += gridDim.y) {  // (gridDim.y < NC only past 65535)
        float t4[4][4], tn[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            tn[i] = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) t4[i][jj] = 0.f;
        }
        const int t0 = c * C, t1 = min(t0 + C, T);
        for (int s0 = t0; s0 < t1; s0 += 64) {
            for (int e = tid; e < 64 * kD; e += 256) {
                const int j = e / kD, r = e % kD, tok = s0 + j;
                sm.ks[j][r] = tok < t1 ? to_f32(kb[size_t(tok) * kD + r]) : 0.f;
                sm.B[j][r] = tok < t1 ? to_f32(vb[size_t(tok) * kDV + r]) : 0.f;
            }
            if (tid < 64) {
                const bool ok = s0 + tid < t1;
                sm.ks[tid][kD] = ok ? 1.f : 0.f;
                sm.ks[tid][kD + 1] = 0.f;
                sm.B[tid][kDV] = ok ? 1.f : 0.f;
            }
            __syncthreads();
            for (int j = cg; j < 64; j += 4) sm.A[j][fi] = sm.ks[j][rt.r] * sm.ks[j][rt.t];
            __syncthreads();
            tile_acc_simt(sm.A, sm.B, t4, tn);
            __syncthreads();
        }
        tile_store_simt(Hc + (size_t(bkv) * NC + c) * kW * kFP, slab * 64, t4, tn);
    }
}

// In place over X[bkv][c][n][f] (fp32, [65][2176] per chunk): the exclusive prefix over chunks
// (reverse = 0: X_c <- sum_{c' < c} X_c') or suffix (reverse = 1: X_c <- sum_{c' > c} X_c'),
// the chunks added one at a time in that order.  With `body`, the sum over all chunks goes to
// the state of (b, kv) (rows [f][64], then z[f]).  Thread = one (n, f) entry of one (b, kv).
__global__ void __launch_bounds__(256) chunk_scan_kernel(float* __restrict__ X, int NC,
                                                         int reverse, float* __restrict__ body)
{
    constexpr int kPer = kW * kFP;
    const int e = blockIdx.x * blockDim.x + threadIdx.x, bkv = blockIdx.y;
    if (e >= kPer) return;
    float* x = X + size_t(bkv) * NC * kPer + e;
    constexpr int kAhead = 8;  // chunks requested ahead of the running sum
    float run = 0.f;
    for (int i0 = 0; i0 < NC; i0 += kAhead) {
        float d[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const int i = i0 + u, c = reverse ? NC - 1 - i : i;
            d[u] = i < NC ? x[size_t(c) * kPer] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const int i = i0 + u, c = reverse ? NC - 1 - i : i;
            if (i < NC) {
                x[size_t(c) * kPer] = run;
                run += d[u];
            }
        }
    }
    if (body) {
        const int n = e / kFP, f = e - n * kFP;
        float* unit = body + size_t(bkv) * kFP * kW;
        if (n < kDV) unit[size_t(f) * kDV + n] = run;
        else unit[size_t(kFP) * kDV + f] = run;
    }
}

// The chunk states of the fp32 path: chunk-parallel when there is an Hc to hold the chunk
// sums, else the walking kernel (the final state alone).
template <typename Tin>
int launch_chunk_states_simt(const Tin* k, const Tin* v, int T, int C, int NC, float* Hc,
                             float* body, int nbkv, cudaStream_t st)
{
    if (Hc == nullptr || NC <= 1 || nbkv > 65535) {
        state_simt_kernel<Tin><<<dim3(kFP / 64, nbkv), 256, 0, st>>>(k, v, T, C, NC, Hc, body);
        OAL_LAUNCH_CHECK();
        return OAL_OK;
    }
    OAL_CUDA_TRY(cudaFuncSetAttribute(chunk_delta_simt_kernel<Tin>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(sizeof(DeltaSmem))));
    chunk_delta_simt_kernel<Tin><<<dim3(kFP / 64, std::min(NC, 65535), nbkv), 256,
                                   sizeof(DeltaSmem), st>>>(k, v, T, C, NC, Hc);
    OAL_LAUNCH_CHECK();
    chunk_scan_kernel<<<dim3((kW * kFP + 255) / 256, nbkv), 256, 0, st>>>(Hc, NC, 0, body);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

template <typename Tin>
static int launch_prefill_simt_t(const Tin* q, const Tin* k, const Tin* v,
                                 const int32_t* gid, const float* L, const int32_t* G,
                                 float eps, float* out, void* state, float* Hc, int B, int T,
                                 int Hq, int Hkv, int C, cudaStream_t st)
{
    const int NC = (T + C - 1) / C;
    float* coef = reinterpret_cast<float*>(static_cast<unsigned char*>(state) + kHeaderBytes);
    float* body = reinterpret_cast<float*>(static_cast<unsigned char*>(state) + kHeaderBytes +
                                           coef_bytes(Hq));
    {
        LaunchScope ls("state_simt", st);
        const int rc = launch_chunk_states_simt(k, v, T, C, NC, Hc, body, B * Hkv, st);
        if (rc) return rc;
    }
    if (T == 0 || out == nullptr) return OAL_OK;  // no out: the state alone is wanted
    const size_t smem = sizeof(ReadoutSmem);
    auto kern = readout_simt_kernel<Tin, false>;
    OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    LaunchScope ls("readout_simt", st);
    kern<<<dim3((T + 63) / 64, B * Hq), 256, smem, st>>>(q, k, v, gid, L, G, eps, coef, Hc, out,
                                                         Hq, Hkv, T, C, NC, nullptr);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

int launch_prefill_simt(const void* q, const void* k, const void* v, const int32_t* gid,
                        const float* L, const int32_t* G, float eps, float* out, void* state,
                        float* Hc, int B, int T, int Hq, int Hkv, int C, int dtype,
                        cudaStream_t st)
{
    if (dtype == OAL_BF16)
        return launch_prefill_simt_t(static_cast<const __nv_bfloat16*>(q),
                                     static_cast<const __nv_bfloat16*>(k),
                                     static_cast<const __nv_bfloat16*>(v), gid, L, G, eps, out,
                                     state, Hc, B, T, Hq, Hkv, C, st);
    return launch_prefill_simt_t(static_cast<const float*>(q), static_cast<const float*>(k),
                                 static_cast<const float*>(v), gid, L, G, eps, out, state, Hc,
                                 B, T, Hq, Hkv, C, st);
}

template <typename Tin>
static int launch_dense_t(const Tin* q, const Tin* k, const Tin* v, const int32_t* gid,
                          const float* L, const int32_t* G, float eps, float* out, int B, int T,
                          int Hq, int Hkv, cudaStream_t st)
{
    if (T == 0 || B == 0) return OAL_OK;
    const size_t smem = sizeof(ReadoutSmem);
    auto kern = readout_simt_kernel<Tin, true>;
    OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    LaunchScope ls("dense_simt", st);
    kern<<<dim3((T + 63) / 64, B * Hq), 256, smem, st>>>(q, k, v, gid, L, G, eps, nullptr,
                                                         nullptr, out, Hq, Hkv, T, 64, 1,
                                                         nullptr);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

int launch_dense(const void* q, const void* k, const void* v, const int32_t* gid, const float* L,
                 const int32_t* G, float eps, float* out, int B, int T, int Hq, int Hkv,
                 int dtype, cudaStream_t st)
{
    if (dtype == OAL_BF16)
        return launch_dense_t(static_cast<const __nv_bfloat16*>(q),
                              static_cast<const __nv_bfloat16*>(k),
                              static_cast<const __nv_bfloat16*>(v), gid, L, G, eps, out, B, T,
                              Hq, Hkv, st);
    return launch_dense_t(static_cast<const float*>(q), static_cast<const float*>(k),
                          static_cast<const float*>(v), gid, L, G, eps, out, B, T, Hq, Hkv, st);
}

int decode_slabs() { return (kF + kDecRows - 1) / kDecRows; }

int launch_decode(const void* q, const void* k, const void* v, void* state, float* out,
                  float* part, int B, int Hq, int Hkv, int dtype, cudaStream_t st)
{
    if (B == 0) return OAL_OK;
    const dim3 grid(decode_slabs(), B * Hkv);
    unsigned char* s = static_cast<unsigned char*>(state);
    const int grp = Hq / Hkv;
    const bool bf = dtype == OAL_BF16;
    auto go = [&](auto G) -> cudaError_t {
        constexpr int g = decltype(G)::value;
        {
            LaunchScope ls("decode", st);
            if (bf)
                decode_kernel<__nv_bfloat16, g><<<grid, kDecThreads, 0, st>>>(
                    static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                    static_cast<const __nv_bfloat16*>(v), s, out, part, Hq, Hkv);
            else
                decode_kernel<float, g><<<grid, kDecThreads, 0, st>>>(
                    static_cast<const float*>(q), static_cast<const float*>(k),
                    static_cast<const float*>(v), s, out, part, Hq, Hkv);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        LaunchScope ls("decode_finish", st);
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(B * Hkv);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, decode_finish_kernel<g>, static_cast<const float*>(part),
                                  out, s, Hq, Hkv, int(grid.x));
    };
    cudaError_t e;
    switch (grp) {
        case 1: e = go(std::integral_constant<int, 1>{}); break;
        case 2: e = go(std::integral_constant<int, 2>{}); break;
        case 3: e = go(std::integral_constant<int, 3>{}); break;
        case 4: e = go(std::integral_constant<int, 4>{}); break;
        case 5: e = go(std::integral_constant<int, 5>{}); break;
        case 6: e = go(std::integral_constant<int, 6>{}); break;
        case 7: e = go(std::integral_constant<int, 7>{}); break;
        case 8: e = go(std::integral_constant<int, 8>{}); break;
        default: return OAL_ERR_UNSUPPORTED;
    }
    OAL_CUDA_TRY(e);
    return OAL_OK;
}

int read_device_error(int* code, cudaStream_t st)
{
    int val = 0;
    OAL_CUDA_TRY(cudaMemcpyFromSymbolAsync(&val, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                  st));
    OAL_CUDA_TRY(cudaStreamSynchronize(st));
    const int zero = 0;
    OAL_CUDA_TRY(cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                                st));
    OAL_CUDA_TRY(cudaStreamSynchronize(st));
    *code = val;
    return OAL_OK;
}

}  // namespace oal
