// oal_hadamard.cu -- the ungrouped Hadamard form on the CUDA-core path.
//
// "Not All Dimensions Are Equal: Outlier-Aware Attention Linearization with Grouped Quadratic
// Kernels" (arXiv 2610.13674, abstract) relaxes the second-order Taylor kernel's shared
// coefficients into per-dimension linear terms and cross-dimensional quadratic terms; eq. (5)
// of "OAL: 按 QK 离群贡献分组的正二次注意力核" (section 核心公式) is that form's readout with free
// coefficients a, b_r, C_rt.  Summing eq. (4) inside eq. (5), the kernel it evaluates is
//   kappa(q, k) = a + sum_r b_r x_r + sum_{r,t} C_rt x_r x_t,   x_r = q_r k_r / sqrt(d_h),
// which need not be positive; yhat = u[:dv] / u[dv] is a plain division.
//
// Only two steps differ from the grouped kernel:
//  - the packed coefficient table (prep_hadamard_kernel) comes from (a, b, C) instead of L L^T;
//    the chunk states (state_simt_kernel) carry no coefficients and are shared as they are;
//  - the intra-chunk kernel values (readout_hadamard_kernel) are a + x . (b + C x).
// The decode step reads only the coefficient table and the packed state, so oal_decode_step
// continues a sequence prefilled here unchanged.
#pragma once

#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

// Packed readout weight of row f (r <= t of qhat = [q; 1]) such that
// sum_f coef_f qhat_r qhat_t khat_r khat_t = a + sum_r b_r x_r + sum_{r,t} C_rt x_r x_t:
//   (64, 64): a;  (r, 64): b_r / sqrt(d_h);  (r, r): C_rr / d_h;  (r < t): (C_rt + C_tr) / d_h.
// One block per query head; block 0 also writes the state header (eps = 0: a holds the
// constant term).
__global__ void __launch_bounds__(256) prep_hadamard_kernel(const float* __restrict__ a,
                                                            const float* __restrict__ b,
                                                            const float* __restrict__ C,
                                                            unsigned char* __restrict__ state,
                                                            int B, int Hq, int Hkv,
                                                            long long tokens,
                                                            unsigned char* __restrict__ rtab)
{
    const int h = blockIdx.x, tid = threadIdx.x;
    const float* bh = b + size_t(h) * kD;
    const float* Ch = C + size_t(h) * kD * kD;
    float* coef = reinterpret_cast<float*>(state + kHeaderBytes) + size_t(h) * kFP;
    for (int f = tid; f < kFP; f += blockDim.x) {
        double val = 0.0;
        if (f < kF) {
            const RT rt = feature_rt(f);
            if (rt.r == kD) val = double(a[h]);
            else if (rt.t == kD) val = double(bh[rt.r]) * 0.125;
            else if (rt.r == rt.t) val = double(Ch[rt.r * kD + rt.r]) / 64.0;
            else val = (double(Ch[rt.r * kD + rt.t]) + double(Ch[rt.t * kD + rt.r])) / 64.0;
        }
        coef[f] = float(val);
        if (rtab) {  // tensor-core readout table: bf16 off-diagonal coefficients, fp32 the rest
            unsigned char* tb = rtab + size_t(h) * kTabBytes;
            if (f < kOffDiagRows)
                reinterpret_cast<__nv_bfloat16*>(tb + kTabCoefH)[f] = __float2bfloat16_rn(float(val));
            else
                reinterpret_cast<float*>(tb + kTabCoefT)[f - kOffDiagRows] = float(val);
        }
    }
    if (rtab) {  // no 8-dim block shares its weights across rows ("pure" flags 0), rest zero
        unsigned char* tb = rtab + size_t(h) * kTabBytes;
        for (uint32_t x = kTabW + tid; x < kTabBytes; x += blockDim.x) tb[x] = 0;
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
        hd->tokens = tokens;
        hd->eps = 0.f;
        for (int i = 0; i < int(sizeof(hd->reserved) / sizeof(hd->reserved[0])); ++i)
            hd->reserved[i] = 0;
    }
}

struct HadamardSmem {
    float qs[64][kDA + 1];
    float ps[64][65];
    union {
        InterTiles t;
        struct {
            float ks[64][kD + 1];
            float vs[64][kW];
        } kv;
    } u;
    float Cs[kD][kD];  // C of this head, row r, column t
    float bs[kD];
    float as;
};

// Readout of 64 query rows of one (b, h), as readout_simt_kernel with the Hadamard kernel:
// inter (prefill only): u_i += phi(q_i)^T S_c from the packed coefficient table and the fp32
// chunk state; intra: u_i += sum_{j in [j0, i]} kappa_ij [v_j; 1] with
// kappa_ij = a + sum_r x_r (b_r + sum_t C_rt x_t); then yhat_i = u_i[0:64] / u_i[64].
// Thread (ri = row, cg = column group): columns n = cg + 4u of u.
template <typename Tin, bool kDense>
__global__ void __launch_bounds__(256) readout_hadamard_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ a, const float* __restrict__ b, const float* __restrict__ C,
    const float* __restrict__ coef, const float* __restrict__ Hc, float* __restrict__ out,
    int Hq, int Hkv, int T, int Cn, int NC)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    HadamardSmem& sm = *reinterpret_cast<HadamardSmem*>(smem_raw);
    const int tile = blockIdx.x, bh = blockIdx.y;
    const int b_ = bh / Hq, h = bh % Hq, kv = h / (Hq / Hkv), bkv = b_ * Hkv + kv;
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
    for (int e = tid; e < kD * kD; e += 256) (&sm.Cs[0][0])[e] = C[size_t(h) * kD * kD + e];
    if (tid < kD) sm.bs[tid] = b[size_t(h) * kD + tid];
    if (tid == 0) sm.as = a[h];
    __syncthreads();

    float acc[17];
#pragma unroll
    for (int u = 0; u < 17; ++u) acc[u] = 0.f;

    const int c = i0 / Cn;
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

    const int j0 = kDense ? 0 : c * Cn;
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
                float x[kD];
#pragma unroll
                for (int t = 0; t < kD; ++t) x[t] = sm.qs[ri][t] * sm.u.kv.ks[key][t] * 0.125f;
                kap = sm.as;
                for (int r = 0; r < kD; ++r) {
                    float y = sm.bs[r];
#pragma unroll
                    for (int t = 0; t < kD; ++t) y = fmaf(sm.Cs[r][t], x[t], y);
                    kap = fmaf(sm.qs[ri][r] * sm.u.kv.ks[key][r] * 0.125f, y, kap);
                }
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
    }
}

template <typename Tin>
static int launch_hadamard_t(const Tin* q, const Tin* k, const Tin* v, const float* a,
                             const float* b, const float* C, float* out, void* state,
                             float* Hc, int B, int T, int Hq, int Hkv, int Cn, bool dense,
                             cudaStream_t st)
{
    const size_t smem = sizeof(HadamardSmem);
    if (!dense) {
        {
            LaunchScope ls("prep_hadamard", st);
            prep_hadamard_kernel<<<Hq, 256, 0, st>>>(a, b, C, static_cast<unsigned char*>(state),
                                                    B, Hq, Hkv, T, nullptr);
            OAL_LAUNCH_CHECK();
        }
        if (B == 0) return OAL_OK;
        float* body = reinterpret_cast<float*>(static_cast<unsigned char*>(state) +
                                               kHeaderBytes + coef_bytes(Hq));
        const int NC = (T + Cn - 1) / Cn;
        {
            LaunchScope ls("state_simt", st);
            const int rc = launch_chunk_states_simt(k, v, T, Cn, NC, Hc, body, B * Hkv, st);
            if (rc) return rc;
        }
        if (T == 0) return OAL_OK;
        const float* coef = reinterpret_cast<const float*>(static_cast<unsigned char*>(state) +
                                                           kHeaderBytes);
        auto kern = readout_hadamard_kernel<Tin, false>;
        OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          int(smem)));
        LaunchScope ls("readout_hadamard", st);
        kern<<<dim3((T + 63) / 64, B * Hq), 256, smem, st>>>(q, k, v, a, b, C, coef, Hc, out, Hq,
                                                             Hkv, T, Cn, NC);
        OAL_LAUNCH_CHECK();
        return OAL_OK;
    }
    if (T == 0 || B == 0) return OAL_OK;
    auto kern = readout_hadamard_kernel<Tin, true>;
    OAL_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(smem)));
    LaunchScope ls("dense_hadamard", st);
    kern<<<dim3((T + 63) / 64, B * Hq), 256, smem, st>>>(q, k, v, a, b, C, nullptr, nullptr, out,
                                                         Hq, Hkv, T, 64, 1);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

int launch_hadamard(const void* q, const void* k, const void* v, const float* a, const float* b,
                    const float* C, float* out, void* state, float* Hc, int B, int T, int Hq,
                    int Hkv, int Cn, int dtype, bool dense, cudaStream_t st)
{
    if (dtype == OAL_BF16)
        return launch_hadamard_t(static_cast<const __nv_bfloat16*>(q),
                                 static_cast<const __nv_bfloat16*>(k),
                                 static_cast<const __nv_bfloat16*>(v), a, b, C, out, state, Hc,
                                 B, T, Hq, Hkv, Cn, dense, st);
    return launch_hadamard_t(static_cast<const float*>(q), static_cast<const float*>(k),
                             static_cast<const float*>(v), a, b, C, out, state, Hc, B, T, Hq,
                             Hkv, Cn, dense, st);
}

}  // namespace oal

extern "C" {

int oal_prefill_hadamard(const void* q, const void* k, const void* v, const float* a,
                         const float* b, const float* C, float* out, void* state,
                         void* workspace, size_t workspace_bytes, const oal_shape* s,
                         void* stream)
{
    using namespace oal;
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_chunk(s))) return rc;
    const bool tensor = use_tensor_path(s) && out != nullptr;
    if ((rc = tensor ? check_prefill_planes(s) : check_planes((long long)s->B * s->Hq)))
        return rc;
    if (!a || !b || !C || !state) return OAL_ERR_NULL;
    if ((rc = check_io(s, q, k, v, out))) return rc;
    if (!aligned16(a) || !aligned16(b) || !aligned16(C) || !aligned16(state)) return OAL_ERR_ALIGN;
    const size_t need = tensor ? tc_workspace_bytes(s->B, s->Hq, s->Hkv, s->T)
                               : simt_chunk_state_bytes(s);
    if (need > 0 && (!workspace || workspace_bytes < need)) return OAL_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return OAL_ERR_ALIGN;
    if (tensor) {
        // the coefficient tables (state and readout) first; then the tensor-core prefill with
        // the intra-chunk part through the feature map
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        {
            LaunchScope ls("prep_hadamard", st);
            prep_hadamard_kernel<<<s->Hq, 256, 0, st>>>(
                a, b, C, static_cast<unsigned char*>(state), s->B, s->Hq, s->Hkv, s->T,
                tc_rtab(workspace, s->B, s->Hkv, s->T));
            OAL_LAUNCH_CHECK();
        }
        return launch_prefill_tc(q, k, v, nullptr, nullptr, nullptr, 0.f, out, state, workspace,
                                 s->B, s->T, s->Hq, s->Hkv, g_prefill_overlap.load() != 0, false,
                                 st, true);
    }
    return launch_hadamard(q, k, v, a, b, C, out, state, static_cast<float*>(workspace), s->B,
                           s->T, s->Hq, s->Hkv, s->chunk, s->dtype, false,
                           static_cast<cudaStream_t>(stream));
}

int oal_dense_hadamard_gpu(const void* q, const void* k, const void* v, const float* a,
                           const float* b, const float* C, float* out, const oal_shape* s,
                           void* stream)
{
    using namespace oal;
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hq))) return rc;
    if (!a || !b || !C) return OAL_ERR_NULL;
    if ((rc = check_io(s, q, k, v, out))) return rc;
    if (!aligned16(a) || !aligned16(b) || !aligned16(C)) return OAL_ERR_ALIGN;
    return launch_hadamard(q, k, v, a, b, C, out, nullptr, nullptr, s->B, s->T, s->Hq, s->Hkv,
                           64, s->dtype, true, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
