// oal_backward.cu -- gradients of the dense causal form, on CUDA cores (reference scale).
//
// "OAL: 按 QK 离群贡献分组的正二次注意力核" trains the kernel coefficients jointly with the
// model (its pipeline figure: LoRA and kernel parameters trained together); the pages print
// no gradient.  This is the chain rule through eqs. (2)-(3) summed over j <= i and
// normalised: with D_i = sum_{j<=i} kappa_ij and yhat_i = sum_{j<=i} kappa_ij v_j / D_i,
//   dkappa_ij = dy_i . (v_j - yhat_i) / D_i,        dv_j += kappa_ij dy_i / D_i,
//   dkappa/dsbar = 2 M sbar,  ds_g/dq_ir = [g(r) = g] k_jr / sqrt(d_h)  (and q <-> k),
//   dM += dkappa sbar sbar^T,  deps += dkappa,  dL = (dM + dM^T) L.
// Three passes, each thread owning what it writes, so the result does not depend on timing:
//   rows  (thread = (b, h, i)):  D_i, yhat_i, dq_i, and the row's partial dM and deps;
//   keys  (thread = (b, kv, j)): dk_j, dv_j over the query heads of the group and rows i >= j;
//   heads (block = h):           dM_h and deps_h summed over (b, i) in order, dL_h; then one
//                                thread sums deps over the heads.
// Work is O(B Hq T^2 d_h): this is the reference-scale gradient, not the training-scale one.
#pragma once

#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

constexpr int kBwdThreads = 128;
constexpr int kMM = kGM1 * kGM1;  // 81 entries of M or dM

struct BwdArgs {
    int B, T, Hq, Hkv;
    float eps;
    const int32_t* gid;
    const float* L;
    const int32_t* G;
    const float* dy;
    float* dq;
    float* dk;
    float* dv;
    float* dL;
    float* deps;
    float* rowD;    // [B][Hq][T]
    float* rowY;    // [B][Hq][T][64]
    float* rowM;    // [B][Hq][T][81]
    float* rowE;    // [B][Hq][T]
    float* headE;   // [Hq]
};

// M = L L^T of head h (leading (G+1) block) into m[81], group ids into g[64]; out-of-range
// values raise OAL_ERR_GROUPS and are clamped.  Returns G.
__device__ __forceinline__ int bwd_head_setup(const BwdArgs& A, int h, float* m, int* g)
{
    int Gh = A.G[h];
    if (Gh < 1 || Gh > kGMax) {
        raise_error(OAL_ERR_GROUPS);
        Gh = Gh < 1 ? 1 : kGMax;
    }
    for (int r = 0; r < kD; ++r) {
        int x = A.gid[h * kD + r];
        if (x < 1 || x > Gh) {
            raise_error(OAL_ERR_GROUPS);
            x = x < 1 ? 1 : Gh;
        }
        g[r] = x;
    }
    const float* Lh = A.L + size_t(h) * kMM;
    for (int a = 0; a < kGM1; ++a)
        for (int c = 0; c < kGM1; ++c) {
            float acc = 0.f;
            if (a <= Gh && c <= Gh)
                for (int mm = 0; mm <= Gh; ++mm) acc = fmaf(Lh[a * kGM1 + mm], Lh[c * kGM1 + mm], acc);
            m[a * kGM1 + c] = acc;
        }
    return Gh;
}

// kappa of one pair (eqs. (2)-(3)); leaves sbar and M sbar.
template <typename Tin>
__device__ __forceinline__ float bwd_kappa(const Tin* qi, const Tin* kj, const int* g,
                                           const float* m, int Gh, float eps, float* sb,
                                           float* ms)
{
    for (int c = 0; c < kGM1; ++c) sb[c] = 0.f;
    sb[0] = 1.f;
    for (int r = 0; r < kD; ++r) sb[g[r]] = fmaf(to_f32(qi[r]) * to_f32(kj[r]), 0.125f, sb[g[r]]);
    float kap = eps;
    for (int c = 0; c <= Gh; ++c) {
        float acc = 0.f;
        for (int e = 0; e <= Gh; ++e) acc = fmaf(m[c * kGM1 + e], sb[e], acc);
        ms[c] = acc;
        kap = fmaf(sb[c], acc, kap);
    }
    return kap;
}

template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads) bwd_rows_kernel(const Tin* __restrict__ q,
                                                               const Tin* __restrict__ k,
                                                               const Tin* __restrict__ v,
                                                               BwdArgs A)
{
    const int bh = blockIdx.y, b = bh / A.Hq, h = bh % A.Hq, kv = h / (A.Hq / A.Hkv);
    const int i = blockIdx.x * kBwdThreads + threadIdx.x;
    __shared__ float m[kMM];
    __shared__ int g[kD];
    __shared__ int sG;
    if (threadIdx.x == 0) sG = bwd_head_setup(A, h, m, g);
    __syncthreads();
    if (i >= A.T) return;
    const int Gh = sG;
    const Tin* qi = q + (size_t(bh) * A.T + i) * kD;
    const Tin* kb = k + size_t(b * A.Hkv + kv) * A.T * kD;
    const Tin* vb = v + size_t(b * A.Hkv + kv) * A.T * kDV;
    const float* gi = A.dy + (size_t(bh) * A.T + i) * kDV;
    float sb[kGM1], ms[kGM1];
    // pass 1: normaliser and output of row i
    float y[kDV];
    for (int n = 0; n < kDV; ++n) y[n] = 0.f;
    float D = 0.f;
    for (int j = 0; j <= i; ++j) {
        const float kap = bwd_kappa(qi, kb + size_t(j) * kD, g, m, Gh, A.eps, sb, ms);
        D += kap;
        for (int n = 0; n < kDV; ++n) y[n] = fmaf(kap, to_f32(vb[size_t(j) * kDV + n]), y[n]);
    }
    for (int n = 0; n < kDV; ++n) y[n] /= D;
    // pass 2: dq_i, this row's dM and deps
    float dqr[kD], dM[kMM];
    for (int r = 0; r < kD; ++r) dqr[r] = 0.f;
    for (int e = 0; e < kMM; ++e) dM[e] = 0.f;
    float de = 0.f;
    for (int j = 0; j <= i; ++j) {
        const Tin* kj = kb + size_t(j) * kD;
        bwd_kappa(qi, kj, g, m, Gh, A.eps, sb, ms);
        float dk_ = 0.f;
        for (int n = 0; n < kDV; ++n) dk_ = fmaf(gi[n], to_f32(vb[size_t(j) * kDV + n]) - y[n], dk_);
        dk_ /= D;
        for (int r = 0; r < kD; ++r) dqr[r] = fmaf(dk_ * 2.f * ms[g[r]] * 0.125f, to_f32(kj[r]), dqr[r]);
        for (int c = 0; c <= Gh; ++c)
            for (int e = 0; e <= Gh; ++e) dM[c * kGM1 + e] = fmaf(dk_ * sb[c], sb[e], dM[c * kGM1 + e]);
        de += dk_;
    }
    const size_t row = size_t(bh) * A.T + i;
    for (int r = 0; r < kD; ++r) A.dq[row * kD + r] = dqr[r];
    for (int n = 0; n < kDV; ++n) A.rowY[row * kDV + n] = y[n];
    for (int e = 0; e < kMM; ++e) A.rowM[row * kMM + e] = dM[e];
    A.rowD[row] = D;
    A.rowE[row] = de;
}

template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads) bwd_keys_kernel(const Tin* __restrict__ q,
                                                               const Tin* __restrict__ k,
                                                               const Tin* __restrict__ v,
                                                               BwdArgs A)
{
    const int bkv = blockIdx.y, b = bkv / A.Hkv, kv = bkv % A.Hkv, grp = A.Hq / A.Hkv;
    const int j = blockIdx.x * kBwdThreads + threadIdx.x;
    __shared__ float m[kMaxGroup][kMM];
    __shared__ int g[kMaxGroup][kD];
    __shared__ int sG[kMaxGroup];
    if (threadIdx.x < grp) sG[threadIdx.x] = bwd_head_setup(A, kv * grp + threadIdx.x,
                                                            m[threadIdx.x], g[threadIdx.x]);
    __syncthreads();
    if (j >= A.T) return;
    const Tin* kj = k + (size_t(bkv) * A.T + j) * kD;
    const Tin* vj = v + (size_t(bkv) * A.T + j) * kDV;
    float dkr[kD], dvr[kDV], sb[kGM1], ms[kGM1];
    for (int r = 0; r < kD; ++r) dkr[r] = 0.f;
    for (int n = 0; n < kDV; ++n) dvr[n] = 0.f;
    for (int x = 0; x < grp; ++x) {
        const int h = kv * grp + x, bh = b * A.Hq + h;
        for (int i = j; i < A.T; ++i) {
            const size_t row = size_t(bh) * A.T + i;
            const Tin* qi = q + row * kD;
            const float kap = bwd_kappa(qi, kj, g[x], m[x], sG[x], A.eps, sb, ms);
            const float* gi = A.dy + row * kDV;
            const float* yi = A.rowY + row * kDV;
            const float invD = 1.f / A.rowD[row];
            float dk_ = 0.f;
            for (int n = 0; n < kDV; ++n) {
                dk_ = fmaf(gi[n], to_f32(vj[n]) - yi[n], dk_);
                dvr[n] = fmaf(kap * invD, gi[n], dvr[n]);
            }
            dk_ *= invD;
            for (int r = 0; r < kD; ++r)
                dkr[r] = fmaf(dk_ * 2.f * ms[g[x][r]] * 0.125f, to_f32(qi[r]), dkr[r]);
        }
    }
    for (int r = 0; r < kD; ++r) A.dk[(size_t(bkv) * A.T + j) * kD + r] = dkr[r];
    for (int n = 0; n < kDV; ++n) A.dv[(size_t(bkv) * A.T + j) * kDV + n] = dvr[n];
}

// dM_h and deps_h summed over (b, i) in order; dL_h = (dM + dM^T) L over the live block.
__global__ void __launch_bounds__(kMM) bwd_heads_kernel(BwdArgs A)
{
    const int h = blockIdx.x, e = threadIdx.x;
    __shared__ float dM[kMM];
    __shared__ int sG;
    if (e == 0) {
        int Gh = A.G[h];
        sG = Gh < 1 ? 1 : (Gh > kGMax ? kGMax : Gh);
    }
    float s = 0.f, de = 0.f;
    for (int b = 0; b < A.B; ++b)
        for (int i = 0; i < A.T; ++i) {
            const size_t row = (size_t(b) * A.Hq + h) * A.T + i;
            s += A.rowM[row * kMM + e];
            if (e == 0) de += A.rowE[row];
        }
    dM[e] = s;
    __syncthreads();
    const int Gh = sG, a = e / kGM1, mm = e % kGM1;
    float val = 0.f;
    if (a <= Gh && mm <= Gh) {
        const float* Lh = A.L + size_t(h) * kMM;
        for (int c = 0; c <= Gh; ++c) val = fmaf(dM[a * kGM1 + c] + dM[c * kGM1 + a], Lh[c * kGM1 + mm], val);
    }
    A.dL[size_t(h) * kMM + e] = val;
    if (e == 0) A.headE[h] = de;
}

__global__ void bwd_eps_kernel(BwdArgs A)
{
    float s = 0.f;
    for (int h = 0; h < A.Hq; ++h) s += A.headE[h];
    *A.deps = s;
}

size_t bwd_workspace_bytes(int B, int T, int Hq)
{
    const size_t rows = size_t(B) * Hq * T;
    return align256(rows * 4) + align256(rows * kDV * 4) + align256(rows * kMM * 4) +
           align256(rows * 4) + align256(size_t(Hq) * 4);
}

template <typename Tin>
static int launch_backward_t(const Tin* q, const Tin* k, const Tin* v, BwdArgs A,
                             cudaStream_t st)
{
    if (A.B > 0 && A.T > 0) {
        {
            LaunchScope ls("backward_rows", st);
            bwd_rows_kernel<Tin><<<dim3((A.T + kBwdThreads - 1) / kBwdThreads, A.B * A.Hq),
                                   kBwdThreads, 0, st>>>(q, k, v, A);
            OAL_LAUNCH_CHECK();
        }
        {
            LaunchScope ls("backward_keys", st);
            bwd_keys_kernel<Tin><<<dim3((A.T + kBwdThreads - 1) / kBwdThreads, A.B * A.Hkv),
                                   kBwdThreads, 0, st>>>(q, k, v, A);
            OAL_LAUNCH_CHECK();
        }
    }
    {
        LaunchScope ls("backward_heads", st);
        bwd_heads_kernel<<<A.Hq, kMM, 0, st>>>(A);
        OAL_LAUNCH_CHECK();
    }
    LaunchScope ls("backward_eps", st);
    bwd_eps_kernel<<<1, 1, 0, st>>>(A);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

int launch_backward(const void* q, const void* k, const void* v, BwdArgs A, int dtype,
                    cudaStream_t st)
{
    if (dtype == OAL_BF16)
        return launch_backward_t(static_cast<const __nv_bfloat16*>(q),
                                 static_cast<const __nv_bfloat16*>(k),
                                 static_cast<const __nv_bfloat16*>(v), A, st);
    return launch_backward_t(static_cast<const float*>(q), static_cast<const float*>(k),
                             static_cast<const float*>(v), A, st);
}

}  // namespace oal

extern "C" {

int oal_dense_backward_workspace_bytes(const oal_shape* s, size_t* bytes)
{
    using namespace oal;
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hq))) return rc;
    if (!bytes) return OAL_ERR_NULL;
    *bytes = bwd_workspace_bytes(s->B, s->T, s->Hq);
    return OAL_OK;
}

int oal_dense_backward_gpu(const void* q, const void* k, const void* v, const int32_t* group_id,
                           const float* L, const int32_t* G, float eps, const float* dy,
                           float* dq, float* dk, float* dv, float* dL, float* deps,
                           void* workspace, size_t workspace_bytes, const oal_shape* s,
                           void* stream)
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
    const size_t need = bwd_workspace_bytes(s->B, s->T, s->Hq);
    if (!workspace || workspace_bytes < need) return OAL_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return OAL_ERR_ALIGN;
    const size_t rows = size_t(s->B) * s->Hq * s->T;
    unsigned char* w = static_cast<unsigned char*>(workspace);
    BwdArgs A;
    A.B = s->B;
    A.T = s->T;
    A.Hq = s->Hq;
    A.Hkv = s->Hkv;
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
    A.rowD = reinterpret_cast<float*>(w);
    w += align256(rows * 4);
    A.rowY = reinterpret_cast<float*>(w);
    w += align256(rows * kDV * 4);
    A.rowM = reinterpret_cast<float*>(w);
    w += align256(rows * kMM * 4);
    A.rowE = reinterpret_cast<float*>(w);
    w += align256(rows * 4);
    A.headE = reinterpret_cast<float*>(w);
    return launch_backward(q, k, v, A, s->dtype, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
