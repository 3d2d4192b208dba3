// oal_chi.cu -- contribution statistic of eq. (1), "OAL: 按 QK 离群贡献分组的正二次注意力核"
// (reproduction note of arXiv 2610.13674), section 核心公式:
//   chi_{p,r} = (1/|Omega_p|) sum_{j<=i} |q_{p,i,r} k_{p,j,r}| / sqrt(d_h)
// per prompt p = (b, query head h), |Omega_p| = T (T + 1) / 2 causal pairs.  The pair sum
// factors as sum_i |q_{i,r}| S_{i,r} with the running sum S_{i,r} = sum_{j<=i} |k_{j,r}|, an
// O(T d) prefix scan per (b, h, r).
#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

constexpr int kChiSegs = 16;  // sequence segments per (b, h): thread = (dim, segment)

template <typename Tin>
__global__ void __launch_bounds__(kD * kChiSegs) chi_kernel(const Tin* __restrict__ q,
                                                            const Tin* __restrict__ k,
                                                            float* __restrict__ chi, int Hq,
                                                            int Hkv, int T)
{
    const int bh = blockIdx.x, b = bh / Hq, h = bh % Hq, kv = h / (Hq / Hkv);
    const int r = threadIdx.x % kD, sg = threadIdx.x / kD;
    const Tin* qh = q + size_t(bh) * T * kD + r;
    const Tin* kh = k + (size_t(b) * Hkv + kv) * T * kD + r;
    const int seg = (T + kChiSegs - 1) / kChiSegs;
    const int t0 = min(T, sg * seg), t1 = min(T, t0 + seg);
    __shared__ double segsum[kChiSegs][kD];
    __shared__ double part[kChiSegs][kD];
    // pass 1: |k| summed over this segment; pass 2: running prefix and sum_i |q_i| S_i
    double ks = 0.0;
    for (int t = t0; t < t1; ++t) ks += fabs(double(to_f32(kh[size_t(t) * kD])));
    segsum[sg][r] = ks;
    __syncthreads();
    double S = 0.0, acc = 0.0;
    for (int x = 0; x < sg; ++x) S += segsum[x][r];
    for (int t = t0; t < t1; ++t) {
        S += fabs(double(to_f32(kh[size_t(t) * kD])));
        acc = fma(fabs(double(to_f32(qh[size_t(t) * kD]))), S, acc);
    }
    part[sg][r] = acc;
    __syncthreads();
    if (sg == 0) {
        double tot = 0.0;
        for (int x = 0; x < kChiSegs; ++x) tot += part[x][r];
        const double pairs = 0.5 * double(T) * double(T + 1);
        chi[size_t(bh) * kD + r] = float(tot * 0.125 / pairs);  // 1 / sqrt(d_h), d_h = 64
    }
}

int launch_chi(const void* q, const void* k, float* chi, int B, int T, int Hq, int Hkv,
               int dtype, cudaStream_t st)
{
    if (B == 0 || T == 0) return OAL_OK;
    LaunchScope ls("chi", st);
    if (dtype == OAL_BF16)
        chi_kernel<__nv_bfloat16><<<B * Hq, kD * kChiSegs, 0, st>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), chi, Hq,
            Hkv, T);
    else
        chi_kernel<float><<<B * Hq, kD * kChiSegs, 0, st>>>(static_cast<const float*>(q),
                                                             static_cast<const float*>(k), chi,
                                                             Hq, Hkv, T);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

}  // namespace oal
