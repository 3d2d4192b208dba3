// oal_stateops.cu -- sums of prefix states.
//
// The prefix state of eq. (4) ("OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式) is a
// sum over tokens, so the state of a sequence's first segments is the sum of the states those
// segments produce alone; a sequence-parallel prefill combines the gathered segment states
// this way.  out[i] = parts[0][i] + parts[1][i] + ... + parts[n_parts-1][i], added in that
// order (bit-reproducible).  Memory-bound: float4 loads, a grid of a few waves.
#pragma once

#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

__global__ void __launch_bounds__(256) state_prefix_sum_kernel(const float* __restrict__ parts,
                                                               int n_parts, size_t n,
                                                               float* __restrict__ out)
{
    const size_t n4 = n / 4;
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < n_parts; ++r) {
            const float4 p = __ldcs(reinterpret_cast<const float4*>(parts + size_t(r) * n) + i);
            s.x += p.x;
            s.y += p.y;
            s.z += p.z;
            s.w += p.w;
        }
        reinterpret_cast<float4*>(out)[i] = s;
    }
    for (size_t i = 4 * n4 + size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        float s = 0.f;
        for (int r = 0; r < n_parts; ++r) s += parts[size_t(r) * n + i];
        out[i] = s;
    }
}

}  // namespace oal

extern "C" {

int oal_state_prefix_sum(const float* parts, int n_parts, size_t n, float* out, void* stream)
{
    using namespace oal;
    if (n_parts < 0) return OAL_ERR_SHAPE;
    if (n == 0) return OAL_OK;
    if (!out || (n_parts > 0 && !parts)) return OAL_ERR_NULL;
    if ((n_parts > 0 && !aligned16(parts)) || !aligned16(out) || (n_parts > 0 && n % 4 != 0))
        return OAL_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t n4 = (n + 3) / 4;
    const int blocks = int(std::min<size_t>((n4 + 255) / 256, size_t(sm_count()) * 8));
    LaunchScope ls("state_prefix_sum", st);
    state_prefix_sum_kernel<<<std::max(blocks, 1), 256, 0, st>>>(parts, n_parts, n, out);
    OAL_LAUNCH_CHECK();
    return OAL_OK;
}

}  // extern "C"
