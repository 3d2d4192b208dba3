// oal_common.cuh -- shared definitions of the OAL CUDA library (sm_100a).
//
// Packed feature map.  With qhat = [q; 1] and khat = [k; 1] (65 entries), eq. (3) of the OAL
// reproduction note (section 核心公式) expands to
//     kappa(q, k) = sum_{r<=t} Cp_rt (qhat_r qhat_t) (khat_r khat_t),
//     Cp_rt = (r == t ? 1 : 2) * M_{g(r),g(t)} * sc_r * sc_t  (+ eps on the (64,64) entry),
// where M = L L^T, g(64) = 0, sc_r = 1/sqrt(d_h) for r < 64 and sc_64 = 1.  The 65*66/2 = 2145
// products khat_r khat_t (r <= t) are exactly the rows of the eq. (4) prefix states
// (H2_rt for r,t < 64, H1_r for t = 64, H0 for r = t = 64), and phi_f(q) = Cp_f qhat_r qhat_t
// collects a, b_r/sqrt(d_h) and C_rt/d_h of eq. (5).  So one packed state S (2145 rows x
// [v; 1]) carries H0, H1 and the symmetric-packed H2, and u_i = phi(q_i)^T S_i.
//
// Packed order of the 2176 (= 17 * 128) feature rows:
//   [0, 1792)     28 off-diagonal 8x8 blocks (R < T of the 8 dim-blocks), 64 rows each:
//                 f = 64*beta + 8*a + b  <->  (r, t) = (8R + a, 8T + b)
//   [1792, 2080)  8 diagonal blocks, 36 rows each: (8R + a, 8R + b), a <= b
//   [2080, 2144)  linear rows (r, 64)
//   2144          constant row (64, 64)
//   [2145, 2176)  padding, (65, 65) with khat_65 = qhat_65 = 0: always zero
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/oal.h"
#include "oal_prof.cuh"

namespace oal {

constexpr int kD = OAL_HEAD_DIM;        // 64
constexpr int kDV = OAL_VALUE_DIM;      // 64
constexpr int kDA = kD + 2;             // augmented q/k length incl. the 1 and a 0 pad slot
constexpr int kW = kDV + 1;             // [v; 1]
constexpr int kGMax = OAL_G_MAX;        // 8
constexpr int kGM1 = kGMax + 1;         // L slot side
constexpr int kF = OAL_FEATURES;        // 2145
constexpr int kFP = OAL_FEATURES_PAD;   // 2176
constexpr int kOffDiagRows = 1792;
constexpr int kDiagRows = 288;
constexpr int kLinStart = 2080;
constexpr int kConstRow = 2144;
constexpr int kMaxGroup = 8;            // Hq / Hkv supported

// Per-query-head table of the tensor-core readout, written into the prefill workspace by the
// coefficient expansion (a1) and copied into shared memory once per readout item:
constexpr uint32_t kTabCoefH = 0;      // bf16 [1792]: coefficients of the off-diagonal rows
constexpr uint32_t kTabCoefT = 3584;   // fp32 [384]: coefficients of rows 1792..2175
constexpr uint32_t kTabW = 5120;       // fp32 [9][64]: L_{g(r),m} / sqrt(d_h) (0 for m > G)
constexpr uint32_t kTabC0 = 7424;      // fp32 [9]: L_{0,m} (0 for m > G)
constexpr uint32_t kTabG = 7460;       // int32: G of the head (clamped to 1..8)
constexpr uint32_t kTabPure = 7464;    // uint8 [8]: 1 if the 8 dims of block R share one group
constexpr uint32_t kTabBytes = 7680;   // a multiple of 256

constexpr uint32_t kStateMagic = 0x534C414Fu;  // "OALS"
constexpr size_t kHeaderBytes = 256;

struct StateHeader {
    uint32_t magic;
    int32_t abi;
    int32_t B, Hq, Hkv, dh, dv, feat_pad;
    long long tokens;
    float eps;
    int32_t reserved[53];
};
static_assert(sizeof(StateHeader) == kHeaderBytes, "header must be 256 bytes");

__host__ __device__ constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ constexpr size_t coef_bytes(int Hq) { return align256(size_t(Hq) * kFP * 4); }
__host__ __device__ constexpr size_t state_unit_bytes() { return size_t(kFP) * kW * 4; }
__host__ __device__ constexpr size_t state_bytes(int B, int Hq, int Hkv) {
    return kHeaderBytes + coef_bytes(Hq) + size_t(B) * Hkv * state_unit_bytes();
}

// (r, t) of packed feature row f; padding rows map to (65, 65).
struct RT { int r, t; };

__host__ __device__ constexpr RT feature_rt(int f) {
    if (f < kOffDiagRows) {
        int beta = f >> 6, R = 0, s = 0;
        while (beta >= s + 7 - R) { s += 7 - R; ++R; }
        const int T = R + 1 + (beta - s);
        return RT{8 * R + ((f >> 3) & 7), 8 * T + (f & 7)};
    }
    if (f < kLinStart) {
        const int e = f - kOffDiagRows, R = e / 36;
        int p = e - 36 * R, a = 0;
        while (p >= 8 - a) { p -= 8 - a; ++a; }
        return RT{8 * R + a, 8 * R + a + p};
    }
    if (f < kConstRow) return RT{f - kLinStart, kD};
    if (f == kConstRow) return RT{kD, kD};
    return RT{kD + 1, kD + 1};
}

// Device-side error word (OAL_OK or a negative oal_status); first error wins.  The library
// is built as one translation unit (oal_lib.cu), so this is the only copy.
__device__ int g_device_error = 0;

__device__ __forceinline__ void raise_error(int code) { atomicCAS(&g_device_error, 0, code); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

// The CUDA error behind the most recent OAL_ERR_CUDA (process-wide, last writer wins).
inline std::atomic<int>& last_cuda_error()
{
    static std::atomic<int> e{0};
    return e;
}

inline int cuda_fail(cudaError_t e)
{
    last_cuda_error().store(int(e));
    return OAL_ERR_CUDA;
}

// Launch-side error check: returns OAL_ERR_CUDA from the calling function.
#define OAL_LAUNCH_CHECK()                                \
    do {                                                  \
        const cudaError_t oal_e_ = cudaGetLastError();    \
        if (oal_e_ != cudaSuccess) return cuda_fail(oal_e_); \
    } while (0)

// Evaluates a CUDA runtime call; on failure returns OAL_ERR_CUDA from the calling function.
#define OAL_CUDA_TRY(call)                                \
    do {                                                  \
        const cudaError_t oal_e_ = (call);                \
        if (oal_e_ != cudaSuccess) return cuda_fail(oal_e_); \
    } while (0)

}  // namespace oal
