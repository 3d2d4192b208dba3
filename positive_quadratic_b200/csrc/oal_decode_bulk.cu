// oal_decode_bulk.cu -- decode step whose state slab reaches shared memory by bulk copies.
//
// The arithmetic, the partition and the summation order are those of decode_kernel
// (oal_simt.cu), so both kernels give bit-identical results ("OAL: 按 QK 离群贡献分组的正二次注意力核",
// section 核心公式, eq. (4) with one new token, then eq. (5)).  For each (b, kv) head, slab s holds
// packed rows [240 s, 240 s + 240).  Each row of Hv gets psi_f(k) v added, z gets psi_f(k), and
// the updated row is read out against phi_{h,f}(q_h) for the Hq/Hkv query heads of that kv head.
//
// What differs is how the slab's 61 KB of Hv rows and its z entries reach the SM. At block start,
// one thread issues five 12 KB bulk copies (cp.async.bulk global -> shared, each completing on
// its own mbarrier) plus the 960-byte z slab. So the whole slab is in flight while the block
// loads q, k and v and forms psi and phi. Each 48-row part is consumed as soon as its copy lands.
// Updated rows leave through streaming 128-bit stores from registers, as in decode_kernel. The
// register-batched loads of decode_kernel keep at most 16 KB per block in flight; this kernel
// keeps the whole slab in flight.  Two blocks share an SM (about 78 KB of shared memory each).
#pragma once

#include <atomic>

#include "oal_common.cuh"
#include "oal_kernels.cuh"
#include "oal_tc_util.cuh"

namespace oal {

constexpr int kDbRows = kDecRows;                                         // 240, as decode_kernel
constexpr int kDbParts = 5;
constexpr int kDbPartRows = kDbRows / kDbParts;                           // 48 = 3 x 16 rows
constexpr uint32_t kDbPartBytes = uint32_t(kDbPartRows) * kDV * sizeof(float);  // 12288
constexpr uint32_t kDbZBytes = uint32_t(kDbRows) * sizeof(float);               // 960
constexpr size_t kDbSmemBytes = size_t(kDbRows) * kDV * sizeof(float) + kDbZBytes;

static_assert(kDbRows % kDbParts == 0, "the parts tile the slab");
// a part is a whole number of 16-row strides, so every thread meets its rows in the order
// decode_kernel uses (rows = rsub mod 16, ascending) and the sums round identically
static_assert(kDbPartRows % (kDecThreads / 16) == 0, "parts keep decode_kernel's row order");
static_assert(kDbPartBytes % 16 == 0 && kDbZBytes % 16 == 0, "bulk copies move 16-byte multiples");
// the last slab's copy runs past row kF into the padding rows, never past the padded state
static_assert(((kF + kDbRows - 1) / kDbRows) * kDbRows <= kFP, "slab copies stay inside the unit");
// source addresses: unit base, the z array and every slab start are 16-byte aligned
static_assert((size_t(kFP) * kW * sizeof(float)) % 16 == 0, "units keep 16-byte alignment");
static_assert((size_t(kFP) * kDV * sizeof(float)) % 16 == 0, "z keeps 16-byte alignment");
static_assert((size_t(kDbRows) * sizeof(float)) % 16 == 0, "z slab starts are 16-byte aligned");
static_assert(kHeaderBytes % 16 == 0, "the header keeps 16-byte alignment");
static_assert(kMaxGroup == 8, "phi rows are read as two 16-byte vectors");

// Process-wide decode kernel choice: 0 = decode_kernel (default), 1 = decode_bulk_kernel.
std::atomic<int> g_decode_variant{0};

template <typename Tin, int kGrp>  // kGrp = Hq / Hkv query heads per kv head
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_bulk_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                       const Tin* __restrict__ v, unsigned char* __restrict__ state,
                       float* __restrict__ out, float* __restrict__ part,
                       unsigned int* __restrict__ tickets, int Hq, int Hkv)
{
    extern __shared__ __align__(128) unsigned char db_smem[];
    float* sh_hv = reinterpret_cast<float*>(db_smem);  // [kDbRows][kDV], the slab's Hv rows
    float* sh_z = sh_hv + size_t(kDbRows) * kDV;         // [kDbRows], the slab's z entries

    __shared__ __align__(8) uint64_t bars[kDbParts];
    __shared__ __align__(16) float vh[kW + 3];
    __shared__ float kh[kDA];
    __shared__ float qh[kMaxGroup][kDA];
    __shared__ __align__(16) float phis[kDbRows][kMaxGroup];
    __shared__ float psis[kDbRows];
    __shared__ float red[kMaxGroup][kW];
    __shared__ float ufin[kMaxGroup][kW];
    __shared__ int s_last;
    __shared__ int s_abort;

    const int slab = blockIdx.x, bkv = blockIdx.y, nslab = gridDim.x;
    constexpr int grp = kGrp;
    const int b = bkv / Hkv, kv = bkv % Hkv, h0 = kv * grp;
    const int tid = threadIdx.x, lane4 = tid & 15, rsub = tid >> 4;
    const float* coef = reinterpret_cast<const float*>(state + kHeaderBytes);
    float* unit = reinterpret_cast<float*>(state + kHeaderBytes + coef_bytes(Hq)) +
                  size_t(bkv) * kFP * kW;
    float* Hv = unit;
    float* z = unit + size_t(kFP) * kDV;
    const int f0 = slab * kDbRows;
    const int nrows = max(0, min(kDbRows, kF - f0));

    if (tid == 0) {
        for (int p = 0; p < kDbParts; ++p) tc::mbar_init(&bars[p], 1);
        tc::fence_mbar_init();
        s_abort = 0;
    }
    __syncthreads();
    if (tid == 0) {
        // every part is always copied (and waited for below), whatever nrows is, so that no
        // copy is still writing into this block's shared memory when the block exits
        tc::mbar_expect_tx(&bars[0], kDbPartBytes + kDbZBytes);
        tc::bulk_g2s(sh_z, z + f0, kDbZBytes, &bars[0]);
        tc::bulk_g2s(sh_hv, Hv + size_t(f0) * kDV, kDbPartBytes, &bars[0]);
        for (int p = 1; p < kDbParts; ++p) {
            tc::mbar_expect_tx(&bars[p], kDbPartBytes);
            tc::bulk_g2s(sh_hv + size_t(p) * kDbPartRows * kDV,
                         Hv + size_t(f0 + p * kDbPartRows) * kDV, kDbPartBytes, &bars[p]);
        }
    }

    // while the copies fly: the new token, the query heads, psi and phi of the slab's rows
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
    for (int e = tid; e < kMaxGroup * kW; e += kDecThreads) (&red[0][0])[e] = 0.f;
    __syncthreads();
    for (int row = tid; row < nrows; row += kDecThreads) {
        const int f = f0 + row;
        const RT rt = feature_rt(f);
        psis[row] = kh[rt.r] * kh[rt.t];
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g)
            phis[row][g] = g < grp ? coef[size_t(h0 + g) * kFP + f] * qh[g][rt.r] * qh[g][rt.t]
                                   : 0.f;
    }
    __syncthreads();

    float acc[kGrp][4];
#pragma unroll
    for (int g = 0; g < kGrp; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
    const float4 v4 = *reinterpret_cast<const float4*>(&vh[lane4 * 4]);
    constexpr int kRowStep = kDecThreads / 16;
    bool good = true;
#pragma unroll 1
    for (int p = 0; p < kDbParts; ++p) {
        // bounded (1 s); once any thread gives up, the others stop waiting too
        if (!tc::mbar_wait(&bars[p], 0, reinterpret_cast<volatile int*>(&s_abort))) {
            good = false;
            continue;
        }
        const int rend = min((p + 1) * kDbPartRows, nrows);
#pragma unroll 3
        for (int row = p * kDbPartRows + rsub; row < rend; row += kRowStep) {
            float4 h = *reinterpret_cast<const float4*>(sh_hv + size_t(row) * kDV + lane4 * 4);
            const float psi = psis[row];
            h.x = fmaf(psi, v4.x, h.x);
            h.y = fmaf(psi, v4.y, h.y);
            h.z = fmaf(psi, v4.z, h.z);
            h.w = fmaf(psi, v4.w, h.w);
            __stcs(reinterpret_cast<float4*>(Hv + size_t(f0 + row) * kDV) + lane4, h);
            const float4 pa = *reinterpret_cast<const float4*>(&phis[row][0]);
            const float4 pb = *reinterpret_cast<const float4*>(&phis[row][4]);
            const float ph[kMaxGroup] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                acc[g][0] = fmaf(ph[g], h.x, acc[g][0]);
                acc[g][1] = fmaf(ph[g], h.y, acc[g][1]);
                acc[g][2] = fmaf(ph[g], h.z, acc[g][2]);
                acc[g][3] = fmaf(ph[g], h.w, acc[g][3]);
            }
        }
    }
    float accz[kGrp];
#pragma unroll
    for (int g = 0; g < kGrp; ++g) accz[g] = 0.f;
    if (good) {  // sh_z arrived with part 0
        for (int row = tid; row < nrows; row += kDecThreads) {
            const float zz = sh_z[row] + psis[row];
            z[f0 + row] = zz;
#pragma unroll
            for (int g = 0; g < kGrp; ++g) accz[g] = fmaf(phis[row][g], zz, accz[g]);
        }
    }
    // From here on, the same reduction as decode_kernel.  It also runs after a timed-out
    // wait, so that the ticket of this (b, kv) is re-armed; the error word reports the failure.
#pragma unroll
    for (int g = 0; g < kGrp; ++g) {
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[g][c] += __shfl_xor_sync(0xffffffffu, acc[g][c], 16);
        float zz = accz[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
        if ((tid & 31) < 16) {
#pragma unroll
            for (int c = 0; c < 4; ++c) atomicAdd(&red[g][lane4 * 4 + c], acc[g][c]);
        }
        if ((tid & 31) == 0) atomicAdd(&red[g][kDV], zz);
    }
    __syncthreads();
    float* mypart = part + (size_t(bkv) * nslab + slab) * grp * kW;
    for (int e = tid; e < grp * kW; e += kDecThreads) mypart[e] = red[e / kW][e % kW];
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned int prev = atomicAdd(&tickets[bkv], 1u);
        s_last = (prev == unsigned(nslab - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float* allpart = part + size_t(bkv) * nslab * grp * kW;
    for (int e = tid; e < grp * kW; e += kDecThreads) {
        float s = 0.f;
        for (int sl = 0; sl < nslab; ++sl) s += __ldcg(allpart + size_t(sl) * grp * kW + e);
        ufin[e / kW][e % kW] = s;
    }
    __syncthreads();
    for (int e = tid; e < grp * kDV; e += kDecThreads) {
        const int g = e / kDV, n = e % kDV;
        out[(size_t(b) * Hq + h0 + g) * kDV + n] = ufin[g][n] / ufin[g][kDV];
    }
    if (tid == 0) {
        tickets[bkv] = 0u;
        if (bkv == 0) reinterpret_cast<StateHeader*>(state)->tokens += 1;
    }
}

template <typename Tin, int kGrp>
static cudaError_t launch_decode_bulk_t(const void* q, const void* k, const void* v,
                                        unsigned char* s, float* out, float* part,
                                        unsigned int* tickets, int B, int Hq, int Hkv,
                                        cudaStream_t st)
{
    auto kern = decode_bulk_kernel<Tin, kGrp>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kDbSmemBytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(decode_slabs(), B * Hkv);
    kern<<<grid, kDecThreads, kDbSmemBytes, st>>>(static_cast<const Tin*>(q),
                                                  static_cast<const Tin*>(k),
                                                  static_cast<const Tin*>(v), s, out, part,
                                                  tickets, Hq, Hkv);
    return cudaGetLastError();
}

// Same arguments, workspace layout (tickets, then per-slab partial sums) and results as
// launch_decode.
int launch_decode_bulk(const void* q, const void* k, const void* v, void* state, float* out,
                       float* part, unsigned int* tickets, int B, int Hq, int Hkv, int dtype,
                       cudaStream_t st)
{
    if (B == 0) return OAL_OK;
    unsigned char* s = static_cast<unsigned char*>(state);
    LaunchScope ls("decode_bulk", st);
    const bool bf = dtype == OAL_BF16;
    cudaError_t e = cudaSuccess;
    auto go = [&](auto G) {
        constexpr int g = decltype(G)::value;
        e = bf ? launch_decode_bulk_t<__nv_bfloat16, g>(q, k, v, s, out, part, tickets, B, Hq,
                                                        Hkv, st)
               : launch_decode_bulk_t<float, g>(q, k, v, s, out, part, tickets, B, Hq, Hkv, st);
    };
    switch (Hq / Hkv) {
        case 1: go(std::integral_constant<int, 1>{}); break;
        case 2: go(std::integral_constant<int, 2>{}); break;
        case 3: go(std::integral_constant<int, 3>{}); break;
        case 4: go(std::integral_constant<int, 4>{}); break;
        case 5: go(std::integral_constant<int, 5>{}); break;
        case 6: go(std::integral_constant<int, 6>{}); break;
        case 7: go(std::integral_constant<int, 7>{}); break;
        case 8: go(std::integral_constant<int, 8>{}); break;
        default: return OAL_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return cuda_fail(e);
    return OAL_OK;
}

int set_decode_variant(int variant) { return g_decode_variant.exchange(variant); }

// The decode kernel chosen by g_decode_variant.
int launch_decode_selected(const void* q, const void* k, const void* v, void* state, float* out,
                           float* part, unsigned int* tickets, int B, int Hq, int Hkv,
                           int dtype, cudaStream_t st)
{
    return g_decode_variant.load() == 1
               ? launch_decode_bulk(q, k, v, state, out, part, tickets, B, Hq, Hkv, dtype, st)
               : launch_decode(q, k, v, state, out, part, tickets, B, Hq, Hkv, dtype, st);
}

}  // namespace oal
