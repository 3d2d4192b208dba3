// oal_kernels.cuh -- internal launchers behind the C ABI (not part of the public header).
#pragma once

#include <cstddef>
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace oal {

int launch_prep(const int32_t* gid, const float* L, const int32_t* G, float eps, void* state,
                int B, int Hq, int Hkv, long long tokens, cudaStream_t st);

int launch_prefill_simt(const void* q, const void* k, const void* v, const int32_t* gid,
                        const float* L, const int32_t* G, float eps, float* out, void* state,
                        float* Hc, int B, int T, int Hq, int Hkv, int C, int dtype,
                        cudaStream_t st);

int launch_dense(const void* q, const void* k, const void* v, const int32_t* gid, const float* L,
                 const int32_t* G, float eps, float* out, int B, int T, int Hq, int Hkv,
                 int dtype, cudaStream_t st);

int decode_slabs();

int launch_decode(const void* q, const void* k, const void* v, void* state, float* out,
                  float* part, int B, int Hq, int Hkv, int dtype,
                  cudaStream_t st);

// ungrouped Hadamard form (oal_hadamard.cu): prefill on CUDA cores, or the dense O(T^2) form
int launch_hadamard(const void* q, const void* k, const void* v, const float* a, const float* b,
                    const float* C, float* out, void* state, float* Hc, int B, int T, int Hq,
                    int Hkv, int Cn, int dtype, bool dense, cudaStream_t st);

int read_device_error(int* code, cudaStream_t st);

// tensor-core (tcgen05) bf16 prefill, chunk 128.  fm_intra: the coefficient tables and the
// state header were written by the caller (free coefficients; gid, L, G unused) and the
// intra-chunk part goes through the feature map.
size_t tc_image_bytes(int B, int Hkv, int T);
size_t tc_workspace_bytes(int B, int Hq, int Hkv, int T);
unsigned char* tc_rtab(void* ws, int B, int Hkv, int T);  // per-head readout tables in ws
int launch_prefill_tc(const void* q, const void* k, const void* v, const int32_t* gid,
                      const float* L, const int32_t* G, float eps, float* out, void* state,
                      void* ws, int B, int T, int Hq, int Hkv, bool overlap, bool cont,
                      cudaStream_t st, bool fm_intra = false);

// The same kernels over a packed variable-length batch in one launch each: sequence i is the
// B = 1 problem of lens[i] tokens whose q block [Hq][T_i][64] starts at row tok_i * Hq (tok_i:
// tokens before it), likewise k, v ([Hkv]) and out; its state is at states + i * stride.
// The workspace holds the chunk states of every sequence, one readout table per head, the
// intra-chunk normalisers, the sequence descriptors and three tensor maps per sequence.
struct TcPackedLayout {
    size_t img, dS, rtab, zin, seqs, maps, total;  // byte offsets and total size
    long long chunks, tokens;                      // sums over the sequences
};
TcPackedLayout tc_packed_layout(int Hq, int Hkv, const int32_t* lens, int n);
int launch_prefill_tc_packed(const void* q, const void* k, const void* v, const int32_t* gid,
                             const float* L, const int32_t* G, float eps, float* out,
                             unsigned char* states, size_t stride, void* ws, const int32_t* lens,
                             int n, int Hq, int Hkv, bool overlap, cudaStream_t st);

// test hook of oal_set_debug_skip_copies
extern std::atomic<int> g_skip_copies;

int launch_chi(const void* q, const void* k, float* chi, int B, int T, int Hq, int Hkv,
               int dtype, cudaStream_t st);

}  // namespace oal
