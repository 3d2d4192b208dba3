// oal_noalloc.cu -- oal_decode_step_noalloc: the decode step with its scratch memory inside
// the library, for callers that cannot allocate device memory or pass a workspace.
//
// The scratch is a file-scope device array of fixed size.  Host code never uses the array's
// name as an address (on the host it is only a stand-in for the symbol): the device address
// is looked up once per device with cudaGetSymbolAddress, with that device current, on the
// first call made on that device, and cached.
#include <mutex>

#include "oal_common.cuh"
#include "oal_kernels.cuh"

namespace oal {

// 4 MiB: room for the reserved leading block and the per-slab partial readouts (9 slabs x 65
// fp32 per query head) of a decode step with B*Hq up to 1789 query heads, whatever Hkv
// (batch 64 x 14 heads needs 2.1 MB).
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int noalloc_scratch(void** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
        return OAL_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return OAL_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return OAL_OK;
}

}  // namespace
}  // namespace oal

extern "C" int oal_decode_step_noalloc(const void* q, const void* k, const void* v,
                                       void* state, float* out, const oal_shape* s,
                                       void* stream)
{
    using namespace oal;
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hkv))) return rc;
    oal_shape one = *s;
    one.T = 1;
    if (!state) return OAL_ERR_NULL;
    if ((rc = check_io(&one, q, k, v, out))) return rc;
    if (!aligned16(state)) return OAL_ERR_ALIGN;
    size_t need = 0;
    if ((rc = oal_decode_workspace_bytes(s, &need))) return rc;
    if (need > kNoAllocScratchBytes) return OAL_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(scratch);
    // every word of the scratch that a step reads, the step itself wrote first
    return launch_decode(q, k, v, state, out,
                         reinterpret_cast<float*>(ws + decode_ticket_bytes(s)), s->B, s->Hq,
                         s->Hkv, s->dtype, st);
}
