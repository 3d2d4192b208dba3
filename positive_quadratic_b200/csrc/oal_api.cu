// oal_api.cu -- the extern "C" boundary declared in include/oal.h: argument validation on the
// host, workspace layout, and dispatch to the kernels.  No device memory is allocated here.
#include <atomic>
#include <cstdio>
#include <cstring>

#include "oal_common.cuh"
#include "oal_kernels.cuh"

using namespace oal;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// q, k, v, out: required and aligned only when there is at least one token to process.
int check_io(const oal_shape* s, const void* q, const void* k, const void* v, const void* out)
{
    if ((long long)s->B * s->T == 0) return OAL_OK;
    if (!q || !k || !v || !out) return OAL_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return OAL_ERR_ALIGN;
    return OAL_OK;
}

int check_common(const oal_shape* s)
{
    if (!s) return OAL_ERR_NULL;
    if (s->B < 0 || s->T < 0 || s->Hq < 1 || s->Hkv < 1 || s->Hq % s->Hkv != 0)
        return OAL_ERR_SHAPE;
    if (s->dh != OAL_HEAD_DIM || s->dv != OAL_VALUE_DIM) return OAL_ERR_UNSUPPORTED;
    if (s->Hq / s->Hkv > kMaxGroup) return OAL_ERR_UNSUPPORTED;
    if (s->dtype != OAL_F32 && s->dtype != OAL_BF16) return OAL_ERR_UNSUPPORTED;
    const long long rows = (long long)s->B * s->Hq * (long long)(s->T > 0 ? s->T : 1);
    if (rows >= (1LL << 31)) return OAL_ERR_SHAPE;
    return OAL_OK;
}

int check_chunk(const oal_shape* s)
{
    return (s->chunk == 64 || s->chunk == 128 || s->chunk == 256) ? OAL_OK
                                                                   : OAL_ERR_UNSUPPORTED;
}

// A grid's y and z dimensions hold at most 65535 blocks.  The CUDA-core kernels put the
// B*Hq query-head planes there, the decode step the B*Hkv state planes, and the tensor-core
// scan the B*Hkv state planes plus one for the coefficient tables.
constexpr long long kMaxGridPlanes = 65535;

int check_planes(long long planes) { return planes > kMaxGridPlanes ? OAL_ERR_SHAPE : OAL_OK; }

size_t simt_chunk_state_bytes(const oal_shape* s)
{
    const size_t NC = s->T > 0 ? size_t((s->T + s->chunk - 1) / s->chunk) : 0;
    return size_t(s->B) * s->Hkv * NC * kW * kFP * sizeof(float);
}

// bf16 inputs with chunk 128 run on the tcgen05 kernels; everything else on CUDA cores.
bool use_tensor_path(const oal_shape* s) { return s->dtype == OAL_BF16 && s->chunk == 128; }

// The prefill's size limits on the path the shape takes: its grid planes, and on tensor cores
// the 32-bit row coordinate (tc::kImgRows rows per slice) of the chunk-state images that the
// readout loads.
int check_prefill_planes(const oal_shape* s)
{
    if (!use_tensor_path(s)) return check_planes((long long)s->B * s->Hq);
    const long long NC = (s->T + tc::kC - 1) / tc::kC;
    if ((long long)s->B * s->Hkv * NC * tc::kSlices * tc::kImgRows >= (1LL << 31))
        return OAL_ERR_SHAPE;
    return check_planes((long long)s->B * s->Hkv + 1);
}

std::atomic<int> g_prefill_overlap{1};

size_t decode_ticket_bytes(const oal_shape* s) { return align256(size_t(s->B) * s->Hkv * 4); }

size_t decode_part_bytes(const oal_shape* s)
{
    return size_t(s->B) * s->Hkv * decode_slabs() * (s->Hq / s->Hkv) * kW * sizeof(float);
}

}  // namespace

extern "C" {

int oal_abi_version(void) { return OAL_ABI_VERSION; }

const char* oal_status_string(int status)
{
    switch (status) {
    case OAL_OK: return "ok";
    case OAL_ERR_NULL: return "a required pointer is NULL";
    case OAL_ERR_SHAPE: return "inconsistent or out-of-range sizes";
    case OAL_ERR_UNSUPPORTED: return "unsupported size, chunk or dtype";
    case OAL_ERR_ALIGN: return "pointer not 16-byte aligned";
    case OAL_ERR_GROUPS: return "group id or group count out of range (clamped on device)";
    case OAL_ERR_CUDA: return "CUDA launch or runtime error";
    case OAL_ERR_TIMEOUT: return "a bounded device wait gave up";
    case OAL_ERR_WORKSPACE: return "workspace missing or too small";
    case OAL_ERR_STATE: return "state buffer does not match the shape";
    default: return "unknown status";
    }
}

int oal_state_bytes(const oal_shape* s, size_t* bytes)
{
    const int rc = check_common(s);
    if (rc) return rc;
    if (!bytes) return OAL_ERR_NULL;
    *bytes = state_bytes(s->B, s->Hq, s->Hkv);
    return OAL_OK;
}

int oal_prefill_workspace_bytes(const oal_shape* s, size_t* bytes)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_chunk(s))) return rc;
    if ((rc = check_prefill_planes(s))) return rc;
    if (!bytes) return OAL_ERR_NULL;
    const size_t tc = use_tensor_path(s) ? tc_workspace_bytes(s->B, s->Hq, s->Hkv, s->T) : 0;
    *bytes = simt_chunk_state_bytes(s) > tc ? simt_chunk_state_bytes(s) : tc;
    if (*bytes == 0) *bytes = 256;
    return OAL_OK;
}

int oal_prefill_path(const oal_shape* s, int* path)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_chunk(s))) return rc;
    if (!path) return OAL_ERR_NULL;
    *path = use_tensor_path(s) ? OAL_PATH_TENSOR : OAL_PATH_CUDA_CORE;
    return OAL_OK;
}

int oal_decode_workspace_bytes(const oal_shape* s, size_t* bytes)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hkv))) return rc;
    if (!bytes) return OAL_ERR_NULL;
    *bytes = decode_ticket_bytes(s) + decode_part_bytes(s);
    return OAL_OK;
}

namespace {

int prefill_impl(const void* q, const void* k, const void* v, const int32_t* group_id,
                 const float* L, const int32_t* G, float eps, float* out, void* state,
                 void* workspace, size_t workspace_bytes, const oal_shape* s, void* stream,
                 bool cont)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_chunk(s))) return rc;
    if (cont && !use_tensor_path(s)) return OAL_ERR_UNSUPPORTED;
    if ((rc = check_prefill_planes(s))) return rc;
    if (!group_id || !L || !G || !state) return OAL_ERR_NULL;
    // out == NULL asks for the state alone (no readout); q is then not read either
    if ((rc = check_io(s, out ? q : k, k, v, out ? out : v))) return rc;
    if (!aligned16(state) || !aligned16(group_id) || !aligned16(L) || !aligned16(G))
        return OAL_ERR_ALIGN;
    size_t need = 0;
    oal_prefill_workspace_bytes(s, &need);
    if (!workspace || workspace_bytes < need) return OAL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return OAL_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cont && (long long)s->B * s->T == 0) return OAL_OK;  // nothing appended
    // the tensor-core path builds the coefficient tables inside its scan kernel
    const bool tc = use_tensor_path(s) && s->B > 0 && s->T > 0;
    if (!tc) {
        rc = launch_prep(group_id, L, G, eps, state, s->B, s->Hq, s->Hkv, s->T, st);
        if (rc) return rc;
    }
    if (s->B == 0) return OAL_OK;
    if (use_tensor_path(s))
        return launch_prefill_tc(q, k, v, group_id, L, G, eps, out, state, workspace, s->B, s->T,
                                 s->Hq, s->Hkv, g_prefill_overlap.load() != 0, cont, st);
    return launch_prefill_simt(q, k, v, group_id, L, G, eps, out, state,
                               static_cast<float*>(workspace), s->B, s->T, s->Hq, s->Hkv,
                               s->chunk, s->dtype, st);
}

}  // namespace

int oal_prefill(const void* q, const void* k, const void* v, const int32_t* group_id,
                const float* L, const int32_t* G, float eps, float* out, void* state,
                void* workspace, size_t workspace_bytes, const oal_shape* s, void* stream)
{
    return prefill_impl(q, k, v, group_id, L, G, eps, out, state, workspace,
                             workspace_bytes, s, stream, false);
}

int oal_prefill_continue(const void* q, const void* k, const void* v, const int32_t* group_id,
                         const float* L, const int32_t* G, float eps, float* out, void* state,
                         void* workspace, size_t workspace_bytes, const oal_shape* s,
                         void* stream)
{
    return prefill_impl(q, k, v, group_id, L, G, eps, out, state, workspace,
                             workspace_bytes, s, stream, true);
}

int oal_decode_step(const void* q, const void* k, const void* v, void* state, float* out,
                    void* workspace, size_t workspace_bytes, const oal_shape* s, void* stream)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hkv))) return rc;
    oal_shape one = *s;
    one.T = 1;
    if (!state) return OAL_ERR_NULL;
    if ((rc = check_io(&one, q, k, v, out))) return rc;
    if (!aligned16(state)) return OAL_ERR_ALIGN;
    size_t need = 0;
    oal_decode_workspace_bytes(s, &need);
    if (!workspace || workspace_bytes < need) return OAL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return OAL_ERR_ALIGN;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    return launch_decode(q, k, v, state, out,
                         reinterpret_cast<float*>(ws + decode_ticket_bytes(s)), s->B, s->Hq,
                         s->Hkv, s->dtype, static_cast<cudaStream_t>(stream));
}

int oal_dense_ref_gpu(const void* q, const void* k, const void* v, const int32_t* group_id,
                      const float* L, const int32_t* G, float eps, float* out,
                      const oal_shape* s, void* stream)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_planes((long long)s->B * s->Hq))) return rc;
    if (!group_id || !L || !G) return OAL_ERR_NULL;
    if ((rc = check_io(s, q, k, v, out))) return rc;
    if (!aligned16(group_id) || !aligned16(L) || !aligned16(G)) return OAL_ERR_ALIGN;
    if ((long long)s->B * s->T == 0) return OAL_OK;
    return launch_dense(q, k, v, group_id, L, G, eps, out, s->B, s->T, s->Hq, s->Hkv, s->dtype,
                        static_cast<cudaStream_t>(stream));
}

int oal_contribution_stat(const void* q, const void* k, float* chi, const oal_shape* s,
                          void* stream)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((long long)s->B * s->T == 0) return OAL_OK;
    if (!q || !k || !chi) return OAL_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(chi)) return OAL_ERR_ALIGN;
    return launch_chi(q, k, chi, s->B, s->T, s->Hq, s->Hkv, s->dtype,
                      static_cast<cudaStream_t>(stream));
}

unsigned long long oal_launch_count(void) { return tracer().launches.load(); }

int oal_set_prefill_overlap(int overlap) { return g_prefill_overlap.exchange(overlap ? 1 : 0); }

int oal_set_debug_skip_copies(int on) { return oal::g_skip_copies.exchange(on ? 1 : 0); }

int oal_profile_enable(int on)
{
    Tracer& t = tracer();
    if (on) {
        std::lock_guard<std::mutex> g(t.mu);
        if (!tracer_fill_pool(t)) return OAL_ERR_CUDA;
    }
    t.enabled.store(on ? 1 : 0);
    return OAL_OK;
}

int oal_profile_read(oal_kernel_stat* stats, int max_stats, int* n_stats)
{
    if (!n_stats || (max_stats > 0 && !stats)) return OAL_ERR_NULL;
    Tracer& t = tracer();
    std::vector<TraceRecord> recs;
    {
        std::lock_guard<std::mutex> g(t.mu);
        recs.swap(t.records);
    }
    std::vector<cudaEvent_t> back;
    int n = 0, rc = OAL_OK;
    for (const TraceRecord& r : recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess ||
            cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
            rc = OAL_ERR_CUDA;
        back.push_back(r.start);
        back.push_back(r.stop);
        int i = 0;
        while (i < n && std::strncmp(stats[i].name, r.name, sizeof(stats[i].name)) != 0) ++i;
        if (i == n) {
            if (n == max_stats) continue;
            std::memset(&stats[n], 0, sizeof(stats[n]));
            std::strncpy(stats[n].name, r.name, sizeof(stats[n].name) - 1);
            ++n;
        }
        stats[i].launches += 1;
        stats[i].total_ms += ms;
    }
    {
        std::lock_guard<std::mutex> g(t.mu);
        t.pool.insert(t.pool.end(), back.begin(), back.end());
    }
    *n_stats = n;
    return rc;
}

int oal_last_cuda_error(char* buf, size_t len)
{
    const int e = last_cuda_error().load();
    if (buf && len > 0) {
        const char* name = e ? cudaGetErrorName(cudaError_t(e)) : "cudaSuccess";
        const char* text = e ? cudaGetErrorString(cudaError_t(e)) : "no error";
        std::snprintf(buf, len, "%s: %s", name, text);
    }
    return e;
}

int oal_device_error(int* code, void* stream)
{
    if (!code) return OAL_ERR_NULL;
    return read_device_error(code, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
