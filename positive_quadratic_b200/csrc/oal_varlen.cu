// oal_varlen.cu -- prefill of a batch of independent sequences of different lengths.
//
// Each sequence is its own causal problem ("OAL: 按 QK 离群贡献分组的正二次注意力核", section
// 核心公式: the prefix sums of eq. (4) run over one sequence), so the batch needs no exchange:
// sequence i is an ordinary B = 1 prefill on its block of the packed arrays, with its own state
// buffer.  The sequences are spread round-robin over the caller's streams, each with its own
// slice of the workspace, so that short sequences, which fill only part of the GPU alone, run
// side by side.  The call's work is ordered after earlier work on the first stream, and later
// work on that stream is ordered after every sequence.
#pragma once

#include <algorithm>

#include "oal_common.cuh"
#include "oal_events.cuh"
#include "oal_kernels.cuh"

namespace oal {
namespace {

struct VarlenPlan {
    size_t ws_one = 0;    // prefill workspace of the longest sequence (one per stream)
    size_t ws_slice = 0;  // ws_one rounded up to 256 bytes
    size_t state_one = 0; // oal_state_bytes of one sequence
    long long total = 0;  // tokens over all sequences
};

int plan_varlen(const oal_shape* s, const int32_t* seq_lens, int n_seq, int n_streams,
                VarlenPlan* p)
{
    if (!s || (n_seq > 0 && !seq_lens)) return OAL_ERR_NULL;
    if (n_seq < 0 || n_streams < 1) return OAL_ERR_SHAPE;
    oal_shape one = *s;
    one.B = 1;
    int tmax = 0;
    long long total = 0;
    for (int i = 0; i < n_seq; ++i) {
        if (seq_lens[i] < 0) return OAL_ERR_SHAPE;
        tmax = std::max(tmax, int(seq_lens[i]));
        total += seq_lens[i];
    }
    // the packed arrays are indexed as one [H][total][64] run per head count
    if (total * (long long)s->Hq >= (1LL << 31)) return OAL_ERR_SHAPE;
    one.T = tmax;
    int rc = check_common(&one);
    if (rc) return rc;
    if ((rc = check_chunk(&one))) return rc;
    VarlenPlan v;
    if ((rc = oal_prefill_workspace_bytes(&one, &v.ws_one))) return rc;
    v.ws_slice = align256(v.ws_one);
    if ((rc = oal_state_bytes(&one, &v.state_one))) return rc;
    v.total = total;
    *p = v;
    return OAL_OK;
}

// The packed batch in one launch per kernel: the tensor-core path only (bf16, chunk 128).
int plan_packed(const oal_shape* s, const int32_t* seq_lens, int n_seq, TcPackedLayout* lay,
                size_t* state_one)
{
    if (!s || (n_seq > 0 && !seq_lens)) return OAL_ERR_NULL;
    if (n_seq < 0) return OAL_ERR_SHAPE;
    oal_shape one = *s;
    one.B = 1;
    int tmax = 0;
    long long total = 0;
    for (int i = 0; i < n_seq; ++i) {
        if (seq_lens[i] < 0) return OAL_ERR_SHAPE;
        tmax = std::max(tmax, int(seq_lens[i]));
        total += seq_lens[i];
    }
    if (total * (long long)s->Hq >= (1LL << 31)) return OAL_ERR_SHAPE;
    one.T = tmax;
    int rc = check_common(&one);
    if (rc) return rc;
    if ((rc = check_chunk(&one))) return rc;
    if (!use_tensor_path(&one)) return OAL_ERR_UNSUPPORTED;
    // the scan's grid planes: every sequence's kv heads and the coefficient tables
    if ((rc = check_planes((long long)n_seq * s->Hkv + 1))) return rc;
    *lay = tc_packed_layout(s->Hq, s->Hkv, seq_lens, n_seq);
    // tensor-copy row coordinates of the chunk-state images are 32-bit
    if (lay->chunks * s->Hkv * 34 * 80 >= (1LL << 31)) return OAL_ERR_SHAPE;
    return oal_state_bytes(&one, state_one);
}

}  // namespace
}  // namespace oal

extern "C" {

int oal_prefill_packed_workspace_bytes(const oal_shape* s, const int32_t* seq_lens, int n_seq,
                                       size_t* bytes)
{
    using namespace oal;
    if (!bytes) return OAL_ERR_NULL;
    TcPackedLayout lay;
    size_t state_one = 0;
    const int rc = plan_packed(s, seq_lens, n_seq, &lay, &state_one);
    if (rc) return rc;
    *bytes = lay.total;
    return OAL_OK;
}

int oal_prefill_packed(const void* q, const void* k, const void* v, const int32_t* group_id,
                       const float* L, const int32_t* G, float eps, float* out, void* states,
                       size_t state_stride, void* workspace, size_t workspace_bytes,
                       const oal_shape* s, const int32_t* seq_lens, int n_seq, void* stream)
{
    using namespace oal;
    TcPackedLayout lay;
    size_t state_one = 0;
    int rc = plan_packed(s, seq_lens, n_seq, &lay, &state_one);
    if (rc) return rc;
    if (!states || !group_id || !L || !G) return OAL_ERR_NULL;
    if (state_stride < state_one || state_stride % 256 != 0) return OAL_ERR_SHAPE;
    if (!workspace || workspace_bytes < lay.total) return OAL_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return OAL_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(states) & 255) != 0) return OAL_ERR_ALIGN;
    if (lay.tokens > 0 && (!q || !k || !v || !out)) return OAL_ERR_NULL;
    if (lay.tokens > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)))
        return OAL_ERR_ALIGN;
    if (!aligned16(group_id) || !aligned16(L) || !aligned16(G)) return OAL_ERR_ALIGN;
    return launch_prefill_tc_packed(q, k, v, group_id, L, G, eps, out,
                                    static_cast<unsigned char*>(states), state_stride, workspace,
                                    seq_lens, n_seq, s->Hq, s->Hkv, g_prefill_overlap.load() != 0,
                                    static_cast<cudaStream_t>(stream));
}

int oal_prefill_varlen_workspace_bytes(const oal_shape* s, const int32_t* seq_lens, int n_seq,
                                       int n_streams, size_t* bytes)
{
    using namespace oal;
    if (!bytes) return OAL_ERR_NULL;
    VarlenPlan p;
    const int rc = plan_varlen(s, seq_lens, n_seq, n_streams, &p);
    if (rc) return rc;
    *bytes = std::max<size_t>(256, p.ws_slice * size_t(n_streams));
    return OAL_OK;
}

int oal_prefill_varlen(const void* q, const void* k, const void* v, const int32_t* group_id,
                       const float* L, const int32_t* G, float eps, float* out, void* states,
                       size_t state_stride, void* workspace, size_t workspace_bytes,
                       const oal_shape* s, const int32_t* seq_lens, int n_seq,
                       void* const* streams, int n_streams)
{
    using namespace oal;
    VarlenPlan p;
    int rc = plan_varlen(s, seq_lens, n_seq, n_streams, &p);
    if (rc) return rc;
    if (!streams || !states || !group_id || !L || !G) return OAL_ERR_NULL;
    if (state_stride < p.state_one || state_stride % 256 != 0) return OAL_ERR_SHAPE;
    if (!workspace || workspace_bytes < p.ws_slice * size_t(n_streams)) return OAL_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return OAL_ERR_ALIGN;
    if (p.total > 0 && (!q || !k || !v || !out)) return OAL_ERR_NULL;
    if (n_seq == 0) return OAL_OK;

    const size_t es = s->dtype == OAL_BF16 ? 2 : 4, D = OAL_HEAD_DIM, DV = OAL_VALUE_DIM;
    const int nst = std::min(n_streams, n_seq);
    cudaStream_t first = static_cast<cudaStream_t>(streams[0]);
    CallEvents evs;
    cudaEvent_t ev_start;
    OAL_CUDA_TRY(evs.make(&ev_start));
    OAL_CUDA_TRY(cudaEventRecord(ev_start, first));
    for (int j = 1; j < nst; ++j)
        OAL_CUDA_TRY(cudaStreamWaitEvent(static_cast<cudaStream_t>(streams[j]), ev_start, 0));

    long long off = 0;  // tokens before sequence i
    for (int i = 0; i < n_seq; ++i) {
        const int j = i % nst;
        oal_shape one = *s;
        one.B = 1;
        one.T = seq_lens[i];
        const size_t o = size_t(off);
        const unsigned char* qi = static_cast<const unsigned char*>(q) + o * s->Hq * D * es;
        const unsigned char* ki = static_cast<const unsigned char*>(k) + o * s->Hkv * D * es;
        const unsigned char* vi = static_cast<const unsigned char*>(v) + o * s->Hkv * DV * es;
        float* oi = out + o * s->Hq * DV;
        void* st = static_cast<unsigned char*>(states) + size_t(i) * state_stride;
        void* ws = static_cast<unsigned char*>(workspace) + size_t(j) * p.ws_slice;
        rc = prefill_impl(qi, ki, vi, group_id, L, G, eps, oi, st, ws, p.ws_one, &one,
                          streams[j], false);
        if (rc) break;
        off += seq_lens[i];
    }
    // join every side stream back into the first, also after a failed sequence, so that later
    // work on streams[0] is ordered after everything already enqueued and no fork stays open
    for (int j = 1; j < nst; ++j) {
        cudaEvent_t ev;
        OAL_CUDA_TRY(evs.make(&ev));
        OAL_CUDA_TRY(cudaEventRecord(ev, static_cast<cudaStream_t>(streams[j])));
        OAL_CUDA_TRY(cudaStreamWaitEvent(first, ev, 0));
    }
    return rc;
}

}  // extern "C"
