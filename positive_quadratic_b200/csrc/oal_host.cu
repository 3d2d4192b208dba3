// oal_host.cu -- prefill from host memory, with the copies overlapped with the kernels.
//
// The sequence is cut into contiguous token segments whose boundaries fall on chunk
// boundaries.  Segment i is copied in on the caller's copy-in stream.  It is computed on the
// compute stream, the first segment by a fresh prefill and the others by continuing the
// prefix state ("OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式: the state of
// eq. (4) is a running sum, so each segment starts from the state the previous one left).
// Its yhat is copied out on the copy-out stream while segment i+1 computes.  The boundaries
// are chunk boundaries, and the continued scan adds the chunk deltas in the same order as one
// whole prefill does, so the results are those of one oal_prefill over the whole sequence.
#pragma once

#include <algorithm>

#include "oal_common.cuh"
#include "oal_events.cuh"
#include "oal_kernels.cuh"

namespace oal {
namespace {

struct HostPlan {
    int nseg = 0;       // segments actually used
    int seg_len = 0;    // tokens per segment (the last one may be shorter)
    size_t esize = 0;   // bytes per q/k/v element
    size_t off_k = 0, off_v = 0, off_out = 0, off_ws = 0;  // byte offsets in the workspace
    size_t ws_bytes = 0;    // prefill workspace of the longest segment
    size_t total = 0;       // whole workspace
};

int plan_host(const oal_shape* s, int segments, HostPlan* p)
{
    int rc = check_common(s);
    if (rc) return rc;
    if ((rc = check_chunk(s))) return rc;
    if (segments < 1) return OAL_ERR_SHAPE;
    if (segments > 1 && !use_tensor_path(s)) return OAL_ERR_UNSUPPORTED;
    HostPlan h;
    h.esize = s->dtype == OAL_BF16 ? 2 : 4;
    const long long T = s->T;
    if (T > 0) {
        const long long per = (T + segments - 1) / segments;
        h.seg_len = int((per + s->chunk - 1) / s->chunk * s->chunk);
        h.nseg = int((T + h.seg_len - 1) / h.seg_len);
    }
    const size_t rows_q = size_t(s->B) * s->Hq, rows_kv = size_t(s->B) * s->Hkv;
    const size_t tok = size_t(T) * OAL_HEAD_DIM;
    h.off_k = align256(rows_q * tok * h.esize);
    h.off_v = h.off_k + align256(rows_kv * tok * h.esize);
    h.off_out = h.off_v + align256(rows_kv * tok * h.esize);
    h.off_ws = h.off_out + align256(rows_q * size_t(T) * OAL_VALUE_DIM * sizeof(float));
    oal_shape seg = *s;
    seg.T = h.nseg > 0 ? h.seg_len : 0;
    if ((rc = oal_prefill_workspace_bytes(&seg, &h.ws_bytes))) return rc;
    h.total = h.off_ws + align256(h.ws_bytes);
    *p = h;
    return OAL_OK;
}

// dst/src rows of `width` bytes: rows x width, with the given pitches
cudaError_t copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                      size_t rows, cudaMemcpyKind kind, cudaStream_t st)
{
    if (rows == 0 || width == 0) return cudaSuccess;
    return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, kind, st);
}

}  // namespace
}  // namespace oal

extern "C" {

int oal_prefill_host_workspace_bytes(const oal_shape* s, int segments, size_t* bytes)
{
    using namespace oal;
    if (!bytes) return OAL_ERR_NULL;
    HostPlan p;
    const int rc = plan_host(s, segments, &p);
    if (rc) return rc;
    *bytes = p.total;
    return OAL_OK;
}

int oal_prefill_host(const void* q_host, const void* k_host, const void* v_host,
                     const int32_t* group_id, const float* L, const int32_t* G, float eps,
                     float* out_host, void* state, void* workspace, size_t workspace_bytes,
                     const oal_shape* s, int segments, void* stream, void* copy_in,
                     void* copy_out)
{
    using namespace oal;
    HostPlan p;
    int rc = plan_host(s, segments, &p);
    if (rc) return rc;
    if (!group_id || !L || !G || !state) return OAL_ERR_NULL;
    if (!workspace || workspace_bytes < p.total) return OAL_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return OAL_ERR_ALIGN;
    if ((long long)s->B * s->T > 0 && (!q_host || !k_host || !v_host || !out_host))
        return OAL_ERR_NULL;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    void* pws = ws + p.off_ws;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t cin = copy_in ? static_cast<cudaStream_t>(copy_in) : st;
    cudaStream_t cout = copy_out ? static_cast<cudaStream_t>(copy_out) : st;
    if (p.nseg == 0 || s->B == 0)  // no tokens: what oal_prefill does for an empty input
        return prefill_impl(ws, ws, ws, group_id, L, G, eps, reinterpret_cast<float*>(ws),
                            state, pws, p.ws_bytes, s, stream, false);

    CallEvents evs;
    cudaEvent_t ev_start, ev_end;
    OAL_CUDA_TRY(evs.make(&ev_start));
    OAL_CUDA_TRY(evs.make(&ev_end));
    // everything earlier on the compute stream (a previous call reading the same staging
    // buffers, for instance) precedes this call's copies
    OAL_CUDA_TRY(cudaEventRecord(ev_start, st));
    if (cin != st) OAL_CUDA_TRY(cudaStreamWaitEvent(cin, ev_start, 0));
    if (cout != st) OAL_CUDA_TRY(cudaStreamWaitEvent(cout, ev_start, 0));

    const size_t rows_q = size_t(s->B) * s->Hq, rows_kv = size_t(s->B) * s->Hkv;
    const size_t T = size_t(s->T), D = OAL_HEAD_DIM, DV = OAL_VALUE_DIM, es = p.esize;
    const unsigned char* qh = static_cast<const unsigned char*>(q_host);
    const unsigned char* kh = static_cast<const unsigned char*>(k_host);
    const unsigned char* vh = static_cast<const unsigned char*>(v_host);
    for (int i = 0; i < p.nseg; ++i) {
        const size_t t0 = size_t(i) * p.seg_len;
        const size_t ts = std::min(size_t(p.seg_len), T - t0);
        // segment i's staging blocks: [B][H][ts][64], packed after segments 0..i-1
        unsigned char* dq = ws + rows_q * t0 * D * es;
        unsigned char* dk = ws + p.off_k + rows_kv * t0 * D * es;
        unsigned char* dv = ws + p.off_v + rows_kv * t0 * D * es;
        float* dout = reinterpret_cast<float*>(ws + p.off_out) + rows_q * t0 * DV;
        OAL_CUDA_TRY(copy_rows(dq, ts * D * es, qh + t0 * D * es, T * D * es, ts * D * es,
                               rows_q, cudaMemcpyHostToDevice, cin));
        OAL_CUDA_TRY(copy_rows(dk, ts * D * es, kh + t0 * D * es, T * D * es, ts * D * es,
                               rows_kv, cudaMemcpyHostToDevice, cin));
        OAL_CUDA_TRY(copy_rows(dv, ts * DV * es, vh + t0 * DV * es, T * DV * es, ts * DV * es,
                               rows_kv, cudaMemcpyHostToDevice, cin));
        cudaEvent_t ev_in, ev_out;
        OAL_CUDA_TRY(evs.make(&ev_in));
        OAL_CUDA_TRY(evs.make(&ev_out));
        OAL_CUDA_TRY(cudaEventRecord(ev_in, cin));
        if (cin != st) OAL_CUDA_TRY(cudaStreamWaitEvent(st, ev_in, 0));
        oal_shape seg = *s;
        seg.T = int(ts);
        rc = prefill_impl(dq, dk, dv, group_id, L, G, eps, dout, state, pws, p.ws_bytes, &seg,
                          stream, i > 0);
        if (rc) return rc;
        OAL_CUDA_TRY(cudaEventRecord(ev_out, st));
        if (cout != st) OAL_CUDA_TRY(cudaStreamWaitEvent(cout, ev_out, 0));
        OAL_CUDA_TRY(copy_rows(out_host + t0 * DV, T * DV * sizeof(float), dout,
                               ts * DV * sizeof(float), ts * DV * sizeof(float), rows_q,
                               cudaMemcpyDeviceToHost, cout));
    }
    // later work on the compute stream (and a synchronisation of it) covers the last copy out
    OAL_CUDA_TRY(cudaEventRecord(ev_end, cout));
    if (cout != st) OAL_CUDA_TRY(cudaStreamWaitEvent(st, ev_end, 0));
    return OAL_OK;
}

}  // extern "C"
