/*
 * oal.h -- C ABI of the B200 (sm_100a) library for OAL causal grouped positive-quadratic
 * attention.
 *
 * What it computes.  "OAL: 按 QK 离群贡献分组的正二次注意力核" (reproduction note of arXiv
 * 2610.13674), section 核心公式, equations in order of appearance:
 *   (2) s_g = sum_{r in G_g} q_r k_r / sqrt(d_h),  sbar = [1, s_1, ..., s_G]
 *   (3) kappa(q, k) = eps + sbar^T L L^T sbar > 0
 *   (4) H0_i = sum_{j<=i} [v_j; 1],  H1_{i,r} = sum_{j<=i} k_{j,r} [v_j; 1],
 *       H2_{i,rt} = sum_{j<=i} k_{j,r} k_{j,t} [v_j; 1]
 *   (5) u_i = a H0_i + (1/sqrt(d_h)) sum_r b_r q_{i,r} H1_{i,r}
 *             + (1/d_h) sum_{r,t} C_rt q_{i,r} q_{i,t} H2_{i,rt},   yhat_i = u_{i,1:dv}/u_{i,dv+1}
 * i.e. yhat_i = sum_{j<=i} kappa(q_i,k_j) v_j / sum_{j<=i} kappa(q_i,k_j) (causal, j <= i
 * inclusive).  The coefficients are a = eps + M_00, b_r = 2 M_{0,g(r)}, C_rt = M_{g(r),g(t)}
 * with M = L L^T (the pages do not print them; this expansion is the one that makes (5) equal
 * (3) summed over j).  The abstract of arXiv 2610.13674 states the linear-time evaluation in
 * sequence length for a fixed head dimension that oal_prefill and oal_decode_step implement.
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers to contiguous row-major arrays, allocated and
 *    owned by the caller (for example through PyTorch), except the *_host arrays of
 *    oal_prefill_host, which are host memory.  The library allocates no device memory and
 *    keeps no pointer after a call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream).  A return of OAL_OK means the work was validated and enqueued.
 *  - Return value: OAL_OK (0) or a negative oal_status.  Nothing aborts or throws.  Argument
 *    errors are found on the host before anything is enqueued.  Errors that only the device
 *    can see (a group id outside 1..G[h], G[h] outside 1..OAL_G_MAX, a bounded wait that ran
 *    out) set a device-side error word instead; read and clear it with oal_device_error().
 *  - Layouts: q [B][Hq][T][dh], k [B][Hkv][T][dh], v [B][Hkv][T][dv] in the element type of
 *    oal_shape.dtype; out [B][Hq][T][dv] fp32.  Query head h reads key/value head
 *    floor(h * Hkv / Hq) (grouped-query attention; Hq must be a multiple of Hkv).
 *    group_id [Hq][dh] int32 with values 1..G[h]; G [Hq] int32 in 1..OAL_G_MAX;
 *    L [Hq][OAL_G_MAX+1][OAL_G_MAX+1] fp32, of which the leading (G[h]+1)x(G[h]+1) block is
 *    used as given (M = L L^T; L need not be triangular).
 *  - Supported sizes: dh = dv = 64; Hq/Hkv <= 8; chunk in {64, 128, 256}; B, T >= 0 with
 *    B*Hq*T < 2^31.  Pointers must be 16-byte aligned.  When B*T == 0 the q, k, v and out
 *    pointers are not used and may be NULL.
 */
#ifndef OAL_H
#define OAL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OAL_ABI_VERSION 1
#define OAL_HEAD_DIM 64
#define OAL_VALUE_DIM 64
#define OAL_G_MAX 8
/* packed features of the prefix state: the upper triangle of qhat qhat^T, qhat = [q; 1] */
#define OAL_FEATURES 2145
#define OAL_FEATURES_PAD 2176

typedef enum { OAL_F32 = 0, OAL_BF16 = 1 } oal_dtype;

typedef enum {
    OAL_OK = 0,
    OAL_ERR_NULL = -1,        /* a required pointer is NULL */
    OAL_ERR_SHAPE = -2,       /* inconsistent or out-of-range sizes */
    OAL_ERR_UNSUPPORTED = -3, /* valid but unsupported (dh/dv != 64, chunk size, dtype) */
    OAL_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned */
    OAL_ERR_GROUPS = -5,      /* device: group id or G out of range (inputs were clamped) */
    OAL_ERR_CUDA = -6,        /* a CUDA launch or runtime call failed */
    OAL_ERR_TIMEOUT = -7,     /* device: a bounded wait gave up */
    OAL_ERR_WORKSPACE = -8,   /* workspace NULL or smaller than the query function says */
    OAL_ERR_STATE = -9        /* state buffer does not match the shape */
} oal_status;

/* Problem description shared by every call.  Size limits checked on the host (OAL_ERR_SHAPE):
 * B*Hq*max(T, 1) < 2^31 rows; and, because a grid holds at most 65535 blocks in its y and z
 * dimensions, B*Hq <= 65535 for the CUDA-core prefill, the Hadamard and dense forms and both
 * backward passes, B*Hkv <= 65535 for the decode step, and B*Hkv + 1 <= 65535 for the
 * tensor-core prefill (n_seq*Hkv + 1 for the packed batch).  The tensor-core prefill also
 * needs B*Hkv*ceil(T/128)*34*80 < 2^31 (32-bit row coordinates of its chunk-state images;
 * chunks*Hkv*34*80 for the packed batch).  The size queries (*_workspace_bytes) apply the
 * same limits. */
typedef struct {
    int32_t B;     /* batch */
    int32_t T;     /* tokens per sequence (oal_decode_step: ignored, one token) */
    int32_t Hq;    /* query heads */
    int32_t Hkv;   /* key/value heads; Hq % Hkv == 0 */
    int32_t dh;    /* head dim of q and k (64) */
    int32_t dv;    /* head dim of v (64) */
    int32_t chunk; /* prefill chunk size C in {64, 128, 256}; ignored by decode and dense */
    int32_t dtype; /* oal_dtype of q, k, v */
} oal_shape;

/* Size in bytes of the recurrent state buffer for `s` (B, Hq, Hkv used).
 * Layout: a 256-byte header; then the readout coefficients of every query head,
 * coef [Hq][OAL_FEATURES_PAD] fp32 (padded to 256 bytes); then, per (b, kv) in row-major
 * order, Hv [OAL_FEATURES_PAD][dv] fp32 followed by z [OAL_FEATURES_PAD] fp32.  Row f of
 * (Hv | z) is sum_j psi_f(k_j) [v_j; 1] over the tokens seen so far, where psi_f(k) =
 * khat_r khat_t for the f-th pair (r <= t) of khat = [k; 1] (index 64 is the constant 1) in
 * this packed order:
 *   f in [0, 1792):     28 off-diagonal 8x8 blocks, (R, T) with R < T over the 8 blocks of 8
 *                       dims in lexicographic order; f = 64*block + 8*a + b <-> (8R+a, 8T+b)
 *   f in [1792, 2080):  8 diagonal blocks of 36 rows: (8R+a, 8R+b), a <= b, a-major
 *   f in [2080, 2144):  (r, 64): sum_j k_{j,r} [v_j; 1]   (H1 of eq. (4))
 *   f = 2144:           (64, 64): sum_j [v_j; 1]           (H0 of eq. (4))
 *   f in [2145, 2176):  zero padding
 * so rows with r, t < 64 hold H2_rt (= H2_tr) of eq. (4).  coef[h][f] is the readout weight
 * of row f for head h: (r == t ? 1 : 2) * M_{g(r),g(t)} * s_r * s_t with g(64) = 0,
 * s_r = 1/sqrt(dh) for r < 64, s_64 = 1, plus eps on f = 2144; u = sum_f coef[h][f] *
 * qhat_r qhat_t * (Hv | z)[f].  The header holds magic 0x534C414F ("OALS"), the ABI version,
 * B, Hq, Hkv, dh, dv, OAL_FEATURES_PAD (int32 each), the token count (int64 at byte 32) and
 * eps (fp32 at byte 40); bytes 44..255 are zero.  The buffer is the resumable artifact of
 * a sequence: copying it saves the sequence, copying it back resumes it. */
int oal_state_bytes(const oal_shape* s, size_t* bytes);

/* Scratch needed by oal_prefill for `s` (all fields used).  The contents need no
 * initialisation and are meaningless after the call.  On the tensor-core path (bf16, chunk
 * 128) it holds the bf16 chunk-state images and the fp32 chunk deltas, 913,920 bytes per
 * (b, kv head, chunk of 128 tokens), plus one 7,680-byte readout table per query head and
 * the fp32 intra-chunk normalisers (4 bytes per (b, query head, token)); on the CUDA-core
 * path the fp32 chunk states. */
int oal_prefill_workspace_bytes(const oal_shape* s, size_t* bytes);

/* Which kernels oal_prefill, oal_prefill_continue and oal_prefill_host run for `s`:
 * *path = OAL_PATH_TENSOR (bf16 inputs, chunk 128: tcgen05 tensor cores, bf16 operands and
 * fp32 accumulation) or OAL_PATH_CUDA_CORE (fp32 inputs, or chunk 64 or 256: fp32 CUDA-core
 * kernels).  Both compute eqs. (2)-(5); the choice changes speed and rounding, not the
 * result's definition.  Returns the shape-validation status of oal_prefill_workspace_bytes. */
typedef enum { OAL_PATH_CUDA_CORE = 0, OAL_PATH_TENSOR = 1 } oal_path;
int oal_prefill_path(const oal_shape* s, int* path);

/* Scratch needed by oal_decode_step for `s` (B, Hq, Hkv used): per-call partial readouts
 * (one per 240-row slab of each (b, kv) and query head), written and then read by the same
 * call, so its contents between calls do not matter.  (Its first 256-byte-aligned block is
 * reserved; earlier versions kept completion tickets there.) */
int oal_decode_workspace_bytes(const oal_shape* s, size_t* bytes);

/* Causal prefill of T tokens: writes out = yhat for every token (eqs. (2)-(5)) and fills
 * `state` (oal_state_bytes) with the prefix state after the last token plus the readout
 * coefficients, ready for oal_decode_step.  Chunked evaluation: within each chunk of C tokens
 * the kernel kappa is evaluated densely (eqs. (2)-(3)); across chunks the exclusive prefix
 * state of eq. (4) is built and read out with eq. (5).  Linear in T for fixed d_h.
 * bf16 inputs with chunk 128 run on tcgen05 tensor cores (bf16 operands, fp32 accumulation,
 * exact fp32 final state); fp32 inputs, and bf16 with chunk 64 or 256, run on CUDA cores in
 * fp32.  `workspace` must hold oal_prefill_workspace_bytes(s) bytes.  out == NULL computes
 * the state alone (no readout; q may then be NULL too), e.g. the per-segment state of a
 * sequence-parallel prefill. */
int oal_prefill(const void* q, const void* k, const void* v, const int32_t* group_id,
                const float* L, const int32_t* G, float eps, float* out, void* state,
                void* workspace, size_t workspace_bytes, const oal_shape* s, void* stream);

/* Prefill continuation: appends T tokens to the sequence whose prefix state `state` already
 * holds (a previous oal_prefill / oal_prefill_continue / oal_decode_step of the same B, Hq,
 * Hkv and the same group_id, L, G, eps).  out[b][h][t] is yhat of the t-th appended token,
 * which attends causally to every earlier token of the sequence (eqs. (2)-(5) with the
 * prefix sums of eq. (4) starting from the state); the state then holds the prefix after the
 * last appended token and its token count grows by T.  Equivalent to one oal_prefill over
 * the whole sequence, to the path's tolerance.  Only the tensor-core path (bf16, chunk 128)
 * continues a prefix; other dtypes or chunk sizes return OAL_ERR_UNSUPPORTED.  T == 0 or
 * B == 0 leaves the state untouched.  Other arguments and errors as oal_prefill. */
int oal_prefill_continue(const void* q, const void* k, const void* v, const int32_t* group_id,
                         const float* L, const int32_t* G, float eps, float* out, void* state,
                         void* workspace, size_t workspace_bytes, const oal_shape* s,
                         void* stream);

/* One autoregressive step for every sequence of the batch: q [B][Hq][1][dh],
 * k [B][Hkv][1][dh], v [B][Hkv][1][dv] (dtype of s).  Adds the new token to `state`
 * (eq. (4), rank-one update of every packed row) and writes out [B][Hq][1][dv] = yhat of the
 * new token (eq. (5), inclusive of it).  `state` must come from oal_prefill with the same
 * B, Hq, Hkv.  Memory-bound: every state row is read and written once. */
int oal_decode_step(const void* q, const void* k, const void* v, void* state, float* out,
                    void* workspace, size_t workspace_bytes, const oal_shape* s,
                    void* stream);

/* oal_decode_step without a workspace: allocates nothing and takes no scratch argument.
 * The paper has no counterpart; this is an interface for callers that cannot allocate
 * device memory: for example a serving engine that reserves all GPU memory for its own pool
 * at start-up and forbids allocation afterwards, a host framework whose plugin interface
 * hands an operator only its input and output buffers, or a latency-critical loop that
 * cannot afford cudaMalloc's implicit device-wide synchronisation.
 * Same arguments and results as oal_decode_step, minus the workspace.  The scratch is a
 * fixed 4 MiB array inside the library (one copy on every GPU that loads the library, held
 * until the process exits).  A step needs align256(4*B*Hkv) + 2340*B*Hq bytes of it; a step
 * that needs more than 4 MiB returns OAL_ERR_UNSUPPORTED without launching anything.  Every
 * B*Hq up to 1789 fits, whatever Hkv (batch 64 x 14 heads needs 2.1 MB).
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 * and caches it; make that first call before any stream capture.  cudaDeviceReset discards
 * the library's device code and data on that device, and with them the array the cached
 * address points to: do not call this entry point on a device after resetting it in the
 * same process.  Every call shares the one array, so calls that overlap on the GPU (on
 * different streams, or from threads that do not order their calls) race and corrupt each
 * other's results: issue them one after another. */
int oal_decode_step_noalloc(const void* q, const void* k, const void* v, void* state,
                            float* out, const oal_shape* s, void* stream);

/* The exact O(T^2) dense form (eqs. (2)-(3) summed over j <= i and normalised), for
 * cross-checking and timing against the linear-time path.  Same arguments as oal_prefill
 * without the state; `chunk` is ignored.  Computes in fp32 for both dtypes. */
int oal_dense_ref_gpu(const void* q, const void* k, const void* v, const int32_t* group_id,
                      const float* L, const int32_t* G, float eps, float* out,
                      const oal_shape* s, void* stream);

/* Contribution statistic of eq. (1) (same page, section 核心公式), per prompt p = (b, query
 * head h) and dimension r:
 *   chi[b][h][r] = (1/|Omega|) sum over causal pairs j <= i of |q_{b,h,i,r} k_{b,kv,j,r}| / sqrt(d_h)
 * with kv = floor(h * Hkv / Hq) and |Omega| = T (T + 1) / 2, the number of causal pairs of the
 * prompt (the page does not define Omega; this is the reading).  The page's chi_r is the mean
 * of chi[b][h][r] over the prompts b of a head.  q [B][Hq][T][64], k [B][Hkv][T][64] in the
 * dtype of `s`; chi [B][Hq][64] fp32; caller-owned device memory, 16-byte aligned.  Uses B, T,
 * Hq, Hkv, dh and dtype of `s` (chunk is ignored).  Accumulates in fp64 (an O(T d) prefix scan
 * of |k| per head).  B*T == 0 writes nothing and allows NULL pointers.  Errors: as
 * oal_prefill (shape, NULL, alignment). */
int oal_contribution_stat(const void* q, const void* k, float* chi, const oal_shape* s,
                          void* stream);

/* Launch mode of the tensor-core prefill (bf16, chunk 128), which runs as three kernels:
 * chunk deltas, the prefix scan over chunks, and the readout.  1 (default): the scan and the
 * readout are launched as programmatic dependents, so each is scheduled while its predecessor
 * drains and waits for it on the device.  0: plain stream order.  Both produce identical
 * results.  Process-wide; returns the previous setting. */
int oal_set_prefill_overlap(int overlap);

/* Test hook for the failure path of the tensor-core kernels.  While on, the inter-chunk
 * readout kernel of the tensor-core prefill (bf16, chunk 128, T > 128 or a continuation)
 * issues none of its copies, so every bounded wait in it runs out: after about one second the
 * kernel sets OAL_ERR_TIMEOUT in the device error word and every role leaves its loop (no copy
 * or MMA left in flight, tensor memory freed), and the context stays usable.  The output of
 * that call is undefined; the state and later calls are not affected.  Process-wide; returns
 * the previous setting.  Off by default; not for production use. */
int oal_set_debug_skip_copies(int on);

/* Prefill with the ungrouped Hadamard form: eq. (5) with free coefficients, that is
 *   kappa(q, k) = a + sum_r b_r x_r + sum_{r,t} C_rt x_r x_t,   x_r = q_r k_r / sqrt(d_h),
 * the relaxation of the Taylor kernel's shared coefficients that the abstract of arXiv
 * 2610.13674 describes (the grouped kernel of eq. (3) is the case a = eps + M_00,
 * b_r = 2 M_{0,g(r)}, C_rt = M_{g(r),g(t)}).  a [Hq], b [Hq][64], C [Hq][64][64] (row r,
 * column t) fp32 device arrays, 16-byte aligned; only the symmetric part of C matters.  The
 * kernel need not be positive: yhat = u[:dv] / u[dv] is a plain IEEE division.
 * bf16 inputs with chunk 128 run on tcgen05 tensor cores: the chunk states, prefix scan and
 * inter-chunk readout of oal_prefill with this coefficient table, and the intra-chunk part as
 * Phi(Q_c) Psi(K_c)^T over the 2176 packed rows (bf16 operands, fp32 accumulation).  fp32
 * inputs, and other chunk sizes, run on CUDA cores in fp32 with an O(T * chunk * d_h^2)
 * intra-chunk part.  Other arguments, the state (eps = 0 in its header; a holds the
 * constant), the workspace (oal_prefill_workspace_bytes) and errors as oal_prefill.
 * oal_decode_step continues the sequence. */
int oal_prefill_hadamard(const void* q, const void* k, const void* v, const float* a,
                         const float* b, const float* C, float* out, void* state,
                         void* workspace, size_t workspace_bytes, const oal_shape* s,
                         void* stream);

/* The dense O(T^2) form of the same kernel (causal, j <= i), fp32 on CUDA cores. */
int oal_dense_hadamard_gpu(const void* q, const void* k, const void* v, const float* a,
                           const float* b, const float* C, float* out, const oal_shape* s,
                           void* stream);

/* Scratch needed by oal_prefill_host for `s` cut into `segments` segments: device staging
 * for q, k, v and yhat of the whole call plus the prefill workspace of the longest segment. */
int oal_prefill_host_workspace_bytes(const oal_shape* s, int segments, size_t* bytes);

/* Prefill from HOST memory, with the copies overlapped with the kernels.  q_host, k_host and
 * v_host are host arrays in oal_prefill's layouts, and out_host receives yhat
 * [B][Hq][T][dv] fp32 in host memory.  They should be page-locked, or the copies will not
 * overlap.  group_id, L, G and state are device memory, as for oal_prefill.
 * The T tokens are cut into `segments` contiguous segments whose boundaries fall on chunk
 * boundaries (fewer when T is short). For each segment:
 *  - it is copied to the device on `copy_in`;
 *  - it is computed on `stream`: oal_prefill for the first segment, oal_prefill_continue for
 *    the others;
 *  - its yhat is copied back on `copy_out` while the next segment computes.
 * The continued prefix scan adds the chunk deltas in the order one whole prefill does, so
 * yhat and the state equal those of oal_prefill over the whole sequence.
 * `workspace` is device memory of oal_prefill_host_workspace_bytes(s, segments) bytes,
 * 256-byte aligned.  `stream`, `copy_in` and `copy_out` are caller-owned; a NULL copy stream
 * means `stream` (no overlap on that side).  The call returns once everything is enqueued.
 * The work is ordered after earlier work on `stream`, and later work on `stream` is ordered
 * after the last copy back.  Synchronise `stream` before reading out_host or reusing the host
 * inputs.
 * Errors: as oal_prefill; OAL_ERR_UNSUPPORTED for segments > 1 off the tensor-core path
 * (bf16, chunk 128); OAL_ERR_SHAPE for segments < 1; OAL_ERR_CUDA if a copy or event call
 * fails. */
int oal_prefill_host(const void* q_host, const void* k_host, const void* v_host,
                     const int32_t* group_id, const float* L, const int32_t* G, float eps,
                     float* out_host, void* state, void* workspace, size_t workspace_bytes,
                     const oal_shape* s, int segments, void* stream, void* copy_in,
                     void* copy_out);

/* Scratch needed by oal_prefill_varlen: n_streams slices of oal_prefill_workspace_bytes for
 * the longest sequence, each rounded up to 256 bytes.  seq_lens is host memory. */
int oal_prefill_varlen_workspace_bytes(const oal_shape* s, const int32_t* seq_lens, int n_seq,
                                       int n_streams, size_t* bytes);

/* Prefill of n_seq independent sequences of different lengths, packed back to back
 * (a variable-length batch).  seq_lens [n_seq] (host int32, each >= 0) gives T_i; with
 * o_i = T_0 + ... + T_{i-1}, sequence i is the B = 1 problem whose q block [Hq][T_i][dh]
 * starts at element o_i*Hq*dh of q, k and v blocks [Hkv][T_i][dh|dv] at o_i*Hkv*dh, and out
 * block [Hq][T_i][dv] (fp32) at o_i*Hq*dv.  Its state is written at states + i*state_stride
 * (state_stride: a multiple of 256, at least oal_state_bytes for B = 1).  Every sequence is
 * exactly an oal_prefill of its block; s gives Hq, Hkv, dh, dv, chunk and dtype (B and T are
 * ignored).  streams [n_streams] (host array of caller-owned streams): sequence i runs on
 * streams[i % n_streams] with workspace slice i % n_streams, so short sequences overlap.  The
 * work is ordered after earlier work on streams[0], and later work on streams[0] is ordered
 * after every sequence.  workspace: oal_prefill_varlen_workspace_bytes, 256-byte aligned.
 * Errors: as oal_prefill, OAL_ERR_SHAPE for a negative length, n_streams < 1 or a bad
 * stride. */
int oal_prefill_varlen(const void* q, const void* k, const void* v, const int32_t* group_id,
                       const float* L, const int32_t* G, float eps, float* out, void* states,
                       size_t state_stride, void* workspace, size_t workspace_bytes,
                       const oal_shape* s, const int32_t* seq_lens, int n_seq,
                       void* const* streams, int n_streams);

/* Scratch needed by oal_prefill_packed: the chunk states of every sequence (913,920 bytes per
 * (sequence, kv head, chunk of 128 tokens)), one 7,680-byte readout table per query head, the
 * intra-chunk normalisers (4 bytes per (token, query head)), 32 bytes of descriptor and three
 * 128-byte tensor maps per sequence.  seq_lens is host memory. */
int oal_prefill_packed_workspace_bytes(const oal_shape* s, const int32_t* seq_lens, int n_seq,
                                       size_t* bytes);

/* The variable-length batch of oal_prefill_varlen (same packed layout of q, k, v, out and the
 * states, same meaning of every argument) computed by one launch of each tensor-core kernel
 * for the whole batch on `stream`: the chunk deltas, intra-chunk sums, prefix scans and
 * readouts of all sequences share one grid each, so many short sequences fill the GPU
 * together.  Each sequence's results are those of an oal_prefill of its block (the same
 * per-chunk arithmetic and summation order).  Tensor-core path only: bf16 inputs with chunk
 * 128, else OAL_ERR_UNSUPPORTED.  workspace: oal_prefill_packed_workspace_bytes, 256-byte
 * aligned; states 256-byte aligned.  The descriptors and tensor maps are copied into the
 * workspace on `stream` from host memory that the call owns, so seq_lens may be reused on
 * return.  Errors: as oal_prefill_varlen. */
int oal_prefill_packed(const void* q, const void* k, const void* v, const int32_t* group_id,
                       const float* L, const int32_t* G, float eps, float* out, void* states,
                       size_t state_stride, void* workspace, size_t workspace_bytes,
                       const oal_shape* s, const int32_t* seq_lens, int n_seq, void* stream);

/* Scratch needed by oal_dense_backward_gpu for `s` (B, T, Hq used): per row of every query
 * head its normaliser, output, partial dM (81 floats) and partial deps. */
int oal_dense_backward_workspace_bytes(const oal_shape* s, size_t* bytes);

/* Gradients of the dense causal form (eqs. (2)-(3) summed over j <= i and normalised) for
 * the joint training of the kernel coefficients with the model.  dy = dLoss/dyhat
 * [B][Hq][T][dv] fp32.  Outputs (fp32, device): dq [B][Hq][T][dh]; dk [B][Hkv][T][dh] and
 * dv [B][Hkv][T][dv], summed over the query heads of each group; dL [Hq][OAL_G_MAX+1]^2,
 * zero outside each head's leading (G+1)x(G+1) block; deps, one float (eps is shared).
 * By the chain rule: dkappa_ij = dy_i . (v_j - yhat_i) / D_i, dkappa/dsbar = 2 M sbar,
 * dL = (dM + dM^T) L.  Deterministic: every output is summed in a fixed order.  O(B Hq T^2
 * dh) on CUDA cores in fp32 for both input dtypes: a reference-scale gradient.  workspace:
 * oal_dense_backward_workspace_bytes, 256-byte aligned.  Errors as oal_prefill. */
int oal_dense_backward_gpu(const void* q, const void* k, const void* v, const int32_t* group_id,
                           const float* L, const int32_t* G, float eps, const float* dy,
                           float* dq, float* dk, float* dv, float* dL, float* deps,
                           void* workspace, size_t workspace_bytes, const oal_shape* s,
                           void* stream);

/* Scratch needed by oal_backward for `s` (B, T, Hq, Hkv used): a state buffer
 * (oal_state_bytes), the fp32 prefix and suffix chunk states (2 x 565,760 bytes per
 * (b, kv head, chunk of 64 tokens)), per row of every query head its normaliser (1 float),
 * output (64), upstream gradient of u (65), partial dM (81) and deps (1), one partial dC'
 * (2176 floats) per (b, query head, chunk) and one float per query head; each part starts
 * on a 256-byte boundary. */
int oal_backward_workspace_bytes(const oal_shape* s, size_t* bytes);

/* Training-scale gradients: the same outputs, layouts and conventions as
 * oal_dense_backward_gpu (dq, dk, dv, dL, deps for dy = dLoss/dyhat), computed as the chunked
 * reverse of the prefill in O(T) per head instead of O(T^2).  With g_i = dLoss/du_i =
 * [dy_i / D_i ; -(dy_i . yhat_i) / D_i] and the packed feature map of eq. (5), pairs inside a
 * 64-token chunk are differentiated directly (eqs. (2)-(3)); pairs across chunks through the
 * exclusive prefix states S_c = sum psi_j [v_j; 1]^T (eq. (4), as in the prefill) and the
 * exclusive suffix states R_c = sum phi_i g_i^T of the readout gradient: dphi(q_i) = S_c g_i,
 * dpsi(k_j) = R_c [v_j; 1], d[v_j; 1] += R_c^T psi(k_j), and dC' = sum_i dphi(q_i) o
 * (qhat_r qhat_t) mapped through C' = (2 - [r = t]) M_{g(r)g(t)} s_r s_t (+ eps) to dM and
 * dL = (dM + dM^T) L.  It recomputes yhat and D_i with the fp32 prefill first.  fp32 on CUDA
 * cores for both input dtypes; deterministic (every sum in a fixed order).  workspace:
 * oal_backward_workspace_bytes, 256-byte aligned.  Errors as oal_dense_backward_gpu. */
int oal_backward(const void* q, const void* k, const void* v, const int32_t* group_id,
                 const float* L, const int32_t* G, float eps, const float* dy, float* dq,
                 float* dk, float* dv, float* dL, float* deps, void* workspace,
                 size_t workspace_bytes, const oal_shape* s, void* stream);

/* Sum of prefix states: out[i] = parts[0*n + i] + parts[1*n + i] + ... for the n_parts
 * arrays of n floats stored back to back in `parts`, added in that order (the prefix state of
 * eq. (4) is a sum over tokens, so summing the states of a sequence's first segments, each
 * computed alone, gives the state after them).  Used on the fp32 body of state buffers (the
 * part after the header and the coefficient tables) by the sequence-parallel prefill.
 * n_parts = 0 writes zeros.  Device pointers, 16-byte aligned; n a multiple of 4 when
 * n_parts > 0.  `out` must not overlap `parts`. */
int oal_state_prefix_sum(const float* parts, int n_parts, size_t n, float* out, void* stream);

/* Reads the device-side error word (OAL_OK or a negative oal_status set by a kernel since
 * the last read), synchronising `stream`, and clears it. */
int oal_device_error(int* code, void* stream);

/* Tracing.  Every kernel launch of the library is counted; while tracing is on, each launch
 * also records a CUDA event pair on its own stream.  oal_profile_read waits for the recorded
 * events, returns per-kernel totals (launches, summed device time) since the previous read,
 * and forgets them.  Tracing costs two event records per launch; leave it off in production. */
typedef struct {
    char name[40];
    int32_t launches;
    double total_ms;
} oal_kernel_stat;

int oal_profile_enable(int on);
int oal_profile_read(oal_kernel_stat* stats, int max_stats, int* n_stats);
/* Kernels launched by this library since it was loaded (all devices, all streams). */
unsigned long long oal_launch_count(void);

/* The CUDA runtime error (cudaError_t value; 0 = none) behind the most recent OAL_ERR_CUDA
 * returned by any call in this process, with its name and description written into buf
 * (NUL-terminated, truncated to len bytes; buf may be NULL). */
int oal_last_cuda_error(char* buf, size_t len);

/* Static description of a status code. */
const char* oal_status_string(int status);

/* OAL_ABI_VERSION of the loaded library. */
int oal_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OAL_H */
