"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on the same seeded
inputs.  Tolerances (row-relative max error, tests/_metrics.py): 1e-4 for fp32 inputs, 2e-2
for bf16 inputs with fp32 accumulation.  Full-size workloads run in the benchmark's launch
configuration and are checked on outputs the oracle can afford (sampled batch elements,
layers or rows)."""
import numpy as np
import pytest

import oracle
from positive_quadratic_b200 import inputs as I
from tests._metrics import TOL_BF16, TOL_F32, row_rel_err
from tests._packed import F, FP, coef_from_header, pack_oracle_state, read_state

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def oal(cuda):
    from positive_quadratic_b200 import build, oal as binding
    build.build()
    binding.lib()
    return binding


def dev_inputs(p, dev):
    dt = torch.bfloat16 if p.dtype == "bf16" else torch.float32
    t = lambda a, d=None: torch.from_numpy(np.ascontiguousarray(a)).to(dev, d)  # noqa: E731
    return (t(p.q, dt), t(p.k, dt), t(p.v, dt), t(p.group_id), t(p.L), t(p.G))


def tol(p):
    return TOL_BF16 if p.dtype == "bf16" else TOL_F32


def gpu_prefill(oal, p, dev, chunk=128):
    q, k, v, g, L, G = dev_inputs(p, dev)
    out, state = oal.prefill(q, k, v, g, L, G, p.eps, chunk)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    return out.cpu().numpy(), state


# --- config 0: tiny fp32 ---------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_config0_prefill_f32(oal, cuda, chunk):
    p = I.config0()
    ref = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    y, _ = gpu_prefill(oal, p, cuda, chunk)
    assert row_rel_err(y, ref) <= TOL_F32


def test_config0_dense_ref_f32(oal, cuda):
    p = I.config0()
    ref = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    q, k, v, g, L, G = dev_inputs(p, cuda)
    y = oal.dense_ref(q, k, v, g, L, G, p.eps).cpu().numpy()
    assert row_rel_err(y, ref) <= TOL_F32


# --- ragged sizes, GQA, both dtypes ---------------------------------------------------------

@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 127, 128, 129, 255, 257, 700])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_prefill(oal, cuda, T, dtype):
    p = I.small_layer(200 + T, B=2, T=T, Hq=4, Hkv=2, dtype=dtype)
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    for chunk in (64, 128, 256):
        y, _ = gpu_prefill(oal, p, cuda, chunk)
        assert row_rel_err(y, ref) <= tol(p), (chunk, row_rel_err(y, ref))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_ref_gqa(oal, cuda, dtype):
    p = I.small_layer(300, B=2, T=333, Hq=14, Hkv=2, dtype=dtype)
    ref = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    q, k, v, g, L, G = dev_inputs(p, cuda)
    y = oal.dense_ref(q, k, v, g, L, G, p.eps).cpu().numpy()
    assert row_rel_err(y, ref) <= tol(p)


def test_group_count_extremes(oal, cuda):
    rng = np.random.default_rng(5)
    p = I.small_layer(301, B=1, T=300, Hq=4, Hkv=1, dtype="f32")
    p.G[:] = [1, 8, 8, 2]
    p.group_id[0] = 1
    for h in (1, 2):
        p.group_id[h] = rng.integers(1, 9, size=64)
        p.group_id[h, :8] = np.arange(1, 9)
        p.L[h] = I.random_L(rng, 8)
    p.group_id[3] = 1
    p.group_id[3, 5] = 2
    p.L[0] = I.random_L(rng, 1)
    p.L[3] = I.random_L(rng, 2)
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    y, _ = gpu_prefill(oal, p, cuda, 128)
    assert row_rel_err(y, ref) <= TOL_F32


def test_empty_inputs(oal, cuda):
    p = I.small_layer(302, B=1, T=0, Hq=2, Hkv=1, dtype="bf16")
    y, state = gpu_prefill(oal, p, cuda, 128)
    assert y.shape == (1, 2, 0, 64)
    hdr, _, S = read_state(state.cpu().numpy(), 1, 2, 1)
    assert hdr["tokens"] == 0 and np.all(S == 0)
    p0 = I.small_layer(303, B=0, T=16, Hq=2, Hkv=1, dtype="bf16")
    y0, _ = gpu_prefill(oal, p0, cuda, 128)
    assert y0.shape == (0, 2, 16, 64)


def test_output_canary(oal, cuda):
    """Nothing is written past the end of `out`."""
    p = I.small_layer(304, B=1, T=190, Hq=2, Hkv=1, dtype="bf16")
    q, k, v, g, L, G = dev_inputs(p, cuda)
    n = 1 * 2 * 190 * 64
    big = torch.full((n + 4096,), 12345.0, device=cuda)
    out = big[:n].view(1, 2, 190, 64)
    oal.prefill(q, k, v, g, L, G, p.eps, 128, out=out)
    torch.cuda.synchronize()
    assert torch.all(big[n:] == 12345.0)


def test_bad_group_id_sets_error_word(oal, cuda):
    p = I.small_layer(305, B=1, T=64, Hq=2, Hkv=1, dtype="bf16")
    p.group_id[1, 3] = 0
    q, k, v, g, L, G = dev_inputs(p, cuda)
    out, _ = oal.prefill(q, k, v, g, L, G, p.eps, 128)
    torch.cuda.synchronize()
    assert oal.device_error() == -5
    assert oal.device_error() == 0  # cleared by the read
    assert torch.isfinite(out).all()


# --- state layout, coefficients, decode ------------------------------------------------------

def _coef_reference(p):
    """Readout weights of the packed rows per include/oal.h, from L and the group ids."""
    return coef_from_header(p.group_id, p.L, p.G, p.eps)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_state_and_coefficients(oal, cuda, dtype):
    p = I.small_layer(306, B=2, T=333, Hq=4, Hkv=2, dtype=dtype)
    _, st = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_state=True)
    _, state = gpu_prefill(oal, p, cuda, 128)
    hdr, coef, S = read_state(state.cpu().numpy(), 2, 4, 2)
    assert hdr["magic"] == 0x534C414F and hdr["tokens"] == 333 and hdr["feat_pad"] == FP
    assert (hdr["B"], hdr["Hq"], hdr["Hkv"], hdr["dh"], hdr["dv"]) == (2, 4, 2, 64, 64)
    np.testing.assert_allclose(coef, _coef_reference(p), rtol=1e-6, atol=1e-9)
    ref = pack_oracle_state(st)
    scale = np.abs(ref).max(axis=2, keepdims=True)
    assert np.max(np.abs(S[:, :, :F] - ref) / scale) < 1e-5
    assert np.all(S[:, :, F:] == 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_continuation(oal, cuda, dtype):
    """prefill(T) + n decode steps == prefill(T + n) (outputs and state)."""
    T0, n = 200, 6
    p = I.small_layer(307, B=3, T=T0 + n, Hq=14, Hkv=2, dtype=dtype)
    y_all, st_all = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps,
                                     return_state=True)
    pre = p.slice_tokens(0, T0)
    _, state = gpu_prefill(oal, pre, cuda, 128)
    ws = oal.decode_workspace(3, 14, 2, cuda)
    q, k, v, _, _, _ = dev_inputs(p, cuda)
    for t in range(T0, T0 + n):
        sl = lambda x: x[:, :, t:t + 1].contiguous()  # noqa: E731
        y = oal.decode_step(sl(q), sl(k), sl(v), state, ws)
        torch.cuda.synchronize()
        assert row_rel_err(y.cpu().numpy()[:, :, 0], y_all[:, :, t]) <= tol(p)
    assert oal.device_error() == 0
    assert torch.all(ws[:256] == 0)  # the reserved leading block is never written
    hdr, _, S = read_state(state.cpu().numpy(), 3, 14, 2)
    assert hdr["tokens"] == T0 + n
    ref = pack_oracle_state(st_all)
    assert np.max(np.abs(S[:, :, :F] - ref) / np.abs(ref).max(axis=2, keepdims=True)) < 1e-5


def test_decode_workspace_contents_do_not_matter(oal, cuda):
    """A decode step writes every scratch word it reads: a workspace full of garbage gives the
    same outputs and state, bit for bit, as a zero-filled one."""
    p = I.small_layer(309, B=2, T=65, Hq=14, Hkv=2, dtype="bf16")
    pre = p.slice_tokens(0, 64)
    q, k, v, _, _, _ = dev_inputs(p, cuda)
    sl = lambda x: x[:, :, 64:65].contiguous()  # noqa: E731
    res = []
    for fill in (0, 0xFF):
        _, state = gpu_prefill(oal, pre, cuda, 128)
        ws = oal.decode_workspace(2, 14, 2, cuda)
        ws.fill_(fill)
        y = oal.decode_step(sl(q), sl(k), sl(v), state, ws)
        torch.cuda.synchronize()
        res.append((y.clone(), state.clone()))
    assert oal.device_error() == 0
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


def test_chunk_size_independence(oal, cuda):
    p = I.small_layer(308, B=1, T=1000, Hq=4, Hkv=2, dtype="f32")
    ys = [gpu_prefill(oal, p, cuda, c)[0] for c in (64, 128, 256)]
    assert row_rel_err(ys[1], ys[0]) < 2e-5 and row_rel_err(ys[2], ys[0]) < 2e-5


# --- full-size workloads (benchmark launch configuration), sampled checks ---------------------

def test_config1_full(oal, cuda):
    p = I.config1()
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    y, _ = gpu_prefill(oal, p, cuda, 128)
    err = row_rel_err(y, ref)
    print(f"config1 max row-relative error {err:.3e}")
    assert err <= TOL_BF16


@pytest.mark.parametrize("layer", [0, 17])
def test_config2_sampled(oal, cuda, layer):
    p = I.config2_layer(layer)
    y, _ = gpu_prefill(oal, p, cuda, 128)
    for b in (0, 7):
        s = p.slice_batch(b, b + 1)
        ref = oracle.recurrent(s.q, s.k, s.v, s.group_id, s.L, s.G, s.eps)
        assert row_rel_err(y[b:b + 1], ref) <= TOL_BF16, (layer, b)


@pytest.mark.parametrize("T", [16384, 32768, 65536])
def test_config3_sampled_rows(oal, cuda, T):
    p = I.config3(T)
    rng = np.random.default_rng(T)
    rows = [(0, int(h), int(i)) for h, i in zip(rng.integers(0, 14, 12), rng.integers(0, T, 12))]
    rows += [(0, 0, 0), (0, 13, T - 1), (0, 6, T // 2)]
    ref = oracle.dense_rows(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, rows)
    for chunk in ((64, 128, 256) if T == 16384 else (128,)):
        y, _ = gpu_prefill(oal, p, cuda, chunk)
        got = np.stack([y[b, h, i] for b, h, i in rows])
        assert row_rel_err(got, ref) <= TOL_BF16, chunk


def test_config4_decode_sampled(oal, cuda):
    p = I.config4(batch=64, context=4096, steps=4)
    pre = p.slice_tokens(0, 4096)
    _, state = gpu_prefill(oal, pre, cuda, 128)
    ws = oal.decode_workspace(64, 14, 2, cuda)
    q, k, v, _, _, _ = dev_inputs(p, cuda)
    ys = []
    for t in range(4096, 4100):
        sl = lambda x: x[:, :, t:t + 1].contiguous()  # noqa: E731
        ys.append(oal.decode_step(sl(q), sl(k), sl(v), state, ws).cpu().numpy()[:, :, 0])
    assert oal.device_error() == 0
    for b in (0, 41):
        s = p.slice_batch(b, b + 1)
        ref = oracle.recurrent(s.q, s.k, s.v, s.group_id, s.L, s.G, s.eps)
        for n, t in enumerate(range(4096, 4100)):
            assert row_rel_err(ys[n][b:b + 1], ref[:, :, t]) <= TOL_BF16, (b, t)


def test_config4_decode_all_steps(oal, cuda):
    """Config 4 as the benchmark runs it: batch 64, 4096-token context prefilled, then all 256
    single-token steps.  Sampled batch elements are checked against the oracle's recurrence
    over the whole 4352-token sequence at every step, and their fp32 states after the last
    step against the oracle's prefix state."""
    steps, ctx = 256, 4096
    p = I.config4(batch=64, context=ctx, steps=steps)
    pre = p.slice_tokens(0, ctx)
    _, state = gpu_prefill(oal, pre, cuda, 128)
    ws = oal.decode_workspace(64, 14, 2, cuda)
    q, k, v, _, _, _ = dev_inputs(p, cuda)
    out = torch.empty(64, 14, steps, 64, dtype=torch.float32, device=cuda)
    y1 = torch.empty(64, 14, 1, 64, dtype=torch.float32, device=cuda)
    for n, t in enumerate(range(ctx, ctx + steps)):
        sl = lambda x: x[:, :, t:t + 1].contiguous()  # noqa: E731
        oal.decode_step(sl(q), sl(k), sl(v), state, ws, out=y1)
        out[:, :, n] = y1[:, :, 0]
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    y = out.cpu().numpy()
    _, _, S = read_state(state.cpu().numpy(), 64, 14, 2)
    for b in (3, 50):
        s = p.slice_batch(b, b + 1)
        ref, st = oracle.recurrent(s.q, s.k, s.v, s.group_id, s.L, s.G, s.eps,
                                   return_state=True)
        assert row_rel_err(y[b:b + 1], ref[:, :, ctx:]) <= TOL_BF16, b
        refS = pack_oracle_state(st)
        err = np.max(np.abs(S[b:b + 1, :, :F] - refS) / np.abs(refS).max(axis=2, keepdims=True))
        assert err < 1e-5, (b, err)


# --- tensor-core prefill schedules --------------------------------------------------------------

@pytest.mark.parametrize("overlap", [True, False])
@pytest.mark.parametrize("T,B", [(129, 1), (300, 2), (1000, 3), (2048, 1)])
def test_tensor_prefill_schedules(oal, cuda, overlap, T, B):
    """bf16, chunk 128 runs on the tcgen05 kernels (chunk deltas, prefix scan, readout),
    with and without programmatic dependent launch: outputs and exact final state match the
    oracle."""
    p = I.small_layer(500 + T, B=B, T=T, Hq=14, Hkv=2, dtype="bf16")
    ref, st = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_state=True)
    prev = oal.set_prefill_overlap(overlap)
    try:
        oal.profile_read()
        oal.profile_enable(True)
        y, state = gpu_prefill(oal, p, cuda, 128)
        oal.profile_enable(False)
        names = set(oal.profile_read())
    finally:
        oal.set_prefill_overlap(prev)
    assert {"delta_tc", "scan", "readout_tc"} <= names, names
    assert row_rel_err(y, ref) <= TOL_BF16
    _, _, S = read_state(state.cpu().numpy(), B, 14, 2)
    refS = pack_oracle_state(st)
    assert np.max(np.abs(S[:, :, :F] - refS) / np.abs(refS).max(axis=2, keepdims=True)) < 1e-5


def test_tensor_schedules_agree(oal, cuda):
    p = I.config1()
    prev = oal.set_prefill_overlap(True)
    try:
        y1, _ = gpu_prefill(oal, p, cuda, 128)
        oal.set_prefill_overlap(False)
        y2, _ = gpu_prefill(oal, p, cuda, 128)
    finally:
        oal.set_prefill_overlap(prev)
    np.testing.assert_array_equal(y1, y2)


# --- contribution statistic, eq. (1) -----------------------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 7, 300, 1000])
def test_contribution_stat(oal, cuda, T, dtype):
    p = I.small_layer(900 + T, B=2, T=T, Hq=4, Hkv=2, dtype=dtype)
    ref = oracle.chi(p.q, p.k)
    q, k, *_ = dev_inputs(p, cuda)
    chi = oal.contribution_stat(q, k).cpu().numpy()
    assert oal.device_error() == 0
    np.testing.assert_allclose(chi, ref, rtol=1e-5, atol=0)


@pytest.mark.gpu
def test_contribution_stat_config1(oal, cuda):
    """Config-1 layer shape (14/2 heads, outliers), first 2048 tokens; the page's chi_r is
    the mean over prompts, here the single prompt of each head."""
    p = I.config1().slice_tokens(0, 2048)
    ref = oracle.chi(p.q, p.k)
    q, k, *_ = dev_inputs(p, cuda)
    chi = oal.contribution_stat(q, k).cpu().numpy()
    np.testing.assert_allclose(chi, ref, rtol=1e-5, atol=0)
    # the outlier dimensions dominate the statistic, as the grouping assumes
    assert np.all(chi.max(axis=-1) > 4 * np.median(chi, axis=-1))


# --- prefill continuation ----------------------------------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("T1,T2", [(200, 1), (256, 300), (129, 700), (1000, 128)])
def test_prefill_continuation(oal, cuda, T1, T2):
    """prefill(T1) then continue(T2) = one prefill of T1 + T2 tokens: outputs of the appended
    tokens and the final state match the oracle run over the whole sequence."""
    p = I.small_layer(700 + T1 + T2, B=2, T=T1 + T2, Hq=14, Hkv=2, dtype="bf16")
    ref, st = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_state=True)
    a, b = p.slice_tokens(0, T1), p.slice_tokens(T1, T1 + T2)
    qa, ka, va, g, L, G = dev_inputs(a, cuda)
    qb, kb, vb, *_ = dev_inputs(b, cuda)
    _, state = oal.prefill(qa, ka, va, g, L, G, p.eps, 128)
    yb = oal.prefill_continue(qb, kb, vb, g, L, G, p.eps, state)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    assert row_rel_err(yb.cpu().numpy(), ref[:, :, T1:]) <= TOL_BF16
    hdr, _, S = read_state(state.cpu().numpy(), 2, 14, 2)
    assert hdr["tokens"] == T1 + T2
    refS = pack_oracle_state(st)
    assert np.max(np.abs(S[:, :, :F] - refS) / np.abs(refS).max(axis=2, keepdims=True)) < 1e-5


@pytest.mark.gpu
def test_state_saved_to_a_file_resumes_the_sequence(oal, cuda, tmp_path):
    """The state buffer is the resumable artifact of a sequence: written to a file after a
    prefill and read back into another device buffer (at another address), it continues the
    sequence exactly as the original buffer does -- a prefill continuation, then decode
    steps -- outputs and state bit for bit."""
    T1, T2, n = 256, 300, 3
    p = I.small_layer(733, B=2, T=T1 + T2 + n, Hq=14, Hkv=2, dtype="bf16")
    a, b = p.slice_tokens(0, T1), p.slice_tokens(T1, T1 + T2)
    qa, ka, va, g, L, G = dev_inputs(a, cuda)
    qb, kb, vb, *_ = dev_inputs(b, cuda)
    q, k, v, *_ = dev_inputs(p, cuda)
    _, state = oal.prefill(qa, ka, va, g, L, G, p.eps, 128)
    torch.cuda.synchronize()
    path = tmp_path / "sequence.state"
    state.cpu().numpy().tofile(path)
    raw = torch.from_numpy(np.fromfile(path, dtype=np.uint8))
    arena = torch.zeros(raw.numel() + 1024, dtype=torch.uint8, device=cuda)
    resumed = arena[512:512 + raw.numel()]
    resumed.copy_(raw.to(cuda))
    assert torch.equal(resumed, state)
    ws = oal.decode_workspace(2, 14, 2, cuda)
    runs = []
    for st in (state, resumed):
        ys = [oal.prefill_continue(qb, kb, vb, g, L, G, p.eps, st)]
        for t in range(T1 + T2, T1 + T2 + n):
            sl = lambda x: x[:, :, t:t + 1].contiguous()  # noqa: E731
            ys.append(oal.decode_step(sl(q), sl(k), sl(v), st, ws))
        torch.cuda.synchronize()
        runs.append(([y.clone() for y in ys], st.clone()))
    assert oal.device_error() == 0
    for y0, y1 in zip(runs[0][0], runs[1][0]):
        assert torch.equal(y0, y1)
    assert torch.equal(runs[0][1], runs[1][1])
    assert torch.all(arena[:512] == 0) and torch.all(arena[512 + raw.numel():] == 0)
    hdr, _, _ = read_state(runs[1][1].cpu().numpy(), 2, 14, 2)
    assert hdr["tokens"] == T1 + T2 + n


@pytest.mark.gpu
def test_prefill_continuation_unsupported_paths(oal, cuda):
    """Continuation runs on the tensor-core path only; fp32 inputs are refused before any
    launch."""
    p = I.small_layer(31, B=1, T=64, Hq=4, Hkv=2, dtype="f32")
    q, k, v, g, L, G = dev_inputs(p, cuda)
    _, state = oal.prefill(q, k, v, g, L, G, p.eps, 128)
    with pytest.raises(oal.OALError):
        oal.prefill_continue(q, k, v, g, L, G, p.eps, state)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,chunk", [("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_state_only_prefill(oal, cuda, dtype, chunk):
    """out = NULL computes the same state as a full prefill, without the readout."""
    p = I.small_layer(77, B=2, T=300, Hq=4, Hkv=2, dtype=dtype)
    q, k, v, g, L, G = dev_inputs(p, cuda)
    _, full = oal.prefill(q, k, v, g, L, G, p.eps, chunk)
    oal.profile_read()
    oal.profile_enable(True)
    alone = oal.prefill_state(k, v, g, L, G, p.eps, 4, chunk)
    oal.profile_enable(False)
    names = set(oal.profile_read())
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    assert not any(n.startswith("readout") for n in names), names
    # defined bytes: header fields (0..44), coefficient tables and prefix states (256..)
    assert torch.equal(full[:44], alone[:44])
    assert torch.equal(full[256:], alone[256:])


@pytest.mark.gpu
@pytest.mark.parametrize("T,segments,B", [(1000, 4, 2), (512, 2, 1), (130, 4, 1), (256, 1, 2)])
def test_prefill_from_host_buffers(oal, cuda, T, segments, B):
    """oal_prefill_host: host q/k/v, segments copied in and yhat copied out on their own
    streams while the next segment computes.  Chunk-aligned segments continue the prefix
    scan in one prefill's order, so yhat and the state equal a device-resident oal_prefill
    bit for bit; both match the oracle."""
    p = I.small_layer(900 + T, B=B, T=T, Hq=14, Hkv=2, dtype="bf16")
    q, k, v, g, L, G = dev_inputs(p, cuda)
    ref_out, ref_state = oal.prefill(q, k, v, g, L, G, p.eps, 128)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    bufs = oal.host_prefill_buffers(hq, hk, hv, g, L, G, 128, segments, device=cuda)
    hout = oal.prefill_from_host(hq, hk, hv, p.eps, bufs)
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    # the same kernels and the same order of every floating-point sum: bit-equal
    assert torch.equal(hout, ref_out.cpu())
    st, rs = bufs["state"], ref_state
    assert torch.equal(st[:44], rs[:44])
    assert torch.equal(st[256:], rs[256:])
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    assert row_rel_err(hout.numpy(), ref) <= TOL_BF16
