"""The seeded input generator (positive_quadratic_b200/inputs.py) against the recipe it states:
bf16 rounding, rotary rotation, outlier scaling, tail-group partitions and the L factors.
Both the CUDA path and the oracle receive these arrays, so a mistake here would hide from the
parity tests; these checks use only properties that hold by definition."""
import numpy as np
import pytest
import torch

from positive_quadratic_b200 import inputs as I


def test_round_bf16_matches_torch():
    """Round to nearest even onto the bf16 grid, as torch's float32 -> bfloat16 cast does,
    including exact ties, subnormals, signed zeros and infinities."""
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact ties: a bf16 value plus half an ulp (bit 15 set, lower bits zero)
        (rng.integers(0, 1 << 15, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 1e-40, -1e-40, 3.4e38], np.float32),
    ]).astype(np.float32)
    x = x[np.isfinite(x) | np.isinf(x)]
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float32).numpy()
    got = I.round_bf16(x)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_rope_rotation_properties():
    """Rotate-half rotary embedding: position 0 is the identity, each pair (r, r + 32) keeps
    its norm, and the dot product of a rotated pair depends only on the position offset."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    y = rng.standard_normal((5, 64)).astype(np.float32)
    np.testing.assert_allclose(I.rope_rotate(x[:1], 0), x[:1], rtol=0, atol=1e-7)
    rx = I.rope_rotate(x, 17)
    pair = lambda a: a[:, :32] ** 2 + a[:, 32:] ** 2  # noqa: E731
    np.testing.assert_allclose(pair(rx), pair(x), rtol=2e-5, atol=1e-5)
    # <R(a) x, R(b) y> = <R(a + s) x, R(b + s) y> for single tokens at positions a, b
    d1 = (I.rope_rotate(x[:1], 3) * I.rope_rotate(y[:1], 11)).sum()
    d2 = (I.rope_rotate(x[:1], 1003) * I.rope_rotate(y[:1], 1011)).sum()
    assert abs(d1 - d2) < 1e-3 * (1 + abs(d1))
    # the first pair (r = 0, frequency base^0 = 1) turns by one radian per position
    e = np.zeros((1, 64), np.float32)
    e[0, 0] = 1.0
    r = I.rope_rotate(e, 1)
    np.testing.assert_allclose([r[0, 0], r[0, 32]], [np.cos(1.0), np.sin(1.0)], atol=1e-6)


@pytest.mark.parametrize("seed,Hq,Hkv", [(1, 14, 2), (2, 8, 1), (3, 4, 4)])
def test_groups_partition_the_outlier_dims(seed, Hq, Hkv):
    p = I.small_layer(seed, B=1, T=8, Hq=Hq, Hkv=Hkv, dtype="bf16")
    grp = Hq // Hkv
    for kv, (dims, scales) in enumerate(p.meta["outliers"]):
        assert 2 <= len(dims) <= 6 and len(set(dims)) == len(dims)
        assert all(4 <= s <= 12 and float(s).is_integer() for s in scales)
        for h in range(kv * grp, (kv + 1) * grp):
            G = int(p.G[h])
            assert 2 <= G <= 1 + min(5, len(dims)) <= I.GMAX
            gid = p.group_id[h]
            assert set(np.flatnonzero(gid != 1)) == set(dims)       # tail = the outliers
            assert set(gid.tolist()) == set(range(1, G + 1))          # every group non-empty
            Lh = p.L[h]
            n = G + 1
            assert np.all(np.triu(Lh[:n, :n], 1) == 0)                # lower triangular
            assert np.all((np.diag(Lh)[:n] >= 0.5) & (np.diag(Lh)[:n] <= 1.5))
            assert not Lh[n:].any() and not Lh[:, n:].any()           # zero outside its slot


def test_outlier_energy_survives_the_rotation():
    """Rotation keeps each pair's energy, so a pair (r, r + 32) of q or k holds on average
    s_r^2 + s_{r+32}^2, with s = the outlier scale (1 for bulk dims)."""
    p = I.small_layer(9, B=1, T=4096, Hq=2, Hkv=1, dtype="f32")
    dims, scales = p.meta["outliers"][0]
    s = np.ones(64)
    s[dims] = scales
    want = s[:32] ** 2 + s[32:] ** 2
    for x in (p.k[0, 0], p.q[0, 0], p.q[0, 1]):
        e = (x[:, :32].astype(np.float64) ** 2 + x[:, 32:] ** 2).mean(axis=0)
        np.testing.assert_allclose(e, want, rtol=0.12)


def test_generator_is_deterministic_and_rounded():
    a = I.small_layer(4, B=2, T=50, Hq=4, Hkv=2, dtype="bf16")
    b = I.small_layer(4, B=2, T=50, Hq=4, Hkv=2, dtype="bf16")
    for name in ("q", "k", "v", "group_id", "L", "G"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    for x in (a.q, a.k, a.v):
        assert np.array_equal(I.round_bf16(x), x)                     # on the bf16 grid
    c = I.small_layer(5, B=2, T=50, Hq=4, Hkv=2, dtype="bf16")
    assert not np.array_equal(a.q, c.q)
    s = a.slice_tokens(10, 30)
    assert np.array_equal(s.q, a.q[:, :, 10:30]) and s.group_id is a.group_id


def test_config_shapes():
    p = I.config1()
    assert p.shape == dict(B=1, Hq=14, Hkv=2, T=4096, dh=64, dv=64) and p.dtype == "bf16"
    z = I.config0()
    assert z.shape == dict(B=1, Hq=1, Hkv=1, T=256, dh=64, dv=64) and z.dtype == "f32"
    assert int(z.G[0]) == 4 and np.bincount(z.group_id[0])[1:].tolist() == [60, 2, 1, 1]
