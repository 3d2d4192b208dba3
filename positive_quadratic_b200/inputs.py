"""Seeded synthetic inputs for OAL attention, shared by the tests, the benchmark and the oracle.

This module holds random draws and data shaping only (outlier scaling, rotary position
rotation of the inputs, bf16 rounding, group partitions); none of the attention arithmetic.
Both the CUDA path and the fp64 oracle receive exactly the arrays produced here.

Workload shapes follow the OAL reproduction note of arXiv 2610.13674 ("OAL: 按 QK 离群贡献
分组的正二次注意力核"): Qwen2.5-0.5B attention layers (14 query heads, 2 key/value heads, head
dim 64, post-RoPE q/k, middle layers 3-20 converted; section 数据协议 and Figure 2(a), where one
head has 60 bulk dimensions sharing a group and the high-contribution tail split into a few
small groups).  The pages publish no tensors, so every value here is synthetic:

* q, k, v ~ N(0, 1); per key/value head 2-6 "outlier" dimensions of q and k are scaled by an
  integer factor in 4..12 (config 0: 4 tail dimensions scaled by 8).
* q and k are then rotated by rotary position embedding with base 1e6 (rotate-half pairing
  of dims r and r+32), positions starting at ``pos0``; the kernels never apply it.
* each query head draws 1..min(5, n_outliers) tail groups as a random partition of its
  key/value head's outlier dims; every other dim is in the bulk group 1 (G = 1 + n_tail).
* L per query head is (G+1)x(G+1) lower triangular, diagonal ~ U(0.5, 1.5), strictly lower
  entries ~ N(0, 0.3^2); stored in a [Gmax+1, Gmax+1] slot (Gmax = 8), zero elsewhere.
* bf16 workloads are rounded to the bf16 grid (round to nearest even) here, so both sides
  see identical values and parity measures the computation, not input quantisation.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GMAX = 8
ROPE_BASE = 1.0e6


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); result stays float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) & np.uint32(0xFFFF0000)).view(np.float32)


@dataclass
class Problem:
    """One attention layer's inputs.  q [B,Hq,T,dh], k [B,Hkv,T,dh], v [B,Hkv,T,dv] float32
    (on the bf16 grid when dtype == 'bf16'); group_id [Hq,dh] int32 in 1..G[h];
    L [Hq,GMAX+1,GMAX+1] float32; G [Hq] int32."""
    name: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    group_id: np.ndarray
    L: np.ndarray
    G: np.ndarray
    eps: float
    dtype: str
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, Hq, T, dh = self.q.shape
        return dict(B=B, Hq=Hq, Hkv=self.k.shape[1], T=T, dh=dh, dv=self.v.shape[3])

    def slice_tokens(self, t0: int, t1: int) -> "Problem":
        return Problem(self.name + f"[{t0}:{t1}]", self.q[:, :, t0:t1].copy(),
                       self.k[:, :, t0:t1].copy(), self.v[:, :, t0:t1].copy(), self.group_id,
                       self.L, self.G, self.eps, self.dtype, dict(self.meta))

    def slice_batch(self, b0: int, b1: int) -> "Problem":
        return Problem(self.name + f"[b{b0}:{b1}]", self.q[b0:b1].copy(), self.k[b0:b1].copy(),
                       self.v[b0:b1].copy(), self.group_id, self.L, self.G, self.eps,
                       self.dtype, dict(self.meta))


def random_L(rng: np.random.Generator, G: int) -> np.ndarray:
    """(G+1)x(G+1) lower-triangular factor in a zero [GMAX+1, GMAX+1] slot."""
    L = np.zeros((GMAX + 1, GMAX + 1), np.float32)
    n = G + 1
    low = rng.normal(0.0, 0.3, size=(n, n)).astype(np.float32)
    L[:n, :n] = np.tril(low, -1)
    L[np.arange(n), np.arange(n)] = rng.uniform(0.5, 1.5, size=n).astype(np.float32)
    return L


def rope_rotate(x: np.ndarray, pos0: int, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate-half rotary embedding of x [..., T, d] at positions pos0..pos0+T-1 (data shaping
    of the inputs only)."""
    T, d = x.shape[-2], x.shape[-1]
    half = d // 2
    inv_freq = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = (pos0 + np.arange(T, dtype=np.float64))[:, None] * inv_freq[None, :]
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1).astype(np.float32)


def _tail_partition(rng: np.random.Generator, dims: np.ndarray, n_tail: int):
    perm = rng.permutation(dims)
    cuts = np.sort(rng.choice(np.arange(1, len(perm)), size=n_tail - 1, replace=False)) \
        if n_tail > 1 else np.array([], dtype=np.int64)
    return np.split(perm, cuts)


def config0() -> Problem:
    """Tiny dense-vs-recurrent check: B=1, one head, T=256, d_h=dv=64, fp32; 4 tail dims of
    q and k scaled by 8; G=4 (60 bulk dims, tail split 2/1/1); L 5x5; eps=1e-6; seed 0."""
    rng = np.random.default_rng(0)
    B, H, T, d = 1, 1, 256, 64
    q = rng.standard_normal((B, H, T, d)).astype(np.float32)
    k = rng.standard_normal((B, H, T, d)).astype(np.float32)
    v = rng.standard_normal((B, H, T, d)).astype(np.float32)
    tail = rng.choice(d, size=4, replace=False)
    q[..., tail] *= 8.0
    k[..., tail] *= 8.0
    gid = np.ones((H, d), np.int32)
    gid[0, tail[0:2]] = 2
    gid[0, tail[2]] = 3
    gid[0, tail[3]] = 4
    G = np.array([4], np.int32)
    L = random_L(rng, 4)[None]
    return Problem("config0", q, k, v, gid, L, G, 1e-6, "f32", dict(tail=tail.tolist()))


def qwen_layer(seed_key, B: int, T: int, Hq: int = 14, Hkv: int = 2, d: int = 64,
               dv: int = 64, pos0: int = 0, dtype: str = "bf16", eps: float = 1e-6,
               name: str = "qwen_layer", extra_tokens: int = 0) -> Problem:
    """One Qwen2.5-0.5B-shaped layer: GQA 14/2, d=64, outlier dims per key/value head,
    per-query-head tail groups and L, RoPE base 1e6.  ``extra_tokens`` appends that many
    further positions (for decode continuation) drawn from the same stream."""
    rng = np.random.default_rng(np.random.SeedSequence(list(np.atleast_1d(seed_key))))
    grp = Hq // Hkv
    Ttot = T + extra_tokens
    q = rng.standard_normal((B, Hq, Ttot, d), dtype=np.float32)
    k = rng.standard_normal((B, Hkv, Ttot, d), dtype=np.float32)
    v = rng.standard_normal((B, Hkv, Ttot, dv), dtype=np.float32)
    gid = np.ones((Hq, d), np.int32)
    G = np.ones(Hq, np.int32)
    L = np.zeros((Hq, GMAX + 1, GMAX + 1), np.float32)
    outliers = []
    for kv in range(Hkv):
        n_out = int(rng.integers(2, 7))
        dims = rng.choice(d, size=n_out, replace=False)
        scale = rng.integers(4, 13, size=n_out).astype(np.float32)
        outliers.append((dims.tolist(), scale.tolist()))
        kview = k[:, kv]
        kview[..., dims] *= scale
        for h in range(kv * grp, (kv + 1) * grp):
            qview = q[:, h]
            qview[..., dims] *= scale
            n_tail = int(rng.integers(1, min(5, n_out) + 1))
            for gi, part in enumerate(_tail_partition(rng, dims, n_tail)):
                gid[h, part] = 2 + gi
            G[h] = 1 + n_tail
            L[h] = random_L(rng, int(G[h]))
    for h in range(Hq):  # per head, to bound peak host memory on large batches
        q[:, h] = rope_rotate(q[:, h], pos0)
    for kv in range(Hkv):
        k[:, kv] = rope_rotate(k[:, kv], pos0)
    if dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return Problem(name, q, k, v, gid, L, G, eps, dtype,
                   dict(outliers=outliers, seed_key=list(np.atleast_1d(seed_key)), pos0=pos0))


def config1() -> Problem:
    """Qwen2.5-0.5B-shaped single-layer prefill: B=1, T=4096, 14/2 heads, bf16."""
    return qwen_layer([1], B=1, T=4096, name="config1")


def config2_layer(layer: int) -> Problem:
    """Batched prefill: B=8, T=4096; one of 18 independent layers (converted layers 3-20),
    each with its own groups and L."""
    return qwen_layer([2, layer], B=8, T=4096, name=f"config2_layer{layer}")


def config3(T: int) -> Problem:
    """Long-context prefill: B=1, T in {16384, 32768, 65536}."""
    return qwen_layer([3, T], B=1, T=T, name=f"config3_T{T}")


def config4(batch: int = 64, context: int = 4096, steps: int = 256) -> Problem:
    """Autoregressive decode: ``context`` tokens to prefill, then ``steps`` single-token
    steps (tokens context..context+steps-1 of the returned arrays)."""
    return qwen_layer([4], B=batch, T=context, extra_tokens=steps, name="config4")


def small_layer(seed: int, B: int, T: int, Hq: int, Hkv: int, dtype: str, d: int = 64,
                dv: int = 64) -> Problem:
    """A Qwen-like layer at small, test-friendly sizes (same recipe as the full configs)."""
    return qwen_layer([100, seed], B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, dv=dv, dtype=dtype,
                      name=f"small_s{seed}_B{B}_T{T}_H{Hq}x{Hkv}_{dtype}")
