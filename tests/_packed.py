"""Test-side reader of the state buffer layout documented in include/oal.h.

Written from the header's description (not from the library's code) so that tests can
compare the library's packed state with the oracle's unpacked H0/H1/H2."""
import numpy as np

F, FP = 2145, 2176
HEADER = 256


def packed_pairs():
    """(r, t) of every packed row f < 2145, following the order stated in include/oal.h."""
    pairs = []
    for R in range(8):
        for T in range(R + 1, 8):
            for a in range(8):
                for b in range(8):
                    pairs.append((8 * R + a, 8 * T + b))
    for R in range(8):
        for a in range(8):
            for b in range(a, 8):
                pairs.append((8 * R + a, 8 * R + b))
    for r in range(64):
        pairs.append((r, 64))
    pairs.append((64, 64))
    assert len(pairs) == F
    return np.array(pairs, dtype=np.int64)


def coef_offset():
    return HEADER


def body_offset(Hq):
    return HEADER + ((Hq * FP * 4 + 255) // 256) * 256


def read_state(buf: np.ndarray, B, Hq, Hkv, dv=64):
    """buf: uint8 numpy copy of the state.  Returns (header dict, coef [Hq,FP],
    S [B,Hkv,FP,dv+1] with S[..., :dv] = Hv and S[..., dv] = z)."""
    hdr = buf[:HEADER]
    i32 = hdr[:32].view(np.int32)
    header = dict(magic=int(hdr[:4].view(np.uint32)[0]), abi=int(i32[1]), B=int(i32[2]),
                  Hq=int(i32[3]), Hkv=int(i32[4]), dh=int(i32[5]), dv=int(i32[6]),
                  feat_pad=int(i32[7]), tokens=int(hdr[32:40].view(np.int64)[0]),
                  eps=float(hdr[40:44].view(np.float32)[0]))
    coef = buf[HEADER:HEADER + Hq * FP * 4].view(np.float32).reshape(Hq, FP)
    unit = FP * (dv + 1)
    body = buf[body_offset(Hq):body_offset(Hq) + B * Hkv * unit * 4].view(np.float32)
    body = body.reshape(B, Hkv, unit)
    Hv = body[:, :, :FP * dv].reshape(B, Hkv, FP, dv)
    z = body[:, :, FP * dv:].reshape(B, Hkv, FP, 1)
    return header, coef, np.concatenate([Hv, z], axis=-1)


def pack_oracle_state(st, pairs=None):
    """Oracle State (H0 [B,Hkv,w], H1 [B,Hkv,d,w], H2 [B,Hkv,d,d,w]) -> packed [B,Hkv,F,w]."""
    pairs = packed_pairs() if pairs is None else pairs
    B, Hkv, w = st.H0.shape
    out = np.zeros((B, Hkv, F, w))
    for f, (r, t) in enumerate(pairs):
        if r < 64 and t < 64:
            out[:, :, f] = st.H2[:, :, r, t]
        elif r < 64:
            out[:, :, f] = st.H1[:, :, r]
        else:
            out[:, :, f] = st.H0
    return out


def coef_from_header(group_id, L, G, eps):
    """Readout weights [Hq, FP] of the packed rows as include/oal.h states them:
    (r == t ? 1 : 2) * M_{g(r),g(t)} * s_r * s_t with M = L L^T, g(64) = 0, s_r = 1/8 for
    r < 64 and s_64 = 1, plus eps on the constant row 2144; zero on the padding rows."""
    pairs = packed_pairs()
    Hq = G.shape[0]
    out = np.zeros((Hq, FP))
    for h in range(Hq):
        Gh = int(G[h])
        Lh = L[h, :Gh + 1, :Gh + 1].astype(np.float64)
        M = Lh @ Lh.T
        g = np.concatenate([group_id[h], [0]])
        s = np.concatenate([np.full(64, 0.125), [1.0]])
        r, t = pairs[:, 0], pairs[:, 1]
        out[h, :F] = np.where(r == t, 1.0, 2.0) * M[g[r], g[t]] * s[r] * s[t]
        out[h, 2144] += eps
    return out
