"""Independent NumPy textbook forms used to pin the oracle (tests only).

Written from the mathematics, not from the oracle: RoPE as a complex rotation
of the (i, i+d/2) pairs, attention as masked matrix products, span scores as
one matrix product of the summed group query with the middle keys.
"""
import numpy as np


def bits_to_f64(a):
    """float32 array, or bf16 given as uint16 bits, to float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rope(x, pos, base):
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    h = d // 2
    inv = base ** (-2.0 * np.arange(h) / d)
    ang = np.asarray(pos, np.float64)[:, None] * inv[None, :]
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], axis=-1)


def causal_attention(q, q_pos, k, v, base):
    """q [n, d] at positions q_pos; keys/values [m, d] at positions 0..m-1."""
    d = q.shape[-1]
    m = k.shape[0]
    qr = rope(q, q_pos, base)
    kr = rope(k, np.arange(m), base)
    lg = qr @ kr.T / np.sqrt(d)
    lg[np.arange(m)[None, :] > np.asarray(q_pos)[:, None]] = -np.inf
    w = np.exp(lg - lg.max(axis=1, keepdims=True))
    w /= w.sum(axis=1, keepdims=True)
    return w @ v


def span_scores(q, kc, G, L, S):
    """q [B,Hq,C,d], kc [B,Hkv,T,d] (float64) -> [B,Hkv,NS] via (sum_j Q_j) @ K_mid^T."""
    B, Hq, C, d = q.shape
    _, Hkv, T, _ = kc.shape
    g = Hq // Hkv
    M = max(0, T - G - L)
    NS = -(-M // S)
    out = np.zeros((B, Hkv, NS))
    for b in range(B):
        for h in range(Hkv):
            qs = q[b, h * g:(h + 1) * g].sum(axis=0)          # [C, d]
            tok = (qs @ kc[b, h, G:G + M].T).max(axis=0)      # [M]
            pad = np.full(NS * S, -np.inf)
            pad[:M] = tok
            out[b, h] = pad.reshape(NS, S).max(axis=1)
    return out


def window_attention(q, kc, vc, kcur, vcur, rows, base):
    """Attention of every query over an explicit window: rows = list of cache
    rows (per b, h) followed by the C current tokens.  Returns [B,Hq,C,d]."""
    B, Hq, C, d = q.shape
    Hkv = kc.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, C, d))
    for b in range(B):
        for h in range(Hkv):
            r = rows[b][h]
            K = np.concatenate([kc[b, h, r], kcur[b, h]], axis=0)
            V = np.concatenate([vc[b, h, r], vcur[b, h]], axis=0)
            W = K.shape[0]
            for j in range(h * g, (h + 1) * g):
                out[b, j] = causal_attention(q[b, j], W - C + np.arange(C), K, V, base)
    return out
