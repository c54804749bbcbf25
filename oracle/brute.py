"""numpy fp64 full-matrix brute force, for pinning the C oracle on tiny inputs.

TEST INFRASTRUCTURE ONLY.  Plain, unsharded causal attention in natural order:
the S x S score matrix, a -inf mask above the diagonal (key k visible to query p
iff k <= p), a two-pass softmax, O = P V.  No zigzag, no blocking, no online
softmax: the point is that sharded-then-unpermuted oracle results must equal this.
The backward is the textbook gradient of <dO, O> in matrix form.
"""
import numpy as np


def causal_attention(q, k, v, causal=True, scale=None):
    """q [B][S][Hq][d], k/v [B][S][Hkv][d] (natural order) -> (o, lse [B][Hq][S])."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, S))
    mask = np.triu(np.ones((S, S), bool), 1) if causal else np.zeros((S, S), bool)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = scale * q[b, :, h, :] @ k[b, :, kv, :].T
            s = np.where(mask, -np.inf, s)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            p = e / l
            o[b, :, h, :] = p @ v[b, :, kv, :]
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return o, lse


def causal_attention_bwd(q, k, v, do, causal=True, scale=None):
    """Gradients of L = <do, O> w.r.t. q, k, v (natural order)."""
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    mask = np.triu(np.ones((S, S), bool), 1) if causal else np.zeros((S, S), bool)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = scale * q[b, :, h, :] @ k[b, :, kv, :].T
            s = np.where(mask, -np.inf, s)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o = p @ v[b, :, kv, :]
            dp = do[b, :, h, :] @ v[b, :, kv, :].T
            ds = p * (dp - (do[b, :, h, :] * o).sum(axis=1, keepdims=True))
            dq[b, :, h, :] = scale * ds @ k[b, :, kv, :]
            dk[b, :, kv, :] += scale * ds.T @ q[b, :, h, :]
            dv[b, :, kv, :] += p.T @ do[b, :, h, :]
    return dq, dk, dv


def key_range_attention(q, k, v, key_lo, key_hi, causal=True, scale=None):
    """Attention restricted to the keys at positions [key_lo, key_hi) (natural order),
    full-matrix: keys outside the range (or above the diagonal when causal) are masked to
    -inf; a row with every key masked gets lse = -inf and O = 0.
    Returns (o [B][S][Hq][d], lse [B][Hq][S])."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    B, S, Hq, d = q.shape
    G = Hq // k.shape[2]
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    pos = np.arange(S)
    visible = (pos[None, :] >= key_lo) & (pos[None, :] < key_hi)
    if causal:
        visible = visible & (pos[None, :] <= pos[:, None])
    else:
        visible = np.broadcast_to(visible, (S, S))
    o = np.zeros_like(q)
    lse = np.full((B, Hq, S), -np.inf)
    rows = visible.any(axis=1)
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, :, h, :] @ k[b, :, h // G, :].T
            s = np.where(visible, s, -np.inf)[rows]
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, rows, h, :] = (e / l) @ v[b, :, h // G, :]
            lse[b, h, rows] = (m + np.log(l))[:, 0]
    return o, lse
