"""Seeded synthetic inputs shared by the tests and the bench.

This module holds random-number generation and plain gathers only; it contains
none of the attention arithmetic and no zigzag rule (a caller that wants the
shard-major layout passes in the permutation it trusts).

Recipe (the pages name no dataset; these stand in for activations of the pages'
model shapes): Q, K, V and dO are drawn i.i.d. N(0, 1) in fp32 from one
torch.Generator seeded with `seed`, in the order Q, K, V, dO, each in natural
position order [B][S][H][d], then rounded to bf16 (round-to-nearest-even).
The long-context stress variant draws n = round(frac * S) positions with
randperm(S)[:n] from the same generator after dO and multiplies the Q and K rows
at those positions (all heads) by 8 in fp32 before rounding (exact).
"""
import torch


def make_inputs(B, S, Hq, Hkv, d, seed, stress_frac=0.0, device="cpu"):
    """Natural-order bf16 tensors q, do [B][S][Hq][d] and k, v [B][S][Hkv][d].

    Returns (q, k, v, do, stress_positions) where stress_positions is an int64
    tensor (empty unless stress_frac > 0).
    """
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    f32 = dict(generator=g, dtype=torch.float32, device=device)
    q = torch.randn(B, S, Hq, d, **f32)
    k = torch.randn(B, S, Hkv, d, **f32)
    v = torch.randn(B, S, Hkv, d, **f32)
    do = torch.randn(B, S, Hq, d, **f32)
    pos = torch.empty(0, dtype=torch.int64, device=device)
    if stress_frac > 0.0:
        n = int(round(stress_frac * S))
        pos = torch.randperm(S, generator=g, device=device)[:n]
        q[:, pos] *= 8.0
        k[:, pos] *= 8.0
    bf = torch.bfloat16
    return q.to(bf), k.to(bf), v.to(bf), do.to(bf), pos


def to_shard_major(x, perm, D):
    """Gather natural-order x [B][S][H][d] into shard-major [D][B][S/D][H][d].

    perm[r*(S/D) + j] is the position placed at row j of shard r.
    """
    B, S, H, d = x.shape
    perm = torch.as_tensor(perm, dtype=torch.int64, device=x.device)
    y = x.index_select(1, perm)                       # [B][S][H][d] in shard-major row order
    return y.reshape(B, D, S // D, H, d).transpose(0, 1).contiguous()


def from_shard_major(y, perm):
    """Inverse of to_shard_major: [D][B][2C][H][d] -> natural [B][S][H][d]."""
    D, B, twoC, H, d = y.shape
    S = D * twoC
    perm = torch.as_tensor(perm, dtype=torch.int64, device=y.device)
    flat = y.transpose(0, 1).reshape(B, S, H, d)     # shard-major row order
    out = torch.empty_like(flat)
    out[:, perm] = flat
    return out


def stats_from_shard_major(s, perm):
    """Per-row statistics [D][B][H][2C] -> natural [B][H][S]."""
    D, B, H, twoC = s.shape
    S = D * twoC
    perm = torch.as_tensor(perm, dtype=torch.int64, device=s.device)
    flat = s.permute(1, 2, 0, 3).reshape(B, H, S)
    out = torch.empty_like(flat)
    out[:, :, perm] = flat
    return out
