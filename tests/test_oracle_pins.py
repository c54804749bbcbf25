"""Pins for the fp64 CPU oracle, against things other than the oracle itself.

- zigzag map: a hand-worked golden example, D=1 identity, bijection, the
  causal-balance property the zigzag exists for (equal causal pairs per shard,
  closed form C^2(2D-1) + C(C+1)) and the imbalance of a contiguous split;
- schedule: per-shard tile work equal and equal to its closed form, kend equal to
  brute-force tile visibility counting, every slot covered exactly once;
- forward: equality with an independent numpy full-matrix causal attention on the
  un-permuted result for every valid D, closed forms (row 0, equal keys, equal
  values, zero queries, one-hot values exposing P itself);
- backward: central finite differences in fp64, the numpy matrix-form gradient,
  dO = 0.
"""
import os

import numpy as np
import pytest
import torch

from oracle import brute
from sequence_sharded_causal_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng):
    return rng.standard_normal(shape)


def _shard(x_nat, perm, D):
    return inputs.to_shard_major(torch.from_numpy(x_nat), perm, D).numpy()


def _unshard(y, perm):
    return inputs.from_shard_major(torch.from_numpy(y), perm).numpy()


def _unshard_stats(s, perm):
    return inputs.stats_from_shard_major(torch.from_numpy(s), perm).numpy()


# ---------------------------------------------------------------- partition

def test_partition_golden(oracle):
    lines = [l for l in open(os.path.join(GOLDEN, "zigzag_S16_D2.txt"))
             if l.strip() and not l.startswith("#")]
    want = np.array([int(x) for x in (lines[0] + " " + lines[1]).split()])
    perm, inv = oracle.partition(16, 2)
    assert np.array_equal(perm, want)
    pairs = [int(x) for x in lines[2].split()]
    got = [int((perm[r * 8:(r + 1) * 8] + 1).sum()) for r in range(2)]
    assert got == pairs


@pytest.mark.parametrize("S", [2, 8, 64, 256, 1024])
def test_partition_D1_identity(oracle, S):
    perm, inv = oracle.partition(S, 1)
    assert np.array_equal(perm, np.arange(S))
    assert np.array_equal(inv, np.arange(S))


def test_partition_bijection_and_balance(oracle):
    for S in range(2, 1025, 2):
        for D in range(1, S // 2 + 1):
            if S % (2 * D):
                continue
            if S > 256 and D not in (1, 2, 4, 8, 16):
                continue
            perm, inv = oracle.partition(S, D)
            assert np.array_equal(np.sort(perm), np.arange(S))
            assert np.array_equal(inv[perm], np.arange(S))
            C = S // (2 * D)
            twoC = 2 * C
            pairs = [(perm[r * twoC:(r + 1) * twoC].astype(np.int64) + 1).sum()
                     for r in range(D)]
            assert len(set(pairs)) == 1, (S, D, pairs)
            assert pairs[0] == C * C * (2 * D - 1) + C * (C + 1)
            assert sum(pairs) == S * (S + 1) // 2


def test_contiguous_split_is_imbalanced():
    # the imbalance the zigzag removes: a contiguous split gives the last shard
    # about 2D-1 times the first shard's causal pairs
    S, D = 4096, 8
    L = S // D
    pairs = [sum(p + 1 for p in range(r * L, (r + 1) * L)) for r in range(D)]
    assert pairs[-1] / pairs[0] > 2 * D - 2


def test_partition_rejects_bad_shapes(oracle):
    with pytest.raises(ValueError):
        oracle.partition(10, 3)


# ---------------------------------------------------------------- schedule

def _brute_kend(perm, S, D, r, i, bq, bk, causal):
    twoC = S // D
    if not causal:
        return S // bk
    rows = perm[r * twoC + i * bq: r * twoC + (i + 1) * bq]
    n = 0
    for kt in range(S // bk):
        keys = np.arange(kt * bk, (kt + 1) * bk)
        if (keys[None, :] <= rows[:, None]).any():
            n = kt + 1
    return n


@pytest.mark.parametrize("S,D,B,Hq,Hkv,bq,bk", [
    (256, 2, 1, 2, 2, 64, 64), (256, 2, 1, 2, 2, 128, 128), (1024, 4, 2, 4, 2, 128, 64),
    (768, 2, 1, 3, 1, 128, 128), (1536, 4, 1, 6, 2, 64, 128), (640, 5, 1, 2, 1, 128, 64)])
def test_schedule_brute(oracle, S, D, B, Hq, Hkv, bq, bk):
    perm, _ = oracle.partition(S, D)
    G = Hq // Hkv
    T = (S // D) // bq
    for causal in (True, False):
        for slots in (1, 2):
            st, units = oracle.schedule(S, D, B, Hq, Hkv, causal, bq, bk, slots)
            kend = {(r, i): _brute_kend(perm, S, D, r, i, bq, bk, causal)
                    for r in range(D) for i in range(T)}
            for r in range(D):
                assert st[r] == B * Hq * sum(kend[(r, i)] for i in range(T))
            seen = set()
            for u in units:
                r, b, g, i0, h0, i1, h1, k0, k1 = (int(x) for x in u)
                assert h0 // G == g and k0 == kend[(r, i0)]
                seen.add((r, b, i0, h0))
                if slots == 1:
                    assert (i1, h1, k1) == (-1, -1, 0)
                elif i1 >= 0:
                    assert h1 // G == g and k1 == kend[(r, i1)]
                    seen.add((r, b, i1, h1))
            assert len(seen) == D * B * T * Hq
            work = np.maximum(units[:, 7], units[:, 8])
            grp = units[:, 1] * Hkv + units[:, 2]
            assert (np.diff(grp) >= 0).all()                      # (b, g)-major
            same = np.diff(grp) == 0
            assert (np.diff(work)[same] <= 0).all()               # longest first within a group


@pytest.mark.parametrize("S,D,Hq,Hkv,bq,bk,per_head", [
    (256, 2, 2, 2, 64, 64, 5), (16384, 8, 32, 32, 128, 128, 1032),
    (32768, 8, 32, 8, 128, 128, 4112), (65536, 4, 24, 4, 128, 128, 32832),
    (131072, 16, 32, 8, 128, 128, 32800), (65536, 4, 24, 4, 128, 64, 65664)])
def test_schedule_closed_form_balance(oracle, S, D, Hq, Hkv, bq, bk, per_head):
    st, _ = oracle.schedule(S, D, 1, Hq, Hkv, True, bq, bk, 2)
    C = S // (2 * D)
    T = C // bq
    closed = (bq // bk) * (T * T * (2 * D - 1) + T * (T + 1))
    assert closed == per_head
    assert (st == Hq * closed).all()


# ---------------------------------------------------------------- forward

def _valid_D(S):
    return [D for D in range(1, S // 2 + 1) if S % (2 * D) == 0]


@pytest.mark.parametrize("S,Hq,Hkv,d", [(32, 2, 2, 8), (48, 3, 1, 4), (64, 4, 2, 16)])
def test_fwd_sharded_equals_unsharded_every_D(oracle, S, Hq, Hkv, d):
    rng = np.random.default_rng(S + Hq + d)
    B = 2
    q, k, v = _rand((B, S, Hq, d), rng), _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    for causal in (True, False):
        o_ref, lse_ref = brute.causal_attention(q, k, v, causal)
        for D in _valid_D(S):
            perm, _ = oracle.partition(S, D)
            o, lse = oracle.attn_fwd(_shard(q, perm, D), k, v, D, causal)
            assert np.abs(_unshard(o, perm) - o_ref).max() < 1e-12
            assert np.abs(_unshard_stats(lse, perm) - lse_ref).max() < 1e-12


def test_fwd_brute_tiny_config_shape(oracle):
    # the tiny configuration's shape: B=1, S=256, 2 heads, d=64, D=2
    S, H, d, D = 256, 2, 64, 2
    rng = np.random.default_rng(0)
    q, k, v = _rand((1, S, H, d), rng), _rand((1, S, H, d), rng), _rand((1, S, H, d), rng)
    perm, _ = oracle.partition(S, D)
    o, lse = oracle.attn_fwd(_shard(q, perm, D), k, v, D)
    o_ref, lse_ref = brute.causal_attention(q, k, v)
    assert np.abs(_unshard(o, perm) - o_ref).max() < 1e-12
    assert np.abs(_unshard_stats(lse, perm) - lse_ref).max() < 1e-12


def test_fwd_closed_forms(oracle):
    rng = np.random.default_rng(7)
    B, S, Hq, Hkv, d, D = 1, 32, 4, 2, 8, 4
    scale = float(np.float32(1 / np.sqrt(d)))
    perm, _ = oracle.partition(S, D)
    pos = np.arange(S)
    q = _rand((B, S, Hq, d), rng)
    k = _rand((B, S, Hkv, d), rng)
    v = _rand((B, S, Hkv, d), rng)
    # (i) position 0 sees only key 0: O = v0, lse = scale q0.k0
    o, lse = oracle.attn_fwd(_shard(q, perm, D), k, v, D)
    o, lse = _unshard(o, perm), _unshard_stats(lse, perm)
    for h in range(Hq):
        kv = h // (Hq // Hkv)
        assert np.allclose(o[0, 0, h], v[0, 0, kv], atol=1e-14)
        assert abs(lse[0, h, 0] - scale * q[0, 0, h] @ k[0, 0, kv]) < 1e-13
    # (ii) all keys equal: P uniform over the p+1 visible keys
    ke = np.repeat(k[:, :1], S, axis=1)
    o, lse = oracle.attn_fwd(_shard(q, perm, D), ke, v, D)
    o, lse = _unshard(o, perm), _unshard_stats(lse, perm)
    for h in range(Hq):
        kv = h // (Hq // Hkv)
        prefix_mean = np.cumsum(v[0, :, kv], axis=0) / (pos + 1)[:, None]
        assert np.abs(o[0, :, h] - prefix_mean).max() < 1e-13
        want = scale * q[0, :, h] @ k[0, 0, kv] + np.log(pos + 1)
        assert np.abs(lse[0, h] - want).max() < 1e-12
    # (iii) all values equal c: O = c
    c = rng.standard_normal(d)
    vc = np.broadcast_to(c, v.shape).copy()
    o, _ = oracle.attn_fwd(_shard(q, perm, D), k, vc, D)
    assert np.abs(o - c).max() < 1e-13
    # (iv) zero queries: prefix means, lse = ln(p+1)
    o, lse = oracle.attn_fwd(_shard(np.zeros_like(q), perm, D), k, v, D)
    o, lse = _unshard(o, perm), _unshard_stats(lse, perm)
    for h in range(Hq):
        kv = h // (Hq // Hkv)
        assert np.abs(o[0, :, h] - np.cumsum(v[0, :, kv], 0) / (pos + 1)[:, None]).max() < 1e-13
        assert np.abs(lse[0, h] - np.log(pos + 1)).max() < 1e-13


def test_fwd_one_hot_values_expose_P(oracle):
    # with v_k = e_k (d = S), O row p is the probability row itself: it must sum to 1,
    # vanish above the diagonal and equal softmax(scale q.K) over the visible keys
    rng = np.random.default_rng(3)
    B, S, H, D = 1, 16, 1, 2
    d = S
    q = _rand((B, S, H, d), rng)
    k = _rand((B, S, H, d), rng)
    v = np.eye(S)[None, :, None, :].copy()
    perm, _ = oracle.partition(S, D)
    o, _ = oracle.attn_fwd(_shard(q, perm, D), k, v, D)
    P = _unshard(o, perm)[0, :, 0, :]
    assert np.abs(P.sum(1) - 1).max() < 1e-14
    assert np.abs(np.triu(P, 1)).max() == 0.0
    scale = float(np.float32(1 / np.sqrt(d)))
    for p in range(S):
        s = scale * k[0, :p + 1, 0] @ q[0, p, 0]
        e = np.exp(s - s.max())
        assert np.abs(P[p, :p + 1] - e / e.sum()).max() < 1e-14


def test_fwd_rows_matches_full(oracle):
    rng = np.random.default_rng(11)
    B, S, Hq, Hkv, d, D = 2, 64, 4, 1, 8, 4
    q = _rand((D, B, S // D, Hq, d), rng)
    k, v = _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    o, lse = oracle.attn_fwd(q, k, v, D)
    rows = np.array([0, 5, 17, 31, 63, 100, 127])
    qf = q.reshape(-1, Hq, d)
    o_r, lse_r = oracle.attn_fwd_rows(qf[rows], rows, k, v, D, Hq)
    assert np.array_equal(o_r, o.reshape(-1, Hq, d)[rows])
    twoC = S // D
    lse_rows = np.stack([lse[r // (B * twoC), (r // twoC) % B, :, r % twoC] for r in rows])
    assert np.array_equal(lse_r, lse_rows)


# ---------------------------------------------------------------- backward

def _loss(oracle, q, k, v, do, D, causal):
    o, _ = oracle.attn_fwd(q, k, v, D, causal)
    return float((o * do).sum())


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_finite_differences(oracle, causal):
    rng = np.random.default_rng(5)
    B, S, Hq, Hkv, d, D = 1, 16, 2, 1, 4, 2
    twoC = S // D
    q = _rand((D, B, twoC, Hq, d), rng)
    k, v = _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    do = _rand((D, B, twoC, Hq, d), rng)
    g = oracle.attn_bwd(q, k, v, do, D, causal)
    h = 1e-6
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"dq": (xp, k, v), "dk": (q, xp, v), "dv": (q, k, xp)}[name]
            argm = {"dq": (xm, k, v), "dk": (q, xm, v), "dv": (q, k, xm)}[name]
            fd[idx] = (_loss(oracle, *args, do, D, causal) - _loss(oracle, *argm, do, D, causal)) / (2 * h)
        rel = np.linalg.norm(g[name] - fd) / np.linalg.norm(fd)
        assert rel < 1e-6, (name, rel)


@pytest.mark.parametrize("S,Hq,Hkv,d", [(64, 2, 2, 8), (96, 6, 2, 4)])
def test_bwd_matches_matrix_form_every_D(oracle, S, Hq, Hkv, d):
    rng = np.random.default_rng(S * d)
    B = 1
    q, k, v = _rand((B, S, Hq, d), rng), _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    do = _rand((B, S, Hq, d), rng)
    dq_ref, dk_ref, dv_ref = brute.causal_attention_bwd(q, k, v, do)
    o_ref, _ = brute.causal_attention(q, k, v)
    for D in _valid_D(S)[:6]:
        perm, _ = oracle.partition(S, D)
        g = oracle.attn_bwd(_shard(q, perm, D), k, v, _shard(do, perm, D), D)
        assert np.abs(_unshard(g["dq"], perm) - dq_ref).max() < 1e-11
        assert np.abs(g["dk"] - dk_ref).max() < 1e-11
        assert np.abs(g["dv"] - dv_ref).max() < 1e-11
        assert np.abs(_unshard(g["o"], perm) - o_ref).max() < 1e-12
        delta = (o_ref * do).sum(-1).transpose(0, 2, 1)
        assert np.abs(_unshard_stats(g["delta"], perm) - delta).max() < 1e-11


def test_dq_rows_match_full_backward(oracle):
    rng = np.random.default_rng(13)
    B, S, Hq, Hkv, d, D = 2, 64, 4, 2, 8, 4
    q = _rand((D, B, S // D, Hq, d), rng)
    do = _rand((D, B, S // D, Hq, d), rng)
    k, v = _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    for causal in (True, False):
        g = oracle.attn_bwd(q, k, v, do, D, causal)
        rows = np.array([0, 3, 15, 16, 31, 40, 63, 64, 101, 127])
        qf, dof = q.reshape(-1, Hq, d), do.reshape(-1, Hq, d)
        dq = oracle.attn_dq_rows(qf[rows], dof[rows], rows, k, v, D, Hq, causal)
        assert np.abs(dq - g["dq"].reshape(-1, Hq, d)[rows]).max() < 1e-13


def test_gradient_identities(oracle):
    # rows of P sum to 1 and rows of dS sum to 0, so per kv head
    # sum_k dV_k = sum over the group's q rows of dO, and sum_k dK_k = 0
    rng = np.random.default_rng(17)
    B, S, Hq, Hkv, d, D = 1, 64, 4, 2, 8, 2
    q = _rand((D, B, S // D, Hq, d), rng)
    do = _rand((D, B, S // D, Hq, d), rng)
    k, v = _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    g = oracle.attn_bwd(q, k, v, do, D)
    G = Hq // Hkv
    for kv in range(Hkv):
        want = do[:, :, :, kv * G:(kv + 1) * G, :].sum(axis=(0, 2, 3))[0]
        assert np.abs(g["dv"][0, :, kv].sum(0) - want).max() < 1e-12
        assert np.abs(g["dk"][0, :, kv].sum(0)).max() < 1e-12


def test_bwd_zero_upstream_gradient(oracle):
    rng = np.random.default_rng(9)
    B, S, Hq, Hkv, d, D = 1, 32, 2, 2, 8, 2
    q = _rand((D, B, S // D, Hq, d), rng)
    k, v = _rand((B, S, Hkv, d), rng), _rand((B, S, Hkv, d), rng)
    g = oracle.attn_bwd(q, k, v, np.zeros_like(q), D)
    assert np.abs(g["dq"]).max() == 0 and np.abs(g["dk"]).max() == 0
    assert np.abs(g["dv"]).max() == 0
