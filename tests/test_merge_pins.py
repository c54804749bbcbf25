"""Pins for the oracle's key-range forward (attn_fwd_keys) and partial-result merge
(attn_merge), the ring-attention pieces ("AutoSP" summary, sections 1 and 4).

Pinned against things other than themselves:
  * attn_fwd_keys against the numpy full-matrix brute force with a key-range mask, for
    several ranges, causal and not, GQA, through the zigzag layout;
  * a one-key range: lse = scale * q . k_k and O = v_k exactly (closed form), and rows
    that see no key get lse = -inf, O = 0;
  * the whole range equals the pinned full forward;
  * merging the results of any split of the key range -- two or three pieces, empty
    pieces included, in any order -- equals the full forward (the identity a softmax
    over a union of disjoint key sets satisfies);
  * a single part merges to itself.
"""
import numpy as np
import pytest
import torch

from oracle import brute
from sequence_sharded_causal_b200 import inputs


def _setup(oracle, B=1, S=64, Hq=4, Hkv=2, d=8, D=2, seed=5):
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    return q_nat, k, v, perm, inputs.to_shard_major(q_nat, perm, D)


@pytest.mark.parametrize("lo,hi,causal", [(0, 64, True), (10, 40, True), (33, 64, True),
                                          (0, 1, True), (20, 21, False), (5, 60, False)])
def test_fwd_keys_matches_brute_force(oracle, lo, hi, causal):
    D = 2
    q_nat, k, v, perm, q = _setup(oracle, D=D)
    o, lse = oracle.attn_fwd_keys(q, k, v, D, lo, hi, causal)
    o_ref, lse_ref = brute.key_range_attention(q_nat.double().numpy(), k.double().numpy(),
                                               v.double().numpy(), lo, hi, causal)
    o_nat = inputs.from_shard_major(torch.from_numpy(o), perm).numpy()
    lse_nat = inputs.stats_from_shard_major(torch.from_numpy(lse), perm).numpy()
    assert np.array_equal(np.isinf(lse_nat), np.isinf(lse_ref))
    fin = np.isfinite(lse_ref)
    assert np.abs(lse_nat[fin] - lse_ref[fin]).max() <= 1e-12
    assert np.abs(o_nat - o_ref).max() <= 1e-12


def test_one_key_closed_form(oracle):
    D, S, kk = 2, 64, 37
    q_nat, k, v, perm, q = _setup(oracle, D=D, S=S)
    o, lse = oracle.attn_fwd_keys(q, k, v, D, kk, kk + 1)
    o_nat = inputs.from_shard_major(torch.from_numpy(o), perm).numpy()
    lse_nat = inputs.stats_from_shard_major(torch.from_numpy(lse), perm).numpy()
    qd, kd, vd = (x.double().numpy() for x in (q_nat, k, v))
    scale = float(np.float32(1.0 / np.sqrt(qd.shape[-1])))
    G = qd.shape[2] // kd.shape[2]
    for p in range(S):
        for h in range(qd.shape[2]):
            if p < kk:       # the key lies above the diagonal: nothing visible
                assert lse_nat[0, h, p] == -np.inf and not o_nat[0, p, h].any()
            else:
                assert abs(lse_nat[0, h, p] - scale * qd[0, p, h] @ kd[0, kk, h // G]) <= 1e-12
                assert np.abs(o_nat[0, p, h] - vd[0, kk, h // G]).max() <= 1e-15


@pytest.mark.parametrize("cuts", [(23,), (0,), (64,), (1, 63), (16, 40), (8, 9, 50)])
@pytest.mark.parametrize("causal", [True, False])
def test_merge_of_any_split_equals_full_forward(oracle, cuts, causal):
    D, S = 4, 64
    q_nat, k, v, perm, q = _setup(oracle, D=D, S=S, Hq=6, Hkv=2, seed=9)
    o_full, lse_full = oracle.attn_fwd(q, k, v, D, causal)
    bounds = [0, *cuts, S]
    parts = [oracle.attn_fwd_keys(q, k, v, D, a, b, causal) for a, b in zip(bounds, bounds[1:])]
    for order in (parts, parts[::-1]):
        o, lse = oracle.attn_merge([x[0] for x in order], [x[1] for x in order])
        assert np.abs(lse - lse_full).max() <= 1e-12
        assert np.abs(o - o_full).max() <= 1e-12


def test_single_part_merges_to_itself(oracle):
    D = 2
    _, k, v, _, q = _setup(oracle, D=D)
    o1, l1 = oracle.attn_fwd_keys(q, k, v, D, 7, 50)
    o, lse = oracle.attn_merge([o1], [l1])
    assert np.array_equal(np.isinf(lse), np.isinf(l1))
    assert np.abs(o - o1).max() <= 1e-15
    fin = np.isfinite(l1)
    assert np.abs(lse[fin] - l1[fin]).max() <= 1e-15
