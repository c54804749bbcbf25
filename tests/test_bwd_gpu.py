"""Backward parity on the GPU: dQ, dK, dV from libzsa vs the fp64 CPU oracle.

The GPU backward consumes the GPU forward's bf16 O and fp32 lse (as a training step
does); the oracle recomputes everything in fp64 from the same bf16 inputs.  Tolerance
(stated for this path): relative Frobenius error <= 1e-2 per tensor.  dK and dV are
sums over every shard and every q head of the kv group.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import inputs

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2

CASES = [  # (B, S, Hq, Hkv, d, D, causal, seed)
    (1, 256, 2, 2, 64, 2, True, 0),        # the tiny configuration
    (1, 1024, 4, 2, 128, 2, True, 1),
    (1, 768, 2, 2, 128, 2, True, 2),       # C = 192: 64-row tiles cover each chunk exactly
    (2, 768, 6, 2, 64, 2, False, 3),       # non-causal, GQA 3, B = 2
    (1, 2048, 8, 8, 128, 4, True, 5),
    (1, 1536, 4, 1, 128, 3, True, 6),      # GQA 4, D = 3
    (1, 1024, 4, 4, 128, 1, True, 7),      # D = 1
    (1, 2048, 4, 2, 64, 8, True, 8),       # D = 8
    (1, 1024, 6, 1, 256, 2, True, 9),      # d = 256 (two-CTA cluster per key tile), GQA 6
    (1, 512, 4, 2, 256, 2, True, 10),      # d = 256, 64-row q slots, C = 128
    (2, 512, 2, 2, 256, 1, False, 11),     # d = 256, non-causal, D = 1, B = 2
    # more units than CTAs, so every CTA carries state from one key tile to the next
    (1, 4096, 16, 8, 64, 4, True, 12),     # 256 units (d = 64)
    (1, 4096, 6, 1, 256, 4, True, 13),     # 32 key tiles over the clusters, long slot walks
]


def rel_fro(x, ref):
    return float(np.linalg.norm((x - ref).ravel()) / np.linalg.norm(ref.ravel()))


def gpu_fwd_bwd(q, k, v, do, D, causal):
    B, S, Hkv, d = k.shape
    problem = zsa.make_problem(B, S, q.shape[3], Hkv, d, D, causal)
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = zsa.attn_fwd(q, k, v, D, causal)
    ws = torch.empty(zsa.zsa_workspace_bytes(problem, 1), dtype=torch.uint8, device="cuda")
    dq, dk, dv = zsa.attn_bwd(q, k, v, o, lse, do, D, causal, workspace=ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    return [x.float().cpu().numpy() for x in (dq, dk, dv)]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,causal,seed", CASES)
def test_bwd_matches_oracle(oracle, B, S, Hq, Hkv, d, D, causal, seed):
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    ref = oracle.attn_bwd(q, k, v, do, D, causal)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, D, causal)
    errs = {n: rel_fro(x, ref[n]) for n, x in (("dq", dq), ("dk", dk), ("dv", dv))}
    assert all(np.isfinite(x).all() for x in (dq, dk, dv))
    assert max(errs.values()) <= REL_TOL, errs


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,seed,frac", [
    (1, 2048, 4, 2, 128, 4, 41, 0.01), (1, 1024, 2, 2, 64, 2, 42, 0.02),
    (1, 1024, 6, 1, 256, 2, 43, 0.02),
    (1, 2048, 12, 2, 256, 4, 44, 0.01),    # the wide-head shape's G = 6 and D = 4
    (1, 4096, 8, 2, 128, 16, 45, 0.01)])   # the long-context G = 4 and D = 16
def test_bwd_stress_rows(oracle, B, S, Hq, Hkv, d, D, seed, frac):
    q_nat, k, v, do_nat, pos = inputs.make_inputs(B, S, Hq, Hkv, d, seed, stress_frac=frac)
    assert pos.numel() > 0
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    ref = oracle.attn_bwd(q, k, v, do, D)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, D, True)
    errs = {n: rel_fro(x, ref[n]) for n, x in (("dq", dq), ("dk", dk), ("dv", dv))}
    assert all(np.isfinite(x).all() for x in (dq, dk, dv))
    assert max(errs.values()) <= REL_TOL, errs


def test_bwd_wait_timeout_reports_status(oracle):
    B, S, Hq, Hkv, d, D = 1, 1024, 4, 2, 128, 2
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 21)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D).cuda()
    do = inputs.to_shard_major(do_nat, perm, D).cuda()
    k, v = k.cuda(), v.cuda()
    o, lse = zsa.attn_fwd(q, k, v, D)
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    ws = torch.empty(zsa.zsa_workspace_bytes(problem, 1), dtype=torch.uint8, device="cuda")
    try:
        zsa.zsa_set_wait_limit_ns(20_000_000)
        zsa.zsa_debug_inject_stall(True)
        zsa.attn_bwd(q, k, v, o, lse, do, D, workspace=ws)
        assert zsa.zsa_device_status(ws) == zsa.ZSA_ERR_TIMEOUT
    finally:
        zsa.zsa_debug_inject_stall(False)
        zsa.zsa_set_wait_limit_ns(2_000_000_000)
    dq, dk, dv = zsa.attn_bwd(q, k, v, o, lse, do, D, workspace=ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    ref = oracle.attn_bwd(q.cpu(), k.cpu(), v.cpu(), do.cpu(), D)
    assert rel_fro(dk.float().cpu().numpy(), ref["dk"]) <= REL_TOL
