"""Forward parity on the GPU: libzsa's sm_100a kernel vs the fp64 CPU oracle.

Inputs are seeded N(0,1) bf16 (sequence_sharded_causal_b200.inputs); Q is laid out
shard-major with the ORACLE's zigzag map, so a wrong map or mask inside the kernel
shows up as a mismatch.  Tolerances (stated for this path): O max-abs <= 1e-2 beyond
the half-ulp rounding of its bf16 output format, lse max-abs <= 1e-3.  Cases span several 128-row tiles, tiles that straddle the two
chunks of a shard, odd tile counts (single-slot units), every supported head dim,
GQA groups of 1, 2, 3, 4, 6, non-causal, B = 2.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import inputs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def bf16_half_ulp(x):
    """Half the bf16 spacing at |x|: the rounding any bf16 output of x may carry."""
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def o_err(o, o_ref):
    """Max-abs O error beyond the output format's own rounding (O is stored as bf16)."""
    return float((np.abs(o - o_ref) - bf16_half_ulp(o_ref)).max())

CASES = [  # (B, S, Hq, Hkv, d, D, causal, seed)
    (1, 256, 2, 2, 64, 2, True, 0),        # the tiny configuration
    (1, 1024, 4, 2, 128, 2, True, 1),      # GQA 2, four tiles per shard
    (1, 768, 2, 2, 128, 2, True, 2),       # MHA, a straddling tile, odd tile count
    (2, 768, 6, 2, 64, 2, False, 3),       # GQA 3 (slot pairs span tiles), non-causal, B=2
    (1, 1024, 6, 1, 256, 2, True, 4),      # d=256, GQA 6
    (1, 2048, 8, 8, 128, 4, True, 5),      # MHA, D=4
    (1, 1536, 4, 1, 128, 3, True, 6),      # D=3, GQA 4
    (1, 1024, 4, 4, 128, 1, True, 7),      # D=1: plain causal attention
    (1, 2048, 4, 2, 64, 8, True, 8),       # D=8, C=128
]


def _gpu_fwd(q, k, v, D, causal):
    B, S, Hkv, d = k.shape
    problem = zsa.make_problem(B, S, q.shape[3], Hkv, d, D, causal)
    ws = torch.empty(zsa.zsa_workspace_bytes(problem, 0), dtype=torch.uint8, device="cuda")
    o, lse = zsa.attn_fwd(q.cuda(), k.cuda(), v.cuda(), D, causal, workspace=ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    return o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,causal,seed", CASES)
def test_fwd_matches_oracle(oracle, B, S, Hq, Hkv, d, D, causal, seed):
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, D, causal)
    o, lse = _gpu_fwd(q, k, v, D, causal)
    err_o = o_err(o, o_ref)
    err_l = np.abs(lse - lse_ref).max()
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert err_o <= O_TOL and err_l <= LSE_TOL, (err_o, err_l)


STRESS = [  # (B, S, Hq, Hkv, d, D, seed, frac): Q and K rows at random positions scaled x8
    (1, 2048, 4, 2, 128, 4, 31, 0.01),
    (1, 4096, 4, 1, 128, 16, 32, 0.005),
    (1, 1024, 2, 2, 64, 2, 33, 0.02),
    (1, 1024, 6, 1, 256, 2, 34, 0.02),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,seed,frac", STRESS)
def test_fwd_stress_rows(oracle, B, S, Hq, Hkv, d, D, seed, frac):
    # scores of scaled rows reach |s| ~ 300: the running max jumps after the first key
    # tile for some rows of a warp and not others (O rescaling, lse stability)
    q_nat, k, v, _, pos = inputs.make_inputs(B, S, Hq, Hkv, d, seed, stress_frac=frac)
    assert pos.numel() > 0
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, D)
    o, lse = _gpu_fwd(q, k, v, D, True)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    err_o = o_err(o, o_ref)
    err_l = np.abs(lse - lse_ref).max()
    assert err_o <= O_TOL and err_l <= LSE_TOL, (err_o, err_l)


def test_fwd_repeatable_and_stream_async(oracle):
    # two launches on a side stream give identical bytes (the forward is deterministic)
    q_nat, k, v, _, _ = inputs.make_inputs(1, 1024, 4, 2, 128, 11)
    perm, _ = oracle.partition(1024, 2)
    q = inputs.to_shard_major(q_nat, perm, 2).cuda()
    k, v = k.cuda(), v.cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o1, l1 = zsa.attn_fwd(q, k, v, 2)
        o2, l2 = zsa.attn_fwd(q, k, v, 2)
    s.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_wait_timeout_reports_status_and_context_survives(oracle):
    # The stall hook makes the MMA threads wait on a barrier nothing arrives at; with a
    # 20 ms limit the wait gives up, the kernel drains what it has in flight, releases
    # TMEM and records ZSA_ERR_TIMEOUT; the context stays usable for a normal launch.
    B, S, Hq, Hkv, d, D = 1, 2048, 4, 2, 128, 2
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 12)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D).cuda()
    k, v = k.cuda(), v.cuda()
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    ws = torch.empty(zsa.zsa_workspace_bytes(problem, 0), dtype=torch.uint8, device="cuda")
    try:
        zsa.zsa_set_wait_limit_ns(20_000_000)
        zsa.zsa_debug_inject_stall(True)
        zsa.attn_fwd(q, k, v, D, workspace=ws)
        assert zsa.zsa_device_status(ws) == zsa.ZSA_ERR_TIMEOUT
    finally:
        zsa.zsa_debug_inject_stall(False)
        zsa.zsa_set_wait_limit_ns(2_000_000_000)
    o, lse = zsa.attn_fwd(q, k, v, D, workspace=ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    o_ref, lse_ref = oracle.attn_fwd(q.cpu(), k.cpu(), v.cpu(), D)
    assert o_err(o.float().cpu().numpy(), o_ref) <= O_TOL
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= LSE_TOL
