"""GPU parity of the sharded forms of the path, against the fp64 oracle.

1. Shard-major K/V (ZSA_KV_SHARD_MAJOR): the kernels read K/V in the all-gather's
   order and write dK/dV in it; un-permuted, everything equals the oracle's natural-order
   result.  Cases include C = 64 (a 128-key tile spans two zigzag chunks), d = 256, GQA.
2. Shard ranges: each rank of an N-rank run launches over its own shards only (the
   launches run one after another here; none waits on another).  Its O, lse and dQ
   rows equal the oracle's rows, its partial dK / dV equal the oracle's gradient from
   that rank's queries alone (other shards' dO set to zero), and the sum over ranks --
   what the reduce-scatter delivers -- equals the full dK / dV.
Tolerances: O max-abs 1e-2 beyond bf16 output rounding, lse max-abs 1e-3, dQ/dK/dV
relative Frobenius 1e-2.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import dist as zdist
from sequence_sharded_causal_b200 import inputs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, REL_TOL = 1e-2, 1e-3, 1e-2


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def o_err(o, ref):
    return float((np.abs(o - ref) - bf16_half_ulp(ref)).max())


def rel_fro(x, ref):
    return float(np.linalg.norm((x - ref).ravel()) / np.linalg.norm(ref.ravel()))


def _np(x):
    return x.float().cpu().numpy()


KV_CASES = [  # (B, S, Hq, Hkv, d, D, causal, seed, stress)
    (1, 256, 2, 2, 64, 2, True, 60, 0.0),        # C = 64: key tiles span two chunks
    (1, 2048, 8, 2, 128, 4, True, 61, 0.01),     # GQA 4, stressed rows
    (2, 1024, 4, 4, 128, 2, True, 62, 0.0),      # B = 2
    (1, 1024, 6, 1, 256, 2, True, 63, 0.0),      # d = 256
    (1, 1536, 4, 2, 64, 3, False, 64, 0.0),      # non-causal, D = 3
    (1, 4096, 8, 2, 128, 16, True, 65, 0.0),     # D = 16, C = 128
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,causal,seed,stress", KV_CASES)
def test_shard_major_kv_matches_oracle(oracle, B, S, Hq, Hkv, d, D, causal, seed, stress):
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed, stress_frac=stress)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    k_sm = inputs.to_shard_major(k, perm, D)
    v_sm = inputs.to_shard_major(v, perm, D)
    ref = oracle.attn_bwd(q, k, v, do, D, causal)
    kw = dict(kv_layout=zsa.ZSA_KV_SHARD_MAJOR)
    qc, kc, vc, doc = q.cuda(), k_sm.cuda(), v_sm.cuda(), do.cuda()
    o, lse = zsa.attn_fwd(qc, kc, vc, D, causal, **kw)
    dq, dk, dv = zsa.attn_bwd(qc, kc, vc, o, lse, doc, D, causal, **kw)
    torch.cuda.synchronize()
    assert o_err(_np(o), ref["o"]) <= O_TOL
    assert float(np.abs(lse.cpu().numpy() - ref["lse"]).max()) <= LSE_TOL
    assert rel_fro(_np(dq), ref["dq"]) <= REL_TOL
    dk_nat = _np(inputs.from_shard_major(dk.cpu(), perm))
    dv_nat = _np(inputs.from_shard_major(dv.cpu(), perm))
    assert rel_fro(dk_nat, ref["dk"]) <= REL_TOL
    assert rel_fro(dv_nat, ref["dv"]) <= REL_TOL


RANK_CASES = [  # (B, S, Hq, Hkv, d, D, world, kv_layout, seed)
    (1, 2048, 4, 2, 128, 4, 2, zsa.ZSA_KV_SHARD_MAJOR, 70),
    (1, 2048, 4, 2, 128, 4, 4, zsa.ZSA_KV_SHARD_MAJOR, 71),
    (1, 4096, 8, 2, 128, 16, 8, zsa.ZSA_KV_SHARD_MAJOR, 72),
    (1, 1024, 4, 4, 64, 2, 2, zsa.ZSA_KV_NATURAL, 73),
    (1, 1024, 6, 1, 256, 2, 2, zsa.ZSA_KV_SHARD_MAJOR, 74),
    (1, 2048, 8, 2, 256, 4, 4, zsa.ZSA_KV_NATURAL, 75),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,world,kv_layout,seed", RANK_CASES)
def test_rank_launches_match_oracle(oracle, B, S, Hq, Hkv, d, D, world, kv_layout, seed):
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    ref = oracle.attn_bwd(q, k, v, do, D)
    sm = kv_layout == zsa.ZSA_KV_SHARD_MAJOR
    kc = (inputs.to_shard_major(k, perm, D) if sm else k).cuda()
    vc = (inputs.to_shard_major(v, perm, D) if sm else v).cuda()
    dk_sum = torch.zeros(kc.shape, dtype=torch.float64)
    dv_sum = torch.zeros(vc.shape, dtype=torch.float64)
    for rank in range(world):
        s0, ns = zdist.shard_range(rank, world, D)
        kw = dict(kv_layout=kv_layout, shard_begin=s0, shard_count=ns)
        qr, dor = q[s0:s0 + ns].contiguous().cuda(), do[s0:s0 + ns].contiguous().cuda()
        o, lse = zsa.attn_fwd(qr, kc, vc, D, **kw)
        dq, dk, dv = zsa.attn_bwd(qr, kc, vc, o, lse, dor, D, **kw)
        torch.cuda.synchronize()
        assert o_err(_np(o), ref["o"][s0:s0 + ns]) <= O_TOL
        assert float(np.abs(lse.cpu().numpy() - ref["lse"][s0:s0 + ns]).max()) <= LSE_TOL
        assert rel_fro(_np(dq), ref["dq"][s0:s0 + ns]) <= REL_TOL
        # the rank's partial dK / dV: the gradient from its own queries alone
        do_mine = torch.zeros_like(do)
        do_mine[s0:s0 + ns] = do[s0:s0 + ns]
        part = oracle.attn_bwd(q, k, v, do_mine, D)
        dk_n = inputs.from_shard_major(dk.cpu(), perm) if sm else dk.cpu()
        dv_n = inputs.from_shard_major(dv.cpu(), perm) if sm else dv.cpu()
        assert rel_fro(_np(dk_n), part["dk"]) <= REL_TOL
        assert rel_fro(_np(dv_n), part["dv"]) <= REL_TOL
        dk_sum += dk.cpu().double()
        dv_sum += dv.cpu().double()
    # the sum over ranks is what the reduce-scatter delivers to the owners
    dk_tot = inputs.from_shard_major(dk_sum, perm) if sm else dk_sum
    dv_tot = inputs.from_shard_major(dv_sum, perm) if sm else dv_sum
    assert rel_fro(dk_tot.numpy(), ref["dk"]) <= REL_TOL
    assert rel_fro(dv_tot.numpy(), ref["dv"]) <= REL_TOL


def test_rank_launch_zeroes_key_tiles_it_does_not_see(oracle):
    # shard 0 of D = 4 at S = 2048 holds positions 0..255 and 1792..2047, so every key
    # tile sees some of its queries; shard 3 holds 768..1279: key tiles past 1279 are seen
    # by none of its rows and must come back as zeros (not stale accumulators), even
    # after a launch that filled every tile.
    B, S, Hq, Hkv, d, D = 1, 2048, 4, 2, 128, 4
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 76)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D).cuda()
    do = inputs.to_shard_major(do_nat, perm, D).cuda()
    kc, vc = k.cuda(), v.cuda()
    o, lse = zsa.attn_fwd(q, kc, vc, D)
    zsa.attn_bwd(q, kc, vc, o, lse, do, D)           # every tile's accumulators in use
    kw = dict(shard_begin=3, shard_count=1)
    o3, l3 = zsa.attn_fwd(q[3:4].contiguous(), kc, vc, D, **kw)
    dq3, dk3, dv3 = zsa.attn_bwd(q[3:4].contiguous(), kc, vc, o3, l3, do[3:4].contiguous(), D, **kw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dk3[:, 1280:]).item() == 0
    assert torch.count_nonzero(dv3[:, 1280:]).item() == 0
    assert torch.count_nonzero(dv3[:, :1280]).item() > 0
