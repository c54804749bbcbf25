"""GPU check of zsa_permute (K5), the natural <-> zigzag shard-major copy.

A byte copy: the result must equal, bit for bit, the rows of x taken in the order of the
ORACLE's zigzag map (oracle.partition's perm: row j of shard r holds position
perm[r*2C + j]).  Cases: Q-like and K/V-like head counts, d = 64/128/256, B = 2, D = 1,
a single 64-row chunk (C = 64), shard ranges (only the range's chunks read / written),
and a round trip.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa

pytestmark = pytest.mark.gpu

CASES = [  # (B, S, H, d, D)
    (1, 1024, 4, 128, 2),
    (2, 768, 3, 64, 3),
    (1, 1024, 6, 256, 4),
    (1, 2048, 1, 128, 16),     # C = 64
    (1, 512, 2, 128, 1),       # D = 1: the identity
]


def _expected_shard_major(x, perm, D):
    B, S, H, d = x.shape
    y = x[:, torch.as_tensor(perm, dtype=torch.int64)]
    return y.reshape(B, D, S // D, H, d).transpose(0, 1).contiguous()


@pytest.mark.parametrize("B,S,H,d,D", CASES)
def test_permute_matches_oracle_map(oracle, B, S, H, d, D):
    g = torch.Generator().manual_seed(B * 7 + S + H + d + D)
    x = torch.randn((B, S, H, d), generator=g).to(torch.bfloat16)
    perm, _ = oracle.partition(S, D)
    want = _expected_shard_major(x, perm, D)
    xs = x.cuda()
    y = zsa.to_shard_major(xs, D)
    back = zsa.from_shard_major(y, D)
    torch.cuda.synchronize()
    assert torch.equal(y.cpu(), want)
    assert torch.equal(back.cpu(), x)


def test_permute_shard_range(oracle):
    B, S, H, d, D = 2, 2048, 4, 128, 4
    g = torch.Generator().manual_seed(5)
    x = torch.randn((B, S, H, d), generator=g).to(torch.bfloat16)
    perm, _ = oracle.partition(S, D)
    want = _expected_shard_major(x, perm, D)
    xs = x.cuda()
    for sb, sc in ((1, 2), (3, 1), (0, 4)):
        y = zsa.to_shard_major(xs, D, shard_begin=sb, shard_count=sc)
        torch.cuda.synchronize()
        assert torch.equal(y.cpu(), want[sb:sb + sc])
        # shard-major -> natural writes the range's positions and nothing else
        out = torch.full((B, S, H, d), 7.0, dtype=torch.bfloat16, device="cuda")
        zsa.from_shard_major(y, D, shard_begin=sb, shard_count=sc, out=out)
        torch.cuda.synchronize()
        got = out.cpu()
        pos = np.asarray(perm).reshape(D, S // D)[sb:sb + sc].ravel()
        mask = np.zeros(S, bool)
        mask[pos] = True
        assert torch.equal(got[:, torch.from_numpy(mask)], x[:, torch.from_numpy(mask)])
        assert (got[:, torch.from_numpy(~mask)] == 7.0).all()


def test_permuted_inputs_drive_the_attention(oracle):
    # Q and K/V brought to shard-major order by K5 feed the attention kernels directly:
    # the same values reach the same tiles in the same order as with the generator's own
    # layout and natural-order K/V, so the results are identical
    B, S, Hq, Hkv, d, D = 1, 2048, 4, 2, 128, 4
    from sequence_sharded_causal_b200 import inputs
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 11)
    perm, _ = oracle.partition(S, D)
    q_ref = inputs.to_shard_major(q_nat, perm, D).cuda()
    kc, vc = k.cuda(), v.cuda()
    q_k5 = zsa.to_shard_major(q_nat.cuda(), D)
    assert torch.equal(q_k5, q_ref)
    o_ref, l_ref = zsa.attn_fwd(q_ref, kc, vc, D)
    k_sm, v_sm = zsa.to_shard_major(kc, D), zsa.to_shard_major(vc, D)
    o_sm, l_sm = zsa.attn_fwd(q_k5, k_sm, v_sm, D, kv_layout=zsa.ZSA_KV_SHARD_MAJOR)
    torch.cuda.synchronize()
    assert torch.equal(o_sm, o_ref) and torch.equal(l_sm, l_ref)
    # and back: O in position order
    o_nat = zsa.from_shard_major(o_sm, D)
    torch.cuda.synchronize()
    assert torch.equal(o_nat.cpu(), inputs.from_shard_major(o_ref.cpu(), perm))
    # the backward with shard-major K/V writes dK / dV in that order; K5 brings them back
    _, _, _, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 11)
    do = zsa.to_shard_major(do_nat.cuda(), D)
    dq_ref, dk_ref, dv_ref = zsa.attn_bwd(q_ref, kc, vc, o_ref, l_ref, do, D)
    dq_sm, dk_sm, dv_sm = zsa.attn_bwd(q_k5, k_sm, v_sm, o_sm, l_sm, do, D,
                                       kv_layout=zsa.ZSA_KV_SHARD_MAJOR)
    torch.cuda.synchronize()
    # dK / dV are accumulated inside one CTA per key tile: identical.  dQ sums the key
    # tiles' contributions with fp32 reduce-adds whose order between CTAs is not fixed,
    # so two runs agree to fp32 summation-order rounding before the bf16 rounding
    assert torch.equal(zsa.from_shard_major(dk_sm, D), dk_ref)
    assert torch.equal(zsa.from_shard_major(dv_sm, D), dv_ref)
    diff = (dq_sm.float() - dq_ref.float()).norm() / dq_ref.float().norm()
    assert float(diff) < 1e-3, float(diff)
