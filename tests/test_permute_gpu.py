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
