"""GPU parity of zsa_attn_fwd_block, the forward over one block of keys (a ring step).

Each case compares the kernel's partial (O, lse) with the oracle's key-range forward on
the same seeded inputs: O max-abs 1e-2 beyond bf16 output rounding, lse max-abs 1e-3,
and rows that see no key of the block exactly O = 0, lse = -inf.  Blocks are unaligned
to the 128-key tiles, empty, whole, past every query, and given both inside a full
natural K/V buffer and as a compact copy.  The ring test runs a whole ring attention on
one GPU: for each rank's shard, the K/V block of every shard in ring order (two chunk
calls per block, read straight from the shard-major buffer the all-gather would fill),
merged with zsa_attn_merge, against the oracle's full forward.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import inputs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def check(o, lse, o_ref, lse_ref):
    """Partial results: finite rows within tolerance, empty rows exact."""
    assert np.array_equal(np.isinf(lse), np.isinf(lse_ref))
    assert not np.isnan(lse).any() and np.isfinite(o).all()
    empty = np.isinf(lse_ref)                                   # [D'][B][Hq][2C]
    o_empty = np.broadcast_to(empty.transpose(0, 1, 3, 2)[..., None], o.shape)
    assert (o[o_empty] == 0).all()
    fin = ~empty
    err_l = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    err_o = float((np.abs(o - o_ref) - bf16_half_ulp(o_ref)).max())
    assert err_o <= O_TOL and err_l <= LSE_TOL, (err_o, err_l)


def _gpu_block(q, k, v, D, lo, hi, causal=True, compact=False):
    B, S = k.shape[0], k.shape[1]
    if compact:
        kb = k[:, lo:hi].contiguous().cuda()
        vb = v[:, lo:hi].contiguous().cuda()
        o, lse = zsa.attn_fwd_block(q.cuda(), kb, vb, D, lo, hi, causal=causal)
    else:
        o, lse = zsa.attn_fwd_block(q.cuda(), k.cuda(), v.cuda(), D, lo, hi, rows_per_batch=S,
                                    row_offset=lo, causal=causal)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


CASES = [  # (B, S, Hq, Hkv, d, D, causal, (lo, hi), compact, seed)
    (1, 1024, 4, 2, 128, 2, True, (0, 1024), False, 90),     # every key: the full forward
    (1, 1024, 4, 2, 128, 2, True, (100, 612), False, 91),    # unaligned both ends
    (1, 1024, 4, 2, 128, 2, True, (256, 384), True, 92),     # one zigzag chunk, compact
    (1, 1024, 4, 2, 128, 2, True, (900, 1024), False, 93),   # most rows see no key
    (1, 1024, 4, 2, 128, 2, True, (300, 300), False, 94),    # empty block
    (2, 768, 6, 2, 64, 2, False, (64, 700), True, 95),       # non-causal, B = 2, GQA 3
    (1, 1024, 6, 1, 256, 2, True, (130, 1000), False, 96),   # d = 256, GQA 6
    (1, 2048, 4, 1, 128, 8, True, (1, 2047), True, 97),      # D = 8, C = 128
    (2, 1536, 4, 2, 128, 3, True, (640, 1100), True, 98),    # D = 3, B = 2
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,causal,rng,compact,seed", CASES)
def test_block_matches_oracle(oracle, B, S, Hq, Hkv, d, D, causal, rng, compact, seed):
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    lo, hi = rng
    o_ref, lse_ref = oracle.attn_fwd_keys(q, k, v, D, lo, hi, causal)
    o, lse = _gpu_block(q, k, v, D, lo, hi, causal, compact)
    check(o, lse, o_ref, lse_ref)


def test_block_stress_rows(oracle):
    # x8 rows: scores near 300 inside a block that starts mid-tile
    B, S, Hq, Hkv, d, D = 1, 2048, 4, 2, 128, 4
    q_nat, k, v, _, pos = inputs.make_inputs(B, S, Hq, Hkv, d, 99, stress_frac=0.01)
    assert pos.numel() > 0
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    o_ref, lse_ref = oracle.attn_fwd_keys(q, k, v, D, 200, 1800)
    o, lse = _gpu_block(q, k, v, D, 200, 1800)
    check(o, lse, o_ref, lse_ref)


def test_block_whole_range_equals_forward(oracle):
    # with every key in the block the kernel runs the same tiles, masks and order as
    # zsa_attn_fwd: the two results are identical
    B, S, Hq, Hkv, d, D = 1, 1024, 4, 2, 128, 4
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 100)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D).cuda()
    o_f, l_f = zsa.attn_fwd(q, k.cuda(), v.cuda(), D)
    o_b, l_b = zsa.attn_fwd_block(q, k.cuda(), v.cuda(), D, 0, S, rows_per_batch=S)
    assert torch.equal(o_f, o_b) and torch.equal(l_f, l_b)


RING = [  # (B, S, Hq, Hkv, d, D, seed)
    (1, 1024, 4, 2, 128, 4, 101),
    (2, 768, 2, 2, 64, 3, 102),
    (1, 1024, 6, 1, 256, 2, 103),
    (1, 4096, 8, 2, 128, 8, 104),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,seed", RING)
def test_ring_attention_on_one_gpu(oracle, B, S, Hq, Hkv, d, D, seed):
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, D)
    C = S // (2 * D)
    k_sm = inputs.to_shard_major(k, perm, D).cuda()     # [D][B][2C][Hkv][d]: the gathered K/V
    v_sm = inputs.to_shard_major(v, perm, D).cuda()
    qc = q.cuda()
    for r in range(D):                                  # rank r's queries
        q_r = qc[r:r + 1]
        problem = zsa.make_problem(B, S, Hq, Hkv, d, D, shard_begin=r, shard_count=1)
        o_parts, l_parts = [], []
        for step in range(D):                           # the block rank r holds at this step
            s = (r - step) % D
            for lo, off in ((s * C, 0), ((2 * D - 1 - s) * C, C)):
                o, lse = zsa.attn_fwd_block(q_r, k_sm[s], v_sm[s], D, lo, lo + C,
                                            rows_per_batch=2 * C, row_offset=off,
                                            shard_begin=r, shard_count=1)
                o_parts.append(o)
                l_parts.append(lse)
        o = torch.empty_like(o_parts[0])
        lse = torch.empty_like(l_parts[0])
        zsa.zsa_attn_merge(problem, o_parts, l_parts, o, lse)
        torch.cuda.synchronize()
        o_np, l_np = o.float().cpu().numpy(), lse.cpu().numpy()
        assert np.isfinite(o_np).all() and np.isfinite(l_np).all()
        err_o = float((np.abs(o_np - o_ref[r:r + 1]) - bf16_half_ulp(o_ref[r:r + 1])).max())
        err_l = float(np.abs(l_np - lse_ref[r:r + 1]).max())
        # the parts are bf16: the merged O carries their rounding too (up to one more
        # half-ulp of the largest part), within the same 1e-2 bound
        assert err_o <= O_TOL and err_l <= LSE_TOL, (r, err_o, err_l)
