"""GPU parity of zsa_attn_merge, the ring-attention (O, lse) merge, against the oracle.

The partial results come from the oracle's key-range forward, rounded to the formats the
GPU stores (O bf16, lse fp32).  zsa_attn_merge of those parts is compared with the
oracle's merge of the SAME rounded parts (O max-abs 1e-2 beyond bf16 output rounding,
lse max-abs 1e-3) and with the full forward.  The splits include the ring order of a
zigzag run (each step's K/V block is one shard's two chunks), empty parts (rows that see
no key of a block), an in-place running merge, a shard range, and 32 parts.
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


def o_err(o, ref):
    return float((np.abs(o - ref) - bf16_half_ulp(ref)).max())


def lse_err(lse, ref):
    assert np.array_equal(np.isinf(lse), np.isinf(ref))
    fin = np.isfinite(ref)
    return float(np.abs(lse[fin] - ref[fin]).max()) if fin.any() else 0.0


def _parts(oracle, q, k, v, D, ranges, causal=True):
    """Oracle partials over key ranges, rounded as the GPU stores them."""
    o_p, l_p = [], []
    for lo, hi in ranges:
        o, lse = oracle.attn_fwd_keys(q, k, v, D, lo, hi, causal)
        o_p.append(torch.from_numpy(o).to(torch.bfloat16))
        l_p.append(torch.from_numpy(lse).to(torch.float32))
    return o_p, l_p


def _ring_ranges(S, D):
    """Key blocks in the order a ring hands them to shard 0: shard s's two chunks."""
    C = S // (2 * D)
    out = []
    for s in range(D):
        out += [(s * C, (s + 1) * C), ((2 * D - 1 - s) * C, (2 * D - s) * C)]
    return out


CASES = [  # (B, S, Hq, Hkv, d, D, split, seed)
    (1, 1024, 4, 2, 128, 4, "ring", 80),
    (1, 512, 2, 2, 64, 2, "ring", 81),
    (1, 1024, 6, 1, 256, 2, "ring", 82),
    (2, 768, 4, 4, 128, 3, [(0, 100), (100, 101), (101, 768)], 83),
    (1, 2048, 4, 2, 128, 16, "ring", 84),     # 32 parts
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,D,split,seed", CASES)
def test_merge_matches_oracle(oracle, B, S, Hq, Hkv, d, D, split, seed):
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, seed)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    ranges = _ring_ranges(S, D) if split == "ring" else split
    assert len(ranges) <= zsa.ZSA_MERGE_MAX_PARTS
    o_p, l_p = _parts(oracle, q, k, v, D, ranges)
    ref_o, ref_l = oracle.attn_merge([x.double() for x in o_p], [x.double() for x in l_p])
    full_o, full_l = oracle.attn_fwd(q, k, v, D)
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    oc, lc = [x.cuda() for x in o_p], [x.cuda() for x in l_p]
    o = torch.empty_like(oc[0])
    lse = torch.empty_like(lc[0])
    zsa.zsa_attn_merge(problem, oc, lc, o, lse)
    torch.cuda.synchronize()
    o_np, l_np = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(o_np).all()
    assert o_err(o_np, ref_o) <= O_TOL
    assert lse_err(l_np, ref_l) <= LSE_TOL
    assert o_err(o_np, full_o) <= O_TOL
    assert lse_err(l_np, full_l) <= LSE_TOL


def test_running_merge_in_place_and_empty_rows(oracle):
    # a ring step at a time: (O, lse) <- merge((O, lse), (O_s, lse_s)), output aliasing
    # the first part; the first blocks leave many rows empty (lse = -inf)
    B, S, Hq, Hkv, d, D = 1, 1024, 4, 2, 128, 4
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 85)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    ranges = _ring_ranges(S, D)[::-1]        # late chunks first: many empty rows early on
    o_p, l_p = _parts(oracle, q, k, v, D, ranges)
    assert torch.isinf(l_p[0]).any()
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    o_run, l_run = o_p[0].cuda(), l_p[0].cuda()
    for o_s, l_s in zip(o_p[1:], l_p[1:]):
        zsa.zsa_attn_merge(problem, [o_run, o_s.cuda()], [l_run, l_s.cuda()], o_run, l_run)
    torch.cuda.synchronize()
    full_o, full_l = oracle.attn_fwd(q, k, v, D)
    # one bf16 rounding per step: still well inside the O tolerance
    assert o_err(o_run.float().cpu().numpy(), full_o) <= O_TOL
    assert lse_err(l_run.cpu().numpy(), full_l) <= LSE_TOL


def test_merge_on_a_shard_range_and_all_empty_rows(oracle):
    # shard range: the parts hold shards 1..2 of D = 4 only; a key block above every
    # row's position leaves those rows empty in all parts: O = 0, lse = -inf
    B, S, Hq, Hkv, d, D = 1, 1024, 2, 1, 64, 4
    q_nat, k, v, _, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 86)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    ranges = [(896, 960), (960, 1024)]         # the last chunk: only shard 0 sees it
    o_p, l_p = _parts(oracle, q, k, v, D, ranges)
    o_p = [x[1:3].contiguous() for x in o_p]
    l_p = [x[1:3].contiguous() for x in l_p]
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D, shard_begin=1, shard_count=2)
    o = torch.full(o_p[0].shape, 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(l_p[0].shape, dtype=torch.float32, device="cuda")
    zsa.zsa_attn_merge(problem, [x.cuda() for x in o_p], [x.cuda() for x in l_p], o, lse)
    torch.cuda.synchronize()
    assert torch.isinf(lse).all() and (lse < 0).all()
    assert torch.count_nonzero(o).item() == 0
