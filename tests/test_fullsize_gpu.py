"""Parity at the benchmark configurations' FULL sizes, in the launch configuration bench.py
times: one zsa_attn_fwd and one zsa_attn_bwd over the whole problem, all D shards in one
launch each.

The fp64 oracle cannot run full-size attention, so:
  * forward: O and lse on sampled query rows (oracle_attn_fwd_rows), 256 per head: the
    global positions 0 and S-1, the first and last position of every zigzag chunk (the
    diagonal-tile cases), every stressed position of the long-context configuration,
    then random positions (generator seeded seed+1000) up to 256;
  * dQ on the same sampled rows (oracle_attn_dq_rows);
  * dK and dV through identities that hold at any size (rows of P sum to 1, rows of dS
    sum to 0): per kv head, sum_k dV_k = sum of dO over the group's q rows (to 1e-2 of
    that sum), and sum_k dK_k = 0 (to 1e-2 of sum_k |dK_k|, the mass that cancels);
and, at a reduced sequence length with the same heads, d and D, a full elementwise
forward + backward check against the full oracle (for the long-context configuration
with 1% of the Q and K rows scaled x8, so every stressed row is compared elementwise).

Inputs follow the recipe of sequence_sharded_causal_b200.inputs (seeds 1..4 for the
four configurations).  Tolerances: O max-abs 1e-2 beyond bf16 output rounding, lse
max-abs 1e-3, dQ/dK/dV relative Frobenius 1e-2.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import inputs

pytestmark = pytest.mark.gpu

FULL = {  # name: (B, S, Hq, Hkv, d, D, seed, stress_frac, reduced S, reduced-S stress_frac)
    "7b_mha": (1, 16384, 32, 32, 128, 8, 1, 0.0, 4096, 0.0),
    "8b_gqa": (1, 32768, 32, 8, 128, 8, 2, 0.0, 4096, 0.0),
    "wide_gqa": (1, 65536, 24, 4, 256, 4, 3, 0.0, 2048, 0.0),
    # the long-context heads and shard count (D = 16, C = 128 at S = 4096), with 1% of
    # the Q and K rows scaled x8 so that about 41 stressed rows land in the reduced case
    "long": (1, 131072, 32, 8, 128, 16, 4, 0.001, 4096, 0.01),
}
O_TOL, LSE_TOL, REL_TOL = 1e-2, 1e-3, 1e-2


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def rel_fro(x, ref):
    return float(np.linalg.norm((x - ref).ravel()) / np.linalg.norm(ref.ravel()))


def sample_positions(S, D, seed, extra):
    C = S // (2 * D)
    chosen = [0, S - 1]
    for c in range(2 * D):
        chosen += [c * C, c * C + C - 1]
    chosen += [int(p) for p in extra]
    chosen = list(dict.fromkeys(chosen))
    g = torch.Generator().manual_seed(seed + 1000)
    for p in torch.randperm(S, generator=g).tolist():
        if len(chosen) >= 256:
            break
        if p not in chosen:
            chosen.append(p)
    return np.array(sorted(chosen[:max(256, len(chosen))]), np.int64)


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_sampled_rows(oracle, name):
    B, S, Hq, Hkv, d, D, seed, frac, _, _ = FULL[name]
    q_nat, k, v, do_nat, stress = inputs.make_inputs(B, S, Hq, Hkv, d, seed, stress_frac=frac)
    perm, inv = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    del q_nat, do_nat
    dev = torch.device("cuda", 0)
    qc, kc, vc, doc = (x.to(dev) for x in (q, k, v, do))
    o, lse = zsa.attn_fwd(qc, kc, vc, D)
    dq, dk, dv = zsa.attn_bwd(qc, kc, vc, o, lse, doc, D)
    torch.cuda.synchronize(dev)
    del qc, kc, vc, doc
    # sampled rows (B = 1): shard-major row index of each sampled position
    pos = sample_positions(S, D, seed, stress.tolist())
    assert set(stress.tolist()) <= set(pos.tolist())
    rows = inv[pos].astype(np.int64)
    qf = q.reshape(-1, Hq, d)[rows]
    dof = do.reshape(-1, Hq, d)[rows]
    o_ref, lse_ref = oracle.attn_fwd_rows(qf, rows, k, v, D, Hq)
    o_got = o.reshape(-1, Hq, d)[torch.from_numpy(rows).to(o.device)].float().cpu().numpy()
    twoC = S // D
    lse_np = lse.cpu().numpy()                                  # [D][B][Hq][2C]
    lse_got = np.stack([lse_np[r // twoC, 0, :, r % twoC] for r in rows])
    err_o = float((np.abs(o_got - o_ref) - bf16_half_ulp(o_ref)).max())
    err_l = float(np.abs(lse_got - lse_ref).max())
    assert np.isfinite(o_got).all() and np.isfinite(lse_got).all()
    assert err_o <= O_TOL and err_l <= LSE_TOL, (err_o, err_l)
    dq_ref = oracle.attn_dq_rows(qf, dof, rows, k, v, D, Hq)
    dq_got = dq.reshape(-1, Hq, d)[torch.from_numpy(rows).to(dq.device)].float().cpu().numpy()
    assert rel_fro(dq_got, dq_ref) <= REL_TOL
    # identities for dK, dV at full size (sums in fp64 of the bf16 results)
    # Each identity is held to the relative tolerance of the quantities it compares:
    # sum_k dV_k against sum_q dO_q, and the cancellation sum_k dK_k = 0 against the
    # mass that cancels, sum_k |dK_k|.
    G = Hq // Hkv
    dv_c, dk_c = dv.cpu()[0], dk.cpu()[0]                        # [S][Hkv][d] bf16
    for g in range(Hkv):
        want = do[:, 0, :, g * G:(g + 1) * G, :].double().sum(dim=(0, 1, 2))
        dvg, dkg = dv_c[:, g].double(), dk_c[:, g].double()
        assert float((dvg.sum(0) - want).norm()) <= REL_TOL * float(want.norm())
        assert float(dkg.sum(0).norm()) <= REL_TOL * float(dkg.abs().sum(0).norm())


@pytest.mark.parametrize("name", [n for n in FULL if FULL[n][8]])
def test_reduced_length_full_check(oracle, name):
    B, _, Hq, Hkv, d, D, seed, _, S, frac = FULL[name]
    q_nat, k, v, do_nat, stress = inputs.make_inputs(B, S, Hq, Hkv, d, seed + 100,
                                                     stress_frac=frac)
    assert (stress.numel() > 0) == (frac > 0)
    perm, _ = oracle.partition(S, D)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    dev = torch.device("cuda", 0)
    qc, kc, vc, doc = (x.to(dev) for x in (q, k, v, do))
    o, lse = zsa.attn_fwd(qc, kc, vc, D)
    dq, dk, dv = zsa.attn_bwd(qc, kc, vc, o, lse, doc, D)
    torch.cuda.synchronize(dev)
    ref = oracle.attn_bwd(q, k, v, do, D)
    o_np = o.float().cpu().numpy()
    assert float((np.abs(o_np - ref["o"]) - bf16_half_ulp(ref["o"])).max()) <= O_TOL
    assert float(np.abs(lse.cpu().numpy() - ref["lse"]).max()) <= LSE_TOL
    for nm, x in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert rel_fro(x.float().cpu().numpy(), ref[nm]) <= REL_TOL, nm
