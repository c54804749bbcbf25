"""Full-size checks of the kernels beyond the attention path, in the launch configuration
bench.py times, on sampled outputs the oracle computes one by one.

- TSP projection step at the wide-head shape (T = 16384 tokens per rank, hidden 5120):
  the QKV step (N = 2048, the 128 x 256 tile build) and the output-projection step into
  an fp32 accumulator (K = 1536, N = 5120), 64 sampled rows each against the fp64
  product of the same bf16 values.
- Ring-attention merge at the long-context Q layout (S = 131072, Hq = 32, d = 128,
  D = 16): two seeded partials merged in place; 512 sampled (row, head) pairs against
  the oracle's merge of the same parts.
- K5 permute of the long-context Q tensor (1 GiB): 512 sampled rows bit-exact against the
  oracle's zigzag map.
Tolerances are those of the small-size tests of the same kernels.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa

pytestmark = pytest.mark.gpu


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def test_tsp_steps_full_size_sampled_rows(oracle):
    T, hidden, nq, nqkv = 16384, 5120, 1536, 2048
    g = torch.Generator(device="cuda").manual_seed(21)
    x = torch.randn(T, hidden, generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn(hidden, nqkv, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    o = torch.randn(T, nq, generator=g, device="cuda").to(torch.bfloat16)
    wo = (torch.randn(nq, hidden, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    y = torch.empty(T, nqkv, dtype=torch.bfloat16, device="cuda")
    y32 = torch.full((T, hidden), 0.5, dtype=torch.float32, device="cuda")
    zsa.zsa_tsp_project(x, w, [(y, nqkv, nqkv, 0)], ws)
    zsa.zsa_tsp_project(o, wo, [(y32, hidden, hidden, 1)], ws)
    torch.cuda.synchronize()
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    rows = torch.randperm(T, generator=torch.Generator().manual_seed(22))[:64]
    ref = oracle.project(x[rows.cuda()].cpu(), w.cpu())
    got = y[rows.cuda()].float().cpu().numpy()
    rms = float(np.sqrt((ref ** 2).mean()))
    assert float((np.abs(got - ref) - bf16_half_ulp(ref)).max()) <= 1e-3 * rms
    ref32 = oracle.project(o[rows.cuda()].cpu(), wo.cpu()) + 0.5
    got32 = y32[rows.cuda()].cpu().numpy()
    rms32 = float(np.sqrt((ref32 ** 2).mean()))
    assert float(np.abs(got32 - ref32).max()) <= 1e-4 * rms32


def test_merge_full_size_sampled_pairs(oracle):
    B, S, Hq, Hkv, d, D = 1, 131072, 32, 8, 128, 16
    twoC = S // D
    g = torch.Generator(device="cuda").manual_seed(23)
    shp, lshp = (D, B, twoC, Hq, d), (D, B, Hq, twoC)
    o1 = torch.randn(shp, generator=g, device="cuda").to(torch.bfloat16)
    o2 = torch.randn(shp, generator=g, device="cuda").to(torch.bfloat16)
    l1 = torch.randn(lshp, generator=g, device="cuda")
    l2 = torch.randn(lshp, generator=g, device="cuda")
    # a few (row, head) pairs with an empty second part
    l2[0, 0, 0, :4] = float("-inf")
    o2[0, 0, :4, 0] = 0
    gen = torch.Generator().manual_seed(24)
    r = torch.randint(0, D, (512,), generator=gen)
    j = torch.randint(0, twoC, (512,), generator=gen)
    h = torch.randint(0, Hq, (512,), generator=gen)
    r[:4], j[:4], h[:4] = 0, torch.arange(4), 0
    parts = [(x[r, 0, j, h].cpu(), y[r, 0, h, j].cpu()) for x, y in ((o1, l1), (o2, l2))]
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    zsa.zsa_attn_merge(problem, [o1, o2], [l1, l2], o1, l1)       # in place, as a ring step
    torch.cuda.synchronize()
    # the oracle merges the sampled pairs as a [1][1][n][1][d] Q layout
    o_ref, l_ref = oracle.attn_merge([p[0].double().numpy().reshape(1, 1, -1, 1, d) for p in parts],
                                     [p[1].double().numpy().reshape(1, 1, 1, -1) for p in parts])
    o_got = o1[r, 0, j, h].float().cpu().numpy()
    l_got = l1[r, 0, h, j].cpu().numpy()
    o_ref = o_ref.reshape(-1, d)
    l_ref = l_ref.reshape(-1)
    assert float((np.abs(o_got - o_ref) - bf16_half_ulp(o_ref)).max()) <= 1e-2
    assert float(np.abs(l_got - l_ref).max()) <= 1e-3


def test_permute_full_size_sampled_rows(oracle):
    B, S, H, d, D = 1, 131072, 32, 128, 16
    g = torch.Generator(device="cuda").manual_seed(25)
    x = torch.randn((B, S, H, d), generator=g, device="cuda").to(torch.bfloat16)
    y = zsa.to_shard_major(x, D)
    torch.cuda.synchronize()
    perm, _ = oracle.partition(S, D)
    perm = np.asarray(perm)
    gen = torch.Generator().manual_seed(26)
    r = torch.randint(0, D, (512,), generator=gen)
    j = torch.randint(0, S // D, (512,), generator=gen)
    pos = torch.from_numpy(perm[(r * (S // D) + j).numpy()])
    assert torch.equal(y[r.cuda(), 0, j.cuda()].cpu(), x[0, pos.cuda()].cpu())
