"""GPU parity of zsa_tsp_project, the local projection GEMM of a TSP broadcast step,
against the oracle (fp64 matmul of the same bf16 values).

Tolerances: bf16 outputs may differ from the fp64 product by their own rounding (half a
bf16 ulp) plus 1e-3 of the output's RMS (fp32 accumulation over K); fp32-accumulated
outputs by 1e-4 of the RMS.  The schedule test emulates every rank of a D-rank run one
after another on one GPU (the broadcast is the local shard; no launch waits on another)
with the packed shards of sequence_sharded_causal_b200.dist, and checks Q, K, V and the
summed output projection against the unsharded products.
"""
import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import dist as zdist

pytestmark = pytest.mark.gpu


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def check_bf16(y, ref):
    rms = float(np.sqrt((ref ** 2).mean()))
    err = float((np.abs(y - ref) - bf16_half_ulp(ref)).max())
    assert err <= 1e-3 * rms, (err, rms)


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("T,K,N", [(128, 64, 128), (256, 512, 384), (1024, 4096, 768),
                                   (384, 1280, 1024),
                                   (200, 72, 160),     # ragged: T, N, K past the tile edges
                                   (4096, 512, 2560),  # 128 x 256 tiles (N = 256 MMAs)
                                   (4000, 264, 2560)]) # 128 x 256 tiles, ragged T and K
def test_project_bf16_matches_oracle(oracle, T, K, N):
    x, w = _rand((T, K), 1), _rand((K, N), 2, 0.05)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    y = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
    zsa.zsa_tsp_project(x.cuda(), w.cuda(), [(y, N, N, 0)], ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    check_bf16(y.float().cpu().numpy(), oracle.project(x, w))


def test_project_segments_and_fp32_accumulate(oracle):
    T, K, N = 256, 256, 512
    x1, x2 = _rand((T, K), 3), _rand((T, K), 4)
    w = _rand((K, N), 5, 0.05)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    # segments: 96 columns into a strided bf16 view, 160 into another, the rest (256)
    # added into an fp32 accumulator, twice
    a = torch.zeros(T, 200, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(T, 160, dtype=torch.bfloat16, device="cuda")
    acc = torch.zeros(T, 256, dtype=torch.float32, device="cuda")
    segs = [(a[:, 40:], 200, 96, 0), (b, 160, 160, 0), (acc, 256, 256, 1)]
    zsa.zsa_tsp_project(x1.cuda(), w.cuda(), segs, ws)
    zsa.zsa_tsp_project(x2.cuda(), w.cuda(), segs, ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    ref2 = oracle.project(x2, w)
    check_bf16(a[:, 40:136].float().cpu().numpy(), ref2[:, :96])
    assert torch.count_nonzero(a[:, :40]).item() == 0 and torch.count_nonzero(a[:, 136:]).item() == 0
    check_bf16(b.float().cpu().numpy(), ref2[:, 96:256])
    ref_acc = oracle.project(x1, w)[:, 256:] + ref2[:, 256:]
    rms = float(np.sqrt((ref_acc ** 2).mean()))
    assert float(np.abs(acc.cpu().numpy() - ref_acc).max()) <= 1e-4 * rms


def test_project_wide_tiles_fp32_accumulate(oracle):
    # enough 128 x 256 tiles for the wide-tile build: a bf16 segment and an fp32 one
    T, K, N = 4096, 256, 2560
    x, w = _rand((T, K), 6), _rand((K, N), 7, 0.05)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    a = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    acc = torch.full((T, 2048), 1.0, dtype=torch.float32, device="cuda")
    zsa.zsa_tsp_project(x.cuda(), w.cuda(), [(a, 512, 512, 0), (acc, 2048, 2048, 1)], ws)
    assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
    ref = oracle.project(x, w)
    check_bf16(a.float().cpu().numpy(), ref[:, :512])
    ref_acc = ref[:, 512:] + 1.0
    rms = float(np.sqrt((ref_acc ** 2).mean()))
    assert float(np.abs(acc.cpu().numpy() - ref_acc).max()) <= 1e-4 * rms


@pytest.mark.parametrize("T,hidden,Hq,Hkv,d,D", [(256, 512, 8, 2, 64, 4),
                                                 (512, 1024, 8, 4, 128, 8),
                                                 (256, 640, 6, 1, 256, 2)])
def test_emulated_rank_schedule(oracle, T, hidden, Hq, Hkv, d, D):
    wq, wk, wv = (_rand((hidden, n), 10 + i, 0.05) for i, n in enumerate((Hq * d, Hkv * d, Hkv * d)))
    wo = _rand((Hq * d, hidden), 13, 0.05)
    nq, nk, nv = zdist.qkv_columns(Hq, Hkv, d, D)
    shards = [zdist.pack_qkv_shard(wq, wk, wv, s, D).cuda() for s in range(D)]
    wo_sh = [zdist.wo_shard(wo, s, D).cuda() for s in range(D)]
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    for r in range(D):
        x = _rand((T, hidden), 20 + r)
        o = _rand((T, Hq * d), 40 + r)
        xc, oc = x.cuda(), o.cuda()
        q = torch.empty(T, Hq * d, dtype=torch.bfloat16, device="cuda")
        k = torch.empty(T, Hkv * d, dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        y32 = torch.zeros(T, hidden, dtype=torch.float32, device="cuda")
        for s in range(D):        # the D broadcast steps of rank r (shard s "received")
            zsa.zsa_tsp_project(xc, shards[s], [(q[:, s * nq:], Hq * d, nq, 0),
                                                (k[:, s * nk:], Hkv * d, nk, 0),
                                                (v[:, s * nv:], Hkv * d, nv, 0)], ws)
            zsa.zsa_tsp_project(oc[:, s * nq:], wo_sh[s], [(y32, hidden, hidden, 1)], ws,
                                T=T, K=nq, N=hidden, ldx=Hq * d)
        assert zsa.zsa_device_status(ws) == zsa.ZSA_OK
        check_bf16(q.float().cpu().numpy(), oracle.project(x, wq))
        check_bf16(k.float().cpu().numpy(), oracle.project(x, wk))
        check_bf16(v.float().cpu().numpy(), oracle.project(x, wv))
        ref_y = oracle.project(o, wo)
        rms = float(np.sqrt((ref_y ** 2).mean()))
        assert float(np.abs(y32.cpu().numpy() - ref_y).max()) <= 1e-4 * rms
