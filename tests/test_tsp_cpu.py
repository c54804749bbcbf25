"""The TSP attention-layer weight schedule ("Folding Tensor and Sequence Parallelism"
summary, section 2, attention layer), on CPU.

- oracle.project is pinned by a brute-force triple loop on tiny inputs, and by special
  cases (identity and permutation weights);
- gloo ranks (world 2 and 4) run sequence_sharded_causal_b200.dist's broadcast schedule
  on CPU tensors, with the oracle's projection in place of the GPU GEMM: after the D
  steps every rank's Q, K, V equal its tokens times the UNSHARDED W_Q, W_K, W_V, and the
  summed output-projection partials equal O W_O;
- zsa_tsp_project rejects bad arguments before touching a device.
"""
import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_project_brute_force_and_special_cases(oracle):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 7))
    w = rng.standard_normal((7, 4))
    y = oracle.project(x, w)
    for i in range(5):
        for j in range(4):
            assert abs(y[i, j] - sum(x[i, t] * w[t, j] for t in range(7))) <= 1e-12
    assert np.array_equal(oracle.project(x, np.eye(7)), x)
    perm = rng.permutation(7)
    assert np.array_equal(oracle.project(x, np.eye(7)[:, perm]), x[:, perm])
    xb = torch.from_numpy(x).to(torch.bfloat16)       # bf16 values are widened exactly
    assert np.array_equal(oracle.project(xb, np.eye(7)), xb.double().numpy())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPE = dict(T=16, hidden=32, Hq=4, Hkv=2, d=8)


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import oracle
    from sequence_sharded_causal_b200 import dist as zd
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, hidden, Hq, Hkv, d = (SHAPE[k] for k in ("T", "hidden", "Hq", "Hkv", "d"))
        g = torch.Generator().manual_seed(11)
        wq = torch.randn(hidden, Hq * d, generator=g, dtype=torch.float64)
        wk = torch.randn(hidden, Hkv * d, generator=g, dtype=torch.float64)
        wv = torch.randn(hidden, Hkv * d, generator=g, dtype=torch.float64)
        wo = torch.randn(Hq * d, hidden, generator=g, dtype=torch.float64)
        xs = torch.randn(world, T, hidden, generator=g, dtype=torch.float64)
        os_ = torch.randn(world, T, Hq * d, generator=g, dtype=torch.float64)
        x, o = xs[rank], os_[rank]
        nq, nk, nv = zd.qkv_columns(Hq, Hkv, d, world)
        q = torch.zeros(T, Hq * d, dtype=torch.float64)
        k = torch.zeros(T, Hkv * d, dtype=torch.float64)
        v = torch.zeros(T, Hkv * d, dtype=torch.float64)

        def qkv_step(s, w_s):      # the oracle in place of the GPU GEMM
            y = torch.from_numpy(oracle.project(x, w_s))
            q[:, s * nq:(s + 1) * nq] = y[:, :nq]
            k[:, s * nk:(s + 1) * nk] = y[:, nq:nq + nk]
            v[:, s * nv:(s + 1) * nv] = y[:, nq + nk:]

        zd.tsp_qkv_projection(x, zd.pack_qkv_shard(wq, wk, wv, rank, world), q, k, v, Hq,
                              Hkv, d, project=qkv_step)
        y32 = torch.empty(T, hidden, dtype=torch.float64)

        def out_step(s, w_s):
            y32.add_(torch.from_numpy(oracle.project(o[:, s * nq:(s + 1) * nq], w_s)))

        zd.tsp_out_projection(o, zd.wo_shard(wo, rank, world), y32, Hq, d, project=out_step)
        errs = [float((q - x @ wq).abs().max()), float((k - x @ wk).abs().max()),
                float((v - x @ wv).abs().max()), float((y32 - o @ wo).abs().max())]
        out[rank] = errs
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_broadcast_schedule_equals_unsharded_projections(world):
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert max(out[r]) <= 1e-10, out[r]


def test_tsp_project_argument_errors():
    build.build()
    L = zsa.lib()
    seg = (zsa.zsa_proj_segment * 1)(zsa.zsa_proj_segment(16, 256, 256, 0))
    sp = ctypes.cast(seg, ctypes.c_void_p)

    def rc(T=256, K=128, N=256, x=16, ldx=128, w=16, ldw=256, segs=sp, n=1, ws=256):
        return L.zsa_tsp_project(T, K, N, x, ldx, w, ldw, segs, n, ws, None)
    assert rc(N=250) == zsa.ZSA_ERR_SHAPE          # N % 32
    assert rc(K=100) == zsa.ZSA_ERR_SHAPE          # K % 8
    assert rc(x=None) == zsa.ZSA_ERR_INVALID
    assert rc(x=24) == zsa.ZSA_ERR_INVALID         # misaligned
    assert rc(ldx=100) == zsa.ZSA_ERR_INVALID      # ldx < K
    assert rc(ws=272) == zsa.ZSA_ERR_INVALID       # status workspace alignment
    assert rc(n=0) == zsa.ZSA_ERR_INVALID
    assert rc(N=384) == zsa.ZSA_ERR_INVALID        # segments do not cover N
    bad = (zsa.zsa_proj_segment * 1)(zsa.zsa_proj_segment(16, 256, 250, 0))
    assert rc(segs=ctypes.cast(bad, ctypes.c_void_p)) == zsa.ZSA_ERR_INVALID   # cols % 32
