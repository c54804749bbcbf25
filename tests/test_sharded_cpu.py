"""The D-GPU realisation's host logic, on CPU.

- zsa_partition restricted to a shard range lists exactly the units the full schedule
  has for those shards, in the same order (bit-exact against the oracle's schedule);
- argument errors for the new problem fields;
- gloo ranks (world 2 and 4) run sequence_sharded_causal_b200.dist's collectives on CPU
  tensors: the all-gather of each rank's own K/V rows yields the whole sequence in the
  shard-major order the kernels read, and the reduce-scatter of every rank's partial
  dK / dV (here computed by the fp64 oracle from the rank's own queries, in place of the
  GPU kernels) hands each rank exactly the oracle's dK / dV rows it owns.
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
from sequence_sharded_causal_b200 import build, inputs
from sequence_sharded_causal_b200 import dist as zdist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return zsa.lib()


CONFIGS = [  # (B, S, Hq, Hkv, d, D): the five benchmark shapes
    (1, 256, 2, 2, 64, 2), (1, 16384, 32, 32, 128, 8), (1, 32768, 32, 8, 128, 8),
    (1, 65536, 24, 4, 256, 4), (1, 131072, 32, 8, 128, 16)]


@pytest.mark.parametrize("cfg", CONFIGS)
@pytest.mark.parametrize("world", [1, 2, 4])
def test_rank_units_are_the_full_schedules_units_of_its_shards(L, oracle, cfg, world):
    B, S, Hq, Hkv, d, D = cfg
    if D % world:
        pytest.skip("ranks must divide D")
    full = zsa.zsa_partition(zsa.make_problem(B, S, Hq, Hkv, d, D))
    bq, bk, slots = full["tiling"]
    _, units = oracle.schedule(S, D, B, Hq, Hkv, True, bq, bk, slots)
    seen = []
    for rank in range(world):
        s0, ns = zdist.shard_range(rank, world, D)
        got = zsa.zsa_partition(zsa.make_problem(B, S, Hq, Hkv, d, D, shard_begin=s0,
                                                 shard_count=ns))
        mine = units[(units[:, 0] >= s0) & (units[:, 0] < s0 + ns)]
        assert np.array_equal(got["sched"], mine)
        assert np.array_equal(got["perm"], full["perm"])
        seen.append(got["sched"])
    # every unit of the full schedule belongs to exactly one rank
    assert sum(len(x) for x in seen) == len(units)


def test_shard_field_errors(L):
    def rc(**kw):
        p = zsa.make_problem(1, 1024, 4, 2, 128, 4, **kw)
        out = ctypes.c_size_t(0)
        return L.zsa_workspace_bytes(ctypes.byref(p), 0, ctypes.byref(out))
    assert rc() == zsa.ZSA_OK
    assert rc(shard_begin=1, shard_count=2) == zsa.ZSA_OK
    assert rc(kv_layout=zsa.ZSA_KV_SHARD_MAJOR) == zsa.ZSA_OK
    assert rc(kv_layout=2) == zsa.ZSA_ERR_INVALID
    assert rc(shard_begin=3, shard_count=2) == zsa.ZSA_ERR_INVALID    # past D
    assert rc(shard_begin=-1, shard_count=1) == zsa.ZSA_ERR_INVALID
    assert rc(shard_begin=1, shard_count=0) == zsa.ZSA_ERR_INVALID    # 0 means all D
    assert rc(shard_count=-2) == zsa.ZSA_ERR_INVALID
    # the workspaces shrink with the shard range
    p_all = zsa.make_problem(1, 1024, 4, 2, 128, 4)
    p_one = zsa.make_problem(1, 1024, 4, 2, 128, 4, shard_begin=2, shard_count=1)
    assert zsa.zsa_workspace_bytes(p_one, 1) < zsa.zsa_workspace_bytes(p_all, 1)
    with pytest.raises(ValueError):
        zdist.shard_range(0, 3, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPE = dict(B=1, S=512, Hq=4, Hkv=2, d=16, D=4)


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import oracle
    from sequence_sharded_causal_b200 import dist as zd
    from sequence_sharded_causal_b200 import inputs as inp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, S, Hq, Hkv, d, D = (SHAPE[k] for k in ("B", "S", "Hq", "Hkv", "d", "D"))
        q_nat, k_nat, v_nat, do_nat, _ = inp.make_inputs(B, S, Hq, Hkv, d, 7)
        perm, _ = oracle.partition(S, D)
        s0, ns = zd.shard_range(rank, world, D)
        # what the rank holds: its own rows of Q, dO, K, V (shard-major)
        q_all = inp.to_shard_major(q_nat, perm, D)
        do_all = inp.to_shard_major(do_nat, perm, D)
        k_sm = inp.to_shard_major(k_nat, perm, D)
        v_sm = inp.to_shard_major(v_nat, perm, D)
        k_all, v_all = zd.gather_kv(k_sm[s0:s0 + ns].clone(), v_sm[s0:s0 + ns].clone())
        gathered_ok = bool(torch.equal(k_all, k_sm) and torch.equal(v_all, v_sm))
        # the rank's partial dK/dV from its own queries (other shards' dO set to 0: their
        # rows then add nothing), computed by the oracle in place of the GPU backward
        do_mine = torch.zeros_like(do_all)
        do_mine[s0:s0 + ns] = do_all[s0:s0 + ns]
        k_g = inp.from_shard_major(k_all, perm)
        v_g = inp.from_shard_major(v_all, perm)
        part = oracle.attn_bwd(q_all, k_g, v_g, do_mine, D)
        dk_part = inp.to_shard_major(torch.from_numpy(part["dk"]), perm, D)
        dv_part = inp.to_shard_major(torch.from_numpy(part["dv"]), perm, D)
        dk_mine, dv_mine = zd.reduce_scatter_kv_grads(dk_part, dv_part)
        full = oracle.attn_bwd(q_all, k_nat, v_nat, do_all, D)
        dk_ref = inp.to_shard_major(torch.from_numpy(full["dk"]), perm, D)[s0:s0 + ns]
        dv_ref = inp.to_shard_major(torch.from_numpy(full["dv"]), perm, D)[s0:s0 + ns]
        err = max(float((dk_mine - dk_ref).abs().max()), float((dv_mine - dv_ref).abs().max()))
        # the rank's dQ rows do not depend on other ranks' queries
        dq_err = float(np.abs(part["dq"][s0:s0 + ns] - full["dq"][s0:s0 + ns]).max())
        out[rank] = (gathered_ok, err, dq_err, tuple(dk_mine.shape))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_gather_and_reduce_scatter_index_maps(world):
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    D, twoC = SHAPE["D"], SHAPE["S"] // SHAPE["D"]
    for r in range(world):
        gathered_ok, err, dq_err, shape = out[r]
        assert gathered_ok
        assert err <= 1e-12, err
        assert dq_err <= 1e-12, dq_err
        assert shape == (D // world, SHAPE["B"], twoC, SHAPE["Hkv"], SHAPE["d"])


def test_shard_major_kv_rows_match_the_zigzag_map(L, oracle):
    # the Q layout's zigzag rows applied to K is what the kernels read as shard-major K:
    # row r*2C + j of the shard-major tensor holds position perm[r*2C + j]
    S, D = 1024, 4
    perm, inv = oracle.partition(S, D)
    k = torch.arange(S, dtype=torch.float32).reshape(1, S, 1, 1)
    sm = inputs.to_shard_major(k, perm, D)          # [D][1][2C][1][1]
    assert np.array_equal(sm.reshape(-1).numpy().astype(np.int64), perm.astype(np.int64))
    assert np.array_equal(inputs.from_shard_major(sm, perm).reshape(-1).numpy(),
                          np.arange(S, dtype=np.float32))
