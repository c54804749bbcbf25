"""The allocation-free backward entry point (zsa_attn_bwd_noalloc).

Some callers cannot allocate device memory where they call the backward (a plugin
inside a host runtime that owns and pre-plans all device memory, a C caller without
an allocator): zsa_attn_bwd_noalloc runs the same backward with a fixed static
scratch.  This file checks, through the C ABI, that two calls in a row give the same
dQ/dK/dV as zsa_attn_bwd with a caller workspace, within the backward's parity
tolerance (relative Frobenius 1e-2); that a problem too large for the scratch is
refused before anything runs; and that the wait limit and stall hook reach this entry
point, with a timeout reported by zsa_noalloc_status.  It is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import inputs

REL_TOL = 1e-2


def rel_fro(x, ref):
    x, ref = x.float().cpu().numpy(), ref.float().cpu().numpy()
    return float(np.linalg.norm(x - ref) / np.linalg.norm(ref))


def test_noalloc_rejects_oversized_problem_on_cpu():
    # S*Hq*(d+1)*4 bytes of scratch far beyond 64 MiB: refused before any CUDA call
    L = zsa.lib()
    big = zsa.make_problem(1, 131072, 32, 8, 128, 16)
    rc = L.zsa_attn_bwd_noalloc(ctypes.byref(big), *([16] * 9), None)
    assert rc == zsa.ZSA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_twice():
    B, S, Hq, Hkv, d, D = 1, 2048, 4, 2, 128, 4
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 51)
    perm = zsa.zsa_partition(zsa.make_problem(B, S, Hq, Hkv, d, D), want_schedule=False)["perm"]
    dev = torch.device("cuda", 0)
    q = inputs.to_shard_major(q_nat, perm, D).to(dev)
    do = inputs.to_shard_major(do_nat, perm, D).to(dev)
    k, v = k.to(dev), v.to(dev)
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    assert zsa.zsa_workspace_bytes(problem, 1) <= zsa.ZSA_NOALLOC_SCRATCH_BYTES
    o, lse = zsa.attn_fwd(q, k, v, D)
    ref = zsa.attn_bwd(q, k, v, o, lse, do, D)          # existing entry point, with workspace
    L = zsa.lib()
    for _ in range(2):                                   # two calls in a row share the scratch
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        stream = torch.cuda.current_stream(dev).cuda_stream
        rc = L.zsa_attn_bwd_noalloc(ctypes.byref(problem), q.data_ptr(), k.data_ptr(),
                                    v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                                    dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), stream)
        assert rc == zsa.ZSA_OK, zsa.status_string(rc)
        torch.cuda.synchronize(dev)
        for got, want in zip((dq, dk, dv), ref):
            assert torch.isfinite(got.float()).all()
            assert rel_fro(got, want) <= REL_TOL


@pytest.mark.gpu
def test_noalloc_timeout_is_reported_and_next_call_is_clean():
    # The stall hook makes the MMA threads wait on a barrier nothing arrives at; with a
    # 20 ms limit that wait gives up, the kernel tears down and records a timeout in the
    # status word inside the static scratch.  zsa_noalloc_status reports and clears it.
    B, S, Hq, Hkv, d, D = 1, 1024, 4, 2, 128, 2
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, 52)
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    perm = zsa.zsa_partition(problem, want_schedule=False)["perm"]
    dev = torch.device("cuda", 0)
    q = inputs.to_shard_major(q_nat, perm, D).to(dev)
    do = inputs.to_shard_major(do_nat, perm, D).to(dev)
    k, v = k.to(dev), v.to(dev)
    o, lse = zsa.attn_fwd(q, k, v, D)
    ref = zsa.attn_bwd(q, k, v, o, lse, do, D)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    assert zsa.zsa_noalloc_status() == zsa.ZSA_OK
    try:
        zsa.zsa_set_wait_limit_ns(20_000_000)
        zsa.zsa_debug_inject_stall(True)
        zsa.zsa_attn_bwd_noalloc(problem, q, k, v, o, lse, do, dq, dk, dv)
        assert zsa.zsa_noalloc_status() == zsa.ZSA_ERR_TIMEOUT
    finally:
        zsa.zsa_debug_inject_stall(False)
        zsa.zsa_set_wait_limit_ns(2_000_000_000)
    assert zsa.zsa_noalloc_status() == zsa.ZSA_OK        # read-and-clear
    zsa.zsa_attn_bwd_noalloc(problem, q, k, v, o, lse, do, dq, dk, dv)
    assert zsa.zsa_noalloc_status() == zsa.ZSA_OK
    for got, want in zip((dq, dk, dv), ref):
        assert rel_fro(got, want) <= REL_TOL
