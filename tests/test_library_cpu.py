"""Host-side checks of libzsa that need no GPU.

- the library loads and exports every entry point include/zsa.h declares;
- zsa_partition (zigzag map, per-shard tile work, unit schedule) equals the oracle's
  independently written partition and schedule, bit for bit, over a sweep of shapes
  and tilings including the five benchmark configurations;
- argument errors come back as the documented status codes before anything touches
  a device.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import sequence_sharded_causal_b200 as zsa
from sequence_sharded_causal_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return zsa.lib()


def test_exports_every_declared_symbol(L):
    header = open(os.path.join(ROOT, "include", "zsa.h")).read()
    declared = set(re.findall(r"^\s*ZSA_API\s+(?:int|const char\*)\s+(zsa_\w+)\s*\(", header, re.M))
    assert declared == set(zsa.EXPORTED), declared
    for name in declared:
        assert hasattr(L, name), name
    assert zsa.status_string(zsa.ZSA_ERR_TIMEOUT).startswith("a bounded")


CONFIGS = [  # (B, S, Hq, Hkv, d, D): the five benchmark shapes
    (1, 256, 2, 2, 64, 2), (1, 16384, 32, 32, 128, 8), (1, 32768, 32, 8, 128, 8),
    (1, 65536, 24, 4, 256, 4), (1, 131072, 32, 8, 128, 16)]


@pytest.mark.parametrize("cfg", CONFIGS)
def test_partition_matches_oracle_on_configs(L, oracle, cfg):
    B, S, Hq, Hkv, d, D = cfg
    p = zsa.make_problem(B, S, Hq, Hkv, d, D)
    got = zsa.zsa_partition(p)
    perm, inv = oracle.partition(S, D)
    assert np.array_equal(got["perm"], perm)
    assert np.array_equal(got["inv_perm"], inv)
    bq, bk, slots = got["tiling"]
    st, units = oracle.schedule(S, D, B, Hq, Hkv, True, bq, bk, slots)
    assert np.array_equal(got["shard_tiles"], st)
    assert np.array_equal(got["sched"], units)
    assert len(set(got["shard_tiles"].tolist())) == 1


SWEEP = [(S, D, B, Hq, Hkv, bq, bk, slots, causal)
         for (S, D) in ((256, 2), (512, 1), (768, 2), (1536, 4), (2560, 5), (4096, 8))
         for (B, Hq, Hkv) in ((1, 2, 2), (2, 6, 2), (1, 3, 1), (1, 8, 8))
         for (bq, bk) in ((128, 128), (128, 64), (64, 64))
         for slots in (1, 2) for causal in (0, 1)
         if (S // D) % bq == 0]


@pytest.mark.parametrize("S,D,B,Hq,Hkv,bq,bk,slots,causal", SWEEP[::3])
def test_schedule_sweep_bit_exact(L, oracle, S, D, B, Hq, Hkv, bq, bk, slots, causal):
    p = zsa.make_problem(B, S, Hq, Hkv, 128, D, causal)
    got = zsa.zsa_partition(p, bq, bk, slots)
    st, units = oracle.schedule(S, D, B, Hq, Hkv, bool(causal), bq, bk, slots)
    assert np.array_equal(got["shard_tiles"], st)
    assert np.array_equal(got["sched"], units)


def _rc_fwd(L, problem, ptrs=(16,) * 5, ws=256, ws_bytes=1 << 30):
    return L.zsa_attn_fwd(ctypes.byref(problem), *ptrs, ws, ws_bytes, None)


def test_argument_errors(L):
    good = zsa.make_problem(1, 1024, 4, 2, 128, 2)
    assert _rc_fwd(L, good, ptrs=(None, 16, 16, 16, 16)) == zsa.ZSA_ERR_INVALID
    assert _rc_fwd(L, good, ptrs=(24, 16, 16, 16, 16)) == zsa.ZSA_ERR_INVALID   # misaligned
    assert _rc_fwd(L, good, ws=272) == zsa.ZSA_ERR_INVALID                        # ws not 256-aligned
    assert _rc_fwd(L, zsa.make_problem(1, 1024, 4, 3, 128, 2)) == zsa.ZSA_ERR_SHAPE   # Hq % Hkv
    assert _rc_fwd(L, zsa.make_problem(1, 1000, 4, 2, 128, 2)) == zsa.ZSA_ERR_SHAPE   # S % 2D*64
    assert _rc_fwd(L, zsa.make_problem(1, 768, 4, 2, 128, 4)) == zsa.ZSA_ERR_SHAPE
    assert _rc_fwd(L, zsa.make_problem(1, 1024, 4, 2, 96, 2)) == zsa.ZSA_ERR_UNSUPPORTED
    assert _rc_fwd(L, zsa.make_problem(0, 1024, 4, 2, 128, 2)) == zsa.ZSA_ERR_INVALID
    assert _rc_fwd(L, zsa.make_problem(1, 1024, 4, 2, 128, 2, scale=-1.0)) == zsa.ZSA_ERR_INVALID
    assert _rc_fwd(L, good, ws_bytes=64) == zsa.ZSA_ERR_WORKSPACE
    assert L.zsa_attn_fwd(None, 16, 16, 16, 16, 16, 256, 1 << 30, None) == zsa.ZSA_ERR_INVALID
    bw = [16] * 9
    assert L.zsa_attn_bwd(ctypes.byref(good), *bw, 256, 64, None) == zsa.ZSA_ERR_WORKSPACE
    bw[3] = None
    assert L.zsa_attn_bwd(ctypes.byref(good), *bw, 256, 1 << 40, None) == zsa.ZSA_ERR_INVALID
    out = ctypes.c_size_t(0)
    assert L.zsa_workspace_bytes(ctypes.byref(good), 2, ctypes.byref(out)) == zsa.ZSA_ERR_INVALID
    assert L.zsa_workspace_bytes(ctypes.byref(good), 1, ctypes.byref(out)) == zsa.ZSA_OK
    assert out.value >= 1024 * 4 * (128 + 1) * 4
    n = ctypes.c_int64(0)
    t = zsa.zsa_tiling(0, 0, 0)
    sched = (zsa.zsa_work * 1)()
    rc = L.zsa_partition(ctypes.byref(good), ctypes.byref(t), None, None, None,
                         ctypes.cast(sched, ctypes.c_void_p), 1, ctypes.byref(n))
    assert rc == zsa.ZSA_ERR_WORKSPACE and n.value > 1
    assert (t.block_q, t.block_k, t.slots) == (128, 128, 2)


def test_size_limits(L):
    # key-tile counts are packed in 16 bits: S / 128 must stay below 65536
    assert _rc_fwd(L, zsa.make_problem(1, 65536 * 128, 4, 2, 128, 1)) == zsa.ZSA_ERR_SHAPE
    assert _rc_fwd(L, zsa.make_problem(1, 65535 * 128, 4, 2, 128, 1), ws_bytes=64) == zsa.ZSA_ERR_WORKSPACE
    # B * S < 2^31: TMA row coordinates are int32
    assert _rc_fwd(L, zsa.make_problem(2 ** 15, 2 ** 16, 4, 2, 128, 2)) == zsa.ZSA_ERR_SHAPE
    assert _rc_fwd(L, zsa.make_problem(2 ** 14, 2 ** 16, 4, 2, 128, 2), ws_bytes=64) == zsa.ZSA_ERR_WORKSPACE
    # the merge indexes rows * Hq * d in 32 bits
    big = zsa.make_problem(1, 2 ** 20, 32, 8, 128, 16)          # 2^20 * 32 * 128 = 2^32
    parts = (ctypes.c_void_p * 2)(16, 16)
    lses = (ctypes.c_void_p * 2)(16, 16)
    assert L.zsa_attn_merge(ctypes.byref(big), 2, parts, lses, 16, 16, None) == zsa.ZSA_ERR_SHAPE
    ok = zsa.make_problem(1, 2 ** 18, 32, 8, 128, 16)            # 2^30: below the limit
    assert L.zsa_attn_merge(ctypes.byref(ok), 2, parts, lses, 16, 16, None) not in (
        zsa.ZSA_ERR_SHAPE, zsa.ZSA_ERR_INVALID)
    assert L.zsa_attn_merge(ctypes.byref(ok), 0, parts, lses, 16, 16, None) == zsa.ZSA_ERR_INVALID
    assert L.zsa_attn_merge(ctypes.byref(ok), zsa.ZSA_MERGE_MAX_PARTS + 1, parts, lses, 16, 16,
                            None) == zsa.ZSA_ERR_INVALID


def test_permute_argument_errors(L):
    good = zsa.make_problem(2, 1024, 4, 2, 128, 2)
    P = ctypes.byref(good)
    n = 2 * 1024 * 4 * 128 * 2                      # bytes of a [B][S][4][d] bf16 tensor
    assert L.zsa_permute(P, 4, 1, 16, 16, None) == zsa.ZSA_ERR_INVALID          # overlap
    assert L.zsa_permute(P, 4, 1, 16, 16 + n - 16, None) == zsa.ZSA_ERR_INVALID
    # a shard range: the shard-major side is that range's rows only
    one = zsa.make_problem(2, 1024, 4, 2, 128, 2, shard_begin=1, shard_count=1)
    P1 = ctypes.byref(one)
    assert L.zsa_permute(P1, 4, 1, 16 + n // 2 - 16, 16, None) == zsa.ZSA_ERR_INVALID
    assert L.zsa_permute(P1, 4, 0, 16, 16 + n // 2 - 16, None) == zsa.ZSA_ERR_INVALID
    # adjacent, not overlapping: passes the argument checks (then fails for want of a GPU)
    assert L.zsa_permute(P1, 4, 1, 16 + n // 2, 16, None) not in (zsa.ZSA_OK, zsa.ZSA_ERR_INVALID)
    assert L.zsa_permute(P1, 4, 0, 16, 16 + n // 2, None) not in (zsa.ZSA_OK, zsa.ZSA_ERR_INVALID)
    assert L.zsa_permute(P, 4, 1, 16, 24 + n, None) == zsa.ZSA_ERR_INVALID       # misaligned
    assert L.zsa_permute(P, 0, 1, 16, 16 + n, None) == zsa.ZSA_ERR_INVALID       # heads
    assert L.zsa_permute(P, 4, 2, 16, 16 + n, None) == zsa.ZSA_ERR_INVALID       # direction
    assert L.zsa_permute(P, 4, 1, None, 16 + n, None) == zsa.ZSA_ERR_INVALID
    assert L.zsa_permute(None, 4, 1, 16, 16 + n, None) == zsa.ZSA_ERR_INVALID
    bad = zsa.make_problem(1, 1000, 4, 2, 128, 2)
    assert L.zsa_permute(ctypes.byref(bad), 4, 1, 16, 16 + n, None) == zsa.ZSA_ERR_SHAPE
    big = zsa.make_problem(40000, 1024, 4, 2, 128, 2)
    assert L.zsa_permute(ctypes.byref(big), 1, 1, 16, 1 << 40, None) == zsa.ZSA_ERR_SHAPE


def test_key_block_argument_errors(L):
    # B = 2, S = 1024: a compact block of keys [100, 612) needs 2 * 512 rows
    good = zsa.make_problem(2, 1024, 4, 2, 128, 2)

    def rc(lo, hi, rpb, off, rows, ws_bytes=64):
        kb = zsa.zsa_key_block(lo, hi, rpb, off, rows)
        return L.zsa_attn_fwd_block(ctypes.byref(good), ctypes.byref(kb), *((16,) * 5), 256,
                                    ws_bytes, None)

    assert rc(100, 612, 512, 0, 1024) == zsa.ZSA_ERR_WORKSPACE      # valid: reaches the size check
    assert rc(0, 0, 0, 0, 1) == zsa.ZSA_ERR_WORKSPACE               # an empty block is valid
    assert rc(100, 612, 512, 0, 1023) == zsa.ZSA_ERR_INVALID        # last row outside the tensor
    assert rc(100, 612, 511, 0, 4096) == zsa.ZSA_ERR_INVALID        # batches overlap
    assert rc(612, 100, 512, 0, 1024) == zsa.ZSA_ERR_INVALID        # hi < lo
    assert rc(-1, 100, 512, 0, 1024) == zsa.ZSA_ERR_INVALID
    assert rc(0, 1025, 1025, 0, 4096) == zsa.ZSA_ERR_INVALID        # past S
    assert rc(0, 100, 100, -1, 1024) == zsa.ZSA_ERR_INVALID
    assert rc(0, 100, 100, 0, 1 << 31) == zsa.ZSA_ERR_INVALID       # int32 TMA coordinates
    assert L.zsa_attn_fwd_block(ctypes.byref(good), None, *((16,) * 5), 256, 1 << 30,
                                None) == zsa.ZSA_ERR_INVALID
