"""fp64 CPU oracle for zigzag-sharded causal (GQA) attention.

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import this package; the product path (the
CUDA library and its binding) never does.  It shares no code with the CUDA path.

The arithmetic lives in oracle.c (plain fp64 loops, OpenMP over rows); this module
only marshals numpy arrays.  Sources followed:
  * "Folding Tensor and Sequence Parallelism" (gist.science 2604.26294), section 2,
    attention-layer schedule: all-gathered K/V, FlashAttention, zigzag partition.
  * "AutoSP" (gist.science 2604.27089), section 2.A, step 4: causal masks are
    recomputed in global positions under sequence sharding.
  * "Tensor, pipeline e sequence parallelism" (llmdeepdive 5.8), "01 Conceito":
    grouped-query heads (q heads share kv heads).
  * "AutoSP" (gist.science 2604.27089), sections 1 and 4: ring attention, the
    sequence-parallel baseline whose per-block partial results attn_fwd_keys computes
    and attn_merge combines (log-sum-exp merge; the reading is stated in oracle.c).

Every function here is pinned by tests/test_oracle_pins.py (brute force, closed
forms, finite differences, invariants); none is "parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        p = ctypes.c_void_p
        lib.oracle_partition.argtypes = [i64, i32, p, p]
        lib.oracle_partition.restype = ctypes.c_int
        lib.oracle_schedule.argtypes = [i64, i32, i32, i32, i32, i32, i32, i32, i32, p, p, i64]
        lib.oracle_schedule.restype = i64
        lib.oracle_attn_fwd.argtypes = [i32, i64, i32, i32, i32, i32, i32, dbl, p, p, p, p, p]
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_fwd_rows.argtypes = [i32, i64, i32, i32, i32, i32, i32, dbl, p, i64,
                                             p, p, p, p, p]
        lib.oracle_attn_fwd_rows.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [i32, i64, i32, i32, i32, i32, i32, dbl] + [p] * 10
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_dq_rows.argtypes = [i32, i64, i32, i32, i32, i32, i32, dbl, p, i64,
                                            p, p, p, p, p]
        lib.oracle_attn_dq_rows.restype = ctypes.c_int
        lib.oracle_attn_fwd_keys.argtypes = [i32, i64, i32, i32, i32, i32, i32, dbl, i64, i64,
                                             p, p, p, p, p]
        lib.oracle_attn_fwd_keys.restype = ctypes.c_int
        lib.oracle_attn_merge.argtypes = [i32, i64, i32, p, p, p, p]
        lib.oracle_attn_merge.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    """Exact widening to a C-contiguous float64 array (bf16/f32 -> f64 is exact)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return np.ascontiguousarray(a.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def partition(S, D):
    """Zigzag map: (perm, inv_perm), int32 [S] each.

    perm[r*2C + j] is the global position of row j of shard r; inv_perm inverts it.
    """
    perm = np.empty(S, np.int32)
    inv = np.empty(S, np.int32)
    if _load().oracle_partition(S, D, _ptr(perm), _ptr(inv)) != 0:
        raise ValueError(f"invalid partition S={S} D={D}")
    return perm, inv


def schedule(S, D, B, Hq, Hkv, causal=True, block_q=128, block_k=128, slots=2):
    """(shard_tiles int64 [D], units int32 [n][9]) of the tile schedule.

    unit row: r, b, g, tile0, head0, tile1, head1, kend0, kend1 (absent slot: -1,-1,0).
    """
    lib = _load()
    st = np.empty(D, np.int64)
    n = lib.oracle_schedule(S, D, B, Hq, Hkv, int(bool(causal)), block_q, block_k, slots,
                            _ptr(st), None, 0)
    if n < 0:
        raise ValueError("invalid tiling")
    units = np.empty((n, 9), np.int32)
    lib.oracle_schedule(S, D, B, Hq, Hkv, int(bool(causal)), block_q, block_k, slots,
                        _ptr(st), _ptr(units), n)
    return st, units


def attn_fwd(q, k, v, D, causal=True, scale=None):
    """Full forward.  q [D][B][2C][Hq][d] (shard-major), k/v [B][S][Hkv][d].

    Returns (o [D][B][2C][Hq][d], lse [D][B][Hq][2C]) in float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    Dq, B, twoC, Hq, d = q.shape
    assert Dq == D
    Bk, S, Hkv, dk = k.shape
    assert Bk == B and dk == d and S == D * twoC and v.shape == k.shape
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    o = np.empty_like(q)
    lse = np.empty((D, B, Hq, twoC), np.float64)
    rc = _load().oracle_attn_fwd(B, S, Hq, Hkv, d, D, int(bool(causal)), float(scale),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_fwd: invalid problem")
    return o, lse


def attn_fwd_rows(q_rows, rows, k, v, D, Hq, causal=True, scale=None):
    """Forward of selected shard-major rows.

    rows: int64 [n] flattened (r*B + b)*2C + j; q_rows: [n][Hq][d].
    Returns (o_rows [n][Hq][d], lse_rows [n][Hq]) in float64.
    """
    q_rows, k, v = _f64(q_rows), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    n = rows.shape[0]
    B, S, Hkv, d = k.shape
    assert q_rows.shape == (n, Hq, d)
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    o = np.empty((n, Hq, d), np.float64)
    lse = np.empty((n, Hq), np.float64)
    rc = _load().oracle_attn_fwd_rows(B, S, Hq, Hkv, d, D, int(bool(causal)), float(scale),
                                      _ptr(rows), n, _ptr(q_rows), _ptr(k), _ptr(v), _ptr(o),
                                      _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_fwd_rows: invalid problem")
    return o, lse


def attn_dq_rows(q_rows, do_rows, rows, k, v, D, Hq, causal=True, scale=None):
    """dQ of selected shard-major rows (rows as in attn_fwd_rows). Returns [n][Hq][d]."""
    q_rows, do_rows, k, v = _f64(q_rows), _f64(do_rows), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    n = rows.shape[0]
    B, S, Hkv, d = k.shape
    assert q_rows.shape == (n, Hq, d) and do_rows.shape == (n, Hq, d)
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    dq = np.empty((n, Hq, d), np.float64)
    rc = _load().oracle_attn_dq_rows(B, S, Hq, Hkv, d, D, int(bool(causal)), float(scale),
                                     _ptr(rows), n, _ptr(q_rows), _ptr(do_rows), _ptr(k), _ptr(v),
                                     _ptr(dq))
    if rc != 0:
        raise ValueError("oracle_attn_dq_rows: invalid problem")
    return dq


def attn_bwd(q, k, v, dout, D, causal=True, scale=None):
    """Full backward of L = <dout, O>.

    Returns dict of float64 arrays: dq, dk, dv, o, lse, delta.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    Dq, B, twoC, Hq, d = q.shape
    Bk, S, Hkv, _ = k.shape
    assert Dq == D and S == D * twoC and dout.shape == q.shape
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    o = np.empty_like(q)
    lse = np.empty((D, B, Hq, twoC), np.float64)
    delta = np.empty_like(lse)
    rc = _load().oracle_attn_bwd(B, S, Hq, Hkv, d, D, int(bool(causal)), float(scale),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                 _ptr(dv), _ptr(o), _ptr(lse), _ptr(delta))
    if rc != 0:
        raise ValueError("oracle_attn_bwd: invalid problem")
    return dict(dq=dq, dk=dk, dv=dv, o=o, lse=lse, delta=delta)


def attn_fwd_keys(q, k, v, D, key_lo, key_hi, causal=True, scale=None):
    """Forward restricted to the keys at positions [key_lo, key_hi) (and k <= p when
    causal).  Layouts as attn_fwd; rows seeing no key get lse = -inf, O = 0."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Dq, B, twoC, Hq, d = q.shape
    Bk, S, Hkv, dk = k.shape
    assert Dq == D and Bk == B and dk == d and S == D * twoC and v.shape == k.shape
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    o = np.empty_like(q)
    lse = np.empty((D, B, Hq, twoC), np.float64)
    rc = _load().oracle_attn_fwd_keys(B, S, Hq, Hkv, d, D, int(bool(causal)), float(scale),
                                      int(key_lo), int(key_hi), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_fwd_keys: invalid problem or key range")
    return o, lse


def attn_merge(o_parts, lse_parts):
    """Merge partial results over disjoint key sets.

    o_parts: list of Q-layout arrays [D'][B][2C][Hq][d]; lse_parts: matching lists of
    [D'][B][Hq][2C].  Returns (o, lse) in the same layouts, float64.
    """
    o_parts = [_f64(x) for x in o_parts]
    lse_parts = [_f64(x) for x in lse_parts]
    n = len(o_parts)
    Dq, B, twoC, Hq, d = o_parts[0].shape
    m = Dq * B * twoC * Hq
    # lse [D'][B][Hq][2C] -> the O layout's pair order [D'][B][2C][Hq]
    lse_pairs = np.ascontiguousarray(np.stack([x.transpose(0, 1, 3, 2) for x in lse_parts]))
    o_stack = np.ascontiguousarray(np.stack(o_parts))
    o = np.empty((Dq, B, twoC, Hq, d), np.float64)
    lse_flat = np.empty((Dq, B, twoC, Hq), np.float64)
    rc = _load().oracle_attn_merge(n, m, d, _ptr(o_stack), _ptr(lse_pairs), _ptr(o),
                                   _ptr(lse_flat))
    if rc != 0:
        raise ValueError("oracle_attn_merge: invalid arguments")
    return o, np.ascontiguousarray(lse_flat.transpose(0, 1, 3, 2))


def project(x, w):
    """One local projection of the TSP attention-layer schedule, Y = X W, in fp64 from the
    (bf16) input values.  "Folding Tensor and Sequence Parallelism" summary, section 2,
    attention layer: every broadcast step multiplies the rank's tokens by the shard of
    the packed attention weights it received.  The matmul is a library step."""
    return _f64(x) @ _f64(w)
