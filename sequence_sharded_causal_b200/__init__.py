"""Zigzag-sharded causal (GQA) attention for B200 -- Python binding of libzsa.

The functions named zsa_* mirror the C ABI in include/zsa.h one to one: they only
marshal arguments (tensor data pointers, the current CUDA stream) and turn status
codes into exceptions.  Every step of the computation runs in the library's sm_100a
kernels; there is no CPU or PyTorch fallback: if libzsa.so is missing the calls raise.

attn_fwd / attn_bwd are conveniences that allocate outputs and the workspace through
PyTorch (device memory only) and then call the same entry points.

Layouts (see include/zsa.h): Q, O, dO, dQ are shard-major [D][B][2C][Hq][d]; K, V, dK,
dV are natural-order [B][S][Hkv][d] (kv_layout=ZSA_KV_NATURAL) or shard-major
[D][B][2C][Hkv][d] (ZSA_KV_SHARD_MAJOR); lse is fp32 [D][B][Hq][2C]; tensors are bf16.
A call restricted to the shards [shard_begin, shard_begin + shard_count) takes the
Q-layout tensors of those shards only.
"""
import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzsa.so")

ZSA_OK = 0
ZSA_ERR_INVALID = -1
ZSA_ERR_SHAPE = -2
ZSA_ERR_UNSUPPORTED = -3
ZSA_ERR_WORKSPACE = -4
ZSA_ERR_CUDA = -5
ZSA_ERR_TIMEOUT = -6
ZSA_KV_NATURAL = 0
ZSA_KV_SHARD_MAJOR = 1

EXPORTED = ("zsa_partition", "zsa_workspace_bytes", "zsa_attn_fwd", "zsa_attn_bwd",
            "zsa_device_status", "zsa_set_wait_limit_ns", "zsa_debug_inject_stall",
            "zsa_trace_events", "zsa_attn_merge", "zsa_tsp_project", "zsa_attn_bwd_noalloc",
            "zsa_noalloc_status", "zsa_attn_fwd_block", "zsa_permute", "zsa_status_string")
ZSA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024
(ZSA_TRACE_FWD, ZSA_TRACE_BWD_PRE, ZSA_TRACE_BWD_MAIN, ZSA_TRACE_BWD_DQ, ZSA_TRACE_MERGE,
 ZSA_TRACE_PROJ, ZSA_TRACE_PERMUTE) = range(7)
ZSA_PROJ_MAX_SEGMENTS = 8
ZSA_MERGE_MAX_PARTS = 32


class zsa_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("S", ctypes.c_int64), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("D", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("kv_layout", ctypes.c_int32), ("shard_begin", ctypes.c_int32),
                ("shard_count", ctypes.c_int32)]


class zsa_tiling(ctypes.Structure):
    _fields_ = [("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32), ("slots", ctypes.c_int32)]


class zsa_work(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("shard", "b", "kv_head", "q_tile0", "q_head0",
                                              "q_tile1", "q_head1", "k_tile_end0", "k_tile_end1")]


class zsa_proj_segment(ctypes.Structure):
    _fields_ = [("out", ctypes.c_void_p), ("ld", ctypes.c_int64), ("cols", ctypes.c_int32),
                ("fp32_accumulate", ctypes.c_int32)]


class zsa_key_block(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("key_lo", "key_hi", "rows_per_batch", "row_offset",
                                              "rows")]


class ZsaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib = None


def lib():
    """The loaded libzsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sequence_sharded_causal_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        vp = ctypes.c_void_p
        L.zsa_partition.argtypes = [P(zsa_problem), P(zsa_tiling), vp, vp, vp, vp, ctypes.c_int64,
                                    P(ctypes.c_int64)]
        L.zsa_workspace_bytes.argtypes = [P(zsa_problem), ctypes.c_int, P(ctypes.c_size_t)]
        L.zsa_attn_fwd.argtypes = [P(zsa_problem), vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.zsa_attn_bwd.argtypes = [P(zsa_problem)] + [vp] * 10 + [ctypes.c_size_t, vp]
        L.zsa_device_status.argtypes = [vp, vp]
        L.zsa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.zsa_debug_inject_stall.argtypes = [ctypes.c_int]
        L.zsa_trace_events.argtypes = [ctypes.c_int, vp, vp]
        L.zsa_attn_merge.argtypes = [P(zsa_problem), ctypes.c_int32, vp, vp, vp, vp, vp]
        i64 = ctypes.c_int64
        L.zsa_tsp_project.argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, ctypes.c_int32, vp, vp]
        L.zsa_attn_bwd_noalloc.argtypes = [P(zsa_problem)] + [vp] * 10
        L.zsa_noalloc_status.argtypes = [vp]
        L.zsa_permute.argtypes = [P(zsa_problem), ctypes.c_int32, ctypes.c_int32, vp, vp, vp]
        L.zsa_attn_fwd_block.argtypes = [P(zsa_problem), P(zsa_key_block), vp, vp, vp, vp, vp, vp,
                                         ctypes.c_size_t, vp]
        L.zsa_status_string.argtypes = [ctypes.c_int]
        L.zsa_status_string.restype = ctypes.c_char_p
        for name in EXPORTED[:-1]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status):
    return lib().zsa_status_string(int(status)).decode()


def _check(rc, where):
    if rc != ZSA_OK:
        raise ZsaError(rc, where)


def make_problem(B, S, Hq, Hkv, d, D, causal=True, scale=None, kv_layout=ZSA_KV_NATURAL,
                 shard_begin=0, shard_count=0):
    """zsa_problem; shard_count = 0 means all D shards (one launch)."""
    if scale is None:
        scale = float(np.float32(1.0 / math.sqrt(d)))
    return zsa_problem(int(B), int(S), int(Hq), int(Hkv), int(d), int(D), int(bool(causal)),
                       float(scale), int(kv_layout), int(shard_begin), int(shard_count))


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ C ABI mirrors

def zsa_partition(problem, block_q=0, block_k=0, slots=0, want_schedule=True):
    """Zigzag map + forward schedule (host only).

    Returns dict: perm, inv_perm (int32 [S]), shard_tiles (int64 [D]), sched (int32
    [n][9]: shard, b, kv_head, q_tile0, q_head0, q_tile1, q_head1, k_tile_end0,
    k_tile_end1) and the tiling actually used.
    """
    t = zsa_tiling(block_q, block_k, slots)
    S, D = int(problem.S), int(problem.D)
    perm = np.empty(S, np.int32)
    inv = np.empty(S, np.int32)
    st = np.empty(D, np.int64)
    n = ctypes.c_int64(0)
    _check(lib().zsa_partition(ctypes.byref(problem), ctypes.byref(t), perm.ctypes.data,
                               inv.ctypes.data, st.ctypes.data, None, 0, ctypes.byref(n)),
           "zsa_partition")
    sched = None
    if want_schedule:
        sched = np.empty((n.value, 9), np.int32)
        _check(lib().zsa_partition(ctypes.byref(problem), ctypes.byref(t), None, None, None,
                                   sched.ctypes.data, n.value, ctypes.byref(n)), "zsa_partition")
    return dict(perm=perm, inv_perm=inv, shard_tiles=st, sched=sched,
                tiling=(t.block_q, t.block_k, t.slots))


def zsa_workspace_bytes(problem, pass_):
    out = ctypes.c_size_t(0)
    _check(lib().zsa_workspace_bytes(ctypes.byref(problem), int(pass_), ctypes.byref(out)),
           "zsa_workspace_bytes")
    return out.value


def zsa_attn_fwd(problem, q, k, v, o, lse, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().zsa_attn_fwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                              _ptr(lse), _ptr(workspace), int(ws_bytes), _stream(stream)),
           "zsa_attn_fwd")


def zsa_attn_fwd_block(problem, block, q, k, v, o, lse, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().zsa_attn_fwd_block(ctypes.byref(problem), ctypes.byref(block), _ptr(q), _ptr(k),
                                    _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace), int(ws_bytes),
                                    _stream(stream)), "zsa_attn_fwd_block")


def zsa_permute(problem, heads, to_shard_major, src, dst, stream=None):
    _check(lib().zsa_permute(ctypes.byref(problem), int(heads), int(to_shard_major), _ptr(src),
                             _ptr(dst), _stream(stream)), "zsa_permute")


def zsa_attn_bwd(problem, q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes=None,
                 stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().zsa_attn_bwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                              _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                              _ptr(workspace), int(ws_bytes), _stream(stream)), "zsa_attn_bwd")


def zsa_attn_merge(problem, o_parts, lse_parts, o, lse, stream=None):
    """Merge partial results (O_i bf16 Q layout, lse_i fp32) over disjoint key sets into
    o / lse (which may alias a part)."""
    n = len(o_parts)
    if n != len(lse_parts):
        raise ValueError("o_parts and lse_parts differ in length")
    op = (ctypes.c_void_p * n)(*[_ptr(x) for x in o_parts])
    lp = (ctypes.c_void_p * n)(*[_ptr(x) for x in lse_parts])
    _check(lib().zsa_attn_merge(ctypes.byref(problem), n, ctypes.cast(op, ctypes.c_void_p),
                                ctypes.cast(lp, ctypes.c_void_p), _ptr(o), _ptr(lse),
                                _stream(stream)), "zsa_attn_merge")


def zsa_tsp_project(x, w, segments, status_ws, T=None, K=None, N=None, ldx=None, ldw=None,
                    stream=None):
    """Y = X W for one TSP step, Y's columns routed to `segments`: a list of
    (out, ld, cols, fp32_accumulate), out a tensor / device pointer."""
    if T is None:
        T, K = x.shape[0], x.shape[1]
    if N is None:
        N = w.shape[1]
    ldx = x.stride(0) if ldx is None else ldx
    ldw = w.stride(0) if ldw is None else ldw
    segs = (zsa_proj_segment * len(segments))(
        *[zsa_proj_segment(_ptr(o), int(ld), int(c), int(bool(acc))) for o, ld, c, acc in segments])
    _check(lib().zsa_tsp_project(int(T), int(K), int(N), _ptr(x), int(ldx), _ptr(w), int(ldw),
                                 ctypes.cast(segs, ctypes.c_void_p), len(segments),
                                 _ptr(status_ws), _stream(stream)), "zsa_tsp_project")


def zsa_attn_bwd_noalloc(problem, q, k, v, o, lse, dout, dq, dk, dv, stream=None):
    """zsa_attn_bwd with the library's fixed static scratch instead of a workspace.

    For callers that cannot allocate device memory at the call site (a host runtime
    that owns all device memory, a C caller without an allocator); see include/zsa.h
    for the size limit and the sharing rules.
    """
    _check(lib().zsa_attn_bwd_noalloc(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                      _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                      _stream(stream)), "zsa_attn_bwd_noalloc")


def zsa_noalloc_status(stream=None):
    """Synchronise; status word of the allocation-free backward's scratch (clears it)."""
    return lib().zsa_noalloc_status(_stream(stream))


def zsa_device_status(workspace, stream=None):
    """Synchronise and return the device status word (0 or ZSA_ERR_TIMEOUT); clears it."""
    return lib().zsa_device_status(_ptr(workspace), _stream(stream))


def zsa_set_wait_limit_ns(limit_ns):
    _check(lib().zsa_set_wait_limit_ns(int(limit_ns)), "zsa_set_wait_limit_ns")


def zsa_debug_inject_stall(enable):
    _check(lib().zsa_debug_inject_stall(int(bool(enable))), "zsa_debug_inject_stall")


def zsa_trace_events(which, begin_event=None, end_event=None):
    """Record torch.cuda.Event (or raw cudaEvent_t) pairs around kernel `which`."""
    def raw(e):
        if e is None or isinstance(e, int):
            return e
        if not e.cuda_event:   # torch creates the event lazily on first record
            e.record()
        return e.cuda_event
    _check(lib().zsa_trace_events(int(which), raw(begin_event), raw(end_event)),
           "zsa_trace_events")


def zsa_status_string(status):
    return status_string(status)


# ------------------------------------------------------------------ conveniences

def _check_tensor(x, shape, dtype, name):
    import torch
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(x.shape) != tuple(shape) or x.dtype != dtype or not x.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got "
                         f"{x.dtype} {tuple(x.shape)} contiguous={x.is_contiguous()}")


def _shapes(problem):
    """(Q-layout shape, K/V shape, lse shape) of a problem."""
    B, S, Hq, Hkv, d, D = (int(problem.B), int(problem.S), int(problem.Hq), int(problem.Hkv),
                           int(problem.d), int(problem.D))
    ns = int(problem.shard_count) or D
    kv = (B, S, Hkv, d) if problem.kv_layout == ZSA_KV_NATURAL else (D, B, S // D, Hkv, d)
    return (ns, B, S // D, Hq, d), kv, (ns, B, Hq, S // D)


def _problem_from(q, k, D, causal, scale, kv_layout, shard_begin, shard_count):
    ns, B, twoC, Hq, d = q.shape
    S = D * twoC
    Hkv = k.shape[2] if kv_layout == ZSA_KV_NATURAL else k.shape[3]
    if shard_count == 0 and ns != D:
        raise ValueError(f"q holds {ns} shards; pass shard_begin / shard_count for a subset of D={D}")
    return make_problem(B, S, Hq, Hkv, d, D, causal, scale, kv_layout, shard_begin, shard_count)


def attn_fwd(q, k, v, D, causal=True, scale=None, workspace=None, kv_layout=ZSA_KV_NATURAL,
             shard_begin=0, shard_count=0):
    """O, lse = attention(Q, K, V): all D zigzag shards in one launch, or the shards
    [shard_begin, shard_begin + shard_count) when shard_count > 0."""
    import torch
    problem = _problem_from(q, k, D, causal, scale, kv_layout, shard_begin, shard_count)
    qs, ks, ls = _shapes(problem)
    _check_tensor(q, qs, torch.bfloat16, "q")
    _check_tensor(k, ks, torch.bfloat16, "k")
    _check_tensor(v, ks, torch.bfloat16, "v")
    o = torch.empty_like(q)
    lse = torch.empty(ls, dtype=torch.float32, device=q.device)
    nbytes = zsa_workspace_bytes(problem, 0)
    if workspace is None or workspace.numel() * workspace.element_size() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    zsa_attn_fwd(problem, q, k, v, o, lse, workspace)
    return o, lse


def attn_fwd_block(q, k, v, D, key_lo, key_hi, rows_per_batch=None, row_offset=0, causal=True,
                   scale=None, workspace=None, shard_begin=0, shard_count=0, out=None):
    """Partial O, lse over the keys at positions [key_lo, key_hi) only (one ring step).

    k, v: contiguous (..., Hkv, d) tensors whose leading dims flatten to the K/V rows; the
    key at position p of batch b is row b * rows_per_batch + row_offset + p - key_lo
    (rows_per_batch defaults to key_hi - key_lo: a [B][key_hi - key_lo][Hkv][d] block).
    out: optional (o, lse) to write into."""
    import torch
    ns, B, twoC, Hq, d = q.shape
    Hkv = k.shape[-2]
    if shard_count == 0 and ns != D:
        raise ValueError(f"q holds {ns} shards; pass shard_begin / shard_count for a subset of D={D}")
    problem = make_problem(B, D * twoC, Hq, Hkv, d, D, causal, scale, ZSA_KV_NATURAL, shard_begin,
                           shard_count)
    qs, _, ls = _shapes(problem)
    _check_tensor(q, qs, torch.bfloat16, "q")
    rows = k.numel() // (Hkv * d)
    _check_tensor(k, tuple(k.shape), torch.bfloat16, "k")
    _check_tensor(v, tuple(k.shape), torch.bfloat16, "v")
    if k.shape[-1] != d:
        raise ValueError(f"k head dim {k.shape[-1]} != q head dim {d}")
    block = zsa_key_block(int(key_lo), int(key_hi),
                          int(key_hi - key_lo if rows_per_batch is None else rows_per_batch),
                          int(row_offset), int(rows))
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(ls, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
        _check_tensor(o, qs, torch.bfloat16, "o")
        _check_tensor(lse, ls, torch.float32, "lse")
    nbytes = zsa_workspace_bytes(problem, 0)
    if workspace is None or workspace.numel() * workspace.element_size() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    zsa_attn_fwd_block(problem, block, q, k, v, o, lse, workspace)
    return o, lse


def to_shard_major(x, D, shard_begin=0, shard_count=0, out=None):
    """K5: natural [B][S][H][d] bf16 -> zigzag shard-major [shards][B][2C][H][d]."""
    import torch
    B, S, H, d = x.shape
    ns = shard_count or D
    problem = make_problem(B, S, H, H, d, D, shard_begin=shard_begin, shard_count=shard_count)
    _check_tensor(x, (B, S, H, d), torch.bfloat16, "x")
    if out is None:
        out = torch.empty((ns, B, S // D, H, d), dtype=torch.bfloat16, device=x.device)
    _check_tensor(out, (ns, B, S // D, H, d), torch.bfloat16, "out")
    zsa_permute(problem, H, 1, x, out)
    return out


def from_shard_major(y, D, shard_begin=0, shard_count=0, out=None):
    """K5: zigzag shard-major [shards][B][2C][H][d] bf16 -> natural [B][S][H][d] (with a
    shard range, only that range's positions of `out` are written)."""
    import torch
    ns, B, twoC, H, d = y.shape
    S = D * twoC
    problem = make_problem(B, S, H, H, d, D, shard_begin=shard_begin, shard_count=shard_count)
    _check_tensor(y, ((shard_count or D), B, twoC, H, d), torch.bfloat16, "y")
    if out is None:
        out = torch.empty((B, S, H, d), dtype=torch.bfloat16, device=y.device)
    _check_tensor(out, (B, S, H, d), torch.bfloat16, "out")
    zsa_permute(problem, H, 0, y, out)
    return out


def attn_bwd(q, k, v, o, lse, do, D, causal=True, scale=None, workspace=None,
             kv_layout=ZSA_KV_NATURAL, shard_begin=0, shard_count=0):
    """dQ, dK, dV of <dO, O>: dK/dV summed over the launch's shards (all D by default)
    and the q heads of a group."""
    import torch
    problem = _problem_from(q, k, D, causal, scale, kv_layout, shard_begin, shard_count)
    qs, ks, ls = _shapes(problem)
    for name, x, shp in (("q", q, qs), ("k", k, ks), ("v", v, ks), ("o", o, qs), ("do", do, qs)):
        _check_tensor(x, shp, torch.bfloat16, name)
    _check_tensor(lse, ls, torch.float32, "lse")
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    nbytes = zsa_workspace_bytes(problem, 1)
    if workspace is None or workspace.numel() * workspace.element_size() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    zsa_attn_bwd(problem, q, k, v, o, lse, do, dq, dk, dv, workspace)
    return dq, dk, dv
