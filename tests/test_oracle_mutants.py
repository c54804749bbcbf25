"""Planted-mistake check for the oracle pins.

Each case copies oracle.c, plants one plausible mistake (wrong chunk index, a
dropped diagonal, a wrong sign, a transposed operand, a wrong GQA map, a dropped
scale ...), builds it on the CPU into a temporary directory and runs the pin
checks against it: every mutant must fail at least one of them.  Nothing here
touches a GPU or the product library.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from sequence_sharded_causal_b200 import inputs

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "second_chunk_index": ("(int64_t)(2 * D - 1 - r) * C", "(int64_t)(2 * D - 2 - r) * C"),
    "chunks_swapped": ("if (j < C)\n        return (int64_t)r * C + j;",
                       "if (j >= C)\n        return (int64_t)r * C + (j - C);"),
    "diagonal_dropped": ("causal ? p + 1 : S", "causal ? (p > 0 ? p : 1) : S"),
    "lse_sign": ("double lse = m + log(l);", "double lse = m - log(l);"),
    "gqa_modulo": ("v, b, h / G, s_buf, o + (row * Hq + h) * d, &nk);",
                   "v, b, h % Hkv, s_buf, o + (row * Hq + h) * d, &nk);"),
    "scale_dropped_fwd": ("s_buf[key] = scale * dot;", "s_buf[key] = dot;"),
    "dk_scale_dropped": ("dk[kofs + t] += scale * ds_buf[key] * q_row[t];",
                         "dk[kofs + t] += ds_buf[key] * q_row[t];"),
    "ds_sign": ("ds_buf[key] = p_buf[key] * (dp - dlt);", "ds_buf[key] = p_buf[key] * (dlt - dp);"),
    "dq_uses_v": ("dq_row[t] += scale * ds_buf[key] * k[kofs + t];",
                  "dq_row[t] += scale * ds_buf[key] * v[kofs + t];"),
    "dv_uses_ds": ("dv[kofs + t] += p_buf[key] * do_row[t];",
                   "dv[kofs + t] += ds_buf[key] * do_row[t];"),
    "delta_dropped": ("dlt += do_row[t] * o_row[t];", "dlt += 0.0 * o_row[t];"),
    "kend_off_by_one": ("return largest / bk + 1;", "return largest / bk;"),
    "order_ascending": ("return a->key_work > b->key_work ? -1 : 1;",
                        "return a->key_work < b->key_work ? -1 : 1;"),
    "keys_diagonal_dropped": ("if (causal && p + 1 < end) end = p + 1;",
                              "if (causal && p < end) end = p;"),
    "keys_range_shifted": ("for (int64_t key = key_lo; key < end; ++key)",
                           "for (int64_t key = key_lo + (key_lo > 0); key < end; ++key)"),
    "merge_weights_unnormalised": ("double w = exp(lse_parts[(int64_t)i * m + x] - lse_x);",
                                   "double w = exp(lse_parts[(int64_t)i * m + x] - mx);"),
    "merge_lse_max_dropped": ("double lse_x = mx + log(l);", "double lse_x = log(l);"),
}


def _build_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, name      # planted wherever the line occurs
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(path), "-o",
                    str(lib), "-lm"], check=True)
    return str(lib)


def _pins_pass():
    """A compact subset of the pin suite; returns False at the first failure."""
    rng = np.random.default_rng(1)
    # zigzag balance + bijection
    for S, D in ((16, 2), (48, 3), (64, 4)):
        perm, _ = oracle.partition(S, D)
        if not np.array_equal(np.sort(perm), np.arange(S)):
            return False
        C, twoC = S // (2 * D), S // D
        pairs = {int((perm[r * twoC:(r + 1) * twoC].astype(np.int64) + 1).sum()) for r in range(D)}
        if pairs != {C * C * (2 * D - 1) + C * (C + 1)}:
            return False
    # schedule kend vs brute visibility, and order
    S, D, bq, bk = 512, 2, 64, 64
    perm, _ = oracle.partition(S, D)
    B_, Hq_, Hkv_ = 1, 2, 1
    st, units = oracle.schedule(S, D, B_, Hq_, Hkv_, True, bq, bk, 2)
    for u in units:
        r, i0, k0 = int(u[0]), int(u[3]), int(u[7])
        rows = perm[r * (S // D) + i0 * bq: r * (S // D) + (i0 + 1) * bq]
        if k0 != int(rows.max()) // bk + 1:
            return False
    work = np.maximum(units[:, 7], units[:, 8])
    grp = units[:, 1] * Hkv_ + units[:, 2]
    if not (np.diff(grp) >= 0).all() or not (np.diff(work)[np.diff(grp) == 0] <= 0).all():
        return False
    # forward vs unsharded brute force (GQA, causal)
    B, S, Hq, Hkv, d, D = 1, 32, 4, 2, 8, 2
    q = rng.standard_normal((B, S, Hq, d))
    k = rng.standard_normal((B, S, Hkv, d))
    v = rng.standard_normal((B, S, Hkv, d))
    do = rng.standard_normal((B, S, Hq, d))
    perm, _ = oracle.partition(S, D)
    qs = inputs.to_shard_major(torch.from_numpy(q), perm, D).numpy()
    dos = inputs.to_shard_major(torch.from_numpy(do), perm, D).numpy()
    o, lse = oracle.attn_fwd(qs, k, v, D)
    o_ref, lse_ref = brute.causal_attention(q, k, v)
    if np.abs(inputs.from_shard_major(torch.from_numpy(o), perm).numpy() - o_ref).max() > 1e-12:
        return False
    if np.abs(inputs.stats_from_shard_major(torch.from_numpy(lse), perm).numpy()
              - lse_ref).max() > 1e-12:
        return False
    # backward vs matrix form
    g = oracle.attn_bwd(qs, k, v, dos, D)
    dq_ref, dk_ref, dv_ref = brute.causal_attention_bwd(q, k, v, do)
    if np.abs(inputs.from_shard_major(torch.from_numpy(g["dq"]), perm).numpy() - dq_ref).max() > 1e-11:
        return False
    if np.abs(g["dk"] - dk_ref).max() > 1e-11 or np.abs(g["dv"] - dv_ref).max() > 1e-11:
        return False
    # dQ of selected rows vs the matrix form
    rows = np.array([0, 7, 16, 31])
    dq_rows = oracle.attn_dq_rows(qs.reshape(-1, Hq, d)[rows], dos.reshape(-1, Hq, d)[rows],
                                  rows, k, v, D, Hq)
    dq_nat = inputs.to_shard_major(torch.from_numpy(dq_ref), perm, D).numpy().reshape(-1, Hq, d)
    if np.abs(dq_rows - dq_nat[rows]).max() > 1e-11:
        return False
    # key-range forward vs the masked brute force, and the merge of a split
    S2, D2 = 32, 2
    perm2, _ = oracle.partition(S2, D2)
    qk = rng.standard_normal((1, S2, 2, 8))
    kk = rng.standard_normal((1, S2, 1, 8))
    vk = rng.standard_normal((1, S2, 1, 8))
    qs2 = inputs.to_shard_major(torch.from_numpy(qk), perm2, D2).numpy()
    for lo, hi in ((5, 20), (11, 32)):
        ok_, lk = oracle.attn_fwd_keys(qs2, kk, vk, D2, lo, hi)
        o_b, l_b = brute.key_range_attention(qk, kk, vk, lo, hi)
        o_n = inputs.from_shard_major(torch.from_numpy(ok_), perm2).numpy()
        if np.abs(o_n - o_b).max() > 1e-12:
            return False
    o_f, l_f = oracle.attn_fwd(qs2, kk, vk, D2)
    pa = oracle.attn_fwd_keys(qs2, kk, vk, D2, 0, 13)
    pb = oracle.attn_fwd_keys(qs2, kk, vk, D2, 13, 32)
    o_m, l_m = oracle.attn_merge([pa[0], pb[0]], [pa[1], pb[1]])
    if np.abs(o_m - o_f).max() > 1e-12 or np.abs(l_m - l_f).max() > 1e-12:
        return False
    return True


def test_unmutated_oracle_passes():
    oracle._load()
    assert _pins_pass()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name, monkeypatch):
    lib_path = _build_mutant(tmp_path, name)
    real = oracle._load()
    mutant = ctypes.CDLL(lib_path)
    for fn in ("oracle_partition", "oracle_schedule", "oracle_attn_fwd", "oracle_attn_fwd_rows",
               "oracle_attn_bwd", "oracle_attn_dq_rows", "oracle_attn_fwd_keys",
               "oracle_attn_merge"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    try:
        ok = _pins_pass()
    except Exception:
        ok = False
    assert not ok, f"mutant {name} slipped through the pins"
