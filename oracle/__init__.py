"""fp64 CPU oracle for certified Top-k attention truncation (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does: it
shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64); this module only loads
the compiled library, marshals numpy arrays and names the statistic columns.
Definitions follow the abstract of "A Mathematical Theory of Top-k Sparse
Attention via Total Variation Distance" (arXiv 2512.07647, fugumt.com page):
TV = discarded tail mass = 1 - exp(-KL), minimal k_eps with TV <= eps, the
head-tail factorisation of the output error and its diameter bound.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle_cta.so")

F32, BF16 = 0, 1

# Column names of the per-row statistics array, in the order of the enum in oracle.c.
STAT_NAMES = (
    "tv", "tv_def", "kl", "one_minus_exp_neg_kl", "err", "err_direct", "tv_km1",
    "gap_u", "tie_bound", "var_p", "diam", "max_s", "log_z", "head_mass",
    "gap_bound", "min_head_u",
)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle_cta.so (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC", "-pthread",
            _SRC, "-o", _LIB, "-lm",
        ])
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.ora_nstat.restype = ctypes.c_int
        lib.ora_certified_topk_attn.restype = ctypes.c_int
        lib.ora_certified_topk_attn.argtypes = [
            vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64, dbl, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp,
        ]
        lib.ora_dense_attn.restype = ctypes.c_int
        lib.ora_dense_attn.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64, vp]
        lib.ora_eval_kept_set.restype = ctypes.c_int
        lib.ora_eval_kept_set.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64,
                                          vp, vp, vp, vp]
        assert lib.ora_nstat() == len(STAT_NAMES)
        _lib = lib
    return _lib


def _raw(a: np.ndarray, dtype: int) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if dtype == F32:
        assert a.dtype == np.float32
    else:
        assert a.dtype in (np.uint16, np.int16), "bf16 inputs are passed as their raw 16-bit words"
    return a


def certified_topk_attn(q, K, V, eps, *, n_heads, n_kv_heads, dtype=F32, batch=1, m=1,
                        threads=None, want_diam=False, want_attn=True, select_only=False):
    """Run the oracle on raw input arrays.

    q: [batch, n_heads, m, d]; K, V: [batch, n_kv_heads, n, d]; fp32 arrays, or
    bf16 as uint16 words.  Returns a dict with ``out`` [rows, d] (fp64),
    ``attn`` [rows, d], ``k`` [rows], ``idx`` (list of int32 arrays, ascending),
    ``idx_full`` [rows, n] and one fp64 array per statistic in STAT_NAMES.
    ``select_only`` stops after k, idx and the TV values (no value rows read).
    """
    lib = _load()
    q, K, V = _raw(q, dtype), _raw(K, dtype), _raw(V, dtype)
    d = q.shape[-1]
    n = K.shape[-2]
    rows = batch * n_heads * m
    assert q.size == rows * d and K.size == batch * n_kv_heads * n * d and V.size == K.size
    out = np.zeros((rows, d), np.float64)
    attn = np.zeros((rows, d), np.float64) if want_attn else None
    k = np.zeros(rows, np.int32)
    idx = np.full((rows, n), -1, np.int32)
    stats = np.zeros((rows, len(STAT_NAMES)), np.float64)
    if threads is None:
        threads = os.cpu_count() or 1
    rc = lib.ora_certified_topk_attn(
        q.ctypes.data, K.ctypes.data, V.ctypes.data, dtype, batch, n_heads, n_kv_heads, m, n, d,
        float(eps), int(threads), int(bool(want_diam)), int(bool(select_only)), out.ctypes.data,
        attn.ctypes.data if attn is not None else None, k.ctypes.data, idx.ctypes.data,
        stats.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle failed with status {rc}")
    res = {"out": out, "attn": attn, "k": k, "idx_full": idx,
           "idx": [idx[r, : k[r]] for r in range(rows)]}
    for j, name in enumerate(STAT_NAMES):
        res[name] = stats[:, j].copy()
    return res


def dense_attn(q, K, V, *, n_heads, n_kv_heads, dtype=F32, batch=1, m=1):
    """Plain fp64 softmax attention over all keys; returns [rows, d]."""
    lib = _load()
    q, K, V = _raw(q, dtype), _raw(K, dtype), _raw(V, dtype)
    d = q.shape[-1]
    n = K.shape[-2]
    rows = batch * n_heads * m
    out = np.zeros((rows, d), np.float64)
    rc = lib.ora_dense_attn(q.ctypes.data, K.ctypes.data, V.ctypes.data, dtype, batch, n_heads,
                            n_kv_heads, m, n, d, out.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle dense attention failed with status {rc}")
    return out


def eval_kept_set(q, K, V, sets, *, n_heads, n_kv_heads, dtype=F32, batch=1, m=1):
    """The truncation to given kept sets, in fp64 (see ora_eval_kept_set).

    ``sets`` is a list of one index array per row (distinct key indices, any
    order, at least one).  Returns a dict with ``tv``, ``kl``, ``err``,
    ``tv_drop_lowest`` (TV after removing the set's lowest-ranked key) [rows]
    and ``out`` [rows, d].
    """
    lib = _load()
    q, K, V = _raw(q, dtype), _raw(K, dtype), _raw(V, dtype)
    d = q.shape[-1]
    n = K.shape[-2]
    rows = batch * n_heads * m
    assert len(sets) == rows
    packed = np.full((rows, n), -1, np.int32)
    counts = np.zeros(rows, np.int32)
    for r, s in enumerate(sets):
        s = np.asarray(s, np.int64)
        packed[r, : len(s)] = s
        counts[r] = len(s)
    out = np.zeros((rows, d), np.float64)
    res = np.zeros((rows, 4), np.float64)
    rc = lib.ora_eval_kept_set(q.ctypes.data, K.ctypes.data, V.ctypes.data, dtype, batch, n_heads,
                               n_kv_heads, m, n, d, packed.ctypes.data, counts.ctypes.data,
                               out.ctypes.data, res.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle set evaluation failed with status {rc}")
    return {"tv": res[:, 0].copy(), "kl": res[:, 1].copy(), "err": res[:, 2].copy(),
            "tv_drop_lowest": res[:, 3].copy(), "out": out}
