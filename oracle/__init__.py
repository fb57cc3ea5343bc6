"""CPU oracle for MLA-absorb tree-verify attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library
and its binding in ``mla_speculative_verify_absorb_b200``) never imports it;
the two share no code. Inputs come from the separate ``workloads`` module,
which holds none of the method's arithmetic.

The arithmetic lives in ``mla_verify_oracle.c`` (plain C, float64, every
definition cited there); this module only compiles it with gcc and passes
numpy arrays through ctypes. ``brute.py`` is a separately written numpy
brute force used as one of the pins on tiny inputs.

Parity of every function here is pinned by ``tests/test_oracle_pins.py``
(causal special case against torch's float64 SDPA, exact single-token and
equal-score cases, permutation invariance, merge identity, closed-form mask
counts, numpy brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_verify_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libmla_verify_oracle.so")
_lock = threading.Lock()
_lib = None

D_LATENT = 512
D_ROPE = 64


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_build`` (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            lib.oracle_ancestor_masks.argtypes = [P, i32, P]
            lib.oracle_ancestor_masks.restype = ctypes.c_int
            lib.oracle_verify_rows.argtypes = [i32, i32, P, P, P, P, P, P, P, i64, f64, P, i64, P, P, P, i32]
            lib.oracle_verify_rows.restype = ctypes.c_int
            lib.oracle_partial_rows.argtypes = [i32, i32, P, P, P, P, P, P, P, i64, f64, P, i64, i64, i64, P, P, P]
            lib.oracle_partial_rows.restype = ctypes.c_int
            lib.oracle_merge_states.argtypes = [i32, i64, P, P, P, P, P]
            lib.oracle_merge_states.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def ancestor_masks(parents, qo_indptr) -> np.ndarray:
    """uint64 ancestor-or-self mask of every tree node of every request."""
    lib = _load()
    parents = _c(parents, np.int32)
    qo_indptr = _c(qo_indptr, np.int32)
    anc = np.zeros(parents.shape[0], dtype=np.uint64)
    for b in range(qo_indptr.shape[0] - 1):
        lo, hi = int(qo_indptr[b]), int(qo_indptr[b + 1])
        seg_p = _c(parents[lo:hi], np.int32)
        seg_a = np.zeros(hi - lo, dtype=np.uint64)
        if lib.oracle_ancestor_masks(_ptr(seg_p), hi - lo, _ptr(seg_a)) != 0:
            raise ValueError(f"invalid tree in request {b}")
        anc[lo:hi] = seg_a
    return anc


def _problem(inp, anc):
    return (
        _c(inp.qo_indptr, np.int32), _c(inp.kv_indptr, np.int32), _c(inp.kv_indices, np.int32),
        _c(anc, np.uint64), _c(inp.q_latent, np.uint16), _c(inp.q_rope, np.uint16),
        _c(inp.kv_pool, np.uint16),
    )


def verify_rows(inp, anc, rows=None, threads: int = 0):
    """Oracle output for query rows ``q = token*H + head`` (all rows if None).

    Returns (out float64 [n, 512], lse float64 [n], visible int32 [n]).
    """
    lib = _load()
    qo, kvp, kvi, anc_c, ql, qr, pool = _problem(inp, anc)
    H = int(inp.q_latent.shape[1])
    n_all = int(qo[-1]) * H
    rows_c = None if rows is None else _c(rows, np.int64)
    n = n_all if rows is None else int(rows_c.shape[0])
    out = np.zeros((n, D_LATENT), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    vis = np.zeros(n, dtype=np.int32)
    rc = lib.oracle_verify_rows(int(qo.shape[0] - 1), H, _ptr(qo), _ptr(kvp), _ptr(kvi), _ptr(anc_c),
                                _ptr(ql), _ptr(qr), _ptr(pool), int(pool.shape[0]), float(inp.sm_scale),
                                _ptr(rows_c), n, _ptr(out), _ptr(lse), _ptr(vis), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the problem (bad row, slot or tree)")
    return out, lse, vis


def partial_rows(inp, anc, key_lo: int, key_hi: int, rows=None):
    """Partial states (m, l, O) over KV positions [key_lo, key_hi) of each request."""
    lib = _load()
    qo, kvp, kvi, anc_c, ql, qr, pool = _problem(inp, anc)
    H = int(inp.q_latent.shape[1])
    rows_c = None if rows is None else _c(rows, np.int64)
    n = int(qo[-1]) * H if rows is None else int(rows_c.shape[0])
    m = np.zeros(n, dtype=np.float64)
    l = np.zeros(n, dtype=np.float64)
    o = np.zeros((n, D_LATENT), dtype=np.float64)
    rc = lib.oracle_partial_rows(int(qo.shape[0] - 1), H, _ptr(qo), _ptr(kvp), _ptr(kvi), _ptr(anc_c),
                                 _ptr(ql), _ptr(qr), _ptr(pool), int(pool.shape[0]), float(inp.sm_scale),
                                 _ptr(rows_c), n, int(key_lo), int(key_hi), _ptr(m), _ptr(l), _ptr(o))
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return m, l, o


def merge_states(ms, ls, os_):
    """Merge stacked partial states ([S, n], [S, n], [S, n, 512]) into (out, lse)."""
    lib = _load()
    ms, ls, os_ = _c(ms, np.float64), _c(ls, np.float64), _c(os_, np.float64)
    S, n = ms.shape
    out = np.zeros((n, D_LATENT), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    lib.oracle_merge_states(int(S), int(n), _ptr(ms), _ptr(ls), _ptr(os_), _ptr(out), _ptr(lse))
    return out, lse
