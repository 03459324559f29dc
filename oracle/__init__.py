"""TokenButler decode-path oracle (test infrastructure only).

Only the tests, the package smoke check and the CPU-baseline leg of the
benchmark may import this package.  It shares no code with the CUDA library:
the arithmetic lives in ``tb_oracle.c`` (plain C, double precision), this file
only marshals numpy arrays into it and strings the steps together per head.

bf16 tensors are handled as ``numpy.uint16`` arrays holding the raw bits.

Function-level citations are in ``tb_oracle.c``; the decode-loop schedule is in
``oracle/schedule.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tb_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


_SAN_LIB_PATH = os.path.join(_HERE, "liboracle_san.so")
_SAN_FLAGS = ["-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH, sanitize: bool = False) -> str:
    """Compile the C oracle with gcc (plain -O2, no fast-math).  sanitize=True
    adds AddressSanitizer and UBSan, for checking the oracle's own memory
    accesses (the process then needs the sanitizer runtimes preloaded)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off"] + (_SAN_FLAGS if sanitize else []) + ["-o", out, src, "-lm"])
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_double.restype = f64
    lib.orc_double_to_bf16.argtypes = [f64]
    lib.orc_double_to_bf16.restype = ctypes.c_uint16
    lib.orc_project_keys.argtypes = [P, P, P, i64, i32, i32]
    lib.orc_project_keys.restype = None
    lib.orc_predict_queries.argtypes = [P, P, P, P, i32, i32, i32, i32]
    lib.orc_predict_queries.restype = None
    lib.orc_scores.argtypes = [P, P, i32, i64, i64, P]
    lib.orc_scores.restype = None
    lib.orc_group_scores.argtypes = [P, i32, P, i32, i64, i64, i32, P]
    lib.orc_group_scores.restype = None
    lib.orc_select.argtypes = [P, i64, i64, i64, i64, i32, P]
    lib.orc_select.restype = i64
    lib.orc_select_inclusive.argtypes = [P, i64, i64, i64, i64, i32, P]
    lib.orc_select_inclusive.restype = i64
    lib.orc_attention_set.argtypes = [i64, i64, i64, P, i64, P]
    lib.orc_attention_set.restype = i64
    lib.orc_attention.argtypes = [P, P, P, i32, P, i64, f64, P]
    lib.orc_attention.restype = None
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(path)
    if _lib is None:
        if os.environ.get("TB_ORACLE_SANITIZE") == "1":
            _lib = _bind(build(out=_SAN_LIB_PATH, sanitize=True))
        else:
            _lib = _bind(build())
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 arrays are passed as uint16 bit patterns"
    return a


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (the upper half of a binary32)."""
    u = (np.asarray(bits, dtype=np.uint32) << 16).astype(np.uint32)
    return u.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# the five steps, one head (or one KV head) at a time
# --------------------------------------------------------------------------

def project_keys(K: np.ndarray, Wk: np.ndarray, lib=None) -> np.ndarray:
    """K' = bf16(K @ Wk^T) for one KV head.  K: [rows][d], Wk: [d'][d]."""
    lib = lib or load()
    K, Wk = _u16(K), _u16(Wk)
    rows, d = K.shape
    dp = Wk.shape[0]
    assert Wk.shape[1] == d
    out = np.empty((rows, dp), dtype=np.uint16)
    lib.orc_project_keys(_ptr(K), _ptr(Wk), _ptr(out), rows, d, dp)
    return out


def predict_queries(h: np.ndarray, W1: np.ndarray, W2: np.ndarray, lib=None) -> np.ndarray:
    """q' = bf16(SiLU(h W1^T)) W2^T in fp32.  h: [B][hidden], W1: [inter][hidden],
    W2: [n_out][inter]; returns [B][n_out] float32."""
    lib = lib or load()
    h, W1, W2 = _u16(h), _u16(W1), _u16(W2)
    batch, hidden = h.shape
    inter = W1.shape[0]
    n_out = W2.shape[0]
    assert W1.shape[1] == hidden and W2.shape[1] == inter
    out = np.empty((batch, n_out), dtype=np.float32)
    lib.orc_predict_queries(_ptr(h), _ptr(W1), _ptr(W2), _ptr(out), batch, hidden, inter, n_out)
    return out


def scores(qp: np.ndarray, Kp: np.ndarray, t_begin: int, t_end: int, lib=None) -> np.ndarray:
    """fp32 scores of positions [t_begin, t_end) for one query head."""
    lib = lib or load()
    qp = np.ascontiguousarray(qp, dtype=np.float32)
    Kp = _u16(Kp)
    dp = Kp.shape[1]
    assert qp.shape == (dp,)
    n = max(0, t_end - t_begin)
    out = np.empty(n, dtype=np.float32)
    if n:
        lib.orc_scores(_ptr(qp), _ptr(Kp), dp, t_begin, t_end, _ptr(out))
    return out


GROUP_REDUCE = {"max": 0, "sum": 1}


def group_scores(qp: np.ndarray, Kp: np.ndarray, t_begin: int, t_end: int, reduce: str,
                 lib=None) -> np.ndarray:
    """fp32 group scores of positions [t_begin, t_end) for the G heads of one
    GQA group (qp [G][d']): the largest or the fp32 sum, in head order, of the
    heads' fp32 scores."""
    lib = lib or load()
    qp = np.ascontiguousarray(qp, dtype=np.float32)
    Kp = _u16(Kp)
    dp = Kp.shape[1]
    assert qp.ndim == 2 and qp.shape[1] == dp
    n = max(0, t_end - t_begin)
    out = np.empty(n, dtype=np.float32)
    if n:
        lib.orc_group_scores(_ptr(qp), qp.shape[0], _ptr(Kp), dp, t_begin, t_end, GROUP_REDUCE[reduce],
                             _ptr(out))
    return out


def select(s_cand: np.ndarray, T: int, S: int, N: int, B: int, nbr: int, lib=None) -> np.ndarray:
    """Top-B of the candidates [S, T-N) by (score desc, position asc), expanded
    by +-nbr and clipped to the candidate range; sorted int32 positions."""
    lib = lib or load()
    nC = max(0, T - N - S)
    s_cand = np.ascontiguousarray(s_cand, dtype=np.float32)
    assert s_cand.shape == (nC,)
    out = np.empty(max(nC, 1), dtype=np.int32)
    n = lib.orc_select(_ptr(s_cand), T, S, N, B, nbr, _ptr(out)) if nC else 0
    return out[:n].copy()


def select_inclusive(s_cand: np.ndarray, T: int, S: int, N: int, B: int, nbr: int, lib=None) -> np.ndarray:
    """Budget-inclusive variant: candidates in (score desc, position asc) order
    while the union of their +-nbr neighbourhoods, clipped to [S, T-N), holds
    at most B positions; sorted int32 positions."""
    lib = lib or load()
    nC = max(0, T - N - S)
    s_cand = np.ascontiguousarray(s_cand, dtype=np.float32)
    assert s_cand.shape == (nC,)
    out = np.empty(max(nC, 1), dtype=np.int32)
    n = lib.orc_select_inclusive(_ptr(s_cand), T, S, N, B, nbr, _ptr(out)) if nC else 0
    return out[:n].copy()


def attention_set(T: int, S: int, N: int, I: np.ndarray, lib=None) -> np.ndarray:
    """Sorted attended positions: sink U window U I."""
    lib = lib or load()
    I = np.ascontiguousarray(I, dtype=np.int32)
    out = np.empty(T + I.size + 1, dtype=np.int32)
    n = lib.orc_attention_set(T, S, N, _ptr(I), I.size, _ptr(out))
    return out[:n].copy()


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, A: np.ndarray, scale: float,
              lib=None) -> np.ndarray:
    """fp32 attention output of one query head over the rows A of one KV head."""
    lib = lib or load()
    q, K, V = _u16(q), _u16(K), _u16(V)
    d = q.shape[0]
    A = np.ascontiguousarray(A, dtype=np.int32)
    out = np.empty(d, dtype=np.float32)
    lib.orc_attention(_ptr(q), _ptr(K), _ptr(V), d, _ptr(A), A.size, float(scale), _ptr(out))
    return out
