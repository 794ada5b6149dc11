"""ctypes front end of the plain C oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path never imports this
package.  It shares no code with the CUDA library; the two meet only through
the seeded input generators, which hold none of the method's arithmetic.

The oracle follows the verification step of speculative sampling as the pages
state it (page titles and sections are cited in ``oracle.c``): temperature
softmaxes q and p, left-to-right acceptance with probability min(1, q/p)
stopping at the first rejection, a draw from max(0, q - p) normalised at the
rejection, and a bonus draw from q when every draft is accepted.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SRCS = [_SRC, os.path.join(_HERE, "gate.c"), os.path.join(_HERE, "sampling.c")]
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1
DTYPE_F64 = 2

OK = 0
ERR_TOKEN_RANGE = 16
ERR_NONFINITE = 17
WARN_ZERO_MASS = 18


def build(force: bool = False) -> str:
    """Compile the oracle's C files into ``liboracle.so`` (plain gcc, IEEE semantics)."""
    stale = not os.path.exists(_LIB) or any(
        os.path.getmtime(_LIB) < os.path.getmtime(src) for src in _SRCS)
    if force or stale:
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", _LIB, *_SRCS, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("gamma", ctypes.c_int),
        ("vocab", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("target_logits", ctypes.c_void_p),
        ("draft_logits", ctypes.c_void_p),
        ("draft_tokens", ctypes.c_void_p),
        ("u_accept", ctypes.c_void_p),
        ("u_resample", ctypes.c_void_p),
        ("temperature", ctypes.c_double),
    ]


_RESULT_FIELDS = [
    "out_tokens", "out_num_accepted", "seq_status", "target_max", "target_sum",
    "draft_max", "draft_sum", "q_tok", "p_tok", "ratio", "accept_margin",
    "resid_mass", "cdf_margin_mass", "cdf_margin_norm", "sampled",
]


class _Result(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in _RESULT_FIELDS]


class _GateProblem(ctypes.Structure):
    _fields_ = [
        ("branches", ctypes.c_int),
        ("positions", ctypes.c_int),
        ("dim", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("hidden", ctypes.c_void_p),
        ("parent", ctypes.c_void_p),
        ("tau", ctypes.c_double),
    ]


_GATE_FIELDS = ["rel_diff", "margin", "recompute", "provenance", "source", "packed", "n_packed",
                "parent_used"]


class _GateResult(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in _GATE_FIELDS]


class _SampProblem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("gamma", ctypes.c_int),
        ("vocab", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("target_logits", ctypes.c_void_p),
        ("draft_logits", ctypes.c_void_p),
        ("draft_tokens", ctypes.c_void_p),
        ("u_accept", ctypes.c_void_p),
        ("u_resample", ctypes.c_void_p),
        ("temperature", ctypes.c_void_p),
        ("top_k", ctypes.c_int),
        ("top_p", ctypes.c_double),
    ]


_SAMP_FIELDS = ["out_tokens", "out_num_accepted", "seq_status", "q_tok", "p_tok",
                "accept_margin", "resid_mass", "cdf_margin_norm", "kept_target", "kept_draft",
                "filter_margin"]


class _SampResult(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in _SAMP_FIELDS]


ERR_TEMPERATURE = 21

GATE_OK = 0
GATE_ERR_PARENT = 20

_lib = None
_lib_lock = threading.Lock()


def _load():
    global _lib
    with _lib_lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_verify.argtypes = [ctypes.POINTER(_Problem), ctypes.POINTER(_Result),
                                          ctypes.c_int, ctypes.c_int]
            lib.oracle_verify.restype = ctypes.c_int
            lib.oracle_softmax_row.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t,
                                               ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_softmax_row.restype = ctypes.c_int
            lib.oracle_gate.argtypes = [ctypes.POINTER(_GateProblem), ctypes.POINTER(_GateResult)]
            lib.oracle_gate.restype = ctypes.c_int
            lib.oracle_verify_sampling.argtypes = [ctypes.POINTER(_SampProblem),
                                                   ctypes.POINTER(_SampResult),
                                                   ctypes.c_int, ctypes.c_int]
            lib.oracle_verify_sampling.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _dtype_code(arr: np.ndarray) -> int:
    if arr.dtype == np.float32:
        return DTYPE_F32
    if arr.dtype == np.uint16:
        return DTYPE_BF16
    if arr.dtype == np.float64:
        return DTYPE_F64
    raise TypeError(f"logits must be float32, float64 or uint16 (bf16 bits), got {arr.dtype}")


def lm_logits(hidden: np.ndarray, weight: np.ndarray) -> np.ndarray:
    """Logits of an output layer, exactly as the plain definition states them:
    hidden [..., d] . weight [V, d]^T in float64 (hidden and weight given as
    float32 values, e.g. the values of bf16 inputs).  A library matmul is the
    one step; the product of two bf16 values is exact in float64 and the sum
    of d of them is rounded at most d times at double precision."""
    h = np.asarray(hidden, np.float64)
    w = np.asarray(weight, np.float64)
    return np.ascontiguousarray(h @ w.T)


def softmax(row: np.ndarray, temperature: float = 1.0):
    """Softmax of one row of logits (float32, or uint16 holding bf16 bits).

    Returns ``(prob float64[V], raw_max, sum)``; raises ValueError on a row the
    oracle rejects (NaN, +inf, or no finite entry).
    """
    row = np.ascontiguousarray(row)
    V = row.shape[-1]
    prob = np.empty(V, np.float64)
    mx = ctypes.c_double()
    sm = ctypes.c_double()
    st = _load().oracle_softmax_row(_ptr(row), _dtype_code(row), 0, V, float(temperature),
                                    _ptr(prob), ctypes.addressof(mx), ctypes.addressof(sm))
    if st != OK:
        raise ValueError(f"oracle rejected the row (status {st})")
    return prob, mx.value, sm.value


def verify(target: np.ndarray, draft: np.ndarray, tokens: np.ndarray, u_accept: np.ndarray,
           u_resample: np.ndarray, temperature: float, threads: int = 1,
           b_range: tuple[int, int] | None = None) -> dict:
    """Run the oracle over a batch.

    ``target`` is [B, gamma+1, V], ``draft`` is [B, gamma, V] (float32, or
    uint16 bf16 bits), ``tokens`` int32 [B, gamma], ``u_accept`` float32
    [B, gamma], ``u_resample`` float32 [B].  ``threads`` splits the batch's
    sequences over host threads (the C call releases the GIL); ``b_range``
    restricts the work to sequences [lo, hi).  Returns a dict of numpy arrays
    named like the fields of ``oracle_result`` plus ``errors``.
    """
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    u_accept = np.ascontiguousarray(u_accept, dtype=np.float32)
    u_resample = np.ascontiguousarray(u_resample, dtype=np.float32)
    B, Gp1, V = target.shape
    G = Gp1 - 1
    if draft.shape != (B, G, V) or draft.dtype != target.dtype:
        raise ValueError("draft logits must be [B, gamma, V] with the target's dtype")
    if tokens.shape != (B, G) or u_accept.shape != (B, G) or u_resample.shape != (B,):
        raise ValueError("tokens/u_accept must be [B, gamma] and u_resample [B]")
    lo, hi = (0, B) if b_range is None else b_range
    out = {
        "out_tokens": np.full((B, G + 1), -1, np.int32),
        "out_num_accepted": np.zeros(B, np.int32),
        "seq_status": np.zeros(B, np.int32),
        "target_max": np.full((B, G + 1), np.nan),
        "target_sum": np.full((B, G + 1), np.nan),
        "draft_max": np.full((B, G), np.nan),
        "draft_sum": np.full((B, G), np.nan),
        "q_tok": np.full((B, G), np.nan),
        "p_tok": np.full((B, G), np.nan),
        "ratio": np.full((B, G), np.nan),
        "accept_margin": np.full((B, G), np.nan),
        "resid_mass": np.full(B, np.nan),
        "cdf_margin_mass": np.full(B, np.nan),
        "cdf_margin_norm": np.full(B, np.nan),
        "sampled": np.full(B, -1, np.int32),
    }
    prob = _Problem(B, G, V, _dtype_code(target), _ptr(target), _ptr(draft), _ptr(tokens),
                    _ptr(u_accept), _ptr(u_resample), float(temperature))
    res = _Result(*[_ptr(out[name]) for name in _RESULT_FIELDS])
    lib = _load()
    threads = max(1, min(int(threads), hi - lo)) if hi > lo else 1
    if threads == 1:
        errs = [lib.oracle_verify(ctypes.byref(prob), ctypes.byref(res), lo, hi)]
    else:
        bounds = np.linspace(lo, hi, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            errs = list(ex.map(
                lambda k: lib.oracle_verify(ctypes.byref(prob), ctypes.byref(res),
                                            int(bounds[k]), int(bounds[k + 1])),
                range(threads)))
    if any(e < 0 for e in errs):
        raise MemoryError("oracle could not allocate its row buffers")
    out["errors"] = int(sum(errs))
    return out


def gate(hidden: np.ndarray, parent: np.ndarray, tau: float) -> dict:
    """The multi-branch fold gate (``gate.c``) on hidden states [branches, positions, dim]
    (float32, or uint16 bf16 bits) with one parent index per branch (-1: none).

    Returns numpy arrays ``rel_diff``, ``margin`` (float64 [branches, positions]),
    ``recompute``, ``provenance``, ``source`` (int32 [branches, positions]),
    ``packed`` (int32 [n_packed]), ``parent_used`` (int32 [branches]) and
    ``status`` (GATE_OK or GATE_ERR_PARENT).
    """
    hidden = np.ascontiguousarray(hidden)
    parent = np.ascontiguousarray(parent, dtype=np.int32)
    nb, npos, dim = hidden.shape
    if parent.shape != (nb,):
        raise ValueError("parent must hold one entry per branch")
    out = {
        "rel_diff": np.empty((nb, npos), np.float64),
        "margin": np.empty((nb, npos), np.float64),
        "recompute": np.empty((nb, npos), np.int32),
        "provenance": np.empty((nb, npos), np.int32),
        "source": np.empty((nb, npos), np.int32),
        "packed": np.empty(max(1, nb * npos), np.int32),
        "n_packed": np.zeros(1, np.int32),
        "parent_used": np.empty(max(1, nb), np.int32),
    }
    prob = _GateProblem(nb, npos, dim, _dtype_code(hidden), _ptr(hidden), _ptr(parent), float(tau))
    res = _GateResult(*[_ptr(out[name]) for name in _GATE_FIELDS])
    st = _load().oracle_gate(ctypes.byref(prob), ctypes.byref(res))
    if st < 0:
        raise MemoryError("oracle could not allocate its buffers")
    n = int(out.pop("n_packed")[0])
    out["packed"] = out["packed"][:n]
    out["parent_used"] = out["parent_used"][:nb]
    out["status"] = st
    return out


def verify_sampling(target: np.ndarray, draft: np.ndarray, tokens: np.ndarray,
                    u_accept: np.ndarray, u_resample: np.ndarray, temperature,
                    top_k: int = 0, top_p: float = 1.0, threads: int = 1,
                    b_range: tuple[int, int] | None = None) -> dict:
    """The verification step on adjusted distributions (``sampling.c``): a
    temperature per sequence (0: greedy), top-k (0: off) and top-p (1: off)
    applied to every target and draft row.  Shapes as in ``verify``;
    ``temperature`` is a scalar or float32 [B]."""
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    u_accept = np.ascontiguousarray(u_accept, dtype=np.float32)
    u_resample = np.ascontiguousarray(u_resample, dtype=np.float32)
    B, Gp1, V = target.shape
    G = Gp1 - 1
    temps = np.ascontiguousarray(np.broadcast_to(np.asarray(temperature, np.float32), (B,)))
    if draft.shape != (B, G, V) or draft.dtype != target.dtype:
        raise ValueError("draft logits must be [B, gamma, V] with the target's dtype")
    lo, hi = (0, B) if b_range is None else b_range
    out = {
        "out_tokens": np.full((B, G + 1), -1, np.int32),
        "out_num_accepted": np.zeros(B, np.int32),
        "seq_status": np.zeros(B, np.int32),
        "q_tok": np.full((B, G), np.nan),
        "p_tok": np.full((B, G), np.nan),
        "accept_margin": np.full((B, G), np.nan),
        "resid_mass": np.full(B, np.nan),
        "cdf_margin_norm": np.full(B, np.nan),
        "kept_target": np.zeros((B, G + 1), np.int32),
        "kept_draft": np.zeros((B, G), np.int32),
        "filter_margin": np.full(B, np.inf),
    }
    prob = _SampProblem(B, G, V, _dtype_code(target), _ptr(target), _ptr(draft), _ptr(tokens),
                        _ptr(u_accept), _ptr(u_resample), _ptr(temps), int(top_k), float(top_p))
    res = _SampResult(*[_ptr(out[name]) for name in _SAMP_FIELDS])
    lib = _load()
    threads = max(1, min(int(threads), hi - lo)) if hi > lo else 1
    bounds = np.linspace(lo, hi, threads + 1).astype(int)
    with ThreadPoolExecutor(threads) as ex:
        errs = list(ex.map(
            lambda k: lib.oracle_verify_sampling(ctypes.byref(prob), ctypes.byref(res),
                                                 int(bounds[k]), int(bounds[k + 1])),
            range(threads)))
    if any(e < 0 for e in errs):
        raise MemoryError("oracle could not allocate its row buffers")
    out["errors"] = int(sum(errs))
    return out
