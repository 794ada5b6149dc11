"""Thin Python binding of ``libspecverify.so`` (the C ABI in include/specverify.h).

Argument marshalling only: every step of the verification runs in the CUDA
library.  The functions keep the C names; ``SpecVerify`` wraps a handle and
takes torch tensors (device memory and streams come from PyTorch).

Importing this module loads the library and fails loudly if it has not been
built (``python -m speculative_decoding_verification_90_b200.build``).  There
is no CPU fallback.  With SPECVERIFY_DEBUG_BOUNDS=1 in the environment it
loads ``libspecverify_debug.so`` instead: the same library compiled with
device bounds checks that report SV_ERR_BOUNDS instead of touching memory
outside a buffer.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
DEBUG_BOUNDS = os.environ.get("SPECVERIFY_DEBUG_BOUNDS", "0") == "1"
LIB_PATH = os.path.join(_PKG, "libspecverify_debug.so" if DEBUG_BOUNDS else "libspecverify.so")

SV_DTYPE_F32 = 0
SV_DTYPE_BF16 = 1

SV_OK = 0
SV_ERR_INVALID_ARG = 1
SV_ERR_CUDA = 2
SV_ERR_OOM = 3
SV_ERR_UNSUPPORTED = 4
SV_ERR_TOKEN_RANGE = 16
SV_ERR_NONFINITE = 17
SV_WARN_ZERO_MASS = 18
SV_ERR_ROW_INDEX = 19
SV_ERR_PARENT = 20
SV_ERR_TEMPERATURE = 21
SV_ERR_PIPELINE = 22
SV_ERR_BOUNDS = 23

# every function declared in include/*.h, with its ctypes signature
_vp, _i, _f, _u32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_uint32)
SIGNATURES = {
    "specverify_create": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i]),
    "specverify_run": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp]),
    "specverify_run_host": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp]),
    "specverify_run_sampling": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp]),
    "specverify_debug_kept": (_i, [_vp, _vp, _vp, _vp]),
    "specverify_run_mapped": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                                   _vp]),
    "specverify_destroy": (None, [_vp]),
    "specverify_get_status": (_i, [_vp, _vp, _u32p]),
    "specverify_debug_readback": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "specverify_set_launch": (_i, [_vp, _i, _i, _i]),
    "specverify_get_launch": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i),
                                   ctypes.POINTER(_i)]),
    "specverify_kernels_per_run": (_i, [_vp, _i, ctypes.POINTER(_i)]),
    "specverify_set_fused": (_i, [_vp, _i, _i, _i, _i]),
    "specverify_get_fused": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i),
                                  ctypes.POINTER(_i)]),
    "specverify_profile_begin": (_i, [_vp, _i]),
    "specverify_profile_end": (_i, [_vp, ctypes.POINTER(_f), ctypes.POINTER(_f), ctypes.POINTER(_i)]),
    "specverify_run_noalloc": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp]),
    "specfold_gate_create": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i]),
    "specfold_gate_run": (_i, [_vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "specfold_gate_get_status": (_i, [_vp, _vp, _u32p]),
    "specfold_gate_profile_begin": (_i, [_vp, _i]),
    "specfold_gate_profile_end": (_i, [_vp, ctypes.POINTER(_f), ctypes.POINTER(_f),
                                       ctypes.POINTER(_i)]),
    "specfold_gate_destroy": (None, [_vp]),
    "specverify_lmhead_create": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i]),
    "specverify_lmhead_run": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp]),
    "specverify_lmhead_logits": (_i, [_vp, _vp, _i, _vp, _vp, _vp]),
    "specverify_lmhead_get_status": (_i, [_vp, _vp, _u32p]),
    "specverify_lmhead_readback": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "specverify_lmhead_profile_begin": (_i, [_vp, _i]),
    "specverify_lmhead_profile_end": (_i, [_vp, ctypes.POINTER(_f), ctypes.POINTER(_f),
                                           ctypes.POINTER(_i)]),
    "specverify_lmhead_destroy": (None, [_vp]),
    "specverify_lmhead_set_keep_logits": (_i, [_vp, _i]),
    "specverify_lmhead_get_keep_logits": (_i, [_vp, ctypes.POINTER(_i)]),
    "specverify_status_string": (ctypes.c_char_p, [_i]),
    "specverify_last_error": (ctypes.c_char_p, []),
}


def _load_library():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m speculative_decoding_verification_90_b200.build` (nvcc, sm_100a). "
            "There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load_library()


class SpecVerifyError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.specverify_status_string(status).decode()
        extra = _lib.specverify_last_error().decode()
        super().__init__(f"{where}: {msg} (status {status})" + (f" [{extra}]" if extra else ""))
        self.status = status


def _check(status: int, where: str) -> int:
    if status != SV_OK:
        raise SpecVerifyError(status, where)
    return status


# ---- the C entry points, one Python function each (raw pointers as ints) ----

def specverify_create(batch: int, gamma: int, vocab: int, dtype: int, device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(_lib.specverify_create(ctypes.byref(h), batch, gamma, vocab, dtype, device),
           "specverify_create")
    return h.value


def specverify_run(h, target, draft, tokens, u_accept, u_resample, temperature, out_tokens,
                   out_num_accepted, stream=0) -> int:
    return _check(_lib.specverify_run(h, target, draft, tokens, u_accept, u_resample,
                                      float(temperature), out_tokens, out_num_accepted, stream),
                  "specverify_run")


def specverify_run_host(h, target, draft, tokens, u_accept, u_resample, temperature, out_tokens,
                        out_num_accepted, stream=0) -> int:
    return _check(_lib.specverify_run_host(h, target, draft, tokens, u_accept, u_resample,
                                           float(temperature), out_tokens, out_num_accepted,
                                           stream),
                  "specverify_run_host")


def specverify_run_mapped(h, target_rows, n_target_rows, target_map, draft_rows, n_draft_rows,
                          draft_map, tokens, u_accept, u_resample, temperature, out_tokens,
                          out_num_accepted, stream=0) -> int:
    return _check(_lib.specverify_run_mapped(h, target_rows, n_target_rows, target_map, draft_rows,
                                             n_draft_rows, draft_map, tokens, u_accept, u_resample,
                                             float(temperature), out_tokens, out_num_accepted,
                                             stream),
                  "specverify_run_mapped")


def specverify_run_sampling(h, target, draft, tokens, u_accept, u_resample, temperatures, top_k,
                            top_p, out_tokens, out_num_accepted, stream=0) -> int:
    return _check(_lib.specverify_run_sampling(h, target, draft, tokens, u_accept, u_resample,
                                               temperatures, int(top_k), float(top_p), out_tokens,
                                               out_num_accepted, stream),
                  "specverify_run_sampling")


def specverify_debug_kept(h, kept_target, kept_draft, stream=0) -> int:
    return _check(_lib.specverify_debug_kept(h, kept_target, kept_draft, stream),
                  "specverify_debug_kept")


def specverify_destroy(h) -> None:
    _lib.specverify_destroy(h)


def specverify_get_status(h, stream=0) -> tuple[int, int]:
    bits = ctypes.c_uint32()
    st = _lib.specverify_get_status(h, stream, ctypes.byref(bits))
    if st in (SV_ERR_INVALID_ARG, SV_ERR_CUDA, SV_ERR_OOM, SV_ERR_UNSUPPORTED):
        _check(st, "specverify_get_status")
    return st, bits.value


def specverify_debug_readback(h, *ptrs, stream=0) -> int:
    return _check(_lib.specverify_debug_readback(h, *ptrs, stream), "specverify_debug_readback")


def specverify_set_launch(h, slices: int, threads: int, draw_slices: int = 0) -> int:
    return _check(_lib.specverify_set_launch(h, slices, threads, draw_slices),
                  "specverify_set_launch")


def specverify_get_launch(h) -> tuple[int, int, int, int]:
    """(slices, threads, max_slices, draw_slices) of the handle."""
    c, t, m, k = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(_lib.specverify_get_launch(h, ctypes.byref(c), ctypes.byref(t), ctypes.byref(m),
                                      ctypes.byref(k)), "specverify_get_launch")
    return c.value, t.value, m.value, k.value


def specverify_kernels_per_run(h, mapped: bool = False) -> int:
    """Kernels one run of the handle enqueues."""
    k = ctypes.c_int()
    _check(_lib.specverify_kernels_per_run(h, 1 if mapped else 0, ctypes.byref(k)),
           "specverify_kernels_per_run")
    return k.value


def specverify_set_fused(h, enable: bool, unit_groups: int = 0, chunk_tiles: int = 0,
                         lag: int = -1) -> int:
    return _check(_lib.specverify_set_fused(h, 1 if enable else 0, unit_groups, chunk_tiles, lag),
                  "specverify_set_fused")


def specverify_get_fused(h) -> tuple[int, int, int, int]:
    """(enabled for an aligned unmapped run, unit_groups, chunk_tiles, lag) of the handle."""
    e, u, c, g = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(_lib.specverify_get_fused(h, ctypes.byref(e), ctypes.byref(u), ctypes.byref(c),
                                     ctypes.byref(g)), "specverify_get_fused")
    return e.value, u.value, c.value, g.value


def specverify_profile_begin(h, max_runs: int) -> int:
    return _check(_lib.specverify_profile_begin(h, max_runs), "specverify_profile_begin")


def specverify_profile_end(h) -> dict:
    """Mean device milliseconds per run of each kernel since profile_begin."""
    a, c, n = ctypes.c_float(), ctypes.c_float(), ctypes.c_int()
    _check(_lib.specverify_profile_end(h, ctypes.byref(a), ctypes.byref(c), ctypes.byref(n)),
           "specverify_profile_end")
    return {"stats_ms": a.value, "draw_ms": c.value, "runs": n.value}


def specverify_run_noalloc(batch, gamma, vocab, dtype, target, draft, tokens, u_accept, u_resample,
                           temperature, out_tokens, out_num_accepted, stream=0) -> int:
    """The step without a handle; its workspace is a static device array (no allocation)."""
    return _check(_lib.specverify_run_noalloc(batch, gamma, vocab, dtype, target, draft, tokens,
                                              u_accept, u_resample, float(temperature), out_tokens,
                                              out_num_accepted, stream),
                  "specverify_run_noalloc")


def specfold_gate_create(branches: int, positions: int, dim: int, dtype: int,
                         device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(_lib.specfold_gate_create(ctypes.byref(h), branches, positions, dim, dtype, device),
           "specfold_gate_create")
    return h.value


def specfold_gate_run(h, hidden, parent, tau, rel_diff, provenance, source, packed_rows,
                      n_packed, packed_hidden, stream=0) -> int:
    return _check(_lib.specfold_gate_run(h, hidden, parent, float(tau), rel_diff, provenance,
                                         source, packed_rows, n_packed, packed_hidden, stream),
                  "specfold_gate_run")


def specfold_gate_get_status(h, stream=0) -> tuple[int, int]:
    bits = ctypes.c_uint32()
    st = _lib.specfold_gate_get_status(h, stream, ctypes.byref(bits))
    if st in (SV_ERR_INVALID_ARG, SV_ERR_CUDA, SV_ERR_OOM, SV_ERR_UNSUPPORTED):
        _check(st, "specfold_gate_get_status")
    return st, bits.value


def specfold_gate_profile_begin(h, max_runs: int) -> int:
    return _check(_lib.specfold_gate_profile_begin(h, max_runs), "specfold_gate_profile_begin")


def specfold_gate_profile_end(h) -> dict:
    """Mean device milliseconds per run of the difference and packing kernels."""
    a, c, n = ctypes.c_float(), ctypes.c_float(), ctypes.c_int()
    _check(_lib.specfold_gate_profile_end(h, ctypes.byref(a), ctypes.byref(c), ctypes.byref(n)),
           "specfold_gate_profile_end")
    return {"rows_ms": a.value, "pack_ms": c.value, "runs": n.value}


def specfold_gate_destroy(h) -> None:
    _lib.specfold_gate_destroy(h)


def specverify_lmhead_create(batch, gamma, vocab, hidden, device=0) -> int:
    h = ctypes.c_void_p()
    _check(_lib.specverify_lmhead_create(ctypes.byref(h), batch, gamma, vocab, hidden, device),
           "specverify_lmhead_create")
    return h.value


def specverify_lmhead_run(h, target_hidden, target_weight, draft_hidden, draft_weight, tokens,
                          u_accept, u_resample, temperature, out_tokens, out_num_accepted,
                          stream=0) -> int:
    return _check(_lib.specverify_lmhead_run(h, target_hidden, target_weight, draft_hidden,
                                             draft_weight, tokens, u_accept, u_resample,
                                             float(temperature), out_tokens, out_num_accepted,
                                             stream),
                  "specverify_lmhead_run")


def specverify_lmhead_logits(h, hidden_rows, rows, weight, out_logits, stream=0) -> int:
    return _check(_lib.specverify_lmhead_logits(h, hidden_rows, rows, weight, out_logits, stream),
                  "specverify_lmhead_logits")


def specverify_lmhead_get_status(h, stream=0) -> tuple[int, int]:
    bits = ctypes.c_uint32()
    st = _lib.specverify_lmhead_get_status(h, stream, ctypes.byref(bits))
    if st in (SV_ERR_INVALID_ARG, SV_ERR_CUDA, SV_ERR_OOM, SV_ERR_UNSUPPORTED):
        _check(st, "specverify_lmhead_get_status")
    return st, bits.value


def specverify_lmhead_readback(h, *ptrs, stream=0) -> int:
    return _check(_lib.specverify_lmhead_readback(h, *ptrs, stream), "specverify_lmhead_readback")


def specverify_lmhead_profile_begin(h, max_runs: int) -> int:
    return _check(_lib.specverify_lmhead_profile_begin(h, max_runs),
                  "specverify_lmhead_profile_begin")


def specverify_lmhead_profile_end(h) -> dict:
    a, c, n = ctypes.c_float(), ctypes.c_float(), ctypes.c_int()
    _check(_lib.specverify_lmhead_profile_end(h, ctypes.byref(a), ctypes.byref(c),
                                              ctypes.byref(n)), "specverify_lmhead_profile_end")
    return {"stats_ms": a.value, "rest_ms": c.value, "runs": n.value}


def specverify_lmhead_set_keep_logits(h, keep: bool) -> int:
    return _check(_lib.specverify_lmhead_set_keep_logits(h, 1 if keep else 0),
                  "specverify_lmhead_set_keep_logits")


def specverify_lmhead_get_keep_logits(h) -> bool:
    k = ctypes.c_int()
    _check(_lib.specverify_lmhead_get_keep_logits(h, ctypes.byref(k)),
           "specverify_lmhead_get_keep_logits")
    return bool(k.value)


def specverify_lmhead_destroy(h) -> None:
    _lib.specverify_lmhead_destroy(h)


def specverify_status_string(status: int) -> str:
    return _lib.specverify_status_string(status).decode()


def specverify_last_error() -> str:
    return _lib.specverify_last_error().decode()


# ---- tensor-level wrapper ----

class SpecVerify:
    """A handle for fixed (batch, gamma, vocab, dtype) on one CUDA device.

    ``run`` takes torch CUDA tensors and enqueues on the current torch stream
    (or ``stream``); ``run_host`` takes host numpy arrays or CPU tensors.
    """

    def __init__(self, batch: int, gamma: int, vocab: int, dtype: str = "bf16", device: int = 0):
        self.batch, self.gamma, self.vocab, self.dtype = batch, gamma, vocab, dtype
        self.device = device
        code = {"f32": SV_DTYPE_F32, "bf16": SV_DTYPE_BF16}[dtype]
        self.handle = specverify_create(batch, gamma, vocab, code, device)

    def close(self):
        if getattr(self, "handle", None):
            specverify_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # shapes the C ABI expects
    def _shapes(self):
        B, G, V = self.batch, self.gamma, self.vocab
        return {"target": (B, G + 1, V), "draft": (B, G, V), "tokens": (B, G),
                "u_accept": (B, G), "u_resample": (B,), "temperatures": (B,),
                "out_tokens": (B, G + 1),
                "out_num_accepted": (B,)}

    def _check_tensor(self, name, t, dtype, cuda):
        import torch
        want = self._shapes()[name]
        if tuple(t.shape) != want:
            raise ValueError(f"{name}: shape {tuple(t.shape)} != {want}")
        if t.dtype != dtype:
            raise ValueError(f"{name}: dtype {t.dtype} != {dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        if cuda and (t.device.type != "cuda" or t.device.index != self.device):
            raise ValueError(f"{name}: must live on cuda:{self.device}")
        if not cuda and t.device.type != "cpu":
            raise ValueError(f"{name}: must be a host tensor")
        return t.data_ptr() if t.numel() else 0

    def _logit_dtype(self):
        import torch
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def run(self, target, draft, tokens, u_accept, u_resample, temperature, out_tokens,
            out_num_accepted, stream=None):
        import torch
        ld = self._logit_dtype()
        ptrs = [self._check_tensor("target", target, ld, True),
                self._check_tensor("draft", draft, ld, True),
                self._check_tensor("tokens", tokens, torch.int32, True),
                self._check_tensor("u_accept", u_accept, torch.float32, True),
                self._check_tensor("u_resample", u_resample, torch.float32, True)]
        outs = [self._check_tensor("out_tokens", out_tokens, torch.int32, True),
                self._check_tensor("out_num_accepted", out_num_accepted, torch.int32, True)]
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specverify_run(self.handle, *ptrs, temperature, *outs, sp)

    def run_mapped(self, target_rows, target_map, draft_rows, draft_map, tokens, u_accept,
                   u_resample, temperature, out_tokens, out_num_accepted, stream=None):
        """Shared-row step: ``target_rows[target_map[b, j]]`` is position (b, j)'s target row."""
        import torch
        B, G, V = self.batch, self.gamma, self.vocab
        ld = self._logit_dtype()

        def rows(name, t, cap):
            if t.dim() != 2 or t.shape[1] != V or not 1 <= t.shape[0] <= cap:
                raise ValueError(f"{name}: shape {tuple(t.shape)} is not [1..{cap}, {V}]")
            if t.dtype != ld or not t.is_contiguous() or t.device.type != "cuda" \
                    or t.device.index != self.device:
                raise ValueError(f"{name}: must be a contiguous {ld} tensor on cuda:{self.device}")
            return t.data_ptr(), t.shape[0]

        def index(name, t, shape):
            if tuple(t.shape) != shape or t.dtype != torch.int32 or not t.is_contiguous() \
                    or t.device.type != "cuda" or t.device.index != self.device:
                raise ValueError(f"{name}: must be a contiguous int32 {shape} tensor on "
                                 f"cuda:{self.device}")
            return t.data_ptr() if t.numel() else 0

        tp, nt = rows("target_rows", target_rows, B * (G + 1))
        tm = index("target_map", target_map, (B, G + 1))
        if G > 0:
            dp, nd = rows("draft_rows", draft_rows, B * G)
            dm = index("draft_map", draft_map, (B, G))
        else:
            dp, nd, dm = 0, 0, 0
        ptrs = [self._check_tensor("tokens", tokens, torch.int32, True),
                self._check_tensor("u_accept", u_accept, torch.float32, True),
                self._check_tensor("u_resample", u_resample, torch.float32, True)]
        outs = [self._check_tensor("out_tokens", out_tokens, torch.int32, True),
                self._check_tensor("out_num_accepted", out_num_accepted, torch.int32, True)]
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specverify_run_mapped(self.handle, tp, nt, tm, dp, nd, dm, *ptrs, temperature, *outs, sp)

    def run_sampling(self, target, draft, tokens, u_accept, u_resample, temperatures, out_tokens,
                     out_num_accepted, top_k=0, top_p=1.0, stream=None):
        """Sampling variants: ``temperatures`` float32 [B] on the device (0: greedy)."""
        import torch
        ld = self._logit_dtype()
        ptrs = [self._check_tensor("target", target, ld, True),
                self._check_tensor("draft", draft, ld, True),
                self._check_tensor("tokens", tokens, torch.int32, True),
                self._check_tensor("u_accept", u_accept, torch.float32, True),
                self._check_tensor("u_resample", u_resample, torch.float32, True),
                self._check_tensor("temperatures", temperatures, torch.float32, True)]
        outs = [self._check_tensor("out_tokens", out_tokens, torch.int32, True),
                self._check_tensor("out_num_accepted", out_num_accepted, torch.int32, True)]
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specverify_run_sampling(self.handle, *ptrs, top_k, top_p, *outs, sp)

    def kept(self, stream=None):
        """Entries kept by each row's adjusted distribution after run_sampling."""
        import torch
        B, G = self.batch, self.gamma
        kt = np.zeros((B, G + 1), np.int32)
        kd = np.zeros((B, G), np.int32)
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specverify_debug_kept(self.handle, kt.ctypes.data, kd.ctypes.data if kd.size else None, sp)
        return kt, kd

    def run_host(self, target, draft, tokens, u_accept, u_resample, temperature, out_tokens,
                 out_num_accepted, stream=None):
        """Host buffers in and out (torch CPU tensors, ideally pinned); returns when done."""
        import torch
        ld = self._logit_dtype()
        ptrs = [self._check_tensor("target", target, ld, False),
                self._check_tensor("draft", draft, ld, False),
                self._check_tensor("tokens", tokens, torch.int32, False),
                self._check_tensor("u_accept", u_accept, torch.float32, False),
                self._check_tensor("u_resample", u_resample, torch.float32, False)]
        outs = [self._check_tensor("out_tokens", out_tokens, torch.int32, False),
                self._check_tensor("out_num_accepted", out_num_accepted, torch.int32, False)]
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specverify_run_host(self.handle, *ptrs, temperature, *outs, sp)

    def status(self, stream=None) -> tuple[int, int]:
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        return specverify_get_status(self.handle, sp)

    def set_launch(self, slices: int, threads: int, draw_slices: int = 0):
        specverify_set_launch(self.handle, slices, threads, draw_slices)

    @property
    def draw_slices(self) -> int:
        return specverify_get_launch(self.handle)[3]

    def launch(self) -> tuple[int, int]:
        """(slices per position, threads per block)."""
        return specverify_get_launch(self.handle)[:2]

    def kernels_per_run(self, mapped: bool = False) -> int:
        return specverify_kernels_per_run(self.handle, mapped)

    def set_fused(self, enable: bool, unit_groups: int = 0, chunk_tiles: int = 0, lag: int = -1):
        """Single launch (True) or three kernels (False) for aligned unmapped runs."""
        specverify_set_fused(self.handle, enable, unit_groups, chunk_tiles, lag)

    def fused(self) -> tuple[int, int, int, int]:
        return specverify_get_fused(self.handle)

    def profile_begin(self, max_runs: int):
        specverify_profile_begin(self.handle, max_runs)

    def profile_end(self) -> dict:
        return specverify_profile_end(self.handle)

    @property
    def max_slices(self) -> int:
        return specverify_get_launch(self.handle)[2]

    def readback(self, stream=None) -> dict:
        """Intermediate values of the last step (see specverify_debug_readback)."""
        import torch
        B, G = self.batch, self.gamma
        out = {"target_lse": np.zeros((B, G + 1), np.float64),
               "draft_lse": np.zeros((B, G), np.float64),
               "q_tok": np.zeros((B, G), np.float64),
               "p_tok": np.zeros((B, G), np.float64),
               "ratio": np.zeros((B, G), np.float64),
               "resid_mass": np.zeros(B, np.float64)}
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specverify_debug_readback(self.handle, *[a.ctypes.data for a in out.values()], stream=sp)
        return out


class FoldGate:
    """A fold-gate handle for fixed (branches, positions, dim, dtype) on one CUDA device.

    ``run`` takes torch CUDA tensors and enqueues on the current torch stream
    (or ``stream``).
    """

    def __init__(self, branches: int, positions: int, dim: int, dtype: str = "bf16",
                 device: int = 0):
        self.branches, self.positions, self.dim, self.dtype = branches, positions, dim, dtype
        self.device = device
        code = {"f32": SV_DTYPE_F32, "bf16": SV_DTYPE_BF16}[dtype]
        self.handle = specfold_gate_create(branches, positions, dim, code, device)

    def close(self):
        if getattr(self, "handle", None):
            specfold_gate_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _ptr(self, name, t, shape, dtype, optional=False):
        if t is None:
            if optional:
                return 0
            raise ValueError(f"{name} is required")
        if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous() \
                or t.device.type != "cuda" or t.device.index != self.device:
            raise ValueError(f"{name}: must be a contiguous {dtype} {shape} tensor on "
                             f"cuda:{self.device}")
        return t.data_ptr()

    def run(self, hidden, parent, tau, packed_rows, n_packed, rel_diff=None, provenance=None,
            source=None, packed_hidden=None, stream=None):
        import torch
        nb, npos, dim = self.branches, self.positions, self.dim
        hd = torch.bfloat16 if self.dtype == "bf16" else torch.float32
        rows = nb * npos
        args = [self._ptr("hidden", hidden, (nb, npos, dim), hd),
                self._ptr("parent", parent, (nb,), torch.int32), float(tau),
                self._ptr("rel_diff", rel_diff, (nb, npos), torch.float32, True),
                self._ptr("provenance", provenance, (nb, npos), torch.int32, True),
                self._ptr("source", source, (nb, npos), torch.int32, True),
                self._ptr("packed_rows", packed_rows, (rows,), torch.int32),
                self._ptr("n_packed", n_packed, (1,), torch.int32),
                self._ptr("packed_hidden", packed_hidden, (rows, dim), hd, True)]
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        specfold_gate_run(self.handle, *args, sp)

    def status(self, stream=None) -> tuple[int, int]:
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        return specfold_gate_get_status(self.handle, sp)

    def profile_begin(self, max_runs: int):
        specfold_gate_profile_begin(self.handle, max_runs)

    def profile_end(self) -> dict:
        return specfold_gate_profile_end(self.handle)


class LmHeadVerify:
    """The verification step fused with the LM head, for fixed (batch, gamma,
    vocab, hidden) on one CUDA device; bf16 hidden states and weights."""

    def __init__(self, batch: int, gamma: int, vocab: int, hidden: int, device: int = 0):
        self.batch, self.gamma, self.vocab, self.hidden = batch, gamma, vocab, hidden
        self.device = device
        self.handle = specverify_lmhead_create(batch, gamma, vocab, hidden, device)

    def close(self):
        if getattr(self, "handle", None):
            specverify_lmhead_destroy(self.handle)
            self.handle = None

    @property
    def keep_logits(self) -> bool:
        """Whether the statistics GEMMs keep every row's logits for the draw."""
        return specverify_lmhead_get_keep_logits(self.handle)

    @keep_logits.setter
    def keep_logits(self, keep: bool):
        specverify_lmhead_set_keep_logits(self.handle, keep)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _t(self, name, t, shape, dtype):
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous() \
                or t.device.type != "cuda" or t.device.index != self.device:
            raise ValueError(f"{name}: must be a contiguous {dtype} {tuple(shape)} tensor on "
                             f"cuda:{self.device}")
        return t.data_ptr() if t.numel() else 0

    def _stream(self, stream):
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)

    def run(self, target_hidden, target_weight, draft_hidden, draft_weight, tokens, u_accept,
            u_resample, temperature, out_tokens, out_num_accepted, stream=None):
        import torch
        B, G, V, D = self.batch, self.gamma, self.vocab, self.hidden
        bf = torch.bfloat16
        args = [self._t("target_hidden", target_hidden, (B, G + 1, D), bf),
                self._t("target_weight", target_weight, (V, D), bf),
                self._t("draft_hidden", draft_hidden, (B, G, D), bf),
                self._t("draft_weight", draft_weight, (V, D), bf),
                self._t("tokens", tokens, (B, G), torch.int32),
                self._t("u_accept", u_accept, (B, G), torch.float32),
                self._t("u_resample", u_resample, (B,), torch.float32)]
        outs = [self._t("out_tokens", out_tokens, (B, G + 1), torch.int32),
                self._t("out_num_accepted", out_num_accepted, (B,), torch.int32)]
        specverify_lmhead_run(self.handle, *args, temperature, *outs, self._stream(stream))

    def logits(self, hidden_rows, weight, out, stream=None):
        import torch
        rows = hidden_rows.shape[0]
        specverify_lmhead_logits(
            self.handle, self._t("hidden_rows", hidden_rows, (rows, self.hidden), torch.bfloat16),
            rows, self._t("weight", weight, (self.vocab, self.hidden), torch.bfloat16),
            self._t("out", out, (rows, self.vocab), torch.float32), self._stream(stream))

    def status(self, stream=None) -> tuple[int, int]:
        return specverify_lmhead_get_status(self.handle, self._stream(stream))

    def readback(self, stream=None) -> dict:
        B, G = self.batch, self.gamma
        out = {"target_lse": np.zeros((B, G + 1)), "draft_lse": np.zeros((B, G)),
               "q_tok": np.zeros((B, G)), "p_tok": np.zeros((B, G)),
               "resid_mass": np.zeros(B)}
        specverify_lmhead_readback(self.handle, *[out[k].ctypes.data if out[k].size else None
                                                  for k in ("target_lse", "draft_lse", "q_tok",
                                                            "p_tok", "resid_mass")],
                                   stream=self._stream(stream))
        return out

    def profile_begin(self, max_runs: int):
        specverify_lmhead_profile_begin(self.handle, max_runs)

    def profile_end(self) -> dict:
        return specverify_lmhead_profile_end(self.handle)
