"""Oracle for the draft-sample-and-verify step -- TEST INFRASTRUCTURE ONLY.

A plain, slow, double-precision CPU implementation (``oracle.c``) of what the
CUDA path computes, loaded through ctypes.  Only the test suite, the smoke
check and the benchmark's CPU-baseline leg may import this package; the
product library never does, and the two share no source.

What is computed, the readings of the pages and the pins are documented in
``oracle.h``.  Functions here only marshal numpy arrays in and out.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

TAG_DRAFT, TAG_ACCEPT, TAG_RESAMPLE = 0, 1, 2
_DT = {"f32": 0, "bf16": 1}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP over batch rows)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                           os.path.getmtime(os.path.join(_HERE, "oracle.h"))))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("K", ctypes.c_int32), ("V", ctypes.c_int32),
                ("r", ctypes.c_int32), ("dtype", ctypes.c_int32), ("draft_dtype", ctypes.c_int32),
                ("temperature", ctypes.c_double), ("greedy", ctypes.c_int32),
                ("seed", ctypes.c_uint64), ("cycle", ctypes.c_uint64),
                ("verify_len", ctypes.c_void_p), ("Wh", ctypes.c_void_p)]


class _Outputs(ctypes.Structure):
    _fields_ = [("draft", ctypes.c_void_p), ("out", ctypes.c_void_p), ("tau", ctypes.c_void_p),
                ("p_draft", ctypes.c_void_p), ("q_draft", ctypes.c_void_p),
                ("flag_draft", ctypes.c_void_p), ("flag_accept", ctypes.c_void_p),
                ("flag_final", ctypes.c_void_p), ("biased", ctypes.c_void_p)]


_lib = None


def build_planted(plant: int, outdir: str):
    """Build a copy of the oracle with planted mistake number `plant` (see the
    ORC_PLANT hooks in oracle.c) into `outdir`; used only to show that the pins
    reject a wrong oracle."""
    path = os.path.join(outdir, f"liboracle_plant{plant}.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           f"-DORC_PLANT={int(plant)}", "-o", path, _SRC, "-lm"])
    h = ctypes.CDLL(path)
    h.orc_cycle.restype = ctypes.c_int
    return h


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.orc_u01.restype = ctypes.c_double
        _lib.orc_uniform.restype = ctypes.c_double
        _lib.orc_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                     ctypes.c_uint32, ctypes.c_uint32]
        _lib.orc_icdf.restype = ctypes.c_int32
        _lib.orc_verify_probs.restype = ctypes.c_int32
        for name in ("orc_cycle", "orc_draft", "orc_verify", "orc_biased_row"):
            getattr(_lib, name).restype = ctypes.c_int
    return _lib


@dataclass
class Params:
    B: int
    K: int
    V: int
    r: int
    dtype: str = "bf16"          # base, target, U, W: "bf16" or "f32"
    temperature: float = 1.0
    greedy: bool = False
    seed: int = 0
    cycle: int = 0
    draft_dtype: str | None = None  # verify-only: dtype of the given draft logits
    verify_len: np.ndarray | None = None  # [B] int32 per-row verify length K_b (1..K), or None
    Wh: np.ndarray | None = None  # [r, r] RNN head weights (raw storage of dtype), or None (Markov)

    def c(self) -> _Params:
        dd = self.draft_dtype or self.dtype
        # the temperature is the fp32 value the GPU receives, widened exactly
        T = float(np.float32(self.temperature))
        vl = None
        if self.verify_len is not None:
            self._vl = np.ascontiguousarray(self.verify_len, dtype=np.int32)  # kept alive
            vl = self._vl.ctypes.data_as(ctypes.c_void_p)
        wh = None
        if self.Wh is not None:
            self._wh = _raw(self.Wh, self.dtype)  # kept alive
            assert self._wh.size == self.r * self.r
            wh = self._wh.ctypes.data_as(ctypes.c_void_p)
        return _Params(self.B, self.K, self.V, self.r, _DT[self.dtype], _DT[dd], T,
                       1 if self.greedy else 0, self.seed & (2**64 - 1), self.cycle & (2**64 - 1),
                       vl, wh)


def _raw(a: np.ndarray, dtype: str) -> np.ndarray:
    """Contiguous raw storage: bf16 as uint16 bit patterns, f32 as float32."""
    if dtype == "bf16":
        if a.dtype != np.uint16:
            raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    elif a.dtype != np.float32:
        raise TypeError("f32 inputs are passed as float32")
    return np.ascontiguousarray(a)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _alloc_outputs(n, K, V=None, biased=False):
    o = dict(draft=np.full((n, K), -7, np.int32), out=np.full((n, K + 1), -7, np.int32),
             tau=np.zeros(n, np.int32), p_draft=np.full((n, K), np.nan),
             q_draft=np.full((n, K), np.nan), flag_draft=np.zeros(n, np.int32),
             flag_accept=np.zeros(n, np.int32), flag_final=np.zeros(n, np.int32))
    if biased:
        o["biased"] = np.zeros((n, K, V))
    c = _Outputs(*[_ptr(o.get(k)) for k in
                   ("draft", "out", "tau", "p_draft", "q_draft", "flag_draft", "flag_accept",
                    "flag_final", "biased")])
    return o, c


def cycle(P: Params, base, target, U, W, last_token, b_begin=0, b_end=None, handle=None):
    """Sequential Markov-biased drafting then verification, rows [b_begin, b_end)."""
    h = handle or lib()
    b_end = P.B if b_end is None else b_end
    base, target = _raw(base, P.dtype), _raw(target, P.dtype)
    U, W = _raw(U, P.dtype), _raw(W, P.dtype)
    lt = np.ascontiguousarray(last_token, dtype=np.int32)
    o, c = _alloc_outputs(b_end - b_begin, P.K)
    rc = h.orc_cycle(ctypes.byref(P.c()), _ptr(base), _ptr(target), _ptr(U), _ptr(W),
                     _ptr(lt), b_begin, b_end, ctypes.byref(c))
    if rc != 0:
        raise ValueError(f"orc_cycle failed: {rc}")
    o["threads"] = h.orc_threads_used()
    return o


def draft(P: Params, base, U, W, last_token, b_begin=0, b_end=None, biased=False):
    b_end = P.B if b_end is None else b_end
    base, U, W = _raw(base, P.dtype), _raw(U, P.dtype), _raw(W, P.dtype)
    lt = np.ascontiguousarray(last_token, dtype=np.int32)
    o, c = _alloc_outputs(b_end - b_begin, P.K, P.V, biased)
    rc = lib().orc_draft(ctypes.byref(P.c()), _ptr(base), _ptr(U), _ptr(W), _ptr(lt),
                         b_begin, b_end, ctypes.byref(c))
    if rc != 0:
        raise ValueError(f"orc_draft failed: {rc}")
    return o


def verify(P: Params, target, draft_logits, draft_tokens, b_begin=0, b_end=None):
    b_end = P.B if b_end is None else b_end
    target = _raw(target, P.dtype)
    dl = _raw(draft_logits, P.draft_dtype or P.dtype)
    dt = np.ascontiguousarray(draft_tokens, dtype=np.int32)
    o, c = _alloc_outputs(b_end - b_begin, P.K)
    rc = lib().orc_verify(ctypes.byref(P.c()), _ptr(target), _ptr(dl), _ptr(dt),
                          b_begin, b_end, ctypes.byref(c))
    if rc != 0:
        raise ValueError(f"orc_verify failed: {rc}")
    return o


def philox(ctr, key):
    c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
    out = (ctypes.c_uint32 * 4)()
    lib().orc_philox4x32_10(c, k, out)
    return [int(x) for x in out]


def u01(x: int) -> float:
    return lib().orc_u01(ctypes.c_uint32(x & 0xFFFFFFFF))


def uniform(seed, cyc, b, pos, tag) -> float:
    return lib().orc_uniform(seed & (2**64 - 1), cyc & (2**64 - 1), b, pos, tag)


def icdf(w, u):
    w = np.ascontiguousarray(w, dtype=np.float64)
    near = ctypes.c_int32(0)
    idx = lib().orc_icdf(_ptr(w), len(w), ctypes.c_double(u), ctypes.byref(near))
    return int(idx), bool(near.value)


def row_stats(x, T):
    x = np.ascontiguousarray(x, dtype=np.float64)
    m, Z = ctypes.c_double(), ctypes.c_double()
    lib().orc_row_stats(_ptr(x), len(x), ctypes.c_double(T), ctypes.byref(m), ctypes.byref(Z))
    return m.value, Z.value


def verify_probs(p, q, d, u_acc, u_res):
    """The verification rule on explicit probabilities and uniforms."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    q = np.ascontiguousarray(q, dtype=np.float64)
    K, V = q.shape
    assert p.shape == (K + 1, V)
    d = np.ascontiguousarray(d, dtype=np.int32)
    ua = np.ascontiguousarray(u_acc, dtype=np.float64)
    ur = np.ascontiguousarray(u_res, dtype=np.float64)
    out = np.zeros(K + 1, np.int32)
    tau = ctypes.c_int32()
    pd = np.zeros(K)
    fa, ff = ctypes.c_int32(), ctypes.c_int32()
    lib().orc_verify_probs(K, V, _ptr(p), _ptr(q), _ptr(d), _ptr(ua), _ptr(ur), _ptr(out),
                           ctypes.byref(tau), _ptr(pd), ctypes.byref(fa), ctypes.byref(ff))
    return dict(out=out, tau=tau.value, p_draft=pd, flag_accept=fa.value, flag_final=ff.value)


def biased_row(P: Params, base, U, W, b, i, prev):
    z = np.zeros(P.V)
    rc = lib().orc_biased_row(ctypes.byref(P.c()), _ptr(_raw(base, P.dtype)),
                              _ptr(_raw(U, P.dtype)), _ptr(_raw(W, P.dtype)), b, i, prev, _ptr(z))
    if rc != 0:
        raise ValueError("orc_biased_row failed")
    return z
