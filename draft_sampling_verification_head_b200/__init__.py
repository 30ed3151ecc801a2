"""Thin Python binding of libspecdec.so (include/specdec.h).

Argument marshalling only: every step of the method runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  The
library must have been built (``build.py``); importing this module on a
machine without it raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libspecdec.so")

SPEC_OK, SPEC_ERR_INVALID_ARG, SPEC_ERR_UNSUPPORTED, SPEC_ERR_CUDA = 0, -1, -2, -3
SPEC_ERR_TIMEOUT, SPEC_ERR_WORKSPACE, SPEC_ERR_TOKEN_RANGE = -4, -5, -6
SPEC_F32, SPEC_BF16 = 0, 1
SPEC_FLAG_FMA_BIAS = 1
SPEC_FLAG_TRACE = 2

# (name, restype, argtypes) of every exported symbol declared in include/*.h
_P = ctypes.c_void_p
_SIGS = {
    "spec_workspace_size": (ctypes.c_size_t, [_P]),
    "spec_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "spec_markov_bias": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P]),
    "spec_markov_bias_sample": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_verify_block": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_verify_block_kb": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_cycle": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_cycle_kb": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_decode_loop": (ctypes.c_int, [_P, ctypes.c_int32, _P, _P, _P, ctypes.c_float, _P, _P, _P,
                                         _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_cycle_rnn": (ctypes.c_int, [_P] * 14),
    "spec_sync_status": (ctypes.c_int, [_P, _P]),
    "spec_cycle_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "spec_l2_persist": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "spec_schedule_verify_len": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P,
                                                 ctypes.c_int32, _P, _P]),
    "spec_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "spec_last_launch_count": (ctypes.c_int32, []),
    "spec_debug_philox": (ctypes.c_int, [_P, _P, _P, ctypes.c_int32, _P]),
    "spec_debug_curand_philox": (ctypes.c_int, [_P, _P, _P, ctypes.c_int32, _P]),
}


class SpecParams(ctypes.Structure):
    """Mirror of spec_params."""
    _fields_ = [("B", ctypes.c_int32), ("K", ctypes.c_int32), ("V", ctypes.c_int32),
                ("r", ctypes.c_int32), ("dtype", ctypes.c_int32), ("draft_dtype", ctypes.c_int32),
                ("temperature", ctypes.c_float), ("greedy", ctypes.c_int32),
                ("seed", ctypes.c_uint64), ("cycle", ctypes.c_uint64),
                ("spin_limit", ctypes.c_uint64), ("flags", ctypes.c_uint32),
                ("row_offset", ctypes.c_uint32)]


_lib = None


def lib():
    """Load libspecdec.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run draft_sampling_verification_head_b200/build.py")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


class SpecError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


def status_string(code: int) -> str:
    return lib().spec_status_string(code).decode()


@dataclass
class Params:
    B: int
    K: int
    V: int
    r: int
    dtype: str = "bf16"
    temperature: float = 1.0
    greedy: bool = False
    seed: int = 0
    cycle: int = 0
    spin_limit: int = 0
    flags: int = 0
    draft_dtype: str | None = None
    row_offset: int = 0  # global index of batch row 0 (Philox counter word 1)

    def c(self) -> SpecParams:
        dt = {"f32": SPEC_F32, "bf16": SPEC_BF16}
        return SpecParams(self.B, self.K, self.V, self.r, dt[self.dtype],
                          dt[self.draft_dtype or self.dtype], float(self.temperature),
                          1 if self.greedy else 0, self.seed & (2**64 - 1),
                          self.cycle & (2**64 - 1), self.spin_limit, self.flags,
                          self.row_offset)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, what):
    if code != SPEC_OK:
        raise SpecError(code, what)


def workspace_size(p: Params) -> int:
    return int(lib().spec_workspace_size(ctypes.byref(p.c())))


def make_workspace(p: Params, device="cuda"):
    """Allocate and zero a workspace for these parameters (torch memory)."""
    import torch
    n = workspace_size(p)
    if n == 0:
        raise SpecError(SPEC_ERR_INVALID_ARG, "spec_workspace_size")
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    _check(lib().spec_workspace_init(_ptr(ws), n, _stream(None)), "spec_workspace_init")
    return ws


def workspace_init(ws, stream=None):
    _check(lib().spec_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "spec_workspace_init")


def markov_bias(p: Params, U, W, prev, bias, ws, stream=None):
    _check(lib().spec_markov_bias(ctypes.byref(p.c()), _ptr(U), _ptr(W), _ptr(prev), _ptr(bias),
                                  _ptr(ws), _stream(stream)), "spec_markov_bias")


def markov_bias_sample(p: Params, base, U, W, last_token, draft, q_draft, biased_out, ws,
                       stream=None):
    _check(lib().spec_markov_bias_sample(ctypes.byref(p.c()), _ptr(base), _ptr(U), _ptr(W),
                                         _ptr(last_token), _ptr(draft), _ptr(q_draft),
                                         _ptr(biased_out), _ptr(ws), _stream(stream)),
           "spec_markov_bias_sample")


def verify_block(p: Params, target, draft_logits, draft, out, tau, p_draft, q_draft, ws,
                 stream=None):
    _check(lib().spec_verify_block(ctypes.byref(p.c()), _ptr(target), _ptr(draft_logits),
                                   _ptr(draft), _ptr(out), _ptr(tau), _ptr(p_draft),
                                   _ptr(q_draft), _ptr(ws), _stream(stream)), "spec_verify_block")


def verify_block_kb(p: Params, target, draft_logits, draft, verify_len, out, tau, p_draft, q_draft,
                    ws, stream=None):
    """spec_verify_block_kb: verification with a verify length K_b per row."""
    _check(lib().spec_verify_block_kb(ctypes.byref(p.c()), _ptr(target), _ptr(draft_logits),
                                      _ptr(draft), _ptr(verify_len), _ptr(out), _ptr(tau),
                                      _ptr(p_draft), _ptr(q_draft), _ptr(ws), _stream(stream)),
           "spec_verify_block_kb")


def cycle(p: Params, base, target, U, W, last_token, draft, out, tau, p_draft, q_draft, ws,
          stream=None):
    _check(lib().spec_cycle(ctypes.byref(p.c()), _ptr(base), _ptr(target), _ptr(U), _ptr(W),
                            _ptr(last_token), _ptr(draft), _ptr(out), _ptr(tau), _ptr(p_draft),
                            _ptr(q_draft), _ptr(ws), _stream(stream)), "spec_cycle")


def cycle_kb(p: Params, base, target, U, W, last_token, verify_len, draft, out, tau, p_draft,
             q_draft, ws, stream=None):
    """spec_cycle_kb: one cycle with a verify length K_b per row (int32 [B], 1..K)."""
    _check(lib().spec_cycle_kb(ctypes.byref(p.c()), _ptr(base), _ptr(target), _ptr(U), _ptr(W),
                               _ptr(last_token), _ptr(verify_len), _ptr(draft), _ptr(out),
                               _ptr(tau), _ptr(p_draft), _ptr(q_draft), _ptr(ws),
                               _stream(stream)), "spec_cycle_kb")


def decode_loop(p: Params, n_cycles, base, target, U, W, last_token, draft, out, tau, p_draft,
                q_draft, next_token, ws, conf=None, conf_threshold=0.0, verify_len=None,
                stream=None):
    """spec_decode_loop: n_cycles chained cycles in one launch; inputs and
    outputs carry a leading cycle axis, next_token [B] the last cycle's last
    emitted tokens."""
    _check(lib().spec_decode_loop(ctypes.byref(p.c()), int(n_cycles), _ptr(base), _ptr(target),
                                  _ptr(conf), float(conf_threshold), _ptr(verify_len), _ptr(U),
                                  _ptr(W), _ptr(last_token), _ptr(draft), _ptr(out), _ptr(tau),
                                  _ptr(p_draft), _ptr(q_draft), _ptr(next_token), _ptr(ws),
                                  _stream(stream)), "spec_decode_loop")


def cycle_rnn(p: Params, base, target, U, W, Wh, last_token, draft, out, tau, p_draft, q_draft, ws,
              stream=None):
    """spec_cycle_rnn: one cycle with the RNN sequential head (Wh [r, r] bf16)."""
    _check(lib().spec_cycle_rnn(ctypes.byref(p.c()), _ptr(base), _ptr(target), _ptr(U), _ptr(W),
                                _ptr(Wh), _ptr(last_token), _ptr(draft), _ptr(out), _ptr(tau),
                                _ptr(p_draft), _ptr(q_draft), _ptr(ws), _stream(stream)),
           "spec_cycle_rnn")


def cycle_noalloc(p: Params, base, target, U, W, last_token, draft, out, tau, p_draft, q_draft,
                  status_out=None, stream=None):
    """spec_cycle on the library's built-in scratch array (no workspace)."""
    _check(lib().spec_cycle_noalloc(ctypes.byref(p.c()), _ptr(base), _ptr(target), _ptr(U),
                                    _ptr(W), _ptr(last_token), _ptr(draft), _ptr(out), _ptr(tau),
                                    _ptr(p_draft), _ptr(q_draft), _ptr(status_out),
                                    _stream(stream)), "spec_cycle_noalloc")


def sync_status(ws, stream=None) -> int:
    return int(lib().spec_sync_status(_ptr(ws), _stream(stream)))


def l2_persist(t, nbytes=None, stream=None):
    """Keep tensor `t` (e.g. the Markov factor W) resident in L2 for kernels
    launched on the stream; t=None clears the window."""
    ptr = None if t is None else ctypes.c_void_p(t.data_ptr())
    n = 0 if t is None else (t.numel() * t.element_size() if nbytes is None else nbytes)
    _check(lib().spec_l2_persist(ptr, n, _stream(stream)), "spec_l2_persist")


def schedule_verify_len(conf, sps):
    """Verify length per request from confidence scores conf [B, K] and the
    steps-per-second table sps [n] (host arrays).  Returns (verify_len [B]
    int32, expected tokens per step, expected tokens per second)."""
    import numpy as np
    c = np.ascontiguousarray(conf, dtype=np.float32)
    s = np.ascontiguousarray(sps, dtype=np.float64)
    if c.ndim != 2 or s.ndim != 1:
        raise ValueError("conf must be [B, K] and sps one-dimensional")
    kb = np.empty(c.shape[0], np.int32)
    ex = np.zeros(2, np.float64)
    _check(lib().spec_schedule_verify_len(c.ctypes.data, c.shape[0], c.shape[1], s.ctypes.data,
                                          s.shape[0], kb.ctypes.data, ex.ctypes.data),
           "spec_schedule_verify_len")
    return kb, float(ex[0]), float(ex[1])


def last_launch_count() -> int:
    return int(lib().spec_last_launch_count())


def debug_philox(ctr, key, out, stream=None):
    _check(lib().spec_debug_philox(_ptr(ctr), _ptr(key), _ptr(out), ctr.shape[0],
                                   _stream(stream)), "spec_debug_philox")


def debug_curand_philox(ctr, key, out, stream=None):
    _check(lib().spec_debug_curand_philox(_ptr(ctr), _ptr(key), _ptr(out), ctr.shape[0],
                                          _stream(stream)), "spec_debug_curand_philox")


def alloc_outputs(p: Params, device="cuda", n_cycles=None):
    """Output tensors for one cycle, or with a leading axis of n_cycles."""
    import torch
    lead = () if n_cycles is None else (int(n_cycles),)
    return dict(draft=torch.full(lead + (p.B, p.K), -7, dtype=torch.int32, device=device),
                out=torch.full(lead + (p.B, p.K + 1), -7, dtype=torch.int32, device=device),
                tau=torch.zeros(lead + (p.B,), dtype=torch.int32, device=device),
                p_draft=torch.full(lead + (p.B, p.K), -1.0, dtype=torch.float32, device=device),
                q_draft=torch.full(lead + (p.B, p.K), -1.0, dtype=torch.float32, device=device))
