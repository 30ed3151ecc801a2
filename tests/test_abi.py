"""The C-ABI library loads and exports every symbol the headers declare; host
argument checks answer before any launch (CPU only, no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

import draft_sampling_verification_head_b200 as sd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(spec_[a-z_0-9]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared()
    assert {"spec_cycle", "spec_markov_bias_sample", "spec_verify_block"} <= declared
    lib = ctypes.CDLL(sd.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(sd._SIGS), "binding signatures out of sync with the headers"


def test_status_strings():
    for code, name in [(0, "SPEC_OK"), (-1, "SPEC_ERR_INVALID_ARG"), (-4, "SPEC_ERR_TIMEOUT"),
                       (-6, "SPEC_ERR_TOKEN_RANGE")]:
        assert sd.status_string(code) == name


def _p(**kw):
    d = dict(B=4, K=4, V=1024, r=16, dtype="bf16", temperature=1.0)
    d.update(kw)
    return sd.Params(**d)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), sd.SPEC_ERR_INVALID_ARG),
    (dict(K=0), sd.SPEC_ERR_INVALID_ARG),
    (dict(r=300), sd.SPEC_ERR_INVALID_ARG),
    (dict(temperature=0.0), sd.SPEC_ERR_INVALID_ARG),
    (dict(V=1001), sd.SPEC_ERR_UNSUPPORTED),
    (dict(row_offset=2**31 - 3), sd.SPEC_ERR_INVALID_ARG),  # row_offset + B beyond 2^31
    (dict(K=1025), sd.SPEC_ERR_INVALID_ARG),
    (dict(r=-1), sd.SPEC_ERR_INVALID_ARG),
])
def test_host_validation_before_launch(kw, code):
    L = sd.lib()
    p = _p(**kw).c()
    fake = ctypes.c_void_p(0x1000)
    rc = L.spec_cycle(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None, None,
                      fake, None)
    assert rc == code
    assert L.spec_workspace_size(ctypes.byref(p)) == 0


def test_null_pointers_rejected():
    L = sd.lib()
    p = _p().c()
    rc = L.spec_cycle(ctypes.byref(p), None, None, None, None, None, None, None, None, None, None,
                      None, None)
    assert rc == sd.SPEC_ERR_INVALID_ARG
    assert L.spec_cycle(None, *([None] * 12)) == sd.SPEC_ERR_INVALID_ARG
    assert L.spec_workspace_init(None, 0, None) == sd.SPEC_ERR_WORKSPACE


def test_greedy_allows_zero_temperature_shape_check():
    L = sd.lib()
    p = _p(temperature=0.0, greedy=True, V=1001).c()
    fake = ctypes.c_void_p(0x1000)
    # passes the temperature rule, then fails on the vocabulary alignment rule
    assert L.spec_cycle(ctypes.byref(p), *([fake] * 6), fake, fake, None, None, fake,
                        None) == sd.SPEC_ERR_UNSUPPORTED


def test_params_struct_matches_header():
    """The ctypes mirror lists spec_params' fields in the header's order, with
    the header's integer widths, so the binding and the library agree on
    every offset."""
    text = open(os.path.join(ROOT, "include", "specdec.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} spec_params;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"\b(u?int\d+_t|float)\s+(\w+)\s*;", body)
    ctype = {"int32_t": ctypes.c_int32, "uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64,
             "float": ctypes.c_float}
    assert [(n, ctype[t]) for t, n in fields] == list(sd.SpecParams._fields_)


def test_params_offsets_match_the_c_compiler(tmp_path):
    """Field offsets and size of spec_params as the host C compiler lays them
    out, against the ctypes mirror."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no host C compiler")
    names = [n for n, _ in sd.SpecParams._fields_]
    src = tmp_path / "probe.c"
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "specdec.h"', "int main(void) {",
             '  printf("%zu\\n", sizeof(spec_params));']
    lines += [f'  printf("%zu\\n", offsetof(spec_params, {n}));' for n in names]
    lines += ["  return 0;", "}"]
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    want = [ctypes.sizeof(sd.SpecParams)] + [getattr(sd.SpecParams, n).offset for n in names]
    assert got == want


def test_valid_params_pass_host_validation():
    """Greedy needs no temperature, and the largest row offset that still fits
    is accepted: validation passes and the call only fails for want of a GPU
    (or launches, on a machine that has one)."""
    import torch
    L = sd.lib()
    if torch.cuda.is_available():
        # a GPU is present: the call would launch; host validation is the same
        # one spec_workspace_size applies, which launches nothing
        for kw in (dict(greedy=True, temperature=0.0), dict(row_offset=2**31 - 4)):
            assert sd.workspace_size(_p(**kw)) > 0, kw
        return
    fake = ctypes.c_void_p(0x1000)
    for kw in (dict(greedy=True, temperature=0.0), dict(row_offset=2**31 - 4)):
        p = _p(**kw).c()
        rc = L.spec_cycle(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None,
                          None, fake, None)
        assert rc not in (sd.SPEC_ERR_INVALID_ARG, sd.SPEC_ERR_UNSUPPORTED), (kw, rc)


def _loop_call(p, n_cycles, conf=None, vlen=None, next_token=True, nulls=()):
    L = sd.lib()
    fake = ctypes.c_void_p(0x1000)
    args = dict(base=fake, target=fake, conf=conf, vlen=vlen, U=fake, W=fake, last=fake,
                draft=None, out=fake, tau=fake, pd=None, qd=None,
                nt=fake if next_token else None, ws=ctypes.c_void_p(0x10000))
    for k in nulls:
        args[k] = None
    return L.spec_decode_loop(ctypes.byref(p.c()), n_cycles, args["base"], args["target"],
                              args["conf"], ctypes.c_float(0.5), args["vlen"], args["U"],
                              args["W"], args["last"], args["draft"], args["out"], args["tau"],
                              args["pd"], args["qd"], args["nt"], args["ws"], None)


@pytest.mark.parametrize("case", ["zero_cycles", "too_many_cycles", "no_next_token",
                                  "conf_and_vlen", "no_target", "no_last_token", "bad_params"])
def test_decode_loop_host_validation(case):
    """spec_decode_loop rejects bad arguments on the host, before any launch."""
    fake = ctypes.c_void_p(0x2000)
    p = _p(r=64)
    kw = {}
    n = 3
    if case == "zero_cycles":
        n = 0
    elif case == "too_many_cycles":
        n = (1 << 16) + 1
    elif case == "no_next_token":
        kw = dict(next_token=False)
    elif case == "conf_and_vlen":
        kw = dict(conf=fake, vlen=fake)
    elif case == "no_target":
        kw = dict(nulls=("target",))
    elif case == "no_last_token":
        kw = dict(nulls=("last",))
    elif case == "bad_params":
        p = _p(B=0, r=64)
    assert _loop_call(p, n, **kw) == sd.SPEC_ERR_INVALID_ARG


def test_decode_loop_one_cycle_needs_no_next_token():
    """One cycle carries nothing over: next_token may be NULL (the call passes
    host validation and fails only for want of a GPU, or launches)."""
    import torch
    if torch.cuda.is_available():
        return  # a fake pointer would reach the device
    rc = _loop_call(_p(r=64), 1, next_token=False)
    assert rc not in (sd.SPEC_ERR_INVALID_ARG, sd.SPEC_ERR_UNSUPPORTED), rc
