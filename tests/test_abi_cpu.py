"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export every function declared in include/attn.h with
the signature the binding declares, and reject bad arguments on the host
before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import exact_tiled_attention_38_b200 as eta
from exact_tiled_attention_38_b200 import build as eta_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def clib():
    eta_build.build()
    return eta.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("attn_fwd", "attn_decode", "attn_fwd_f16", "attn_decode_f16", "attn_strerror",
              "attn_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(clib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(clib, n), f"{n} not exported"
    assert set(names) == set(eta.SIGNATURES), "binding and header disagree"


def test_argument_counts_match_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for name, (_, args) in eta.SIGNATURES.items():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", text)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(args), name


def test_strerror_covers_codes(clib):
    for code in (eta.ATTN_OK, eta.ATTN_ERR_INVALID, eta.ATTN_ERR_UNSUPPORTED, eta.ATTN_ERR_CUDA,
                 eta.ATTN_ERR_TIMEOUT, 12345):
        s = clib.attn_strerror(code)
        assert s and len(s) > 1


def test_strerror_messages_state_the_real_limits(clib):
    msg = lambda c: clib.attn_strerror(c).decode()  # noqa: E731
    unsup = msg(eta.ATTN_ERR_UNSUPPORTED)
    # head sizes: any multiple of 8 in [8, 256] is supported (not just 64 / 128)
    assert "multiple of 8 in [8, 256]" in unsup and "not 64 or 128" not in unsup
    assert "65,535" in unsup and "sm_100" in unsup
    scr = msg(eta.ATTN_ERR_SCRATCH)
    assert "attn_decode_noalloc" in scr and "2,097,152" in scr
    assert msg(12345) == "unknown error code"


# Calls that the host rejects (or finds empty) before touching CUDA.
FAKE = ctypes.c_void_p(0x10000)


def fwd(clib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=4, Hkv=2, Nq=8, Nk=8, d=128,
             scale=0.1, causal=1)
    a.update(kw)
    return clib.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                         a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], None)


def test_fwd_host_validation(clib):
    assert fwd(clib, Hq=3) == eta.ATTN_ERR_INVALID
    assert fwd(clib, Hkv=0) == eta.ATTN_ERR_INVALID
    assert fwd(clib, B=-1) == eta.ATTN_ERR_INVALID
    assert fwd(clib, Nq=-5) == eta.ATTN_ERR_INVALID
    assert fwd(clib, scale=0.0) == eta.ATTN_ERR_INVALID
    assert fwd(clib, scale=float("inf")) == eta.ATTN_ERR_INVALID
    # head sizes: multiples of 8 in [8, 256] are taken (64 and 128 on the
    # tensor cores, the rest on the generic kernel); nothing else is
    for d in (0, 4, 12, 100, 264, 512):
        assert fwd(clib, d=d) == eta.ATTN_ERR_UNSUPPORTED, d
    for d in (8, 96, 256):  # accepted: an empty problem is a no-op
        assert fwd(clib, d=d, B=0) == eta.ATTN_OK, d
    assert fwd(clib, o=None) == eta.ATTN_ERR_INVALID
    assert fwd(clib, q=ctypes.c_void_p(0x10008)) == eta.ATTN_ERR_INVALID
    assert fwd(clib, lse=ctypes.c_void_p(0x10002)) == eta.ATTN_ERR_INVALID
    assert fwd(clib, Nq=65535 * 256 + 1) == eta.ATTN_ERR_INVALID
    # empty problems are a no-op
    assert fwd(clib, B=0) == eta.ATTN_OK
    assert fwd(clib, Nq=0) == eta.ATTN_OK
    assert clib.attn_fwd_f16(FAKE, FAKE, FAKE, FAKE, None, 0, 1, 1, 4, 4, 64, 0.1, 0,
                             None) == eta.ATTN_OK


def dec(clib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, s=FAKE, o=FAKE, lse=None, B=2, Hq=8, Hkv=2, d=128,
             scale=0.1)
    a.update(kw)
    return clib.attn_decode(a["q"], a["k"], a["v"], a["s"], a["o"], a["lse"], a["B"], a["Hq"],
                            a["Hkv"], a["d"], a["scale"], None)


def test_decode_host_validation(clib):
    assert dec(clib, Hq=6, Hkv=4) == eta.ATTN_ERR_INVALID
    assert dec(clib, scale=-0.5) == eta.ATTN_ERR_INVALID
    assert dec(clib, d=84) == eta.ATTN_ERR_UNSUPPORTED
    assert dec(clib, d=272) == eta.ATTN_ERR_UNSUPPORTED
    assert dec(clib, d=80, B=0) == eta.ATTN_OK
    assert dec(clib, s=None) == eta.ATTN_ERR_INVALID
    assert dec(clib, s=ctypes.c_void_p(0x10002)) == eta.ATTN_ERR_INVALID
    assert dec(clib, k=ctypes.c_void_p(0x10004)) == eta.ATTN_ERR_INVALID
    assert dec(clib, B=0) == eta.ATTN_OK
    assert clib.attn_decode_num_splits(2, 6, 4, 128) == eta.ATTN_ERR_INVALID
    assert clib.attn_decode_num_splits(2, 8, 2, 100) == eta.ATTN_ERR_UNSUPPORTED
    assert clib.attn_decode_num_splits(2, 8, 2, 96) == 1  # generic kernel: no split


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(eta, "_lib", None)
    with pytest.raises(RuntimeError):
        eta.load_library(str(tmp_path / "missing.so"))


def test_stall_hook_rejects_bad_wait(clib):
    # checked on the host before any CUDA call
    for bad in (0, 1000001):
        assert clib.attn_fwd_stall_test(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 1, 8, 8, 128, 0.1, 1,
                                        bad, None) == eta.ATTN_ERR_INVALID
    # the generic head-size kernel has no waits to stall
    assert clib.attn_fwd_stall_test(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 1, 8, 8, 96, 0.1, 1,
                                    1000, None) == eta.ATTN_ERR_UNSUPPORTED


def test_window_entry_points_reject_bad_windows(clib):
    for bad in (0, -3):
        assert clib.attn_fwd_window(FAKE, FAKE, FAKE, FAKE, None, 1, 2, 1, 8, 8, 128, 0.1, bad,
                                    None) == eta.ATTN_ERR_INVALID
        assert clib.attn_decode_window(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 1, 128, 0.1,
                                       bad, None) == eta.ATTN_ERR_INVALID


def test_merge_host_validation(clib):
    def merge(**kw):
        a = dict(oa=FAKE, la=FAKE, op=FAKE, lp=FAKE, out=None, rows=10, d=128)
        a.update(kw)
        return clib.attn_merge(a["oa"], a["la"], a["op"], a["lp"], a["out"], a["rows"], a["d"],
                               None)

    assert merge(rows=-1) == eta.ATTN_ERR_INVALID
    assert merge(d=12) == eta.ATTN_ERR_UNSUPPORTED
    assert merge(d=264) == eta.ATTN_ERR_UNSUPPORTED
    assert merge(rows=0) == eta.ATTN_OK
    assert merge(oa=None) == eta.ATTN_ERR_INVALID
    assert merge(lp=None) == eta.ATTN_ERR_INVALID
    assert merge(op=ctypes.c_void_p(0x10008)) == eta.ATTN_ERR_INVALID
    assert merge(la=ctypes.c_void_p(0x10002)) == eta.ATTN_ERR_INVALID
    assert merge(out=ctypes.c_void_p(0x10004)) == eta.ATTN_ERR_INVALID
    assert clib.attn_merge_f16(FAKE, FAKE, FAKE, FAKE, None, 0, 64, None) == eta.ATTN_OK


def test_build_tracks_every_source():
    # A change to any kernel source must trigger a rebuild of the library.
    csrc = os.path.join(ROOT, "exact_tiled_attention_38_b200", "csrc")
    srcs = {os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))}
    assert srcs <= set(eta_build.DEPS)
    assert HEADER in eta_build.DEPS


def test_decode_batch_limit_of_the_split_passes(clib):
    # d = 64 / 128 decode launches one grid z slice per sequence
    assert dec(clib, B=65536, Hq=1, Hkv=1) == eta.ATTN_ERR_UNSUPPORTED
    assert clib.attn_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 65536, 1, 1, 128, 0.1,
                                    None) == eta.ATTN_ERR_UNSUPPORTED


def test_binding_refuses_tensors_on_different_devices():
    import torch

    class FakeDev:  # stands in for CUDA tensors on two devices (no GPU needed)
        def __init__(self, dev):
            self.device = torch.device(dev)

    with pytest.raises(ValueError):
        eta._on_device(FakeDev("cuda:0"), FakeDev("cuda:1"))
    eta._on_device(FakeDev("cuda:1"), None, FakeDev("cuda:1"))  # one device: fine


def test_header_is_plain_c_and_links(tmp_path, clib):
    # The boundary is a C ABI: the header compiles as C99 with warnings as
    # errors, and a C program that takes the address of every entry point links
    # against the library.
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    src = tmp_path / "abi.c"
    src.write_text('#include "attn.h"\n#include <stdio.h>\n'
                   "int main(void) {\n  void* fns[] = {\n" +
                   "".join(f"    (void*)&{n},\n" for n in names) +
                   "  };\n  printf(\"%d\\n\", (int)(sizeof fns / sizeof fns[0]));\n"
                   "  return 0;\n}\n")
    lib_dir = os.path.dirname(eta.LIB_PATH)
    res = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                          "-Wno-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
                          "-L", lib_dir, "-lattn", "-o", str(tmp_path / "abi")],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_last_cuda_error_starts_clear(clib):
    # No CUDA call has failed on this thread through the library's launch paths.
    assert clib.attn_last_cuda_error() == 0
