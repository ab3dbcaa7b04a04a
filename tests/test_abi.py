"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/pba.h declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re
import subprocess

import pytest

import pair_biased_attention_b200 as pba
from pair_biased_attention_b200 import build as pba_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pba.h")


@pytest.fixture(scope="module")
def lib():
    pba_build.build()
    return pba.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^PBA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("pba_forward", "pba_partial", "softmax_merge", "tri_attn_forward", "tri_proj_forward",
              "tri_out_proj_forward", "pwa_forward",
              "pba_status_string",
              "pba_last_device_error", "pba_set_wait_timeout_ns", "pba_selftest_wait_timeout",
              "pba_selftest_exp2"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", pba.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing else of ours leaks out of the hidden-visibility build
    ours = {s for s in exported if s.startswith(("pba", "softmax", "tri_", "pwa"))}
    assert ours == set(declared_functions())


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "pba.h"\nint main(void){ pba_attn_desc d; (void)d; return (int)PBA_OK; }\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-c",
                           str(src), "-o", str(tmp_path / "use.o")])


def test_status_strings(lib):
    for code, name in [(0, "PBA_OK"), (1, "PBA_ERR_INVALID_ARG"), (2, "PBA_ERR_UNSUPPORTED"), (3, "PBA_ERR_CUDA"),
                       (4, "PBA_ERR_TIMEOUT")]:
        assert pba.pba_status_string(code) == name
    assert pba.pba_status_string(77) == "PBA_ERR_UNKNOWN"


def test_wait_timeout_setting_roundtrip(lib):
    prev = pba.pba_set_wait_timeout_ns(123456)
    assert prev == 1_000_000_000
    assert pba.pba_set_wait_timeout_ns(0) == 123456  # 0 restores the default
    assert pba.pba_set_wait_timeout_ns(0) == 1_000_000_000


def _desc(**kw):
    d = pba.PbaAttnDesc()
    d.B, d.H, d.Nq, d.Nk, d.D, d.dtype = 1, 2, 16, 16, 64, pba.PBA_BF16
    for k, v in kw.items():
        setattr(d, k, v)
    return d


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: each call below fails its checks first


@pytest.mark.parametrize("kw,expect", [
    ({"B": 0}, pba.PBA_ERR_INVALID_ARG),
    ({"H": -1}, pba.PBA_ERR_INVALID_ARG),
    ({"Nq": -5}, pba.PBA_ERR_INVALID_ARG),
    ({"D": 48}, pba.PBA_ERR_UNSUPPORTED),
    ({"D": 128}, pba.PBA_ERR_UNSUPPORTED),
    ({"dtype": 7}, pba.PBA_ERR_UNSUPPORTED),
    ({"softmax_scale": -1.0}, pba.PBA_ERR_INVALID_ARG),
    ({"softmax_scale": float("nan")}, pba.PBA_ERR_INVALID_ARG),
    ({"Nk": 1 << 40}, pba.PBA_ERR_INVALID_ARG),
])
def test_forward_rejects_bad_descriptors(lib, kw, expect):
    d = _desc(**kw)
    assert lib.pba_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None) == expect
    assert lib.pba_partial(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None) == expect


def test_null_pointers_rejected(lib):
    d = _desc()
    assert lib.pba_forward(None, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None) == pba.PBA_ERR_INVALID_ARG
    assert lib.pba_forward(ctypes.byref(d), None, FAKE, FAKE, FAKE, None, FAKE, None, None) == pba.PBA_ERR_INVALID_ARG
    assert lib.pba_forward(ctypes.byref(d), FAKE, FAKE, FAKE, None, None, FAKE, None, None) == pba.PBA_ERR_INVALID_ARG
    assert lib.pba_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, None, None, None) == pba.PBA_ERR_INVALID_ARG
    # a partial needs all three outputs
    assert lib.pba_partial(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE,
                           None) == pba.PBA_ERR_INVALID_ARG


@pytest.mark.parametrize("args,expect", [
    ((0, 4, 64), pba.PBA_ERR_INVALID_ARG),    # P < 1
    ((2, -1, 64), pba.PBA_ERR_INVALID_ARG),   # rows < 0
    ((2, 4, 6), pba.PBA_ERR_INVALID_ARG),     # D not a multiple of 4
    ((2, 4, 512), pba.PBA_ERR_INVALID_ARG),   # D too large
])
def test_merge_rejects_bad_sizes(lib, args, expect):
    assert lib.softmax_merge(*args, FAKE, FAKE, FAKE, pba.PBA_BF16, FAKE, None, None) == expect


def test_merge_rejects_dtype_and_nulls(lib):
    assert lib.softmax_merge(2, 4, 64, FAKE, FAKE, FAKE, 9, FAKE, None, None) == pba.PBA_ERR_UNSUPPORTED
    assert lib.softmax_merge(2, 4, 64, None, FAKE, FAKE, pba.PBA_F32, FAKE, None, None) == pba.PBA_ERR_INVALID_ARG
    unaligned = ctypes.c_void_p(0x10004)
    assert lib.softmax_merge(2, 4, 64, unaligned, FAKE, FAKE, pba.PBA_F32, FAKE, None,
                             None) == pba.PBA_ERR_INVALID_ARG


@pytest.mark.parametrize("N,H,D,orient,expect", [
    (16, 4, 16, 0, pba.PBA_ERR_UNSUPPORTED),   # head dim
    (16, 4, 32, 2, pba.PBA_ERR_INVALID_ARG),   # orientation
    (12, 4, 32, 0, pba.PBA_ERR_INVALID_ARG),   # N not a multiple of 8
    (-8, 4, 32, 0, pba.PBA_ERR_INVALID_ARG),
    (16, 0, 32, 1, pba.PBA_ERR_INVALID_ARG),
])
def test_tri_rejects_bad_arguments(lib, N, H, D, orient, expect):
    assert lib.tri_attn_forward(N, H, D, orient, 0.0, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None,
                                None) == expect


def test_tri_rejects_unaligned_pointer(lib):
    unaligned = ctypes.c_void_p(0x10008)
    assert lib.tri_attn_forward(16, 4, 32, 0, 0.0, unaligned, FAKE, FAKE, FAKE, None, None, FAKE, None,
                                None) == pba.PBA_ERR_INVALID_ARG


@pytest.mark.parametrize("N,c,H,D,expect", [
    (16, 96, 4, 32, pba.PBA_ERR_UNSUPPORTED),    # c not 64 or 128
    (16, 128, 4, 16, pba.PBA_ERR_UNSUPPORTED),   # H*D != 128
    (16, 128, 3, 32, pba.PBA_ERR_UNSUPPORTED),   # H not a power of two up to 8
    (-1, 128, 4, 32, pba.PBA_ERR_INVALID_ARG),
    (40000, 128, 4, 32, pba.PBA_ERR_INVALID_ARG),  # N*N row coordinates past int32
])
def test_proj_rejects_bad_shapes(lib, N, c, H, D, expect):
    assert lib.tri_proj_forward(N, c, H, D, *([FAKE] * 8), None) == expect


def test_proj_rejects_null_and_unaligned(lib):
    args = [FAKE] * 8
    for i in range(8):
        bad = list(args)
        bad[i] = None
        assert lib.tri_proj_forward(16, 128, 4, 32, *bad, None) == pba.PBA_ERR_INVALID_ARG
    bad = list(args)
    bad[0] = ctypes.c_void_p(0x10008)  # z not 16-byte aligned
    assert lib.tri_proj_forward(16, 128, 4, 32, *bad, None) == pba.PBA_ERR_INVALID_ARG


@pytest.mark.parametrize("S,N,H,D,expect", [
    (4, 64, 2, 16, pba.PBA_ERR_UNSUPPORTED),   # head dim
    (4, 60, 2, 32, pba.PBA_ERR_INVALID_ARG),   # N not a multiple of 8
    (-1, 64, 2, 32, pba.PBA_ERR_INVALID_ARG),
    (4, 64, 0, 32, pba.PBA_ERR_INVALID_ARG),
])
def test_pwa_rejects_bad_shapes(lib, S, N, H, D, expect):
    assert lib.pwa_forward(S, N, H, D, FAKE, FAKE, None, None, FAKE, None, None) == expect


def test_pwa_rejects_null_and_unaligned(lib):
    assert lib.pwa_forward(4, 64, 2, 32, None, FAKE, None, None, FAKE, None, None) == pba.PBA_ERR_INVALID_ARG
    assert lib.pwa_forward(4, 64, 2, 32, FAKE, FAKE, None, None, None, None, None) == pba.PBA_ERR_INVALID_ARG
    odd = ctypes.c_void_p(0x10008)
    assert lib.pwa_forward(4, 64, 2, 32, FAKE, FAKE, None, odd, FAKE, FAKE, None) == pba.PBA_ERR_INVALID_ARG
    # lse is required: the softmax takes it as its first pass
    assert lib.pwa_forward(4, 64, 2, 32, FAKE, FAKE, None, None, FAKE, None, None) == pba.PBA_ERR_INVALID_ARG
    assert lib.pwa_forward(4, 64, 2, 32, FAKE, FAKE, None, None, FAKE, ctypes.c_void_p(0x10002),
                           None) == pba.PBA_ERR_INVALID_ARG


@pytest.mark.parametrize("N,c,H,D,expect", [
    (16, 96, 4, 32, pba.PBA_ERR_UNSUPPORTED),   # pair channels
    (16, 128, 4, 16, pba.PBA_ERR_UNSUPPORTED),  # H*D != 128
    (-1, 128, 4, 32, pba.PBA_ERR_INVALID_ARG),
    (40000, 128, 4, 32, pba.PBA_ERR_INVALID_ARG),
])
def test_out_proj_rejects_bad_shapes(lib, N, c, H, D, expect):
    assert lib.tri_out_proj_forward(N, c, H, D, FAKE, FAKE, FAKE, None) == expect


def test_out_proj_rejects_null_and_unaligned(lib):
    assert lib.tri_out_proj_forward(0, 128, 4, 32, None, None, None, None) == pba.PBA_OK  # nothing to do
    for i in range(3):
        args = [FAKE, FAKE, FAKE]
        args[i] = None
        assert lib.tri_out_proj_forward(16, 128, 4, 32, *args, None) == pba.PBA_ERR_INVALID_ARG
        args[i] = ctypes.c_void_p(0x10008)
        assert lib.tri_out_proj_forward(16, 128, 4, 32, *args, None) == pba.PBA_ERR_INVALID_ARG


def test_selftest_rejects_bad_limit(lib):
    assert lib.pba_selftest_wait_timeout(0, None) == pba.PBA_ERR_INVALID_ARG
