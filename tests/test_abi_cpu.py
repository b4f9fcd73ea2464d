"""The C-ABI library builds, loads and exports every symbol include/flce.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from lm_head_linear_tmem_b200 import _native, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flce.h")

FAKE = 0x10000  # a 256-aligned, never-dereferenced address for argument-check tests


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flce_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("flce_forward", "flce_backward", "flce_workspace_bytes", "flce_get_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _native.SIGNATURES, name


def test_version_and_strings(lib):
    assert lib.flce_version() >= 100
    for code, name in _native.STATUS_NAMES.items():
        assert lib.flce_status_string(code).decode() == name
    assert lib.flce_status_string(99).decode() == "FLCE_ERR_UNKNOWN"


def test_workspace_bytes(lib):
    ws = lib.flce_workspace_bytes
    assert ws(-1, 64, 512, 0) == 0
    assert ws(64, 4, 512, 0) == 0
    assert ws(64, 64, 0, 0) == 0
    assert ws(64, 64, 512, 7) == 0
    tiny = ws(64, 64, 512, 0)
    assert tiny > 0 and tiny % 256 == 0
    big = ws(16384, 4096, 131072, 0)
    # forward partials: 512 vocab tiles x 16384 rows x (m, s) fp32 = 64 MiB;
    # backward: compact hidden 16384 x 4096 bf16 = 128 MiB + dZ block
    # 16384 x 16384 bf16 = 512 MiB + compact-order dHidden of a token chunk
    # 16384 x 4096 fp32 = 256 MiB + row-compaction, label-sort and residual arrays
    assert 896 * 2 ** 20 <= big < 898 * 2 ** 20
    with _native.options(bwd_compact=0):  # dHidden goes straight to its output
        assert ws(16384, 4096, 131072, 0) <= big - 256 * 2 ** 20
    assert ws(0, 64, 512, 0) > 0
    assert ws(64, 64, 512, 1) > 0
    ex = lib.flce_workspace_bytes_ex
    for dtype in (0, 1):
        base = ws(300, 64, 1000, dtype)
        assert ex(300, 64, 1000, dtype, 0) == base
        assert ex(300, 64, 1000, dtype, 3) == base  # accumulate flags need no scratch
        assert ex(300, 64, 1000, dtype, 4) >= base + 4 * 300 * 64
        assert ex(300, 64, 1000, dtype, 8) >= base + 4 * 1000 * 64
        assert ex(300, 64, 1000, dtype, 12) >= base + 4 * 1300 * 64
        assert ex(300, 64, 1000, dtype, 16) == 0
    assert ex(-1, 64, 1000, 0, 4) == 0


def _fwd(lib, N=64, H=64, V=512, softcap=0.0, reduction=0, dtype=0, ws_size=None,
         hidden=FAKE, weight=FAKE, labels=FAKE, loss=FAKE, ntok=FAKE, lse=FAKE):
    if ws_size is None:
        ws_size = lib.flce_workspace_bytes(N, H, V, dtype) or 1 << 20
    return lib.flce_forward(hidden, weight, labels, N, H, V, -100, softcap, reduction, dtype,
                            loss, ntok, lse, FAKE, ws_size, None)


def test_argument_errors_are_synchronous(lib):
    ARG, SHAPE, WS = 1, 2, 7
    assert _fwd(lib, reduction=5) == ARG
    assert _fwd(lib, dtype=3) == ARG
    assert _fwd(lib, softcap=-1.0) == ARG
    assert _fwd(lib, softcap=float("nan")) == ARG
    assert _fwd(lib, softcap=float("inf")) == ARG
    assert _fwd(lib, H=68) == SHAPE          # bf16 rows must be 16-byte multiples
    assert _fwd(lib, H=4) == SHAPE
    assert _fwd(lib, V=0) == SHAPE
    assert _fwd(lib, N=-3) == SHAPE
    assert _fwd(lib, hidden=None) == ARG
    assert _fwd(lib, weight=FAKE + 8) == ARG  # misaligned for TMA
    assert _fwd(lib, labels=FAKE + 4) == ARG
    assert _fwd(lib, ws_size=1024) == WS
    assert _fwd(lib, loss=None) == ARG
    wsb = lib.flce_workspace_bytes(64, 64, 512, 0)
    bad_bwd = lib.flce_backward(FAKE, FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, None,
                                float("nan"), None, FAKE, FAKE, 0, FAKE, wsb, None)
    assert bad_bwd == ARG
    bad_flags = lib.flce_backward(FAKE, FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, None,
                                  1.0, None, FAKE, FAKE, 16, FAKE, wsb, None)
    assert bad_flags == ARG
    no_outputs = lib.flce_backward(FAKE, FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, None,
                                   1.0, None, None, None, 0, FAKE, wsb, None)
    assert no_outputs == ARG
    # bf16 gradient outputs need the larger workspace of flce_workspace_bytes_ex
    for flags in (4, 8, 12):
        assert lib.flce_backward(FAKE, FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, None,
                                 1.0, None, FAKE, FAKE, flags, FAKE, wsb, None) == WS
    assert lib.flce_get_status(None, None) == ARG
    for bad_scale in (float("nan"), float("inf")):
        assert lib.flce_forward_ex(FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, bad_scale,
                                   FAKE, FAKE, FAKE, FAKE, wsb, None) == ARG


def test_options_host_side(lib):
    """Options are set and read through the ABI (no environment variable reaches
    the library); out-of-range values and unknown options are refused and leave
    the option unchanged; the workspace size follows the chunk options."""
    v = ctypes.c_int64()
    defaults = {"cta_group": 2, "bwd_compact": 1, "bwd_fuse": 1, "mn3d": 1,
                "chunk_tokens": 16384, "chunk_vocab": 16384, "wait_timeout_ms": 1000,
                "grad_tile_n": 512, "dz_tile_n": 0, "fwd_tile_n": 512, "fwd_group_m": 16,
                "dz_group_m": 16, "grad_group_m": 8, "fwd_dynamic": 1,
                "dz_buffers": 1, "fwd_compact": 1}
    assert set(defaults) == set(_native.OPTIONS)
    for name, dflt in defaults.items():
        assert _native.get_option(name) == dflt, name
    ARG = 1
    for name, bad in (("cta_group", 3), ("cta_group", 0), ("bwd_compact", 2),
                      ("chunk_tokens", 100), ("chunk_vocab", 1 << 21),
                      ("wait_timeout_ms", 5), ("grad_tile_n", 384), ("dz_tile_n", 128),
                      ("grad_tile_n", 0), ("fwd_tile_n", 0),
                      ("fwd_tile_n", 1024), ("fwd_group_m", 0), ("grad_group_m", 65)):
        assert lib.flce_set_option(_native.OPTIONS[name], bad) == ARG, (name, bad)
        assert _native.get_option(name) == defaults[name]
    assert lib.flce_set_option(-1, 0) == ARG and lib.flce_set_option(99, 0) == ARG
    assert lib.flce_get_option(99, ctypes.byref(v)) == ARG
    assert lib.flce_get_option(0, None) == ARG
    big = lib.flce_workspace_bytes(16384, 4096, 131072, 0)
    with _native.options(chunk_tokens=1024, chunk_vocab=2048, grad_tile_n=256):
        assert _native.get_option("chunk_tokens") == 1024
        assert _native.get_option("grad_tile_n") == 256
        small = lib.flce_workspace_bytes(16384, 4096, 131072, 0)
        assert small < big  # the dZ block is 1024 x 2048 bf16 instead of 16384 x 16384
    assert _native.get_option("chunk_tokens") == 16384
    assert _native.get_option("grad_tile_n") == 512
    assert lib.flce_workspace_bytes(16384, 4096, 131072, 0) == big
    # a chunk size that is not a multiple of 256 is rounded up
    with _native.options(chunk_vocab=512):
        ws512 = lib.flce_workspace_bytes(8192, 64, 5000, 0)
    with _native.options(chunk_vocab=300):
        assert _native.get_option("chunk_vocab") == 300
        assert lib.flce_workspace_bytes(8192, 64, 5000, 0) == ws512


def test_label_token_count_entry_points_host_side(lib):
    """flce_forward_ex2 / flce_backward_ex check their arguments like the calls they
    extend (the count itself is any int64: negative means none)."""
    ARG = 1
    wsb = lib.flce_workspace_bytes(64, 64, 512, 0)
    assert lib.flce_forward_ex2(FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 5, 0, 1.0, 10,
                                FAKE, FAKE, FAKE, FAKE, wsb, None) == ARG
    assert lib.flce_forward_ex2(FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, float("nan"),
                                10, FAKE, FAKE, FAKE, FAKE, wsb, None) == ARG
    assert lib.flce_backward_ex(FAKE, FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, None,
                                float("inf"), 10, None, FAKE, FAKE, 0, FAKE, wsb, None) == ARG
    assert lib.flce_backward_ex(FAKE, FAKE, FAKE, FAKE, 64, 64, 512, -100, 0.0, 0, 0, None,
                                1.0, 10, None, None, None, 0, FAKE, wsb, None) == ARG


def test_profile_api_host_side(lib):
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    assert lib.flce_profile_read(0, ctypes.byref(ms), ctypes.byref(n)) == 0
    assert n.value == 0
    assert lib.flce_profile_read(99, ctypes.byref(ms), ctypes.byref(n)) == 1
    assert lib.flce_profile_enable(0) == 0


def test_header_is_plain_c_and_a_c_program_links(tmp_path):
    """include/flce.h compiles as C99 with all warnings as errors, and a C caller
    links against the library and the CUDA runtime (it runs in the GPU tests)."""
    from tests import _c_driver
    exe = _c_driver.build_driver(str(tmp_path))
    res = subprocess.run([exe], capture_output=True, text=True)
    assert res.returncode == 1 and "usage" in res.stderr  # no GPU call without arguments
