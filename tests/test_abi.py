"""CPU checks of the C-ABI boundary: the library builds, loads, and exports
every symbol include/nvfp4sk.h declares (no compute calls without a GPU)."""
import ctypes
import os
import subprocess

from nvfp4_skinny_gemm_b200 import build, lib


def test_library_builds_and_exports_every_declared_symbol():
    path = build.build()
    assert os.path.exists(path)
    declared = lib.header_symbols()
    assert len(declared) >= 19
    L = ctypes.CDLL(path)
    for name in declared:
        assert hasattr(L, name), f"{name} declared in nvfp4sk.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared) <= exported
    # the binding covers exactly the declared API
    assert set(lib._SIGS) == set(declared)


def test_version_and_options_without_gpu():
    L = lib.load()
    assert L.nvfp4sk_version() == 100
    assert L.nvfp4sk_get_option(lib.OPT_PDL) in (0, 1)
    assert L.nvfp4sk_set_option(lib.OPT_ATTN_SPLITS, 7) == 0
    assert L.nvfp4sk_get_option(lib.OPT_ATTN_SPLITS) == 7
    assert L.nvfp4sk_set_option(lib.OPT_ATTN_SPLITS, 0) == 0
    assert L.nvfp4sk_set_option(99, 1) == -1
    assert b"unknown option" in L.nvfp4sk_last_error()


def test_prepared_sizes():
    L = lib.load()
    unit = 2 * 128 * 128 + 8 * 512              # 128 rows x 512 K: codes + scale images
    assert L.nvfp4_prepared_weight_bytes(128, 512) == unit
    assert L.nvfp4_prepared_weight_bytes(129, 576) == 2 * 2 * unit
    assert L.nvfp4_prepared_weight_bytes(151936, 5120) == 1187 * 10 * unit
    assert L.nvfp4_prepared_act_bytes(5120) == 10 * (2 * 16 * 128 + 8 * 512)
    assert L.nvfp4_prepared_act_bytes(17408) == 34 * 8192


def test_header_is_plain_c():
    """The public header compiles as C99 with no CUDA or torch headers."""
    hdr = lib.HEADER
    r = subprocess.run(["gcc", "-std=c99", "-fsyntax-only", "-x", "c", hdr], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_arity_matches_header():
    """Every ctypes signature of the binding has as many arguments as the C
    declaration in include/nvfp4sk.h (a missing one shifts the stream handle)."""
    import re
    from nvfp4_skinny_gemm_b200 import lib
    txt = open(lib.HEADER).read()
    seen = 0
    for m in re.finditer(r"NVFP4SK_API [^(]*?\b([a-z_0-9]+)\(([^)]*)\);", txt, re.S):
        name, args = m.group(1), m.group(2).strip()
        n = 0 if args in ("", "void") else len(args.split(","))
        assert len(lib._SIGS[name][1]) == n, (name, n, len(lib._SIGS[name][1]))
        seen += 1
    assert seen == len(lib._SIGS)
