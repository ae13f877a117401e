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


# Fake device addresses: every call below is rejected by a host-side check
# before the library looks at the device, so nothing is dereferenced or
# launched (on a machine with or without a GPU).
A = 1 << 20                 # 16-byte aligned, non-null
MIS = A + 8                 # 8 bytes off a 16-byte boundary


def _rc(name, *args):
    return getattr(lib.load(), name)(*args)


def test_host_checks_reject_bad_arguments_before_the_device():
    E_ARG, E_SHAPE, E_ALIGN = -1, -2, -3
    cases = [
        # nvfp4_quantize_act(x, dtype, rows, K, ld_x, g_in, codes, scales, g_out, act, ws, ws_bytes, stream)
        (E_ARG, "nvfp4_quantize_act", None, 0, 16, 64, 64, None, A, A, None, None, A, 1 << 20, None),
        (E_ARG, "nvfp4_quantize_act", A, 7, 16, 64, 64, None, A, A, A, None, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_quantize_act", A, 0, 16, 24, 24, None, A, A, A, None, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_quantize_act", A, 0, 17, 64, 64, None, None, None, A, A, A, 1 << 20, None),
        (E_ALIGN, "nvfp4_quantize_act", MIS, 0, 16, 64, 64, None, A, A, A, None, A, 1 << 20, None),
        # nvfp4_prepare_act(codes, scales, rows, K, act, stream)
        (E_SHAPE, "nvfp4_prepare_act", A, A, 17, 64, A, None),
        (E_ALIGN, "nvfp4_prepare_act", A, A, 16, 64, MIS, None),
        # nvfp4_prepare_weight(codes, scales, N, K, prepared, stream)
        (E_SHAPE, "nvfp4_prepare_weight", A, A, 128, 100, A, None),
        (E_ALIGN, "nvfp4_prepare_weight", A, A, 128, 128, MIS, None),
        (E_ALIGN, "nvfp4_prepare_weight", MIS, A, 128, 128, A, None),
        (E_ALIGN, "nvfp4_prepare_weight", A, A + 2, 128, 128, A, None),
        # nvfp4_linear(a, g_a, M, w, g_w, N, K, residual, y, ldy, ws, ws_bytes, stream)
        (E_ARG, "nvfp4_linear", None, A, 16, A, A, 128, 128, None, A, 128, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_linear", A, A, 17, A, A, 128, 128, None, A, 128, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_linear", A, A, 16, A, A, 524289, 128, None, A, 524289, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_linear", A, A, 16, A, A, 128, 96, None, A, 128, A, 1 << 20, None),
        (E_ALIGN, "nvfp4_linear", MIS, A, 16, A, A, 128, 128, None, A, 128, A, 1 << 20, None),
        # nvfp4_linear_wide(a, g_a, S, w, g_w, N, K, residual, y, ldy, stream)
        (E_ARG, "nvfp4_linear_wide", None, A, 100, A, A, 128, 128, None, A, 128, None),
        (E_SHAPE, "nvfp4_linear_wide", A, A, 0, A, A, 128, 128, None, A, 128, None),
        (E_SHAPE, "nvfp4_linear_wide", A, A, 100, A, A, 128, 96, None, A, 128, None),
        (E_SHAPE, "nvfp4_linear_wide", A, A, 100, A, A, 128, 128, None, A, 64, None),
        (E_ALIGN, "nvfp4_linear_wide", MIS, A, 100, A, A, 128, 128, None, A, 128, None),
        # nvfp4_linear_swiglu(a, g_a, M, w, g_w, F, K, g_out, act_out, ws, ws_bytes, stream)
        (E_ARG, "nvfp4_linear_swiglu", A, A, 16, A, A, 256, 128, None, A, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_linear_swiglu", A, A, 0, A, A, 256, 128, A, A, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_linear_swiglu", A, A, 16, A, A, 192, 128, A, A, A, 1 << 20, None),
        (E_SHAPE, "nvfp4_linear_swiglu", A, A, 16, A, A, 256, 96, A, A, A, 1 << 20, None),
        (E_ALIGN, "nvfp4_linear_swiglu", A, A, 16, A, A, 256, 128, A, MIS, A, 1 << 20, None),
        # nvfp4_quantize_act_tiles(x, dtype, rows, K, ld_x, g_in, g_out, tiles, stream)
        (E_ARG, "nvfp4_quantize_act_tiles", A, 0, 942, 3072, 3072, None, A, A, None),
        (E_SHAPE, "nvfp4_quantize_act_tiles", A, 0, 942, 3008, 3072, A, A, A, None),
        (E_ALIGN, "nvfp4_quantize_act_tiles", A, 0, 942, 3072, 3072, A, A, MIS, None),
        # nvfp4_rmsnorm_quantize_tiles(x, w, eps, rows, n, g_in, g_out, tiles, stream)
        (E_ARG, "nvfp4_rmsnorm_quantize_tiles", A, None, 1e-6, 942, 5120, A, A, A, None),
        (E_SHAPE, "nvfp4_rmsnorm_quantize_tiles", A, A, 1e-6, 942, 8704, A, A, A, None),
        (E_SHAPE, "nvfp4_rmsnorm_quantize_tiles", A, A, 1e-6, 0, 5120, A, A, A, None),
        # nvfp4_swiglu_quantize_tiles(gu, rows, F, g_in, g_out, tiles, stream)
        (E_ARG, "nvfp4_swiglu_quantize_tiles", A, 942, 17408, A, None, A, None),
        (E_SHAPE, "nvfp4_swiglu_quantize_tiles", A, 942, 17344, A, A, A, None),
        (E_ALIGN, "nvfp4_swiglu_quantize_tiles", MIS, 942, 17408, A, A, A, None),
        # nvfp4_linear_noalloc(a, g_a, M, w, g_w, N, K, residual, y, ldy, stream)
        (E_SHAPE, "nvfp4_linear_noalloc", A, A, 16, A, A, 524289, 128, None, A, 524289, None),
        # tree_attn_fp8kv(q, ld_q, T, Hq, Hkv, D, k_pool, v_pool, n_pool, P, page_table, ctx_len, parent,
        #                 k_scale, v_scale, sm_scale, out, g_act, act, ws, ws_bytes, stream)
        (E_SHAPE, "tree_attn_fp8kv", A, 3072, 17, 24, 4, 128, A, A, 8, 64, A, 100, A, A, A, 0.088, A, None,
         None, A, 1 << 20, None),
        (E_SHAPE, "tree_attn_fp8kv", A, 3072, 16, 24, 4, 64, A, A, 8, 64, A, 100, A, A, A, 0.088, A, None,
         None, A, 1 << 20, None),
        (E_SHAPE, "tree_attn_fp8kv", A, 3072, 16, 36, 4, 128, A, A, 8, 64, A, 100, A, A, A, 0.088, A, None,
         None, A, 1 << 20, None),
        (E_ALIGN, "tree_attn_fp8kv", MIS, 3072, 16, 24, 4, 128, A, A, 8, 64, A, 100, A, A, A, 0.088, A, None,
         None, A, 1 << 20, None),
        (E_ARG, "tree_attn_fp8kv", A, 3072, 16, 24, 4, 128, A, A, 8, 64, A, 100, A, A, A, 0.088, A, None,
         A, A, 1 << 20, None),
        # causal_attn_fp8kv(q, ld_q, T, Hq, Hkv, D, k_pool, v_pool, n_pool, P, page_table, ctx_len,
        #                   k_scale, v_scale, sm_scale, out, ws, ws_bytes, stream)
        (E_ARG, "causal_attn_fp8kv", None, 3072, 128, 24, 4, 128, A, A, 8, 64, A, 100, A, A, 0.088, A, A, 1 << 20,
         None),
        (E_SHAPE, "causal_attn_fp8kv", A, 3072, 129, 24, 4, 128, A, A, 8, 64, A, 100, A, A, 0.088, A, A, 1 << 20,
         None),
        (E_SHAPE, "causal_attn_fp8kv", A, 3072, 64, 24, 5, 128, A, A, 8, 64, A, 100, A, A, 0.088, A, A, 1 << 20,
         None),
        (E_ALIGN, "causal_attn_fp8kv", MIS, 3072, 64, 24, 4, 128, A, A, 8, 64, A, 100, A, A, 0.088, A, A, 1 << 20,
         None),
        # kv_page_restore(src, src_ids, dst, dst_ids, n, page_bytes, n_src, n_dst, stream)
        (E_SHAPE, "kv_page_restore", A, A, A, A, 4, 15, 8, 8, None),
        (E_ALIGN, "kv_page_restore", MIS, A, A, A, 4, 32768, 8, 8, None),
        # nvfp4_rmsnorm_quantize(x, w, eps, rows, n, g_in, codes, scales, g_out, act, ws, ws_bytes, stream)
        (E_SHAPE, "nvfp4_rmsnorm_quantize", A, A, 1e-6, 16, 8256, None, A, A, A, None, None, 0, None),
        (E_SHAPE, "nvfp4_rmsnorm_quantize", A, A, 1e-6, 17, 5120, None, A, A, A, None, None, 0, None),
        (E_SHAPE, "nvfp4_rmsnorm_quantize", A, A, 1e-6, 17, 5120, A, A, A, A, A, None, 0, None),
        # nvfp4_swiglu_quantize(gu, rows, F, g_in, codes, scales, g_out, act, ws, ws_bytes, stream)
        (E_SHAPE, "nvfp4_swiglu_quantize", A, 0, 17408, None, A, A, A, None, None, 0, None),
        (E_SHAPE, "nvfp4_swiglu_quantize", A, 17, 17408, None, A, A, A, None, None, 0, None),
        (E_SHAPE, "nvfp4_swiglu_quantize", A, 17, 17408, A, A, A, A, A, None, 0, None),
        # kv_append_fp8(k, v, ld, T, Hkv, D, k_pool, v_pool, n_pool, P, page_table, ctx_len, k_s, v_s, stream)
        (E_SHAPE, "kv_append_fp8", A, A, 4096, 16, 4, 12, A, A, 8, 64, A, 100, A, A, None),
        # argmax_rows_bf16(x, rows, n, ld, idx, ws, ws_bytes, stream)
        (E_SHAPE, "argmax_rows_bf16", A, 5000, 151936, 151936, A, A, 1 << 24, None),
        # tree_accept_greedy(draft, target, parent, T, path, n, next, stream)
        (E_SHAPE, "tree_accept_greedy", A, A, A, 33, A, A, A, None),
        # kv_compact_accepted(k, v, layer_stride, n_layers, Hkv, D, n_pool, P, page_table, ctx_len, path, n, T, stream)
        (E_SHAPE, "kv_compact_accepted", A, A, 1 << 20, 64, 4, 136, 8, 64, A, 100, A, A, 16, None),
        # kv_v_pages_to_tiled(src, dst, n_planes, D, page_size, stream)
        (E_SHAPE, "kv_v_pages_to_tiled", A, A + (1 << 20), 4, 12, 64, None),
        (E_SHAPE, "kv_v_pages_to_tiled", A, A + (1 << 20), 4, 256, 128, None),
        (E_ALIGN, "kv_v_pages_to_tiled", MIS, A + (1 << 20), 4, 128, 64, None),
        (E_ARG, "kv_v_pages_to_tiled", A, A + 8192, 4, 128, 64, None),
        # nvfp4sk_debug_encode(x, n, e2m1, e4m3, stream)
        (E_ARG, "nvfp4sk_debug_encode", A, -1, A, A, None),
    ]
    for want, name, *args in cases:
        got = _rc(name, *args)
        assert got == want, (name, args, got, lib.load().nvfp4sk_last_error())
        assert lib.load().nvfp4sk_last_error(), name
    # an empty restore is a no-op that needs no device
    assert _rc("kv_page_restore", A, A, A, A, 0, 32768, 8, 8, None) == 0


def test_calls_fail_loudly_without_a_gpu():
    """Without a device the library reports an error (no CPU fallback), and
    the binding raises it."""
    import pytest
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = _rc("nvfp4sk_debug_wait_timeout", None)
    assert rc in (-5, -8), rc
    assert lib.load().nvfp4sk_last_error()
    with pytest.raises(lib.NvFp4Error):
        lib._call("nvfp4sk_debug_wait_timeout", None)


def test_binding_rejects_host_tensors():
    """Every tensor argument of the C ABI is a device pointer: the binding
    raises on a host tensor instead of passing its address to a kernel."""
    import pytest
    import torch

    class HostWs:                                   # stands in for a device workspace
        def get(self, n):
            return torch.zeros(max(int(n), 256), dtype=torch.uint8)

    h = lambda *s, dt=torch.uint8: torch.zeros(*s, dtype=dt)
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    g = torch.ones(1)
    calls = [
        lambda: lib.rmsnorm_quantize(bf(16, 64), bf(64), 1e-6, (None, None, g), act=h(8192)),
        lambda: lib.swiglu_quantize(bf(16, 128), (None, None, g), act=h(8192)),
        lambda: lib.prepare_weight(h(128, 32), h(128, 4), 128, 64),
        lambda: lib.prepare_act(h(16, 32), h(16, 4), 64, act=h(8192)),
        lambda: lib.kv_page_restore(h(64), h(1, dt=torch.int32), h(64), h(1, dt=torch.int32), 32),
        lambda: lib.kv_append(bf(16, 384), bf(16, 384), 384, 16, h(2, 1, 64, 128), h(2, 1, 8192),
                              h(2, dt=torch.int32), 0, g, g),
        lambda: lib.tree_accept(h(16, dt=torch.int32), h(16, dt=torch.int32), h(16, dt=torch.int32),
                                out=(h(16, dt=torch.int32), h(1, dt=torch.int32), h(1, dt=torch.int32))),
        lambda: lib.linear(h(8192), g, 16, h(36864), g, 128, 512, y=bf(16, 128), ws=HostWs()),
        lambda: lib.tree_attn(bf(16, 24, 128), h(2, 4, 64, 128), h(2, 4, 8192), h(2, dt=torch.int32), 10,
                              h(16, dt=torch.int32), g, g, out=bf(16, 24, 128), ws=HostWs()),
        lambda: lib.argmax(bf(16, 4096), idx=h(16, dt=torch.int32), ws=HostWs()),
        lambda: lib.v_pages_to_tiled(h(2, 64, 128), h(2, 8192)),
        lambda: lib.linear_wide(h(36864), g, 20, h(36864), g, 128, 512, y=bf(20, 128)),
        lambda: lib.causal_attn(bf(32, 24, 128), h(2, 4, 64, 128), h(2, 4, 8192), h(2, dt=torch.int32), 10,
                                g, g, out=bf(32, 24, 128), ws=HostWs()),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(ValueError, match="device tensor"):
            call()


def test_failing_status_rezeroes_counter_workspaces(monkeypatch):
    """After a failing device status the binding zeroes its default linear,
    argmax and attention workspaces (their arrival counters may be stale after
    a wait ran out) and leaves the others alone; a clean status touches nothing."""
    import torch

    class FakeWs:
        def __init__(self):
            self.buf = torch.full((64,), 7, dtype=torch.uint8)

    spaces = {(0, k): FakeWs() for k in ("linear", "argmax", "attn", "quantize")}
    monkeypatch.setattr(lib, "_default_ws", spaces)
    state = {"rc": 0}

    class FakeLib:
        def nvfp4sk_get_device_status(self, stream, site):
            return state["rc"]

    monkeypatch.setattr(lib, "load", lambda path=None: FakeLib())
    monkeypatch.setattr(lib, "_stream", lambda s=None: None)
    assert lib.device_status()[0] == 0
    assert all(int(w.buf.min()) == 7 for w in spaces.values())
    state["rc"] = -6
    assert lib.device_status()[0] == -6
    for (_, kind), w in spaces.items():
        want = 0 if kind in ("linear", "argmax", "attn") else 7
        assert int(w.buf.min()) == want and int(w.buf.max()) == want, kind


def test_option_block_restores_the_previous_value():
    """lib.option sets a library option for the calls inside the block and
    puts the previous value back, on an exception too."""
    lib.load()
    assert lib.get_option(lib.OPT_ATTN_SPLITS) == 0
    with lib.option(lib.OPT_ATTN_SPLITS, 3):
        assert lib.get_option(lib.OPT_ATTN_SPLITS) == 3
    assert lib.get_option(lib.OPT_ATTN_SPLITS) == 0
    try:
        with lib.option(lib.OPT_ATTN_SPLITS, 5):
            raise KeyError("inside")
    except KeyError:
        pass
    assert lib.get_option(lib.OPT_ATTN_SPLITS) == 0


def test_attention_launch_count_follows_the_split_grid():
    """One launch (split kernel with the combine fused) only when the fused
    combine is on and the split grid fits on the GPU at once; an explicit
    split count whose grid is not given counts two."""
    lib.load()
    assert lib.attn_launches() == 2
    with lib.option(lib.OPT_ATTN_FUSED_COMBINE, 1):
        assert lib.attn_launches() == 1
        with lib.option(lib.OPT_ATTN_SPLITS, 3):
            assert lib.attn_launches() == 2
            assert lib.attn_launches(3 * 24, 148) == 1
            assert lib.attn_launches(7 * 24, 148) == 2
    assert lib.attn_launches(3 * 24, 148) == 2


def test_prefill_split_count_rule():
    """The prefill gives its causal calls PREFILL_ATTN_SPLITS splits only on
    the GPU with at least four blocks in flight, and leaves a split count the
    caller set alone."""
    import types
    import torch
    from nvfp4_skinny_gemm_b200 import step
    lib.load()
    gpu = types.SimpleNamespace(dev=torch.device("cuda", 0))
    cpu = types.SimpleNamespace(dev=torch.device("cpu"))
    f = step.VerifyModel._causal_splits
    assert f(gpu, 8) == f(gpu, 4) == step.PREFILL_ATTN_SPLITS
    assert f(gpu, 3) == f(gpu, 1) == 0
    assert f(cpu, 8) == 0
    with lib.option(lib.OPT_ATTN_SPLITS, 5):
        assert f(gpu, 8) == 0
