"""ctypes binding of libnvfp4sk (C ABI in include/nvfp4sk.h).

Argument marshalling only: every step runs in the CUDA library.  Functions
take torch CUDA tensors (or None), pass their device pointers and the current
CUDA stream, and raise NvFp4Error on a non-zero status.  If the shared library
is missing, the first call raises -- there is no CPU fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libnvfp4sk.so")
HEADER = os.path.join(ROOT, "include", "nvfp4sk.h")

BF16, FP32 = 0, 1
OPT_PDL, OPT_TIMEOUT_NS, OPT_ATTN_SPLITS, OPT_LINEAR_CTAS, OPT_ATTN_FUSED_COMBINE = 0, 1, 2, 3, 4
STATUS = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED_SHAPE", -3: "MISALIGNED", -4: "WORKSPACE",
          -5: "CUDA", -6: "TIMEOUT", -7: "OUT_OF_RANGE", -8: "DEVICE"}


class NvFp4Error(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn}: {STATUS.get(code, code)} ({code}): {msg}")
        self.code = code


_lib = None
_vp, _i64, _int, _sz, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float

_SIGS = {
    "nvfp4_quantize_workspace_bytes": (_sz, [_i64, _i64]),
    "nvfp4_prepared_act_bytes": (_sz, [_i64]),
    "nvfp4_quantize_act": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_prepare_act": (_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "nvfp4_prepared_weight_bytes": (_sz, [_i64, _i64]),
    "nvfp4_prepare_weight": (_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "nvfp4_linear_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "nvfp4_linear": (_int, [_vp, _vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _sz, _vp]),
    "nvfp4_linear_wide": (_int, [_vp, _vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp]),
    "nvfp4_linear_swiglu_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "nvfp4_linear_swiglu": (_int, [_vp, _vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_linear_noalloc_scratch_bytes": (_sz, []),
    "nvfp4_linear_noalloc": (_int, [_vp, _vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp]),
    "tree_attn_workspace_bytes": (_sz, [_int, _int, _int, _int, _int, _i64]),
    "tree_attn_fp8kv": (_int, [_vp, _i64, _int, _int, _int, _int, _vp, _vp, _i64, _int, _vp, _i64, _vp, _vp,
                               _vp, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "causal_attn_workspace_bytes": (_sz, [_int, _int, _int, _int, _int, _i64]),
    "causal_attn_fp8kv": (_int, [_vp, _i64, _int, _int, _int, _int, _vp, _vp, _i64, _int, _vp, _i64, _vp, _vp,
                                 _f32, _vp, _vp, _sz, _vp]),
    "kv_page_restore": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp]),
    "kv_v_pages_to_tiled": (_int, [_vp, _vp, _i64, _int, _int, _vp]),
    "nvfp4_rmsnorm_quantize": (_int, [_vp, _vp, _f32, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_swiglu_quantize": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_quantize_act_tiles": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "nvfp4_rmsnorm_quantize_tiles": (_int, [_vp, _vp, _f32, _i64, _i64, _vp, _vp, _vp, _vp]),
    "nvfp4_swiglu_quantize_tiles": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "kv_append_fp8": (_int, [_vp, _vp, _i64, _int, _int, _int, _vp, _vp, _i64, _int, _vp, _i64, _vp, _vp, _vp]),
    "argmax_workspace_bytes": (_sz, [_i64, _i64]),
    "argmax_rows_bf16": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _sz, _vp]),
    "nvfp4sk_get_device_status": (_int, [_vp, ctypes.POINTER(_int)]),
    "nvfp4sk_last_error": (ctypes.c_char_p, []),
    "nvfp4sk_version": (_int, []),
    "nvfp4sk_set_option": (_int, [_int, _i64]),
    "nvfp4sk_get_option": (_i64, [_int]),
    "nvfp4sk_debug_encode": (_int, [_vp, _i64, _vp, _vp, _vp]),
    "nvfp4sk_debug_wait_timeout": (_int, [_vp]),
    "tree_accept_greedy": (_int, [_vp, _vp, _vp, _int, _vp, _vp, _vp, _vp]),
    "kv_compact_accepted": (_int, [_vp, _vp, _i64, _int, _int, _int, _i64, _int, _vp, _i64, _vp, _vp, _int, _vp]),
}


def header_symbols():
    """Names of the functions include/nvfp4sk.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^NVFP4SK_API [^(]*?\b([a-z_0-9]+)\(", txt, re.M)))


def load(path: str = LIB_PATH):
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libnvfp4sk.so not found at {path}; build it with "
                               "`python -m nvfp4_skinny_gemm_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _d(t):
    """Device address of a CUDA tensor; an int passes through as a raw device
    address.  A host tensor raises here rather than reaching a kernel."""
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"a device tensor is expected, got one on {t.device}")
    return t.data_ptr()


def _p(t):
    return None if t is None else _d(t)


def _stream(stream=None):
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def _check(name, rc):
    if rc != 0:
        raise NvFp4Error(name, rc, load().nvfp4sk_last_error().decode())


def _call(name, *args):
    _check(name, getattr(load(), name)(*args))


class Workspace:
    """Zero-filled device scratch that grows on demand (kept zeroed by the calls)."""

    def __init__(self, device=None):
        self.buf = None
        self.device = device

    def get(self, nbytes: int) -> torch.Tensor:
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device or "cuda")
        return self.buf


_default_ws = {}


def default_workspace(kind, slot=0):
    """The library's default workspace of an op kind on the current device;
    slot > 0: another one of the same kind (for calls of that kind that run
    at the same time on other streams), zeroed like the default after a
    failing device status."""
    dev = torch.cuda.current_device()
    key = kind if slot == 0 else f"{kind}#{slot}"
    return _default_ws.setdefault((dev, key), Workspace(f"cuda:{dev}"))


def _ws(ws, nbytes, kind):
    """Workspace pointer and size; by default one zero-filled buffer per
    (device, op kind): the linear and argmax workspaces hold arrival counters
    that must read zero at call start, which another op's partials would break."""
    if ws is None:
        ws = default_workspace(kind)
    buf = ws.get(nbytes)
    return buf.data_ptr(), buf.numel()


# ------------------------------------------------------------------ calls
def set_option(opt, value):
    _call("nvfp4sk_set_option", opt, int(value))


def attn_launches(ctas=None, sms=None):
    """Kernel launches per tree_attn / causal_attn call: 1 with the fused
    combine (OPT_ATTN_FUSED_COMBINE on and the whole split grid resident at
    once, one CTA per SM), else 2 (split, then combine).  The library's own
    split counts always give a grid that fits; for a call made at an explicit
    OPT_ATTN_SPLITS, pass its grid size (ctas = splits x heads) and the
    device's SM count (sms), else 2 is assumed."""
    if not get_option(OPT_ATTN_FUSED_COMBINE):
        return 2
    if get_option(OPT_ATTN_SPLITS) <= 0:
        return 1
    return 1 if ctas is not None and sms is not None and ctas <= sms else 2


@contextlib.contextmanager
def option(opt, value):
    """Set a library option for the calls made inside the block, then put its
    previous value back."""
    old = get_option(opt)
    set_option(opt, value)
    try:
        yield
    finally:
        set_option(opt, old)


def get_option(opt):
    return load().nvfp4sk_get_option(opt)


# default workspaces whose arrival counters must read zero when a call starts
_COUNTER_KINDS = ("linear", "linear_swiglu", "argmax", "attn")


def _rezero_counter_workspaces():
    """Zero the default linear / argmax / attention workspaces of every device: a call whose
    device wait ran out can leave their arrival counters non-zero, and the next
    call on the same workspace would count stale arrivals."""
    for (dev, kind), ws in _default_ws.items():
        if kind.split("#")[0] in _COUNTER_KINDS and ws.buf is not None:
            ws.buf.zero_()


def device_status(stream=None):
    """(status code, site): synchronises the stream, reads and clears the error
    word.  On a non-zero status the default linear, argmax and attention workspaces are
    zeroed again (stream-ordered on the current stream), as the C ABI's
    workspace rule asks of every caller-owned workspace after a failure."""
    site = _int(0)
    rc = load().nvfp4sk_get_device_status(_stream(stream), ctypes.byref(site))
    if rc != 0:
        _rezero_counter_workspaces()
    return rc, site.value


def act_buffer(K: int, device=None) -> torch.Tensor:
    """Zero-filled prepared-activation buffer for K input features."""
    return torch.zeros(load().nvfp4_prepared_act_bytes(K), dtype=torch.uint8, device=device or "cuda")


def quantize(x: torch.Tensor, g_in: torch.Tensor | None = None, out=None, act: torch.Tensor | None = None,
             canonical: bool = True, ws=None, stream=None):
    """NVFP4-quantise x [rows, K] (bf16 or fp32, row stride x.stride(0)).

    Returns (codes u8 [rows, K/2], scales u8 [rows, K/16], g f32 [1]); with
    act (a buffer from act_buffer) the prepared tile image is written too;
    canonical=False skips the canonical outputs (codes/scales are None)."""
    rows, K = x.shape
    assert x.stride(1) == 1
    dt = BF16 if x.dtype == torch.bfloat16 else FP32
    if out is None:
        out = (torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device) if canonical else None,
               torch.empty(rows, K // 16, dtype=torch.uint8, device=x.device) if canonical else None,
               torch.empty(1, dtype=torch.float32, device=x.device))
    codes, scales, g = out
    wp, wn = _ws(ws, load().nvfp4_quantize_workspace_bytes(rows, K), "quantize")
    _call("nvfp4_quantize_act", _d(x), dt, rows, K, x.stride(0), _p(g_in), _p(codes), _p(scales),
          _d(g), _p(act), wp, wn, _stream(stream))
    return codes, scales, g


def prepare_act(codes: torch.Tensor, scales: torch.Tensor, K: int, act=None, stream=None):
    rows = codes.shape[0]
    if act is None:
        act = act_buffer(K, codes.device)
    _call("nvfp4_prepare_act", _d(codes), _d(scales), rows, K, _d(act), _stream(stream))
    return act


def prepared_weight_bytes(N: int, K: int) -> int:
    return load().nvfp4_prepared_weight_bytes(N, K)


def prepare_weight(codes: torch.Tensor, scales: torch.Tensor, N: int, K: int, out=None, stream=None):
    """Tile image of an NVFP4 matrix (a weight, or an activation of many tokens
    for nvfp4_linear_wide); out: a device buffer of at least
    prepared_weight_bytes(N, K) bytes, or None to allocate one."""
    if out is None:
        out = torch.empty(load().nvfp4_prepared_weight_bytes(N, K), dtype=torch.uint8, device=codes.device)
    elif out.numel() < load().nvfp4_prepared_weight_bytes(N, K):
        raise ValueError("prepare_weight: out is too small")
    _call("nvfp4_prepare_weight", _d(codes), _d(scales), N, K, _d(out), _stream(stream))
    return out


def linear(a_act, g_a, M, w_prep, g_w, N, K, y=None, residual=None, ws=None, stream=None):
    """Y [M, N] bf16 = NVFP4 linear (+ residual) on prepared operands."""
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=a_act.device)
    wp, wn = _ws(ws, load().nvfp4_linear_workspace_bytes(M, N, K), "linear")
    _call("nvfp4_linear", _d(a_act), _d(g_a), M, _d(w_prep), _d(g_w), N, K,
          _p(residual), _d(y), y.stride(0), wp, wn, _stream(stream))
    return y


def linear_swiglu(a_act, g_a, M, w_prep, g_w, F, K, g_out, act, ws=None, stream=None):
    """gate+up linear ([2F, K] weight, gate rows first) with SwiGLU and its NVFP4
    quantisation (static scale g_out) in the epilogue: writes the prepared
    F-wide activation of the down linear into act (rows < M)."""
    wp, wn = _ws(ws, load().nvfp4_linear_swiglu_workspace_bytes(M, F, K), "linear_swiglu")
    _call("nvfp4_linear_swiglu", _d(a_act), _d(g_a), M, _d(w_prep), _d(g_w), F, K, _d(g_out), _d(act), wp, wn,
          _stream(stream))
    return act


def linear_wide(a_prep, g_a, S, w_prep, g_w, N, K, y=None, residual=None, stream=None):
    """Y [S, N] bf16 = NVFP4 linear (+ residual) for S tokens; a_prep is the
    activation in the weight tile image (prepare_weight of its codes/scales)."""
    if y is None:
        y = torch.empty(S, N, dtype=torch.bfloat16, device=a_prep.device)
    _call("nvfp4_linear_wide", _d(a_prep), _d(g_a), S, _d(w_prep), _d(g_w), N, K,
          _p(residual), _d(y), y.stride(0), _stream(stream))
    return y


def tree_attn(q, k_pool, v_pool, page_table, ctx_len, parent, k_scale, v_scale, sm_scale=None, out=None,
              ld_q=None, T=None, Hq=None, ws=None, stream=None, g_act=None, act=None):
    """q bf16 [T, Hq, D] (or a strided [T, >= Hq*D] view with ld_q); pools u8
    [pages, Hkv, P, D] / [pages, Hkv, D*P] (tiled V planes); returns bf16 [T, Hq, D].
    With act (prepared activation buffer) and g_act (static tensor scale), the
    output is also quantised to NVFP4 in the same launch."""
    n_pages, Hkv, P, D = k_pool.shape
    if T is None:
        T, Hq = q.shape[0], q.shape[1]
    if ld_q is None:
        ld_q = q.stride(0)
    if sm_scale is None:
        sm_scale = D ** -0.5
    if out is None:
        out = torch.empty(T, Hq, D, dtype=torch.bfloat16, device=q.device)
    wp, wn = _ws(ws, load().tree_attn_workspace_bytes(T, Hq, Hkv, D, P, int(ctx_len)), "attn")
    _call("tree_attn_fp8kv", _d(q), ld_q, T, Hq, Hkv, D, _d(k_pool), _d(v_pool), n_pages, P,
          _d(page_table), int(ctx_len), _d(parent), _d(k_scale), _d(v_scale),
          float(sm_scale), _d(out), _p(g_act), _p(act), wp, wn, _stream(stream))
    return out


def causal_attn(q, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale, sm_scale=None, out=None, ld_q=None,
                T=None, Hq=None, ws=None, stream=None):
    """Causal attention of T <= 128 new tokens (positions ctx_len ..) over the
    FP8 paged cache; q bf16 [T, Hq, D] or a strided view with ld_q; returns
    bf16 [T, Hq, D]."""
    n_pages, Hkv, P, D = k_pool.shape
    if T is None:
        T, Hq = q.shape[0], q.shape[1]
    if ld_q is None:
        ld_q = q.stride(0)
    if sm_scale is None:
        sm_scale = D ** -0.5
    if out is None:
        out = torch.empty(T, Hq, D, dtype=torch.bfloat16, device=q.device)
    wp, wn = _ws(ws, load().causal_attn_workspace_bytes(T, Hq, Hkv, D, P, int(ctx_len)), "attn")
    _call("causal_attn_fp8kv", _d(q), ld_q, T, Hq, Hkv, D, _d(k_pool), _d(v_pool), n_pages, P,
          _d(page_table), int(ctx_len), _d(k_scale), _d(v_scale), float(sm_scale), _d(out), wp, wn,
          _stream(stream))
    return out


def kv_page_restore(src_pool, src_ids, dst_pool, dst_ids, page_bytes, n=None, stream=None):
    n = src_ids.numel() if n is None else n
    _call("kv_page_restore", _d(src_pool), _d(src_ids), _d(dst_pool), _d(dst_ids), n,
          page_bytes, src_pool.numel() // page_bytes, dst_pool.numel() // page_bytes, _stream(stream))


def v_pages_to_tiled(v_token_major, v_tiled=None, stream=None):
    """Token-major V planes u8 [n, page_size, D] -> the tiled plane layout the
    attention reads, u8 [n, D*page_size] (a byte permutation)."""
    n, P, D = v_token_major.shape
    if v_tiled is None:
        v_tiled = torch.empty(n, D * P, dtype=torch.uint8, device=v_token_major.device)
    _call("kv_v_pages_to_tiled", _d(v_token_major), _d(v_tiled), n, D, P, _stream(stream))
    return v_tiled


def rmsnorm_quantize(x, w, eps, out, act=None, stream=None, g_in=None):
    """out = (codes or None, scales or None, g); act: prepared buffer or None;
    g_in: static tensor scale (device [1]) or None for the dynamic one."""
    rows, n = x.shape
    codes, scales, g = out
    _call("nvfp4_rmsnorm_quantize", _d(x), _d(w), float(eps), rows, n, _p(g_in), _p(codes),
          _p(scales), _d(g), _p(act), None, 0, _stream(stream))
    return out


def swiglu_quantize(gu, out, act=None, stream=None, g_in=None):
    rows, F2 = gu.shape
    codes, scales, g = out
    _call("nvfp4_swiglu_quantize", _d(gu), rows, F2 // 2, _p(g_in), _p(codes), _p(scales), _d(g),
          _p(act), None, 0, _stream(stream))
    return out


def quantize_tiles(x, g_in, tiles, g_out, stream=None):
    """NVFP4 of x [rows, K] with the static scale g_in straight into the tile
    image nvfp4_linear_wide streams (tokens as rows); g_out receives g_in."""
    rows, K = x.shape
    assert x.stride(1) == 1
    dt = BF16 if x.dtype == torch.bfloat16 else FP32
    _call("nvfp4_quantize_act_tiles", _d(x), dt, rows, K, x.stride(0), _d(g_in), _d(g_out), _d(tiles),
          _stream(stream))
    return tiles


def rmsnorm_quantize_tiles(x, w, eps, g_in, tiles, g_out, stream=None):
    """rmsnorm_quantize with a static scale into the wide tile image."""
    rows, n = x.shape
    _call("nvfp4_rmsnorm_quantize_tiles", _d(x), _d(w), float(eps), rows, n, _d(g_in), _d(g_out), _d(tiles),
          _stream(stream))
    return tiles


def swiglu_quantize_tiles(gu, g_in, tiles, g_out, stream=None):
    """swiglu_quantize with a static scale into the wide tile image."""
    rows, F2 = gu.shape
    _call("nvfp4_swiglu_quantize_tiles", _d(gu), rows, F2 // 2, _d(g_in), _d(g_out), _d(tiles), _stream(stream))
    return tiles


def kv_append(k_new, v_new, ld_new, T, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale, stream=None):
    n_pages, Hkv, P, D = k_pool.shape
    _call("kv_append_fp8", _d(k_new),
          _d(v_new), ld_new, T, Hkv, D, _d(k_pool),
          _d(v_pool), n_pages, P, _d(page_table), int(ctx_len), _d(k_scale),
          _d(v_scale), _stream(stream))


def tree_accept(draft_tokens, target_argmax, parent, out=None, stream=None):
    """Greedy acceptance: returns device tensors (path i32 [T], n i32 [1], next i32 [1])."""
    T = parent.numel()
    if out is None:
        dev = parent.device
        out = (torch.empty(T, dtype=torch.int32, device=dev), torch.empty(1, dtype=torch.int32, device=dev),
               torch.empty(1, dtype=torch.int32, device=dev))
    path, n, nxt = out
    _call("tree_accept_greedy", _d(draft_tokens), _d(target_argmax), _d(parent), T,
          _d(path), _d(n), _d(nxt), _stream(stream))
    return out


def kv_compact(k_base, v_base, layer_stride, n_layers, Hkv, D, n_pool_pages, P, page_table, ctx_len, path, n, T,
               stream=None):
    """Move the accepted tokens' K/V to ctx_len .. in every layer (see kv_compact_accepted)."""
    _call("kv_compact_accepted", k_base, v_base, int(layer_stride), n_layers, Hkv, D, int(n_pool_pages), P,
          _d(page_table), int(ctx_len), _d(path), _d(n), T, _stream(stream))


def argmax(x, idx=None, ws=None, stream=None):
    rows, n = x.shape
    if idx is None:
        idx = torch.empty(rows, dtype=torch.int32, device=x.device)
    wp, wn = _ws(ws, load().argmax_workspace_bytes(rows, n), "argmax")
    _call("argmax_rows_bf16", _d(x), rows, n, x.stride(0), _d(idx), wp, wn, _stream(stream))
    return idx


def debug_encode(x: torch.Tensor, stream=None):
    n = x.numel()
    e2 = torch.empty(n, dtype=torch.uint8, device=x.device)
    e4 = torch.empty(n, dtype=torch.uint8, device=x.device)
    _call("nvfp4sk_debug_encode", _d(x), n, _d(e2), _d(e4), _stream(stream))
    return e2, e4
