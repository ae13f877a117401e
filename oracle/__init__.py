"""CPU oracle for the tree-MTP verification step (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` import this package.  It is a thin
numpy/ctypes wrapper over ``oracle.c`` (plain fp64 C) plus a few plain numpy
compositions; it imports nothing from the CUDA package.

What is computed, and where the pages leave it open, is documented in
``oracle.c``; the codec definitions follow the OCP MX v1.0 (E2M1) and OCP OFP8
(E4M3) specifications.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_int = ctypes.c_int


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_e2m1_value.argtypes = [_int]; L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [_int]; L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e2m1_encode.argtypes = [ctypes.c_double]; L.oracle_e2m1_encode.restype = _int
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]; L.oracle_e4m3_encode.restype = _int
        L.oracle_e2m1_table.argtypes = [_f64p]; L.oracle_e2m1_table.restype = None
        L.oracle_e4m3_table.argtypes = [_f64p]; L.oracle_e4m3_table.restype = None
        L.oracle_encode_many.argtypes = [_f32p, _i64, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_encode_many.restype = None
        L.oracle_nvfp4_tensor_scale.argtypes = [_f32p, _i64]
        L.oracle_nvfp4_tensor_scale.restype = ctypes.c_float
        L.oracle_nvfp4_quantize.argtypes = [_f32p, _i64, _i64, ctypes.c_void_p, _u8p, _u8p,
                                            ctypes.POINTER(ctypes.c_float)]
        L.oracle_nvfp4_quantize.restype = _int
        L.oracle_nvfp4_dequantize.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _i64, _f64p]
        L.oracle_nvfp4_dequantize.restype = None
        L.oracle_nvfp4_linear.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _u8p, _u8p,
                                          ctypes.c_float, _i64, _i64, _f64p]
        L.oracle_nvfp4_linear.restype = None
        L.oracle_nvfp4_linear_sampled.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                                  ctypes.c_float, _i64, _i64p, _i64p, _i64, _f64p]
        L.oracle_nvfp4_linear_sampled.restype = None
        L.oracle_tree_attn.argtypes = [_f32p, _int, _int, _int, _int, _u8p, _u8p, _i64, _int,
                                       _i32p, _i64, _i32p, _f32p, _f32p, ctypes.c_double, _f64p]
        L.oracle_tree_attn.restype = _int
        L.oracle_kv_append.argtypes = [_f32p, _f32p, _int, _int, _int, _u8p, _u8p, _i64, _int,
                                       _i32p, _i64, _f32p, _f32p]
        L.oracle_kv_append.restype = _int
        L.oracle_kv_page_restore.argtypes = [_u8p, _i32p, _u8p, _i32p, _i64, _i64, _i64, _i64]
        L.oracle_kv_page_restore.restype = _int
        L.oracle_rmsnorm.argtypes = [_f32p, _i64, _i64, _f32p, ctypes.c_double, _f64p]
        L.oracle_rmsnorm.restype = None
        L.oracle_swiglu.argtypes = [_f32p, _i64, _i64, _f64p]
        L.oracle_swiglu.restype = None
        _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- codecs
def e2m1_table() -> np.ndarray:
    t = np.zeros(16, np.float64)
    lib().oracle_e2m1_table(t)
    return t


def e4m3_table() -> np.ndarray:
    t = np.zeros(256, np.float64)
    lib().oracle_e4m3_table(t)
    return t


def e2m1_encode(v: float) -> int:
    return lib().oracle_e2m1_encode(float(v))


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(v))


def encode_many(x):
    """One E2M1 code and one E4M3 code per float (RNE, satfinite)."""
    x = _f32(x).ravel()
    e2 = np.zeros(x.size, np.uint8)
    e4 = np.zeros(x.size, np.uint8)
    lib().oracle_encode_many(x, x.size, e2.ctypes.data, e4.ctypes.data)
    return e2, e4


# ---------------------------------------------------------------- NVFP4
def tensor_scale(x) -> float:
    x = _f32(x).ravel()
    return float(lib().oracle_nvfp4_tensor_scale(x, x.size))


def quantize(x, g_in=None):
    """NVFP4-quantise x [rows, K] (fp32 values, e.g. exact bf16 widened).

    Returns (codes u8 [rows, K/2], scales u8 [rows, K/16], g float)."""
    x = _f32(x)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    g = ctypes.c_float(0.0)
    gin = None
    if g_in is not None:
        gin_arr = (ctypes.c_float * 1)(float(g_in))
        gin = ctypes.cast(gin_arr, ctypes.c_void_p)
    rc = lib().oracle_nvfp4_quantize(x, rows, K, gin, codes, scales, ctypes.byref(g))
    if rc != 0:
        raise ValueError("K must be a multiple of 16")
    return codes, scales, float(g.value)


def dequantize(codes, scales, g):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, K), np.float64)
    lib().oracle_nvfp4_dequantize(codes, scales, float(g), rows, K, out)
    return out


def linear(a_codes, a_scales, g_a, w_codes, w_scales, g_w):
    """Y [M, N] = (A W^T) in fp64 from NVFP4 operands."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    w_codes = np.ascontiguousarray(w_codes, np.uint8)
    w_scales = np.ascontiguousarray(w_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    y = np.zeros((M, N), np.float64)
    lib().oracle_nvfp4_linear(a_codes, a_scales, float(g_a), M, w_codes, w_scales, float(g_w), N, K, y)
    return y


def linear_sampled(a_codes, a_scales, g_a, w_codes, w_scales, g_w, idx_m, idx_n):
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    w_codes = np.ascontiguousarray(w_codes, np.uint8)
    w_scales = np.ascontiguousarray(w_scales, np.uint8)
    K = a_codes.shape[1] * 2
    im = np.ascontiguousarray(idx_m, np.int64)
    inn = np.ascontiguousarray(idx_n, np.int64)
    y = np.zeros(im.size, np.float64)
    lib().oracle_nvfp4_linear_sampled(a_codes, a_scales, float(g_a), w_codes, w_scales, float(g_w),
                                      K, im, inn, im.size, y)
    return y


# ---------------------------------------------------------------- attention
def tree_attn(q, k_pool, v_pool, page_table, ctx_len, parent, k_scale, v_scale, sm_scale=None):
    """q [T, Hq, D]; k_pool u8 [pages, Hkv, P, D]; v_pool u8 [pages, Hkv, D*P]
    (8-dimension x 16-slot tiles of 128 bytes, tile (d//8, slot//16) at index
    (d//8)*(P//16) + slot//16)."""
    q = _f32(q)
    T, Hq, D = q.shape
    k_pool = np.ascontiguousarray(k_pool, np.uint8)
    v_pool = np.ascontiguousarray(v_pool, np.uint8)
    n_pages, Hkv, P, D2 = k_pool.shape
    assert D2 == D and v_pool.shape == (n_pages, Hkv, D * P) and D % 8 == 0 and P % 16 == 0
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.zeros((T, Hq, D), np.float64)
    rc = lib().oracle_tree_attn(q, T, Hq, Hkv, D, k_pool, v_pool, n_pages, P,
                                np.ascontiguousarray(page_table, np.int32), int(ctx_len),
                                np.ascontiguousarray(parent, np.int32), _f32(k_scale), _f32(v_scale),
                                float(sm_scale), out)
    if rc != 0:
        raise ValueError(f"oracle_tree_attn failed ({rc})")
    return out


def kv_append(k_new, v_new, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale):
    """In place: write T new tokens' K/V [T, Hkv, D] at positions ctx_len.. as E4M3."""
    k_new = _f32(k_new)
    v_new = _f32(v_new)
    T, Hkv, D = k_new.shape
    n_pages, _, P, _ = k_pool.shape
    rc = lib().oracle_kv_append(k_new, v_new, T, Hkv, D, k_pool, v_pool, n_pages, P,
                                np.ascontiguousarray(page_table, np.int32), int(ctx_len),
                                _f32(k_scale), _f32(v_scale))
    if rc != 0:
        raise ValueError("page id out of range")


def kv_page_restore(src_pool, src_ids, dst_pool, dst_ids, page_bytes):
    """In place on dst_pool (flat u8 arrays)."""
    src_ids = np.ascontiguousarray(src_ids, np.int32)
    dst_ids = np.ascontiguousarray(dst_ids, np.int32)
    rc = lib().oracle_kv_page_restore(src_pool, src_ids, dst_pool, dst_ids, src_ids.size, page_bytes,
                                      src_pool.size // page_bytes, dst_pool.size // page_bytes)
    if rc != 0:
        raise ValueError("page id out of range")


# ---------------------------------------------------------------- glue
def rmsnorm(x, w, eps=1e-6):
    x = _f32(x)
    rows, n = x.shape
    out = np.zeros((rows, n), np.float64)
    lib().oracle_rmsnorm(x, rows, n, _f32(w), float(eps), out)
    return out


def swiglu(gu):
    gu = _f32(gu)
    rows, F2 = gu.shape
    out = np.zeros((rows, F2 // 2), np.float64)
    lib().oracle_swiglu(gu, rows, F2 // 2, out)
    return out


def ancestors(parent, i):
    """anc(i) = {i} u anc(parent(i)), anc(-1) = {}."""
    out = []
    while i >= 0:
        out.append(i)
        i = int(parent[i])
    return out


# ---------------------------------------------------------------- greedy tree acceptance
# The step after the verify forward ("Tree multi-token prediction": one target
# pass checks every candidate of the tree and the path that agrees with the
# target is kept; at temperature 0 that is exact): node 0 (the root, the
# last accepted token) is accepted; node i >= 1 is accepted when its parent is
# accepted and its draft token equals the target's greedy choice after the
# parent.  The accepted path ends at the deepest accepted node (lowest index
# among equally deep ones); the next token is the target's choice after it.
def tree_accept_greedy(draft_tokens, target_argmax, parent):
    """Returns (path [root .. end] as a list of node indices, next token)."""
    T = len(parent)
    accepted = [False] * T
    depth = [0] * T
    for i in range(T):                       # parents precede children
        p = int(parent[i])
        if p < 0:
            accepted[i] = i == 0
            depth[i] = 0
        else:
            depth[i] = depth[p] + 1
            accepted[i] = accepted[p] and int(draft_tokens[i]) == int(target_argmax[p])
    end = 0
    for i in range(T):
        if accepted[i] and depth[i] > depth[end]:
            end = i
    path = []
    i = end
    while i >= 0:
        path.append(i)
        i = int(parent[i])
    path.reverse()
    return path, int(target_argmax[end])


def kv_compact_accepted(k_pool, v_pool, page_table, ctx_len, path):
    """In place on one layer's pools (k [pages, Hkv, P, D], v [pages, Hkv, D*P]
    in the tiled plane layout): the K/V of path node path[k], stored at logical
    position ctx_len + path[k], is moved to position ctx_len + k, so that the
    accepted tokens follow the context contiguously.  Each moved token is read
    before anything is written."""
    n_pages, Hkv, P, D = k_pool.shape

    def v_off(d, t):                         # tile (d//8, t//16) of 8 x 16 bytes
        return ((d // 8) * (P // 16) + t // 16) * 128 + (d % 8) * 16 + t % 16

    def where(pos):
        return int(page_table[pos // P]), pos % P

    ks, vs = [], []
    for node in path:
        pg, sl = where(ctx_len + node)
        ks.append(k_pool[pg, :, sl, :].copy())
        vs.append(np.array([[v_pool[pg, h, v_off(d, sl)] for d in range(D)] for h in range(Hkv)], np.uint8))
    for k in range(len(path)):
        pg, sl = where(ctx_len + k)
        k_pool[pg, :, sl, :] = ks[k]
        for h in range(Hkv):
            for d in range(D):
                v_pool[pg, h, v_off(d, sl)] = vs[k][h, d]


# ---------------------------------------------------------------- one decoder layer
def bf16(x):
    """Nearest bf16 of each value, as an fp64 array: round to fp32 first (as
    the kernels hold their results), then to the upper 16 bits of the fp32
    pattern, ties to even.  Finite, in-range inputs only."""
    f = np.asarray(x, np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def decoder_layer(h, norm_w1, norm_w2, weights, G, k_pool, v_pool, page_table, ctx_len, parent, k_scale,
                  v_scale, Hq, eps=1e-6):
    """One pre-norm decoder layer of the verify step on the T rows of h, as
    the step composes it ("NVFP4 and FP8": NVFP4 weights and activations, FP8
    KV cache; "Tree multi-token prediction": the T rows are the tree's nodes):

        y1 = bf16(RMSNorm(h)),            qkv = bf16(NVFP4(y1) x W_qkv^T),
        FP8 append of the rows' K/V at ctx_len .., a = bf16(tree attention),
        h1 = bf16(h + NVFP4(a) x W_o^T),  y2 = bf16(RMSNorm(h1)),
        gu = bf16(NVFP4(y2) x W_gu^T),    s = bf16(SwiGLU(gu)),
        h2 = bf16(h1 + NVFP4(s) x W_down^T).

    weights: name -> (codes, scales, g) of 'qkv', 'o', 'gate_up', 'down';
    G: the four activation scales (norm1, attention out, norm2, SwiGLU) of a
    calibrated checkpoint, or None for the dynamic amax/2688 of each tensor.
    The pools (k [pages, Hkv, P, D], v [pages, Hkv, D*P]) are updated in place.
    Returns a dict of every intermediate (fp64 arrays of bf16 values)."""
    h = np.asarray(h, np.float64)
    T = h.shape[0]
    _, Hkv, _, D = k_pool.shape
    qd, kd = Hq * D, Hkv * D

    def lin(x, name, site):
        ac, asc, ga = quantize(x, g_in=None if G is None else float(G[site]))
        return linear(ac, asc, ga, *weights[name])

    r = {"h": h}
    r["y1"] = bf16(rmsnorm(h, norm_w1, eps))
    r["qkv"] = bf16(lin(r["y1"], "qkv", 0))
    kv_append(r["qkv"][:, qd:qd + kd].reshape(T, Hkv, D), r["qkv"][:, qd + kd:].reshape(T, Hkv, D),
              k_pool, v_pool, page_table, ctx_len, k_scale, v_scale)
    a = tree_attn(r["qkv"][:, :qd].reshape(T, Hq, D), k_pool, v_pool, page_table, ctx_len, parent,
                  k_scale, v_scale)
    r["attn"] = bf16(a.reshape(T, qd))
    r["h1"] = bf16(h + lin(r["attn"], "o", 1))
    r["y2"] = bf16(rmsnorm(r["h1"], norm_w2, eps))
    r["gu"] = bf16(lin(r["y2"], "gate_up", 2))
    r["s"] = bf16(swiglu(r["gu"]))
    r["h2"] = bf16(r["h1"] + lin(r["s"], "down", 3))
    return r
