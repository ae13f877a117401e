"""Seeded synthetic inputs for the verify-step workloads.

This module is the ONE piece shared by the CUDA path's tests/bench and the CPU
oracle.  It draws random tensors with the shapes and value distributions of
the workloads and holds none of the method's arithmetic (no NVFP4 recipe, no
attention, no restore).  The FP8 KV cache it builds is an input state of the
attention call: per (KV head, K|V) it divides by a scale and casts with
torch's own float8_e4m3fn conversion.

Seeds: numpy ``default_rng([42, workload_id, tensor_id, ...])``; 42 is the
seed the benchmark pages use for their runs ("How to reproduce": temperature
0, seed 42).

Workload shapes (27B-class dense layer, tree verification):
hidden 5120, 24 query heads, 4 KV heads, head_dim 128, FFN 17408, vocab
151936, page size 64, 16 tree nodes, context up to 23,552 tokens
("What MLPerf Edge Agentic measures": input grows to ~23.5K tokens; "Tree
multi-token prediction": 8 draft steps, top-2 per depth, 16-node tree).
"""
from __future__ import annotations

import math

import numpy as np
import torch

HIDDEN = 5120
N_Q_HEADS = 24
N_KV_HEADS = 4
HEAD_DIM = 128
FFN = 17408
VOCAB = 151936
PAGE = 64
TREE_NODES = 16
CTX_MAX = 23552
N_LAYERS = 64

# (K, N) of the four linears of one layer: QKV, O, gate+up, down.
LAYER_LINEARS = {
    "qkv": (HIDDEN, (N_Q_HEADS + 2 * N_KV_HEADS) * HEAD_DIM),   # 5120 -> 4096
    "o": (N_Q_HEADS * HEAD_DIM, HIDDEN),                        # 3072 -> 5120
    "gate_up": (HIDDEN, 2 * FFN),                               # 5120 -> 34816
    "down": (FFN, HIDDEN),                                      # 17408 -> 5120
}

W_STD = 0.02


def rng(*ids) -> np.random.Generator:
    return np.random.default_rng([42, *[int(i) for i in ids]])


def weight_fp32(workload: int, tensor: int, N: int, K: int, sub: int = 0) -> np.ndarray:
    """W [N, K] ~ N(0, 0.02^2), float32."""
    g = rng(workload, tensor, sub)
    w = g.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(W_STD)
    return w


def activation_bf16(workload: int, tensor: int, M: int, K: int, outlier_frac: float = 0.0,
                    outlier_gain: float = 20.0, sub: int = 0) -> torch.Tensor:
    """A [M, K] ~ N(0,1) rounded to bf16; round(outlier_frac*K) channels chosen
    by the seed without replacement are multiplied by outlier_gain in every row
    before rounding (the 1%-outlier-channel activation of the layer workload)."""
    g = rng(workload, tensor, sub)
    a = g.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(outlier_frac * K))
    if n_out:
        ch = g.choice(K, size=n_out, replace=False)
        a[:, ch] *= np.float32(outlier_gain)
    return torch.from_numpy(a).to(torch.bfloat16)


def bf16_normal(workload: int, tensor: int, shape, sub: int = 0) -> torch.Tensor:
    g = rng(workload, tensor, sub)
    return torch.from_numpy(g.standard_normal(shape, dtype=np.float32)).to(torch.bfloat16)


def tree_parent(workload: int, T: int = TREE_NODES, sub: int = 0) -> np.ndarray:
    """Parent array of the verification tree (-1 for the root).

    Reading of "8 draft steps, top-2 candidates per depth, 16 nodes": node 0 is
    the root (depth 0); node i >= 1 sits at depth ceil(i/2), so depths 1..7
    hold two nodes and depth 8 holds node 15; the parent of node i is drawn
    uniformly from the nodes at depth(i) - 1.  Nodes are in topological order.
    """
    g = rng(workload, 900, sub)
    depth = [0] + [math.ceil(i / 2) for i in range(1, T)]
    parent = np.full(T, -1, np.int32)
    for i in range(1, T):
        cands = [j for j in range(i) if depth[j] == depth[i] - 1]
        parent[i] = cands[int(g.integers(len(cands)))]
    return parent


def chain_parent(T: int) -> np.ndarray:
    return np.arange(-1, T - 1, dtype=np.int32)


def fp8_codes(x: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 bytes of x / scale via torch's float8_e4m3fn cast (RNE), clamped
    to +-448 first so that out-of-range values saturate."""
    y = (x.astype(np.float32) / np.float32(scale)).astype(np.float32)
    y = np.clip(y, -448.0, 448.0)
    return torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def v_plane_offsets(D: int = HEAD_DIM, P: int = PAGE) -> np.ndarray:
    """[D, P] byte offsets of (dimension d, slot t) inside one (page, head)
    plane of the V pool: the plane is cut into tiles of 8 dimensions x 16 slots
    (128 bytes), tile (d // 8, t // 16) stored at tile index
    (d // 8) * (P // 16) + t // 16, row d % 8 of 16 slot bytes inside."""
    assert D % 8 == 0 and P % 16 == 0
    d = np.arange(D)[:, None]
    t = np.arange(P)[None, :]
    return ((d // 8) * (P // 16) + t // 16) * 128 + (d % 8) * 16 + t % 16


class KVCache:
    """A synthetic FP8 paged cache for one layer.

    k_pool u8 [n_pages, Hkv, P, D] (token-major pages), v_pool u8
    [n_pages, Hkv, D * P] (tiled planes, see v_plane_offsets), page_table i32
    over the logical pages covering ctx_len + T positions, k_scale/v_scale
    f32 [Hkv].
    """

    def __init__(self, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale, T):
        self.k_pool, self.v_pool, self.page_table = k_pool, v_pool, page_table
        self.ctx_len, self.k_scale, self.v_scale, self.T = ctx_len, k_scale, v_scale, T


def kv_cache(workload: int, ctx_len: int, T: int = TREE_NODES, Hkv: int = N_KV_HEADS,
             D: int = HEAD_DIM, P: int = PAGE, extra_pages: int = 0, fill_tree: bool = True,
             sub: int = 0, unused_nan: bool = False) -> KVCache:
    """K/V ~ N(0,1) for positions 0..ctx_len+T-1, per-(head, K|V) scale =
    amax over the context / 448, stored as FP8 in a randomly permuted pool.
    If fill_tree, the tree slots ctx_len..ctx_len+T-1 are filled too (with the
    same scales, saturating); otherwise they are left as zero bytes.  Pool
    bytes that hold no position are random finite codes, or the E4M3 NaN code
    0x7F if unused_nan (a pool that was never cleared)."""
    g = rng(workload, 800, sub)
    total = ctx_len + T
    n_log = (total + P - 1) // P
    n_pages = n_log + extra_pages
    k = g.standard_normal((total, Hkv, D), dtype=np.float32)
    v = g.standard_normal((total, Hkv, D), dtype=np.float32)
    ctx = max(ctx_len, 1)
    k_scale = np.array([np.abs(k[:ctx, h]).max() / 448.0 for h in range(Hkv)], np.float32)
    v_scale = np.array([np.abs(v[:ctx, h]).max() / 448.0 for h in range(Hkv)], np.float32)
    page_table = g.permutation(n_pages)[:n_log].astype(np.int32)
    # unused pool bytes get random codes (never NaN) so that stray reads show
    k_pool = g.integers(0, 0x7E, (n_pages, Hkv, P, D), dtype=np.uint8)
    v_pool = g.integers(0, 0x7E, (n_pages, Hkv, D * P), dtype=np.uint8)
    if unused_nan:
        k_pool[:] = 0x7F
        v_pool[:] = 0x7F
    off = v_plane_offsets(D, P)
    upto = total if fill_tree else ctx_len
    for h in range(Hkv):
        kc = fp8_codes(k[:upto, h], k_scale[h])          # [pos, D]
        vc = fp8_codes(v[:upto, h], v_scale[h])
        for p in range(0, upto, P):
            n = min(P, upto - p)
            pg = page_table[p // P]
            k_pool[pg, h, :n, :] = kc[p:p + n]
            v_pool[pg, h, off[:, :n].ravel()] = vc[p:p + n].T.ravel()
    if not fill_tree:
        for i in range(T):
            p = ctx_len + i
            k_pool[page_table[p // P], :, p % P, :] = 0
            v_pool[page_table[p // P], :, off[:, p % P]] = 0
    return KVCache(k_pool, v_pool, page_table, ctx_len, k_scale, v_scale, T)


def query_bf16(workload: int, T: int = TREE_NODES, Hq: int = N_Q_HEADS, D: int = HEAD_DIM,
               sub: int = 0):
    return bf16_normal(workload, 700, (T, Hq, D), sub)
