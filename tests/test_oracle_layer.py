"""Pins for the oracle's composed decoder layer (oracle.decoder_layer), on
tiny shapes (hidden 64, 4 query heads and 2 KV heads of 16 dims, FFN 64,
pages of 16 tokens):

(1) its bf16 rounding equals torch's bf16 cast, ties included;
(2) with the O and down weights zero the layer is the identity on h (both
    residual branches add exactly 0);
(3) with static scales a chain is causal: changing row k leaves every output
    row before k bit-identical and changes row k;
(4) in a tree, changing node k changes exactly k and its descendants;
(5) with static scales, rows 0..15 and then rows 16..S-1 (attending to the
    first group's appended K/V as context) give the bits of one pass over all
    S rows, pools included: the suffix prefill's decomposition;
(6) with dynamic scales rows are coupled through the tensor amax, which is
    why the decomposition of (5) needs static scales;
(7) one token with no context attends only to itself: each query head's
    attention output is the FP8 round trip (torch's float8_e4m3fn cast) of
    the V part of its own QKV row, for the KV head of its group.
"""
import numpy as np
import torch

from nvfp4_skinny_gemm_b200 import inputs as I

H, HQ, HKV, D, F, P = 64, 4, 2, 16, 64, 16
SHAPES = {"qkv": (H, (HQ + 2 * HKV) * D), "o": (HQ * D, H), "gate_up": (H, 2 * F), "down": (F, H)}


def _weights(oracle, zero=()):
    w = {}
    for t, (name, (K, N)) in enumerate(SHAPES.items()):
        x = I.weight_fp32(21, t, N, K) * 5.0                   # std 0.1: O(1) outputs at K = 64
        if name in zero:
            x[:] = 0.0
        w[name] = oracle.quantize(x)
    return w


def _setup(ctx, T, seed=0):
    cache = I.kv_cache(22, ctx, T=T, Hkv=HKV, D=D, P=P, extra_pages=2, fill_tree=False, sub=seed)
    h = I.bf16_normal(23, 0, (T, H), seed).double().numpy()
    return cache, h


def _run(oracle, w, G, cache, h, parent, ctx=None):
    kp, vp = cache.k_pool.copy(), cache.v_pool.copy()
    r = oracle.decoder_layer(h, np.ones(H, np.float32), np.ones(H, np.float32), w, G, kp, vp,
                             cache.page_table, cache.ctx_len if ctx is None else ctx, parent,
                             cache.k_scale, cache.v_scale, HQ)
    return r, kp, vp


G_STATIC = [0.3 / 2688, 2.0 / 2688, 3.0 / 2688, 2.0 / 2688]


def test_bf16_rounding_matches_torch(oracle):
    g = np.random.default_rng(5)
    x = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-20, 20, 20000),
                        # exact ties between two bf16 neighbours, both parities of the kept bit
                        (1.0 + (np.arange(256) * 2 + 1) * 2.0 ** -8) * 2.0 ** g.integers(-30, 30, 256)])
    want = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.bf16(x), want)


def test_zero_o_and_down_is_the_identity(oracle):
    w = _weights(oracle, zero=("o", "down"))
    cache, h = _setup(37, 8)
    r, _, _ = _run(oracle, w, G_STATIC, cache, h, I.tree_parent(7, 8))
    assert np.array_equal(r["h2"], h) and np.array_equal(r["h1"], h)
    assert np.abs(r["attn"]).max() > 0.1                       # the attention branch did run


def test_chain_is_causal_with_static_scales(oracle):
    w = _weights(oracle)
    cache, h = _setup(29, 12)
    chain = I.chain_parent(12)
    base, _, _ = _run(oracle, w, G_STATIC, cache, h, chain)
    for k in (0, 5, 11):
        h2 = h.copy()
        h2[k] = -h2[k] + 0.25
        r, _, _ = _run(oracle, w, G_STATIC, cache, h2, chain)
        assert np.array_equal(r["h2"][:k], base["h2"][:k]), k
        assert not np.array_equal(r["h2"][k], base["h2"][k]), k


def test_tree_changes_only_descendants(oracle):
    w = _weights(oracle)
    T = 16
    cache, h = _setup(41, T)
    parent = I.tree_parent(8, T)
    base, _, _ = _run(oracle, w, G_STATIC, cache, h, parent)
    for k in (1, 4, 9):
        h2 = h.copy()
        h2[k] = -h2[k] + 0.25
        r, _, _ = _run(oracle, w, G_STATIC, cache, h2, parent)
        desc = {i for i in range(T) if k in oracle.ancestors(parent, i)}
        changed = {i for i in range(T) if not np.array_equal(r["h2"][i], base["h2"][i])}
        assert changed == desc, (k, changed, desc)


def test_row_groups_equal_one_pass_with_static_scales(oracle):
    w = _weights(oracle)
    S, ctx = 20, 33
    cache, h = _setup(ctx, S)
    whole, kp_w, vp_w = _run(oracle, w, G_STATIC, cache, h, I.chain_parent(S))
    kp, vp = cache.k_pool.copy(), cache.v_pool.copy()
    parts = []
    for r0, t in ((0, 16), (16, 4)):
        parts.append(oracle.decoder_layer(h[r0:r0 + t], np.ones(H, np.float32), np.ones(H, np.float32), w,
                                          G_STATIC, kp, vp, cache.page_table, ctx + r0, I.chain_parent(t),
                                          cache.k_scale, cache.v_scale, HQ))
    assert np.array_equal(np.concatenate([p["h2"] for p in parts]), whole["h2"])
    assert np.array_equal(kp, kp_w) and np.array_equal(vp, vp_w)


def test_dynamic_scales_couple_rows(oracle):
    w = _weights(oracle)
    cache, h = _setup(29, 12)
    chain = I.chain_parent(12)
    base, _, _ = _run(oracle, w, None, cache, h, chain)
    h2 = h.copy()
    h2[11] = 0.0
    h2[11, 0] = 100.0              # RMSNorm maps row 11 to one value of 8: the amax of y1 grows
    r, _, _ = _run(oracle, w, None, cache, h2, chain)
    assert np.array_equal(r["y1"][0], base["y1"][0])           # RMSNorm itself is row-local
    assert not np.array_equal(r["qkv"][0], base["qkv"][0])     # the shared tensor scale is not
    # the same change with static scales leaves row 0 alone (pin 3)
    s0, _, _ = _run(oracle, w, G_STATIC, cache, h, chain)
    s1, _, _ = _run(oracle, w, G_STATIC, cache, h2, chain)
    assert np.array_equal(s1["h2"][:11], s0["h2"][:11])


def test_lone_token_attends_to_its_own_v(oracle):
    w = _weights(oracle)
    cache, h = _setup(0, 1)
    r, _, _ = _run(oracle, w, G_STATIC, cache, h, np.array([-1], np.int32))
    qd, kd = HQ * D, HKV * D
    v = r["qkv"][0, qd + kd:].reshape(HKV, D)
    vs = cache.v_scale.astype(np.float32)
    y = np.clip((v.astype(np.float32) / vs[:, None]).astype(np.float32), -448, 448)
    fp8 = torch.from_numpy(y).to(torch.float8_e4m3fn).double().numpy() * vs[:, None].astype(np.float64)
    group = HQ // HKV
    want = np.stack([fp8[hq // group] for hq in range(HQ)]).reshape(1, qd)
    want = torch.from_numpy(want).to(torch.float32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(r["attn"], want)
