"""Pins for the oracle's tree-masked attention over the FP8 paged cache.

(1) a chain-shaped tree equals causal attention (torch SDPA, fp64, explicit
    causal mask) over context + tree tokens;
(2) a tree equals running each root-to-node path as its own chain;
(3) one node with no context returns its own V;
(4) identical keys give the mean of the visible V;
(5) pure-Python brute force at L=3, D=8, T=4;
(6) a random permutation of the physical pool (with the page table) changes
    nothing; bytes outside the visible positions change nothing;
(7) the tiled V plane layout: hand-computed byte offsets, a bijection;
(8) causal attention over a suffix of S tokens, split into row groups of at
    most 16 that each attend to the context before them plus their own chain
    (the suffix prefill's decomposition), gives the same rows as the chain of
    all S tokens at once, bit for bit.
"""
import math

import numpy as np
import torch

from nvfp4_skinny_gemm_b200 import inputs


def _dense(cache, Hkv, D, P):
    """Dequantised dense K, V [L+T, Hkv, D] (torch float8 view x scale)."""
    total = cache.ctx_len + cache.T
    kp = torch.from_numpy(cache.k_pool.copy()).view(torch.float8_e4m3fn).double().numpy()
    vp = torch.from_numpy(cache.v_pool.copy()).view(torch.float8_e4m3fn).double().numpy()
    off = inputs.v_plane_offsets(D, P)
    K = np.zeros((total, Hkv, D))
    V = np.zeros((total, Hkv, D))
    for p in range(total):
        pg = cache.page_table[p // P]
        K[p] = kp[pg, :, p % P, :] * cache.k_scale[:, None]
        V[p] = vp[pg][:, off[:, p % P]] * cache.v_scale[:, None]
    return K, V


def _run(oracle, q, cache, parent):
    return oracle.tree_attn(q, cache.k_pool, cache.v_pool, cache.page_table, cache.ctx_len, parent,
                            cache.k_scale, cache.v_scale)


def test_chain_equals_causal_sdpa(oracle):
    T, Hq, Hkv, D, P, L = 5, 6, 2, 16, 16, 21
    cache = inputs.kv_cache(100, L, T=T, Hkv=Hkv, D=D, P=P, extra_pages=3)
    q = inputs.query_bf16(100, T, Hq, D).float().numpy()
    out = _run(oracle, q, cache, inputs.chain_parent(T))
    K, V = _dense(cache, Hkv, D, P)
    grp = Hq // Hkv
    qt = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)                 # [Hq, T, D]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(grp, 0)          # [Hq, L+T, D]
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(grp, 0)
    mask = torch.tensor([[p <= L + i for p in range(L + T)] for i in range(T)])
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    assert np.allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_tree_equals_per_path_chains(oracle):
    T, Hq, Hkv, D, P, L = 16, 4, 2, 8, 16, 37
    cache = inputs.kv_cache(101, L, T=T, Hkv=Hkv, D=D, P=P)
    parent = inputs.tree_parent(101, T)
    q = inputs.query_bf16(101, T, Hq, D).float().numpy()
    out = _run(oracle, q, cache, parent)
    total = L + T
    for i in range(T):
        path = sorted(oracle.ancestors(parent, i))                  # root .. i
        d = len(path)
        # a fresh cache: same context pages, the path's tree slots in order
        n_log = (L + d + P - 1) // P
        kp = np.zeros((n_log, Hkv, P, D), np.uint8)
        vp = np.zeros((n_log, Hkv, D * P), np.uint8)
        off = inputs.v_plane_offsets(D, P)
        for p in range(L + d):
            src = p if p < L else L + path[p - L]
            spg, sslot = cache.page_table[src // P], src % P
            kp[p // P, :, p % P, :] = cache.k_pool[spg, :, sslot, :]
            vp[p // P][:, off[:, p % P]] = cache.v_pool[spg][:, off[:, sslot]]
        sub = oracle.tree_attn(q[path], kp, vp, np.arange(n_log, dtype=np.int32), L,
                               inputs.chain_parent(d), cache.k_scale, cache.v_scale)
        assert np.allclose(sub[-1], out[i], rtol=1e-12, atol=1e-14), i
    assert total == L + T


def test_single_node_no_context_returns_v0(oracle):
    Hq, Hkv, D, P = 2, 1, 8, 16
    cache = inputs.kv_cache(102, 0, T=1, Hkv=Hkv, D=D, P=P)
    cache.k_scale[:] = 0.5
    cache.v_scale[:] = 0.25
    q = inputs.query_bf16(102, 1, Hq, D).float().numpy()
    out = _run(oracle, q, cache, np.array([-1], np.int32))
    _, V = _dense(cache, Hkv, D, P)
    for h in range(Hq):
        assert np.array_equal(out[0, h], V[0, 0])


def test_identical_keys_give_mean_of_visible_v(oracle):
    T, Hq, Hkv, D, P, L = 6, 2, 1, 8, 16, 13
    cache = inputs.kv_cache(103, L, T=T, Hkv=Hkv, D=D, P=P)
    for p in range(L + T):
        cache.k_pool[cache.page_table[p // P], 0, p % P, :] = 0x30   # same key everywhere
    parent = np.array([-1, 0, 0, 1, 2, 3], np.int32)
    q = inputs.query_bf16(103, T, Hq, D).float().numpy()
    out = _run(oracle, q, cache, parent)
    _, V = _dense(cache, Hkv, D, P)
    for i in range(T):
        vis = list(range(L)) + [L + j for j in oracle.ancestors(parent, i)]
        want = V[vis, 0].mean(axis=0)
        for h in range(Hq):
            assert np.allclose(out[i, h], want, rtol=1e-12, atol=1e-14)


def test_bruteforce_tiny(oracle):
    T, Hq, Hkv, D, P, L = 4, 2, 1, 8, 16, 3
    cache = inputs.kv_cache(104, L, T=T, Hkv=Hkv, D=D, P=P, extra_pages=2)
    parent = np.array([-1, 0, 0, 2], np.int32)
    q = inputs.query_bf16(104, T, Hq, D).float().numpy()
    out = _run(oracle, q, cache, parent)
    K, V = _dense(cache, Hkv, D, P)
    anc = {0: [0], 1: [0, 1], 2: [0, 2], 3: [0, 2, 3]}
    for i in range(T):
        for h in range(Hq):
            pos = [0, 1, 2] + [L + j for j in anc[i]]
            s = [sum(float(q[i, h, d]) * K[p, 0, d] for d in range(D)) / math.sqrt(D) for p in pos]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            o = [sum(w[j] * V[p, 0, d] for j, p in enumerate(pos)) / sum(w) for d in range(D)]
            assert np.allclose(out[i, h], o, rtol=1e-12, atol=1e-14)


def test_page_permutation_and_unseen_bytes_do_not_matter(oracle):
    T, Hq, Hkv, D, P, L = 16, 6, 2, 16, 16, 45
    cache = inputs.kv_cache(105, L, T=T, Hkv=Hkv, D=D, P=P, extra_pages=5)
    parent = inputs.tree_parent(105, T)
    q = inputs.query_bf16(105, T, Hq, D).float().numpy()
    out = _run(oracle, q, cache, parent)
    rng = np.random.default_rng(9)
    perm = rng.permutation(cache.k_pool.shape[0])        # new physical id of old page j = perm[j]
    kp = np.empty_like(cache.k_pool); vp = np.empty_like(cache.v_pool)
    kp[perm] = cache.k_pool; vp[perm] = cache.v_pool
    out2 = oracle.tree_attn(q, kp, vp, perm[cache.page_table].astype(np.int32), L, parent,
                            cache.k_scale, cache.v_scale)
    assert np.array_equal(out, out2)
    # scribble over every byte that no node may see
    used = {(cache.page_table[p // P], p % P) for p in range(L + T)}
    kp3, vp3 = cache.k_pool.copy(), cache.v_pool.copy()
    off = inputs.v_plane_offsets(D, P)
    for pg in range(kp3.shape[0]):
        for slot in range(P):
            if (pg, slot) not in used:
                kp3[pg, :, slot, :] = 0x7E
                vp3[pg][:, off[:, slot]] = 0x7E
    out3 = oracle.tree_attn(q, kp3, vp3, cache.page_table, L, parent, cache.k_scale, cache.v_scale)
    assert np.array_equal(out, out3)


def test_v_plane_layout():
    off = inputs.v_plane_offsets(16, 32)
    # tile (d//8, t//16) at index (d//8)*2 + t//16, 128 bytes; row d%8 of 16 bytes
    assert off[0, 0] == 0 and off[0, 15] == 15 and off[1, 0] == 16 and off[7, 15] == 127
    assert off[0, 16] == 128 and off[8, 0] == 256 and off[9, 17] == 401 and off[15, 31] == 511
    for D, P in [(8, 16), (16, 32), (128, 64)]:
        o = inputs.v_plane_offsets(D, P)
        assert sorted(o.ravel().tolist()) == list(range(D * P))


def test_suffix_groups_equal_whole_causal(oracle):
    """Row group (r, t) of a causal suffix sees positions < start + r + i for
    its row i, which is a chain of t tokens after a context of start + r: the
    oracle visits the same positions in the same order, so the results match
    exactly.  Groups of 16 (S = 37: two full groups and a ragged one) and the
    prefill's blocks of 128 queries (S = 150: one full block and a ragged one)."""
    from nvfp4_skinny_gemm_b200.step import PREFILL_CHUNK, prefill_chunks
    Hq, Hkv, D, P, start = 4, 2, 16, 16, 29
    for S, C, sizes in [(37, 16, [16, 16, 5]), (150, PREFILL_CHUNK, [128, 22])]:
        cache = inputs.kv_cache(104, start, T=S, Hkv=Hkv, D=D, P=P, extra_pages=2)
        q = inputs.query_bf16(104, S, Hq, D).float().numpy()
        whole = _run(oracle, q, cache, inputs.chain_parent(S))
        groups = prefill_chunks(start, S, C)
        assert [t for _, t, _ in groups] == sizes
        for r, t, ctx in groups:
            part = oracle.tree_attn(q[r:r + t], cache.k_pool, cache.v_pool, cache.page_table, ctx,
                                    inputs.chain_parent(t), cache.k_scale, cache.v_scale)
            assert np.array_equal(part, whole[r:r + t]), (S, r, t)
    S = 37
    cache = inputs.kv_cache(104, start, T=S, Hkv=Hkv, D=D, P=P, extra_pages=2)
    q = inputs.query_bf16(104, S, Hq, D).float().numpy()
    whole = _run(oracle, q, cache, inputs.chain_parent(S))
    # the check has teeth: rows that skip the earlier rows of their own group differ
    wrong = oracle.tree_attn(q[16:32], cache.k_pool, cache.v_pool, cache.page_table, start + 16,
                             np.full(16, -1, np.int32), cache.k_scale, cache.v_scale)
    assert not np.allclose(wrong, whole[16:32])
