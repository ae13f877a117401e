"""GPU greedy tree acceptance and accepted-KV compaction against the oracle:
path, length and next token identical on random trees (ties included) and on
chains; compaction byte-identical in every layer of a multi-layer pool; a
malformed parent array is flagged and only the root is accepted."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda, to_dev
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def _run(tok, amax, parent):
    path, n, nxt = nv.tree_accept(to_dev(tok), to_dev(amax), to_dev(parent))
    n = int(n.cpu()[0])
    return path.cpu().numpy()[:n].tolist(), int(nxt.cpu()[0])


def test_accept_matches_oracle_random_trees(oracle):
    cuda()
    rng = np.random.default_rng(61)
    for trial in range(200):
        T = int(rng.integers(1, 17))
        parent = inputs.tree_parent(51, 16, sub=trial)[:T]
        amax = rng.integers(0, 3, T).astype(np.int32)
        tok = rng.integers(0, 3, T).astype(np.int32)
        assert _run(tok, amax, parent) == oracle.tree_accept_greedy(tok, amax, parent), trial
    assert nv.device_status()[0] == 0


def test_accept_chain_and_bad_parent(oracle):
    cuda()
    T = 16
    parent = inputs.chain_parent(T)
    amax = np.arange(100, 100 + T, dtype=np.int32)
    tok = np.concatenate([[7], amax[:-1]]).astype(np.int32)
    tok[9] = 0
    assert _run(tok, amax, parent) == oracle.tree_accept_greedy(tok, amax, parent) == (list(range(9)), 108)
    bad = parent.copy()
    bad[5] = 7                                  # not topologically ordered
    nv.device_status()
    assert _run(tok, amax, bad) == ([0], 100)
    rc, site = nv.device_status()
    assert (rc, site) == (-7, 501)


def test_compaction_all_layers_matches_oracle(oracle):
    cuda()
    n_layers, T, Hkv, D, P, L = 3, 16, 4, 128, 64, 1000
    caches = [inputs.kv_cache(62, L, T=T, sub=l, extra_pages=2) for l in range(n_layers)]
    pt = caches[0].page_table                          # same page table for every layer
    for c in caches[1:]:
        c.page_table = pt
    kp = np.stack([c.k_pool for c in caches])          # [layer, pages, Hkv, P, D]
    vp = np.stack([c.v_pool for c in caches])
    parent = inputs.tree_parent(62)
    rng = np.random.default_rng(63)
    amax = rng.integers(0, 2, T).astype(np.int32)
    tok = rng.integers(0, 2, T).astype(np.int32)
    path, nxt = oracle.tree_accept_greedy(tok, amax, parent)
    kd, vd = to_dev(kp), to_dev(vp)
    dpath, dn, dnext = nv.tree_accept(to_dev(tok), to_dev(amax), to_dev(parent))
    stride = kp[0].nbytes
    nv.kv_compact(kd.data_ptr(), vd.data_ptr(), stride, n_layers, Hkv, D, kp.shape[1], P, to_dev(pt), L, dpath, dn, T)
    for l in range(n_layers):
        wk, wv = kp[l].copy(), vp[l].copy()
        oracle.kv_compact_accepted(wk, wv, pt, L, path)
        assert np.array_equal(kd[l].cpu().numpy(), wk), l
        assert np.array_equal(vd[l].cpu().numpy(), wv), l
    assert int(dn.cpu()[0]) == len(path) and int(dnext.cpu()[0]) == nxt
    assert nv.device_status()[0] == 0
