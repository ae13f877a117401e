"""Pins for the oracle's greedy tree acceptance and accepted-KV compaction.

(1) a chain accepts exactly the matching prefix; (2) the result equals an
explicit enumeration of every root-to-node path (brute force, different
algorithm) on random trees; (3) hand-worked examples, incl. ties between
equally deep nodes; (4) compaction moves exactly the accepted tokens' bytes to
consecutive positions and leaves every other byte alone.
"""
import numpy as np

from nvfp4_skinny_gemm_b200 import inputs


def _brute(tok, amax, parent):
    T = len(parent)
    best, best_end = None, None
    for end in range(T):
        path = []
        i = end
        while i >= 0:
            path.append(i)
            i = int(parent[i])
        path.reverse()
        if path[0] != 0:
            continue
        ok = all(tok[path[k]] == amax[path[k - 1]] for k in range(1, len(path)))
        if ok and (best is None or len(path) > len(best)):
            best, best_end = path, end
    return best, int(amax[best_end])


def test_chain_accepts_matching_prefix(oracle):
    T = 8
    parent = inputs.chain_parent(T)
    amax = np.array([11, 12, 13, 14, 15, 16, 17, 18], np.int32)
    tok = np.array([99, 11, 12, 13, 0, 15, 16, 17], np.int32)     # node 4 mismatches
    path, nxt = oracle.tree_accept_greedy(tok, amax, parent)
    assert path == [0, 1, 2, 3] and nxt == 14
    tok_all = np.concatenate([[5], amax[:-1]]).astype(np.int32)
    path, nxt = oracle.tree_accept_greedy(tok_all, amax, parent)
    assert path == list(range(T)) and nxt == 18
    path, nxt = oracle.tree_accept_greedy(np.full(T, -1, np.int32), amax, parent)
    assert path == [0] and nxt == 11


def test_hand_worked_tree_and_ties(oracle):
    #        0
    #      /   \
    #     1     2          amax[0] = 7: node 1 (tok 7) and node 2 (tok 7) both match
    #    / \     \         amax[1] = 3: node 3 (tok 3) matches, node 4 (tok 9) does not
    #   3   4     5        amax[2] = 4: node 5 (tok 4) matches
    parent = np.array([-1, 0, 0, 1, 1, 2], np.int32)
    tok = np.array([0, 7, 7, 3, 9, 4], np.int32)
    amax = np.array([7, 3, 4, 8, 1, 6], np.int32)
    path, nxt = oracle.tree_accept_greedy(tok, amax, parent)
    assert path == [0, 1, 3] and nxt == 8                  # depth-2 tie: node 3 < node 5
    tok[3] = 2
    path, nxt = oracle.tree_accept_greedy(tok, amax, parent)
    assert path == [0, 2, 5] and nxt == 6


def test_matches_brute_force_on_random_trees(oracle):
    rng = np.random.default_rng(31)
    for trial in range(300):
        T = int(rng.integers(1, 17))
        parent = inputs.tree_parent(50, 16, sub=trial)[:T]
        amax = rng.integers(0, 4, T).astype(np.int32)
        tok = rng.integers(0, 4, T).astype(np.int32)
        assert oracle.tree_accept_greedy(tok, amax, parent) == _brute(tok, amax, parent), trial


def test_compaction_moves_exactly_the_accepted_tokens(oracle):
    T, Hkv, D, P, L = 16, 2, 16, 16, 40
    cache = inputs.kv_cache(60, L, T=T, Hkv=Hkv, D=D, P=P, extra_pages=3)
    kp, vp = cache.k_pool.copy(), cache.v_pool.copy()
    off = inputs.v_plane_offsets(D, P)
    path = [0, 2, 5, 11]

    def tok(k_pool, v_pool, pos):
        pg, sl = cache.page_table[pos // P], pos % P
        return k_pool[pg, :, sl, :].copy(), v_pool[pg][:, off[:, sl]].copy()

    want = [tok(kp, vp, L + n) for n in path]
    oracle.kv_compact_accepted(kp, vp, cache.page_table, L, path)
    for k in range(len(path)):
        gk, gv = tok(kp, vp, L + k)
        assert np.array_equal(gk, want[k][0]) and np.array_equal(gv, want[k][1])
    # every byte outside positions L .. L+3 is unchanged
    mk = np.ones(kp.shape, bool)
    mv = np.ones(vp.shape, bool)
    for k in range(len(path)):
        pg, sl = cache.page_table[(L + k) // P], (L + k) % P
        mk[pg, :, sl, :] = False
        mv[pg][:, off[:, sl]] = False
    assert np.array_equal(kp[mk], cache.k_pool[mk]) and np.array_equal(vp[mv], cache.v_pool[mv])
