"""Host logic of the suffix prefill (VerifyModel.prefill), on the CPU.

The library calls are replaced by a recording fake that moves symbolic labels
instead of numbers: every buffer row (and every cache position of every
layer) holds a label that spells out how its value was produced, e.g.
("norm", w, site, x) = RMSNorm with weight row w of the row labelled x,
quantised with site scale `site`.  Each fake op builds its output labels from
the labels of what it reads, and the test compares the final labels with the
ones the layer definition gives row by row, without groups.  So it fails if a
group reads a buffer that another group has overwritten, attends before the
K/V it needs is written or to K/V it must not see, reads another layer's pool
or weights, or quantises with another site's scale.
No kernel and no oracle runs here; the numbers are checked by the GPU tests.
"""
import numpy as np
import pytest
import torch

from nvfp4_skinny_gemm_b200 import inputs as I
from nvfp4_skinny_gemm_b200 import step


def _row0(x):
    """(storage id, first row) of a row-major view."""
    base = x.untyped_storage().data_ptr()
    return base, (x.data_ptr() - base) // (x.stride(0) * x.element_size())


class FakeLib:
    def __init__(self):
        self.labels = {}          # (storage, row) -> label
        self.kv = {}              # (layer, position) -> label
        self.gl = {}              # g tensor data_ptr -> site label
        self.launches = 0
        self.m = None
        self.wmap = {}

    # ---- helpers
    def rows(self, x, n=None):
        s, r0 = _row0(x)
        n = x.shape[0] if n is None else n
        return [(s, r0 + i) for i in range(n)]

    def get(self, x, n=None):
        return [self.labels.get(k) for k in self.rows(x, n)]

    def put(self, x, labels):
        for k, v in zip(self.rows(x, len(labels)), labels):
            self.labels[k] = v

    def site_of(self, g):
        off = g.data_ptr() - self.m.G.data_ptr()
        assert 0 <= off < self.m.G.numel() * 4 and off % 4 == 0
        return off // 4

    def layer_of_pool(self, k_pool):
        for l in range(self.m.n_layers):
            if k_pool.data_ptr() == self.m.k_pool(l).data_ptr():
                return l
        raise AssertionError("not a layer's K pool")

    # ---- library surface
    def act_buffer(self, K, device=None):
        return torch.zeros(16, dtype=torch.uint8)

    def rmsnorm_quantize(self, x, w, eps, out, act=None, stream=None, g_in=None):
        self.launches += 1
        assert g_in is not None and x.shape[0] <= 16
        src = self.get(x)
        widx = (w.data_ptr() - self.m.norm_w.data_ptr()) // (I.HIDDEN * 2)
        site = self.site_of(g_in)
        self.gl[out[2].data_ptr()] = site
        self.put(act, [("norm", widx, site, v) for v in src])

    def swiglu_quantize(self, gu, out, act=None, stream=None, g_in=None):
        self.launches += 1
        assert g_in is not None and gu.shape[0] <= 16
        site = self.site_of(g_in)
        self.gl[out[2].data_ptr()] = site
        self.put(act, [("swiglu", site, v) for v in self.get(gu)])

    def linear(self, a_act, g_a, M, w_prep, g_w, N, K, y=None, residual=None, ws=None, stream=None):
        self.launches += 1
        assert 1 <= M <= 16 and y.shape[0] == M
        l, name = self.wmap[id(w_prep)]
        a = self.get(a_act, M)
        res = None
        if residual is not None:
            assert residual.data_ptr() == y.data_ptr()
            res = self.get(residual)
        self.put(y, [("linear", l, name, self.gl[g_a.data_ptr()], v, None if res is None else res[i])
                     for i, v in enumerate(a)])

    def kv_append(self, k_new, v_new, ld_new, T, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale,
                  stream=None):
        self.launches += 1
        l = self.layer_of_pool(k_pool)
        assert v_pool.data_ptr() == self.m.v_pool(l).data_ptr()
        assert k_scale.data_ptr() == self.m.k_scale[l].data_ptr()
        qd, kd = I.N_Q_HEADS * I.HEAD_DIM, I.N_KV_HEADS * I.HEAD_DIM
        assert _row0(k_new)[1] == _row0(v_new)[1]
        assert (k_new.data_ptr() - _row0(k_new)[0]) % (k_new.stride(0) * 2) == qd * 2
        assert (v_new.data_ptr() - _row0(v_new)[0]) % (v_new.stride(0) * 2) == (qd + kd) * 2
        src = self.get(k_new, T)
        pt = page_table.numpy()
        for i in range(T):
            assert 0 <= pt[(ctx_len + i) // I.PAGE] < self.m.n_pool
            self.kv[(l, ctx_len + i)] = ("kv", src[i])

    def tree_attn(self, q, k_pool, v_pool, page_table, ctx_len, parent, k_scale, v_scale, sm_scale=None,
                  out=None, ld_q=None, T=None, Hq=None, ws=None, stream=None, g_act=None, act=None):
        self.launches += 2
        l = self.layer_of_pool(k_pool)
        assert 1 <= T <= 16 and Hq == I.N_Q_HEADS and ld_q == q.stride(0)
        assert np.array_equal(parent.numpy()[:T], I.chain_parent(T))
        assert (ctx_len + T + I.PAGE - 1) // I.PAGE <= self.m.n_log
        qs = self.get(q, T)
        seen = [self.kv.get((l, p)) for p in range(self.start, ctx_len + T)]
        site = self.site_of(g_act)
        self.gl[g_act.data_ptr()] = site
        labels = [("attn", site, qs[i], tuple(seen[:ctx_len - self.start + i + 1])) for i in range(T)]
        self.put(out, labels)
        self.put(act, labels)

    def argmax(self, x, idx=None, ws=None, stream=None):
        self.launches += 1
        self.put(idx.view(-1, 1), [("argmax", v) for v in self.get(x)])


class _FakeWeight:
    def __init__(self, *shape):
        self.shape = shape[:2]

    def mul_(self, s):
        return self


def _model(monkeypatch, n_layers, ctx_len, lm_head=True):
    fake = FakeLib()
    monkeypatch.setattr(step, "nv", fake)
    monkeypatch.setattr(step.torch, "randn", lambda *a, **k: _FakeWeight(*a))
    monkeypatch.setattr(step.Linear, "from_fp32",
                        staticmethod(lambda w: step.Linear(object(), torch.ones(1), *w.shape)))
    m = step.VerifyModel(n_layers=n_layers, ctx_len=ctx_len, T=16, weights="device", device="cpu",
                         lm_head=lm_head)
    fake.m = m
    for l, lay in enumerate(m.layers):
        for name, lin in lay.items():
            fake.wmap[id(lin.prep)] = (l, name)
    if lm_head:
        fake.wmap[id(m.lm_head.prep)] = (None, "lm_head")
    m.static = True
    return m, fake


def _expected(n_layers, start, S):
    """Labels the layer definition gives, row by row (no groups anywhere)."""
    sites = step.VerifyModel.SITES
    h = [("in", r) for r in range(S)]
    kv = {}
    for l in range(n_layers):
        s0 = l * sites
        y1 = [("norm", 2 * l, s0, v) for v in h]
        qkv = [("linear", l, "qkv", s0, v, None) for v in y1]
        for r in range(S):
            kv[(l, start + r)] = ("kv", qkv[r])
        att = [("attn", s0 + 1, qkv[r], tuple(kv[(l, start + j)] for j in range(r + 1))) for r in range(S)]
        h1 = [("linear", l, "o", s0 + 1, att[r], h[r]) for r in range(S)]
        y2 = [("norm", 2 * l + 1, s0 + 2, v) for v in h1]
        gu = [("linear", l, "gate_up", s0 + 2, v, None) for v in y2]
        s = [("swiglu", s0 + 3, v) for v in gu]
        h = [("linear", l, "down", s0 + 3, s[r], h1[r]) for r in range(S)]
    return h, kv


@pytest.mark.parametrize("S", [1, 16, 37, 48])
def test_prefill_dataflow(monkeypatch, S):
    L = 1040
    start = L - S
    m, fake = _model(monkeypatch, 2, L)
    fake.start = start
    h = torch.zeros(S, I.HIDDEN, dtype=torch.bfloat16)
    fake.put(h, [("in", r) for r in range(S)])
    ids = m.prefill(h, start)
    h_exp, kv_exp = _expected(2, start, S)
    assert fake.get(h) == h_exp
    for key, v in kv_exp.items():
        assert fake.kv[key] == v, key
    # nothing outside the suffix's positions was written
    assert set(fake.kv) == set(kv_exp)
    # the head: the last row through the final norm (site 2 * SITES), the LM head, argmax
    i = m.n_layers * m.SITES
    assert fake.get(ids.view(-1, 1)) == [
        ("argmax", ("linear", None, "lm_head", i, ("norm", 2 * m.n_layers, i, h_exp[-1]), None))]
    assert fake.launches == m.prefill_launches(S)


def test_prefill_groups():
    assert step.prefill_chunks(100, 0) == []
    assert step.prefill_chunks(100, 5) == [(0, 5, 100)]
    assert step.prefill_chunks(7, 40) == [(0, 16, 7), (16, 16, 23), (32, 8, 39)]
    for start, S in [(0, 1), (3, 16), (998, 42), (0, 1000)]:
        g = step.prefill_chunks(start, S)
        assert sum(t for _, t, _ in g) == S
        assert all(1 <= t <= step.PREFILL_CHUNK and ctx == start + r for r, t, ctx in g)
        assert [r for r, _, _ in g] == list(range(0, S, step.PREFILL_CHUNK))
    with pytest.raises(ValueError):
        step.prefill_chunks(-1, 4)


def test_prefill_arguments(monkeypatch):
    m, fake = _model(monkeypatch, 1, 1040, lm_head=False)
    h = torch.zeros(8, I.HIDDEN, dtype=torch.bfloat16)
    assert m.prefill(h[:0], 100) is None and fake.launches == 0
    with pytest.raises(ValueError):
        m.prefill(h, m.n_log * I.PAGE - 7)           # last position past the page table
    with pytest.raises(ValueError):
        m.prefill(h.float(), 100)
    with pytest.raises(ValueError):
        m.prefill(torch.zeros(8, 2 * I.HIDDEN, dtype=torch.bfloat16)[:, ::2], 100)
    m.static = False
    with pytest.raises(RuntimeError):
        m.prefill(h, 100)


def test_prefill_layer_ranges(monkeypatch):
    """Layers 0..k-1 and then k..n-1 in two calls give the labels of one call;
    the head runs only in the call that ends with the last layer."""
    L, S = 1040, 21
    start = L - S
    m, fake = _model(monkeypatch, 3, L)
    fake.start = start
    h = torch.zeros(S, I.HIDDEN, dtype=torch.bfloat16)
    fake.put(h, [("in", r) for r in range(S)])
    assert m.prefill(h, start, layers=range(0, 1)) is None
    n1 = fake.launches
    ids = m.prefill(h, start, layers=range(1, 3))
    h_exp, kv_exp = _expected(3, start, S)
    assert fake.get(h) == h_exp and ids is not None
    assert all(fake.kv[k] == v for k, v in kv_exp.items())
    assert n1 > 0 and fake.launches == m.prefill_launches(S)
    with pytest.raises(ValueError):
        m.prefill(h, start, layers=[3])
