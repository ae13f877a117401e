"""A label-moving stand-in for the library binding, for CPU tests of the host
logic that sequences library calls (VerifyModel.step / prefill).

Every buffer row (and every cache position of every layer) holds a label that
spells out how its value was produced, e.g. ("norm", w, site, x) = RMSNorm
with weight row w of the row labelled x, quantised with site scale `site`.
Each fake op builds its output labels from the labels of what it reads, so a
test can compare the final labels with the ones the layer definition gives.
Labels are hash-consed: a label is the integer id of a flat tuple whose parts
are strings, numbers or the ids of other labels, so deep layer stacks compare
in constant time.
No kernel and no oracle runs; launches are counted as the library would
launch kernels (an attention call is two launches, split and combine: the
library's default, which attn_launches() reports).
"""
import numpy as np
import torch

from nvfp4_skinny_gemm_b200 import inputs as I
from nvfp4_skinny_gemm_b200 import step


def row0(x):
    """(storage id, first row) of a row-major view."""
    base = x.untyped_storage().data_ptr()
    return base, (x.data_ptr() - base) // (x.stride(0) * x.element_size())


def ancestors(parent, i):
    """Tree slots node i sees: its ancestors and itself, in slot order."""
    out = []
    while i >= 0:
        out.append(i)
        i = int(parent[i])
    return sorted(out)


class Labels:
    """Hash-consing table: L(*parts) is the id of the label with these parts."""

    def __init__(self):
        self.ids = {}

    def __call__(self, *parts):
        return self.ids.setdefault(parts, len(self.ids))


class FakeLib:
    def __init__(self):
        self.L = Labels()
        self.labels = {}          # (storage, row) -> label
        self.kv = {}              # (layer, position) -> label
        self.gl = {}              # g tensor data_ptr -> scale label
        self.launches = 0
        self.m = None
        self.wmap = {}
        self.start = 0            # first labelled cache position (earlier ones are context)
        self.restores = 0
        self.accepted = None

    # ---- helpers
    def rows(self, x, n=None):
        s, r0 = row0(x)
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

    def scale(self, g_in, g_out, src):
        """Label of the tensor scale a quantiser uses: the static site, or a
        dynamic scale that depends on every row it quantised."""
        lab = self.L("site", self.site_of(g_in)) if g_in is not None else self.L("dynamic", *src)
        self.gl[g_out.data_ptr()] = lab
        return lab

    def layer_of_pool(self, k_pool):
        for l in range(self.m.n_layers):
            if k_pool.data_ptr() == self.m.k_pool(l).data_ptr():
                return l
        raise AssertionError("not a layer's K pool")

    # ---- library surface
    def act_buffer(self, K, device=None):
        return torch.zeros(16, dtype=torch.uint8)

    def kv_page_restore(self, src_pool, src_ids, dst_pool, dst_ids, page_bytes, n=None, stream=None):
        self.launches += 1
        self.restores += 1

    def tree_accept(self, draft_tokens, target_argmax, parent, out=None, stream=None):
        self.launches += 1
        self.accepted = (self.get(draft_tokens.view(-1, 1)), self.get(target_argmax.view(-1, 1)))
        return ("path", "n", "next")

    def kv_compact(self, k_base, v_base, layer_stride, n_layers, Hkv, D, n_pool_pages, P, page_table, ctx_len,
                   path, n, T, stream=None):
        self.launches += 1
        assert (path, n) == ("path", "n") and ctx_len == self.m.L and n_layers == self.m.n_layers

    def _quant_out(self, out, act, labels):
        """A quantiser writes the 16-row prepared image (act) or, for any row
        count with a static scale, the canonical codes (out[0])."""
        if act is not None:
            assert len(labels) <= 16
            self.put(act, labels)
        else:
            assert out[0] is not None and out[0].shape[0] == len(labels)
            self.put(out[0], labels)

    def quantize(self, x, g_in=None, out=None, act=None, canonical=True, ws=None, stream=None):
        self.launches += 1
        assert act is not None or g_in is not None
        src = self.get(x)
        lab = self.scale(g_in, out[2], src)
        self._quant_out(out, act, [self.L("quant", lab, v) for v in src])
        return out

    def rmsnorm_quantize(self, x, w, eps, out, act=None, stream=None, g_in=None):
        self.launches += 1
        assert x.shape[0] <= 16 or (g_in is not None and act is None)
        src = self.get(x)
        widx = (w.data_ptr() - self.m.norm_w.data_ptr()) // (I.HIDDEN * 2)
        lab = self.scale(g_in, out[2], src)
        self._quant_out(out, act, [self.L("norm", widx, lab, v) for v in src])

    def swiglu_quantize(self, gu, out, act=None, stream=None, g_in=None):
        self.launches += 1
        assert gu.shape[0] <= 16 or (g_in is not None and act is None)
        src = self.get(gu)
        lab = self.scale(g_in, out[2], src)
        self._quant_out(out, act, [self.L("swiglu", lab, v) for v in src])

    def _tiles_out(self, tiles, labels):
        """A quantiser writing the wide tile image: rows 0 .. S-1 of tiles."""
        self.put(tiles[:len(labels)], labels)
        return tiles

    def quantize_tiles(self, x, g_in, tiles, g_out, stream=None):
        self.launches += 1
        src = self.get(x)
        lab = self.scale(g_in, g_out, src)
        return self._tiles_out(tiles, [self.L("quant", lab, v) for v in src])

    def rmsnorm_quantize_tiles(self, x, w, eps, g_in, tiles, g_out, stream=None):
        self.launches += 1
        src = self.get(x)
        widx = (w.data_ptr() - self.m.norm_w.data_ptr()) // (I.HIDDEN * 2)
        lab = self.scale(g_in, g_out, src)
        return self._tiles_out(tiles, [self.L("norm", widx, lab, v) for v in src])

    def swiglu_quantize_tiles(self, gu, g_in, tiles, g_out, stream=None):
        self.launches += 1
        src = self.get(gu)
        lab = self.scale(g_in, g_out, src)
        return self._tiles_out(tiles, [self.L("swiglu", lab, v) for v in src])

    def prepared_weight_bytes(self, N, K):
        return N * K

    def prepare_weight(self, codes, scales, N, K, out=None, stream=None):
        """Tile image of canonical codes: moves row labels (rows 0 .. N-1 of out)."""
        self.launches += 1
        assert codes.shape[0] == N and out is not None
        self.put(out[:N], self.get(codes))
        return out

    def linear_wide(self, a_prep, g_a, S, w_prep, g_w, N, K, y=None, residual=None, stream=None):
        self.launches += 1
        assert y.shape[0] == S
        l, name = self.wmap[id(w_prep)]
        a = self.get(a_prep[:S])
        res = None
        if residual is not None:
            assert residual.data_ptr() == y.data_ptr()
            res = self.get(residual)
        self.put(y, [self.L("linear", l, name, self.gl[g_a.data_ptr()], v, None if res is None else res[i])
                     for i, v in enumerate(a)])

    def causal_attn(self, q, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale, sm_scale=None, out=None,
                    ld_q=None, T=None, Hq=None, ws=None, stream=None):
        """Query i (position ctx_len + i) attends to every labelled context
        position and to the new positions ctx_len .. ctx_len + i."""
        self.launches += self.attn_launches()
        l = self.layer_of_pool(k_pool)
        assert 1 <= T <= 128 and Hq == I.N_Q_HEADS and ld_q == q.stride(0)
        assert (ctx_len + T + I.PAGE - 1) // I.PAGE <= self.m.n_log
        qs = self.get(q, T)
        ctx = [self.kv.get((l, p)) for p in range(self.start, ctx_len)]
        self.put(out, [self.L("attn", qs[i], *ctx, *[self.kv.get((l, ctx_len + j)) for j in range(i + 1)])
                       for i in range(T)])

    def linear(self, a_act, g_a, M, w_prep, g_w, N, K, y=None, residual=None, ws=None, stream=None):
        self.launches += 1
        assert 1 <= M <= 16 and y.shape[0] == M
        l, name = self.wmap[id(w_prep)]
        a = self.get(a_act, M)
        res = None
        if residual is not None:
            assert residual.data_ptr() == y.data_ptr()
            res = self.get(residual)
        self.put(y, [self.L("linear", l, name, self.gl[g_a.data_ptr()], v, None if res is None else res[i])
                     for i, v in enumerate(a)])

    def linear_swiglu(self, a_act, g_a, M, w_prep, g_w, F, K, g_out, act, ws=None, stream=None):
        """gate+up linear, SwiGLU and its quantisation with the static scale
        g_out, in one launch: the labels the two-launch sequence gives."""
        self.launches += 1
        assert 1 <= M <= 16
        l, name = self.wmap[id(w_prep)]
        assert name == "gate_up" and 2 * F == I.LAYER_LINEARS[name][1]
        gu = [self.L("linear", l, name, self.gl[g_a.data_ptr()], v, None) for v in self.get(a_act, M)]
        lab = self.scale(g_out, g_out, gu)
        self.put(act, [self.L("swiglu", lab, v) for v in gu])
        return act

    def kv_append(self, k_new, v_new, ld_new, T, k_pool, v_pool, page_table, ctx_len, k_scale, v_scale,
                  stream=None):
        self.launches += 1
        l = self.layer_of_pool(k_pool)
        assert v_pool.data_ptr() == self.m.v_pool(l).data_ptr()
        assert k_scale.data_ptr() == self.m.k_scale[l].data_ptr()
        qd, kd = I.N_Q_HEADS * I.HEAD_DIM, I.N_KV_HEADS * I.HEAD_DIM
        assert row0(k_new)[1] == row0(v_new)[1]
        assert (k_new.data_ptr() - row0(k_new)[0]) % (k_new.stride(0) * 2) == qd * 2
        assert (v_new.data_ptr() - row0(v_new)[0]) % (v_new.stride(0) * 2) == (qd + kd) * 2
        src = self.get(k_new, T)
        pt = page_table.numpy()
        for i in range(T):
            assert 0 <= pt[(ctx_len + i) // I.PAGE] < self.m.n_pool
            self.kv[(l, ctx_len + i)] = self.L("kv", src[i])

    @staticmethod
    def attn_launches(ctas=None, sms=None):
        return 2

    def tree_attn(self, q, k_pool, v_pool, page_table, ctx_len, parent, k_scale, v_scale, sm_scale=None,
                  out=None, ld_q=None, T=None, Hq=None, ws=None, stream=None, g_act=None, act=None):
        self.launches += self.attn_launches()
        l = self.layer_of_pool(k_pool)
        assert 1 <= T <= 16 and Hq == I.N_Q_HEADS and ld_q == q.stride(0)
        assert (ctx_len + T + I.PAGE - 1) // I.PAGE <= self.m.n_log
        par = parent.numpy()[:T]
        assert all(-1 <= par[i] < i for i in range(T))
        qs = self.get(q, T)
        ctx = [self.kv.get((l, p)) for p in range(self.start, ctx_len)]
        labels = [self.L("attn", qs[i], *ctx, *[self.kv.get((l, ctx_len + j)) for j in ancestors(par, i)])
                  for i in range(T)]
        self.put(out, labels)
        if act is not None:
            lab = self.L("site", self.site_of(g_act))
            self.gl[g_act.data_ptr()] = lab
            self.put(act, [self.L("quant", lab, v) for v in labels])

    def argmax(self, x, idx=None, ws=None, stream=None):
        self.launches += 1
        self.put(idx.view(-1, 1), [self.L("argmax", v) for v in self.get(x)])


class FakeWeight:
    def __init__(self, *shape):
        self.shape = shape[:2]

    def mul_(self, s):
        return self


def fake_model(monkeypatch, n_layers, ctx_len, T=16, lm_head=True, static=True):
    """A VerifyModel on the CPU whose library calls go to a FakeLib (weights
    are placeholders: no numbers are ever computed)."""
    fake = FakeLib()
    monkeypatch.setattr(step, "nv", fake)
    monkeypatch.setattr(step.torch, "randn", lambda *a, **k: FakeWeight(*a))
    monkeypatch.setattr(step.VerifyModel, "_fill_cache", lambda self, seed: None)
    monkeypatch.setattr(step.Linear, "from_fp32",
                        staticmethod(lambda w: step.Linear(object(), torch.ones(1), *w.shape)))
    m = step.VerifyModel(n_layers=n_layers, ctx_len=ctx_len, T=T, weights="device", device="cpu",
                         lm_head=lm_head)
    fake.m = m
    for l, lay in enumerate(m.layers):
        for name, lin in lay.items():
            fake.wmap[id(lin.prep)] = (l, name)
    if lm_head:
        fake.wmap[id(m.lm_head.prep)] = (None, "lm_head")
    m.static = static
    return m, fake


def scale_label(L, static, site, rows):
    """The tensor scale the definition uses at a quantisation site: the static
    per-site scale, or the dynamic one over all the rows it quantises."""
    return L("site", site) if static else L("dynamic", *rows)


def expected_layers(L, n_layers, start, S, parent, h, static=True, ctx_kv=None):
    """Labels the layer definition gives for S rows at cache positions
    start .. start+S-1, row i attending to the labelled context ctx_kv[l]
    (a list per layer, default none) and to the rows parent makes visible,
    with no grouping of rows anywhere.  Returns (h labels, {(layer, pos): kv})."""
    sites = step.VerifyModel.SITES
    kv = {}
    for l in range(n_layers):
        ctx = list(ctx_kv[l]) if ctx_kv is not None else []
        s0 = l * sites
        n_sc = scale_label(L, static, s0, h)
        y1 = [L("norm", 2 * l, n_sc, v) for v in h]
        qkv = [L("linear", l, "qkv", n_sc, v, None) for v in y1]
        for r in range(S):
            kv[(l, start + r)] = L("kv", qkv[r])
        att = [L("attn", qkv[r], *ctx, *[kv[(l, start + j)] for j in ancestors(parent, r)]) for r in range(S)]
        a_sc = scale_label(L, static, s0 + 1, att)
        aq = [L("quant", a_sc, v) for v in att]
        h1 = [L("linear", l, "o", a_sc, aq[r], h[r]) for r in range(S)]
        n2_sc = scale_label(L, static, s0 + 2, h1)
        y2 = [L("norm", 2 * l + 1, n2_sc, v) for v in h1]
        gu = [L("linear", l, "gate_up", n2_sc, v, None) for v in y2]
        s_sc = scale_label(L, static, s0 + 3, gu)
        s = [L("swiglu", s_sc, v) for v in gu]
        h = [L("linear", l, "down", s_sc, s[r], h1[r]) for r in range(S)]
    return h, kv
