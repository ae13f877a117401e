"""Host logic of the suffix prefill (VerifyModel.prefill), on the CPU, with
the label-moving fake of the library (tests/fake_lib.py): the final labels of
the hidden rows, of every layer's cache positions and of the returned token
must be those of the layer definition applied to all suffix rows at once, as
one causal chain.  So the test fails if an attention block attends before
the K/V it needs is written or to K/V it must not see, a linear reads another
site's activation, another layer's pool or weights, or a quantiser uses
another site's scale.
"""
import pytest
import torch

from fake_lib import expected_layers, fake_model, scale_label
from nvfp4_skinny_gemm_b200 import inputs as I
from nvfp4_skinny_gemm_b200 import step


def _model(monkeypatch, n_layers, ctx_len, lm_head=True):
    return fake_model(monkeypatch, n_layers, ctx_len, lm_head=lm_head)


def _inputs(fake, S):
    return [fake.L("in", r) for r in range(S)]


def _expected(fake, n_layers, start, S):
    return expected_layers(fake.L, n_layers, start, S, I.chain_parent(S), _inputs(fake, S))


@pytest.mark.parametrize("S", [1, 16, 37, 130, 300])
def test_prefill_dataflow(monkeypatch, S):
    L = 1040
    start = L - S
    m, fake = _model(monkeypatch, 2, L)
    fake.start = start
    h = torch.zeros(S, I.HIDDEN, dtype=torch.bfloat16)
    fake.put(h, _inputs(fake, S))
    ids = m.prefill(h, start)
    h_exp, kv_exp = _expected(fake, 2, start, S)
    assert fake.get(h) == h_exp
    for key, v in kv_exp.items():
        assert fake.kv[key] == v, key
    # nothing outside the suffix's positions was written
    assert set(fake.kv) == set(kv_exp)
    # the head: the last row through the final norm (site 2 * SITES), the LM head, argmax
    L, sc = fake.L, scale_label(fake.L, True, m.n_layers * m.SITES, None)
    assert fake.get(ids.view(-1, 1)) == [
        L("argmax", L("linear", None, "lm_head", sc, L("norm", 2 * m.n_layers, sc, h_exp[-1]), None))]
    assert fake.launches == m.prefill_launches(S)


def test_prefill_groups():
    assert step.prefill_chunks(100, 0) == []
    assert step.prefill_chunks(100, 5) == [(0, 5, 100)]
    assert step.prefill_chunks(7, 300) == [(0, 128, 7), (128, 128, 135), (256, 44, 263)]
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
        m.prefill(h.to("meta"), 100)                 # another device than the model's
    with pytest.raises(ValueError):
        m.prefill(torch.zeros(8, 2 * I.HIDDEN, dtype=torch.bfloat16)[:, ::2], 100)
    m.static = False
    with pytest.raises(RuntimeError):
        m.prefill(h, 100)


def test_prefill_layer_ranges(monkeypatch):
    """Layers 0..k-1 and then k..n-1 in two calls give the labels of one call;
    the head runs only in the call that ends with the last layer."""
    L, S = 1040, 150
    start = L - S
    m, fake = _model(monkeypatch, 3, L)
    fake.start = start
    h = torch.zeros(S, I.HIDDEN, dtype=torch.bfloat16)
    fake.put(h, _inputs(fake, S))
    assert m.prefill(h, start, layers=range(0, 1)) is None
    n1 = fake.launches
    ids = m.prefill(h, start, layers=range(1, 3))
    h_exp, kv_exp = _expected(fake, 3, start, S)
    assert fake.get(h) == h_exp and ids is not None
    assert all(fake.kv[k] == v for k, v in kv_exp.items())
    assert n1 > 0 and fake.launches == m.prefill_launches(S)
    with pytest.raises(ValueError):
        m.prefill(h, start, layers=[3])
