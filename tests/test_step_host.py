"""Host logic of the verify step (VerifyModel.step), on the CPU, with the
label-moving fake of the library (tests/fake_lib.py).

For a 16-node tree and a chain of 4, with static and dynamic activation
scales, the final labels of the hidden rows, of every layer's tree slots and
of the argmax ids must be those of the layer definition (node i attends to
the context plus its ancestors and itself), and the number of launches must
be launches_per_step(), the count bench.py reports.
"""
import pytest
import torch

from fake_lib import expected_layers, fake_model, scale_label
from nvfp4_skinny_gemm_b200 import inputs as I


@pytest.mark.parametrize("static,T,chain", [(True, 16, False), (False, 16, False), (True, 4, True)])
def test_step_dataflow_and_launch_count(monkeypatch, static, T, chain):
    L, n_layers = 1000, 3
    m, fake = fake_model(monkeypatch, n_layers, L, T=T, static=static)
    fake.start = L
    parent = I.chain_parent(T) if chain else I.tree_parent(4, T)
    m.parent.copy_(torch.from_numpy(parent))
    inp = [fake.L("in", r) for r in range(T)]
    fake.put(m.h, inp)
    m.step()
    h_exp, kv_exp = expected_layers(fake.L, n_layers, L, T, parent, inp, static=static)
    assert fake.get(m.h) == h_exp
    for key, v in kv_exp.items():
        assert fake.kv[key] == v, key
    assert set(fake.kv) == set(kv_exp)
    Lb = fake.L
    sc = scale_label(Lb, static, n_layers * m.SITES, h_exp)
    assert fake.get(m.ids.view(-1, 1)) == [
        Lb("argmax", Lb("linear", None, "lm_head", sc, Lb("norm", 2 * n_layers, sc, v), None)) for v in h_exp]
    assert fake.launches == m.launches_per_step(restore=True)
    assert m.launches_per_layer == (9 if static else 11)


def test_launch_count_of_the_benchmarked_step(monkeypatch):
    """64 layers, static scales: 1 restore + 64 x 9 + 3 = 580 launches."""
    m, fake = fake_model(monkeypatch, 64, 1024)
    fake.start = 1024
    m.parent.copy_(torch.from_numpy(I.tree_parent(4)))
    m.step()
    assert fake.launches == m.launches_per_step() == 580


def test_agent_turn_restore_prefill_verify_accept(monkeypatch):
    """turn(): one restore, the suffix prefilled at positions prefix .. ctx-1,
    then the verify step whose every node attends to the whole prefilled
    suffix (and its ancestors), then acceptance on the step's argmax."""
    L, n_layers = 1000, 2
    m, fake = fake_model(monkeypatch, n_layers, L)
    S = L - m.prefix_tokens
    fake.start = m.prefix_tokens
    h_suf = torch.zeros(S, I.HIDDEN, dtype=torch.bfloat16)
    suf_in = [fake.L("suffix", r) for r in range(S)]
    fake.put(h_suf, suf_in)
    parent = I.tree_parent(4)
    m.parent.copy_(torch.from_numpy(parent))
    tree_in = [fake.L("node", r) for r in range(16)]
    fake.put(m.h, tree_in)
    draft = torch.zeros(16, dtype=torch.int32)
    fake.put(draft.view(-1, 1), [fake.L("draft", r) for r in range(16)])
    nxt, ids, acc = m.turn(h_suf, draft)
    assert fake.restores == 1 and acc == ("path", "n", "next")
    _, suf_kv = expected_layers(fake.L, n_layers, m.prefix_tokens, S, I.chain_parent(S), suf_in)
    ctx = [[suf_kv[(l, m.prefix_tokens + r)] for r in range(S)] for l in range(n_layers)]
    h_exp, tree_kv = expected_layers(fake.L, n_layers, L, 16, parent, tree_in, ctx_kv=ctx)
    assert fake.get(m.h) == h_exp
    assert all(fake.kv[k] == v for k, v in {**suf_kv, **tree_kv}.items())
    assert fake.accepted[0] == [fake.L("draft", r) for r in range(16)]
    assert fake.accepted[1] == fake.get(m.ids.view(-1, 1))
    assert fake.launches == 1 + m.prefill_launches(S) + m.launches_per_step(restore=False) + 2
    with pytest.raises(ValueError):
        m.turn(h_suf[:-1])
