"""The composed verify step on the GPU: a 2-layer model with the LM head run
twice from the same inputs gives bit-identical hidden states and argmax ids
(every reduction in the library has a fixed order), in both activation-scale
modes; greedy acceptance of a draft that agrees with the target's first two
choices along a chain accepts exactly those nodes and compacts their K/V."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda
from nvfp4_skinny_gemm_b200 import inputs as I

pytestmark = pytest.mark.gpu


def test_step_is_deterministic_and_acceptance_runs(oracle):
    cuda()
    from nvfp4_skinny_gemm_b200.step import VerifyModel
    T = I.TREE_NODES
    m = VerifyModel(n_layers=2, ctx_len=1024, weights="device")
    h0 = I.bf16_normal(4, 300, (T, I.HIDDEN)).cuda()
    parent = torch.from_numpy(I.chain_parent(T)).cuda()

    def run():
        m.h.copy_(h0)
        m.parent.copy_(parent)
        m.step()
        torch.cuda.synchronize()
        return m.h.clone(), m.ids.clone()

    h1, ids1 = run()
    h2, ids2 = run()
    assert torch.equal(h1, h2) and torch.equal(ids1, ids2)
    m.calibrate()
    h3, ids3 = run()
    h4, ids4 = run()
    assert torch.equal(h3, h4) and torch.equal(ids3, ids4)
    # a draft whose nodes 1 and 2 match the target's choices after nodes 0 and 1
    ids = ids4.cpu().numpy()
    draft = np.full(T, -1, np.int32)
    draft[1], draft[2] = ids[0], ids[1]
    draft[3] = ids[2] + 1                   # node 3 disagrees
    kv_before = m.kv[:, :, :, :].clone()
    path, n, nxt = m.accept(torch.from_numpy(draft).cuda())
    n = int(n.cpu()[0])
    assert n == 3 and path.cpu().numpy()[:3].tolist() == [0, 1, 2] and int(nxt.cpu()[0]) == ids[2]
    # chain: path == [0, 1, 2] keeps every token in place, so the cache is unchanged
    assert torch.equal(m.kv, kv_before)
    assert oracle.tree_accept_greedy(draft, ids, I.chain_parent(T)) == ([0, 1, 2], int(ids[2]))
