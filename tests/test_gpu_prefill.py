"""Suffix prefill on the GPU (VerifyModel.prefill): S prompt tokens that the
prefix cache does not hold go through every layer, all rows at once in the
linears; the attention runs in blocks of 128 queries, each block attending to
the context before it (earlier blocks included) plus its own causal chain.

(1) Per layer, teacher-forced against the oracle run over all S rows at once
    (no groups): RMSNorm + NVFP4 with the static site scales, the NVFP4
    linears with M = S, the FP8 append of the S tokens' K/V (bit-exact pool),
    causal attention as ONE chain of S tokens after the context, SwiGLU.  The
    bars are those of the one-layer verify test (rel-Frobenius 1e-2 on the
    composed outputs; attention 2e-3 + 2^-8 |o| against the oracle fed the
    GPU's own Q and cache).  S = 20 spans a full group and a ragged one.
(1b) The attention blocks of a 5-block suffix as prefill() runs them (spread
    over streams at the prefill's split count): against the oracle's one
    causal chain, and bit-identical to the same calls made one after another.
(2) The whole call with the LM head: the returned token is the first argmax
    of the last row's logits; two calls over layer ranges [0, 1) and [1, 2)
    give the bits of one call; a second run gives the same bits.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import ATTN_ABS_TOL, cuda, rel_fro
from nvfp4_skinny_gemm_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _calibrated(L, weights, lm_head):
    from nvfp4_skinny_gemm_b200.step import VerifyModel
    m = VerifyModel(n_layers=2, ctx_len=L, T=I.TREE_NODES, weights=weights, lm_head=lm_head)
    m.parent.copy_(torch.from_numpy(I.tree_parent(4)))
    m.restore()
    m.h.copy_(I.bf16_normal(4, 300, (I.TREE_NODES, I.HIDDEN)) * 0.5)
    m.calibrate(restore=False)
    m.restore()
    return m


def test_prefill_layers_teacher_forced(oracle):
    cuda()
    L, S = 1024, 20
    start = L - S
    m = _calibrated(L, "host", lm_head=False)
    G = m.G.cpu().numpy()
    hs = (I.bf16_normal(4, 301, (S, I.HIDDEN)) * 0.5).cuda()
    ones = np.ones(I.HIDDEN, np.float32)
    qd, kd = I.N_Q_HEADS * I.HEAD_DIM, I.N_KV_HEADS * I.HEAD_DIM
    pt = m.page_table_h
    for l in range(m.n_layers):
        s0 = l * m.SITES
        kp = m.k_pool(l).cpu().numpy().copy()
        vp = m.v_pool(l).cpu().numpy().copy()
        h = hs.float().cpu().numpy()
        assert m.prefill(hs, start, layers=[l]) is None
        torch.cuda.synchronize()
        qkv_gpu = m._pf["qkv"][:S].float().cpu().numpy()
        attn_gpu = m._pf["attn"][:S].float().cpu().numpy()
        h2_gpu = hs.float().cpu().numpy()

        wq = {name: oracle.quantize(I.weight_fp32(4, t, N, K, sub=l))
              for t, (name, (K, N)) in enumerate(I.LAYER_LINEARS.items())}

        def lin(x_bf16, name, site):
            ac, asc, ga = oracle.quantize(x_bf16, g_in=float(G[site]))
            return oracle.linear(ac, asc, ga, *wq[name])

        y1 = _bf16(oracle.rmsnorm(h, ones, eps=m.eps))
        qkv = _bf16(lin(y1, "qkv", s0))
        assert rel_fro(qkv_gpu, qkv) <= 1e-2, (l, rel_fro(qkv_gpu, qkv))
        ks, vs = m.k_scale[l].cpu().numpy(), m.v_scale[l].cpu().numpy()
        oracle.kv_append(qkv_gpu[:, qd:qd + kd].reshape(S, I.N_KV_HEADS, I.HEAD_DIM),
                         qkv_gpu[:, qd + kd:].reshape(S, I.N_KV_HEADS, I.HEAD_DIM), kp, vp, pt, start, ks, vs)
        assert np.array_equal(m.k_pool(l).cpu().numpy(), kp)
        assert np.array_equal(m.v_pool(l).cpu().numpy(), vp)
        # one causal chain of all S tokens after the context, no groups
        a = oracle.tree_attn(qkv_gpu[:, :qd].reshape(S, I.N_Q_HEADS, I.HEAD_DIM), kp, vp, pt, start,
                             I.chain_parent(S), ks, vs)
        err_a = np.abs(attn_gpu.reshape(a.shape) - a)
        assert np.all(err_a <= 2e-3 + 2.0 ** -8 * np.abs(a)), (l, err_a.max())
        h1 = _bf16(h + lin(attn_gpu, "o", s0 + 1))
        y2 = _bf16(oracle.rmsnorm(h1, ones, eps=m.eps))
        gu = _bf16(lin(y2, "gate_up", s0 + 2))
        s = _bf16(oracle.swiglu(gu))
        h2 = _bf16(h1 + lin(s, "down", s0 + 3))
        err = rel_fro(h2_gpu, h2)
        print(f"prefill layer {l}: rel-Frobenius {err:.2e}")
        assert err <= 1e-2 and np.isfinite(h2_gpu).all()


def test_prefill_attention_blocks_on_streams(oracle):
    """A 520-token suffix after 4,000 cached tokens: 5 blocks, which prefill()
    spreads over its streams at PREFILL_ATTN_SPLITS splits per query head."""
    cuda()
    from nvfp4_skinny_gemm_b200 import lib as nv
    from nvfp4_skinny_gemm_b200.step import PREFILL_ATTN_SPLITS, VerifyModel, prefill_chunks
    start, S = 4000, 520
    L = start + S
    m = VerifyModel(n_layers=1, ctx_len=L, T=I.TREE_NODES, weights="device", lm_head=False)
    m.restore()
    qd, kd = I.N_Q_HEADS * I.HEAD_DIM, I.N_KV_HEADS * I.HEAD_DIM
    pf = m._prefill_buffers(S)
    qkv, attn = pf["qkv"][:S], pf["attn"][:S]
    qkv.copy_(I.bf16_normal(4, 303, (S, qkv.shape[1])) * 0.5)
    kp_d, vp_d, ks, vs = m.k_pool(0), m.v_pool(0), m.k_scale[0], m.v_scale[0]
    nv.kv_append(qkv[:, qd:], qkv[:, qd + kd:], qkv.stride(0), S, kp_d, vp_d, m.page_table, start, ks, vs)
    chunks = prefill_chunks(start, S)
    assert len(chunks) == 5 and m._causal_splits(len(chunks)) == PREFILL_ATTN_SPLITS
    m._causal_blocks(pf, 0, qkv, attn, start, S)
    seq = torch.empty_like(attn)
    with nv.option(nv.OPT_ATTN_SPLITS, PREFILL_ATTN_SPLITS):
        for r, t, ctx in chunks:
            nv.causal_attn(qkv[r:r + t], kp_d, vp_d, m.page_table, ctx, ks, vs, out=seq[r:r + t],
                           ld_q=qkv.stride(0), T=t, Hq=I.N_Q_HEADS)
    torch.cuda.synchronize()
    assert nv.get_option(nv.OPT_ATTN_SPLITS) == 0
    assert torch.equal(attn, seq)
    got = attn.float().cpu().numpy()
    a = oracle.tree_attn(qkv[:, :qd].float().cpu().numpy().reshape(S, I.N_Q_HEADS, I.HEAD_DIM),
                         kp_d.cpu().numpy(), vp_d.cpu().numpy(), m.page_table_h, start, I.chain_parent(S),
                         ks.cpu().numpy(), vs.cpu().numpy())
    assert np.isfinite(got).all()
    err = np.abs(got.reshape(a.shape) - a)
    assert np.all(err <= ATTN_ABS_TOL + 2.0 ** -8 * np.abs(a)), err.max()


def test_prefill_head_ranges_determinism():
    cuda()
    L, S = 1024, 37
    start = L - S
    m = _calibrated(L, "device", lm_head=True)
    h0 = (I.bf16_normal(4, 302, (S, I.HIDDEN)) * 0.5).cuda()
    kv0 = m.kv.clone()

    def run(ranges):
        m.kv.copy_(kv0)
        h = h0.clone()
        for r in ranges:
            ids = m.prefill(h, start, layers=r)
        torch.cuda.synchronize()
        return h, ids.clone(), m.kv.clone(), m._pf["logits"].clone()

    h_a, ids_a, kv_a, lg_a = run([None])
    h_b, ids_b, kv_b, lg_b = run([None])
    h_c, ids_c, kv_c, lg_c = run([range(0, 1), range(1, 2)])
    assert torch.equal(h_a, h_b) and torch.equal(kv_a, kv_b) and torch.equal(ids_a, ids_b)
    assert torch.equal(h_a, h_c) and torch.equal(kv_a, kv_c) and torch.equal(ids_a, ids_c)
    assert torch.isfinite(lg_a.float()).all()
    lg = lg_a.float().cpu().numpy()[0]
    assert int(ids_a.cpu()[0]) == int(np.flatnonzero(lg == lg.max())[0])
    # only the suffix's cache positions changed, in both layers
    changed = (kv_a != kv0).cpu().numpy()             # [layers, 2, pool pages, 32 KB]
    P = I.PAGE
    pages = {int(m.page_table_h[p // P]) for p in range(start, L)}
    assert changed[:, :, sorted(pages)].any(axis=(2, 3)).all()
    others = [pg for pg in range(m.n_pool) if pg not in pages]
    assert not changed[:, :, others].any()


@pytest.mark.parametrize("rows", [942, 130, 1, 256])
def test_quantisers_write_the_wide_tile_image(rows):
    """The prefill's quantisation sites write the wide linear's tile image
    directly: byte for byte what nvfp4_prepare_weight makes of the same
    quantiser's canonical codes and scales (rows past `rows` in the last
    128-row tile are left as they were: zero here, as prepare_weight pads)."""
    cuda()
    from nvfp4_skinny_gemm_b200 import lib as nv
    dev = torch.device("cuda")
    g_in = torch.full((1,), 0.0023, dtype=torch.float32, device=dev)
    g_out = torch.empty(1, dtype=torch.float32, device=dev)

    def check(K, canon, tiles_call):
        ref = nv.prepare_weight(*canon, rows, K)
        tiles = torch.zeros(nv.prepared_weight_bytes(rows, K), dtype=torch.uint8, device=dev)
        tiles_call(tiles)
        torch.cuda.synchronize()
        assert nv.device_status() == (0, 0)
        assert float(g_out.cpu()[0]) == float(g_in.cpu()[0])
        assert torch.equal(tiles.cpu(), ref.cpu())

    def canon_out(K):
        return (torch.empty(rows, K // 2, dtype=torch.uint8, device=dev),
                torch.empty(rows, K // 16, dtype=torch.uint8, device=dev),
                torch.empty(1, dtype=torch.float32, device=dev))

    H, F, QD = I.HIDDEN, I.FFN, I.N_Q_HEADS * I.HEAD_DIM
    x = (I.bf16_normal(95, 0, (rows, H)) * 2).to(dev)
    w = (I.bf16_normal(95, 1, (H,)) * 0.1 + 1).to(dev)
    out = canon_out(H)
    nv.rmsnorm_quantize(x, w, 1e-6, out, g_in=g_in)
    check(H, out[:2], lambda t: nv.rmsnorm_quantize_tiles(x, w, 1e-6, g_in, t, g_out))

    a = I.bf16_normal(95, 2, (rows, QD)).to(dev)
    out = canon_out(QD)
    nv.quantize(a, g_in=g_in, out=out)
    check(QD, out[:2], lambda t: nv.quantize_tiles(a, g_in, t, g_out))
    a32 = a.float()
    out = canon_out(QD)
    nv.quantize(a32, g_in=g_in, out=out)
    check(QD, out[:2], lambda t: nv.quantize_tiles(a32, g_in, t, g_out))

    gu = (I.bf16_normal(95, 3, (rows, 2 * F)) * 2).to(dev)
    out = canon_out(F)
    nv.swiglu_quantize(gu, out, g_in=g_in)
    check(F, out[:2], lambda t: nv.swiglu_quantize_tiles(gu, g_in, t, g_out))
