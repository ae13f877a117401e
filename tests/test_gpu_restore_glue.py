"""GPU parity of the prefix-cache restore (byte-exact), the FP8 KV append
(bit-exact), the fused RMSNorm/SwiGLU quantisers (every 16-block bit-exact,
up to the bf16 rounding of op outputs that sit at a rounding midpoint; see
tests/quant_check.py), the row argmax and the V-plane conversion."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda, host, to_dev
from quant_check import bf16_of, check_quant_bytes
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_src,n_dst,n,page_bytes", [(40, 50, 30, 32768), (10, 12, 7, 8208), (5, 5, 5, 96),
                                                      (2000, 2100, 1500, 65536)])
def test_restore_bytes(oracle, n_src, n_dst, n, page_bytes):
    cuda()
    rng = np.random.default_rng(90 + n)
    src = rng.integers(0, 256, n_src * page_bytes, dtype=np.uint8)
    dst = rng.integers(0, 256, n_dst * page_bytes, dtype=np.uint8)
    sid = rng.permutation(n_src)[:n].astype(np.int32)
    did = rng.permutation(n_dst)[:n].astype(np.int32)
    d_src, d_dst = to_dev(src), to_dev(dst)
    nv.kv_page_restore(d_src, to_dev(sid), d_dst, to_dev(did), page_bytes)
    want = dst.copy()
    oracle.kv_page_restore(src, sid, want, did, page_bytes)
    assert np.array_equal(d_dst.cpu().numpy(), want)


def test_restore_empty_and_bad_ids():
    cuda()
    pb = 1024
    src = torch.arange(8 * pb, dtype=torch.int64).to(torch.uint8).cuda()
    dst = torch.zeros(8 * pb, dtype=torch.uint8, device="cuda")
    ids = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    nv.kv_page_restore(src, ids, dst, ids, pb, n=0)
    assert int(dst.sum()) == 0
    nv.device_status()
    bad = torch.tensor([1, 9], dtype=torch.int32, device="cuda")
    nv.kv_page_restore(src, bad, dst, ids, pb)
    rc, _ = nv.device_status()
    assert rc == -7
    assert torch.equal(dst[:pb], src[pb:2 * pb])          # the valid pair was still copied
    assert int(dst[pb:2 * pb].sum()) == 0                 # the invalid one was skipped


def test_kv_append_bitexact(oracle):
    cuda()
    T, Hkv, D, P, L = 16, 4, 128, 64, 1000
    cache = inputs.kv_cache(91, L, fill_tree=False)
    qkv = inputs.bf16_normal(91, 3, (T, 4096))
    qkv[:, 3072:] *= 3.0
    kp, vp = to_dev(cache.k_pool), to_dev(cache.v_pool)
    d = to_dev(qkv)
    nv.kv_append(d[:, 3072:], d[:, 3584:], 4096, T, kp, vp, to_dev(cache.page_table), L, to_dev(cache.k_scale),
                 to_dev(cache.v_scale))
    kn = qkv[:, 3072:3584].float().numpy().reshape(T, Hkv, D)
    vn = qkv[:, 3584:].float().numpy().reshape(T, Hkv, D)
    wk, wv = cache.k_pool.copy(), cache.v_pool.copy()
    oracle.kv_append(kn, vn, wk, wv, cache.page_table, L, cache.k_scale, cache.v_scale)
    assert np.array_equal(kp.cpu().numpy(), wk)
    assert np.array_equal(vp.cpu().numpy(), wv)


def _dequant_err(oracle, codes, scales, g, want):
    deq = oracle.dequantize(codes.cpu().numpy(), scales.cpu().numpy(), float(g.cpu()[0]))
    return np.linalg.norm(deq - want) / np.linalg.norm(want)


@pytest.mark.parametrize("g_static", [None, 0.0019])
def test_rmsnorm_quantize(oracle, g_static):
    """g_static None: dynamic tensor scale; else the one-launch static-scale path."""
    cuda()
    rows, n = 16, inputs.HIDDEN
    x = inputs.bf16_normal(92, 0, (rows, n)) * 3
    w = inputs.bf16_normal(92, 1, (n,)) * 0.1 + 1
    out = (torch.empty(rows, n // 2, dtype=torch.uint8, device="cuda"),
           torch.empty(rows, n // 16, dtype=torch.uint8, device="cuda"),
           torch.empty(1, dtype=torch.float32, device="cuda"))
    g_in = None if g_static is None else to_dev(np.array([g_static], np.float32))
    nv.rmsnorm_quantize(to_dev(x), to_dev(w), 1e-6, out, g_in=g_in)
    y = oracle.rmsnorm(x.float().numpy(), w.float().numpy(), eps=1e-6)
    # codes and scales = NVFP4 of the bf16-rounded RMSNorm output, block by
    # block bit-exact against the oracle's, except where the exact value sits
    # at a bf16 rounding midpoint (then either rounding's bytes are correct)
    og = oracle.quantize(bf16_of(y).astype(np.float32), g_in=g_static)[2]
    assert np.float32(out[2].cpu()[0]) == np.float32(og)
    n_bad, _ = check_quant_bytes(oracle, y, out[0].cpu().numpy(), out[1].cpu().numpy(), og)
    print(f"rmsnorm quantise: {n_bad} of {y.size // 16} blocks at a bf16 rounding midpoint")
    assert _dequant_err(oracle, *out, y) < 0.12           # NVFP4 quantisation noise of N(0,1) data


@pytest.mark.parametrize("g_static", [None, 0.015])
def test_swiglu_quantize(oracle, g_static):
    cuda()
    rows, F = 16, inputs.FFN
    gu = inputs.bf16_normal(93, 0, (rows, 2 * F)) * 2
    out = (torch.empty(rows, F // 2, dtype=torch.uint8, device="cuda"),
           torch.empty(rows, F // 16, dtype=torch.uint8, device="cuda"),
           torch.empty(1, dtype=torch.float32, device="cuda"))
    g_in = None if g_static is None else to_dev(np.array([g_static], np.float32))
    nv.swiglu_quantize(to_dev(gu), out, g_in=g_in)
    h = oracle.swiglu(gu.float().numpy())
    og = oracle.quantize(bf16_of(h).astype(np.float32), g_in=g_static)[2]
    assert np.float32(out[2].cpu()[0]) == np.float32(og)
    n_bad, _ = check_quant_bytes(oracle, h, out[0].cpu().numpy(), out[1].cpu().numpy(), og)
    print(f"swiglu quantise: {n_bad} of {h.size // 16} blocks at a bf16 rounding midpoint")
    assert _dequant_err(oracle, *out, h) < 0.2


@pytest.mark.parametrize("rows,n", [(16, 151936), (1, 151936), (3, 1000), (16, 7)])
def test_argmax(rows, n):
    cuda()
    x = inputs.bf16_normal(94, n % 7, (rows, n))
    if n > 100:
        x[0, 17] = 50.0
        x[0, n - 3] = 50.0          # tie: lowest index wins
    got = nv.argmax(to_dev(x)).cpu().numpy()
    want = np.argmax(x.float().numpy(), axis=1)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("n,D,P", [(37, 128, 64), (5, 8, 16), (3, 64, 128), (1, 128, 128)])
def test_v_pages_to_tiled(n, D, P):
    """Token-major V planes -> tiled planes: every byte lands at the offset the
    tiled layout gives for its (dimension, slot)."""
    cuda()
    src = np.random.default_rng(95 + n).integers(0, 256, (n, P, D), dtype=np.uint8)
    got = nv.v_pages_to_tiled(to_dev(src)).cpu().numpy()
    off = inputs.v_plane_offsets(D, P)                 # [D, P]
    want = np.empty((n, D * P), np.uint8)
    want[:, off.ravel()] = src.transpose(0, 2, 1).reshape(n, D * P)
    assert np.array_equal(got, want)
