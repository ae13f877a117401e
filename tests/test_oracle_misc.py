"""Pins for the oracle's restore, KV append and layer glue.

Restore: byte equality of every restored page, every other page unchanged,
out-of-range ids rejected.  KV append: torch's float8_e4m3fn cast of the
same fp32 quotient.  RMSNorm / SwiGLU: torch's own rms_norm and silu in
fp64, and closed forms (constant row; silu(0) = 0).
"""
import numpy as np
import pytest
import torch

from nvfp4_skinny_gemm_b200 import inputs


def test_restore_bytes(oracle):
    rng = np.random.default_rng(11)
    pb = 96
    src = rng.integers(0, 256, 20 * pb, dtype=np.uint8)
    dst = rng.integers(0, 256, 30 * pb, dtype=np.uint8)
    before = dst.copy()
    src_ids = rng.permutation(20)[:12].astype(np.int32)
    dst_ids = rng.permutation(30)[:12].astype(np.int32)
    oracle.kv_page_restore(src, src_ids, dst, dst_ids, pb)
    for s, d in zip(src_ids, dst_ids):
        assert np.array_equal(dst[d * pb:(d + 1) * pb], src[s * pb:(s + 1) * pb])
    for d in set(range(30)) - set(dst_ids.tolist()):
        assert np.array_equal(dst[d * pb:(d + 1) * pb], before[d * pb:(d + 1) * pb])
    with pytest.raises(ValueError):
        oracle.kv_page_restore(src, np.array([20], np.int32), dst, np.array([0], np.int32), pb)


def test_kv_append_matches_torch_cast(oracle):
    T, Hkv, D, P, L = 16, 4, 128, 64, 100
    cache = inputs.kv_cache(110, L, T=T, Hkv=Hkv, D=D, P=P, fill_tree=False)
    rng = np.random.default_rng(12)
    kn = (rng.standard_normal((T, Hkv, D)) * 3).astype(np.float32)
    vn = (rng.standard_normal((T, Hkv, D)) * 3).astype(np.float32)
    kp, vp = cache.k_pool.copy(), cache.v_pool.copy()
    oracle.kv_append(kn, vn, kp, vp, cache.page_table, L, cache.k_scale, cache.v_scale)
    for i in range(T):
        p = L + i
        pg, slot = cache.page_table[p // P], p % P
        for h in range(Hkv):
            qk = np.clip(kn[i, h] / cache.k_scale[h], -448, 448).astype(np.float32)
            qv = np.clip(vn[i, h] / cache.v_scale[h], -448, 448).astype(np.float32)
            wk = torch.from_numpy(qk).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            wv = torch.from_numpy(qv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(kp[pg, h, slot], wk)
            assert np.array_equal(vp[pg, h, inputs.v_plane_offsets(D, P)[:, slot]], wv)
    # context untouched
    for p in range(L):
        pg, slot = cache.page_table[p // P], p % P
        assert np.array_equal(kp[pg, :, slot], cache.k_pool[pg, :, slot])


def test_rmsnorm(oracle):
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, 640)).astype(np.float32) * 5
    w = rng.uniform(0.5, 1.5, 640).astype(np.float32)
    got = oracle.rmsnorm(x, w, eps=1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (640,),
                                       torch.from_numpy(w).double(), eps=1e-6).numpy()
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-15)
    c = np.full((1, 64), -3.0, np.float32)
    assert np.allclose(oracle.rmsnorm(c, np.ones(64, np.float32), eps=0.0), -1.0, rtol=1e-15)


def test_swiglu(oracle):
    rng = np.random.default_rng(14)
    gu = rng.standard_normal((2, 2 * 300)).astype(np.float32) * 4
    got = oracle.swiglu(gu)
    t = torch.from_numpy(gu).double()
    ref = (torch.nn.functional.silu(t[:, :300]) * t[:, 300:]).numpy()
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-15)
    z = np.zeros((1, 2), np.float32); z[0, 1] = 7.0
    assert oracle.swiglu(z)[0, 0] == 0.0
