"""Host-side logic of bench.py that needs no GPU: the nvidia-smi clock
sampler's parsing and the reporting of throttle reasons."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

def test_clock_sampler_parses_and_flags_throttling():
    """bench.Clocks reads `nvidia-smi --query-gpu=... --format=csv,noheader,nounits`
    samples; the median SM clock and every active slowdown reason are reported."""
    sys.path.insert(0, ROOT)
    import bench

    class FakeProc:
        def __init__(self, out):
            self.out = out

        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return self.out, ""

    rows = ["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1950, 1965, 980.5, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1965, 1965, 990.0, 0x4, Not Active, Active, Not Active, Active",
            "garbage line"]
    c = bench.Clocks.__new__(bench.Clocks)
    c.proc = FakeProc("\n".join(rows))
    d = c.stop()
    assert d["sm_mhz"] == 1965.0 and d["sm_max_mhz"] == 1965.0 and d["samples"] == 3
    assert d["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    c.proc = None
    assert c.stop()["sm_mhz"] is None


def test_prefill_flops_brute_force():
    """bench.prefill_flops against a count over rows, positions and weights."""
    sys.path.insert(0, ROOT)
    import bench
    from nvfp4_skinny_gemm_b200 import inputs as I
    S, start, layers = 7, 11, 3
    lin, attn = bench.prefill_flops(S, start, layers)
    macs = 0
    for _ in range(layers):
        for K, N in I.LAYER_LINEARS.values():
            macs += S * N * K
    macs += I.VOCAB * I.HIDDEN                       # LM head, last row only
    assert lin == 2 * macs
    seen = sum(len(range(0, start + i + 1)) for i in range(S))
    # QK^T and PV: 2 x D multiply-adds per (row, head, visible position)
    assert attn == layers * I.N_Q_HEADS * seen * 2 * 2 * I.HEAD_DIM


def test_verify_step_algorithmic_linear_bytes(monkeypatch):
    """The bytes the bench divides by for the linears' roofline: per launch the
    weight codes + E4M3 scales, the activation codes + scales, the output (and
    the residual read of O and down), 64 layers + LM head at 16 rows.  The
    output is bf16, except gate+up with static scales, whose launch writes the
    NVFP4 codes + E4M3 scales of SwiGLU's N/2 features."""
    from fake_lib import fake_model
    from nvfp4_skinny_gemm_b200 import inputs as I
    m, _ = fake_model(monkeypatch, 64, 1024)
    T, tot = 16, 0
    for name, (K, N) in list(I.LAYER_LINEARS.items()) * 64:
        res = 2 if name in ("o", "down") else 1
        out = T * (N // 2) // 2 + T * (N // 2) // 16 if name == "gate_up" else res * T * N * 2
        tot += N * K // 2 + N * K // 16 + T * K // 2 + T * K // 16 + out
    K, N = I.HIDDEN, I.VOCAB
    tot += N * K // 2 + N * K // 16 + T * K // 2 + T * K // 16 + T * N * 2
    assert m.static and m.linear_bytes() == tot == 11_467_670_528
    m.static = False        # dynamic scales: gate+up writes bf16 gate and up
    assert m.linear_bytes() == 11_528_946_688


def test_verify_step_attention_and_restore_bytes(monkeypatch):
    """K+V bytes read per step (layers x 4 heads x 128 dims x 2 for K and V
    over the context and the 16 tree slots) and the restore's read + write of
    the reused prefix pages (32 KB planes, K and V, every layer)."""
    import math
    from fake_lib import fake_model
    n = 2                                            # both counts are linear in the layers
    for L in (1024, 8192, 23552):
        m, _ = fake_model(monkeypatch, n, L)
        assert m.attn_bytes() == n * 2 * (L + 16) * 4 * 128
        pages = math.ceil(round(0.96 * L) / 64)
        assert m.restore_bytes() == 2 * n * 2 * pages * 32768
    assert pages == 354                              # 22,610 prefix tokens at 23,552


def test_oracle_sample_on_one_thread():
    """The single-thread CPU baseline runs the same sample in a child process
    limited to one OpenMP thread (smaller than the multi-threaded figure)."""
    sys.path.insert(0, ROOT)
    import bench
    v1 = bench.oracle_sample_one_thread(1024, 2)
    assert v1 is not None and v1 > 0
    assert bench.oracle_sample_one_thread(1024, 2, timeout=0.01) is None


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """The DRAM traffic the bench reports next to each roofline comes from the
    committed ncu summary only while the summary's source hash matches the
    current kernel source; any other hash (an edited kernel) gives None."""
    import bench
    lin = bench.recorded_traffic()
    att = bench.recorded_attn_traffic()
    # when present (the kernels unchanged since the capture), close to the algorithmic bytes
    assert lin is None or 0.99 < lin / 11_468_270_000 < 1.01
    assert att is None or 0.99 < att / 24_133_632 < 1.02
    (tmp_path / "profiles").mkdir()
    for name, key in (("nvfp4_linear_verify_step.md", "traffic_bytes_per_step_of_linears"),
                      ("tree_attn_fp8kv_ctx23552_t16.md", "traffic_bytes_per_call_of_split")):
        (tmp_path / "profiles" / name).write_text(f"{key}: 1.0e+07 source: 0123456789abcdef\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0123456789abcdef")
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "fedcba9876543210")
    assert bench.recorded_traffic() == 1.0e7
    assert bench.recorded_attn_traffic() is None
