"""bench.py's flop accounting, checked on CPU against the step it describes:
the algorithmic flops of one training step rebuilt from its matrix products
(forward, input-gradient and weight-gradient GEMMs) plus causal attention
(forward: Q K^T and P V over the keys j <= i; backward: twice that), and the
per-configuration values of the scope table."""
import pytest

import bench
import oracle


def _step_flops_per_token(depth, V, T):
    D = oracle.dims(depth, V)
    C, F, H = D["C"], D["F"], D["H"]
    M = T  # per token: divide everything by the token count M = B*T (B drops out)
    gemms = [(M, C + 256, C), (M, C, C), (M, F, C), (M, C, F)] * depth + [(M, V, C)]
    fwd = sum(2.0 * m * n * k for m, n, k in gemms)
    # causal attention: key j <= i, so T(T+1)/2 pairs per (row, head); two products of d = 128
    attn_fwd = depth * H * 2 * (2.0 * 128 * T * (T + 1) / 2)
    return (3 * fwd + 3 * attn_fwd) / M  # backward: dgrad + wgrad per GEMM, 2x the attention forward


@pytest.mark.parametrize("name,depth,T,listed", [("d4", 4, 256, 1.195e8), ("d12", 12, 1024, 7.974e8),
                                                  ("d20", 20, 2048, 2.823e9), ("d24", 24, 2048, 4.511e9),
                                                  ("d32", 32, 2048, 9.764e9)])
def test_model_flops_per_token(name, depth, T, listed):
    C = oracle.dims(depth, 65536)["C"]
    got = bench.model_flops_per_token(depth, C, 65536, T)
    # the formula counts T/2 keys per query where the step has (T+1)/2
    assert got == pytest.approx(_step_flops_per_token(depth, 65536, T), rel=1e-3)
    assert got == pytest.approx(listed, rel=5e-4)
    nc = bench.model_flops_per_token_noncausal(depth, C, 65536, T)
    assert nc - got == pytest.approx(6.0 * T * C * depth)


def test_job_rate_and_shard_seed():
    assert bench.job_rate(32768, 100.0, 1) == pytest.approx(327680.0)
    assert bench.job_rate(32768, 100.0, 8) == pytest.approx(8 * 327680.0)
    assert len({bench.shard_seed(2, r) for r in range(8)}) == 8


def test_mufu_fraction():
    # two operations per logit for B*T = 32768 tokens of V = 65536 logits at 148 SMs x 1485 MHz:
    # 4.29e9 operations over 3.52e12 per second = 1.22 ms is the bound
    bound_ms = 2.0 * 65536 * 32768 / (16 * 148 * 1485e6) * 1e3
    assert bench.mufu_fraction(bound_ms, 32768, 65536, 148, 1485.0) == pytest.approx(1.0)
    assert bench.mufu_fraction(2 * bound_ms, 32768, 65536, 148, 1485.0) == pytest.approx(0.5)


def test_window_flop_count():
    import bench
    # no window, or windows covering T, give the causal count
    base = bench.model_flops_per_token(20, 1280, 65536, 2048)
    assert bench.model_flops_per_token(20, 1280, 65536, 2048, [0] * 20) == base
    assert bench.model_flops_per_token(20, 1280, 65536, 2048, [2048] * 20) == base
    # a window of w keys: w - w^2/(2T) pairs per query instead of T/2
    one = bench.model_flops_per_token(1, 1280, 65536, 2048, [1024]) - bench.model_flops_per_token(1, 1280, 65536, 2048, [0])
    assert abs(one - 12.0 * 1280 * (1024 - 1024 ** 2 / 4096 - 1024)) < 1e-6


def test_traffic_is_reported_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    # roofline.traffic comes from a committed ncu summary, and only while the
    # kernel source still hashes to the one recorded there
    import hashlib
    src = tmp_path / "k.cuh"
    src.write_text("// kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    (prof / "k_traffic.txt").write_text(
        f"source_file: k.cuh\nsource_sha256: {sha}\ntraffic_bytes_per_launch: 1234.5\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k") == 1234.5
    src.write_text("// kernel v2\n")  # the kernel changed after the capture
    assert bench.traffic_record("k") is None
    assert bench.traffic_record("other") is None  # no summary at all
    (prof / "k_traffic.txt").write_text("traffic_bytes_per_launch: 1.0\n")  # no source recorded
    assert bench.traffic_record("k") is None
