"""CPU checks of the bench's work accounting: the admitted-pair count that
every TFLOP/s figure divides by equals the number of pairs the oracle's mask
admits (a plain count of the mask, written from the method's definition), and
the flop and byte conventions hold on hand-computed cases."""

import numpy as np
import pytest

import bench
from oracle import attention as oatt
from sink_augmented_gqa_b200 import workloads as wl


@pytest.mark.parametrize("off,T,window", [(0, 1, 0), (0, 64, 0), (0, 64, 16), (37, 19, 16), (0, 200, 128),
                                          (1000, 96, 128), (5, 3, 1), (0, 130, 200)])
def test_pairs_match_the_oracle_mask(off, T, window):
    want = int(oatt.allowed_mask(off, T, off + T, window).sum())
    assert bench.pairs(off, T, window) == want


def test_pairs_closed_forms():
    # full causal from offset 0: T (T + 1) / 2; a band of W keys: W per row once
    # the row has W keys behind it, so T W - W (W - 1) / 2 for T >= W
    assert bench.pairs(0, 4096, 0) == 4096 * 4097 // 2
    assert bench.pairs(0, 4096, 128) == 4096 * 128 - 128 * 127 // 2
    # at a large offset every band row sees exactly W keys
    assert bench.pairs(65536, 512, 128) == 512 * 128
    # one decode row at offset off sees off + 1 keys
    assert bench.pairs(131071, 1, 0) == 131072


def test_flops_convention():
    # 4 d flops per admitted pair and query head (QK^T and PV, 2 each)
    cfg = wl.CONFIGS["lite"]
    assert bench.flops(cfg, 0, cfg.T, 0) == 4 * cfg.d * cfg.B * cfg.n_q * (cfg.T * (cfg.T + 1) // 2)
    # the Lite full layer is ~0.206 TFLOP
    assert bench.flops(cfg, 0, cfg.T, 0) == pytest.approx(0.2062e12, rel=1e-3)


def test_job_throughput_sums_ranks():
    # whole-job value: units of all ranks over the slowest rank's time
    assert bench.job_throughput(4, 1e12, 1.0) == pytest.approx(4e15)
    assert np.isclose(bench.job_throughput(1, 5e11, 0.5), 1e15)


def test_handoff_work_and_bytes():
    cfg = wl.CONFIGS["handoff"]
    # the full layer's chunk: 16 sequences x 64 heads x 512 rows at offset 65,536
    f = bench.flops(cfg, cfg.offset, cfg.T, 0)
    assert f == 4 * 64 * 16 * 64 * (512 * 65536 + 512 * 513 // 2)
    assert f == pytest.approx(8.83e12, rel=2e-3)
    # decode rows read: the whole prefix on full layers, W rows on band layers
    assert bench.decode_rows(cfg.offset + cfg.T, 0) == cfg.offset + cfg.T + 1
    assert bench.decode_rows(cfg.offset + cfg.T, 128) == 128
    assert bench.decode_rows(5, 128) == 6
    # one decode step of the full layer reads ~2.16 GB of K and V
    assert cfg.B * bench.decode_rows(cfg.offset + cfg.T, 0) * bench.kv_row_bytes(cfg) == pytest.approx(
        2.165e9, rel=1e-3)
    # prefill bytes: q and out, the new k/v rows read and appended, and the
    # admitted prefix rows (W - 1 per sequence on the band layer)
    qo = 2 * 16 * 512 * 64 * 64 * 2
    new = 2 * 16 * 512 * 8 * 64 * 4
    assert bench.prefill_bytes(cfg, cfg.offset, cfg.T, 128) == qo + new + 16 * 127 * 8 * 64 * 4
    assert bench.prefill_bytes(cfg, 0, 100, 0) == 2 * 16 * 100 * 64 * 64 * 2 + 2 * 16 * 100 * 8 * 64 * 4


def test_roofline_fraction_takes_the_lower_roof():
    peaks = dict(tf=1000.0, hbm=5000.0)
    # 1 TFLOP over 1 GB in 2 ms: AI = 1000 flop/B, 500 TFLOP/s against the tensor roof
    r = bench.roofline_frac(500.0, 1e9, 2e-3, peaks)
    assert r["bound"] == "tensor" and r["frac_of_roofline"] == pytest.approx(0.5)
    # 10 GFLOP over 1 GB in 0.4 ms: AI = 10, roof 50 TFLOP/s (HBM), achieved 25
    r = bench.roofline_frac(25.0, 1e9, 0.4e-3, peaks)
    assert r["bound"] == "hbm" and r["roofline_TFLOP/s"] == pytest.approx(50.0)
    assert r["frac_of_roofline"] == pytest.approx(0.5)
