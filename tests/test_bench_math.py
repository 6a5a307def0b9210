"""The benchmark's roofline numerators: the algorithmic bytes and FLOPs it
divides by measured times, checked against the figures worked out by hand for
the workloads (no GPU)."""
import types

import numpy as np

import bench


def _case(seq_lens, HI, DI=128, K=2048, H=128, Dqk=576, Dv=512):
    seq_lens = np.asarray(seq_lens, np.int32)
    return types.SimpleNamespace(seq_lens=seq_lens, T=len(seq_lens), HI=HI, DI=DI, K=K, H=H, Dqk=Dqk, Dv=Dv)


def test_decode_128k_bytes():
    # layer: keys 8*131072*128 + queries/weights 8*32*(128+4) + gathered rows 8*2048*1152
    #        + q 8*128*1152 + gate 8*128*2 + out 8*128*1024 = 155,356,160
    # indexer (algorithmic): keys + queries/weights = 134,251,520; with its 8*131072*4 score writes 138,445,824
    c = _case([131072] * 8, HI=32)
    layer, indexer = bench.decode_bytes(c)
    assert layer == 155_356_160 and indexer == 134_251_520
    assert indexer + bench.score_write_bytes(c) == 138_445_824


def test_decode_1m_bytes():
    # 134,217,728 + 32*132 + 2048*1152 + 128*1152 + 256 + 128*1024 = 136,860,032
    layer, _ = bench.decode_bytes(_case([1 << 20], HI=32))
    assert layer == 136_860_032


def test_short_sequences_gather_only_what_they_hold():
    # a 1000-token sequence keeps all 1000 rows (< K)
    layer, _ = bench.decode_bytes(_case([1000], HI=16))
    assert layer == 1000 * 128 + 16 * 132 + 1000 * 1152 + 128 * 1152 + 256 + 128 * 1024


def test_swa_layer_bytes():
    # 64 sequences x 64 heads x 128 dims x 2 bytes x (2 x 128 window rows + q + out) = 270,532,608
    assert bench.swa_bytes(64, 64, 128, 128, 4096) == 270_532_608
    assert bench.swa_bytes(1, 1, 128, 128, 10) == 1 * 1 * 128 * 2 * (2 * 10 + 2)  # shorter than the window


def test_prefill_indexer_flops_and_topk_bytes():
    assert bench.prefill_indexer_flops(32768, 16, 128) == 2_199_090_364_416  # about 2.199e12
    assert bench.prefill_topk_bytes(32768, 2048) == 2_147_549_184 + 268_435_456


def _sampler(samples, max_mhz=1965):
    """A sampler holding the given (MHz, reason bits) readings, 1 ms apart."""
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.ok, c.samples, c.max_mhz = True, [(m, r, 1e-3 * i) for i, (m, r) in enumerate(samples)], max_mhz
    return c


def test_clock_record_rejects_slowdowns_and_unexplained_low_clocks():
    full, cap, hw, therm = 0, 0x4, 0x8, 0x40
    assert not _sampler([(1965, full)] * 10).rejected()
    assert not _sampler([(1300, cap)] * 10).rejected()          # power-capped: kept and noted
    assert _sampler([(1965, full)] * 9 + [(1965, hw)]).rejected()  # any hardware slowdown
    assert _sampler([(1800, therm)] * 10).rejected()
    assert _sampler([(1200, full)] * 10).rejected()              # stuck low with no reason: a clock lock
    s = _sampler([(1965, full)] * 6 + [(1300, cap)] * 4).summary()
    assert s["sm_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"] and s["samples"] == 10
    assert s["span_ms"] == 9.0  # first to last reading


def test_nominal_peaks_reported_beside_the_measured_ones():
    assert bench.SPEC_HBM_GBS == 7700.0 and bench.SPEC_FP8_TFLOPS == 4500.0
