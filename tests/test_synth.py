"""The seeded input recipes: shapes, dtypes, structure and determinism."""
import numpy as np
import pytest

from memory_bound_fk_b200 import synth


def test_workload_table_sizes():
    w = synth.WORKLOADS
    assert w["cfg1_softmax"].shape == (256, 1000)
    assert w["cfg2_gelu"].numel * 4 == 32 * 2 ** 20
    assert w["cfg3_softmax"].algorithmic_bytes == 2 * 8192 * 4096 * 4
    assert w["cfg4_softmax"].shape == (1048576, 2048) and w["cfg4_softmax"].itemsize == 2
    assert w["cfg5_softmax"].numel * 4 == 256 * 2 ** 20


def test_cfg1_is_seed0_normal_sigma3_and_gelu_shares_it():
    a = synth.make("cfg1_softmax")
    g = synth.make("cfg1_gelu")
    assert a.dtype == np.float32 and np.array_equal(a.ravel(), g)
    assert abs(float(a.std()) - 3.0) < 0.02 and abs(float(a.mean())) < 0.02
    assert np.array_equal(a, synth.make("cfg1_softmax"))


def test_cfg2_recipe():
    x = synth.make("cfg2_gelu")
    assert x.shape == (8388608,) and x.dtype == np.float32
    assert np.all(np.abs(x) <= 20.0)
    # |x| > 6 essentially only comes from the 83886 uniform entries, of which
    # 70% land outside [-6, 6]
    big = int(np.count_nonzero(np.abs(x) > 6))
    assert abs(big - 0.7 * 83886) < 5 * np.sqrt(0.7 * 0.3 * 83886)


def test_cfg3_rows_have_exactly_410_neg_inf_and_chunking_is_consistent():
    rows = synth.cfg3_rows(60, 70)
    assert rows.shape == (10, 4096)
    assert np.all(np.isneginf(rows).sum(axis=1) == 410)
    fin = rows[np.isfinite(rows)]
    assert abs(float(fin.std()) - 4.0) < 0.1
    again = synth.cfg3_rows(64, 66)
    assert np.array_equal(again, rows[4:6])


def test_cfg4_head_causal_structure():
    h = synth.cfg4_head(7)
    assert h.shape == (2048, 2048) and h.dtype == np.uint16
    iu = np.triu_indices(2048, 1)
    assert np.all(h[iu] == 0xFF80)
    il = np.tril_indices(2048)
    vals = synth.bf16_bits_to_f32(h[il])
    assert np.all(np.isfinite(vals))
    assert abs(float(vals.std()) - 8.0) < 0.05
    assert np.array_equal(h, synth.cfg4_head(7))
    assert not np.array_equal(h, synth.cfg4_head(8))


def test_cfg5_one_offset_entry_per_row():
    r = synth.cfg5_rows(8, 16)
    assert r.shape == (8, 131072)
    assert np.all((r > 30).sum(axis=1) == 1)
    assert np.array_equal(synth.cfg5_rows(10, 12), r[2:4])


def test_bf16_packing_rounds_to_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    b = synth.f32_to_bf16_bits(v)
    assert list(b) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F81]
    assert np.array_equal(synth.bf16_bits_to_f32(b)[:4], np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5], np.float32))


@pytest.mark.parametrize("threads", [1, 3])
def test_threaded_generation_is_thread_count_invariant(threads):
    a = synth._cfg5(rows=16, cols=4096, threads=threads)
    b = synth._cfg5(rows=16, cols=4096, threads=8)
    assert np.array_equal(a, b)
