"""Seeded input generators: shapes, determinism and page-table validity."""
import numpy as np
import pytest

import workloads as W


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_shapes_and_tables(name):
    w = W.WORKLOADS[name]
    lens = W.seq_lens(w)
    assert lens.shape == (w.batch,)
    if w.seq_len is None:
        lo, hi = w.len_range
        assert lens.min() >= lo and lens.max() <= hi
    bt, npages = W.block_table(w, lens)
    used = bt[bt >= 0]
    # every page of the pool is owned by exactly one (sequence, slot)
    assert np.array_equal(np.sort(used), np.arange(npages))
    for b in range(w.batch):
        n = (lens[b] + W.PAGE - 1) // W.PAGE
        assert np.all(bt[b, :n] >= 0) and np.all(bt[b, n:] == -1)
    if not w.paged:
        assert np.array_equal(used, np.arange(npages))
    qn, qp = W.queries(w)
    assert qn.shape == (w.batch * w.q_len, w.n_heads, 128) and qp.shape == (w.batch * w.q_len, w.n_heads, 64)
    wuk, wuv = W.weights(w)
    assert wuk.shape == wuv.shape == (w.n_heads, 128, 512)
    sid, pos = W.new_token_positions(w, lens)
    assert len(sid) == len(pos) == w.batch * w.q_len
    assert np.all(pos == np.repeat(lens, w.q_len) - w.q_len + np.tile(np.arange(w.q_len), w.batch))


def test_determinism_and_windows():
    w = W.WORKLOADS["v3_b1"]
    a = W.kv_rows(w, 0)
    b = W.kv_rows(w, 0)
    assert np.array_equal(a, b)
    # any window equals the same slice of the full draw
    assert np.array_equal(W.kv_rows(w, 0, 4000, 4096), a[4000:4096])
    assert np.array_equal(W.kv_rows(w, 0, 17, 5000 if a.shape[0] > 5000 else a.shape[0]), a[17:])
    # bf16 workloads hold bf16-representable values
    assert np.array_equal(W.round_bf16(a), a)
    q1 = W.queries(w)[0]
    assert np.array_equal(q1, W.queries(w)[0])
    w2 = W.with_overrides(w, seed=1)
    assert not np.array_equal(W.queries(w2)[0], q1)


def test_value_distributions():
    w = W.WORKLOADS["tiny"]
    wuk, _ = W.weights(w)
    assert abs(wuk.std() * np.sqrt(512) - 1.0) < 0.02
    rows = W.kv_rows(w, 0)
    assert abs(rows.mean()) < 0.02 and abs(rows.std() - 1.0) < 0.02


def test_round_bf16_cast():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], dtype=np.float32)
    y = W.round_bf16(x)
    assert list(y) == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0]
    assert np.array_equal(W.bf16_bits(np.array([1.0], np.float32)), np.array([0x3F80], np.uint16))
