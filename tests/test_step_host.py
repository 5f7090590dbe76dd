"""DecodeStep's host-side choices, on CPU tensors (no kernel runs): which
attention form a step uses and the buffers it owns for it."""
import numpy as np
import pytest

from latent_attention_decode_absorbed_b200 import DecodeStep

torch = pytest.importorskip("torch")


def _step(**kw):
    args = dict(batch=2, q_len=2, n_heads=128, dtype="bf16", cache_dtype="e4m3",
                block_table=np.arange(8, dtype=np.int32).reshape(2, 4), num_pages=8, split_tokens=128,
                device="cpu")
    args.update(kw)
    return DecodeStep(**args)


def test_e4m3_cache_with_65_to_128_heads_takes_the_8bit_form():
    for h in (65, 96, 128):
        st = _step(n_heads=h)
        assert st.q8
        assert tuple(st.q_e4m3.shape) == (4, 2, h, 576) and st.q_e4m3.dtype == torch.uint8
        assert tuple(st.q_scale.shape) == (4, h) and st.q_scale.dtype == torch.float32


def test_other_steps_keep_mla_decode_fwd():
    for kw in (dict(n_heads=64), dict(cache_dtype="bf16"), dict(n_heads=128, q8=False)):
        st = _step(**kw)
        assert not st.q8 and st.q_e4m3 is None and st.q_scale is None


def test_q8_asked_where_it_cannot_run():
    with pytest.raises(ValueError):
        _step(cache_dtype="bf16", q8=True)
    with pytest.raises(ValueError):
        _step(n_heads=16, q8=True)
