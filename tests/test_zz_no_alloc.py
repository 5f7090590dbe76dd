"""mla_decode_static, the entry point for callers that cannot allocate device
memory themselves (it keeps the split partials in a scratch array the library
holds), against the workspace path mla_decode_fwd + mla_combine and against
the fp64 oracle's split partials and combine.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process (the first call on the device performs the scratch lookup)."""
import math

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

TOL = 1e-2          # the bf16-cache parity gate


def _problem(seed, lens, T, H, split_tokens, host=None):
    g = np.random.default_rng(seed)
    npg = [(L + 63) // 64 for L in lens]
    num_pages = sum(npg) + 1
    ids = g.permutation(num_pages)
    bt = np.full((len(lens), max(npg)), -1, np.int32)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = ids[off:off + n]; off += n
    rows = round_bf16(g.standard_normal((num_pages * 64, 576)).astype(np.float32))
    qh = round_bf16(g.standard_normal((len(lens) * T, H, 576)).astype(np.float32) * 0.25)
    cache = to_device(rows, "bf16")
    q = to_device(qh, "bf16")
    S = -(-bt.shape[1] * 64 // split_tokens)
    if host is not None:
        host.update(rows=rows, q=qh, bt=bt, lens=list(lens), T=T, S=S, split_tokens=split_tokens)
    return dict(q_abs=q, q_dtype=mla.MLA_BF16, cache=mla.pack_cache_rows(cache), cache_scale=None,
                cache_dtype=mla.MLA_BF16, num_pages=num_pages, block_table=torch.from_numpy(bt).cuda(),
                max_pages_per_seq=bt.shape[1], page_size=64,
                seq_lens=torch.tensor(lens, dtype=torch.int32).cuda(), batch=len(lens), q_len=T, n_heads=H,
                num_splits=S, split_tokens=split_tokens, softmax_scale=1 / math.sqrt(192))


def _with_workspace(p):
    rows = p["batch"] * p["q_len"]
    o_part = torch.empty((rows, p["n_heads"], p["num_splits"], 512), device="cuda")
    lse_part = torch.empty((rows, p["n_heads"], p["num_splits"]), device="cuda")
    o_lat = torch.empty((rows, p["n_heads"], 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((rows, p["n_heads"]), device="cuda")
    mla.mla_decode_fwd(**p, o_part=o_part, lse_part=lse_part)
    mla.mla_combine(o_part, lse_part, rows, p["n_heads"], p["num_splits"], o_lat, mla.MLA_BF16, lse)
    torch.cuda.synchronize()
    return to_host_f64(o_lat), to_host_f64(lse)


def _static(p):
    rows = p["batch"] * p["q_len"]
    o_lat = torch.full((rows, p["n_heads"], 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((rows, p["n_heads"]), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_decode_static(**p, o_lat=o_lat, o_dtype=mla.MLA_BF16, lse_out=lse, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return to_host_f64(o_lat), to_host_f64(lse)


def _oracle(h):
    """fp64 oracle: split partials of every sequence, then their combine."""
    o_all, l_all = [], []
    T = h["T"]
    for b, L in enumerate(h["lens"]):
        slots = np.concatenate([h["bt"][b, j] * 64 + np.arange(64) for j in range((L + 63) // 64)])[:L]
        c = h["rows"][slots].astype(np.float64)
        q = h["q"][b * T:(b + 1) * T].astype(np.float64)
        o, l = oracle.attention_partials(q[..., :512], q[..., 512:], c[:, :512], c[:, 512:],
                                         h["split_tokens"], h["S"])
        oc, lc = oracle.combine_partials(o, l)
        o_all.append(oc); l_all.append(lc)
    return np.concatenate(o_all), np.concatenate(l_all)


def test_static_scratch_matches_workspace_path_and_oracle_on_consecutive_calls():
    ha, hb = {}, {}
    a = _problem(1, [70, 300, 129], 1, 128, 128, ha)
    b = _problem(2, [5, 1000], 2, 64, 256, hb)
    refs = {id(a): _oracle(ha), id(b): _oracle(hb)}
    # two calls in a row with different shapes, then the first again: the
    # scratch keeps the previous call's contents, which must not leak through
    for p in (a, b, a):
        ref_o, ref_l = _with_workspace(p)
        got_o, got_l = _static(p)
        assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_l))
        assert oracle.normwise_rel_err(got_o, ref_o) < TOL
        np.testing.assert_allclose(got_l, ref_l, atol=1e-3)
        or_o, or_l = refs[id(p)]
        assert oracle.normwise_rel_err(got_o, or_o) < TOL
        np.testing.assert_allclose(got_l, or_l, atol=1e-3)


def test_static_scratch_at_exactly_its_capacity():
    # 1 row x 128 heads x 64 splits = 8192 partial rows: the last partial's
    # o_part row ends where the lse_part area of the scratch begins
    h = {}
    p = _problem(4, [64 * 64], 1, 128, 64, h)
    assert p["batch"] * p["q_len"] * p["n_heads"] * p["num_splits"] == mla.MLA_STATIC_MAX_PARTIALS
    ref_o, ref_l = _with_workspace(p)
    for _ in range(2):
        got_o, got_l = _static(p)
        assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_l))
        assert oracle.normwise_rel_err(got_o, ref_o) < TOL
        np.testing.assert_allclose(got_l, ref_l, atol=1e-3)
    or_o, or_l = _oracle(h)
    assert oracle.normwise_rel_err(got_o, or_o) < TOL
    np.testing.assert_allclose(got_l, or_l, atol=1e-3)


def test_static_scratch_rejects_requests_above_its_capacity():
    p = _problem(3, [64 * 40], 1, 128, 64)          # 1 row x 128 heads x 40 splits = 5120 partials
    big = dict(p, num_splits=65)                    # 128 x 65 = 8320 > 8192
    o_lat = torch.empty((1, 128, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_static(**big, o_lat=o_lat, o_dtype=mla.MLA_BF16)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    assert "exceeds the static scratch capacity" in str(e.value)
    assert mla.MLA_STATIC_MAX_PARTIALS == 8192
