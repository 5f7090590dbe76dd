"""The projections on either side of the attention core against the oracle,
on the GPU through the C ABI, at the DeepSeek-V3 model width d = 7168:

  mla_out_proj        u = W_O [o_1; ...; o_H]   (after mla_out_uv)
  mla_kv_proj_append  kv_a = W_kv,a h, then the cache rows of kv_a, in one kernel

Weights are synthetic (N(0, 1/fan_in)).  Tolerances come from the
arithmetic: bf16 inputs are exact, products are accumulated in fp32 over
K = 16384 (W_O) or 7168 (W_kv,a), in a split-K order that varies between
runs, so the fp32 results carry a relative error of order 1e-6."""
import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from gpu_common import bf16_exact_or_boundary
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

D_MODEL = 7168
DT = {"f32": mla.MLA_F32, "bf16": mla.MLA_BF16, "e4m3": mla.MLA_E4M3}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}


@pytest.mark.parametrize("rows,H", [(1, 128), (8, 128), (130, 128), (5, 16)])
def test_out_proj_matches_oracle(rows, H):
    g = np.random.default_rng(rows * 1000 + H)
    out = round_bf16(g.standard_normal((rows, H, 128)).astype(np.float32) * 0.3)
    w_o = round_bf16((g.standard_normal((D_MODEL, H * 128)) / np.sqrt(H * 128)).astype(np.float32))
    u = torch.full((rows, D_MODEL), float("nan"), device="cuda")
    mla.mla_out_proj(to_device(out, "bf16"), to_device(w_o, "bf16"), u, rows, H, D_MODEL)
    torch.cuda.synchronize()
    got = to_host_f64(u)
    ref = oracle.out_projection(out.astype(np.float64), w_o.astype(np.float64))
    assert np.all(np.isfinite(got))
    # one row = one vector: normwise relative error over the model width
    assert oracle.normwise_rel_err(got[:, None, :], ref[:, None, :]) < 1e-5
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-5)


def test_out_proj_rejects_a_width_it_does_not_tile():
    x = torch.zeros((1, 16, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((100, 16 * 128), dtype=torch.bfloat16, device="cuda")
    u = torch.zeros((1, 100), device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_out_proj(x, w, u, 1, 16, 100)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED


def _pool(lens, spare, seed):
    g = np.random.default_rng(seed)
    npg = [(L + 63) // 64 for L in lens]
    total = sum(npg) + spare
    ids = g.permutation(total)
    bt = np.full((len(lens), max(npg)), -1, np.int32)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = ids[off:off + n]
        off += n
    return bt, total


@pytest.mark.parametrize("cache_dt", ["bf16", "f32", "e4m3"])
@pytest.mark.parametrize("lens", [[1], [70, 5, 64], [130, 71]])
def test_kv_proj_append_matches_oracle(cache_dt, lens):
    bt, num_pages = _pool(lens, spare=3, seed=len(lens))
    g = np.random.default_rng(sum(lens))
    seq = np.concatenate([np.full(L, b) for b, L in enumerate(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(L) for L in lens]).astype(np.int32)
    order = g.permutation(len(seq))
    seq, pos = seq[order], pos[order]
    n = len(seq)
    h = round_bf16(g.standard_normal((n, D_MODEL)).astype(np.float32))
    w = round_bf16((g.standard_normal((576, D_MODEL)) / np.sqrt(D_MODEL)).astype(np.float32))
    gain = (1.0 + 0.3 * g.standard_normal(512)).astype(np.float32)
    eps, max_pos = 1e-6, 256
    cos = np.empty((max_pos, 32), np.float32); sin = np.empty_like(cos)
    mla.mla_rope_table(10000.0, max_pos, cos, sin)
    cache = torch.zeros((num_pages, 9, 64, 64), dtype=TDT[cache_dt], device="cuda")
    cache.view(torch.uint8).fill_(0xFF)                     # sentinel: every byte 0xFF
    scale = torch.full((num_pages, 64), float("nan"), device="cuda") if cache_dt == "e4m3" else None
    ws = torch.full((mla.mla_kv_proj_workspace_bytes(n),), 0x7F, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_kv_proj_append(to_device(h, "bf16"), to_device(w, "bf16"), n, D_MODEL, ws,
                           torch.from_numpy(seq).cuda(), torch.from_numpy(pos).cuda(), torch.from_numpy(bt).cuda(),
                           len(lens), bt.shape[1], 64, torch.from_numpy(gain).cuda(), eps,
                           torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda(), max_pos, cache, scale,
                           DT[cache_dt], num_pages, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows_dev = mla.unpack_cache_rows(cache)
    raw = rows_dev.contiguous().view(torch.uint8).cpu().numpy().reshape(num_pages * 64, -1)
    slot = bt[seq, pos // 64].astype(np.int64) * 64 + pos % 64
    # indexing: exactly the appended slots changed
    touched = np.zeros(num_pages * 64, bool); touched[slot] = True
    assert np.all(raw[~touched] == 0xFF)
    assert not np.any(np.all(raw[touched] == 0xFF, axis=1))
    # (1) the projection: the call leaves the fp32 kv_a rows in its workspace;
    # they must match the oracle's fp64 W_kv,a h to fp32-accumulation accuracy
    kv_gpu = ws[:n * 576 * 4].view(torch.float32).view(n, 576).cpu().numpy().astype(np.float64)
    kv_ref = oracle.kv_a_projection(h.astype(np.float64), w.astype(np.float64))
    assert oracle.normwise_rel_err(kv_gpu[:, None, :], kv_ref[:, None, :]) < 1e-5
    np.testing.assert_allclose(kv_gpu, kv_ref, rtol=0, atol=1e-4)
    # (2) the rows written from it: as exact as mla_cache_append on the same
    # fp32 rows (RMSNorm, RoPE, rounding of the oracle applied to kv_gpu)
    ref = oracle.cache_rows(kv_gpu, pos, gain, eps)
    if cache_dt == "f32":
        got = rows_dev.cpu().numpy().astype(np.float64)[slot]
        np.testing.assert_allclose(got, ref, rtol=2e-6, atol=1e-6)
    elif cache_dt == "bf16":
        got = rows_dev.to(torch.float64).cpu().numpy()[slot]
        bad = bf16_exact_or_boundary(got, ref)
        assert not bad.any(), f"{bad.sum()} bf16 values off (first at {np.argwhere(bad)[:3]})"
    else:
        codes = rows_dev.cpu().numpy()[slot]
        sc = scale.view(-1).cpu().numpy().astype(np.float64)
        assert np.all(np.isnan(np.delete(sc, slot)))
        ref_codes, ref_scale = oracle.quantize_rows_e4m3(ref)
        np.testing.assert_allclose(sc[slot], ref_scale, rtol=2e-6)
        diff = codes != ref_codes
        if diff.any():
            # only where x*448/a sits within fp32 error of a rounding tie
            y = ref * (448.0 / np.max(np.abs(ref), axis=1, keepdims=True))
            a, bq = oracle.e4m3_decode(codes[diff]), oracle.e4m3_decode(ref_codes[diff])
            mid = 0.5 * (a + bq)
            assert np.all(np.abs(y[diff] - mid) <= 1e-5 * np.abs(y[diff])), "e4m3 codes differ away from a tie"
            assert diff.mean() < 1e-3
    # and the end-to-end error of the cached values against the fp64 chain
    # h -> W_kv,a h -> rows stays within the storage rounding
    full = oracle.stored_rows(oracle.cache_rows_from_hidden(h.astype(np.float64), w.astype(np.float64), pos, gain,
                                                            eps), cache_dt)[0]
    stored = oracle.stored_rows(ref, cache_dt)[0]
    assert oracle.normwise_rel_err(stored[:, None, :], full[:, None, :]) < {"f32": 1e-5, "bf16": 1e-2, "e4m3": 3e-2}[cache_dt]


@pytest.mark.parametrize("cache_dt", ["bf16", "e4m3"])
def test_layer_chain_from_hidden_states(cache_dt):
    """One layer end to end through DecodeStep: the step's new tokens enter as
    hidden states (append_from_hidden: W_kv,a, then the cache rows), attention
    over the whole cache, W_UV per head, then W_O over all heads
    (project_model); against the oracle's fp64 chain on the same inputs."""
    import workloads as W
    from gpu_common import TOL
    from workloads.device import DeviceWorkload
    w = W.Workload("chain_" + cache_dt, 3, 2, 128, None, (130, 400), "bf16", cache_dt, True, 256, seed=21)
    dw = DeviceWorkload(w)            # the cache holds the workload's rows at every position
    st = dw.step
    g = np.random.default_rng(77)
    n = w.batch * w.q_len
    h = round_bf16(g.standard_normal((n, D_MODEL)).astype(np.float32))
    w_kva = round_bf16((g.standard_normal((576, D_MODEL)) / np.sqrt(D_MODEL)).astype(np.float32))
    w_o = round_bf16((g.standard_normal((D_MODEL, w.n_heads * 128)) / np.sqrt(w.n_heads * 128)).astype(np.float32))
    # the new tokens (the last q_len positions of each sequence) come from h
    st.append_from_hidden(to_device(h, "bf16"), to_device(w_kva, "bf16"), dw.seq_ids, dw.positions)
    st.absorb(dw.q_nope, dw.q_pe, dw.w_uk)
    st.attend()
    st.combine()
    st.project_out(dw.w_uv)
    u = st.project_model(to_device(w_o, "bf16"))
    torch.cuda.synchronize()
    assert int(st.err.item()) == 0
    got = to_host_f64(u).reshape(w.batch, w.q_len, D_MODEL)
    qn, qp = W.queries(w)
    wuk, wuv = W.weights(w)
    sid, pos = dw.seq_ids.cpu().numpy(), dw.positions.cpu().numpy()
    for b, L in enumerate(dw.lens):
        L = int(L)
        old = oracle.sequence_cache(W.kv_rows(w, b)[:L - w.q_len], cache_dt, None, w.eps, w.theta)
        mine = np.flatnonzero(sid == b)
        mine = mine[np.argsort(pos[mine])]
        new = oracle.stored_rows(oracle.cache_rows_from_hidden(h[mine].astype(np.float64), w_kva.astype(np.float64),
                                                               pos[mine], None, w.eps, w.theta), cache_dt)[0]
        c_hat = np.concatenate([old[0], new[:, :512]])
        k_r = np.concatenate([old[1], new[:, 512:]])
        rows = slice(b * w.q_len, (b + 1) * w.q_len)
        out = oracle.attention_absorbed(qn[rows], qp[rows], wuk, wuv, c_hat, k_r)[0]
        ref = oracle.out_projection(out, w_o.astype(np.float64))
        assert oracle.normwise_rel_err(got[b][:, None, :], ref[:, None, :]) < TOL[cache_dt], f"seq {b}"
