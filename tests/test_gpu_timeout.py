"""The decode kernel's bounded waits, driven to run out without faulting or
hanging the GPU: a test hook makes every CTA pair's leader leave its first
query load out, so the MMA issuer's wait for it gives up after a short bound.
The launch must return on its own with MLA_DEVERR_TIMEOUT in err_word, and
the next launch in the same process (whose unit counter the aborted launch
must have reset) must be correct again."""
import math

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _problem(seed, lens, T, H, split_tokens):
    g = np.random.default_rng(seed)
    npg = [(L + 63) // 64 for L in lens]
    num_pages = sum(npg)
    ids = g.permutation(num_pages)
    bt = np.full((len(lens), max(npg)), -1, np.int32)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = ids[off:off + n]; off += n
    rows = round_bf16(g.standard_normal((num_pages * 64, 576)).astype(np.float32))
    qh = round_bf16(g.standard_normal((len(lens) * T, H, 576)).astype(np.float32) * 0.25)
    S = -(-bt.shape[1] * 64 // split_tokens)
    host = dict(rows=rows, q=qh, bt=bt, lens=list(lens), T=T, S=S, split=split_tokens)
    dev = dict(q_abs=to_device(qh, "bf16"), q_dtype=mla.MLA_BF16, cache=mla.pack_cache_rows(to_device(rows, "bf16")),
               cache_scale=None, cache_dtype=mla.MLA_BF16, num_pages=num_pages,
               block_table=torch.from_numpy(bt).cuda(), max_pages_per_seq=bt.shape[1], page_size=64,
               seq_lens=torch.tensor(lens, dtype=torch.int32).cuda(), batch=len(lens), q_len=T, n_heads=H,
               num_splits=S, split_tokens=split_tokens, softmax_scale=1 / math.sqrt(192))
    return host, dev


def _run(dev):
    rows = dev["batch"] * dev["q_len"]
    o_part = torch.full((rows, dev["n_heads"], dev["num_splits"], 512), float("nan"), device="cuda")
    lse_part = torch.full((rows, dev["n_heads"], dev["num_splits"]), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_decode_fwd(**dev, o_part=o_part, lse_part=lse_part, err_word=err)
    torch.cuda.synchronize()
    return o_part, lse_part, int(err.item())


def test_wait_bound_runs_out_then_next_launch_is_correct():
    host, dev = _problem(5, [300, 1000, 64], 1, 128, 256)
    try:
        # about 1 ms at 2 GHz: far above any wait of this small launch, far below a hang
        mla.mla_test_set_decode_wait(2_000_000, withhold_q_load=True)
        _, _, err = _run(dev)
        assert err & mla.MLA_DEVERR_TIMEOUT, f"err_word {err:#x} lacks MLA_DEVERR_TIMEOUT"
    finally:
        mla.mla_test_set_decode_wait(0, withhold_q_load=False)
    # the same process, the next launch: unit counter reset, results right
    o_part, lse_part, err = _run(dev)
    assert err == 0
    rows = dev["batch"] * dev["q_len"]
    o_lat = torch.empty((rows, dev["n_heads"], 512), device="cuda")
    lse = torch.empty((rows, dev["n_heads"]), device="cuda")
    mla.mla_combine(o_part, lse_part, rows, dev["n_heads"], dev["num_splits"], o_lat, mla.MLA_F32, lse)
    torch.cuda.synchronize()
    got_o, got_l = to_host_f64(o_lat), to_host_f64(lse)
    for b, L in enumerate(host["lens"]):
        slots = np.concatenate([host["bt"][b, j] * 64 + np.arange(64) for j in range((L + 63) // 64)])[:L]
        c = host["rows"][slots].astype(np.float64)
        q = host["q"][b:b + 1].astype(np.float64)
        o, l = oracle.attention_partials(q[..., :512], q[..., 512:], c[:, :512], c[:, 512:], host["split"], host["S"])
        oc, lc = oracle.combine_partials(o, l)
        assert oracle.normwise_rel_err(got_o[b:b + 1], oc) < 1e-2
        np.testing.assert_allclose(got_l[b:b + 1], lc, atol=1e-3)
