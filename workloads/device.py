"""Put a seeded workload on the GPU through the library's own calls.

GPU side only (the oracle never imports this).  It uploads the generator's
raw inputs and builds each sequence's cache with ``mla_cache_append``; it
holds no arithmetic of the method itself.
"""
from __future__ import annotations

import numpy as np

from . import (WORKLOADS, Workload, bf16_bits, block_table, kv_rows, new_token_positions, queries,
               seq_lens, weights)


def to_device(x: np.ndarray, dtype: str, device="cuda"):
    """float32 array (bf16-representable when dtype == 'bf16') -> torch tensor."""
    import torch
    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(device)


def to_host_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


class DeviceWorkload:
    """A workload's weights, step inputs and a filled cache on the GPU."""

    def __init__(self, w: Workload, split_tokens=None, device="cuda", build_cache=True, norm_gain=None, q8=None):
        import torch
        from latent_attention_decode_absorbed_b200 import DecodeStep
        self.w = w
        self.lens = seq_lens(w)
        self.bt, self.num_pages = block_table(w, self.lens)
        self.step = DecodeStep(batch=w.batch, q_len=w.q_len, n_heads=w.n_heads, dtype=w.dtype,
                               cache_dtype=w.cache_dtype, block_table=self.bt, num_pages=self.num_pages,
                               split_tokens=split_tokens or w.split_tokens, max_pos=int(self.lens.max()),
                               theta=w.theta, eps=w.eps, norm_gain=norm_gain, softmax_scale=w.softmax_scale,
                               device=device, q8=q8)
        self.step.seq_lens.copy_(torch.from_numpy(self.lens))
        qn, qp = queries(w)
        wuk, wuv = weights(w)
        self.q_nope, self.q_pe = to_device(qn, w.dtype, device), to_device(qp, w.dtype, device)
        self.w_uk, self.w_uv = to_device(wuk, w.dtype, device), to_device(wuv, w.dtype, device)
        sid, pos = new_token_positions(w, self.lens)
        self.seq_ids = torch.from_numpy(sid).to(device)
        self.positions = torch.from_numpy(pos).to(device)
        rows = np.concatenate([kv_rows(w, b, int(L) - w.q_len, int(L)) for b, L in enumerate(self.lens)])
        self.kv_new = to_device(rows, w.dtype, device)
        if build_cache:
            self.build_cache()

    def build_cache(self, chunk=65536):
        """Append every row of every sequence (positions 0..L_b-1)."""
        import torch
        dev = self.step.device
        for b, L in enumerate(self.lens):
            for lo in range(0, int(L), chunk):
                hi = min(int(L), lo + chunk)
                rows = to_device(kv_rows(self.w, b, lo, hi), self.w.dtype, dev)
                sid = torch.full((hi - lo,), b, dtype=torch.int32, device=dev)
                pos = torch.arange(lo, hi, dtype=torch.int32, device=dev)
                self.step.append(rows, sid, pos)
        torch.cuda.synchronize()

    def run(self, stream=None):
        return self.step.run(self.kv_new, self.seq_ids, self.positions, self.q_nope, self.q_pe,
                             self.w_uk, self.w_uv, stream)


def get(name: str, **kw) -> DeviceWorkload:
    return DeviceWorkload(WORKLOADS[name], **kw)
