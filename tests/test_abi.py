"""The C ABI without a GPU: libmla.so loads, exports every function that
the headers in include/ declare with the signature the binding uses, validates
arguments on the host, and its host-only RoPE table is right."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
from latent_attention_decode_absorbed_b200 import build as mla_build

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))


@pytest.fixture(scope="module")
def lib():
    mla_build.build()
    return mla.lib()


def _declarations():
    text = "\n".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = {}
    for m in re.finditer(r"(?:^|\n)\s*([A-Za-z_][\w\s\*]*?)\b(mla_\w+)\s*\(([^;{]*?)\)\s*;", text):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3)
        ps = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
        decls[name] = (ret, ps)
    return decls


def _code(param: str) -> str:
    if "*" in param or param.startswith("cudaStream_t"):
        return "p"
    if param.startswith("unsigned long long"):
        return "Q"
    t = param.split()[0] if not param.startswith("const") else param.split()[1]
    return {"int": "i", "mla_dtype": "i", "float": "f", "double": "d"}[t]


def test_header_declares_the_path():
    names = set(_declarations())
    for n in ["mla_cache_append", "mla_absorb_q", "mla_decode_fwd", "mla_combine", "mla_out_uv",
              "mla_rope_table", "mla_decode_workspace_bytes", "mla_status_string", "mla_last_error_message",
              "mla_version"]:
        assert n in names


def test_every_declared_symbol_is_exported_with_matching_signature(lib):
    decls = _declarations()
    assert decls, "no declarations parsed"
    for name, (ret, params) in decls.items():
        assert hasattr(lib, name), f"{name} not exported"
        assert name in mla._SIGS, f"binding lacks {name}"
        sig = "".join(_code(p) for p in params)
        assert sig == mla._SIGS[name][1], (name, sig, mla._SIGS[name][1])


def test_status_strings(lib):
    assert mla.status_string(0) == "ok"
    assert mla.status_string(mla.MLA_ERR_INVALID_ARG) == "invalid argument"
    assert mla.status_string(99) == "unknown status"
    assert mla.mla_version() >= 10000


def test_rope_table_host(lib):
    n = 4096
    cos = np.empty((n, 32), np.float32)
    sin = np.empty((n, 32), np.float32)
    mla.mla_rope_table(10000.0, n, cos, sin)
    i = np.arange(32)
    ang = np.arange(n)[:, None] * 10000.0 ** (-2.0 * i / 64.0)
    assert np.array_equal(cos, np.cos(ang).astype(np.float32))
    assert np.array_equal(sin, np.sin(ang).astype(np.float32))
    with pytest.raises(mla.MlaError):
        mla.mla_rope_table(10000.0, 0, cos, sin)
    with pytest.raises(mla.MlaError):
        mla.mla_rope_table(0.5, 4, cos, sin)


FAKE = 1 << 20   # a non-null, 128-byte-aligned value; never dereferenced (validation fails first)


def _decode_kwargs(**over):
    kw = dict(q_abs=FAKE, q_dtype=mla.MLA_BF16, cache=FAKE, cache_scale=None, cache_dtype=mla.MLA_BF16,
              num_pages=4, block_table=FAKE, max_pages_per_seq=4, page_size=64, seq_lens=FAKE, batch=1,
              q_len=1, n_heads=128, num_splits=2, split_tokens=128, softmax_scale=1 / math.sqrt(192),
              o_part=FAKE, lse_part=FAKE, err_word=None, stream=0)
    kw.update(over)
    return kw


@pytest.mark.parametrize("over,status", [
    (dict(page_size=32), mla.MLA_ERR_UNSUPPORTED),
    (dict(split_tokens=100), mla.MLA_ERR_INVALID_ARG),
    (dict(num_splits=1), mla.MLA_ERR_INVALID_ARG),            # 1*128 < 4*64
    (dict(n_heads=0), mla.MLA_ERR_INVALID_ARG),
    (dict(n_heads=129), mla.MLA_ERR_INVALID_ARG),
    (dict(q_dtype=mla.MLA_F32), mla.MLA_ERR_UNSUPPORTED),      # f32 q with bf16 cache
    (dict(cache_dtype=mla.MLA_E4M3), mla.MLA_ERR_INVALID_ARG),  # no cache_scale
    (dict(o_part=None), mla.MLA_ERR_INVALID_ARG),
    (dict(cache=FAKE + 64), mla.MLA_ERR_INVALID_ARG),          # cache not 128-byte aligned
    (dict(softmax_scale=float("nan")), mla.MLA_ERR_INVALID_ARG),
    (dict(batch=0), mla.MLA_ERR_INVALID_ARG),
])
def test_decode_validation(lib, over, status):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_fwd(**_decode_kwargs(**over))
    assert e.value.status == status
    assert lib.mla_last_error_message().decode().startswith("mla_decode_fwd")


def test_other_validation(lib):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_absorb_q(FAKE, FAKE, FAKE, FAKE, 4, 0, mla.MLA_BF16, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_out_uv(FAKE, FAKE, FAKE, 4, 8, mla.MLA_E4M3, 0)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
    with pytest.raises(mla.MlaError) as e:
        mla.mla_combine(FAKE, FAKE, 4, 8, 0, FAKE, mla.MLA_BF16, None, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_cache_append(FAKE, mla.MLA_BF16, 8, FAKE, FAKE, FAKE, 1, 4, 64, None, 1e-6, FAKE, FAKE, 256,
                             FAKE, None, mla.MLA_E4M3, 4, None, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG       # e4m3 without scale
    with pytest.raises(mla.MlaError) as e:
        mla.mla_cache_append(FAKE, mla.MLA_BF16, 8, FAKE, FAKE, FAKE, 1, 4, 64, None, -1.0, FAKE, FAKE, 256,
                             FAKE, None, mla.MLA_BF16, 4, None, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG       # negative eps
    with pytest.raises(mla.MlaError) as e:
        mla.mla_combine_shards(FAKE, None, 2, 4, 8, FAKE, mla.MLA_F32, None, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG       # null lse_shard
    with pytest.raises(mla.MlaError) as e:
        mla.mla_combine_shards(FAKE, FAKE, 0, 4, 8, FAKE, mla.MLA_F32, None, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG       # no shards
    with pytest.raises(mla.MlaError) as e:
        mla.mla_combine_shards(FAKE, FAKE, 2, 4, 8, FAKE, mla.MLA_E4M3, None, 0)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
    mla.mla_combine_shards(None, None, 2, 0, 8, None, mla.MLA_F32, None, 0)   # zero rows
    # zero-size work is accepted and enqueues nothing (no GPU touched)
    mla.mla_cache_append(None, mla.MLA_BF16, 0, None, None, None, 1, 4, 64, None, 1e-6, None, None, 256,
                         None, None, mla.MLA_BF16, 4, None, 0)
    mla.mla_absorb_q(None, None, None, None, 0, 8, mla.MLA_BF16, 0)


def test_decode_workspace_bytes_host(lib):
    # o_part [B*T, H, S, 512] + lse_part [B*T, H, S], fp32: the long workload's 134 MB + 262 KB
    assert mla.mla_decode_workspace_bytes(8, 1, 128, 64) == 8 * 128 * 64 * 513 * 4
    assert mla.mla_decode_workspace_bytes(128, 2, 128, 4) == 256 * 128 * 4 * 513 * 4
    assert mla.mla_decode_workspace_bytes(0, 1, 128, 4) == 0
    assert mla.mla_decode_workspace_bytes(1, 1, 16, -1) == 0


def _q8_kwargs(**over):
    kw = dict(q8=FAKE, q_scale=FAKE, cache=FAKE, cache_scale=FAKE, num_pages=4, block_table=FAKE,
              max_pages_per_seq=4, page_size=64, seq_lens=FAKE, batch=1, q_len=1, n_heads=128, num_splits=2,
              split_tokens=128, softmax_scale=1 / math.sqrt(192), o_part=FAKE, lse_part=FAKE, err_word=None,
              stream=0)
    kw.update(over)
    return kw


@pytest.mark.parametrize("over,status", [
    (dict(n_heads=64), mla.MLA_ERR_UNSUPPORTED),            # the 8-bit form is the pair kernel's: 65..128 heads
    (dict(n_heads=129), mla.MLA_ERR_UNSUPPORTED),
    (dict(page_size=32), mla.MLA_ERR_UNSUPPORTED),
    (dict(num_splits=1), mla.MLA_ERR_INVALID_ARG),          # 1*128 < 4*64
    (dict(q_scale=None), mla.MLA_ERR_INVALID_ARG),
    (dict(cache_scale=None), mla.MLA_ERR_INVALID_ARG),
    (dict(q8=FAKE + 8), mla.MLA_ERR_INVALID_ARG),
    (dict(softmax_scale=0.0), mla.MLA_ERR_INVALID_ARG),
    (dict(batch=40000, q_len=2), mla.MLA_ERR_UNSUPPORTED),   # more than 65535 query rows
])
def test_decode_q8_validation(lib, over, status):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_fwd_q8(**_q8_kwargs(**over))
    assert e.value.status == status
    assert lib.mla_last_error_message().decode().startswith("mla_decode_fwd_q8")


def test_split_q_validation(lib):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_split_q_e4m3(FAKE, 4, 0, FAKE, FAKE, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_split_q_e4m3(FAKE, 4, 128, None, FAKE, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_split_q_e4m3(FAKE + 2, 4, 128, FAKE, FAKE, 0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    mla.mla_split_q_e4m3(None, 0, 128, None, None, 0)        # zero rows: nothing enqueued
