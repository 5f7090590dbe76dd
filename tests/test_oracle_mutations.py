"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch each one.  A pin set that let one of these through would not be
evidence that the oracle is right."""
import math

import numpy as np
import pytest

import oracle
import oracle.mla_oracle as om
import pins

ORIG = {name: getattr(om, name) for name in
        ["attention_naive", "attention_absorbed", "rope_angles", "rope", "rms_norm",
         "e4m3_encode", "combine_partials", "absorb_q", "out_uv", "round_to_bf16",
          "normwise_rel_err", "out_projection", "kv_a_projection", "decompress_kv",
          "split_query_e4m3"]}


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(om, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _drop_rope_term(monkeypatch):
    _patch(monkeypatch, "attention_naive", lambda qn, qp, *a, **k: ORIG["attention_naive"](qn, qp * 0, *a, **k))
    _patch(monkeypatch, "attention_absorbed", lambda qn, qp, *a, **k: ORIG["attention_absorbed"](qn, qp * 0, *a, **k))


def _scale_128(monkeypatch):
    s = 1.0 / math.sqrt(128.0)
    _patch(monkeypatch, "attention_naive", lambda *a, **k: ORIG["attention_naive"](*a, softmax_scale=s))
    _patch(monkeypatch, "attention_absorbed", lambda *a, **k: ORIG["attention_absorbed"](*a, softmax_scale=s))


def _rope_wrong_direction(monkeypatch):
    _patch(monkeypatch, "rope_angles", lambda *a, **k: -ORIG["rope_angles"](*a, **k))


def _rope_half_split(monkeypatch):
    def rope(x, pos, theta=10000.0):
        x = np.asarray(x, np.float64)
        ang = om.rope_angles(pos, theta, x.shape[-1])
        h = x.shape[-1] // 2
        x0, x1 = x[..., :h], x[..., h:]
        return np.concatenate([x0 * np.cos(ang) - x1 * np.sin(ang), x0 * np.sin(ang) + x1 * np.cos(ang)], -1)
    _patch(monkeypatch, "rope", rope)


def _rms_no_sqrt(monkeypatch):
    def rms(c, gain=None, eps=1e-6):
        c = np.asarray(c, np.float64)
        y = c / (np.mean(c * c, axis=-1, keepdims=True) + eps)
        return y if gain is None else y * gain
    _patch(monkeypatch, "rms_norm", rms)


def _causal_excludes_self(monkeypatch):
    def naive(q_nope, q_pe, w_uk, w_uv, c, kr, softmax_scale=None):
        T = q_nope.shape[0]
        out = np.zeros((T, q_nope.shape[1], 128))
        for t in range(T):
            n = c.shape[0] - T + t            # one row short
            out[t] = ORIG["attention_naive"](q_nope[t:t + 1], q_pe[t:t + 1], w_uk, w_uv,
                                             c[:max(n, 1)], kr[:max(n, 1)])[0]
        return out
    _patch(monkeypatch, "attention_naive", naive)


def _e4m3_ties_away(monkeypatch):
    def enc(x):
        x = np.asarray(x, np.float64)
        nudged = x + np.sign(x) * np.abs(x) * 1e-12   # breaks ties away from zero
        return ORIG["e4m3_encode"](nudged)
    _patch(monkeypatch, "e4m3_encode", enc)


def _combine_no_weights(monkeypatch):
    def comb(o_part, lse_part):
        o = np.asarray(o_part).mean(axis=-2)
        return o, np.max(lse_part, axis=-1)
    _patch(monkeypatch, "combine_partials", comb)


def _wrong_value_matrix(monkeypatch):
    _patch(monkeypatch, "attention_absorbed",
           lambda qn, qp, wuk, wuv, *a, **k: ORIG["attention_absorbed"](qn, qp, wuk, wuk, *a, **k))


def _bf16_truncates(monkeypatch):
    def rb(x):
        x = np.asarray(x, np.float64)
        e = np.floor(np.log2(np.abs(np.where(x == 0, 1, x))))
        q = np.ldexp(1.0, (e - 7).astype(np.int64))
        return np.where(x == 0, 0.0, np.trunc(x / q) * q)
    _patch(monkeypatch, "round_to_bf16", rb)


def _gate_mean(monkeypatch):
    def gate(got, ref):
        got = np.asarray(got, np.float64); ref = np.asarray(ref, np.float64)
        return float(np.mean(np.linalg.norm(got - ref, axis=-1) / np.linalg.norm(ref, axis=-1)))
    _patch(monkeypatch, "normwise_rel_err", gate)


def _gate_den_from_got(monkeypatch):
    _patch(monkeypatch, "normwise_rel_err", lambda got, ref: ORIG["normwise_rel_err"](ref, got))


def _gate_wrong_axis(monkeypatch):
    def gate(got, ref):
        got = np.asarray(got, np.float64); ref = np.asarray(ref, np.float64)
        return float(np.max(np.linalg.norm(got - ref, axis=-2) / np.linalg.norm(ref, axis=-2)))
    _patch(monkeypatch, "normwise_rel_err", gate)


def _gate_zero(monkeypatch):
    _patch(monkeypatch, "normwise_rel_err", lambda got, ref: 0.0)


def _gate_global_norm(monkeypatch):
    def gate(got, ref):
        got = np.asarray(got, np.float64); ref = np.asarray(ref, np.float64)
        return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    _patch(monkeypatch, "normwise_rel_err", gate)


def _concat_interleaved(monkeypatch):
    def proj(out, w_o):
        out = np.asarray(out, np.float64)
        T, H, dv = out.shape
        return out.transpose(0, 2, 1).reshape(T, H * dv) @ np.asarray(w_o, np.float64).T   # i*H + h order
    _patch(monkeypatch, "out_projection", proj)


def _kv_a_transposed_halves(monkeypatch):
    def proj(h, w):
        kv = ORIG["kv_a_projection"](h, w)
        return np.concatenate([kv[:, 64:], kv[:, :64]], axis=1)      # rope channels first
    _patch(monkeypatch, "kv_a_projection", proj)


def _decompress_swapped(monkeypatch):
    def dec(c, w_uk, w_uv):
        k, v = ORIG["decompress_kv"](c, w_uk, w_uv)
        return v, k                                                  # keys from W_UV, values from W_UK
    _patch(monkeypatch, "decompress_kv", dec)


def _decompress_heads_reversed(monkeypatch):
    def dec(c, w_uk, w_uv):
        k, v = ORIG["decompress_kv"](c, w_uk, w_uv)
        return k[:, ::-1], v[:, ::-1]                                # head i gets head H-1-i's weights
    _patch(monkeypatch, "decompress_kv", dec)



def _split_lo_own_scale(monkeypatch):
    def split(q):
        hi, lo, sc = ORIG["split_query_e4m3"](q)
        y = om.e4m3_decode(lo) * 16.0                              # lo kept on a scale 16x finer
        return hi, om.e4m3_encode(y), sc
    _patch(monkeypatch, "split_query_e4m3", split)


def _split_scale_inverted(monkeypatch):
    def split(q):
        hi, lo, sc = ORIG["split_query_e4m3"](q)
        return hi, lo, np.where(sc > 0, 1.0 / np.where(sc > 0, sc, 1.0), 0.0).astype(np.float32)
    _patch(monkeypatch, "split_query_e4m3", split)

MUTATIONS = [_drop_rope_term, _scale_128, _rope_wrong_direction, _rope_half_split, _rms_no_sqrt,
             _causal_excludes_self, _e4m3_ties_away, _combine_no_weights, _wrong_value_matrix,
             _bf16_truncates, _gate_mean, _gate_den_from_got, _gate_wrong_axis, _gate_zero,
             _gate_global_norm, _concat_interleaved, _kv_a_transposed_halves, _decompress_swapped,
             _decompress_heads_reversed, _split_lo_own_scale, _split_scale_inverted]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__.strip("_"))
def test_pins_catch_mutation(monkeypatch, mutate):
    mutate(monkeypatch)
    caught = []
    for pin in pins.ALL_PINS:
        if pin is pins.pin_brute_force:
            continue                                  # slow; the others suffice
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught {mutate.__name__}"
