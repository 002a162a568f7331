"""The fp64 oracle against its pins (CPU only), and the pins' own sensitivity:
each plausible mistake, planted in a CPU stand-in of the oracle, must trip at
least one pin."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def oracle_impl(q, kv, sl, scale, d_v):
    return oracle.mla_decode(q, kv, sl, scale, d_v=d_v)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle_impl)


def sink_oracle_impl(q, kv, sl, scale, d_v, sinks):
    return oracle.mla_decode(q, kv, sl, scale, d_v=d_v, sinks=sinks)


@pytest.mark.parametrize("pin", pins.SINK_PINS, ids=lambda p: p.__name__)
def test_oracle_sink_pin(pin):
    pin(sink_oracle_impl)


def test_sink_rows_entry_matches_full():
    g = torch.Generator().manual_seed(5)
    q = (torch.randn(2, 2, 3, 576, generator=g)).to(torch.bfloat16)
    kv = (torch.randn(2, 30, 576, generator=g)).to(torch.bfloat16)
    sl = np.array([30, 0], np.int32)
    sinks = np.array([0.5, -1.0, 3.0])
    out, lse = oracle.mla_decode(q, kv, sl, pins.SCALE, sinks=sinks)
    rows = np.array([0, 4, 7, 11])
    o2, l2 = oracle.mla_decode_rows(q, kv, sl, pins.SCALE, rows, sinks=sinks)
    np.testing.assert_array_equal(o2, out.reshape(-1, 512)[rows])
    np.testing.assert_array_equal(l2, lse.reshape(-1)[rows])


def test_rows_entry_matches_full():
    g = torch.Generator().manual_seed(3)
    q = (torch.randn(3, 2, 5, 576, generator=g)).to(torch.bfloat16)
    kv = (torch.randn(3, 40, 576, generator=g)).to(torch.bfloat16)
    sl = np.array([40, 1, 0], np.int32)
    out, lse = oracle.mla_decode(q, kv, sl, pins.SCALE)
    rows = np.array([0, 7, 12, 13, 29, 10], np.int64)
    o2, l2 = oracle.mla_decode_rows(q, kv, sl, pins.SCALE, rows)
    np.testing.assert_array_equal(o2, out.reshape(-1, 512)[rows])
    np.testing.assert_array_equal(l2, lse.reshape(-1)[rows])


def test_rejects_bad_lengths():
    q = torch.zeros(1, 1, 1, 576, dtype=torch.bfloat16)
    kv = torch.zeros(1, 4, 576, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        oracle.mla_decode(q, kv, np.array([5], np.int32), pins.SCALE)
    with pytest.raises(ValueError):
        oracle.mla_decode(q, kv, np.array([-1], np.int32), pins.SCALE)


def test_golden_fixture_reproduces():
    """tests/golden/tiny_oracle.json was written by tests/golden/make_golden.py,
    which calls only oracle/; the oracle must keep reproducing it."""
    from mla_decode_attention_11_b200 import workloads as W
    with open(os.path.join(GOLDEN, "tiny_oracle.json")) as f:
        gold = json.load(f)
    w = W.WORKLOADS[gold["workload"]]
    q, kv, sl = W.generate(w)
    out, lse = oracle.mla_decode(q, kv, sl, w.scale)
    np.testing.assert_allclose(lse.reshape(-1), np.array(gold["lse"]), rtol=0, atol=1e-12)
    flat = out.reshape(-1)
    idx = np.array(gold["out_index"], dtype=np.int64)
    np.testing.assert_allclose(flat[idx], np.array(gold["out_value"]), rtol=0, atol=1e-12)


def test_fp8_golden_fixture_reproduces():
    """tests/golden/tiny_fp8_oracle.json: the FP8-cache oracle on the tiny
    workload's quantised cache, written by tests/golden/make_golden.py."""
    from mla_decode_attention_11_b200 import workloads as W
    with open(os.path.join(GOLDEN, "tiny_fp8_oracle.json")) as f:
        gold = json.load(f)
    w = W.WORKLOADS[gold["workload"]]
    q, codes, ks, sl = W.generate_fp8(w)
    assert ks == gold["kv_scale"]
    out, lse = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale)
    np.testing.assert_allclose(lse.reshape(-1), np.array(gold["lse"]), rtol=0, atol=1e-12)
    idx = np.array(gold["out_index"], dtype=np.int64)
    np.testing.assert_allclose(out.reshape(-1)[idx], np.array(gold["out_value"]), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- mutants
# CPU stand-ins of the oracle with one planted mistake each.  They are never
# used as references; they exist only to show the pins would catch the mistake.

def _np_attention(q, kv, sl, scale, d_v, *, qk_cols=None, v_cols=None, lse_base=math.e,
                  scale_used=True, sign=1.0, len_delta=0, add_max_to_lse=True,
                  normalise=True, head_mixup=False, sinks=None, sink_mode="correct"):
    qd = q.to(torch.float64).numpy()
    kd = kv.to(torch.float64).numpy()
    B, Sq, H, d = qd.shape
    out = np.zeros((B, Sq, H, d_v))
    lse = np.zeros((B, Sq, H))
    qc = slice(0, d) if qk_cols is None else qk_cols
    vc = slice(0, d_v) if v_cols is None else slice(d - d_v, d)  # "last d_v columns"
    for b in range(B):
        L = int(sl[b]) + len_delta
        L = max(0, min(L, kd.shape[1]))
        for t in range(Sq):
            for h in range(H):
                sg = -np.inf if sinks is None else float(sinks[0 if sink_mode == "first_head" else h])
                if sink_mode == "scaled":
                    sg *= scale
                if L == 0:
                    lse[b, t, h] = -np.inf if (sink_mode == "empty_minus_inf" or sinks is None) else sg
                    continue
                qrow = qd[b, t, 0 if head_mixup else h]
                s = sign * (kd[b, :L, qc] @ qrow[qc]) * (scale if scale_used else 1.0)
                m = s.max()
                if sink_mode != "not_in_max":
                    m = max(m, sg)
                w = np.exp(s - m)
                l = w.sum()
                if sink_mode != "ignored":
                    l += np.exp(sg - m)
                o = w @ kd[b, :L, vc]
                if sink_mode == "carries_first_value":
                    o = o + np.exp(sg - m) * kd[b, 0, vc]
                out[b, t, h] = o / l if normalise else o
                lse[b, t, h] = ((m if add_max_to_lse else 0.0) + np.log(l)) / math.log(lse_base)
    return out, lse


MUTANTS = {
    "correct": {},
    "drop_rope_columns": dict(qk_cols=slice(0, 512)),
    "values_from_last_columns": dict(v_cols="last"),
    "lse_in_base_2": dict(lse_base=2.0),
    "scale_ignored": dict(scale_used=False),
    "score_sign_flipped": dict(sign=-1.0),
    "one_key_short": dict(len_delta=-1),
    "one_key_past_end": dict(len_delta=+1),
    "max_missing_from_lse": dict(add_max_to_lse=False),
    "output_not_normalised": dict(normalise=False),
    "heads_mixed_up": dict(head_mixup=True),
}


SINK_MUTANTS = {
    "correct": {},
    "sink_ignored": dict(sink_mode="ignored"),
    "sink_multiplied_by_scale": dict(sink_mode="scaled"),
    "sink_left_out_of_max": dict(sink_mode="not_in_max"),
    "sink_carries_a_value": dict(sink_mode="carries_first_value"),
    "first_head_sink_for_all": dict(sink_mode="first_head"),
    "empty_sequence_lse_minus_inf": dict(sink_mode="empty_minus_inf"),
}


def _run_sink_pins(kwargs):
    def impl(q, kv, sl, scale, d_v, sinks):
        return _np_attention(q, kv, sl, scale, d_v, sinks=sinks, **kwargs)
    failed = []
    for pin in pins.SINK_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(SINK_MUTANTS))
def test_sink_pins_catch_planted_mistakes(name):
    failed = _run_sink_pins(SINK_MUTANTS[name])
    if name == "correct":
        assert failed == [], f"a correct stand-in must pass every sink pin, failed: {failed}"
    else:
        assert failed, f"planted mistake '{name}' passed every sink pin"


def _run_pins(kwargs):
    def impl(q, kv, sl, scale, d_v):
        return _np_attention(q, kv, sl, scale, d_v, **kwargs)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name):
    failed = _run_pins(MUTANTS[name])
    if name == "correct":
        assert failed == [], f"a correct stand-in must pass every pin, failed: {failed}"
    else:
        assert failed, f"planted mistake '{name}' passed every pin"



# ---------------------------------------------------------------- MHA decode oracle

def mha_oracle_impl(q, k, v, sl, scale):
    return oracle.mha_decode(q, k, v, sl, scale)


@pytest.mark.parametrize("pin", pins.MHA_PINS, ids=lambda p: p.__name__)
def test_mha_oracle_pin(pin):
    pin(mha_oracle_impl)


def _np_mha(q, k, v, sl, scale, *, group_map="div", values_from_k=False, scale_used=True, len_delta=0):
    qd, kd, vd = (x.to(torch.float64).numpy() for x in (q, k, v))
    B, Sq, H, D = qd.shape
    Hkv, Dv = kd.shape[2], vd.shape[3]
    out = np.zeros((B, Sq, H, Dv))
    lse = np.zeros((B, Sq, H))
    for b in range(B):
        L = max(0, min(int(sl[b]) + len_delta, kd.shape[1]))
        for t in range(Sq):
            for h in range(H):
                hk = h // (H // Hkv) if group_map == "div" else h % Hkv
                if L == 0:
                    lse[b, t, h] = -np.inf
                    continue
                s = (kd[b, :L, hk] @ qd[b, t, h]) * (scale if scale_used else 1.0)
                m = s.max()
                w = np.exp(s - m)
                vals = kd[b, :L, hk, :Dv] if values_from_k else vd[b, :L, hk]
                out[b, t, h] = (w @ vals) / w.sum()
                lse[b, t, h] = m + np.log(w.sum())
    return out, lse


MHA_MUTANTS = {
    "correct": {},
    "kv_head_h_mod_hkv": dict(group_map="mod"),
    "values_from_k": dict(values_from_k=True),
    "scale_ignored": dict(scale_used=False),
    "one_key_short": dict(len_delta=-1),
}


@pytest.mark.parametrize("name", sorted(MHA_MUTANTS))
def test_mha_pins_catch_planted_mistakes(name):
    def impl(q, k, v, sl, scale):
        return _np_mha(q, k, v, sl, scale, **MHA_MUTANTS[name])
    failed = []
    for pin in pins.MHA_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    if name == "correct":
        assert failed == [], f"a correct stand-in must pass every MHA pin, failed: {failed}"
    else:
        assert failed, f"planted mistake '{name}' passed every MHA pin"


# ---------------------------------------------------------------- MHA decode oracle with sinks

@pytest.mark.parametrize("pin", pins.MHA_SINK_PINS, ids=lambda p: p.__name__)
def test_mha_oracle_sink_pin(pin):
    pin(lambda q, k, v, sl, scale, sinks: oracle.mha_decode(q, k, v, sl, scale, sinks=sinks))


def _np_mha_sinks(q, k, v, sl, scale, sinks, *, sink_mode="correct"):
    qd, kd, vd = (x.to(torch.float64).numpy() for x in (q, k, v))
    B, Sq, H, D = qd.shape
    Hkv, Dv = kd.shape[2], vd.shape[3]
    out = np.zeros((B, Sq, H, Dv))
    lse = np.zeros((B, Sq, H))
    for b in range(B):
        L = int(sl[b])
        for t in range(Sq):
            for h in range(H):
                hk = h // (H // Hkv)
                sg = -np.inf if sinks is None else float(sinks[0 if sink_mode == "first_head" else h])
                if sink_mode == "scaled":
                    sg *= scale
                if L == 0:
                    lse[b, t, h] = -np.inf if sink_mode == "empty_minus_inf" else sg
                    continue
                s = (kd[b, :L, hk] @ qd[b, t, h]) * scale
                m = s.max() if sink_mode == "not_in_max" else max(s.max(), sg)
                w = np.exp(s - m)
                l = w.sum() + (0.0 if sink_mode == "ignored" else np.exp(sg - m))
                o = w @ vd[b, :L, hk]
                if sink_mode == "carries_first_value":
                    o = o + np.exp(sg - m) * vd[b, 0, hk]
                out[b, t, h] = o / l
                lse[b, t, h] = m + np.log(l)
    return out, lse


MHA_SINK_MUTANTS = {
    "correct": {},
    "sink_ignored": dict(sink_mode="ignored"),
    "sink_multiplied_by_scale": dict(sink_mode="scaled"),
    "sink_left_out_of_max": dict(sink_mode="not_in_max"),
    "sink_carries_a_value": dict(sink_mode="carries_first_value"),
    "first_head_sink_for_all": dict(sink_mode="first_head"),
    "empty_sequence_lse_minus_inf": dict(sink_mode="empty_minus_inf"),
}


@pytest.mark.parametrize("name", sorted(MHA_SINK_MUTANTS))
def test_mha_sink_pins_catch_planted_mistakes(name):
    def impl(q, k, v, sl, scale, sinks):
        return _np_mha_sinks(q, k, v, sl, scale, sinks, **MHA_SINK_MUTANTS[name])
    failed = []
    for pin in pins.MHA_SINK_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    if name == "correct":
        assert failed == [], f"a correct stand-in must pass every MHA sink pin, failed: {failed}"
    else:
        assert failed, f"planted mistake '{name}' passed every MHA sink pin"


# ---------------------------------------------------------------- FP8 latent cache oracle

def _oracle_fp8_attend(q, codes, ks, sl, scale, d_v, sinks):
    return oracle.mla_decode_fp8(q, codes, ks, sl, scale, d_v=d_v, sinks=sinks)


@pytest.mark.parametrize("pin", pins.FP8_PINS, ids=lambda p: p.__name__)
def test_fp8_oracle_pin(pin):
    pin(oracle.e4m3_decode, _oracle_fp8_attend)


def test_fp8_rows_entry_matches_full():
    g = torch.Generator().manual_seed(65)
    q = torch.randn(2, 2, 3, 576, generator=g).to(torch.bfloat16)
    codes = (torch.randn(2, 21, 576, generator=g) * 20).to(torch.float8_e4m3fn).view(torch.uint8)
    sl = np.array([21, 0], np.int32)
    sinks = np.array([0.5, -1.0, 3.0])
    out, lse = oracle.mla_decode_fp8(q, codes, 0.05, sl, pins.SCALE, sinks=sinks)
    rows = np.array([0, 4, 7, 11, 5])
    o2, l2 = oracle.mla_decode_fp8(q, codes, 0.05, sl, pins.SCALE, sinks=sinks, row_ids=rows)
    np.testing.assert_array_equal(o2, out.reshape(-1, 512)[rows])
    np.testing.assert_array_equal(l2, lse.reshape(-1)[rows])


def test_fp8_oracle_is_the_bf16_oracle_on_exact_values():
    """Same operations in the same order on the same doubles: bit-identical."""
    g = torch.Generator().manual_seed(66)
    codes = torch.randint(0, 256, (2, 33, 576), generator=g, dtype=torch.uint8)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0x7E
    q = (torch.randn(2, 1, 4, 576, generator=g) * 0.05).to(torch.bfloat16)
    sl = np.array([33, 9], np.int32)
    ks = 2.0 ** -6
    kv = (codes.view(torch.float8_e4m3fn).to(torch.float64) * ks).to(torch.bfloat16)
    out, lse = oracle.mla_decode_fp8(q, codes, ks, sl, pins.SCALE)
    ro, rl = oracle.mla_decode(q, kv, sl, pins.SCALE)
    np.testing.assert_array_equal(out, ro)
    np.testing.assert_array_equal(lse, rl)


def test_fp8_rejects_non_finite_scale():
    q = torch.zeros(1, 1, 1, 576, dtype=torch.bfloat16)
    codes = np.zeros((1, 4, 576), np.uint8)
    with pytest.raises(ValueError):
        oracle.mla_decode_fp8(q, codes, float("nan"), np.array([4], np.int32), 0.1)


def _np_e4m3(codes, *, bias=7, subnormal_as_normal=False, sign=True, man_bits=3, nan_code=True):
    c = np.asarray(codes, dtype=np.int64)
    s = c >> 7
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    frac = m / (2 ** man_bits)
    if subnormal_as_normal:
        v = (1.0 + frac) * np.exp2(np.maximum(e, 1) - bias)
    else:
        v = np.where(e == 0, frac * 2.0 ** (1 - bias), (1.0 + frac) * np.exp2(e - bias))
    if sign:
        v = np.where(s == 1, -v, v)
    if nan_code:
        v = np.where((e == 15) & (c & 7 == 7), np.nan, v)
    return v


def _np_fp8_attend(q, codes, ks, sl, scale, d_v, sinks, *, dec=None, ks_keys="mul", ks_values="mul"):
    dec = dec or {}
    vals = _np_e4m3(np.asarray(codes), **dec)
    kscale = {"mul": ks, "none": 1.0, "div": 1.0 / ks}
    kd = vals * kscale[ks_keys]
    vd = vals[..., :d_v] * kscale[ks_values]
    qd = q.to(torch.float64).numpy()
    B, Sq, H, _ = qd.shape
    out = np.zeros((B, Sq, H, d_v))
    lse = np.zeros((B, Sq, H))
    for b in range(B):
        L = int(sl[b])
        for t in range(Sq):
            for h in range(H):
                sg = -np.inf if sinks is None else float(sinks[h])
                if L == 0:
                    lse[b, t, h] = sg
                    continue
                s = (kd[b, :L] @ qd[b, t, h]) * scale
                m = max(s.max(), sg)
                w = np.exp(s - m)
                l = w.sum() + np.exp(sg - m)
                out[b, t, h] = (w @ vd[b, :L]) / l
                lse[b, t, h] = m + np.log(l)
    return out, lse


FP8_MUTANTS = {
    "correct": {},
    "exponent_bias_8": dict(dec=dict(bias=8)),
    "subnormals_read_as_normals": dict(dec=dict(subnormal_as_normal=True)),
    "sign_bit_ignored": dict(dec=dict(sign=False)),
    "mantissa_read_as_4_bits": dict(dec=dict(man_bits=4)),
    "nan_code_read_as_finite": dict(dec=dict(nan_code=False)),
    "kv_scale_not_on_keys": dict(ks_keys="none"),
    "kv_scale_not_on_values": dict(ks_values="none"),
    "kv_scale_divides": dict(ks_keys="div", ks_values="div"),
}


@pytest.mark.parametrize("name", sorted(FP8_MUTANTS))
def test_fp8_pins_catch_planted_mistakes(name):
    kw = FP8_MUTANTS[name]

    def decode(codes):
        return _np_e4m3(codes, **kw.get("dec", {}))

    def attend(q, codes, ks, sl, scale, d_v, sinks):
        return _np_fp8_attend(q, codes, ks, sl, scale, d_v, sinks, **kw)

    failed = []
    for pin in pins.FP8_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(decode, attend)
        except AssertionError:
            failed.append(pin.__name__)
    if name == "correct":
        assert failed == [], f"a correct stand-in must pass every FP8 pin, failed: {failed}"
    else:
        assert failed, f"planted mistake '{name}' passed every FP8 pin"
