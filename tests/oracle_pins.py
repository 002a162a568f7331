"""Checks that pin the fp64 oracle to facts other than itself.

Each ``pin_*`` takes an implementation ``impl(q, kv, seqlens, scale, d_v) ->
(out, lse)`` (numpy float64 results) and raises AssertionError when the
implementation disagrees with a closed form, an invariant fixed by the
definition, a high-precision brute force, or an independent library routine.
tests/test_oracle.py runs them on the oracle, and also on deliberately broken
variants to show that each plausible mistake trips at least one pin.
"""
from __future__ import annotations

import math
from decimal import Decimal, getcontext

import numpy as np
import torch

SCALE = float(torch.tensor(576 ** -0.5, dtype=torch.float32).item())


def _rand_bf16(shape, gen, sigma=1.0):
    return (torch.randn(*shape, generator=gen) * sigma).to(torch.bfloat16)


def _f64(x):
    return x.to(torch.float64).numpy()


def pin_single_key(impl):
    """L = 1: the only weight is 1, so out is that key's value row and lse is
    its scaled score."""
    g = torch.Generator().manual_seed(11)
    q = _rand_bf16((2, 1, 4, 576), g)
    kv = _rand_bf16((2, 3, 576), g)
    sl = np.array([1, 1], dtype=np.int32)
    out, lse = impl(q, kv, sl, SCALE, 512)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(out[b, 0, h], _f64(kv[b, 0, :512]))
            s0 = SCALE * float(torch.dot(q[b, 0, h].double(), kv[b, 0].double()))
            assert abs(lse[b, 0, h] - s0) <= 1e-12 * max(1.0, abs(s0))


def pin_identical_keys(impl):
    """L identical rows: uniform weights, out = that row's value, lse = s + ln L."""
    g = torch.Generator().manual_seed(12)
    q = _rand_bf16((1, 1, 3, 576), g)
    row = _rand_bf16((576,), g)
    L = 37
    kv = row.expand(1, L, 576).contiguous()
    out, lse = impl(q, kv, np.array([L], np.int32), SCALE, 512)
    for h in range(3):
        np.testing.assert_allclose(out[0, 0, h], _f64(row[:512]), rtol=0, atol=1e-14)
        s = SCALE * float(torch.dot(q[0, 0, h].double(), row.double()))
        assert abs(lse[0, 0, h] - (s + math.log(L))) <= 1e-12


def pin_zero_query(impl):
    """q = 0: all scores are 0, weights uniform: out = mean of value rows,
    lse = ln L."""
    g = torch.Generator().manual_seed(13)
    q = torch.zeros((2, 1, 2, 576), dtype=torch.bfloat16)
    kv = _rand_bf16((2, 50, 576), g)
    sl = np.array([50, 17], np.int32)
    out, lse = impl(q, kv, sl, SCALE, 512)
    for b, L in enumerate(sl):
        mean = kv[b, :L, :512].double().mean(dim=0).numpy()
        for h in range(2):
            np.testing.assert_allclose(out[b, 0, h], mean, rtol=0, atol=1e-13)
            assert abs(lse[b, 0, h] - math.log(L)) <= 1e-13


def pin_two_keys(impl):
    """Closed form: q = a e_0, k_0 = e_0, k_1 = e_1 (q . k_1 = 0): weights
    sigma(a*scale) and 1 - sigma(a*scale); lse = ln(exp(a*scale) + 1)."""
    a = 6.5  # exactly representable in bf16
    q = torch.zeros((1, 1, 1, 576), dtype=torch.bfloat16)
    q[0, 0, 0, 0] = a
    g = torch.Generator().manual_seed(14)
    kv = _rand_bf16((1, 2, 576), g)
    kv[0, 0, :] = 0
    kv[0, 1, :] = 0
    kv[0, 0, 0] = 1.0
    kv[0, 1, 1] = 1.0
    v0 = torch.zeros(512, dtype=torch.float64)
    v0[0] = 1.0
    v1 = torch.zeros(512, dtype=torch.float64)
    v1[1] = 1.0
    z = a * SCALE
    w0 = 1.0 / (1.0 + math.exp(-z))
    out, lse = impl(q, kv, np.array([2], np.int32), SCALE, 512)
    np.testing.assert_allclose(out[0, 0, 0], (w0 * v0 + (1 - w0) * v1).numpy(), rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - math.log(math.exp(z) + 1.0)) <= 1e-14


def pin_rope_shift(impl):
    """A shared additive score term: setting the last rope column of q to 1 and
    of every key to 2 adds 2*scale to every score, which leaves out unchanged
    and shifts lse by exactly 2*scale (and proves the rope columns count)."""
    g = torch.Generator().manual_seed(15)
    q = _rand_bf16((1, 1, 4, 576), g)
    kv = _rand_bf16((1, 29, 576), g)
    q[..., 575] = 0
    kv[..., 575] = 0
    out0, lse0 = impl(q, kv, np.array([29], np.int32), SCALE, 512)
    q[..., 575] = 1.0
    kv[..., 575] = 2.0
    out1, lse1 = impl(q, kv, np.array([29], np.int32), SCALE, 512)
    np.testing.assert_allclose(out1, out0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse1 - lse0, 2.0 * SCALE, rtol=0, atol=1e-12)


def pin_value_columns(impl):
    """Values are the first 512 columns: with every key equal except for
    columns >= 512, the output must be identical (those columns feed scores
    only), and changing column 0 of one key must move out[..., 0]."""
    g = torch.Generator().manual_seed(16)
    q = torch.zeros((1, 1, 1, 576), dtype=torch.bfloat16)
    kv = _rand_bf16((1, 5, 576), g)
    out, _ = impl(q, kv, np.array([5], np.int32), SCALE, 512)
    mean = kv[0, :5, :512].double().mean(dim=0).numpy()
    np.testing.assert_allclose(out[0, 0, 0], mean, rtol=0, atol=1e-13)
    kv2 = kv.clone()
    kv2[0, :, 512:] = 0  # rope columns never contribute to values
    out2, _ = impl(q, kv2, np.array([5], np.int32), SCALE, 512)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-15)


def pin_permutation(impl):
    """Reordering the keys (with their values) leaves out and lse unchanged."""
    g = torch.Generator().manual_seed(17)
    q = _rand_bf16((1, 2, 3, 576), g)
    kv = _rand_bf16((1, 41, 576), g)
    perm = torch.randperm(41, generator=g)
    out0, lse0 = impl(q, kv, np.array([41], np.int32), SCALE, 512)
    out1, lse1 = impl(q, kv[:, perm].contiguous(), np.array([41], np.int32), SCALE, 512)
    np.testing.assert_allclose(out1, out0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse1, lse0, rtol=0, atol=1e-13)


def pin_independence(impl):
    """Rows do not interact: each (token, head) equals a run on that row alone,
    and each sequence sees only its own cache and length."""
    g = torch.Generator().manual_seed(18)
    q = _rand_bf16((2, 2, 3, 576), g)
    kv = _rand_bf16((2, 23, 576), g)
    sl = np.array([23, 9], np.int32)
    out, lse = impl(q, kv, sl, SCALE, 512)
    for b in range(2):
        for t in range(2):
            for h in range(3):
                o1, l1 = impl(q[b:b + 1, t:t + 1, h:h + 1].contiguous(), kv[b:b + 1].contiguous(),
                              sl[b:b + 1], SCALE, 512)
                np.testing.assert_allclose(o1[0, 0, 0], out[b, t, h], rtol=0, atol=1e-14)
                assert abs(l1[0, 0, 0] - lse[b, t, h]) <= 1e-14


def pin_tail_ignored(impl):
    """Rows at or past a sequence's length are never read (NaN there changes
    nothing), and an empty sequence gives out = 0, lse = -inf."""
    g = torch.Generator().manual_seed(19)
    q = _rand_bf16((3, 1, 2, 576), g)
    kv = _rand_bf16((3, 16, 576), g)
    sl = np.array([16, 5, 0], np.int32)
    out0, lse0 = impl(q, kv, sl, SCALE, 512)
    kv_nan = kv.clone()
    kv_nan[1, 5:] = float("nan")
    kv_nan[2, :] = float("nan")
    out1, lse1 = impl(q, kv_nan, sl, SCALE, 512)
    np.testing.assert_array_equal(out1, out0)
    np.testing.assert_array_equal(lse1, lse0)
    assert np.all(out1[2] == 0.0) and np.all(np.isneginf(lse1[2]))


def _decimal_reference(q, kv, sl, scale, d_v, digits=50):
    getcontext().prec = digits
    qd = q.to(torch.float64).numpy()
    kd = kv.to(torch.float64).numpy()
    B, Sq, H, d = qd.shape
    out = np.zeros((B, Sq, H, d_v))
    lse = np.zeros((B, Sq, H))
    sc = Decimal(scale)
    for b in range(B):
        L = int(sl[b])
        for t in range(Sq):
            for h in range(H):
                s = [sc * sum(Decimal(float(qd[b, t, h, i])) * Decimal(float(kd[b, j, i])) for i in range(d))
                     for j in range(L)]
                m = max(s)
                w = [(x - m).exp() for x in s]
                l = sum(w)
                for e in range(d_v):
                    out[b, t, h, e] = float(sum(w[j] * Decimal(float(kd[b, j, e])) for j in range(L)) / l)
                lse[b, t, h] = float(m + l.ln())
    return out, lse


def pin_brute_force_decimal(impl):
    """50-digit decimal brute force on tiny shapes (d_qk = 6, d_v = 4), with
    generic dimensions, large score spread and ragged lengths."""
    g = torch.Generator().manual_seed(20)
    q = _rand_bf16((2, 2, 2, 6), g, sigma=3.0)
    kv = _rand_bf16((2, 5, 6), g, sigma=3.0)
    sl = np.array([5, 3], np.int32)
    scale = 0.37
    out, lse = impl(q, kv, sl, scale, 4)
    ro, rl = _decimal_reference(q, kv, sl, scale, 4)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-13)


def pin_sdpa_library(impl):
    """torch's fp64 scaled_dot_product_attention (math path) with k = kv rows
    and v = their first 512 columns, and torch.logsumexp of the fp64 scores for
    lse, at the real 576/512 dimensions with ragged lengths and two tokens."""
    g = torch.Generator().manual_seed(21)
    q = _rand_bf16((2, 2, 4, 576), g)
    kv = _rand_bf16((2, 67, 576), g)
    sl = np.array([67, 30], np.int32)
    out, lse = impl(q, kv, sl, SCALE, 512)
    for b in range(2):
        L = int(sl[b])
        qq = q[b].double().reshape(1, -1, 576)           # [1, Sq*H, 576]
        kk = kv[b, :L].double().reshape(1, L, 576)
        vv = kv[b, :L, :512].double().reshape(1, L, 512)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=SCALE)
        np.testing.assert_allclose(out[b].reshape(-1, 512), ref[0].numpy(), rtol=0, atol=1e-12)
        scores = (qq[0] @ kk[0].T) * SCALE
        np.testing.assert_allclose(lse[b].reshape(-1), torch.logsumexp(scores, dim=-1).numpy(),
                                   rtol=0, atol=1e-12)


ALL_PINS = [pin_single_key, pin_identical_keys, pin_zero_query, pin_two_keys, pin_rope_shift,
            pin_value_columns, pin_permutation, pin_independence, pin_tail_ignored,
            pin_brute_force_decimal, pin_sdpa_library]


# ---------------------------------------------------------------- attention sinks
# impl(q, kv, seqlens, scale, d_v, sinks) with sinks a float64 [H] array of
# per-head sink logits (one extra softmax term without a value) or None.

def pin_sink_absent_is_minus_inf(impl):
    """A sink of -inf adds exp(-inf) = 0 to the denominator and cannot be the
    max: the result equals the sink-free one."""
    g = torch.Generator().manual_seed(31)
    q = _rand_bf16((2, 2, 3, 576), g)
    kv = _rand_bf16((2, 40, 576), g)
    sl = np.array([40, 9], np.int32)
    o0, l0 = impl(q, kv, sl, SCALE, 512, None)
    o1, l1 = impl(q, kv, sl, SCALE, 512, np.full(3, -np.inf))
    np.testing.assert_array_equal(o1, o0)
    np.testing.assert_array_equal(l1, l0)


def pin_sink_zero_query(impl):
    """q = 0: every score is 0, so with sink sigma the weights are 1 / (L + e^sigma)
    each: out = mean(V) * L / (L + e^sigma) and lse = ln(L + e^sigma).  The
    sinks span both signs and one far above the scores (e^800 overflows a
    double, so the sink must take part in the max)."""
    g = torch.Generator().manual_seed(32)
    q = torch.zeros((2, 1, 4, 576), dtype=torch.bfloat16)
    kv = _rand_bf16((2, 30, 576), g)
    sl = np.array([30, 7], np.int32)
    sinks = np.array([-3.0, 0.0, 2.5, 800.0])
    out, lse = impl(q, kv, sl, SCALE, 512, sinks)
    for b, L in enumerate(sl):
        mean = kv[b, :L, :512].double().mean(dim=0).numpy()
        for h, sg in enumerate(sinks):
            # ln(L + e^sg) and L / (L + e^sg) written to stay finite for sg = 800
            ref_lse = max(sg, math.log(L)) + math.log1p(math.exp(-abs(sg - math.log(L))))
            frac = math.exp(math.log(L) - ref_lse)
            np.testing.assert_allclose(out[b, 0, h], mean * frac, rtol=1e-12, atol=1e-300)
            assert abs(lse[b, 0, h] - ref_lse) <= 1e-12 * max(1.0, abs(ref_lse))


def pin_sink_is_a_value_free_key(impl):
    """A sink equals one more key whose value is zero: append a row that is 0
    in the 512 value columns and has rope columns r, and set the sink to that
    row's score scale * <q_rope, r> (computed exactly in fp64).  The sink
    result must equal the sink-free result over L + 1 keys.  One query row per
    case (B = Sq = H = 1), so each case's sink is that row's own score."""
    g = torch.Generator().manual_seed(33)
    for case, L in enumerate([1, 5, 64]):
        q = _rand_bf16((1, 1, 1, 576), g)
        kv = _rand_bf16((1, L + 1, 576), g)
        kv[0, L, :512] = 0
        kv[0, L, 512:] = _rand_bf16((64,), g, sigma=4.0 + case)
        sigma = SCALE * float(torch.dot(q[0, 0, 0, 512:].double(), kv[0, L, 512:].double()))
        o_s, l_s = impl(q, kv, np.array([L], np.int32), SCALE, 512, np.array([sigma]))
        o_k, l_k = impl(q, kv, np.array([L + 1], np.int32), SCALE, 512, None)
        np.testing.assert_allclose(o_s, o_k, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l_s, l_k, rtol=0, atol=1e-12)


def pin_sink_empty_sequence(impl):
    """L = 0: nothing to attend to; out = 0 and the log-sum-exp is the sink
    alone."""
    g = torch.Generator().manual_seed(34)
    q = _rand_bf16((2, 1, 2, 576), g)
    kv = _rand_bf16((2, 8, 576), g)
    sl = np.array([0, 8], np.int32)
    sinks = np.array([1.25, -7.0])
    out, lse = impl(q, kv, sl, SCALE, 512, sinks)
    np.testing.assert_array_equal(out[0], 0.0)
    np.testing.assert_array_equal(lse[0, 0], sinks)


SINK_PINS = [pin_sink_absent_is_minus_inf, pin_sink_zero_query, pin_sink_is_a_value_free_key,
             pin_sink_empty_sequence]


# ---------------------------------------------------------------- MHA decode
# impl(q, k, v, seqlens, scale) with q [B,Sq,H,D], k [B,L,Hkv,D], v [B,L,Hkv,Dv].

def pin_mha_mqa_equals_latent_definition(impl):
    """One kv head shared by all query heads, with v = the first Dv columns of
    k, is exactly the latent-cache definition (keys are kv rows, values their
    first Dv columns): compare with the MLA oracle's generic entry point."""
    import oracle
    g = torch.Generator().manual_seed(41)
    q = _rand_bf16((2, 2, 4, 96), g)
    k = _rand_bf16((2, 23, 1, 96), g)
    v = k[..., :64].contiguous()
    sl = np.array([23, 9], np.int32)
    out, lse = impl(q, k, v, sl, 0.1)
    ro, rl = oracle.mla_decode(q, k[:, :, 0, :].contiguous(), sl, 0.1, d_v=64)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-13)


def pin_mha_sdpa_library(impl):
    """torch's fp64 scaled_dot_product_attention with the kv heads repeated
    over their query-head groups (GQA), and torch.logsumexp, at D = Dv = 128
    with ragged lengths and two tokens."""
    g = torch.Generator().manual_seed(42)
    B, Sq, H, Hkv, L, D = 2, 2, 8, 2, 41, 128
    q = _rand_bf16((B, Sq, H, D), g)
    k = _rand_bf16((B, L, Hkv, D), g)
    v = _rand_bf16((B, L, Hkv, D), g)
    sl = np.array([41, 13], np.int32)
    scale = D ** -0.5
    out, lse = impl(q, k, v, sl, scale)
    for b in range(B):
        Lb = int(sl[b])
        qq = q[b].double().permute(1, 0, 2)                                 # [H, Sq, D]
        kk = k[b, :Lb].double().permute(1, 0, 2).repeat_interleave(H // Hkv, dim=0)  # [H, L, D]
        vv = v[b, :Lb].double().permute(1, 0, 2).repeat_interleave(H // Hkv, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)  # [H, Sq, D]
        np.testing.assert_allclose(out[b], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
        sc = torch.einsum("hsd,hld->hsl", qq, kk) * scale
        np.testing.assert_allclose(lse[b], torch.logsumexp(sc, dim=-1).permute(1, 0).numpy(), rtol=0, atol=1e-12)


def pin_mha_head_groups(impl):
    """Head h reads kv head h // (H / Hkv): with every value of kv head hk equal
    to hk + 1, head h's output is exactly h // (H / Hkv) + 1 (the weights sum
    to one), whatever the scores."""
    g = torch.Generator().manual_seed(43)
    B, H, Hkv, L, D = 1, 12, 3, 17, 64
    q = _rand_bf16((B, 1, H, D), g, sigma=2.0)
    k = _rand_bf16((B, L, Hkv, D), g, sigma=2.0)
    v = torch.empty((B, L, Hkv, 32), dtype=torch.bfloat16)
    for hk in range(Hkv):
        v[:, :, hk, :] = hk + 1
    out, _ = impl(q, k, v, np.array([L], np.int32), 0.2)
    for h in range(H):
        np.testing.assert_allclose(out[0, 0, h], h // (H // Hkv) + 1, rtol=1e-14, atol=0)


def pin_mha_single_key(impl):
    """L = 1: out is that key's value row of the head's kv head; lse its score."""
    g = torch.Generator().manual_seed(44)
    q = _rand_bf16((1, 1, 4, 128), g)
    k = _rand_bf16((1, 3, 2, 128), g)
    v = _rand_bf16((1, 3, 2, 128), g)
    out, lse = impl(q, k, v, np.array([1], np.int32), 0.09)
    for h in range(4):
        hk = h // 2
        np.testing.assert_array_equal(out[0, 0, h], _f64(v[0, 0, hk]))
        s0 = 0.09 * float(torch.dot(q[0, 0, h].double(), k[0, 0, hk].double()))
        assert abs(lse[0, 0, h] - s0) <= 1e-12 * max(1.0, abs(s0))


MHA_PINS = [pin_mha_mqa_equals_latent_definition, pin_mha_sdpa_library, pin_mha_head_groups, pin_mha_single_key]


# ---------------------------------------------------------------- MHA decode with attention sinks
# impl(q, k, v, seqlens, scale, sinks) with sinks a float64 [H] array or None.

def pin_mha_sink_absent_is_minus_inf(impl):
    """A sink of -inf changes nothing: the result equals the sink-free one,
    bit for bit."""
    g = torch.Generator().manual_seed(71)
    q = _rand_bf16((2, 2, 4, 64), g)
    k = _rand_bf16((2, 19, 2, 64), g)
    v = _rand_bf16((2, 19, 2, 48), g)
    sl = np.array([19, 6], np.int32)
    o0, l0 = impl(q, k, v, sl, 0.125, None)
    o1, l1 = impl(q, k, v, sl, 0.125, np.full(4, -np.inf))
    np.testing.assert_array_equal(o1, o0)
    np.testing.assert_array_equal(l1, l0)


def pin_mha_sink_is_a_value_free_key(impl):
    """A sink equals one more key, in the head's own kv head, whose value row
    is zero and whose score is the sink: append key L with k = (a, 0, ..., 0)
    and v = 0, one query head per kv head (so each kv head's extra key serves
    exactly one head), and set sink_h = scale * q_h[0] * a exactly.  The
    sink result over L keys must equal the sink-free result over L + 1."""
    g = torch.Generator().manual_seed(72)
    for L in (1, 4, 33):
        Hkv = 3
        q = _rand_bf16((1, 1, Hkv, 32), g)
        k = _rand_bf16((1, L + 1, Hkv, 32), g)
        v = _rand_bf16((1, L + 1, Hkv, 16), g)
        k[0, L] = 0
        v[0, L] = 0
        a = torch.tensor([1.5, -2.0, 3.25], dtype=torch.bfloat16)
        k[0, L, :, 0] = a
        scale = 0.25
        sinks = np.array([scale * float(q[0, 0, h, 0]) * float(a[h]) for h in range(Hkv)])
        o_s, l_s = impl(q, k, v, np.array([L], np.int32), scale, sinks)
        o_k, l_k = impl(q, k, v, np.array([L + 1], np.int32), scale, None)
        np.testing.assert_allclose(o_s, o_k, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l_s, l_k, rtol=0, atol=1e-12)


def pin_mha_sink_zero_query(impl):
    """q = 0: all scores are 0, so the weights are 1 / (L + e^sigma): out =
    mean of the kv head's values * L / (L + e^sigma), lse = ln(L + e^sigma),
    with a sink far above the scores (e^800 overflows a double, so the sink
    must take part in the max)."""
    g = torch.Generator().manual_seed(73)
    H, Hkv, L = 4, 2, 11
    q = torch.zeros((1, 1, H, 32), dtype=torch.bfloat16)
    k = _rand_bf16((1, L, Hkv, 32), g)
    v = _rand_bf16((1, L, Hkv, 24), g)
    sinks = np.array([-2.0, 0.5, 3.0, 800.0])
    out, lse = impl(q, k, v, np.array([L], np.int32), 0.3, sinks)
    for h, sg in enumerate(sinks):
        mean = v[0, :, h // 2].double().mean(dim=0).numpy()
        ref_lse = max(sg, math.log(L)) + math.log1p(math.exp(-abs(sg - math.log(L))))
        np.testing.assert_allclose(out[0, 0, h], mean * math.exp(math.log(L) - ref_lse), rtol=1e-12, atol=1e-300)
        assert abs(lse[0, 0, h] - ref_lse) <= 1e-12 * max(1.0, abs(ref_lse))


def pin_mha_sink_empty_sequence(impl):
    """L = 0: out = 0 and the log-sum-exp is the head's sink alone."""
    g = torch.Generator().manual_seed(74)
    q = _rand_bf16((2, 1, 2, 32), g)
    k = _rand_bf16((2, 5, 1, 32), g)
    v = _rand_bf16((2, 5, 1, 32), g)
    sinks = np.array([0.75, -4.0])
    out, lse = impl(q, k, v, np.array([0, 5], np.int32), 0.2, sinks)
    np.testing.assert_array_equal(out[0], 0.0)
    np.testing.assert_array_equal(lse[0, 0], sinks)


MHA_SINK_PINS = [pin_mha_sink_absent_is_minus_inf, pin_mha_sink_is_a_value_free_key, pin_mha_sink_zero_query,
                 pin_mha_sink_empty_sequence]


# ---------------------------------------------------------------- FP8 latent cache
# FP8 pins take (decode, attend): decode(codes uint8 array) -> float64 values
# of the E4M3 codes; attend(q, codes, kv_scale, seqlens, scale, d_v, sinks)
# -> (out, lse) for a cache of codes whose values are kv_scale * e4m3(code).

def _codes_from_normal(shape, gen, sigma, kv_scale):
    """Random E4M3 codes of N(0, sigma) values quantised with kv_scale (torch's
    own rounding; this only makes inputs)."""
    x = torch.randn(*shape, generator=gen, dtype=torch.float64) * sigma / kv_scale
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def _torch_e4m3_values(codes):
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


def pin_fp8_decode_library(decode, attend):
    """All 256 codes against torch's float8_e4m3fn -> float64 conversion (an
    independent library routine); the two NaN codes must decode to NaN."""
    codes = np.arange(256, dtype=np.uint8)
    got = decode(codes)
    ref = _torch_e4m3_values(torch.from_numpy(codes)).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])
    np.testing.assert_array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))


def pin_fp8_decode_closed_forms(decode, attend):
    """Values fixed by the format: 1 sign, 4 exponent bits (bias 7), 3 mantissa
    bits, subnormals (m/8) 2^-6 at exponent field 0, S.1111.111 = NaN."""
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
             0x38: 1.0, 0x3F: 1.875, 0x40: 2.0, 0x77: 240.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0,
             0xFE: -448.0, 0x81: -(2.0 ** -9)}
    got = decode(np.array(sorted(table), dtype=np.uint8))
    for v, (c, want) in zip(got, sorted(table.items())):
        assert v == want and math.copysign(1.0, v) == math.copysign(1.0, want), (hex(c), v, want)
    assert np.isnan(decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def pin_fp8_sdpa_library(decode, attend):
    """torch's fp64 scaled_dot_product_attention over the dequantised cache
    (kv_scale * torch's own E4M3 values; keys all 576 columns, values the
    first 512) and torch.logsumexp, with a scale that is not a power of two,
    ragged lengths and two tokens."""
    g = torch.Generator().manual_seed(61)
    ks = 0.0123
    q = _rand_bf16((2, 2, 4, 576), g)
    codes = _codes_from_normal((2, 53, 576), g, 1.0, ks)
    sl = np.array([53, 19], np.int32)
    out, lse = attend(q, codes, ks, sl, SCALE, 512, None)
    kvd = _torch_e4m3_values(codes) * ks
    for b in range(2):
        L = int(sl[b])
        qq = q[b].double().reshape(1, -1, 576)
        kk = kvd[b, :L].reshape(1, L, 576)
        vv = kvd[b, :L, :512].reshape(1, L, 512)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=SCALE)
        np.testing.assert_allclose(out[b].reshape(-1, 512), ref[0].numpy(), rtol=0, atol=1e-12)
        sc = (qq[0] @ kk[0].T) * SCALE
        np.testing.assert_allclose(lse[b].reshape(-1), torch.logsumexp(sc, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_fp8_single_key(decode, attend):
    """L = 1: out is the key's dequantised value row (kv_scale * e4m3), exactly;
    lse is its scaled score."""
    g = torch.Generator().manual_seed(62)
    ks = 0.037
    q = _rand_bf16((1, 1, 3, 576), g)
    codes = _codes_from_normal((1, 2, 576), g, 1.0, ks)
    out, lse = attend(q, codes, ks, np.array([1], np.int32), SCALE, 512, None)
    vals = _torch_e4m3_values(codes[0, 0]) * ks
    for h in range(3):
        np.testing.assert_array_equal(out[0, 0, h], vals[:512].numpy())
        s0 = SCALE * float(torch.dot(q[0, 0, h].double(), vals))
        assert abs(lse[0, 0, h] - s0) <= 1e-12 * max(1.0, abs(s0))


def pin_fp8_scale_trade(decode, attend):
    """Doubling kv_scale while halving the softmax scale leaves every score,
    hence the weights and lse, unchanged and doubles every value: out doubles."""
    g = torch.Generator().manual_seed(63)
    ks = 0.02
    q = _rand_bf16((2, 1, 3, 576), g)
    codes = _codes_from_normal((2, 31, 576), g, 1.0, ks)
    sl = np.array([31, 8], np.int32)
    o1, l1 = attend(q, codes, ks, sl, 0.08, 512, None)
    o2, l2 = attend(q, codes, 2 * ks, sl, 0.04, 512, None)
    np.testing.assert_allclose(o2, 2 * o1, rtol=1e-13, atol=0)
    np.testing.assert_allclose(l2, l1, rtol=1e-13, atol=1e-13)


def pin_fp8_all_codes_equal_bf16_cache(decode, attend):
    """Every finite code, with a power-of-two kv_scale (2^-7), gives values that
    bf16 holds exactly, so the FP8 definition must reproduce the (separately
    pinned) bf16-cache oracle on that bf16 cache -- sinks, an empty sequence
    and a ragged length included -- up to summation order (the oracle itself
    matches bit for bit: tests/test_oracle.py)."""
    import oracle  # the bf16 definition, pinned by ALL_PINS and SINK_PINS
    g = torch.Generator().manual_seed(64)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    B, L = 3, 40
    codes = np.empty((B, L, 576), dtype=np.uint8)
    rng = np.random.default_rng(64)
    for b in range(B):
        for j in range(L):
            codes[b, j] = rng.choice(finite, size=576)
    ks = 2.0 ** -7
    q = _rand_bf16((B, 2, 2, 576), g, sigma=0.05)
    sl = np.array([40, 0, 23], np.int32)
    sinks = np.array([0.3, -2.0])
    codes_t = torch.from_numpy(codes)
    kv_bf16 = (_torch_e4m3_values(codes_t) * ks).to(torch.bfloat16)
    assert torch.equal(kv_bf16.double(), _torch_e4m3_values(codes_t) * ks)  # exact in bf16
    out, lse = attend(q, codes_t, ks, sl, SCALE, 512, sinks)
    ro, rl = oracle.mla_decode(q, kv_bf16, sl, SCALE, sinks=sinks)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-13)


FP8_PINS = [pin_fp8_decode_library, pin_fp8_decode_closed_forms, pin_fp8_sdpa_library, pin_fp8_single_key,
            pin_fp8_scale_trade, pin_fp8_all_codes_equal_bf16_cache]
