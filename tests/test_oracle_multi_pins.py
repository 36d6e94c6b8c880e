"""Pins for the oracle's multi-token decode (q_len new tokens per sequence, causal among
them).  New token j of a sequence with ctx cached tokens sits at position ctx-q_len+j and
attends to positions 0..ctx-q_len+j.  Each test checks the oracle against something
other than itself: 50-digit brute force, torch SDPA with an explicit causal mask, a
closed form.  CPU only."""
from __future__ import annotations

import mpmath
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_348_b200 import inputs
from tests.helpers import bits, bits_to_f64, make_case


def _multi_q(case, q_len, seed):
    return bits(inputs.randn((case["B"], q_len, case["Hq"], case["D"]), case["dtype"], seed,
                             stream=11))


def _mp_causal(case, q, s, j, h):
    """Brute force with 50 digits, written independently of the oracle: positions are
    enumerated from the block table and the causal limit is stated as a position test."""
    mpmath.mp.dps = 50
    q_len = q.shape[1]
    g = case["Hq"] // case["Hkv"]
    kvh = h // g
    ctx, bs, D = int(case["ctx"][s]), case["bs"], case["D"]
    pos_j = ctx - q_len + j                         # position of new token j
    keep = [t for t in range(ctx) if t <= pos_j]
    if not keep:
        return [0.0] * D
    qf = bits_to_f64(q[s, j, h], case["dtype"])
    rows = [(int(case["tables"][s, t // bs]), t % bs) for t in keep]
    kf = [bits_to_f64(case["k"][b, kvh, o], case["dtype"]) for b, o in rows]
    vf = [bits_to_f64(case["v"][b, kvh, o], case["dtype"]) for b, o in rows]
    sc = mpmath.mpf(case["scale"])
    w = [mpmath.exp(sc * mpmath.fsum(mpmath.mpf(qf[d]) * mpmath.mpf(k[d]) for d in range(D)))
         for k in kf]
    den = mpmath.fsum(w)
    return [float(mpmath.fsum(w[i] * mpmath.mpf(vf[i][d]) for i in range(len(keep))) / den)
            for d in range(D)]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_multi_brute_force_tiny(dtype):
    ctx = [1, 2, 3, 6, 9]
    case = make_case(len(ctx), 4, 2, 8, 2, ctx, dtype=dtype, seed=13)
    q_len = 3
    q = _multi_q(case, q_len, 13)
    out64, _ = oracle.decode_multi(q, case["k"], case["v"], case["tables"], case["ctx"],
                                   case["scale"], dtype)
    for s in range(len(ctx)):
        for j in range(q_len):
            for h in range(4):
                np.testing.assert_allclose(out64[s, j, h], _mp_causal(case, q, s, j, h),
                                           rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("q_len", [1, 2, 5])
def test_multi_contiguous_equals_sdpa_with_causal_mask(q_len):
    Hq, Hkv, D, bs = 8, 2, 16, 4
    ctx = [5, 8, 13, 24]
    case = make_case(len(ctx), Hq, Hkv, D, bs, ctx, dtype="f16", seed=17, shuffle=False,
                     poison=False)
    q = _multi_q(case, q_len, 17)
    out64, _ = oracle.decode_multi(q, case["k"], case["v"], case["tables"], case["ctx"],
                                   case["scale"], "f16")
    k = torch.from_numpy(bits_to_f64(case["k"], "f16"))
    v = torch.from_numpy(bits_to_f64(case["v"], "f16"))
    qf = torch.from_numpy(bits_to_f64(q, "f16"))
    start = 0
    for s, c in enumerate(ctx):
        nb = -(-c // bs)
        Ks = k[start:start + nb].permute(1, 0, 2, 3).reshape(Hkv, nb * bs, D)[:, :c]
        Vs = v[start:start + nb].permute(1, 0, 2, 3).reshape(Hkv, nb * bs, D)[:, :c]
        Ks = Ks.repeat_interleave(Hq // Hkv, dim=0)
        Vs = Vs.repeat_interleave(Hq // Hkv, dim=0)
        # query row j may see key t iff t <= c - q_len + j (bottom-right aligned causal mask)
        mask = torch.arange(c)[None, :] <= (c - q_len + torch.arange(q_len))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qf[s].permute(1, 0, 2), Ks, Vs, attn_mask=mask, scale=case["scale"])  # [Hq,q_len,D]
        np.testing.assert_allclose(out64[s], ref.permute(1, 0, 2).numpy(), rtol=1e-12,
                                   atol=1e-13)
        start += nb


def test_multi_identical_keys_give_mean_of_visible_values():
    q_len, bs = 4, 4
    ctx = [6, 11]
    case = make_case(2, 4, 2, 16, bs, ctx, seed=19, poison=False)
    k = case["k"]
    for s in range(2):
        for t in range(ctx[s]):
            k[case["tables"][s, t // bs], :, t % bs] = k[case["tables"][s, 0], :, 0]
    q = _multi_q(case, q_len, 19)
    out64, _ = oracle.decode_multi(q, k, case["v"], case["tables"], case["ctx"], case["scale"],
                                   "f16")
    for s in range(2):
        for j in range(q_len):
            n = ctx[s] - q_len + 1 + j
            for h in range(4):
                rows = [bits_to_f64(case["v"][case["tables"][s, t // bs], h // 2, t % bs], "f16")
                        for t in range(n)]
                np.testing.assert_allclose(out64[s, j, h], np.mean(rows, axis=0), rtol=1e-14,
                                           atol=1e-15)


def test_multi_tokens_before_the_context_are_zero_and_q_len_1_is_decode():
    # ctx < q_len: new tokens at negative positions see nothing -> zero rows
    case = make_case(3, 4, 4, 8, 4, [2, 0, 7], seed=23)
    q = _multi_q(case, 4, 23)
    out64, out16 = oracle.decode_multi(q, case["k"], case["v"], case["tables"], case["ctx"],
                                       case["scale"], "f16")
    assert not out64[0, :2].any() and out64[0, 2:].any()
    assert not out64[1].any() and not out16[1].any()
    # q_len 1 reads the same rows as single-token decode
    one, _ = oracle.decode_multi(q[:, 3:], case["k"], case["v"], case["tables"], case["ctx"],
                                 case["scale"], "f16")
    ref, _ = oracle.decode(q[:, 3], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], "f16")
    assert np.array_equal(one[:, 0], ref)
