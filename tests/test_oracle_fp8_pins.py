"""Pins for the oracle's 8-bit E4M3 KV cache: the code table and the rounding against
torch's own float8_e4m3fn type, the saturation rule, the binary32 quantisation step,
and decode over E4M3 pools against the pinned 16-bit decode and a 50-digit brute force.
CPU only."""
from __future__ import annotations

import mpmath
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import bits, bits_to_f64, make_case


def test_e4m3_code_table_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref)) and np.isnan(got).sum() == 2
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.5, 20000),
        np.linspace(-463.9, 463.9, 4001),
        np.arange(-512, 513) * 2.0 ** -10,                 # exact subnormal midpoints
    ]).astype(np.float32)
    x = x[np.abs(x) < 464]             # torch turns larger magnitudes into NaN, not 448
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f64_to_e4m3(float(v)) for v in x], dtype=np.uint8)
    assert len(x) > 24000 and np.array_equal(got, ref)


def test_e4m3_ties_to_even_between_every_pair_of_codes():
    vals = [(c, oracle.e4m3_to_f64(c)) for c in range(0x7F)]        # 0 .. 448, ascending
    for (ca, va), (cb, vb) in zip(vals, vals[1:]):
        mid = (va + vb) / 2
        assert oracle.f64_to_e4m3(mid) == (ca if ca % 2 == 0 else cb)
        assert oracle.f64_to_e4m3(np.nextafter(mid, 0)) == ca
        assert oracle.f64_to_e4m3(np.nextafter(mid, np.inf)) == cb
        assert oracle.f64_to_e4m3(-va) == (0x80 | ca)


def test_e4m3_saturates_instead_of_overflowing():
    for x, code in [(448.0, 0x7E), (463.9, 0x7E), (464.0, 0x7E), (470.0, 0x7E), (1e30, 0x7E),
                    (-1e30, 0xFE), (float("inf"), 0x7E)]:
        assert oracle.f64_to_e4m3(x) == code, x
    assert oracle.f64_to_e4m3(float("nan")) & 0x7F == 0x7F


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_quantise_divides_in_binary32(dtype):
    rng = np.random.default_rng(1)
    x16 = (rng.standard_normal(3000) * 3).astype(np.float16)
    if dtype == "bf16":
        b = (x16.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    else:
        b = x16.view(np.uint16)
    for scale in (0.0137, 0.5, 1.0 / 3.0):
        xf = bits_to_f64(b, dtype).astype(np.float32)
        q = (xf / np.float32(scale)).astype(np.float32)
        ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sat = np.abs(q) >= 464
        ref[sat] = np.where(np.signbit(q[sat]), 0xFE, 0x7E)
        got = np.array([oracle.quantize_e4m3(int(v), dtype, scale) for v in b], dtype=np.uint8)
        assert np.array_equal(got, ref), scale


def _e4m3_case(seed, ctx, Hq=8, Hkv=2, D=16, bs=4, dtype="f16"):
    case = make_case(len(ctx), Hq, Hkv, D, bs, ctx, dtype=dtype, seed=seed, poison=False)
    rng = np.random.default_rng(seed)
    case["k8"] = rng.integers(0, 256, size=case["k"].shape).astype(np.uint8)
    case["v8"] = rng.integers(0, 256, size=case["v"].shape).astype(np.uint8)
    for a in (case["k8"], case["v8"]):
        a[(a & 0x7F) == 0x7F] ^= 0x01                        # no NaN codes
    return case


def test_e4m3_decode_equals_16bit_decode_of_the_dequantised_values():
    # power-of-two scales keep scale * code exact in fp16, so the pinned 16-bit decode
    # of those values must give the same fp64 bits
    case = _e4m3_case(2, [1, 7, 13, 30])
    ks, vs = 0.25, 2.0
    deq = lambda a, sc: np.vectorize(lambda c: sc * oracle.e4m3_to_f64(int(c)))(a)
    k16 = deq(case["k8"], ks).astype(np.float16).view(np.uint16)
    v16 = deq(case["v8"], vs).astype(np.float16).view(np.uint16)
    assert np.array_equal(bits_to_f64(k16, "f16"), deq(case["k8"], ks))     # exact
    a, _ = oracle.decode_e4m3(case["q"], case["k8"], case["v8"], ks, vs, case["tables"],
                              case["ctx"], case["scale"], "f16")
    b, _ = oracle.decode(case["q"], k16, v16, case["tables"], case["ctx"], case["scale"], "f16")
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64))


def test_e4m3_decode_brute_force():
    case = _e4m3_case(3, [2, 5, 9], Hq=4, Hkv=2, D=8, bs=2, dtype="bf16")
    ks, vs = 0.0311, 0.173
    out, _ = oracle.decode_e4m3(case["q"], case["k8"], case["v8"], ks, vs, case["tables"],
                                case["ctx"], case["scale"], "bf16")
    mpmath.mp.dps = 50
    for s in range(3):
        for h in range(4):
            kvh = h // 2
            qf = bits_to_f64(case["q"][s, h], "bf16")
            rows = [(int(case["tables"][s, t // 2]), t % 2) for t in range(int(case["ctx"][s]))]
            kf = [[mpmath.mpf(ks) * mpmath.mpf(oracle.e4m3_to_f64(int(c)))
                   for c in case["k8"][b, kvh, o]] for b, o in rows]
            vf = [[mpmath.mpf(vs) * mpmath.mpf(oracle.e4m3_to_f64(int(c)))
                   for c in case["v8"][b, kvh, o]] for b, o in rows]
            w = [mpmath.exp(mpmath.mpf(case["scale"]) * mpmath.fsum(mpmath.mpf(qf[d]) * k[d]
                                                                    for d in range(8)))
                 for k in kf]
            ref = [float(mpmath.fsum(w[t] * vf[t][d] for t in range(len(w))) / mpmath.fsum(w))
                   for d in range(8)]
            np.testing.assert_allclose(out[s, h], ref, rtol=1e-12, atol=1e-14)


def test_e4m3_append_writes_the_quantised_codes_and_nothing_else():
    N, Hkv, bs, D, T = 12, 2, 4, 16, 9
    rng = np.random.default_rng(4)
    k8 = rng.integers(0, 256, size=(N, Hkv, bs, D)).astype(np.uint8)
    v8 = k8.copy()
    before_k, before_v = k8.copy(), v8.copy()
    k = bits(torch.from_numpy((rng.standard_normal((T, Hkv, D)) * 4).astype(np.float32)).to(
        torch.bfloat16))
    v = bits(torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).to(
        torch.bfloat16))
    slots = rng.choice(N * bs, size=T, replace=False).astype(np.int64)
    slots[4] = -1
    oracle.cache_append_e4m3(k8, v8, k, v, slots, "bf16", 0.05, 0.02)
    touched = np.zeros((N, bs), dtype=bool)
    for i, sl in enumerate(slots):
        if sl < 0:
            continue
        b, o = divmod(int(sl), bs)
        touched[b, o] = True
        for h in range(Hkv):
            assert [int(c) for c in k8[b, h, o]] == [oracle.quantize_e4m3(int(x), "bf16", 0.05)
                                                     for x in k[i, h]]
            assert [int(c) for c in v8[b, h, o]] == [oracle.quantize_e4m3(int(x), "bf16", 0.02)
                                                     for x in v[i, h]]
    mask = ~touched
    assert np.array_equal(k8.transpose(0, 2, 1, 3)[mask], before_k.transpose(0, 2, 1, 3)[mask])
    assert np.array_equal(v8.transpose(0, 2, 1, 3)[mask], before_v.transpose(0, 2, 1, 3)[mask])


# ---- per-(block, kv head) scales: the scale a block's offset-0 token fixes is the power
# of two s with s/16 < amax/448 <= s/8 (amax/448 in binary32), 1 for an all-zero row.

def _is_pow2(x: float) -> bool:
    m, _ = np.frexp(x)
    return x > 0 and m == 0.5


def test_block_scale_closed_forms_and_boundaries():
    assert oracle.e4m3_block_scale(448.0) == 8.0                  # amax/448 = 1 = 2^0
    assert oracle.e4m3_block_scale(14.0) == 0.25                  # 2^-5 exactly
    nxt = float(np.nextafter(np.float32(14.0), np.float32(20.0)))
    assert oracle.e4m3_block_scale(nxt) == 0.5                    # just above: next power
    assert oracle.e4m3_block_scale(0.0) == 1.0
    assert oracle.e4m3_block_scale(448.0 * 2.0 ** -20) == 2.0 ** -17


def test_block_scale_brackets_the_row_for_any_amax():
    rng = np.random.default_rng(7)
    amax = np.concatenate([10.0 ** rng.uniform(-30, 4, 4000),
                           np.float32(448.0) * 2.0 ** rng.integers(-40, 8, 200)]).astype(np.float32)
    for a in amax:
        s = oracle.e4m3_block_scale(float(a))
        y = float(np.float32(a) / np.float32(448.0))
        assert _is_pow2(s) and s / 16 < y <= s / 8, (a, s)


def _bs_case(dtype, seed, N=12, Hkv=2, bs=4, D=32):
    rng = np.random.default_rng(seed)
    k8 = rng.integers(0, 256, size=(N, Hkv, bs, D), dtype=np.uint8)
    v8 = rng.integers(0, 256, size=(N, Hkv, bs, D), dtype=np.uint8)
    ks = np.full((N, Hkv), 3.0, np.float32)
    vs = np.full((N, Hkv), 5.0, np.float32)
    return k8, v8, ks, vs


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_block_scaled_append_fixes_scales_at_offset_zero_in_any_order(dtype):
    N, Hkv, bs, D = 12, 2, 4, 32
    k8, v8, ks, vs = _bs_case(dtype, 1)
    rng = np.random.default_rng(2)
    T = 5
    k = bits(torch.from_numpy(rng.standard_normal((T, Hkv, D)) * 3).to(
        torch.float16 if dtype == "f16" else torch.bfloat16))
    v = bits(torch.from_numpy(rng.standard_normal((T, Hkv, D)) * 0.01).to(
        torch.float16 if dtype == "f16" else torch.bfloat16))
    # block 7 gets offsets 3 then 0 (the offset-0 token comes later in the batch), block 2
    # gets offset 1 only (keeps its scale), one padding token
    slots = np.array([7 * bs + 3, 2 * bs + 1, -1, 7 * bs + 0, 9 * bs + 0], np.int64)
    k8b, v8b, ksb, vsb = k8.copy(), v8.copy(), ks.copy(), vs.copy()
    oracle.cache_append_e4m3_bs(k8b, v8b, ksb, vsb, k, v, slots, dtype)
    kf, vf = bits_to_f64(k, dtype), bits_to_f64(v, dtype)
    for blk, tok in ((7, 3), (9, 4)):
        for h in range(Hkv):
            for x, scl in ((kf[tok, h], ksb[blk, h]), (vf[tok, h], vsb[blk, h])):
                y = float(np.float32(np.abs(x).max()) / np.float32(448.0))
                assert _is_pow2(float(scl)) and scl / 16 < y <= scl / 8
    assert ksb[2].tolist() == [3.0, 3.0] and vsb[2].tolist() == [5.0, 5.0]
    changed = {7, 9}
    assert all(ksb[b].tolist() == ks[b].tolist() for b in range(N) if b not in changed)
    # every written code is the pinned quantiser's code with its block's scale
    for i, sl in enumerate(slots):
        if sl < 0:
            continue
        b, o = divmod(int(sl), bs)
        for h in range(Hkv):
            for d in range(D):
                assert k8b[b, h, o, d] == oracle.quantize_e4m3(k[i, h, d], dtype, ksb[b, h])
                assert v8b[b, h, o, d] == oracle.quantize_e4m3(v[i, h, d], dtype, vsb[b, h])
    # nothing else in the pools changed
    mask = np.zeros((N, Hkv, bs), bool)
    for sl in slots:
        if sl >= 0:
            mask[int(sl) // bs, :, int(sl) % bs] = True
    assert np.array_equal(k8b[~mask], k8[~mask]) and np.array_equal(v8b[~mask], v8[~mask])
    # the first row of a block: its largest value maps into (28, 56] of the code range
    top = max(abs(oracle.e4m3_to_f64(c)) for c in k8b[9, 0, 0])
    assert 28 <= top <= 56


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_block_scaled_decode_equals_16bit_decode_of_the_dequantised_pools(dtype):
    # power-of-two scales keep scale * code exact in fp16 / bf16 at these magnitudes, so
    # the 8-bit decode must give exactly the pinned 16-bit decode of the dequantised rows
    case = make_case(4, 8, 2, 64, 8, [5, 16, 17, 40], dtype=dtype, seed=31, poison=False)
    rng = np.random.default_rng(3)
    N, Hkv, bs, D = case["k"].shape
    k8 = rng.integers(0, 0x78, size=(N, Hkv, bs, D), dtype=np.uint8) | \
        (rng.integers(0, 2, size=(N, Hkv, bs, D), dtype=np.uint8) << 7)
    v8 = rng.integers(0, 0x78, size=(N, Hkv, bs, D), dtype=np.uint8)
    ks = (2.0 ** rng.integers(-6, 1, size=(N, Hkv))).astype(np.float32)
    vs = (2.0 ** rng.integers(-6, 1, size=(N, Hkv))).astype(np.float32)
    deq = lambda c8, sc: np.vectorize(oracle.e4m3_to_f64)(c8) * sc[:, :, None, None]
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    k16 = bits(torch.from_numpy(deq(k8, ks)).to(tdt))
    v16 = bits(torch.from_numpy(deq(v8, vs)).to(tdt))
    assert np.array_equal(bits_to_f64(k16, dtype), deq(k8, ks))      # exact in 16 bits
    a, _ = oracle.decode_e4m3_bs(case["q"], k8, v8, ks, vs, case["tables"], case["ctx"],
                                 case["scale"], dtype)
    b, _ = oracle.decode(case["q"], k16, v16, case["tables"], case["ctx"], case["scale"], dtype)
    assert np.array_equal(a, b)
    # equal block scales everywhere: exactly the per-tensor-scale decode
    c, _ = oracle.decode_e4m3_bs(case["q"], k8, v8, np.full_like(ks, 0.25),
                                 np.full_like(vs, 0.5), case["tables"], case["ctx"],
                                 case["scale"], dtype)
    e, _ = oracle.decode_e4m3(case["q"], k8, v8, 0.25, 0.5, case["tables"], case["ctx"],
                              case["scale"], dtype)
    assert np.array_equal(c, e)
