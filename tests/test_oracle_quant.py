"""Pins of the oracle's e4m3 quantiser and fp8 expert arithmetic (CPU only).

Each check ties the oracle to something other than itself: torch's float8_e4m3fn conversion (a
library routine) for the code table and for rounding, closed forms for saturation, ties and the
error bound, and the pinned bf16 MoE oracle for the fp8 expert stages on operands that already
lie on the e4m3 grid (there quantisation is the identity, so the two must agree).
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from oracle.quant import (decode_e4m3, e4m3_table, encode_e4m3, quantize_matrix, quantize_rows,
                          round_e4m3)


def _torch_e4m3(x):
    """torch's RNE conversion of binary32 values to float8_e4m3fn, widened to float64."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_code_table_matches_torch_bit_patterns():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    tab = e4m3_table()
    assert np.array_equal(np.isnan(tab), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(tab[ok], ref[ok])
    assert np.array_equal(np.signbit(tab[ok]), np.signbit(ref[ok]))
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9 and tab[0x08] == 2.0 ** -6


def test_encode_decode_round_trip():
    tab = e4m3_table()
    c = np.arange(256, dtype=np.uint8)
    ok = ~np.isnan(tab)
    assert np.array_equal(encode_e4m3(tab[ok]), c[ok])
    assert np.array_equal(decode_e4m3(c[ok]), tab[ok])
    with pytest.raises(ValueError):
        encode_e4m3(np.array([1.0625]))  # between 1 and 1.125


def test_rounding_matches_torch_everywhere_below_the_clamp():
    rng = np.random.default_rng(0)
    # random binary32 values over every binade of the format, plus the subnormal range
    mags = np.exp2(rng.uniform(-14, 8.85, 200000)).astype(np.float32)
    x = np.where(rng.random(mags.shape) < 0.5, -mags, mags).astype(np.float32)
    # every grid point, every midpoint between neighbours, and their binary32 neighbours
    tab = e4m3_table()[:0x7F]
    mids = ((tab[1:] + tab[:-1]) / 2).astype(np.float32)
    pts = np.concatenate([tab.astype(np.float32), mids, [np.float32(456.0)]])
    near = np.concatenate([pts, np.nextafter(pts, np.float32(np.inf)),
                           np.nextafter(pts, np.float32(0))])
    x = np.concatenate([x, near, -near]).astype(np.float32)
    x = x[np.abs(x) < 464.0]  # torch turns larger values into NaN; the oracle saturates
    got = round_e4m3(x.astype(np.float64))
    ref = _torch_e4m3(x)
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))


def test_ties_go_to_the_even_significand():
    # 1 + 1/16 lies halfway between 1 (mantissa 0) and 1.125 (mantissa 1): even is 1
    assert round_e4m3(np.array([1.0625]))[0] == 1.0
    # 1.1875 lies between 1.125 (m 1) and 1.25 (m 2): even is 1.25
    assert round_e4m3(np.array([1.1875]))[0] == 1.25
    # halfway between the two smallest subnormals 2^-9 and 2^-8: even is 2^-8 (m 2)
    assert round_e4m3(np.array([1.5 * 2.0 ** -9]))[0] == 2.0 ** -8
    # halfway between 0 and 2^-9 goes to zero
    assert round_e4m3(np.array([2.0 ** -10]))[0] == 0.0


def test_saturation_to_448():
    x = np.array([448.0, 460.0, 464.0, 465.0, 1e6, 3e38, -1e9])
    assert np.array_equal(round_e4m3(x), [448, 448, 448, 448, 448, 448, -448])


def test_row_quantisation_bounds():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal((64, 300)) * np.exp2(rng.uniform(-20, 20, (64, 1)))).astype(np.float32)
    v[3] = 0.0
    q, s = quantize_rows(v)
    assert s.dtype == np.float32 and s[3] == 0 and not q[3].any()
    nz = np.arange(64) != 3
    amax = np.abs(v[nz]).max(axis=1)
    assert np.array_equal(s[nz], (amax / np.float32(448)).astype(np.float32))
    # the largest element of each row lands on +-448
    assert np.all(np.abs(q[nz]).max(axis=1) == 448.0)
    # dequantisation error: half a quantum of the element's binade (2^-4 relative for normals,
    # 2^-10 absolute in scaled units for subnormals), plus the binary32 quotient's rounding
    deq = q * s[:, None].astype(np.float64)
    err = np.abs(deq - v)
    scaled = np.abs(v) / np.where(s > 0, s, 1)[:, None]
    bound = np.where(scaled >= 2.0 ** -6, 2.0 ** -4 * np.abs(v), 2.0 ** -10 * s[:, None])
    assert np.all(err[nz] <= bound[nz] * (1 + 2.0 ** -20))


def test_rows_already_on_the_grid_are_exact():
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 0x7F, (16, 64))
    codes[:, 5] = 0x7E  # each row's largest magnitude is 448
    vals = e4m3_table()[codes] * np.where(rng.random((16, 64)) < 0.5, -1, 1)
    sigma = np.exp2(rng.integers(-12, 4, 16)).astype(np.float64)
    q, s = quantize_rows(vals * sigma[:, None])
    assert np.array_equal(q, vals)
    assert np.array_equal(s.astype(np.float64), sigma)


def _on_grid(rng, shape, lo=-15, hi=-10):
    """Rows of e4m3 values times a power of two per row, each row's max magnitude 448 x 2^j."""
    rows = int(np.prod(shape[:-1]))
    codes = rng.integers(0, 0x7F, (rows, shape[-1]))
    codes[np.arange(rows), rng.integers(0, shape[-1], rows)] = 0x7E
    sign = np.where(rng.random((rows, shape[-1])) < 0.5, -1.0, 1.0)
    sigma = np.exp2(rng.integers(lo, hi, rows)).astype(np.float64)
    return (e4m3_table()[codes] * sign * sigma[:, None]).reshape(shape)


def test_fp8_stages_equal_the_bf16_expert_on_grid_operands():
    rng = np.random.default_rng(3)
    n, d, hid = 24, 128, 48
    x = _on_grid(rng, (n, d), -9, -6)
    w_gu = _on_grid(rng, (2 * hid, d))
    w_d = _on_grid(rng, (d, hid))
    xq, xs = quantize_rows(x)
    gq, gs = quantize_matrix(w_gu)
    h8 = om.gate_up_fp8(xq, xs, gq, gs)
    y16, h16 = om.expert_glu(x, w_gu, w_d, "bf16")
    assert np.array_equal(h8, h16)
    # the down stage on an h that lies on the grid reproduces the plain product
    hg = _on_grid(rng, (n, hid), -6, -2)
    dq, ds = quantize_matrix(w_d)
    ref = hg @ w_d.T
    got = om.down_fp8(hg, dq, ds)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # a transposed or per-column scale would break this: check that scales vary along rows
    assert len(np.unique(gs)) > 1 and len(np.unique(ds)) > 1


def test_fp8_moe_within_the_quantisation_bound_of_the_bf16_moe():
    rng = np.random.default_rng(4)
    t, d, e, k, hid, hs = 48, 128, 8, 2, 64, 96
    wr = (rng.standard_normal((e, d)) * 0.02).astype(np.float32)
    w_gu = _on_grid(rng, (e, 2 * hid, d))
    w_d = _on_grid(rng, (e, d, hid))
    s_gu = _on_grid(rng, (2 * hs, d))
    s_d = _on_grid(rng, (d, hs))
    xg = _on_grid(rng, (t, d), -9, -6)
    y8, info8 = om.moe_ffn_fp8(xg, wr, w_gu, w_d, k, (s_gu, s_d))
    y16, info16 = om.moe_ffn(xg, wr, w_gu, w_d, k, "bf16", (s_gu, s_d))
    assert np.array_equal(info8["ids"], info16["ids"])
    # the only difference left is h's quantisation: |dh| <= 2^-4 |h| + 2^-10 s_h elementwise, so
    # |dy_slot| <= sum_j (2^-4 |h_j| + 2^-10 s_h) |w_d[., j]|
    bound = np.zeros((t, d))
    for s in range(k):
        for tok in range(t):
            ex = info16["ids"][tok, s]
            _, h = om.expert_glu(xg[tok:tok + 1], w_gu[ex], w_d[ex], "bf16")
            sh = np.abs(h).max() / 448
            bound[tok] += info16["weights"][tok, s] * (
                (2.0 ** -4 * np.abs(h) + 2.0 ** -10 * sh) @ np.abs(w_d[ex]).T)[0]
    _, hsh = om.expert_glu(xg, s_gu, s_d, "bf16")
    sh = np.abs(hsh).max(axis=1, keepdims=True) / 448
    bound += (2.0 ** -4 * np.abs(hsh) + 2.0 ** -10 * sh) @ np.abs(s_d).T
    err = np.abs(y8 - y16)
    assert np.all(err <= bound * 1.001 + 1e-12)
    assert err.max() > 0  # h quantisation did change something


# ---- NVFP4 ---------------------------------------------------------------------------------

from oracle.quant import (dequantize_nvfp4, e2m1_table, encode_e2m1, quantize_nvfp4_rows,  # noqa: E402
                          round_e2m1)


def test_e2m1_code_table():
    # the eight magnitudes the format admits: exponent field 0 holds 0 and 0.5, then 1, 1.5 /
    # 2, 3 / 4, 6; bit 3 is the sign
    tab = e2m1_table()
    assert tab[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(tab[8:], -tab[:8]) and np.signbit(tab[8])
    assert np.array_equal(encode_e2m1(tab), np.arange(16, dtype=np.uint8))


def test_e2m1_rounding_brute_force():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-8, 8, 20000), np.arange(-7, 7.01, 0.125)])
    got = round_e2m1(x)
    grid = e2m1_table()[:8]
    for v, g in zip(x, got):
        a = abs(v)
        if a >= 6:
            assert g == np.copysign(6.0, v)
            continue
        dist = np.abs(grid - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) == 2:  # a tie: the even code (mantissa bit 0) wins
            pick = best[0] if best[0] % 2 == 0 else best[1]
        else:
            pick = best[0]
        assert g == np.copysign(grid[pick], v), (v, g)


def _nvfp4_on_grid(rng, rows, k, j_lo=-14, j_hi=-8):
    """Rows code * block scale * 2^j where every 16-block holds a +-6 code and the row's largest
    block scale is 448: NVFP4 quantisation returns them exactly."""
    codes = e2m1_table()[rng.integers(0, 8, (rows, k // 16, 16))]
    codes[:, :, rng.integers(0, 16)] = 6.0
    codes *= np.where(rng.random(codes.shape) < 0.5, -1.0, 1.0)
    sb = e4m3_table()[rng.integers(0x30, 0x7F, (rows, k // 16))]
    sb[:, 0] = 448.0
    g = np.exp2(rng.integers(j_lo, j_hi, rows)).astype(np.float64)
    return (codes * sb[:, :, None] * g[:, None, None]).reshape(rows, k), codes.reshape(rows, k), sb, g


def test_nvfp4_rows_on_grid_are_exact():
    rng = np.random.default_rng(6)
    x, codes, sb, g = _nvfp4_on_grid(rng, 12, 64)
    q, sb2, g2 = quantize_nvfp4_rows(x)
    assert np.array_equal(q, codes) and np.array_equal(sb2, sb)
    assert np.array_equal(g2.astype(np.float64), g)
    assert np.array_equal(dequantize_nvfp4(q, sb2, g2), x)


def test_nvfp4_error_bound_and_max_block():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((32, 128)) * np.exp2(rng.uniform(-10, 10, (32, 1)))).astype(np.float32)
    x[4] = 0.0
    q, sb, g = quantize_nvfp4_rows(x)
    assert g[4] == 0 and not q[4].any()
    d = dequantize_nvfp4(q, sb, g)
    blocks = np.abs(x.astype(np.float64)).reshape(32, 8, 16)
    bmax = np.repeat(blocks.max(axis=2), 16, axis=1)
    # half an e2m1 spacing (<= |x| / 4, or 1/4 of the block step below 1) with a block step of
    # at most (block max / 6) * (1 + 1/16) after the e4m3 rounding of the block scale
    bound = 0.25 * np.abs(x) + 0.25 * bmax / 6 * (17 / 16)
    assert np.all(np.abs(d - x) <= bound * (1 + 1e-6))
    nz = g > 0
    amax_blk = blocks.max(axis=2).argmax(axis=1)
    assert np.all(sb[nz, amax_blk[nz]] == 448.0)  # the block holding the row maximum
    assert np.all(np.abs(q[nz]).max(axis=1) == 6.0)


def test_nvfp4_stages_equal_the_bf16_expert_on_grid_operands():
    rng = np.random.default_rng(8)
    n, d, hid = 8, 64, 32
    x, *_ = _nvfp4_on_grid(rng, n, d, -6, -4)
    w_gu, *_ = _nvfp4_on_grid(rng, 2 * hid, d, -16, -12)
    w_d, *_ = _nvfp4_on_grid(rng, d, hid, -16, -12)
    y16, h16 = om.expert_glu(x, w_gu, w_d, "bf16")
    assert np.array_equal(om.gate_up_nvfp4(x, w_gu), h16)
    hg, *_ = _nvfp4_on_grid(rng, n, hid, -8, -6)
    ref = hg @ w_d.T
    assert np.allclose(om.down_nvfp4(hg, w_d), ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_nvfp4_moe_runs_and_routes_like_bf16():
    rng = np.random.default_rng(9)
    t, d, e, k, hid, hs = 32, 64, 8, 2, 32, 48
    x = rng.standard_normal((t, d))
    wr = rng.standard_normal((e, d)) * 0.02
    w_gu = rng.standard_normal((e, 2 * hid, d)) * 0.02
    w_d = rng.standard_normal((e, d, hid)) * 0.02
    sh = (rng.standard_normal((2 * hs, d)) * 0.02, rng.standard_normal((d, hs)) * 0.02)
    y4, i4 = om.moe_ffn_nvfp4(x, wr, w_gu, w_d, k, sh)
    y16, i16 = om.moe_ffn(x, wr, w_gu, w_d, k, "bf16", sh)
    assert np.array_equal(i4["ids"], i16["ids"])
    # 4-bit elements: the outputs agree to the format's precision, not to bf16's
    rel = np.linalg.norm(y4 - y16) / np.linalg.norm(y16)
    assert 1e-3 < rel < 0.25, rel


# ---- the LM head on e4m3 operands ---------------------------------------------------------------

def test_lm_head_fp8_equals_bf16_head_on_grid_operands():
    # rows already on the e4m3 grid whose maximum is 448: quantisation is the identity (scale 1),
    # so the fp8 head equals the plain product exactly
    from oracle import model as om
    from oracle.quant import e4m3_table
    rng = np.random.default_rng(5)
    grid = e4m3_table()
    grid = grid[np.isfinite(grid) & (np.abs(grid) <= 448)]
    xf = rng.choice(grid, (6, 64))
    emb = rng.choice(grid, (40, 64))
    xf[:, 0] = 448.0
    emb[:, 3] = -448.0
    got = om.lm_head_fp8(xf, emb)
    assert np.array_equal(got, (xf @ emb.T).astype(np.float32).astype(np.float64))


def test_lm_head_fp8_error_bound_and_planted_mistake():
    from oracle import model as om
    from oracle.quant import quantize_rows
    rng = np.random.default_rng(6)
    xf = rng.standard_normal((8, 96))
    emb = rng.standard_normal((50, 96)) * 0.02
    got = om.lm_head_fp8(xf, emb)
    exact = xf @ emb.T
    # each element moves by at most half an e4m3 step: 2^-4 relative to a normal value, plus the
    # subnormal quantum (2^-9 of the row scale, halved) near zero
    ex = np.abs(xf) * 2.0 ** -4 + np.max(np.abs(xf), 1, keepdims=True) / 448 * 2.0 ** -10
    ee = np.abs(emb) * 2.0 ** -4 + np.max(np.abs(emb), 1, keepdims=True) / 448 * 2.0 ** -10
    bound = (np.abs(xf) + ex) @ ee.T + ex @ np.abs(emb).T + 1e-12
    assert np.all(np.abs(got - exact) <= bound)
    assert np.max(np.abs(got - exact)) > 0  # the quantisation does act
    # a dropped vocabulary-row scale does not pass the bound
    xq, xs = quantize_rows(xf)
    eq, es = quantize_rows(emb)
    wrong = (xq @ eq.T) * xs[:, None]
    assert not np.all(np.abs(wrong - exact) <= bound)
