"""Pins of the CPU oracle against facts fixed outside it.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden/pages_examples.txt), library routines (torch's
float8 dtypes, float32->bf16 cast, silu, autograd), brute-force searches,
closed forms and invariants.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import mx
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_examples.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, inp, exp, _cite = line.split(maxsplit=3)
        rows.append((kind, inp, exp))
    return rows


def _f(s):
    return float.fromhex(s) if "0x" in s else float(s)


# ---------------------------------------------------------------- formats
def test_e4m3_table_closed_form():
    t = mx.E4M3_TABLE
    assert t[0x7E] == 448.0
    assert t[0xFE] == -448.0
    assert t[0x08] == 2.0 ** -6          # smallest normal
    assert t[0x01] == 2.0 ** -9          # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert t[0x38] == 1.0 and t[0x40] == 2.0 and t[0x3C] == 1.5
    assert t[0x00] == 0.0 and not math.copysign(1, t[0x00]) < 0
    assert t[0x80] == 0.0 and math.copysign(1, t[0x80]) < 0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.isfinite(t).sum() == 254


def test_e4m3_table_vs_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = mx.e4m3_decode(np.arange(256))
    np.testing.assert_array_equal(np.isnan(ref), np.isnan(ours))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ref[fin], ours[fin])
    np.testing.assert_array_equal(np.signbit(ref[fin]), np.signbit(ours[fin]))


def test_e8m0_golden_from_pages():
    for kind, inp, exp in _golden():
        if kind != "e8m0":
            continue
        got = float(mx.e8m0_decode(np.array([int(inp)]))[0])
        if exp == "nan":
            assert math.isnan(got)
        else:
            assert got == _f(exp), (inp, got, exp)


def test_e8m0_vs_torch():
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = b.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    ours = mx.e8m0_decode(np.arange(256))
    np.testing.assert_array_equal(np.isnan(ref), np.isnan(ours))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ref[fin], ours[fin])


def test_mx_worked_example_from_pages():
    for kind, inp, exp in _golden():
        if kind != "mx":
            continue
        val, byte = inp.split(",")
        code = mx.e4m3_code_of(np.array([float(val)]))
        deq = mx.dequantize_rows(code.reshape(1, 1), np.array([[int(byte)]], dtype=np.uint8))
        got = float(deq[0, 0])
        assert got == _f(exp)
        # "representable in bf16": rounding to bf16 leaves it unchanged
        assert float(mx.round_to_bf16(np.array([got]))[0]) == got
        assert float(torch.tensor(got, dtype=torch.float64).to(torch.bfloat16).double()) == got


# ---------------------------------------------------------------- bf16
def test_round_to_bf16_vs_torch_from_fp32():
    g = np.random.default_rng(1)
    a = g.standard_normal(200000).astype(np.float32) * np.float32(2.0) ** g.integers(-140, 127, 200000).astype(np.float32)
    a = np.concatenate([a, np.array([3.4e38, -3.4e38, 1e-45, -1e-45, 0.0, -0.0], dtype=np.float32)])
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    ours = mx.round_to_bf16(a.astype(np.float64))
    np.testing.assert_array_equal(ref, ours)


def _bf16_neighbours_bruteforce(x):
    """Nearest bf16 to float64 x by enumerating the two bracketing bf16 values."""
    f = np.float32(x)                      # may itself be rounded; bracket around it
    bits = int(np.array(f).view(np.uint32)) >> 16
    best = None
    for b in range(bits - 2, bits + 3):
        if b < 0 or b > 0xFFFF:
            continue
        v = float(mx.bf16_bits_to_f64(np.array([b], dtype=np.uint16))[0])
        if not math.isfinite(v) or math.copysign(1, v) != math.copysign(1, x):
            continue
        d = abs(v - x)
        key = (d, b & 1)                    # ties -> even last mantissa bit
        if best is None or key < best[0]:
            best = (key, v)
    return best[1]


def test_round_to_bf16_bruteforce_f64():
    g = np.random.default_rng(2)
    xs = g.standard_normal(3000) * 2.0 ** g.integers(-130, 120, 3000)
    # exact ties between two bf16 values (midpoints)
    mids = (mx.bf16_bits_to_f64(np.arange(0x3F80, 0x3F90, dtype=np.uint16)) +
            mx.bf16_bits_to_f64(np.arange(0x3F81, 0x3F91, dtype=np.uint16))) / 2
    xs = np.concatenate([xs, mids, -mids])
    ours = mx.round_to_bf16(xs)
    for x, o in zip(xs, ours):
        assert o == _bf16_neighbours_bruteforce(float(x)), x


# ---------------------------------------------------------------- E4M3 element encoder
_POS = np.arange(0x7F)                    # finite non-negative codes 0x00..0x7E
_POS_VAL = mx.E4M3_TABLE[_POS]


def _e4m3_bruteforce(v):
    """Nearest finite E4M3 by search over the decode table, ties -> even code."""
    # past 1e6 every candidate is absorbed in float64 distances; the nearest
    # finite value there is 448 either way
    a = np.minimum(np.abs(v), 1e6)
    d = np.abs(a[:, None] - _POS_VAL[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = np.where(d == dmin, _POS[None, :], 10 ** 6)
    even = np.where((cand % 2 == 0) & (cand < 10 ** 6), cand, 10 ** 6)
    pick = np.where(even.min(axis=1) < 10 ** 6, even.min(axis=1), cand.min(axis=1))
    return (pick | (np.signbit(v).astype(np.int64) << 7)).astype(np.uint8)


@pytest.mark.parametrize("byte", [0, 100, 119, 127, 134, 254])
def test_e4m3_encoder_exhaustive_bf16(byte):
    x = mx.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    x = x[np.isfinite(x)]
    v = np.ldexp(x, -(byte - 127))
    ours = mx.e4m3_code_of(mx.e4m3_round(v))
    for lo in range(0, v.size, 8192):
        ref = _e4m3_bruteforce(v[lo:lo + 8192])
        np.testing.assert_array_equal(ours[lo:lo + 8192], ref)


def test_e4m3_encoder_vs_torch_in_range():
    x = mx.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    for byte in (119, 127, 131):
        v = np.ldexp(x, -(byte - 127))
        v = v[np.isfinite(v) & (np.abs(v) <= 448.0)]
        ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        ours = mx.e4m3_code_of(mx.e4m3_round(v))
        np.testing.assert_array_equal(ours, ref)


# ---------------------------------------------------------------- E5M2 element format
def test_e5m2_table_closed_form():
    t = mx.E5M2_TABLE
    assert t[0x7B] == 57344.0 and t[0xFB] == -57344.0       # largest finite
    assert t[0x04] == 2.0 ** -14                            # smallest normal
    assert t[0x01] == 2.0 ** -16                            # smallest subnormal
    assert t[0x03] == 3 * 2.0 ** -16                        # largest subnormal
    assert t[0x3C] == 1.0 and t[0x40] == 2.0 and t[0x3E] == 1.5
    assert t[0x7C] == np.inf and t[0xFC] == -np.inf
    assert np.isnan(t[[0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF]]).all()
    assert t[0x80] == 0.0 and math.copysign(1, t[0x80]) < 0
    assert np.isfinite(t).sum() == 248


def test_e5m2_table_vs_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e5m2).to(torch.float64).numpy()
    ours = mx.e5m2_decode(np.arange(256))
    np.testing.assert_array_equal(np.isnan(ref), np.isnan(ours))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ref[ok], ours[ok])
    np.testing.assert_array_equal(np.signbit(ref[ok]), np.signbit(ours[ok]))


_POS5 = np.arange(0x7C)                   # finite non-negative E5M2 codes 0x00..0x7B
_POS5_VAL = mx.E5M2_TABLE[_POS5]


def _e5m2_bruteforce(v):
    """Nearest finite E5M2 by search over the decode table, ties -> even code."""
    a = np.minimum(np.abs(v), 1e9)
    d = np.abs(a[:, None] - _POS5_VAL[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = np.where(d == dmin, _POS5[None, :], 10 ** 6)
    even = np.where((cand % 2 == 0) & (cand < 10 ** 6), cand, 10 ** 6)
    pick = np.where(even.min(axis=1) < 10 ** 6, even.min(axis=1), cand.min(axis=1))
    return (pick | (np.signbit(v).astype(np.int64) << 7)).astype(np.uint8)


@pytest.mark.parametrize("byte", [0, 100, 112, 127, 141, 254])
def test_e5m2_encoder_exhaustive_bf16(byte):
    x = mx.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    x = x[np.isfinite(x)]
    v = np.ldexp(x, -(byte - 127))
    ours = mx.e5m2_code_of(mx.e5m2_round(v))
    for lo in range(0, v.size, 8192):
        ref = _e5m2_bruteforce(v[lo:lo + 8192])
        np.testing.assert_array_equal(ours[lo:lo + 8192], ref)


def test_e5m2_encoder_vs_torch_in_range():
    x = mx.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    for byte in (112, 127, 135):
        v = np.ldexp(x, -(byte - 127))
        v = v[np.isfinite(v) & (np.abs(v) <= 57344.0)]
        ref = torch.from_numpy(v).to(torch.float8_e5m2).view(torch.uint8).numpy()
        ours = mx.e5m2_code_of(mx.e5m2_round(v))
        np.testing.assert_array_equal(ours, ref)


def test_e5m2_scale_rule_and_special_blocks():
    g = np.random.default_rng(13)
    x = mx.round_to_bf16(g.standard_normal((16, 256)) * 2.0 ** g.integers(-90, 90, (16, 1)))
    codes, sc = mx.quantize_rows(x, "e5m2")
    amax = np.abs(x).reshape(16, 8, 32).max(axis=2)
    ratio = amax / np.ldexp(1.0, sc.astype(np.int64) - 127)
    assert ((ratio >= 2.0 ** 15) & (ratio < 2.0 ** 16)).all()       # emax 15: max lands in [2^15, 2^16)
    deq = mx.dequantize_rows(codes, sc, "e5m2")
    s = np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1)
    a = np.abs(x) / s
    ulp = np.ldexp(1.0, np.maximum(np.frexp(a)[1] - 3, -16))
    unsat = a <= 57344
    assert (np.abs(deq - x)[unsat] <= 0.5 * ulp[unsat] * s[unsat]).all()
    y = np.zeros((1, 96))
    y[0, 0] = np.inf
    y[0, 1] = -2.0
    y[0, 32:64] = -0.0
    c, b = mx.quantize_rows(y, "e5m2")
    assert b[0, 0] == 0xFF and c[0, 0] == 0x7F and c[0, 1] == 0xFF
    assert b[0, 1] == 0 and (c[0, 32:64] == 0x80).all() and b[0, 2] == 0


# ---------------------------------------------------------------- block quantizer
def test_scale_rule_puts_block_max_in_256_512():
    g = np.random.default_rng(3)
    x = mx.round_to_bf16(g.standard_normal((64, 256)) * 2.0 ** g.integers(-100, 100, (64, 1)))
    codes, sc = mx.quantize_rows(x)
    amax = np.abs(x).reshape(64, 8, 32).max(axis=2)
    ratio = amax / np.ldexp(1.0, sc.astype(np.int64) - 127)
    assert ((ratio >= 256) & (ratio < 512)).all()
    # the largest element is saturated to 448 or lands on 256..448 exactly
    deq = mx.dequantize_rows(codes, sc)
    assert (np.abs(deq) <= 448 * np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1) + 0).all()


def test_scale_is_power_of_two_and_roundtrip_bound():
    g = np.random.default_rng(4)
    x = mx.round_to_bf16(g.standard_normal((32, 320)) * 3.0)
    codes, sc = mx.quantize_rows(x)
    s = np.repeat(mx.e8m0_decode(sc), 32, axis=1)
    v = x / s
    deq = mx.dequantize_rows(codes, sc)
    a = np.abs(v)
    ulp = np.ldexp(1.0, np.maximum(np.frexp(a)[1] - 4, -9))
    unsat = a <= 448
    assert (np.abs(deq - x)[unsat] <= 0.5 * ulp[unsat] * s[unsat]).all()
    assert (np.abs(deq - x)[~unsat] <= 64 * s[~unsat]).all()
    m, e = np.frexp(mx.e8m0_decode(sc))
    assert (m == 0.5).all()


def test_special_blocks():
    x = np.zeros((1, 160))
    x[0, 32:64] = mx.bf16_bits_to_f64(np.array([0x0001], dtype=np.uint16))[0]  # bf16 subnormal
    x[0, 64] = np.nan
    x[0, 65] = -1.0
    x[0, 96] = np.inf
    x[0, 128:160] = -0.0
    codes, sc = mx.quantize_rows(x)
    assert sc[0, 0] == 0 and (codes[0, :32] == 0).all()            # all-zero block
    assert sc[0, 1] == 0                                           # amax below 2^-126 clamps to 0
    assert sc[0, 2] == 0xFF and codes[0, 64] == 0x7F and codes[0, 65] == 0xFF
    assert sc[0, 3] == 0xFF and (codes[0, 96:128] & 0x7F == 0x7F).all()
    assert sc[0, 4] == 0 and (codes[0, 128:160] == 0x80).all()     # -0 keeps its sign


def test_short_last_group():
    g = np.random.default_rng(5)
    x = mx.round_to_bf16(g.standard_normal((4, 100)))
    x[:, 96:] *= 1000.0                                            # last block of 4
    x = mx.round_to_bf16(x)
    codes, sc = mx.quantize_rows(x)
    assert sc.shape == (4, 4) and codes.shape == (4, 100)
    amax = np.abs(x[:, 96:]).max(axis=1)
    assert (sc[:, 3] == mx.scale_byte(amax)).all()
    # the first three blocks do not see the large tail
    assert (sc[:, :3] < sc[:, 3:]).all()
    np.testing.assert_allclose(mx.dequantize_rows(codes, sc), x, rtol=2 ** -3)


def test_cols_are_rows_of_transpose_with_row_blocks():
    g = np.random.default_rng(6)
    x = mx.round_to_bf16(g.standard_normal((64, 48)))
    x[5, 7] = 1e4
    x = mx.round_to_bf16(x)
    cc, cs = mx.quantize_cols(x)
    assert cc.shape == (48, 64) and cs.shape == (48, 2)
    # only the block holding (row 5, col 7) sees the outlier
    big = cs == cs.max()
    assert big.sum() == 1 and big[7, 0]


# ---------------------------------------------------------------- grouped GEMMs
_EXACT_VALS = np.array([0, 1, 2, 3, 4, 6, 8, 12, 16, -1, -2, -3, -4, -6, -8, -12, -16], dtype=np.int64)


def _exact_ints(g, shape):
    """Integers whose MX quantization is exact (values {1,1.5}*2^k, |v| <= 16)."""
    return g.choice(_EXACT_VALS, size=shape)


def test_exact_values_roundtrip_exactly():
    g = np.random.default_rng(7)
    x = _exact_ints(g, (64, 96)).astype(np.float64)
    c, s = mx.quantize_rows(x)
    np.testing.assert_array_equal(mx.dequantize_rows(c, s), x)


def test_grouped_gemm_exact_integer_closed_form():
    g = np.random.default_rng(8)
    E, N, K = 3, 40, 64
    offsets = np.array([0, 64, 64, 160], dtype=np.int32)          # expert 1 empty
    M = 192
    a = _exact_ints(g, (M, K))
    w = _exact_ints(g, (E, N, K))
    ac, as_ = mx.quantize_rows(a.astype(np.float64))
    wc, ws = mx.quantize_weights_rows(w.astype(np.float64))
    out = mx.grouped_gemm(ac, as_, wc, ws, offsets)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        np.testing.assert_array_equal(out[lo:hi], (a[lo:hi] @ w[e].T).astype(np.float64))
    assert np.isnan(out[160:]).all()                               # tail never written


def test_wgrad_exact_integer_closed_form_and_empty_expert():
    g = np.random.default_rng(9)
    E, N, Kx, M = 3, 64, 96, 256
    offsets = np.array([0, 128, 128, 224], dtype=np.int32)
    G = _exact_ints(g, (M, N))
    X = _exact_ints(g, (M, Kx))
    gc, gs = mx.quantize_cols(G.astype(np.float64))
    xc, xs = mx.quantize_cols(X.astype(np.float64))
    dw = mx.grouped_gemm_wgrad(gc, gs, xc, xs, offsets)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        np.testing.assert_array_equal(dw[e], (G[lo:hi].T @ X[lo:hi]).astype(np.float64))
    assert (dw[1] == 0).all() and not np.signbit(dw[1]).any()


# ---------------------------------------------------------------- SwiGLU
def test_swiglu_vs_torch_silu():
    g = np.random.default_rng(10)
    h13 = mx.round_to_bf16(g.standard_normal((16, 64)) * 4)
    F = 32
    ta = torch.from_numpy(h13[:, :F])
    tb = torch.from_numpy(h13[:, F:])
    ref = mx.round_to_bf16((torch.nn.functional.silu(ta) * tb).numpy())
    np.testing.assert_array_equal(mx.swiglu(h13), ref)


def test_dswiglu_finite_difference():
    g = np.random.default_rng(11)
    F = 64
    h13 = mx.round_to_bf16(g.standard_normal((8, 2 * F)) * 3)
    dh = mx.round_to_bf16(g.standard_normal((8, F)))
    a, b = h13[:, :F], h13[:, F:]
    f = lambda aa, bb: aa / (1 + np.exp(-aa)) * bb
    eps = 1e-6
    dga = (f(a + eps, b) - f(a - eps, b)) / (2 * eps) * dh
    dgb = (f(a, b + eps) - f(a, b - eps)) / (2 * eps) * dh
    got = mx.dswiglu(dh, h13)
    ref = np.concatenate([dga, dgb], axis=1)
    np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-8)


# ---------------------------------------------------------------- composites
def _tiny(seed=0, E=3, D=64, F=64, counts=(40, 0, 70), pad=32):
    spec = synth.Spec("t", E, D, F, sum(counts), 1, pad, None, 0, 0.05)
    inp = synth.make_moe_inputs(spec, seed, counts_override=list(counts))
    f = lambda t: t.float().double().numpy()
    return inp, f(inp.x), f(inp.w13), f(inp.w2), f(inp.dy), inp.routing.offsets


def _torch_moe(x, w13, w2, dy, offsets):
    """Independent float64 autograd MLP over expert segments."""
    x = torch.tensor(x, requires_grad=True)
    w13 = torch.tensor(w13, requires_grad=True)
    w2 = torch.tensor(w2, requires_grad=True)
    F = w13.shape[1] // 2
    ys = []
    for e in range(w13.shape[0]):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        xe = x[lo:hi]
        gate = xe @ w13[e, :F].T
        up = xe @ w13[e, F:].T
        ys.append((torch.nn.functional.silu(gate) * up) @ w2[e].T)
    y = torch.cat(ys)
    y.backward(torch.tensor(dy[: y.shape[0]]))
    return y.detach().numpy(), x.grad.numpy(), w13.grad.numpy(), w2.grad.numpy()


def test_composite_exact_mode_vs_torch_autograd():
    inp, x, w13, w2, dy, off = _tiny()
    f = mx.moe_mlp_fwd(x, w13, w2, off, exact=True)
    b = mx.moe_mlp_bwd(dy, f, x, w13, w2, off, exact=True)
    y, dx, dw13, dw2 = _torch_moe(x, w13, w2, dy, off)
    M = int(off[-1])
    np.testing.assert_allclose(f["y"][:M], y, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b["dx"][:M], dx[:M], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b["dw13"], dw13, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b["dw2"], dw2, rtol=1e-12, atol=1e-14)
    assert (b["dw13"][1] == 0).all() and (b["dw2"][1] == 0).all()


def test_composite_mx_mode_close_to_exact_and_zero_expert():
    inp, x, w13, w2, dy, off = _tiny(seed=1)
    fe = mx.moe_mlp_fwd(x, w13, w2, off, exact=True)
    be = mx.moe_mlp_bwd(dy, fe, x, w13, w2, off, exact=True)
    fq = mx.moe_mlp_fwd(x, w13, w2, off)
    bq = mx.moe_mlp_bwd(dy, fq, x, w13, w2, off)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(fq["y"], fe["y"]) < 0.15
    assert rel(bq["dx"], be["dx"]) < 0.15
    assert rel(bq["dw13"], be["dw13"]) < 0.15
    assert rel(bq["dw2"], be["dw2"]) < 0.15
    assert (bq["dw13"][1] == 0).all() and (bq["dw2"][1] == 0).all()


def test_composite_mx_fc1_exact_on_representable_inputs():
    """With inputs whose quantization is exact, MX-mode h13 equals the exact h13."""
    g = np.random.default_rng(12)
    E, D, F = 2, 64, 32
    off = np.array([0, 32, 96], dtype=np.int32)
    tern = lambda shape: g.choice(np.array([-1.0, 0.0, 1.0]), size=shape)
    x = tern((96, D))
    w13 = tern((E, 2 * F, D)) / 16
    w2 = tern((E, D, F)) / 16
    fe = mx.moe_mlp_fwd(x, w13, w2, off, exact=True)
    fq = mx.moe_mlp_fwd(x, w13, w2, off)
    assert np.abs(fe["h13"]).max() <= 4                      # k/16, |k| <= 64: exact in bf16
    np.testing.assert_array_equal(fq["h13"], fe["h13"])


def test_pad_rows_inert_pad128_vs_pad256():
    spec128 = synth.Spec("p", 4, 64, 64, 300, 2, 128, None, 0, 0.05)
    spec256 = synth.Spec("p", 4, 64, 64, 300, 2, 256, None, 0, 0.05)
    a = synth.make_moe_inputs(spec128, 3)
    b = synth.make_moe_inputs(spec256, 3)
    np.testing.assert_array_equal(a.routing.counts, b.routing.counts)
    f = lambda t: t.float().double().numpy()
    outs = []
    for inp in (a, b):
        fw = mx.moe_mlp_fwd(f(inp.x), f(inp.w13), f(inp.w2), inp.routing.offsets)
        bw = mx.moe_mlp_bwd(f(inp.dy), fw, f(inp.x), f(inp.w13), f(inp.w2), inp.routing.offsets)
        real = inp.routing.src_token >= 0
        outs.append((fw["y"][real], bw["dx"][real], bw["dw13"], bw["dw2"]))
        # pad rows produce exact zeros
        pad = np.ones(inp.routing.M, bool)
        pad[real] = False
        assert (fw["y"][pad] == 0).all() and (bw["dx"][pad] == 0).all()
    for u, v in zip(*outs):
        np.testing.assert_array_equal(u, v)


def test_nan_tail_never_read():
    inp, x, w13, w2, dy, off = _tiny(seed=2, counts=(40, 0, 70))
    M = int(off[-1])
    xt = np.concatenate([x, np.full((64, x.shape[1]), np.nan)])
    dyt = np.concatenate([dy, np.full((64, x.shape[1]), np.nan)])
    f0 = mx.moe_mlp_fwd(x, w13, w2, off)
    b0 = mx.moe_mlp_bwd(dy, f0, x, w13, w2, off)
    f1 = mx.moe_mlp_fwd(xt, w13, w2, off)
    b1 = mx.moe_mlp_bwd(dyt, f1, xt, w13, w2, off)
    np.testing.assert_array_equal(f0["y"][:M], f1["y"][:M])
    np.testing.assert_array_equal(b0["dx"][:M], b1["dx"][:M])
    np.testing.assert_array_equal(b0["dw13"], b1["dw13"])
    np.testing.assert_array_equal(b0["dw2"], b1["dw2"])


# ---------------------------------------------------------------- blocking axis of each GEMM operand
# MX blocks run along the contraction dimension of every GEMM operand (the
# MX definition scales 32 elements that enter the same dot product; the
# fully-fused plan page, "What it adds": row-wise quantization for the forward,
# column-wise for the backward contractions).  Each operand below is drawn so
# that its quantization is the identity when its blocks run along its
# contraction axis and destroys entries when they run along the other axis:
# signed powers of two whose exponent is constant along the contraction axis
# and sweeps 24 binades across any 32 consecutive positions of the other axis
# (a block that mixes them holds magnitudes 2^24 apart; relative to the block
# scale E4M3 reaches down to 2^-9 * 2^-8 only, so its small entries flush).
# The GEMM outputs then have closed forms in terms of the unquantized operand.
_NB = 160                     # expert rows (a multiple of 32, unlike every other dimension)
_D, _F = 192, 128


def _axis_exact(g, shape, contraction_axis):
    """Powers of two (10 % zeros), exponent constant along contraction_axis."""
    n_other = shape[1 - contraction_axis]
    exp = (7 * np.arange(n_other)) % 25 - 12          # every 25 consecutive positions: all of -12..12
    e = exp[:, None] if contraction_axis == 1 else exp[None, :]
    sign = g.choice(np.array([-1.0, 1.0]), size=shape)
    zero = g.random(shape) < 0.1
    return np.where(zero, 0.0, sign * np.ldexp(1.0, np.broadcast_to(e, shape)))


def _bf16_generic(g, shape, std):
    return mx.round_to_bf16(g.normal(0.0, std, size=shape))


def test_axis_pin_operands_of_the_exact_inputs_are_unchanged():
    """The construction itself: exact under the contraction-axis blocking,
    altered under the other blocking."""
    g = np.random.default_rng(31)
    a = _axis_exact(g, (_NB, _D), 1)                  # contraction along columns
    np.testing.assert_array_equal(mx.dequantize_rows(*mx.quantize_rows(a)), a)
    assert (mx.dequantize_rows(*mx.quantize_cols(a)).T != a).mean() > 0.2
    b = _axis_exact(g, (_NB, _D), 0)                  # contraction along rows
    np.testing.assert_array_equal(mx.dequantize_rows(*mx.quantize_cols(b)).T, b)
    assert (mx.dequantize_rows(*mx.quantize_rows(b)) != b).mean() > 0.2


def test_axis_pin_forward_operands():
    """x, W13 blocked along D and W2 along F (and h along F): h13 and y
    equal their closed forms on the unquantized x, W13, W2."""
    g = np.random.default_rng(32)
    x = _axis_exact(g, (_NB, _D), 1)                  # FC1 contracts D
    w13 = _axis_exact(g, (2 * _F, _D), 1)             # FC1 contracts D
    w2 = _axis_exact(g, (_D, _F), 1)                  # FC2 contracts F
    r = mx.expert_fwd(x, w13, w2)
    # every h13 entry is 2^k times an integer of at most 192: exact in float64 and bf16
    np.testing.assert_array_equal(r["h13"], x @ w13.T)
    hq = mx.dequantize_rows(*r["h_row"])
    np.testing.assert_array_equal(r["y"], hq @ w2.T)
    assert (np.abs(r["h13"]) > 0).mean() > 0.5 and (np.abs(r["y"]) > 0).mean() > 0.5


def test_axis_pin_backward_dgrad_operands():
    """dY blocked along D and W2 along D (dh), dh13 along 2F and W13 along 2F
    (dx): dh and dx equal their closed forms on the unquantized dY, W2, W13."""
    g = np.random.default_rng(33)
    x = _bf16_generic(g, (_NB, _D), 1.0)
    w13 = _axis_exact(g, (2 * _F, _D), 0)             # dx contracts 2F (the rows of W13)
    w2 = _axis_exact(g, (_D, _F), 0)                  # dh contracts D (the rows of W2)
    dy = _axis_exact(g, (_NB, _D), 1)                 # dh contracts D
    f = mx.expert_fwd(x, w13, w2)
    r = mx.expert_bwd(dy, f, x, w13, w2)
    np.testing.assert_array_equal(r["dh"], dy @ w2)   # 2^k times integers of at most 192: exact
    gq = mx.dequantize_rows(*r["dh13_row"])
    np.testing.assert_array_equal(r["dx"], gq @ w13)
    assert (np.abs(r["dh"]) > 0).mean() > 0.5 and (np.abs(r["dx"]) > 0).mean() > 0.5


def test_axis_pin_backward_wgrad_operands():
    """dY, h, dh13 and x blocked along the token rows (dW2, dW13): the weight
    gradients equal their closed forms on the unquantized dY and x."""
    g = np.random.default_rng(34)
    x = _axis_exact(g, (_NB, _D), 0)                  # dW13 contracts the rows
    dy = _axis_exact(g, (_NB, _D), 0)                 # dW2 contracts the rows
    w13 = _bf16_generic(g, (2 * _F, _D), 0.05)
    w2 = _bf16_generic(g, (_D, _F), 0.05)
    f = mx.expert_fwd(x, w13, w2)
    r = mx.expert_bwd(dy, f, x, w13, w2)
    hc = mx.dequantize_rows(*f["h_col"])              # [F, n]
    gc = mx.dequantize_rows(*r["dh13_col"])           # [2F, n]
    np.testing.assert_array_equal(r["dw2"], dy.T @ hc.T)
    np.testing.assert_array_equal(r["dw13"], gc @ x)
    np.testing.assert_array_equal(mx.dequantize_rows(*f["x_col"]).T, x)
    np.testing.assert_array_equal(mx.dequantize_rows(*r["dy_col"]).T, dy)
    assert (np.abs(r["dw2"]) > 0).mean() > 0.5 and (np.abs(r["dw13"]) > 0).mean() > 0.5
