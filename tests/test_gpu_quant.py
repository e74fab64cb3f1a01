"""GPU parity of the cast kernels against the oracle (bit-exact codes and scales).

Casts are integer decisions taken from bf16 inputs with exact power-of-two
scaling, so the bar is bit equality of every code and scale byte.
"""
import numpy as np
import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk
import synth
from oracle import mx
from mxtest import bf16_np, mma_to_plain, u8, assert_codes_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits_to_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def _check_rows(xt: torch.Tensor, out, plain=True):
    x = bf16_np(xt)
    rc, rs = mx.quantize_rows(x)
    np.testing.assert_array_equal(u8(out["row_codes"]), rc)
    gs = u8(out["row_scales"]) if plain else mma_to_plain(u8(out["row_scales"]), *x.shape)
    np.testing.assert_array_equal(gs.reshape(rs.shape), rs)


def _check_cols(xt: torch.Tensor, out, plain=True):
    x = bf16_np(xt)
    cc, cs = mx.quantize_cols(x)
    np.testing.assert_array_equal(u8(out["col_codes"]), cc)
    gs = u8(out["col_scales"]) if plain else mma_to_plain(u8(out["col_scales"]), x.shape[1], x.shape[0])
    np.testing.assert_array_equal(gs.reshape(cs.shape), cs)


def test_every_bf16_pattern_random_blocks():
    """All 65,536 bf16 bit patterns (NaN/Inf included) in random blocks of 32."""
    g = np.random.default_rng(0)
    bits = g.permutation(65536).reshape(512, 128)
    xt = _bits_to_bf16(bits).to(DEV)
    out = mxk.mxfp8_quantize(xt, mxk.ROW | mxk.COL)
    _check_rows(xt.cpu(), out)
    _check_cols(xt.cpu(), out)


@pytest.mark.parametrize("byte", [0, 1, 100, 119, 127, 134, 200, 246])
def test_every_finite_pattern_under_fixed_scale(byte):
    """Each finite bf16 pattern below the block maximum, quantized under a fixed scale byte."""
    k = byte - 127 + 8 if byte > 0 else -119          # block max in [2^k, 2^(k+1))
    allv = mx.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    fin = np.isfinite(allv) & (np.abs(allv) < 2.0 ** (k + 1))
    pats = np.arange(65536)[fin]
    nblk = -(-pats.size // 31)
    pats = np.concatenate([pats, np.zeros(nblk * 31 - pats.size, dtype=pats.dtype)]).reshape(nblk, 31)
    setter = mx.f64_to_bf16_bits(np.array([2.0 ** k]))[0]
    blocks = np.concatenate([np.full((nblk, 1), setter), pats], axis=1)     # [nblk, 32]
    rows = -(-nblk // 4) * 4
    blocks = np.concatenate([blocks, np.zeros(((rows - nblk), 32), dtype=blocks.dtype)])
    xt = _bits_to_bf16(blocks.reshape(rows // 4, 128))
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW)
    _check_rows(xt, out)
    assert (u8(out["row_scales"]).reshape(-1)[:nblk] == byte).all()


@pytest.mark.parametrize("layout", [mxk.PLAIN, mxk.MMA])
def test_dual_quant_random_with_outliers(layout):
    g = synth.rng(3)
    xt = synth.to_bf16(synth.normal(g, (384, 640), 1.0, 0.01, 100.0))
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW | mxk.COL, layout)
    _check_rows(xt, out, layout == mxk.PLAIN)
    _check_cols(xt, out, layout == mxk.PLAIN)


def test_batched_col_weights():
    g = synth.rng(4)
    w = synth.to_bf16(synth.normal(g, (3, 256, 384), 0.02))
    out = mxk.mxfp8_quantize(w.to(DEV), mxk.COL, mxk.MMA)
    cc = u8(out["col_codes"])
    cs = mma_to_plain(u8(out["col_scales"]), 3 * 384, 256).reshape(3, 384, 8)
    for b in range(3):
        rc, rs = mx.quantize_cols(bf16_np(w[b]))
        np.testing.assert_array_equal(cc[b], rc)
        np.testing.assert_array_equal(cs[b], rs)


@pytest.mark.parametrize("shape", [(64, 100), (8, 7170), (3, 31), (5, 1)])
def test_short_last_group(shape):
    g = synth.rng(5)
    xt = synth.to_bf16(synth.normal(g, shape, 2.0, 0.05, 30.0))
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW)
    assert out["row_scales"].shape[-1] == -(-shape[1] // 32)
    _check_rows(xt, out)


def test_transport_payload_cast_full_size():
    """The A2E payload cast: x [8192, 7168] bf16 ~N(0,1), row-wise, every element."""
    xt = synth.make_cast_input()
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW)
    _check_rows(xt, out)


def test_swiglu_quant_small_bitexact_or_one_code():
    g = synth.rng(6)
    h13 = synth.to_bf16(synth.normal(g, (256, 2 * 384), 1.0, 0.01, 100.0))
    out = mxk.mxfp8_swiglu_quant(h13.to(DEV), mxk.ROW | mxk.COL)
    rc, rs, cc, cs = mx.swiglu_quant(bf16_np(h13))
    assert_codes_close(u8(out["row_codes"]), rc, u8(out["row_scales"]), rs, "swiglu ROW")
    assert_codes_close(u8(out["col_codes"]), cc, u8(out["col_scales"]), cs, "swiglu COL")


def test_swiglu_quant_full_size_sampled():
    """h13 [16384, 2x4096] with 1 % outliers x100; 16 sampled 32-row blocks checked."""
    h13 = synth.make_swiglu_input()
    hd = h13.to(DEV)
    out = mxk.mxfp8_swiglu_quant(hd, mxk.ROW | mxk.COL, mxk.MMA)
    torch.cuda.synchronize()
    g = np.random.default_rng(7)
    rb = np.sort(g.choice(16384 // 32, size=16, replace=False))
    rows = (rb[:, None] * 32 + np.arange(32)[None, :]).reshape(-1)
    x = bf16_np(h13[torch.from_numpy(rows)])
    rc, rs, _, _ = mx.swiglu_quant(x)
    got_rc = u8(out["row_codes"])[rows]
    got_rs = mma_to_plain(u8(out["row_scales"]), 16384, 4096)[rows]
    assert_codes_close(got_rc, rc, got_rs, rs, "swiglu ROW full")
    gcc = u8(out["col_codes"])
    gcs = mma_to_plain(u8(out["col_scales"]), 4096, 16384)
    for i, b in enumerate(rb):
        _, _, cc, cs = mx.swiglu_quant(x[i * 32:(i + 1) * 32])
        assert_codes_close(gcc[:, b * 32:(b + 1) * 32], cc, gcs[:, b:b + 1], cs, "swiglu COL full")


def test_dequantize_endpoints_and_random():
    g = np.random.default_rng(8)
    codes = g.integers(0, 256, (64, 96), dtype=np.uint8)
    scales = g.integers(0, 256, (64, 3), dtype=np.uint8)
    scales[0, :] = 0          # 2^-127: an E4M3 16 restores to 2^-123 (representable in bf16)
    scales[1, :] = 255        # NaN
    scales[2, :] = 127
    codes[0, 0] = 0x58        # 16.0
    out = mxk.mxfp8_dequantize(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV))
    got = bf16_np(out)
    ref = mx.round_to_bf16(mx.dequantize_rows(codes, scales))
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])
    assert got[0, 0] == 2.0 ** -123
    assert np.isnan(got[1]).all()


def _dequant_check(codes, scales):
    out = mxk.mxfp8_dequantize(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV))
    got = bf16_np(out)
    ref = mx.round_to_bf16(mx.dequantize_rows(codes, scales))
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])


def test_dequantize_every_code_with_every_scale():
    # Row r carries scale byte r on all its blocks and every code once: all
    # 65536 (code, scale) pairs, including overflow to inf, bf16 subnormals
    # and both NaN sources.
    codes = np.tile(np.arange(256, dtype=np.uint8), (256, 1))
    scales = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 8, axis=1)
    _dequant_check(codes, scales)


@pytest.mark.parametrize("rows,cols", [(37, 48), (130, 40), (5, 16), (2048, 7168)])
def test_dequantize_shapes(rows, cols):
    # cols % 32 == 16 (a half block at the row end), cols % 16 != 0 (scalar
    # path) and a payload-sized tensor on the vector path.
    g = np.random.default_rng(rows * 7 + cols)
    codes = g.integers(0, 256, (rows, cols), dtype=np.uint8)
    scales = g.integers(100, 150, (rows, (cols + 31) // 32), dtype=np.uint8)
    _dequant_check(codes, scales)


# ---------------------------------------------------------------- E5M2 elements
def _check_e5m2(xt, out, rows=True, cols=True, plain=True):
    x = bf16_np(xt)
    if rows:
        rc, rs = mx.quantize_rows(x, "e5m2")
        np.testing.assert_array_equal(u8(out["row_codes"]), rc)
        gs = u8(out["row_scales"]) if plain else mma_to_plain(u8(out["row_scales"]), *x.shape)
        np.testing.assert_array_equal(gs.reshape(rs.shape), rs)
    if cols:
        cc, cs = mx.quantize_cols(x, "e5m2")
        np.testing.assert_array_equal(u8(out["col_codes"]), cc)
        gs = u8(out["col_scales"]) if plain else mma_to_plain(u8(out["col_scales"]), x.shape[1], x.shape[0])
        np.testing.assert_array_equal(gs.reshape(cs.shape), cs)


def test_e5m2_every_bf16_pattern_random_blocks():
    g = np.random.default_rng(1)
    bits = g.permutation(65536).reshape(512, 128)
    xt = _bits_to_bf16(bits)
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW | mxk.COL, elem="e5m2")
    _check_e5m2(xt, out)


@pytest.mark.parametrize("byte", [0, 1, 100, 112, 127, 141, 200, 239])
def test_e5m2_every_finite_pattern_under_fixed_scale(byte):
    k = byte - 127 + 15 if byte > 0 else -112         # block max in [2^k, 2^(k+1))
    allv = mx.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    fin = np.isfinite(allv) & (np.abs(allv) < 2.0 ** (k + 1))
    pats = np.arange(65536)[fin]
    nblk = -(-pats.size // 31)
    pats = np.concatenate([pats, np.zeros(nblk * 31 - pats.size, dtype=pats.dtype)]).reshape(nblk, 31)
    setter = mx.f64_to_bf16_bits(np.array([2.0 ** k]))[0]
    blocks = np.concatenate([np.full((nblk, 1), setter), pats], axis=1)
    rows = -(-nblk // 4) * 4
    blocks = np.concatenate([blocks, np.zeros(((rows - nblk), 32), dtype=blocks.dtype)])
    xt = _bits_to_bf16(blocks.reshape(rows // 4, 128))
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW, elem="e5m2")
    _check_e5m2(xt, out, cols=False)
    assert (u8(out["row_scales"]).reshape(-1)[:nblk] == byte).all()


@pytest.mark.parametrize("layout", [mxk.PLAIN, mxk.MMA])
def test_e5m2_dual_and_short_group(layout):
    g = synth.rng(6)
    xt = synth.to_bf16(synth.normal(g, (256, 384), 1.0, 0.01, 1000.0))
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW | mxk.COL, layout, elem="e5m2")
    _check_e5m2(xt, out, plain=layout == mxk.PLAIN)
    xs = synth.to_bf16(synth.normal(g, (9, 7170), 3.0))
    out = mxk.mxfp8_quantize(xs.to(DEV), mxk.ROW, elem="e5m2")
    _check_e5m2(xs, out, cols=False)


def test_e5m2_transport_roundtrip_full_size():
    """The A2E payload in E5M2: cast [8192, 7168] and restore, every element."""
    xt = synth.make_cast_input()
    out = mxk.mxfp8_quantize(xt.to(DEV), mxk.ROW, elem="e5m2")
    back = mxk.mxfp8_dequantize(out["row_codes"], out["row_scales"], elem="e5m2")
    torch.cuda.synchronize()
    x = bf16_np(xt)
    rc, rs = mx.quantize_rows(x, "e5m2")
    np.testing.assert_array_equal(u8(out["row_codes"]), rc)
    np.testing.assert_array_equal(u8(out["row_scales"]), rs)
    ref = mx.round_to_bf16(mx.dequantize_rows(rc, rs, "e5m2"))
    np.testing.assert_array_equal(bf16_np(back), ref)


def test_e5m2_dequantize_every_code_with_every_scale():
    codes = np.tile(np.arange(256, dtype=np.uint8), (256, 1))
    scales = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 8, axis=1)
    for shape_cols in (256, 40):           # vector path and scalar path
        c = np.ascontiguousarray(codes[:, :shape_cols])
        s = np.ascontiguousarray(scales[:, :(shape_cols + 31) // 32])
        out = mxk.mxfp8_dequantize(torch.from_numpy(c).to(DEV), torch.from_numpy(s).to(DEV), elem="e5m2")
        got = bf16_np(out)
        ref = mx.round_to_bf16(mx.dequantize_rows(c, s, "e5m2"))
        np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
        fin = ~np.isnan(ref)
        np.testing.assert_array_equal(got[fin], ref[fin])
