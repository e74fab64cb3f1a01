"""GPU parity of the tcgen05 grouped GEMMs against the oracle.

Operands are quantized by the oracle from the same bf16 tensors the GPU
quantizes itself (the casts are bit-exact, checked in test_gpu_quant), so
both sides multiply identical MXFP8 operands.
"""
import numpy as np
import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk
import synth
from oracle import mx
from mxtest import (assert_codes_close, assert_gemm_close, bf16_np, mma_to_plain, plain_to_mma, u8)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _offsets(counts, pad):
    padded = [((c + pad - 1) // pad) * pad for c in counts]
    return np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)


def _bf16(a):
    return synth.to_bf16(np.asarray(a, dtype=np.float32))


def _mx_rows_dev(x_bf16: torch.Tensor):
    """GPU ROW quantization with MMA scales (the GEMM operand form)."""
    o = mxk.mxfp8_quantize(x_bf16.to(DEV), mxk.ROW, mxk.MMA)
    return o["row_codes"].reshape(-1, x_bf16.shape[-1]), o["row_scales"]


def _exact_pow2_ternary(g, shape, spread=3):
    """t * 2^e with t in {-1,0,1} and e constant per 32-block: quantization is exact."""
    t = g.choice(np.array([-1.0, 0.0, 1.0]), size=shape)
    t[..., ::32] = 1.0                                   # every block has a nonzero
    e = g.integers(-spread, spread + 1, size=shape[:-1] + (shape[-1] // 32,))
    return t * np.repeat(np.ldexp(1.0, e), 32, axis=-1)


# ------------------------------------------------------------------ ragged M
@pytest.mark.parametrize("N,pad", [(256, 128), (384, 128), (512, 256), (256, 256)])
def test_grouped_gemm_exact_closed_form(N, pad):
    """Exactly representable operands: fp32 accumulation is exact, so the bf16
    output must equal round_to_bf16 of the exact product bit for bit.
    pad 256 with N % 256 == 0 runs the CTA-pair (256 x 256 tile) kernel."""
    g = np.random.default_rng(1)
    E, K = 3, 512
    off = _offsets([200, 0, 300], pad)
    M = int(off[-1]) + 128
    a = _exact_pow2_ternary(g, (M, K))
    w = _exact_pow2_ternary(g, (E, N, K))
    ac, as_ = _mx_rows_dev(_bf16(a))
    wc, ws = _mx_rows_dev(_bf16(w.reshape(E * N, K)))
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxk.mxfp8_grouped_gemm(ac, as_, wc.reshape(E, N, K), ws, _dev(off), pad, out=out)
    got = bf16_np(out)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        np.testing.assert_array_equal(got[lo:hi], mx.round_to_bf16(a[lo:hi] @ w[e].T))
    assert np.isnan(got[off[-1]:]).all()          # rows past offsets[E] untouched
    assert mxk.device_error() == 0


@pytest.mark.parametrize("pad,N,K", [(128, 512, 256), (256, 384, 640), (128, 256, 1408), (256, 512, 768)])
def test_grouped_gemm_random_vs_oracle(pad, N, K):
    g = synth.rng(2)
    E = 4
    off = _offsets([130, 0, 77, 300], pad)
    M = int(off[-1])
    a = _bf16(synth.normal(g, (M, K)))
    w = _bf16(synth.normal(g, (E, N, K), 0.02))
    ac, as_ = _mx_rows_dev(a)
    wc, ws = _mx_rows_dev(w.reshape(E * N, K))
    out = mxk.mxfp8_grouped_gemm(ac, as_, wc.reshape(E, N, K), ws, _dev(off), pad)
    arc, ars = mx.quantize_rows(bf16_np(a))
    wrc, wrs = mx.quantize_weights_rows(bf16_np(w))
    ref = mx.grouped_gemm(arc, ars, wrc, wrs, off)
    assert_gemm_close(bf16_np(out), ref, "grouped_gemm")


def test_grouped_gemm_nan_tail_not_read():
    g = synth.rng(3)
    E, N, K = 2, 256, 256
    off = _offsets([100, 60], 128)
    M = int(off[-1]) + 256
    a = synth.normal(g, (M, K))
    a[off[-1]:] = np.nan                                  # poisoned tail
    at = _bf16(a)
    w = _bf16(synth.normal(g, (E, N, K), 0.02))
    ac, as_ = _mx_rows_dev(at)
    wc, ws = _mx_rows_dev(w.reshape(E * N, K))
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device=DEV)
    mxk.mxfp8_grouped_gemm(ac, as_, wc.reshape(E, N, K), ws, _dev(off), 128, out=out)
    got = bf16_np(out)
    assert np.isfinite(got[: off[-1]]).all()
    assert (got[off[-1]:] == 7.0).all()


def test_bad_offsets_raise_device_error_and_write_nothing():
    E, N, K, M = 2, 256, 256, 256
    a = torch.zeros(M, K, dtype=torch.uint8, device=DEV)
    sa = torch.zeros(M * K // 32, dtype=torch.uint8, device=DEV)
    w = torch.zeros(E, N, K, dtype=torch.uint8, device=DEV)
    sw = torch.zeros(E * N * K // 32, dtype=torch.uint8, device=DEV)
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device=DEV)
    assert mxk.device_error() == 0
    for bad in ([0, 256, 128], [0, 64, 256], [0, 128, 512], [128, 128, 256]):
        mxk.mxfp8_grouped_gemm(a, sa, w, sw, _dev(np.array(bad, np.int32)), 128, out=out)
        assert mxk.device_error(reset=True) == 4, bad
    assert (bf16_np(out) == 3.0).all()


def test_bindings_reject_mismatched_shapes_before_launch():
    """A tensor whose shape disagrees with the others would make the kernel
    read or write outside it; the binding refuses it before any launch."""
    E, N, K, M, F = 2, 256, 256, 256, 128
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8, device=DEV)
    off = _dev(np.array([0, 128, 256], np.int32))
    out = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    good = (u8(M, K), u8(M * K // 32), u8(E, N, K), u8(E * N * K // 32))
    bad_cases = [
        (u8(M, K), u8(M * K // 32), u8(E, N, K + 128), u8(E * N * (K + 128) // 32)),   # K of w
        (u8(M, K), u8(M * K // 32 - 1), u8(E, N, K), u8(E * N * K // 32)),             # a_scales size
        (u8(M, K), u8(M * K // 32), u8(E + 1, N, K), u8((E + 1) * N * K // 32)),       # experts of w
    ]
    for a, sa, w, sw in bad_cases:
        with pytest.raises(ValueError):
            mxk.mxfp8_grouped_gemm(a, sa, w, sw, off, 128, out=out)
    with pytest.raises(ValueError):
        mxk.mxfp8_grouped_gemm(*good, off, 128, out=torch.zeros(M, N + 128, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(ValueError):   # xt with another M
        mxk.mxfp8_grouped_gemm_wgrad(u8(N, M), u8(N * M // 32), u8(K, M + 128), u8(K * (M + 128) // 32), off, 128)
    with pytest.raises(ValueError):   # w13 with an odd row count
        mxk.mxfp8_grouped_gemm_swiglu_quant(u8(M, K), u8(M * K // 32), u8(E, 2 * F + 1, K),
                                            u8(E * (2 * F + 1) * K // 32), off, 128)
    h13 = torch.zeros(M, 2 * F, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):   # w2t laid out as [E, 2F, D]: h13 would be read past its end
        mxk.mxfp8_grouped_gemm_dswiglu_quant(u8(M, K), u8(M * K // 32), u8(E, 2 * F, K), u8(E * 2 * F * K // 32),
                                             off, h13, 128)
    with pytest.raises(ValueError):
        mxk.mxfp8_dequantize(u8(M, K), u8(M * K // 32 + 1))
    assert mxk.device_error() == 0


# ------------------------------------------------------------------ ragged K
def _mx_cols_dev(x_bf16: torch.Tensor):
    o = mxk.mxfp8_quantize(x_bf16.to(DEV), mxk.COL, mxk.MMA)
    return o["col_codes"], o["col_scales"]


@pytest.mark.parametrize("N,Kx", [(256, 384), (512, 512), (128, 128), (256, 256), (2048, 1536)])
def test_wgrad_exact_closed_form_and_empty_expert(N, Kx):
    """Kx = 384 and 128 take the 128-wide tile, 512 and 256 the 256-wide one;
    N x Kx = 2048 x 1536 gives 3 x 96 tiles, more than the SMs, so CTAs walk
    on to the next expert's tiles."""
    g = np.random.default_rng(4)
    E = 3
    off = _offsets([256, 0, 300], 128)
    M = int(off[-1])
    # COL quantization of G and X is exact when each 32-row block of a column
    # is t * 2^e: build the transposes with the helper and transpose back.
    Gt = _exact_pow2_ternary(g, (N, M))
    Xt = _exact_pow2_ternary(g, (Kx, M))
    gc, gs = _mx_cols_dev(_bf16(Gt.T))
    xc, xs = _mx_cols_dev(_bf16(Xt.T))
    out = torch.full((E, N, Kx), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxk.mxfp8_grouped_gemm_wgrad(gc, gs, xc, xs, _dev(off), 128, out=out)
    got = bf16_np(out)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        np.testing.assert_array_equal(got[e], mx.round_to_bf16(Gt[:, lo:hi] @ Xt[:, lo:hi].T))
    assert (got[1] == 0).all() and not np.signbit(got[1]).any()


@pytest.mark.parametrize("N,Kx", [(256, 384), (256, 512)])
def test_wgrad_expert_rows_skip_only_padding(N, Kx):
    """With each expert's token-row count given, the weight gradient stops at
    the last 128-row K block holding a token row.  Kx = 384 runs the single-CTA
    kernel, 512 the CTA pairs.  With zero pad rows the result equals the full
    sum; codes planted in the all-padding K blocks are ignored with the counts
    (and seen without them); a count beyond its segment writes nothing and
    raises the offsets error."""
    g = synth.rng(9)
    counts = [300, 0, 129, 256]
    E, pad = len(counts), 256
    off = _offsets(counts, pad)
    M = int(off[-1])
    G = np.zeros((M, N), np.float32)
    X = np.zeros((M, Kx), np.float32)
    for e, c in enumerate(counts):
        G[off[e]:off[e] + c] = synth.normal(g, (c, N), 1e-2)
        X[off[e]:off[e] + c] = synth.normal(g, (c, Kx))
    gc, gs = _mx_cols_dev(_bf16(G))
    xc, xs = _mx_cols_dev(_bf16(X))
    rows = _dev(np.array(counts, np.int32))
    full = mxk.mxfp8_grouped_gemm_wgrad(gc, gs, xc, xs, _dev(off), pad)
    skip = mxk.mxfp8_grouped_gemm_wgrad(gc, gs, xc, xs, _dev(off), pad, expert_rows=rows)
    assert torch.equal(full, skip)
    # plant codes (and unit scales) in the K blocks that hold only padding
    gc2, xc2, gs2, xs2 = gc.clone(), xc.clone(), gs.clone(), xs.clone()
    for e, c in enumerate(counts):
        lo, hi = int(off[e]) + (c + 127) // 128 * 128, int(off[e + 1])
        if hi > lo:
            gc2[:, lo:hi] = 0x38      # E4M3 1.0
            xc2[:, lo:hi] = 0x38
    gs2.fill_(127)
    xs2.fill_(127)
    gs2.copy_(torch.where(gs == 0, gs2, gs))   # real blocks keep their scales
    xs2.copy_(torch.where(xs == 0, xs2, xs))
    planted = mxk.mxfp8_grouped_gemm_wgrad(gc2, gs2, xc2, xs2, _dev(off), pad, expert_rows=rows)
    assert torch.equal(planted, full)
    unskipped = mxk.mxfp8_grouped_gemm_wgrad(gc2, gs2, xc2, xs2, _dev(off), pad)
    assert not torch.equal(unskipped, full)
    # a count larger than its segment
    out = torch.full((E, N, Kx), 3.0, dtype=torch.bfloat16, device=DEV)
    bad = _dev(np.array([300, 1, 129, 256], np.int32))
    assert mxk.device_error() == 0
    mxk.mxfp8_grouped_gemm_wgrad(gc, gs, xc, xs, _dev(off), pad, out=out, expert_rows=bad)
    assert mxk.device_error(reset=True) == 4
    assert (bf16_np(out) == 3.0).all()


@pytest.mark.parametrize("pad,N,Kx", [(128, 256, 256), (256, 384, 512), (256, 512, 768)])
def test_wgrad_random_vs_oracle(pad, N, Kx):
    g = synth.rng(5)
    E = 4
    off = _offsets([300, 0, 129, 60], pad)
    M = int(off[-1])
    G = _bf16(synth.normal(g, (M, N), 1e-2))
    X = _bf16(synth.normal(g, (M, Kx)))
    gc, gs = _mx_cols_dev(G)
    xc, xs = _mx_cols_dev(X)
    out = mxk.mxfp8_grouped_gemm_wgrad(gc, gs, xc, xs, _dev(off), pad)
    gcc, gcs = mx.quantize_cols(bf16_np(G))
    xcc, xcs = mx.quantize_cols(bf16_np(X))
    ref = mx.grouped_gemm_wgrad(gcc, gcs, xcc, xcs, off)
    assert_gemm_close(bf16_np(out), ref, "wgrad")
    assert (bf16_np(out)[1] == 0).all()


# ------------------------------------------------------------------ fused epilogues
@pytest.mark.parametrize("pad", [128, 256])
def test_fc1_swiglu_dual_quant_vs_oracle_and_standalone(pad):
    g = synth.rng(6)
    E, D, F = 3, 256, 384
    off = _offsets([200, 0, 140], pad)
    M = int(off[-1])
    x = _bf16(synth.normal(g, (M, D)))
    w13 = _bf16(synth.normal(g, (E, 2 * F, D), 0.05))
    xc, xs = _mx_rows_dev(x)
    wc, ws = _mx_rows_dev(w13.reshape(E * 2 * F, D))
    o = mxk.mxfp8_grouped_gemm_swiglu_quant(xc, xs, wc.reshape(E, 2 * F, D), ws, _dev(off), pad)
    # oracle: h13 per expert, then SwiGLU + dual quantization
    xr = mx.quantize_rows(bf16_np(x))
    wr = mx.quantize_weights_rows(bf16_np(w13))
    h13_ref = mx.round_to_bf16(mx.grouped_gemm(*xr, *wr, off))
    h13_got = bf16_np(o["h13"])
    assert_gemm_close(h13_got, h13_ref, "h13")
    rc, rs, cc, cs = mx.swiglu_quant(h13_ref)
    got_rs = mma_to_plain(u8(o["h_row_scales"]), M, F)
    got_cs = mma_to_plain(u8(o["h_col_scales"]), F, M)
    assert_codes_close(u8(o["h_row_codes"]), rc, got_rs, rs, "FC1 h ROW")
    assert_codes_close(u8(o["h_col_codes"]), cc, got_cs, cs, "FC1 h COL")
    # the fused epilogue equals the standalone SwiGLU cast of its own h13, bit for bit
    s = mxk.mxfp8_swiglu_quant(o["h13"], mxk.ROW | mxk.COL, mxk.MMA)
    for k in ("row_codes", "row_scales", "col_codes", "col_scales"):
        assert torch.equal(s[k].reshape(-1), o["h_" + k].reshape(-1)), k


@pytest.mark.parametrize("pad", [128, 256])
def test_fc2_dgrad_dswiglu_dual_quant_vs_oracle(pad):
    g = synth.rng(7)
    E, D, F = 3, 384, 256
    off = _offsets([150, 0, 250], pad)
    M = int(off[-1])
    dy = _bf16(synth.normal(g, (M, D), 1e-2))
    w2 = _bf16(synth.normal(g, (E, D, F), 0.05))
    h13 = _bf16(synth.normal(g, (M, 2 * F), 2.0))
    dr, ds = _mx_rows_dev(dy)
    w2t = mxk.mxfp8_quantize(w2.to(DEV), mxk.COL, mxk.MMA)        # [E, F, D]
    o = mxk.mxfp8_grouped_gemm_dswiglu_quant(dr, ds, w2t["col_codes"], w2t["col_scales"], _dev(off),
                                             h13.to(DEV), pad)
    dyr = mx.quantize_rows(bf16_np(dy))
    w2c = mx.quantize_weights_cols(bf16_np(w2))
    dh = mx.round_to_bf16(np.nan_to_num(mx.grouped_gemm(*dyr, *w2c, off)))
    dh13 = mx.dswiglu(dh, bf16_np(h13))
    dh13[off[-1]:] = 0
    rc, rs = mx.quantize_rows(dh13)
    cc, cs = mx.quantize_cols(dh13)
    got_rs = mma_to_plain(u8(o["g_row_scales"]), M, 2 * F)
    got_cs = mma_to_plain(u8(o["g_col_scales"]), 2 * F, M)
    assert_codes_close(u8(o["g_row_codes"]), rc, got_rs, rs, "dh13 ROW")
    assert_codes_close(u8(o["g_col_codes"]), cc, got_cs, cs, "dh13 COL")


def test_bounded_wait_times_out_and_reports():
    """A wait on a barrier nothing arrives on gives up (about 2 s), records
    MXMOE_ERR_DEVICE_TIMEOUT and leaves the context usable."""
    import ctypes
    L = mxk.lib()
    assert mxk.device_error() == 0
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.mxmoe_selftest_wait_timeout(st) == 0
    assert mxk.device_error(reset=True) == 7
    # the context still works
    x = torch.ones(128, 128, dtype=torch.bfloat16, device=DEV)
    o = mxk.mxfp8_quantize(x, mxk.ROW)
    assert (o["row_codes"] == 0x78).all()           # 1.0 under scale 2^-8 is 256 = E4M3 0x78
    assert mxk.device_error() == 0
