"""GPU parity of the moe_mlp_fwd / moe_mlp_bwd composites against the oracle."""
import numpy as np
import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk
import synth
from oracle import mx
from mxtest import assert_gemm_close, bf16_np, mma_to_plain, u8, assert_codes_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(inp):
    off = torch.from_numpy(inp.routing.offsets).to(DEV)
    pad = inp.spec.pad
    x, w13, w2, dy = (t.to(DEV) for t in (inp.x, inp.w13, inp.w2, inp.dy))
    y, saved = mxk.moe_mlp_fwd(x, w13, w2, off, pad)
    dx, dw13, dw2 = mxk.moe_mlp_bwd(dy, w13, w2, off, saved, pad)
    torch.cuda.synchronize()
    assert mxk.device_error() == 0
    return y, saved, dx, dw13, dw2


def _np(inp):
    return (bf16_np(inp.x), bf16_np(inp.w13), bf16_np(inp.w2), bf16_np(inp.dy))


def _compare_expert(e, lo, hi, ref_f, ref_b, y, saved, dx, dw13, dw2, M, F, D):
    assert_gemm_close(bf16_np(y[lo:hi]), ref_f["y"], f"y[e={e}]")
    assert_gemm_close(bf16_np(saved["h13"][lo:hi]), ref_f["h13"], f"h13[e={e}]")
    assert_gemm_close(bf16_np(dx[lo:hi]), ref_b["dx"], f"dx[e={e}]")
    assert_gemm_close(bf16_np(dw13[e]), ref_b["dw13"], f"dw13[e={e}]")
    assert_gemm_close(bf16_np(dw2[e]), ref_b["dw2"], f"dw2[e={e}]")
    # the saved COL-quantized x is exact; the saved h codes meet the fused bar
    xcc = u8(saved["x_col_codes"])[:, lo:hi]
    xcs = mma_to_plain(u8(saved["x_col_scales"]), D, M)[:, lo // 32:hi // 32]
    np.testing.assert_array_equal(xcc, ref_f["x_col"][0])
    np.testing.assert_array_equal(xcs, ref_f["x_col"][1])
    hcc = u8(saved["h_col_codes"])[:, lo:hi]
    hcs = mma_to_plain(u8(saved["h_col_scales"]), F, M)[:, lo // 32:hi // 32]
    assert_codes_close(hcc, ref_f["h_col"][0], hcs, ref_f["h_col"][1], f"h COL[e={e}]")


def test_tiny_fwd_bwd_all_experts():
    """E=4, D=F=256, 512 tokens, top-2 uniform, pad 128 (every element compared)."""
    inp = synth.make_moe_inputs("tiny", 0)
    y, saved, dx, dw13, dw2 = _run(inp)
    x, w13, w2, dy = _np(inp)
    off = inp.routing.offsets
    rf = mx.moe_mlp_fwd(x, w13, w2, off)
    rb = mx.moe_mlp_bwd(dy, rf, x, w13, w2, off)
    M, D = x.shape
    F = w13.shape[1] // 2
    assert_gemm_close(bf16_np(y), rf["y"], "y")
    assert_gemm_close(bf16_np(dx), rb["dx"], "dx")
    assert_gemm_close(bf16_np(dw13), rb["dw13"], "dw13")
    assert_gemm_close(bf16_np(dw2), rb["dw2"], "dw2")
    for e in rf["experts"]:
        lo, hi = int(off[e]), int(off[e + 1])
        _compare_expert(e, lo, hi, rf["experts"][e], rb["experts"][e], y, saved, dx, dw13, dw2, M, F, D)


def test_zero_token_experts_exact_zero_grads_and_pad_rows():
    spec = synth.Spec("zero", 4, 256, 256, 400, 1, 128, None, 0, 0.02)
    inp = synth.make_moe_inputs(spec, 1, counts_override=[0, 250, 0, 150])
    y, saved, dx, dw13, dw2 = _run(inp)
    for e in (0, 2):
        assert (bf16_np(dw13[e]) == 0).all() and (bf16_np(dw2[e]) == 0).all()
    pad = inp.routing.src_token < 0
    assert (bf16_np(y)[pad] == 0).all() and (bf16_np(dx)[pad] == 0).all()


def test_zero_routed_tokens_backward():
    """No token routed anywhere: the forward writes nothing, all grads are zero."""
    spec = synth.Spec("none", 3, 256, 256, 0, 1, 128, None, 0, 0.02)
    inp = synth.make_moe_inputs(spec, 2, counts_override=[0, 0, 0])
    M = 128
    off = torch.zeros(4, dtype=torch.int32, device=DEV)
    x = torch.zeros(M, 256, dtype=torch.bfloat16, device=DEV)
    w13, w2 = inp.w13.to(DEV), inp.w2.to(DEV)
    y = torch.full((M, 256), 5.0, dtype=torch.bfloat16, device=DEV)
    y, saved = mxk.moe_mlp_fwd(x, w13, w2, off, 128, y=y)
    dx = torch.full_like(x, 5.0)
    dx, dw13, dw2 = mxk.moe_mlp_bwd(x, w13, w2, off, saved, 128, dx=dx)
    torch.cuda.synchronize()
    assert (bf16_np(y) == 5.0).all() and (bf16_np(dx) == 5.0).all()
    assert (bf16_np(dw13) == 0).all() and (bf16_np(dw2) == 0).all()
    assert mxk.device_error() == 0


def test_pad128_vs_pad256_same_real_rows():
    s128 = synth.Spec("p", 4, 256, 256, 300, 2, 128, None, 0, 0.02)
    s256 = synth.Spec("p", 4, 256, 256, 300, 2, 256, None, 0, 0.02)
    a, b = synth.make_moe_inputs(s128, 3), synth.make_moe_inputs(s256, 3)
    ra, rb = _run(a), _run(b)
    ma, mb = a.routing.src_token >= 0, b.routing.src_token >= 0
    assert torch.equal(ra[0][torch.from_numpy(ma).to(DEV)], rb[0][torch.from_numpy(mb).to(DEV)])
    assert torch.equal(ra[2][torch.from_numpy(ma).to(DEV)], rb[2][torch.from_numpy(mb).to(DEV)])
    assert torch.equal(ra[3], rb[3]) and torch.equal(ra[4], rb[4])


def test_dsv3_16b_full_size_sampled_experts():
    """E=64, D=2048, F=1408, 8192 tokens top-6, Zipf(1.1), pad 256: the heaviest,
    the median and a zero-token expert checked against the oracle."""
    inp = synth.make_moe_inputs("dsv3_16b", 0)
    y, saved, dx, dw13, dw2 = _run(inp)
    counts = inp.routing.counts
    order = np.argsort(counts)
    zero = [int(e) for e in np.nonzero(counts == 0)[0]]
    assert len(zero) >= 2
    nz = [int(e) for e in order if counts[e] > 0]
    sample = [nz[-1], nz[len(nz) // 2]]
    off = inp.routing.offsets
    x, w13, w2, dy = _np(inp)
    M, D = x.shape
    F = w13.shape[1] // 2
    for e in sample:
        lo, hi = int(off[e]), int(off[e + 1])
        rf = mx.expert_fwd(x[lo:hi], w13[e], w2[e])
        rb = mx.expert_bwd(dy[lo:hi], rf, x[lo:hi], w13[e], w2[e])
        _compare_expert(e, lo, hi, rf, rb, y, saved, dx, dw13, dw2, M, F, D)
    for e in zero:
        assert (bf16_np(dw13[e]) == 0).all() and (bf16_np(dw2[e]) == 0).all()


def test_prequantized_weights_path_matches_bf16_weight_composites():
    """mxmoe_quantize_weights + the _q composites give the same bits as the
    composites that cast the bf16 weights themselves."""
    inp = synth.make_moe_inputs("tiny", 4)
    y, saved, dx, dw13, dw2 = _run(inp)
    off = torch.from_numpy(inp.routing.offsets).to(DEV)
    pad = inp.spec.pad
    x, w13, w2, dy = (t.to(DEV) for t in (inp.x, inp.w13, inp.w2, inp.dy))
    qw = mxk.mxmoe_quantize_weights(w13, w2)
    yq, sq = mxk.moe_mlp_fwd_q(x, qw, off, pad)
    dxq, dw13q, dw2q = mxk.moe_mlp_bwd_q(dy, qw, off, sq, pad)
    torch.cuda.synchronize()
    for a, b in ((y, yq), (dx, dxq), (dw13, dw13q), (dw2, dw2q), (saved["h13"], sq["h13"])):
        assert torch.equal(a, b)
    # the dual weight cast equals the separate ROW and COL casts
    E, F2, D = w13.shape
    r = mxk.mxfp8_quantize(w13, mxk.ROW | mxk.COL, mxk.MMA)
    assert torch.equal(r["row_codes"].reshape(-1), qw["w13_codes"].reshape(-1))
    assert torch.equal(r["col_codes"].reshape(-1), qw["w13t_codes"].reshape(-1))
    assert torch.equal(r["row_scales"], qw["w13_scales"]) and torch.equal(r["col_scales"], qw["w13t_scales"])
