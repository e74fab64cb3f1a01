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


def _oracle_ragged_m(a_codes, a_scales, w_codes, w_scales):
    """Oracle grouped GEMM of one expert segment on given codes (plain scales)."""
    n = a_codes.shape[0]
    return mx.grouped_gemm(a_codes, a_scales, w_codes[None], w_scales[None], np.array([0, n]))


def _oracle_ragged_k(gt_codes, gt_scales, xt_codes, xt_scales):
    """Oracle weight-gradient GEMM of one expert segment on given COL codes."""
    n = gt_codes.shape[1]
    return mx.grouped_gemm_wgrad(gt_codes, gt_scales, xt_codes, xt_scales, np.array([0, n]))[0]


def _weight_codes_plain(qw, key, e, R, C):
    """Expert e's codes and plain scales out of a batched MMA-layout weight cast."""
    codes = u8(qw[key + "_codes"][e])
    per = R * C // 32
    flat = u8(qw[key + "_scales"][e * per:(e + 1) * per])
    return codes, mma_to_plain(flat, R, C)


def test_dsv3_full_size_prequantized_path_sampled_experts():
    """The configuration bench.py times: E=256, D=7168, F=2048, 16384 tokens
    top-8, Zipf(1.0), pad 256, inputs drawn on the device, one training step
    through mxmoe_quantize_weights + moe_mlp_fwd_q + moe_mlp_bwd_q.

    Checked, for the median-sized and the largest expert, without any bar
    fitted to a run:
    * the weight casts bit for bit (experts 0, E/2 and E-1 as well; E-1's
      codes lie past 2^32 bytes into the W13 buffers);
    * the composite equals the same step issued call by call, bit for bit,
      which exposes the operands the composites keep in their workspace;
    * each link of the chain against the oracle applied to that link's own
      inputs as the GPU produced them: every GEMM output at the GEMM bar on the
      operand codes it consumed (h13 on the exact x and W13 casts, so on the
      oracle's own chain; y on the GPU's h codes; dx and dW13 on its dh13
      codes; dW2 on its h codes), and each fused epilogue's codes at the fused
      bar (>= 99.9 % equal, the rest one code) on the GPU's h13 (SwiGLU; the
      dSwiGLU's dh GEMM runs on exact operands).  A code that may legitimately
      differ by one step, or an h13 one bf16 ulp off after fp32 accumulation,
      is not charged to the next link: near the zero of silu' a one-ulp h13
      moves dgate by more than one E4M3 step of its own size;
    * end to end against the oracle's own chain: relative Frobenius 2e-3.
    """
    inp = synth.device_moe_inputs("dsv3", 0, device=DEV)
    r = inp.routing
    off = torch.from_numpy(r.offsets).to(DEV)
    pad = inp.spec.pad
    M, E, D, F = r.M, inp.spec.E, inp.spec.D, inp.spec.F
    qw = mxk.mxmoe_quantize_weights(inp.w13, inp.w2)
    y, saved = mxk.moe_mlp_fwd_q(inp.x, qw, off, pad)
    dx, dw13, dw2 = mxk.moe_mlp_bwd_q(inp.dy, qw, off, saved, pad)
    torch.cuda.synchronize()
    assert mxk.device_error() == 0

    # the weight casts, bit for bit, per expert on the host
    counts = r.counts
    order = [int(e) for e in np.argsort(counts) if counts[e] > 0]
    sample = [order[len(order) // 2], order[-1]]
    for e in sorted({0, E // 2, E - 1} | set(sample)):
        w13_e, w2_e = bf16_np(inp.w13[e]), bf16_np(inp.w2[e])
        for key, ref, R, C in (("w13", mx.quantize_rows(w13_e), 2 * F, D), ("w13t", mx.quantize_cols(w13_e), D, 2 * F),
                               ("w2", mx.quantize_rows(w2_e), D, F), ("w2t", mx.quantize_cols(w2_e), F, D)):
            codes, scales = _weight_codes_plain(qw, key, e, R, C)
            np.testing.assert_array_equal(codes, ref[0], err_msg=f"{key} codes, expert {e}")
            np.testing.assert_array_equal(scales, ref[1], err_msg=f"{key} scales, expert {e}")

    # the same step call by call
    xq = mxk.mxfp8_quantize(inp.x, mxk.ROW | mxk.COL, mxk.MMA)
    f1 = mxk.mxfp8_grouped_gemm_swiglu_quant(xq["row_codes"], xq["row_scales"], qw["w13_codes"], qw["w13_scales"],
                                              off, pad)
    assert torch.equal(f1["h13"], saved["h13"]) and torch.equal(xq["col_codes"], saved["x_col_codes"])
    assert torch.equal(f1["h_col_codes"], saved["h_col_codes"])
    assert torch.equal(f1["h_col_scales"], saved["h_col_scales"])
    assert torch.equal(xq["col_scales"], saved["x_col_scales"])
    assert torch.equal(mxk.mxfp8_grouped_gemm(f1["h_row_codes"], f1["h_row_scales"], qw["w2_codes"], qw["w2_scales"],
                                              off, pad), y)
    del xq["row_codes"], xq["row_scales"]
    dyq = mxk.mxfp8_quantize(inp.dy, mxk.ROW | mxk.COL, mxk.MMA)
    g = mxk.mxfp8_grouped_gemm_dswiglu_quant(dyq["row_codes"], dyq["row_scales"], qw["w2t_codes"], qw["w2t_scales"],
                                             off, saved["h13"], pad)
    assert torch.equal(mxk.mxfp8_grouped_gemm(g["g_row_codes"], g["g_row_scales"], qw["w13t_codes"],
                                              qw["w13t_scales"], off, pad), dx)
    assert torch.equal(mxk.mxfp8_grouped_gemm_wgrad(g["g_col_codes"], g["g_col_scales"], xq["col_codes"],
                                                    xq["col_scales"], off, pad), dw13)
    assert torch.equal(mxk.mxfp8_grouped_gemm_wgrad(dyq["col_codes"], dyq["col_scales"], f1["h_col_codes"],
                                                    f1["h_col_scales"], off, pad), dw2)
    torch.cuda.synchronize()
    assert mxk.device_error() == 0

    # the fused epilogues' codes on the host, plain scales
    hr_c, hr_s = u8(f1["h_row_codes"]), mma_to_plain(u8(f1["h_row_scales"]), M, F)
    hc_c, hc_s = u8(f1["h_col_codes"]), mma_to_plain(u8(f1["h_col_scales"]), F, M)
    gr_c, gr_s = u8(g["g_row_codes"]), mma_to_plain(u8(g["g_row_scales"]), M, 2 * F)
    gc_c, gc_s = u8(g["g_col_codes"]), mma_to_plain(u8(g["g_col_scales"]), 2 * F, M)
    xcol = u8(saved["x_col_codes"])
    dycol = u8(dyq["col_codes"])
    for e in sample:
        lo, hi = int(r.offsets[e]), int(r.offsets[e + 1])
        b0, b1 = lo // 32, hi // 32
        x_e, dy_e = bf16_np(inp.x[lo:hi]), bf16_np(inp.dy[lo:hi])
        w13_e, w2_e = bf16_np(inp.w13[e]), bf16_np(inp.w2[e])
        rf = mx.expert_fwd(x_e, w13_e, w2_e)
        h13_e = bf16_np(saved["h13"][lo:hi])
        h_row = (hr_c[lo:hi], hr_s[lo:hi])
        h_col = (np.ascontiguousarray(hc_c[:, lo:hi]), np.ascontiguousarray(hc_s[:, b0:b1]))
        g_row = (gr_c[lo:hi], gr_s[lo:hi])
        g_col = (np.ascontiguousarray(gc_c[:, lo:hi]), np.ascontiguousarray(gc_s[:, b0:b1]))
        # the casts are exact
        np.testing.assert_array_equal(xcol[:, lo:hi], rf["x_col"][0])
        # FC1: exact operands -> the oracle's own h13
        assert_gemm_close(h13_e, rf["h13"], f"h13[e={e}]")
        # the SwiGLU epilogue on this h13
        sq = mx.swiglu_quant(h13_e)
        assert_codes_close(h_row[0], sq[0], h_row[1], sq[1], f"h ROW[e={e}]")
        assert_codes_close(h_col[0], sq[2], h_col[1], sq[3], f"h COL[e={e}]")
        # FC2 on the h codes it consumed
        assert_gemm_close(bf16_np(y[lo:hi]), _oracle_ragged_m(*h_row, *mx.quantize_rows(w2_e)), f"y[e={e}]")
        # backward on the saved tensors the GPU forward left (h13, h COL; x COL is exact)
        rb_on = mx.expert_bwd(dy_e, {"h13": h13_e, "h_col": h_col, "x_col": rf["x_col"]}, x_e, w13_e, w2_e)
        np.testing.assert_array_equal(dycol[:, lo:hi], rb_on["dy_col"][0])
        # the dSwiGLU epilogue (its dh GEMM on exact operands) on this h13
        assert_codes_close(g_row[0], rb_on["dh13_row"][0], g_row[1], rb_on["dh13_row"][1], f"dh13 ROW[e={e}]")
        assert_codes_close(g_col[0], rb_on["dh13_col"][0], g_col[1], rb_on["dh13_col"][1], f"dh13 COL[e={e}]")
        # dx, dW13 and dW2 on the codes they consumed
        assert_gemm_close(bf16_np(dx[lo:hi]), _oracle_ragged_m(*g_row, *mx.quantize_cols(w13_e)),
                          f"dx[e={e}] on the GPU's dh13 codes")
        assert_gemm_close(bf16_np(dw13[e]), _oracle_ragged_k(*g_col, *rf["x_col"]), f"dW13[e={e}] on the GPU's dh13 codes")
        assert_gemm_close(bf16_np(dw2[e]), rb_on["dw2"], f"dW2[e={e}] on the GPU's h codes")
        # end to end against the oracle's own chain
        rb = mx.expert_bwd(dy_e, rf, x_e, w13_e, w2_e)
        for what, got, ref in (("y", bf16_np(y[lo:hi]), rf["y"]), ("dx", bf16_np(dx[lo:hi]), rb["dx"]),
                               ("dW13", bf16_np(dw13[e]), rb["dw13"]), ("dW2", bf16_np(dw2[e]), rb["dw2"])):
            rf_, ma = assert_gemm_close(got, ref, f"{what}[e={e}] end to end", rel=2e-3, absf=np.inf)
            print(f"{what}[e={e}] end to end: rel Frobenius {rf_:.2e}, max abs {ma:.2e} of max|ref|")


def _full_mma(plain_full):
    """Plain [R, C/32] scales -> flat MMA-layout bytes on the device."""
    from mxtest import plain_to_mma
    return torch.from_numpy(plain_to_mma(plain_full)).to(DEV)


def test_dsv3_full_size_step_gemms_on_oracle_operands():
    """Each grouped GEMM of the step at the DSv3-scale launch configuration
    (full routing, M = 162,560 padded rows, E = 256) on operands the oracle
    quantized: one expert's rows/columns hold the oracle's codes and scales,
    every other expert's are zero.  The GPU result for that expert must meet
    the GEMM bar against the oracle's float64 product of the same codes."""
    spec = synth.SPECS["dsv3"]
    r = synth.make_routing(spec, 0)
    M, E, D, F = r.M, spec.E, spec.D, spec.F
    order = [int(e) for e in np.argsort(r.counts) if r.counts[e] > 0]
    e = order[len(order) // 2]
    lo, hi = int(r.offsets[e]), int(r.offsets[e + 1])
    n = hi - lo
    g = synth.rng(11)
    f = lambda a: synth.to_bf16(a).float().double().numpy()
    x_e = f(synth.normal(g, (n, D), 1.0, 1e-3, 50.0))
    x_e[int(r.counts[e]):] = 0.0                                   # pad rows
    dy_e = f(synth.normal(g, (n, D), 1e-2))
    dy_e[int(r.counts[e]):] = 0.0
    w13_e = f(synth.normal(g, (2 * F, D), spec.w_std))
    w2_e = f(synth.normal(g, (D, F), spec.w_std))
    rf = mx.expert_fwd(x_e, w13_e, w2_e)
    rb = mx.expert_bwd(dy_e, rf, x_e, w13_e, w2_e)
    off = torch.from_numpy(r.offsets).to(DEV)
    u8z = lambda *sh: np.zeros(sh, dtype=np.uint8)

    def rows_operand(codes_e, scales_e, K):           # [M, K] with rows lo:hi filled
        c, s_ = u8z(M, K), u8z(M, K // 32)
        c[lo:hi], s_[lo:hi] = codes_e, scales_e
        return torch.from_numpy(c).to(DEV), _full_mma(s_)

    def cols_operand(codes_e, scales_e, N):           # [N, M] with columns lo:hi filled
        c, s_ = u8z(N, M), u8z(N, M // 32)
        c[:, lo:hi], s_[:, lo // 32:hi // 32] = codes_e, scales_e
        return torch.from_numpy(c).to(DEV), _full_mma(s_)

    def weight_operand(codes_e, scales_e, N, K):      # [E, N, K] with expert e filled
        c, s_ = u8z(E, N, K), u8z(E * N, K // 32)
        c[e] = codes_e
        s_[e * N:(e + 1) * N] = scales_e
        return torch.from_numpy(c).to(DEV), _full_mma(s_)

    # a3: h13 = x_ROW . W13_ROW^T, SwiGLU + dual quant
    a, sa = rows_operand(*rf["x_row"], D)
    w, sw = weight_operand(*mx.quantize_rows(w13_e), 2 * F, D)
    o = mxk.mxfp8_grouped_gemm_swiglu_quant(a, sa, w, sw, off, spec.pad)
    assert_gemm_close(bf16_np(o["h13"][lo:hi]), rf["h13"], "h13 (a3)")
    rs = mma_to_plain(u8(o["h_row_scales"]), M, F)[lo:hi]
    assert_codes_close(u8(o["h_row_codes"])[lo:hi], rf["h_row"][0], rs, rf["h_row"][1], "h ROW (a3)")
    del a, sa, w, sw, o
    # a6: dh = dY_ROW . W2_COL, dSwiGLU with the oracle's h13, dual quant
    a, sa = rows_operand(*rb["dy_row"], D)
    w, sw = weight_operand(*mx.quantize_cols(w2_e), F, D)
    h13 = np.zeros((M, 2 * F), dtype=np.float32)
    h13[lo:hi] = rf["h13"]
    o = mxk.mxfp8_grouped_gemm_dswiglu_quant(a, sa, w, sw, off, synth.to_bf16(h13).to(DEV), spec.pad)
    gs_ = mma_to_plain(u8(o["g_row_scales"]), M, 2 * F)[lo:hi]
    assert_codes_close(u8(o["g_row_codes"])[lo:hi], rb["dh13_row"][0], gs_, rb["dh13_row"][1], "dh13 ROW (a6)")
    gcs = mma_to_plain(u8(o["g_col_scales"]), 2 * F, M)[:, lo // 32:hi // 32]
    assert_codes_close(u8(o["g_col_codes"])[:, lo:hi], rb["dh13_col"][0], gcs, rb["dh13_col"][1], "dh13 COL (a6)")
    del a, sa, w, sw, o, h13
    torch.cuda.empty_cache()
    # a4: y = h_ROW . W2_ROW^T
    a, sa = rows_operand(*rf["h_row"], F)
    w, sw = weight_operand(*mx.quantize_rows(w2_e), D, F)
    y = mxk.mxfp8_grouped_gemm(a, sa, w, sw, off, spec.pad)
    assert_gemm_close(bf16_np(y[lo:hi]), rf["y"], "y (a4)")
    del a, sa, w, sw, y
    # a8: dx = dh13_ROW . W13_COL (W13 COL codes stored [E, D, 2F])
    a, sa = rows_operand(*rb["dh13_row"], 2 * F)
    w, sw = weight_operand(*mx.quantize_cols(w13_e), D, 2 * F)
    dx = mxk.mxfp8_grouped_gemm(a, sa, w, sw, off, spec.pad)
    assert_gemm_close(bf16_np(dx[lo:hi]), rb["dx"], "dx (a8)")
    del a, sa, w, sw, dx
    torch.cuda.empty_cache()
    # a7: dW2 = dY_COL^T . h_COL ; a9: dW13 = dh13_COL^T . x_COL
    gt, gs = cols_operand(*rb["dy_col"], D)
    xt, xs = cols_operand(*rf["h_col"], F)
    dw2 = mxk.mxfp8_grouped_gemm_wgrad(gt, gs, xt, xs, off, spec.pad)
    assert_gemm_close(bf16_np(dw2[e]), rb["dw2"], "dW2 (a7)")
    del gt, gs, xt, xs, dw2
    torch.cuda.empty_cache()
    gt, gs = cols_operand(*rb["dh13_col"], 2 * F)
    xt, xs = cols_operand(*rf["x_col"], D)
    dw13 = mxk.mxfp8_grouped_gemm_wgrad(gt, gs, xt, xs, off, spec.pad)
    assert_gemm_close(bf16_np(dw13[e]), rb["dw13"], "dW13 (a9)")
    assert mxk.device_error() == 0


@pytest.mark.parametrize("name", ["tiny", "dsv3_16b"])
def test_unfused_plan_forward_equals_fused_bitwise(name):
    """The unfused "swiglu" plan (FC1 -> bf16 h13 in HBM -> standalone SwiGLU +
    dual quant -> FC2) and the fused FC1 epilogue give the same bits
    (SwiGLU-boundary page: fused forward bitwise equal to the standalone cast)."""
    inp = synth.make_moe_inputs(name, 5)
    off = torch.from_numpy(inp.routing.offsets).to(DEV)
    pad = inp.spec.pad
    x, w13, w2 = inp.x.to(DEV), inp.w13.to(DEV), inp.w2.to(DEV)
    qw = mxk.mxmoe_quantize_weights(w13, w2)
    yf, sf = mxk.moe_mlp_fwd_q(x, qw, off, pad)
    yu, su = mxk.moe_mlp_fwd_unfused_q(x, qw, off, pad)
    torch.cuda.synchronize()
    M = int(inp.routing.offsets[-1])
    assert torch.equal(yf[:M], yu[:M])
    assert torch.equal(sf["h13"][:M], su["h13"][:M])
    for k in ("h_col_codes", "h_col_scales", "x_col_codes", "x_col_scales"):
        assert torch.equal(sf[k], su[k]), k


def test_dense_feedforward_is_the_one_expert_case():
    """E = 1 (a dense SwiGLU FeedForward in MXFP8) against the oracle."""
    spec = synth.Spec("dense", 1, 256, 384, 300, 1, 128, None, 0, 0.05)
    inp = synth.make_moe_inputs(spec, 6)
    y, saved, dx, dw13, dw2 = _run(inp)
    x, w13, w2, dy = _np(inp)
    off = inp.routing.offsets
    rf = mx.moe_mlp_fwd(x, w13, w2, off)
    rb = mx.moe_mlp_bwd(dy, rf, x, w13, w2, off)
    assert_gemm_close(bf16_np(y), rf["y"], "y")
    assert_gemm_close(bf16_np(dx), rb["dx"], "dx")
    assert_gemm_close(bf16_np(dw13), rb["dw13"], "dw13")
    assert_gemm_close(bf16_np(dw2), rb["dw2"], "dw2")


def _sqnr_db(x, ref):
    err = np.linalg.norm(np.asarray(x, dtype=np.float64) - ref)
    return float(20.0 * np.log10(np.linalg.norm(ref) / max(err, 1e-300)))


@pytest.mark.parametrize("name", ["tiny", "dsv3_16b"])
def test_sqnr_against_the_unquantized_layer_tracks_the_oracle(name):
    # SQNR tracking (SwiGLU-boundary page, "Numerics and tests"): the GPU
    # MXFP8 outputs, measured against the same layer without quantization
    # (oracle exact mode, float64), lose no more signal than the oracle's own
    # MXFP8 arithmetic does: within 0.3 dB of it, and above 20 dB.
    spec = synth.SPECS[name]
    inp = synth.make_moe_inputs(spec, 3)
    y, saved, dx, dw13, dw2 = _run(inp)
    x, w13, w2, dy = _np(inp)
    off = inp.routing.offsets
    experts = None if name == "tiny" else sorted(int(e) for e in np.argsort(-inp.routing.counts)[:2])
    segs = ([(e, off[e], off[e + 1]) for e in experts] if experts else [(None, 0, int(off[-1]))])
    f_mx = mx.moe_mlp_fwd(x, w13, w2, off, experts)
    b_mx = mx.moe_mlp_bwd(dy, f_mx, x, w13, w2, off, experts)
    f_ex = mx.moe_mlp_fwd(x, w13, w2, off, experts, exact=True)
    b_ex = mx.moe_mlp_bwd(dy, f_ex, x, w13, w2, off, experts, exact=True)
    rows = np.concatenate([np.arange(lo, hi) for _, lo, hi in segs])
    ex = slice(None) if experts is None else experts
    for what, got, mxv, exv in (
            ("y", bf16_np(y)[rows], f_mx["y"][rows], f_ex["y"][rows]),
            ("dx", bf16_np(dx)[rows], b_mx["dx"][rows], b_ex["dx"][rows]),
            ("dW13", bf16_np(dw13)[ex], b_mx["dw13"][ex], b_ex["dw13"][ex]),
            ("dW2", bf16_np(dw2)[ex], b_mx["dw2"][ex], b_ex["dw2"][ex])):
        s_gpu, s_oracle = _sqnr_db(got, exv), _sqnr_db(mxv, exv)
        assert s_gpu >= 20.0, f"{what}: SQNR {s_gpu:.1f} dB"
        assert s_gpu >= s_oracle - 0.3, f"{what}: GPU {s_gpu:.2f} dB vs oracle MXFP8 {s_oracle:.2f} dB"


def _kernels_launched(fn):
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    return [n for n in names if "grouped_gemm" in n or "mx_" in n or "route_" in n or "combine" in n]


def test_kernel_launch_counts():
    # op-count contract (SwiGLU-boundary page, "Numerics and tests": profiler
    # op-count contracts; "Summary": the fused boundary replaces the 6 + 6
    # standalone casts): forward = x cast, FC1 with the fused SwiGLU + dual
    # quant, FC2; the unfused plan adds one standalone SwiGLU cast; backward =
    # dY cast, FC2 dgrad with the fused dSwiGLU + dual quant, dW2, dx, dW13.
    inp = synth.make_moe_inputs("tiny", 0)
    off = torch.from_numpy(inp.routing.offsets).to(DEV)
    pad = inp.spec.pad
    x, w13, w2, dy = (t.to(DEV) for t in (inp.x, inp.w13, inp.w2, inp.dy))
    qw = mxk.mxmoe_quantize_weights(w13, w2)
    y, saved = mxk.moe_mlp_fwd_q(x, qw, off, pad)
    fwd = _kernels_launched(lambda: mxk.moe_mlp_fwd_q(x, qw, off, pad, y=y, saved=saved))
    unf = _kernels_launched(lambda: mxk.moe_mlp_fwd_unfused_q(x, qw, off, pad, y=y, saved=saved))
    bwd = _kernels_launched(lambda: mxk.moe_mlp_bwd_q(dy, qw, off, saved, pad))
    assert len(fwd) == 3 and sum("mx_cast" in n for n in fwd) == 1, fwd
    assert len(unf) == 4 and sum("mx_cast" in n for n in unf) == 2, unf
    assert len(bwd) == 5 and sum("mx_cast" in n for n in bwd) == 1, bwd
    # the token-major layer: 3 routing kernels, gather + cast, FC1, FC2, combine;
    # backward: gather + cast, 4 GEMMs, unpermute, router-weight gradient
    spec = inp.spec
    tk = torch.from_numpy(inp.routing.topk).to(DEV)
    wt = torch.from_numpy(synth.router_weights(spec.tokens, spec.top_k)).to(DEV)
    xt = torch.randn(spec.tokens, spec.D, device=DEV).to(torch.bfloat16)
    out, ls = mxk.moe_layer_fwd_q(xt, tk, wt, qw, pad)
    lf = _kernels_launched(lambda: mxk.moe_layer_fwd_q(xt, tk, wt, qw, pad, out=out, saved=ls))
    lb = _kernels_launched(lambda: mxk.moe_layer_bwd_q(xt, wt, qw, ls, pad))
    assert len(lf) == 7 and sum("route_" in n for n in lf) == 3, lf
    assert len(lb) == 7 and sum("combine" in n for n in lb) == 2, lb
    assert mxk.device_error() == 0
