"""GPU parity of the token dispatcher (route, gather + quantize, combine and its
weight gradient) against oracle.routing.

Layout construction is integer work: offsets, row_slot and slot_row must
equal the oracle's exactly.  The gather + quantize is a cast of gathered (and
for the backward, weight-scaled) rows: bit-exact codes and scales.  The
combine sums k fp32 products and rounds once to bf16; its bar is
|got - ref| <= 2^-8 |ref| + 2^-20 sum_j |w_j y_j| per element (one bf16
rounding plus the fp32 accumulation of at most 64 terms).  The weight
gradient is an fp32 dot product of D terms: |got - ref| <= 2^-14 sum |dout y|.
"""
import numpy as np
import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk
import synth
from oracle import mx, routing
from mxtest import assert_gemm_close, bf16_np, mma_to_plain, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _route_gpu(topk, E, pad, m_cap=None):
    out = mxk.mxmoe_route(torch.from_numpy(np.ascontiguousarray(topk, dtype=np.int32)).to(DEV), E, pad, m_cap)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy().astype(np.int64) for k, v in out.items()}


def _assert_route_equal(topk, E, pad):
    ref = routing.route(topk, E, pad)
    got = _route_gpu(topk, E, pad)
    M = int(ref["offsets"][-1])
    np.testing.assert_array_equal(got["offsets"], ref["offsets"])
    np.testing.assert_array_equal(got["row_slot"][:M], ref["row_slot"])
    assert (got["row_slot"][M:] == -1).all()
    np.testing.assert_array_equal(got["slot_row"], ref["slot_row"])
    assert mxk.device_error() == 0
    return ref, got


@pytest.mark.parametrize("name", ["tiny", "dsv3_16b", "dsv3"])
def test_route_matches_oracle_on_workloads(name):
    spec = synth.SPECS[name]
    topk = synth.make_routing(spec).topk
    _assert_route_equal(topk, spec.E, spec.pad)


@pytest.mark.parametrize("T,k,E,pad,zipf", [
    (300, 4, 16, 32, None),     # ragged last chunk
    (4096, 1, 3, 128, 2.0),     # exactly one chunk
    (9000, 8, 1024, 128, 1.0),  # E at the maximum: the large shared-memory path
    (5000, 1, 1, 256, None),    # one expert: the dense case (top-1)
    (20000, 6, 64, 256, 3.0),   # most slots on a few experts
])
def test_route_matches_oracle_random(T, k, E, pad, zipf):
    assert k <= E
    topk = synth.topk_ids(T, k, E, seed=T + E, zipf_s=zipf) if E > 1 else np.zeros((T, 1), np.int32)
    _assert_route_equal(topk, E, pad)


def test_route_empty_and_overflow_and_bad_ids():
    # no tokens: all offsets zero, every row a pad row
    got = _route_gpu(np.zeros((0, 2), np.int32), 4, 128, m_cap=256)
    np.testing.assert_array_equal(got["offsets"], 0)
    assert (got["row_slot"] == -1).all()
    # a capacity too small for the routing: flagged, nothing written out of range
    topk = np.zeros((300, 1), np.int32)
    got = _route_gpu(topk, 2, 128, m_cap=128)
    assert mxk.device_error() == 2
    assert got["offsets"][-1] == 384
    np.testing.assert_array_equal(got["row_slot"], np.arange(128))
    # an id outside [0, E)
    topk = np.array([[0, 1], [1, 7]], np.int32)
    got = _route_gpu(topk, 4, 32, m_cap=128)
    assert mxk.device_error() == 9
    assert got["slot_row"][3] == -1
    np.testing.assert_array_equal(got["offsets"], [0, 32, 64, 64, 64])


def _x_tokens(T, D, seed, outliers=0.0):
    return synth.to_bf16(synth.normal(synth.rng(seed), (T, D), 1.0, outliers, 50.0))


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("layout", [mxk.PLAIN, mxk.MMA])
def test_permute_quant_matches_oracle(weighted, layout):
    T, k, E, D, pad = 700, 3, 5, 256, 128
    topk = synth.topk_ids(T, k, E, seed=11)
    r = routing.route(topk, E, pad)
    m_cap = mxk.mxmoe_route_capacity(T, k, E, pad)
    row_slot = np.full(m_cap, -1, np.int64)
    row_slot[:len(r["row_slot"])] = r["row_slot"]
    x = _x_tokens(T, D, 12, 1e-3)
    w = synth.router_weights(T, k, seed=3) if weighted else None
    out = mxk.mxmoe_permute_quant(x.to(DEV), torch.from_numpy(row_slot.astype(np.int32)).to(DEV), k,
                                  None if w is None else torch.from_numpy(w).to(DEV), scale_layout=layout)
    torch.cuda.synchronize()
    rc, rs, cc, cs = routing.permute_quant(bf16_np(x), row_slot, k, w)
    np.testing.assert_array_equal(u8(out["row_codes"]), rc)
    np.testing.assert_array_equal(u8(out["col_codes"]), cc)
    if layout == mxk.PLAIN:
        np.testing.assert_array_equal(u8(out["row_scales"]), rs)
        np.testing.assert_array_equal(u8(out["col_scales"]), cs)
    else:
        np.testing.assert_array_equal(mma_to_plain(u8(out["row_scales"]), m_cap, D), rs)
        np.testing.assert_array_equal(mma_to_plain(u8(out["col_scales"]), D, m_cap), cs)
    assert mxk.device_error() == 0


@pytest.mark.parametrize("layout", [mxk.PLAIN, mxk.MMA])
def test_permute_quant_respects_the_device_row_limit(layout):
    # pad 32: the layout ends inside a 128-row tile; nothing at or past the
    # limit (codes or scales) may be written
    T, k, E, D, pad = 200, 2, 5, 128, 32
    topk = synth.topk_ids(T, k, E, seed=4)
    rt = mxk.mxmoe_route(torch.from_numpy(topk).to(DEV), E, pad)
    M = int(rt["offsets"][-1].item())
    m_cap = rt["row_slot"].numel()
    assert M % 128 != 0
    x = _x_tokens(T, D, 5).to(DEV)
    bufs = [torch.full((m_cap * D,), 0xAB, dtype=torch.uint8, device=DEV) for _ in range(2)]
    scl = [torch.full((m_cap * D // 32,), 0xAB, dtype=torch.uint8, device=DEV) for _ in range(2)]
    L = mxk.lib()
    p = lambda t: t.data_ptr()
    st = torch.cuda.current_stream().cuda_stream
    assert L.mxmoe_permute_quant(p(x), T, D, p(rt["row_slot"]), k, None, m_cap, p(rt["offsets"][E:]), 3, layout,
                                 p(bufs[0]), p(scl[0]), p(bufs[1]), p(scl[1]), st) == 0
    torch.cuda.synchronize()
    ref = routing.route(topk, E, pad)
    rc, rs, cc, cs = routing.permute_quant(bf16_np(x.cpu()), ref["row_slot"], k)
    grc = u8(bufs[0]).reshape(m_cap, D)
    gcc = u8(bufs[1]).reshape(D, m_cap)
    np.testing.assert_array_equal(grc[:M], rc)
    np.testing.assert_array_equal(gcc[:, :M], cc)
    assert (grc[M:] == 0xAB).all() and (gcc[:, M:] == 0xAB).all()
    if layout == mxk.PLAIN:
        grs, gcs = u8(scl[0]).reshape(m_cap, D // 32), u8(scl[1]).reshape(D, m_cap // 32)
    else:
        grs, gcs = mma_to_plain(u8(scl[0]), m_cap, D), mma_to_plain(u8(scl[1]), D, m_cap)
    np.testing.assert_array_equal(grs[:M], rs)
    np.testing.assert_array_equal(gcs[:, :M // 32], cs)
    assert (grs[M:] == 0xAB).all() and (gcs[:, M // 32:] == 0xAB).all()


def test_permute_quant_full_size_sampled():
    # DSv3 layer: 16384 tokens x top-8 over 256 experts, D = 7168, pad 256;
    # 12 sampled 32-row blocks (ROW rows and COL blocks are self-contained)
    spec = synth.SPECS["dsv3"]
    topk = synth.make_routing(spec).topk
    T, k, D = spec.tokens, spec.top_k, spec.D
    gen = torch.Generator(device=DEV)
    gen.manual_seed(21)
    x = torch.randn(T, D, generator=gen, device=DEV).to(torch.bfloat16)
    w = synth.router_weights(T, k, seed=2)
    rt = mxk.mxmoe_route(torch.from_numpy(topk).to(DEV), spec.E, spec.pad)
    row_slot = rt["row_slot"].cpu().numpy().astype(np.int64)
    m_cap = len(row_slot)
    M = int(rt["offsets"][-1].item())
    blocks = np.random.default_rng(0).choice(M // 32, size=12, replace=False)
    for weighted in (False, True):
        wt = torch.from_numpy(w).to(DEV) if weighted else None
        out = mxk.mxmoe_permute_quant(x, rt["row_slot"], k, wt, rows_dev=rt["offsets"][spec.E:])
        torch.cuda.synchronize()
        grs = mma_to_plain(u8(out["row_scales"]), m_cap, D)
        gcs = mma_to_plain(u8(out["col_scales"]), D, m_cap)
        for b in blocks:
            rows = np.arange(b * 32, b * 32 + 32)
            s = row_slot[rows]
            toks = np.unique(s[s >= 0] // k)
            # the block's tokens as a compact table, slots renumbered into it
            idx = {int(t): i for i, t in enumerate(toks)}
            s2 = np.array([-1 if v < 0 else idx[int(v // k)] * k + int(v % k) for v in s])
            x2 = bf16_np(x[torch.from_numpy(toks).to(DEV)]) if len(toks) else np.zeros((0, D))
            w2 = w[toks] if weighted else None
            rc, rs, cc, cs = routing.permute_quant(x2, s2, k, w2)
            np.testing.assert_array_equal(u8(out["row_codes"][b * 32:(b + 1) * 32]), rc)
            np.testing.assert_array_equal(grs[rows], rs)
            np.testing.assert_array_equal(u8(out["col_codes"][:, b * 32:(b + 1) * 32]), cc)
            np.testing.assert_array_equal(gcs[:, b:b + 1], cs)
    assert mxk.device_error() == 0


def _combine_bound(y, slot_row, T, k, w):
    ww = np.ones((T, k)) if w is None else w.astype(np.float64)
    return routing.unpermute_combine(np.abs(y), slot_row, T, k, np.abs(ww))


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("T,k,E,D", [(300, 4, 16, 256), (64, 1, 3, 7168), (1000, 8, 32, 1024)])
def test_combine_and_weight_grad_match_oracle(weighted, T, k, E, D):
    topk = synth.topk_ids(T, k, E, seed=T)
    r = routing.route(topk, E, 128)
    M = len(r["row_slot"])
    y = synth.to_bf16(synth.normal(synth.rng(T + 1), (M, D)))
    dout = synth.to_bf16(synth.normal(synth.rng(T + 2), (T, D)))
    w = synth.router_weights(T, k, seed=T) if weighted else None
    sr = torch.from_numpy(r["slot_row"].astype(np.int32)).to(DEV)
    wt = None if w is None else torch.from_numpy(w).to(DEV)
    out = mxk.mxmoe_unpermute_combine(y.to(DEV), sr, k, wt)
    dw = mxk.mxmoe_combine_weight_grad(dout.to(DEV), y.to(DEV), sr, k)
    torch.cuda.synchronize()
    yn, dn = bf16_np(y), bf16_np(dout)
    ref = routing.unpermute_combine(yn, r["slot_row"], T, k, w)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * _combine_bound(yn, r["slot_row"], T, k, w)
    assert (np.abs(bf16_np(out) - ref) <= bound).all()
    dref = routing.combine_weight_grad(dn, yn, r["slot_row"], T, k)
    dbound = 2.0 ** -14 * routing.combine_weight_grad(np.abs(dn), np.abs(yn), r["slot_row"], T, k) + 1e-30
    assert (np.abs(dw.cpu().numpy() - dref) <= dbound).all()
    assert mxk.device_error() == 0


def test_layer_forward_routes_runs_the_mlp_and_combines():
    # tokens -> route -> gather + quantize -> FC1 + SwiGLU + quant -> FC2 -> combine
    spec = synth.SPECS["tiny"]
    T, k, E, D, F, pad = spec.tokens, spec.top_k, spec.E, spec.D, spec.F, spec.pad
    topk = synth.make_routing(spec).topk
    g = synth.rng(31)
    x = synth.to_bf16(synth.normal(g, (T, D)))
    w13 = synth.to_bf16(synth.normal(g, (E, 2 * F, D), spec.w_std))
    w2 = synth.to_bf16(synth.normal(g, (E, D, F), spec.w_std))
    wr = synth.router_weights(T, k, seed=31)
    rt = mxk.mxmoe_route(torch.from_numpy(topk).to(DEV), E, pad)
    qx = mxk.mxmoe_permute_quant(x.to(DEV), rt["row_slot"], k, rows_dev=rt["offsets"][E:])
    qw = mxk.make_qweights(E, D, F, DEV)
    mxk.mxmoe_quantize_weights(w13.to(DEV), w2.to(DEV), qw)
    o1 = mxk.mxfp8_grouped_gemm_swiglu_quant(qx["row_codes"], qx["row_scales"], qw["w13_codes"],
                                             qw["w13_scales"], rt["offsets"], pad)
    y = mxk.mxfp8_grouped_gemm(o1["h_row_codes"], o1["h_row_scales"], qw["w2_codes"], qw["w2_scales"],
                               rt["offsets"], pad)
    out = mxk.mxmoe_unpermute_combine(y, rt["slot_row"], k, torch.from_numpy(wr).to(DEV))
    torch.cuda.synchronize()
    assert mxk.device_error() == 0
    r = routing.route(topk, E, pad)
    xr = routing.permute(bf16_np(x), r["row_slot"], k)
    fwd = mx.moe_mlp_fwd(xr, bf16_np(w13), bf16_np(w2), r["offsets"])
    # the FC2 output is bf16 at the GEMM boundary: the combine reads bf16 y
    ref = routing.unpermute_combine(mx.round_to_bf16(fwd["y"]), r["slot_row"], T, k, wr)
    assert_gemm_close(bf16_np(out), ref, "layer output")


def _layer_inputs(spec, seed):
    g = synth.rng(seed)
    T, k, E, D, F = spec.tokens, spec.top_k, spec.E, spec.D, spec.F
    topk = synth.make_routing(spec).topk
    x = synth.to_bf16(synth.normal(g, (T, D)))
    w13 = synth.to_bf16(synth.normal(g, (E, 2 * F, D), spec.w_std))
    w2 = synth.to_bf16(synth.normal(g, (E, D, F), spec.w_std))
    dout = synth.to_bf16(synth.normal(g, (T, D), spec.dy_std))
    wr = synth.router_weights(T, k, seed=seed)
    return topk, x, w13, w2, dout, wr


def test_layer_composites_match_oracle_tiny():
    spec = synth.SPECS["tiny"]
    topk, x, w13, w2, dout, wr = _layer_inputs(spec, 41)
    qw = mxk.mxmoe_quantize_weights(w13.to(DEV), w2.to(DEV))
    tk, wt = torch.from_numpy(topk).to(DEV), torch.from_numpy(wr).to(DEV)
    out, saved = mxk.moe_layer_fwd_q(x.to(DEV), tk, wt, qw, spec.pad)
    dx, dw13, dw2, dwr = mxk.moe_layer_bwd_q(dout.to(DEV), wt, qw, saved, spec.pad)
    torch.cuda.synchronize()
    assert mxk.device_error() == 0
    xn, w13n, w2n, dn = bf16_np(x), bf16_np(w13), bf16_np(w2), bf16_np(dout)
    f = routing.layer_fwd(xn, topk, wr, w13n, w2n, spec.E, spec.pad)
    b = routing.layer_bwd(dn, f, xn, topk, wr, w13n, w2n, spec.pad)
    M = int(f["route"]["offsets"][-1])
    np.testing.assert_array_equal(saved["offsets"].cpu().numpy(), f["route"]["offsets"])
    np.testing.assert_array_equal(saved["row_slot"].cpu().numpy()[:M], f["route"]["row_slot"])
    np.testing.assert_array_equal(saved["slot_row"].cpu().numpy(), f["route"]["slot_row"])
    assert_gemm_close(bf16_np(out), f["out"], "layer out")
    assert_gemm_close(bf16_np(dx), b["dx"], "layer dx")
    assert_gemm_close(bf16_np(dw13), b["dw13"], "layer dW13")
    assert_gemm_close(bf16_np(dw2), b["dw2"], "layer dW2")
    assert_gemm_close(dwr.cpu().numpy(), b["dweights"], "layer router-weight gradient")


@pytest.mark.parametrize("name", ["dsv3_16b", "dsv3"])
def test_layer_composites_equal_the_row_composites_bitwise(name):
    # the token-major layer = (torch gather) + the row-level composites +
    # combine, bit for bit, at the DSv3-16B-like size and at the DSv3 size the
    # end-to-end measurement runs (there with device-drawn inputs)
    spec = synth.SPECS[name]
    T, k, E, D, F = spec.tokens, spec.top_k, spec.E, spec.D, spec.F
    if name == "dsv3":
        dinp = synth.device_moe_inputs(spec, 43, device=DEV)
        topk, w13, w2 = dinp.routing.topk, dinp.w13, dinp.w2
        x = dinp.x_tok
        del dinp
        gen = torch.Generator(device=DEV)
        gen.manual_seed(44)
        dout = (torch.randn(T, D, generator=gen, device=DEV) * spec.dy_std).to(torch.bfloat16)
        wr = synth.router_weights(T, k, seed=43)
    else:
        topk, x, w13, w2, dout, wr = _layer_inputs(spec, 43)
    x, dout = x.to(DEV), dout.to(DEV)
    qw = mxk.mxmoe_quantize_weights(w13.to(DEV), w2.to(DEV))
    del w13, w2
    tk, wt = torch.from_numpy(topk).to(DEV), torch.from_numpy(wr).to(DEV)
    out, saved = mxk.moe_layer_fwd_q(x, tk, wt, qw, spec.pad)
    dx, dw13, dw2, dwr = mxk.moe_layer_bwd_q(dout, wt, qw, saved, spec.pad)
    # the same layout fed to the row composites
    off, rs, sr = saved["offsets"], saved["row_slot"].long(), saved["slot_row"]
    real = rs >= 0
    tok = torch.where(real, rs // k, 0)
    x_rows = torch.where(real[:, None], x[tok], torch.zeros((), dtype=x.dtype, device=DEV))
    wflat = wt.reshape(-1)
    dy_rows = (wflat[torch.where(real, rs, 0)][:, None] * dout[tok].float()).to(torch.bfloat16)
    dy_rows = torch.where(real[:, None], dy_rows, torch.zeros((), dtype=dy_rows.dtype, device=DEV))
    y_rows, s2 = mxk.moe_mlp_fwd_q(x_rows, qw, off, spec.pad)
    dx_rows, dw13b, dw2b = mxk.moe_mlp_bwd_q(dy_rows, qw, off, s2, spec.pad)
    torch.cuda.synchronize()
    assert mxk.device_error() == 0
    M = int(off[-1].item())
    assert torch.equal(saved["y"][:M], y_rows[:M])
    assert torch.equal(out, mxk.mxmoe_unpermute_combine(y_rows, sr, k, wt))
    assert torch.equal(dw13, dw13b) and torch.equal(dw2, dw2b)
    assert torch.equal(dx, mxk.mxmoe_unpermute_combine(dx_rows, sr, k))
    assert torch.equal(dwr, mxk.mxmoe_combine_weight_grad(dout, y_rows, sr, k))
