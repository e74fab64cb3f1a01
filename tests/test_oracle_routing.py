"""Pins of the dispatcher oracle (oracle.routing) against values fixed by hand,
an independently built layout, closed forms and finite differences."""
import numpy as np
import pytest

import synth
from oracle import mx, routing


def test_route_hand_example():
    # Three tokens, top-2 over three experts, worked by hand:
    # slots 0:(t0,e0) 1:(t0,e2) 2:(t1,e2) 3:(t1,e1) 4:(t2,e0) 5:(t2,e1)
    topk = np.array([[0, 2], [2, 1], [0, 1]])
    r = routing.route(topk, 3, 2)
    np.testing.assert_array_equal(r["counts"], [2, 2, 2])
    np.testing.assert_array_equal(r["offsets"], [0, 2, 4, 6])
    np.testing.assert_array_equal(r["row_slot"], [0, 4, 3, 5, 1, 2])
    np.testing.assert_array_equal(r["slot_row"], [0, 4, 5, 2, 1, 3])
    r = routing.route(topk, 3, 4)
    np.testing.assert_array_equal(r["offsets"], [0, 4, 8, 12])
    np.testing.assert_array_equal(r["row_slot"], [0, 4, -1, -1, 3, 5, -1, -1, 1, 2, -1, -1])
    # an expert nobody picks keeps an empty segment
    r = routing.route(np.array([[1], [1], [3]]), 4, 2)
    np.testing.assert_array_equal(r["offsets"], [0, 0, 2, 2, 4])
    np.testing.assert_array_equal(r["row_slot"], [0, 1, 2, -1])


@pytest.mark.parametrize("name", ["tiny", "dsv3_16b"])
def test_route_matches_the_input_generator_layout(name):
    # synth builds the same layout by a lexsort; the oracle by per-token lists.
    spec = synth.SPECS[name]
    rt = synth.make_routing(spec)
    r = routing.route(rt.topk, spec.E, spec.pad)
    np.testing.assert_array_equal(r["offsets"], rt.offsets)
    real = r["row_slot"] >= 0
    np.testing.assert_array_equal(real, rt.src_token >= 0)
    np.testing.assert_array_equal(r["row_slot"][real] // spec.top_k, rt.src_token[real])


@pytest.mark.parametrize("T,k,E,pad,zipf", [(300, 4, 16, 32, None), (257, 3, 9, 128, 1.2), (64, 1, 5, 32, 2.0)])
def test_route_invariants(T, k, E, pad, zipf):
    topk = synth.topk_ids(T, k, E, seed=T, zipf_s=zipf)
    r = routing.route(topk, E, pad)
    off, rs, sr = r["offsets"], r["row_slot"], r["slot_row"]
    np.testing.assert_array_equal(r["counts"], np.bincount(topk.reshape(-1), minlength=E))
    assert (off % pad == 0).all() and (np.diff(off) >= 0).all()
    np.testing.assert_array_equal(np.sort(rs[rs >= 0]), np.arange(T * k))   # every slot once
    np.testing.assert_array_equal(rs[sr], np.arange(T * k))
    for e in range(E):
        seg = rs[off[e]:off[e + 1]]
        c = r["counts"][e]
        assert (seg[c:] == -1).all()
        assert (topk.reshape(-1)[seg[:c]] == e).all()
        assert (np.diff(seg[:c]) > 0).all()                                   # ascending slots


def test_route_rejects_bad_ids():
    with pytest.raises(ValueError):
        routing.route(np.array([[0, 4]]), 4, 32)


def test_permute_identity_and_power_of_two_weights():
    g = synth.rng(3)
    x = mx.round_to_bf16(g.standard_normal((5, 64)))
    r = routing.route(np.arange(5)[:, None] % 2, 2, 1)
    rows = routing.permute(x, r["row_slot"], 1)
    np.testing.assert_array_equal(rows[r["slot_row"]], x)
    # power-of-two weights scale without rounding
    w = np.array([[0.5], [2.0], [0.25], [1.0], [4.0]], dtype=np.float32)
    rows = routing.permute(x, r["row_slot"], 1, w)
    np.testing.assert_array_equal(rows[r["slot_row"]], x * w)


def test_weighted_permute_rounds_the_fp32_product_to_bf16():
    # near 1 the bf16 spacing is 2^-7, so 1 + 2^-8 and 1 + 3*2^-8 are ties
    def one(w, x=1.0):
        return routing.permute(np.array([[x]]), np.array([0]), 1, np.array([[w]], dtype=np.float32))[0, 0]
    assert one(1 + 2.0 ** -8) == 1.0                        # tie, even mantissa below
    assert one(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6          # tie, even mantissa above
    assert one(1 + 2.0 ** -8 + 2.0 ** -20) == 1 + 2.0 ** -7  # past the tie
    # (1 + 2^-7)(1 - 2^-8) = 1 + 2^-8 - 2^-15: just below the tie
    assert one(1 - 2.0 ** -8, 1 + 2.0 ** -7) == 1.0
    assert one(-0.5, 3.0) == -1.5


def test_combine_of_permute_is_weight_sum_times_token():
    T, k, E = 40, 3, 7
    topk = synth.topk_ids(T, k, E, seed=5)
    w = synth.router_weights(T, k, seed=5)
    r = routing.route(topk, E, 32)
    x = synth.rng(1).standard_normal((T, 48))
    y = routing.permute(x, r["row_slot"], k)
    out = routing.unpermute_combine(y, r["slot_row"], T, k, w)
    np.testing.assert_allclose(out, x * w.astype(np.float64).sum(1, keepdims=True), rtol=1e-12, atol=1e-12)
    out = routing.unpermute_combine(y, r["slot_row"], T, k)
    np.testing.assert_allclose(out, k * x, rtol=1e-12)


def test_weight_grad_is_the_derivative_of_the_combine():
    T, k, E, D = 6, 2, 3, 16
    topk = synth.topk_ids(T, k, E, seed=9)
    r = routing.route(topk, E, 32)
    g = synth.rng(2)
    y = g.standard_normal((len(r["row_slot"]), D))
    dout = g.standard_normal((T, D))
    w = g.random((T, k))
    dw = routing.combine_weight_grad(dout, y, r["slot_row"], T, k)
    h = 1e-6
    for t in range(T):
        for j in range(k):
            wp, wm = w.copy(), w.copy()
            wp[t, j] += h
            wm[t, j] -= h
            fp = np.sum(dout * routing.unpermute_combine(y, r["slot_row"], T, k, wp))
            fm = np.sum(dout * routing.unpermute_combine(y, r["slot_row"], T, k, wm))
            assert abs((fp - fm) / (2 * h) - dw[t, j]) < 1e-6 * max(1.0, abs(dw[t, j]))


def test_layer_exact_mode_vs_torch_autograd():
    # the whole token-major layer (route, permute, MLP, weighted combine) and
    # its backward, without quantization, against float64 autograd of
    # out[t] = sum_j w[t, j] * MLP_{topk[t, j]}(x[t])
    import torch
    T, k, E, D, F, pad = 24, 2, 3, 16, 8, 4
    g = synth.rng(21)
    topk = synth.topk_ids(T, k, E, seed=21)
    w = g.random((T, k))
    x = g.standard_normal((T, D))
    w13 = g.standard_normal((E, 2 * F, D)) * 0.3
    w2 = g.standard_normal((E, D, F)) * 0.3
    dout = g.standard_normal((T, D))
    fwd = routing.layer_fwd(x, topk, w, w13, w2, E, pad, exact=True)
    bwd = routing.layer_bwd(dout, fwd, x, topk, w, w13, w2, pad, exact=True)

    X = torch.tensor(x, requires_grad=True)
    W13 = torch.tensor(w13, requires_grad=True)
    W2 = torch.tensor(w2, requires_grad=True)
    WR = torch.tensor(w, requires_grad=True)
    outs = []
    for t in range(T):
        acc = torch.zeros(D, dtype=torch.float64)
        for j in range(k):
            e = int(topk[t, j])
            h13 = W13[e] @ X[t]
            h = torch.nn.functional.silu(h13[:F]) * h13[F:]
            acc = acc + WR[t, j] * (W2[e] @ h)
        outs.append(acc)
    out = torch.stack(outs)
    (out * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(fwd["out"], out.detach().numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(bwd["dx"], X.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(bwd["dw13"], W13.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(bwd["dw2"], W2.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(bwd["dweights"], WR.grad.numpy(), rtol=1e-9, atol=1e-12)
