"""CPU oracle of the token dispatcher around the routed-experts MLP.
TEST INFRASTRUCTURE ONLY: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; it shares no code with the
CUDA path.

The MLP consumes its tokens in an expert-major layout whose per-expert
segments are padded to a multiple of ``pad_multiple`` rows: the "padded
dispatcher" that the fully-fused plan installs (fully-fused plan page, "What
it adds": the pad_multiple=256 dispatcher the kernels' per-expert alignment
requires; SwiGLU-boundary page, "Usage": the token dispatcher produces the
padded expert-major layout the kernels consume).  The pages name the steps
(routing, padding, permutation generation: HiFloat8/AutoEP page,
"Implementation") but print no definition of them, so the reading here is the
plainest one:

* slot s = t*k + j is token t's j-th routed copy, sent to expert topk[t, j];
* expert e's segment holds its slots in ascending slot order (so tokens in
  ascending order), followed by zero pad rows up to the next multiple of
  ``pad_multiple`` (an expert with no tokens has an empty segment);
* forward permute: row m of the layout is the source token's row (zero for a
  pad row);
* forward combine: out[t] = sum_j w[t, j] * y[row(t, j)], w the router
  weights;
* backward: d y[row(t, j)] = w[t, j] * dout[t], rounded to bf16 after an fp32
  product; d w[t, j] = <dout[t], y[row(t, j)]>; d x[t] = sum_j dx[row(t, j)].

Float64 except where a value is rounded to bf16 for the next step: the
weighted gradient rows are fp32 products rounded to bf16, as the CUDA path
forms them before quantizing (both sides take the code decision in the same
precision).
"""
from __future__ import annotations

import numpy as np

from . import mx


def route(topk: np.ndarray, E: int, pad: int):
    """Expert-major padded layout of a top-k routing.

    topk [T, k] expert ids.  Returns a dict with
      counts   [E]     real rows per expert
      offsets  [E+1]   int32 start of each padded segment (offsets[E] = M)
      row_slot [M]     slot t*k+j of each row, -1 for a pad row
      slot_row [T*k]   row of each slot
    """
    topk = np.asarray(topk)
    T, k = topk.shape
    if topk.size and (topk.min() < 0 or topk.max() >= E):
        raise ValueError("expert id outside [0, E)")
    per_expert = [[] for _ in range(E)]
    for t in range(T):                      # ascending slots, so tokens in order
        for j in range(k):
            per_expert[int(topk[t, j])].append(t * k + j)
    counts = np.array([len(s) for s in per_expert], dtype=np.int64)
    offsets = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        padded = -(-counts[e] // pad) * pad
        offsets[e + 1] = offsets[e] + padded
    M = int(offsets[E])
    row_slot = -np.ones(M, dtype=np.int64)
    slot_row = np.empty(T * k, dtype=np.int64)
    for e in range(E):
        for i, s in enumerate(per_expert[e]):
            row_slot[offsets[e] + i] = s
            slot_row[s] = offsets[e] + i
    return {"counts": counts, "offsets": offsets, "row_slot": row_slot, "slot_row": slot_row}


def permute(x_tok: np.ndarray, row_slot: np.ndarray, k: int, weights=None, exact=False) -> np.ndarray:
    """Rows of the padded layout: x_tok[slot // k] (zero for pad rows).

    With ``weights`` [T, k] (fp32) every row is multiplied by its slot's
    weight in fp32 and rounded to bf16 (the backward of the combine);
    exact=True multiplies in float64 without rounding.
    """
    D = x_tok.shape[1]
    out = np.zeros((len(row_slot), D))
    for m, s in enumerate(row_slot):
        if s < 0:
            continue
        row = x_tok[s // k]
        if weights is not None and exact:
            row = float(np.asarray(weights, dtype=np.float64).reshape(-1)[s]) * row
        elif weights is not None:
            w = np.float32(np.asarray(weights, dtype=np.float32).reshape(-1)[s])
            row = mx.round_to_bf16((w * row.astype(np.float32)).astype(np.float64))
        out[m] = row
    return out


def permute_quant(x_tok, row_slot, k, weights=None):
    """permute() followed by ROW and COL MX quantization of the layout."""
    rows = permute(x_tok, row_slot, k, weights)
    rc, rs = mx.quantize_rows(rows)
    cc, cs = mx.quantize_cols(rows)
    return rc, rs, cc, cs


def unpermute_combine(y: np.ndarray, slot_row: np.ndarray, T: int, k: int, weights=None) -> np.ndarray:
    """out[t] = sum_j w[t, j] * y[row(t, j)] in float64 (w = 1 without weights)."""
    out = np.zeros((T, y.shape[1]))
    w = None if weights is None else np.asarray(weights, dtype=np.float64).reshape(T, k)
    for t in range(T):
        for j in range(k):
            r = slot_row[t * k + j]
            out[t] += (1.0 if w is None else w[t, j]) * y[r]
    return out


def combine_weight_grad(dout: np.ndarray, y: np.ndarray, slot_row: np.ndarray, T: int, k: int) -> np.ndarray:
    """d w[t, j] = <dout[t], y[row(t, j)]> in float64, shape [T, k]."""
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            dw[t, j] = float(np.dot(dout[t], y[slot_row[t * k + j]]))
    return dw


def layer_fwd(x_tok, topk, weights, w13, w2, E, pad, exact=False):
    """Token-major layer forward: route, permute, the MLP over the padded
    layout (oracle.mx.moe_mlp_fwd), combine with the router weights.

    The MLP output rows are bf16 at the GEMM boundary, so the combine reads
    them rounded (exact=True: unrounded).  Returns a dict with the route
    tables, x_rows, the MLP forward ('mlp'), y_rows and out [T, D].
    """
    T, k = np.asarray(topk).shape
    r = route(topk, E, pad)
    x_rows = permute(x_tok, r["row_slot"], k)
    fwd = mx.moe_mlp_fwd(x_rows, w13, w2, r["offsets"], exact=exact)
    y_rows = np.nan_to_num(fwd["y"]) if exact else mx.round_to_bf16(np.nan_to_num(fwd["y"]))
    out = unpermute_combine(y_rows, r["slot_row"], T, k, weights)
    return dict(route=r, x_rows=x_rows, mlp=fwd, y_rows=y_rows, out=out)


def layer_bwd(dout, fwd, x_tok, topk, weights, w13, w2, pad, exact=False):
    """Token-major layer backward: dY rows = w * dout[token] (bf16), the MLP
    backward (oracle.mx.moe_mlp_bwd), dx_tok = sum of a token's dx rows (bf16
    rows, float64 sum), dweights = <dout, y row>.  Returns dict(dx, dw13, dw2,
    dweights)."""
    T, k = np.asarray(topk).shape
    r = fwd["route"]
    dy_rows = permute(dout, r["row_slot"], k, weights, exact=exact)
    bwd = mx.moe_mlp_bwd(dy_rows, fwd["mlp"], fwd["x_rows"], w13, w2, r["offsets"], exact=exact)
    dx_rows = np.nan_to_num(bwd["dx"]) if exact else mx.round_to_bf16(np.nan_to_num(bwd["dx"]))
    dx = unpermute_combine(dx_rows, r["slot_row"], T, k)
    dweights = combine_weight_grad(dout, fwd["y_rows"], r["slot_row"], T, k)
    return dict(dx=dx, dw13=bwd["dw13"], dw2=bwd["dw2"], dweights=dweights, dy_rows=dy_rows)
