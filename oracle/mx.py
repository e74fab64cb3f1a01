"""CPU oracle for the MXFP8 routed-experts MLP.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the library never does.  It shares no
code with the CUDA path.

Everything is plain numpy in float64, written as the definition of each step:

* MXFP8 tensor = E4M3 element codes plus one E8M0 power-of-two scale per
  block of 32 consecutive elements (A2E MXFP8 page, "Add support for MXFP8
  input to the A2E operator"; A2E transport page, "quant_mode").
* Block scale: OCP Microscaling (MX) v1.0 rule, shared exponent
  floor(log2(amax)) - 8 (8 = largest E4M3 exponent), stored as E8M0 byte
  exponent + 127 and clamped to [0, 254].  The pages do not print this rule;
  it is the reading they support ("E8M0 block scale", power-of-two scales).
* Element: value / 2^shared_exp rounded to the nearest E4M3 value, ties to
  even mantissa, magnitudes past 448 saturated to 448, sign kept (so negative
  underflow is -0, code 0x80).
* A block holding NaN or Inf gets scale byte 0xFF (the E8M0 NaN) and every
  element code 0x7F | sign (the E4M3 NaN).
* E8M0 decode: byte b -> 2^(b-127) for b in [0, 254], 0xFF -> NaN; byte 0x00
  is 2^-127, not zero (A2E transport page, review "[P2] Handle the two E8M0
  endpoint encodings before shifting").
* Row-wise (ROW) blocks run along the last, contiguous dimension; the last
  block of a row may be short (A2E transport page, unit tests: "a hidden size
  that is not a multiple of the group size").  Column-wise (COL) blocks run
  over 32 consecutive rows of one column and are stored transposed, i.e. COL
  quantization of X is ROW quantization of X^T.
* SwiGLU: h = bf16(silu(a) * b), a = first F columns of h13 (gate, w1),
  b = last F columns (up, w3); h is rounded to bf16 before it is quantized
  (SwiGLU-boundary page, "Numerics and tests": the fused kernel matches the
  standalone cast bit for bit in the forward).
* dSwiGLU: s = sigmoid(a); dgate = dh*b*s*(1 + a*(1-s)); dup = dh*a*s; dh is
  the bf16 output of the dgrad GEMM and both results are rounded to bf16
  (fully-fused plan page, "fused dSwiGLU backward").
* Grouped GEMMs: per expert segment [offsets[e], offsets[e+1]), float64
  matmul over dequantized operands (fully-fused plan page, "What it adds":
  FC1 grouped GEMM, FC2 GEMM, dSwiGLU backward, wgrad).  Zero-token experts
  give exactly zero weight gradients.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8          # 448 = 1.75 * 2^8
E8M0_BIAS = 127
E8M0_NAN = 0xFF
E4M3_NAN = 0x7F


# ----------------------------------------------------------------------------
# element and scale formats
# ----------------------------------------------------------------------------
def e4m3_decode_table() -> np.ndarray:
    """All 256 E4M3 codes decoded from the format definition.

    sign bit, 4-bit exponent (bias 7), 3-bit mantissa; exponent field 0 is
    subnormal m/8 * 2^-6; S.1111.111 is NaN; there is no infinity.
    """
    t = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            t[c] = np.nan
        elif e == 0:
            t[c] = s * (m / 8.0) * 2.0 ** -6
        else:
            t[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3_TABLE = e4m3_decode_table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e8m0_decode(b: np.ndarray) -> np.ndarray:
    """E8M0 byte -> 2^(b-127); 0xFF -> NaN."""
    b = np.asarray(b, dtype=np.int64)
    out = np.ldexp(1.0, b - E8M0_BIAS)
    return np.where(b == E8M0_NAN, np.nan, out)


# ----------------------------------------------------------------------------
# bf16
# ----------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest bf16 value, ties to even (returns float64).

    bf16 has 8 significant bits and the float32 exponent range: in the binade
    [2^k, 2^(k+1)), k >= -126, the spacing is 2^(k-7); below 2^-126 it is 2^-133.
    Magnitudes that round past the largest finite bf16 become infinite.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e = np.frexp(xf)                 # |x| in [2^(e-1), 2^e)
    ulp_exp = np.maximum(e - 8, -133)
    q = np.rint(np.ldexp(xf, -ulp_exp))  # round half to even
    r = np.ldexp(q, ulp_exp)
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(np.abs(r) > bf16_max, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 values that are exactly bf16 -> uint16 bit patterns."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------
# MX quantization
# ----------------------------------------------------------------------------
def scale_byte(amax: np.ndarray) -> np.ndarray:
    """E8M0 byte of a block from its largest magnitude (OCP MX v1.0 rule).

    shared_exp = floor(log2(amax)) - 8, byte = clamp(shared_exp + 127, 0, 254);
    amax == 0 gives byte 0; a non-finite amax gives 0xFF.
    """
    amax = np.asarray(amax, dtype=np.float64)
    out = np.zeros(amax.shape, dtype=np.int64)
    pos = np.isfinite(amax) & (amax > 0)
    _, e = np.frexp(amax[pos])          # amax in [2^(e-1), 2^e) -> floor(log2) = e-1
    out[pos] = np.clip((e - 1) - E4M3_EMAX + E8M0_BIAS, 0, 254)
    out[~np.isfinite(amax)] = E8M0_NAN
    return out.astype(np.uint8)


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round float64 to the E4M3 grid: nearest, ties to even, saturate at 448.

    In the binade [2^k, 2^(k+1)), k >= -6, E4M3 values are spaced 2^(k-3);
    below 2^-6 (subnormals) the spacing is 2^-9.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros_like(a)
    nz = a > 0
    _, e = np.frexp(a[nz])
    ulp_exp = np.maximum(e - 4, -9)
    out[nz] = np.ldexp(np.rint(np.ldexp(a[nz], -ulp_exp)), ulp_exp)
    out = np.minimum(out, E4M3_MAX)
    return np.copysign(out, v)


def e4m3_code_of(q: np.ndarray) -> np.ndarray:
    """Bit pattern of a float64 already on the E4M3 grid (|q| <= 448)."""
    q = np.asarray(q, dtype=np.float64)
    a = np.abs(q)
    sign = np.signbit(q).astype(np.int64) << 7
    code = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** -6
    code[sub] = np.rint(a[sub] / 2.0 ** -9).astype(np.int64)
    nrm = ~sub
    _, e = np.frexp(a[nrm])             # a in [2^(e-1), 2^e)
    k = e - 1
    mant = np.rint((np.ldexp(a[nrm], -k) - 1.0) * 8).astype(np.int64)
    code[nrm] = ((k + 7) << 3) | mant
    return (code | sign).astype(np.uint8)


def quantize_rows(x: np.ndarray):
    """ROW MX quantization of a 2-D array of bf16 values (given as float64).

    Blocks of 32 along the last dimension; the last block of a row may be
    shorter.  Returns (codes uint8 [rows, cols], scales uint8 [rows, ceil(cols/32)]).
    """
    x = np.asarray(x, dtype=np.float64)
    rows, cols = x.shape
    nb = -(-cols // BLOCK)
    padc = nb * BLOCK
    xp = np.zeros((rows, padc))
    xp[:, :cols] = x
    blocks = xp.reshape(rows, nb, BLOCK)
    absb = np.abs(blocks)
    bad = ~np.isfinite(absb).all(axis=2)
    amax = np.where(bad, np.inf, np.nanmax(np.where(np.isfinite(absb), absb, 0.0), axis=2))
    sb = scale_byte(amax)                                   # [rows, nb]
    shared = sb.astype(np.int64) - E8M0_BIAS
    v = np.ldexp(blocks, -shared[:, :, None])               # exact: power-of-two scaling
    with np.errstate(invalid="ignore"):
        q = e4m3_round(np.where(np.isfinite(v), v, 0.0))
    codes = e4m3_code_of(q)
    nan_code = (np.signbit(blocks).astype(np.uint8) << 7) | E4M3_NAN
    codes = np.where(bad[:, :, None], nan_code, codes).astype(np.uint8)
    codes = codes.reshape(rows, padc)[:, :cols]
    return np.ascontiguousarray(codes), sb


def quantize_cols(x: np.ndarray):
    """COL MX quantization: blocks of 32 consecutive rows of one column.

    Stored transposed: codes [cols, rows], scales [cols, rows/32].  It is the
    ROW quantization of x^T.
    """
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[0] % BLOCK == 0, "COL quantization needs rows % 32 == 0"
    return quantize_rows(x.T)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """codes [rows, cols] * per-block scale -> float64 [rows, cols]."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    s = e8m0_decode(scales)                                 # [rows, nb]
    s_full = np.repeat(s, BLOCK, axis=1)[:, :cols]
    return e4m3_decode(codes) * s_full


# ----------------------------------------------------------------------------
# SwiGLU and its derivative
# ----------------------------------------------------------------------------
def _sigmoid(a):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-a))


def swiglu(h13: np.ndarray) -> np.ndarray:
    """h = bf16(silu(a) * b), a = h13[:, :F] (gate), b = h13[:, F:] (up)."""
    h13 = np.asarray(h13, dtype=np.float64)
    F = h13.shape[1] // 2
    a, b = h13[:, :F], h13[:, F:]
    return round_to_bf16(a * _sigmoid(a) * b)


def dswiglu(dh: np.ndarray, h13: np.ndarray) -> np.ndarray:
    """dh13 = [dgate | dup] in bf16 for h = silu(a) * b.

    d silu(a)/da = s * (1 + a * (1 - s)) with s = sigmoid(a).
    """
    h13 = np.asarray(h13, dtype=np.float64)
    dh = np.asarray(dh, dtype=np.float64)
    F = h13.shape[1] // 2
    a, b = h13[:, :F], h13[:, F:]
    s = _sigmoid(a)
    dgate = dh * b * s * (1.0 + a * (1.0 - s))
    dup = dh * a * s
    return round_to_bf16(np.concatenate([dgate, dup], axis=1))


def swiglu_quant(h13: np.ndarray):
    """Standalone SwiGLU + dual quantization: (h_row codes, scales, h_col codes, scales)."""
    h = swiglu(h13)
    rc, rs = quantize_rows(h)
    cc, cs = quantize_cols(h)
    return rc, rs, cc, cs


# ----------------------------------------------------------------------------
# grouped GEMMs
# ----------------------------------------------------------------------------
def _experts(offsets, experts):
    E = len(offsets) - 1
    return range(E) if experts is None else experts


def grouped_gemm(a_codes, a_scales, w_codes, w_scales, offsets, experts=None):
    """out[m] = A[m] . W[e]^T for m in expert e's segment (ragged M).

    A: codes [M, K] + ROW scales [M, K/32]; W: codes [E, N, K] + scales
    [E, N, K/32].  Rows outside the listed experts' segments are NaN.
    """
    M, K = a_codes.shape
    E, N, _ = w_codes.shape
    out = np.full((M, N), np.nan)
    for e in _experts(offsets, experts):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        a = dequantize_rows(a_codes[lo:hi], a_scales[lo:hi])
        w = dequantize_rows(w_codes[e], w_scales[e])
        out[lo:hi] = a @ w.T
    return out


def grouped_gemm_wgrad(g_codes_t, g_scales_t, x_codes_t, x_scales_t, offsets, experts=None):
    """dW[e] = G_e^T . X_e summed over expert e's token rows (ragged K).

    Operands are COL-quantized and stored transposed: G^T codes [N, M] with
    scales [N, M/32], X^T codes [Kx, M] with scales [Kx, M/32].  An expert with
    no rows gets dW[e] = 0 exactly.
    """
    N = g_codes_t.shape[0]
    Kx = x_codes_t.shape[0]
    E = len(offsets) - 1
    ex = list(_experts(offsets, experts))
    out = np.full((E, N, Kx), np.nan)
    for e in ex:
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            out[e] = 0.0
            continue
        b0, b1 = lo // BLOCK, hi // BLOCK
        g = dequantize_rows(g_codes_t[:, lo:hi], g_scales_t[:, b0:b1])
        x = dequantize_rows(x_codes_t[:, lo:hi], x_scales_t[:, b0:b1])
        out[e] = g @ x.T
    return out


def quantize_weights_rows(w: np.ndarray):
    """ROW quantization of each expert matrix: w [E, R, C] -> codes, scales [E, R, C/32]."""
    cs, ss = zip(*(quantize_rows(w[e]) for e in range(w.shape[0])))
    return np.stack(cs), np.stack(ss)


def quantize_weights_cols(w: np.ndarray):
    """COL quantization of each expert matrix: w [E, R, C] -> codes [E, C, R], scales [E, C, R/32]."""
    cs, ss = zip(*(quantize_cols(w[e]) for e in range(w.shape[0])))
    return np.stack(cs), np.stack(ss)


# ----------------------------------------------------------------------------
# composites
# ----------------------------------------------------------------------------
def _seg_matmul(a, b_of_e, offsets, experts, n_out):
    """out[seg_e] = a[seg_e] @ b_of_e(e) for each listed expert (float64)."""
    out = np.full((a.shape[0], n_out), np.nan)
    for e in _experts(offsets, experts):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            out[lo:hi] = a[lo:hi] @ b_of_e(e)
    return out


def _seg_wgrad(g, x, offsets, experts, E):
    """dW[e] = g[seg_e]^T @ x[seg_e]; zero for an expert without rows."""
    out = np.full((E, g.shape[1], x.shape[1]), np.nan)
    for e in _experts(offsets, experts):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        out[e] = g[lo:hi].T @ x[lo:hi] if hi > lo else 0.0
    return out


def moe_mlp_fwd(x, w13, w2, offsets, experts=None, exact=False):
    """Forward of the MXFP8 routed-experts MLP.

    x [M, D] bf16 values, w13 [E, 2F, D] (rows 0..F-1 gate, F..2F-1 up),
    w2 [E, D, F], given as float64 arrays.  Every GEMM operand is the
    dequantized MX tensor: x and h ROW-quantized along the contraction
    dimension, w13 and w2 ROW-quantized per expert along theirs.  h13 is
    rounded to bf16, h = bf16(silu(gate) * up).  y is returned unrounded.

    exact=True drops every quantization and bf16 rounding (a plain float64
    MLP with the same structure); the tests use it to pin the composition.
    """
    x = np.asarray(x, dtype=np.float64)
    E = w13.shape[0]
    F = w13.shape[1] // 2
    D = x.shape[1]
    out = {}
    if exact:
        xq, w13q, w2q = x, w13, w2
    else:
        x_rc, x_rs = quantize_rows(x)
        out["x_row"] = (x_rc, x_rs)
        out["x_col"] = quantize_cols(x)
        xq = dequantize_rows(x_rc, x_rs)
        w13q = np.stack([dequantize_rows(*quantize_rows(w13[e])) for e in range(E)])
        w2q = np.stack([dequantize_rows(*quantize_rows(w2[e])) for e in range(E)])
    h13 = _seg_matmul(xq, lambda e: w13q[e].T, offsets, experts, 2 * F)
    h13 = np.nan_to_num(h13, nan=0.0)        # rows of experts not listed: inert
    if exact:
        a, b = h13[:, :F], h13[:, F:]
        h = a * _sigmoid(a) * b
        hq = h
    else:
        h13 = round_to_bf16(h13)
        h = swiglu(h13)
        h_rc, h_rs = quantize_rows(h)
        out["h_row"] = (h_rc, h_rs)
        out["h_col"] = quantize_cols(h)
        hq = dequantize_rows(h_rc, h_rs)
    y = _seg_matmul(hq, lambda e: w2q[e].T, offsets, experts, D)
    out.update(y=y, h13=h13, h=h)
    return out


def moe_mlp_bwd(dy, fwd, x, w13, w2, offsets, experts=None, exact=False):
    """Backward of :func:`moe_mlp_fwd`: dx [M, D], dW13 [E, 2F, D], dW2 [E, D, F].

    dh = dY . W2[e] with dY ROW-quantized and W2 COL-quantized along D;
    dh is rounded to bf16 and turned into dh13 = [dgate | dup] (bf16) by
    dSwiGLU.  dW2[e] = dY_e^T . h_e and dW13[e] = dh13_e^T . x_e over the
    expert's rows with both operands COL-quantized along the token dimension;
    dx = dh13 . W13[e] with dh13 ROW-quantized and W13 COL-quantized along 2F.
    """
    dy = np.asarray(dy, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    E = w13.shape[0]
    F = w13.shape[1] // 2
    D = dy.shape[1]
    h13 = fwd["h13"]
    out = {}
    if exact:
        dyr = dyc = dy
        w2c = w2
        w13c = w13
        hc, xc = fwd["h"], x
    else:
        dy_rc, dy_rs = quantize_rows(dy)
        dy_cc, dy_cs = quantize_cols(dy)
        dyr = dequantize_rows(dy_rc, dy_rs)
        dyc = dequantize_rows(dy_cc, dy_cs).T
        # W2[e] is [D, F]: COL blocks run along D (the contraction of dh)
        w2c = np.stack([dequantize_rows(*quantize_cols(w2[e])).T for e in range(E)])
        # W13[e] is [2F, D]: COL blocks run along 2F (the contraction of dx)
        w13c = np.stack([dequantize_rows(*quantize_cols(w13[e])).T for e in range(E)])
        hc = dequantize_rows(*fwd["h_col"]).T
        xc = dequantize_rows(*fwd["x_col"]).T
    dh = _seg_matmul(dyr, lambda e: w2c[e], offsets, experts, F)
    dh = np.nan_to_num(dh, nan=0.0)
    if exact:
        a, b = h13[:, :F], h13[:, F:]
        s = _sigmoid(a)
        dh13 = np.concatenate([dh * b * s * (1.0 + a * (1.0 - s)), dh * a * s], axis=1)
        gr = gc = dh13
    else:
        dh = round_to_bf16(dh)
        dh13 = dswiglu(dh, h13)
        g_rc, g_rs = quantize_rows(dh13)
        g_cc, g_cs = quantize_cols(dh13)
        out["dh13_row"] = (g_rc, g_rs)
        out["dh13_col"] = (g_cc, g_cs)
        out["dy_row"] = (dy_rc, dy_rs)
        out["dy_col"] = (dy_cc, dy_cs)
        gr = dequantize_rows(g_rc, g_rs)
        gc = dequantize_rows(g_cc, g_cs).T
    dw2 = _seg_wgrad(dyc, hc, offsets, experts, E)
    dx = _seg_matmul(gr, lambda e: w13c[e], offsets, experts, D)
    dw13 = _seg_wgrad(gc, xc, offsets, experts, E)
    out.update(dx=dx, dw13=dw13, dw2=dw2, dh=dh, dh13=dh13)
    return out
