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
* E5M2 elements (A2E transport page, "quant_mode=4": the activation goes out
  as E4M3 or E5M2 with its E8M0 block scale): same block rule with the E5M2
  largest exponent 15 (floor(log2(amax)) - 15), nearest-even rounding onto the
  E5M2 grid (subnormal spacing 2^-16), saturation at 57344, NaN/Inf blocks
  -> 0xFF and codes 0x7F | sign.
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
E5M2_MAX = 57344.0     # 1.75 * 2^15
E5M2_EMAX = 15


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


def e5m2_decode_table() -> np.ndarray:
    """All 256 E5M2 codes decoded from the format definition.

    sign bit, 5-bit exponent (bias 15), 2-bit mantissa; exponent field 0 is
    subnormal m/4 * 2^-14; exponent field 31 is infinity (m = 0) or NaN.
    """
    t = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 2) & 0x1F
        m = c & 0x3
        if e == 0x1F:
            t[c] = s * np.inf if m == 0 else np.nan
        elif e == 0:
            t[c] = s * (m / 4.0) * 2.0 ** -14
        else:
            t[c] = s * (1.0 + m / 4.0) * 2.0 ** (e - 15)
    return t


E5M2_TABLE = e5m2_decode_table()


def e5m2_decode(codes: np.ndarray) -> np.ndarray:
    return E5M2_TABLE[np.asarray(codes, dtype=np.uint8)]


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
def scale_byte(amax: np.ndarray, emax: int = E4M3_EMAX) -> np.ndarray:
    """E8M0 byte of a block from its largest magnitude (OCP MX v1.0 rule).

    shared_exp = floor(log2(amax)) - emax (8 for E4M3, 15 for E5M2),
    byte = clamp(shared_exp + 127, 0, 254); amax == 0 gives byte 0; a
    non-finite amax gives 0xFF.
    """
    amax = np.asarray(amax, dtype=np.float64)
    out = np.zeros(amax.shape, dtype=np.int64)
    pos = np.isfinite(amax) & (amax > 0)
    _, e = np.frexp(amax[pos])          # amax in [2^(e-1), 2^e) -> floor(log2) = e-1
    out[pos] = np.clip((e - 1) - emax + E8M0_BIAS, 0, 254)
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


def e5m2_round(v: np.ndarray) -> np.ndarray:
    """Round float64 to the E5M2 grid: nearest, ties to even, saturate at 57344.

    In the binade [2^k, 2^(k+1)), k >= -14, E5M2 values are spaced 2^(k-2);
    below 2^-14 (subnormals) the spacing is 2^-16.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros_like(a)
    nz = a > 0
    _, e = np.frexp(a[nz])
    ulp_exp = np.maximum(e - 3, -16)
    out[nz] = np.ldexp(np.rint(np.ldexp(a[nz], -ulp_exp)), ulp_exp)
    out = np.minimum(out, E5M2_MAX)
    return np.copysign(out, v)


def e5m2_code_of(q: np.ndarray) -> np.ndarray:
    """Bit pattern of a float64 already on the E5M2 grid (|q| <= 57344)."""
    q = np.asarray(q, dtype=np.float64)
    a = np.abs(q)
    sign = np.signbit(q).astype(np.int64) << 7
    code = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** -14
    code[sub] = np.rint(a[sub] / 2.0 ** -16).astype(np.int64)
    nrm = ~sub
    _, e = np.frexp(a[nrm])
    k = e - 1
    mant = np.rint((np.ldexp(a[nrm], -k) - 1.0) * 4).astype(np.int64)
    code[nrm] = ((k + 15) << 2) | mant
    return (code | sign).astype(np.uint8)


# element formats: (largest exponent, rounding onto the grid, bit pattern, decode)
ELEMENTS = {
    "e4m3": (E4M3_EMAX, e4m3_round, e4m3_code_of, e4m3_decode),
    "e5m2": (E5M2_EMAX, e5m2_round, e5m2_code_of, e5m2_decode),
}


def quantize_rows(x: np.ndarray, elem: str = "e4m3"):
    """ROW MX quantization of a 2-D array of bf16 values (given as float64).

    Blocks of 32 along the last dimension; the last block of a row may be
    shorter.  Returns (codes uint8 [rows, cols], scales uint8 [rows, ceil(cols/32)]).
    ``elem`` picks the element format (E4M3 by default, or E5M2; the A2E
    transport page, "quant_mode=4": E4M3 or E5M2 with an E8M0 block scale).
    """
    emax, rnd, code_of, _ = ELEMENTS[elem]
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
    sb = scale_byte(amax, emax)                             # [rows, nb]
    shared = sb.astype(np.int64) - E8M0_BIAS
    v = np.ldexp(blocks, -shared[:, :, None])               # exact: power-of-two scaling
    with np.errstate(invalid="ignore"):
        q = rnd(np.where(np.isfinite(v), v, 0.0))
    codes = code_of(q)
    nan_code = (np.signbit(blocks).astype(np.uint8) << 7) | E4M3_NAN
    codes = np.where(bad[:, :, None], nan_code, codes).astype(np.uint8)
    codes = codes.reshape(rows, padc)[:, :cols]
    return np.ascontiguousarray(codes), sb


def quantize_cols(x: np.ndarray, elem: str = "e4m3"):
    """COL MX quantization: blocks of 32 consecutive rows of one column.

    Stored transposed: codes [cols, rows], scales [cols, rows/32].  It is the
    ROW quantization of x^T.
    """
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[0] % BLOCK == 0, "COL quantization needs rows % 32 == 0"
    return quantize_rows(x.T, elem)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, elem: str = "e4m3") -> np.ndarray:
    """codes [rows, cols] * per-block scale -> float64 [rows, cols]."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    s = e8m0_decode(scales)                                 # [rows, nb]
    s_full = np.repeat(s, BLOCK, axis=1)[:, :cols]
    with np.errstate(invalid="ignore"):
        return ELEMENTS[elem][3](codes) * s_full


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
# Every quantization block of the composite lies inside one expert segment:
# ROW blocks are within a row, COL blocks are 32-row groups and segments start
# at multiples of the pad (itself a multiple of 128).  The composite is
# therefore written per expert segment and the full-tensor forms below just
# loop over the experts.
def expert_fwd(x_e, w13_e, w2_e, exact=False):
    """Forward for the rows x_e [n, D] routed to one expert.

    h13 = x_e . w13_e^T with x ROW-quantized along D and w13_e [2F, D]
    ROW-quantized along D; h13 rounded to bf16; h = bf16(silu(gate) * up);
    y = h . w2_e^T with h ROW-quantized along F and w2_e [D, F] along F
    (y is returned unrounded).  exact=True drops every quantization and bf16
    rounding (a plain float64 MLP with the same structure).
    """
    x_e = np.asarray(x_e, dtype=np.float64)
    F = w13_e.shape[0] // 2
    out = {}
    if exact:
        xq, w13q, w2q = x_e, w13_e, w2_e
    else:
        out["x_row"] = quantize_rows(x_e)
        out["x_col"] = quantize_cols(x_e)
        xq = dequantize_rows(*out["x_row"])
        w13q = dequantize_rows(*quantize_rows(w13_e))
        w2q = dequantize_rows(*quantize_rows(w2_e))
    h13 = xq @ w13q.T
    if exact:
        a, b = h13[:, :F], h13[:, F:]
        h = a * _sigmoid(a) * b
        hq = h
    else:
        h13 = round_to_bf16(h13)
        h = swiglu(h13)
        out["h_row"] = quantize_rows(h)
        out["h_col"] = quantize_cols(h)
        hq = dequantize_rows(*out["h_row"])
    out.update(y=hq @ w2q.T, h13=h13, h=h)
    return out


def expert_bwd(dy_e, fwd_e, x_e, w13_e, w2_e, exact=False):
    """Backward for one expert segment.

    dh = dY . W2 with dY ROW-quantized along D and W2 [D, F] COL-quantized
    along D; dh rounded to bf16; dh13 = [dgate | dup] = dSwiGLU(dh, h13) in
    bf16; dW2 = dY^T . h and dW13 = dh13^T . x with both operands
    COL-quantized along the token rows; dx = dh13 . W13 with dh13
    ROW-quantized and W13 [2F, D] COL-quantized along 2F.
    """
    dy_e = np.asarray(dy_e, dtype=np.float64)
    F = w13_e.shape[0] // 2
    h13 = fwd_e["h13"]
    out = {}
    if exact:
        dyr = dyc = dy_e
        w2c, w13c = w2_e, w13_e
        hc, xc = fwd_e["h"], np.asarray(x_e, dtype=np.float64)
    else:
        out["dy_row"] = quantize_rows(dy_e)
        out["dy_col"] = quantize_cols(dy_e)
        dyr = dequantize_rows(*out["dy_row"])
        dyc = dequantize_rows(*out["dy_col"]).T
        w2c = dequantize_rows(*quantize_cols(w2_e)).T       # [D, F], blocks along D
        w13c = dequantize_rows(*quantize_cols(w13_e)).T     # [2F, D], blocks along 2F
        hc = dequantize_rows(*fwd_e["h_col"]).T
        xc = dequantize_rows(*fwd_e["x_col"]).T
    dh = dyr @ w2c
    if exact:
        a, b = h13[:, :F], h13[:, F:]
        s = _sigmoid(a)
        dh13 = np.concatenate([dh * b * s * (1.0 + a * (1.0 - s)), dh * a * s], axis=1)
        gr = gc = dh13
    else:
        dh = round_to_bf16(dh)
        dh13 = dswiglu(dh, h13)
        out["dh13_row"] = quantize_rows(dh13)
        out["dh13_col"] = quantize_cols(dh13)
        gr = dequantize_rows(*out["dh13_row"])
        gc = dequantize_rows(*out["dh13_col"]).T
    out.update(dw2=dyc.T @ hc, dx=gr @ w13c, dw13=gc.T @ xc, dh=dh, dh13=dh13)
    return out


def _segments(offsets, experts):
    E = len(offsets) - 1
    for e in (range(E) if experts is None else experts):
        yield e, int(offsets[e]), int(offsets[e + 1])


def moe_mlp_fwd(x, w13, w2, offsets, experts=None, exact=False):
    """Forward of the routed-experts MLP over the expert-major padded layout.

    x [M, D], w13 [E, 2F, D] (rows 0..F-1 gate = w1, F..2F-1 up = w3),
    w2 [E, D, F], as float64 arrays of bf16 values.  Returns full-size arrays
    y, h13, h (rows outside the listed experts' segments are NaN) and
    'experts': {e: per-expert dict of expert_fwd}.
    """
    x = np.asarray(x, dtype=np.float64)
    M, D = x.shape
    F = w13.shape[1] // 2
    y = np.full((M, D), np.nan)
    h13 = np.full((M, 2 * F), np.nan)
    h = np.full((M, F), np.nan)
    per = {}
    for e, lo, hi in _segments(offsets, experts):
        if hi == lo:
            continue
        r = expert_fwd(x[lo:hi], w13[e], w2[e], exact)
        y[lo:hi], h13[lo:hi], h[lo:hi] = r["y"], r["h13"], r["h"]
        per[e] = r
    return dict(y=y, h13=h13, h=h, experts=per)


def moe_mlp_bwd(dy, fwd, x, w13, w2, offsets, experts=None, exact=False):
    """Backward: dx [M, D] (NaN outside the listed segments), dW13 [E, 2F, D],
    dW2 [E, D, F] (NaN for experts not listed, exact zeros for listed experts
    without rows), plus 'experts': {e: per-expert dict of expert_bwd}."""
    dy = np.asarray(dy, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    M, D = dy.shape
    E, F2, _ = w13.shape
    dx = np.full((M, D), np.nan)
    dw13 = np.full((E, F2, D), np.nan)
    dw2 = np.full((E, D, F2 // 2), np.nan)
    per = {}
    for e, lo, hi in _segments(offsets, experts):
        if hi == lo:
            dw13[e] = 0.0
            dw2[e] = 0.0
            continue
        r = expert_bwd(dy[lo:hi], fwd["experts"][e], x[lo:hi], w13[e], w2[e], exact)
        dx[lo:hi], dw13[e], dw2[e] = r["dx"], r["dw13"], r["dw2"]
        per[e] = r
    return dict(dx=dx, dw13=dw13, dw2=dw2, experts=per)
