"""Shared helpers of the test suite (layout reference, comparisons, seeded inputs)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import mx


def has_gpu() -> bool:
    return torch.cuda.is_available()


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> float64 numpy (exact)."""
    return t.detach().float().cpu().double().numpy()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def mma_index(R: int, C: int) -> np.ndarray:
    """Index map plain [R, C/32] -> offset in the tensor-core (MMA) scale layout.

    512-byte atoms of 128 rows x 4 column blocks; atom (r/128, kb/4) at
    ((r/128)*(C/128) + kb/4)*512; inside it row r, block kb at
    (r%32)*16 + ((r%128)/32)*4 + kb%4.
    """
    r = np.arange(R)[:, None]
    kb = np.arange(C // 32)[None, :]
    return ((r // 128) * (C // 128) + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4


def mma_to_plain(flat: np.ndarray, R: int, C: int) -> np.ndarray:
    return np.asarray(flat).reshape(-1)[mma_index(R, C)]


def plain_to_mma(plain: np.ndarray) -> np.ndarray:
    R, nb = plain.shape
    out = np.zeros(R * nb, dtype=np.uint8)
    out[mma_index(R, nb * 32)] = plain
    return out


def rel_fro(a: np.ndarray, ref: np.ndarray) -> float:
    d = np.linalg.norm(a - ref)
    n = np.linalg.norm(ref)
    return float(d / n) if n > 0 else float(d)


def assert_gemm_close(got: np.ndarray, ref: np.ndarray, what: str, rel=2e-3, absf=1e-2):
    """The GEMM bar: relative Frobenius <= 2e-3 and max-abs <= 1e-2 * max|ref|."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    rf = rel_fro(got, ref)
    ma = float(np.abs(got - ref).max()) if ref.size else 0.0
    mr = float(np.abs(ref).max()) if ref.size else 0.0
    assert rf <= rel, f"{what}: rel Frobenius {rf:.3e} > {rel}"
    assert ma <= absf * mr + 1e-30, f"{what}: max abs {ma:.3e} > {absf} * {mr:.3e}"
    return rf, ma / (mr + 1e-30)


def code_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance between E4M3 codes in representable steps (sign-magnitude order)."""
    def lin(c):
        c = c.astype(np.int64)
        mag = c & 0x7F
        return np.where(c & 0x80, -mag, mag)
    return np.abs(lin(a) - lin(b))


def assert_codes_close(got_codes, ref_codes, got_scales, ref_scales, what, frac=0.999):
    """Fused-epilogue bar: >= 99.9 % of codes equal, the rest off by at most one code.

    Both operands are [rows, cols] codes with plain [rows, cols/32] scales.
    Where the block scales agree "one code" is one step of the E4M3 grid.
    Where they differ (the block maximum crossed a power of two after a
    one-ulp bf16 difference upstream) the two dequantized values are compared
    on the coarser block's grid: they must be at most one step apart there.
    """
    gc, rc = np.asarray(got_codes), np.asarray(ref_codes)
    gs, rs = np.asarray(got_scales).astype(np.int64), np.asarray(ref_scales).astype(np.int64)
    n = gc.shape[-1]
    gse = np.repeat(gs, 32, axis=-1)[..., :n]
    rse = np.repeat(rs, 32, axis=-1)[..., :n]
    eq = (gc == rc) & (gse == rse)
    f = float(eq.mean())
    assert f >= frac, f"{what}: only {f:.6f} of codes equal"
    idx = np.nonzero(~eq)
    if idx[0].size:
        s = np.maximum(gse[idx], rse[idx]) - 127
        vg = mx.e4m3_decode(gc[idx]) * np.ldexp(1.0, gse[idx] - 127 - s)
        vr = mx.e4m3_decode(rc[idx]) * np.ldexp(1.0, rse[idx] - 127 - s)
        big = np.maximum(np.abs(vg), np.abs(vr))
        step = np.ldexp(1.0, np.maximum(np.frexp(big)[1] - 4, -9))
        off = np.abs(vg - vr) > step * (1 + 1e-12)
        assert not off.any(), f"{what}: {int(off.sum())} codes off by more than one step"
    return f, float((gs != rs).mean())
