"""moe_mlp_fwd_noalloc: the forward composite for callers that cannot allocate.

Some callers (a plugin inside a host runtime that owns all device memory, or
code with a fixed memory budget) cannot hand the library a workspace.  This
entry point uses a scratch area compiled into the library instead.  It runs
the same kernels as the workspace-taking moe_mlp_fwd on the same inputs, so
its outputs must be the same bits; the test calls it through the C ABI twice
for one layer, with a different layer's call in between (so the second call
starts on another layer's leftovers in the shared scratch), compares every
output with moe_mlp_fwd bit for bit and the result with the oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk
import synth
from mxtest import assert_codes_close, assert_gemm_close, bf16_np, mma_to_plain, u8
from oracle import mx

pytestmark = pytest.mark.gpu
DEV = "cuda"
SAVED_KEYS = ("h13", "h_col_codes", "h_col_scales", "x_col_codes", "x_col_scales")


def _saved_struct(s):
    return mxk._Saved(*(s[k].data_ptr() for k in SAVED_KEYS))


def _filled_outputs(M, D, F):
    """y and saved buffers holding a sentinel (NaN / 0x5A), so bytes a call
    leaves untouched compare equal and bytes it writes are checked."""
    y = torch.full((M, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    saved = mxk.make_saved(M, D, F, DEV)
    for k in SAVED_KEYS:
        saved[k].fill_(0x5A if saved[k].dtype == torch.uint8 else float("nan"))
    return y, saved


def _noalloc(L, x, w13, w2, off, pad):
    M, D = x.shape
    E = off.numel() - 1
    F = w13.shape[1] // 2
    y, saved = _filled_outputs(M, D, F)
    st = _saved_struct(saved)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    s = L.moe_mlp_fwd_noalloc(x.data_ptr(), M, D, w13.data_ptr(), w2.data_ptr(), E, F, off.data_ptr(), pad,
                              y.data_ptr(), ctypes.byref(st), stream)
    assert s == 0, L.mxmoe_last_error_message().decode()
    torch.cuda.synchronize()
    return y, saved


def _same(a, b):
    """Bitwise equality (NaN sentinels included)."""
    return torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def _dev(inp):
    return (torch.from_numpy(inp.routing.offsets).to(DEV), inp.x.to(DEV), inp.w13.to(DEV), inp.w2.to(DEV))


def test_noalloc_forward_equals_workspace_forward_twice():
    L = mxk.lib()
    inp = synth.make_moe_inputs("tiny", 0)                               # pad 128
    other = synth.make_moe_inputs(synth.Spec("other", 4, 256, 256, 700, 2, 256, None, 0, 0.02), 9)
    off, x, w13, w2 = _dev(inp)
    pad = inp.spec.pad
    M, D = x.shape
    F = w13.shape[1] // 2
    y_ref, saved_ref = _filled_outputs(M, D, F)
    mxk.moe_mlp_fwd(x, w13, w2, off, pad, y=y_ref, saved=saved_ref)
    torch.cuda.synchronize()
    rows = int(inp.routing.offsets[-1])
    for call in range(2):
        y, saved = _noalloc(L, x, w13, w2, off, pad)
        assert _same(y, y_ref), f"y differs (call {call})"
        for k in SAVED_KEYS:
            assert _same(saved[k], saved_ref[k]), f"{k} differs (call {call})"
        # another layer (more rows, pad 256) through the same scratch before the next call
        o_off, o_x, o_w13, o_w2 = _dev(other)
        _noalloc(L, o_x, o_w13, o_w2, o_off, other.spec.pad)
    assert mxk.device_error() == 0

    # the no-allocation result against the oracle
    f = lambda t: t.float().double().cpu().numpy()
    ro = inp.routing.offsets
    rf = mx.moe_mlp_fwd(f(inp.x), f(inp.w13), f(inp.w2), ro)
    assert_gemm_close(bf16_np(y)[:rows], rf["y"][:rows], "y (no-alloc vs oracle)")
    assert_gemm_close(bf16_np(saved["h13"])[:rows], rf["h13"][:rows], "h13 (no-alloc vs oracle)")
    for e in rf["experts"]:
        lo, hi = int(ro[e]), int(ro[e + 1])
        ref = rf["experts"][e]
        np.testing.assert_array_equal(u8(saved["x_col_codes"])[:, lo:hi], ref["x_col"][0])
        hcs = mma_to_plain(u8(saved["h_col_scales"]), F, M)[:, lo // 32:hi // 32]
        assert_codes_close(u8(saved["h_col_codes"])[:, lo:hi], ref["h_col"][0], hcs, ref["h_col"][1],
                           f"h COL[e={e}] (no-alloc vs oracle)")


def test_noalloc_rejects_layers_larger_than_its_scratch():
    L = mxk.lib()
    M, D, E, F = 8192, 2048, 4, 1024            # forward workspace > 32 MiB
    assert L.mxmoe_workspace_size(M, D, E, F, 1) > (32 << 20)
    saved = mxk._Saved(0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    s = L.moe_mlp_fwd_noalloc(0x10000, M, D, 0x10000, 0x10000, E, F, 0x10000, 128, 0x10000, ctypes.byref(saved),
                              None)
    assert s == 8
    assert "static scratch" in L.mxmoe_last_error_message().decode()
