"""moe_mlp_fwd_noalloc: the forward composite for callers that cannot allocate.

Some callers (a plugin inside a host runtime that owns all device memory, or
code with a fixed memory budget) cannot hand the library a workspace.  This
entry point uses a scratch area compiled into the library instead.  The test
calls it through the C ABI twice in a row and checks both results against the
workspace-taking moe_mlp_fwd with the GEMM tolerance the other tests use.
"""
import ctypes

import numpy as np
import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk
import synth
from mxtest import assert_gemm_close, bf16_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _saved_struct(s):
    return mxk._Saved(s["h13"].data_ptr(), s["h_col_codes"].data_ptr(), s["h_col_scales"].data_ptr(),
                      s["x_col_codes"].data_ptr(), s["x_col_scales"].data_ptr())


def _noalloc(L, x, w13, w2, off, pad):
    M, D = x.shape
    E = off.numel() - 1
    F = w13.shape[1] // 2
    y = torch.full((M, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    saved = mxk.make_saved(M, D, F, DEV)
    st = _saved_struct(saved)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    s = L.moe_mlp_fwd_noalloc(x.data_ptr(), M, D, w13.data_ptr(), w2.data_ptr(), E, F, off.data_ptr(), pad,
                              y.data_ptr(), ctypes.byref(st), stream)
    assert s == 0, L.mxmoe_last_error().decode()
    torch.cuda.synchronize()
    return y, saved


def test_noalloc_forward_matches_workspace_forward_twice():
    L = mxk.lib()
    inp = synth.make_moe_inputs("tiny", 0)
    off = torch.from_numpy(inp.routing.offsets).to(DEV)
    pad = inp.spec.pad
    x, w13, w2 = inp.x.to(DEV), inp.w13.to(DEV), inp.w2.to(DEV)
    y_ref, saved_ref = mxk.moe_mlp_fwd(x, w13, w2, off, pad)
    torch.cuda.synchronize()
    for _ in range(2):
        y, saved = _noalloc(L, x, w13, w2, off, pad)
        assert_gemm_close(bf16_np(y), bf16_np(y_ref), "y (no-alloc vs workspace)")
        assert_gemm_close(bf16_np(saved["h13"]), bf16_np(saved_ref["h13"]), "h13 (no-alloc vs workspace)")
        for k in ("h_col_codes", "h_col_scales", "x_col_codes", "x_col_scales"):
            same = (saved[k] == saved_ref[k]).float().mean().item()
            assert same >= 0.999, (k, same)
    assert mxk.device_error() == 0


def test_noalloc_rejects_layers_larger_than_its_scratch():
    L = mxk.lib()
    M, D, E, F = 8192, 2048, 4, 1024            # forward workspace > 32 MiB
    assert L.mxmoe_workspace_size(M, D, E, F, 1) > (32 << 20)
    saved = mxk._Saved(0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    s = L.moe_mlp_fwd_noalloc(0x10000, M, D, 0x10000, 0x10000, E, F, 0x10000, 128, 0x10000, ctypes.byref(saved),
                              None)
    assert s == 8
    assert "static scratch" in L.mxmoe_last_error().decode()
