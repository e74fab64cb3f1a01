"""C-ABI library: loads, exports every declared symbol, rejects bad arguments
on the host before touching the GPU (these run without a GPU)."""
import ctypes

import pytest
import torch

import mxfp8_block_scaled_routed_b200 as mxk

P = ctypes.c_void_p
FAKE = 0x10000          # aligned dummy device address: never dereferenced on the paths below
MIS = 0x10001           # misaligned


@pytest.fixture(scope="module")
def L():
    return mxk.lib()


def test_every_header_function_is_exported(L):
    names = mxk.header_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n


def test_version_and_error_string(L):
    assert b"sm_100a" in L.mxmoe_version()
    assert isinstance(L.mxmoe_last_error_message(), bytes)


def _err(L):
    return L.mxmoe_last_error_message().decode()


def test_gemm_rejects_bad_pad_and_shapes(L):
    s = L.mxfp8_grouped_gemm(P(FAKE), P(FAKE), 256, 256, P(FAKE), P(FAKE), 4, 256, P(FAKE), 100, P(FAKE), None)
    assert s == 2 and "pad_multiple" in _err(L)
    s = L.mxfp8_grouped_gemm(P(FAKE), P(FAKE), 200, 256, P(FAKE), P(FAKE), 4, 256, P(FAKE), 128, P(FAKE), None)
    assert s == 2 and "M=200" in _err(L)
    s = L.mxfp8_grouped_gemm(P(FAKE), P(FAKE), 256, 256, P(FAKE), P(FAKE), 4, 256, None, 128, P(FAKE), None)
    assert s == 1 and "expert_offsets" in _err(L)
    s = L.mxfp8_grouped_gemm(P(MIS), P(FAKE), 256, 256, P(FAKE), P(FAKE), 4, 256, P(FAKE), 128, P(FAKE), None)
    assert s == 3 and "a is not 16-byte aligned" in _err(L)
    s = L.mxfp8_grouped_gemm(P(FAKE), P(FAKE), 256, 256, P(FAKE), P(FAKE), 0, 256, P(FAKE), 128, P(FAKE), None)
    assert s == 2 and "E=0" in _err(L)


def test_wgrad_and_fused_reject(L):
    s = L.mxfp8_grouped_gemm_wgrad(P(FAKE), P(FAKE), 256, P(FAKE), P(FAKE), 100, 256, P(FAKE), None, 4, 128, P(FAKE),
                                   None)
    assert s == 2 and "Kx=100" in _err(L)
    s = L.mxfp8_grouped_gemm_swiglu_quant(P(FAKE), P(FAKE), 256, 256, P(FAKE), P(FAKE), 4, 96, P(FAKE), 128,
                                          None, P(FAKE), P(FAKE), P(FAKE), P(FAKE), None)
    assert s == 2 and "F=96" in _err(L)
    s = L.mxfp8_grouped_gemm_dswiglu_quant(P(FAKE), P(FAKE), 256, 256, P(FAKE), P(FAKE), 4, 128, P(FAKE), 128,
                                           None, P(FAKE), P(FAKE), P(FAKE), P(FAKE), None)
    assert s == 1 and "h13" in _err(L)


def test_quantize_rejects(L):
    s = L.mxfp8_quantize(P(FAKE), 1, 64, 64, 0, 0, None, None, None, None, None)
    assert s == 9
    s = L.mxfp8_quantize(P(FAKE), 1, 48, 64, 2, 0, None, None, P(FAKE), P(FAKE), None)
    assert s == 2 and "rows % 32" in _err(L)
    s = L.mxfp8_quantize(P(FAKE), 1, 64, 64, 1, 0, None, P(FAKE), None, None, None)
    assert s == 1
    s = L.mxfp8_quantize(P(FAKE), 1, 256, 200, 1, 1, P(FAKE), P(FAKE), None, None, None)
    assert s == 2 and "MMA" in _err(L)
    s = L.mxfp8_swiglu_quant(P(FAKE), 64, 48, 1, 0, P(FAKE), P(FAKE), None, None, None)
    assert s == 2


def test_composite_workspace_checks(L):
    M, D, E, F = 512, 256, 4, 256
    need_f = L.mxmoe_workspace_size(M, D, E, F, 1)
    need_b = L.mxmoe_workspace_size(M, D, E, F, 2)
    # x_row + w13 + w2 + h_row codes (+ scales, alignment)
    assert need_f >= M * D + E * 2 * F * D + E * D * F + M * F
    assert need_b >= 2 * M * D + E * 3 * F * D + 2 * M * 2 * F
    saved = mxk._Saved(FAKE, FAKE, FAKE, FAKE, FAKE)
    s = L.moe_mlp_fwd(P(FAKE), M, D, P(FAKE), P(FAKE), E, F, P(FAKE), 128, P(FAKE), ctypes.byref(saved),
                      P(FAKE), need_f - 1, None)
    assert s == 8 and "workspace" in _err(L)
    s = L.moe_mlp_bwd(P(FAKE), M, D, P(FAKE), P(FAKE), E, F, P(FAKE), 128, ctypes.byref(saved), P(FAKE), P(FAKE),
                      P(FAKE), None, need_b, None)
    assert s == 8


def test_binding_refuses_cpu_tensors():
    x = torch.zeros(128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        mxk.mxfp8_quantize(x)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mxk, "_lib", None)
    monkeypatch.setattr(mxk, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        mxk.lib()


def test_route_capacity_and_workspace_arithmetic(L):
    # 16384 tokens x top-8 over 256 experts padded to 256: at most 255 pad rows per expert
    assert L.mxmoe_route_capacity(16384, 8, 256, 256) == 131072 + 256 * 255
    assert L.mxmoe_route_capacity(3, 2, 3, 4) == 128                 # 6 + 3*3 = 15 -> one 128-row tile
    assert L.mxmoe_route_capacity(1, 1, 64, 128) == 128               # only one expert can be busy
    assert L.mxmoe_route_capacity(0, 8, 64, 256) == 0
    assert L.mxmoe_route_capacity(-1, 8, 64, 256) == -1
    assert L.mxmoe_route_capacity(10, 2, 4, 0) == -1
    assert L.mxmoe_route_workspace_size(16384, 8, 256) == 32 * 256 * 4
    assert L.mxmoe_route_workspace_size(1, 1, 7) == 7 * 4
    assert L.mxmoe_route_workspace_size(0, 1, 7) == 0


def test_dispatcher_rejects(L):
    s = L.mxmoe_route(P(FAKE), 16, 2, 2048, 128, 1024, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1 << 20, None)
    assert s == 2 and "E=2048" in _err(L)
    s = L.mxmoe_route(P(FAKE), 16, 2, 8, 0, 1024, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1 << 20, None)
    assert s == 9
    s = L.mxmoe_route(P(FAKE), 16, 2, 8, 128, 1024, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 4, None)
    assert s == 8 and "workspace" in _err(L)
    s = L.mxmoe_route(None, 16, 2, 8, 128, 1024, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1 << 20, None)
    assert s == 1
    s = L.mxmoe_permute_quant(P(FAKE), 16, 200, P(FAKE), 2, None, 256, None, 3, 1, P(FAKE), P(FAKE), P(FAKE),
                              P(FAKE), None)
    assert s == 2
    s = L.mxmoe_permute_quant(P(MIS), 16, 256, P(FAKE), 2, None, 256, None, 3, 1, P(FAKE), P(FAKE), P(FAKE),
                              P(FAKE), None)
    assert s == 3
    s = L.mxmoe_permute_quant(P(FAKE), 16, 256, P(FAKE), 2, None, 256, None, 2, 1, P(FAKE), P(FAKE), None,
                              P(FAKE), None)
    assert s == 1
    s = L.mxmoe_unpermute_combine(P(FAKE), 256, 100, P(FAKE), None, 16, 2, P(FAKE), None)
    assert s == 2 and "D=100" in _err(L)
    s = L.mxmoe_unpermute_combine(P(FAKE), 256, 128, P(FAKE), None, 16, 65, P(FAKE), None)
    assert s == 2
    s = L.mxmoe_combine_weight_grad(P(FAKE), P(MIS), 256, 128, P(FAKE), 16, 2, P(FAKE), None)
    assert s == 3


def test_layer_composites_reject(L):
    T, k, D, E, F, pad = 512, 2, 256, 4, 256, 128
    need_f = L.moe_layer_workspace_size(T, k, D, E, F, pad, 1)
    need_b = L.moe_layer_workspace_size(T, k, D, E, F, pad, 2)
    m_cap = L.mxmoe_route_capacity(T, k, E, pad)
    assert need_f >= m_cap * D + m_cap * F and need_b >= 2 * m_cap * D + 4 * m_cap * F + 2 * m_cap * D
    assert L.moe_layer_workspace_size(T, k, D, E, F, pad, 3) == 0
    saved = mxk._LayerSaved(FAKE, FAKE, FAKE, FAKE, mxk._Saved(FAKE, FAKE, FAKE, FAKE, FAKE))
    qw = mxk._QWeights(*([FAKE] * 8))
    s = L.moe_layer_fwd_q(P(FAKE), T, D, P(FAKE), P(FAKE), k, ctypes.byref(qw), E, F, 100, P(FAKE),
                          ctypes.byref(saved), P(FAKE), need_f, None)
    assert s == 2 and "pad_multiple" in _err(L)
    s = L.moe_layer_fwd_q(P(FAKE), T, D, P(FAKE), P(FAKE), 5, ctypes.byref(qw), E, F, pad, P(FAKE),
                          ctypes.byref(saved), P(FAKE), need_f, None)
    assert s == 2 and "top_k" in _err(L)
    s = L.moe_layer_fwd_q(P(FAKE), T, D, P(FAKE), P(FAKE), k, ctypes.byref(qw), E, F, pad, P(FAKE),
                          ctypes.byref(saved), P(FAKE), need_f - 1, None)
    assert s == 8 and "workspace" in _err(L)
    s = L.moe_layer_bwd_q(P(FAKE), T, D, None, k, ctypes.byref(qw), E, F, pad, ctypes.byref(saved), P(FAKE),
                          P(FAKE), P(FAKE), None, P(FAKE), need_b, None)
    assert s == 1
