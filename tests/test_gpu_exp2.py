"""The kernels' FMA-pipe exp2 (range reduction + fitted cubic) against CUDA's exp2f (GPU)."""

import ctypes

import pytest

pytestmark = pytest.mark.gpu


def test_poly_exp2_relative_error(splitkv):
    import torch
    x = torch.cat([torch.linspace(-126.0, 9.0, 1 << 20, device="cuda"),
                   torch.rand(1 << 20, device="cuda") * -20.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 8.0, -125.5], device="cuda")])
    y = torch.empty_like(x)
    st = splitkv._lib.splitkv_selftest_exp2(x.data_ptr(), y.data_ptr(), ctypes.c_int64(x.numel()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    ref = torch.exp2(x.double())
    keep = x > -120.0                       # far below fp32 normal range the result is only "tiny"
    rel = ((y.double() - ref).abs() / ref)[keep]
    assert float(rel.max()) < 1e-4, float(rel.max())
    tiny = y[~keep]
    assert bool((tiny >= 0).all()) and float(tiny.max()) < 1e-30


def test_poly_exp2_is_zero_below_the_normal_range_and_for_minus_infinity(splitkv):
    """Masked scores reach the exponential as -inf: the FMA-pipe exp2 gives exactly 0 there,
    as the MUFU one does, and for any input below -126."""
    import torch
    x = torch.tensor([float("-inf"), -1e30, -300.0, -127.0, -126.5], device="cuda")
    y = torch.full_like(x, 1.0)
    st = splitkv._lib.splitkv_selftest_exp2(x.data_ptr(), y.data_ptr(), ctypes.c_int64(x.numel()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert y.cpu().tolist() == [0.0] * 5
