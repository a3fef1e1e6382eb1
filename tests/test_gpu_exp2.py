"""The FMA-pipe exp2 used for a share of the attention softmax exponentials
(Cody-Waite split plus a fitted degree-3 minimax polynomial) against the
hardware exp2 (torch.exp2 on the GPU) and against float64, within the bound
the fit guarantees (8.6e-5 relative, plus float32 rounding)."""
import ctypes

import numpy as np
import pytest
import torch

from kv_cache_compression_fkv_b200 import _lib

pytestmark = pytest.mark.gpu
BOUND = 8.6e-5 + 4 * 2.0 ** -24


def _emulated(x: torch.Tensor) -> torch.Tensor:
    y = torch.empty_like(x)
    st = _lib.load().fkv_exp2_emulated(x.data_ptr(), y.data_ptr(), x.numel(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    return y


def test_exp2_poly_relative_error(cuda_device):
    # the softmax feeds it x = s*scale*log2e - m, in (-inf, 8]
    x = torch.cat([torch.linspace(-126.0, 8.0, 2_000_001),
                   torch.arange(-126, 9, dtype=torch.float32),          # integers: exact
                   torch.rand(100_000) * 134.0 - 126.0]).cuda()
    y = _emulated(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= BOUND, rel
    hw = torch.exp2(x)  # the hardware / CUDA exp2 in float32
    rel_hw = ((y.double() - hw.double()).abs() / hw.double()).max().item()
    assert rel_hw <= BOUND + 2.0 ** -22, rel_hw
    ints = torch.arange(-126, 9, dtype=torch.float32).cuda()
    assert torch.equal(_emulated(ints), torch.exp2(ints.double()).float())  # exact powers of 2


def test_exp2_poly_special_inputs(cuda_device):
    x = torch.tensor([float("-inf"), -1000.0, -127.0, -126.5, 0.0, -0.0, 8.0], device="cuda")
    y = _emulated(x).cpu().numpy()
    assert y[0] == 0.0 and y[1] == 0.0 and y[2] == 0.0      # clamped to 2^-127 -> exact zero
    assert 0.0 <= y[3] < 2.0 ** -126                          # below the normal range
    assert y[4] == 1.0 and y[5] == 1.0 and y[6] == 256.0
