"""The hardware rates the attention kernel's design rests on, measured by the
library's diagnostics (one CTA per SM, clock64 in CTA 0):

  * one thread issuing tcgen05.mma back to back keeps the tensor pipe at its
    nominal rate for the attention's M128 N128 K16 shapes (Q.K^T from shared
    memory, P.V with A from tensor memory and V MN-major), with either B
    layout and either A source, and through the attention's grouped issue
    helpers: the issue is not what bounds the kernel;  an N = 256 MMA takes
    twice as long, an N = 64 one is bound by the issue itself;
  * an M = 64 MMA takes as long as an M = 128 one (half the FLOP rate);
  * one warp keeps its sub-partition's MUFU busy (about 8 cycles per ex2 warp
    instruction); two warps share it (about twice as long each).

The bounds below are loose: they check the shape of the behaviour, not an
exact cycle count."""
import ctypes

import pytest
import torch

from kv_cache_compression_fkv_b200 import _lib

pytestmark = pytest.mark.gpu


def _mma(shape, busy=0, n=256):
    lib = _lib.load()
    cyc = torch.zeros(4, dtype=torch.int64, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for _ in range(2):  # the second launch is timed warm
        assert lib.fkv_diag_mma_rate(shape, n, busy, cyc.data_ptr(), ws.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert int(ws.view(torch.int32)[0]) == 0
    issue, total = (int(v) / n for v in cyc[:2].tolist())
    return issue, total


def _ex2(warps, n=4096):
    lib = _lib.load()
    cyc = torch.zeros(2, dtype=torch.int64, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        assert lib.fkv_diag_ex2_rate(n, warps, cyc.data_ptr(), s) == 0
    torch.cuda.synchronize()
    return int(cyc[0]) / n


def test_mma_issue_keeps_the_tensor_pipe_busy(cuda_device):
    r = {shape: _mma(shape) for shape in range(11)}
    busy_issue, _ = _mma(6, busy=1)
    names = ["QK", "PV", "N256", "N64", "SS MN-major B", "TS K-major B", "QK probe", "PV probe",
             "e4m3 QK", "e4m3 PV", "M64"]
    print("cycles per MMA (issue/complete): " +
          ", ".join(f"{names[k]} {r[k][0]:.1f}/{r[k][1]:.1f}" for k in range(11)) +
          f", QK probe with busy neighbours {busy_issue:.1f}")
    qk = r[0][0]
    # M128 N128 K16 bf16 = 64 cycles of tensor work: every operand source and
    # layout, and the attention's grouped issue, keep pace with it
    for k in (0, 1, 4, 5, 6, 7):
        assert 60.0 <= r[k][1] <= 75.0, names[k]
    assert 1.8 <= r[2][0] / qk <= 2.2       # N = 256: twice the work, twice the time
    assert r[3][0] < 0.9 * qk               # N = 64: faster, though not half
    assert busy_issue <= 1.1 * r[6][0]      # busy warps beside the issuer cost nothing
    # e4m3 M128 N128 K32: 64 cycles at the nominal rate (twice bf16's FLOPs per
    # cycle); never faster than that
    for k in (8, 9):
        assert 60.0 <= r[k][1] <= 200.0, names[k]
    # M = 64: half the work of shape 0 in the same time (half the FLOP rate),
    # so a 64-row tile saves no tensor time over a padded 128-row one
    assert 0.9 * r[0][1] <= r[10][1] <= 1.1 * r[0][1]


def test_one_warp_saturates_its_mufu(cuda_device):
    one, two, four = _ex2(1), _ex2(2), _ex2(4)
    print(f"cycles per ex2 warp instruction: 1 warp {one:.2f}, 2 warps {two:.2f}, 4 warps {four:.2f}")
    assert 7.5 <= one <= 12.0
    assert 1.7 <= two / one <= 2.3 and 3.4 <= four / one <= 4.6


def test_diag_rejects_bad_sizes(cuda_device):
    lib = _lib.load()
    cyc = torch.zeros(4, dtype=torch.int64, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert lib.fkv_diag_mma_rate(11, 256, 0, cyc.data_ptr(), ws.data_ptr(), s) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_diag_mma_rate(0, 5000, 0, cyc.data_ptr(), ws.data_ptr(), s) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_diag_mma_rate(0, 12, 0, cyc.data_ptr(), ws.data_ptr(), s) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_diag_ex2_rate(12, 1, cyc.data_ptr(), s) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_diag_ex2_rate(4096, 5, cyc.data_ptr(), s) == _lib.FKV_ERR_SHAPE
