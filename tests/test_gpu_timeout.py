"""Failure detection on the GPU without a GPU fault: a bounded device wait that
runs out.

``fkv_diag_attend_timeout`` runs the bf16 tensor-core attention with a short
wait limit while CTA 0 withholds the completion signal of its first logit
tile (the MMAs behind it are issued and complete).  The softmax warps of CTA 0
give up waiting, every role of that CTA winds down (bounded waits for its own
copies and MMAs, tensor memory freed), the kernel returns, and the workspace
status word reads FKV_ERR_TIMEOUT with CTA 0 as the detail.  The other CTAs
finish their work units normally, and the same context then runs the normal
attention again, bit-identical to the call before the failure.
"""
import ctypes

import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from kv_cache_compression_fkv_b200 import _lib
from tests import parity

pytestmark = pytest.mark.gpu

WAIT_CYCLES = 1 << 22  # about 2 ms at the B200's clocks


def _attend(lib, p, d, o, out, diag):
    ptr = lambda t: t.data_ptr()  # noqa: E731
    stream = torch.cuda.current_stream().cuda_stream
    args = (ctypes.byref(p), ptr(d["q_cur"]), ptr(d["k_cur"]), ptr(d["v_cur"]), ptr(o["k_comp"]),
            ptr(o["v_comp"]), ptr(o["kept_cnt"]), ptr(out))
    if diag:
        return lib.fkv_diag_attend_timeout(*args, WAIT_CYCLES, ptr(o["ws"]), stream)
    return lib.fkv_attend_compressed(*args, ptr(o["ws"]), stream)


def _reset_status(lib, o):
    st = lib.fkv_workspace_init(o["ws"].data_ptr(), o["ws"].numel(),
                                torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FKV_OK


def test_withheld_signal_times_out_and_the_context_stays_usable(cuda_device):
    w = wl.scaled(wl.get("480p"), name="timeout", H=2, T=256, F=4, Fc=2, n_static=1,
                  static_frames=(0, 2), k_dynamic=2, score_stride=3, seed=51)
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    fkv.step(p, d, o)
    assert fkv.read_status(o["ws"]) == (0, -1)
    ref = o["out"].clone()
    lib = _lib.load()

    # the failing call: returns FKV_OK (launched), the device status records the timeout
    out = torch.full_like(ref, float("nan"))
    assert _attend(lib, p, d, o, out, diag=True) == _lib.FKV_OK
    torch.cuda.synchronize()
    assert fkv.read_status(o["ws"]) == (_lib.FKV_ERR_TIMEOUT, 0)
    # CTA 0 owns the first work unit only (8 units, 8 CTAs): query tile 0 of
    # head 0 is left unwritten; every other unit is the attention, bit for bit
    assert bool(torch.isnan(out[0, 0, :128]).all())
    assert torch.equal(out[0, 0, 128:], ref[0, 0, 128:])
    assert torch.equal(out[0, 1:], ref[0, 1:])

    # the same context afterwards: the normal call, twice, equals the earlier result
    for _ in range(2):
        _reset_status(lib, o)
        again = torch.full_like(ref, float("nan"))
        assert _attend(lib, p, d, o, again, diag=False) == _lib.FKV_OK
        torch.cuda.synchronize()
        assert fkv.read_status(o["ws"]) == (0, -1)
        assert torch.equal(again, ref)


def test_diag_rejects_unsupported_requests(cuda_device):
    w = wl.scaled(wl.get("480p"), name="timeout_args", H=2, T=256, F=4, Fc=2, n_static=1,
                  static_frames=(0, 2), k_dynamic=2, score_stride=3, seed=52)
    p = fkv.params_for(w)
    d = parity.upload(wl.generate(w))
    o = fkv.allocate(p)
    lib = _lib.load()
    ptr = lambda t: t.data_ptr()  # noqa: E731
    base = (ctypes.byref(p), ptr(d["q_cur"]), ptr(d["k_cur"]), ptr(d["v_cur"]), ptr(o["k_comp"]),
            ptr(o["v_comp"]), ptr(o["kept_cnt"]), ptr(o["out"]))
    s = torch.cuda.current_stream().cuda_stream
    assert lib.fkv_diag_attend_timeout(*base, 100, ptr(o["ws"]), s) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_diag_attend_timeout(*base, 1 << 40, ptr(o["ws"]), s) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_diag_attend_timeout(*base, WAIT_CYCLES, None, s) == _lib.FKV_ERR_WORKSPACE
