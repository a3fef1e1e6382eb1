"""fkv_score_segments_noalloc, the scoring entry point for callers that cannot
allocate device memory (for example a plugin that its host runtime hands only
input and output buffers, or a serving loop that reserved all of HBM up front).

It must give the same segment scores as fkv_score_segments with a caller
workspace, on two calls in a row (the static scratch it uses is shared and
keeps the previous call's contents), and must refuse sizes whose scratch is
above its static maximum without launching anything.  This file is collected
last so that a run stopping at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from kv_cache_compression_fkv_b200 import _lib
from tests import parity

pytestmark = pytest.mark.gpu


def _noalloc(p, d, seg_score):
    lib = _lib.load()
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    return lib.fkv_score_segments_noalloc(
        ctypes.byref(p), ptr(d.get("q_cur")), ptr(d.get("q_score")), ptr(d["k_hist"]),
        ptr(d.get("k_cur")), ptr(d.get("head_role")), seg_score.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def _assert_close(got, ref):
    g, r = got.double().cpu().numpy(), ref.double().cpu().numpy()
    for idx in np.ndindex(r.shape[:2]):
        scale = np.max(np.abs(r[idx]))
        if scale == 0:
            assert np.array_equal(g[idx], r[idx])
            continue
        rel = np.max(np.abs(g[idx] - r[idx])) / scale
        assert rel <= parity.SCORE_REL, (idx, rel)


@pytest.mark.parametrize("case", ["480p", "token_small"])
def test_noalloc_matches_workspace_scoring_twice(cuda_device, case):
    if case == "480p":
        w = wl.get("480p")
    else:
        w = wl.scaled(wl.get("token14b"), name="token_small", H=4, T=96, F=9, Fc=2, n_score_q=96,
                      sink_tokens=192, recent_tokens=192, keep_tokens=300, seed=41)
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    fkv.score_segments(p, d["q_cur"], d.get("q_score"), d["k_hist"], d.get("head_role"),
                       o["seg_score"], o["ws"])
    ref = o["seg_score"].clone()
    for _ in range(2):
        got = torch.full_like(ref, float("nan"))
        assert _noalloc(p, d, got) == _lib.FKV_OK
        torch.cuda.synchronize()
        _assert_close(got, ref)


def test_noalloc_rejects_scratch_above_its_maximum(cuda_device):
    w = wl.get("480p_30layer")  # 30 layers of per-block partial statistics: about 200 MB
    p = fkv.params_for(w)
    assert fkv.sizes(p)["ws_bytes"] > 16 << 20  # above the static maximum
    sentinel = torch.full((w.L, w.H, w.F), 7.0, device="cuda")
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    st = _noalloc(p, {"q_cur": dummy, "k_hist": dummy,
                      "head_role": torch.ones(1, dtype=torch.uint8, device="cuda")}, sentinel)
    assert st == _lib.FKV_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((sentinel == 7.0).all())
