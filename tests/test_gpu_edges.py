"""Edge cases of the CUDA path against the oracle: budgets at 0 and at the
maximum, all-static and all-dynamic layers, an empty history, engineered
exact ties (lower index wins), 0% pruning equal to full attention, and the
device-side error reporting (no fault: the kernels clamp and record)."""
import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def _small(**kw):
    base = wl.scaled(wl.get("480p"), name="edge", H=4, T=130, F=6, Fc=1, n_static=2,
                     static_frames=(0, 5), k_dynamic=2, score_stride=2, seed=31)
    return wl.scaled(base, **kw)


@pytest.mark.parametrize("k", [0, 1, 6])
def test_dynamic_budget_extremes(cuda_device, k):
    w = _small()
    x = wl.generate(w)
    x["k_per_head"][x["head_role"] == 1] = k
    res = parity.run_step(w, x, comp_rows=w.F * w.T)
    parity.check_step(w, x, res)
    assert (res["kept_cnt"][x["head_role"] == 1] == k).all()


@pytest.mark.parametrize("role", [0, 1])
def test_all_static_or_all_dynamic(cuda_device, role):
    w = _small()
    x = wl.generate(w)
    x["head_role"][:] = role
    x["static_mask"][:] = 0
    x["static_mask"][..., [1, 2, 4]] = 1
    x["k_per_head"][:] = 3
    res = parity.run_step(w, x, comp_rows=3 * w.T)
    parity.check_step(w, x, res)


def test_empty_history(cuda_device):
    w = _small(F=0, static_frames=(), k_dynamic=0)
    x = wl.generate(w)
    res = parity.run_step(w, x, comp_rows=0)
    assert (res["kept_cnt"] == 0).all()
    parity.check_step(w, x, res)


@pytest.mark.parametrize("T,F", [(96, 0), (40, 2), (128, 1), (128, 2)])
def test_few_key_blocks(cuda_device, T, F):
    """One to three 128-key blocks in total: one attention stream may be
    empty, or one block shorter than the other (its last PV then follows the
    other stream's extra S)."""
    w = _small(T=T, F=F, Fc=1, static_frames=tuple(range(F)), k_dynamic=F)
    x = wl.generate(w)
    res = parity.run_step(w, x, comp_rows=max(F * T, 0))
    parity.check_step(w, x, res)


def test_zero_pruning_is_full_attention_and_bit_identical(cuda_device):
    """mask = every frame, k = F: the output equals full attention over
    history + chunk, and is bit-identical to attending the raw history."""
    w = _small()
    x = wl.generate(w)
    x["static_mask"][:] = 1
    x["k_per_head"][:] = w.F
    res = parity.run_step(w, x, comp_rows=w.F * w.T)
    parity.check_step(w, x, res)
    p = fkv.params_for(w, comp_rows=w.F * w.T)
    d = parity.upload(x)
    o = fkv.allocate(p)
    cnt = torch.full((w.L, w.H), w.F, dtype=torch.int32, device="cuda")
    fkv.attend_compressed(p, d["q_cur"], d["k_cur"], d["v_cur"], d["k_hist"], d["v_hist"], cnt,
                          o["out"], o["ws"])
    assert torch.equal(o["out"].cpu(), res["out"])


def test_exact_frame_ties_pick_lower_index(cuda_device):
    """Every history frame of the dynamic heads is the same block of keys, so all
    frame masses are exactly equal; top-k must be frames 0..k-1.  T is a
    multiple of 128 so every frame is reduced in the same order."""
    w = _small(T=128, k_dynamic=3)
    x = wl.generate(w)
    blk = x["k_hist"][:, :, : w.T].clone()
    x["k_hist"].copy_(blk.repeat(1, 1, w.F, 1))
    res = parity.run_step(w, x)
    for h in range(w.H):
        if x["head_role"][0, h]:
            s = res["seg_score"][0, h]
            assert torch.all(s == s[0]), s
            assert parity.gpu_kept(res, 0, h).tolist() == [0, 1, 2]
    parity.check_step(w, x, res)


def test_exact_token_ties_pick_lower_index(cuda_device):
    w = wl.scaled(wl.get("token14b"), name="tok_ties", H=2, T=32, F=6, Fc=1, n_score_q=16,
                  sink_tokens=32, recent_tokens=32, keep_tokens=40, seed=33)
    x = wl.generate(w)
    # candidates come in identical pairs (2i, 2i+1): equal phi within each pair
    c0, c1 = w.sink_tokens, w.N - w.recent_tokens
    cand = x["k_hist"][:, :, c0:c1]
    cand[:, :, 1::2] = cand[:, :, 0::2]
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)
    for h in range(w.H):
        phi = res["seg_score"][0, h]
        assert torch.equal(phi[0::2], phi[1::2])
        kept = parity.gpu_kept(res, 0, h)[w.sink_tokens: w.sink_tokens + w.keep_tokens] - c0
        ref = orc.top_k(phi.double().numpy(), w.keep_tokens)
        assert kept.tolist() == ref.tolist()


def test_device_errors_are_recorded_not_faulted(cuda_device):
    w = _small()
    x = wl.generate(w)
    x["k_per_head"][0, 2] = 99  # k > F on a dynamic head
    x["head_role"][0, 2] = 1
    res = parity.run_step(w, x)
    assert res["status"] == (fkv._lib.FKV_ERR_DEVICE_ARG, 2)
    assert int(res["kept_cnt"][0, 2]) == w.F  # clamped
    # capacity below the kept rows: copy clamped, error recorded
    y = wl.generate(w)
    res = parity.run_step(w, y, comp_rows=w.T)
    assert res["status"][0] == fkv._lib.FKV_ERR_DEVICE_ARG


def test_fp32_odd_head_dim(cuda_device):
    w = wl.scaled(wl.get("tiny"), name="tiny_d36", D=36, T=21, seed=34)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)
