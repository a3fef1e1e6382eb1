"""Cache lifecycle across chunks and denoising steps, against the oracle.

* fkv_cache_advance: the next history = the most recent kept segments of the
  compressed cache, then the chunk's own K/V (bit-exact copy);
* a second chunk step on that advanced history matches the oracle running the
  same two-chunk sequence;
* later denoising steps of a chunk reuse its selection and compressed cache
  through fkv_attend_compressed alone (new chunk Q/K/V each step).
"""
import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def _frame_w(**kw):
    base = wl.scaled(wl.get("480p"), name="life", H=4, T=160, F=6, Fc=2, n_static=2,
                     static_frames=(0, 2, 4, 5), k_dynamic=4, score_stride=3, seed=51)
    return wl.scaled(base, **kw)


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


@pytest.mark.parametrize("mode", ["frame", "token"])
def test_cache_advance_bit_exact(cuda_device, mode):
    if mode == "frame":
        w = _frame_w()
        out_segments = 4 + w.Fc            # all 4 kept frames + the chunk
        seg_len = w.T
    else:
        w = wl.scaled(wl.get("token14b"), name="life_tok", H=3, T=64, F=8, Fc=2, n_score_q=64,
                      sink_tokens=64, recent_tokens=64, keep_tokens=150, seed=52)
        out_segments = 200 + w.Lq          # the 200 most recent of 278 kept tokens + chunk
        seg_len = 1
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    fkv.step(p, d, o)
    rows = out_segments * seg_len
    k_next = torch.empty((w.L, w.H, rows, w.D), dtype=torch.bfloat16, device="cuda")
    v_next = torch.empty_like(k_next)
    fkv.cache_advance(p, o["k_comp"], o["v_comp"], o["kept_cnt"], d["k_cur"], d["v_cur"],
                      out_segments, k_next, v_next, o["ws"])
    assert fkv.read_status(o["ws"])[0] == 0
    kept_cnt = o["kept_cnt"].cpu()
    for l in range(w.L):
        for h in range(w.H):
            kept = parity.gpu_kept({"kept_cnt": kept_cnt, "kept_idx": o["kept_idx"].cpu()}, l, h)
            for name, hist, cur, got in (("k", "k_hist", "k_cur", k_next), ("v", "v_hist", "v_cur", v_next)):
                comp = orc.compact(wl.as_float64(x[hist][l, h]), kept, seg_len)
                exp = orc.advance(comp, len(kept), seg_len, wl.as_float64(x[cur][l, h]), out_segments)
                assert np.array_equal(_f64(got[l, h]), exp), (mode, name, l, h)


def test_advance_with_too_few_kept_segments_records_error(cuda_device):
    w = _frame_w()
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    fkv.step(p, d, o)
    out_segments = 5 + w.Fc                # asks for 5 kept frames, heads have 4
    k_next = torch.full((w.L, w.H, out_segments * w.T, w.D), 7.0, dtype=torch.bfloat16, device="cuda")
    v_next = torch.empty_like(k_next)
    fkv.cache_advance(p, o["k_comp"], o["v_comp"], o["kept_cnt"], d["k_cur"], d["v_cur"],
                      out_segments, k_next, v_next, o["ws"])
    assert fkv.read_status(o["ws"])[0] == fkv._lib.FKV_ERR_DEVICE_ARG
    assert bool((k_next[:, :, : 5 * w.T] == 0).all())


def test_two_chunks_through_the_advanced_cache(cuda_device):
    w = _frame_w()
    x1 = wl.generate(w)
    # the second chunk's queries and own K/V come from an independent draw
    x2_new = wl.generate(wl.scaled(w, seed=w.seed + 100))
    p = fkv.params_for(w)
    d1 = parity.upload(x1)
    o1 = fkv.allocate(p)
    fkv.step(p, d1, o1)
    window = 4 + w.Fc                      # keeps the history at F = 6 frames
    k_next = torch.empty((w.L, w.H, window * w.T, w.D), dtype=torch.bfloat16, device="cuda")
    v_next = torch.empty_like(k_next)
    fkv.cache_advance(p, o1["k_comp"], o1["v_comp"], o1["kept_cnt"], d1["k_cur"], d1["v_cur"],
                      window, k_next, v_next, o1["ws"])
    x2 = dict(x1)
    for k in ("q_cur", "k_cur", "v_cur"):
        x2[k] = x2_new[k]
    x2["k_hist"], x2["v_hist"] = k_next.cpu(), v_next.cpu()
    w2 = wl.scaled(w, F=window)
    res2 = parity.run_step(w2, x2)
    # oracle: the same sequence computed from the first chunk's inputs alone
    for l in range(w.L):
        for h in range(w.H):
            kept1, _ = orc.head_keep(
                granularity="frame", dynamic=bool(x1["head_role"][l, h]),
                mask_row=x1["static_mask"][l, h].numpy(), k=int(x1["k_per_head"][l, h]),
                q_cur=wl.as_float64(x1["q_cur"][l, h]), k_hist=wl.as_float64(x1["k_hist"][l, h]),
                T=w.T, scale=w.scale, score_stride=w.score_stride)
            kh = orc.advance(orc.compact(wl.as_float64(x1["k_hist"][l, h]), kept1, w.T), len(kept1),
                             w.T, wl.as_float64(x1["k_cur"][l, h]), window)
            vh = orc.advance(orc.compact(wl.as_float64(x1["v_hist"][l, h]), kept1, w.T), len(kept1),
                             w.T, wl.as_float64(x1["v_cur"][l, h]), window)
            assert np.array_equal(_f64(k_next[l, h]), kh) and np.array_equal(_f64(v_next[l, h]), vh)
    parity.check_step(w2, x2, res2)


def test_denoising_steps_reuse_the_selection(cuda_device):
    w = _frame_w()
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    fkv.step(p, d, o)                       # first denoising step: select + compact + attend
    kept_cnt = o["kept_cnt"].cpu()
    kept_idx = o["kept_idx"].cpu()
    for s in range(1, 4):                   # later steps: the chunk's Q/K/V change
        y = wl.generate(wl.scaled(w, seed=w.seed + 1000 + s))
        dy = {k: y[k].cuda() for k in ("q_cur", "k_cur", "v_cur")}
        out = torch.empty_like(o["out"])
        fkv.attend_compressed(p, dy["q_cur"], dy["k_cur"], dy["v_cur"], o["k_comp"], o["v_comp"],
                              o["kept_cnt"], out, o["ws"])
        for l in range(w.L):
            for h in range(w.H):
                kept = parity.gpu_kept({"kept_cnt": kept_cnt, "kept_idx": kept_idx}, l, h)
                keys = np.concatenate([orc.compact(wl.as_float64(x["k_hist"][l, h]), kept, w.T),
                                       wl.as_float64(y["k_cur"][l, h])])
                vals = np.concatenate([orc.compact(wl.as_float64(x["v_hist"][l, h]), kept, w.T),
                                       wl.as_float64(y["v_cur"][l, h])])
                exp = orc.attention(wl.as_float64(y["q_cur"][l, h]), keys, vals, w.scale)
                parity.compare_attention(_f64(out[l, h]), exp, "bf16", f"step {s} l={l} h={h}")
    assert fkv.read_status(o["ws"])[0] == 0
