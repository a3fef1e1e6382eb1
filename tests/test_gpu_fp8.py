"""The e4m3 compressed cache on the GPU against the oracle.

Codes and scales are integers / fp32 values decided in fp32 on both sides,
so they must match bit for bit.  The fp8 attention is compared with the exact
softmax attention over the oracle's own dequantised cache, within the bound
``fkv_fp8.attention_tolerance`` derives from rounding the probabilities to
e4m3 (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "与现有产品/工作流的接口"
item 3: the compression composes with KV quantization).

Kept lists come from a seeded host generator (``fkv_workloads.random_kept``),
the same for both sides.
"""
import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_fp8 as f8
from oracle import fkv_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def _f32(t):
    return wl.as_float64(t).astype(np.float32)


def _setup(w, kept_seed, n_keep=None, zero_frame=False):
    x = wl.generate(w)
    if zero_frame:  # an all-zero K segment and V segment: scale 1, codes 0
        x["k_hist"][0, min(2, w.H - 1), w.T:2 * w.T] = 0
        x["v_hist"][0, min(2, w.H - 1), w.T:2 * w.T] = 0
    p = fkv.params_for(w, comp_rows=w.F * w.T)  # room for every frame: the lists are random
    d = parity.upload(x)
    o = fkv.allocate(p)
    kept_idx, kept_cnt = wl.random_kept(w, kept_seed, n_keep)
    c = fkv.allocate_fp8(p)
    for k, t in c.items():  # sentinels: rows / scales the calls must not touch stay as they are
        t.fill_(0x5A if t.dtype == torch.uint8 else float("nan"))
    fkv.compact_gather_fp8(p, d["k_hist"], d["v_hist"], kept_idx.cuda(), kept_cnt.cuda(), c, o["ws"])
    fkv.quantize_chunk_fp8(p, d["q_cur"], d["k_cur"], d["v_cur"], c, o["ws"])
    return x, p, d, o, c, kept_idx, kept_cnt


def _small(T, F, Fc, H, seed):
    return wl.scaled(wl.get("480p"), name=f"fp8_{T}_{F}_{Fc}_{H}", H=H, D=128, T=T, F=F, Fc=Fc,
                     n_static=1, static_frames=(0,), k_dynamic=1, score_stride=1, dtype="bf16",
                     seed=seed, style="video")


@pytest.mark.parametrize("T,F,Fc,H", [(128, 5, 1, 3), (160, 6, 2, 4), (37, 4, 1, 3), (200, 3, 3, 2)])
def test_codes_and_scales_bit_exact(cuda_device, T, F, Fc, H):
    w = _small(T, F, Fc, H, seed=T + F)
    x, p, d, o, c, kept_idx, kept_cnt = _setup(w, kept_seed=T, zero_frame=True)
    assert fkv.read_status(o["ws"])[0] == 0
    g = {k: t.cpu().numpy() for k, t in c.items()}
    for l in range(w.L):
        for h in range(w.H):
            n = int(kept_cnt[l, h])
            kept = kept_idx[l, h, :n].numpy()
            kc, sk, vc, sv = f8.compact_quantized(_f32(x["k_hist"][l, h]), _f32(x["v_hist"][l, h]),
                                                  kept, T)
            rows = n * T
            assert np.array_equal(g["k_comp"][l, h, :rows], kc), (l, h)
            assert np.array_equal(g["v_comp"][l, h, :rows], vc), (l, h)
            assert np.array_equal(g["k_comp_scale"][l, h, :n].view(np.uint32), sk.view(np.uint32))
            assert np.array_equal(g["v_comp_scale"][l, h, :n].view(np.uint32), sv.view(np.uint32))
            # nothing past the kept rows / scales is written
            assert np.all(g["k_comp"][l, h, rows:] == 0x5A) and np.all(g["v_comp"][l, h, rows:] == 0x5A)
            assert np.all(np.isnan(g["k_comp_scale"][l, h, n:]))
            kq, skq = f8.quantize_segments(_f32(x["k_cur"][l, h]), T)
            vq, svq = f8.quantize_segments(_f32(x["v_cur"][l, h]), T)
            qq, sqq = f8.quantize_rows(_f32(x["q_cur"][l, h]))
            assert np.array_equal(g["k_cur"][l, h], kq) and np.array_equal(g["v_cur"][l, h], vq)
            assert np.array_equal(g["k_cur_scale"][l, h].view(np.uint32), skq.view(np.uint32))
            assert np.array_equal(g["v_cur_scale"][l, h].view(np.uint32), svq.view(np.uint32))
            assert np.array_equal(g["q_cur"][l, h], qq)
            assert np.array_equal(g["q_scale"][l, h].view(np.uint32), sqq.view(np.uint32))
    # the zeroed segment, where kept, has scale 1 and all-zero codes
    hz = min(2, w.H - 1)
    kept = list(kept_idx[0, hz, :int(kept_cnt[0, hz])].numpy())
    if 1 in kept:
        pz = kept.index(1)
        assert g["k_comp_scale"][0, hz, pz] == 1.0 and not g["k_comp"][0, hz, pz * T:(pz + 1) * T].any()


def _oracle_fp8_attention(x, w, l, h, kept, rows=None):
    """Exact attention over the oracle's dequantised fp8 cache, and its tolerance."""
    T = w.T
    kc, sk, vc, sv = f8.compact_quantized(_f32(x["k_hist"][l, h]), _f32(x["v_hist"][l, h]), kept, T)
    kq, skq = f8.quantize_segments(_f32(x["k_cur"][l, h]), T)
    vq, svq = f8.quantize_segments(_f32(x["v_cur"][l, h]), T)
    qq, sqq = f8.quantize_rows(_f32(x["q_cur"][l, h]))
    if rows is not None:
        qq, sqq = qq[rows], sqq[rows]
    q = f8.e4m3_decode(qq) * sqq.astype(np.float64)[:, None]
    keys = np.concatenate([f8.dequantize(kc, sk, T), f8.dequantize(kq, skq, T)])
    vals = np.concatenate([f8.dequantize(vc, sv, T), f8.dequantize(vq, svq, T)])
    v_codes = np.concatenate([vc, vq])
    sv_key = np.concatenate([np.repeat(sv.astype(np.float64), T), np.repeat(svq.astype(np.float64), T)])
    scale = 1.0 / np.sqrt(w.D)
    ref = orc.attention(q, keys, vals, scale)
    tol = f8.attention_tolerance(q, keys, v_codes, sv_key, scale, ref)
    return ref, tol


@pytest.mark.parametrize("T,F,Fc,H,seed", [(128, 5, 1, 3, 1), (160, 6, 2, 3, 2), (200, 4, 1, 2, 3),
                                           (136, 3, 3, 2, 4), (1560, 2, 1, 2, 5)])
def test_attend_fp8_within_rounding_model(cuda_device, T, F, Fc, H, seed):
    w = _small(T, F, Fc, H, seed=seed)
    x, p, d, o, c, kept_idx, kept_cnt = _setup(w, kept_seed=seed + 10)
    out = torch.full_like(o["out"], float("nan"))
    fkv.attend_compressed_fp8(p, c, kept_cnt.cuda(), out, o["ws"])
    assert fkv.read_status(o["ws"])[0] == 0
    got = out.cpu().double().numpy()
    for l in range(w.L):
        for h in range(w.H):
            kept = kept_idx[l, h, :int(kept_cnt[l, h])].numpy()
            ref, tol = _oracle_fp8_attention(x, w, l, h, kept)
            err = np.abs(got[l, h] - ref)
            assert np.all(err <= tol), (l, h, float(err.max()), float((err / tol).max()))
            assert err.mean() <= 2.0 ** -6 * np.abs(ref).mean()


def test_attend_fp8_480p_sampled_rows(cuda_device):
    w = wl.get("480p")
    x, p, d, o, c, kept_idx, kept_cnt = _setup(w, kept_seed=480, n_keep=13)
    out = torch.empty_like(o["out"])
    fkv.attend_compressed_fp8(p, c, kept_cnt.cuda(), out, o["ws"])
    assert fkv.read_status(o["ws"])[0] == 0
    # the bf16 path on the same kept lists, for the size of the fp8 departure
    fkv.compact_gather(p, d["k_hist"], d["v_hist"], kept_idx.cuda(), kept_cnt.cuda(), o["k_comp"],
                       o["v_comp"], o["ws"])
    out16 = torch.empty_like(o["out"])
    fkv.attend_compressed(p, d["q_cur"], d["k_cur"], d["v_cur"], o["k_comp"], o["v_comp"],
                          kept_cnt.cuda(), out16, o["ws"])
    rows = wl.sample_rows(w.Fc * w.T, 48, seed=7)
    for l, h in [(0, 0), (0, 1), (0, 5), (0, 11)]:
        kept = kept_idx[l, h, :int(kept_cnt[l, h])].numpy()
        ref, tol = _oracle_fp8_attention(x, w, l, h, kept, rows)
        got = out[l, h, rows].cpu().double().numpy()
        assert np.all(np.abs(got - ref) <= tol), (l, h)
        # fp8 against bf16 operands: the quantisation error, well below the signal
        g16 = out16[l, h, rows].cpu().double().numpy()
        assert np.abs(got - g16).mean() <= 0.05 * np.abs(g16).mean()


def test_step_fp8_equals_the_separate_calls(cuda_device):
    w = wl.scaled(wl.get("480p"), name="step_fp8", H=4, T=256, F=6, Fc=2, n_static=2,
                  static_frames=(0, 2, 5), k_dynamic=3, score_stride=4, seed=31)
    x = parity.upload(wl.generate(w))
    p = fkv.params_for(w)
    o = fkv.allocate(p)
    c = fkv.allocate_fp8(p)
    fkv.step_fp8(p, x, o, c)
    assert fkv.read_status(o["ws"])[0] == 0
    # the same steps one call at a time
    r = fkv.allocate(p)
    c2 = fkv.allocate_fp8(p)
    fkv.score_segments(p, x["q_cur"], None, x["k_hist"], x["head_role"], r["seg_score"], r["ws"])
    fkv.select_topk(p, r["seg_score"], x["head_role"], x["static_mask"], x["k_per_head"],
                    r["kept_idx"], r["kept_cnt"], r["ws"])
    fkv.compact_gather_fp8(p, x["k_hist"], x["v_hist"], r["kept_idx"], r["kept_cnt"], c2, r["ws"])
    fkv.quantize_chunk_fp8(p, x["q_cur"], x["k_cur"], x["v_cur"], c2, r["ws"])
    out2 = torch.empty_like(r["out"])
    fkv.attend_compressed_fp8(p, c2, r["kept_cnt"], out2, r["ws"])
    assert fkv.read_status(r["ws"])[0] == 0
    assert torch.equal(o["kept_cnt"], r["kept_cnt"]) and torch.equal(o["seg_score"], r["seg_score"])
    assert torch.equal(o["out"], out2)
    for k in ("k_cur", "v_cur", "q_cur", "q_scale", "k_cur_scale", "v_cur_scale"):
        assert torch.equal(c[k], c2[k]), k
    cnt = o["kept_cnt"].cpu()
    for h in range(w.H):
        rows, n = int(cnt[0, h]) * w.T, int(cnt[0, h])
        for k in ("k_comp", "v_comp"):
            assert torch.equal(c[k][0, h, :rows], c2[k][0, h, :rows]), (k, h)
        for k in ("k_comp_scale", "v_comp_scale"):
            assert torch.equal(c[k][0, h, :n], c2[k][0, h, :n]), (k, h)


def test_attend_fp8_1080p_sampled_rows(cuda_device):
    w = wl.get("1080p")
    x, p, d, o, c, kept_idx, kept_cnt = _setup(w, kept_seed=1080, n_keep=13)
    out = torch.empty_like(o["out"])
    fkv.attend_compressed_fp8(p, c, kept_cnt.cuda(), out, o["ws"])
    assert fkv.read_status(o["ws"])[0] == 0
    rows = wl.sample_rows(w.Fc * w.T, 24, seed=8)
    for l, h in [(0, 2), (0, 9)]:
        kept = kept_idx[l, h, :int(kept_cnt[l, h])].numpy()
        ref, tol = _oracle_fp8_attention(x, w, l, h, kept, rows)
        got = out[l, h, rows].cpu().double().numpy()
        assert np.all(np.abs(got - ref) <= tol), (l, h)


# Bar of the e4m3 path against the UNQUANTISED fp64 oracle, per head, fixed from
# the format before any GPU comparison: e4m3 keeps 3 mantissa bits, so every
# rounding of Q, K, V and P moves an element by at most u = 2^-4 of itself; the
# output may sit on average half a unit roundoff, and at its worst element one
# unit roundoff, away from the exact attention, relative to the output's own
# scale (mean |O| and max |O| of the head).
FP8_MEAN_REL, FP8_MAX_REL = 2.0 ** -5, 2.0 ** -4


def test_step_fp8_480p_against_the_unquantised_oracle(cuda_device):
    """The whole e4m3 step at 480P, every query row of every head, against the
    exact fp64 attention over the unquantised kept cache (the kept lists are the
    GPU's, which the bf16 parity tests check against the oracle's selection)."""
    w = wl.get("480p")
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    c = fkv.allocate_fp8(p)
    fkv.step_fp8(p, d, o, c)
    assert fkv.read_status(o["ws"])[0] == 0
    got_all = o["out"].cpu()
    worst = (0.0, 0.0)
    for h in range(w.H):
        kept = parity.gpu_kept({"kept_cnt": o["kept_cnt"].cpu(), "kept_idx": o["kept_idx"].cpu()}, 0, h)
        f64 = lambda k: wl.as_float64(x[k][0, h])  # noqa: E731
        keys = np.concatenate([orc.compact(f64("k_hist"), kept, w.T), f64("k_cur")])
        vals = np.concatenate([orc.compact(f64("v_hist"), kept, w.T), f64("v_cur")])
        ref = orc.attention(f64("q_cur"), keys, vals, w.scale)
        err = np.abs(got_all[0, h].double().numpy() - ref)
        mean_rel = err.mean() / np.abs(ref).mean()
        max_rel = err.max() / np.abs(ref).max()
        worst = (max(worst[0], mean_rel), max(worst[1], max_rel))
        assert mean_rel <= FP8_MEAN_REL and max_rel <= FP8_MAX_REL, (h, mean_rel, max_rel)
    print("e4m3 vs unquantised oracle (mean/mean|O|, max/max|O|):", worst)
