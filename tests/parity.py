"""Helpers of the GPU parity tests: run the library and the oracle on the same
seeded inputs and compare them under the stated tolerances.

Tolerances (written here, derived in the design notes):
  * kept indices and compacted K/V: bit-exact;
  * selection sets may differ from the oracle's only where the oracle's k-th
    and (k+1)-th scores are within 1e-5 relative, and only by segments whose
    scores lie inside that window;
  * attention output: bf16 max-abs 2e-2, mean-abs 2e-3; fp32 1e-4 / 1e-5;
  * segment scores (float32 on the GPU): relative 1e-4 of the largest score of
    the head.
"""
from __future__ import annotations

import numpy as np
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_oracle as orc

SEL_REL = 1e-5
SCORE_REL = 1e-4
ATTN_TOL = {"bf16": (2e-2, 2e-3), "fp32": (1e-4, 1e-5)}


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def upload(inputs, device="cuda"):
    return {k: v.to(device) for k, v in inputs.items()}


def run_step(w, inputs_cpu, comp_rows=None, p=None):
    """fkv_step on the GPU; returns CPU copies of every output + device status."""
    p = p or fkv.params_for(w, comp_rows)
    dev = upload(inputs_cpu)
    outs = fkv.allocate(p)
    fkv.step(p, dev, outs)
    status = fkv.read_status(outs["ws"])
    torch.cuda.synchronize()
    res = {k: v.cpu() for k, v in outs.items() if k != "ws"}
    res["status"] = status
    res["params"] = p
    return res


class HeadView:
    """Exact float64 views of one (layer, head) of the generated inputs, made
    on demand so that large workloads are never upcast as a whole."""

    def __init__(self, inputs_cpu):
        self.t = inputs_cpu

    def __call__(self, key, l, h):
        v = self.t[key][l, h]
        return wl.as_float64(v) if v.is_floating_point() else v.numpy()


def gpu_kept(res, l, h):
    c = int(res["kept_cnt"][l, h])
    return res["kept_idx"][l, h, :c].numpy().astype(np.int64)


def check_selection(orc_kept, orc_score, g_kept, k, where):
    """Equal sets, or a difference confined to a near-tie at the k-th score."""
    if len(g_kept) == len(orc_kept) and np.array_equal(g_kept, orc_kept):
        return True
    assert orc_score is not None, f"{where}: static selection differs: {g_kept} vs {orc_kept}"
    assert len(g_kept) == len(orc_kept) == k, f"{where}: count {len(g_kept)} vs {len(orc_kept)}"
    srt = np.sort(orc_score)[::-1]
    sk, sk1 = srt[k - 1], srt[k]
    win = SEL_REL * abs(sk)
    assert abs(sk - sk1) <= win, f"{where}: selection differs outside a near-tie ({sk} vs {sk1})"
    diff = np.setxor1d(g_kept, orc_kept)
    cand = orc_score[diff]
    assert np.all(np.abs(cand - sk) <= win), f"{where}: differing segments not at the threshold"
    return False


def compare_attention(got, exp, dtype, where):
    amax, amean = ATTN_TOL[dtype]
    err = np.abs(got - exp)
    assert err.max() <= amax and err.mean() <= amean, (
        f"{where}: attention max-abs {err.max():.3g} (tol {amax}), mean-abs {err.mean():.3g} (tol {amean})")
    return float(err.max()), float(err.mean())


def check_step(w, inputs_cpu, res, heads=None, rows=None, check_comp=True):
    """Compares one fkv_step result with the oracle on the given (l, h) and
    query rows (None = all).  Returns summary statistics."""
    x = HeadView(inputs_cpu)
    L, H = w.L, w.H
    todo = heads if heads is not None else [(l, h) for l in range(L) for h in range(H)]
    token_mask = getattr(w, "static_token_mask", False)
    seg_len = w.T if (w.granularity == "frame" and not token_mask) else 1
    assert res["status"][0] == 0, f"device status {res['status']}"
    stats = {"attn_max": 0.0, "attn_mean": 0.0, "score_rel": 0.0, "sel_exact": 0, "sel_tie": 0}
    for (l, h) in todo:
        where = f"{w.name} l={l} h={h}"
        dynamic = w.granularity == "token" or bool(x("head_role", l, h))
        k_hist, v_hist = x("k_hist", l, h), x("v_hist", l, h)
        q_cur = x("q_cur", l, h)
        k_sel = int(x("k_per_head", l, h))
        kept_o, score_o = orc.head_keep(
            granularity=w.granularity, dynamic=dynamic, mask_row=x("static_mask", l, h),
            k=k_sel, q_cur=q_cur, k_hist=k_hist,
            T=w.T, scale=w.scale, score_stride=w.score_stride,
            q_score=None if "q_score" not in inputs_cpu else x("q_score", l, h),
            sink=w.sink_tokens, recent=w.recent_tokens,
            k_chunk=x("k_cur", l, h) if getattr(w, "score_with_chunk", False) else None,
            token_static_mask=token_mask)
        kept_g = gpu_kept(res, l, h)
        if score_o is not None and len(score_o) > 0:
            sg = res["seg_score"][l, h].numpy().astype(np.float64)
            rel = np.max(np.abs(sg - score_o)) / np.max(np.abs(score_o))
            assert rel <= SCORE_REL, f"{where}: segment scores rel err {rel:.3g}"
            stats["score_rel"] = max(stats["score_rel"], float(rel))
        if w.granularity == "token":
            exact = check_selection(kept_o[w.sink_tokens:len(kept_o) - w.recent_tokens] - w.sink_tokens,
                                    score_o, kept_g[w.sink_tokens:len(kept_g) - w.recent_tokens] - w.sink_tokens,
                                    k_sel, where)
            assert np.array_equal(kept_g[:w.sink_tokens], np.arange(w.sink_tokens))
            assert np.array_equal(kept_g[len(kept_g) - w.recent_tokens:],
                                  np.arange(w.N - w.recent_tokens, w.N))
        elif token_mask and dynamic:
            # token lists of whole frames: compare the frames, then the expansion
            fr_g = np.unique(kept_g // w.T)
            assert np.array_equal(kept_g, orc.frames_to_tokens(fr_g, w.T)), f"{where}: not whole frames"
            exact = check_selection(np.unique(kept_o // w.T), score_o, fr_g, k_sel, where)
        else:
            exact = check_selection(kept_o, score_o, kept_g, k_sel, where)
        stats["sel_exact" if exact else "sel_tie"] += 1
        # compaction: bit-exact copy of the (validated) GPU selection
        n_rows = len(kept_g) * seg_len
        kc = orc.compact(k_hist, kept_g, seg_len)
        vc = orc.compact(v_hist, kept_g, seg_len)
        if check_comp:
            assert np.array_equal(to_f64(res["k_comp"][l, h, :n_rows]), kc), f"{where}: k_comp differs"
            assert np.array_equal(to_f64(res["v_comp"][l, h, :n_rows]), vc), f"{where}: v_comp differs"
        keys = np.concatenate([kc, x("k_cur", l, h)])
        vals = np.concatenate([vc, x("v_cur", l, h)])
        q = q_cur if rows is None else q_cur[rows]
        exp = orc.attention(q, keys, vals, w.scale)
        got = to_f64(res["out"][l, h]) if rows is None else to_f64(res["out"][l, h][torch.as_tensor(rows)])
        mx, mn = compare_attention(got, exp, w.dtype, where)
        stats["attn_max"] = max(stats["attn_max"], mx)
        stats["attn_mean"] = max(stats["attn_mean"], mn)
    return stats
