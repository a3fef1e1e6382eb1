"""Compaction with temporal RoPE re-positioning of the kept keys, against the
oracle (fp64 rotation of the same inputs, rounded once by the GPU).  The kept
lists come from a seeded host generator, the same for both sides."""
import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,n_pairs", [("bf16", 22), ("bf16", 64), ("fp32", 9), ("bf16", 0)])
def test_compact_gather_rope(cuda_device, dtype, n_pairs):
    D = 128 if dtype == "bf16" else 36
    w = wl.scaled(wl.get("480p"), name=f"rope_{dtype}", H=4, D=D, T=96, F=7, Fc=1, n_static=2,
                  static_frames=(0, 3, 6), k_dynamic=3, score_stride=2, dtype=dtype, seed=61,
                  style="video")
    x = wl.generate(w)
    p = fkv.params_for(w, comp_rows=w.F * w.T)  # room for every frame: the lists are random
    d = parity.upload(x)
    o = fkv.allocate(p)
    # seeded kept lists from the host, the same for both sides
    o["kept_idx"], o["kept_cnt"] = (t.cuda() for t in wl.random_kept(w, seed=62))
    omega = torch.tensor(10000.0 ** (-np.arange(n_pairs) / max(n_pairs, 1)), dtype=torch.float32)
    kc = torch.full_like(o["k_comp"], float("nan"))
    vc = torch.full_like(o["v_comp"], float("nan"))
    fkv.compact_gather_rope(p, d["k_hist"], d["v_hist"], o["kept_idx"], o["kept_cnt"],
                            omega.cuda() if n_pairs else None, kc, vc, o["ws"])
    assert fkv.read_status(o["ws"])[0] == 0
    kept_cnt, kept_idx = o["kept_cnt"].cpu(), o["kept_idx"].cpu()
    # rounding of the fp32 rotation to the activation dtype: half an ulp, plus
    # the fp32 rotation error
    rel = 2.0 ** -8 if dtype == "bf16" else 1e-6
    for l in range(w.L):
        for h in range(w.H):
            kept = parity.gpu_kept({"kept_cnt": kept_cnt, "kept_idx": kept_idx}, l, h)
            rows = len(kept) * w.T
            exp_k = orc.compact_repositioned(wl.as_float64(x["k_hist"][l, h]), kept, w.T, w.F,
                                             omega.double().numpy())
            got_k = kc[l, h, :rows].cpu().double().numpy()
            assert np.all(np.abs(got_k - exp_k) <= rel * np.abs(exp_k) + 1e-6), (l, h)
            # the dims past the band and the values are exact copies
            plain = orc.compact(wl.as_float64(x["k_hist"][l, h]), kept, w.T)
            assert np.array_equal(got_k[:, 2 * n_pairs:], plain[:, 2 * n_pairs:])
            assert np.array_equal(vc[l, h, :rows].cpu().double().numpy(),
                                  orc.compact(wl.as_float64(x["v_hist"][l, h]), kept, w.T))
            if n_pairs == 0:
                assert np.array_equal(got_k, plain)


def test_compact_gather_rope_480p(cuda_device):
    w = wl.get("480p")
    x = wl.generate(w)
    p = fkv.params_for(w, comp_rows=w.F * w.T)
    d = parity.upload(x)
    o = fkv.allocate(p)
    kept_idx, kept_cnt = wl.random_kept(w, seed=480, n_keep=13)
    omega = torch.tensor(10000.0 ** (-np.arange(22) / 22), dtype=torch.float32)
    kc = torch.full_like(o["k_comp"], float("nan"))
    vc = torch.full_like(o["v_comp"], float("nan"))
    fkv.compact_gather_rope(p, d["k_hist"], d["v_hist"], kept_idx.cuda(), kept_cnt.cuda(),
                            omega.cuda(), kc, vc, o["ws"])
    assert fkv.read_status(o["ws"])[0] == 0
    for h in (0, 1, 5, 11):  # head 0 keeps nothing, head 1 every frame, the others 13
        kept = kept_idx[0, h, :int(kept_cnt[0, h])].numpy()
        rows = len(kept) * w.T
        exp_k = orc.compact_repositioned(wl.as_float64(x["k_hist"][0, h]), kept, w.T, w.F,
                                         omega.double().numpy())
        got_k = kc[0, h, :rows].cpu().double().numpy()
        assert np.all(np.abs(got_k - exp_k) <= 2.0 ** -8 * np.abs(exp_k) + 1e-6), h
        assert np.array_equal(vc[0, h, :rows].cpu().double().numpy(),
                              orc.compact(wl.as_float64(x["v_hist"][0, h]), kept, w.T))
