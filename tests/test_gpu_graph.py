"""fkv_step captured in a CUDA graph: the call does no host synchronisation and
no allocation, so a serving loop can capture it once and replay it.  Replays
on new inputs copied into the captured buffers must give exactly the outputs
of eager calls on the same inputs (the same kernels, the same launch
configurations)."""
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["480p", "token14b"])
def test_step_graph_replay_matches_eager(cuda_device, name):
    base = wl.get(name)
    w = wl.scaled(base, name=f"graph_{name}", H=4, F=6, T=256, Fc=1) if name == "480p" else \
        wl.scaled(base, name=f"graph_{name}", H=4, T=96, F=10, sink_tokens=192, recent_tokens=96,
                  keep_tokens=300, n_score_q=96)
    if name == "480p":
        w = wl.scaled(w, static_frames=(0, 2, 5), k_dynamic=3, n_static=2)
    p = fkv.params_for(w)
    xs = [parity.upload(wl.generate(wl.scaled(w, seed=w.seed + i))) for i in range(3)]
    x = {k: v.clone() for k, v in xs[0].items()}   # the captured input buffers
    o = fkv.allocate(p)
    io = fkv.make_step_io(p, x, o)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                         # warm-up outside the capture
        fkv.step(p, x, o, io=io, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fkv.step(p, x, o, io=io, stream=torch.cuda.current_stream())
    for xi in xs:
        for k, v in xi.items():
            x[k].copy_(v)
        g.replay()
        torch.cuda.synchronize()
        got = {k: o[k].clone() for k in ("out", "kept_idx", "kept_cnt", "seg_score")}
        ref = fkv.allocate(p)
        fkv.step(p, xi, ref)
        torch.cuda.synchronize()
        assert fkv.read_status(o["ws"])[0] == 0 and fkv.read_status(ref["ws"])[0] == 0
        for k in ("out", "kept_cnt", "seg_score"):
            assert torch.equal(got[k], ref[k]), k
        # kept lists: entries past the count are left untouched by design
        cnt = ref["kept_cnt"].cpu()
        gi, ri = got["kept_idx"].cpu(), ref["kept_idx"].cpu()
        for l in range(w.L):
            for h in range(w.H):
                c = int(cnt[l, h])
                assert torch.equal(gi[l, h, :c], ri[l, h, :c]), (l, h)


def test_marshalled_calls_repeat_the_wrapper_calls(cuda_device):
    """fkv.marshal: one wrapper call checked and converted once, repeated as a
    bare C-ABI call, gives the same results as the wrapper."""
    w = wl.scaled(wl.get("480p"), name="marshal", H=4, T=256, F=6, Fc=2, n_static=2,
                  static_frames=(0, 2, 5), k_dynamic=3, score_stride=4, seed=33)
    x = parity.upload(wl.generate(w))
    p = fkv.params_for(w)
    ref, o = fkv.allocate(p), fkv.allocate(p)
    fkv.step(p, x, ref)
    calls = [
        fkv.marshal(fkv.score_segments, p, x["q_cur"], None, x["k_hist"], x["head_role"],
                    o["seg_score"], o["ws"]),
        fkv.marshal(fkv.select_topk, p, o["seg_score"], x["head_role"], x["static_mask"],
                    x["k_per_head"], o["kept_idx"], o["kept_cnt"], o["ws"]),
        fkv.marshal(fkv.compact_gather, p, x["k_hist"], x["v_hist"], o["kept_idx"],
                    o["kept_cnt"], o["k_comp"], o["v_comp"], o["ws"]),
        fkv.marshal(fkv.attend_compressed, p, x["q_cur"], x["k_cur"], x["v_cur"], o["k_comp"],
                    o["v_comp"], o["kept_cnt"], o["out"], o["ws"]),
    ]
    for _ in range(2):
        for fn, args in calls:
            assert fn(*args) == 0
    assert fkv.read_status(o["ws"])[0] == 0
    for k in ("seg_score", "kept_cnt", "out"):
        assert torch.equal(o[k], ref[k]), k
