"""fkv_step_launches is what the bench reports as its kernel launches per
step: check it against the kernels one fkv_step call actually launches, as
recorded by the CUDA profiler (CUPTI, through torch.profiler), for the
tensor-core frame path, the token path and the fp32 path."""
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from tests import parity

pytestmark = pytest.mark.gpu


def _cases():
    return [
        wl.scaled(wl.get("480p"), name="lc_frame", H=4, T=256, F=6, Fc=2, n_static=2,
                  static_frames=(0, 2, 5), k_dynamic=3, score_stride=4, seed=61),
        wl.scaled(wl.get("token14b"), name="lc_token", H=4, T=96, F=9, Fc=2, n_score_q=96,
                  sink_tokens=192, recent_tokens=192, keep_tokens=300, seed=62),
        wl.get("tiny"),
    ]


@pytest.mark.parametrize("w", _cases(), ids=lambda w: w.name)
def test_step_launch_count_matches_the_profiler(cuda_device, w):
    x = parity.upload(wl.generate(w))
    p = fkv.params_for(w)
    o = fkv.allocate(p)
    io = fkv.make_step_io(p, x, o)
    fkv.step(p, x, o, io=io)  # warm-up (first-call set-up stays outside the profile)
    torch.cuda.synchronize()
    acts = [torch.profiler.ProfilerActivity.CUDA]
    with torch.profiler.profile(activities=acts) as prof:
        fkv.step(p, x, o, io=io)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events()
             if e.device_type == torch.autograd.DeviceType.CUDA and
             ("fkv::" in e.name or "sm100::" in e.name)]
    print(w.name, len(names), sorted(set(n.split("(")[0] for n in names)))
    assert len(names) == fkv.step_launches(p), names
    assert fkv.read_status(o["ws"])[0] == 0
