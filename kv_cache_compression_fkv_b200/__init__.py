"""Forcing-KV hybrid head-wise KV-cache compression for NVIDIA B200.

Python binding of the C library ``libfkv.so`` (include/fkv.h).  The functions
below only check and marshal arguments -- device pointers of contiguous torch
CUDA tensors and the current CUDA stream -- and call the library; every step
of the chunk step runs in the library's CUDA kernels.  torch provides device
memory and streams.  There is no CPU fallback: without the built library the
import of ``_lib`` functions raises.

Steps (one call of :func:`step`, per layer and head):
  static heads keep their profiled frames; dynamic heads score the history
  frames by the softmax mass of the chunk's scoring queries and keep the top
  k; the kept K/V are compacted; the chunk attends to the compressed cache
  plus its own K/V (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "关键模块"
  2-3, "输出与工程收益").  ``granularity="token"`` is Deep Forcing's
  participative compression (bxzpzcl.cn/news/2125000, section 3.1).
"""
from __future__ import annotations

import ctypes
import math
from typing import Dict, Optional

import torch

from . import _lib
from ._lib import Params, StepIO

__all__ = [
    "FkvError", "Params", "make_params", "params_for", "sizes", "allocate", "score_segments",
    "select_topk", "compact_gather", "attend_compressed", "step", "read_status", "library",
    "step_launches", "make_step_io", "score_segments_noalloc", "cache_advance",
    "compact_gather_rope", "marshal",
]


class FkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = _lib.load().fkv_status_string(int(status)).decode()
        super().__init__(f"{where}: {msg}")


def library():
    return _lib.load()


def _check(status: int, where: str):
    if status != _lib.FKV_OK:
        raise FkvError(status, where)


def make_params(*, L: int, H: int, D: int, T: int, F: int, Fc: int, dtype: str = "bf16",
                granularity: str = "frame", score_stride: int = 1, n_score_q: int = 0,
                sink_tokens: int = 0, recent_tokens: int = 0, comp_rows: Optional[int] = None,
                scale: Optional[float] = None, score_with_chunk: bool = False,
                static_token_mask: bool = False) -> Params:
    """fkv_params_t from keyword sizes.  comp_rows defaults to the worst case
    (every history row kept).  score_with_chunk / static_token_mask set
    FKV_FLAG_SCORE_WITH_CHUNK / FKV_FLAG_STATIC_TOKEN_MASK."""
    p = Params()
    p.num_layers, p.num_heads, p.head_dim = L, H, D
    p.frame_tokens, p.hist_frames, p.chunk_frames = T, F, Fc
    p.score_stride, p.n_score_q = score_stride, n_score_q
    p.sink_tokens, p.recent_tokens = sink_tokens, recent_tokens
    p.comp_rows = F * T if comp_rows is None else comp_rows
    p.scale = 1.0 / math.sqrt(D) if scale is None else scale
    p.dtype = {"bf16": _lib.FKV_DTYPE_BF16, "fp32": _lib.FKV_DTYPE_FP32}[dtype]
    p.granularity = {"frame": _lib.FKV_GRAN_FRAME, "token": _lib.FKV_GRAN_TOKEN}[granularity]
    p.flags = ((_lib.FKV_FLAG_SCORE_WITH_CHUNK if score_with_chunk else 0) |
               (_lib.FKV_FLAG_STATIC_TOKEN_MASK if static_token_mask else 0))
    return p


def params_for(w, comp_rows: Optional[int] = None) -> Params:
    """Params of a workload description (an object with the fields of
    ``fkv_workloads.Workload``).  comp_rows defaults to the rows the budgets
    keep: max(static mask size, k) * T in frame mode, S + C + R in token mode."""
    token_mask = getattr(w, "static_token_mask", False)
    if comp_rows is None:
        if w.granularity == "frame" and token_mask:
            edge = max(1, w.T // 8)
            static_rows = (w.T + (w.F - 1) * 2 * edge) if w.F > 0 else 0
            comp_rows = max(static_rows, w.k_dynamic * w.T)
        elif w.granularity == "frame":
            comp_rows = max(len(w.static_frames), w.k_dynamic) * w.T
        else:
            comp_rows = w.sink_tokens + w.keep_tokens + w.recent_tokens
    return make_params(L=w.L, H=w.H, D=w.D, T=w.T, F=w.F, Fc=w.Fc, dtype=w.dtype,
                       granularity=w.granularity, score_stride=w.score_stride,
                       n_score_q=w.n_score_q, sink_tokens=w.sink_tokens,
                       recent_tokens=w.recent_tokens, comp_rows=comp_rows, scale=w.scale,
                       score_with_chunk=getattr(w, "score_with_chunk", False),
                       static_token_mask=token_mask)


def sizes(p: Params) -> Dict[str, int]:
    """Derived sizes: nseg, max_kept, max_comp_rows, ws_bytes (and the
    activation dtype)."""
    lib = _lib.load()
    _check(lib.fkv_check_params(ctypes.byref(p)), "fkv_check_params")
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    ws = ctypes.c_size_t()
    _check(lib.fkv_num_segments(ctypes.byref(p), ctypes.byref(a)), "fkv_num_segments")
    _check(lib.fkv_max_kept(ctypes.byref(p), ctypes.byref(b)), "fkv_max_kept")
    _check(lib.fkv_max_comp_rows(ctypes.byref(p), ctypes.byref(c)), "fkv_max_comp_rows")
    _check(lib.fkv_workspace_size(ctypes.byref(p), ctypes.byref(ws)), "fkv_workspace_size")
    return {"nseg": a.value, "max_kept": b.value, "max_comp_rows": c.value, "ws_bytes": ws.value}


def step_launches(p: Params) -> int:
    """Kernel launches one fkv_step call enqueues (the library's own count)."""
    n = ctypes.c_int32()
    _check(_lib.load().fkv_step_launches(ctypes.byref(p), ctypes.byref(n)), "fkv_step_launches")
    return n.value


def _act_dtype(p: Params):
    return torch.bfloat16 if p.dtype == _lib.FKV_DTYPE_BF16 else torch.float32


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, numel: Optional[int] = None,
         optional: bool = False) -> Optional[int]:
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {numel}")
    return t.data_ptr()


def _shapes(p: Params) -> Dict[str, int]:
    s = sizes(p)
    L, H, D = p.num_layers, p.num_heads, p.head_dim
    Lq = p.chunk_frames * p.frame_tokens
    N = p.hist_frames * p.frame_tokens
    return {
        "act_cur": L * H * Lq * D, "act_hist": L * H * N * D, "q_score": L * H * p.n_score_q * D,
        "heads": L * H,
        "mask": L * H * (N if p.flags & _lib.FKV_FLAG_STATIC_TOKEN_MASK else p.hist_frames),
        "seg": L * H * s["nseg"],
        "kept": L * H * s["max_kept"], "comp": L * H * p.comp_rows * D, "ws": s["ws_bytes"],
    }


def allocate(p: Params, device="cuda") -> Dict[str, torch.Tensor]:
    """Output tensors and a zero-initialised workspace for these params."""
    s = sizes(p)
    L, H, D = p.num_layers, p.num_heads, p.head_dim
    Lq = p.chunk_frames * p.frame_tokens
    dt = _act_dtype(p)
    out = {
        "seg_score": torch.empty((L, H, s["nseg"]), dtype=torch.float32, device=device),
        "kept_idx": torch.full((L, H, s["max_kept"]), -1, dtype=torch.int32, device=device),
        "kept_cnt": torch.zeros((L, H), dtype=torch.int32, device=device),
        "k_comp": torch.empty((L, H, p.comp_rows, D), dtype=dt, device=device),
        "v_comp": torch.empty((L, H, p.comp_rows, D), dtype=dt, device=device),
        "out": torch.empty((L, H, Lq, D), dtype=dt, device=device),
        # 256-byte alignment: torch's caching allocator returns 512-B aligned blocks
        "ws": torch.empty((s["ws_bytes"],), dtype=torch.uint8, device=device),
    }
    _check(_lib.load().fkv_workspace_init(out["ws"].data_ptr(), s["ws_bytes"], _stream(None)),
           "fkv_workspace_init")
    return out


def score_segments(p: Params, q_cur, q_score, k_hist, head_role, seg_score, ws, stream=None,
                   k_cur=None):
    """Segment scores; k_cur (the chunk's keys) is needed with score_with_chunk."""
    n, dt = _shapes(p), _act_dtype(p)
    token = p.granularity == _lib.FKV_GRAN_TOKEN
    st = _lib.load().fkv_score_segments(
        ctypes.byref(p), _ptr(q_cur, "q_cur", dt, n["act_cur"], optional=token),
        _ptr(q_score, "q_score", dt, n["q_score"], optional=not token),
        _ptr(k_hist, "k_hist", dt, n["act_hist"]),
        _ptr(k_cur, "k_cur", dt, n["act_cur"], optional=not (p.flags & _lib.FKV_FLAG_SCORE_WITH_CHUNK)),
        _ptr(head_role, "head_role", torch.uint8, n["heads"], optional=token),
        _ptr(seg_score, "seg_score", torch.float32, n["seg"]),
        _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_score_segments")


def score_segments_noalloc(p: Params, q_cur, q_score, k_hist, head_role, seg_score, stream=None,
                           k_cur=None):
    """score_segments without a workspace: for callers that cannot allocate
    device memory.  The library's own static 16 MiB device scratch is used, so
    sizes needing more are rejected, and calls must not overlap on the GPU."""
    n, dt = _shapes(p), _act_dtype(p)
    token = p.granularity == _lib.FKV_GRAN_TOKEN
    st = _lib.load().fkv_score_segments_noalloc(
        ctypes.byref(p), _ptr(q_cur, "q_cur", dt, n["act_cur"], optional=token),
        _ptr(q_score, "q_score", dt, n["q_score"], optional=not token),
        _ptr(k_hist, "k_hist", dt, n["act_hist"]),
        _ptr(k_cur, "k_cur", dt, n["act_cur"], optional=not (p.flags & _lib.FKV_FLAG_SCORE_WITH_CHUNK)),
        _ptr(head_role, "head_role", torch.uint8, n["heads"], optional=token),
        _ptr(seg_score, "seg_score", torch.float32, n["seg"]), _stream(stream))
    _check(st, "fkv_score_segments_noalloc")


def select_topk(p: Params, seg_score, head_role, static_mask, k_per_head, kept_idx, kept_cnt, ws,
                stream=None):
    n = _shapes(p)
    token = p.granularity == _lib.FKV_GRAN_TOKEN
    st = _lib.load().fkv_select_topk(
        ctypes.byref(p), _ptr(seg_score, "seg_score", torch.float32, n["seg"]),
        _ptr(head_role, "head_role", torch.uint8, n["heads"], optional=token),
        _ptr(static_mask, "static_mask", torch.uint8, n["mask"], optional=token),
        _ptr(k_per_head, "k_per_head", torch.int32, n["heads"]),
        _ptr(kept_idx, "kept_idx", torch.int32, n["kept"]),
        _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]), _ptr(ws, "ws", torch.uint8, n["ws"]),
        _stream(stream))
    _check(st, "fkv_select_topk")


def select_heuristic(p: Params, policy: str, seed: int, k_per_head, kept_idx, kept_cnt, ws,
                     seg_score=None, stream=None):
    """Comparison selector of every head (fkv_select_heuristic): policy
    "uniform" (evenly spaced segments) or "random" (largest Philox4x64-10
    priorities; written to seg_score, which is then required)."""
    n = _shapes(p)
    pol = {"uniform": _lib.FKV_POLICY_UNIFORM, "random": _lib.FKV_POLICY_RANDOM}[policy]
    st = _lib.load().fkv_select_heuristic(
        ctypes.byref(p), pol, int(seed) & ((1 << 64) - 1),
        _ptr(k_per_head, "k_per_head", torch.int32, n["heads"]),
        _ptr(seg_score, "seg_score", torch.float32, n["seg"], optional=policy == "uniform"),
        _ptr(kept_idx, "kept_idx", torch.int32, n["kept"]),
        _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]), _ptr(ws, "ws", torch.uint8, n["ws"]),
        _stream(stream))
    _check(st, "fkv_select_heuristic")


def compact_gather(p: Params, k_hist, v_hist, kept_idx, kept_cnt, k_comp, v_comp, ws, stream=None):
    n, dt = _shapes(p), _act_dtype(p)
    st = _lib.load().fkv_compact_gather(
        ctypes.byref(p), _ptr(k_hist, "k_hist", dt, n["act_hist"]),
        _ptr(v_hist, "v_hist", dt, n["act_hist"]), _ptr(kept_idx, "kept_idx", torch.int32, n["kept"]),
        _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]), _ptr(k_comp, "k_comp", dt, n["comp"]),
        _ptr(v_comp, "v_comp", dt, n["comp"]), _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_compact_gather")


def attend_compressed(p: Params, q_cur, k_cur, v_cur, k_comp, v_comp, kept_cnt, out, ws,
                      stream=None):
    n, dt = _shapes(p), _act_dtype(p)
    st = _lib.load().fkv_attend_compressed(
        ctypes.byref(p), _ptr(q_cur, "q_cur", dt, n["act_cur"]), _ptr(k_cur, "k_cur", dt, n["act_cur"]),
        _ptr(v_cur, "v_cur", dt, n["act_cur"]), _ptr(k_comp, "k_comp", dt, n["comp"]),
        _ptr(v_comp, "v_comp", dt, n["comp"]), _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]),
        _ptr(out, "out", dt, n["act_cur"]), _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_attend_compressed")


def compact_gather_rope(p: Params, k_hist, v_hist, kept_idx, kept_cnt, omega, k_comp, v_comp, ws,
                        stream=None):
    """Compaction with temporal RoPE re-positioning of the kept keys
    (fkv_compact_gather_rope); omega: float32 CUDA tensor of the temporal
    RoPE frequencies, one per rotated dim pair."""
    n, dt = _shapes(p), _act_dtype(p)
    n_pairs = 0 if omega is None else int(omega.numel())
    st = _lib.load().fkv_compact_gather_rope(
        ctypes.byref(p), _ptr(k_hist, "k_hist", dt, n["act_hist"]),
        _ptr(v_hist, "v_hist", dt, n["act_hist"]), _ptr(kept_idx, "kept_idx", torch.int32, n["kept"]),
        _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]),
        _ptr(omega, "omega", torch.float32, n_pairs, optional=n_pairs == 0), n_pairs,
        _ptr(k_comp, "k_comp", dt, n["comp"]), _ptr(v_comp, "v_comp", dt, n["comp"]),
        _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_compact_gather_rope")


def cache_advance(p: Params, k_comp, v_comp, kept_cnt, k_cur, v_cur, out_segments: int, k_next,
                  v_next, ws, stream=None):
    """Next history cache (fkv_cache_advance): the last out_segments - chunk
    kept segments of the compressed cache, then the chunk's own K/V."""
    n, dt = _shapes(p), _act_dtype(p)
    seg_len = p.frame_tokens if p.granularity == _lib.FKV_GRAN_FRAME else 1
    out_n = p.num_layers * p.num_heads * out_segments * seg_len * p.head_dim
    chunk_segs = (p.chunk_frames * p.frame_tokens) // seg_len
    old = out_segments > chunk_segs
    st = _lib.load().fkv_cache_advance(
        ctypes.byref(p), _ptr(k_comp, "k_comp", dt, n["comp"], optional=not old),
        _ptr(v_comp, "v_comp", dt, n["comp"], optional=not old),
        _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]),
        _ptr(k_cur, "k_cur", dt, n["act_cur"]), _ptr(v_cur, "v_cur", dt, n["act_cur"]),
        int(out_segments), _ptr(k_next, "k_next", dt, out_n), _ptr(v_next, "v_next", dt, out_n),
        _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_cache_advance")


def make_step_io(p: Params, inputs: Dict[str, torch.Tensor], outputs: Dict[str, torch.Tensor]) -> StepIO:
    """fkv_step_io_t of tensors already checked for device, dtype and size."""
    n, dt = _shapes(p), _act_dtype(p)
    token = p.granularity == _lib.FKV_GRAN_TOKEN
    io = StepIO()
    io.q_cur = _ptr(inputs["q_cur"], "q_cur", dt, n["act_cur"])
    io.k_cur = _ptr(inputs["k_cur"], "k_cur", dt, n["act_cur"])
    io.v_cur = _ptr(inputs["v_cur"], "v_cur", dt, n["act_cur"])
    io.k_hist = _ptr(inputs["k_hist"], "k_hist", dt, n["act_hist"])
    io.v_hist = _ptr(inputs["v_hist"], "v_hist", dt, n["act_hist"])
    io.q_score = _ptr(inputs.get("q_score"), "q_score", dt, n["q_score"], optional=not token)
    io.head_role = _ptr(inputs.get("head_role"), "head_role", torch.uint8, n["heads"], optional=token)
    io.static_mask = _ptr(inputs.get("static_mask"), "static_mask", torch.uint8, n["mask"], optional=token)
    io.k_per_head = _ptr(inputs["k_per_head"], "k_per_head", torch.int32, n["heads"])
    io.seg_score = _ptr(outputs["seg_score"], "seg_score", torch.float32, n["seg"])
    io.kept_idx = _ptr(outputs["kept_idx"], "kept_idx", torch.int32, n["kept"])
    io.kept_cnt = _ptr(outputs["kept_cnt"], "kept_cnt", torch.int32, n["heads"])
    io.k_comp = _ptr(outputs["k_comp"], "k_comp", dt, n["comp"])
    io.v_comp = _ptr(outputs["v_comp"], "v_comp", dt, n["comp"])
    io.out = _ptr(outputs["out"], "out", dt, n["act_cur"])
    _ptr(outputs["ws"], "ws", torch.uint8, n["ws"])
    return io


def step(p: Params, inputs: Dict[str, torch.Tensor], outputs: Dict[str, torch.Tensor], stream=None,
         io: Optional[StepIO] = None):
    """The whole chunk step (fkv_step).  ``inputs`` holds q_cur, k_cur, v_cur,
    k_hist, v_hist, k_per_head and head_role / static_mask (frame mode) or
    q_score (token mode); ``outputs`` is what :func:`allocate` returns.  A
    prebuilt ``io`` (from :func:`make_step_io`) skips the per-call checks."""
    if io is None:
        io = make_step_io(p, inputs, outputs)
    st = _lib.load().fkv_step(ctypes.byref(p), ctypes.byref(io), outputs["ws"].data_ptr(),
                              _stream(stream))
    _check(st, "fkv_step")


def allocate_fp8(p: Params, device="cuda") -> Dict[str, torch.Tensor]:
    """Buffers of the e4m3 compressed cache (fkv_fp8_cache_t): codes as uint8,
    scales as float32 (k_comp_scale / v_comp_scale: one per kept segment,
    k_cur_scale / v_cur_scale: one per chunk frame, q_scale: one per query)."""
    L, H, D = p.num_layers, p.num_heads, p.head_dim
    Lq = p.chunk_frames * p.frame_tokens
    u8, f32 = torch.uint8, torch.float32
    return {
        "k_comp": torch.empty((L, H, p.comp_rows, D), dtype=u8, device=device),
        "v_comp": torch.empty((L, H, p.comp_rows, D), dtype=u8, device=device),
        "k_comp_scale": torch.empty((L, H, p.hist_frames), dtype=f32, device=device),
        "v_comp_scale": torch.empty((L, H, p.hist_frames), dtype=f32, device=device),
        "k_cur": torch.empty((L, H, Lq, D), dtype=u8, device=device),
        "v_cur": torch.empty((L, H, Lq, D), dtype=u8, device=device),
        "k_cur_scale": torch.empty((L, H, p.chunk_frames), dtype=f32, device=device),
        "v_cur_scale": torch.empty((L, H, p.chunk_frames), dtype=f32, device=device),
        "q_cur": torch.empty((L, H, Lq, D), dtype=u8, device=device),
        "q_scale": torch.empty((L, H, Lq), dtype=f32, device=device),
    }


def make_fp8_cache(p: Params, c: Dict[str, torch.Tensor]) -> _lib.Fp8Cache:
    """fkv_fp8_cache_t over the tensors of allocate_fp8 (shapes checked)."""
    L, H, D = p.num_layers, p.num_heads, p.head_dim
    Lq = p.chunk_frames * p.frame_tokens
    need = {
        "k_comp": (torch.uint8, L * H * p.comp_rows * D), "v_comp": (torch.uint8, L * H * p.comp_rows * D),
        "k_comp_scale": (torch.float32, L * H * p.hist_frames),
        "v_comp_scale": (torch.float32, L * H * p.hist_frames),
        "k_cur": (torch.uint8, L * H * Lq * D), "v_cur": (torch.uint8, L * H * Lq * D),
        "k_cur_scale": (torch.float32, L * H * p.chunk_frames),
        "v_cur_scale": (torch.float32, L * H * p.chunk_frames),
        "q_cur": (torch.uint8, L * H * Lq * D), "q_scale": (torch.float32, L * H * Lq),
    }
    fp = _lib.Fp8Cache()
    for name in _lib.FP8_CACHE_FIELDS:
        dt, n = need[name]
        setattr(fp, name, _ptr(c.get(name), name, dt, n, optional=n == 0))
    return fp


def compact_gather_fp8(p: Params, k_hist, v_hist, kept_idx, kept_cnt, cache, ws, stream=None):
    """Step 4 into the e4m3 cache (fkv_compact_gather_fp8): kept frames
    quantised per segment into cache["k_comp"] / ["v_comp"] and their scales."""
    n, dt = _shapes(p), _act_dtype(p)
    fp = make_fp8_cache(p, cache)
    st = _lib.load().fkv_compact_gather_fp8(
        ctypes.byref(p), _ptr(k_hist, "k_hist", dt, n["act_hist"]),
        _ptr(v_hist, "v_hist", dt, n["act_hist"]), _ptr(kept_idx, "kept_idx", torch.int32, n["kept"]),
        _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]), ctypes.byref(fp),
        _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_compact_gather_fp8")


def quantize_chunk_fp8(p: Params, q_cur, k_cur, v_cur, cache, ws, stream=None):
    """The chunk's own operands in e4m3 (fkv_quantize_chunk_fp8): K / V per
    frame, Q per row."""
    n, dt = _shapes(p), _act_dtype(p)
    fp = make_fp8_cache(p, cache)
    st = _lib.load().fkv_quantize_chunk_fp8(
        ctypes.byref(p), _ptr(q_cur, "q_cur", dt, n["act_cur"]),
        _ptr(k_cur, "k_cur", dt, n["act_cur"]), _ptr(v_cur, "v_cur", dt, n["act_cur"]),
        ctypes.byref(fp), _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_quantize_chunk_fp8")


def attend_compressed_fp8(p: Params, cache, kept_cnt, out, ws, stream=None):
    """Step 5 over the e4m3 cache (fkv_attend_compressed_fp8), bf16 out."""
    n, dt = _shapes(p), _act_dtype(p)
    fp = make_fp8_cache(p, cache)
    st = _lib.load().fkv_attend_compressed_fp8(
        ctypes.byref(p), ctypes.byref(fp), _ptr(kept_cnt, "kept_cnt", torch.int32, n["heads"]),
        _ptr(out, "out", dt, n["act_cur"]), _ptr(ws, "ws", torch.uint8, n["ws"]), _stream(stream))
    _check(st, "fkv_attend_compressed_fp8")


def step_fp8(p: Params, inputs: Dict[str, torch.Tensor], outputs: Dict[str, torch.Tensor],
             cache: Dict[str, torch.Tensor], stream=None, io: Optional[StepIO] = None):
    """The whole chunk step with the e4m3 cache (fkv_step_fp8): ``inputs`` and
    ``outputs`` as for :func:`step` (the bf16 k_comp / v_comp are not used),
    ``cache`` from :func:`allocate_fp8`."""
    if io is None:
        io = make_step_io(p, inputs, outputs)
    fp = make_fp8_cache(p, cache)
    st = _lib.load().fkv_step_fp8(ctypes.byref(p), ctypes.byref(io), ctypes.byref(fp),
                                  outputs["ws"].data_ptr(), _stream(stream))
    _check(st, "fkv_step_fp8")


class _Recorder:
    """Stands in for the loaded library while one wrapper runs: records the C
    function and its converted arguments instead of calling it."""

    def __init__(self, lib):
        self._lib = lib
        self.call = None

    def __getattr__(self, name):
        fn = getattr(self._lib, name)

        def record(*args):
            self.call = (fn, args)
            return _lib.FKV_OK
        return record


def marshal(wrapper, *args, **kwargs):
    """(c_function, c_args) of one call of an entry-point wrapper of this
    module, checked and converted once: ``c_function(*c_args)`` repeats the
    call with no Python-side work (for timing loops, or a serving loop that
    calls the same entry point on the same buffers; the status it returns is
    the caller's to check).  Nothing is launched by marshal itself.  The
    recorded arguments refer to the given tensors and params, which must
    stay alive."""
    real = _lib.load
    rec = _Recorder(real())
    _lib.load = lambda: rec
    try:
        wrapper(*args, **kwargs)
    finally:
        _lib.load = real
    if rec.call is None:
        raise ValueError(f"{getattr(wrapper, '__name__', wrapper)} made no library call")
    return rec.call


def read_status(ws: torch.Tensor, stream=None):
    """(first device-side status since init, (layer*H + head) it was seen on or -1).
    Synchronises the stream."""
    a, b = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.load().fkv_read_status(ws.data_ptr(), _stream(stream), ctypes.byref(a), ctypes.byref(b)),
           "fkv_read_status")
    return a.value, b.value
