"""fp64 CPU oracle of the Forcing-KV chunk step -- TEST INFRASTRUCTURE ONLY.

Nothing on the product path may import, call or execute this package: only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use
it.  It shares no code with the CUDA library (no kernels, headers, helpers,
tables or constants); the only thing both sides consume is the seeded input
generator in ``fkv_workloads``, which holds none of the method's arithmetic.

Modules
  fkv_oracle  numpy float64, usable up to the 1080P and 30-layer workloads
              (attention may be evaluated on a subset of query rows).
  fkv_loops   pure-Python loops over ``math``; tiny inputs only.  A second,
              independent spelling of the same definitions.
  fkv_fp8     the e4m3 compressed cache: codes and per-segment scales (fp32
              decisions, as the kernels take them), dequantisation, and the
              error model of an fp8 tensor-core attention.
  fkv_heuristics  the comparison selectors (uniform eviction, random drop
              with a Philox4x64-10 priority per segment).

Sources (page title and section):
  Forcing-KV (ai-feeds.com/i/paper/2605.09681): "关键模块" items 2 (static
    structural pruning: a fixed keep-mask extracted at inference) and 3
    (dynamic similarity pruning: history grouped by frame, each group scored by
    the current queries' attention, the top few groups kept); "输出与工程收益"
    (the compressed KV replaces the cache inside attention).
  Deep Forcing (bxzpzcl.cn/news/2125000), section 3.1: sink / recent /
    candidate partition, phi_j = sum_r q_r^T k_j, top-C with C = N - S - R;
    section 5.1: budget N = 70-80% of the window.

Parity status: every function is pinned by a ``-m "not gpu"`` test against a
closed form, a library routine, brute force or an invariant, except the
segment-score semantics beyond the one sentence the Forcing-KV page gives
(softmax mass over history keys, summed over the scoring queries): that
reading is a choice, and is "parity unpinned" as to the pages.
"""
