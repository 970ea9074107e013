"""Measurement of the hot-path rows other than the headline decode step (`bench.py
--workload score|encode|attn4|attn3big|search|search4|compare`): one JSON line each, same keys as the headline
line (metric, value, roofline of the row's dominant kernel, clocks, launches) plus the CPU
oracle timed on a bounded sample of the same workload.

Workloads (all synthetic, seeded; the big inputs are drawn on the GPU):
  score   64 sequences x 8 KV heads, context 16384 growing by one token per step; prod
          2+1 keys (m = 128), fp16 norms; a step appends one bf16 token per (sequence,
          head) and scores 32 query heads (4 per KV head) over every key.
  encode  the prefill of that cache: 8,388,608 bf16 vectors, prod 2+1, d = 128.
  attn4   4 sequences x 8 KV heads x context 131072, K and V 4-bit MSE, fp16 norms, bf16
          K/V with a per-(sequence, head) scale ~ U(0.5, 2); one tq_decode_step per step.
  attn3big  the 3-bit prod decode step (2-bit codes + 128 QJL signs, fp16 norms) over 64
          sequences x 8 KV heads x context 16384 (872 MB of packed K/V: HBM-bound).
  search  1,000,000 x 1536 L2-normalised fp32 database vectors, 2-bit MSE codes, 1024
          queries, top-10.
"""

import json
import os
import time

import bench

ROWS = ("score", "encode", "attn4", "search")

# When a list, _line appends each row's line here instead of printing it (the default bench run
# folds every row into the headline line, see collect_rows).
COLLECT = None


def _events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def _peak(kind):
    peaks, src = bench.measured_peaks()
    if kind == "hbm":
        return float(peaks.get("hbm_gbs", bench.FALLBACK_HBM_GBS)), f"{src} hbm_gbs"
    return float(peaks.get("bf16_tflops", 1590.0)), f"{src} bf16_tflops"


def _line(args, metric, value, unit, ms_per_step, config, roofline, launches, clocks, extra=None, cpu=None):
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": config.pop("dtype"), "data": "synthetic", "config": config,
            "roofline": roofline, "gpu_launches": launches, "clocks": clocks}
    if extra:
        line.update(extra)
    if cpu:
        line["cpu_baseline"] = cpu
    if COLLECT is not None:
        COLLECT.append(line)
        return
    print(json.dumps(line), flush=True)


def _encode_into(tq, h, cache, x_of, L, slice_len, torch):
    """Encodes the cache prefill in slices of `slice_len` tokens (x_of(l0, n) -> [B, Hkv, n, d]);
    returns the device milliseconds spent in the encode calls."""
    ms = 0.0
    for l0 in range(0, L, slice_len):
        n = min(slice_len, L - l0)
        x = x_of(l0, n)
        a, b = _events(torch)
        a.record()
        out = h.encode(x)
        b.record()
        torch.cuda.synchronize()
        ms += a.elapsed_time(b)
        for name in ("codes", "signs", "norms", "rnorms"):   # (QJL-only rows have no codes or rnorms)
            if out[name] is not None:
                getattr(cache, name)[:, :, l0:l0 + n].copy_(out[name])
        del x, out
    return ms


# ------------------------------------------------------------------ score (cfg 5)

S5 = dict(B=64, Hkv=8, Hq=32, L0=16384, d=128, bits=3, m=128, seed_handle=0, seed_prefill=10, seed_step=11)


def run_score(args):
    import torch
    import embedding_vector_quantization_b200 as tq
    if args.small:
        S5["B"] = 16        # 109 MB of packed keys + 34 MB of logits
    B, Hkv, Hq, L0, d = S5["B"], S5["Hkv"], S5["Hq"], S5["L0"], S5["d"]
    T = min(args.steps, 256)
    L_cap = L0 + 256
    h = tq.Handle(d, S5["bits"], S5["seed_handle"], qjl_m=S5["m"])
    cache = tq.Cache(h, B, Hkv, L_cap)
    g = torch.Generator(device="cuda").manual_seed(S5["seed_prefill"])
    enc_ms = _encode_into(tq, h, cache,
                          lambda l0, n: torch.randn(B, Hkv, n, d, generator=g, device="cuda").to(torch.bfloat16),
                          L0, 2048, torch)
    gs = torch.Generator(device="cuda").manual_seed(S5["seed_step"])
    W = args.warmup
    toks = torch.randn(T + W, B, Hkv, d, generator=gs, device="cuda").to(torch.bfloat16)
    qs = torch.randn(T + W, B, Hq, d, generator=gs, device="cuda")
    lens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, Hq, L_cap, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_score_workspace_bytes(h.ptr, B, Hq), dtype=torch.uint8, device="cuda")
    k_in, q_in = toks[0].clone(), qs[0].clone()

    def step():
        tq.tq_append(h.ptr, k_in, B, Hkv, cache.struct, lens, 1)
        tq.tq_score(h.ptr, q_in, B, Hq, Hkv, cache.struct, lens, logits, ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    tq.tq_timer_read(None, forget=True)
    tq.tq_timer_enable(True)
    graph_k = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_k):
        step()
    tq.tq_timer_enable(False)
    return _score_timed(args, torch, tq, h, graph, graph_k, step, toks, qs, k_in, q_in, lens, T, W, L0, enc_ms)


def _score_timed(args, torch, tq, h, graph, graph_k, step, toks, qs, k_in, q_in, lens, T, W, L0, enc_ms):
    B, Hkv, Hq = S5["B"], S5["Hkv"], S5["Hq"]
    G = Hq // Hkv

    def run(gr, t0, timed):
        evs = []
        for t in range(t0, t0 + T):
            k_in.copy_(toks[W + t - t0])
            q_in.copy_(qs[W + t - t0])
            ev = _events(torch)
            ev[0].record()
            gr.replay()
            ev[1].record()
            evs.append(ev)
            if not timed:
                torch.cuda.synchronize()
                yield t
        torch.cuda.synchronize()
        if timed:
            yield sum(a.elapsed_time(b) for a, b in evs)

    lens.fill_(L0 - W)
    for t in range(W):
        k_in.copy_(toks[t])
        q_in.copy_(qs[t])
        graph.replay()
    torch.cuda.synchronize()
    sampler = bench.ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    sampler.start()
    total_ms = next(run(graph, 0, True))
    clocks = sampler.stop()
    # score-kernel time per launch from the instrumented capture (same steps again)
    lens.fill_(L0)
    score_ms, score_n = 0.0, 0
    for _ in run(graph_k, 0, False):
        ms_k, n_k = tq.tq_timer_read("score", forget=False)
        score_ms += ms_k
        score_n += n_k
    _, kernels_per_step = tq.tq_timer_read(None, forget=False)
    keys = sum(B * Hkv * (L0 + t + 1) for t in range(T))          # KV-head keys scored
    packed = keys * 52                                              # codes 32 + signs 16 + norm 2 + rnorm 2
    written = keys * G * 4                                          # fp32 logits of 4 query heads
    peak, src = _peak("hbm")
    ach = (packed + written) / (score_ms / 1e3) / 1e9
    cfg = {"workload": "score step, TurboQuant prod 3-bit (2-bit Lloyd-Max + 1-bit QJL m=128), d=128, "
                       "64 sequences x 8 KV heads, 32 query heads, context 16384 growing by 1 per step",
           "B": B, "Hkv": Hkv, "Hq": Hq, "context_start": L0, "d": 128, "dtype": "int8 mma / f32",
           "l2": "not flushed: each step reads 440 MB of packed keys and writes 135 MB of logits (> 126 MB L2)",
           "step": "tq_append (one bf16 token per sequence and head, len += 1) + tq_score, one CUDA graph replay"}
    roof = {"bound": "hbm", "kernel": "score_prod2_kernel", "achieved": ach, "peak": peak, "unit": "GB/s",
            "frac": ach / peak, "traffic": None, "peak_source": src, "launch_ms": score_ms / max(score_n, 1),
            "algorithmic_bytes_per_launch": (packed + written) / T}
    extra = {"keys_scored_per_s": keys / (total_ms / 1e3), "query_key_pairs_per_s": keys * G / (total_ms / 1e3),
             "packed_gb_per_s": packed / (total_ms / 1e3) / 1e9,
             "prefill_encode": {"vectors": B * Hkv * L0, "ms": enc_ms,
                                "vectors_per_s": B * Hkv * L0 / (enc_ms / 1e3)}}
    cpu = None if args.no_cpu_baseline else oracle_score_sample()
    if args.small:
        cfg["workload"] += " [reduced for profiling: 16 sequences]"
    _line(args, "keys scored/sec (cfg 5 score step)", extra["keys_scored_per_s"], "keys/s", total_ms / T, cfg, roof,
          kernels_per_step * T, clocks, extra, cpu)


def oracle_score_sample(budget_s=12.0):
    """The oracle scoring 4 query heads over 16384 prod-encoded keys of one (sequence, KV
    head), repeated for about budget_s seconds (setup untimed); keys/s."""
    import numpy as np
    import torch
    from oracle import codebook, ops, quant, rotation
    d, m, L = 128, 128, S5["L0"]
    Pi, S = rotation.rotation(d, S5["seed_handle"], m)
    c, beta = codebook.lloyd_max(d, 2)
    x = torch.randn(L, d, generator=torch.Generator().manual_seed(S5["seed_prefill"])).to(torch.bfloat16).double().numpy()
    e = quant.encode_prod(x, Pi, S, c, beta, "f16")
    q = torch.randn(4, d, generator=torch.Generator().manual_seed(S5["seed_step"])).double().numpy()
    reps, t0 = 0, time.perf_counter()
    while True:
        for hq in range(4):
            ops.score_prod(q[hq], e["idx"], e["n_stored"], e["sigma"], e["rnorm_stored"], Pi, S, c)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": reps * L / el, "unit": "keys/s", "cores": bench.blas_threads(), "kind": "oracle",
            "sample": f"{reps} x (4 query heads over 16384 keys of one sequence and KV head) in {el:.1f} s, "
                      f"fp64 NumPy oracle"}


# ------------------------------------------------------------------ encode (cfg 5 prefill)

def run_encode(args):
    """Prefill encode of the score workload's cache: 8,388,608 bf16 vectors, prod 2+1, in
    launches of 1,048,576 vectors (each pass re-encodes the whole prefill)."""
    import torch
    import embedding_vector_quantization_b200 as tq
    B, Hkv, L0, d, m = S5["B"], S5["Hkv"], S5["L0"], S5["d"], S5["m"]
    h = tq.Handle(d, S5["bits"], S5["seed_handle"], qjl_m=m)
    n_all = B * Hkv * L0 if not args.small else 1 << 20   # small: one launch, 268 MB of input
    per = 1 << 20
    g = torch.Generator(device="cuda").manual_seed(S5["seed_prefill"])
    x = torch.randn(n_all, d, generator=g, device="cuda").to(torch.bfloat16)      # 2.15 GB
    out = h.alloc_rows((per,), x.device)
    passes = max(1, args.steps)

    def one_pass():
        for r0 in range(0, n_all, per):
            h.encode(x[r0:r0 + per], out=out)

    for _ in range(max(1, args.warmup)):
        one_pass()
    torch.cuda.synchronize()
    tq.tq_timer_read(None, forget=True)
    sampler = bench.ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    sampler.start()
    a, b = _events(torch)
    a.record()
    for _ in range(passes):
        one_pass()
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = a.elapsed_time(b) / passes
    # per-launch kernel time, timed separately with the library's event pairs
    tq.tq_timer_enable(True)
    one_pass()
    torch.cuda.synchronize()
    tq.tq_timer_enable(False)
    k_ms, k_n = tq.tq_timer_read("encode", forget=True)
    launches_per_pass = (n_all + per - 1) // per
    flops = 2 * d * d + 2 * m * d                     # algorithmic: rotation + QJL projection, per vector
    peak, src = _peak("tensor")
    ach = per * flops / (k_ms / max(k_n, 1) / 1e3) / 1e12
    cfg = {"workload": "prefill encode, TurboQuant prod 3-bit (2-bit Lloyd-Max + 1-bit QJL m=128), d=128, "
                       "bf16 input, 8,388,608 vectors (64 sequences x 8 KV heads x 16384)",
           "vectors": n_all, "launch_vectors": per, "d": d, "dtype": "bf16 hi/lo tcgen05, f32 accumulate",
           "l2": "not flushed: each pass reads 2.15 GB of input (> 126 MB L2)"}
    roof = {"bound": "tensor", "kernel": "encode_tc_kernel", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak, "traffic": None, "peak_source": src, "launch_ms": k_ms / max(k_n, 1),
            "algorithmic_flops_per_launch": per * flops,
            "note": "algorithmic flops (2d^2 + 2md per vector); the hi/lo split runs 5 MMA passes of that size"}
    hbm_bytes = n_all * (2 * d + 32 + 16 + 2 + 2)
    extra = {"vectors_encoded_per_s": n_all / (ms / 1e3), "hbm_gb_per_s": hbm_bytes / (ms / 1e3) / 1e9}
    cpu = None if args.no_cpu_baseline else oracle_encode_sample()
    if args.small:
        cfg["workload"] += " [reduced for profiling: 1,048,576 vectors]"
    _line(args, "vectors encoded/sec (cfg 5 prefill encode)", extra["vectors_encoded_per_s"], "vectors/s", ms, cfg,
          roof, launches_per_pass * passes, clocks, extra, cpu)


def oracle_encode_sample(budget_s=12.0, rows=16384):
    """The oracle's prod encode of `rows` bf16 vectors, repeated for about budget_s seconds."""
    import torch
    from oracle import codebook, quant, rotation
    Pi, S = rotation.rotation(128, S5["seed_handle"], 128)
    c, beta = codebook.lloyd_max(128, 2)
    x = torch.randn(rows, 128, generator=torch.Generator().manual_seed(S5["seed_prefill"])).to(torch.bfloat16)
    x = x.double().numpy()
    reps, t0 = 0, time.perf_counter()
    while True:
        quant.encode_prod(x, Pi, S, c, beta, "f16")
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": reps * rows / el, "unit": "vectors/s", "cores": bench.blas_threads(), "kind": "oracle",
            "sample": f"{reps} x {rows} bf16 vectors, prod 2+1, d=128, in {el:.1f} s, fp64 NumPy oracle"}


# ------------------------------------------------------------------ attention, 4-bit MSE (cfg 3)

S3 = dict(B=4, Hkv=8, Hq=32, L=131072, d=128, bits=4, seed_k=5, seed_v=6, seed_q=7)
# the 3-bit prod decode step over a cache of the streaming workload's size: 64 sequences x 8 KV
# heads x 16384 tokens (872 MB of packed K/V), an HBM-bound read
S5A = dict(B=64, Hkv=8, Hq=32, L=16384, d=128, bits=3, m=128, seed_k=10, seed_v=12, seed_q=13)


def run_attn4(args):
    import torch
    import embedding_vector_quantization_b200 as tq
    if args.small:
        S3["B"] = 1         # 138 MB of packed K/V
    hk = tq.Handle(S3["d"], S3["bits"], 0, norm_dtype=tq.TQ_F16)
    hv = tq.Handle(S3["d"], S3["bits"], 1, norm_dtype=tq.TQ_F16)
    spec = dict(S3, bytes_per_token=2 * (64 + 2), kernel="attn_mse4_kernel", scaled=True,
                workload="GQA decode step, TurboQuant MSE 4-bit K and V, d=128, B=%d, 8 KV heads / 32 query heads, "
                         "context 131072, bf16 K/V N(0,1) x U(0.5,2) per (sequence, head)" % S3["B"],
                dtype="s8xs8->s32 MMA (22-bit fixed-point queries, Walsh planes), u8xu8->s32 MMA (16-bit "
                      "weights), f32 softmax/combine",
                metric="packed-KV GB/s (cfg 3 decode step, 4-bit MSE)")
    cpu = None if args.no_cpu_baseline else oracle_attn4_sample()
    _run_decode_row(args, tq, torch, hk, hv, spec, cpu)


def run_attn3big(args):
    import torch
    import embedding_vector_quantization_b200 as tq
    if args.small:
        S5A["B"] = 8        # 109 MB of packed K/V
    hk = tq.Handle(S5A["d"], S5A["bits"], 0, qjl_m=S5A["m"])
    hv = tq.Handle(S5A["d"], S5A["bits"], 1, qjl_m=S5A["m"])
    # caches of 256 MB and more take the two-kernel form (scores, then values; timed together)
    env2k = os.environ.get("TQ_ATTN_2K", "")
    two = env2k not in ("", "0") or (env2k == "" and S5A["B"] * S5A["Hkv"] * S5A["L"] * 104 >= 256e6)
    spec = dict(S5A, bytes_per_token=2 * (32 + 16 + 2 + 2),
                kernel="score_prod2_kernel<true> + value_prod2_kernel" if two else "attn_prod2_kernel",
                scaled=False,
                workload="GQA decode step, TurboQuant prod 3-bit (2-bit Lloyd-Max + 1-bit QJL m=128), d=128, "
                         "B=%d, 8 KV heads / 32 query heads, context 16384, bf16 K/V N(0,1)" % S5A["B"],
                dtype="s8xs8->s32 MMA (22-bit fixed-point queries), u8xu8->s32 MMA (16-bit weights), "
                      "f32 softmax/combine",
                metric="packed-KV GB/s (3-bit decode step over an HBM-sized cache)")
    _run_decode_row(args, tq, torch, hk, hv, spec, None)


def _run_decode_row(args, tq, torch, hk, hv, spec, cpu):
    """One decode step (tq_decode_step in a CUDA graph) over a cache larger than L2, timed per step."""
    B, Hkv, Hq, L, d = spec["B"], spec["Hkv"], spec["Hq"], spec["L"], spec["d"]
    kc, vc = tq.Cache(hk, B, Hkv, L), tq.Cache(hv, B, Hkv, L)
    enc_ms = 0.0
    for h, cache, seed in ((hk, kc, spec["seed_k"]), (hv, vc, spec["seed_v"])):
        g = torch.Generator(device="cuda").manual_seed(seed)
        if spec["scaled"]:
            scl = (0.5 + 1.5 * torch.rand(B, Hkv, 1, 1, generator=g, device="cuda"))      # U(0.5, 2) per (b, head)
        else:
            scl = torch.ones(B, Hkv, 1, 1, device="cuda")
        enc_ms += _encode_into(tq, h, cache, lambda l0, n: (torch.randn(B, Hkv, n, d, generator=g, device="cuda")
                                                           * scl).to(torch.bfloat16), L, 8192, torch)
    gq = torch.Generator(device="cuda").manual_seed(spec["seed_q"])
    W, T = args.warmup, args.steps
    qs = torch.randn(T + W, B, Hq, d, generator=gq, device="cuda")
    kn = torch.randn(T + W, B, Hkv, d, generator=gq, device="cuda").to(torch.bfloat16)
    vn = torch.randn(T + W, B, Hkv, d, generator=gq, device="cuda").to(torch.bfloat16)
    L0 = L - 1
    lens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L), dtype=torch.uint8, device="cuda")
    q_in, k_in, v_in = qs[0].clone(), kn[0].clone(), vn[0].clone()

    def step():
        tq.tq_decode_step(hk.ptr, hv.ptr, q_in, k_in, v_in, B, Hq, Hkv, kc.struct, vc.struct, lens, 1 / d ** 0.5,
                          out, ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    tq.tq_timer_read(None, forget=True)
    tq.tq_timer_enable(True)
    graph_k = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_k):
        step()
    tq.tq_timer_enable(False)

    def set_inputs(t):
        q_in.copy_(qs[t])
        k_in.copy_(kn[t])
        v_in.copy_(vn[t])
        lens.fill_(L0)

    for t in range(W):
        set_inputs(t)
        graph.replay()
    torch.cuda.synchronize()
    sampler = bench.ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    sampler.start()
    evs = []
    for t in range(T):
        set_inputs(W + t)
        ev = _events(torch)
        ev[0].record()
        graph.replay()
        ev[1].record()
        evs.append(ev)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    total_ms = sum(a.elapsed_time(b) for a, b in evs)
    split_ms, split_n = 0.0, 0
    kern = {}
    for t in range(T):
        set_inputs(W + t)
        graph_k.replay()
        torch.cuda.synchronize()
        for name in ("prologue", "attn_split", "attn_combine"):
            ms_k, n_k = tq.tq_timer_read(name, forget=False)
            kern[name] = kern.get(name, 0.0) + ms_k
            if name == "attn_split":
                split_ms += ms_k
                split_n += n_k
    _, kernels_per_step = tq.tq_timer_read(None, forget=False)
    bytes_step = B * Hkv * L * spec["bytes_per_token"]
    peak, src = _peak("hbm")
    ach = bytes_step / (split_ms / max(split_n, 1) / 1e3) / 1e9
    cfg = {"workload": spec["workload"], "B": B, "Hkv": Hkv, "Hq": Hq, "context": L, "d": d, "dtype": spec["dtype"],
           "l2": "not flushed: each step reads %.1f MB of packed K/V (> 126 MB L2)" % (bytes_step / 1e6),
           "step": "tq_decode_step, one CUDA graph replay; len reset outside the timed bracket"}
    roof = {"bound": "hbm", "kernel": spec["kernel"], "achieved": ach, "peak": peak, "unit": "GB/s",
            "frac": ach / peak, "traffic": None, "peak_source": src, "launch_ms": split_ms / max(split_n, 1),
            "algorithmic_bytes_per_launch": bytes_step}
    value = bytes_step * T / (total_ms / 1e3) / 1e9
    extra = {"tokens_per_s": B * Hkv * L * T / (total_ms / 1e3),
             "kernel_us_per_step": {k: round(1e3 * v / T, 2) for k, v in kern.items()},
             "prefill_encode": {"vectors": 2 * B * Hkv * L, "ms": enc_ms,
                                "vectors_per_s": 2 * B * Hkv * L / (enc_ms / 1e3)}}
    if args.small:
        cfg["workload"] += " [reduced for profiling]"
    _line(args, spec["metric"], value, "GB/s", total_ms / T, cfg, roof, kernels_per_step * T, clocks, extra, cpu)


def oracle_attn4_sample(budget_s=12.0, L=32768):
    """The oracle's decode attention of 4 query heads over L tokens of one (sequence, KV head)
    of 4-bit MSE K/V (encoded once, untimed); packed GB/s."""
    import numpy as np
    import torch
    from oracle import codebook, ops, quant, rotation
    d = 128
    c, beta = codebook.lloyd_max(d, 4)
    caches = []
    for seed, hseed in ((S3["seed_k"], 0), (S3["seed_v"], 1)):
        Pi = rotation.rotation(d, hseed, 0)[0]
        x = torch.randn(L, d, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16).double().numpy()
        e = quant.encode_mse(x, Pi, c, beta, "f16")
        caches.append({"idx": e["idx"].reshape(1, 1, L, d), "n": e["n_stored"].reshape(1, 1, L), "Pi": Pi, "c": c})
    q = torch.randn(1, 4, d, generator=torch.Generator().manual_seed(S3["seed_q"])).double().numpy()
    reps, t0 = 0, time.perf_counter()
    while True:
        ops.decode_attention(q, caches[0], caches[1], [L], 1 / np.sqrt(d))
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": reps * L * 2 * 66 / el / 1e9, "unit": "GB/s", "cores": bench.blas_threads(), "kind": "oracle",
            "sample": f"{reps} x (4 query heads over {L} tokens of one sequence and KV head) in {el:.1f} s, "
                      f"fp64 NumPy oracle"}


# ------------------------------------------------------------------ search (cfg 4)

S4 = dict(n=1_000_000, nq=1024, d=1536, bits=2, k=10, seed_handle=0, seed_db=8, seed_q=9)


FP32_LANES_PER_SM = 128   # fp32 FMA lanes per B200 SM (4 partitions x 32)


def run_search(args, bits=None):
    """cfg-4 search at 2 or 4 bits on the tcgen05 kernel (TQ_SIMT=1: the SIMT kernel)."""
    import torch
    import embedding_vector_quantization_b200 as tq
    bits = S4["bits"] if bits is None else bits
    if args.small:
        S4["n"] = 400_000   # 154 MB of 2-bit codes
    n, nq, d, k = S4["n"], S4["nq"], S4["d"], S4["k"]
    h = tq.Handle(d, bits, S4["seed_handle"])
    g = torch.Generator(device="cuda").manual_seed(S4["seed_db"])
    db = torch.randn(n, d, generator=g, device="cuda")
    db /= db.norm(dim=1, keepdim=True)
    gq = torch.Generator(device="cuda").manual_seed(S4["seed_q"])
    q = torch.randn(nq, d, generator=gq, device="cuda")
    q /= q.norm(dim=1, keepdim=True)
    a, b = _events(torch)
    a.record()
    enc = h.encode(db)
    b.record()
    torch.cuda.synchronize()
    enc_ms = a.elapsed_time(b)
    ws = torch.empty(tq.tq_search_workspace_bytes(h.ptr, nq, n, k), dtype=torch.uint8, device="cuda")
    T = max(1, min(args.steps, 5))
    for _ in range(max(1, min(args.warmup, 3))):
        idx, sc = h.search_topk(q, enc["codes"], enc["norms"], k, workspace=ws)
    torch.cuda.synchronize()
    sampler = bench.ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    sampler.start()
    a.record()
    for _ in range(T):
        idx, sc = h.search_topk(q, enc["codes"], enc["norms"], k, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = a.elapsed_time(b) / T
    tq.tq_timer_read(None, forget=True)
    tq.tq_timer_enable(True)
    h.search_topk(q, enc["codes"], enc["norms"], k, workspace=ws)
    torch.cuda.synchronize()
    tq.tq_timer_enable(False)
    s_ms, s_n = tq.tq_timer_read("search", forget=False)
    _, launches = tq.tq_timer_read(None, forget=True)
    # recall@10 against exact fp32 inner products (no TF32), in database chunks
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    best_s = torch.full((nq, k), -float("inf"), device="cuda")
    best_i = torch.zeros((nq, k), dtype=torch.int64, device="cuda")
    for r0 in range(0, n, 131072):
        s_ = q @ db[r0:r0 + 131072].T
        ts, ti = s_.topk(k, dim=1)
        cs, ci = torch.cat([best_s, ts], 1), torch.cat([best_i, ti + r0], 1)
        best_s, sel = cs.topk(k, dim=1)
        best_i = ci.gather(1, sel)
    torch.backends.cuda.matmul.allow_tf32 = prev
    hits = sum(len(set(x.tolist()) & set(y.tolist())) for x, y in zip(idx.cpu(), best_i.cpu()))
    recall = hits / (nq * k)
    flops = 2.0 * d * nq * n
    ach = flops / (s_ms / max(s_n, 1) / 1e3) / 1e12
    cfg = {"workload": f"top-10 inner-product search, TurboQuant MSE {bits}-bit, d=1536, 1,000,000 L2-normalised "
                       "N(0,I) database vectors, 1024 queries (stands in for the pages' vector-search benchmarks)",
           "n": n, "nq": nq, "d": d, "k": k,
           "l2": f"not flushed: the {n * d * bits // 8 // 1000000} MB of codes exceed the 126 MB L2"}
    if not os.environ.get("TQ_SIMT") and d % 64 == 0 and d >= 128:
        # tcgen05 int8 contractions into tensor memory: the measured bf16 dense peak x 2 (the
        # nominal int8 : bf16 ratio, 4.5 : 2.25 PFLOP/s)
        bf16, src = _peak("tensor")
        peak = 2.0 * bf16
        cfg["dtype"] = ("int8 tcgen05 mma (15-bit centroid and query pieces: three contractions into two "
                        "int32 accumulators in tensor memory)")
        roof = {"bound": "tensor", "kernel": "search_tc_kernel", "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                "peak_source": f"{src} x 2 (int8 : bf16 nominal ratio)",
                "launch_ms": s_ms / max(s_n, 1), "algorithmic_flops_per_launch": flops,
                "note": "algorithmic 2d flops per (query, vector); the kernel executes 3x that in int8 MMA "
                        "operations (C_h Q_h, C_h Q_l, C_l Q_h), so its tensor-bound ceiling is 1/3 of the peak"}
    else:
        # fp32 FMAs on the CUDA cores: SMs x 128 lanes x 2 flop x the median sampled SM clock
        sm_mhz = clocks.get("sm_mhz") or 1965.0
        peak = torch.cuda.get_device_properties(0).multi_processor_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12
        cfg["dtype"] = "f32 SIMT (centroid table in shared memory)"
        roof = {"bound": "alu", "kernel": "search_simt_kernel", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": None,
                "peak_source": "derived: SMs x 128 fp32 FMA lanes x 2 flop x median sampled SM clock",
                "launch_ms": s_ms / max(s_n, 1), "algorithmic_flops_per_launch": flops}
    extra = {"queries_per_s": nq / (ms / 1e3), "recall_at_10": recall,
             "db_encode": {"vectors": n, "ms": enc_ms, "vectors_per_s": n / (enc_ms / 1e3), "input": "fp32"}}
    cpu = None if args.no_cpu_baseline else oracle_search_sample(bits=bits)
    if args.small:
        cfg["workload"] += " [reduced for profiling: 400,000 vectors]"
    _line(args, f"queries/sec (cfg 4 top-10 search, 1M x 1536, {bits}-bit)", extra["queries_per_s"], "queries/s", ms,
          cfg, roof, launches * T, clocks, extra, cpu)


def oracle_search_sample(budget_s=12.0, n=32768, nq=64, bits=None):
    """The oracle's top-10 search of nq queries over n vectors (d = 1536; encode untimed)."""
    import torch
    from oracle import codebook, ops, quant, rotation
    d = S4["d"]
    bits = S4["bits"] if bits is None else bits
    Pi = rotation.rotation(d, S4["seed_handle"], 0)[0]
    c, beta = codebook.lloyd_max(d, bits)
    x = torch.randn(n, d, generator=torch.Generator().manual_seed(S4["seed_db"])).double()
    x = (x / x.norm(dim=1, keepdim=True)).numpy()
    e = quant.encode_mse(x, Pi, c, beta, "f32")
    q = torch.randn(nq, d, generator=torch.Generator().manual_seed(S4["seed_q"])).double()
    q = (q / q.norm(dim=1, keepdim=True)).numpy()
    reps, t0 = 0, time.perf_counter()
    while True:
        s = ops.search_scores(q, e["idx"], e["n_stored"], Pi, c)
        ops.topk(s, S4["k"])
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    scale = S4["n"] / n
    return {"value": reps * nq / el / scale, "unit": "queries/s", "cores": bench.blas_threads(), "kind": "oracle",
            "sample": f"{reps} x ({nq} queries over {n} vectors) in {el:.1f} s, scaled to 1,000,000 vectors; "
                      f"fp64 NumPy oracle"}


def run_compare(args):
    """Uncompressed-attention comparator: the cfg-2 decode attention (B = 1, 8 KV / 32 query heads,
    context 32768, d = 128) over the 3-bit TurboQuant cache (tq.attn_decode: query rotation, int8
    tensor-core attention, combine) against the same attention over the K/V held uncompressed in
    bf16 and in fp32 ("TurboQuant: redefining AI efficiency", "Experimental results":
    attention-logit speed of 4-bit keys against 32-bit keys). The uncompressed attention is two
    batched GEMMs (cuBLAS) with a softmax between them, which streams K and V at these decode
    shapes; torch's fused scaled_dot_product_attention is timed too, as context (it spreads a
    decode of one sequence over only its 8 (batch, head) units). Every call is timed cold: L2 is
    flushed (256 MB write) before each one. A comparator, not a target."""
    import torch
    import torch.nn.functional as F
    import embedding_vector_quantization_b200 as tq
    import workloads as synth
    Wc = bench.W
    B, Hkv, Hq, L, d, m = Wc["B"], Wc["Hkv"], Wc["Hq"], Wc["L"], Wc["d"], Wc["m"]
    dev = torch.device("cuda", 0)
    hk = tq.Handle(d, Wc["bits"], Wc["seed_k_handle"], qjl_m=m)
    hv = tq.Handle(d, Wc["bits"], Wc["seed_v_handle"], qjl_m=m)
    K = synth.outlier_kv(seed=Wc["seed_k"]).to(dev)   # [B, Hkv, L, d] bf16
    V = synth.outlier_kv(seed=Wc["seed_v"]).to(dev)
    kc, vc = tq.Cache(hk, B, Hkv, L, dev), tq.Cache(hv, B, Hkv, L, dev)
    kc.fill(K)
    vc.fill(V)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(Wc["seed_q"])).to(dev)
    scale = 1.0 / d ** 0.5
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    # the G query heads of KV head h (query heads G h .. G h + G - 1) as a query length of G over that
    # head's keys: plain multi-head attention, the same result as the GQA decode, no K/V repetition
    G = Hq // Hkv
    qf = q.view(B, Hkv, G, d)
    qb, Kf, Vf = qf.to(torch.bfloat16), K.float(), V.float()
    Kt, Kft = K.transpose(-1, -2), Kf.transpose(-1, -2)

    def gemm_attn(qq, KT, VV):   # [B, Hkv, G, L] scores, softmax, [B, Hkv, G, d] output
        return torch.softmax(torch.matmul(qq, KT) * scale, dim=-1, dtype=torch.float32).to(VV.dtype) @ VV

    calls = {
        "turboquant_3bit": lambda: tq.attn_decode(hk, hv, q, kc, vc, lens, scale, out=out, workspace=ws),
        "gemm_bf16": lambda: gemm_attn(qb, Kt, V),
        "gemm_fp32": lambda: gemm_attn(qf, Kft, Vf),
        "sdpa_bf16": lambda: F.scaled_dot_product_attention(qb, K, V, scale=scale),
        "sdpa_fp32": lambda: F.scaled_dot_product_attention(qf, Kf, Vf, scale=scale),
    }
    reps = max(5, min(args.steps, 50))
    a, b = _events(torch)
    us = {}
    sampler = bench.ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    sampler.start()
    for name, fn in calls.items():
        for _ in range(max(3, args.warmup)):
            fn()
        t = []
        for _ in range(reps):
            flush.zero_()
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            t.append(a.elapsed_time(b) * 1e3)
        us[name] = sorted(t)[len(t) // 2]
    clocks = sampler.stop()
    kv_bytes = {"turboquant_3bit": B * Hkv * L * bench.PACKED_BYTES_PER_TOKEN,
                "gemm_bf16": 2 * B * Hkv * L * d * 2, "gemm_fp32": 2 * B * Hkv * L * d * 4,
                "sdpa_bf16": 2 * B * Hkv * L * d * 2, "sdpa_fp32": 2 * B * Hkv * L * d * 4}
    cfg = {"workload": bench.WORKLOAD_NAME + "; the same K/V uncompressed in bf16 and fp32 for the comparator",
           "dtype": "int8 mma / f32 (TurboQuant); bf16 and f32 (torch scaled_dot_product_attention)",
           "l2": "flushed before every timed call (256 MB write)"}
    extra = {"median_us": us, "kv_bytes": kv_bytes,
             "kv_gb_per_s": {k: kv_bytes[k] / (us[k] * 1e-6) / 1e9 for k in us},
             "speedup_vs_bf16": us["gemm_bf16"] / us["turboquant_3bit"],
             "speedup_vs_fp32": us["gemm_fp32"] / us["turboquant_3bit"],
             "note": "a comparator: uncompressed attention as cuBLAS batched GEMMs + softmax (the faster of the two "
                     "uncompressed forms timed here). The fp32 GEMMs at these skinny shapes stream at a few hundred "
                     "GB/s, so the ratio against fp32 overstates the gain; the line's value is the ratio against "
                     "bf16. The pages quote up to 8x for 4-bit keys against 32-bit keys on H100, attention-logit "
                     "computation alone"}
    roof = {"bound": "hbm", "kernel": "tq_attn_decode (3 launches)", "achieved": kv_bytes["turboquant_3bit"] /
            (us["turboquant_3bit"] * 1e-6) / 1e9, "peak": _peak("hbm")[0], "unit": "GB/s",
            "frac": kv_bytes["turboquant_3bit"] / (us["turboquant_3bit"] * 1e-6) / 1e9 / _peak("hbm")[0],
            "traffic": None, "peak_source": _peak("hbm")[1]}
    _line(args, "decode attention speedup of 3-bit TurboQuant K/V over uncompressed bf16 K/V (cfg-2 shapes)",
          extra["speedup_vs_bf16"], "x", us["turboquant_3bit"] / 1e3, cfg, roof, 3 * reps, clocks, extra)


# ------------------------------------------------------------------ polar and QJL-only scores (next rows)

def run_score_kind(args, kind):
    """Scores of 32 query heads (4 per KV head) over a cache of the next rows' formats, d = 128:
    kind "polar" (recursive polar transform, 4 bits at level 1, 2 bits above: 48-byte rows,
    fp32 norms; 32 sequences x 8 KV heads x 16384 keys) or "qjl" (QJL-only 1-bit rows: 128 sign
    bits and an fp16 norm; 64 x 8 x 16384). One tq_score per step in a CUDA graph; the prefill
    encode is timed too. Both score kernels run on the CUDA cores (table lookups and fp32 FMAs
    for polar, sign-weighted sums for QJL-only), so the roofline is the fp32 SIMT peak."""
    import torch
    import embedding_vector_quantization_b200 as tq
    d, Hkv, G, L = 128, 8, 4, 16384
    B = 32 if kind == "polar" else 64
    if args.small:
        B = 4
    Hq = Hkv * G
    h = tq.PolarHandle(d, 4, 2, seed=0) if kind == "polar" else tq.Handle(d, 1, 0, qjl_m=128)
    cache = tq.Cache(h, B, Hkv, L)
    g = torch.Generator(device="cuda").manual_seed(10)
    enc_ms = _encode_into(tq, h, cache, lambda l0, n: torch.randn(B, Hkv, n, d, generator=g, device="cuda")
                          .to(torch.bfloat16), L, 2048, torch)
    gq = torch.Generator(device="cuda").manual_seed(11)
    W, T = args.warmup, args.steps
    qs = torch.randn(T + W, B, Hq, d, generator=gq, device="cuda")
    q_in = qs[0].clone()
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, Hq, L, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_score_workspace_bytes(h.ptr, B, Hq), dtype=torch.uint8, device="cuda")

    def step():
        tq.tq_score(h.ptr, q_in, B, Hq, Hkv, cache.struct, lens, logits, ws)

    s_ = torch.cuda.Stream()
    s_.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_):
        step()
    torch.cuda.current_stream().wait_stream(s_)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    tq.tq_timer_read(None, forget=True)
    tq.tq_timer_enable(True)
    graph_k = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_k):
        step()
    tq.tq_timer_enable(False)
    for t in range(W):
        q_in.copy_(qs[t])
        graph.replay()
    torch.cuda.synchronize()
    sampler = bench.ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    sampler.start()
    evs = []
    for t in range(T):
        q_in.copy_(qs[W + t])
        ev = _events(torch)
        ev[0].record()
        graph.replay()
        ev[1].record()
        evs.append(ev)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    total_ms = sum(a.elapsed_time(b) for a, b in evs)
    sc_ms, sc_n = 0.0, 0
    for t in range(T):
        q_in.copy_(qs[W + t])
        graph_k.replay()
        torch.cuda.synchronize()
        ms_k, n_k = tq.tq_timer_read("score", forget=False)
        sc_ms += ms_k
        sc_n += n_k
    _, kernels_per_step = tq.tq_timer_read(None, forget=False)
    keys = B * Hkv * L
    row = h.codes_B + h.signs_B + (4 if h.norm_dtype == tq.TQ_F32 else 2)
    # fp32 flops the kernel's arithmetic needs per (key, query head): polar, a product and an FMA
    # per fold of the d - 1 tree nodes above the level-1 table lookups; QJL-only, an FMA per sign
    flops_per = (4 * (d // 2 - 1) + 2) if kind == "polar" else 2 * 128
    flops = keys * G * flops_per
    sm_mhz = clocks.get("sm_mhz") or 1965.0
    peak = torch.cuda.get_device_properties(0).multi_processor_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12
    launch_ms = sc_ms / max(sc_n, 1)
    ach = flops / (launch_ms / 1e3) / 1e12
    name = {"polar": "recursive polar transform (PolarQuant), d=128, 4 bits at level 1 and 2 bits at levels 2-7 "
                     "(2.98 bits per coordinate)",
            "qjl": "QJL-only 1-bit keys (128 sign bits + fp16 norm), d=128"}[kind]
    cfg = {"workload": f"scores of 4 query heads per KV head over {name}; {B} sequences x 8 KV heads x 16384 keys",
           "B": B, "Hkv": Hkv, "Hq": Hq, "context": L, "d": d,
           "dtype": "f32 SIMT (per-query tables)" if kind == "polar" else "f32 SIMT",
           "l2": "not flushed: each step reads %.0f MB of packed keys and writes %.0f MB of logits"
                 % (keys * row / 1e6, keys * G * 4 / 1e6)}
    roof = {"bound": "alu", "kernel": "polar_score_kernel" if kind == "polar" else "score_simt_kernel",
            "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
            "peak_source": "derived: SMs x 128 fp32 lanes x 2 flop x median sampled SM clock",
            "launch_ms": launch_ms, "algorithmic_flops_per_launch": flops,
            "hbm_gbs_of_the_same_launch": (keys * row + keys * G * 4) / (launch_ms / 1e3) / 1e9}
    extra = {"keys_scored_per_s": keys * T / (total_ms / 1e3),
             "prefill_encode": {"vectors": keys, "ms": enc_ms, "vectors_per_s": keys / (enc_ms / 1e3)}}
    _line(args, f"keys scored/sec ({kind} keys)", extra["keys_scored_per_s"], "keys/s", total_ms / T, cfg, roof,
          kernels_per_step * T, clocks, extra, None)


# ------------------------------------------------------------------ the small MSE workload (cfg 1)

def _unpack_rows(codes, d, bits):
    """Indices of LSB-first packed rows (uint8 [n, B] numpy) -> int64 [n, d]."""
    import numpy as np
    stream = np.unpackbits(codes, axis=1, bitorder="little")[:, : d * bits].reshape(codes.shape[0], d, bits)
    return (stream.astype(np.int64) << np.arange(bits)).sum(axis=2)


def run_cfg1(args):
    """MSE-only 3-bit TurboQuant, d = 128: 4096 fp32 N(0,1) keys (seed 0) encoded, one N(0,1) query
    (seed 1) scored against all of them. Reports the index usage, norms, scores and the empirical
    distortion mean ||x - x_hat||^2 / ||x||^2 (x_hat rebuilt on the host from the GPU's codes with
    the handle's Pi and codebook); the CPU leg (the oracle) adds the near-boundary index mismatch
    fraction and the largest score difference."""
    import numpy as np
    import torch
    import embedding_vector_quantization_b200 as tq
    import workloads
    d, bits, n = 128, 3, 4096
    h = tq.Handle(d, bits, 0)
    x = workloads.mse_keys(n, d, seed=0)
    q = workloads.queries((1, 1, d), 1)
    xg = x.cuda()
    cache = tq.Cache(h, 1, 1, n)
    lens = torch.full((1,), n, dtype=torch.int32, device="cuda")
    ws = torch.empty(tq.tq_score_workspace_bytes(h.ptr, 1, 1), dtype=torch.uint8, device="cuda")
    logits = torch.zeros(1, 1, n, dtype=torch.float32, device="cuda")
    for _ in range(3):
        cache.fill(xg.view(1, 1, n, d))
        tq.score(h, q.cuda(), cache, lens, logits=logits, workspace=ws)
    torch.cuda.synchronize()
    reps = 20
    e_ms = s_ms = 0.0
    for _ in range(reps):
        a, b = _events(torch)
        a.record()
        cache.fill(xg.view(1, 1, n, d))
        b.record()
        c, e = _events(torch)
        c.record()
        tq.score(h, q.cuda(), cache, lens, logits=logits, workspace=ws)
        e.record()
        torch.cuda.synchronize()
        e_ms += a.elapsed_time(b)
        s_ms += c.elapsed_time(e)
    codes = cache.codes.cpu().numpy().reshape(n, -1)
    norms = cache.norms.cpu().numpy().reshape(n)
    scores = logits.cpu().numpy().reshape(n)
    idx = _unpack_rows(codes, d, bits)
    cent, _ = h.codebook()
    Pi, _ = h.rotation()
    xh = norms.astype(np.float64)[:, None] * (cent[idx] @ Pi)
    xd = x.double().numpy()
    dist = float(np.mean(np.sum((xd - xh) ** 2, axis=1) / np.sum(xd * xd, axis=1)))
    rec = {"workload": "MSE-only TurboQuant, d=128, b=3: 4096 fp32 N(0,1) keys (seed 0), 1 N(0,1) query (seed 1)",
           "encode_us": 1e3 * e_ms / reps, "score_us": 1e3 * s_ms / reps,
           "index_histogram": np.bincount(idx.ravel(), minlength=8).tolist(),
           "norms": {"mean": float(norms.mean()), "min": float(norms.min()), "max": float(norms.max())},
           "scores": {"first": [float(v) for v in scores[:4]], "mean": float(scores.mean()),
                      "std": float(scores.std())},
           "empirical_mse_distortion": dist,
           "expected_mse_distortion": "d * MSE(3 bits, d = 128) = 0.0340 (the Lloyd-Max codebook's own MSE)"}
    if not args.no_cpu_baseline:
        from oracle import codebook, ops, quant, rotation
        t0 = time.perf_counter()
        Pio, _ = rotation.rotation(d, 0)
        co, bo = codebook.lloyd_max(d, bits)
        eo = quant.encode_mse(xd, Pio, co, bo, "f32")
        so = ops.score_mse(q.double().numpy().reshape(d), eo["idx"], eo["n_stored"], Pio, co)
        el = time.perf_counter() - t0
        mism = idx != eo["idx"]
        near = np.abs(eo["y"][mism] - bo[np.minimum(idx[mism], eo["idx"][mism])]) if mism.any() else np.zeros(0)
        # scores against the oracle scoring the GPU's own codes (the parity rule), and end to end
        # against the oracle's own encode (a code inside the 1e-5 band moves its key's score a step)
        sg = ops.score_mse(q.double().numpy().reshape(d), idx, norms.astype(np.float64), Pio, co)
        floor = np.linalg.norm(q.double().numpy()) * norms.astype(np.float64) / np.sqrt(d)
        rec["oracle"] = {"index_mismatch_fraction": float(mism.mean()),
                         "mismatches_within_1e-5_of_a_boundary": bool(np.all(near < 1e-5)),
                         "max_score_error_on_gpu_codes_rel_to_floor": float(np.max(np.abs(scores - sg) / floor)),
                         "max_abs_score_difference_end_to_end": float(np.max(np.abs(scores - so))),
                         "oracle_seconds": el, "kind": "oracle", "cores": bench.blas_threads()}
        # the same keys through the 3-bit prod encode (2-bit codes + 128 QJL signs, fp16 norms; the
        # tensor-core encode at d = 128): index and sign mismatch fractions against the oracle's
        # encode. An index may differ only within 1e-5 of a boundary, a sign only for a projection
        # within 1e-5 ||x|| of zero (or in a row whose index differs, which moves the residual).
        hp = tq.Handle(d, 3, 0, qjl_m=128)
        pc = tq.Cache(hp, 1, 1, n)
        pc.fill(xg.view(1, 1, n, d))
        torch.cuda.synchronize()
        pidx = _unpack_rows(pc.codes.cpu().numpy().reshape(n, -1), d, 2)
        psig = np.unpackbits(pc.signs.cpu().numpy().reshape(n, -1), axis=1, bitorder="little")[:, :128]
        Pip, Sp = rotation.rotation(d, 0, 128)
        cp_, bp_ = codebook.lloyd_max(d, 2)
        ep = quant.encode_prod(xd, Pip, Sp, cp_, bp_, "f16")
        imis = pidx != ep["idx"]
        inear = (np.abs(ep["y"][imis] - bp_[np.minimum(pidx[imis], ep["idx"][imis])])
                 if imis.any() else np.zeros(0))
        smis = psig.astype(np.int64) != ep["sigma"]
        smis[np.any(imis, axis=1)] = False
        r_, j_ = np.nonzero(smis)
        snear = np.abs(ep["z"][r_, j_]) < 1e-5 * ep["n_exact"][r_]
        rec["oracle"]["prod_3bit"] = {"index_mismatch_fraction": float(imis.mean()),
                                      "index_mismatches_within_1e-5_of_a_boundary": bool(np.all(inear < 1e-5)),
                                      "sign_mismatch_fraction": float(smis.mean()),
                                      "sign_mismatches_within_1e-5_of_zero": bool(np.all(snear))}
    if COLLECT is not None:
        COLLECT.append({"metric": "cfg1", "record": rec})
    else:
        print(json.dumps({"metric": "MSE-only 3-bit encode + score record (cfg 1)", "record": rec}), flush=True)


def collect_rows(args, rows=("cfg1", "score", "encode", "attn4", "attn3big", "search", "search4", "polar", "qjl")):
    """Runs every other hot-path row with a few steps and returns {row: its line}. The rows'
    own CPU baselines are skipped (the cfg-1 record keeps its oracle check)."""
    import copy
    global COLLECT
    out = {}
    fns = {"cfg1": run_cfg1, "score": run_score, "encode": run_encode, "attn4": run_attn4, "attn3big": run_attn3big,
           "search": lambda a: run_search(a, bits=2), "search4": lambda a: run_search(a, bits=4),
           "polar": lambda a: run_score_kind(a, "polar"), "qjl": lambda a: run_score_kind(a, "qjl")}
    for name in rows:
        a = copy.copy(args)
        a.steps, a.warmup, a.small = 10, 3, False
        a.no_cpu_baseline = name != "cfg1" or args.no_cpu_baseline
        COLLECT = []
        try:
            fns[name](a)
            line = COLLECT[-1] if COLLECT else {"error": "no line"}
        except Exception as exc:   # a row that fails is reported, the headline line still prints
            line = {"error": f"{type(exc).__name__}: {exc}"}
        finally:
            COLLECT = None
        out[name] = line
        import torch
        torch.cuda.empty_cache()
    return out


def run(args):
    if args.workload == "compare":
        run_compare(args)
        return
    if args.workload == "search4":
        run_search(args, bits=4)
        return
    {"score": run_score, "encode": run_encode, "attn4": run_attn4, "attn3big": run_attn3big,
     "search": run_search, "cfg1": run_cfg1, "polar": lambda a: run_score_kind(a, "polar"),
     "qjl": lambda a: run_score_kind(a, "qjl")}[args.workload](args)
