#!/usr/bin/env python
"""Benchmark of the quantized-KV decode path on B200 (one JSON line on rank 0).

Workload (3-bit prod TurboQuant, d = 128): one GQA decode step over a
compressed cache -- batch 1, 8 KV heads, 32 query heads, context 32768, K and V
each 2-bit Lloyd-Max MSE + 1-bit QJL sketch (m = 128), fp16 norms and residual
norms; bf16 K/V with per-(head, channel) std ~ LogNormal(0, 0.5) and 2 outlier
channels x10 per head. A step is the whole hot path for one new token, one
tq_decode_step call: append of the new key and value (norm, rotate, bucketize,
pack, QJL sign-pack) together with the query rotation, then scores, online
softmax and value accumulate, then the combine that also advances len. The
step is captured once in a CUDA graph; each timed step replays it. `len` is reset between steps (outside the timed
bracket) so every step attends over exactly 32768 tokens; L2 is flushed
between steps (the packed cache, 27 MB, would otherwise sit in the 126 MB L2).

value   = packed K+V bytes read by the attention per step / device time per step (GB/s)
e2e     = same metric through the C ABI with host buffers: per step one CUDA
          graph copies the new token and the queries (one block) from a pinned
          staging buffer, runs the step and copies the attention output back to
          pinned memory, all inside the timed bracket; the host fills the
          staging buffer between steps.
rows    = (N = 1, unless --no-rows) every other hot-path row measured after the headline's
          timed region with a few steps each and folded into the same line: the cfg-1 encode
          + score record, the streaming score step, the prefill encode, the 4-bit decode step,
          the 3-bit decode step over an HBM-sized cache, the 2- and 4-bit searches, and the
          scores over polar-transform and QJL-only keys.
Multi-GPU (--gpus N under torchrun): every rank runs its own independent
instance of the workload (weak scaling, no collective on the data path); the
reported time is the max over ranks.
"""

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed-KV GB/s and keys scored/sec (3-bit, d=128) vs HBM roofline; vectors encoded/sec"
W = dict(B=1, Hkv=8, Hq=32, L=32768, d=128, bits=3, m=128, seed_k_handle=0, seed_v_handle=1,
         seed_k=2, seed_v=3, seed_q=4)
PACKED_BYTES_PER_TOKEN = 2 * (32 + 16 + 2 + 2)   # K and V: 2-bit codes + sign bits + fp16 norm + fp16 rnorm
WORKLOAD_NAME = ("GQA decode step, TurboQuant prod 3-bit (2-bit Lloyd-Max + 1-bit QJL m=128), d=128, "
                 "B=1, 8 KV heads / 32 query heads, context 32768, bf16 K/V with lognormal channel scales "
                 "and 2 outlier channels")
# Arithmetic of the timed path: int8 x int8 -> int32 tensor-core MMAs on fixed-point queries (22-bit
# against the codes, 15-bit against the QJL signs) and 16-bit fixed-point softmax weights, fp32
# softmax, combine and output.
DTYPE = "s8xs8->s32 MMA (22/15-bit fixed-point queries, 16-bit weights), f32 softmax/combine"
FALLBACK_HBM_GBS = 6650.0
# DRAM bytes (read + write) of one attn_prod2_kernel launch on this workload, from
# `ncu --set full` (the attention kernel's profile summary in the repository); set to None whenever
# that kernel changes until it is captured again.
ATTN_TRAFFIC_BYTES = 27_368_192


def decode_config(world):
    """The `config` object of the decode-step line (identical in both arms)."""
    return {"workload": WORKLOAD_NAME, "B": W["B"], "Hkv": W["Hkv"], "Hq": W["Hq"], "context": W["L"],
            "d": W["d"], "bits": "2 MSE + 1 QJL (m=128)", "l2": "flushed between steps (256 MB write)",
            "step": "tq_decode_step (append K and V, rotate q, attend, advance len), one CUDA graph replay",
            "parallelism": f"independent replica per GPU x{world}"}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["tq", "reference"], default="tq")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--workload", choices=["decode", "score", "encode", "attn4", "attn3big", "search", "search4",
                                          "compare", "cfg1", "polar", "qjl"],
                   default="decode",
                   help="decode: the headline decode step (default); the others measure the remaining hot-path "
                        "rows on their own workloads, one JSON line each (attn3big: the 3-bit decode step over a "
                        "64 x 8 x 16384-token cache; search: 2-bit codes, search4: 4-bit; "
                        "compare: the cfg-2 attention against uncompressed bf16 / fp32 K/V)")
    p.add_argument("--no-rows", action="store_true",
                   help="decode only: skip the other hot-path rows that the default run folds into its line")
    p.add_argument("--small", action="store_true",
                   help="row workloads only: a reduced size (still above the 126 MB L2, a few hundred MB in "
                        "all) for profiler captures; the numbers of such a run are not bench values")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for name, val in zip(names, f[3:7]):
                if val.lower() in ("active", "1", "yes"):
                    reasons.add(name)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------- oracle (CPU) leg

class OracleSample:
    """The CPU oracle on a bounded sample of the same workload: `group_heads` KV head(s)
    of the decode step (encode of the new K and V token, then attention of the group's
    4 query heads over 32768 cached tokens). Setup (the prefill encode) is untimed."""

    def __init__(self, group_heads=1):
        import numpy as np
        import workloads as synth
        from oracle import codebook, ops, quant, rotation
        self.np, self.ops, self.quant = np, ops, quant
        d, m, L = W["d"], W["m"], W["L"]
        G = W["Hq"] // W["Hkv"]
        self.gh, self.d, self.m, self.L = group_heads, d, m, L
        self.P = [rotation.rotation(d, W["seed_k_handle"], m), rotation.rotation(d, W["seed_v_handle"], m)]
        self.c, self.beta = codebook.lloyd_max(d, W["bits"] - 1)
        self.X = [synth.outlier_kv(seed=W["seed_k"])[:, :group_heads].double().numpy(),
                  synth.outlier_kv(seed=W["seed_v"])[:, :group_heads].double().numpy()]
        self.q = synth.queries((1, W["Hq"], d), W["seed_q"]).double().numpy()[:, : G * group_heads]
        self.caches = [self._encode(self.X[i][:, :, : L - 1], *self.P[i]) for i in range(2)]

    def _encode(self, x, P, S):
        e = self.quant.encode_prod(x.reshape(-1, self.d), P, S, self.c, self.beta, "f16")
        sh = (1, self.gh, x.shape[2])
        return {"idx": e["idx"].reshape(sh + (self.d,)), "n": e["n_stored"].reshape(sh),
                "sigma": e["sigma"].reshape(sh + (self.m,)), "rnorm": e["rnorm_stored"].reshape(sh),
                "Pi": P, "S": S, "c": self.c}

    def step(self):
        """One decode step; returns the packed bytes the attention reads."""
        full = []
        for i in range(2):
            new = self._encode(self.X[i][:, :, self.L - 1:self.L], *self.P[i])
            f = dict(self.caches[i])
            for key in ("idx", "n", "sigma", "rnorm"):
                f[key] = self.np.concatenate([self.caches[i][key], new[key]], axis=2)
            full.append(f)
        self.ops.decode_attention(self.q, full[0], full[1], [self.L], 1.0 / self.np.sqrt(self.d))
        return self.L * PACKED_BYTES_PER_TOKEN * self.gh


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def oracle_decode_sample(budget_s=12.0):
    """Times OracleSample.step repeatedly for about `budget_s` seconds: (GB/s, seconds, steps, threads)."""
    s = OracleSample()
    s.step()
    reps, nbytes, t0 = 0, 0, time.perf_counter()
    while True:
        nbytes += s.step()
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return nbytes / el / 1e9, el, reps, blas_threads()


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = OracleSample()
    for _ in range(args.warmup):
        s.step()
    t_total, nbytes = 0.0, 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        nbytes += s.step()
        t_total += time.perf_counter() - t0
    value = nbytes / t_total / 1e9 if t_total > 0 else 0.0
    threads = blas_threads()
    sample = "each step: 1 of 8 KV-head groups (new-token encode + attention of 4 query heads over 32768 tokens)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- GPU leg

def run_tq(args):
    import torch
    import torch.distributed as dist
    import embedding_vector_quantization_b200 as tq
    from embedding_vector_quantization_b200 import dist as tqdist
    import workloads as synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    B, Hkv, Hq, L, d, m = W["B"], W["Hkv"], W["Hq"], W["L"], W["d"], W["m"]
    L0 = L - 1                                            # prefill; each step appends token L0 -> context L
    hk = tq.Handle(d, W["bits"], W["seed_k_handle"], qjl_m=m)
    hv = tq.Handle(d, W["bits"], W["seed_v_handle"], qjl_m=m)
    K = synth.outlier_kv(seed=W["seed_k"] + 100 * rank).to(dev)
    V = synth.outlier_kv(seed=W["seed_v"] + 100 * rank).to(dev)
    kc, vc = tq.Cache(hk, B, Hkv, L, dev), tq.Cache(hv, B, Hkv, L, dev)
    kc.fill(K[:, :, :L0])
    vc.fill(V[:, :, :L0])
    lens = torch.full((B,), L0, dtype=torch.int32, device=dev)

    n_tok = max(args.steps, 1) + args.warmup
    g = torch.Generator().manual_seed(W["seed_q"] + 100 * rank)
    q_all = torch.randn(n_tok, B, Hq, d, generator=g).to(dev)
    k_all = K[:, :, L0].unsqueeze(0).expand(n_tok, B, Hkv, d).contiguous()   # the workload's token 32768
    v_all = V[:, :, L0].unsqueeze(0).expand(n_tok, B, Hkv, d).contiguous()
    # the step's inputs live in one device block (query, new key, new value), so that the end-to-end
    # path moves them from pinned host memory in one copy
    qb, kb = q_all[0].numel() * 4, k_all[0].numel() * 2
    in_dev = torch.empty(qb + 2 * kb, dtype=torch.uint8, device=dev)
    q_in = in_dev[:qb].view(torch.float32).view(q_all[0].shape)
    k_in = in_dev[qb:qb + kb].view(torch.bfloat16).view(k_all[0].shape)
    v_in = in_dev[qb + kb:].view(torch.bfloat16).view(v_all[0].shape)
    q_in.copy_(q_all[0])
    k_in.copy_(k_all[0])
    v_in.copy_(v_all[0])
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L), dtype=torch.uint8, device=dev)
    scale = 1.0 / (d ** 0.5)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)   # 2x the 126 MB L2

    def step():   # append the new key and value of every head at slot len[b], attend over len[b] + 1 tokens
        tq.tq_decode_step(hk.ptr, hv.ptr, q_in, k_in, v_in, B, Hq, Hkv, kc.struct, vc.struct, lens, scale, out, ws)

    # eager warm-up (sets kernel attributes), then capture the step with kernel timers inside
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            step()
            lens.fill_(L0)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    # two captures of the same step: `graph` (timed, nothing but the step's kernels) and
    # `graph_k` (the same with an event pair around every kernel, for the per-kernel split)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    tq.tq_timer_read(None, forget=True)
    tq.tq_timer_enable(True)
    graph_k = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_k):
        step()
    tq.tq_timer_enable(False)
    lens.fill_(L0)
    graph_k.replay()                    # the captured event pairs exist only after a replay
    lens.fill_(L0)
    torch.cuda.synchronize()
    _, kernels_per_step = tq.tq_timer_read(None, forget=False)

    def set_inputs(t):
        q_in.copy_(q_all[t])
        k_in.copy_(k_all[t])
        v_in.copy_(v_all[t])

    for t in range(args.warmup):
        set_inputs(t)
        flush.zero_()
        graph.replay()
        lens.fill_(L0)
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    split_ms, split_n = 0.0, 0
    names = ("prologue", "attn_split", "attn_combine")
    kern_ms = {k: 0.0 for k in names}
    for i in range(args.steps):
        set_inputs(args.warmup + i)
        flush.zero_()
        evs[i][0].record()
        graph.replay()
        evs[i][1].record()
        lens.fill_(L0)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    step_ms = [a.elapsed_time(b) for a, b in evs]
    # per-kernel device time: the same steps replayed through the instrumented capture
    for i in range(args.steps):
        set_inputs(args.warmup + i)
        flush.zero_()
        graph_k.replay()
        lens.fill_(L0)
        torch.cuda.synchronize()                # captured event pairs are re-recorded by every replay
        for k in names:
            ms_k, n_k = tq.tq_timer_read(k, forget=False)
            kern_ms[k] += ms_k
            if k == "attn_split":
                split_ms += ms_k
                split_n += n_k
    max_ms = tqdist.max_over_ranks(sum(step_ms))   # the job's time: the slowest rank

    # --- end to end through the C ABI with host buffers (pinned), same workload
    in_h = torch.empty(n_tok, in_dev.numel(), dtype=torch.uint8).pin_memory()   # [step][query | key | value]
    in_h[:, :qb].view(torch.float32).copy_(q_all.cpu().reshape(n_tok, -1))
    in_h[:, qb:qb + kb].view(torch.bfloat16).copy_(k_all.cpu().reshape(n_tok, -1))
    in_h[:, qb + kb:].view(torch.bfloat16).copy_(v_all.cpu().reshape(n_tok, -1))
    o_h = torch.empty(args.steps, B, Hq, d, dtype=torch.float32)
    # one graph per step: the copy of the step's inputs from a pinned staging buffer, the step's
    # kernels and the copy of the output to pinned host memory
    stage_h = torch.empty(in_dev.numel(), dtype=torch.uint8).pin_memory()
    out_h = torch.empty(B, Hq, d, dtype=torch.float32).pin_memory()
    graph_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        stage_h.copy_(in_h[0])
        for _ in range(2):
            in_dev.copy_(stage_h, non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
            lens.fill_(L0)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph_e2e):
        in_dev.copy_(stage_h, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
    lens.fill_(L0)
    torch.cuda.synchronize()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        stage_h.copy_(in_h[args.warmup + i])   # the host places the step's inputs (outside the bracket)
        flush.zero_()
        e2e_ev[i][0].record()
        graph_e2e.replay()
        e2e_ev[i][1].record()
        lens.fill_(L0)
        torch.cuda.synchronize()               # the output is in out_h; the staging buffer is free again
        o_h[i].copy_(out_h)
    del graph_e2e
    e2e_ms = tqdist.max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev))
    h2d = (q_in.numel() * 4 + k_in.numel() * 2 + v_in.numel() * 2)
    d2h = out.numel() * 4

    # --- encode throughput (vectors encoded / s): prefill encode of the K and V caches
    enc_ms = 0.0
    reps = 5
    for r in range(reps + 1):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        tq.tq_encode(hk.ptr, K, B * Hkv * L, kc.codes, kc.signs, kc.norms, kc.rnorms)
        tq.tq_encode(hv.ptr, V, B * Hkv * L, vc.codes, vc.signs, vc.norms, vc.rnorms)
        b.record()
        torch.cuda.synchronize()
        if r:
            enc_ms += a.elapsed_time(b)
    enc_vectors = 2 * B * Hkv * L
    enc_vps = enc_vectors * reps / (enc_ms / 1e3)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    del graph, graph_k
    tokens = B * Hkv * L                               # key (and value) rows read per step per rank
    bytes_step = tokens * PACKED_BYTES_PER_TOKEN
    value = world * bytes_step * args.steps / (max_ms / 1e3) / 1e9
    keys_s = world * tokens * args.steps / (max_ms / 1e3)
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    split_avg_ms = split_ms / max(split_n, 1)
    achieved = bytes_step / (split_avg_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
        "config": decode_config(world),
        "keys_scored_per_s": keys_s,
        "query_key_pairs_per_s": keys_s * (Hq // Hkv),
        "vectors_encoded_per_s": enc_vps,
        "encode": {"vectors": enc_vectors, "ms_per_pass": enc_ms / reps, "input": "bf16 K and V prefill"},
        "hbm_frac_nominal_8tbs": value / world / 8000.0,
        "roofline": {"bound": "hbm", "kernel": "attn_split", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": ATTN_TRAFFIC_BYTES,
                     "peak_source": f"{peak_src} hbm_gbs", "launch_ms": split_avg_ms,
                     "algorithmic_bytes_per_launch": bytes_step},
        "e2e": {"value": world * bytes_step * args.steps / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps},
        "kernel_us_per_step": {k: round(1e3 * v / args.steps, 3) for k, v in kern_ms.items()},
        "gpu_launches": kernels_per_step * args.steps,
        "kernels_per_step": kernels_per_step,
        "clocks": clocks,
    }
    if world == 1 and not args.no_rows:
        # every other hot-path row, a few steps each, after the headline's timed region
        import bench_rows
        line["rows"] = bench_rows.collect_rows(args)
    if world == 1 and not args.no_cpu_baseline:
        gbs, el, reps_c, threads = oracle_decode_sample()
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{reps_c} decode steps of 1 of 8 KV-head groups (4 query heads, "
                                          f"32768 tokens) in {el:.1f} s, fp64 NumPy oracle"}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "decode":
        run_tq(args)
    else:
        import bench_rows
        bench_rows.run(args)


if __name__ == "__main__":
    main()
