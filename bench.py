"""Prefill throughput of one Qwen3-VL decoder layer on B200, as one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the MRoPE position
ids (P0) and one decoder layer (P1..P9) through the C ABI. The default
workload is the Qwen3-VL-4B-shape layer at S = 4096 with a 32x24 image span
and Q/K/V bias (bf16, random weights, synthetic input). Its working set
(weights ~200 MB, activations ~180 MB) exceeds the 126 MB L2, so no flush is
needed between steps.

  value     tokens/s per layer, inputs resident in HBM, CUDA events on the
            launching stream, max over ranks;
  e2e       the same through the public API with host buffers: pinned x and
            token types copied in, x' copied out, every step (uploads and
            downloads on their own streams, overlapping other steps' kernels);
  roofline  the dominant kernel (gate/up GEMM with SiLU*up epilogue), timed
            live by stage events the library records inside the timed steps;
  cpu_baseline the CPU oracle (fp32 NumPy) on a bounded sample.

With N > 1 (torchrun) every rank runs an independent replica on its own GPU
(the layer does not shard across GPUs here): weak scaling, no collective on
the data path. --impl reference times the CPU oracle itself on the host.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import q3vl_synth as syn  # noqa: E402

METRIC = "prefill tokens/s per layer (bf16, 1xB200); % of BF16 tensor peak and HBM BW"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gate_up_traffic.json")
GEMM_SRC = os.path.join(ROOT, "qwen3_vl_decoder_b200", "csrc", "gemm_tc.cu")
STAGES = ["table", "rms1", "qkv", "attention", "o_proj", "rms2", "gate_up", "down"]
CPU_SAMPLE_TOKENS = 512


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=syn.Q4B_LAYER.name, choices=sorted(syn.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the one-token decode measurement of the 36-layer stack")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode measurement and print its JSON (for profiling)")
    ap.add_argument("--decode-batches", default="1,32",
                    help="comma-separated decode batch sizes")
    ap.add_argument("--decode-layers", type=int, default=36,
                    help="layers of the decode stack (36 = the 4B shape)")
    return ap.parse_args()


def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE {world}")
    return rank, world, local


def layer_flops(w, S=None):
    """Algorithmic FLOPs of one layer: GEMMs plus causal attention (S(S+1)/2 pairs)."""
    S = w.seq if S is None else S
    H, Dq, Dkv, I = w.hidden, w.q_dim, w.kv_dim, w.intermediate
    gemm = 2 * S * H * (Dq + 2 * Dkv) + 2 * S * Dq * H + 4 * S * H * I + 2 * S * I * H
    attn = 4 * w.n_heads * 128 * S * (S + 1) // 2
    return gemm, attn


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, 6650.0, "fallback"


def src_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for_current_kernel():
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        if t.get("gemm_tc_sha") == src_hash(GEMM_SRC):
            return t.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows]
        smax = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Not" not in v
                          and v.strip() not in ("", "[N/A]")})
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


def setup(w, dev):
    import qwen3_vl_decoder_b200 as q3
    cfg = q3.config_of(w)
    raw = syn.layer_weights(w, 0)
    packed = q3.pack_layer(cfg, {k: v.to(dev) for k, v in raw.items()})
    del raw
    st = {"q3": q3, "cfg": cfg, "packed": packed}
    st["x_host"] = syn.hidden_input(w).pin_memory()
    st["x"] = st["x_host"].to(dev)
    st["tt_host"] = torch.tensor(syn.token_types(w), dtype=torch.uint8).pin_memory()
    st["tt"] = st["tt_host"].to(dev)
    g = syn.grids(w)
    st["g_host"] = torch.tensor(g, dtype=torch.int32).reshape(-1, 3).pin_memory() if g else None
    st["g"] = st["g_host"].to(dev) if g else None
    st["slab"] = st["rows"] = None
    if w.images and w.deepstack_layers:
        st["slab"] = syn.deepstack_slabs(w)[0].to(dev)
        st["rows"] = torch.tensor(syn.image_rows(w), dtype=torch.int32, device=dev)
    st["ws"] = q3.workspace(cfg, w.seq, dev)
    st["out_host"] = torch.empty_like(st["x_host"]).pin_memory()
    torch.cuda.synchronize()
    return st


def device_step(st, events=None):
    q3 = st["q3"]
    pos, _ = q3.mrope_positions(st["tt"], st["g"], check=False)
    if events is not None:
        q3.set_stage_events(events)
    q3.layer_prefill(st["cfg"], st["packed"], st["x"], pos, st["slab"], st["rows"], st["ws"])


class E2EPipeline:
    """End-to-end steps through the public API with host buffers.

    Every step copies its inputs (x, token types, grids) from pinned host
    memory to the device, runs P0..P9, and copies x' back to pinned host
    memory. Uploads, compute and downloads run on three streams with
    double-buffered device inputs, so step k+1's upload and step k-1's
    download overlap step k's kernels, as a serving loop would.
    """

    def __init__(self, st, dev):
        self.st = st
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.current_stream(dev)
        self.x = [st["x"], torch.empty_like(st["x"])]
        self.tt = [st["tt"], torch.empty_like(st["tt"])]
        self.g = [st["g"], None if st["g"] is None else torch.empty_like(st["g"])]
        self.out = [st["out_host"], torch.empty_like(st["out_host"]).pin_memory()]
        self.in_done = [torch.cuda.Event() for _ in range(2)]
        self.comp_done = [torch.cuda.Event() for _ in range(2)]
        self.out_done = [torch.cuda.Event() for _ in range(2)]
        self.started = [False, False]

    def step(self, k):
        st, q3, b = self.st, self.st["q3"], k % 2
        with torch.cuda.stream(self.s_in):
            if self.started[b]:
                self.s_in.wait_event(self.out_done[b])   # x[b] was read by its download
            self.x[b].copy_(st["x_host"], non_blocking=True)
            self.tt[b].copy_(st["tt_host"], non_blocking=True)
            if self.g[b] is not None:
                self.g[b].copy_(st["g_host"], non_blocking=True)
            self.in_done[b].record(self.s_in)
        self.s_comp.wait_event(self.in_done[b])
        pos, _ = q3.mrope_positions(self.tt[b], self.g[b], check=False, stream=self.s_comp)
        q3.layer_prefill(st["cfg"], st["packed"], self.x[b], pos, st["slab"], st["rows"], st["ws"],
                         stream=self.s_comp)
        self.comp_done[b].record(self.s_comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.comp_done[b])
            self.out[b].copy_(self.x[b], non_blocking=True)
            self.out_done[b].record(self.s_out)
        self.started[b] = True

    def finish(self):
        self.s_comp.wait_stream(self.s_in)
        self.s_comp.wait_stream(self.s_out)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(v, world, dev):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def timed(fn, steps, world, dev):
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(steps):
        fn(k)
    b.record()
    barrier(world)
    return max_over_ranks(a.elapsed_time(b) / 1e3, world, dev)


def cpu_oracle_rate(w, seconds=10.0, min_reps=1, max_reps=1000, reps=None,
                    tokens=CPU_SAMPLE_TOKENS):
    """tokens/s of the fp32 NumPy oracle on the first `tokens` tokens of w."""
    from oracle import q3vl_oracle as O
    n = min(tokens, w.seq)
    ws = w.with_seq(n, images=tuple(im for im in w.images if im[0] + im[1] * im[2] <= n))
    raw = syn.layer_weights(ws, 0)
    x = syn.hidden_input(ws).float().numpy()
    pos, _ = O.mrope_positions_tokens(syn.token_types(ws), syn.grids(ws))
    cfg = O.Config.of(ws)
    W = {k: v.float().numpy() for k, v in raw.items()}
    times = []
    t_end = time.perf_counter() + seconds
    while True:
        t0 = time.perf_counter()
        O.layer(cfg, W, x, pos, dtype=np.float32)
        times.append(time.perf_counter() - t0)
        if reps is not None:
            if len(times) >= reps:
                break
        elif (time.perf_counter() >= t_end and len(times) >= min_reps) or len(times) >= max_reps:
            break
    return n, times


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def reference_arm(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # size the per-step sample so that the whole run takes about a minute
    total = max(1, args.warmup) + max(1, args.steps)
    tokens = 64
    _, t64 = cpu_oracle_rate(w, reps=2, tokens=64)
    for cand in (128, 256, 512):
        if min(t64) * cand / 64 * total <= 90.0:
            tokens = cand
    n, warm = cpu_oracle_rate(w, reps=max(1, args.warmup), tokens=tokens)
    n, times = cpu_oracle_rate(w, reps=max(1, args.steps), tokens=tokens)
    total = sum(times)
    rate = n * len(times) / total
    sample = (f"first {n} tokens of {w.name} ({w.seq} tokens), one fp32 NumPy layer pass per "
              f"step, {len(times)} steps")
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "seq_len": w.seq, "sample_tokens": n},
            "cpu_baseline": {"value": rate, "unit": UNIT, "cores": cpu_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def decode_leg(dev, steps, warmup, batches=(1, 32), w=None):
    """One-token decode through the 36-layer 4B-shape stack after a 4096-row prompt.

    The prompt is prefilled into slot 0 of every layer's cache (q3vl_stack_prefill_kv)
    and copied to the other slots. One decode step (a static input copied into x, the
    36-layer q3vl_stack_decode, q3vl_decode_advance) is captured in a CUDA graph and
    replayed; the context grows by one row per step. Bytes per step are the packed
    projection weights of every layer plus each token's cache rows (K and V of all
    rows up to and including its own), which bound the step by HBM bandwidth.
    """
    import qwen3_vl_decoder_b200 as q3
    w = syn.Q4B_DECODE if w is None else w
    cfg = q3.config_of(w)
    layers = []
    for l in range(w.n_layers):
        raw = syn.layer_weights(w, l, device=dev)
        layers.append(q3.pack_layer(cfg, raw))
        del raw
    S, Bmax = w.seq, max(batches)
    cap = S + warmup + steps + 16
    kvs = q3.kv_caches(cfg, w.n_layers, n_seq=Bmax, cap=cap, device=dev)
    tt = torch.tensor(syn.token_types(w), dtype=torch.uint8, device=dev)
    g = syn.grids(w)
    gd = torch.tensor(g, dtype=torch.int32, device=dev).reshape(-1, 3)
    pos_p, nxt = q3.mrope_positions(tt, gd)
    q3.stack_prefill_kv(cfg, layers, syn.hidden_input(w, dev), pos_p, kvs, 0)
    for kv in kvs:
        kv.k[1:, :S].copy_(kv.k[0, :S].expand(Bmax - 1, -1, -1))
        kv.v[1:, :S].copy_(kv.v[0, :S].expand(Bmax - 1, -1, -1))
    q3.check_device()
    w_bytes = q3.packed_layer_bytes(cfg)
    dkv_bytes = 2 * 2 * w.n_kv_heads * w.head_dim          # K and V of one row, bf16
    out = {"workload": w.name, "prompt_rows": S, "layers": w.n_layers}
    burst, sustained, hbm, src = peaks()
    for B in batches:
        gen = torch.Generator(device=dev).manual_seed(17)
        x_in = torch.randn(B, w.hidden, generator=gen, device=dev).to(torch.bfloat16)
        x = torch.empty_like(x_in)
        seq = torch.arange(B, dtype=torch.int32, device=dev)
        ws = q3.decode_workspace(cfg, B, cap, dev)

        def reset():
            return (torch.full((3, B), nxt, dtype=torch.int32, device=dev),
                    torch.full((B,), S, dtype=torch.int32, device=dev))
        pos, lens = reset()

        def step():
            x.copy_(x_in)
            q3.stack_decode(cfg, layers, x, pos, kvs, seq, lens, None, ws)
            q3.decode_advance(pos, lens)
        n0 = q3.launch_count()
        step()
        launches = q3.launch_count() - n0
        torch.cuda.synchronize()
        p0, l0 = reset()
        pos.copy_(p0)
        lens.copy_(l0)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(warmup):
            graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(steps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        q3.check_device()
        assert torch.isfinite(x.float()).all(), "non-finite decode output"
        t = e0.elapsed_time(e1) / 1e3
        ctx_mean = S + warmup + (steps - 1) / 2.0          # rows cached before the token
        step_bytes = w.n_layers * (w_bytes + B * (ctx_mean + 1) * dkv_bytes)
        gbs = step_bytes * steps / t / 1e9
        out[f"B{B}"] = {"value": B * steps / t, "unit": "tokens/s", "batch": B,
                        "ms_per_step": 1e3 * t / steps,
                        "us_per_layer": 1e6 * t / steps / w.n_layers, "steps": steps,
                        "kernel_launches_per_step": launches,
                        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                     "frac": gbs / hbm, "bytes_per_step": step_bytes,
                                     "peak_source": f"{src} copy bandwidth"}}
        del graph
    del kvs, layers
    torch.cuda.empty_cache()
    # final norm + LM head of the decoded rows (tied: the embedding table is
    # the head), Qwen3-VL's vocabulary; bytes = the [vocab, H] bf16 weight
    vocab = 151936
    gen = torch.Generator(device=dev).manual_seed(23)
    table = (0.02 * torch.randn(vocab, w.hidden, generator=gen, device=dev)).to(torch.bfloat16)
    gain = (1.0 + 0.1 * torch.randn(w.hidden, generator=gen, device=dev)).to(torch.bfloat16)
    head = {}
    for B in batches:
        xr = torch.randn(B, w.hidden, generator=gen, device=dev).to(torch.bfloat16)
        logits = torch.empty((B, vocab), dtype=torch.float32, device=dev)
        hws = torch.empty(int(q3.lib().q3vl_lm_head_workspace_bytes(ctypes.byref(cfg), B)),
                          dtype=torch.uint8, device=dev)
        for _ in range(3):
            q3.lm_head(cfg, xr, gain, table, logits, hws)
        n = 50
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(n):
            q3.lm_head(cfg, xr, gain, table, logits, hws)
        e1.record()
        torch.cuda.synchronize()
        q3.check_device()
        t = e0.elapsed_time(e1) / 1e3 / n
        head_bytes = vocab * w.hidden * 2 + B * (w.hidden * 4 + vocab * 4)
        head[f"B{B}"] = {"us": 1e6 * t, "vocab": vocab,
                         "roofline": {"bound": "hbm", "achieved": head_bytes / t / 1e9, "peak": hbm,
                                      "unit": "GB/s", "frac": head_bytes / t / 1e9 / hbm}}
    out["lm_head"] = head
    del table
    torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    w = syn.WORKLOADS[args.workload]
    if w.n_layers != 1 or w.dtype != "bf16":
        w = w.with_layers(1)
    if args.impl == "reference":
        reference_arm(args, w)
        return
    if args.decode_only:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        batches = tuple(int(b) for b in args.decode_batches.split(","))
        out = decode_leg(dev, args.steps, max(3, args.warmup), batches,
                         syn.Q4B_DECODE.with_layers(args.decode_layers))
        print(json.dumps(out), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    st = setup(w, dev)
    q3 = st["q3"]
    S = w.seq

    # warm-up (also the first positions check)
    pos, nxt = q3.mrope_positions(st["tt"], st["g"])
    for _ in range(max(3, args.warmup)):
        device_step(st)
    q3.check_device()

    # device-resident timed region, with stage events inside every step
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    n0 = q3.launch_count()
    with ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else 0) as clk:
        t_dev = timed(lambda k: device_step(st, evs[k]), args.steps, world, dev)
    launches = q3.launch_count() - n0
    q3.set_stage_events(None)
    q3.check_device()
    stage_ms = {name: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1])
                                      for k in range(args.steps))
                for i, name in enumerate(STAGES)}

    # end-to-end through the public API with host buffers
    pipe = E2EPipeline(st, dev)
    for k in range(3):
        pipe.step(k)
    pipe.finish()

    def e2e_steps(k):
        if k == 0:   # the copy streams start after the timed region's start event
            pipe.s_in.wait_stream(pipe.s_comp)
            pipe.s_out.wait_stream(pipe.s_comp)
        pipe.step(k)
        if k == args.steps - 1:
            pipe.finish()   # the timed region ends after the last download

    t_e2e = timed(e2e_steps, args.steps, world, dev)
    q3.check_device()
    assert torch.isfinite(st["out_host"].float()).all(), "non-finite output"

    # a second workload for reference: the 2B-shape layer at S = 1024 (one GPU only)
    also = {}
    if world == 1 and args.workload != syn.Q2B_LAYER.name:
        w2 = syn.Q2B_LAYER
        st2 = setup(w2, dev)
        for _ in range(5):
            device_step(st2)
        n2 = max(50, args.steps // 2)
        t2 = timed(lambda k: device_step(st2), n2, world, dev)
        st2["q3"].check_device()
        g2, a2 = layer_flops(w2)
        also[w2.name] = {"value": w2.seq * n2 / t2, "unit": UNIT, "ms_per_step": 1e3 * t2 / n2,
                         "steps": n2, "tflops": (g2 + a2) * n2 / t2 / 1e12}
        del st2
        torch.cuda.empty_cache()

    decode = None
    if world == 1 and not args.no_decode:
        decode = decode_leg(dev, min(args.steps, 400), max(3, min(args.warmup, 20)),
                            tuple(int(b) for b in args.decode_batches.split(",")),
                            syn.Q4B_DECODE.with_layers(args.decode_layers))

    burst, sustained, hbm, src = peaks()
    gemm_f, attn_f = layer_flops(w)
    H, I = w.hidden, w.intermediate
    gu_flops = 4 * S * H * I
    gu_s = stage_ms["gate_up"] / 1e3
    achieved = gu_flops / gu_s / 1e12
    tc_s = sum(stage_ms[k] for k in ("qkv", "attention", "o_proj", "gate_up", "down")) / 1e3
    # P2 (the input row statistic) is the one standalone HBM pass of a bf16
    # layer: P7 is fused into the o-projection / gate-up epilogues.
    rms_bytes = S * H * 2 + S * 4
    rms_gbs = rms_bytes / (stage_ms["rms1"] / 1e3) / 1e9
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        n, times = cpu_oracle_rate(w, seconds=10.0)
        cpu = {"value": n * len(times) / sum(times), "unit": UNIT, "cores": cpu_cores(),
               "kind": "oracle",
               "sample": f"first {n} tokens of {w.name}, fp32 NumPy oracle layer, "
                         f"{len(times)} passes in {sum(times):.1f} s"}
    h2d = st["x_host"].numel() * 2 + st["tt_host"].numel() + \
        (st["g_host"].numel() * 4 if st["g_host"] is not None else 0)
    line = {
        "metric": METRIC, "value": world * S * args.steps / t_dev, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_dev / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded random-init weights N(0,0.02), gains 1+N(0,0.1), x N(0,1)",
        "config": {"workload": w.name, "seq_len": S, "global_batch": world,
                   "parallelism": f"replicas x{world}",
                   "l2": "working set larger than L2 (no flush)"},
        "roofline": {"bound": "tensor", "kernel": "gate_up GEMM + SiLU*up epilogue",
                     "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                     "frac": achieved / sustained,
                     "peak_source": f"{src} bf16 sustained (timed inside the layer step)",
                     "traffic": traffic_for_current_kernel(),
                     "flops_per_launch": gu_flops},
        "tensor_work": {"gemm_gflop": gemm_f / 1e9, "attn_gflop": attn_f / 1e9,
                        "tflops": (gemm_f + attn_f) / tc_s / 1e12,
                        "frac_of_sustained": (gemm_f + attn_f) / tc_s / 1e12 / sustained,
                        "frac_of_burst": (gemm_f + attn_f) / tc_s / 1e12 / burst},
        "hbm_passes": {"rms1_gbs": rms_gbs, "frac": rms_gbs / hbm, "peak_gbs": hbm,
                       "bytes": rms_bytes,
                       "note": "P2 input row statistic, timed with its launch gap; P7 fused "
                               "into the o-projection epilogue (no pass)"},
        "stages_ms": stage_ms,
        "cpu_baseline": cpu,
        "e2e": {"value": world * S * args.steps / t_e2e, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": st["out_host"].numel() * 2},
        "also": also,
        "decode": decode,
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "next_position": nxt,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
