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
            live by stage events the library records inside every 10th timed
            step (--stage-every); `kernels` has the same for every kernel;
  also      the 2B-shape layer, the 2B 28-layer stack and the 32B-shape
            50-layer encoder (S = 1064 and 8192), with the final-norm pass;
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
    ap.add_argument("--stage-every", type=int, default=10,
                    help="record the per-kernel stage events on every n-th timed step")
    ap.add_argument("--no-stacks", action="store_true",
                    help="skip the 2B 28-layer stack and 32B 50-layer encoder measurements")
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
    """SM clock, power and clock-event reasons sampled during the timed region.

    A child process (a fresh interpreter, not a fork of this CUDA process)
    polls NVML with read-only queries every half millisecond between
    __enter__ and __exit__, so even a timed region of a few tens of
    milliseconds gets samples: a thread of this process would wait for the
    interpreter lock while the timed loop launches and synchronises. Without
    NVML it falls back to nvidia-smi.
    """
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    POLLER = (
        "import signal, sys, time\n"
        "import pynvml\n"
        "signal.signal(signal.SIGTERM, lambda *a: (sys.stdout.flush(), sys.exit(0)))\n"
        "pynvml.nvmlInit()\n"
        "key, period = sys.argv[1], float(sys.argv[2])\n"
        "h = (pynvml.nvmlDeviceGetHandleByUUID(key) if key.startswith('GPU-')\n"
        "     else pynvml.nvmlDeviceGetHandleByIndex(int(key)))\n"
        "smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)\n"
        "print('ready', flush=True)\n"
        "k, pw = 0, 0.0\n"
        "while True:\n"
        "    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)\n"
        "    mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)\n"
        "    if k % 8 == 0:\n"
        "        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1e3\n"
        "    print(f'{sm},{smax},{mask},{pw}')\n"
        "    k += 1\n"
        "    time.sleep(period)\n")

    def __init__(self, dev, period_s=0.0005):
        self.dev = dev
        self.period = period_s
        self.samples = []      # (sm_mhz, sm_max_mhz, reason mask, power W)
        self.source = None
        self.proc = None
        self.lines = []
        self.out = ""

    def _key(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            return str(self.dev.index or 0)

    def __enter__(self):
        import threading
        self.reader = None
        try:
            import pynvml  # noqa: F401  (the child needs it)
            self.proc = subprocess.Popen(
                [sys.executable, "-c", self.POLLER, self._key(), str(self.period)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            if self.proc.stdout.readline().strip() != "ready":
                raise RuntimeError("NVML poller did not start")
            self.source = "nvml"
            # drain the pipe so the child never blocks on a full buffer
            self.reader = threading.Thread(
                target=lambda: self.lines.extend(self.proc.stdout), daemon=True)
            self.reader.start()
        except Exception:
            if self.proc is not None:
                self.proc.kill()
                self.proc.wait()
            self.proc = None
            self.source = "nvidia-smi"
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.dev.index or 0), f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                time.sleep(0.5)   # its first sample comes a moment after start
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        if self.source == "nvml":
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)
            for r in self.lines:
                f = r.strip().split(",")
                if len(f) == 4:
                    try:
                        self.samples.append((float(f[0]), float(f[1]), int(f[2]), float(f[3])))
                    except ValueError:
                        continue
            return
        self.proc.terminate()
        try:
            self.out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.out, _ = self.proc.communicate()
        for r in (self.out or "").strip().splitlines():
            f = r.split(",")
            if len(f) < 9:
                continue
            try:
                mask = sum(bit for (n, bit), v in zip(self.REASONS[:4], f[5:9])
                           if v.strip() not in ("", "[N/A]") and "Not" not in v)
                self.samples.append((float(f[1]), float(f[2]), mask, float(f[3] or 0)))
            except ValueError:
                continue

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"],
                    "source": self.source}
        sm = [s[0] for s in self.samples]
        smax = max(s[1] for s in self.samples)
        reasons = sorted({n for s in self.samples for n, bit in self.REASONS if s[2] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": smax,
                "reasons": reasons, "power_w_max": max(s[3] for s in self.samples),
                "samples": len(self.samples), "source": self.source}


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
    """P0 and one layer call; with `events` the library records the 9 stage
    boundaries of this call (and none when events is None)."""
    q3 = st["q3"]
    pos, _ = q3.mrope_positions(st["tt"], st["g"], check=False)
    if events is not None or st.get("events_on"):
        q3.set_stage_events(events)
        st["events_on"] = events is not None
    q3.layer_prefill(st["cfg"], st["packed"], st["x"], pos, st["slab"], st["rows"], st["ws"])


class E2EPipeline:
    """End-to-end steps through the public API with host buffers.

    Every step copies its inputs (x, token types, grids) from pinned host
    memory to the device, runs P0..P9, and copies x' back to pinned host
    memory. Uploads, compute and downloads run on three streams with
    triple-buffered device inputs, so step k+1's upload and step k-1's
    download overlap each other and step k's kernels, as a serving loop
    would (with two buffers, step k+1's upload would have to wait for step
    k-1's download of the same buffer).
    """

    NBUF = 3

    def __init__(self, st, dev):
        self.st = st
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.current_stream(dev)
        n = self.NBUF
        self.x = [st["x"]] + [torch.empty_like(st["x"]) for _ in range(n - 1)]
        self.tt = [st["tt"]] + [torch.empty_like(st["tt"]) for _ in range(n - 1)]
        self.g = [st["g"]] + [None if st["g"] is None else torch.empty_like(st["g"])
                              for _ in range(n - 1)]
        self.out = [st["out_host"]] + [torch.empty_like(st["out_host"]).pin_memory()
                                       for _ in range(n - 1)]
        self.in_done = [torch.cuda.Event() for _ in range(n)]
        self.comp_done = [torch.cuda.Event() for _ in range(n)]
        self.out_done = [torch.cuda.Event() for _ in range(n)]
        self.started = [False] * n

    def step(self, k):
        st, q3, b = self.st, self.st["q3"], k % self.NBUF
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


def stack_leg(w, dev, steps, warmup, final_norm_reps=50):
    """Whole-stack prefill of workload w (all its layers, DeepStack slabs and the
    final norm as the workload has them), weights drawn and packed on the device.
    Per-pass time from CUDA events around the stack call (x is restored from a
    copy between passes, outside the events)."""
    import qwen3_vl_decoder_b200 as q3
    cfg = q3.config_of(w)
    layers = []
    for l in range(w.n_layers):
        raw = syn.layer_weights(w, l, device=dev)
        layers.append(q3.pack_layer(cfg, raw))
        del raw
    tt = torch.tensor(syn.token_types(w), dtype=torch.uint8, device=dev)
    g = syn.grids(w)
    gd = torch.tensor(g, dtype=torch.int32, device=dev).reshape(-1, 3) if g else None
    pos, _ = q3.mrope_positions(tt, gd)
    slabs = [s.to(dev) for s in syn.deepstack_slabs(w)]
    rows = (torch.tensor(syn.image_rows(w), dtype=torch.int32, device=dev) if slabs else None)
    gain = syn.final_norm(w, dev)
    x0 = syn.hidden_input(w, dev)
    x = x0.clone()
    ws = q3.workspace(cfg, w.seq, dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for k in range(warmup + steps):
        x.copy_(x0)
        if k >= warmup:
            evs[k - warmup][0].record()
        q3.stack_prefill(cfg, layers, x, pos, gain, slabs, rows, ws)
        if k >= warmup:
            evs[k - warmup][1].record()
    torch.cuda.synchronize()
    q3.check_device()
    assert torch.isfinite(x.float()).all(), f"non-finite {w.name} output"
    t = statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3
    g_f, a_f = layer_flops(w)
    burst, sustained, hbm, src = peaks()
    tfl = (g_f + a_f) * w.n_layers / t / 1e12
    out = {"layers": w.n_layers, "seq_len": w.seq, "final_norm": gain is not None,
           "deepstack_slabs": len(slabs), "ms_per_stack": 1e3 * t, "steps": steps,
           "value": w.seq / t, "unit": "tokens/s",
           "layer_tokens_per_s": w.seq * w.n_layers / t,
           "tflops": tfl, "frac_of_burst": tfl / burst, "frac_of_sustained": tfl / sustained}
    if gain is not None:
        # P10 alone on the stack's output: [S, H] read and written once
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            q3.final_norm(cfg, x, gain)
        e0.record()
        for _ in range(final_norm_reps):
            q3.final_norm(cfg, x, gain)
        e1.record()
        torch.cuda.synchronize()
        q3.check_device()
        tn = e0.elapsed_time(e1) / 1e3 / final_norm_reps
        nb = 4 * w.seq * w.hidden + 2 * w.hidden
        out["final_norm_pass"] = {"us": 1e6 * tn, "bytes": nb,
                                  "roofline": {"bound": "hbm", "achieved": nb / tn / 1e9,
                                               "peak": hbm, "unit": "GB/s",
                                               "frac": nb / tn / 1e9 / hbm}}
    del layers, ws, x, x0
    torch.cuda.empty_cache()
    return out


def elementwise_leg(dev, hbm, rows=65536, reps=20):
    """The standalone row-statistic (P2) and final-norm (P10) kernels on a
    4B-width activation of `rows` rows (335 MB of bf16 at 65536), far larger
    than one layer call's 21 MB, where launch and ramp latency dominate: the
    kernels' own bandwidth. Bytes: P2 reads x and writes 1/rms; P10 reads x
    and the gain and writes x."""
    import qwen3_vl_decoder_b200 as q3
    w = syn.Q4B_LAYER
    cfg = q3.config_of(w)
    H = w.hidden
    g = torch.Generator(device=dev).manual_seed(5)
    x = torch.randn(rows, H, generator=g, device=dev).to(torch.bfloat16)
    gain = (1 + 0.1 * torch.randn(H, generator=g, device=dev)).to(torch.bfloat16)
    out = {"rows": rows, "width": H}
    for name, fn, nb in (("rowstat", lambda: q3.rms_rowstat(cfg, x), 2 * rows * H + 4 * rows),
                         ("final_norm", lambda: q3.final_norm(cfg, x, gain),
                          4 * rows * H + 2 * H)):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / reps
        out[name] = {"us": 1e6 * t, "bytes": nb,
                     "roofline": {"bound": "hbm", "achieved": nb / t / 1e9, "peak": hbm,
                                  "unit": "GB/s", "frac": nb / t / 1e9 / hbm}}
    q3.check_device()
    del x
    torch.cuda.empty_cache()
    return out


def kernel_rooflines(w, stage_ms, peak, peak_name, hbm):
    """Per-kernel algorithmic work over its live stage time."""
    S, H, I = w.seq, w.hidden, w.intermediate
    Dq, Dkv = w.q_dim, w.kv_dim
    flops = {
        "qkv": 2 * S * H * (Dq + 2 * Dkv),
        "attention": 4 * w.n_heads * 128 * S * (S + 1) // 2,
        "o_proj": 2 * S * Dq * H,
        "gate_up": 4 * S * H * I,
        "down": 2 * S * I * H,
    }
    out = {}
    for k, f in flops.items():
        ms = stage_ms[k]
        a = f / (ms / 1e3) / 1e12
        out[k] = {"bound": "tensor", "ms": ms, "gflop": f / 1e9, "achieved": a,
                  "unit": "TFLOP/s", "peak": peak, "frac": a / peak, "peak_source": peak_name}
    # The bf16 layer's prologue kernel (the "table" stage): P1's cos/sin table
    # written, the positions read, and P2's pass over x (read once, 1/rms
    # written). P2 has no stage of its own in a bf16 layer call.
    b = S * 64 * 2 * 4 + 3 * S * 4 + S * H * 2 + S * 4
    ms = stage_ms["table"]
    a = b / (ms / 1e3) / 1e9
    out["prologue"] = {"bound": "hbm", "ms": ms, "bytes": b, "achieved": a, "unit": "GB/s",
                       "peak": hbm, "frac": a / hbm, "peak_source": "measured copy bandwidth",
                       "note": "P1 + P2 in one launch, timed with its launch gap"}
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

    # Device-resident timed region. Every `stage_every`-th step records the
    # stage-boundary events the per-kernel times come from. An event between
    # two kernels keeps the second from starting early as a programmatic
    # dependent of the first, so those steps run their kernels back to back
    # without overlap (clean per-kernel times); the other steps do not record.
    every = max(1, args.stage_every)
    sampled = [k for k in range(args.steps) if k % every == 0]
    evs = {k: [torch.cuda.Event(enable_timing=True) for _ in range(9)] for k in sampled}
    for row in evs.values():
        for e in row:
            e.record()
    torch.cuda.synchronize()
    n0 = q3.launch_count()
    with ClockSampler(dev) as clk:
        t_dev = timed(lambda k: device_step(st, evs.get(k)), args.steps, world, dev)
    launches = q3.launch_count() - n0
    q3.set_stage_events(None)
    st["events_on"] = False
    q3.check_device()
    clocks = clk.summary()
    stage_ms = {name: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in sampled)
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
    h2d = st["x_host"].numel() * 2 + st["tt_host"].numel() + \
        (st["g_host"].numel() * 4 if st["g_host"] is not None else 0)
    d2h = st["out_host"].numel() * 2
    del st, pipe
    torch.cuda.empty_cache()

    # the other workloads, for reference (one GPU only): the 2B-shape layer, the
    # 2B 28-layer stack and the 32B-shape 50-layer encoder at both lengths
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
    if world == 1 and not args.no_stacks:
        also[syn.Q2B_STACK.name] = stack_leg(syn.Q2B_STACK, dev, steps=10, warmup=3)
        also[syn.Q32B_ENC_1064.name] = stack_leg(syn.Q32B_ENC_1064, dev, steps=5, warmup=2)
        also[syn.Q32B_ENC.name] = stack_leg(syn.Q32B_ENC, dev, steps=3, warmup=1)
        also["elementwise-4b-width-s65536"] = elementwise_leg(dev, peaks()[2])
        also["context"] = ("the pages time one workload of this path: a 1064-token encode through "
                           "the 32B-shape encoder truncated at layer 50, 29 s (55 s with the "
                           "dequantize-and-host-GEMM arm) on a 28-core AVX2 host with quantized "
                           "weights; context only, not a baseline")

    decode = None
    if world == 1 and not args.no_decode:
        decode = decode_leg(dev, min(args.steps, 400), max(3, min(args.warmup, 20)),
                            tuple(int(b) for b in args.decode_batches.split(",")),
                            syn.Q4B_DECODE.with_layers(args.decode_layers))

    burst, sustained, hbm, src = peaks()
    # The burst peak applies to a kernel timed in a short region at full clock;
    # the sustained peak (the power-capped clock of a seconds-long loop) when
    # the timed region is long or the sampled SM clock sat well below its max.
    at_max = clocks.get("sm_mhz") is not None and clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"]
    if t_dev < 1.0 or at_max:
        peak, peak_name = burst, (f"{src} bf16 burst (timed region {t_dev:.3f} s, median SM clock "
                                  f"{clocks.get('sm_mhz')} of {clocks.get('sm_max_mhz')} MHz)")
    else:
        peak, peak_name = sustained, (f"{src} bf16 sustained (timed region {t_dev:.1f} s, median "
                                      f"SM clock {clocks.get('sm_mhz')} MHz below max)")
    gemm_f, attn_f = layer_flops(w)
    kr = kernel_rooflines(w, stage_ms, peak, peak_name, hbm)
    gu = kr["gate_up"]
    tc_s = sum(stage_ms[k] for k in ("qkv", "attention", "o_proj", "gate_up", "down")) / 1e3
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        n, times = cpu_oracle_rate(w, seconds=10.0)
        cpu = {"value": n * len(times) / sum(times), "unit": UNIT, "cores": cpu_cores(),
               "kind": "oracle",
               "sample": f"first {n} tokens of {w.name} (of {w.seq}), fp32 NumPy oracle layer, "
                         f"{len(times)} passes in {sum(times):.1f} s; attention cost grows with "
                         f"S, so the rate overstates the oracle at the full length"}
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
                     "achieved": gu["achieved"], "peak": peak, "unit": "TFLOP/s",
                     "frac": gu["frac"], "peak_source": peak_name,
                     "frac_of_sustained": gu["achieved"] / sustained,
                     "traffic": traffic_for_current_kernel(),
                     "flops_per_launch": gu["gflop"] * 1e9, "ms": gu["ms"]},
        "kernels": kr,
        "tensor_work": {"gemm_gflop": gemm_f / 1e9, "attn_gflop": attn_f / 1e9,
                        "tflops": (gemm_f + attn_f) / tc_s / 1e12,
                        "frac": (gemm_f + attn_f) / tc_s / 1e12 / peak,
                        "frac_of_burst": (gemm_f + attn_f) / tc_s / 1e12 / burst,
                        "frac_of_sustained": (gemm_f + attn_f) / tc_s / 1e12 / sustained},
        "stages_ms": stage_ms,
        "cpu_baseline": cpu,
        "e2e": {"value": world * S * args.steps / t_e2e, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "also": also,
        "decode": decode,
        "gpu_launches": launches,
        "clocks": clocks,
        "next_position": nxt,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
