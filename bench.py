#!/usr/bin/env python
"""Benchmark of the TokenGate prefill hot path on B200: prefill tokens/s through
gate -> top-K -> gather -> (QKV projection, RoPE) -> token-gated attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tokengate|reference]
                    [--workload NAME]

One step = one pass of the whole path over one workload.  The default is the
128k-token workload (Qwen3-1.7B gate layer: N = 131072 tokens, document 130560,
question 512, hidden 2048, gate 2048 -> 256 -> 1, K_doc = 4096 so K = 4608 kept
tokens, 16 query / 8 KV heads of 128, 3% of the rows scaled x3); --workload
picks the 16k one or one of the 32k budget sweep (K_doc 512 / 2048 / 8192 /
16384, and K = N with zero gains and tau = 1).  Inputs are synthetic and seeded.
Where h is smaller than twice the 126 MB L2 (16k, 32k) a 256 MB buffer is
written between timed steps; at 128k h (537 MB) already is larger.

Multi-GPU (torchrun): every rank runs its own replica (independent prefills,
"scaling": "weak"); the only collectives are the barrier and the max-over-ranks
of the device time.  Rank 0 prints one JSON line.

--impl reference runs the CPU oracle (single thread) on a bounded sample of
each step's work and extrapolates to the full workload; only rank 0 works.
"""
import argparse
import faulthandler
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from learned_token_pruning_tg_b200 import synth  # noqa: E402

METRIC = "prefill tokens/s through gate+top-K+gated attention at 16k–128k; % roofline"
WORKLOAD = synth.L128K
BENCH_WORKLOADS = {name: w for name, w in synth.WORKLOADS.items() if w.bf16}
L2_BYTES = 126 * 1000 * 1000


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def config_dict(w):
    return {"workload": f"{w.name}: gate layer, N={w.N} (document {w.n_doc}, question {w.N - w.n_doc}), "
                        f"K_doc={w.k_doc} -> K={w.K}",
            "N": w.N, "doc_span": [w.doc_begin, w.doc_end], "k_doc": w.k_doc, "K": w.K, "d": w.d, "d_g": w.d_g,
            "Hq": w.Hq, "Hkv": w.Hkv, "d_h": w.d_h, "heavy_rows": f"{w.n_scaled} rows x{w.scale}",
            "l2": (f"256 MB written between timed steps (h is {w.N * w.d * 2 / 1e6:.0f} MB < 2 x 126 MB L2)"
                   if needs_flush(w) else
                   f"inputs larger than L2 (h is {w.N * w.d * 2 / 1e6:.0f} MB > 2 x 126 MB L2); no flush"),
            "path": "gate, select, gather, projection with RoPE (fused), attention", "seed": w.seed,
            **({"tau": 1.0, "gain": 0.0} if w.zero_gain else {})}


def needs_flush(w) -> bool:
    """True when the step's main input (h) is not at least twice the L2: then the L2 is flushed by a
    256 MB write between timed steps."""
    return w.N * w.d * 2 < 2 * L2_BYTES


def make_layer(w, gi, ap, dev, gather_into_projection=False):
    """The gate layer the benchmark times (and the end-to-end parity test checks), for one workload."""
    from learned_token_pruning_tg_b200.path import GatedPrefillLayer
    Wqkv = torch.cat([ap.Wq, ap.Wk, ap.Wv], dim=0)
    return GatedPrefillLayer(w.N, w.doc_begin, w.doc_end, w.k_doc, gi.W1.to(torch.bfloat16), gi.w2, Wqkv, w.Hq,
                             w.Hkv, w.d_h, ap.gain, ap.tau, eps=w.eps, rope_base=w.rope_base, device=dev,
                             gather_into_projection=gather_into_projection)


# ---------------------------------------------------------------- multi-rank plumbing
def reduce_max(x: float, device) -> float:
    """Max of x over all ranks (a no-op on one process).  Replicas run independent prefills,
    so the job's time is that of its slowest rank."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(w, rank: int) -> int:
    """Each rank prefills its own prompt (independent problems): a different seed per rank."""
    return w.seed + rank


def job_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: tokens all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


# ---------------------------------------------------------------- algorithmic work per stage
def stage_work(w):
    """Algorithmic FLOPs and bytes of each stage (per step)."""
    N, d, dg, K, Hq, Hkv, dh = w.N, w.d, w.d_g, w.K, w.Hq, w.Hkv, w.d_h
    return {
        "gate": {"flops": 2.0 * N * d * dg, "bytes": N * d * 2 + dg * d * 2 + dg * 4 + N * 4},
        "select": {"flops": 0.0, "bytes": N * 4 + K * 4},
        "gather": {"flops": 0.0, "bytes": 2.0 * K * d * 2 + K * 4 * 4},
        "rope": {"flops": 0.0, "bytes": 2.0 * K * (Hq + Hkv) * dh * 2 + K * 4},
        "attn": {"flops": 4.0 * (K * K / 2.0) * dh * Hq,
                 "bytes": (K * Hq * dh + 2 * K * Hkv * dh + K * Hq * dh) * 2 + K * 4},
        "qkv": {"flops": 2.0 * K * d * (Hq + 2 * Hkv) * dh, "bytes": (K * d + d * (Hq + 2 * Hkv) * dh +
                                                                   K * (Hq + 2 * Hkv) * dh) * 2},
        # the fused projection: x [K, d] and W read once, qkv written in bf16 and V again in fp16
        "proj": {"flops": 2.0 * K * d * (Hq + 2 * Hkv) * dh,
                 "bytes": (K * d + d * (Hq + 2 * Hkv) * dh + K * (Hq + 2 * Hkv) * dh + K * Hkv * dh) * 2 + K * 4},
    }


KERNEL_SOURCES = {
    "gate": ["gate_score.cu"], "select": ["topk_select.cu"], "gather": ["gather_compact.cu"],
    "rope": ["rope_apply.cu"], "attn": ["gated_attention.cu"], "proj": ["project_rope.cu"],
}


def kernel_src_hash(stage):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "learned_token_pruning_tg_b200", "csrc")
    for f in KERNEL_SOURCES[stage] + ["tg_device.cuh"]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(stage):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            j = json.load(f)
        e = j.get(stage)
        if e and e.get("src_sha") == kernel_src_hash(stage):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- clocks during the timed region
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle", 0x2: "applications_clocks_setting"}

    def __init__(self, cuda_index, period=0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(cuda_index)
            dom, bus, dev = (getattr(props, k, None) for k in ("pci_domain_id", "pci_bus_id", "pci_device_id"))
            if all(isinstance(x, int) for x in (dom, bus, dev)):
                # NVML wants the bus id as a string "dddddddd:bb:dd.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0".encode())
            else:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[cuda_index]) if vis else cuda_index
                self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = self._reasons_fn(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = sorted(r for r in self.reasons if r != "gpu_idle")
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------- oracle (CPU) timing
_ORACLE_CACHE = {}



def host_info():
    """The host's core count and CPU model (the oracle baseline runs on one of those cores)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def oracle_sample(w, gi, ap, budget_s, seed=0):
    """Time the single-threaded oracle on a bounded sample of one step of this workload's own data and
    extrapolate the step time.

    Sample (every step on the workload's hidden states and weights):
      gate        n_g rows of h drawn at random, scaled by N / n_g;
      select      in full, over a score vector of length N made of the sampled rows' scores repeated
                  (the select's cost depends on N, not on the values);
      gather      in full (the kept set of that select);
      projection  the first K_a gathered rows times Wq, Wk, Wv, scaled by K / K_a;
      RoPE        the same K_a rows, scaled by K / K_a;
      attention   n_a query rows spread over the first K_a rows, every head, over their causal keys among
                  those rows, scaled by the causal (query, key) pairs of the whole kept set over the
                  pairs timed.
    Every part is timed as it runs; the extrapolation only multiplies each part by its stated factor."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(seed)
    N, K, d_h, Hq, Hkv, d = w.N, w.K, w.d_h, w.Hq, w.Hkv, w.d
    cols = (Hq + 2 * Hkv) * d_h
    n_g = max(8, int(0.35 * budget_s / (d * w.d_g * 9e-10)))
    K_a = int(min(K, max(16, 0.25 * budget_s / (d * cols * 1.1e-9))))
    c = _ORACLE_CACHE.get((w.name, gi.h.data_ptr()))
    if c is None:
        c = {"W1": gi.W1.float().numpy(), "w2": gi.w2.numpy(),
             "h_bits": gi.h.view(torch.int16).numpy().view(np.uint16),
             "Wqkv": torch.cat([ap.Wq, ap.Wk, ap.Wv]).float().numpy()}
        _ORACLE_CACHE[(w.name, gi.h.data_ptr())] = c
    rows_g = np.sort(rng.choice(N, size=min(n_g, N), replace=False))
    hs = gi.h[torch.from_numpy(rows_g)].float().numpy()
    t0 = time.perf_counter()
    s_g = oracle.gate_score(hs, c["W1"], c["w2"], eps=w.eps)
    t_gate = (time.perf_counter() - t0) * N / len(rows_g)
    scores = np.resize(s_g.astype(np.float32), N)
    t0 = time.perf_counter()
    kept = oracle.topk_select(scores, w.doc_begin, w.doc_end, w.k_doc)
    t_select = time.perf_counter() - t0
    t0 = time.perf_counter()
    h_kept, pos, s_kept = oracle.gather_compact(c["h_bits"], kept, scores=scores)
    t_gather = time.perf_counter() - t0
    x = (h_kept[:K_a].astype(np.uint32) << 16).view(np.float32)
    t0 = time.perf_counter()
    qkv = oracle.project(x, c["Wqkv"])
    t_proj = (time.perf_counter() - t0) * K / K_a
    qf = qkv[:, : Hq * d_h].astype(np.float32).reshape(K_a, Hq, d_h)
    kf = qkv[:, Hq * d_h: (Hq + Hkv) * d_h].astype(np.float32).reshape(K_a, Hkv, d_h)
    t0 = time.perf_counter()
    q = oracle.rope(qf, pos[:K_a], w.rope_base)
    k = oracle.rope(kf, pos[:K_a], w.rope_base)
    t_rope = (time.perf_counter() - t0) * K / K_a
    v = qkv[:, (Hq + Hkv) * d_h:].reshape(K_a, Hkv, d_h)
    per_pair = 4.0 * d_h * Hq * 1.1e-9
    n_a = int(max(1, min(K_a, 0.3 * budget_s / (per_pair * K_a / 2.0))))
    rows_a = np.unique(np.linspace(0, K_a - 1, n_a).astype(np.int64))
    t0 = time.perf_counter()
    oracle.gated_attention(q, k, v, s=s_kept[:K_a], g=ap.gain.numpy(), tau=ap.tau, rows=rows_a)
    t_attn = (time.perf_counter() - t0) * (K * (K + 1) / 2.0) / float(np.sum(rows_a + 1))
    total = t_gate + t_select + t_gather + t_proj + t_rope + t_attn
    sample = (f"oracle, 1 thread, on this workload's data: gate {len(rows_g)}/{N} rows, select and gather in full, "
              f"projection and RoPE {K_a}/{K} kept rows, attention {len(rows_a)} query rows x {Hq} heads over the "
              f"first {K_a} kept rows (scaled by causal pairs); each part extrapolated by its factor")
    parts = {"gate_s": t_gate, "select_s": t_select, "gather_s": t_gather, "proj_s": t_proj, "rope_s": t_rope,
             "attn_s": t_attn}
    return total, sample, parts


def oracle_backward_sample(K, Hq, Hkv, d_h, budget_s=10.0, seed=0):
    """Time the single-threaded oracle backward on a bounded sample and extrapolate one full backward.

    Sample: one KV head and its G = Hq / Hkv query heads (an independent problem) over the first K' of
    the K tokens, K' chosen so the sample takes about budget_s; the causal work grows as K'(K'+1)/2,
    so the time is scaled by K(K+1) / (K'(K'+1)) and by the Hkv KV heads."""
    import numpy as np

    import oracle

    G = Hq // Hkv
    # about 5 multiply-adds of d_h per visible (query, key, head) pair at ~1.2e9 per second
    per_pair = 5.0 * d_h / 1.2e9 * G
    Ks = int(min(K, max(64, (2.0 * budget_s / per_pair) ** 0.5)))
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((Ks, G, d_h)).astype(np.float32)
    k = rng.standard_normal((Ks, 1, d_h)).astype(np.float32)
    v = rng.standard_normal((Ks, 1, d_h)).astype(np.float32)
    do = rng.standard_normal((Ks, G, d_h)).astype(np.float32)
    s = rng.standard_normal(Ks).astype(np.float32)
    g = rng.random(G).astype(np.float32)
    t0 = time.perf_counter()
    oracle.gated_attention_backward(q, k, v, do, s=s, g=g, tau=1.1)
    t = time.perf_counter() - t0
    total = t * (K * (K + 1.0)) / (Ks * (Ks + 1.0)) * Hkv
    sample = (f"oracle backward, 1 thread: 1 of {Hkv} KV heads ({G} query heads) over the first {Ks} of {K} "
              f"tokens, extrapolated by the causal pair count and the KV heads")
    return total, sample


def oracle_decode_sample(keys_per_layer, Hq, Hkv, d_h, budget_s=5.0, seed=0):
    """Time the single-threaded oracle on one decoding query over a T_s-key cache (the oracle's gated
    attention for the last row) and extrapolate by the keys of every layer (work is linear in keys)."""
    import numpy as np

    import oracle

    per_key = 2.0 * d_h * Hq / 1.2e9
    Ts = int(min(max(keys_per_layer), max(256, budget_s / per_key)))
    rng = np.random.default_rng(seed)
    q = np.zeros((Ts, Hq, d_h), dtype=np.float32)
    q[-1] = rng.standard_normal((Hq, d_h))
    k = rng.standard_normal((Ts, Hkv, d_h)).astype(np.float32)
    v = rng.standard_normal((Ts, Hkv, d_h)).astype(np.float32)
    s = rng.standard_normal(Ts).astype(np.float32)
    g = rng.random(Hq).astype(np.float32)
    t0 = time.perf_counter()
    oracle.gated_attention(q, k, v, s=s, g=g, tau=1.1, rows=[Ts - 1])
    t = time.perf_counter() - t0
    total = t / Ts * float(sum(keys_per_layer))
    sample = (f"oracle, 1 thread: one decoding query over a {Ts}-key cache ({Hq} heads), extrapolated by the "
              f"{sum(keys_per_layer)} cached keys of the {len(keys_per_layer)} layer(s)")
    return total, sample


def decode_cpu_baseline(args, keys_per_layer, Hq, Hkv, d_h, unit_scale, unit):
    if args.no_cpu_baseline:
        return {}
    cores = pin_one_core()
    t, sample = oracle_decode_sample(keys_per_layer, Hq, Hkv, d_h, budget_s=min(args.cpu_budget, 5.0))
    return {"cpu_baseline": {"value": t * unit_scale, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample}}


def pin_one_core():
    try:
        os.sched_setaffinity(0, {sorted(os.sched_getaffinity(0))[0]})
        return 1
    except Exception:
        return 1


# ---------------------------------------------------------------- arms
def run_reference(args, rank, world):
    """The reference arm: the oracle, single-threaded, on a bounded sample of each step (rank 0 only).
    A step here is the sample actually run: `steps` samples are timed, `ms_per_step` is their mean
    wall time, and `value` is the tokens/s that sample rate represents (N over the extrapolated time
    of a whole step)."""
    w = BENCH_WORKLOADS[args.workload]
    if rank != 0:
        return None
    gi = synth.gate_inputs(w)
    ap = synth.attn_params(w)
    budget = min(15.0, 100.0 / max(1, args.steps + args.warmup))
    cores = pin_one_core()
    for _ in range(args.warmup):
        oracle_sample(w, gi, ap, budget)
    walls, fulls = [], []
    for i in range(args.steps):
        t0 = time.perf_counter()
        t, sample, _ = oracle_sample(w, gi, ap, budget, seed=i)
        walls.append(time.perf_counter() - t0)
        fulls.append(t)
    t_full = statistics.mean(fulls)
    value = w.N / t_full
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_dict(w),
            "impl": "reference", "extrapolated": True,
            "step": "one bounded oracle sample of the workload's step; value = N / (the sample's time "
                    "extrapolated to the whole step)",
            "full_step_s_extrapolated": t_full,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample, **host_info()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_tokengate(args, rank, world, local_rank):
    from learned_token_pruning_tg_b200 import tokengate as tg
    from learned_token_pruning_tg_b200.path import nvtx_marks

    if not os.path.exists(tg.LIB_PATH):
        from learned_token_pruning_tg_b200 import build as tg_build
        tg_build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = BENCH_WORKLOADS[args.workload]
    gi = synth.gate_inputs(w, seed=replica_seed(w, rank))
    ap = synth.attn_params(w, seed=replica_seed(w, rank))
    layer = make_layer(w, gi, ap, dev)
    stages = list(layer.stages)
    h = gi.h.to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if needs_flush(w) else None

    def between_steps():
        if flush is not None:
            flush.fill_(1)

    for _ in range(args.warmup):
        # warm-up steps carry NVTX ranges per step when asked (for a profiler's NVTX filter)
        layer.run(h, mark=nvtx_marks() if args.nvtx else None)
    torch.cuda.synchronize()
    assert layer.device_status() == 0, "device status nonzero after the warm-up"

    # The step captured once in a CUDA graph (the same kernels, replayed without host launch cost).
    # Every rank takes the same collective steps whether or not its capture works.
    graph, graph_err = None, None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            layer.run(h)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            layer.run(h)
        for _ in range(max(3, args.warmup)):
            g.replay()
        torch.cuda.synchronize()
        graph = g
    except Exception as e:  # report, do not fail the run
        graph_err = f"{type(e).__name__}: {e}"[:200]
        torch.cuda.synchronize()
    graph_failed = reduce_max(0.0 if graph is not None else 1.0, dev) > 0.0

    # Every timed step has its own events on the launching (current) stream; the L2 flush, where the
    # workload needs one, runs between a step's end event and the next step's start event.
    K = args.steps
    names = stages + ["end"]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in names] for _ in range(K)]

    def marker(i):
        def m(name):
            ev[i][names.index(name)].record()
        return m

    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    # (3) per-step kernel times in the step's own context and without host launch gaps: one CUDA graph
    # per prefix of the step (gate; gate + select; ...), each replayed R times between its own events;
    # a step's time is the difference between the mean times of the prefix that ends with it and the
    # prefix before it.  Every replay follows a 256 MB pass over L2, so each prefix's gate starts from
    # the same L2 state (a gate right after a gate runs ~10% slower than after other work, which would
    # shift time from the gate's prefix into the select's difference): the same write flush the timed
    # steps have where they have one, else a read of 256 MB, which evicts L2 without leaving dirty
    # lines whose write-back the next gate would pay and the timed steps do not.
    R = max(10, min(K, 40))
    evict = None if flush is not None else torch.empty(256 << 20, dtype=torch.uint8, device=dev).view(torch.int32)

    def before_prefix():
        if flush is not None:
            flush.fill_(1)
        else:
            evict.max()
    prefix_graphs, staged_err = [], None
    try:
        calls = list(layer.stage_calls(h).values())
        for n in range(1, len(calls) + 1):
            gs = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gs):
                for call in calls[:n]:
                    call()
            gs.replay()
            prefix_graphs.append(gs)
        torch.cuda.synchronize()
    except Exception as e:  # report, fall back to the kernel-by-kernel stage times
        staged_err = f"{type(e).__name__}: {e}"[:200]
        prefix_graphs = []
        torch.cuda.synchronize()
    staged_failed = reduce_max(0.0 if prefix_graphs else 1.0, dev) > 0.0
    pev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(R)]
           for _ in prefix_graphs]
    with ClockSampler(dev.index) as clk:
        # (1) K steps launched one kernel at a time, with per-stage events
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for i in range(K):
            between_steps()
            layer.run(h, mark=marker(i))
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        # (2) K replays of the captured step
        if not graph_failed:
            torch.cuda.synchronize()
            for e0, e1 in gev:
                between_steps()
                e0.record()
                graph.replay()
                e1.record()
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
        # (3) the step's prefixes
        if not staged_failed:
            for gs, evs in zip(prefix_graphs, pev):
                for e0, e1 in evs:
                    before_prefix()
                    e0.record()
                    gs.replay()
                    e1.record()
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
    ms_launched = reduce_max(sum(e[0].elapsed_time(e[-1]) for e in ev) / K, dev)
    stage_ms = {s: sum(e[j].elapsed_time(e[j + 1]) for e in ev) / K for j, s in enumerate(stages)}
    stage_timing = "kernel-by-kernel launches of the timed steps (host launch gaps included)"
    if not staged_failed:
        prefix_ms = [reduce_max(sum(e0.elapsed_time(e1) for e0, e1 in evs) / R, dev) for evs in pev]
        stage_ms = {s: prefix_ms[j] - (prefix_ms[j - 1] if j else 0.0) for j, s in enumerate(stages)}
        stage_timing = (f"step prefixes (gate; gate + select; ...) each captured in a CUDA graph and replayed {R} "
                        f"times between events, each replay after a 256 MB pass over L2 ({'write' if flush is not None else 'read'}); "
                        f"a step's time is the difference of consecutive prefix means")
    del prefix_graphs
    status = layer.device_status()
    ungraphed = {"ms_per_step": ms_launched, "value": job_throughput(w.N, world, ms_launched), "unit": "tokens/s"}
    if not graph_failed:
        ms_graph = reduce_max(sum(e0.elapsed_time(e1) for e0, e1 in gev) / K, dev)
        graph_line = {"ms_per_step": ms_graph, "value": job_throughput(w.N, world, ms_graph), "unit": "tokens/s"}
        ms_step, value = ms_graph, graph_line["value"]
    else:
        graph_line = {"unavailable": graph_err or "capture failed on another rank"}
        ms_step, value = ms_launched, ungraphed["value"]
    del graph

    # end to end through the same API from pinned host memory: H2D of h, the path, D2H of out + kept
    h_host = gi.h.pin_memory()
    out_host = torch.empty(layer.out.shape, dtype=torch.bfloat16).pin_memory()
    kept_host = torch.empty(layer.K, dtype=torch.int32).pin_memory()
    h_dev = torch.empty_like(h)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        layer.run_host(h_host, h_dev, out_host, kept_host)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        layer.run_host(h_host, h_dev, out_host, kept_host)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = reduce_max(e2e_ms, dev)
    e2e = {"value": job_throughput(w.N, world, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h_host.numel() * h_host.element_size(),
           "d2h_bytes_per_step": out_host.numel() * out_host.element_size() + kept_host.numel() * 4,
           "ms_per_step": e2e_ms}

    # The key bias's cost: the attention call with and without s' and g (the pages put it at <= 1.1x).
    def time_attn(with_bias: bool, reps: int = 20) -> float:
        kw = dict(s_kept=layer.s_kept[: layer.K], gain=layer.gain) if with_bias else {}
        for _ in range(3):
            tg.tg_gated_attention_f16v(layer.q, layer.k, layer.v16, layer.out, layer.ws_attn, tau=layer.tau, **kw)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(reps):
            tg.tg_gated_attention_f16v(layer.q, layer.k, layer.v16, layer.out, layer.ws_attn, tau=layer.tau, **kw)
        a1.record()
        torch.cuda.synchronize()
        return a0.elapsed_time(a1) / reps
    t_bias, t_plain = time_attn(True), time_attn(False)

    if rank != 0:
        return None

    # roofline of the dominant libtokengate kernel, and of the whole path.  The timed region is short
    # (milliseconds) and runs near the maximum clock, so the burst tensor peak is the denominator; the
    # sustained figure is reported beside it.
    peaks = load_peaks()
    work = stage_work(w)
    tensor_peak = peaks["bf16_tflops"]
    dom = max(stages, key=lambda s: stage_ms[s])

    def lower_bound(s, tpk=tensor_peak):
        return max(work[s]["flops"] / (tpk * 1e12), work[s]["bytes"] / (peaks["hbm_gbs"] * 1e9))

    sec = stage_ms[dom] * 1e-3
    if work[dom]["flops"] / (tensor_peak * 1e12) >= work[dom]["bytes"] / (peaks["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": work[dom]["flops"] / sec / 1e12, "peak": tensor_peak,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": work[dom]["bytes"] / sec / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic(dom)
    roof["kernel"] = dom
    roof["algorithmic_per_launch"] = {"flops": work[dom]["flops"], "bytes": work[dom]["bytes"]}
    roof["peak_source"] = peaks["source"] + (" (burst bf16)" if roof["bound"] == "tensor" else " (HBM copy)")
    if roof["bound"] == "tensor":
        roof["frac_of_sustained_peak"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
    # the specification's path (gate, select, gather, attention) and the whole step (plus the projection):
    # the path's steps that run as stages of their own (a layer that gathers inside the projection's
    # operand loads has no gather stage: that work is inside "proj", which the step fractions cover).
    # The path's time is the measured graphed step minus the estimated time of the stages off the path
    # (one estimate instead of the sum of four, each a difference of two prefix means); the sum of the
    # path's own stage estimates is reported beside it.
    path = [s for s in ("gate", "select", "gather", "attn") if s in stages]
    off_path = [s for s in stages if s not in path]
    t_split = sum(stage_ms[s] for s in path) * 1e-3
    t_path, path_method = t_split, "sum of the path's stage times"
    if not graph_failed and not staged_failed:
        t_rest = ms_step * 1e-3 - sum(stage_ms[s] for s in off_path) * 1e-3
        if t_rest > 0:
            t_path = t_rest
            path_method = f"graphed step minus the stage times off the path ({', '.join(off_path)})"
    path_roof = sum(lower_bound(s) for s in path) / t_path
    path_roof_sustained = sum(lower_bound(s, peaks["bf16_tflops_sustained"]) for s in path) / t_path
    path_roof_nominal = sum(max(work[s]["flops"] / 2.25e15, work[s]["bytes"] / 8.0e12) for s in path) / t_path
    step_bound = sum(lower_bound(s) for s in stages)
    kernels = {}
    for s in stages:
        sec_s = stage_ms[s] * 1e-3
        kernels[s] = {"us": stage_ms[s] * 1e3,
                      "tflops": work[s]["flops"] / sec_s / 1e12 if work[s]["flops"] else None,
                      "gbs": work[s]["bytes"] / sec_s / 1e9,
                      "bound_us": lower_bound(s) * 1e6,
                      "roofline_frac": lower_bound(s) / sec_s}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cores = pin_one_core()
        t, sample, parts = oracle_sample(w, gi, ap, args.cpu_budget)
        cpu = {"value": w.N / t, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
               "extrapolated_s_per_step": t, "parts_s": parts, **host_info()}

    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; stands in for NIAH-style prompts)",
            "config": config_dict(w), "impl": "tokengate",
            "path_ms": t_path * 1e3, "path_tokens_per_s": w.N * world / t_path, "path_stages": path,
            "path_method": path_method, "path_ms_from_split": t_split * 1e3,
            "path_roofline_frac_from_split": sum(lower_bound(s) for s in path) / t_split,
            "stage_sum_ms": sum(stage_ms.values()),
            "path_roofline_frac": path_roof, "path_roofline_frac_sustained_peak": path_roof_sustained,
            "path_roofline_frac_nominal_peak": path_roof_nominal,
            "step_roofline_frac_ungraphed": step_bound / (ms_launched * 1e-3),
            "step_roofline_frac": step_bound / (ms_step * 1e-3),
            "timing": "value and ms_per_step: K replays of the step captured in one CUDA graph, each between its "
                      "own events; 'ungraphed': the same K steps launched kernel by kernel; path_ms, the kernels "
                      "and the path fractions come from the step times named in stage_timing",
            "graph": graph_line, "ungraphed": ungraphed,
            "stage_timing": stage_timing if staged_err is None else f"{stage_timing} ({staged_err})",
            "attention_bias_cost": {"with_bias_ms": t_bias, "without_bias_ms": t_plain, "ratio": t_bias / t_plain},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": layer.launches_per_step() * K, "clocks": clk.summary(), "device_status": status,
            "peaks": peaks}


def run_stack(args, rank, world, local_rank):
    """The pruned prefill through a 28-layer stack at 64k (gate after layer 13, 8192 document tokens
    kept) against the same stack with every token kept: device time per prefill and peak memory."""
    from learned_token_pruning_tg_b200 import stack as stk
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = stk.STACK64K
    wts = stk.random_weights(cfg, dev)
    x = stk.random_embeddings(cfg, dev)
    s = stk.PrunedPrefillStack(cfg, wts, device=dev)
    reps = max(1, min(args.steps, 5))

    def timed(prune: bool):
        for _ in range(max(1, min(args.warmup, 2))):
            s.run(x, prune=prune, keep_kv=True)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            s.run(x, prune=prune, keep_kv=True)
        e1.record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        peak = torch.cuda.max_memory_allocated(dev) - base
        return reduce_max(e0.elapsed_time(e1) / reps, dev), peak, s.kv_bytes()

    with ClockSampler(dev.index) as clk:
        ms_pruned, mem_pruned, kv_pruned = timed(True)
        ms_dense, mem_dense, kv_dense = timed(False)
    status = s.device_status()
    if rank != 0:
        return None
    return {"metric": f"prefill latency, {cfg.n_layers}-layer stack at {cfg.N // 1024}k (gate after layer "
                      f"{cfg.gate_layer}, {cfg.k_doc} document tokens kept)",
            "value": ms_pruned, "unit": "ms", "n_gpus": world, "steps": reps, "warmup": args.warmup,
            "ms_per_step": ms_pruned, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded random weights and embeddings)",
            "config": {"workload": cfg.name, "N": cfg.N, "doc_span": [cfg.doc_begin, cfg.doc_end],
                       "k_doc": cfg.k_doc, "K": cfg.K, "layers": cfg.n_layers, "gate_layer": cfg.gate_layer,
                       "d": cfg.d, "d_ff": cfg.d_ff, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d_h": cfg.d_h},
            "impl": "tokengate",
            "dense_ms": ms_dense, "speedup": ms_dense / ms_pruned,
            "kv_cache_gb": {"pruned": kv_pruned / 1e9, "dense": kv_dense / 1e9},
            "peak_memory_gb": {"pruned": mem_pruned / 1e9, "dense": mem_dense / 1e9,
                               "note": "above the weights and inputs, KV cache included"},
            "clocks": clk.summary(), "device_status": status}


def run_decode(args, rank, world, local_rank):
    """One decoding step's attention over the KV cache a 28-layer 64k pruned prefill leaves (layers
    up to the gate layer hold all N keys, the layers above the K kept keys with their scores; plus
    the new token's own key), against the cache of the unpruned stack (N + 1 keys in every layer).
    Each layer's cache is its own buffer (4.3 GB and 7.5 GB in all, far above L2), so every step
    reads it from HBM; the 28 launches of a step are captured in one CUDA graph."""
    from learned_token_pruning_tg_b200 import stack as stk
    from learned_token_pruning_tg_b200 import tokengate as tg
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = stk.STACK64K
    Hq, Hkv, d_h, L = cfg.Hq, cfg.Hkv, cfg.d_h, cfg.gate_layer
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed + 7 + rank)

    def cache(T):
        return (torch.randn(T, Hkv, d_h, generator=gen, device=dev, dtype=torch.bfloat16),
                torch.randn(T, Hkv, d_h, generator=gen, device=dev, dtype=torch.bfloat16),
                torch.randn(T, generator=gen, device=dev))

    T_all, T_kept = cfg.N + 1, cfg.K + 1
    pruned = [cache(T_all if li <= L else T_kept) for li in range(cfg.n_layers)]
    dense = [cache(T_all) for _ in range(cfg.n_layers)]
    q = torch.randn(Hq, d_h, generator=gen, device=dev, dtype=torch.bfloat16)
    gain = 2.0 * torch.rand(Hq, generator=gen, device=dev)
    out = torch.empty(Hq, d_h, dtype=torch.bfloat16, device=dev)
    ws = tg.new_workspace(0, Hq, op=tg.TG_OP_DECODE, device=dev)

    def step(layers, prune):
        for li, (k, v, sc) in enumerate(layers):
            if prune and li > L:
                tg.tg_gated_decode(q, k, v, out, ws, s_cache=sc, gain=gain, tau=1.1)
            else:
                tg.tg_gated_decode(q, k, v, out, ws, tau=1.0)

    def cache_bytes(layers, prune):
        return sum(k.numel() * 2 * 2 + (sc.numel() * 4 if prune and li > L else 0)
                   for li, (k, v, sc) in enumerate(layers))

    reps = max(10, min(args.steps, 200))

    def timed(layers, prune):
        for _ in range(3):
            step(layers, prune)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(layers, prune)
        for _ in range(max(3, args.warmup)):
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        del g
        return reduce_max(e0.elapsed_time(e1) / reps, dev)

    with ClockSampler(dev.index) as clk:
        ms_pruned = timed(pruned, True)
        ms_dense = timed(dense, False)
    status = tg.tg_device_status(ws)
    if rank != 0:
        return None
    peaks = load_peaks()
    b_pruned, b_dense = cache_bytes(pruned, True), cache_bytes(dense, False)
    achieved = b_pruned / (ms_pruned * 1e-3) / 1e9
    return {"metric": f"decode-step attention latency over the KV cache of a {cfg.n_layers}-layer {cfg.N // 1024}k "
                      f"pruned prefill (gate after layer {cfg.gate_layer}, {cfg.k_doc} document tokens kept)",
            "value": ms_pruned, "unit": "ms", "n_gpus": world, "steps": reps, "warmup": args.warmup,
            "ms_per_step": ms_pruned, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded random caches)",
            "config": {"workload": f"{cfg.name} decode", "layers": cfg.n_layers, "gate_layer": L,
                       "keys_per_layer": {"up_to_gate": T_all, "above_gate": T_kept}, "Hq": Hq, "Hkv": Hkv,
                       "d_h": d_h, "timing": "one CUDA graph of the 28 launches per step, replayed"},
            "impl": "tokengate", "dense_ms": ms_dense, "speedup": ms_dense / ms_pruned,
            "bytes_per_step": {"pruned": b_pruned, "dense": b_dense},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": "gated_decode_kernel",
                         "dense_frac": b_dense / (ms_dense * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "gpu_launches": cfg.n_layers * reps, "clocks": clk.summary(), "device_status": status,
            **decode_cpu_baseline(args, [T_all if li <= L else T_kept for li in range(cfg.n_layers)], Hq, Hkv,
                                  d_h, 1e3, "ms")}


def run_decode_layer(args, rank, world, local_rank):
    """One layer's decoding-step attention over a 64k cache (65,537 keys x 8 KV heads x 128, K and V
    268 MB, above L2): the single launch the decode kernel's ncu summary captures."""
    from learned_token_pruning_tg_b200 import stack as stk
    from learned_token_pruning_tg_b200 import tokengate as tg
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = stk.STACK64K
    T = cfg.N + 1
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed + 11 + rank)
    k = torch.randn(T, cfg.Hkv, cfg.d_h, generator=gen, device=dev, dtype=torch.bfloat16)
    v = torch.randn(T, cfg.Hkv, cfg.d_h, generator=gen, device=dev, dtype=torch.bfloat16)
    s = torch.randn(T, generator=gen, device=dev)
    q = torch.randn(cfg.Hq, cfg.d_h, generator=gen, device=dev, dtype=torch.bfloat16)
    gain = 2.0 * torch.rand(cfg.Hq, generator=gen, device=dev)
    out = torch.empty(cfg.Hq, cfg.d_h, dtype=torch.bfloat16, device=dev)
    ws = tg.new_workspace(0, cfg.Hq, op=tg.TG_OP_DECODE, device=dev)
    for _ in range(max(3, args.warmup)):
        tg.tg_gated_decode(q, k, v, out, ws, s_cache=s, gain=gain, tau=1.1)
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 100))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        tg.tg_gated_decode(q, k, v, out, ws, s_cache=s, gain=gain, tau=1.1)
    e1.record()
    torch.cuda.synchronize()
    us = reduce_max(e0.elapsed_time(e1) / reps * 1e3, dev)
    if rank != 0:
        return None
    nbytes = 2 * k.numel() * 2 + s.numel() * 4
    peaks = load_peaks()
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"metric": "one layer's decoding-step attention over a 64k KV cache", "value": us, "unit": "us",
            "n_gpus": world, "steps": reps, "warmup": args.warmup, "ms_per_step": us / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random cache)",
            "config": {"workload": "qwen3-1.7b 64k layer cache", "T": T, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d_h": cfg.d_h,
                       "l2": "cache 268 MB > L2, no flush"},
            "impl": "tokengate",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": None, "kernel": "gated_decode_kernel"},
            "gpu_launches": reps, "device_status": tg.tg_device_status(ws),
            **decode_cpu_baseline(args, [T], cfg.Hq, cfg.Hkv, cfg.d_h, 1e6, "us")}


def run_backward(args, rank, world, local_rank):
    """The gradients of the gated attention above the gate at the 128k workload's kept set (K = 4608,
    16 query / 8 KV heads of 128): one tg_gated_attention_backward call (four launches) per step, after
    one forward that provides the output and log-sum-exp.  The inputs (75 MB) fit in L2, so a 512 MB
    buffer is written between timed calls; each call is timed alone with its own events."""
    from learned_token_pruning_tg_b200 import tokengate as tg
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    K, Hq, Hkv, d_h = WORKLOAD.K, WORKLOAD.Hq, WORKLOAD.Hkv, WORKLOAD.d_h
    d = synth.qkv(K, Hq, Hkv, d_h, seed=4608 + rank, heavy_frac=0.03)
    dout = synth.grad_out(K, Hq, d_h, seed=4609 + rank).to(dev)
    q, k, v, s, g = d.q.to(dev), d.k.to(dev), d.v.to(dev), d.s.to(dev), d.gain.to(dev)
    out = torch.empty(K, Hq, d_h, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(Hq, K, dtype=torch.float32, device=dev)
    ws_f = tg.new_workspace(K, Hkv * d_h, op=tg.TG_OP_ATTENTION, device=dev)
    tg.tg_gated_attention(q, k, v, out, ws_f, s_kept=s, gain=g, tau=d.tau, lse=lse)
    ws = tg.new_workspace(K, Hq, Hkv, op=tg.TG_OP_ATTENTION_BACKWARD, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = torch.empty(K, dtype=torch.float32, device=dev)
    dg = torch.empty(Hq, dtype=torch.float32, device=dev)
    dtau = torch.empty(1, dtype=torch.float32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def call():
        tg.tg_gated_attention_backward(q, k, v, out, dout, lse, dq, dk, dv, ws, s_kept=s, gain=g, tau=d.tau,
                                       ds=ds, dg=dg, dtau=dtau)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 50))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with ClockSampler(dev.index) as clk:
        for e0, e1 in ev:
            flush.fill_(1)
            e0.record()
            call()
            e1.record()
        torch.cuda.synchronize()
    us = reduce_max(sum(e0.elapsed_time(e1) for e0, e1 in ev) / reps * 1e3, dev)
    if rank != 0:
        return None
    pairs = K * (K + 1) / 2
    flop = 5 * 2 * pairs * d_h * Hq     # S, dP, dV, dK, dQ over the causal pairs (S and dP recomputed: 7)
    peaks = load_peaks()
    tf = flop / (us * 1e-6) / 1e12
    return {"metric": "gated attention backward (dq, dk, dv, ds, dg, dtau), 128k workload's kept set",
            "value": us, "unit": "us", "n_gpus": world, "steps": reps, "warmup": args.warmup,
            "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded q, k, v, dO; 3% heavy rows)",
            "config": {"workload": "qwen3-1.7b-128k kept set", "K": K, "Hq": Hq, "Hkv": Hkv, "d_h": d_h,
                       "l2": "inputs 75 MB < L2: 512 MB written between timed calls"},
            "impl": "tokengate",
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16_tflops"], "traffic": None,
                         "kernel": "whole backward (prep, dq, dkdv, finish)",
                         "algorithmic_flop": flop},
            "clocks": clk.summary(), "gpu_launches": 4 * reps, "device_status": tg.tg_device_status(ws),
            **backward_cpu_baseline(args, K, Hq, Hkv, d_h)}


def backward_cpu_baseline(args, K, Hq, Hkv, d_h):
    """The oracle backward beside the GPU one (rank 0 only; skipped with --no-cpu-baseline)."""
    if args.no_cpu_baseline:
        return {}
    cores = pin_one_core()
    t, sample = oracle_backward_sample(K, Hq, Hkv, d_h, budget_s=min(args.cpu_budget, 15.0))
    return {"cpu_baseline": {"value": t * 1e6, "unit": "us", "cores": cores, "kind": "oracle", "sample": sample}}


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["tokengate", "reference"], default="tokengate")
    ap.add_argument("--workload", choices=sorted(BENCH_WORKLOADS), default=WORKLOAD.name,
                    help="the workload one step runs (default: the 128k one)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nvtx", action="store_true", help="NVTX range tg:<step> around each warm-up step")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--decode-layer", action="store_true",
                    help="time one layer's decoding step over a 64k cache (the decode kernel alone)")
    ap.add_argument("--decode", action="store_true",
                    help="time one decoding step's attention over a pruned 28-layer cache (and an unpruned one)")
    ap.add_argument("--backward", action="store_true",
                    help="time the gated attention backward at the 128k workload's kept set")
    ap.add_argument("--stack", action="store_true",
                    help="time the pruned prefill through a 28-layer stack (and the unpruned one) instead")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run = (run_stack if args.stack else run_decode if args.decode else run_backward if args.backward else
               run_decode_layer if args.decode_layer else run_tokengate)
        res = run(args, rank, world, local_rank)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
