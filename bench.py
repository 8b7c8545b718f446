"""Benchmark of the hashed n-gram embedding lookup on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: the fused kernel forms the
bigram/trigram contexts, hashes 16 rows per token, gathers and sums them, applies the
gate and adds the residual ("Qwen Brought Back N-Grams. All 51 Billion Parameters of
Them.", section "N-grams, of all things"; gate of "Qwen3.8-Flash-Next: A 51B N-gram
Embedding Table with Heterogeneous Memory Prefetch", Key point 1).

Default workload: the full-size table of the pages (20,000,000 x 2560 bf16, 95.4 GiB in
HBM) and one 32,768-token prefill of Zipf(1.1) tokens over a 151,936-id vocabulary.
Prints one JSON line (rank 0).  Under torchrun every rank holds its own table replica
and its own token batch (weak scaling, no collective on the data path); the time is
the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

# the DMA host mode copies rows with OpenMP threads: let them sleep between calls instead of
# spinning on the cores the launching thread needs (read by libgomp when it loads)
os.environ.setdefault("OMP_WAIT_POLICY", "PASSIVE")

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ngram_inputs as gen  # noqa: E402

METRIC = "n-gram embed tokens/s and gather GB/s (% of HBM or PCIe H2D roofline), 1 B200"
UNIT = "tokens/s"
HEADS = 16
_CS = "hashed_gram_embedding_ngram_b200/csrc/"
KERNEL_SOURCES = {   # the source files each timed kernel and its processing order are built from
    "bf16": [_CS + "gather.cuh", _CS + "device_common.cuh", _CS + "order.cuh"],
    "int8": [_CS + "gather.cuh", _CS + "gather_int8.cuh", _CS + "device_common.cuh", _CS + "order.cuh"],
    "fp8": [_CS + "gather.cuh", _CS + "gather_int8.cuh", _CS + "device_common.cuh", _CS + "order.cuh"],
    "nvfp4": [_CS + "gather.cuh", _CS + "gather_int8.cuh", _CS + "gather_nvfp4.cuh",
              _CS + "device_common.cuh", _CS + "order.cuh"],
}
KERNEL_NAME = {"bf16": "k_gather_bf16<16>", "int8": "k_gather_int8<16>",
               "fp8": "k_gather_fp8<16>", "nvfp4": "k_gather_nvfp4<16>"}
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# --------------------------------------------------------------------------- helpers
def row_bytes(w) -> int:
    """Bytes the gather reads per row: bf16 2d; int8 / fp8 d codes + the fp32 row scale;
    nvfp4 d/2 code bytes + d/16 block-scale bytes (the padding is never read)."""
    if w.dtype == "bf16":
        return 2 * w.d
    if w.dtype == "nvfp4":
        return w.d // 2 + w.d // 16
    return w.d + 4


def stored_row_bytes(w) -> int:
    if w.dtype == "nvfp4":
        return w.d // 2 + -(-(w.d // 16) // 16) * 16
    return 2 * w.d if w.dtype == "bf16" else w.d + 4


def oracle_dtype(w) -> int:
    import oracle
    return {"bf16": oracle.BF16, "int8": oracle.INT8, "fp8": oracle.FP8, "nvfp4": oracle.NVFP4}[w.dtype]


def algorithmic_bytes(w, n_seq=None, T=None) -> int:
    """Bytes the method must move per call: 16 rows, the residual read and the output
    write per token, the token id, the gate once and the history once per sequence."""
    n_seq = w.n_seq if n_seq is None else n_seq
    T = w.T if T is None else T
    N = n_seq * T
    hist = 8 * n_seq if w.history else 0
    return N * (HEADS * row_bytes(w) + 2 * 2 * w.d + 4) + 4 * w.d + hist


def read_stream_gbs(dev, nbytes=4 << 30, reps=5) -> float:
    """A read-only HBM stream measured in this run (outside every timed region): the best
    of `reps` torch.amax reductions over nbytes of int32 -- a second denominator beside the
    measured copy peak."""
    import torch
    x = torch.ones(nbytes // 4, dtype=torch.int32, device=dev)
    best = float("inf")
    for i in range(reps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        torch.amax(x)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            best = min(best, e0.elapsed_time(e1))
    del x
    torch.cuda.empty_cache()
    return nbytes / (best / 1e3) / 1e9


def write_stream_gbs(dev, nbytes=4 << 30, reps=5) -> float:
    """A write-only HBM stream measured in this run (outside every timed region): the best
    of `reps` fills of nbytes of int32 -- the denominator for kernels that mostly write."""
    import torch
    x = torch.empty(nbytes // 4, dtype=torch.int32, device=dev)
    best = float("inf")
    for i in range(reps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        x.fill_(i)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            best = min(best, e0.elapsed_time(e1))
    del x
    torch.cuda.empty_cache()
    return nbytes / (best / 1e3) / 1e9


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def code_only(text: str) -> str:
    """A source file without its comments and blank lines: the hash below tracks the code,
    so that editing a comment does not orphan a committed ncu summary."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


def kernel_sha(dtype: str = "bf16", read=None) -> str:
    """Hash of the code (comments stripped) of the sources a timed kernel is built from.
    read(rel) -> text; default: the working tree."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[dtype]:
        if read is None:
            with open(os.path.join(ROOT, rel)) as f:
                text = f.read()
        else:
            text = read(rel)
        h.update(code_only(text).encode())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons while running."""

    def __init__(self, gpu_id: str, period_ms: int = 50):
        self.gpu_id, self.period_ms = gpu_id, period_ms
        self.proc, self.path = None, None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + CLOCK_FIELDS, "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms), "-i", self.gpu_id],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) == 9:
                        rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(rows)}


def gpu_id_for(dev) -> str:
    import torch
    p = torch.cuda.get_device_properties(dev)
    bus = getattr(p, "pci_bus_id", None)
    dom = getattr(p, "pci_domain_id", 0)
    devid = getattr(p, "pci_device_id", 0)
    if bus is not None:
        return "%08X:%02X:%02X.0" % (dom, bus, devid)
    return str(dev.index or 0)


# --------------------------------------------------------------------------- ranks
def rank_seeds(rank: int, batch: int):
    """(token seed, history seed) of one rank's batch: every rank draws its own tokens."""
    return gen.TOKEN_SEED + 1000 * rank + batch, gen.HISTORY_SEED + 1000 * rank + batch


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings (ms) over all ranks; a plain list back."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_tokens_per_s(world: int, tokens_per_rank: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (elapsed_ms / 1e3)


# --------------------------------------------------------------------------- CPU oracle
def oracle_tokens_per_s(w, inp, budget_s: float, threads: int, seed: int = 0, table=None):
    """Time the oracle (test infrastructure) on a bounded sample of this workload's tokens.
    table: the materialised table (uint16 [R][d] bf16 bits, e.g. a view of pinned host
    memory) the oracle reads its rows from; None: rows regenerated from the synthetic-table
    definition (one Philox call per two elements).  Returns (tokens/s, tokens, seconds)."""
    import oracle
    rng = np.random.default_rng(seed)
    kw = dict(R=w.R, d=w.d, dtype=oracle_dtype(w), acc=oracle.ACC_F32, n_threads=threads,
              vocab_size=w.vocab)
    if table is None:
        kw["table_seed"] = gen.TABLE_SEED
    else:
        kw["table"] = table
    probe = rng.choice(w.N, size=min(w.N, 4 * threads), replace=False)
    t0 = time.perf_counter()
    oracle.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"], sel=probe, **kw)
    per_tok = (time.perf_counter() - t0) / probe.size
    n = int(max(1, min(w.N, budget_s / max(per_tok, 1e-9))))
    sel = np.sort(rng.choice(w.N, size=n, replace=False))
    t0 = time.perf_counter()
    oracle.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"], sel=sel, **kw)
    dt = time.perf_counter() - t0
    if dt < budget_s / 2:                 # the whole batch took less than the budget: repeat it
        reps = int(min(100, budget_s / max(dt, 1e-9)))
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"], sel=sel, **kw)
        dt = time.perf_counter() - t0
        n *= reps
    return n / dt, n, dt


def cpu_baseline_record(w, inp, budget_s: float, table=None, table_desc: str = "") -> dict:
    """The oracle on all host cores and on one core, reading the materialised table when one
    is given (the rows a CPU lookup would read), plus, as a secondary labelled figure, the
    oracle regenerating its rows from their definition.  Tokens/s and the algorithmic GB/s."""
    threads = os.cpu_count() or 1
    per_tok = algorithmic_bytes(w) / w.N
    src = "materialised" if table is not None else "regenerated"
    v, n, dt = oracle_tokens_per_s(w, inp, budget_s, threads, table=table)
    v1, n1, dt1 = oracle_tokens_per_s(w, inp, min(3.0, budget_s / 4), 1, seed=1, table=table)
    rec = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "row_source": src,
           "gbs": v * per_tok / 1e9,
           "sample": "%d tokens of this %d-token workload (repeated passes when one pass is short), "
                     "%.1f s, rows read from %s" % (
               n, w.N, dt, table_desc if table is not None else
               "their synthetic-table definition (regenerated per element)"),
           "single_thread": {"value": v1, "unit": UNIT, "cores": 1, "gbs": v1 * per_tok / 1e9,
                             "sample": "%d tokens, %.1f s" % (n1, dt1)}}
    if table is not None:
        vr, nr, dtr = oracle_tokens_per_s(w, inp, min(5.0, budget_s / 3), threads, seed=2)
        rec["regenerated_rows"] = {"value": vr, "unit": UNIT, "cores": threads,
                                   "gbs": vr * per_tok / 1e9,
                                   "sample": "%d tokens, %.1f s, rows regenerated from their "
                                             "definition (Philox-bound, secondary)" % (nr, dtr)}
    return rec


# --------------------------------------------------------------------------- arms
def run_reference(args, w):
    """The oracle on the host cores, as the reference arm: each step is a bounded
    sample of the workload's tokens (rank 0 only)."""
    import oracle  # noqa: F401
    threads = os.cpu_count() or 1
    inp = gen.make_inputs(w)
    total_budget = args.reference_seconds
    steps, warm = args.steps, args.warmup
    per_step_budget = total_budget / max(1, steps + warm)
    _, n_probe, dt_probe = oracle_tokens_per_s(w, inp, min(2.0, per_step_budget), threads)
    per_tok = dt_probe / n_probe
    n_step = int(max(1, min(w.N, per_step_budget / per_tok)))
    rng = np.random.default_rng(7)
    import oracle as orc
    kw = dict(R=w.R, d=w.d, dtype=oracle_dtype(w),
              table_seed=gen.TABLE_SEED, acc=orc.ACC_F32, n_threads=threads, vocab_size=w.vocab)
    sels = [np.sort(rng.choice(w.N, size=n_step, replace=False)) for _ in range(steps + warm)]
    for i in range(warm):
        orc.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"], sel=sels[i], **kw)
    t0 = time.perf_counter()
    for i in range(warm, warm + steps):
        orc.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"], sel=sels[i], **kw)
    dt = time.perf_counter() - t0
    value = n_step * steps / dt
    sample = "%d of %d tokens per step (rows regenerated from the synthetic-table definition)" % (
        n_step, w.N)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": 1e3 * dt / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": config_for(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def resolved_launch(w, args) -> str:
    """eager launches, or CUDA graphs of 100 steps (auto: graphs for N <= 1024 tokens)."""
    return args.launch if args.launch != "auto" else ("graph" if w.N <= 1024 else "eager")


def config_for(w, args) -> dict:
    return {
        "workload": w.name, "R": w.R, "d": w.d, "table_dtype": w.dtype,
        "table_gib": round(w.R * stored_row_bytes(w) / 2**30, 2), "n_seq": w.n_seq, "T": w.T,
        "tokens_per_step_per_gpu": w.N, "heads": "8 bigram + 8 trigram",
        "tokens": "%s over vocab %d" % ("Zipf(1.1)" if w.tokens == "zipf" else "uniform", w.vocab),
        "accumulate": "fp32, head order", "residency": "hbm", "variant": args.variant,
        "l2": "inputs larger than L2: %.2f GB moved per step, %d token batches cycle (their rows "
              "span %.0f MB) vs 126 MB L2" % (algorithmic_bytes(w) / 1e9, max(args.batches, batches_for(w)),
                                              max(args.batches, batches_for(w)) * w.N * HEADS * row_bytes(w) / 1e6),
        "parallelism": "replicas x%d (tokens sharded, table replicated)" % args.gpus,
        "launch": resolved_launch(w, args),
    }


def make_table(ng, w, dev):
    """The workload's synthetic table in HBM (set-up, untimed): (dtype, table, scale)."""
    import torch
    dtype = {"bf16": ng.NGRAM_BF16, "int8": ng.NGRAM_INT8_ROWSCALE,
             "fp8": ng.NGRAM_FP8_E4M3_ROWSCALE, "nvfp4": ng.NGRAM_NVFP4}[w.dtype]
    table = torch.empty((w.R, ng.ngram_row_bytes(dtype, w.d)), dtype=torch.uint8, device=dev)
    scale = None
    if dtype != ng.NGRAM_BF16:     # per-row scales, or the one NVFP4 global scale
        scale = torch.empty((1 if dtype == ng.NGRAM_NVFP4 else w.R,), dtype=torch.float32, device=dev)
    ng.ngram_fill_synthetic(table, w.R, w.d, dtype, gen.TABLE_SEED, row_scale=scale)
    return dtype, table, scale


L2_BYTES = 126 * 10**6          # B200 L2


def batches_for(w, minimum: int = 2) -> int:
    """Token batches a timed loop cycles through: enough that the rows they read (16 per
    token) span twice the L2, so that no batch finds its rows left in L2 by its previous
    turn (decode batches are small: 82 KB of rows for one token)."""
    per = w.N * HEADS * row_bytes(w)
    return max(minimum, -(-2 * L2_BYTES // per))


class Batches:
    """One rank's token batches (distinct seeds per rank and batch) and the activations of
    a workload, on the host and on the device.  per_batch: every batch has its own residual
    and output rows too (used when many small batches cycle, so that the activations do not
    stay in L2 either); else one residual and one output serve every batch."""

    def __init__(self, w, dev, rank=0, batches=2, token_gate=False, per_batch=False):
        import torch
        self.host_tok, self.host_hist = [], []
        for b in range(batches):
            ts, hs = rank_seeds(rank, b)
            self.host_tok.append(gen.tokens_for(w, ts))
            self.host_hist.append(gen.history_for(w, hs))
        self.res_bits = gen.residual_bf16_bits(w.N, w.d, gen.RESIDUAL_SEED + rank)
        self.gate_h = gen.gate_f32(w.d)
        tok_all = torch.from_numpy(np.stack(self.host_tok)).to(dev)
        self.tok_d = [tok_all[b] for b in range(batches)]
        if w.history:
            hist_all = torch.from_numpy(np.stack(self.host_hist)).to(dev)
            self.hist_d = [hist_all[b] for b in range(batches)]
        else:
            self.hist_d = [None] * batches
        self.res_cpu = torch.from_numpy(self.res_bits.view(np.int16)).view(torch.bfloat16).view(w.N, w.d)
        self.residual = self.res_cpu.to(dev)
        self.out = torch.empty_like(self.residual)
        n_act = batches if per_batch else 1
        if per_batch:
            bits = gen.residual_bf16_bits(n_act * w.N, w.d, gen.RESIDUAL_SEED + 1000 + rank)
            res_all = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).view(n_act, w.N, w.d).to(dev)
            out_all = torch.empty_like(res_all)
            self.res_b = [res_all[b] for b in range(n_act)]
            self.out_b = [out_all[b] for b in range(n_act)]
        else:
            self.res_b, self.out_b = [self.residual], [self.out]
        self.gate = torch.from_numpy(self.gate_h).to(dev)
        if token_gate:                      # one bf16 gate per token and column
            g = np.random.default_rng(12).uniform(0, 1, (w.N, w.d)).astype(np.float32)
            self.gate = torch.from_numpy(g).to(torch.bfloat16).to(dev)
        self.n = batches

    def inputs(self, b=0):
        return {"tokens": self.host_tok[b], "history": self.host_hist[b], "residual": self.res_bits,
                "gate": self.gate_h}


def time_forward(ng, ctx, bt, stream, steps, warmup, launch, dev, barrier=lambda: None, G=100):
    """W untimed warm-up steps, then K timed steps bracketed by a barrier and a
    synchronize; step i uses token batch i % B (and its own activations when bt has them).
    Eager: one ngram_forward per step, CUDA events around each launch.  Graph: the steps
    are captured in CUDA graphs of G steps (ceil(B / G) graphs, so every batch is used) and
    replayed in turn, events around each replay (decode-sized launches are otherwise bound
    by the Python launch path).  Returns (elapsed_ms, kernel ms per step, K, clocks)."""
    import torch

    def step(i, s=None):
        b = i % bt.n
        a = b % len(bt.res_b)
        ng.ngram_forward(ctx, bt.tok_d[b], bt.res_b[a], bt.gate, out=bt.out_b[a], history=bt.hist_d[b],
                         stream=s if s is not None else stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    K = steps
    graphs = []
    if launch == "graph":
        n_graphs = -(-bt.n // G)
        K = max(G * n_graphs, -(-K // (G * n_graphs)) * G * n_graphs)
        for j in range(n_graphs):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                cap = torch.cuda.current_stream()
                for i in range(G):
                    step(j * G + i, cap)
            graphs.append(gr)
        for gr in graphs:
            gr.replay()
        torch.cuda.synchronize()
    n_ev = K if not graphs else K // G
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id_for(dev)) as clk:
        barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(n_ev):
            ev_s[i].record(stream)
            if not graphs:
                step(i)
            else:
                graphs[i % len(graphs)].replay()
            ev_e[i].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
    elapsed_ms = t0.elapsed_time(t1)
    kern_ms = statistics.fmean(ev_s[i].elapsed_time(ev_e[i]) for i in range(n_ev))
    if graphs:
        kern_ms /= G                          # per step inside the graph (kernel + gap)
        del graphs
    return elapsed_ms, kern_ms, K, clk.summary()


def distinct_bytes(w, unique_rows: int) -> int:
    """The least DRAM traffic of one launch whatever the order or reuse: every distinct row
    once, the residual read and output write per token, the token ids and the gate."""
    return unique_rows * row_bytes(w) + w.N * (2 * 2 * w.d + 4) + 4 * w.d


PROFILE_FOR = {"full_prefill": "gather_bf16_prefill", "int8_uniform": "gather_int8_uniform",
               "fp8_prefill": "gather_fp8_prefill", "nvfp4_prefill": "gather_nvfp4_prefill"}


def profiled_traffic(workload: str, dtype: str, distinct: int, n_tokens: int):
    """DRAM bytes per launch, estimated from the committed ncu summary of a small case of the
    same kernel in the same launch configuration (profiles/<kernel>_<workload>.txt), if it was
    taken on the kernel code as it is now (its kernel_sha line, first word).  The summary
    names its scaling:
      per_token       the small case is the same token batch on a smaller table: its DRAM
                      bytes per token times this launch's tokens;
      distinct_ratio  the small case has fewer tokens (uniform ids: row reuse comes only from
                      hash collisions): its DRAM bytes over its distinct bytes, times this
                      launch's distinct bytes.
    Returns (bytes, source) or (None, reason)."""
    name = PROFILE_FOR.get(workload)
    if name is None:
        return None, "no small-case profile for this workload"
    p = os.path.join(ROOT, "profiles", name + ".txt")
    if not os.path.exists(p):
        return None, "profiles/%s.txt missing" % name
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith(" "):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if (kv.get("kernel_sha", "").split() or [""])[0] != kernel_sha(dtype):
        return None, "profiles/%s.txt was taken on other kernel code" % name
    try:
        dram = float(kv["small_dram_bytes_per_launch"].split()[0])
        small_distinct = float(kv["small_distinct_bytes_per_launch"].split()[0])
        small_tokens = float(kv["small_tokens"].split()[0])
        scaling = kv["scaling"].split()[0]
    except (KeyError, ValueError, IndexError):
        return None, "profiles/%s.txt lacks the small-case figures" % name
    small = kv.get("small_workload", "?").split(" ")[0]
    if scaling == "per_token":
        return dram / small_tokens * n_tokens, (
            "ncu DRAM bytes of %s (%s): %.0f per token, times this launch's %d tokens" % (
                small, name, dram / small_tokens, n_tokens))
    if scaling == "distinct_ratio":
        return dram / small_distinct * distinct, (
            "ncu DRAM bytes of %s (%s) over its distinct bytes = %.4f, times this launch's "
            "distinct bytes" % (small, name, dram / small_distinct))
    return None, "profiles/%s.txt names an unknown scaling %r" % (name, scaling)


def hbm_record(ng, dev, w, dtype, table, scale, steps, launch, read_gbs=None, flags=0) -> dict:
    """One workload on an HBM-resident table, timed like the headline (bounded steps), as a
    sub-record of the bench line: tokens/s, the roofline against the measured copy peak,
    the clocks sampled during its timed region and the device error word."""
    import torch
    hp = ng.ngram_default_hash_params(vocab_size=w.vocab, flags=flags)
    ctx = ng.ngram_init(table, w.R, w.d, dtype, ng.NGRAM_RES_HBM, hp, w.N, row_scale=scale)
    nb = batches_for(w)
    bt = Batches(w, dev, batches=nb, per_batch=nb > 2)
    stream = torch.cuda.current_stream()
    elapsed_ms, kern_ms, K, clocks = time_forward(ng, ctx, bt, stream, steps, 5, launch, dev)
    st, info = ng.ngram_get_device_error(ctx)
    _, _, ucount = ng.ngram_dedup_rows(ctx, bt.tok_d[0], history=bt.hist_d[0])
    U = int(ucount.item())
    ctx.close()
    peaks = measured_peaks()
    nbytes = algorithmic_bytes(w)
    dist_b = distinct_bytes(w, U)
    achieved = nbytes / (kern_ms / 1e3) / 1e9
    traffic, tsrc = profiled_traffic(w.name, w.dtype, dist_b, w.N)
    rec = {
        "workload": w.name,
        "config": {"R": w.R, "d": w.d, "table_dtype": w.dtype, "n_seq": w.n_seq, "T": w.T,
                   "tokens": "%s over vocab %d" % ("Zipf(1.1)" if w.tokens == "zipf" else "uniform", w.vocab),
                   "history": w.history, "residency": "hbm", "launch": launch,
                   "table_gib": round(w.R * stored_row_bytes(w) / 2**30, 2),
                   "l2": "%d token batches cycle%s: their rows span %.0f MB, over twice the 126 MB L2" % (
                       nb, " (each with its own residual and output rows)" if nb > 2 else "",
                       nb * w.N * HEADS * row_bytes(w) / 1e6)},
        "value": w.N * K / (elapsed_ms / 1e3), "unit": UNIT, "ms_per_step": elapsed_ms / K,
        "kernel_ms": kern_ms, "steps": K,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "traffic_source": tsrc,
                     "algorithmic_bytes_per_launch": nbytes, "unique_rows": U,
                     "unique_row_bytes": U * row_bytes(w), "distinct_bytes_per_launch": dist_b,
                     "frac_on_distinct_bytes": dist_b / (kern_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)"},
        "clocks": clocks,
        "device_error": "ok" if st == ng.NGRAM_OK else str(info),
    }
    if read_gbs:
        rec["roofline"]["frac_of_read_stream"] = achieved / read_gbs
    if launch == "graph":
        rec["us_per_step"] = kern_ms * 1e3
        if clocks.get("sm_mhz"):
            rec["kcycles_per_step"] = kern_ms * clocks["sm_mhz"]      # us x MHz / 1000
    return rec


def host_mem_available() -> int:
    """MemAvailable of this host in bytes (0 if unknown)."""
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    return int(line.split()[1]) * 1024
    except OSError:
        pass
    return 0


def run_extras(args, ng, dev, full, bt_full, read_gbs, line):
    """The other configurations on one GPU, each a sub-record of the bench line (bounded:
    fixed step counts, tables filled once).  Called after the headline with the full bf16
    table still resident: mid, the decode batches and the backward; then the host-resident
    configuration and the CPU baseline on the same materialised host table; then the 8- and
    4-bit tables, after the bf16 table is released."""
    import gc

    import torch
    t_start = time.perf_counter()
    W = gen.WORKLOADS
    extra = []
    dtype, table, scale = full
    full.clear()
    # ---- mid (its own 9.5 GiB table), the decode batches and the backward on the full table
    mid = W["mid"]
    mdt, mtab, msc = make_table(ng, mid, dev)
    extra.append(hbm_record(ng, dev, mid, mdt, mtab, msc, 400, "eager", read_gbs))
    if not args.no_cpu_baseline:        # the oracle on a host copy of mid's 9.5 GiB table
        host_mid = mtab.view(torch.int16).cpu().numpy().view(np.uint16).reshape(mid.R, mid.d)
        extra[-1]["cpu_baseline"] = cpu_baseline_record(
            mid, gen.make_inputs(mid), min(args.cpu_seconds, 8.0), table=host_mid,
            table_desc="a host copy of the 2,000,000 x 2560 bf16 table (9.5 GiB)")
        del host_mid
    del mtab, msc
    gc.collect()
    torch.cuda.empty_cache()
    for n in (1, 16, 64, 256):
        extra.append(hbm_record(ng, dev, W["full_decode_%d" % n], dtype, table, scale, 20_000, "graph"))
    fw = W["full_prefill"]
    ctx = ng.ngram_init(table, fw.R, fw.d, dtype, ng.NGRAM_RES_HBM,
                        ng.ngram_default_hash_params(vocab_size=fw.vocab), fw.N)
    bw = backward_record(ng, dev, fw, ctx, 2, 100, 5)
    ctx.close()
    del ctx
    bw.update(workload="full_prefill_backward",
              config={"R": fw.R, "d": fw.d, "table_dtype": "bf16", "n_seq": fw.n_seq, "T": fw.T,
                      "mode": "backward: table gradient + shared-gate gradient"})
    extra.append(bw)
    # ---- the host-resident configuration, then the CPU baseline on the same materialised table
    host_bytes = fw.R * fw.d * 2
    avail = host_mem_available()
    ht = None
    if avail >= host_bytes + (24 << 30):
        t0 = time.perf_counter()
        ht = ng.HostTable((fw.R, fw.d), torch.bfloat16)
        pin_s = time.perf_counter() - t0
        t0 = time.perf_counter()
        ng.ngram_fill_synthetic(ht.tensor, fw.R, fw.d, ng.NGRAM_BF16, gen.TABLE_SEED)
        torch.cuda.synchronize()
        fill_s = time.perf_counter() - t0
    else:
        pin_s = fill_s = None
    if ht is not None:
        with ClockSampler(gpu_id_for(dev)) as clk:
            report, h2d, gemm_ms, gemm_tflops = host_modes(
                ng, ht, fw.R, fw.d, ["host_decode_256", "host_prefill"], dev, 200,
                modes=("uva", "uva_dedup", "dma", "auto"))
        clocks = clk.summary()
        for name, entry in report.items():
            hw = W[name]
            best = entry["auto"]
            extra.append({
                "workload": name,
                "config": {"R": fw.R, "d": fw.d, "table_dtype": "bf16", "n_seq": hw.n_seq, "T": hw.T,
                           "residency": "host (pinned, mapped)", "pin_s": pin_s, "fill_s": fill_s,
                           "stand_in": "bf16 [4096x2560]x[2560x2560] GEMM looped on a second stream"},
                "value": best["tokens_per_s"], "unit": UNIT, "ms_per_step": best["ms"],
                "steps": entry["steps"], "mode": "auto (chose %s)" % best.get("choice"),
                "roofline": {"bound": "pcie_h2d", "achieved": best["nominal_row_gbs"], "peak": h2d,
                             "unit": "GB/s", "frac": best["nominal_row_gbs"] / h2d,
                             "nominal_bytes": "16 x 5120 B per token, every mode",
                             "peak_source": "measured in this run: pinned 1 GiB cudaMemcpyAsync, best of 10"},
                "modes": {m: entry[m] for m in ("uva", "uva_dedup", "dma", "auto")},
                "overlap": {"gemm_alone_tflops": gemm_tflops, "gemm_alone_ms": gemm_ms,
                            "per_mode": {m: {"lookup_alone_ms": entry[m]["ms"],
                                             "lookup_overlapped_ms": entry[m]["overlapped_ms"],
                                             "gemm_tflops_overlapped": entry[m]["gemm_tflops_overlapped"]}
                                         for m in ("uva", "uva_dedup", "dma", "auto")}},
                "prefetch": entry.get("prefetch"),
                "clocks": clocks,
                "device_error": "ok" if all(entry[m]["device_error"] == ng.NGRAM_OK
                                            for m in ("uva", "uva_dedup", "dma", "auto")) else "set",
            })
    # the oracle reads the materialised table after the host-resident timings: rows it leaves in
    # the CPU caches would slow the GPU's reads of them over PCIe
    if not args.no_cpu_baseline:
        tab = None if ht is None else ht.tensor.view(torch.int16).numpy().view(np.uint16)
        line["cpu_baseline"] = cpu_baseline_record(
            fw, bt_full.inputs(0), args.cpu_seconds, table=tab,
            table_desc="the materialised 20,000,000 x 2560 bf16 table (95.4 GiB, pinned host memory)")
        if ht is None:
            line["cpu_baseline"]["note"] = ("host RAM too small for the 95.4 GiB table (%.1f GiB "
                                            "available): rows regenerated" % (avail / 2**30))
        del tab                               # a view of the pinned table: gone before close()
    if ht is not None:
        ht.close()
    else:
        extra.append({"workload": "host_prefill", "skipped": "host RAM: %.1f GiB available, the table "
                                                             "needs 95.4 GiB + 24 GiB margin" % (avail / 2**30)})
    # ---- the 8- and 4-bit tables (the bf16 table is released first)
    del table, scale
    gc.collect()
    torch.cuda.empty_cache()
    for name in ("int8_uniform", "fp8_prefill", "nvfp4_prefill"):
        lw = W[name]
        ldt, ltab, lsc = make_table(ng, lw, dev)
        extra.append(hbm_record(ng, dev, lw, ldt, ltab, lsc, 200, "eager"))
        del ltab, lsc
        gc.collect()
        torch.cuda.empty_cache()
    line["extra"] = extra
    line["extra_wall_s"] = time.perf_counter() - t_start


def run_ours(args, w):
    import datetime

    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_ngram_b200 as ng

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the lookup has no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- table (set-up, untimed): a replica of the whole table on every GPU
    dtype, table, scale = make_table(ng, w, dev)
    flags = {"default": 0, "dedup": ng.NGRAM_FLAG_DEDUP, "tma": ng.NGRAM_FLAG_TMA_STAGING,
             "sort": ng.NGRAM_FLAG_SORT, "batch_order": ng.NGRAM_FLAG_BATCH_ORDER,
             "token_gate": ng.NGRAM_FLAG_TOKEN_GATE}[args.variant]
    grouped = args.variant == "sort" or (args.variant in ("default", "token_gate")
                                         and w.N >= ng.NGRAM_SORT_MIN_TOKENS)
    # grouped bf16 / NVFP4 batches of >= 4096 tokens hash every token once, in the order
    # step's count kernel, and the gather reads the row ids
    prehash = grouped and w.dtype in ("bf16", "nvfp4") and w.N >= 4096
    hp = ng.ngram_default_hash_params(vocab_size=w.vocab, flags=flags)
    ctx = ng.ngram_init(table, w.R, w.d, dtype, ng.NGRAM_RES_HBM, hp, w.N, row_scale=scale)

    # ---- inputs: this rank's token batches (distinct seeds per rank and batch)
    nb = max(args.batches, batches_for(w))
    bt = Batches(w, dev, rank, nb, token_gate=args.variant == "token_gate", per_batch=nb > args.batches)
    stream = torch.cuda.current_stream()

    # ---- distinct rows of the first batch (outside any timed region): U * row bytes is the
    # least a lookup of this batch can read from the table, whatever the order or reuse
    _, _, ucount = ng.ngram_dedup_rows(ctx, bt.tok_d[0], history=bt.hist_d[0])
    unique_rows = int(ucount.item())
    read_gbs = read_stream_gbs(dev)

    # ---- device-resident timing
    launch = resolved_launch(w, args)
    elapsed_ms, kern_ms, K, clocks = time_forward(ng, ctx, bt, stream, args.steps, args.warmup,
                                                  launch, dev, barrier)
    st, info = ng.ngram_get_device_error(ctx)
    if st != ng.NGRAM_OK:
        raise SystemExit("device error word set: %s" % info)

    # ---- end to end through the host-buffer call: every step moves its tokens and
    # residual from pinned host memory to the device and its output back to the host
    # (ngram_forward_host pipelines the copies with the gather in ~8 MB chunks)
    tok_h = [torch.from_numpy(t).pin_memory() for t in bt.host_tok[:64]]
    hist_h = [None if h is None else torch.from_numpy(h).pin_memory() for h in bt.host_hist[:64]]
    res_h = bt.res_cpu.pin_memory()
    out_h = torch.empty_like(res_h).pin_memory()
    gate_h_tok = bt.gate.cpu().pin_memory() if args.variant == "token_gate" else None
    E = max(1, args.e2e_steps)

    def e2e_step(i):
        b = i % len(tok_h)
        if args.variant == "default":
            ng.ngram_forward_host(ctx, tok_h[b], res_h, bt.gate, out=out_h, history=hist_h[b],
                                  stream=stream)
        else:                                 # staged variants: copy in, forward, copy out
            bt.tok_d[b].copy_(tok_h[b], non_blocking=True)
            if hist_h[b] is not None:
                bt.hist_d[b].copy_(hist_h[b], non_blocking=True)
            bt.residual.copy_(res_h, non_blocking=True)
            if gate_h_tok is not None:        # a per-token gate is an activation: it comes in too
                bt.gate.copy_(gate_h_tok, non_blocking=True)
            ng.ngram_forward(ctx, bt.tok_d[b], bt.residual, bt.gate, out=bt.out, history=bt.hist_d[b],
                             stream=stream)
            out_h.copy_(bt.out, non_blocking=True)

    for i in range(min(3, E)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(E):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    h2d = w.N * 4 + (w.n_seq * 8 if w.history else 0) + w.N * w.d * 2 * (2 if args.variant == "token_gate" else 1)
    d2h = w.N * w.d * 2
    bidir = measure_bidir_gbs(dev) if rank == 0 else (0.0, 0.0)

    # ---- max over ranks
    elapsed_ms, kern_ms, e2e_ms = max_over_ranks([elapsed_ms, kern_ms, e2e_ms], world, dev)

    if rank == 0:
        value = weak_scaling_tokens_per_s(world, w.N, K, elapsed_ms)
        e2e_value = weak_scaling_tokens_per_s(world, w.N, E, e2e_ms)
        # the PCIe bound of a call: its input and output bytes at the rates measured with both
        # directions busy at once (one GPU's link; every rank has its own)
        bound_ms = max(h2d / bidir[0], d2h / bidir[1]) / 1e6 if min(bidir) > 0 else None
        peaks = measured_peaks()
        bytes_launch = algorithmic_bytes(w) + (w.N * 2 * w.d if args.variant == "token_gate" else 0)
        achieved = bytes_launch / (kern_ms / 1e3) / 1e9
        dist_b = distinct_bytes(w, unique_rows)
        traffic, tsrc = (profiled_traffic(w.name, w.dtype, dist_b, w.N) if args.variant == "default"
                         else (None, "variant %s: not profiled" % args.variant))
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": config_for(w, args),
            "gather_gbs": bytes_launch * world * K / (elapsed_ms / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": traffic, "traffic_source": tsrc,
                         "kernel": ("hash + dedup + compact + gather (8 kernels)" if args.variant == "dedup"
                                    else "k_gather_bf16_bulk<16>" if args.variant == "tma"
                                    else ("grouped order (3 kernels%s) + " % (
                                        ", row ids hashed once" if prehash else "") if grouped else "")
                                    + KERNEL_NAME[w.dtype]),
                         "kernel_ms": kern_ms, "algorithmic_bytes_per_launch": bytes_launch,
                         "unique_rows": unique_rows,
                         "unique_row_bytes": unique_rows * row_bytes(w),
                         "distinct_bytes_per_launch": dist_b,
                         "frac_on_distinct_bytes": dist_b / (kern_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "read_stream_gbs": read_gbs, "frac_of_read_stream": achieved / read_gbs,
                         "frac_of_8tbs_nominal": achieved / 8000.0,
                         "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": E,
                    "pcie_both_directions_gbs": {"h2d": bidir[0], "d2h": bidir[1]},
                    "pcie_bound_tokens_per_s": (w.N * world / (bound_ms / 1e3)) if bound_ms else None,
                    "frac_of_pcie_bound": (bound_ms / (e2e_ms / E)) if bound_ms else None,
                    "path": ("ngram_forward_host: pinned host tokens + residual in, bf16 out "
                             "back to pinned host, chunked H2D / gather / D2H on 3 streams")
                    if args.variant == "default" else
                            "pinned host tokens + residual -> device, ngram_forward, out -> pinned host"},
            "clocks": clocks,
            "gpu_launches": K * (8 if args.variant == "dedup" else 4 if grouped else 1),
        }
        extras = (world == 1 and not args.no_extra and args.variant == "default"
                  and w.name == "full_prefill")
        ctx.close()
        ctx = None                            # the context object holds the table too
        if extras:
            full = [dtype, table, scale]      # run_extras releases the bf16 table midway
            del table, scale
            run_extras(args, ng, dev, full, bt, read_gbs, line)
        elif world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_record(w, bt.inputs(0), args.cpu_seconds)
        print(json.dumps(line), flush=True)
    else:
        ctx.close()
    if world > 1:
        dist.destroy_process_group()


def measure_bidir_gbs(dev, nbytes=1 << 30, reps=5):
    """Best-of-N pinned copies in both directions at once (H2D on one stream, D2H on
    another, from a common start): (H2D GB/s, D2H GB/s) -- the PCIe bound of a call that
    moves its inputs in and its outputs out."""
    import torch
    src_h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst_h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    a_d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    b_d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    best = (0.0, 0.0)
    for _ in range(reps):
        start = torch.cuda.Event(enable_timing=True)
        e1, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record()
        s1.wait_event(start)
        s2.wait_event(start)
        with torch.cuda.stream(s1):
            a_d.copy_(src_h, non_blocking=True)
            e1.record(s1)
        with torch.cuda.stream(s2):
            dst_h.copy_(b_d, non_blocking=True)
            e2.record(s2)
        torch.cuda.synchronize()
        h2d = nbytes / (start.elapsed_time(e1) / 1e3) / 1e9
        d2h = nbytes / (start.elapsed_time(e2) / 1e3) / 1e9
        if min(h2d, d2h) > min(best):
            best = (h2d, d2h)
    del src_h, dst_h, a_d, b_d
    torch.cuda.empty_cache()
    return best


def measure_h2d_gbs(dev, nbytes=1 << 30, reps=10) -> float:
    """Best-of-N pinned host -> device copy bandwidth (GB/s), the PCIe roofline."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    best = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) / 1e3) / 1e9)
    return best


def prefetch_pipeline(ng, ht, R, d, w, gemm_ms, time_gemms, main_s, dev, A, B):
    """Prefetch pattern on the host-resident table: step i runs its compute (g stand-in
    GEMMs) and its lookup from HBM staging on the main stream while batch i+1's rows are
    staged from host memory on a side stream.  Compared with the same steps doing the
    UVA lookup inline, and with the compute alone."""
    import math

    import torch
    side = torch.cuda.Stream()
    hp = ng.ngram_default_hash_params(vocab_size=w.vocab)
    ctx = ng.ngram_init(ht.tensor, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HOST_UVA, hp, w.N)
    bt = []
    for b in range(2):
        inp = gen.make_inputs(w, token_seed=500 + b)
        bt.append((torch.from_numpy(inp["tokens"]).to(dev),
                   None if inp["history"] is None else torch.from_numpy(inp["history"]).to(dev)))
    res = torch.from_numpy(gen.residual_bf16_bits(w.N, d).view(np.int16)).view(torch.bfloat16).view(w.N, d).to(dev)
    gate = torch.from_numpy(gen.gate_f32(d)).to(dev)
    out = torch.empty_like(res)
    K = max(5, min(100, int(5e4 / w.N)))

    def timed(fn, n):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main_s)
        for i in range(n):
            fn(i)
        b.record(main_s)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    for i in range(2):
        ng.ngram_prefetch(ctx, i, *bt[i], stream=main_s)
    pf_ms = timed(lambda i: ng.ngram_prefetch(ctx, i % 2, *bt[i % 2], stream=main_s), K)
    st_ms = timed(lambda i: ng.ngram_forward_staged(ctx, i % 2, res, gate, out=out, stream=main_s), K)
    g = max(1, math.ceil(pf_ms / gemm_ms))

    def compute():
        for _ in range(g):
            torch.matmul(A, B)

    comp_ms = timed(lambda i: compute(), K)
    inline_ms = timed(lambda i: (compute(), ng.ngram_forward(ctx, bt[i % 2][0], res, gate, out=out,
                                                             history=bt[i % 2][1], stream=main_s)), K)
    ev_pf = [torch.cuda.Event(), torch.cuda.Event()]
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]
    ng.ngram_prefetch(ctx, 0, *bt[0], stream=main_s)
    ev_pf[0].record(main_s)

    def step(i):
        cur, nxt = i % 2, (i + 1) % 2
        side.wait_event(ev_used[nxt])             # the slot's previous lookup is done
        ng.ngram_prefetch(ctx, nxt, *bt[nxt], stream=side)
        ev_pf[nxt].record(side)
        compute()
        main_s.wait_event(ev_pf[cur])
        ng.ngram_forward_staged(ctx, cur, res, gate, out=out, stream=main_s)
        ev_used[cur].record(main_s)

    piped_ms = timed(step, K)
    ctx.close()
    return {"prefetch_ms": pf_ms, "staged_lookup_ms": st_ms, "gemms_per_step": g,
            "compute_only_ms": comp_ms, "step_inline_uva_ms": inline_ms,
            "step_prefetched_ms": piped_ms,
            "lookup_on_critical_path_ms": piped_ms - comp_ms}


HOST_MODES = ("uva", "uva_grouped", "uva_dedup", "dma", "auto")


def host_modes(ng, ht, R, d, names, dev, host_steps, modes=HOST_MODES, prefetch=True):
    """Each host workload in each residency mode: time alone (K calls, CUDA events; wall
    time for the host-blocking DMA mode), time again while a stand-in bf16
    [4096 x 2560] x [2560 x 2560] GEMM loops on a second stream, check bit-identity with
    the first mode and the device error word; then the prefetch pattern.  Returns
    (report, h2d GB/s, GEMM ms alone, GEMM TFLOP/s alone)."""
    import torch
    h2d = measure_h2d_gbs(dev)
    main_s = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    A = torch.randn(4096, 2560, dtype=torch.bfloat16, device=dev)
    B = torch.randn(2560, 2560, dtype=torch.bfloat16, device=dev)
    gemm_flop = 2.0 * 4096 * 2560 * 2560

    def time_gemms(n):
        with torch.cuda.stream(side):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(side)
            for _ in range(n):
                torch.matmul(A, B)
            b.record(side)
        return a, b

    with torch.cuda.stream(side):          # warm cuBLAS on the stream it is timed on
        for _ in range(30):
            torch.matmul(A, B)
    torch.cuda.synchronize()
    a, b = time_gemms(200)
    torch.cuda.synchronize()
    gemm_ms = a.elapsed_time(b) / 200
    report = {}
    table = {"uva": (ng.NGRAM_RES_HOST_UVA, 0), "uva_grouped": (ng.NGRAM_RES_HOST_UVA, ng.NGRAM_FLAG_SORT),
             "uva_dedup": (ng.NGRAM_RES_HOST_UVA, ng.NGRAM_FLAG_DEDUP),
             "dma": (ng.NGRAM_RES_HOST_DMA, 0), "auto": (ng.NGRAM_RES_HOST_AUTO, 0)}
    for name in names:
        w = gen.WORKLOADS[name]
        inp = gen.make_inputs(w)
        tok = torch.from_numpy(inp["tokens"]).to(dev)
        hist = None if inp["history"] is None else torch.from_numpy(inp["history"]).to(dev)
        res = torch.from_numpy(inp["residual"].view(np.int16)).view(torch.bfloat16).view(w.N, w.d).to(dev)
        gate = torch.from_numpy(inp["gate"]).to(dev)
        out = torch.empty_like(res)
        K = max(5, min(host_steps, int(2e5 / w.N)))
        row_bytes = HEADS * 2 * w.d * w.N               # nominal row bytes per call
        entry = {"N": w.N, "steps": K}
        ref = None
        for mname in modes:
            where, flags = table[mname]
            hp = ng.ngram_default_hash_params(vocab_size=w.vocab, flags=flags)
            ctx = ng.ngram_init(ht.tensor, R, d, ng.NGRAM_BF16, where, hp, w.N)
            for _ in range(3):
                ng.ngram_forward(ctx, tok, res, gate, out=out, history=hist, stream=main_s)
            torch.cuda.synchronize()
            # host-blocking modes count wall time: DMA, and AUTO once it has picked DMA
            blocking = mname == "dma" or (where == ng.NGRAM_RES_HOST_AUTO and
                                          ng.ngram_auto_choice(ctx, w.N) == ng.NGRAM_RES_HOST_DMA)
            got = out.clone()
            if ref is None:
                ref = got
            same = bool(torch.equal(got.view(torch.int16), ref.view(torch.int16)))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            w0 = time.perf_counter()
            e0.record(main_s)
            for _ in range(K):
                ng.ngram_forward(ctx, tok, res, gate, out=out, history=hist, stream=main_s)
            e1.record(main_s)
            torch.cuda.synchronize()
            wall = (time.perf_counter() - w0) * 1e3 / K
            ms = max(e0.elapsed_time(e1) / K, wall if blocking else 0.0)
            # overlapped with the GEMM stand-in on the side stream
            n_gemm = max(1, int(ms * K / gemm_ms))
            ga, gb = time_gemms(n_gemm)
            o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            o0.record(main_s)
            for _ in range(K):
                ng.ngram_forward(ctx, tok, res, gate, out=out, history=hist, stream=main_s)
            o1.record(main_s)
            torch.cuda.synchronize()
            ms_ov = o0.elapsed_time(o1) / K
            gemm_ov_ms = ga.elapsed_time(gb) / n_gemm
            st, _ = ng.ngram_get_device_error(ctx)
            entry[mname] = {
                "ms": ms, "tokens_per_s": w.N / (ms / 1e3),
                "nominal_row_gbs": row_bytes / (ms / 1e3) / 1e9,
                "frac_of_h2d": row_bytes / (ms / 1e3) / 1e9 / h2d,
                "overlapped_ms": ms_ov, "gemm_tflops_overlapped": gemm_flop / (gemm_ov_ms / 1e3) / 1e12,
                "bit_identical_to_%s" % modes[0]: same, "device_error": st,
            }
            if where == ng.NGRAM_RES_HOST_AUTO:
                entry[mname]["choice"] = {ng.NGRAM_RES_HOST_UVA: "uva", ng.NGRAM_RES_HOST_DMA: "dma",
                                          ng.NGRAM_AUTO_UVA_DEDUP: "uva_dedup"}.get(
                    ng.ngram_auto_choice(ctx, w.N), "undecided")
            ctx.close()
        if prefetch:
            entry["prefetch"] = prefetch_pipeline(ng, ht, R, d, w, gemm_ms, time_gemms, main_s, dev, A, B)
        report[name] = entry
    return report, h2d, gemm_ms, gemm_flop / (gemm_ms / 1e3) / 1e12


def run_host(args):
    """Host-resident table: the 20M x 2560 bf16 table pinned in host memory, each host
    workload timed in UVA, DMA and AUTO residency, alone and overlapped with a stand-in
    bf16 [4096 x 2560] x [2560 x 2560] GEMM looped on a second stream."""
    import torch

    import hashed_gram_embedding_ngram_b200 as ng

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    names = args.host_workloads.split(",")
    R, d = gen.WORKLOADS[names[0]].R, gen.WORKLOADS[names[0]].d
    if args.host_rows:
        R = args.host_rows
    t0 = time.perf_counter()
    ht = ng.HostTable((R, d), torch.bfloat16)
    pin_s = time.perf_counter() - t0
    t0 = time.perf_counter()
    ng.ngram_fill_synthetic(ht.tensor, R, d, ng.NGRAM_BF16, gen.TABLE_SEED)
    torch.cuda.synchronize()
    fill_s = time.perf_counter() - t0
    with ClockSampler(gpu_id_for(dev)) as clk:
        report, h2d, gemm_ms, gemm_tflops = host_modes(ng, ht, R, d, names, dev, args.host_steps)
    head = names[-1]
    best = report[head]["auto"]
    line = {
        "metric": METRIC, "value": best["tokens_per_s"], "unit": UNIT, "n_gpus": 1,
        "steps": report[head]["steps"], "warmup": 3, "ms_per_step": best["ms"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": head, "R": R, "d": d, "residency": "host (pinned, mapped)",
                   "table_gib": round(R * d * 2 / 2**30, 2), "pin_s": pin_s, "fill_s": fill_s,
                   "stand_in": "bf16 [4096x2560]x[2560x2560] GEMM on a second stream"},
        "roofline": {"bound": "pcie_h2d", "achieved": best["nominal_row_gbs"], "peak": h2d,
                     "unit": "GB/s", "frac": best["nominal_row_gbs"] / h2d, "traffic": None,
                     "peak_source": "measured in this run: pinned 1 GiB cudaMemcpyAsync, best of 10"},
        "gemm_alone_tflops": gemm_tflops,
        "host_modes": report,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    ht.close()


def run_shard(args, w):
    """Column-sharded table (--variant shard): rank r of P holds columns [r d/P, (r+1) d/P)
    of every row; each step, every rank runs ngram_forward_shard on the whole batch, which
    stores its columns into every rank's output buffer through CUDA IPC mappings (the
    fused all-gather), between two one-element NCCL all-reduces that order the ranks.  The
    whole job computes one N-token batch per step (strong scaling).  With one GPU the one
    shard is the whole table and no collective runs."""
    import datetime

    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_ngram_b200 as ng
    from hashed_gram_embedding_ngram_b200 import shard

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    dtype = {"bf16": ng.NGRAM_BF16, "int8": ng.NGRAM_INT8_ROWSCALE,
             "fp8": ng.NGRAM_FP8_E4M3_ROWSCALE, "nvfp4": ng.NGRAM_NVFP4}[w.dtype]
    col0, d = shard.shard_columns(w.d, world, rank, dtype)
    table = torch.empty((w.R, ng.ngram_row_bytes(dtype, d)), dtype=torch.uint8, device=dev)
    scale = None
    if dtype != ng.NGRAM_BF16:
        scale = torch.empty((1 if dtype == ng.NGRAM_NVFP4 else w.R,), dtype=torch.float32, device=dev)
    ng.ngram_fill_synthetic_cols(table, w.R, d, col0, dtype, gen.TABLE_SEED, row_scale=scale)
    ctx = ng.ngram_init(table, w.R, d, dtype, ng.NGRAM_RES_HBM,
                        ng.ngram_default_hash_params(vocab_size=w.vocab), w.N, row_scale=scale)
    toks = [torch.from_numpy(gen.tokens_for(w, gen.TOKEN_SEED + b)).to(dev) for b in range(args.batches)]
    hists = [None if not w.history else torch.from_numpy(gen.history_for(w, gen.HISTORY_SEED + b)).to(dev)
             for b in range(args.batches)]
    res_cpu = torch.from_numpy(gen.residual_bf16_bits(w.N, w.d).view(np.int16)).view(torch.bfloat16).view(w.N, w.d)
    residual = res_cpu.to(dev)
    gate = torch.from_numpy(gen.gate_f32(w.d)).to(dev)
    if world > 1:
        peers = shard.PeerOutputs(w.N, w.d, device=dev)
        outs = peers.ptrs
        out = peers.out
    else:
        peers = None
        out = torch.empty_like(residual)
        outs = [out]
    stream = torch.cuda.current_stream()

    def order():
        if world > 1:
            shard.complete()

    def step(i):
        b = i % args.batches
        order()
        ng.ngram_forward_shard(ctx, toks[b], residual, gate, outs, w.d, col0, history=hists[b],
                               stream=stream)
        order()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id_for(dev)) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(K):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    elapsed_ms = max_over_ranks([t0.elapsed_time(t1)], world, dev)[0]
    # end to end: tokens and residual from pinned host memory, the output back
    tok_h = [t.cpu().pin_memory() for t in toks]
    res_h, out_h = res_cpu.pin_memory(), torch.empty_like(res_cpu).pin_memory()
    E = max(1, args.e2e_steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(E):
        b = i % args.batches
        toks[b].copy_(tok_h[b], non_blocking=True)
        residual.copy_(res_h, non_blocking=True)
        step(i)
        out_h.copy_(out[:w.N], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]
    if rank == 0:
        grouped = w.N >= ng.NGRAM_SORT_MIN_TOKENS
        line = {
            "metric": METRIC, "value": w.N * K / (elapsed_ms / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": dict(config_for(w, args), parallelism="column shard x%d, fused all-gather over "
                                                            "peer memory" % world, shard_columns=d),
            "e2e": {"value": w.N * E / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": w.N * 4 + w.N * w.d * 2,
                    "d2h_bytes_per_step": w.N * w.d * 2, "steps": E},
            "clocks": clk.summary(),
            "gpu_launches": K * (4 if grouped else 1),
        }
        print(json.dumps(line), flush=True)
    if peers is not None:
        dist.barrier()
        peers.close()
    if world > 1:
        dist.destroy_process_group()


def backward_record(ng, dev, w, ctx, batches, steps, warmup) -> dict:
    """The backward pass of the lookup on one batch: the table gradient
    (ngram_backward_rows) then the shared-gate gradient (ngram_backward_gate), CUDA events
    around each call; their algorithmic bytes and stream bounds."""
    import torch
    N, d, H = w.N, w.d, HEADS
    toks = [torch.from_numpy(gen.tokens_for(w, gen.TOKEN_SEED + b)).to(dev) for b in range(batches)]
    hists = [None if not w.history else torch.from_numpy(gen.history_for(w, gen.HISTORY_SEED + b)).to(dev)
             for b in range(batches)]
    rng = np.random.default_rng(11)
    dy = torch.from_numpy(rng.standard_normal((N, d), dtype=np.float32)).to(torch.bfloat16).to(dev)
    gate = torch.from_numpy(gen.gate_f32(d)).to(dev)
    uniq = torch.empty(N * H, dtype=torch.int32, device=dev)
    count = torch.empty(1, dtype=torch.int32, device=dev)
    grad_rows = torch.empty((N * H, d), dtype=torch.float32, device=dev)
    grad_gate = torch.empty(d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def rows(i):
        b = i % batches
        ng.ngram_backward_rows(ctx, toks[b], dy, gate, history=hists[b], uniq_out=uniq,
                               count_out=count, grad_rows=grad_rows, stream=stream)

    def gate_grad(i):
        b = i % batches
        ng.ngram_backward_gate(ctx, toks[b], dy, history=hists[b], out=grad_gate, stream=stream)

    for i in range(warmup):
        rows(i)
        gate_grad(i)
    torch.cuda.synchronize()
    K = steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    Us = []
    with ClockSampler(gpu_id_for(dev)) as clk:
        torch.cuda.synchronize()
        for i in range(K):
            ev[i][0].record(stream)
            rows(i)
            ev[i][1].record(stream)
            gate_grad(i)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    for b in range(batches):               # distinct rows of each batch (outside the timing)
        rows(b)
        Us.append(int(count.item()))
    st, info = ng.ngram_get_device_error(ctx)
    rows_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in ev)
    gate_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in ev)
    step_ms = statistics.fmean(e[0].elapsed_time(e[2]) for e in ev)
    U = statistics.fmean(Us)
    peaks = measured_peaks()
    # algorithmic bytes: table gradient = dy read once + one fp32 row per distinct row
    # written; gate gradient = the forward's row reads + dy read (+ fp64 partials)
    rows_bytes = N * 2 * d + U * 4 * d + 4 * d
    gate_bytes = N * (HEADS * row_bytes(w) + 2 * d + 4) + 2 * 8 * d * ((N + 15) // 16) + 4 * d
    # the table gradient mostly writes: its stream bound is the gradient rows at the
    # measured write stream plus dy at the measured read stream
    wr_gbs, rd_gbs = write_stream_gbs(dev), read_stream_gbs(dev)
    rows_bound_ms = (U * 4 * d / wr_gbs + N * 2 * d / rd_gbs) / 1e6
    del grad_rows
    return {
        "value": N / (step_ms / 1e3), "unit": UNIT, "steps": K, "warmup": warmup,
        "ms_per_step": step_ms, "distinct_rows_per_batch": U,
        "backward_rows": {"ms": rows_ms, "algorithmic_bytes": rows_bytes,
                          "achieved_gbs": rows_bytes / rows_ms / 1e6,
                          "frac": rows_bytes / rows_ms / 1e6 / peaks["hbm_gbs"],
                          "stream_bound_ms": rows_bound_ms, "frac_of_stream_bound": rows_bound_ms / rows_ms,
                          "write_stream_gbs": wr_gbs, "read_stream_gbs": rd_gbs,
                          "kernels": "hash, dedup (5), radix sort (%d passes x 5), segments, k_rows_grad"
                                     % ((max(1, (N * H - 1).bit_length()) + 7) // 8)},
        "backward_gate": {"ms": gate_ms, "algorithmic_bytes": gate_bytes,
                          "achieved_gbs": gate_bytes / gate_ms / 1e6,
                          "frac": gate_bytes / gate_ms / 1e6 / peaks["hbm_gbs"],
                          "kernels": "k_gate_grad + k_gate_reduce"},
        "peak": {"hbm_gbs": peaks["hbm_gbs"], "source": peaks["source"]},
        "clocks": clk.summary(),
        "device_error": "ok" if st == ng.NGRAM_OK else str(info),
    }


def run_backward(args, w):
    """The backward pass of the lookup, timed like the forward: one step = the table
    gradient + the shared-gate gradient of one batch, on one GPU."""
    import torch

    import hashed_gram_embedding_ngram_b200 as ng

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the lookup has no CPU path)")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    dtype, table, scale = make_table(ng, w, dev)
    ctx = ng.ngram_init(table, w.R, w.d, dtype, ng.NGRAM_RES_HBM,
                        ng.ngram_default_hash_params(vocab_size=w.vocab), w.N, row_scale=scale)
    rec = backward_record(ng, dev, w, ctx, args.batches, args.steps, args.warmup)
    line = {
        "metric": "n-gram embed backward tokens/s (table + gate gradients), 1 B200",
        "n_gpus": 1, "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
        "config": dict(config_for(w, args), mode="backward",
                       distinct_rows_per_batch=rec.pop("distinct_rows_per_batch")),
    }
    line.update(rec)
    print(json.dumps(line), flush=True)
    ctx.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="full_prefill", choices=sorted(gen.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batches", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other configurations (mid, decode, backward, host-resident, "
                         "int8 / FP8 / NVFP4) that the default full_prefill run adds as sub-records")
    ap.add_argument("--launch", default="auto", choices=["auto", "eager", "graph"],
                    help="eager launches, or 100-step CUDA graphs (auto: graph for N <= 1024)")
    ap.add_argument("--variant", default="default",
                    choices=["default", "dedup", "tma", "sort", "batch_order", "shard", "token_gate"],
                    help="HBM path: library default (grouped order from 16,384 tokens), dedup + "
                         "staged gather, TMA staging, always grouped, always batch order; shard: "
                         "the table split by columns over the ranks (strong scaling)")
    ap.add_argument("--host-workloads", default="host_decode_1,host_decode_16,host_decode_64,"
                                                "host_decode_256,host_prefill")
    ap.add_argument("--host-steps", type=int, default=200)
    ap.add_argument("--host-rows", type=int, default=0, help="override R for the host table")
    ap.add_argument("--mode", default="forward", choices=["forward", "backward"],
                    help="forward: the lookup (the benchmark); backward: table + gate gradients")
    args = ap.parse_args()
    w = gen.WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    if w.residency == "host" and args.impl == "ours":
        run_host(args)
        return
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return
    if args.mode == "backward":
        if rank == 0:
            run_backward(args, w)
        return
    if args.variant == "shard":
        run_shard(args, w)
        return
    run_ours(args, w)


if __name__ == "__main__":
    main()
