"""Benchmark: paged-attention decode query-tokens/s and achieved K/V-read HBM
bandwidth on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl ours|reference]

A step is one decode step of the whole hot path on one batch: copy-on-write
block copies (when the workload has any), the K/V write of every sequence's
new token, and decode attention (split partitions merged inside the same kernel),
for every layer of the workload. The default workload is the Llama-7B-shaped
single layer: 96 sequences, 32 heads, head_dim 128, block size 16, context
lengths uniform in [128, 2048], an 8192-block pool.

By default each layer's K/V write and decode run as one launch
(pa_write_kv_decode) and the whole step is replayed from a CUDA graph;
--separate uses pa_write_kv + pa_decode, --no-graph launches from the host.

Under torchrun (N > 1) every rank runs an independent replica of the workload
(the path has no exchange step); the time is the maximum over ranks and the
value counts the query tokens of all ranks.

--impl reference times the fp64 CPU oracle on this machine's host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged-attn decode query-tokens/s; achieved KV-read HBM GB/s vs B200 peak"
UNIT = "query-tokens/s"
NOMINAL_PEAK_GBS = 8000.0  # the B200's nominal ~8 TB/s HBM3e bandwidth
FALLBACK_PEAK_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20

WORKLOADS = {
    "tiny": (lambda seed, dt="f16": wl.tiny(seed=seed, dtype=dt),
             "tiny: 4 seqs, 4 heads, head_dim 64, block_size 16, ctx {1,17,33,100}, "
             "64-block pool"),
    "llama7b_layer": (lambda seed, dt="f16": wl.llama_layer(seed=seed, dtype=dt),
                      "llama7b_layer: 96 seqs, 32 heads, head_dim 128, block_size 16, "
                      "ctx U[128,2048], 8192-block pool, write_kv + decode"),
    "long_context": (lambda seed, dt="f16": wl.long_context(seed=seed, dtype=dt),
                     "long_context: 8 seqs, 32 heads, head_dim 128, block_size 16, "
                     "ctx U[16384,32768], 20000-block pool, split decode (partitions merged in-kernel)"),
    "prefix_cow": (lambda seed, dt="f16": wl.prefix_cow(seed=seed, dtype=dt),
                   "prefix_cow: 64 seqs sharing a 1024-token prefix, suffix U[1,512], "
                   "32 heads, head_dim 128, copy_blocks + write_kv + decode"),
    "full_step_bs8": (lambda seed, dt="f16": wl.full_step(seed=seed, block_size=8, dtype=dt),
                      "full_step: 32 layers, 256 seqs, ctx min(Geom(1/300),4096), bs 8"),
    "full_step_bs16": (lambda seed, dt="f16": wl.full_step(seed=seed, block_size=16, dtype=dt),
                       "full_step: 32 layers, 256 seqs, ctx min(Geom(1/300),4096), bs 16"),
    "full_step_bs32": (lambda seed, dt="f16": wl.full_step(seed=seed, block_size=32, dtype=dt),
                       "full_step: 32 layers, 256 seqs, ctx min(Geom(1/300),4096), bs 32"),
    "swap_resume": (lambda seed, dt="f16": wl.llama_layer(seed=seed, dtype=dt),
                    "swap_resume: llama7b_layer whose every 4th sequence (24 of 96) is swapped "
                    "in from pinned host memory (pa_swap_blocks) before each decode"),
    "small_batch_step": (lambda seed, dt="f16": wl.full_step(seed=seed, block_size=16, num_seqs=8, dtype=dt),
                         "small_batch_step: 32 layers, 8 seqs, ctx min(Geom(1/300),4096), "
                         "bs 16 (launch-bound)"),
}
SEEDS = {"tiny": 0, "llama7b_layer": 1, "long_context": 2, "prefix_cow": 3,
         "full_step_bs8": 4, "full_step_bs16": 4, "full_step_bs32": 4, "small_batch_step": 5,
         "swap_resume": 1}


def algorithmic_bytes(step) -> dict:
    """Bytes one decode over one layer must move: every context token's K and
    V row (head_dim x 2 bytes, all heads), the query and output rows and the
    block-table entries it reads. Over-reads of partly filled blocks are not
    counted."""
    H, D = step.num_heads, step.head_dim
    ctx = step.context_lens.astype(np.int64)
    kv = wl.kv_bytes_read(step)      # K and V rows (fp8: codes + a 4-byte scale per row)
    qo = step.num_seqs * H * D * 2 * 2
    table = int(np.sum(-(-ctx // step.block_size))) * 4
    return {"kv": kv, "total": kv + qo + table}


def kernel_source_hash(sources=("decode.cuh", "ptx.cuh")) -> str:
    """Hash of a decode kernel's own sources (an ncu traffic record is void
    once they change)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_417_b200", "csrc")
    for name in sources:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_PEAK_GBS, "fallback"


def traffic_key(args):
    """Name of the workload in profiles/traffic.json: the config, plus the
    K/V dtype and head count when they differ from the config's own."""
    key = args.config
    if args.kv_dtype != "f16":
        key += f"_{args.kv_dtype}"
    if args.kv_heads:
        key += f"_kvh{args.kv_heads}"
    if args.seqs:
        key += f"_s{args.seqs}"
    return key


def recorded_traffic(config):
    """DRAM bytes per decode launch from an ncu capture, if one was taken on
    the current kernel sources (profiles/traffic.json); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(config)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("kernel_source_hash") != kernel_source_hash(
            tuple(rec.get("sources", ("decode.cuh", "ptx.cuh")))):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_uuid):
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if device_uuid:
            cmd[1:1] = ["-i", device_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        sm, smax, reasons = [], [], set()
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def device_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# ----------------------------------------------------------------------------
# The oracle on the host cores (cpu_baseline, and the reference arm).
# ----------------------------------------------------------------------------

def oracle_inputs(sub, layers):
    """Host pools of a sub-step (input generation, outside any timing)."""
    return [wl.host_pools(sub, li) for li in layers]


def time_oracle(sub, layers, pools, results=None):
    """Seconds the oracle takes for the whole step of ``sub`` on ``layers``:
    copy-on-write, K/V write, decode. ``results`` (a list) receives the fp64
    outputs of each layer."""
    import oracle
    t0 = time.perf_counter()
    outs = []
    for li, (kc, vc) in zip(layers, pools):
        outs.append(oracle.default().step_on_pools(sub, li, kc, vc))
    secs = time.perf_counter() - t0
    if results is not None:
        results[:] = outs
    return secs


def oracle_sample(step, target_seconds):
    """A sub-batch of ``step`` whose oracle run on one layer takes about
    ``target_seconds``."""
    order = np.random.default_rng(123).permutation(step.num_seqs)
    probe = wl.subset(step, order[:1])
    t1 = time_oracle(probe, [0], oracle_inputs(probe, [0]))
    per_token = t1 / max(1, int(probe.context_lens.sum()))
    budget = target_seconds / max(per_token, 1e-9)
    ids, tokens = [], 0
    for s in order:
        if ids and tokens + int(step.context_lens[s]) > budget:
            break
        ids.append(int(s))
        tokens += int(step.context_lens[s])
    return wl.subset(step, sorted(ids))


def accuracy(step, sub, layers, refs, gpu_outs):
    """Max and mean |gpu - oracle| over every output element of the sampled
    sequences and layers, the worst element, and whether all are within the
    tolerance: 2e-3 for f16 outputs (fp8 caches have f16 rows), and
    |o| * 2^-8 + 1e-3 for bf16 outputs (bf16 rounding alone can pass 2e-3)."""
    ids = np.asarray(sub.meta["seq_ids"], dtype=np.int64)
    worst, total, count, ok = (0.0, None), 0.0, 0, True
    bf16 = step.io_dtype == "bf16"
    for li, ref in zip(layers, refs):
        got = gpu_outs[li][ids].double().cpu().numpy()
        if not np.all(np.isfinite(got)):
            return {"max_abs_err": float("inf"), "within_tolerance": False,
                    "checked": "non-finite GPU output"}
        err = np.abs(got - ref)
        tol = np.abs(ref) * 2.0 ** -8 + 1e-3 if bf16 else 2e-3
        ok = ok and bool(np.all(err <= tol))
        k = int(np.argmax(err))
        if err.flat[k] >= worst[0]:
            s_, h_, d_ = np.unravel_index(k, err.shape)
            worst = (float(err.flat[k]), {"layer": int(li), "seq": int(ids[s_]),
                                          "head": int(h_), "dim": int(d_)})
        total += float(err.sum())
        count += err.size
    return {"max_abs_err": worst[0], "mean_abs_err": total / max(count, 1),
            "worst": worst[1], "within_tolerance": ok,
            "tolerance": "|o|*2^-8 + 1e-3 (bf16 output)" if bf16 else 2e-3,
            "checked": (f"{sub.num_seqs} of {step.num_seqs} sequences x layers "
                        f"{list(layers)} of {step.num_layers}: outputs of the timed steps "
                        f"vs the fp64 oracle outputs of the CPU-baseline sample")}


def cpu_baseline(step, gpu_outs=None, target_seconds=12.0):
    """The oracle on this host's cores over a bounded sample of the workload,
    repeated until about ``target_seconds`` of oracle work were timed. With
    ``gpu_outs`` (the outputs of the timed steps, per layer) the oracle's
    outputs for the sample are also compared with them."""
    import oracle
    layers = [0] if step.num_layers == 1 else [0, step.num_layers - 1]
    sub = oracle_sample(step, target_seconds / len(layers))
    pools = oracle_inputs(sub, layers)
    secs, reps, refs = 0.0, 0, []
    while reps == 0 or secs < 0.8 * target_seconds:
        secs += time_oracle(sub, layers, pools, refs)
        reps += 1
    value = sub.num_seqs * len(layers) * reps / (secs * step.num_layers)
    line = {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"{sub.num_seqs} of {step.num_seqs} sequences x {len(layers)} of "
                       f"{step.num_layers} layers (copy-on-write, K/V write, decode), "
                       f"{reps} repetition(s), fp64 C + OpenMP, {secs:.1f} s; value scaled "
                       f"to whole decode steps")}
    acc = accuracy(step, sub, layers, refs, gpu_outs) if gpu_outs is not None else None
    return line, acc


def block_manager_timing(step, reps=200):
    """Host cost of producing one decode step's integer inputs (append one
    token per sequence: tables, context lengths, slots, copy-on-write pairs)
    with the library's C++ block manager and with the Python allocator of
    workloads/, on the workload's sequence lengths."""
    from paged_kv_cache_417_b200.block_manager import BlockManager
    S, bs = step.num_seqs, step.block_size
    pre = (step.context_lens - 1).astype(np.int64)
    nb = int(np.sum(-(-(pre + reps + 1) // bs))) + S + 16
    order = np.random.default_rng(7).permutation(nb)
    mb = int(np.max(-(-(pre + reps + 1) // bs)))
    cc = BlockManager(nb, bs, order)
    for i in range(S):
        cc.add_sequence(i)
        cc.allocate_tokens(i, int(pre[i]))
    ids = np.arange(S, dtype=np.int64)
    t0 = time.perf_counter()
    for _ in range(reps):
        cc.prepare_decode(ids, mb)
    cpp = (time.perf_counter() - t0) / reps
    alloc = wl.BlockAllocator(nb, bs, order)
    seqs = [wl.Sequence() for _ in range(S)]
    for i in range(S):
        wl.allocate_tokens(alloc, seqs[i], int(pre[i]))
    t0 = time.perf_counter()
    for _ in range(reps):
        bt = np.full((S, mb), -1, dtype=np.int32)
        for i, sq in enumerate(seqs):
            wl.append_token(alloc, sq)
            bt[i, :len(sq.block_table)] = sq.block_table
    py = (time.perf_counter() - t0) / reps
    return {"seqs": S, "cpp_us_per_step": cpp * 1e6, "python_us_per_step": py * 1e6,
            "reps": reps}


def max_over_ranks(x, dist=None, device=None):
    """The maximum of a per-rank number over all ranks (identity alone)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# The suite's other workloads, measured briefly after the default one's line
# is timed (one GPU, default workload), each by this script in a child
# process with its own warm-up, L2 flushes, CUDA-event timing and clocks.
OTHER_CONFIGS = (
    ("long_context", ["--config", "long_context"], 30),
    ("prefix_cow", ["--config", "prefix_cow"], 100),
    ("full_step_bs16", ["--config", "full_step_bs16"], 10),
    ("llama7b_layer_fp8", ["--kv-dtype", "fp8"], 100),
    ("llama7b_layer_kvh8", ["--kv-heads", "8"], 100),
    ("llama7b_layer_kvh2", ["--kv-heads", "2"], 100),
    ("llama7b_layer_fp8_kvh8", ["--kv-dtype", "fp8", "--kv-heads", "8"], 100),
)


def other_config_runs(warmup):
    """A compact record of each other workload's own JSON line."""
    out = []
    for name, extra, steps in OTHER_CONFIGS:
        cmd = [sys.executable, os.path.abspath(__file__), *extra, "--steps", str(steps),
               "--warmup", str(max(3, warmup)), "--soak-seconds", "0.3", "--no-e2e",
               "--no-cpu-baseline", "--no-other-configs"]
        try:
            res = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
            d = json.loads(res.stdout.strip().splitlines()[-1])
            r = d["roofline"]
            out.append({"config": name, "workload": d["config"]["workload"],
                        "value": d["value"], "unit": d["unit"], "steps": d["steps"],
                        "ms_per_step": d["ms_per_step"], "decode_us": r["decode_us"],
                        "roofline_frac": r["frac"], "frac_of_8tbs": r["frac_of_8tbs"],
                        "traffic": r["traffic"], "partition_size": d["partition_size"],
                        "clocks": d["clocks"]})
            if name == "prefix_cow":
                out[-1]["note"] = ("fractions count logical bytes: the shared prefix is read "
                                   "once from HBM and then from L2, by design of the workload")
        except Exception as e:  # reported in the line, never fatal to it
            out.append({"config": name, "error": f"{type(e).__name__}: {e}"[:300]})
    return out


def job_throughput(world, seqs_per_rank, steps, max_ms):
    """Query tokens of all ranks per second of the slowest rank."""
    return world * seqs_per_rank * steps / (max_ms / 1e3)


def run_reference(args, config_desc):
    step = make_step(args.config, 0, args.kv_dtype, args.kv_heads, args.seqs)
    sub = oracle_sample(step, 2.0)
    layers = [0]
    pools = oracle_inputs(sub, layers)
    for _ in range(args.warmup):
        time_oracle(sub, layers, pools)
    secs = 0.0
    for _ in range(args.steps):
        secs += time_oracle(sub, layers, pools)
    value = sub.num_seqs * len(layers) * args.steps / (secs * step.num_layers)
    import oracle
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": config_desc,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{sub.num_seqs} of {step.num_seqs} sequences, 1 of "
                                   f"{step.num_layers} layers per step, scaled to whole steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# The CUDA path: one step as the benchmark launches it (also driven by the
# GPU tests of the benchmarked path).
# ----------------------------------------------------------------------------

def make_step(config, rank=0, kv_dtype="f16", kv_heads=0, seqs=0):
    """The workload of ``config`` for replica ``rank`` (seed + 1000 * rank),
    optionally with ``kv_heads`` K/V heads or ``seqs`` sequences."""
    seed = SEEDS[config] + 1000 * rank
    if seqs:
        if config != "llama7b_layer":
            raise ValueError("--seqs applies to llama7b_layer only")
        return wl.llama_layer(seed=seed, num_seqs=seqs, num_blocks=max(256, 8192 * seqs // 96),
                              dtype=kv_dtype, num_kv_heads=kv_heads or None)
    if kv_heads:
        if config == "llama7b_layer":
            return wl.llama_layer(seed=seed, dtype=kv_dtype, num_kv_heads=kv_heads)
        if config.startswith("full_step_bs"):
            return wl.full_step(seed=seed, dtype=kv_dtype, num_kv_heads=kv_heads,
                                block_size=int(config[len("full_step_bs"):]))
        raise ValueError("--kv-heads applies to llama7b_layer and full_step_bs*")
    return WORKLOADS[config][0](seed, kv_dtype)


INTEGER_INPUTS = ("block_tables", "context_lens", "slot_mapping", "copy_pairs")


def native_inputs(step):
    """The step's integer inputs (block tables, context lengths, the new
    tokens' slots, copy-on-write pairs) built by the library's C++ block
    manager with pa_bm_prepare_decode, from the allocation history the
    workload's Python allocator followed: the same free order, the shared
    prefix forked to every sequence, each sequence's cached tokens, then one
    appended token per sequence. Where the workload gives each partly filled
    last block a second holder, the C++ side forks the whole sequence (a
    parallel-sampling sibling) while the Python allocator adds a holder to
    that block only: every block of such a sequence then counts one more
    holder on the C++ side, and every decode input is the same. Returns a
    dict of numpy arrays (plus the manager's reference counts under
    "ref_count")."""
    from paged_kv_cache_417_b200.block_manager import BlockManager
    m = step.meta
    S, bs = step.num_seqs, step.block_size
    bm = BlockManager(step.num_blocks, bs, m["free_order"])
    prefix = int(m["prefix_tokens"])
    if prefix and S:
        bm.add_sequence(0)
        bm.allocate_tokens(0, prefix)
        for s in range(1, S):
            bm.fork(0, s)
    else:
        for s in range(S):
            bm.add_sequence(s)
    for s in range(S):
        bm.allocate_tokens(s, int(m["pre_tokens"][s]))
    if m["fork_partial_tail"]:
        for s in range(S):
            if bm.num_tokens(s) % bs:
                bm.fork(s, S + s)
    out = bm.prepare_decode(np.arange(S, dtype=np.int64), step.max_blocks_per_seq)
    out["ref_count"] = bm.ref_counts()
    return out


def upload_step(step, dev, integer_inputs=None):
    """All inputs of ``step`` on ``dev`` (fp8 pools wrapped for the binding).
    ``integer_inputs`` (e.g. from :func:`native_inputs`) replaces the block
    tables, context lengths, slots and copy-on-write pairs."""
    import torch
    import paged_kv_cache_417_b200 as pk
    from workloads.device import device_step
    d = device_step(step, dev)
    if integer_inputs is not None:
        for k in INTEGER_INPUTS:
            d[k] = torch.from_numpy(np.ascontiguousarray(integer_inputs[k])).to(dev)
    if step.dtype == "fp8":
        for key in ("key_caches", "value_caches"):
            d[key] = [pk.Fp8Cache(t, step.block_size, step.head_dim, torch.float16)
                      for t in d[key]]
    return d


class StepLauncher:
    """One decode step of the whole path for every layer of ``step``:
    copy-on-write block copies (when the workload has any), then per layer
    the fused K/V write + decode (``fused``) or pa_write_kv then pa_decode.
    The caches in ``d`` are updated in place; outputs go to ``self.outs``
    unless other output tensors are given. ``swap`` (swap-resume workload)
    swaps the workload's host blocks in first."""

    def __init__(self, step, d, dev, fused=True, partition=0, swap=None):
        import torch
        import paged_kv_cache_417_b200 as pk
        self.pk, self.torch = pk, torch
        self.step, self.d, self.dev = step, d, dev
        self.fused, self.partition, self.swap = fused, partition, swap
        self.outs = [torch.empty_like(q) for q in d["query"]]
        S = step.num_seqs
        self.ws = pk.alloc_workspace(S, step.num_heads, step.head_dim, step.max_context_len,
                                     partition, dev)
        self.P = pk.decode_partition_size(S, step.num_heads, d["key_caches"][0],
                                          step.max_context_len, partition)
        self.split = step.max_context_len > self.P
        # Split partitions are merged by the last CTA of each sequence, unless
        # the grid has more (sequence, head) slots than the workspace has
        # arrival counters (then a separate reduce kernel runs).
        self.reduce_launch = self.split and S * step.num_heads > 65536
        self.has_copy = step.copy_pairs.shape[0] > 0

    @property
    def launches_per_step(self):
        L = self.step.num_layers
        n = (1 if self.has_copy else 0) + L * ((1 if self.fused else 2) +
                                               (1 if self.reduce_launch else 0))
        return n + (1 if self.swap is not None else 0)

    def swap_in(self):
        sw, d = self.swap, self.d
        self.pk.swap_blocks(sw["host_k"], sw["host_v"], d["key_caches"], d["value_caches"],
                            sw["map"])

    def one_step(self, dec_events=None, inputs=None, out_list=None):
        """Enqueue one step on the current stream; ``dec_events`` (two lists)
        receive CUDA events around every decode call."""
        pk, torch, step, d = self.pk, self.torch, self.step, self.d
        src = inputs or d
        dst = out_list or self.outs
        stream = torch.cuda.current_stream(self.dev)
        if self.swap is not None:
            self.swap_in()
        if self.has_copy:
            pk.copy_blocks(d["key_caches"], d["value_caches"], src["copy_pairs"])
        for li in range(step.num_layers):
            kc, vc = d["key_caches"][li], d["value_caches"][li]
            if not self.fused:
                pk.write_kv(src["new_key"][li], src["new_value"][li], src["slot_mapping"], kc,
                            vc)
            if dec_events is not None:
                dec_events[0].append(torch.cuda.Event(enable_timing=True))
                dec_events[0][-1].record(stream)
            if self.fused:
                pk.write_kv_decode(dst[li], src["query"][li], src["new_key"][li],
                                   src["new_value"][li], kc, vc, src["block_tables"],
                                   src["context_lens"], step.max_context_len,
                                   float(step.scale), partition_size=self.partition,
                                   workspace=self.ws)
            else:
                pk.decode(dst[li], src["query"][li], kc, vc, src["block_tables"],
                          src["context_lens"], step.max_context_len, float(step.scale),
                          partition_size=self.partition, workspace=self.ws)
            if dec_events is not None:
                dec_events[1].append(torch.cuda.Event(enable_timing=True))
                dec_events[1][-1].record(stream)

    def capture(self, inputs=None, out_list=None):
        """The whole step recorded once as a CUDA graph (the library only
        enqueues kernels on the current stream, allocates nothing and never
        synchronises, so it can be captured)."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.one_step(inputs=inputs, out_list=out_list)
        torch.cuda.synchronize(self.dev)
        return g


def make_swap(step, d, dev):
    """Swap-resume workload: a pinned host pool holds the blocks of every 4th
    sequence; each step swaps them into their GPU blocks first."""
    import torch
    S, L = step.num_seqs, step.num_layers
    blocks = sorted({int(b) for s_ in range(0, S, 4) for b in step.block_tables[s_] if b >= 0})
    idx = torch.tensor(blocks, device=dev)
    hk = [d["key_caches"][li][idx].cpu().pin_memory() for li in range(L)]
    hv = [d["value_caches"][li][idx].cpu().pin_memory() for li in range(L)]
    return {"host_k": hk, "host_v": hv, "blocks": len(blocks),
            "map": torch.tensor([[i, b] for i, b in enumerate(blocks)], dtype=torch.int64,
                                device=dev),
            "bytes": 2 * L * len(blocks) * hk[0][0].numel() * hk[0].element_size()}


class E2EPipeline:
    """End to end through the public API with host buffers: every step copies
    its inputs from pinned host memory to the device and its outputs back, as
    one packed DMA each way. Two input/output buffer sets and a copy stream
    each way pipeline the steps, so a step's copies overlap its neighbours'
    compute on the copy engines. With ``graph`` every buffer set has its own
    captured step."""

    def __init__(self, launcher, graph=True):
        import torch
        self.torch, self.launcher, self.graph = torch, launcher, graph
        d, dev, L = launcher.d, launcher.dev, launcher.step.num_layers
        names = [(k, i) for k in ("query", "new_key", "new_value") for i in range(L)]
        names += [(k, None) for k in ("slot_mapping", "block_tables", "context_lens")]
        if launcher.has_copy:
            names.append(("copy_pairs", None))

        def tensor_of(name):
            k, i = name
            return d[k][i] if i is not None else d[k]

        layout, off = [], 0
        for nm in names:
            t = tensor_of(nm)
            nbytes = t.numel() * t.element_size()
            layout.append((nm, off, nbytes, t.dtype, t.shape))
            off = (off + nbytes + 255) // 256 * 256
        self.h2d = off
        self.host_in = torch.empty(self.h2d, dtype=torch.uint8, pin_memory=True)
        for nm, o, nbytes, _, _ in layout:
            self.host_in[o:o + nbytes].copy_(tensor_of(nm).reshape(-1).view(torch.uint8).cpu())
        self.out_meta = [(o.dtype, o.shape, o.numel() * o.element_size())
                         for o in launcher.outs]
        self.d2h = sum(m[2] for m in self.out_meta)

        def views(buf):
            v = {"query": [None] * L, "new_key": [None] * L, "new_value": [None] * L,
                 "copy_pairs": d["copy_pairs"]}
            for (k, i), o, nbytes, dt, shape in layout:
                t = buf[o:o + nbytes].view(dt).view(shape)
                if i is None:
                    v[k] = t
                else:
                    v[k][i] = t
            return v

        self.bufs = []
        for _ in range(2):
            dev_in = torch.empty(self.h2d, dtype=torch.uint8, device=dev)
            dev_out = torch.empty(self.d2h, dtype=torch.uint8, device=dev)
            bf = {"dev_in": dev_in, "in": views(dev_in), "dev_out": dev_out,
                  "out": self._split(dev_out),
                  "host_out": torch.empty(self.d2h, dtype=torch.uint8, pin_memory=True)}
            if graph:
                bf["graph"] = launcher.capture(inputs=bf["in"], out_list=bf["out"])
            self.bufs.append(bf)
        self.up, self.down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        self.ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "step", "d2h")}

    def _split(self, flat):
        outs, o = [], 0
        for dt, shape, nb in self.out_meta:
            outs.append(flat[o:o + nb].view(dt).view(shape))
            o += nb
        return outs

    def host_outputs(self, b):
        """The outputs of the last step that ran on buffer set ``b``, as
        copied to pinned host memory (call after synchronising)."""
        return self._split(self.bufs[b]["host_out"])

    def run(self, n, sleep_s=0.0):
        """Enqueue ``n`` end-to-end steps; returns the (start, end) timing
        events, recorded on the upload and download streams."""
        torch, ev, up, down = self.torch, self.ev, self.up, self.down
        stream = torch.cuda.current_stream(self.launcher.dev)
        with torch.cuda.stream(up):
            if sleep_s:
                torch.cuda._sleep(int(sleep_s * 2.0e9))
            t0 = torch.cuda.Event(enable_timing=True)
            t0.record(up)
        for k in range(n):
            b = k % 2
            bf = self.bufs[b]
            with torch.cuda.stream(up):
                if k >= 2:
                    up.wait_event(ev["step"][b])  # step k-2 has read these inputs
                bf["dev_in"].copy_(self.host_in, non_blocking=True)
                ev["h2d"][b].record(up)
            stream.wait_event(ev["h2d"][b])
            if k >= 2:
                stream.wait_event(ev["d2h"][b])  # outputs of step k-2 copied out
            if self.graph:
                bf["graph"].replay()
            else:
                self.launcher.one_step(inputs=bf["in"], out_list=bf["out"])
            ev["step"][b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev["step"][b])
                bf["host_out"].copy_(bf["dev_out"], non_blocking=True)
                ev["d2h"][b].record(down)
        t1 = torch.cuda.Event(enable_timing=True)
        t1.record(down)
        return t0, t1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="llama7b_layer", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition", type=int, default=0)
    ap.add_argument("--seqs", type=int, default=0,
                    help="llama7b_layer only: this many sequences (pool scaled to match), "
                         "for profiler captures on a smaller case of the same kernel")
    ap.add_argument("--soak-seconds", type=float, default=1.0)
    ap.add_argument("--kv-dtype", default="f16", choices=["f16", "bf16", "fp8"],
                    help="cache storage (fp8: e4m3 codes + fp32 row scales, fp16 rows)")
    ap.add_argument("--kv-heads", type=int, default=0,
                    help="llama7b_layer / full_step: K/V heads (grouped query heads)")
    ap.add_argument("--separate", action="store_true",
                    help="pa_write_kv then pa_decode instead of the fused pa_write_kv_decode")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step from the host instead of replaying a CUDA graph")
    ap.add_argument("--inputs", default="native", choices=["native", "python"],
                    help="which block manager builds the step's integer inputs: the "
                         "library's C++ one (default) or the Python allocator of workloads/")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the short runs of the other workloads that a default "
                         "single-GPU run appends to its line")
    args = ap.parse_args()
    args.fused = not args.separate
    args.graph = not args.no_graph
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    flush = args.config != "prefix_cow"  # prefix reuse through L2 is part of that workload
    config_desc = {"workload": WORKLOADS[args.config][1],
                   "l2": "flushed between steps (256 MiB read)" if flush else
                         "not flushed (shared-prefix reuse is part of the workload)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "partition": args.partition or "auto",
                   "launch": ("fused write+decode" if args.fused else "write_kv, decode") +
                             (", CUDA graph" if args.graph else "")}

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, config_desc)
        return

    import torch

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)

    try:
        step = make_step(args.config, rank, args.kv_dtype, args.kv_heads, args.seqs)
    except ValueError as e:
        ap.error(str(e))
    if args.seqs:
        config_desc["workload"] += f" (reduced to {args.seqs} seqs)"
    if args.kv_heads:
        config_desc["workload"] += f" with {args.kv_heads} K/V heads (grouped query heads)"
    if args.kv_dtype != "f16":
        config_desc["kv_dtype"] = args.kv_dtype
    native = None
    if args.inputs == "native":
        native = native_inputs(step)
        for k in INTEGER_INPUTS:
            if not np.array_equal(native[k], getattr(step, k)):
                raise SystemExit(f"C++ block manager's {k} differs from the workload's")
        config_desc["inputs"] = ("block tables, context lengths, slots and copy-on-write pairs "
                                 "from the C++ block manager (pa_bm_prepare_decode); equal to "
                                 "the Python allocator's")
    else:
        config_desc["inputs"] = "integer inputs from the Python allocator of workloads/"
    d = upload_step(step, dev, native)
    S = step.num_seqs
    stream = torch.cuda.current_stream(dev)
    swap = make_swap(step, d, dev) if args.config == "swap_resume" else None
    launcher = StepLauncher(step, d, dev, fused=args.fused, partition=args.partition, swap=swap)
    outs, P, split = launcher.outs, launcher.P, launcher.split
    one_step = launcher.one_step
    # L2 flush by reading 256 MiB: the previous step's lines are evicted and
    # L2 is left holding clean lines, so no write-back lands on the next step.
    flush_buf = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)

    def flush_l2():
        if flush:
            flush_buf.sum()

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # Warm-up (also measures how long the host takes to enqueue a step on the
    # eager path with decode events, the slowest way a timed loop below
    # enqueues one), then an untimed soak so clocks settle and get sampled.
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(args.warmup):
        flush_l2()
        one_step(([], []))
    host_step_s = (time.perf_counter() - t0) / args.warmup
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(device_uuid(torch, dev))
    t_end = time.perf_counter() + args.soak_seconds
    while time.perf_counter() < t_end:
        for _ in range(10):
            flush_l2()
            one_step()
        torch.cuda.synchronize(dev)

    def head_start():
        """Hold the GPU in a bounded sleep while the host queues the timed
        steps, so no step waits for a launch (at most about 1 s)."""
        secs = min(1.0, 2.0 * args.steps * host_step_s + 0.002)
        torch.cuda._sleep(int(secs * 2.0e9))

    run_step = one_step
    if args.graph:
        graph_main = launcher.capture()
        run_step = lambda dec_events=None, inputs=None: graph_main.replay()  # noqa: E731
        for _ in range(args.warmup):
            flush_l2()
            run_step()
        torch.cuda.synchronize(dev)

    def host_paced(n):
        """Steps per second when the host launches each step as it goes (no
        head start): host launch cost shows here when it exceeds GPU time."""
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            run_step()
        b.record(stream)
        barrier()
        return job_throughput(world, S, n, max_over_ranks(a.elapsed_time(b), dist, dev))

    paced = host_paced(args.steps)

    # Timed region: K steps, L2 flushed between them, each step bracketed by
    # CUDA events on the launching stream.
    barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dec_events = ([], [])
    head_start()
    for k in range(args.steps):
        flush_l2()
        starts[k].record(stream)
        run_step(dec_events)
        ends[k].record(stream)
    barrier()
    # The outputs of the timed (graph-replayed) steps, kept for the accuracy
    # check against the oracle's outputs in the CPU-baseline leg.
    timed_outs = [o.clone() for o in outs]
    if args.graph:
        # Decode events cannot sit inside a replayed graph: time the decode
        # calls on the eager path, same steps, for the roofline.
        head_start()
        for k in range(args.steps):
            flush_l2()
            one_step(dec_events)
        barrier()
    clocks = sampler.stop()
    step_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    dec_ms = [a.elapsed_time(b) for a, b in zip(*dec_events)]
    total_ms = max_over_ranks(step_ms, dist, dev)
    value = job_throughput(world, S, args.steps, total_ms)

    # Roofline of the dominant kernel (the decode call; split partitions are
    # merged inside it).
    ab = algorithmic_bytes(step)
    dec_avg_s = statistics.mean(dec_ms) / 1e3
    achieved = ab["total"] / dec_avg_s / 1e9
    peak, peak_kind = measured_peak()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": recorded_traffic(traffic_key(args)),
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs copy bandwidth)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "kernel": "pa_decode (one decode kernel; split partitions merged in-kernel)",
                "algorithmic_bytes_per_launch": ab["total"],
                "kv_bytes_per_launch": ab["kv"],
                "decode_us": dec_avg_s * 1e6,
                "kv_gbs": ab["kv"] / dec_avg_s / 1e9,
                "frac_of_8tbs": achieved / NOMINAL_PEAK_GBS}

    swap_stats = None
    if swap is not None:
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier()
        for k in range(args.steps):
            ev0[k].record(stream)
            launcher.swap_in()
            ev1[k].record(stream)
        barrier()
        swap_s = statistics.mean(a.elapsed_time(b) for a, b in zip(ev0, ev1)) / 1e3
        # Reference: one contiguous pinned-host -> device copy of the same bytes.
        ref_src = torch.empty(swap["bytes"], dtype=torch.uint8).pin_memory()
        ref_dst = torch.empty(swap["bytes"], dtype=torch.uint8, device=dev)
        for _ in range(3):
            ref_dst.copy_(ref_src, non_blocking=True)
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(10):
            ref_dst.copy_(ref_src, non_blocking=True)
        b.record(stream)
        barrier()
        ref_s = a.elapsed_time(b) / 10 / 1e3
        swap_stats = {"blocks": swap["blocks"], "bytes_per_step": swap["bytes"],
                      "swap_us": swap_s * 1e6, "swap_gbs": swap["bytes"] / swap_s / 1e9,
                      "pinned_memcpy_gbs": swap["bytes"] / ref_s / 1e9,
                      "frac_of_memcpy": ref_s / swap_s}

    # End to end through the public API with host buffers (E2EPipeline). No
    # L2 flush here: every step reads more K/V than L2 holds.
    e2e = None
    if not args.no_e2e:
        pipe = E2EPipeline(launcher, graph=args.graph)
        barrier()
        h0 = time.perf_counter()
        pipe.run(args.warmup)
        host_e2e_s = (time.perf_counter() - h0) / args.warmup
        barrier()
        t0, t1 = pipe.run(args.steps, min(1.0, 1.5 * args.steps * host_e2e_s + 0.002))
        barrier()
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
        # What the host received must be what the device-timed steps computed.
        same = all(torch.equal(h.to(dev).view(torch.uint8), o.view(torch.uint8))
                   for b in range(2) for h, o in zip(pipe.host_outputs(b), timed_outs))
        e2e = {"value": job_throughput(world, S, args.steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": pipe.h2d, "d2h_bytes_per_step": pipe.d2h,
               "outputs_equal_device_timed": bool(same),
               "how": "one packed pinned-host DMA each way per step, 2 buffer sets, "
                      "separate upload and download streams overlapping compute"}

    cpu, acc = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, acc = cpu_baseline(step, timed_outs)
    bm_timing = block_manager_timing(step) if rank == 0 else None
    others = None
    if (rank == 0 and world == 1 and args.config == "llama7b_layer" and args.kv_dtype == "f16"
            and not args.kv_heads and not args.seqs and not args.separate and args.graph
            and not args.no_other_configs):
        others = other_config_runs(args.warmup)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": step.dtype,
            "accumulate": "f32", "data": "synthetic", "config": config_desc,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "max_abs_err": acc["max_abs_err"] if acc else None, "accuracy": acc,
            "gpu_launches": launcher.launches_per_step * args.steps, "clocks": clocks,
            "host_paced_value": paced, "host_block_manager": bm_timing, "swap": swap_stats,
            "partition_size": P, "split": split, "other_configs": others,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
