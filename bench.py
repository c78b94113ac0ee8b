#!/usr/bin/env python
"""Benchmark one paged decode step (store_kvcache + paged_attention_decode).

A step is one pass of the whole hot path over one batch: write each
sequence's new K/V row into its slot, then attend every query head over its
paged context (plus the split-K reduce when the plan splits). Inputs are
seeded synthetic tensors of the Qwen3-8B-shaped decode layer by default
(1024 sequences, lengths uniform in [100, 2048], 32 query / 8 KV heads,
head_dim 128, block_size 256, bf16 cache), resident in HBM before timing.
The KV pools (4.6 GB read per step) are far larger than L2, so no flush is
needed between steps.

Prints one JSON line (rank 0). ``--impl reference`` times the fp64 CPU
oracle instead, on bounded samples of the same workload.

Multi-GPU (torchrun): every rank runs its own copy of the workload (weak
scaling, no collective on the data path); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_482_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention tokens/sec and achieved HBM GB/s (% of B200 peak)"
UNIT = "tokens/s"
NOMINAL_HBM_GBS = 8000.0  # the "~8 TB/s" the target percentage refers to
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["paged_kv_cache_482_b200/csrc/decode.cuh", "paged_kv_cache_482_b200/csrc/decode_mma.cuh",
                  "paged_kv_cache_482_b200/csrc/decode.cu",
                  "paged_kv_cache_482_b200/csrc/pkv_common.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="qwen3_8b",
                    choices=sorted(W.CONFIGS) + sorted(W.PREFILL_CONFIGS) + sorted(W.NORM_CONFIGS) +
                    sorted(W.ROPE_CONFIGS),
                    help="a decode workload, a chunked-prefill one (prefill_*), an add + RMSNorm one (norm_*) or a "
                         "fused RoPE + store one (rope_*)")
    ap.add_argument("--partition", type=int, default=0, help="0 auto, -1 never split, >0 tokens per partition")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--num-seqs", type=int, default=0, help="override the workload's sequence count")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU work of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--out", default="", help="also append the JSON line to this file")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step's kernels from Python instead of replaying CUDA graphs of the step")
    ap.add_argument("--natural-order", action="store_true",
                    help="decode: visit the sequences in batch order instead of longest first")
    ap.add_argument("--no-staging", action="store_true",
                    help="E4M3 prefill: widen the codes in every CTA instead of once into a workspace")
    ap.add_argument("--no-shared-prefix", action="store_true",
                    help="attend a shared-prefix batch with the ordinary decode call instead of the cascade")
    ap.add_argument("--component", choices=["decode", "block_manager"], default="decode",
                    help="block_manager: time the host block manager's per-step bookkeeping instead")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers


def emit(line: dict, args) -> None:
    """Print the one JSON line (and append it to --out when given)."""
    text = json.dumps(line)
    print(text, flush=True)
    if getattr(args, "out", ""):
        d = os.path.dirname(os.path.abspath(args.out))
        os.makedirs(d, exist_ok=True)
        with open(args.out, "a") as f:
            f.write(text + "\n")


def workload_desc(cfg: W.DecodeConfig) -> str:
    if cfg.prefix_tokens:
        ctx = f"{cfg.prefix_tokens} shared + U[{cfg.ctx_lo},{cfg.ctx_hi}]"
    else:
        ctx = f"U[{cfg.ctx_lo},{cfg.ctx_hi}]"
    return (f"{cfg.name} paged decode layer: {cfg.num_seqs} seqs, ctx {ctx}, {cfg.num_q_heads}q/{cfg.num_kv_heads}kv "
            f"heads, head_dim {cfg.head_dim}, block_size {cfg.block_size}, {cfg.cache_dtype} cache")


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(cfg_name: str, partition_tokens: int):
    """dram read+write bytes per decode launch from a committed ncu capture, if
    it was taken on the current kernel source and the same workload."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except Exception:  # noqa: BLE001
        return None
    if rec.get("kernel_hash") != kernel_hash() or rec.get("workload") != cfg_name:
        return None
    if rec.get("partition_tokens") != partition_tokens:
        return None
    return rec.get("dram_bytes_per_launch")


def algorithmic_bytes(wl: W.Workload) -> dict:
    """Bytes one decode launch must move at minimum."""
    c = wl.cfg
    esize = 1 if wl.is_fp8 else 2
    ctx = wl.context_lens.long().cpu()
    # per-token E4M3 scales: 4 bytes for K and 4 for V per (token, KV head)
    row = c.head_dim * esize + (4 if wl.token_scales else 0)
    kv = int(ctx.sum()) * c.num_kv_heads * row * 2
    qo = 2 * c.num_seqs * c.num_q_heads * c.head_dim * 2
    nb = int(((ctx + c.block_size - 1) // c.block_size).sum())
    meta = 4 * nb + 4 * c.num_seqs
    if c.prefix_tokens:
        # shared prefix blocks are read once from HBM (they stay in L2)
        shared_tok = c.prefix_tokens
        own = int((ctx - c.prefix_tokens).sum())
        unique_kv = (shared_tok + own) * c.num_kv_heads * row * 2
    else:
        unique_kv = kv
    return dict(kv=kv, unique_kv=unique_kv, q_out=qo, meta=meta, total=kv + qo + meta,
                unique_total=unique_kv + qo + meta)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_ids):
        self.samples = []
        self.proc = None
        self.window = None
        try:
            cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits", "-lms",
                   "200"]
            if device_ids:
                cmd += ["-i", ",".join(str(d) for d in device_ids)]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.samples.append((time.time(), parts))

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while self.proc is not None and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.05)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:  # noqa: BLE001
                self.proc.kill()

    def summary(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        inwin = [p for t, p in self.samples if t0 <= t <= t1 + 0.25]
        used = inwin or [p for _, p in self.samples[-3:]]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        sm, smax, pw = [], [], []
        for p in used:
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
                pw.append(float(p[3]))
            except ValueError:
                pass
            for n, v in zip(names, p[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(pw) if pw else None, "reasons": sorted(reasons), "samples": len(inwin),
                "samples_note": "in the timed window" if inwin else "nearest samples (window shorter than 200 ms)"}


class NvmlSampler:
    """SM clock, power and clock-event reasons read through NVML every 5 ms
    (reads only), so that even a window of a few milliseconds holds samples.
    Same summary() as ClockSampler; make_sampler falls back to nvidia-smi."""

    PERIOD_S = 0.005

    def __init__(self, device_id):
        import pynvml as N

        self.N = N
        N.nvmlInit()
        if isinstance(device_id, str):
            self.h = N.nvmlDeviceGetHandleByUUID(device_id)
        else:
            self.h = N.nvmlDeviceGetHandleByIndex(int(device_id))
        self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM))
        self.bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                     "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                     "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                     "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}
        self.samples = []
        self.running = True
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def _poll(self):
        N = self.N
        while self.running:
            try:
                sm = float(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
                pw = N.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                rs = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.time(), sm, pw, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.PERIOD_S)

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while not self.samples and time.time() - t0 < timeout:
            time.sleep(0.005)

    def stop(self):
        self.running = False
        self.thread.join(timeout=1.0)

    def summary(self, t0, t1):
        inwin = [x for x in self.samples if t0 <= x[0] <= t1]
        used = inwin or self.samples[-3:]
        reasons = sorted({n for _, _, _, rs in used for n, b in self.bits.items() if rs & b})
        sm = [x[1] for x in used]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "power_w_max": max(x[2] for x in used) if used else None, "reasons": reasons,
                "samples": len(inwin), "sampler": "NVML every 5 ms",
                "samples_note": "in the timed window" if inwin else "nearest samples (no sample in the window)"}


def make_sampler(local_rank: int):
    """NVML sampler for this rank's GPU, else the nvidia-smi one."""
    ids = nvsmi_ids(local_rank)
    try:
        return NvmlSampler(ids[0])
    except Exception:  # noqa: BLE001
        return ClockSampler(ids)


def nvsmi_ids(local_rank: int):
    try:
        props = torch.cuda.get_device_properties(local_rank)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            s = str(uuid)
            return ["GPU-" + s if not s.startswith("GPU-") else s]
    except Exception:  # noqa: BLE001
        pass
    return [local_rank]



_HOST_AFFINITY = {"prev": None, "desc": "not bound"}


def bind_host_to_gpu(local_rank: int) -> str:
    """Restrict this process's host thread to the CPU cores that NVML reports
    as local to its GPU, before any pinned host buffer is made. Pinned pages
    then sit on the socket whose PCIe root the GPU hangs off, so host<->device
    copies do not cross the inter-socket link; left unbound, the placement
    follows whichever core the process starts on and the end-to-end numbers
    vary from run to run. The oracle baselines get the full set back
    (restore_host_affinity). Returns a description for the JSON line."""
    try:
        import pynvml as N

        N.nvmlInit()
        ident = nvsmi_ids(local_rank)[0]
        h = N.nvmlDeviceGetHandleByUUID(ident) if isinstance(ident, str) else N.nvmlDeviceGetHandleByIndex(int(ident))
        ncpu = os.cpu_count() or 1
        words = N.nvmlDeviceGetCpuAffinity(h, (ncpu + 63) // 64)
        local = {w * 64 + b for w, word in enumerate(words) for b in range(64) if (int(word) >> b) & 1}
        prev = os.sched_getaffinity(0)
        cores = local & prev
        if not cores:
            _HOST_AFFINITY["desc"] = "not bound (NVML gave no usable local cores)"
        elif cores == prev:
            _HOST_AFFINITY["desc"] = f"all {len(prev)} usable cores are local to the GPU (NVML)"
        else:
            os.sched_setaffinity(0, cores)
            _HOST_AFFINITY["prev"] = prev
            _HOST_AFFINITY["desc"] = f"bound to the {len(cores)} of {len(prev)} cores local to the GPU (NVML affinity)"
    except Exception as e:  # noqa: BLE001
        _HOST_AFFINITY["desc"] = f"not bound ({type(e).__name__})"
    return _HOST_AFFINITY["desc"]


def restore_host_affinity() -> None:
    """Give the process its original cores back (before an oracle baseline)."""
    if _HOST_AFFINITY["prev"] is not None:
        os.sched_setaffinity(0, _HOST_AFFINITY["prev"])
        _HOST_AFFINITY["prev"] = None


class L2Flush:
    """Leaves L2 cold and clean between timed steps: a 256 MB write (the
    flush), then a 256 MB read of a second buffer, which writes the first
    one's dirty lines back before the timed kernel starts. With the write
    alone, the timed kernel would pay for writing back up to 126 MB of the
    flush buffer's dirty lines, which are no part of its work."""

    def __init__(self, device="cuda"):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.r = torch.zeros(64 << 20, dtype=torch.int32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.sum()

    desc = "flushed between steps (256 MB write, then a 256 MB read that leaves L2 clean; untimed)"


def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of a list of floats over all ranks (identity alone)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(world: int, seqs_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank decodes its own batch each step (weak
    scaling); the job takes as long as its slowest rank."""
    return world * seqs_per_rank * steps / (max_ms * 1e-3)


# --------------------------------------------------------------- CPU oracle


def _compact(sub: dict, bs: int):
    """Renumber the blocks a sample uses to 0..n-1 (relabelling physical blocks
    leaves attention unchanged), so the host pools hold only those blocks."""
    bt = sub["block_tables"].long()
    used = torch.unique(bt[bt >= 0])
    remap = torch.full((int(used.max()) + 1,), -1, dtype=torch.long)
    remap[used] = torch.arange(used.numel())
    out = dict(sub)
    out["block_tables"] = torch.where(bt >= 0, remap[bt.clamp(min=0)], bt).to(torch.int32)

    def slots(s):
        s = s.long()
        return torch.where(s >= 0, remap[(s // bs).clamp(min=0)] * bs + s % bs, s).to(torch.int32)

    out["slot_hist"] = slots(sub["slot_hist"])
    out["slot_new"] = slots(sub["slot_new"])
    return out, int(used.numel())


def oracle_sample_runner(wl: W.Workload, ids, threads: int):
    """Prepare host pools for a sample (untimed); return a function that runs
    the sample's step (store the new tokens, attend) on the CPU oracle."""
    import oracle as O

    c = wl.cfg
    sub, nblk = _compact(W.subset_for_seqs(wl, ids), c.block_size)
    fill = W.CANARY_FP8 if wl.is_fp8 else W.CANARY_BF16
    kp = O.new_pool(nblk, c.num_kv_heads, c.block_size, c.head_dim, wl.is_fp8, fill)
    vp = O.new_pool(nblk, c.num_kv_heads, c.block_size, c.head_dim, wl.is_fp8, fill)
    ks = wl.k_scale.cpu() if wl.k_scale is not None else None
    vs = wl.v_scale.cpu() if wl.v_scale is not None else None
    if wl.token_scales:
        ks = O.new_scale_pool(nblk, c.num_kv_heads, c.block_size)
        vs = O.new_scale_pool(nblk, c.num_kv_heads, c.block_size)
    O.store_kvcache(sub["k_hist"], sub["v_hist"], kp, vp, sub["slot_hist"], nblk, c.block_size, ks, vs)

    def step(num_threads=threads):
        O.store_kvcache(sub["k_new"], sub["v_new"], kp, vp, sub["slot_new"], nblk, c.block_size, ks, vs)
        out, st = O.paged_attention_decode(sub["q"], kp, vp, sub["block_tables"], sub["context_lens"],
                                           c.num_kv_heads, c.block_size, c.softmax_scale, ks, vs,
                                           num_threads=num_threads)
        return st

    return step


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def probe_size(wl: W.Workload, order, threads: int, max_tokens: int = 32768) -> int:
    """Sequences in a probe sample: at least one, at most max(threads, 4), and
    no more than max_tokens context tokens beyond the first. Preparing a
    sample stores its history through the oracle, which for an E4M3 cache
    costs far more per token than attending (the plain encoder searches the
    code table), so long contexts get a short probe."""
    lens = wl.context_lens.cpu()
    cap = min(len(order), max(threads, 4))
    n, toks = 0, 0
    while n < cap and (n == 0 or toks + int(lens[order[n]]) <= max_tokens):
        toks += int(lens[order[n]])
        n += 1
    return n


def cpu_baseline(wl: W.Workload, target_s: float) -> dict:
    """Tokens/s of the oracle on a bounded sample: its preparation (untimed) and
    its step (timed) take about target_s together."""
    restore_host_affinity()
    threads = cpu_threads()
    S = wl.cfg.num_seqs
    order = torch.randperm(S, generator=torch.Generator().manual_seed(123)).tolist()
    n = probe_size(wl, order, threads)
    t0 = time.perf_counter()
    probe = oracle_sample_runner(wl, order[:n], threads)
    setup = time.perf_counter() - t0
    t0 = time.perf_counter()
    probe()
    dt = time.perf_counter() - t0
    n2 = int(min(S, max(n, n * target_s / max(dt + setup, 1e-6))))
    run = probe if n2 == n else oracle_sample_runner(wl, order[:n2], threads)
    t0 = time.perf_counter()
    st = run()
    dt = time.perf_counter() - t0
    toks = int(wl.context_lens.cpu()[order[:n2]].sum())
    # the same oracle on one thread, over the first n2 / threads sequences of the sample
    n1 = max(1, n2 // threads)
    run1 = run if n1 == n2 else (probe if n1 == n else oracle_sample_runner(wl, order[:n1], 1))
    t0 = time.perf_counter()
    st1 = run1(1)
    dt1 = time.perf_counter() - t0
    if st != 0 or st1 != 0:
        raise RuntimeError(f"the oracle returned status {st} (all cores) / {st1} (one thread) on its sample")
    return {"value": n2 / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n2} of {S} sequences ({toks} context tokens) of the same step, fp64, {dt:.2f} s, "
                      f"OpenMP over sequences; status {st}",
            "single_thread": {"value": n1 / dt1, "unit": UNIT, "cores": 1,
                              "sample": f"the first {n1} of those sequences, {dt1:.2f} s; status {st1}"}}


# --------------------------------------------------------------- reference


def run_reference(args):
    if rank_env()[1] != 0:
        return 0  # the CPU oracle runs once, on rank 0
    cfg = W.CONFIGS[args.config]
    if args.num_seqs:
        cfg = cfg.with_(num_seqs=args.num_seqs, name=f"{cfg.name}[{args.num_seqs} seqs]")
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = W.generate(cfg, args.seed, device=dev)
    threads = cpu_threads()
    S = cfg.num_seqs
    # size each step's sample so that preparing the (up to four) samples and
    # the warm-up + timed steps take about two minutes
    order = torch.randperm(S, generator=torch.Generator().manual_seed(7)).tolist()
    n0 = probe_size(wl, order, threads)
    t0 = time.perf_counter()
    probe = oracle_sample_runner(wl, order[:n0], threads)
    setup_per_seq = (time.perf_counter() - t0) / n0
    t0 = time.perf_counter()
    probe()
    per_seq = (time.perf_counter() - t0) / n0
    n_runs = min(4, args.steps + args.warmup)
    per_seq_total = n_runs * setup_per_seq + max(1, args.steps + args.warmup) * per_seq
    n = int(min(S, max(1, 120.0 / max(per_seq_total, 1e-9))))
    runs = [oracle_sample_runner(wl, order[(i * n) % S:(i * n) % S + n] or order[:n], threads)
            for i in range(n_runs)]
    for i in range(args.warmup):
        runs[i % len(runs)]()
    t0 = time.perf_counter()
    for i in range(args.steps):
        runs[i % len(runs)]()
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "sample_seqs_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{n} of {S} sequences per step, fp64 oracle, OpenMP over sequences"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line, args)
    return 0


# -------------------------------------------------------------------- ours


def run_block_manager(args):
    """Host time of the block manager on the workload's request mix.

    Admission: every request of the workload is added with its prompt (the
    shared prefix of ``prefix_tokens`` tokens, then its own tokens), hitting
    the cached prefix blocks. A decode step: one token appended to every
    sequence (the slot_mapping of store_kvcache) and the block tables and
    context lengths of all of them (the decode inputs). Timed on the host
    clock; the oracle's Python manager does the same on a bounded sample.
    """
    import numpy as np

    from paged_kv_cache_482_b200.blocks import BlockManager

    cfg = W.CONFIGS[args.config if args.config != "qwen3_8b" else "prefix_shared"]
    if args.num_seqs:
        cfg = cfg.with_(num_seqs=args.num_seqs)
    rng = np.random.default_rng(args.seed)
    S, bs = cfg.num_seqs, cfg.block_size
    prefix = rng.integers(0, 150000, cfg.prefix_tokens).tolist()
    lens = rng.integers(max(cfg.ctx_lo, 1), cfg.ctx_hi + 1, S)
    prompts = [prefix + rng.integers(0, 150000, int(n)).tolist() for n in lens]
    steps, warm = args.steps, args.warmup
    max_len = max(len(p) for p in prompts) + steps + warm
    num_blocks = S * (-(-max_len // bs)) + 16
    ids = np.arange(S, dtype=np.int64)

    def admit(m):
        hits = 0
        for i, p in enumerate(prompts):
            st, cached = m.add_sequence(i, p)
            assert st == 0
            hits += cached
        return hits

    m = BlockManager(num_blocks, bs)
    t0 = time.perf_counter()
    hits = admit(m)
    t_admit = time.perf_counter() - t0
    tokens = rng.integers(0, 150000, (steps + warm, S)).astype(np.int32)
    maxb = -(-max_len // bs)
    tables = np.empty((S, maxb), np.int32)
    lens_out = np.empty(S, np.int32)
    slots = np.empty(S, np.int32)
    for j in range(warm):
        m.append_tokens(ids, tokens[j], out=slots)
        m.block_tables(ids, maxb, tables, lens_out)
    t0 = time.perf_counter()
    for j in range(warm, warm + steps):
        m.append_tokens(ids, tokens[j], out=slots)
        m.block_tables(ids, maxb, tables, lens_out)
    step_us = (time.perf_counter() - t0) / steps * 1e6
    n_prompt = sum(len(p) for p in prompts)
    line = {
        "metric": "block manager host time per decode step (append + block tables)",
        "value": round(step_us, 2), "unit": "us/step", "higher_is_better": False, "n_gpus": 0,
        "steps": steps, "warmup": warm, "dtype": "int32", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: {S} sequences, shared prefix {cfg.prefix_tokens} tokens + "
                               f"[{cfg.ctx_lo}, {cfg.ctx_hi}] own tokens, block_size {bs}, pool {num_blocks} blocks"},
        "admission": {"value": round(n_prompt / t_admit, 1), "unit": "prompt tokens/s",
                      "cached_tokens": int(hits), "prompt_tokens": int(n_prompt)},
    }
    if not args.no_cpu_baseline:
        sys.path.insert(0, ROOT)
        from oracle.block_manager import BlockManagerOracle

        o = BlockManagerOracle(num_blocks, bs)
        t0 = time.perf_counter()
        admit(o)
        o_admit = time.perf_counter() - t0
        n_o = max(1, min(steps, 20))
        t0 = time.perf_counter()
        for j in range(n_o):
            for i in range(S):
                o.append_token(i, int(tokens[j, i]))
            for i in range(S):
                o.block_table(i)
        o_us = (time.perf_counter() - t0) / n_o * 1e6
        line["cpu_baseline"] = {"value": round(o_us, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
                                "sample": f"{n_o} steps of the same {S} sequences; admission of all prompts "
                                          f"{n_prompt / o_admit:.0f} prompt tokens/s"}
    m.close()
    emit(line, args)


# ------------------------------------------------------------------ prefill


def prefill_desc(cfg: W.PrefillConfig) -> str:
    mix = f" + {cfg.decode_seqs} decode requests" if cfg.decode_seqs else ""
    return (f"{cfg.name} chunked-prefill layer: {cfg.num_seqs} seqs x chunk U[{cfg.chunk_lo},{cfg.chunk_hi}] after "
            f"history U[{cfg.hist_lo},{cfg.hist_hi}]{mix}, {cfg.num_q_heads}q/{cfg.num_kv_heads}kv heads, head_dim "
            f"{cfg.head_dim}, block_size {cfg.block_size}, {cfg.cache_dtype} cache")


def prefill_flops(wl) -> int:
    """Causal attention FLOPs of one prefill launch: every (query token, head)
    row takes 2 d FLOPs per key for QK and 2 d per key for PV, over the
    p + 1 keys at or before its position p."""
    c = wl.cfg
    cu, ctx = wl.cu_q_lens.cpu().long(), wl.context_lens.cpu().long()
    n = cu[1:] - cu[:-1]
    keys = int((n * (ctx - n) + n * (n + 1) // 2).sum())
    return keys * c.num_q_heads * 4 * c.head_dim


def prefill_split(wl):
    """(FLOPs of the chunks longer than one token, K/V bytes that the one-token
    chunks -- decode requests, run in the decode kernel -- must read)."""
    c = wl.cfg
    cu, ctx = wl.cu_q_lens.cpu().long(), wl.context_lens.cpu().long()
    n = cu[1:] - cu[:-1]
    long_ = n > 1
    keys = int((n * (ctx - n) + n * (n + 1) // 2)[long_].sum())
    es = 1 if wl.is_fp8 else 2
    row = 2 * c.head_dim * es + (8 if wl.token_scales else 0)
    return keys * c.num_q_heads * 4 * c.head_dim, int(ctx[n == 1].sum()) * c.num_kv_heads * row


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), float(d["bf16_tflops"]), "measured"
    except Exception:  # noqa: BLE001
        return 1400.0, 1590.0, "fallback"


def prefill_oracle_sampler(wl, threads: int):
    """Host pools of the whole step (untimed) and a function that runs the
    oracle on the given (sequence, chunk row) pairs, each as a one-token
    chunk at its position (its result depends on the tokens up to it only)."""
    import oracle as O

    c = wl.cfg
    fill = W.CANARY_FP8 if wl.is_fp8 else W.CANARY_BF16
    kp = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, wl.is_fp8, fill)
    vp = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, wl.is_fp8, fill)
    ks = wl.k_scale.cpu() if wl.k_scale is not None else None
    vs = wl.v_scale.cpu() if wl.v_scale is not None else None
    if wl.token_scales:
        ks = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
        vs = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
    O.store_kvcache(wl.k_hist.cpu(), wl.v_hist.cpu(), kp, vp, wl.slot_hist.cpu(), wl.num_blocks, c.block_size, ks, vs)
    O.store_kvcache(wl.k_new.cpu(), wl.v_new.cpu(), kp, vp, wl.slot_new.cpu(), wl.num_blocks, c.block_size, ks, vs)
    q, bt = wl.q.cpu(), wl.block_tables.cpu()
    cu, cl = wl.cu_q_lens.cpu().long(), wl.context_lens.cpu().long()

    def run(pairs):
        rows = torch.tensor([int(cu[s]) + j for s, j in pairs])
        ctx = torch.tensor([int(cl[s] - (cu[s + 1] - cu[s]) + j + 1) for s, j in pairs], dtype=torch.int32)
        seqs = torch.tensor([s for s, _ in pairs])
        out, st = O.paged_attention_prefill(q[rows], kp, vp, bt[seqs], torch.arange(len(pairs) + 1, dtype=torch.int32),
                                            ctx, c.num_kv_heads, c.block_size, c.softmax_scale, ks, vs,
                                            num_threads=threads)
        return st

    return run


def prefill_sample_pairs(wl, n, seed):
    """n (sequence, chunk row) pairs drawn uniformly from the step's rows."""
    cu = wl.cu_q_lens.cpu().long()
    rows = torch.randperm(wl.total_q, generator=torch.Generator().manual_seed(seed))[:n]
    seq = torch.searchsorted(cu, rows, right=True) - 1
    return [(int(s), int(r - cu[s])) for s, r in zip(seq, rows)]


def prefill_cpu_baseline(wl, target_s: float) -> dict:
    restore_host_affinity()
    threads = cpu_threads()
    run = prefill_oracle_sampler(wl, threads)
    n = max(threads, 8)
    t0 = time.perf_counter()
    run(prefill_sample_pairs(wl, n, 1))
    dt = time.perf_counter() - t0
    n2 = int(min(wl.total_q, max(n, n * target_s / max(dt, 1e-6))))
    t0 = time.perf_counter()
    st = run(prefill_sample_pairs(wl, n2, 2))
    dt = time.perf_counter() - t0
    return {"value": n2 / dt, "unit": "query tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n2} of {wl.total_q} query tokens of the same step, drawn uniformly, each as a one-token "
                      f"chunk at its position; fp64, {dt:.2f} s, OpenMP over tokens; status {st}"}


def run_prefill_reference(args):
    if rank_env()[1] != 0:
        return 0
    cfg = W.PREFILL_CONFIGS[args.config]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = W.generate_prefill(cfg, args.seed, device=dev)
    threads = cpu_threads()
    run = prefill_oracle_sampler(wl, threads)
    n0 = max(threads, 8)
    t0 = time.perf_counter()
    run(prefill_sample_pairs(wl, n0, 1))
    per_row = (time.perf_counter() - t0) / n0
    n = int(min(wl.total_q, max(1, 120.0 / max(1, args.steps + args.warmup) / max(per_row, 1e-9))))
    for i in range(args.warmup):
        run(prefill_sample_pairs(wl, n, 10 + i))
    t0 = time.perf_counter()
    for i in range(args.steps):
        run(prefill_sample_pairs(wl, n, 100 + i))
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    unit = "query tokens/s"
    emit({
        "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": prefill_desc(cfg), "sample_rows_per_step": n},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": f"{n} of {wl.total_q} query tokens per step, each as a one-token chunk"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }, args)
    return 0


PREFILL_METRIC = "chunked-prefill paged attention query tokens/sec and achieved tensor TFLOP/s"


def prefill_dtype(wl):
    """Operand types of the prefill kernels for this cache (the tensor cores accumulate in fp32)."""
    if not wl.is_fp8:
        return "bf16 x bf16 -> fp32 (tcgen05)"
    if wl.token_scales:
        return ("e4m3 cache with per-token scales: S in f16 x f16 (K widened to f16, Q scaled per row), "
                "P V in bf16 x bf16 (V widened to bf16, P times the V scales) -> fp32 (tcgen05); "
                "chunks of one query tile or less: bf16 operands")
    return ("e4m3 cache widened to f16, Q scaled per row into f16; f16 x f16 -> fp32 (tcgen05); "
            "chunks of one query tile or less: bf16 operands")


def run_prefill(args):
    from paged_kv_cache_482_b200 import pagedkv as K

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    host_cores = bind_host_to_gpu(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    cfg = W.PREFILL_CONFIGS[args.config]
    wl = W.generate_prefill(cfg, args.seed + rank, device="cuda")
    c = cfg
    shape = (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)
    if wl.is_fp8:
        kp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device="cuda")
        vp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device="cuda")
    else:
        kp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        vp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if wl.token_scales:  # one scale per (token, KV head), written by the store
        wl.k_scale, wl.v_scale = W.scale_pools(wl.num_blocks, c.num_kv_heads, c.block_size, device="cuda")
    K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, wl.k_scale, wl.v_scale, err)
    cu = wl.cu_q_lens.cpu().long()
    mq = int((cu[1:] - cu[:-1]).max())
    out = torch.empty_like(wl.q)
    # E4M3: the widening workspace (allocated once, like a serving engine would)
    ws = None
    if wl.is_fp8 and not args.no_staging:
        nbytes = K.prefill_workspace_bytes(wl.block_tables.shape[0], c.num_kv_heads, c.head_dim,
                                           wl.block_tables.shape[1], c.block_size,
                                           K.PKV_CACHE_FP8_E4M3_TOKEN if wl.token_scales else K.PKV_CACHE_FP8_E4M3)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda") if nbytes else None
    long_chunks = mq > 128 // c.group

    def step(q, k_new, v_new, slot_new, bt, cu_d, cl):
        K.store_kvcache(k_new, v_new, kp, vp, slot_new, wl.k_scale, wl.v_scale, err)
        K.paged_attention_prefill(q, kp, vp, bt, cu_d, cl, c.softmax_scale, mq, out=out, k_scale=wl.k_scale,
                                  v_scale=wl.v_scale, dev_err=err, workspace=ws)

    inputs = (wl.q, wl.k_new, wl.v_new, wl.slot_new, wl.block_tables, wl.cu_q_lens, wl.context_lens)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        step(*inputs)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())} during warm-up")

    sampler = make_sampler(local) if local == 0 else None
    if sampler:
        sampler.wait_first()
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kst)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    e_start.record(stream)
    for k in range(Kst):
        ev[k][0].record(stream)
        K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale, err)
        ev[k][1].record(stream)
        K.paged_attention_prefill(wl.q, kp, vp, wl.block_tables, wl.cu_q_lens, wl.context_lens, c.softmax_scale, mq,
                                  out=out, k_scale=wl.k_scale, v_scale=wl.v_scale, dev_err=err, workspace=ws)
        ev[k][2].record(stream)
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    elapsed_ms = e_start.elapsed_time(e_end)
    attn_ms = statistics.mean(ev[k][1].elapsed_time(ev[k][2]) for k in range(Kst))
    store_ms = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(Kst))
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None
    if sampler:
        sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())} in the timed steps")

    # end to end: pinned host inputs -> device -> store + prefill -> host output, every step
    host_in = [t.cpu().pin_memory() for t in inputs]
    dev_in = [torch.empty_like(t) for t in inputs]
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out.numel() * host_out.element_size()

    def e2e_step():
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        step(*dev_in)
        host_out.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = x0.elapsed_time(x1)
    elapsed_ms, attn_ms, e2e_ms = max_over_ranks([elapsed_ms, attn_ms, e2e_ms], dist, device="cuda")

    if rank == 0:
        flops = prefill_flops(wl)
        peak_sus, peak_burst, kind = measured_tensor_peak()
        achieved = flops / (attn_ms * 1e-3) / 1e12
        T = wl.total_q
        line = {
            "metric": PREFILL_METRIC, "value": world * T * Kst / (elapsed_ms * 1e-3), "unit": "query tokens/s",
            "n_gpus": world, "steps": Kst, "warmup": args.warmup, "ms_per_step": elapsed_ms / Kst,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": prefill_dtype(wl), "data": "synthetic",
            "config": {"workload": prefill_desc(c), "query_tokens": T, "kv_tokens": int(wl.context_lens.sum()),
                       "max_q_len": mq, "seed": args.seed,
                       "e4m3_widening": (None if not wl.is_fp8 else
                                         "once per call into a workspace" if ws is not None else "in every CTA"),
                       "parallelism": f"replicas x{world} (independent batches, no collective)",
                       "host_cores": host_cores,
                       "l2": "no flush: each step's pools and queries exceed 126 MB of L2"},
            "attention_us": attn_ms * 1e3, "store_us": store_ms * 1e3,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_sus, "unit": "TFLOP/s",
                         "frac": achieved / peak_sus, "traffic": None,
                         "kernel": ("paged_prefill_ws_kernel (+ widen_kv_kernel, paged_prefill_kernel, decode)"
                                    if ws is not None and long_chunks else
                                    "paged_prefill_ws_kernel (+ paged_prefill_kernel, decode)"),
                         "peak_source": f"{kind} cuBLAS bf16 GEMM, sustained (bf16_tflops_sustained); "
                                        f"burst {peak_burst}",
                         "algorithmic_flops_per_launch": flops,
                         "flops_note": "causal: 4 * head_dim FLOPs per (query row, head, key at or before it)"},
            "e2e": {"value": world * T * args.e2e_steps / (e2e_ms * 1e-3), "unit": "query tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
            # per step: the store, the one-tile kernel (short chunks), the decode
            # kernel (one-token chunks) and, when some chunk is longer than
            # 128 / G tokens, the warp-specialised kernel (after the widening
            # kernel when an E4M3 workspace is given)
            "gpu_launches": (2 if mq <= 1 else 3 + (1 + (1 if ws is not None else 0) if long_chunks else 0)) * Kst,
            "clocks": clocks,
        }
        chunk_flops, decode_bytes = prefill_split(wl)
        if decode_bytes:  # a mixed batch: tensor work and a K/V stream at once
            hbm, _ = measured_peak()
            t_tc, t_hbm = chunk_flops / (peak_sus * 1e12) * 1e6, decode_bytes / (hbm * 1e9) * 1e6
            line["mixed_bound"] = {
                "chunk_flops": chunk_flops, "decode_kv_bytes": decode_bytes,
                "tensor_us": t_tc, "hbm_us": t_hbm, "lower_bound_us": max(t_tc, t_hbm),
                "frac": max(t_tc, t_hbm) / (attn_ms * 1e3),
                "note": "the roofline above counts FLOPs only; the one-token chunks are a K/V stream. Lower "
                        "bound of the call: the larger of the chunks' FLOPs at the sustained tensor peak and "
                        "the decode rows' K/V bytes at the measured copy bandwidth (perfect overlap)"}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = prefill_cpu_baseline(wl, args.cpu_seconds)
        emit(line, args)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------ add + RMSNorm

NORM_METRIC = "fused residual add + RMSNorm rows/sec and achieved HBM GB/s"


def norm_desc(cfg) -> str:
    return (f"{cfg.name} residual add + RMSNorm: {cfg.num_tokens} rows x hidden {cfg.hidden}, eps {cfg.eps}, "
            f"{'with' if cfg.residual else 'without'} residual, bf16")


def norm_bytes(cfg) -> int:
    """Bytes one launch must move: x read and out written, the residual read
    and written back, the weight read once."""
    per = (4 if cfg.residual else 2) * 2
    return cfg.num_tokens * cfg.hidden * per + cfg.hidden * 2


def norm_cpu_baseline(wl, target_s: float) -> dict:
    restore_host_affinity()
    import oracle as O

    threads = cpu_threads()
    c = wl.cfg
    x, r, w = wl.x.cpu(), (wl.residual.cpu() if wl.residual is not None else None), wl.weight.cpu()
    n = max(1, min(c.num_tokens, 64))
    t0 = time.perf_counter()
    O.fused_add_rmsnorm(x[:n], r[:n] if r is not None else None, w, c.eps, num_threads=threads)
    dt = time.perf_counter() - t0
    n2 = int(min(c.num_tokens, max(n, n * target_s / max(dt, 1e-6))))
    t0 = time.perf_counter()
    _, _, st = O.fused_add_rmsnorm(x[:n2], r[:n2] if r is not None else None, w, c.eps, num_threads=threads)
    dt = time.perf_counter() - t0
    return {"value": n2 / dt, "unit": "rows/s", "cores": threads, "kind": "oracle",
            "sample": f"the first {n2} of {c.num_tokens} rows, fp64, {dt:.2f} s, OpenMP over rows; status {st}"}


def run_norm_reference(args):
    if rank_env()[1] != 0:
        return 0
    import oracle as O

    cfg = W.NORM_CONFIGS[args.config]
    wl = W.generate_norm(cfg, args.seed, device="cuda" if torch.cuda.is_available() else "cpu")
    threads = cpu_threads()
    x, r, w = wl.x.cpu(), (wl.residual.cpu() if wl.residual is not None else None), wl.weight.cpu()
    n = cfg.num_tokens
    for _ in range(args.warmup):
        O.fused_add_rmsnorm(x, r, w, cfg.eps, num_threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.fused_add_rmsnorm(x, r, w, cfg.eps, num_threads=threads)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    emit({
        "impl": "reference", "metric": NORM_METRIC, "value": value, "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": norm_desc(cfg)},
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": threads, "kind": "oracle",
                         "sample": f"all {n} rows per step, fp64, OpenMP over rows"},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }, args)
    return 0


def run_norm(args):
    from paged_kv_cache_482_b200 import pagedkv as K

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    host_cores = bind_host_to_gpu(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    cfg = W.NORM_CONFIGS[args.config]
    wl = W.generate_norm(cfg, args.seed + rank, device="cuda")
    x, r, w = wl.x, wl.residual, wl.weight
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        K.fused_add_rmsnorm(x, r, w, cfg.eps, out=out)
    torch.cuda.synchronize()
    # inputs larger than L2 (checked) or L2 flushed between steps
    moved = norm_bytes(cfg)
    flush = L2Flush() if moved < (256 << 20) else None
    sampler = make_sampler(local) if local == 0 else None
    if sampler:
        sampler.wait_first()
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kst)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for k in range(Kst):
        if flush is not None:
            flush()
        ev[k][0].record(stream)
        K.fused_add_rmsnorm(x, r, w, cfg.eps, out=out)
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    times = [ev[k][0].elapsed_time(ev[k][1]) for k in range(Kst)]
    total_ms = sum(times)
    kern_ms = statistics.mean(times)
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None
    if sampler:
        sampler.stop()

    host_in = [t.cpu().pin_memory() for t in (x, r) if t is not None]
    dev_in = [torch.empty_like(t) for t in (x, r) if t is not None]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2 if r is not None else 1)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    def e2e_step():
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        K.fused_add_rmsnorm(dev_in[0], dev_in[1] if r is not None else None, w, cfg.eps, out=out)
        host_out[0].copy_(out, non_blocking=True)
        if r is not None:
            host_out[1].copy_(dev_in[1], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = x0.elapsed_time(x1)
    total_ms, kern_ms, e2e_ms = max_over_ranks([total_ms, kern_ms, e2e_ms], dist, device="cuda")
    if rank == 0:
        peak, kind = measured_peak()
        achieved = moved / (kern_ms * 1e-3) / 1e9
        T = cfg.num_tokens
        line = {
            "metric": NORM_METRIC, "value": world * T * Kst / (total_ms * 1e-3), "unit": "rows/s", "n_gpus": world,
            "steps": Kst, "warmup": args.warmup, "ms_per_step": total_ms / Kst, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in/out, fp32 arithmetic", "data": "synthetic",
            "config": {"workload": norm_desc(cfg), "seed": args.seed,
                       "parallelism": f"replicas x{world} (independent rows, no collective)",
                       "host_cores": host_cores,
                       "l2": (L2Flush.desc if flush is not None else
                              f"no flush: {moved / 1e6:.0f} MB moved per step, above the 126 MB L2")},
            "kernel_us": kern_ms * 1e3,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": None, "kernel": "fused_add_rmsnorm_kernel",
                         "peak_source": f"{kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                         "algorithmic_bytes_per_launch": moved,
                         "bytes_note": "x and residual read, residual and out written, weight read once"},
            "e2e": {"value": world * T * args.e2e_steps / (e2e_ms * 1e-3), "unit": "rows/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
            "gpu_launches": Kst,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = norm_cpu_baseline(wl, args.cpu_seconds)
        emit(line, args)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------- rotary embedding + store

ROPE_METRIC = "fused RoPE + store_kvcache tokens/sec and achieved HBM GB/s"


def rope_desc(cfg) -> str:
    style = "half pairs (i, i+d/2)" if cfg.style == W.ROPE_HALF else "neighbour pairs (2i, 2i+1)"
    return (f"{cfg.name}: {cfg.num_tokens} tokens at positions < {cfg.max_position}, {cfg.num_q_heads}q/"
            f"{cfg.num_kv_heads}kv heads, head_dim {cfg.head_dim}, block_size {cfg.block_size}, {cfg.cache_dtype} "
            f"cache, {style}")


def rope_bytes(cfg) -> int:
    """Bytes one launch must move: q in and out, k and v in, the two cache
    rows out (plus per-token scales), each token's table row, positions and
    slots."""
    N, nq, nkv, d = cfg.num_tokens, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    es = 1 if cfg.is_fp8 else 2
    return (N * nq * d * 2 * 2 + N * nkv * d * 2 * 2 + N * nkv * d * es * 2 + (N * nkv * 8 if cfg.token_scales else 0)
            + N * d * 4 + N * 8)


def _rope_pools(wl, device="cuda"):
    c = wl.cfg
    shape = (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)
    if c.is_fp8:
        kp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device=device)
    else:
        kp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device=device).view(torch.bfloat16)
    vp = kp.clone()
    if c.token_scales:
        ks, vs = W.scale_pools(wl.num_blocks, c.num_kv_heads, c.block_size, device=device)
    else:
        ks, vs = wl.k_scale, wl.v_scale
    return kp, vp, ks, vs


def rope_cpu_baseline(wl, target_s: float) -> dict:
    restore_host_affinity()
    import oracle as O

    threads = cpu_threads()
    c = wl.cfg
    q, k, v, pos, sl, cs = (t.cpu() for t in (wl.q, wl.k, wl.v, wl.positions, wl.slot_mapping, wl.cos_sin))
    ks, vs = wl.k_scale, wl.v_scale
    hk = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, c.is_fp8, 0)
    hv = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, c.is_fp8, 0)
    if c.token_scales:
        ks = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
        vs = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
    elif ks is not None:
        ks, vs = ks.cpu(), vs.cpu()

    def run(n):
        return O.store_kvcache_rope(q[:n], k[:n], v[:n], hk, hv, sl[:n], pos[:n], cs, wl.num_blocks, c.block_size,
                                    ks, vs, style=c.style)[1]

    n = max(1, min(c.num_tokens, 64))
    t0 = time.perf_counter()
    run(n)
    dt = time.perf_counter() - t0
    n2 = int(min(c.num_tokens, max(n, n * target_s / max(dt, 1e-6))))
    t0 = time.perf_counter()
    st = run(n2)
    dt = time.perf_counter() - t0
    if st != 0:
        raise RuntimeError(f"the oracle returned status {st} on its sample")
    return {"value": n2 / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"the first {n2} of {c.num_tokens} tokens, binary32 rotation + store, {dt:.2f} s, "
                      f"one thread; status {st}"}


def run_rope_reference(args):
    if rank_env()[1] != 0:
        return 0
    cfg = W.ROPE_CONFIGS[args.config]
    wl = W.generate_rope(cfg, args.seed)
    per_step = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    vals = [rope_cpu_baseline(wl, per_step)["value"] for _ in range(args.warmup + args.steps)][args.warmup:]
    value = statistics.mean(vals)
    emit({
        "impl": "reference", "metric": ROPE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": cfg.num_tokens / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": rope_desc(cfg)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "a bounded prefix of the step's tokens per step, one thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }, args)
    return 0


def run_rope(args):
    from paged_kv_cache_482_b200 import pagedkv as K

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    host_cores = bind_host_to_gpu(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    cfg = W.ROPE_CONFIGS[args.config]
    wl = W.generate_rope(cfg, args.seed + rank, device="cuda")
    kp, vp, ks, vs = _rope_pools(wl)
    q_out = torch.empty_like(wl.q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(q, k, v, pos, sl):
        K.store_kvcache_rope(k, v, kp, vp, sl, pos, wl.cos_sin, q=q, q_out=q_out, style=cfg.style, k_scale=ks,
                             v_scale=vs, dev_err=err)

    args_dev = (wl.q, wl.k, wl.v, wl.positions, wl.slot_mapping)
    for _ in range(max(3, args.warmup)):
        step(*args_dev)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())} during warm-up")
    moved = rope_bytes(cfg)
    flush = L2Flush() if moved < (256 << 20) else None
    stream = torch.cuda.current_stream()
    sampler = make_sampler(local) if local == 0 else None
    if sampler:
        sampler.wait_first()
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kst)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for kk in range(Kst):
        if flush is not None:
            flush()
        ev[kk][0].record(stream)
        step(*args_dev)
        ev[kk][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    times = [ev[kk][0].elapsed_time(ev[kk][1]) for kk in range(Kst)]
    total_ms, kern_ms = sum(times), statistics.mean(times)
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None
    if sampler:
        sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())} in the timed steps")

    host_in = [t.cpu().pin_memory() for t in args_dev]
    dev_in = [torch.empty_like(t) for t in args_dev]
    host_out = torch.empty(q_out.shape, dtype=q_out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out.numel() * host_out.element_size()

    def e2e_step():
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        step(*dev_in)
        host_out.copy_(q_out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = x0.elapsed_time(x1)
    total_ms, kern_ms, e2e_ms = max_over_ranks([total_ms, kern_ms, e2e_ms], dist, device="cuda")
    if rank == 0:
        peak, kind = measured_peak()
        achieved = moved / (kern_ms * 1e-3) / 1e9
        N = cfg.num_tokens
        line = {
            "metric": ROPE_METRIC, "value": world * N * Kst / (total_ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": Kst, "warmup": args.warmup, "ms_per_step": total_ms / Kst, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("bf16 in, binary32 rotation, " + ("e4m3" if cfg.is_fp8 else "bf16") + " cache"),
            "data": "synthetic",
            "config": {"workload": rope_desc(cfg), "seed": args.seed,
                       "parallelism": f"replicas x{world} (independent tokens, no collective)",
                       "host_cores": host_cores,
                       "l2": (L2Flush.desc if flush is not None else
                              f"no flush: {moved / 1e6:.0f} MB moved per step, above the 126 MB L2")},
            "kernel_us": kern_ms * 1e3,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": None, "kernel": "store_kvcache_rope_kernel",
                         "peak_source": f"{kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                         "algorithmic_bytes_per_launch": moved,
                         "bytes_note": "q in/out, k and v in, cache rows (and scales) out, table rows, positions, slots"},
            "e2e": {"value": world * N * args.e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
            "gpu_launches": Kst,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = rope_cpu_baseline(wl, args.cpu_seconds)
        emit(line, args)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.config in W.ROPE_CONFIGS:
        return run_rope_reference(args) if args.impl == "reference" else run_rope(args)
    if args.component == "block_manager":
        return run_block_manager(args)
    if args.config in W.NORM_CONFIGS:
        return run_norm_reference(args) if args.impl == "reference" else run_norm(args)
    if args.config in W.PREFILL_CONFIGS:
        return run_prefill_reference(args) if args.impl == "reference" else run_prefill(args)
    if args.impl == "reference":
        return run_reference(args)

    from paged_kv_cache_482_b200 import pagedkv as K

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    host_cores = bind_host_to_gpu(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    cfg = W.CONFIGS[args.config]
    if args.num_seqs:
        cfg = cfg.with_(num_seqs=args.num_seqs, name=f"{cfg.name}[{args.num_seqs} seqs]")
    wl = W.generate(cfg, args.seed + rank, device="cuda")
    c = cfg
    shape = (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)
    if wl.is_fp8:
        kp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device="cuda")
        vp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device="cuda")
    else:
        kp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        vp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    if wl.token_scales:  # one scale per (token, KV head), written by the store
        wl.k_scale, wl.v_scale = W.scale_pools(wl.num_blocks, c.num_kv_heads, c.block_size, device="cuda")
    H = wl.k_hist.shape[0]
    for i in range(0, H, 1 << 20):
        j = min(H, i + (1 << 20))
        K.store_kvcache(wl.k_hist[i:j], wl.v_hist[i:j], kp, vp, wl.slot_hist[i:j], wl.k_scale, wl.v_scale)
    # a batch whose sequences share a cached prefix goes through the shared-prefix (cascade) call, as an
    # engine with a prefix cache would issue it (the groups come from the block manager's hits)
    shared = bool(c.prefix_tokens) and not args.no_shared_prefix
    groups = (wl.group_bounds, wl.group_prefix, c.num_seqs) if shared else None
    step = K.DecodeStep(kp, vp, c.num_seqs, c.num_q_heads, wl.block_tables.shape[1], c.softmax_scale,
                        wl.k_scale, wl.v_scale, max_context_len=c.max_context, partition_request=args.partition,
                        groups=groups)
    inputs = (wl.q, wl.k_new, wl.v_new, wl.slot_new, wl.block_tables, wl.context_lens)
    # store + decode (+ reduce when split); shared prefix: store + prefix + decode + merge
    launches_per_step = 4 if shared else 2 + (1 if step.plan["partition_tokens"] > 0 else 0)
    # The scheduler knows the lengths on the host: visit the longest sequences first.
    order = None if args.natural_order else K.longest_first(wl.context_lens.cpu()).cuda()

    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        step.run(*inputs, seq_order=order)
    torch.cuda.synchronize()
    if int(step.dev_err.item()) != 0:
        raise RuntimeError(f"device error word {int(step.dev_err.item())} during warm-up")

    sampler = make_sampler(local) if local == 0 else None
    if sampler:
        sampler.wait_first()
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kst)]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    def store():
        K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale, step.dev_err)

    def decode():
        if shared:
            K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                                   step.groups[0], step.groups[1], step.groups[2], out=step.out,
                                                   k_scale=wl.k_scale, v_scale=wl.v_scale,
                                                   max_context_len=c.max_context, partition_request=args.partition,
                                                   workspace=step.workspace, dev_err=step.dev_err)
        else:
            K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale, out=step.out,
                                     k_scale=wl.k_scale, v_scale=wl.v_scale, max_context_len=c.max_context,
                                     partition_request=args.partition, workspace=step.workspace,
                                     dev_err=step.dev_err, seq_order=order)

    if not args.no_graph:  # each half of the step recorded once as a CUDA graph, replayed every step
        store, decode = K.graphed(store), K.graphed(decode)
        torch.cuda.synchronize()
    e_start.record(stream)
    for k in range(Kst):
        ev[k][0].record(stream)
        store()
        ev[k][1].record(stream)
        decode()
        ev[k][2].record(stream)
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    elapsed_ms = e_start.elapsed_time(e_end)
    decode_ms = statistics.mean(ev[k][1].elapsed_time(ev[k][2]) for k in range(Kst))
    store_ms = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(Kst))
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None
    if sampler:
        sampler.stop()
    if int(step.dev_err.item()) != 0:
        raise RuntimeError(f"device error word {int(step.dev_err.item())} in the timed steps")

    # end to end: pinned host inputs -> device -> step -> host output, every step
    host_in = [t.cpu().pin_memory() for t in inputs]
    host_out = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    # inputs plus the longest-first order that run_host computes and uploads each step
    h2d = sum(t.numel() * t.element_size() for t in host_in) + 4 * c.num_seqs
    if shared:  # the groups' bounds and prefix lengths
        h2d += 4 * (2 * len(wl.group_prefix) + 1)
    d2h = host_out.numel() * host_out.element_size()
    for _ in range(3):
        step.run_host(*host_in, host_out)
    step.flush(stream)  # the timed copies start after x0
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    x0 = torch.cuda.Event(enable_timing=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(args.e2e_steps):
        step.run_host(*host_in, host_out)
    step.flush(stream)  # x1 after the last output copy
    x1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = x0.elapsed_time(x1)

    elapsed_ms, decode_ms, e2e_ms = max_over_ranks([elapsed_ms, decode_ms, e2e_ms], dist, device="cuda")

    if rank == 0:
        ab = algorithmic_bytes(wl)
        peak, peak_kind = measured_peak()
        bytes_launch = ab["unique_total"] if c.prefix_tokens else ab["total"]
        achieved = bytes_launch / (decode_ms * 1e-3) / 1e9
        pt = step.plan["partition_tokens"]
        traffic = recorded_traffic(c.name, pt)
        value = job_throughput(world, c.num_seqs, Kst, elapsed_ms)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": Kst, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / Kst, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if wl.is_fp8 else "bf16", "data": "synthetic",
            "config": {
                "workload": workload_desc(c), "num_seqs": c.num_seqs, "seq_len": "ctx " + (
                    f"{c.prefix_tokens}+U[{c.ctx_lo},{c.ctx_hi}]" if c.prefix_tokens else f"U[{c.ctx_lo},{c.ctx_hi}]"),
                "kv_tokens": wl.kv_tokens(), "seed": args.seed, "partition_tokens": pt,
                "schedule": ("shared-prefix cascade: each group's prefix once for all its members (tensor "
                             "cores) beside the suffixes, in batch order" if shared else
                             ("batch order" if args.natural_order else
                              "longest sequence first (order from host lengths)")),
                "launch": "Python calls" if args.no_graph else "CUDA graphs of the store and of the decode, replayed",
                "parallelism": f"replicas x{world} (independent batches, no collective)",
                "host_cores": host_cores,
                "l2": f"no flush: {ab['kv'] / 1e9:.2f} GB of KV read per step, far above the 126 MB L2",
            },
            "attention_us": decode_ms * 1e3,
            "store_us": store_ms * 1e3,
            "hbm_gbs": achieved,
            "hbm_pct_of_8tbs": 100.0 * achieved / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": (("paged_prefix_mma_kernel + " if shared else "") +
                                    ("paged_decode_mma_kernel" if c.head_dim == 128 else "paged_decode_kernel") +
                                    (" + paged_decode_reduce_kernel" if pt > 0 or shared else "")),
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                         "algorithmic_bytes_per_launch": bytes_launch,
                         "bytes_note": ("unique bytes: shared prefix counted once" if c.prefix_tokens else
                                        "KV rows of every context token + q + out + block-table entries")},
            "e2e": {"value": job_throughput(world, c.num_seqs, args.e2e_steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
            "gpu_launches": launches_per_step * Kst,
            "clocks": clocks,
        }
        if c.prefix_tokens:
            line["logical_gbs"] = ab["total"] / (decode_ms * 1e-3) / 1e9
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
        emit(line, args)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
