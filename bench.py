"""Batch-1 decode benchmark of the hybrid Gated-DeltaNet + attention megakernel.

Workload: the 0.8B-shaped hybrid (24 layers, [D,D,D,A] x 6, hidden 1024, vocab
151936, bf16 weights from N(0, 0.02), seed 1), a 128-token uniform random prompt,
then tg128: 128 greedy decode steps at batch 1. One bench step = restore the
post-prompt state, then 128 decode launches (one kernel launch per token).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {mk,reference}] [--workload {tg128,long}]

--workload long times the long-context variant instead: the same model with a seeded
32768-position bf16 KV cache in every attention layer (N(0, 1), RoPE applied) and
DeltaNet states from N(0, 0.1), then 128 greedy decode steps from position 32768.

Prints one JSON line (rank 0). With --gpus N > 1 (launched by torchrun) every rank
runs an independent replica on its own GPU; there is no data-path collective.
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
from typing import Optional

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "batch-1 decode tok/s (hybrid DeltaNet, tg128) and % of B200 HBM roofline"
PROMPT = 128
TG = 128
MAX_CTX = PROMPT + TG + 16
LONG_POS = 32768
WORKLOAD = ("0.8B-shaped hybrid Gated-DeltaNet + attention (24 layers [D,D,D,A]x6, hidden 1024, "
            "vocab 151936 tied, DeltaNet 16 heads dk=dv=128, attention 8q/2kv heads D=256, SwiGLU 3584), "
            "bf16 weights N(0,0.02) seed 1, 128-token random prompt, tg128 greedy decode, batch 1")
LONG_WORKLOAD = ("0.8B-shaped hybrid (as tg128), long context: seeded bf16 KV cache of 32768 positions per "
                 "attention layer (N(0,1), RoPE applied, seed 3), DeltaNet states N(0,0.1), then 128 greedy "
                 "decode steps at batch 1 from position 32768")
LONG_Q8_WORKLOAD = ("0.8B-shaped hybrid (as tg128), long context with the 8-bit KV cache (blocks of 32, fp16 "
                    "scales): a 32768-token random prompt prefilled through the library, then 128 greedy decode "
                    "steps at batch 1 from position 32768")
KERNEL_SOURCES = ["hybrid_deltanet_attention_b200/csrc/decode.cu", "hybrid_deltanet_attention_b200/csrc/dev.cuh",
                  "hybrid_deltanet_attention_b200/csrc/mk_internal.h"]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def bytes_per_token(cfg, pos: int, kv_row_bytes: int = 0) -> dict:
    """Algorithmic bytes one decode step at position `pos` reads (and writes); kv_row_bytes:
    bytes of one cache row (0: bf16, 2 * D)."""
    H, V, F = cfg.hidden, cfg.vocab, cfg.ffn
    w = V * H * 2 + H * 2                                  # tied LM head + final gain
    for kind in cfg.pattern:
        w += 2 * H * 2 + 3 * F * H * 2                     # gains, gate, up, down
        if kind == "D":
            w += cfg.dn_in_rows * H * 2 + cfg.dn_conv_channels * cfg.conv_width * 2
            w += H * cfg.dn_heads * cfg.dn_dv * 2
        else:
            w += cfg.at_in_rows * H * 2 + H * cfg.at_q_heads * cfg.at_head_dim * 2
    s = cfg.n_dn * cfg.dn_heads * cfg.dn_dv * cfg.dn_dk * 4
    conv = cfg.n_dn * cfg.conv_width * cfg.dn_conv_channels * 4
    kv = cfg.n_at * cfg.at_kv_heads * (pos + 1) * (kv_row_bytes or 2 * cfg.at_head_dim) * 2
    return {"weights": w, "state": s, "conv": conv, "kv": kv, "read": w + s + conv + kv,
            "write": s + cfg.n_dn * cfg.dn_conv_channels * 4 + cfg.n_at * cfg.at_kv_heads * cfg.at_head_dim * 4}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(khash: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on this kernel."""
    p = os.path.join(ROOT, "profiles", "decode_0.8b_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as fh:
        for line in fh:
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_hash") != khash:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 6:
                    continue
                try:
                    sms.append(float(parts[0]))
                    mx = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[2:6]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sms)}


class EnergyMeter:
    """Energy this GPU drew over the timed region, from NVML's total-energy counter
    (millijoules since the driver loaded). Read only: nothing is set or reset. The GPU
    is found by its PCI bus id (the CUDA index can differ from NVML's), else by index.
    The counter advances in steps of tens of milliseconds and the board is shared with
    other jobs' idle draw, so the figure is advisory. `nvml` may be a stand-in module."""

    def __init__(self, cuda_index: int, pci_bus_id: Optional[str] = None, nvml=None):
        self.index, self.bus, self.nv = cuda_index, pci_bus_id, nvml
        self.h = None
        self.e0 = self.e1 = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            if self.nv is None:
                import pynvml
                self.nv = pynvml
            self.nv.nvmlInit()
            h = None
            if self.bus:
                try:
                    h = self.nv.nvmlDeviceGetHandleByPciBusId(self.bus)
                except Exception:
                    h = None
            self.h = h if h is not None else self.nv.nvmlDeviceGetHandleByIndex(self.index)
        except Exception:
            self.h = None
        return self

    def _read(self):
        try:
            return float(self.nv.nvmlDeviceGetTotalEnergyConsumption(self.h))
        except Exception:
            return None

    def start(self):
        if self.h is not None:
            self.e0, self.t0 = self._read(), time.perf_counter()

    def stop(self):
        if self.h is not None:
            self.e1, self.t1 = self._read(), time.perf_counter()

    def __exit__(self, *a):
        if self.h is not None:
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self, tokens: int):
        if self.e0 is None or self.e1 is None or self.e1 < self.e0 or tokens <= 0:
            return None
        j = (self.e1 - self.e0) / 1000.0
        sec = max(self.t1 - self.t0, 1e-9)
        return {"joules": j, "seconds": sec, "avg_w": j / sec, "j_per_token": j / tokens,
                "tokens_per_j": tokens / j if j > 0 else None,
                "source": "NVML total-energy counter of this GPU before and after the timed region (read only; "
                          "advisory: counter granularity, shared board)"}


def cuda_pci_bus_id(torch, index: int) -> Optional[str]:
    try:
        p = torch.cuda.get_device_properties(index)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


def dist_setup(n_gpus: int):
    import torch
    if n_gpus > 1 or int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return dist.get_rank(), dist.get_world_size(), local
    torch.cuda.set_device(0)
    return 0, 1, 0


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over the ranks (a time: the slowest replica defines the job's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput of `world` independent replicas that each processed
    `units_per_rank` units, timed by the slowest one (weak scaling)."""
    return world * units_per_rank / seconds


# ------------------------------------------------------------------ oracle (CPU) timing
_ORACLE_W = None


def oracle_sample(seconds_budget: float = 15.0, n_prompt: int = 16, n_decode: int = 64):
    """Time the CPU oracle on a bounded sample of the same workload: weights prepared
    untimed, a short prompt fed untimed, then n_decode greedy steps timed."""
    import oracle
    import synth
    cfg = synth.QWEN_08B
    global _ORACLE_W
    if _ORACLE_W is None:   # prepared once per process (untimed)
        _ORACLE_W = oracle.prepare_weights(cfg, synth.make_weights(cfg))
    W = _ORACLE_W
    st = oracle.new_state(cfg, n_prompt + n_decode + 1)
    z = oracle.prefill(cfg, W, st, synth.make_prompt(cfg, n_prompt))
    tok = int(np.argmax(z))
    t0 = time.perf_counter()
    done = 0
    for _ in range(n_decode):
        z = oracle.decode_step(cfg, W, st, tok)
        tok = int(np.argmax(z))
        done += 1
        if time.perf_counter() - t0 > seconds_budget:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    sample = (f"oracle (numpy float64) on the 0.8B-shaped model: {done} greedy decode steps at positions "
              f"{n_prompt}..{n_prompt + done - 1} after a {n_prompt}-token prompt (prompt and weight preparation untimed)")
    return done / dt, cores, sample


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals = []
    cores, sample = 1, ""
    for _ in range(args.warmup + args.steps):
        v, cores, sample = oracle_sample(seconds_budget=6.0, n_prompt=8, n_decode=16)
        vals.append(v)
    timed = vals[args.warmup:]
    value = float(np.mean(timed))
    line = {
        "metric": METRIC, "impl": "reference", "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 16 * 1000.0 / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "reference": "the CPU oracle (numpy float64), bounded sample per step"},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ the CUDA path
def seed_long_context(m, cfg, n_pos, dev):
    """Write the seeded long-context state into the model's state buffer."""
    import torch
    import synth
    ks, vs, ss = synth.long_context_state(cfg, n_pos)
    m.reset()
    kc, vc, S = m.k_cache, m.v_cache, m.S
    for ai in range(cfg.n_at):
        kc[ai, :, :n_pos] = torch.from_numpy(ks[ai].view(np.int16)).to(dev).view(torch.bfloat16)
        vc[ai, :, :n_pos] = torch.from_numpy(vs[ai].view(np.int16)).to(dev).view(torch.bfloat16)
    for li in range(cfg.n_dn):
        S[li] = torch.from_numpy(ss[li]).to(dev)
    m.set_position(n_pos)
    return int(synth.stream(3, "long.first_token").integers(0, cfg.vocab))


EXTRA_WORKLOADS = ("pp520", "pp4096", "long", "long_q8", "27b")


def extra_workloads(args) -> dict:
    """The other measured configurations, each in its own process (so every one starts from a
    clean device), summarised for the headline line: prefill pp520 / pp4096, long-context
    decode with the bf16 and the 8-bit KV cache, the 27B-shaped 4-bit model (plain decode and
    K = 5 verify). Each runs 3 timed steps after 2 warm-up steps."""
    out = {}
    for w in EXTRA_WORKLOADS:
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", w, "--steps", "3", "--warmup", "2",
               "--no-cpu-baseline"]
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
            lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
            if r.returncode != 0 or not lines:
                out[w] = {"error": (r.stderr or r.stdout).strip().splitlines()[-1:] or ["exit %d" % r.returncode]}
                continue
            d = json.loads(lines[-1])
            keep = {k: d[k] for k in ("metric", "value", "unit", "ms_per_step", "e2e", "roofline", "clocks", "plain_decode",
                                      "sampled_verify") if k in d}
            keep["config"] = d.get("config", {}).get("workload")
            out[w] = keep
        except Exception as ex:   # a failure here never hides the headline line
            out[w] = {"error": repr(ex)}
    return out


def run_mk(args):
    import torch
    import hybrid_deltanet_attention_b200 as hda
    import synth

    rank, world, local = dist_setup(args.gpus)
    cfg = synth.QWEN_08B
    dev = torch.device("cuda", local)
    long_ctx = args.workload in ("long", "long_q8")
    kv_q8 = args.workload == "long_q8"
    P0 = LONG_POS if long_ctx else PROMPT
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw, dev), max_ctx=(LONG_POS + TG + 16) if long_ctx else MAX_CTX,
                  kv_format=hda._abi.MK_KV_Q8 if kv_q8 else hda._abi.MK_KV_BF16)
    del raw
    prompt_np = synth.make_prompt(cfg, PROMPT)
    prompt = torch.from_numpy(prompt_np).to(dev)

    # context after the prompt (or the seeded long context), snapshotted once; every step restores it
    first = torch.empty(1, dtype=torch.int32, device=dev)
    if kv_q8:   # the 8-bit rows are written by the library itself: prefill a random long prompt
        m.reset()
        ctx = torch.from_numpy(synth.make_prompt(cfg, LONG_POS, tag="long.ctx")).to(dev)
        m.prefill(ctx, next_token=first)
    elif long_ctx:
        first.fill_(seed_long_context(m, cfg, LONG_POS, dev))
    else:
        m.reset()
        m.prefill(prompt, next_token=first)
    assert m.sync() == 0
    snap = m.state.clone()
    first_tok = first.clone()
    toks = torch.empty(TG + 1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def one_step(ev=None):
        m.state.copy_(snap)
        m.set_position(P0)              # same value as the snapshot; keeps the handle's position in step
        toks[0:1].copy_(first_tok)
        if ev is not None:
            ev[0].record(stream)
        for i in range(TG):
            m.decode(toks[i:i + 1], toks[i + 1:i + 2])
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        one_step()
    assert m.sync() == 0
    launches0 = m.launches
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_device()
    with ClockSampler(cur) as clk, EnergyMeter(cur, cuda_pci_bus_id(torch, cur)) as energy:
        barrier(world)
        torch.cuda.synchronize()
        energy.start()
        t_start.record(stream)
        for k in range(args.steps):
            one_step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize()
        energy.stop()
        barrier(world)
    dev_err = m.sync()
    if dev_err:
        raise RuntimeError(f"device error word 0x{dev_err:x}")
    launches = m.launches - launches0
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    decode_ms = sum(a.elapsed_time(b) for a, b in evs)
    decode_ms = max_over_ranks(decode_ms, world)
    value = replica_throughput(args.steps * TG, world, total_ms / 1000.0)

    # roofline of the decode kernel: algorithmic bytes per launch / average launch duration
    per = [bytes_per_token(cfg, P0 + i, int(m.sizes.kv_row_bytes)) for i in range(TG)]
    read_avg = float(np.mean([b["read"] for b in per]))
    write_avg = float(np.mean([b["write"] for b in per]))
    t_launch = decode_ms / 1000.0 / (args.steps * TG)
    peak, peak_kind = measured_peaks()
    achieved = read_avg / t_launch / 1e9
    khash = kernel_hash()
    traffic = None if long_ctx else recorded_traffic(khash)

    if long_ctx:
        # end to end: the first token from pinned host memory in, 128 decode launches,
        # the generated tokens back to pinned host memory (the seeded context stays resident)
        h_in = torch.tensor([int(first_tok.item())], dtype=torch.int32).pin_memory()
        h_out = torch.empty(TG + 1, dtype=torch.int32).pin_memory()

        def e2e_step():
            m.state.copy_(snap)
            m.set_position(P0)
            toks[0:1].copy_(h_in, non_blocking=True)
            for i in range(TG):
                m.decode(toks[i:i + 1], toks[i + 1:i + 2])
            h_out.copy_(toks, non_blocking=True)
            torch.cuda.current_stream().synchronize()
        e2e_step()
        e2e_steps = max(1, min(args.steps, 5))
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            e2e_step()
        dt = max_over_ranks(time.perf_counter() - t0, world)
        e2e = replica_throughput(e2e_steps * TG, world, dt)
        e2e_io = (4, (TG + 1) * 4, "first token pinned host -> device, 128 decode launches over the seeded "
                                   "32K context, tokens device -> pinned host")
    else:
        # end to end through the public C call with host buffers: prompt in, tokens out
        pinned_in = torch.from_numpy(prompt_np).pin_memory()
        pinned_out = torch.empty(TG, dtype=torch.int32).pin_memory()
        for _ in range(max(1, args.warmup // 2)):
            m.reset()
            m.generate(pinned_in.numpy(), TG, out=pinned_out.numpy())
        e2e_steps = max(1, min(args.steps, 5))
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            m.reset()
            m.generate(pinned_in.numpy(), TG, out=pinned_out.numpy())
        dt = max_over_ranks(time.perf_counter() - t0, world)
        e2e = replica_throughput(e2e_steps * TG, world, dt)
        e2e_io = (PROMPT * 4, TG * 4, "mk_generate: pinned host prompt (128) -> prefill -> 128 greedy tokens -> pinned host")
    if rank != 0:
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not long_ctx:
        v, cores, sample = oracle_sample()
        cpu = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample}
        try:   # the same oracle on one thread (BLAS pools limited to 1), a shorter sample
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                v1, _, sample1 = oracle_sample(seconds_budget=8.0, n_prompt=8, n_decode=16)
            cpu["one_thread"] = {"value": v1, "unit": "tok/s", "cores": 1, "sample": sample1}
        except Exception as ex:   # the multi-threaded figure stands on its own
            cpu["one_thread"] = {"error": repr(ex)}

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": (LONG_Q8_WORKLOAD if kv_q8 else LONG_WORKLOAD) if long_ctx else WORKLOAD,
                   "tokens_per_step": TG,
                   "context_at_start": P0,
                   "l2": "inputs larger than L2: every step streams 1.23 GB of weights (L2 is 126 MB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_kind": peak_kind,
                     "bytes_per_launch_read": read_avg, "bytes_per_launch_write": write_avg,
                     "kernel": "mk_decode_kernel", "avg_launch_us": t_launch * 1e6, "kernel_hash": khash},
        "e2e": {"value": e2e, "unit": "tok/s", "h2d_bytes_per_step": e2e_io[0], "d2h_bytes_per_step": e2e_io[1],
                "what": e2e_io[2]},
        "gpu_launches": launches,
        "clocks": clocks,
        "energy": energy.summary(args.steps * TG),
        "cpu_baseline": cpu,
    }
    if world == 1 and args.workload == "tg128" and not args.no_extra:
        line["workloads"] = extra_workloads(args)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def linear_macs_per_token(cfg) -> int:
    """Multiply-accumulates of the prefill's linear layers per token (the LM head excluded)."""
    H, F = cfg.hidden, cfg.ffn
    tot = 0
    for kind in cfg.pattern:
        tot += 3 * F * H
        if kind == "D":
            tot += cfg.dn_in_rows * H + H * cfg.dn_heads * cfg.dn_dv
        else:
            tot += cfg.at_in_rows * H + H * cfg.at_q_heads * cfg.at_head_dim
    return tot


def prefill_flops(cfg, T: int, pos0: int = 0) -> dict:
    """Algorithmic FLOPs of a prefill of T tokens after pos0 cached positions: the linear
    layers (LM head for the last token only), causal attention (Q K^T and P V over the keys
    each query sees) and the chunked delta rule (chunk C = 64: K K^T, Q K^T, the triangular
    solve for [U | W], Q S0^T, W S0^T, P Delta and the state update K^T (dec Delta))."""
    lin = 2.0 * linear_macs_per_token(cfg) * T + 2.0 * cfg.vocab * cfg.hidden
    keys = T * pos0 + T * (T + 1) / 2.0                  # sum over queries of the keys they see
    attn = cfg.n_at * cfg.at_q_heads * 2.0 * 2.0 * keys * cfg.at_head_dim
    C, dk, dv = 64, cfg.dn_dk, cfg.dn_dv
    wy_macs_tok = C * dk + C * dk / 2.0 + C * (dk + dv) / 2.0 + 3.0 * dk * dv + C * dv / 2.0
    wy = 2.0 * wy_macs_tok * cfg.dn_heads * cfg.n_dn * T
    return {"linear": lin, "attention": attn, "deltanet": wy, "total": lin + attn + wy}


def run_prefill(args):
    """Prefill throughput: one step = reset + mk_prefill of a uniform random prompt."""
    import torch
    import hybrid_deltanet_attention_b200 as hda
    import synth

    rank, world, local = dist_setup(args.gpus)
    cfg = synth.QWEN_08B
    T = int(args.workload[2:])
    dev = torch.device("cuda", local)
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw, dev), max_ctx=T + 16)
    del raw
    prompt_np = synth.make_prompt(cfg, T, tag=f"pp{T}")
    prompt = torch.from_numpy(prompt_np).to(dev)
    nxt = torch.empty(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def one_step():
        m.reset()
        m.prefill(prompt, next_token=nxt)

    for _ in range(args.warmup):
        one_step()
    assert m.sync() == 0
    launches0 = m.launches
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            one_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    assert m.sync() == 0
    ms = max_over_ranks(a.elapsed_time(b), world) / args.steps
    value = replica_throughput(T, world, ms / 1000.0)
    # end to end: pinned host prompt -> prefill -> next token to pinned host
    h_in = torch.from_numpy(prompt_np).pin_memory()
    h_out = torch.empty(1, dtype=torch.int32).pin_memory()

    def e2e_step():
        m.reset()
        prompt.copy_(h_in, non_blocking=True)
        m.prefill(prompt, next_token=nxt)
        h_out.copy_(nxt, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    e2e_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        e2e_step()
    e2e = replica_throughput(args.steps * T, world, max_over_ranks(time.perf_counter() - t0, world))
    if rank != 0:
        return 0
    fl = prefill_flops(cfg, T)
    useful_tflops = fl["total"] / (ms / 1000.0) / 1e12
    peak = None
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            peak = float(json.load(fh).get("bf16_tflops") or 0) or None
    line = {
        "metric": f"prefill tok/s (pp{T}) and tensor-core FLOP/s of the linear layers", "value": value,
        "unit": "tok/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (fp32 activations as bf16 hi+lo)",
        "data": "synthetic",
        "config": {"workload": f"0.8B-shaped hybrid, bf16 weights N(0,0.02) seed 1, {T}-token uniform random prompt, "
                               "batch 1, reset + prefill per step", "prompt": T},
        "roofline": {"bound": "tensor", "achieved": useful_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": (useful_tflops / peak) if peak else None, "traffic": None,
                     "what": "whole-prefill time against the algorithmic FLOPs of the whole prefill (linear layers, "
                             "causal attention, chunked delta rule: %.3g TFLOP); the bf16 hi/lo split issues about twice "
                             "these on the tensor cores" % (fl["total"] / 1e12),
                     "flops": fl, "peak_kind": "measured, burst (the prefill is timed alone)"},
        "e2e": {"value": e2e, "unit": "tok/s", "h2d_bytes_per_step": T * 4, "d2h_bytes_per_step": 4},
        "gpu_launches": (m.launches - launches0) // max(1, args.steps),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_27b(args):
    """27B-shaped 4-bit model: plain greedy decode after a 1024-token context, and
    speculative verify passes of K = 5 drafts (80 % equal to the model's greedy token)."""
    import torch
    import hybrid_deltanet_attention_b200 as hda
    import synth

    rank, world, local = dist_setup(args.gpus)
    small = args.workload == "verify08"
    cfg = synth.QWEN_08B if small else synth.QWEN_27B
    dev = torch.device("cuda", local)
    CTX, K, TGP = 1024, 5, 32
    n_pass = max(4, args.steps)
    weights = hda.weights_to_device(synth.make_weights(cfg), dev) if small else synth.device_q4_weights(cfg, dev, cfg.seed)
    m = hda.Model(cfg, weights, max_ctx=CTX + TGP + (K + 1) * (n_pass + args.warmup + 2) + 16, max_draft=K)
    del weights
    torch.cuda.empty_cache()
    ctx = torch.from_numpy(synth.make_prompt(cfg, CTX, tag="ctx1024")).to(dev)
    first = torch.empty(1, dtype=torch.int32, device=dev)
    m.reset()
    m.prefill(ctx[:-1])
    assert m.sync() == 0
    snap = m.state.clone()
    stream = torch.cuda.current_stream()
    # plain decode (speculation off)
    toks = torch.empty(TGP + 1, dtype=torch.int32, device=dev)
    toks[0:1].copy_(ctx[-1:])
    for i in range(4):
        m.decode(toks[i:i + 1], toks[i + 1:i + 2])
    m.state.copy_(snap)
    m.set_position(CTX - 1)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        a.record(stream)
        for i in range(TGP):
            m.decode(toks[i:i + 1], toks[i + 1:i + 2])
        b.record(stream)
        torch.cuda.synchronize()
    assert m.sync() == 0
    plain_ms = a.elapsed_time(b) / TGP
    # verify passes
    m.state.copy_(snap)
    m.set_position(CTX - 1)
    last = int(ctx[-1].item())
    committed_total, verify_ms = 0, 0.0
    n_acc = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.empty(K + 1, dtype=torch.int32, device=dev)
    g_t = torch.empty(K + 1, dtype=torch.int32, device=dev)
    for ps in range(args.warmup + n_pass):
        # the model's greedy continuation (untimed): decode K steps, then restore
        pos = int(m.pos_tensor.item())
        keep = m.state.clone()
        g_t[0] = last
        for i in range(K):
            m.decode(g_t[i:i + 1], g_t[i + 1:i + 2])
        greedy = g_t[1:].cpu().numpy()
        m.state.copy_(keep)
        m.set_position(pos)
        use, ids = synth.draft_choices(4, ps, K, cfg.vocab)
        drafts = synth.compose_drafts(greedy, use, ids, cfg.vocab)
        tin = torch.from_numpy(np.concatenate([[last], drafts]).astype(np.int32)).to(dev)
        torch.cuda.synchronize()
        a.record(stream)
        m.verify(tin, n_acc, out)
        b.record(stream)
        torch.cuda.synchronize()
        n = int(n_acc.item())
        last = int(out[n].item())
        if ps >= args.warmup:
            committed_total += n + 1
            verify_ms += a.elapsed_time(b)
    assert m.sync() == 0
    # sampling-mode verify passes at temperature 1 (same draft recipe; the uniforms are
    # seeded inputs drawn on the host before the pass)
    m.state.copy_(snap)
    m.set_position(CTX - 1)
    last = int(ctx[-1].item())
    samp_total, samp_ms = 0, 0.0
    urng = np.random.default_rng(4)
    uni = torch.empty(2 * (K + 1), dtype=torch.float32, device=dev)
    for ps in range(args.warmup + n_pass):
        pos = int(m.pos_tensor.item())
        keep = m.state.clone()
        g_t[0] = last
        for i in range(K):
            m.decode(g_t[i:i + 1], g_t[i + 1:i + 2])
        greedy = g_t[1:].cpu().numpy()
        m.state.copy_(keep)
        m.set_position(pos)
        use, ids = synth.draft_choices(4, ps, K, cfg.vocab)
        drafts = synth.compose_drafts(greedy, use, ids, cfg.vocab)
        tin = torch.from_numpy(np.concatenate([[last], drafts]).astype(np.int32)).to(dev)
        uni.copy_(torch.from_numpy(urng.random(2 * (K + 1)).astype(np.float32)))
        torch.cuda.synchronize()
        a.record(stream)
        m.verify_sampled(tin, 1.0, uni, n_acc, out)
        b.record(stream)
        torch.cuda.synchronize()
        n = int(n_acc.item())
        last = int(out[n].item())
        if ps >= args.warmup:
            samp_total += n + 1
            samp_ms += a.elapsed_time(b)
    assert m.sync() == 0
    if rank != 0:
        return 0
    eff = committed_total / (verify_ms / 1000.0)
    bytes_w = cfg.param_count() * (2.0 if small else 0.5625)
    line = {
        "metric": ("0.8B-shaped hybrid (bf16)" if small else "27B-shaped 4-bit hybrid") +
                  ": effective tok/s with K=5 speculative verify (80% greedy drafts), and plain decode tok/s",
        "value": eff, "unit": "tok/s", "n_gpus": world, "steps": n_pass, "warmup": args.warmup,
        "ms_per_step": verify_ms / n_pass, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 weights, fp32 activations" if small else "q4k weights, fp32 activations",
        "data": "synthetic (seeded weights)" if small else "synthetic (device-generated 4-bit blocks)",
        "config": {"workload": (WORKLOAD.split(", bf16 weights")[0] + ", bf16 weights seed 1" if small else
                                "27B-shaped hybrid (64 layers [D,D,D,A]x16, hidden 5120, vocab 151936, DeltaNet 48 heads "
                                "dk=dv=128, attention 24q/4kv D=256, SwiGLU 17408), Q4_K-style weights") +
                               ", 1024-token context, K=5 drafts per pass",
                   "tokens_per_pass": committed_total / n_pass,
                   "pass_ms": verify_ms / n_pass,
                   "tok_s_at_expected_acceptance": 3.689 / (verify_ms / n_pass / 1000.0),
                   "verify_path": "one pass over the weights (batched layers; linear layers and the LM head on "
                                  "mma.sync bf16 tensor-core tiles over the K+1 tokens; commit of the accepted prefix)"
                   if small else "one pass over the 4-bit weights (batched layers; 4-bit codes fed as exact bf16 to "
                                 "mma.sync tensor-core tiles over the K+1 tokens; commit of the accepted prefix)"},
        "sampled_verify": {"temperature": 1.0, "pass_ms": samp_ms / n_pass, "tokens_per_pass": samp_total / n_pass,
                           "acceptance_cost_ms": (samp_ms - verify_ms) / n_pass,
                           "note": "random-init weights give a near-uniform distribution at temperature 1, so "
                                   "drafts are rarely kept; the pass time is the figure"},
        "plain_decode": {"tok_s": 1000.0 / plain_ms, "ms_per_token": plain_ms,
                         "hbm_frac_of_measured": (bytes_w / (plain_ms / 1000.0) / 1e9) / measured_peaks()[0]},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="tg128 only: skip the other measured configurations (prefill, long context, 27B)")
    ap.add_argument("--workload", default="tg128",
                    choices=["tg128", "long", "long_q8", "pp520", "pp4096", "27b", "verify08"])
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload.startswith("pp"):
        return run_prefill(args)
    if args.workload in ("27b", "verify08"):
        return run_27b(args)
    return run_mk(args)


if __name__ == "__main__":
    sys.exit(main())
