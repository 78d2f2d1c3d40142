"""Benchmark of the IndexCache layer stack (indexer + top-k on Full layers,
sparse attention on every layer) on synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle arm
    python bench.py --measure-fp8-peak       # FP8 dense GEMM peak (context)

A step is one pass of the whole stack over one batch of synthetic input. The
default workload is prefill-200k: one 204800-token sequence through 47 layers
at index_topk_freq=4, FP8 E4M3 indexer, 64-head latent-KV attention. Besides
the headline (tok/s at the workload's own F/S assignment), the line carries
the same stack at index_topk_freq 1 and 2 (the IndexCache speedup), and the
decode workload decode-32x32k (32 requests x 32768 context, 47 layers, freq
4) measured the same way.

Under torchrun every rank runs its own independent sequence (weak scaling)
unless --shard rows splits one sequence's query rows across the ranks; the
timed region is bracketed by a barrier and a synchronize and the reported
time is the maximum over ranks. `--gpus N` without torchrun re-launches this
script under torch.distributed.run with N ranks.

Printed on rank 0: one JSON line (metric, value, unit, the roofline of the
dominant kernel and of the whole stack, e2e through host buffers, the oracle
CPU baseline, clocks).
"""

from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import time

_ROOT = os.path.dirname(os.path.abspath(__file__))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from dsa_indexer_reuse_b200 import workloads as W  # noqa: E402

METRIC = "prefill tok/s & decode tok/s over F/S layer stack; % of tensor/HBM roofline"
DEFAULT_WORKLOAD = "prefill-200k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of a kernel on the named workload, with a hash of the kernel's
# sources at capture time: the figure is reported only while the sources are
# unchanged (profiles/ holds the capture summaries).
MEASURED_TRAFFIC = {
    ("sparse_attn_kernel", "prefill-8k"): {
        "bytes": 681.871104e6 + 498.541312e6, "sources": ("attention.cuh", "common.cuh"),
        "sha": "fc901264c2aff13d"},
    ("sparse_attn_kernel", "decode-32x32k"): {
        "bytes": 78.243840e6 + 4.161792e6, "sources": ("attention.cuh", "common.cuh"),
        "sha": "fc901264c2aff13d"},
}


def sources_sha(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(_ROOT, "dsa_indexer_reuse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    m = MEASURED_TRAFFIC.get((kernel, workload))
    if m is None or sources_sha(m["sources"]) != m["sha"]:
        return None
    return m["bytes"]


# --------------------------------------------------------------------------- launch
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_cmd(gpus: int, argv) -> list:
    """The torch.distributed.run command that runs this script with `gpus`
    ranks on this node (rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            "--nproc-per-node", str(gpus), "--master-addr", "127.0.0.1",
            "--master-port", str(_free_port()), os.path.abspath(__file__)] + list(argv)


def check_world(gpus: int):
    """--gpus must agree with the launcher's WORLD_SIZE when there is one."""
    world = os.environ.get("WORLD_SIZE")
    if world is not None and int(world) != gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE=%s; launch one rank per GPU"
                         % (gpus, world))


# --------------------------------------------------------------------------- setup
def dist_setup(backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=180), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def load_peaks():
    """Roofline denominators: measured HBM copy bandwidth and cuBLAS bf16
    (burst for kernels timed alone, sustained beside it); FP8 is the bf16
    burst peak x the nominal FP8/BF16 ratio (no measured FP8 figure)."""
    path = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    src = "measured"
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
    else:
        d, src = dict(FALLBACK_PEAKS), "fallback"
    bf16 = float(d.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    return {"hbm_gbs": float(d.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])), "bf16_tflops": bf16,
            "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", bf16)),
            "fp8_tflops": FP8_PER_BF16 * bf16, "source": src}


def stack_shape(wl):
    return dict(batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k, q_pos0=wl.q_pos0, H_I=wl.H_I, d_I=wl.d_I,
                topk=wl.topk, qk_dtype=wl.qk_dtype, w_dtype=wl.w_dtype, H=wl.H, d_qk=wl.d_qk,
                d_v=wl.d_v, sm_scale=wl.sm_scale)


def slots_for(wl):
    """Number of distinct buffers for the per-token tensors (q, q_I, w, out):
    every layer keeps its own kv and k_I, but the largest workloads rotate
    the per-token tensors through a few slots to fit in HBM."""
    per_layer = wl.batch * wl.n_q * (wl.H * (wl.d_qk + wl.d_v) * 2 + wl.H_I * wl.d_I * 2)
    if per_layer * wl.n_layers < 60e9:
        return wl.n_layers
    return 2 if per_layer * 2 < 80e9 else 1


def make_layers(wl, seed, device, keys_from=None, all_full=False):
    """Device tensors for every layer, seeded per layer. Every layer has its
    own kv (and k_I where it is Full); the per-token tensors (q_I, w, q, out)
    live in slots_for(wl) rotating slots. Shared layers get no indexer
    tensors unless all_full (every layer then carries indexer tensors, so the
    same layers serve any F/S assignment).
    keys_from: reuse another layer list's k_I, k_scale and kv (same keys)."""
    is_full, _ = _resolve(wl)
    full = np.ones_like(is_full) if all_full else is_full
    n_slots = slots_for(wl)
    slots = []
    for s in range(n_slots):
        d = W.indexer_query_inputs(wl, s, seed=seed, device=device)
        d["q"] = W.attention_query(wl, s, seed=seed, device=device)
        d["out"] = torch.empty((wl.batch, wl.n_q, wl.H, wl.d_v), dtype=torch.bfloat16,
                               device=device)
        slots.append(d)
    layers = []
    for l in range(wl.n_layers):
        sl = slots[l % n_slots]
        if keys_from is not None:
            keys = {"k_I": keys_from[l]["k_I"], "k_scale": keys_from[l]["k_scale"]}
            kv = keys_from[l]["kv"]
        else:
            keys = W.indexer_key_inputs(wl, l, seed=seed, device=device) if full[l] else {}
            kv = W.attention_kv(wl, l, seed=seed, device=device)
        layers.append(dict(q_I=sl["q_I"] if full[l] else None,
                           q_scale=sl["q_scale"] if full[l] else None,
                           w=sl["w"] if full[l] else None,
                           k_I=keys.get("k_I"), k_scale=keys.get("k_scale"),
                           q=sl["q"], kv=kv, out=sl["out"]))
    return layers, is_full


def _resolve(wl, freq=None, pattern=None):
    import dsa_indexer_reuse_b200 as ic
    if freq is None:
        freq, pattern = wl.freq, wl.pattern
    return ic.resolve_pattern(wl.n_layers, freq, pattern)


# --------------------------------------------------------------------------- ranks
def max_over_ranks(ms: float, world: int, device) -> float:
    """The job's time is the slowest rank's (all ranks call this)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tok_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank processes its own sequences, so the job's
    throughput is all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


# --------------------------------------------------------------------------- work counts
def selected_keys(wl):
    """Σ over query rows of the keys each selects: min(topk, visible keys)."""
    keys = 0
    for t in range(wl.n_q):
        keys += min(wl.topk, min(wl.q_pos0 + t + 1, wl.n_k))
    return wl.batch * keys


def attn_flops(wl):
    return selected_keys(wl) * wl.H * (wl.d_qk + wl.d_v) * 2


def attn_bytes(wl):
    """(compulsory HBM bytes, gathered bytes) of one attention launch.
    Compulsory: q, idx and out once, and every distinct selected KV row once;
    a sequence's distinct rows are at most min(n_k, its selected keys), and
    for causal prefill every key is selected by some query (all n_k rows),
    for decode each selected row is distinct (topk rows per request).
    Gathered: every selected row at each use (L2 traffic in prefill)."""
    keys = selected_keys(wl)
    rows = wl.batch * wl.n_q
    distinct = wl.batch * min(wl.n_k, keys // max(wl.batch, 1))
    compulsory = (rows * wl.H * wl.d_qk * 2 + distinct * wl.d_qk * 2 + rows * wl.topk * 4
                  + rows * wl.H * wl.d_v * 2)
    return compulsory, keys * wl.d_qk * 2


def indexer_flops(wl):
    pairs = 0
    for t in range(wl.n_q):
        pairs += min(wl.q_pos0 + t + 1, wl.n_k)
    return wl.batch * pairs * wl.H_I * wl.d_I * 2


def distill_flops(wl, n_served):
    """Multiply-adds of the distillation target of one Full layer: the served
    layers' attention logits over the selected keys plus the indexer scores of
    those keys (2 FLOP each)."""
    keys = attn_flops(wl) // (wl.H * (wl.d_qk + wl.d_v) * 2)
    return keys * (n_served * wl.H * wl.d_qk + wl.H_I * wl.d_I) * 2


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def indexer_bytes(wl):
    esz = 1 if wl.qk_dtype == W.FP8_E4M3 else 2
    wsz = 4 if wl.w_dtype == W.F32 else 2
    rows = wl.batch * wl.n_q
    b = rows * wl.H_I * wl.d_I * esz + wl.batch * wl.n_k * wl.d_I * esz + rows * wl.H_I * wsz
    b += rows * wl.topk * 4
    if wl.qk_dtype == W.FP8_E4M3:
        b += rows * 4 + wl.batch * wl.n_k * 4
    return b


def kernel_roofline(flops, nbytes, ms, tensor_tflops, hbm_gbs):
    """Roofline of one launch: t_roof = max(FLOPs / tensor peak, compulsory
    bytes / HBM bandwidth); `bound` is the term that wins, `achieved` is the
    work of that term over the measured time, and frac = t_roof / time."""
    t_c = flops / (tensor_tflops * 1e12)
    t_m = nbytes / (hbm_gbs * 1e9)
    t = ms / 1e3
    if t_c >= t_m:
        return {"bound": "tensor", "achieved": flops / t / 1e12, "peak": tensor_tflops,
                "unit": "TFLOP/s", "frac": t_c / t, "t_roof_ms": t_c * 1e3}
    return {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": hbm_gbs, "unit": "GB/s",
            "frac": t_m / t, "t_roof_ms": t_m * 1e3}


def tensor_peak_of(wl, peaks, kernel):
    if kernel == "indexer" and wl.qk_dtype == W.FP8_E4M3:
        return peaks["fp8_tflops"]
    return peaks["bf16_tflops"]


def stack_roofline(wl, n_full, ms_per_step, peaks):
    """Σ over the step's launches of t_roof, against the measured step."""
    ri = kernel_roofline(indexer_flops(wl), indexer_bytes(wl), 1.0, tensor_peak_of(wl, peaks, "indexer"),
                         peaks["hbm_gbs"])
    ra = kernel_roofline(attn_flops(wl), attn_bytes(wl)[0], 1.0, peaks["bf16_tflops"], peaks["hbm_gbs"])
    t_roof = n_full * ri["t_roof_ms"] + wl.n_layers * ra["t_roof_ms"]
    return {"t_roof_ms": t_roof, "measured_ms": ms_per_step, "frac": t_roof / ms_per_step,
            "tok_s_at_roofline": wl.batch * wl.n_q / (t_roof / 1e3),
            "terms": "%d Full layers x indexer (%s-bound) + %d layers x attention (%s-bound)"
                     % (n_full, ri["bound"], wl.n_layers, ra["bound"])}


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.path = os.path.join("/tmp", "ic_clocks_%d.csv" % os.getpid())

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
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
        self.f.close()
        sm, smax, power, reasons = [], 0.0, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        dev = str(torch.cuda.current_device()) if torch.cuda.is_available() else "0"
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or parts[0] != dev:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = max(smax, float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_median": statistics.median(power) if power else None}


# --------------------------------------------------------------------------- GPU arm
def workload_of(args):
    """The named workload with the command line's overrides applied."""
    wl = W.WORKLOADS[args.workload]
    if getattr(args, "seq_len", 0):
        wl = wl.with_(n_q=args.seq_len, n_k=args.seq_len)
    if getattr(args, "layers", 0):
        wl = wl.with_(n_layers=args.layers, pattern=None if wl.pattern is None else
                      (wl.pattern * args.layers)[:args.layers])
    if getattr(args, "freq", 0):
        wl = wl.with_(freq=args.freq, pattern=None)
    if getattr(args, "pattern", None):
        wl = wl.with_(pattern=args.pattern, n_layers=len(args.pattern))
    return wl


def launches_per_step(wl, n_full):
    import dsa_indexer_reuse_b200 as ic
    idx_split = ic.indexer_workspace_size(wl.batch, wl.n_q, wl.n_k, wl.H_I, wl.d_I, wl.topk,
                                          wl.qk_dtype) > 0
    attn_split = ic.sparse_attn_workspace_size(wl.batch, wl.n_q, wl.H, wl.d_v, wl.topk) > 0
    return n_full * (2 if idx_split else 1) + wl.n_layers * (2 if attn_split else 1)


def timed_steps(run_step, steps, world, dev, stream):
    """Device time of `steps` calls of run_step, bracketed by a barrier and a
    synchronize, max over ranks (every rank calls this)."""
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        run_step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


def kernel_times(wl, layers, is_full, idx_buf, ws, stream, n_steps):
    """Mean device time per launch of each kernel of the stack over n_steps
    instrumented passes (the same kernels through the standalone entry
    points, CUDA events on the launching stream)."""
    import dsa_indexer_reuse_b200 as ic
    t_idx, t_att = [], []
    for _ in range(n_steps):
        for l, L in enumerate(layers):
            if is_full[l]:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                ic.indexer_topk(L["q_I"], L["w"], L["k_I"], wl.topk, q_scale=L["q_scale"],
                                k_scale=L["k_scale"], q_pos0=wl.q_pos0, idx_out=idx_buf,
                                workspace=ws, stream=stream)
                b.record(stream)
                t_idx.append((a, b))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ic.sparse_attn(L["q"], L["kv"], idx_buf, d_v=wl.d_v, sm_scale=wl.sm_scale,
                           out=L["out"], workspace=ws, stream=stream)
            b.record(stream)
            t_att.append((a, b))
    torch.cuda.synchronize()
    idx_ms = statistics.mean(a.elapsed_time(b) for a, b in t_idx) if t_idx else 0.0
    att_ms = statistics.mean(a.elapsed_time(b) for a, b in t_att)
    return idx_ms, att_ms, len(t_idx), len(t_att)


def gpu_arm(args, world, rank, wl_all, with_sweep):
    import dsa_indexer_reuse_b200 as ic
    dev = torch.device("cuda", torch.cuda.current_device())
    shard = args.shard == "rows" and wl_all.n_q > 1
    if shard:
        # one sequence across the ranks: this rank's zig-zag row chunks, each a
        # stack call with q_pos0 at the chunk's first row and the full key range
        from dsa_indexer_reuse_b200.sharding import zigzag_rows
        subs = [wl_all.with_(n_q=b - a, q_pos0=a) for a, b in zigzag_rows(wl_all.n_q, world, rank)]
    else:
        subs = [wl_all]
    calls, layer_sets, is_full = [], [], None
    for sw in subs:
        layers, is_full = make_layers(sw, seed=0 if shard else rank, device=dev,
                                      keys_from=layer_sets[0] if layer_sets else None,
                                      all_full=with_sweep)
        layer_sets.append(layers)
        calls.append(ic.StackCall(layers, stack_shape(sw), freq=sw.freq, pattern=sw.pattern))
    wl, layers, call = subs[0], layer_sets[0], calls[0]
    n_full = int(is_full.sum())
    launches = sum(launches_per_step(sw, n_full) for sw in subs)
    stream = torch.cuda.current_stream()

    use_graph = wl.n_q == 1  # decode steps are launch-bound: replay them as a CUDA graph
    graph = None
    if use_graph:
        call(stream)  # warm the one-time setup before capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call(torch.cuda.current_stream())
        run_step = graph.replay
    else:
        def run_step():
            for c in calls:
                c(stream)

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    assert ic.get_device_status() == 0

    # ---- device-timed region: K steps through ic_layer_stack
    sampler = ClockSampler()
    sampler.start()
    time.sleep(0.3)
    ms = timed_steps(run_step, args.steps, world, dev, stream)
    clocks = sampler.stop()
    ms_per_step = ms / args.steps
    if shard:
        value = wl_all.batch * wl_all.n_q / (ms_per_step / 1e3)  # one sequence across all ranks
    else:
        value = whole_job_tok_per_s(wl.batch * wl.n_q, world, ms_per_step)
    if graph is not None:
        del graph

    # ---- the same layers at index_topk_freq 1 and 2 (every layer carries its
    # indexer tensors); already warm, so each is timed directly
    sweep = None
    if with_sweep:
        sweep = {}
        for f in (1, 2):
            c = ic.StackCall(layers, stack_shape(wl), freq=f, idx_buffer=call.idx_buffer,
                             workspace=call.workspace)
            msf = timed_steps(lambda: c(stream), args.sweep_steps, world, dev, stream) / args.sweep_steps
            nf = int(_resolve(wl, f, None)[0].sum())
            sweep[str(f)] = {"ms_per_step": msf, "tok_s": whole_job_tok_per_s(wl.batch * wl.n_q, world, msf),
                             "full_layers": nf, "steps": args.sweep_steps}
        sweep[str(wl.freq)] = {"ms_per_step": ms_per_step, "tok_s": value, "full_layers": n_full,
                               "steps": args.steps}
        sweep["speedup_freq%d_vs_freq1" % wl.freq] = sweep["1"]["ms_per_step"] / ms_per_step
        sweep["speedup_freq2_vs_freq1"] = sweep["1"]["ms_per_step"] / sweep["2"]["ms_per_step"]

    # ---- per-kernel timing over instrumented passes
    n_inst = max(1, min(args.steps, 10 if ms_per_step < 1000 else 1))
    idx_ms, att_ms, n_il, n_al = kernel_times(wl, layers, is_full, call.idx_buffer, call.workspace,
                                              stream, n_inst)
    assert ic.get_device_status() == 0
    res = dict(wl=wl, value=value, ms_per_step=ms_per_step, clocks=clocks, idx_ms=idx_ms,
               att_ms=att_ms, n_full=n_full, launches=launches * args.steps, graph=use_graph,
               shard=shard, sweep=sweep, kernel_launches_timed={"indexer": n_il, "attention": n_al})

    # ---- end to end: inputs from pinned host memory, result back to host
    # (the device-resident layers are released first; e2e stages its own)
    host = None
    if not args.no_e2e and not shard:
        host = e2e_host_tensors(wl, layers, is_full)
    del calls, layer_sets, layers, call
    torch.cuda.empty_cache()
    if host is not None:
        res["e2e"] = e2e_arm(args, wl, host, world, dev, ms_per_step)
        del host
    torch.cuda.empty_cache()
    assert ic.get_device_status() == 0
    return res


def e2e_host_tensors(wl, layers, is_full):
    """Pinned host copies of every layer's inputs (and a host buffer for the
    last layer's output). The library stages host inputs through two device
    slots (layer l uses slot l % 2) and skips the copy of a host buffer its
    slot already holds, so the host keeps two buffers per field and hands
    the users of a field in one slot alternate buffers: every layer's inputs
    cross PCIe every step, with at most two pinned copies of each field."""
    fields = ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv")
    resident = ("k_I", "k_scale", "kv") if wl.n_q == 1 else ()
    host_of, uses, hl = {}, {}, []
    for l, L in enumerate(layers):
        d = {}
        for k in fields:
            t = L.get(k)
            if t is None or k in resident:
                d[k] = t
                continue
            n = uses.get((k, l % 2), 0)
            uses[(k, l % 2)] = n + 1
            key = (k, n % 2)
            if key not in host_of:
                h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                h.copy_(t)
                host_of[key] = h
            d[k] = host_of[key]
        # intermediate outputs stay on the device (the next layer's input in a
        # model); the step's result is the last layer's output
        d["out"] = None
        hl.append(d)
    hl[-1]["out"] = torch.empty(layers[-1]["out"].shape, dtype=torch.bfloat16, pin_memory=True)
    return hl


def e2e_arm(args, wl, hl, world, dev, step_ms):
    """Same metric through ic_layer_stack_host, the entry point for tensors in
    host memory. Every step copies each layer's inputs in from pinned host
    memory and reads the step's result back: the last layer's output and the
    index buffer (intermediate outputs stay on the device, where the next
    layer of a model would consume them). The library overlaps layer l+1's
    input copies with layer l's kernels. For prefill every tensor is a
    per-step input; for a decode step the inputs are the new tokens' tensors
    (q_I, q_scale, w, q) and the KV cache and indexer keys stay resident on
    the device, as in serving (the step is then replayed as one CUDA graph,
    like the device-resident arm). Bytes per step are counted from the
    copies the call makes."""
    import dsa_indexer_reuse_b200 as ic
    decode = wl.n_q == 1
    # intermediate outputs: device buffers of the library's staging (a device
    # tensor per layer parity keeps the call's view of them)
    outs = [torch.empty((wl.batch, wl.n_q, wl.H, wl.d_v), dtype=torch.bfloat16, device=dev)
            for _ in range(2)]
    for l, d in enumerate(hl):
        if d["out"] is None:
            d["out"] = outs[l % 2]
    idx_host = torch.empty((wl.batch, wl.n_q, wl.topk), dtype=torch.int32, pin_memory=True)
    hcall = ic.StackHostCall(hl, stack_shape(wl), freq=wl.freq, pattern=wl.pattern, idx_out=idx_host,
                             device=dev)
    stream = torch.cuda.current_stream()
    # long steps (seconds of PCIe each) are timed over --e2e-steps; short
    # ones over the run's --steps
    steps = max(1, args.e2e_steps if step_ms > 1000 else args.steps)
    hcall(stream)  # warm: the library's copy streams are created here
    torch.cuda.synchronize()
    h2d, d2h = hcall.h2d_bytes, hcall.d2h_bytes  # what every call copies (the library's count)
    graph = None
    if decode:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            hcall(torch.cuda.current_stream())
        one = graph.replay
        for _ in range(max(1, args.warmup)):
            one()
    else:
        def one():
            hcall(stream)
    torch.cuda.synchronize()
    ms = timed_steps(one, steps, world, dev, stream)
    if graph is not None:
        del graph
    return {"value": whole_job_tok_per_s(wl.batch * wl.n_q, world, ms / steps), "unit": "tok/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps,
            "resident": "kv cache and indexer keys" if decode else "nothing",
            "api": "ic_layer_stack_host" + (" (CUDA graph)" if decode else "")}


def roofline_block(wl, r, peaks):
    """The dominant kernel's roofline (top level) plus both kernels' and the
    whole stack's."""
    ri = kernel_roofline(indexer_flops(wl), indexer_bytes(wl), r["idx_ms"], tensor_peak_of(wl, peaks, "indexer"),
                         peaks["hbm_gbs"]) if r["idx_ms"] > 0 else None
    ra = kernel_roofline(attn_flops(wl), attn_bytes(wl)[0], r["att_ms"], peaks["bf16_tflops"], peaks["hbm_gbs"])
    att_total = r["att_ms"] * wl.n_layers
    idx_total = r["idx_ms"] * r["n_full"]
    if ri is not None:
        ri.update(kernel="indexer_topk_kernel", ms=r["idx_ms"], flop_per_launch=indexer_flops(wl),
                  bytes_per_launch=indexer_bytes(wl), traffic=measured_traffic("indexer_topk_kernel", wl.name),
                  peak_source="%s bf16 burst x %.0f (nominal FP8/BF16)" % (peaks["source"], FP8_PER_BF16)
                  if wl.qk_dtype == W.FP8_E4M3 else "%s bf16 burst (cuBLAS)" % peaks["source"])
    comp, gath = attn_bytes(wl)
    ra.update(kernel="sparse_attn_kernel", ms=r["att_ms"], flop_per_launch=attn_flops(wl),
              bytes_per_launch=comp, gather_bytes_per_launch=gath,
              gather_gbs=gath / (r["att_ms"] / 1e3) / 1e9,
              traffic=measured_traffic("sparse_attn_kernel", wl.name),
              peak_source="%s bf16 burst (cuBLAS)" % peaks["source"] if ra["bound"] == "tensor"
              else "%s HBM copy" % peaks["source"])
    top = dict(ra if (ri is None or att_total >= idx_total) else ri)
    top["kernels"] = {"indexer_topk_kernel": ri, "sparse_attn_kernel": ra}
    top["stack"] = stack_roofline(wl, r["n_full"], r["ms_per_step"], peaks)
    top["peaks"] = {"bf16_tflops_burst": peaks["bf16_tflops"],
                    "bf16_tflops_sustained": peaks["bf16_tflops_sustained"],
                    "fp8_tflops": peaks["fp8_tflops"], "hbm_gbs": peaks["hbm_gbs"],
                    "source": peaks["source"]}
    return top


# --------------------------------------------------------------------------- oracle
def oracle_sample(wl, rows_target=64, seed=0):
    """Time the CPU oracle on a bounded sample of query rows of one Full and
    one Shared layer and extrapolate to the whole stack.

    The rows are evenly spaced over the sequence (so their mean cost is the
    mean row cost of the causal triangle); each row's indexer + top-k runs as
    its own oracle call (one query at its absolute position over all visible
    keys) in a pool of one thread per host core, then the sampled rows'
    attention runs over the oracle's own index rows. The oracle's work
    depends only on the shapes, so the sample draws its own seeded values
    for just those rows (query tensors) and one sequence's keys and KV.
    Returns (tok/s, cores, description, wall seconds)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    cores = oracle.hardware_threads()
    n_rows = wl.batch * wl.n_q
    rows = np.unique(np.linspace(0, n_rows - 1, min(rows_target, n_rows)).astype(np.int64))
    R = len(rows)
    one = wl.with_(batch=1, n_q=R)
    qi = {k: W.raw_numpy(v) for k, v in W.indexer_query_inputs(one, 0, seed=seed).items()}
    ki = {k: W.raw_numpy(v) for k, v in W.indexer_key_inputs(wl.with_(batch=1), 0, seed=seed).items()}
    q = W.raw_numpy(W.attention_query(one, 0, seed=seed))
    kv = W.raw_numpy(W.attention_kv(wl.with_(batch=1), 0, seed=seed))

    def pos_of(r):  # absolute position of sampled row r
        return wl.q_pos0 + int(r % wl.n_q)

    def one_row(i):
        sl = slice(i, i + 1)
        idx, _ = oracle.indexer_topk(
            qi["q_I"][:, sl], None if qi["q_scale"] is None else qi["q_scale"][:, sl], qi["w"][:, sl],
            ki["k_I"], ki["k_scale"], qk_dtype=wl.qk_dtype, w_dtype=wl.w_dtype, batch=1, n_q=1,
            n_k=wl.n_k, q_pos0=pos_of(rows[i]), H_I=wl.H_I, d_I=wl.d_I, topk=wl.topk, threads=1)
        return idx[0]

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=cores) as ex:
        idx = np.stack(list(ex.map(one_row, range(R))))
    t1 = time.perf_counter()
    oracle.sparse_attn(q, kv, idx, batch=1, n_q=R, n_k=wl.n_k, H=wl.H, d_qk=wl.d_qk, d_v=wl.d_v,
                       topk=wl.topk, sm_scale=wl.sm_scale, threads=cores)
    t2 = time.perf_counter()
    n_full = int(_resolve_oracle(wl)[0].sum())
    scale = n_rows / R
    stack_s = (t1 - t0) * scale * n_full + (t2 - t1) * scale * wl.n_layers
    desc = ("%d evenly spaced query rows of one Full and one Shared layer (indexer+top-k "
            "%.1f s, attention %.1f s on %d threads), extrapolated to %d layers (%d Full) x %d rows"
            % (R, t1 - t0, t2 - t1, cores, wl.n_layers, n_full, n_rows))
    return n_rows / stack_s, cores, desc, t2 - t0


def _resolve_oracle(wl):
    import oracle
    return oracle.resolve_pattern(wl.n_layers, wl.freq, wl.pattern)


# --------------------------------------------------------------------------- fp8 peak
def measure_fp8_peak():
    """Dense E4M3 GEMM throughput of torch._scaled_mm at 8192^3 (burst: best of
    10; sustained: back to back for 4 s), context for the FP8 denominator."""
    n = 8192
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
    one = torch.tensor(1.0, device="cuda")

    def mm():
        return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    best = 1e9
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    flops = 2.0 * n ** 3
    sampler = ClockSampler()
    sampler.start()
    t_end = time.time() + 4.0
    cnt = 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    while time.time() < t_end:
        for _ in range(20):
            mm()
        cnt += 20
        torch.cuda.synchronize()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    sus = flops * cnt / (e0.elapsed_time(e1) / 1e3) / 1e12
    print(json.dumps({"fp8_e4m3_tflops": flops / (best / 1e3) / 1e12, "fp8_e4m3_tflops_sustained": sus,
                      "shape": [n, n, n], "how": "torch._scaled_mm e4m3 x e4m3 -> bf16, best of 10 "
                      "(burst) and back to back for 4 s (sustained)", "clocks": clocks}))


# --------------------------------------------------------------------------- single kernel
def single_kernel(args):
    """Launch one kernel of layer 0 `warmup + steps` times (profiling aid):
    prints the mean device time per launch of the last `steps` launches."""
    import dsa_indexer_reuse_b200 as ic
    wl = workload_of(args)
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    ind = W.indexer_inputs(wl, 0, device=dev)
    idx = ic.indexer_topk(ind["q_I"], ind["w"], ind["k_I"], wl.topk, q_scale=ind["q_scale"],
                          k_scale=ind["k_scale"], q_pos0=wl.q_pos0)
    if args.single == "distill":
        # the first Full layer and the layers it serves (itself first)
        is_full, src = ic.resolve_pattern(wl.n_layers, wl.freq, wl.pattern)
        served = []
        for l in range(wl.n_layers):
            if src[l] == 0:
                att = W.attention_inputs(wl, l, device=dev)
                served.append((att["q"], att["kv"]))
        n_served = len(served)

        def launch():
            ic.distill_target(served, ind["q_I"], ind["w"], ind["k_I"], idx, q_scale=ind["q_scale"],
                              k_scale=ind["k_scale"], sm_scale=wl.sm_scale, with_target=False)
    elif args.single == "attn":
        q = W.attention_query(wl, 0, device=dev)
        kv = W.attention_kv(wl, 0, device=dev)
        out = torch.empty((wl.batch, wl.n_q, wl.H, wl.d_v), dtype=torch.bfloat16, device=dev)

        def launch():
            ic.sparse_attn(q, kv, idx, d_v=wl.d_v, sm_scale=wl.sm_scale, out=out)
    else:
        def launch():
            ic.indexer_topk(ind["q_I"], ind["w"], ind["k_I"], wl.topk, q_scale=ind["q_scale"],
                            k_scale=ind["k_scale"], q_pos0=wl.q_pos0, idx_out=idx)
    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        launch()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    peaks = load_peaks()
    if args.single == "distill":
        f = distill_flops(wl, n_served)
        roof = kernel_roofline(f, 0, ms, peaks["bf16_tflops"], peaks["hbm_gbs"])
        print(json.dumps({"kernel": "distill", "workload": wl.name, "n_q": wl.n_q, "served": n_served,
                          "ms": ms, "tflops": f / (ms / 1e3) / 1e12, "roofline": roof,
                          "status": ic.get_device_status()}))
        return
    if args.single == "attn":
        roof = kernel_roofline(attn_flops(wl), attn_bytes(wl)[0], ms, peaks["bf16_tflops"], peaks["hbm_gbs"])
        f = attn_flops(wl)
    else:
        roof = kernel_roofline(indexer_flops(wl), indexer_bytes(wl), ms, tensor_peak_of(wl, peaks, "indexer"),
                               peaks["hbm_gbs"])
        f = indexer_flops(wl)
    print(json.dumps({"kernel": args.single, "workload": wl.name, "n_q": wl.n_q, "n_k": wl.n_k, "ms": ms,
                      "tflops": f / (ms / 1e3) / 1e12, "roofline": roof, "status": ic.get_device_status()}))


# --------------------------------------------------------------------------- main
def config_of(wl, parallelism, l2=True):
    c = {"workload": wl.name, "batch": wl.batch, "seq_len": wl.n_q, "kv_len": wl.n_k,
         "layers": wl.n_layers, "index_topk_freq": wl.freq, "index_topk_pattern": wl.pattern,
         "topk": wl.topk, "indexer": "H_I=%d d_I=%d %s" % (wl.H_I, wl.d_I,
                                                          "e4m3" if wl.qk_dtype else "bf16"),
         "attention": "H=%d d_qk=%d d_v=%d bf16" % (wl.H, wl.d_qk, wl.d_v),
         "parallelism": parallelism}
    if l2:
        c["l2"] = "inputs larger than L2 (each step streams every layer's tensors)"
    return c


def dtype_of(wl):
    return "fp8-e4m3 indexer, bf16 attention" if wl.qk_dtype == W.FP8_E4M3 else "bf16"


def reference_arm(args, wl):
    """The CPU oracle arm: each step is one bounded sample of the workload
    (oracle_sample), timed on the host's cores; `value` extrapolates the
    sample to the workload's tokens per second."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    cores = oracle.hardware_threads()
    vals, walls = [], []
    desc = ""
    for s in range(args.steps):
        v, cores, desc, secs = oracle_sample(wl, rows_target=args.oracle_rows or 2 * cores, seed=s)
        vals.append(v)
        walls.append(secs)
    value = statistics.mean(vals)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(walls),
        "ms_per_workload_step_extrapolated": 1e3 * wl.batch * wl.n_q / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, "dp%d" % args.gpus),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def cpu_dry_run(args):
    """Launcher self-test without a GPU: every rank joins a gloo group, times
    a trivial host step, and rank 0 prints the job line's rank fields."""
    world, rank, _ = dist_setup("gloo")
    t0 = time.perf_counter()
    time.sleep(0.01 * (rank + 1))
    ms = max_over_ranks((time.perf_counter() - t0) * 1e3, world, torch.device("cpu"))
    if rank == 0:
        print(json.dumps({"metric": METRIC, "n_gpus": world, "dry_run": True, "ms_per_step": ms,
                          "value": whole_job_tok_per_s(1, world, ms), "unit": "tok/s"}))
    if world > 1:
        torch.distributed.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode-32x32k sub-measurement of the default run")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the index_topk_freq 1 / 2 sweep of freq workloads")
    ap.add_argument("--sweep-steps", type=int, default=1)
    ap.add_argument("--oracle-rows", type=int, default=0, help="rows per oracle sample (0: 2 per core)")
    ap.add_argument("--measure-fp8-peak", action="store_true")
    ap.add_argument("--cpu-dry-run", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--single", choices=["indexer", "attn", "distill"], default=None,
                    help="run only one kernel of layer 0 (for profiling)")
    ap.add_argument("--seq-len", type=int, default=0, help="override n_q = n_k (prefill)")
    ap.add_argument("--freq", type=int, default=0, help="override index_topk_freq")
    ap.add_argument("--pattern", default=None, help="override index_topk_pattern (F/S string)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count")
    ap.add_argument("--shard", default="none", choices=["none", "rows"],
                    help="rows: split one prefill sequence's query rows across the ranks (zig-zag, "
                         "strong scaling); default: one independent sequence per rank (weak)")
    argv = sys.argv[1:] if argv is None else argv
    args = ap.parse_args(argv)
    if args.gpus < 1:
        raise SystemExit("bench.py: --gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "ours":
        # one process per GPU: re-launch under torch.distributed.run
        sys.stdout.flush()
        os.execv(sys.executable, relaunch_cmd(args.gpus, argv))
    check_world(args.gpus)
    if args.cpu_dry_run:
        cpu_dry_run(args)
        return
    if args.measure_fp8_peak:
        measure_fp8_peak()
        return
    if args.single:
        single_kernel(args)
        return
    wl = workload_of(args)
    if args.impl == "reference":
        reference_arm(args, wl)
        return

    world, rank, local = dist_setup()
    peaks = load_peaks()
    with_sweep = (not args.no_sweep and wl.freq > 1 and args.shard == "none"
                  and wl.name == DEFAULT_WORKLOAD and not args.freq)
    r = gpu_arm(args, world, rank, wl, with_sweep)
    wk = r["wl"]  # the workload the per-kernel timings ran on (this rank's first chunk when sharded)
    roof = roofline_block(wk, r, peaks)
    line = {
        "metric": METRIC, "value": r["value"], "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
        "higher_is_better": True, "scaling": "strong" if r["shard"] else "weak", "vs_baseline": None,
        "dtype": dtype_of(wl), "data": "synthetic",
        "config": config_of(wl, ("zigzag-rows%d" if r["shard"] else "dp%d") % world),
        "roofline": roof, "gpu_launches": r["launches"], "clocks": r["clocks"],
        "e2e": r.get("e2e"), "cuda_graph": r["graph"],
        "per_kernel_launches_timed": r["kernel_launches_timed"],
    }
    if r["sweep"] is not None:
        line["index_topk_freq_sweep"] = r["sweep"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, _ = oracle_sample(wl, rows_target=args.oracle_rows or 4 * 16)
        line["cpu_baseline"] = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle",
                                "sample": desc}
    # the decode workload, measured the same way (graph replay of the 47-layer step)
    if not args.no_decode and wl.name == DEFAULT_WORKLOAD and args.shard == "none" and not args.freq \
            and not args.seq_len and not args.layers and not args.pattern:
        dwl = W.DECODE_32X32K
        dargs = argparse.Namespace(**vars(args))
        rd = gpu_arm(dargs, world, rank, dwl, False)
        droof = roofline_block(dwl, rd, peaks)
        dec = {"workload": dwl.name, "value": rd["value"], "unit": "tok/s", "ms_per_step": rd["ms_per_step"],
               "tok_s_per_request": rd["value"] / (dwl.batch * world), "steps": args.steps,
               "warmup": args.warmup, "config": config_of(dwl, "dp%d" % world, l2=False),
               "dtype": dtype_of(dwl), "roofline": droof, "clocks": rd["clocks"], "e2e": rd.get("e2e"),
               "gpu_launches": rd["launches"], "cuda_graph": rd["graph"]}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, cores, desc, _ = oracle_sample(dwl, rows_target=args.oracle_rows or 16)
            dec["cpu_baseline"] = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle",
                                   "sample": desc}
        line["decode"] = dec
        line["gpu_launches"] += rd["launches"]
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
