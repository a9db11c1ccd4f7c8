"""Benchmark of the LoopKV decode step on B200.

Workload: the batched long-context decode of a 1.4B-shaped looped model
(4 loops x 24 layers, 16 KV heads, head dim 128, batch 32, 16384 cached
tokens per sequence; loop 3 all 4-bit, loops 0-2 35% 4-bit / 35% 2-bit /
30% SHARE; tau 0.002; keys with 4 outlier channels at 10x, peaked queries;
synthetic, seeded).  One step appends one new token to every cell and
decodes every cell, in serving order (loops 0-2, then loop 3), for all 32
sequences and 16 heads: 96 cell-steps.

Prints one JSON line.  ``value`` is cell-steps/s over all ranks, timed on
the device with CUDA events (max over ranks) with the KV cache resident in
HBM (105 GB, far larger than L2).  ``e2e`` repeats the step through the
public API with each step's inputs copied from pinned host memory and the
outputs read back inside the timed region.  ``roofline`` reports the decode
kernel's algorithmic bytes over its measured time against the measured HBM
copy bandwidth.  ``--impl reference`` times the CPU oracle instead.
"""

import argparse
import gc
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn loop×layer cell-steps/s; achieved HBM GB/s vs ~8 TB/s roofline"
UNIT = "cell-steps/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="loopkv", choices=["loopkv", "reference"])
    ap.add_argument("--config", default="2")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work budget of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--q-per-kv", type=int, default=1, choices=[1, 2, 4],
                    help="query heads per KV head (grouped-query decode); 1 = one query "
                         "per KV head, the workloads' own shape")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per GPU (default: the workload's batch); smaller "
                         "batches are for profiling captures only")
    ap.add_argument("--seq-chunks", type=int, default=1,
                    help="decode the batch as this many sequence sub-batches, one after the "
                         "other, each with its own cache (for a batch whose KV cache exceeds "
                         "the GPU); a step's time is the sum over sub-batches")
    ap.add_argument("--cell-chunks", type=int, default=1,
                    help="decode the cells as this many loop-aligned chunks, each with its own "
                         "cache (plans without SHARE / RES2 cells); a step's time is the sum")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps one call at a time; by default they are "
                         "captured (appends and decodes, in serving order) as one CUDA graph "
                         "after the warm-up and the replay is timed, as a serving engine runs "
                         "its decode step")
    ap.add_argument("--decode-split", type=int, default=0,
                    help="CTAs per decoded unit at least (0: the library chooses); for "
                         "launch-shape sweeps")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        return float(mp["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def per_token_head_bytes(kind, D):
    """Bytes one quantized token of one head occupies in the planes + meta."""
    if kind == 0:
        return 5 * D // 4      # K_hi, K_lo, K_meta, V_hi, V_meta (V_lo counted per selection)
    if kind == 1:
        return 4 * D // 4      # K_hi, K_meta, V_hi, V_meta
    return 4 * D               # bf16 key + value


def decode_bytes(wl, cells, lens_own, lens_src, nsel_total, g=1):
    """Algorithmic HBM bytes of one decode launch over `cells`.

    Per unit (KV head): each attended position at its storage's per-token
    bytes (bf16 residual and the SHARE current token at 4D bytes), read once
    for the g query heads of the group, the low-plane rows of the selected
    positions (D/4 each), the queries (2D each) and the outputs (4D each).
    A RES2 unit reads its residual-coded positions twice over: the
    reference's bytes plus its own 2-bit residual rows (D per token), and
    its bf16 window at 4D per token.
    """
    D, H = wl.head_dim, wl.n_heads
    total = 0
    for c in cells:
        share = wl.kinds[c] == 2
        if wl.kinds[c] == 4:
            rk = int(wl.kinds[wl.source_cell(c)])
            for n in lens_own:
                n = int(n)
                rt = (n // 32 - 1) * 32 if n >= 64 else 0
                ref = rt * (4 * D if rk == 3 else per_token_head_bytes(rk, D))
                tok = ref + rt * per_token_head_bytes(1, D) + (n - rt) * 4 * D
                total += H * (tok + g * (2 * D + 4 * D))
            continue
        dk = int(wl.kinds[wl.data_cell(c)])
        for b, n in enumerate(lens_own):
            n = int(n)
            n_att = n - 1 if share else n
            n_src = int(lens_src[b]) if share else n
            if dk == 3:
                q, r = 0, n_att
            else:
                qtok = n_src // 32 * 32
                q = min(n_att, qtok)
                r = n_att - q
            tok = q * per_token_head_bytes(dk, D) + r * 4 * D + (4 * D if share else 0)
            total += H * (tok + g * (2 * D + 4 * D))
    return int(total) + int(nsel_total) * (D // 4)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        note = None
        if not sm:
            # the timed region was shorter than the sampling interval: one
            # reading right after it
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index),
                                      "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits"],
                                     capture_output=True, text=True, timeout=10).stdout
                parts = [p.strip() for p in out.strip().split(",")]
                sm, smax = [float(parts[0])], [float(parts[1])]
                reasons = {n for n, v in zip(names, parts[4:8]) if v.lower().startswith("active")}
                note = "timed region shorter than the 200 ms sampling interval: read right after it"
            except Exception:
                return None
        rec = {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
               "reasons": sorted(reasons), "samples": len(sm) if note is None else 0}
        if note:
            rec["note"] = note
        return rec


def workload_text(wl, B, g=1):
    """One-line description of the benched workload."""
    k = wl.kinds
    plan = "plan %d Q4 / %d Q2 / %d SHARE / %d BF16 cells" % (
        (k == 0).sum(), (k == 1).sum(), (k == 2).sum(), (k == 3).sum())
    if (k == 4).any():
        plan += " / %d RES2 (2-bit residuals against the final loop)" % (k == 4).sum()
    ctx = ("%d cached tokens" % int(wl.lengths[0]) if len(set(wl.lengths[:B].tolist())) == 1
           else "ragged %d-%d cached tokens" % (int(wl.lengths[:B].min()), int(wl.lengths[:B].max())))
    heads = "%d KV heads" % wl.n_heads
    if g > 1:
        heads += " x %d query heads each (grouped-query)" % g
    return ("%s: %d loops x %d layers, %s, head dim %d, batch %d per GPU, %s + 1 "
            "appended per step, %s, tau %g" % (wl.name, wl.n_loops, wl.n_layers, heads,
                                              wl.head_dim, B, ctx, plan, wl.tau))


def shard_sequences(rank, batch):
    """Global sequence ids a rank serves: weak scaling, `batch` sequences per
    rank, disjoint across ranks (so every rank decodes different data)."""
    return list(range(rank * batch, (rank + 1) * batch))


def max_over_ranks(values, world, device):
    """Element-wise max of a list of floats over all ranks (timing)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(record="decode_traffic.json",
                rec_paths=("loop_aware_quantized_b200/csrc/decode.cu",
                           "loop_aware_quantized_b200/csrc/loopkv_internal.cuh")):
    """DRAM bytes / algorithmic bytes of a kernel from its committed ncu
    capture (profiles/<record>), when it was taken on the current kernel
    source; else None.  Traffic grows with the units a launch processes, so
    a full launch moves this ratio times its algorithmic bytes."""
    path = os.path.join(ROOT, "profiles", record)
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_hash") != source_hash([os.path.join(ROOT, p) for p in rec_paths]):
        return None
    return rec.get("traffic_over_algorithmic")


# --------------------------------------------------------- oracle baseline

class OracleSample:
    """A fixed sample of a workload's units in the CPU oracle, built once;
    rate(seconds) times the oracle's decodes of them on the calling core.

    LoopKV workloads: one unit per cell kind the plan has (Q4, Q2, SHARE,
    BF16, RES2), each with its g query heads, at the workload's context (+1
    token, as in a decode step).
    LoopVQ workloads (vq=True): two units, decoding loop 1."""

    def __init__(self, config, seqs_global, g=1, vq=False):
        from oracle import oracle as orc
        from synth import workloads as W
        self.orc, self.vq, self.g = orc, vq, g
        self.units = []
        if vq:
            wl = self.wl = W.make_vq(config)
            n = self.n = int(wl.lengths[0])
            for layer, b, h in ((3, 5, 7), (17, 30, 2)):
                self.units.append((W.vq_indices(wl, 0, layer, b, h, 0, n),
                                   W.vq_indices(wl, 1, layer, b, h, 0, n),
                                   W.vq_codebook(wl, 0, layer, h), W.vq_codebook(wl, 1, layer, h),
                                   W.vq_query(wl, 1, layer, b, h)))
            return
        wl = self.wl = W.make(config)
        n = int(wl.lengths[0])
        self.n = n + 1
        rng = np.random.default_rng(0)
        picks = []
        for kind in (0, 1, 2, 3, 4):
            cs = [c for c in range(wl.n_cells) if wl.kinds[c] == kind]
            if cs:
                picks.append((int(rng.choice(cs)), int(rng.integers(len(seqs_global))),
                              int(rng.integers(wl.n_heads))))
        self.cells = [c for c, _, _ in picks]
        for c, b, h in picks:
            b = int(seqs_global[b])
            kind = int(wl.kinds[c])
            cap = int(wl.capacity[0])
            own = orc.OracleUnit(kind, wl.head_dim, cap)
            src = None
            if kind == 2:
                k = np.zeros((n + 1, wl.head_dim), np.uint16)
                v = np.zeros_like(k)
                k[-1] = W.raw_keys(wl, c, b, h, n, n + 1)[0]
                v[-1] = W.raw_values(wl, c, b, h, n, n + 1)[0]
                own.append(k, v)
                sc = wl.source_cell(c)
                src = orc.OracleUnit(int(wl.kinds[sc]), wl.head_dim, cap)
                src.append(W.raw_keys(wl, sc, b, h, 0, n), W.raw_values(wl, sc, b, h, 0, n))
            else:
                own.append(W.raw_keys(wl, c, b, h, 0, n + 1), W.raw_values(wl, c, b, h, 0, n + 1))
                if kind == 4:  # the reference, one token behind in serving order
                    sc = wl.source_cell(c)
                    src = orc.OracleUnit(int(wl.kinds[sc]), wl.head_dim, cap)
                    src.append(W.raw_keys(wl, sc, b, h, 0, n), W.raw_values(wl, sc, b, h, 0, n))
            self.units.append((own, src, W.query_group(wl, c, b, h, n + 1, g)))

    def rate(self, seconds):
        """(cell-steps/s, sample description), extrapolated from the sample: a
        cell-step decodes B x H units of one cell, so a step of the workload
        takes sum over its cells of B * H * (mean time of the sampled unit of
        that cell's kind), and the rate is cells / that time."""
        wl, orc = self.wl, self.orc
        done = 0
        spent = [0.0] * len(self.units)
        calls = [0] * len(self.units)
        t0 = time.perf_counter()
        while True:
            for i, u in enumerate(self.units):
                t1 = time.perf_counter()
                if self.vq:
                    orc.vq_decode(*u, 1, wl.n_loops)
                else:
                    orc.decode_group(u[0], u[2], wl.tau, src=u[1])
                spent[i] += time.perf_counter() - t1
                calls[i] += 1
                done += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
        per_unit = [t / c for t, c in zip(spent, calls)]
        if self.vq:
            unit_s = float(np.mean(per_unit))
            step_s = wl.n_cells * wl.batch * wl.n_heads * unit_s
            desc = ("%d oracle LoopVQ decodes of %d sampled units (%d coded tokens each) in %.1f s "
                    "on 1 core" % (done, len(self.units), self.n, el))
        else:
            by_kind = {int(self.wl.kinds[c]): t for c, t in zip(self.cells, per_unit)}
            step_s = sum(by_kind[int(k)] for k in wl.kinds) * wl.batch * wl.n_heads
            desc = ("%d oracle decodes of %d sampled units (one per kind of the plan; %d tokens "
                    "each%s) in %.1f s on 1 core" % (
                        done, len(self.units), self.n,
                        ", %d query heads per unit" % self.g if self.g > 1 else "", el))
        desc += ("; extrapolated: one step = %d cells x %d seqs x %d heads of units, each at its "
                 "kind's sampled time" % (wl.n_cells, wl.batch, wl.n_heads))
        return wl.n_cells / step_s, desc


# --------------------------------------------------------------- LoopVQ leg

VQ_CONFIGS = ("vq16k",)


def vq_unit_bytes(n, D):
    """Algorithmic bytes of one LoopVQ unit decode: n tokens' key and value
    indices (D/4 bytes each), the two codebooks' loop slices (256 entries x
    4 fp32 each), the query (2D) and the output (4D)."""
    return n * (D // 2) + 2 * 256 * 4 * 4 + 2 * D + 4 * D


def oracle_baseline(config, seconds, seqs_global, g=1):
    """The oracle on one core: (cell-steps/s, sample description, cores)."""
    return OracleSample(config, seqs_global, g).rate(seconds) + (1,)


def oracle_baseline_vq(config, seconds):
    """The oracle's LoopVQ decode on one core: (cell-steps/s, sample, cores)."""
    return OracleSample(config, [], vq=True).rate(seconds) + (1,)


def bench_vq(args, rank, world):
    """The LoopVQ workload: per step, the new token of every (layer,
    sequence, KV head) is encoded (keys, values: one launch each, all loops
    at once) and every (loop, layer) cell is decoded (one launch per loop,
    all layers, sequences and KV heads)."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from loop_aware_quantized_b200 import vq_decode, vq_encode
    from synth import workloads as W
    from synth.gpu import VqDeviceGenerator

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = W.make_vq(args.config)
    if args.batch:
        wl.batch = args.batch
        wl.lengths = wl.lengths[:args.batch]
    B, H, D, L = wl.batch, wl.n_heads, wl.head_dim, wl.n_loops
    n0 = wl.lengths[:B].astype(np.int32)
    n_steps = args.warmup + args.steps
    total_steps = n_steps + (0 if args.no_e2e else args.steps)
    wl.capacity = int(n0.max()) + total_steps   # room for one new token per step
    gen = VqDeviceGenerator(wl, dev, seq0=rank * B)   # weak scaling: disjoint sequences
    t_build = time.perf_counter()
    ik, iv = gen.indices(0, T=int(n0.max())), gen.indices(1, T=int(n0.max()))
    cbk, cbv = gen.codebooks(0), gen.codebooks(1)
    torch.cuda.synchronize()
    build_s = time.perf_counter() - t_build

    def inputs(s):
        """Step s: queries per loop ("loop" stream l + 16 s) and the new
        token's keys and values in every loop (streams 1000 + ..., 2000 + ...)."""
        q = [gen.queries(l + 16 * s) for l in range(L)]
        xk = torch.stack([gen.queries(1000 + l + 16 * s) for l in range(L)]).unsqueeze(4)
        xv = torch.stack([gen.queries(2000 + l + 16 * s) for l in range(L)]).unsqueeze(4)
        return q, xk.contiguous(), xv.contiguous()

    ins = [inputs(s) for s in range(n_steps)]
    outs = [torch.empty(ins[0][0][0].shape, dtype=torch.float32, device=dev) for _ in range(L)]
    stream = torch.cuda.current_stream()
    use_graph = not args.eager
    # external: inside a captured graph the records become timed event nodes
    ev = [[(torch.cuda.Event(enable_timing=True, external=use_graph),
            torch.cuda.Event(enable_timing=True, external=use_graph))
           for _ in range(L)] for _ in range(args.steps)]

    def step(s, inp, events=None, st=None):
        """Encode the token at position n0 + s, then decode over n0 + s + 1."""
        q, xk, xv = inp
        vq_encode(n0 + s, xk, cbk, ik, stream=st)
        vq_encode(n0 + s, xv, cbv, iv, stream=st)
        lens = n0 + s + 1
        for loop in range(L):
            if events is not None:
                events[loop][0].record(st or stream)
            vq_decode(loop, lens, ik, iv, cbk, cbv, q[loop], out=outs[loop], stream=st)
            if events is not None:
                events[loop][1].record(st or stream)

    for s in range(args.warmup):
        step(s, ins[s])
    torch.cuda.synchronize()
    graph = None
    if use_graph:
        # every call takes its lengths and positions by value: the K timed
        # steps are captured once and replayed once
        gstream = torch.cuda.Stream(device=dev)
        gstream.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gstream, capture_error_mode="thread_local"):
            for i in range(args.steps):
                step(args.warmup + i, ins[args.warmup + i], events=ev[i], st=gstream)
        stream.wait_stream(gstream)
        torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            step(args.warmup + i, ins[args.warmup + i], events=ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    dec_ms = sum(a.elapsed_time(b) for row in ev for (a, b) in row)
    elapsed_ms, dec_ms = max_over_ranks([elapsed_ms, dec_ms], world, dev)
    ms_per_step = elapsed_ms / args.steps
    value = wl.n_cells * world / (ms_per_step / 1000.0)
    n_launches = args.steps * L
    dec_bytes = sum(L * wl.n_layers * H * sum(vq_unit_bytes(int(n) + args.warmup + i + 1, D)
                                              for n in n0) for i in range(args.steps))
    launch_bytes = dec_bytes / n_launches
    achieved = dec_bytes / (dec_ms / 1000.0) / 1e9
    peak, peak_kind = measured_peaks()
    tr = ncu_traffic("vq_traffic.json", ("loop_aware_quantized_b200/csrc/vq.cu",
                                         "loop_aware_quantized_b200/csrc/loopkv_internal.cuh"))
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": None if tr is None else tr * launch_bytes,
                "peak_kind": peak_kind + " copy bandwidth",
                "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "kernel": "loopkv LoopVQ decode", "bytes_per_launch": launch_bytes,
                "ms_per_launch": dec_ms / n_launches,
                "note": "issue and index-load latency bind the kernel before HBM does (one "
                        "shared-memory wavefront per table lookup)"}

    e2e = None
    if not args.no_e2e:
        host_in = []
        for s in range(args.steps):
            q, xk, xv = inputs(n_steps + s)
            host_in.append(([x.cpu().pin_memory() for x in q], xk.cpu().pin_memory(),
                            xv.cpu().pin_memory()))
        dq = [torch.empty_like(x) for x in ins[0][0]]
        dxk, dxv = torch.empty_like(ins[0][1]), torch.empty_like(ins[0][2])
        host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        h2d = sum(x.numel() * x.element_size() for x in host_in[0][0]) + 2 * dxk.numel() * 2
        d2h = sum(o.numel() * o.element_size() for o in outs)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(args.steps):
            hq, hxk, hxv = host_in[s]
            for dst, src in zip(dq, hq):
                dst.copy_(src, non_blocking=True)
            dxk.copy_(hxk, non_blocking=True)
            dxv.copy_(hxv, non_blocking=True)
            step(n_steps + s, (dq, dxk, dxv))
            for dst, src in zip(host_out, outs):
                dst.copy_(src, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0] / args.steps
        e2e = {"value": wl.n_cells * world / (e2e_ms / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "overlap": "none: copy in, encode + decode, copy out per step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v1, desc, _ = oracle_baseline_vq(args.config, args.cpu_seconds)
        v, cores = oracle_all_cores(args.config, [], vq=True, cpu_seconds=2 * args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": "one process per host core, each timing its own sample like this one: "
                         "%s; on one core alone: %.4g cell-steps/s" % (desc, v1)}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u8 codebook indices, fp32 codebooks and accumulate", "data": "synthetic",
            "config": {"workload": "%s: LoopVQ, %d loops x %d layers, %d KV heads, head "
                                   "dim %d, batch %d per GPU, %d coded tokens + 1 encoded per "
                                   "step, 1 byte per 4 channels x %d loops (%.2f bits per "
                                   "element)" % (wl.name, L, wl.n_layers, H, D, B, int(n0[0]), L,
                                                 8.0 / (4 * L)),
                       "step": "encode the new token (keys, values), then decode every "
                               "(loop, layer) cell: one launch per loop",
                       "launch": ("the timed steps launched one call at a time" if args.eager
                                  else "the timed steps replay as one CUDA graph captured after "
                                       "the warm-up"),
                       "global_batch": B * world, "seq_len": int(n0[0]),
                       "parallelism": "dp%d (independent sequences)" % world,
                       "l2": "inputs larger than L2 (indices %.1f GB)" % (
                           2 * ik.numel() / 1e9), "build_s": build_s},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": (L + 2) * args.steps, "clocks": clocks,
            "token_head_cells_per_s": float(wl.n_cells * H * world *
                                            np.sum(n0 + args.warmup + args.steps // 2 + 1)) /
                                      (ms_per_step / 1000.0),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------- the oracle on every host core

_SAMPLE = None


def _sample_init(config, seqs_global, g, vq):
    global _SAMPLE
    _SAMPLE = OracleSample(config, seqs_global, g, vq)


def _sample_rate(seconds):
    return _SAMPLE.rate(seconds)[0]


class OracleAllCores:
    """The oracle as it stands in one process per host core (spawned, so no
    CUDA state is inherited), each with its own copy of the sample, built
    once; rate(seconds) times them together and sums their cell-steps/s."""

    def __init__(self, config, seqs_global, g=1, vq=False):
        import multiprocessing as mp
        self.cores = os.cpu_count() or 1
        self.pool = mp.get_context("spawn").Pool(
            self.cores, initializer=_sample_init, initargs=(config, list(seqs_global), g, vq))

    def rate(self, seconds):
        return float(sum(self.pool.map(_sample_rate, [seconds] * self.cores, chunksize=1)))

    def close(self):
        self.pool.close()
        self.pool.join()


def oracle_all_cores(config, seqs_global, g=1, vq=False, cpu_seconds=24.0):
    """(summed cell-steps/s, cores) with each core timing its sample for
    max(1 s, cpu_seconds / cores)."""
    oc = OracleAllCores(config, seqs_global, g, vq)
    try:
        return oc.rate(max(1.0, cpu_seconds / oc.cores)), oc.cores
    finally:
        oc.close()


# -------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, one process per host core, timed on
    bounded samples of the same workload (rank 0 only)."""
    if rank != 0:
        return
    from synth import workloads as W
    vq = args.config in VQ_CONFIGS
    if vq:
        wl = W.make_vq(args.config)
        text = "%s: LoopVQ decode (%s)" % (wl.name, wl.description)
    else:
        wl = W.make(args.config)
        text = workload_text(wl, wl.batch, args.q_per_kv)
    seqs = list(range(wl.batch))
    one = OracleSample(args.config, seqs, args.q_per_kv, vq)
    v1, desc = one.rate(max(1.0, min(args.cpu_seconds, 4.0)))
    t_all = time.perf_counter()
    oc = OracleAllCores(args.config, seqs, args.q_per_kv, vq)
    try:
        per = max(1.0, min(args.cpu_seconds, 6.0) / max(1, args.steps))
        for _ in range(args.warmup):
            oc.rate(0.3)
        vals = [oc.rate(per) for _ in range(args.steps)]
    finally:
        oc.close()
    wall = time.perf_counter() - t_all
    value = float(np.mean(vals))
    sample = ("one process per host core (%d), each timing its own copy of this sample for "
              "%.1f s per step: %s; on one core alone: %.4g cell-steps/s" % (oc.cores, per, desc, v1))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wl.n_cells / value if value > 0 else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": text, "impl": "CPU oracle (fp64 C++)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oc.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


def time_chunk(args, wl, dev, world, cells_g, seqs, n0, G, total_steps, sampler, keep=False):
    """Build the cache of `cells_g` (global cell ids, whole loops) for the
    global sequences `seqs` and time args.steps decode steps on it (append
    one token to every cell and decode them, in serving order) after
    args.warmup untimed ones.  Returns the device times, the decode launches'
    algorithmic bytes and, with keep=True, what the end-to-end leg reuses."""
    import torch
    import torch.distributed as dist

    from loop_aware_quantized_b200 import Plan, query_sizes, steps
    from synth.gpu import DeviceGenerator

    B, H, D = len(seqs), wl.n_heads, wl.head_dim
    n_loops = len(cells_g) // wl.n_layers
    kinds = np.asarray(wl.kinds)[cells_g]
    # each sequence's capacity: its context, the steps' new tokens and a group of headroom
    cap = (n0.astype(np.int64) + total_steps + 32 + 31) // 32 * 32
    cap = cap.astype(np.int32)
    _, need = query_sizes(n_loops, wl.n_layers, H, D, cap, kinds, wl.tau, q_per_kv=G)
    free, _ = torch.cuda.mem_get_info(dev)
    if need > 0.92 * free:
        raise SystemExit("the KV cache of %d sequences needs %.1f GB, %.1f GB are free: decode "
                         "the batch in sub-batches (--seq-chunks) or the cells in chunks "
                         "(--cell-chunks)" % (B, need / 1e9, free / 1e9))
    plan = Plan(n_loops, wl.n_layers, H, D, cap, kinds, wl.tau, device=dev, q_per_kv=G,
                decode_split=args.decode_split)
    gen = DeviceGenerator(wl, dev)
    local_of = {c: i for i, c in enumerate(cells_g)}

    # build the cache: every token of every cell through the append kernel
    # (the final loop first: RES2 cells quantize against it)
    t_build = time.perf_counter()
    kbuf = vbuf = None
    final = [c for c in cells_g if c // wl.n_layers == wl.n_loops - 1]
    for c in final + [c for c in cells_g if c not in final]:
        kbuf, vbuf = gen.kv([c], seqs, np.zeros(B, np.int32), int(n0.max()), k=kbuf, v=vbuf)
        plan.append([local_of[c]], kbuf, vbuf, n_new=n0)
    del kbuf, vbuf
    torch.cuda.synchronize()
    build_s = time.perf_counter() - t_build
    torch.cuda.empty_cache()

    phase_l = steps.phases(n_loops, wl.n_layers)
    phase_g = [[cells_g[i] for i in ph] for ph in phase_l]

    def step_inputs(s):
        """Inputs of step s: the token at position n0 + s of every cell, and the
        queries of units holding n0 + s + 1 tokens."""
        q, k, v = [], [], []
        for cells in phase_g:
            kk, vv = gen.kv(list(cells), seqs, n0 + s, 1)
            k.append(kk)
            v.append(vv)
            q.append(gen.queries(list(cells), seqs, np.tile(n0 + s + 1, (len(cells), 1)), g=G))
        return q, k, v

    n_dev_steps = args.warmup + args.steps
    inputs = [step_inputs(s) for s in range(n_dev_steps)]
    oshape = (B, H, G, D) if G > 1 else (B, H, D)
    outs = [torch.empty((len(c),) + oshape, dtype=torch.float32, device=dev) for c in phase_l]
    nsels = [[torch.zeros((len(c), B, H), dtype=torch.int32, device=dev) for c in phase_l]
             for _ in range(args.steps)]
    stream = torch.cuda.current_stream()
    use_graph = not args.eager
    # external: inside a captured graph the records become timed event nodes
    ev = [[(torch.cuda.Event(enable_timing=True, external=use_graph),
            torch.cuda.Event(enable_timing=True, external=use_graph))
           for _ in phase_l] for _ in range(args.steps)]

    for s in range(args.warmup):
        q, k, v = inputs[s]
        steps.decode_step(plan, phase_l, q, k, v, outs)
    torch.cuda.synchronize()

    graph = None
    if use_graph:
        # the library only enqueues kernels (lengths advance on the device),
        # so the K timed steps are captured once and replayed once
        gstream = torch.cuda.Stream(device=dev)
        gstream.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gstream, capture_error_mode="thread_local"):
            for i in range(args.steps):
                q, k, v = inputs[args.warmup + i]
                steps.decode_step(plan, phase_l, q, k, v, outs, nsel=nsels[i], events=ev[i],
                                  stream=gstream)
        stream.wait_stream(gstream)
        torch.cuda.synchronize()

    if sampler.proc is None:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            q, k, v = inputs[args.warmup + i]
            steps.decode_step(plan, phase_l, q, k, v, outs, nsel=nsels[i], events=ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    dec_ms = sum(a.elapsed_time(b) for row in ev for (a, b) in row)
    plan.check()

    # algorithmic bytes of every decode launch in the timed region
    dec_bytes = 0
    for i in range(args.steps):
        s = args.warmup + i
        for pi, cells in enumerate(phase_g):
            lens_own = n0 + s + 1
            # non-final loops decode before the final loop's append of this step
            lens_src = n0 + s if (pi == 0 and len(phase_g) > 1) else n0 + s + 1
            dec_bytes += decode_bytes(wl, cells, lens_own, lens_src, int(nsels[i][pi].sum()), G)
    # per phase: an append and a decode launch for the plain cells and one
    # each for RES2 cells (when the phase has them); the appends commit the
    # lengths themselves
    launches_per_step = sum(2 * (int(any(wl.kinds[c] != 4 for c in cells)) +
                                 int(any(wl.kinds[c] == 4 for c in cells)))
                            for cells in phase_g)
    out = {"elapsed_ms": elapsed_ms, "dec_ms": dec_ms, "dec_bytes": dec_bytes,
           "build_s": build_s, "dec_launches": args.steps * len(phase_g),
           "launches": launches_per_step * args.steps, "cache_bytes": plan.cache_bytes}
    if keep:
        out.update(plan=plan, phase=phase_l, inputs=inputs, outs=outs, step_inputs=step_inputs)
    else:
        # give this chunk's cache back to the device before the next chunk
        plan.close()
        plan.cache = plan.table = None
        del plan, gen, inputs, outs, nsels, ev, graph
        gc.collect()
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.config in VQ_CONFIGS:
        bench_vq(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from loop_aware_quantized_b200 import steps
    from synth import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)

    wl = W.make(args.config)
    if args.batch:
        wl.batch = args.batch
        wl.lengths = wl.lengths[:args.batch]
        wl.capacity = wl.capacity[:args.batch]
    B, H, D = wl.batch, wl.n_heads, wl.head_dim
    G = args.q_per_kv
    # weak scaling: every rank serves its own batch of B sequences
    seqs_all = shard_sequences(rank, B)
    if B % args.seq_chunks:
        raise SystemExit("--seq-chunks must divide the batch (%d)" % B)
    sb = B // args.seq_chunks
    if wl.n_loops % args.cell_chunks:
        raise SystemExit("--cell-chunks must divide the loops (%d)" % wl.n_loops)
    if args.cell_chunks > 1 and any(int(k) in (2, 4) for k in wl.kinds):
        raise SystemExit("--cell-chunks needs a plan without SHARE / RES2 cells")
    lpc = wl.n_loops // args.cell_chunks
    chunks = []
    for si in range(args.seq_chunks):
        for ci in range(args.cell_chunks):
            cells = list(range(ci * lpc * wl.n_layers, (ci + 1) * lpc * wl.n_layers))
            chunks.append((cells, list(range(si * sb, (si + 1) * sb))))
    whole = len(chunks) == 1
    total_steps = args.warmup + args.steps + (0 if (args.no_e2e or not whole)
                                              else args.warmup + args.steps)
    n0_all = wl.lengths[:B].astype(np.int32)

    sampler = ClockSampler(local)
    runs = []
    for cells_g, idx in chunks:
        seqs = [seqs_all[i] for i in idx]
        runs.append(time_chunk(args, wl, dev, world, cells_g, seqs, n0_all[idx], G, total_steps,
                               sampler, keep=whole))
    clocks = sampler.stop()
    elapsed_ms = sum(r["elapsed_ms"] for r in runs)
    dec_ms = sum(r["dec_ms"] for r in runs)
    dec_bytes = sum(r["dec_bytes"] for r in runs)
    build_s = sum(r["build_s"] for r in runs)
    n_dec_launches = sum(r["dec_launches"] for r in runs)
    launches = sum(r["launches"] for r in runs)
    cache_gb = max(r["cache_bytes"] for r in runs) / 1e9
    n0 = n0_all

    elapsed_ms, dec_ms = max_over_ranks([elapsed_ms, dec_ms], world, dev)
    ms_per_step = elapsed_ms / args.steps
    value = wl.n_cells * world / (ms_per_step / 1000.0)

    # ---- end to end through the API: pinned host inputs in, outputs out
    e2e = None
    if not args.no_e2e and whole:
        r0 = runs[0]
        plan, phase, inputs, outs, step_inputs = (r0["plan"], r0["phase"], r0["inputs"],
                                                   r0["outs"], r0["step_inputs"])
        n_dev_steps = args.warmup + args.steps
        stream = torch.cuda.current_stream()
        host_in = []
        for s in range(args.steps):
            q, k, v = step_inputs(n_dev_steps + s)
            host_in.append([[x.cpu().pin_memory() for x in grp] for grp in (q, k, v)])
        # Double-buffered serving loop: step s+1's inputs go to the device
        # (and step s's outputs come back) on a copy stream while step s
        # decodes; the events order every buffer reuse.
        copy = torch.cuda.Stream(device=dev)
        dbuf = [[[torch.empty_like(x) for x in grp] for grp in inputs[0]] for _ in range(2)]
        obuf = [[torch.empty_like(o) for o in outs] for _ in range(2)]
        host_out = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
                    for _ in range(2)]
        h2d = sum(x.numel() * x.element_size() for grp in host_in[0] for x in grp)
        d2h = sum(o.numel() * o.element_size() for o in outs)
        ev_in = [torch.cuda.Event() for _ in range(args.steps)]
        ev_done = [torch.cuda.Event() for _ in range(args.steps)]
        ev_out = [torch.cuda.Event() for _ in range(args.steps)]

        def upload(s):
            with torch.cuda.stream(copy):
                if s >= 2:
                    copy.wait_event(ev_done[s - 2])      # step s-2 has read this buffer
                for dst, src in zip(sum(dbuf[s % 2], []), sum(host_in[s], [])):
                    dst.copy_(src, non_blocking=True)
                ev_in[s].record(copy)

        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy.wait_event(e0)
        upload(0)
        for s in range(args.steps):
            stream.wait_event(ev_in[s])
            if s >= 2:
                stream.wait_event(ev_out[s - 2])         # step s-2's outputs are read back
            dq, dk, dv = dbuf[s % 2]
            steps.decode_step(plan, phase, dq, dk, dv, obuf[s % 2])
            ev_done[s].record(stream)
            if s + 1 < args.steps:
                upload(s + 1)
            with torch.cuda.stream(copy):
                copy.wait_event(ev_done[s])
                for dst, src in zip(host_out[s % 2], obuf[s % 2]):
                    dst.copy_(src, non_blocking=True)
                ev_out[s].record(copy)
        stream.wait_event(ev_out[args.steps - 1])
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0] / args.steps
        e2e = {"value": wl.n_cells * world / (e2e_ms / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "overlap": "double-buffered: a step's copies overlap the neighbouring decodes"}
        plan.check()

    peak, peak_kind = measured_peaks()
    achieved = dec_bytes / (dec_ms / 1000.0) / 1e9 if dec_ms > 0 else 0.0
    tr = ncu_traffic()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": None if tr is None else tr * dec_bytes / n_dec_launches,
                "peak_kind": peak_kind + " copy bandwidth",
                "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "kernel": "loopkv decode", "bytes_per_launch": dec_bytes / n_dec_launches,
                "ms_per_launch": dec_ms / n_dec_launches}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v1, desc, _ = oracle_baseline(args.config, args.cpu_seconds, seqs_all, G)
        v, cores = oracle_all_cores(args.config, seqs_all, G, cpu_seconds=2 * args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": "one process per host core, each timing its own sample like this one: "
                         "%s; on one core alone: %.4g cell-steps/s" % (desc, v1)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u2/u4 codes, fp32 accumulate", "data": "synthetic",
            "config": {"workload": workload_text(wl, B, G),
                       "step": "append 1 token + decode, every cell, serving order",
                       "global_batch": B * world, "seq_len": int(n0[0]),
                       "parallelism": "dp%d (independent sequences)" % world,
                       "q_per_kv": G,
                       "l2": "inputs larger than L2 (KV cache %.1f GB)" % cache_gb,
                       "build_s": build_s},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            # attended (position, KV head) pairs decoded per second, all cells
            "token_head_cells_per_s": float(wl.n_cells * H * world *
                                            np.sum(n0 + args.warmup + args.steps // 2 + 1)) /
                                      (ms_per_step / 1000.0),
            "clocks": clocks,
        }
        if args.decode_split:
            line["config"]["decode_split"] = args.decode_split
        line["config"]["launch"] = (
            "the timed steps launched one call at a time" if args.eager else
            "the timed steps (appends and decodes) replay as one CUDA graph captured after "
            "the warm-up")
        if not whole:
            line["config"]["chunks"] = (
                "%d sequence sub-batch(es) x %d cell chunk(s), decoded one after the other, each "
                "with its own cache (largest %.1f GB); a step's time is the sum over chunks"
                % (args.seq_chunks, args.cell_chunks, cache_gb))
        print(json.dumps(line), flush=True)
    for r in runs:
        if r.get("plan") is not None:
            r["plan"].close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
