"""Benchmark of the DFlash 2 draft -> select -> verify step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: launched one rank per GPU by torch.distributed.run)

Workload: the concurrency-32 case -- 32 sequences, block 8 (7 drafted
positions + 1 bonus row), vocabulary 151,936, bf16 logits, selector
embeddings 151,936 x 128 bf16 and W 128 x 128 fp32, dynconv hidden 5,120 over
32 x 8 tokens; seeded synthetic inputs of that shape (synth "b32").

One step = the whole path over one batch, each call through the C ABI:
  dflash2_topk_softmax_ex (224 draft rows, with their normalisers) ->
  dflash2_pair_select -> dflash2_verify_sample_ex (Philox, softmax q from the
  drafter normalisers: the fused cycle, draft rows not streamed again) ->
  dflash2_verify_greedy -> dflash2_dynconv2.
value = steps per second over all ranks (each rank runs its own batch:
weak scaling, no collective on the data path), from K whole steps run back to
back between two CUDA events (each step captured once in a CUDA graph).  A
step reads ~344 MB of inputs, more than the 126 MB L2: two input sets
alternate between steps and the greedy verify reads the other set's target
rows, so no call finds its streamed rows in L2.  The per-call breakdown
("calls", and the roofline of the dominant call) is a second pass: L2 is
flushed by a 256 MB write followed by a read of the same buffer (no dirty
lines left) before every call, each call timed alone with CUDA events, the
flushes outside the timed intervals.

--impl reference times the CPU oracle (the plain fp64 restatement the tests
check against) on the same workload, metric and unit, one sequence of the
batch per step, on rank 0 only.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft-select-verify cycles/sec and HBM GB/s (% of peak) at B=1/8/32, V=151936"
WORKLOAD = "b32"
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the step with eager launches instead of CUDA graph replays")
    ap.add_argument("--acceptance", action="store_true",
                    help="print the acceptance study (mean accepted tokens per verify step for "
                         "the top-1 path, the pair selector and the top-16 oracle path) instead "
                         "of a bench line")
    ap.add_argument("--only", choices=["topk_softmax", "pair_select", "verify_sample",
                                       "verify_greedy", "dynconv2"], default=None,
                    help="run and time one call of the step only (for profiling); prints a "
                         "per-call line, not a bench line")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def algorithmic_bytes(w, B):
    """Bytes each call must move at least once (inputs read once, outputs written once)."""
    G, V, d, H, T = w.G, w.V, w.d, w.H, w.T
    return {
        "topk_softmax": 2 * B * G * V + B * G * (16 * 12 + 12),
        "pair_select": 2 * B * (1 + 16 * G) * d + 4 * d * d + B * G * (16 * 8) + B * G * 8 + B * 4,
        # fused cycle: the target rows once, and the one draft row a residual
        # draw reads per sequence (drafter normalisers come from topk)
        "verify_sample": 2 * B * (G + 1) * V + 2 * B * V + B * G * 12 + B * (G + 2) * 4,
        "verify_greedy": 2 * B * (G + 1) * V + B * G * 4 + B * (G + 2) * 4,
        "dynconv2": 2 * (2 * H * H) + 2 * 2 * B * T * H + 2 * B * H,
    }


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML (read-only) for SM clock and throttle reasons while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:  # CUDA and NVML may number devices differently: match by UUID
                uuid = "GPU-" + str(torch.cuda.get_device_properties(index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.get_reasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

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
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- traffic
def recorded_traffic(kernel):
    """DRAM bytes per call from the committed ncu summary (profiles/traffic.json),
    if none of the call's source files has changed since it was captured; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        h = hashlib.sha256()
        for name in rec["sources"]:
            h.update(open(os.path.join(ROOT, "block_draft_verification_b200", "csrc", name), "rb").read())
        if h.hexdigest()[:16] != rec["sources_sha256_16"]:
            return None
        return float(rec["dram_bytes_per_call"])
    except Exception:
        return None


# --------------------------------------------------------------------------- CPU oracle
def oracle_step_seconds(w, batch, sel, conv, seqs):
    """The oracle's whole path for the given sequences of the batch (seconds)."""
    import oracle
    t0 = time.perf_counter()
    for s in seqs:
        idx, _, logp, _ = oracle.topk_softmax(batch.draft[s], w.inv_temperature)
        tok, _, _ = oracle.pair_select(idx[None], logp.astype(np.float32)[None],
                                       batch.anchor[s:s + 1], sel.emb, sel.W)
        oracle.verify_sample(batch.target[s:s + 1], batch.draft[s:s + 1], tok, w.seed, 0,
                             batch.seq_id[s:s + 1], w.inv_temperature)
        oracle.verify_greedy(batch.target[s:s + 1], tok)
        oracle.dynconv2(conv.x[s:s + 1], conv.x_prev[s:s + 1], conv.w_tap)
    return time.perf_counter() - t0


def run_reference(args, rank, world):
    import synth
    if rank != 0:
        return
    w = synth.WORKLOADS[WORKLOAD]
    batch = synth.gen_batch(w)
    sel = synth.gen_selector(w)
    conv = synth.gen_conv(w)
    for i in range(args.warmup):
        oracle_step_seconds(w, batch, sel, conv, [i % w.B])
    times = [oracle_step_seconds(w, batch, sel, conv, [i % w.B]) for i in range(args.steps)]
    per_seq = float(np.mean(times))
    value = 1.0 / (per_seq * w.B)                 # full 32-sequence steps per second
    sample = "one of the 32 sequences per step (its 7 draft rows, 8 target rows, selector, " \
             "both verifies and its 8 dynconv tokens), scaled by 32"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "cycles/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_seq * w.B * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "concurrency-32: B=32, block 8, V=151936, bf16 logits, "
                                   "d=128 selector, dynconv H=5120 x 32x8 tokens",
                       "parallelism": "rank 0 only (CPU)"},
            "cpu_baseline": {"value": value, "unit": "cycles/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "cycles/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- acceptance study
def acceptance_paths(dfl, torch, T, Q, anchor, E, Wsel, inv_t):
    """The three drafted paths of a batch, every step in the library's kernels
    (the path choice is a compare and a select on their outputs): the drafter's
    top-1 per position, the pair selector's path, and the top-16 oracle path
    (the target's own token wherever it is among the drafter's 16 candidates,
    else the top-1).  Returns the paths and the per-position hit masks."""
    B, G1, V = T.shape
    G = G1 - 1
    idx, _, logp, _ = dfl.topk_softmax(Q.reshape(-1, V), inv_t)
    cand = idx.view(B, G, 16)
    t = dfl.topk_softmax(T[:, :G].reshape(-1, V), inv_t)[0].view(B, G, 16)[:, :, 0]
    hit16 = (cand == t[:, :, None]).any(-1)
    top1 = cand[:, :, 0].contiguous()
    oracle_path = torch.where(hit16, t, top1).contiguous()
    sel = dfl.pair_select(cand, logp.view(B, G, 16), anchor, E, Wsel)[0]
    return {"top1": top1, "selector": sel, "top16_oracle": oracle_path}, hit16, top1 == t


def run_acceptance(args):
    """Synthetic analog of the pages' top-16 oracle figure (a trained drafter:
    4.27 accepted tokens per step on its top-1 path, 6.79 when told the target
    token whenever it is in the top 16): mean (n + 1) under greedy verification
    for the three paths, on the calibrated synthetic workloads."""
    import torch

    import block_draft_verification_b200 as dfl
    import synth

    dev = torch.device("cuda", 0)

    def dev_t(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    out = {}
    for name, ncyc in (("b1", 128), ("b8", 128), ("b32", 128)):
        w = synth.WORKLOADS[name]
        sel = synth.gen_selector(w)
        E, Wsel = dev_t(sel.emb), dev_t(sel.W)
        acc = {"top1": [], "selector": [], "top16_oracle": []}
        h16, h1 = [], []
        for first in range(0, ncyc, 32):
            b = synth.gen_batch(w, B=min(32, ncyc - first), first=first)
            T = dev_t(b.target)
            paths, hit16, hit1 = acceptance_paths(dfl, torch, T, dev_t(b.draft), dev_t(b.anchor),
                                                  E, Wsel, w.inv_temperature)
            for k, p in paths.items():
                acc[k] += (dfl.verify_greedy(T, p)[0] + 1).cpu().tolist()
            h16.append(hit16.float().mean().item())
            h1.append(hit1.float().mean().item())
        out[name] = {k: round(float(np.mean(v)), 3) for k, v in acc.items()}
        out[name].update(cycles=ncyc, target_in_top16=round(float(np.mean(h16)), 4),
                         target_is_top1=round(float(np.mean(h1)), 4))
    print(json.dumps({"acceptance_study": out, "block": 8,
                      "pages": "trained drafter, top-1 path 4.27 -> top-16 oracle 6.79"}),
          flush=True)


# --------------------------------------------------------------------------- ranks
def rank_first_sequence(rank, k, B):
    """First sequence of input set k (0 or 1) on a rank: every (rank, set)
    pair takes its own block of B sequences, so the ranks' batches are
    disjoint (weak scaling, no data-path collective)."""
    return (rank * 2 + k) * B


def max_over_ranks(values, world, device):
    """Elementwise maximum of per-rank float values (the slowest rank's time),
    as float64 on `device`; one all-reduce when world > 1."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t


# --------------------------------------------------------------------------- GPU
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import block_draft_verification_b200 as dfl
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[WORKLOAD]
    B, G, V = w.B, w.G, w.V

    # inputs: two input sets per rank (alternated between steps), weights once
    sets = [(synth.gen_batch(w, first=rank_first_sequence(rank, k, B)),
             synth.gen_conv(w, first=rank_first_sequence(rank, k, B)))
            for k in range(2)]
    sel = synth.gen_selector(w)
    wtap = sets[0][1].w_tap

    def dev_t(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    E, Wsel, Wtap = dev_t(sel.emb), dev_t(sel.W), dev_t(wtap)
    inputs = []
    for b, c in sets:
        inputs.append(dict(T=dev_t(b.target), Q=dev_t(b.draft), anchor=dev_t(b.anchor),
                           sid=dev_t(b.seq_id.view(np.int32)), x=dev_t(c.x), xp=dev_t(c.x_prev)))
    ws = dfl.Workspace(dev, dfl.workspace_bytes(B, G, V) + dfl.workspace_bytes(B * G, 1, V))
    def topk_out():
        return (torch.empty((B * G, 16), dtype=torch.int32, device=dev),
                torch.empty((B * G, 16), dtype=torch.float32, device=dev),
                torch.empty((B * G, 16), dtype=torch.float32, device=dev),
                torch.empty((B * G,), dtype=torch.float32, device=dev),
                torch.empty((B * G,), dtype=torch.float32, device=dev),
                torch.empty((B * G,), dtype=torch.float32, device=dev))

    for k, inp in enumerate(inputs):
        inp["topk"] = topk_out()  # per input set: the normalisers stay with their rows
    outs = dict(
        sel=(torch.empty((B, G), dtype=torch.int32, device=dev),
             torch.empty((B, G), dtype=torch.int32, device=dev),
             torch.empty((B,), dtype=torch.float32, device=dev)),
        samp=(torch.empty((B,), dtype=torch.int32, device=dev),
              torch.empty((B, G + 1), dtype=torch.int32, device=dev)),
        greedy=(torch.empty((B,), dtype=torch.int32, device=dev),
                torch.empty((B, G + 1), dtype=torch.int32, device=dev)),
        conv=torch.empty((B, w.T, w.H), dtype=torch.bfloat16, device=dev),
    )
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)
    names = ["topk_softmax", "pair_select", "verify_sample", "verify_greedy", "dynconv2"]
    kernels_per_step = {"topk_softmax": 1, "pair_select": 1, "verify_sample": 1,
                        "verify_greedy": 1, "dynconv2": 1}

    def calls(inp, step, t_greedy=None):
        tk = inp["topk"]
        tg = inp["T"] if t_greedy is None else t_greedy
        return [
            lambda: dfl.topk_softmax(inp["Q"].view(B * G, V), w.inv_temperature, out=tk, ws=ws,
                                     stats=True),
            lambda: dfl.pair_select(tk[0].view(B, G, 16), tk[2].view(B, G, 16), inp["anchor"], E,
                                    Wsel, out=outs["sel"], ws=ws),
            lambda: dfl.verify_sample(inp["T"], inp["Q"], outs["sel"][0], w.seed, step, inp["sid"],
                                      w.inv_temperature, out=outs["samp"], ws=ws,
                                      draft_stats=(tk[4].view(B, G), tk[5].view(B, G))),
            lambda: dfl.verify_greedy(tg, outs["sel"][0], out=outs["greedy"], ws=ws),
            lambda: dfl.dynconv2(inp["x"], inp["xp"], Wtap, out=outs["conv"]),
        ]

    stream = torch.cuda.current_stream(dev)

    def run_calls(n, step0, record):
        evs = []
        for s in range(n):
            inp = inputs[(step0 + s) % 2]
            row = []
            for name, fn in zip(names, calls(inp, step0 + s)):
                if record and args.only and name != args.only:
                    continue
                # L2 flush: write a buffer twice the size of L2, then read it,
                # so the timed call starts with no data of its own in L2 and
                # no dirty lines left to write back
                flush.fill_(s & 0xFF)
                flush_sink.add_(flush.view(torch.int64).sum())
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                row.append((e0, e1))
            evs.append(row)
        return evs

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # The step as timed: the five calls back to back, no flush in between.
    # Input sets alternate between steps and the greedy verify reads the
    # other set's target rows, so no call finds the rows it streams in L2
    # from an earlier call (a step reads ~344 MB of inputs, L2 is 126 MB);
    # the sampling verify may find the draft rows topk just read (the fused
    # cycle).  Each set's step is captured once in a CUDA graph (launch cost
    # off the host); replays reuse the captured Philox step, which changes
    # no cost.
    def step_eager(k, step):
        for fn in calls(inputs[k], step, t_greedy=inputs[1 - k]["T"]):
            fn()

    graphs, graph_note = None, "eager launches"
    if not args.no_graph and not args.only:
        try:
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            with torch.cuda.stream(cap):
                for k in range(2):
                    step_eager(k, k)
            cap.synchronize()
            graphs = []
            for k in range(2):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    step_eager(k, k)
                graphs.append(g)
            torch.cuda.synchronize(dev)
            graph_note = "CUDA graph replays (one graph per input set)"
        except Exception as e:  # capture refused: time eager launches instead
            graphs = None
            graph_note = "eager launches (graph capture failed: %s)" % str(e).splitlines()[0][:120]
            torch.cuda.synchronize(dev)

    def run_step_pass(n, step0):
        for s in range(n):
            k = (step0 + s) % 2
            if graphs is not None:
                graphs[k].replay()
            else:
                step_eager(k, step0 + s)

    run_calls(args.warmup, 0, False)
    run_step_pass(max(args.warmup, 3), 0)
    barrier()
    sampler = ClockSampler(local_rank)
    with sampler:
        t_wall0 = time.perf_counter()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        run_step_pass(args.steps, args.warmup)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall0
        barrier()
        evs = run_calls(args.steps, args.warmup, True)
        torch.cuda.synchronize(dev)
    barrier()
    per_call = np.array([[e0.elapsed_time(e1) for (e0, e1) in row] for row in evs])  # ms
    if args.only:  # one call alone: a per-call line for profiling, not a bench line
        if rank == 0:
            us = float(per_call.mean()) * 1e3
            nbytes = algorithmic_bytes(w, B)[args.only]
            print(json.dumps({"only": args.only, "us": round(us, 2), "algorithmic_bytes": nbytes,
                              "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1),
                              "steps": args.steps}), flush=True)
        return
    local = max_over_ranks([s0.elapsed_time(s1), float(per_call.sum(axis=1).mean())] +
                           per_call.mean(axis=0).tolist(), world, dev)
    ms_per_step = float(local[0]) / args.steps
    calls_sum_ms = float(local[1])
    mean_call_ms = local[2:].cpu().numpy()

    # e2e: the public API with host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        b0, c0 = sets[0]
        host = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in
                dict(T=b0.target.view(np.int16), Q=b0.draft.view(np.int16), anchor=b0.anchor,
                     sid=b0.seq_id.view(np.int32), x=c0.x.view(np.int16),
                     xp=c0.x_prev.view(np.int16)).items()}
        res_host = dict(samp_n=torch.empty((B,), dtype=torch.int32).pin_memory(),
                        samp_tok=torch.empty((B, G + 1), dtype=torch.int32).pin_memory(),
                        greedy_tok=torch.empty((B, G + 1), dtype=torch.int32).pin_memory(),
                        path=torch.empty((B, G), dtype=torch.int32).pin_memory(),
                        conv=torch.empty((B, w.T, w.H), dtype=torch.int16).pin_memory())
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in res_host.values())
        dbuf = inputs[0]

        def e2e_step(step):
            dbuf["T"].view(torch.int16).copy_(host["T"], non_blocking=True)
            dbuf["Q"].view(torch.int16).copy_(host["Q"], non_blocking=True)
            dbuf["anchor"].copy_(host["anchor"], non_blocking=True)
            dbuf["sid"].copy_(host["sid"], non_blocking=True)
            dbuf["x"].view(torch.int16).copy_(host["x"], non_blocking=True)
            dbuf["xp"].view(torch.int16).copy_(host["xp"], non_blocking=True)
            for fn in calls(dbuf, step):
                fn()
            res_host["samp_n"].copy_(outs["samp"][0], non_blocking=True)
            res_host["samp_tok"].copy_(outs["samp"][1], non_blocking=True)
            res_host["greedy_tok"].copy_(outs["greedy"][1], non_blocking=True)
            res_host["path"].copy_(outs["sel"][0], non_blocking=True)
            res_host["conv"].copy_(outs["conv"].view(torch.int16), non_blocking=True)

        for s in range(max(1, args.warmup)):
            e2e_step(s)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ne = max(3, min(args.steps, 20))
        e0.record(stream)
        for s in range(ne):
            e2e_step(s)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        t = max_over_ranks([e0.elapsed_time(e1) / ne], world, dev)
        e2e = {"value": world * 1000.0 / float(t[0]), "unit": "cycles/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    if rank != 0:
        return
    peak, peak_kind = peaks()
    alg = algorithmic_bytes(w, B)
    calls_info = {}
    for i, n in enumerate(names):
        us = float(mean_call_ms[i]) * 1e3
        gbs = alg[n] / (us * 1e-6) / 1e9
        calls_info[n] = {"us": round(us, 2), "algorithmic_bytes": alg[n], "GB/s": round(gbs, 1),
                         "frac_of_hbm_peak": round(gbs / peak, 4)}
    dom = max(names, key=lambda n: calls_info[n]["us"])
    kernel_of = {"topk_softmax": "topk_softmax", "pair_select": "pair_select",
                 "verify_sample": "verify_sample", "verify_greedy": "verify_greedy",
                 "dynconv2": "dynconv2"}
    step_bytes = sum(alg.values())
    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9
    sample_cycle_us = sum(calls_info[n]["us"] for n in ("topk_softmax", "pair_select", "verify_sample"))
    greedy_cycle_us = sum(calls_info[n]["us"] for n in ("topk_softmax", "pair_select", "verify_greedy"))

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        b0, c0 = sets[0]
        seqs = list(range(8))
        sec = oracle_step_seconds(w, b0, sel, synth.ConvInputs(c0.x, c0.x_prev, wtap), seqs)
        cpu = {"value": 1.0 / (sec / len(seqs) * B), "unit": "cycles/s", "cores": 1,
               "kind": "oracle",
               "sample": "8 of the 32 sequences of one step (all five calls), scaled by 32/8; "
                         "single-threaded fp64 oracle"}
    value = world * 1000.0 / ms_per_step
    line = {
        "metric": METRIC, "value": value, "unit": "cycles/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "concurrency-32: B=32, block 8 (7 drafted + 1 bonus), V=151936, "
                               "bf16 logits, selector d=128 (emb 151936x128 bf16, W fp32), "
                               "sampling at T=1.0 (fused cycle: drafter normalisers from topk) "
                               "and greedy verify, dynconv H=5120 over 32x8 tokens; one step = "
                               "all five calls",
                   "global_batch": B * world, "parallelism": "dp%d (independent batches)" % world,
                   "timing": "K whole steps between two CUDA events on the launching "
                             "stream, " + graph_note,
                   "l2": "inputs larger than L2: a step reads ~344 MB of inputs (two input sets "
                         "alternated, the greedy verify on the other set's target rows); the "
                         "per-call breakdown ('calls', roofline) flushes L2 (256 MB write + "
                         "read) before every call, outside its timed intervals",
                   "calls_sum_us": round(calls_sum_ms * 1e3, 2),
                   "step_hbm_GBps": round(step_gbs, 1),
                   "step_frac_of_hbm_peak": round(step_gbs / peak, 4),
                   "sampling_cycle_per_s": round(1e6 / sample_cycle_us, 1),
                   "greedy_cycle_per_s": round(1e6 / greedy_cycle_us, 1),
                   "wall_s_timed": round(t_wall, 3)},
        "calls": calls_info,
        "roofline": {"kernel": kernel_of[dom], "bound": "hbm",
                     "achieved": calls_info[dom]["GB/s"], "peak": peak, "unit": "GB/s",
                     "frac": round(calls_info[dom]["GB/s"] / peak, 4),
                     "traffic": recorded_traffic(dom), "peak_kind": peak_kind},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(args.steps * sum(kernels_per_step.values())),
        "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.acceptance:
            if rank == 0:
                run_acceptance(args)
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
