"""Benchmark: CSA indexer distillation loss, forward + backward, on B200.

One step = sai_window_lse -> sai_distill_target -> sai_distill_kl (with
dscores) over one batch of the V4-Flash-width workload (B=1, S=4096, H=64,
D=512, cr=4, K=512, W=128; seeded synthetic inputs). The metric is tokens/s
(B*S per step). Inputs are resident in HBM for `value`; `e2e` repeats the step
through the same C-ABI calls from pinned host buffers, with the host->device
copies of every input and the device->host copy of the loss and dscores inside
the timed region (each step's input copies overlap the previous step's
compute).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs its own batch (independent problems,
weak scaling, no collective on the data path); the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on the host cores instead.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOAD = "flash"
METRIC = "distill-loss tokens/s (fwd+bwd), S=4096 H=64 K=512 D=512; % bf16 TC peak"
UNIT = "tokens/s"
CLOCK_WINDOW_S = 1.5


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="sai", choices=["sai", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--long-steps", type=int, default=30,
                    help="timed steps of the long-context side line (0: skip it)")
    ap.add_argument("--packed-steps", type=int, default=50,
                    help="timed steps of the packed-documents side line (0: skip it)")
    ap.add_argument("--fused-steps", type=int, default=200,
                    help="timed steps of the window-fused route on the main workload (0: skip it)")
    return ap.parse_args()


def workload_config(w, n):
    return {
        "workload": f"{WORKLOAD}: B={w.B} S={w.S} H={w.H} D={w.D} cr={w.cr} K={w.K} W={w.W}, "
                    f"top-K of a random causal score, sorted ascending; bf16 Q/Kw/pool N(0,1), "
                    f"fp32 sink N(0,1), scores N(0,2); "
                    + ("seed 1003" if n == 1 else f"seeds 1003..{1003 + n - 1}, one batch per rank"),
        "global_batch": w.B * n,
        "seq_len": w.S,
        "parallelism": f"dp{n}" if n > 1 else "single",
        "l2": "flushed between timed steps (untimed): a 256 MiB write, then a 256 MiB read of another "
              "buffer, so the L2 holds no line of the inputs and no dirty line of the flush",
    }


def candidate_blocks(w):
    """Blocks every token may select (causal and inside its document): the
    score entries the selection kernel reads."""
    t = np.arange(w.S)
    hi = (t + 1) // w.cr
    n = 0
    for b in range(w.B):
        d0 = np.zeros(w.S, dtype=np.int64) if w.doc_start is None else np.clip(w.doc_start[b], 0, t)
        lo = (d0 + w.cr - 1) // w.cr
        n += int(np.maximum(hi - lo, 0).sum())
    return n


def algorithmic_counts(w):
    """Valid selected slots and window keys: the units behind the flop and byte
    counts (2*H*D flops per slot or key)."""
    t = np.arange(w.S)
    sel = int((w.valid != 0).sum())
    win = 0
    for b in range(w.B):
        d0 = np.zeros(w.S, dtype=np.int64) if w.doc_start is None else w.doc_start[b].astype(np.int64)
        lo = np.maximum(d0, t - w.W + 1)
        win += int((t - lo + 1).sum())
    return sel, win


def to_dev(w, dev):
    import torch
    t = {}
    for k in ("Q", "Kw", "pool"):
        t[k] = torch.from_numpy(getattr(w, k).view(np.int16)).to(dev).view(torch.bfloat16)
    for k in ("idx", "sink", "doc_start", "scores", "valid"):
        a = getattr(w, k)
        t[k] = None if a is None else torch.from_numpy(a).to(dev)
    return t


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("bf16_tflops", 1590.0), d.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


def traffic_record(kernel_src: str):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current sources of the kernel (else null)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    r = rec.get(kernel_src)
    if not r:
        return None
    csrc = os.path.join(ROOT, "sparse_attention_indexer_window_b200", "csrc")
    m = hashlib.sha256()
    for name in r.get("sources", [kernel_src]):
        with open(os.path.join(csrc, name), "rb") as f:
            m.update(f.read())
    if r.get("src_sha256_16") != m.hexdigest()[:16]:
        return None
    return r.get("dram_bytes_per_launch")


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while running.

    Samples carry nvidia-smi's own timestamps, so the summary can say how many
    of them fall inside a given wall-clock window (the timed region)."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 50

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"sai_clocks_{os.getpid()}_{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, window=None, timed=None):
        """Summary over the samples inside `window` (wall-clock (t0, t1)),
        with the count of those inside `timed` as well."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "samples_in_timed_region": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        with open(self.path) as f:
            summary = self.parse(f, window, timed)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return summary

    @staticmethod
    def _stamp(s):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(s, fmt).timestamp()
            except ValueError:
                pass
        return None

    @classmethod
    def parse(cls, lines, window=None, timed=None):
        """Summary of nvidia-smi rows in the order of Q: median SM clock, max
        clock, and every slowdown reason seen active in any sample, over the
        rows whose timestamp lies in `window` (all rows when None)."""
        sm, mx, reasons, n, n_timed = [], None, set(), 0, 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            ts = cls._stamp(parts[0])
            if window is not None and (ts is None or not window[0] <= ts <= window[1]):
                continue
            try:
                sm.append(float(parts[2]))
                mx = float(parts[3])
            except ValueError:
                continue
            n += 1
            if timed is not None and ts is not None and timed[0] <= ts <= timed[1]:
                n_timed += 1
            for nm, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": n, "samples_in_timed_region": n_timed,
                "interval_ms": cls.INTERVAL_MS}


def cpu_baseline(w, seconds: float):
    """The fp64 oracle on a bounded sample of the workload's tokens."""
    import oracle
    rng = np.random.default_rng(11)
    probe = np.sort(rng.choice(w.B * w.S, size=16, replace=False))
    t0 = time.perf_counter()
    oracle.run_all(w, probe)
    dt = max(time.perf_counter() - t0, 1e-3)
    n = int(min(w.B * w.S, max(16, seconds / dt * 16)))
    tok = np.sort(rng.choice(w.B * w.S, size=n, replace=False))
    t0 = time.perf_counter()
    oracle.run_all(w, tok)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of {w.B * w.S} tokens drawn uniformly (seed 11), whole path "
                      f"(window_lse, target, KL rows), fp64, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import synth
    w = synth.make(WORKLOAD)
    per_tok = 0.0
    probe = np.arange(w.S - 8, w.S)
    t0 = time.perf_counter()
    oracle.run_all(w, probe)
    per_tok = (time.perf_counter() - t0) / len(probe)
    budget = 150.0
    n_per_step = int(max(1, min(w.B * w.S, budget / max(args.steps + args.warmup, 1) / max(per_tok, 1e-6))))
    rng = np.random.default_rng(12)
    for _ in range(args.warmup):
        oracle.run_all(w, np.sort(rng.choice(w.B * w.S, n_per_step, replace=False)))
    done, el = 0, 0.0
    for _ in range(args.steps):
        tok = np.sort(rng.choice(w.B * w.S, n_per_step, replace=False))
        t0 = time.perf_counter()
        oracle.run_all(w, tok)
        el += time.perf_counter() - t0
        done += n_per_step
    v = done / el
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, 1),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{n_per_step} uniformly drawn tokens of {w.B * w.S} per step"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0



def side_line(name, steps, dev, stream, rank, err, flush_l2):
    """window_lse -> distill_target -> distill_kl on another workload, `steps`
    timed steps after 3 warm-up steps, L2 flushed before each; the target's
    spill workspace and the KL's are allocated once, outside the timed loop."""
    import torch
    import sparse_attention_indexer_window_b200 as sai
    from sparse_attention_indexer_window_b200 import shard
    import synth
    wX = synth.make(name, seed=shard.rank_seed(synth.CONFIGS[name].seed, rank))
    tX = to_dev(wX, dev)
    wl = torch.empty((wX.B, wX.S, wX.H), device=dev)
    p = torch.empty((wX.B, wX.S, wX.K), device=dev)
    ds = torch.empty((wX.B, wX.S, wX.K), device=dev)
    loss = torch.empty(1, device=dev)
    ws_kl = torch.empty(sai.kl_workspace_bytes(wX.B, wX.S, wX.K), dtype=torch.uint8, device=dev)
    nb = sai.target_workspace_bytes(wX.B, wX.S, wX.H, wX.D, wX.K, dev)
    ws_t = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(3 + steps):
        flush_l2(i)
        if i >= 3:
            ev[i - 3][0].record(stream)
        sai.window_lse(tX["Q"], tX["Kw"], wX.W, wX.scale, tX["doc_start"], out=wl)
        if i >= 3:
            ev[i - 3][1].record(stream)
        sai.distill_target(tX["Q"], tX["pool"], tX["idx"], wl, wX.cr, wX.scale, sink=tX["sink"],
                           doc_start=tX["doc_start"], err=err, out=p, workspace=ws_t)
        if i >= 3:
            ev[i - 3][2].record(stream)
        sai.distill_kl(p, tX["scores"], tX["valid"], wX.coeff, workspace=ws_kl, loss=loss, dscores=ds)
        if i >= 3:
            ev[i - 3][3].record(stream)
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0
    sel, win = algorithmic_counts(wX)
    ms = statistics.mean(e[0].elapsed_time(e[3]) for e in ev)
    tgt = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    recipe = {"long": "random distinct causal blocks, -1 tail",
              "packed": "top-K of a random causal score per document, sorted ascending"}[name]
    line = {
        "workload": f"{name}: B={wX.B} S={wX.S} H={wX.H} D={wX.D} cr={wX.cr} K={wX.K} W={wX.W}, {recipe}; "
                    f"same value distributions",
        "steps": steps, "ms_per_step": ms, "tokens_per_s": wX.B * wX.S / (ms / 1e3),
        "kernels_ms": {"window_lse": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
                       "distill_target": tgt,
                       "distill_kl": statistics.mean(e[2].elapsed_time(e[3]) for e in ev)},
        "selected_slots": sel, "window_keys": win,
        "distill_target_tflops": 2.0 * wX.H * wX.D * sel / (tgt / 1e3) / 1e12,
        "step_tflops": 2.0 * wX.H * wX.D * (sel + win) / (ms / 1e3) / 1e12,
        "target_spill_workspace_bytes": nb,
    }
    del tX
    torch.cuda.empty_cache()
    return line

def fused_window_line(w, t, steps, stream, err, flush_l2, p, ds, loss, ws):
    """The same step as two calls, distill_target_window -> distill_kl (the
    window band inside the target kernel, Q read once), on the main
    workload's inputs, timed like the main line."""
    import torch
    import sparse_attention_indexer_window_b200 as sai
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(3 + steps):
        flush_l2(i)
        if i >= 3:
            ev[i - 3][0].record(stream)
        sai.distill_target_window(t["Q"], t["Kw"], t["pool"], t["idx"], w.W, w.cr, w.scale, sink=t["sink"],
                                  doc_start=t["doc_start"], err=err, out=p)
        if i >= 3:
            ev[i - 3][1].record(stream)
        sai.distill_kl(p, t["scores"], t["valid"], w.coeff, workspace=ws, loss=loss, dscores=ds)
        if i >= 3:
            ev[i - 3][2].record(stream)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sel, win = algorithmic_counts(w)
    ms = statistics.mean(e[0].elapsed_time(e[2]) for e in ev)
    tgt = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    fl = 2.0 * w.H * w.D * (sel + win)
    return {
        "route": "sai_distill_target_window -> sai_distill_kl (two calls, Q read once)",
        "steps": steps, "ms_per_step": ms, "tokens_per_s": w.B * w.S / (ms / 1e3),
        "kernels_ms": {"distill_target_window": tgt,
                       "distill_kl": statistics.mean(e[1].elapsed_time(e[2]) for e in ev)},
        "distill_target_window_tflops": fl / (tgt / 1e3) / 1e12,
        # DRAM bytes of one launch (ncu), against the algorithmic Q + Kw + idx
        # + pool + p: Q is read once for both the window band and the scores
        "traffic": traffic_record("target_tc.cu#window"),
        "algorithmic_bytes": w.B * w.S * (w.H * w.D * 2 + w.D * 2 + w.K * 4 + w.K * 4) + w.B * (w.S // w.cr) * w.D * 2,
        "algorithmic": f"2*H*D flops per selected slot and window key x ({sel} + {win}) = {fl:.4g} flops/launch",
        "gpu_launches": 2 * steps,
    }


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)

    import sparse_attention_indexer_window_b200 as sai
    from sparse_attention_indexer_window_b200 import shard
    import synth

    # weak scaling: every rank runs its own full batch of the workload
    w = synth.make(WORKLOAD, seed=shard.rank_seed(synth.CONFIGS[WORKLOAD].seed, rank))
    t = to_dev(w, dev)
    B, S, H, D, K = w.B, w.S, w.H, w.D, w.K
    wl = torch.empty((B, S, H), device=dev)
    p = torch.empty((B, S, K), device=dev)
    ds = torch.empty((B, S, K), device=dev)
    loss = torch.empty(1, device=dev)
    ws = torch.empty(sai.kl_workspace_bytes(B, S, K), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2(i):
        # The write evicts every line of the inputs; the read of a second
        # buffer then evicts the write's own dirty lines, whose write-back
        # would otherwise land inside the next timed kernel.
        flush.fill_(i & 0xFF)
        flush_r.sum()

    def step():
        sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"], out=wl)
        sai.distill_target(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, sink=t["sink"],
                           doc_start=t["doc_start"], err=err, out=p)
        sai.distill_kl(p, t["scores"], t["valid"], w.coeff, workspace=ws, loss=loss, dscores=ds)

    for _ in range(max(args.warmup, 3)):
        flush_l2(1)
        step()
    torch.cuda.synchronize(dev)

    nsteps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nsteps)]
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.2)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    for i in range(nsteps):
        flush_l2(i)
        e = ev[i]
        e[0].record(stream)
        sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"], out=wl)
        e[1].record(stream)
        sai.distill_target(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, sink=t["sink"],
                           doc_start=t["doc_start"], err=err, out=p)
        e[2].record(stream)
        sai.distill_kl(p, t["scores"], t["valid"], w.coeff, workspace=ws, loss=loss, dscores=ds)
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    # A short timed region holds few clock samples: keep the same steps running
    # (untimed) until the clock window spans at least CLOCK_WINDOW_S, so the
    # record shows the clocks this work runs at. Every rank runs the same count.
    soak = 0
    if wall1 - wall0 < CLOCK_WINDOW_S:
        per = max((wall1 - wall0) / nsteps, 1e-5)
        soak = int(min(200000, (CLOCK_WINDOW_S - (wall1 - wall0)) / per)) + 1
        for i in range(soak):
            flush_l2(i)
            step()
        torch.cuda.synchronize(dev)
    wall2 = time.time()
    if world > 1:
        dist.barrier()
    clk = clocks.stop(window=(wall0, wall2), timed=(wall0, wall1))

    # Warm-L2 figures for reference: the same steps back to back with no
    # flush between them (Q alone, 268 MB, is larger than the 126 MB L2).
    warm_steps = max(3, min(nsteps, 200))
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(warm_steps)]
    for i in range(warm_steps):
        e = wev[i]
        e[0].record(stream)
        sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"], out=wl)
        e[1].record(stream)
        sai.distill_target(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, sink=t["sink"],
                           doc_start=t["doc_start"], err=err, out=p)
        e[2].record(stream)
        sai.distill_kl(p, t["scores"], t["valid"], w.coeff, workspace=ws, loss=loss, dscores=ds)
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    warm = {"steps": warm_steps,
            "ms_per_step": statistics.mean(e[0].elapsed_time(e[3]) for e in wev),
            "kernels_ms": {"window_lse": statistics.mean(e[0].elapsed_time(e[1]) for e in wev),
                           "distill_target": statistics.mean(e[1].elapsed_time(e[2]) for e in wev),
                           "distill_kl": statistics.mean(e[2].elapsed_time(e[3]) for e in wev)},
            "note": "no L2 flush between steps; not the headline"}
    clk["window"] = f"timed region ({wall1 - wall0:.3f} s) plus {soak} more steps of the same work"
    k_win = [e[0].elapsed_time(e[1]) for e in ev]
    k_tgt = [e[1].elapsed_time(e[2]) for e in ev]
    k_kl = [e[2].elapsed_time(e[3]) for e in ev]
    total_ms = shard.max_over_ranks(float(sum(e[0].elapsed_time(e[3]) for e in ev)), device=dev)
    assert int(err.item()) == 0
    ms_step = total_ms / nsteps
    tokens_total = B * S * world * nsteps
    value = tokens_total / (total_ms / 1e3)

    # ---------------------------------------------------------------- e2e
    host = {}
    for k in ("Q", "Kw", "pool", "idx", "sink", "doc_start", "scores", "valid"):
        if t[k] is not None:
            host[k] = t[k].cpu().pin_memory()
    out_loss = torch.empty(1).pin_memory()
    out_ds = torch.empty((B, S, K)).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_loss.numel() * 4 + out_ds.numel() * 4
    # Two device copies of the inputs and a copy stream: step i+1's inputs
    # cross the host link while step i computes (a step's copy waits only for
    # the step two before it, the last one to read that buffer).
    dqs = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    cstream = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    for e in ev_free:
        e.record(stream)

    def e2e_step(i):
        dq = dqs[i & 1]
        cstream.wait_event(ev_free[i & 1])
        with torch.cuda.stream(cstream):
            for k, v in host.items():
                dq[k].copy_(v, non_blocking=True)
        ev_in[i & 1].record(cstream)
        stream.wait_event(ev_in[i & 1])
        sai.window_lse(dq["Q"], dq["Kw"], w.W, w.scale, dq.get("doc_start"), out=wl)
        sai.distill_target(dq["Q"], dq["pool"], dq["idx"], wl, w.cr, w.scale, sink=dq.get("sink"),
                           doc_start=dq.get("doc_start"), err=err, out=p)
        sai.distill_kl(p, dq["scores"], dq["valid"], w.coeff, workspace=ws, loss=loss, dscores=ds)
        ev_free[i & 1].record(stream)
        out_loss.copy_(loss, non_blocking=True)
        out_ds.copy_(ds, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cstream.wait_event(e0)        # no copy of the timed steps starts before e0
    for i in range(args.e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = shard.max_over_ranks(e0.elapsed_time(e1), device=dev)
    e2e_value = B * S * world * args.e2e_steps / (e2e_ms / 1e3)

    # ------------------------------------------- block selection (side line)
    # sai_indexer_topk feeds idx, scores and valid to the step above; it is
    # timed on its own, on this workload's shape, and is not part of `value`.
    isc = torch.from_numpy(synth.index_scores(B, S, w.cr, seed=shard.rank_seed(7001, rank))).to(dev)
    t_idx = torch.empty((B, S, K), dtype=torch.int32, device=dev)
    t_sel = torch.empty((B, S, K), dtype=torch.float32, device=dev)
    t_val = torch.empty((B, S, K), dtype=torch.uint8, device=dev)
    sel_steps = max(3, min(nsteps, 200))
    sel_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(sel_steps)]
    for i in range(3 + sel_steps):
        flush_l2(i)
        if i >= 3:
            sel_ev[i - 3][0].record(stream)
        sai.indexer_topk(isc, w.cr, K, doc_start=t["doc_start"], idx=t_idx, sel_scores=t_sel, valid=t_val)
        if i >= 3:
            sel_ev[i - 3][1].record(stream)
    torch.cuda.synchronize(dev)
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in sel_ev)
    del isc

    # ------------------------------------- the window-fused route (side line)
    fused = fused_window_line(w, t, args.fused_steps, stream, err, flush_l2, p, ds, loss, ws) \
        if args.fused_steps > 0 else None

    # ------------------------------------------- side lines: long, packed
    # The same three calls on the long-context workload (S=16384, K=2048: up
    # to 2048 selected blocks per token) and the packed one (B=4, two
    # documents per row), timed like the step above; not part of `value`.
    del t
    torch.cuda.empty_cache()
    long_line = side_line("long", args.long_steps, dev, stream, rank, err, flush_l2) \
        if args.long_steps > 0 else None
    packed_line = side_line("packed", args.packed_steps, dev, stream, rank, err, flush_l2) \
        if args.packed_steps > 0 else None

    # batch-wide loss over all ranks, for the record (not part of the timed path)
    n_rows = int((w.valid.reshape(-1, K) != 0).any(axis=1).sum())
    loss_all, _ = shard.global_mean_loss(float(loss.item()), n_rows, device=dev)

    if rank == 0:
        peak_tf, hbm_gbs, peak_src = load_peaks()
        sel, win = algorithmic_counts(w)
        fl_tgt = 2.0 * H * D * sel
        fl_win = 2.0 * H * D * win
        fl_step = fl_tgt + fl_win
        tgt_ms = statistics.mean(k_tgt)
        win_ms = statistics.mean(k_win)
        kl_ms = statistics.mean(k_kl)
        achieved = fl_tgt / (tgt_ms / 1e3) / 1e12
        # algorithmic bytes of the two HBM-bound kernels
        win_bytes = B * S * H * D * 2 + B * S * D * 2 + B * S * H * 4
        kl_bytes = B * S * K * (4 + 4 + 1 + 4)
        cand = candidate_blocks(w)
        sel_bytes = 4 * cand + B * S * K * (4 + 4 + 1)
        line = {
            "metric": METRIC,
            "value": value,
            "unit": UNIT,
            "n_gpus": world,
            "steps": nsteps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(w, world),
            "tc_peak_frac_step": fl_step / (ms_step / 1e3) / 1e12 / peak_tf,
            # for transparency: the flops of every slot and a full window per
            # token, as if nothing were masked (the headline counts only the
            # selected slots and the causal window keys)
            "padded_flops_per_step": 2.0 * H * D * B * S * (K + w.W),
            "tc_peak_frac_step_padded": 2.0 * H * D * B * S * (K + w.W) / (ms_step / 1e3) / 1e12 / peak_tf,
            "warm_l2": warm,
            "roofline": {
                "kernel": "distill_target (target_tc_kernel<64>)",
                "bound": "tensor",
                "achieved": achieved,
                "peak": peak_tf,
                "unit": "TFLOP/s",
                "frac": achieved / peak_tf,
                "peak_source": f"{peak_src} bf16 dense (burst)",
                "algorithmic": f"2*H*D flops per selected slot x {sel} selected slots = {fl_tgt:.4g} flops/launch",
                "traffic": traffic_record("target_tc.cu"),
            },
            "kernels_ms": {"window_lse": win_ms, "distill_target": tgt_ms, "distill_kl": kl_ms},
            "kernels_roofline": {
                "window_lse": {"bound": "hbm", "achieved_gbs": win_bytes / (win_ms / 1e3) / 1e9,
                               "peak_gbs": hbm_gbs, "frac": win_bytes / (win_ms / 1e3) / 1e9 / hbm_gbs,
                               "tflops": fl_win / (win_ms / 1e3) / 1e12,
                               "traffic": traffic_record("window_lse_tc.cu")},
                "distill_kl": {"bound": "hbm", "achieved_gbs": kl_bytes / (kl_ms / 1e3) / 1e9,
                               "peak_gbs": hbm_gbs, "frac": kl_bytes / (kl_ms / 1e3) / 1e9 / hbm_gbs},
            },
            "selection": {
                "kernel": "indexer_topk_kernel (sai_indexer_topk), not part of the step",
                "ms": sel_ms, "bound": "hbm", "achieved_gbs": sel_bytes / (sel_ms / 1e3) / 1e9,
                "peak_gbs": hbm_gbs, "frac": sel_bytes / (sel_ms / 1e3) / 1e9 / hbm_gbs,
                "algorithmic": f"4 B per candidate score read ({cand} candidates) + 9 B per slot written "
                               f"({B * S * K} slots) = {sel_bytes} B/launch",
                "launches": sel_steps, "input": "index scores N(0,1) over every block, seed per rank",
            },
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": args.e2e_steps,
                    "pipelining": "two device input buffers; each step's host->device copies run on a copy "
                                  "stream while the previous step computes; loss and dscores read back "
                                  "every step"},
            "fused_window": fused,
            "long": long_line,
            "packed": packed_line,
            "gpu_launches": 3 * nsteps * world,   # window, target, KL (one cooperative launch); every rank
            "clocks": clk,
            "loss": loss_all,
        }
        if fused is not None:
            fused["distill_target_window_frac"] = fused["distill_target_window_tflops"] / peak_tf
        for sl in (long_line, packed_line):
            if sl is not None:
                sl["distill_target_frac"] = sl["distill_target_tflops"] / peak_tf
                sl["step_frac"] = sl["step_tflops"] / peak_tf
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
