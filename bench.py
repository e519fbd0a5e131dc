#!/usr/bin/env python
"""Benchmark of one speculative-decoding step: target verification + P-EAGLE draft-batch
construction, through libpspec's C ABI, on the large-batch workload (B=1024 sequences,
K=7 drafts, vocabulary 201088, hidden 2880, bf16 logits).

A step = one verify call (rejection rule by default, --mode greedy for the greedy rule)
over the B*(K+1) target rows (and B*K draft rows), whose accepted counts and bonus
tokens feed one draft-batch construction call.  Inputs are resident in HBM and larger
than L2 (6.2 GB of logits per step), so every step streams them from DRAM.

Prints one JSON line (rank 0).  Under torchrun each rank runs its own replica of the
workload (the sequences are independent; no collective on the data path) and the
reported time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--mode rejection|greedy]
  python bench.py --impl reference ...   # the CPU oracle on the same workload
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verify+build step/s and achieved HBM GB/s (% of peak) at B=1024,K=7,V=201088"
UNIT = "step/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["pspec", "reference"], default="pspec")
    p.add_argument("--mode", choices=["rejection", "greedy"], default="rejection")
    p.add_argument("--path", choices=["auto", "sweep", "early"], default="auto",
                   help="verify path: automatic selection, full sweep or early exit")
    p.add_argument("--cluster", type=int, default=0, help="early-exit cluster size (0 auto)")
    p.add_argument("--fusion", choices=["auto", "always", "never"], default="auto",
                   help="verify + build in one launch (early-exit path): pspec_set_step_fusion")
    p.add_argument("--tail", type=int, default=0,
                   help="early exit: sequences for the 8-CTA tail launch (0 auto, -1 never)")
    p.add_argument("--e2e-steps", type=int, default=8)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the other workloads (c1, c64, greedy b1024, depth sweep) that a "
                        "one-GPU run adds to its JSON line")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample", type=int, default=512,
                   help="sequences of the workload the CPU oracle baseline verifies")
    p.add_argument("--workload", default="b1024", help="b1024 (default), c64 or c1")
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's number of sequences (profiling and scaling aid)")
    p.add_argument("--graph", action="store_true",
                   help="capture one step in a CUDA graph and time its replays")
    p.add_argument("--separate", action="store_true",
                   help="time verify and build as two calls even where one fused launch can do both")
    p.add_argument("--build-only", action="store_true",
                   help="time the draft-batch construction alone (profiling aid: no logits)")
    p.add_argument("--depth-sweep", action="store_true",
                   help="the depth sweep: B=256, V=128256, K in 1,3,5,7,8, draft noise 0.3,0.7,1.5 "
                        "(one JSON line with a point per (K, sigma))")
    p.add_argument("--depth-k", default="", help="comma-separated K values of the depth sweep (default all)")
    p.add_argument("--sample-only", choices=["sample", "argmax"], default=None,
                   help="time draft-token sampling alone over the workload's drafter rows")
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, or None when there is
    none or it was taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_per_launch_bytes:\s*([0-9.eE+]+)", txt)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", txt)
    if not m or not h or h.group(1) != src_hash:
        return None
    return float(m.group(1))


_SAMPLER = r"""
import sys, time
import pynvml as N
N.nvmlInit()
uuid, idx, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
try:
    h = N.nvmlDeviceGetHandleByUUID(uuid)
except Exception:
    h = N.nvmlDeviceGetHandleByIndex(idx if N.nvmlDeviceGetCount() > idx else 0)
print("max", N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM), flush=True)
while True:
    sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
    pw = N.nvmlDeviceGetPowerUsage(h) / 1000.0
    rs = N.nvmlDeviceGetCurrentClocksEventReasons(h)
    print(time.time(), sm, pw, rs, flush=True)
    time.sleep(period)
"""


class ClockSampler:
    """Samples SM clock, power and clock-event (throttle) reasons through NVML in a child
    process while the timed region runs, so the sampling never waits on this process."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, torch_device: int, period_s: float = 0.002):
        import subprocess
        import torch
        self.samples, self.max_sm, self.err = [], None, None
        try:
            uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:  # noqa: BLE001
            uuid = "unknown"
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        idx = torch_device
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if len(parts) > torch_device and parts[torch_device].isdigit():
            idx = int(parts[torch_device])
        self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, uuid, str(idx), str(period_s)],
                                     stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        first = self.proc.stdout.readline().split()      # waits until NVML is up
        if len(first) == 2 and first[0] == "max":
            self.max_sm = int(first[1])
        else:
            self.err = "nvml sampler failed: " + (self.proc.stderr.read()[-300:] if self.proc.poll() is not None else "?")

    def __enter__(self):
        self.t_start = time.time()
        self.t_timed_end = None
        return self

    def mark_timed_end(self):
        """End of the timed region; samples after it (up to the context's exit) come from
        the same steps run on, untimed, so that a timed region shorter than NVML's update
        interval still has clock readings beside it."""
        self.t_timed_end = time.time()

    def __exit__(self, *a):
        self.t_end = time.time()
        if self.t_timed_end is None:
            self.t_timed_end = self.t_end
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=30)
        for ln in out.splitlines():
            f = ln.split()
            if len(f) == 4 and self.t_start <= float(f[0]) <= self.t_end:
                self.samples.append((float(f[0]), int(f[1]), float(f[2]), int(f[3])))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_sm, "reasons": [], "source": "nvml",
                    "note": self.err or "no samples inside the timed region"}
        timed = [s for s in self.samples if s[0] <= self.t_timed_end]
        use = timed or self.samples
        sms = [s[1] for s in use]
        bits = 0
        for s in self.samples:
            bits |= s[3]
        reasons = sorted(v for k, v in self.REASONS.items() if bits & k)
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_sm,
                "sm_mhz_min": min(s[1] for s in self.samples),
                "power_w_max": round(max(s[2] for s in self.samples), 1),
                "reasons": reasons, "samples_timed_region": len(timed),
                "samples": len(self.samples),
                "source": "nvml, polled every ~2 ms" + (
                    "" if timed else "; sm_mhz from the same steps run on for 0.25 s right "
                    "after the timed region (none of its samples fell inside it)")}


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's elapsed time: every rank contributes its own device-timed ms."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job throughput: every rank ran `steps` steps of its own batch (weak scaling)
    within the slowest rank's elapsed time."""
    return world * steps / (elapsed_ms * 1e-3)


def set_tuning(ps, args):
    """The command line's tuning as the library's process-wide defaults."""
    ps.pspec_set_verify_path({"auto": 0, "sweep": 1, "early": 2}[args.path])
    ps.pspec_set_cluster_size(args.cluster)
    ps.pspec_set_tail_split(args.tail)
    ps.pspec_set_step_fusion({"auto": 0, "always": 1, "never": 2}[args.fusion])


# ----------------------------------------------------------------------------- workload
def make_workload(name, device, rank, batch=0):
    import torch
    from speculative_decoding_step_pspec_b200 import inputs as I
    w = dict(b1024=I.B1024, c64=I.C64, c1=I.C1)[name]
    w = I.scaled(w, seed=w.seed + 1000 * rank)      # each replica draws its own batch
    if batch:
        w = I.scaled(w, B=batch)
    target, draft = I.logits(w, device)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, device)
    binp = I.build_inputs(w, device, drafts=sampled)
    if torch.device(device).type == "cuda":
        torch.cuda.synchronize()
    return w, dict(target=target, draft=draft, sampled=sampled, greedy=greedy, u=u, build=binp)


def verify_rows(w, mode, accepted, early_exit):
    """Logit rows a verify pass must read: every row (full sweep), or with early exit only
    the rows of positions 0..a_i (target and draft rows for the rejection rule; the
    target's row K as well when all K drafts pass)."""
    import numpy as np
    if not early_exit:
        return w.B * ((2 * w.K + 1) if mode == "rejection" else (w.K + 1))
    a = np.asarray(accepted, np.int64)
    if mode == "rejection":
        return int(np.where(a < w.K, 2 * (a + 1), 2 * w.K + 1).sum())
    return int((a + 1).sum())


def algorithmic_bytes(w, mode, accepted, early_exit=False):
    """Bytes the method must move per step (verify + draft-batch build)."""
    import numpy as np
    s = 2 if str(w.dtype).endswith("bfloat16") else 4
    verify = verify_rows(w, mode, accepted, early_exit) * w.V * s
    c = np.asarray(accepted, np.int64) + 1                 # surviving verify rows (L = K+1)
    H, sh = w.H, s
    T_in = w.B * (w.K + 1)
    T_cap = -(-(T_in + w.B * (w.K - 1)) // w.capture_pad) * w.capture_pad
    hidden = int((c.sum() * H * sh) + ((c + w.K - 1).sum() * H * sh))
    live_rows = int((c + w.K - 1).sum())
    meta = T_cap * 21 + T_in * 8 + live_rows * 4 + (w.B + 1) * 8 + w.B * (16 + 4 * w.K)
    return verify, hidden + meta


# ----------------------------------------------------------------------------- pspec arm
def run_pspec(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import speculative_decoding_step_pspec_b200 as ps

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    set_tuning(ps, args)
    w, d = make_workload(args.workload, dev, rank, args.batch)
    rej = args.mode == "rejection"
    ws = ps.Workspace(w.B, w.K, w.V, rej, dev)
    vout = ps.api.verify_outputs(w.B, w.K, dev, False, rej)
    bi = d["build"]
    bout = ps.api.build_outputs(w.B, w.K, w.H, bi["T_cap"], bi["verify_hidden"].dtype, dev)
    drafts = d["sampled"] if rej else d["greedy"]

    def verify(stream=None):
        if rej:
            ps.verify_rejection(d["target"], d["draft"], drafts, d["u"], workspace=ws, out=vout)
        else:
            ps.verify_greedy(d["target"], drafts, workspace=ws, out=vout)

    def build():
        ps.build_draft_batch(K=w.K, block_size=w.block_size, mask_id=bi["mask_id"],
                             pad_id=bi["pad_id"], T_cap=bi["T_cap"], qsl_in=bi["qsl_in"],
                             verify_tokens=bi["verify_tokens"], verify_pos=bi["verify_pos"],
                             accepted_len=vout["accepted_len"], bonus=vout["bonus"],
                             block_table=bi["block_table"], verify_hidden=bi["verify_hidden"],
                             h_shared=bi["h_shared"], out=bout)

    def fused_step():
        ps.step(d["target"], drafts, bi, draft_logits=d["draft"] if rej else None,
                uniforms=d["u"] if rej else None, workspace=ws, out=vout, build_out=bout)

    # one call of the public step API: where a single launch verifies and builds, that is
    # the step that is timed; otherwise the two calls are timed apart
    fused_step()
    n_step = ps.pspec_last_launches()
    verify()
    n_verify = ps.pspec_last_launches()
    fused = (not args.separate) and n_step == n_verify
    for _ in range(max(3, args.warmup)):
        if fused:
            fused_step()
            lv, lb = n_step, 0
        else:
            verify()
            lv = ps.pspec_last_launches()
            build()
            lb = ps.pspec_last_launches()
        path = ps.pspec_last_verify_path()
        cluster = ps.pspec_last_cluster_size()
    launches_per_step = lv + lb
    torch.cuda.synchronize()
    graph = None
    if args.graph:                     # the step's launches, captured once and replayed
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph):
                if fused:
                    fused_step()
                else:
                    verify()
                    build()
        torch.cuda.current_stream().wait_stream(side)
        graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    for e in ev:          # torch only times events it has seen recorded; the library
        e[1].record()     # re-records the split event between the two verify launches
    torch.cuda.synchronize()

    def one_step():
        if graph is not None:
            graph.replay()
        elif fused:
            fused_step()
        else:
            verify()
            build()

    # inputs that L2 could hold across steps: flush before every step (outside its events)
    # and sum the per-step times instead of timing the loop as a whole
    in_bytes = sum(x.numel() * x.element_size() for x in (d["target"], d["draft"]) if x is not None)
    flush_buf = (torch.empty(256 << 20, dtype=torch.uint8, device=dev)
                 if in_bytes < (256 << 20) else None)
    def instrumented_step(e):
        """One step with events at its start, between the verify and the build and at its
        end (the library records e[1] between the sweep's two verify launches)."""
        e[0].record()
        if graph is not None:
            graph.replay()
            e[2].record()
            e[3].record()
        elif fused:
            fused_step()
            e[2].record()
            e[3].record()
        else:
            if rej:
                ps.pspec_set_split_event(e[1])
            verify()
            e[2].record()
            build()
            e[3].record()
            ps.pspec_set_split_event(None)

    # With inputs larger than L2 the K steps are timed as a whole with nothing between their
    # launches: an event recorded between the verify and the build holds the build back
    # until the verify has drained (it is a programmatic dependent that would otherwise be
    # placed while the verify's last clusters run), which costs a few microseconds a step.
    # The per-kernel times then come from up to 50 more steps with events between the launches.
    # With an L2 flush before every step, the steps carry their own events.
    instrument_timed = flush_buf is not None
    n_inst = K if instrument_timed else min(K, 50)
    with sampler:
        # two more untimed steps once the sampler runs, and no synchronisation before t0:
        # the GPU is still busy with them when t0 is reached, so the host has queued the
        # first timed step by then.  (After an idle GPU the first step's events would also
        # hold the host's argument marshalling, ~0.08 ms.)
        for _ in range(2):
            if flush_buf is not None:
                flush_l2(flush_buf)
            one_step()
        t0.record()
        for s in range(K):
            if flush_buf is not None:
                flush_l2(flush_buf)
            if instrument_timed:
                instrumented_step(ev[s])
            else:
                one_step()
        t1.record()
        torch.cuda.synchronize()
        sampler.mark_timed_end()
        if not instrument_timed:
            # right after the timed steps, at most 50 of them (a long run heats the part
            # towards its power cap, and later steps would not be the ones timed)
            one_step()                     # untimed: the GPU is busy when the first is queued
            for s in range(n_inst):
                instrumented_step(ev[s])
        b2b = None
        if not instrument_timed and graph is None and not fused and path == 2:
            # the early-exit verify alone, n_inst calls back to back with nothing recorded
            # between them: the dominant kernel's own duration, without the gap that an event
            # between two launches opens (the front end drains, then starts the next launch)
            b2b = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            b2b[0].record()
            for _ in range(n_inst):
                verify()
            b2b[1].record()
        # clock readings beside a short timed region: the same steps for 0.25 s more
        for _ in range(min(4000, int(math.ceil(250.0 / max(t0.elapsed_time(t1) / K, 1e-3))))):
            one_step()
        torch.cuda.synchronize()
    if not instrument_timed:
        ev = ev[:n_inst]
    if world > 1:
        dist.barrier()
    own_ms = (t0.elapsed_time(t1) if flush_buf is None
              else sum(e[0].elapsed_time(e[3]) for e in ev))
    elapsed_ms = max_over_ranks(own_ms, world, dev)

    verify_ms = [e[0].elapsed_time(e[2]) for e in ev]
    build_ms = [e[2].elapsed_time(e[3]) for e in ev]
    # library-recorded split event between the sweep's statistics and draw launches
    split = rej and not fused and graph is None and path == 1
    stats_ms = [e[0].elapsed_time(e[1]) for e in ev] if split else verify_ms
    draw_ms = [e[1].elapsed_time(e[2]) for e in ev] if split else None
    assert int(vout["err"].item()) == 0 and int(bout["err"].item()) == 0
    acc = vout["accepted_len"].cpu().numpy()
    early = path == 2                       # the path that reads rows only up to a_i
    vbytes, bbytes = algorithmic_bytes(w, args.mode, acc, early)
    full_vbytes, _ = algorithmic_bytes(w, args.mode, acc, False)
    hbm, peak_src = peaks()
    ms_step = elapsed_ms / K
    step_gbs = (vbytes + bbytes) / (ms_step * 1e-3) / 1e9
    if early:
        dom_kernel = "ee_kernel"
        src = ["speculative_decoding_step_pspec_b200/csrc/verify_early_exit.cu",
               "speculative_decoding_step_pspec_b200/csrc/verify_common.cuh",
               "speculative_decoding_step_pspec_b200/csrc/common.cuh"]
        if fused:
            src.append("speculative_decoding_step_pspec_b200/csrc/build_common.cuh")
    else:
        dom_kernel = "rej_stats_kernel" if rej else "greedy_sweep_kernel"
        src = ["speculative_decoding_step_pspec_b200/csrc/verify_rejection.cu" if rej else
               "speculative_decoding_step_pspec_b200/csrc/verify_greedy.cu",
               "speculative_decoding_step_pspec_b200/csrc/verify_common.cuh",
               "speculative_decoding_step_pspec_b200/csrc/common.cuh"]
    src_hash = kernel_source_hash(src)
    dom_ms = statistics.mean(stats_ms)
    dom_ms_events = dom_ms
    if b2b is not None:
        dom_ms = b2b[0].elapsed_time(b2b[1]) / n_inst
    whole = fused or graph is not None                     # one timed unit: the whole step
    dom_bytes = vbytes + bbytes if whole else vbytes       # a fused launch also builds
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    # both rules share the early-exit kernel: its profiles are per rule
    prof_key = dom_kernel + ("_greedy" if not rej and dom_kernel == "ee_kernel" else "")
    # a whole-step timing (fused launch, graph replay) is not one kernel's: no kernel traffic
    # (the profiles hold the named workloads' sizes: none for an overridden batch)
    traffic = None if (whole or args.batch) else profiled_traffic(prof_key, args.workload, src_hash)

    line = {
        "metric": METRIC, "value": round(aggregate_value(K, world, elapsed_ms), 3), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"{args.workload}{'' if not args.batch else ' (B overridden)'}: B={w.B}, K={w.K}, V={w.V}, H={w.H}, block_size="
                        f"{w.block_size}, bf16 logits, {args.mode} verify + P-EAGLE draft-batch build",
            "B": w.B, "K": w.K, "V": w.V, "H": w.H, "mode": args.mode,
            "verify_path": {1: "full sweep", 2: f"early exit ({cluster}-CTA cluster per sequence)"}[path],
            "step": ("one launch (verify + build fused)" if fused else "verify launches + build launch")
                    + (", CUDA graph replay" if graph is not None else ""),
            "l2": ("inputs larger than L2 (%.2f GB of logits per step); no flush; the K steps "
                   "timed as a whole, per-kernel times from min(K, 50) more steps with events "
                   "between the launches" % (vbytes / 1e9)
                   if flush_buf is None else
                   "256 MB buffer written then read before every step, outside the step's events; "
                   "elapsed time = sum of the per-step event times"),
            "parallelism": f"replicas x{world} (independent sequences, no collective)",
        },
        "achieved_gbs": round(step_gbs, 1),
        "pct_of_peak": round(100 * step_gbs / hbm, 2),
        "algorithmic_bytes_per_step": {"verify": int(vbytes), "build": int(bbytes),
                                       "verify_full_sweep": int(full_vbytes)},
        "kernels_ms": {
            dom_kernel + (" (verify + build, one launch)" if fused and lv == 1 else "")
            + (" (verify + build, two launches)" if fused and lv == 2 else "")
            + (" (two launches: the large-batch clusters, then wider ones for the last sequences)"
               if path == 2 and lv == 2 and not fused else "")
            + (" (CUDA graph replay of the step)" if graph is not None else ""): round(dom_ms, 5),
            **({"ee_kernel with events between the step's launches": round(dom_ms_events, 5)}
               if b2b is not None else {}),
            **({"rej_draw_kernel": round(statistics.mean(draw_ms), 5)} if draw_ms else {}),
            **({} if whole else {"build_kernel": round(statistics.mean(build_ms), 5)}),
        },
        **({"kernels_ms_timing": "ee_kernel: min(K, 50) verify calls back to back, nothing "
                                 "recorded between them; build_kernel: min(K, 50) steps with "
                                 "events between the launches"} if b2b is not None else {}),
        **({} if whole else {"build_gbs": round(bbytes / (statistics.mean(build_ms) * 1e-3) / 1e9, 1)}),
        "roofline": {
            "kernel": dom_kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic,
            "launches": lv,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback",
            "algorithmic_bytes_per_launch": int(dom_bytes),
        },
        "gpu_launches": K * launches_per_step,
        "launches_per_step": launches_per_step,
        "acceptance": {"mean_accepted": round(float(acc.mean()), 4),
                       # accepted drafts / drafts tested (a rejection ends a sequence's tests)
                       "rate": round(float(acc.sum()) / float(np.minimum(acc + 1, w.K).sum()), 4),
                       "histogram": np.bincount(acc, minlength=w.K + 1).tolist()},
        "clocks": sampler.summary(),
    }

    if not args.no_e2e:
        line["e2e"] = run_e2e(args, w, d, ps, dev, world)
    else:
        line["e2e"] = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args, w, d, acc)
    if world == 1 and not args.no_extra and not args.batch and args.workload == "b1024":
        line["other_workloads"] = extra_workloads(args, w, d, dev, hbm)
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- other workloads
def flush_l2(buf):
    """Evicts the step's data from L2: a buffer larger than L2 is written, then read back, so
    that L2 ends up holding clean lines of it and the timed launch does not pay for writing
    back the flush's own dirty lines."""
    buf.fill_(1)
    buf.max()


def time_steps(fn, n, flush=None):
    """Device time of each of n calls of fn (CUDA events on the current stream, one pair per
    call); with `flush`, a buffer larger than L2 is written and read before every call,
    outside the timed pair.  Without it (inputs larger than L2) the n calls are timed as a
    whole, nothing recorded between them, and each gets the mean."""
    import torch
    if flush is None:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b) / n] * n
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(n)]
    for a, b in pairs:
        if flush is not None:
            flush_l2(flush)
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in pairs]


def step_summary(w, mode, ms_list, launches, path, acc, hbm, graph_ms=None):
    """One workload's numbers: step time, algorithmic GB/s and fraction of the peak, launches
    per step and the accepted-length histogram."""
    import numpy as np
    early = path == 2
    vbytes, bbytes = algorithmic_bytes(w, mode, acc, early)
    ms = statistics.median(ms_list)
    gbs = (vbytes + bbytes) / (ms * 1e-3) / 1e9
    out = {"workload": f"{w.name}: B={w.B}, K={w.K}, V={w.V}, H={w.H}, bf16, {mode}",
           "ms_per_step": round(ms, 5), "ms_mean": round(statistics.mean(ms_list), 5),
           "step_per_s": round(1e3 / ms, 1), "achieved_gbs": round(gbs, 1),
           "frac_of_peak": round(gbs / hbm, 4), "algorithmic_bytes": int(vbytes + bbytes),
           "launches_per_step": launches,
           "verify_path": {1: "full sweep", 2: "early exit"}[path],
           "acceptance_rate": round(float(acc.sum()) / float(np.minimum(acc + 1, w.K).sum()), 4),
           "histogram": np.bincount(acc, minlength=w.K + 1).tolist()}
    if graph_ms is not None:
        g = statistics.median(graph_ms)
        out["graph_replay_ms_per_step"] = round(g, 5)
        out["graph_replay_step_per_s"] = round(1e3 / g, 1)
    return out


def measure_workload(ps, w, inputs, mode, dev, hbm, n, flush, graph=True):
    """Eager steps through the public step API (and, with `graph`, replays of one step
    captured in a CUDA graph) on resident inputs, timed per step."""
    import torch
    rej = mode == "rejection"
    bi = inputs["build"]
    drafts = inputs["sampled"] if rej else inputs["greedy"]
    ws = ps.Workspace(w.B, w.K, w.V, rej, dev)
    vout = ps.api.verify_outputs(w.B, w.K, dev, False, rej)
    bout = ps.api.build_outputs(w.B, w.K, w.H, bi["T_cap"], bi["verify_hidden"].dtype, dev)

    def step():
        ps.step(inputs["target"], drafts, bi, draft_logits=inputs["draft"] if rej else None,
                uniforms=inputs["u"] if rej else None, workspace=ws, out=vout, build_out=bout)
    for _ in range(3):
        step()
    launches, path = ps.pspec_last_launches(), ps.pspec_last_verify_path()
    ms = time_steps(step, n, flush)
    # the same step with its argument structs filled once (what a C caller or a decode loop
    # with fixed buffers pays per step: the launches alone)
    call, _, _ = ps.api.prepare_step(inputs["target"], drafts, bi,
                                     draft_logits=inputs["draft"] if rej else None,
                                     uniforms=inputs["u"] if rej else None, workspace=ws,
                                     out=vout, build_out=bout)
    stream = torch.cuda.current_stream().cuda_stream
    call(stream)
    p_ms = time_steps(lambda: call(stream), n, flush)
    g_ms = None
    if graph:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g):
                step()
        torch.cuda.current_stream().wait_stream(side)
        g.replay()
        torch.cuda.synchronize()
        g_ms = time_steps(g.replay, n, flush)
        del g
    assert int(vout["err"].item()) == 0 and int(bout["err"].item()) == 0
    acc = vout["accepted_len"].cpu().numpy()
    r = step_summary(w, mode, ms, launches, path, acc, hbm, g_ms)
    r["prepared_call_ms_per_step"] = round(statistics.median(p_ms), 5)
    return r


def extra_workloads(args, w_head, d_head, dev, hbm):
    """The other configurations, measured after the headline in the same run: the greedy
    rule on the large batch, the c=1 and c=64 shapes under both rules (eager and as CUDA
    graph replays, L2 flushed before every step), the c=1 recipe's per-token acceptance
    over 256 independent sequences, and the depth sweep (B=256, V=128256, K in 1,3,5,7,8,
    draft noise 0.3, 0.7, 1.5; L2 flushed before every step)."""
    import numpy as np
    import torch

    import speculative_decoding_step_pspec_b200 as ps
    from speculative_decoding_step_pspec_b200 import inputs as I
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out["b1024_greedy"] = measure_workload(ps, w_head, d_head, "greedy", dev, hbm, 20, None,
                                           graph=False)
    out["b1024_greedy"]["l2"] = "inputs larger than L2; no flush"
    for name in ("c1", "c64"):
        w, d = make_workload(name, dev, 0)
        for mode in ("rejection", "greedy"):
            r = measure_workload(ps, w, d, mode, dev, hbm, 50, flush)
            r["l2"] = "256 MB buffer written then read before every step (outside the timed events)"
            out[f"{name}_{mode}"] = r
        del d
    # the c=1 recipe's acceptance needs more than one sequence: 256 independent draws
    wa = I.scaled(I.C1, B=256, seed=I.C1.seed + 77)
    t, q = I.logits(wa, dev)
    sampled, _ = I.draft_tokens(wa, q)
    u = I.uniforms(wa, dev)
    r = ps.verify_rejection(t, q, sampled, u)
    acc = r["accepted_len"].cpu().numpy()
    out["c1_acceptance"] = {
        "sequences": wa.B, "rule": "rejection",
        "per_token_rate": round(float(acc.sum()) / float(np.minimum(acc + 1, wa.K).sum()), 4),
        "mean_accepted": round(float(acc.mean()), 3),
        "histogram": np.bincount(acc, minlength=wa.K + 1).tolist(),
        "stated_target": "roughly 0.65-0.75 per-token acceptance"}
    del t, q, sampled, u, r
    pts = []
    for K in I.DEPTH_K:
        for sigma in I.DEPTH_SIGMA:
            wd = I.depth(K, sigma)
            target, draft = I.logits(wd, dev)
            sampled, greedy = I.draft_tokens(wd, draft)
            dd = dict(target=target, draft=draft, sampled=sampled, greedy=greedy,
                      u=I.uniforms(wd, dev), build=I.build_inputs(wd, dev, drafts=sampled))
            p = measure_workload(ps, wd, dd, "rejection", dev, hbm, 20, flush, graph=False)
            p.update({"K": K, "sigma": sigma})
            pts.append(p)
            del dd, target, draft, sampled, greedy
            torch.cuda.empty_cache()
    out["depth_sweep"] = {"l2": "256 MB buffer written then read before every step", "points": pts}
    return out


def run_e2e(args, w, d, ps, dev, world):
    """The same step through the public API from pinned HOST buffers: every step copies its
    inputs host->device, runs verify + build, and reads the results back."""
    import torch
    import torch.distributed as dist
    rej = args.mode == "rejection"
    bi = d["build"]
    names = ["target", "draft", "u"] if rej else ["target"]
    host = {k: torch.empty_like(d[k], device="cpu", pin_memory=True) for k in names}
    drafts_dev = d["sampled"] if rej else d["greedy"]
    host["drafts"] = torch.empty_like(drafts_dev, device="cpu", pin_memory=True)
    bnames = ["qsl_in", "verify_tokens", "verify_pos", "block_table", "verify_hidden", "h_shared"]
    for k in bnames:
        host["b_" + k] = torch.empty_like(bi[k], device="cpu", pin_memory=True)
    for k in names:
        host[k].copy_(d[k])
    host["drafts"].copy_(drafts_dev)
    for k in bnames:
        host["b_" + k].copy_(bi[k])
    dv = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    ws = ps.Workspace(w.B, w.K, w.V, rej, dev)
    vout = ps.api.verify_outputs(w.B, w.K, dev, False, rej)
    bout = ps.api.build_outputs(w.B, w.K, w.H, bi["T_cap"], bi["verify_hidden"].dtype, dev)
    res_names = ["out_tokens", "accepted_len", "bonus"]
    bres_names = ["draft_tokens", "draft_pos", "slot_mapping", "row_kind", "hidden_src",
                  "qsl_out", "seq_lens_out", "sample_idx"]
    hres = {k: torch.empty_like(vout[k], device="cpu", pin_memory=True) for k in res_names}
    hres.update({"b_" + k: torch.empty_like(bout[k], device="cpu", pin_memory=True) for k in bres_names})
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in hres.values())

    def step():
        for k, t in host.items():
            dv[k].copy_(t, non_blocking=True)
        binp = dict(K=w.K, block_size=w.block_size, mask_id=bi["mask_id"], pad_id=bi["pad_id"],
                    T_cap=bi["T_cap"], qsl_in=dv["b_qsl_in"], verify_tokens=dv["b_verify_tokens"],
                    verify_pos=dv["b_verify_pos"], block_table=dv["b_block_table"],
                    verify_hidden=dv["b_verify_hidden"], h_shared=dv["b_h_shared"])
        ps.step(dv["target"], dv["drafts"], binp, draft_logits=dv["draft"] if rej else None,
                uniforms=dv["u"] if rej else None, workspace=ws, out=vout, build_out=bout)
        for k in res_names:
            hres[k].copy_(vout[k], non_blocking=True)
        for k in bres_names:
            hres["b_" + k].copy_(bout[k], non_blocking=True)

    step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    n = max(1, args.e2e_steps)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    del host, dv
    return {"value": round(aggregate_value(n, world, ms), 3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": n, "ms_per_step": round(ms / n, 3),
            "path": "pinned host buffers -> cudaMemcpyAsync -> C-ABI step (verify + build) -> results to host"}


def _oracle_inputs(d, seqs):
    import numpy as np
    import torch

    def logits(x):
        x = x[seqs]
        return x.view(torch.int16).cpu().numpy().view(np.uint16) if x.dtype == torch.bfloat16 else x.float().cpu().numpy()
    return (logits(d["target"]), logits(d["draft"]), d["sampled"][seqs].cpu().numpy(),
            d["u"][seqs].cpu().numpy())


def _oracle_build_args(w, d, acc, bonus):
    import torch
    bi = d["build"]
    vh = bi["verify_hidden"]
    vh = vh.view(torch.int16) if vh.dtype == torch.bfloat16 else vh
    hs = bi["h_shared"]
    hs = hs.view(torch.int16) if hs.dtype == torch.bfloat16 else hs
    return dict(K=w.K, block_size=w.block_size, mask_id=bi["mask_id"], pad_id=bi["pad_id"],
                T_cap=bi["T_cap"], qsl_in=bi["qsl_in"].cpu().numpy(),
                verify_tokens=bi["verify_tokens"].cpu().numpy(),
                verify_pos=bi["verify_pos"].cpu().numpy(), accepted_len=acc, bonus=bonus,
                block_table=bi["block_table"].cpu().numpy(), verify_hidden=vh.cpu().numpy(),
                h_shared=hs.cpu().numpy())


def cpu_baseline(args, w, d, acc):
    """The oracle as it stands, on the host cores, over a bounded sample of this workload:
    rejection (or greedy) verify of `cpu_sample` sequences, scaled to the whole batch, plus
    one full draft-batch construction."""
    import numpy as np
    import torch

    import oracle
    S = min(args.cpu_sample, w.B)
    seqs = torch.arange(S, device=d["target"].device)
    t, q, dr, u = _oracle_inputs(d, seqs)
    threads = max(1, min(os.cpu_count() or 1, S))
    bargs = _oracle_build_args(w, d, acc.astype(np.int32), np.zeros(w.B, np.int32))
    t0 = time.perf_counter()
    if args.mode == "rejection":
        oracle.verify_rejection(t, q, dr, u, threads=threads)
    else:
        oracle.verify_greedy(t, d["greedy"][seqs].cpu().numpy(), threads=threads)
    t1 = time.perf_counter()
    oracle.build_draft_batch(**bargs)
    t2 = time.perf_counter()
    step_s = (t1 - t0) * (w.B / S) + (t2 - t1)
    return {"value": round(1.0 / step_s, 5), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{args.mode} verify of {S} of {w.B} sequences (x{w.B / S:.2f}) + one "
                      f"full draft-batch build; {t1 - t0:.2f} s + {t2 - t1:.2f} s wall, "
                      f"{threads} threads"}


def run_build_only(args, local_rank):
    """The draft-batch construction alone on the workload's shapes (accepted counts drawn
    by the input generator): a profiling aid that holds only the build's buffers."""
    import torch

    import speculative_decoding_step_pspec_b200 as ps
    from speculative_decoding_step_pspec_b200 import inputs as I
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = dict(b1024=I.B1024, c64=I.C64, c1=I.C1)[args.workload]
    bi = I.build_inputs(w, dev)
    out = ps.api.build_outputs(w.B, w.K, w.H, bi["T_cap"], bi["verify_hidden"].dtype, dev)

    def build():
        ps.build_draft_batch(K=w.K, block_size=w.block_size, mask_id=bi["mask_id"],
                             pad_id=bi["pad_id"], T_cap=bi["T_cap"], qsl_in=bi["qsl_in"],
                             verify_tokens=bi["verify_tokens"], verify_pos=bi["verify_pos"],
                             accepted_len=bi["accepted_len"], bonus=bi["bonus"],
                             block_table=bi["block_table"], verify_hidden=bi["verify_hidden"],
                             h_shared=bi["h_shared"], out=out)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2: evict between steps
    for _ in range(max(3, args.warmup)):
        build()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush_l2(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        build()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    _, bbytes = algorithmic_bytes(w, "greedy", bi["accepted_len"].cpu().numpy())
    ms = statistics.median(times)
    hbm, _ = peaks()
    print(json.dumps({"metric": "draft-batch build alone (L2 flushed between launches)",
                      "workload": args.workload, "ms_median": round(ms, 5),
                      "ms_p10": round(sorted(times)[len(times) // 10], 5),
                      "algorithmic_bytes": int(bbytes), "gbs": round(bbytes / (ms * 1e-3) / 1e9, 1),
                      "frac_of_peak": round(bbytes / (ms * 1e-3) / 1e9 / hbm, 4),
                      "err": int(out["err"].item())}), flush=True)


def run_sample_only(args, local_rank):
    """Draft-token sampling alone over the workload's B*K drafter rows (the step after the
    drafter forward): inverse-CDF draws with seeded uniforms, or the argmax.  The rows are
    larger than L2 at the large-batch size; smaller workloads flush L2 between launches."""
    import torch

    import speculative_decoding_step_pspec_b200 as ps
    from speculative_decoding_step_pspec_b200 import inputs as I
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = dict(b1024=I.B1024, c64=I.C64, c1=I.C1)[args.workload]
    if args.batch:
        w = I.scaled(w, B=args.batch)
    g = torch.Generator(device=dev).manual_seed(w.seed)
    draft = torch.empty((w.B, w.K, w.V), dtype=w.dtype, device=dev)
    for b0 in range(0, w.B, 64):                   # drafter rows N(0, sigma_t), chunked
        b1 = min(w.B, b0 + 64)
        draft[b0:b1] = (torch.randn((b1 - b0, w.K, w.V), generator=g, device=dev)
                        * w.sigma_t).to(w.dtype)
    u = I.uniforms(w, dev)[:, :w.K].contiguous() if args.sample_only == "sample" else None
    ws = torch.zeros(ps._binding.pspec_sample_workspace_bytes(w.B, w.K, w.V), dtype=torch.uint8,
                     device=dev)
    out = ps.sample_drafts(draft, u, workspace=ws)
    nbytes = draft.numel() * draft.element_size()
    flush = None if nbytes > (256 << 20) else torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        ps.sample_drafts(draft, u, workspace=ws, out=out)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    with sampler:
        for a, b in ev:
            if flush is not None:
                flush_l2(flush)
            a.record()
            ps.sample_drafts(draft, u, workspace=ws, out=out)
            b.record()
        torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in ev]
    assert int(out["err"].item()) == 0
    ms = statistics.mean(times)
    hbm, peak_src = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    src = ["speculative_decoding_step_pspec_b200/csrc/sample_drafts.cu",
           "speculative_decoding_step_pspec_b200/csrc/verify_common.cuh",
           "speculative_decoding_step_pspec_b200/csrc/common.cuh"]
    print(json.dumps({
        "metric": "draft-token sampling alone: rows/s and achieved HBM GB/s",
        "workload": f"{args.workload}: B={w.B}, K={w.K}, V={w.V}, {str(w.dtype).split('.')[-1]} drafter rows",
        "mode": args.sample_only, "rows": w.B * w.K, "steps": args.steps,
        "ms_mean": round(ms, 5), "ms_median": round(statistics.median(times), 5),
        "rows_per_s": round(w.B * w.K / (ms * 1e-3), 1),
        "l2": "rows larger than L2; no flush" if flush is None else "256 MB buffer written then read between launches",
        "roofline": {"kernel": "sample_kernel", "bound": "hbm", "achieved": round(gbs, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                     "traffic": profiled_traffic("sample_kernel", args.workload,
                                                 kernel_source_hash(src)),
                     "peak_source": peak_src, "algorithmic_bytes_per_launch": int(nbytes)},
        "gpu_launches": args.steps, "clocks": sampler.summary()}), flush=True)


def run_depth_sweep(args, local_rank):
    """Step time, achieved GB/s and the accepted-length histogram per (K, sigma) of the
    depth-sweep workload (B=256, V=128256, H=4096), rejection rule, automatic path."""
    import numpy as np
    import torch

    import speculative_decoding_step_pspec_b200 as ps
    from speculative_decoding_step_pspec_b200 import inputs as I
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    set_tuning(ps, args)
    hbm, _ = peaks()
    points = []
    ks = [int(x) for x in args.depth_k.split(",")] if args.depth_k else I.DEPTH_K
    for K in ks:
        for sigma in I.DEPTH_SIGMA:
            w = I.depth(K, sigma)
            target, draft = I.logits(w, dev)
            sampled, _ = I.draft_tokens(w, draft)
            u = I.uniforms(w, dev)
            bi = I.build_inputs(w, dev, drafts=sampled)
            ws = ps.Workspace(w.B, w.K, w.V, True, dev)
            vout = ps.api.verify_outputs(w.B, w.K, dev, False, True)
            bout = ps.api.build_outputs(w.B, w.K, w.H, bi["T_cap"], bi["verify_hidden"].dtype, dev)

            def step():
                ps.step(target, sampled, bi, draft_logits=draft, uniforms=u, workspace=ws,
                        out=vout, build_out=bout)
            for _ in range(max(3, args.warmup)):
                step()
            launches = ps.pspec_last_launches()
            path = ps.pspec_last_verify_path()
            torch.cuda.synchronize()
            n = max(20, args.steps // 5)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(n):
                step()
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / n
            assert int(vout["err"].item()) == 0 and int(bout["err"].item()) == 0
            acc = vout["accepted_len"].cpu().numpy()
            early = path == 2
            vbytes, bbytes = algorithmic_bytes(w, "rejection", acc, early)
            points.append({"K": K, "sigma": sigma, "ms_per_step": round(ms, 4),
                           "step_per_s": round(1e3 / ms, 1),
                           "achieved_gbs": round((vbytes + bbytes) / (ms * 1e-3) / 1e9, 1),
                           "frac_of_peak": round((vbytes + bbytes) / (ms * 1e-3) / 1e9 / hbm, 4),
                           "algorithmic_bytes": int(vbytes + bbytes), "launches": launches,
                           "acceptance_rate": round(float(acc.sum()) / float(np.minimum(acc + 1, K).sum()), 4),
                           "histogram": np.bincount(acc, minlength=K + 1).tolist()})
            del target, draft, bi, ws, vout, bout
            torch.cuda.empty_cache()
    print(json.dumps({"metric": "depth sweep: step time, GB/s and accepted-length histogram per (K, sigma)",
                      "workload": "depth: B=256, V=128256, H=4096, bf16, rejection rule, automatic path",
                      "peak_gbs": hbm, "points": points}), flush=True)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank):
    """The CPU oracle as the reference arm: each step verifies a rotating bounded sample of
    the workload's sequences on the host cores and builds the full draft batch; the step
    time is scaled to the whole batch."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    w, d = make_workload(args.workload, dev, 0)
    threads = max(1, os.cpu_count() or 1)
    acc = np.full(w.B, w.K // 2, np.int32)
    bargs = _oracle_build_args(w, d, acc, np.zeros(w.B, np.int32))
    # size the per-step sample so that warmup + steps take about two minutes
    probe = torch.arange(1, device=dev)
    t, q, dr, u = _oracle_inputs(d, probe)
    a = time.perf_counter()
    oracle.verify_rejection(t, q, dr, u) if args.mode == "rejection" else oracle.verify_greedy(t, dr)
    per_seq = time.perf_counter() - a
    a = time.perf_counter()
    oracle.build_draft_batch(**bargs)
    build_s = time.perf_counter() - a
    budget = 120.0 / max(1, args.steps + args.warmup)
    S = int(max(1, min(w.B, threads * max(0.0, budget - build_s) / max(per_seq, 1e-6))))
    times = []
    for s in range(args.warmup + args.steps):
        seqs = (torch.arange(S, device=dev) + s * S) % w.B
        t, q, dr, u = _oracle_inputs(d, seqs)
        a = time.perf_counter()
        if args.mode == "rejection":
            oracle.verify_rejection(t, q, dr, u, threads=min(threads, S))
        else:
            oracle.verify_greedy(t, dr, threads=min(threads, S))
        b = time.perf_counter()
        oracle.build_draft_batch(**bargs)
        c = time.perf_counter()
        if s >= args.warmup:
            times.append((b - a) * (w.B / S) + (c - b))
    step_s = statistics.mean(times)
    value = round(1.0 / step_s, 5)
    cores = min(threads, S)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{args.workload}: B={w.B}, K={w.K}, V={w.V}, H={w.H}, {args.mode} "
                               f"verify + P-EAGLE draft-batch build (CPU oracle)",
                   "B": w.B, "K": w.K, "V": w.V, "H": w.H, "mode": args.mode},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {args.mode} verify of {S} of {w.B} sequences "
                                   f"(x{w.B / S:.1f}) + one full draft-batch build"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.build_only:
            run_build_only(args, local_rank)
        elif args.sample_only:
            run_sample_only(args, local_rank)
        elif args.depth_sweep:
            run_depth_sweep(args, local_rank)
        else:
            run_pspec(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
