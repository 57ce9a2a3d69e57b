#!/usr/bin/env python
"""Benchmark of the Tail-Replay hot path on B200.

Workload (one step): one hit on one group of 3 Gated DeltaNet layers after a full-attention
layer; d_model 2048, 16 heads of d_k = d_v = 128; cached FA output hiddens h ~ N(0,1) (bf16),
weights N(0, 0.02) (bf16); matched prefix m = 32768, r = 5% -> the last k = 1639 hiddens are
replayed from a zero state through the 3 layers (RMSNorm -> projection + gates + key norm ->
chunked scan -> output projection + residual; the last layer's readout is skipped), and the
rebuilt states S_hat_m are compared with the full-prefill S_m (state error, fp64).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  N > 1 runs under torchrun: every rank replays its own
independent request (no collective on the data path; weak scaling); the time is the max over
ranks.  --impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "replayed tokens/s & GDN scan state-updates/s on 1 B200; % of HBM/TC roofline"
D, H, DH, L, M_PREFIX, R_NUM, R_DEN = 2048, 16, 128, 3, 32768, 5, 100
D_FF = 5632   # FFN width of the FFN cell (2.75 d_model, a multiple of 128)
WORKLOAD = ("one group = 1 FA + 3 LA (Gated DeltaNet) layers, d_model 2048, 16 heads "
            "d_k=d_v=128, bf16 cached h ~N(0,1), weights N(0,0.02), alpha=exp(-softplus), "
            "m=32768, r=0.05 (k=1639), batch 1")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sample-tokens", type=int, default=205,
                   help="reference arm: tail tokens per timed step (a bounded sample)")
    p.add_argument("--profile", choices=["scan", "group"], default=None,
                   help="run only one workload a few times (for ncu captures), no JSON line")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workload configurations (1, 3, 4 and the sweep)")
    return p.parse_args()


def profile_run(args):
    """A short run of one workload for profilers: the scan cell or the group replay step."""
    import torch
    import synth
    import linear_attention_state_zero_b200 as tr
    dev = torch.device("cuda", 0)
    if args.profile == "scan":
        k5 = tr.tail_len(32768, 10, 100)
        case = synth.scan_case([k5], 32, 128, 128, torch.bfloat16, 0.97, 1.0,
                               seed=synth.SEED_BASE + 4)
        t = [x.to(dev) for x in (case.q, case.k, case.v, case.log_alpha, case.beta)]
        for _ in range(args.warmup + args.steps):
            tr.gdn_scan(*t, case.cu_seqlens)
    else:
        k = tr.tail_len(M_PREFIX, R_NUM, R_DEN)
        seed = synth.SEED_BASE + 1
        h = synth.hidden_prefix(M_PREFIX, D, seed)[M_PREFIX - k:].contiguous().to(dev)
        layers = [tr.Layer(l.W_in.to(dev), l.W_o.to(dev))
                  for l in synth.la_layers(L, D, H, DH, DH, seed=seed)]
        rep = tr.GroupReplay(h, [0, k], layers, H, DH, DH, skip_last_output=True)
        S_ref = torch.ones_like(rep.S_hat).reshape(-1, DH, DH)
        for _ in range(args.warmup + args.steps):  # one step: the replay and the state error
            rep.run()
            tr.state_error(S_ref, rep.S_hat.reshape(-1, DH, DH), per_mat=False)
    torch.cuda.synchronize()
    tr.check()
    print("profile run done:", args.profile)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


# ------------------------------------------------------------ multi-rank host logic
# Every rank replays its own independent request (weak scaling): nothing but the
# timing crosses ranks.
def rank_seed(rank):
    """Seed of the request a rank replays: distinct per rank, the same on every run."""
    import synth
    return synth.SEED_BASE + 1 + 1000 * rank


def max_over_ranks(x, world, device):
    """Largest x over all ranks (the slowest rank sets the job time)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms_per_step):
    """Units processed by all ranks per second, given the max-over-ranks step time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


# ------------------------------------------------------------------ flop/byte model
def flops_inproj(T, skip_q):
    n_in = 2 * H * DH + H * DH + 2 * H - (H * DH if skip_q else 0)
    return 2.0 * T * D * n_in


def flops_outproj(T):
    return 2.0 * T * (H * DH) * D


def scan_flops_per_token_head(C=64, dk=DH, dv=DH):
    # chunked form: 6 C dk + 4 C dv + C^2/3 + 6 dk dv per token-head
    return 6 * C * dk + 4 * C * dv + C * C / 3.0 + 6 * dk * dv


def group_model(k):
    """Algorithmic FLOPs and bytes of one step (last layer's readout skipped)."""
    F = 0.0
    Bw = 0.0
    for l in range(L):
        last = l == L - 1
        F += flops_inproj(k, last)
        n_in = 3 * H * DH + 2 * H - (H * DH if last else 0)
        Bw += n_in * D * 2
        if not last:
            F += flops_outproj(k)
            Bw += D * H * DH * 2
    F += L * k * H * scan_flops_per_token_head()
    B = Bw + k * D * 2 + L * H * DH * DH * 4
    return F, B


KERNEL_DESC = {
    "rmsnorm": "RMSNorm (bytes: x in, x_hat out)",
    "in_proj": "in-proj tcgen05 GEMM + gate/key-norm epilogue (flops)",
    "scan_prep": "chunked scan, per-(chunk, head) prep (bytes: q, k, v, log alpha, beta in)",
    "scan_chain": "chunked scan, chunk-to-chunk state chain (bytes: final state out)",
    "scan_out": "chunked scan, readout (bytes: o out)",
    "out_proj": "out-proj tcgen05 GEMM + residual (flops)",
    "scan_recurrent": "token-recurrent scan (bytes: q, k, v, gates in, o out)",
    "scan_fused": "chunked scan, prep and chain in one launch (bytes: q, k, v, gates in, o and "
                  "final state out)",
    "scan_plan": "chunked scan plan (chunk offsets, longest-first order; bytes: none counted)",
}


def kernel_work(name, layer, k):
    """Algorithmic work of one launch: ("tensor", FLOPs) or ("hbm", bytes)."""
    last = layer == L - 1
    if name == "rmsnorm":
        return "hbm", k * D * ((2 if layer == 0 else 4) + 2)
    if name == "in_proj":
        return "tensor", flops_inproj(k, last)
    if name == "scan_prep":
        return "hbm", k * H * ((2 if last else 3) * DH * 2 + 8)
    if name == "scan_chain":
        # the final state out, plus o when the readout is fused into the chain
        return "hbm", H * DH * DH * 4 + (0 if last or "scan_out" in KERNELS_SEEN else k * H * DH * 2)
    if name == "scan_out":
        return "hbm", k * H * DH * 2
    if name == "out_proj":
        return "tensor", flops_outproj(k)
    if name == "scan_fused":
        return "hbm", k * H * ((2 if last else 3) * DH * 2 + 8 + (0 if last else DH * 2)) + \
            H * DH * DH * 4
    if name == "scan_plan":
        return "hbm", 0.0
    if name == "scan_recurrent":
        return "hbm", k * H * ((2 if last else 3) * DH * 2 + 8 + (0 if last else DH * 2))
    raise KeyError(name)


KERNELS_SEEN = set()


def kernel_rooflines(names, avg_ms, k, peaks):
    """Per kernel (summed over the layers): achieved algorithmic rate / measured peak."""
    out = {}
    layer = -1
    work, ms, launches, bound = {}, {}, {}, {}
    KERNELS_SEEN.clear()
    KERNELS_SEEN.update(names)
    for n, t in zip(names, avg_ms):
        # a layer starts at its input projection; an RMSNorm launch (the first layer's; the
        # later layers' is folded into the residual GEMM before them) precedes it
        if n == "in_proj":
            layer += 1
        b, w = kernel_work(n, layer + 1 if n == "rmsnorm" else layer, k)
        bound[n] = b
        work[n] = work.get(n, 0.0) + w
        ms[n] = ms.get(n, 0.0) + t
        launches[n] = launches.get(n, 0) + 1
    for n in work:
        if bound[n] == "tensor":
            ach, peak, unit = work[n] / (ms[n] * 1e-3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        else:
            ach, peak, unit = work[n] / (ms[n] * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
        out[n] = {"bound": bound[n], "achieved": ach, "peak": peak, "unit": unit,
                  "frac": ach / peak, "launches_per_step": launches[n],
                  "us_per_step": ms[n] * 1e3,
                  ("flops" if bound[n] == "tensor" else "bytes") + "_per_launch":
                      work[n] / launches[n],
                  "what": KERNEL_DESC[n]}
    return out


def load_traffic():
    """DRAM bytes per launch (read + write) from the committed ncu summary, per kernel; a
    kernel whose source changed since the capture gets None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic_group_step.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return {}
    out = {}
    for n, r in rec.get("kernels", {}).items():
        h = hashlib.sha256()
        try:
            for src in r["sources"]:
                with open(os.path.join(ROOT, src), "rb") as f:
                    h.update(f.read())
        except OSError:
            continue
        out[n] = r["bytes_per_launch"] if h.hexdigest() == r["sha256"] else None
    return out


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.15)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        text = self.tmp.read()
        os.unlink(self.tmp.name)
        return self.summarize(text)

    @staticmethod
    def summarize(text):
        """Median SM clock, the largest max clock and every throttle reason seen active, from
        `nvidia-smi --query-gpu=FIELDS --format=csv,noheader,nounits` lines."""
        rows = [r for r in csv.reader(io.StringIO(text)) if len(r) >= 9]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------- the other configurations
SWEEP_M = [4096, 8192, 16384, 32768, 65536, 131072]
SWEEP_R = [1, 2, 5, 10, 20, 100]   # percent


def _timer(stream, flush):
    """fn, n -> mean ms of n device-timed calls, L2 flushed before each (outside the timing)."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn, n):
        ts = []
        for _ in range(n):
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return sum(ts) / len(ts)
    return timed


def _group_flops_bytes(T, Dm, Hh, d, n_layers, n_groups, d_in_bytes=2):
    """Algorithmic FLOPs and bytes of replaying n_groups groups of n_layers LA layers over T
    tail tokens (last layer's readout skipped): projections + chunked scan; weights once per
    group, the h tails in, the states out."""
    F = Bw = 0.0
    for l in range(n_layers):
        last = l == n_layers - 1
        n_in = 3 * Hh * d + 2 * Hh - (Hh * d if last else 0)
        F += 2.0 * T * Dm * n_in + (0 if last else 2.0 * T * Hh * d * Dm)
        Bw += n_in * Dm * 2 + (0 if last else Dm * Hh * d * 2)
    F += n_layers * T * Hh * scan_flops_per_token_head(dk=d, dv=d)
    F *= n_groups
    B = n_groups * (Bw + T * Dm * d_in_bytes) + 0.0
    return F, B


def config_cells(dev, peaks, stream, flush, n_rep, cpu):
    """Configurations 1, 3, 4 and the scan sweep: throughput, roofline fraction, state errors
    and (with cpu) the oracle's rate on a bounded sample of each."""
    import torch
    import synth
    import linear_attention_state_zero_b200 as tr
    timed = _timer(stream, flush)
    out = {}

    # ---- 1: single head, fp32, d = 64, m = 4096, r = 5% (k = 205): the fp32 test path
    m1 = 4096
    k1 = tr.tail_len(m1, 5, 100)
    full, tail = synth.scan_case_from_prefix(m1, k1, 1, 64, 64, torch.float32, 0.90, 1.00,
                                             seed=synth.SEED_BASE + 0)
    fd = [x.to(dev) for x in (full.q, full.k, full.v, full.log_alpha, full.beta)]
    td = [x.to(dev) for x in (tail.q, tail.k, tail.v, tail.log_alpha, tail.beta)]
    o1 = torch.empty_like(td[2])
    S1m = torch.empty(1, 1, 64, 64, device=dev)
    S1h = torch.empty_like(S1m)
    cu_t, cu_f = tr.seqlens(tail.cu_seqlens, dev), tr.seqlens(full.cu_seqlens, dev)
    run_tail = lambda: tr.gdn_scan(*td, cu_t, o=o1, S_final=S1h)
    run_full = lambda: tr.gdn_scan(*fd, cu_f, want_o=False, S_final=S1m)
    for _ in range(3):
        run_tail(); run_full()
    t_tail = timed(run_tail, n_rep) * 1e-3
    t_full = timed(run_full, n_rep) * 1e-3
    _, tot1 = tr.state_error(S1m.reshape(-1, 64, 64), S1h.reshape(-1, 64, 64), per_mat=False)
    by1 = k1 * (3 * 64 * 4 + 8 + 64 * 4) + 64 * 64 * 4
    c1 = {"workload": "single-head Gated DeltaNet scan, fp32, d_k=d_v=64, m=4096, r=0.05 "
                      "(k=205), alpha~U[0.90,1]",
          "tail_us": t_tail * 1e6, "state_updates_per_s": k1 / t_tail,
          "full_prefill_us": t_full * 1e6, "full_prefill_state_updates_per_s": m1 / t_full,
          "state_error": float(tot1.item()),
          "roofline": {"bound": "latency", "achieved": by1 / t_tail / 1e9, "unit": "GB/s",
                       "peak": peaks["hbm_gbs"], "frac": by1 / t_tail / 1e9 / peaks["hbm_gbs"],
                       "note": "one head of 205 tokens: a chain of 205 dependent updates; "
                               "reported for information"}}
    if cpu:
        import oracle
        t0 = time.perf_counter()
        reps = 0
        while reps < 3 or time.perf_counter() - t0 < 1.0:
            oracle.gdn_scan(tail.q, tail.k, tail.v, tail.log_alpha, tail.beta, tail.cu_seqlens)
            reps += 1
        c1["cpu_baseline"] = {"value": k1 * reps / (time.perf_counter() - t0),
                              "unit": "state-updates/s", "cores": os.cpu_count(),
                              "kind": "oracle", "sample": "the whole k=205 tail, %d runs" % reps}
    out["config1_fp32_single_head"] = c1
    del fd, td

    # ---- 3: 8 concurrent hits x 8 groups x 3 LA layers, d_model 2048, 16 heads, m = 32768
    Dm, Hh, d, Lg, G, N, m3 = 2048, 16, 128, 3, 8, 8, 32768
    base = synth.SEED_BASE + 2
    layers3 = [synth.la_layers(Lg, Dm, Hh, d, d, seed=base * 16 + g, device=str(dev))
               for g in range(G)]
    for r_num in (5, 10):
        k3 = tr.tail_len(m3, r_num, 100)
        cu3 = synth.cu_seqlens_of([k3] * N)
        hs = [synth.hidden_prefix(N * k3, Dm, base * 1024 + 8 * g + r_num, device=str(dev))
              for g in range(G)]
        reps = [tr.GroupReplay(hs[g], cu3, [tr.Layer(l.W_in, l.W_o) for l in layers3[g]],
                               Hh, d, d, skip_last_output=True) for g in range(G)]
        # the groups one after another, and on 2 and 4 lanes (concurrent streams)
        by_lanes = {}
        for lanes in (1, 2, 4):
            grp = tr.GroupsReplay(reps, lanes=lanes)
            for _ in range(2):
                grp.run(stream)
            by_lanes[lanes] = timed(lambda: grp.run(stream), max(3, n_rep // 4)) * 1e-3
            tr.check()
            del grp
        best3 = min(by_lanes, key=by_lanes.get)
        t3 = by_lanes[best3]
        F3, B3 = _group_flops_bytes(N * k3, Dm, Hh, d, Lg, G)
        t_roof = max(F3 / (peaks["bf16_tflops"] * 1e12), B3 / (peaks["hbm_gbs"] * 1e9))
        c3 = {"workload": "8 concurrent hits x 8 groups x 3 LA layers, d_model 2048, 16 heads "
                          "d=128, m=32768, r=%.2f (k=%d), one tr_replay_groups call" % (r_num / 100, k3),
              "us": t3 * 1e6, "replayed_tokens_per_s": N * k3 / t3,
              "token_layers_per_s": N * k3 * G * Lg / t3,
              "state_updates_per_s": N * k3 * G * Lg * Hh / t3,
              "roofline": {"bound": "tensor", "t_roof_us": t_roof * 1e6, "alg_flops": F3,
                           "alg_bytes": B3, "achieved": F3 / t3 / 1e12, "unit": "TFLOP/s",
                           "peak": peaks["bf16_tflops"], "frac": t_roof / t3},
              "lanes": best3, "us_by_lanes": {str(n): v * 1e6 for n, v in by_lanes.items()}}
        out["config3_8hits_8groups_r%02d" % r_num] = c3
        del reps, hs
    if cpu:
        import oracle
        lc = synth.la_layers(Lg, Dm, Hh, d, d, seed=base * 16)
        hcpu = synth.hidden_prefix(128, Dm, base)
        t0 = time.perf_counter()
        oracle.replay_group(hcpu, [0, 128], lc, Hh, d, d, skip_last_output=True)
        dt = time.perf_counter() - t0
        for r_num in (5, 10):
            out["config3_8hits_8groups_r%02d" % r_num]["cpu_baseline"] = {
                "value": 128 / dt / G, "unit": "replayed tokens/s", "cores": os.cpu_count(),
                "kind": "oracle",
                "sample": "128 tail tokens through one group's 3 LA layers (%.1f s), "
                          "extrapolated to 8 groups" % dt}
    del layers3

    # ---- 4: 64 requests, m ~ U[1024, 131072], r = 10%, d_model 4096, 32 heads, 8 groups x 3
    Dm, Hh, G, n = 4096, 32, 8, 64
    seed = synth.SEED_BASE + 3
    ms = synth.varlen_prefix_lengths(n, 1024, 131072, seed)
    ks = [tr.tail_len(mi, 10, 100) for mi in ms]
    cu4 = synth.cu_seqlens_of(ks)
    T4 = int(cu4[-1])
    # the packed tails (about 3.5 GB), drawn on the device and shared by the 8 groups: the
    # groups' cost does not depend on the values
    h4 = synth.hidden_prefix(T4, Dm, seed, device=str(dev))
    layers4 = [synth.la_layers(Lg, Dm, Hh, d, d, seed=seed * 16 + g, device=str(dev))
               for g in range(G)]
    reps = [tr.GroupReplay(h4, cu4, [tr.Layer(l.W_in, l.W_o) for l in layers4[g]], Hh, d, d,
                           skip_last_output=True) for g in range(G)]
    # the groups one after another, and on 2 lanes (each lane holds a ~46 GB workspace slice;
    # a lane count that does not fit in memory is skipped)
    by4 = {}
    for lanes in (1, 2):
        try:
            grp = tr.GroupsReplay(reps, lanes=lanes)
        except torch.cuda.OutOfMemoryError:
            continue
        grp.run(stream)
        torch.cuda.synchronize()
        by4[lanes] = timed(lambda: grp.run(stream), 2) * 1e-3
        tr.check()
        del grp
        torch.cuda.empty_cache()
    best4 = min(by4, key=by4.get)
    t4 = by4[best4]
    F4, B4 = _group_flops_bytes(T4, Dm, Hh, d, Lg, G)
    t_roof = max(F4 / (peaks["bf16_tflops"] * 1e12), B4 / (peaks["hbm_gbs"] * 1e9))
    c4 = {"workload": "varlen batch of 64 requests, m~U[1024,131072] packed via cu_seqlens, "
                      "r=0.10 (sum k=%d), d_model 4096, 32 heads d=128, 8 groups x 3 LA layers, "
                      "one tr_replay_groups call (the 8 groups share one packed h buffer)" % T4,
          "us": t4 * 1e6, "replayed_tokens_per_s": T4 / t4,
          "token_layers_per_s": T4 * G * Lg / t4, "state_updates_per_s": T4 * G * Lg * Hh / t4,
          "max_k": max(ks), "min_k": min(ks),
          "roofline": {"bound": "tensor", "t_roof_us": t_roof * 1e6, "alg_flops": F4,
                       "alg_bytes": B4, "achieved": F4 / t4 / 1e12, "unit": "TFLOP/s",
                       "peak": peaks["bf16_tflops"], "frac": t_roof / t4},
          "lanes": best4, "us_by_lanes": {str(n): v * 1e6 for n, v in by4.items()}}
    if cpu:
        import oracle
        lc = synth.la_layers(Lg, Dm, Hh, d, d, seed=seed * 16)
        hcpu = synth.hidden_prefix(64, Dm, seed)
        t0 = time.perf_counter()
        oracle.replay_group(hcpu, [0, 64], lc, Hh, d, d, skip_last_output=True)
        dt = time.perf_counter() - t0
        c4["cpu_baseline"] = {"value": 64 / dt / G, "unit": "replayed tokens/s",
                              "cores": os.cpu_count(), "kind": "oracle",
                              "sample": "64 tail tokens through one group's 3 LA layers (%.1f s),"
                                        " extrapolated to 8 groups" % dt}
    out["config4_varlen_64req_d4096"] = c4
    del reps, h4, layers4
    torch.cuda.empty_cache()

    # ---- 5: the scan sweep, 32 heads d = 128, bf16, alpha ~ U[0.80, 1] and U[0.97, 1]
    Hh = 32
    cells = []
    gen = torch.Generator(device=dev)
    for alpha_lo in (0.80, 0.97):
        for mi, m in enumerate(SWEEP_M):
            gen.manual_seed(synth.SEED_BASE + 4 + 16 * mi + (0 if alpha_lo == 0.80 else 8))
            # inputs drawn on the device with the sweep's distributions (unit q, k; N(0,1) v;
            # alpha ~ U[alpha_lo, 1]; beta = sigmoid(N(0,1)))
            def unit(shape):
                x = torch.randn(*shape, generator=gen, device=dev)
                return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
            q, kk = unit((m, Hh, d)), unit((m, Hh, d))
            v = torch.randn(m, Hh, d, generator=gen, device=dev).to(torch.bfloat16)
            la = torch.log(alpha_lo + (1 - alpha_lo) * torch.rand(m, Hh, generator=gen, device=dev))
            be = torch.sigmoid(torch.randn(m, Hh, generator=gen, device=dev))
            S_m = torch.empty(1, Hh, d, d, device=dev)
            tr.gdn_scan(q, kk, v, la, be, [0, m], want_o=False, S_final=S_m)
            for r in SWEEP_R:
                k5 = tr.tail_len(m, r, 100)
                a = m - k5
                o5 = torch.empty(k5, Hh, d, dtype=torch.bfloat16, device=dev)
                Sh = torch.empty_like(S_m)
                args5 = (q[a:], kk[a:], v[a:], la[a:].contiguous(), be[a:].contiguous())
                cu5 = tr.seqlens([0, k5], dev)
                fn = lambda: tr.gdn_scan(*args5, cu5, o=o5, S_final=Sh)
                fn()
                t5 = timed(fn, max(3, min(n_rep, 10))) * 1e-3
                _, tot = tr.state_error(S_m.reshape(-1, d, d), Sh.reshape(-1, d, d),
                                        per_mat=False)
                upd = k5 * Hh
                by = upd * (3 * 256 + 8 + 256) + Hh * d * d * 4
                cells.append({"m": m, "r": r / 100, "k": k5, "alpha": [alpha_lo, 1.0],
                              "us": t5 * 1e6, "state_updates_per_s": upd / t5,
                              "achieved_gbs": by / t5 / 1e9,
                              "frac": by / t5 / 1e9 / peaks["hbm_gbs"],
                              "rel_state_error": float(tot.item())})
            del q, kk, v, la, be
    tr.check()
    c5 = {"workload": "scan sweep m in {4K..128K} x r in {1,2,5,10,20,100}%, 32 heads d=128, "
                      "bf16 q/k/v, alpha~U[0.80,1] and U[0.97,1]; per cell the tail replay "
                      "(readout included) timed, ||S_m - S_hat_m||/||S_m|| against the full "
                      "prefill",
          "roofline_basis": "HBM: 1032 B per token-head + 64 KB state out per head, of the "
                            "measured copy bandwidth",
          "cells": cells}
    if cpu:
        import oracle
        case = synth.scan_case([512], Hh, d, d, torch.bfloat16, 0.97, 1.0, seed=synth.SEED_BASE + 4)
        t0 = time.perf_counter()
        oracle.gdn_scan(case.q, case.k, case.v, case.log_alpha, case.beta, case.cu_seqlens)
        dt = time.perf_counter() - t0
        c5["cpu_baseline"] = {"value": 512 * Hh / dt, "unit": "state-updates/s",
                              "cores": os.cpu_count(), "kind": "oracle",
                              "sample": "512 tokens x 32 heads with readout (%.1f s); the same "
                                        "rate applies to every cell (extrapolated)" % dt}
    out["config5_scan_sweep"] = c5
    return out


# ------------------------------------------------------------------ reference
def reference_arm(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return
    import numpy as np
    import torch
    import oracle
    import synth

    k = oracle.tail_len(M_PREFIX, R_NUM, R_DEN)
    seed = synth.SEED_BASE + 1
    h_tail = synth.hidden_prefix(M_PREFIX, D, seed)[M_PREFIX - k:]
    layers = synth.la_layers(L, D, H, DH, DH, seed=seed)
    sample = args.sample_tokens  # tokens per step (default 205 = 1/8 of the tail), all 3 layers
    cu = [0, sample]
    times = []
    for i in range(args.warmup + args.steps):
        a = (i * sample) % (k - sample)
        t0 = time.perf_counter()
        oracle.replay_group(h_tail[a:a + sample], cu, layers, H, DH, DH, skip_last_output=True)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    mean = sum(times) / len(times)
    value = sample / mean
    cores = os.cpu_count()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "replayed tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "k": k, "sample_tokens": sample},
        "cpu_baseline": {"value": value, "unit": "replayed tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": "%d consecutive tail tokens through all 3 LA layers per step"
                                   % sample},
        "e2e": {"value": value, "unit": "replayed tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- our arm
def cpu_baseline_sample(h_tail_cpu, layers_cpu, k):
    import oracle
    reps, t = 0, 0.0
    oracle.replay_group(h_tail_cpu[:64], [0, 64], layers_cpu, H, DH, DH, skip_last_output=True)
    while reps < 2 or (t < 10.0 and reps < 4):
        t0 = time.perf_counter()
        oracle.replay_group(h_tail_cpu, [0, k], layers_cpu, H, DH, DH, skip_last_output=True)
        t += time.perf_counter() - t0
        reps += 1
    return {"value": k * reps / t, "unit": "replayed tokens/s", "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": "full k=%d tail of the bench workload, %d repetitions (%.1f s)" % (k, reps, t)}


def our_arm(args):
    import torch
    import torch.distributed as dist
    import synth
    import linear_attention_state_zero_b200 as tr

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks, peak_src = load_peaks()

    k = tr.tail_len(M_PREFIX, R_NUM, R_DEN)
    seed = rank_seed(rank)
    h_full_cpu = synth.hidden_prefix(M_PREFIX, D, seed)
    h_tail_cpu = h_full_cpu[M_PREFIX - k:].contiguous()
    layers_cpu = synth.la_layers(L, D, H, DH, DH, seed=seed)
    layers = [tr.Layer(l.W_in.to(dev), l.W_o.to(dev)) for l in layers_cpu]
    h_full = h_full_cpu.to(dev)
    h_tail = h_tail_cpu.to(dev)

    # full-prefill reference states S_m (k = m), untimed
    full = tr.GroupReplay(h_full, [0, M_PREFIX], layers, H, DH, DH, skip_last_output=True)
    S_m = full.run()[0].clone()
    del full
    rep = tr.GroupReplay(h_tail, [0, k], layers, H, DH, DH, skip_last_output=True)
    S_m_flat = S_m.reshape(-1, DH, DH)
    S_hat_flat = rep.S_hat.reshape(-1, DH, DH)
    n_k = rep.kernel_count()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    # one event before the replay, one after each of its kernels, one after the state error
    events = [torch.cuda.Event(enable_timing=True) for _ in range(n_k + 2)]
    stream = torch.cuda.current_stream()
    for e in events:
        e.record(stream)
    handles = [e.cuda_event for e in events]

    def step():
        # the production path: every kernel launched back to back (programmatic
        # dependent launch between them)
        rep.run(stream)
        per, tot = tr.state_error(S_m_flat, S_hat_flat, per_mat=False)
        return tot

    def step_profiled():
        # the same kernels with an event recorded after each one (no overlap of launches)
        rep.run_profiled(handles[:n_k + 1], stream)
        per, tot = tr.state_error(S_m_flat, S_hat_flat, per_mat=False)
        events[-1].record(stream)
        return tot

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        flush.zero_()
        step()
        flush.zero_()
        step_profiled()
    torch.cuda.synchronize()
    tr.check()

    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = []
    err_tot = None
    for _ in range(args.steps):
        flush.zero_()  # L2 flush outside the timed interval
        e0.record(stream)
        err_tot = step()
        e1.record(stream)
        e1.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    tr.check()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(k, world, ms_per_step)

    # per-kernel CUDA-event times over the same number of steps (profiled launches)
    prof_ms, kern_ms = [], [[] for _ in range(n_k)]
    for _ in range(args.steps):
        flush.zero_()
        step_profiled()
        torch.cuda.synchronize()  # read this step's events before they are re-recorded
        prof_ms.append(events[0].elapsed_time(events[-1]))
        for i in range(n_k):
            kern_ms[i].append(events[i].elapsed_time(events[i + 1]))
    tr.check()

    # per-kernel breakdown, in launch order (the library names its launches)
    names = rep.kernel_names()
    assert len(names) == n_k, (names, n_k)
    avg = [sum(x) / len(x) for x in kern_ms]
    brk = {}
    for n, a in zip(names, avg):
        brk[n] = brk.get(n, 0.0) + a * 1e3
    kernels = kernel_rooflines(names, avg, k, peaks)
    dominant = max(kernels, key=lambda n: kernels[n]["us_per_step"])
    traffic = load_traffic()
    F, B = group_model(k)
    t_roof = max(F / (peaks["bf16_tflops"] * 1e12), B / (peaks["hbm_gbs"] * 1e9))

    # end to end through the public API with host buffers: every step copies its h tail
    # from pinned host memory and reads S_hat and the error back.  Two replay contexts
    # (own h, S_hat, workspace) alternate, so step i+1's input copy (copy stream) runs
    # during step i's kernels and step i's read-back (second copy stream) during step
    # i+1's; L2 is flushed before every replay, inside the timed interval.
    h_host = h_tail_cpu.pin_memory()
    reps2 = [rep, tr.GroupReplay(torch.empty_like(h_tail), [0, k], layers, H, DH, DH,
                                 skip_last_output=True)]
    h_dev = [h_tail, reps2[1].h_tail]
    S_host = [torch.empty(rep.S_hat.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    err_host = [torch.empty(1, dtype=torch.float64).pin_memory() for _ in range(2)]
    cp_in, cp_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_done, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    started = [False, False]
    tot_b = [None, None]

    def e2e_step(i):
        b = i % 2
        if started[b]:
            cp_in.wait_event(ev_done[b])   # replay i-2 no longer reads this h buffer
        with torch.cuda.stream(cp_in):
            h_dev[b].copy_(h_host, non_blocking=True)
        ev_in[b].record(cp_in)
        stream.wait_event(ev_in[b])
        if started[b]:
            stream.wait_event(ev_out[b])   # step i-2's S_hat has been read back
        flush.zero_()
        reps2[b].run(stream)
        _, tot_b[b] = tr.state_error(S_m_flat, reps2[b].S_hat.reshape(-1, DH, DH), per_mat=False)
        ev_done[b].record(stream)
        cp_out.wait_event(ev_done[b])
        with torch.cuda.stream(cp_out):
            S_host[b].copy_(reps2[b].S_hat, non_blocking=True)
            err_host[b].copy_(tot_b[b], non_blocking=True)
        ev_out[b].record(cp_out)
        started[b] = True

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    e0.record(stream)
    cp_in.wait_event(e0)
    for i in range(args.warmup, args.warmup + args.steps):
        e2e_step(i)
    for b in range(2):
        stream.wait_event(ev_out[b])
    e1.record(stream)
    e1.synchronize()
    e2e_total = e0.elapsed_time(e1)
    tr.check()
    e2e_value = job_throughput(k, world, max_over_ranks(e2e_total, world, dev) / args.steps)
    assert float(err_host[(args.warmup + args.steps - 1) % 2].item()) == float(err_tot.item())

    # transfer/replay overlap: the group's FA KV (K and V of the m = 32768 prefix; 2 KV heads
    # of 128, bf16: 33.5 MB) copied from pinned host memory on its own stream during the replay
    kv_host = torch.empty(2 * M_PREFIX * 2 * DH * 2, dtype=torch.uint8).pin_memory()
    kv_dev = torch.empty(kv_host.shape, dtype=torch.uint8, device=dev)
    groups = tr.GroupsReplay([rep])
    side = torch.cuda.Stream(device=dev)

    def timed(fn, n):
        ts = []
        for _ in range(n):
            flush.zero_()
            torch.cuda.synchronize()
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return sum(ts) / len(ts)

    def copy_only():
        # the same entry point with no groups: one cudaMemcpyAsync on the copy stream
        tr.kv_transfer(kv_host, kv_dev, stream=stream, copy_stream=side)

    n_ov = max(5, min(args.steps, 30))
    for _ in range(3):
        groups.run_overlapped(kv_host, kv_dev, stream=stream, copy_stream=side)
    t_kv = timed(copy_only, n_ov)
    t_rep = timed(lambda: groups.run(stream), n_ov)
    t_ov = timed(lambda: groups.run_overlapped(kv_host, kv_dev, stream=stream, copy_stream=side),
                 n_ov)
    tr.check()

    # scan-only cell: 32 heads d=128, m=32768, r=0.10 (k=3277), bf16, alpha ~ U[0.97, 1]
    k5 = tr.tail_len(32768, 10, 100)
    case = synth.scan_case([k5], 32, 128, 128, torch.bfloat16, 0.97, 1.0, seed=synth.SEED_BASE + 4)
    sq, sk, sv = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    sla, sb = case.log_alpha.to(dev), case.beta.to(dev)
    so = torch.empty_like(sv)
    sS = torch.empty(1, 32, 128, 128, dtype=torch.float32, device=dev)
    cu_s = tr.seqlens(case.cu_seqlens, dev)
    for _ in range(3):
        tr.gdn_scan(sq, sk, sv, sla, sb, cu_s, o=so, S_final=sS)
    scan_ms = []
    for _ in range(max(5, min(args.steps, 50))):
        flush.zero_()
        e0.record(stream)
        tr.gdn_scan(sq, sk, sv, sla, sb, cu_s, o=so, S_final=sS)
        e1.record(stream)
        e1.synchronize()
        scan_ms.append(e0.elapsed_time(e1))
    scan_t = sum(scan_ms) / len(scan_ms) * 1e-3
    upd = k5 * 32
    scan_bytes = upd * (3 * 256 + 8 + 256) + 32 * 128 * 128 * 4
    scan_gbs = scan_bytes / scan_t / 1e9
    # the same tail's transition product P (32 heads of 128 x 128), the repair operator
    cu5 = cu_s
    Pbuf = torch.empty(1, 32, 128, 128, dtype=torch.float32, device=dev)
    for _ in range(3):
        tr.transition_product(sk, sla, sb, cu5, P=Pbuf)
    tp_ms = []
    for _ in range(max(5, min(args.steps, 50))):
        flush.zero_()
        e0.record(stream)
        tr.transition_product(sk, sla, sb, cu5, P=Pbuf)
        e1.record(stream)
        e1.synchronize()
        tp_ms.append(e0.elapsed_time(e1))
    tp_t = sum(tp_ms) / len(tp_ms) * 1e-3
    tr.check()

    # FFN cell: the same group and tail with a dense SwiGLU FFN (d_ff = D_FF) after each LA
    # layer but the last (the tail-FFN skip), weights drawn on the device
    fl_dev = synth.la_layers(L, D, H, DH, DH, seed=seed + 7, device=str(dev), d_ff=D_FF)
    frep = tr.GroupReplay(h_tail, [0, k], [tr.Layer(l.W_in, l.W_o, None, l.W_gate, l.W_up,
                                                    l.W_down) for l in fl_dev],
                          H, DH, DH, skip_last_output=True)
    n_f = frep.kernel_count()
    fev = [torch.cuda.Event(enable_timing=True) for _ in range(n_f + 1)]
    for e in fev:
        e.record(stream)
    fh = [e.cuda_event for e in fev]
    for _ in range(3):
        frep.run(stream)
    f_t = timed(lambda: frep.run(stream), n_ov)
    f_kern = [0.0] * n_f
    for _ in range(n_ov):
        flush.zero_()
        frep.run_profiled(fh, stream)
        torch.cuda.synchronize()
        for i in range(n_f):
            f_kern[i] += fev[i].elapsed_time(fev[i + 1]) / n_ov
    tr.check()
    # the FFN's launches by name (rmsnorm, gate/up with the SwiGLU epilogue, down)
    f_names = frep.kernel_names()
    def f_sum(name):
        v = [t for n, t in zip(f_names, f_kern) if n == name]
        return sum(v) * 1e3 if v else float("nan")
    sw_us, dn_us, fn_us = f_sum("ffn_gate_up"), f_sum("ffn_down"), f_sum("ffn_rmsnorm")
    sw_flops = 2.0 * k * D * 2 * D_FF          # per launch
    dn_flops = 2.0 * k * D_FF * D
    sw_tf = sw_flops * (L - 1) / (sw_us * 1e-6) / 1e12
    dn_tf = dn_flops * (L - 1) / (dn_us * 1e-6) / 1e12
    del frep, fl_dev

    # GDN-options cell: the same group and tail with the short convolution (width 4), the
    # per-head gate parameters and the gated output norm
    gl_dev = synth.la_layers(L, D, H, DH, DH, seed=seed + 11, device=str(dev), conv_width=4,
                             gate_params=True, output_gate=True)
    grep_ = tr.GroupReplay(h_tail, [0, k], [tr.Layer(l.W_in, l.W_o, conv_w=l.conv_w, A_log=l.A_log,
                                                     dt_bias=l.dt_bias, o_norm_gain=l.o_norm_gain)
                                            for l in gl_dev],
                           H, DH, DH, skip_last_output=True, output_gate=True)
    n_g = grep_.kernel_count()
    gev = [torch.cuda.Event(enable_timing=True) for _ in range(n_g + 1)]
    for e in gev:
        e.record(stream)
    gh = [e.cuda_event for e in gev]
    for _ in range(3):
        grep_.run(stream)
    g_t = timed(lambda: grep_.run(stream), n_ov)
    g_kern = [0.0] * n_g
    for _ in range(n_ov):
        flush.zero_()
        grep_.run_profiled(gh, stream)
        torch.cuda.synchronize()
        for i in range(n_g):
            g_kern[i] += gev[i].elapsed_time(gev[i + 1]) / n_ov
    tr.check()
    g_names = grep_.kernel_names()
    def g_sum(name):
        v = [t for n, t in zip(g_names, g_kern) if n == name]
        return sum(v) * 1e3 if v else float("nan")
    conv_us, gn_us = g_sum("short_conv"), g_sum("gated_norm")
    C_conv = 3 * H * DH
    conv_bytes = (L - 1) * k * C_conv * 4 + k * (2 * H * DH) * 4   # bf16 in + out per channel
    gn_bytes = (L - 1) * k * H * DH * 6                            # o, z in; o out (bf16)
    conv_gbs = conv_bytes / (conv_us * 1e-6) / 1e9
    gn_gbs = gn_bytes / (gn_us * 1e-6) / 1e9
    del grep_, gl_dev

    configs = None
    if world == 1 and not args.no_configs:
        configs = config_cells(dev, peaks, stream, flush, args.steps,
                               cpu=not args.no_cpu_baseline)

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline_sample(h_tail_cpu, layers_cpu, k)
        line = {
            "metric": METRIC, "value": value, "unit": "replayed tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "d_model": D, "n_heads": H, "d_head": DH,
                       "la_layers": L, "m": M_PREFIX, "r": R_NUM / R_DEN, "k": k,
                       "requests_per_gpu": 1, "parallelism": "independent requests per GPU",
                       "l2": "flushed (256 MiB write) before every timed step"},
            "token_layers_per_s": value * L,
            "state_updates_per_s": value * L * H,
            "state_error_vs_full_prefill": float(err_tot.item()),
            # the dominant kernel's figure (the contract), with the whole step's fraction of
            # its own roofline beside it (group_step_frac = t_roof / t_step)
            "roofline": dict(kernels[dominant], kernel=dominant,
                             traffic=traffic.get(dominant),
                             peak_source=peak_src + (" (burst bf16)" if kernels[dominant]["bound"] ==
                                                     "tensor" else " (HBM copy)"),
                             group_step_frac=t_roof / (ms_per_step * 1e-3)),
            "kernel_rooflines": {n: dict(r, traffic=traffic.get(n)) for n, r in kernels.items()},
            "profiled_ms_per_step": sum(prof_ms) / len(prof_ms),
            "group_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": ms_per_step * 1e3,
                               "frac": t_roof / (ms_per_step * 1e-3), "alg_flops": F,
                               "alg_bytes": B},
            "kernel_us_per_step": brk,
            "scan": {"workload": "scan only: 32 heads d=128, bf16, alpha~U[0.97,1], m=32768, "
                                 "r=0.10 (k=%d)" % k5,
                     "state_updates_per_s": upd / scan_t, "us": scan_t * 1e6,
                     "roofline": {"bound": "hbm", "achieved": scan_gbs, "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": scan_gbs / peaks["hbm_gbs"],
                                  "traffic": traffic.get("scan_cell"),
                                  "alg_bytes": scan_bytes}},
            "transfer_overlap": {
                "workload": "group replay with the FA KV (33.5 MB, pinned host) copied on its own "
                            "stream", "kv_bytes": int(kv_host.numel()), "kv_copy_us": t_kv * 1e3,
                "replay_us": t_rep * 1e3, "overlapped_us": t_ov * 1e3,
                "max_over_overlapped": max(t_kv, t_rep) / t_ov},
            "transition_product": {
                "workload": "P = T_t...T_1 of the scan cell's tail (32 heads, k=%d), fp32 out" % k5,
                "us": tp_t * 1e6, "token_heads_per_s": upd / tp_t},
            "ffn_group": {
                "workload": "the headline group and tail with a dense SwiGLU FFN (d_ff=%d) after "
                            "each LA layer but the last (tail-FFN skip)" % D_FF,
                "us": f_t * 1e3, "replayed_tokens_per_s": k / (f_t * 1e-3),
                "kernels_per_step": n_f,
                "ffn_us_per_step": {"rmsnorm": fn_us, "gate_up_swiglu": sw_us, "down": dn_us},
                "gate_up_roofline": {"bound": "tensor", "achieved": sw_tf,
                                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                     "frac": sw_tf / peaks["bf16_tflops"],
                                     "flops_per_launch": sw_flops},
                "down_roofline": {"bound": "tensor", "achieved": dn_tf,
                                  "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                  "frac": dn_tf / peaks["bf16_tflops"],
                                  "flops_per_launch": dn_flops}},
            "gdn_options": {
                "workload": "the headline group and tail with the short convolution (width 4), "
                            "per-head A_log/dt_bias and the gated output norm",
                "us": g_t * 1e3, "replayed_tokens_per_s": k / (g_t * 1e-3),
                "kernels_per_step": n_g,
                "conv": {"us_per_step": conv_us, "bound": "hbm", "achieved": conv_gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": conv_gbs / peaks["hbm_gbs"], "bytes_per_step": conv_bytes},
                "gated_norm": {"us_per_step": gn_us, "bound": "hbm", "achieved": gn_gbs,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": gn_gbs / peaks["hbm_gbs"], "bytes_per_step": gn_bytes}},
            "configs": configs,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "replayed tokens/s",
                    "h2d_bytes_per_step": k * D * 2,
                    "d2h_bytes_per_step": int(S_host[0].numel() * 4 + 8)},
            "gpu_launches": args.steps * (n_k + 2),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.profile:
        profile_run(args)
    elif args.impl == "reference":
        reference_arm(args)
    else:
        our_arm(args)


if __name__ == "__main__":
    main()
