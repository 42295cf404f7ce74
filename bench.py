#!/usr/bin/env python
"""Benchmark of the Dust estimator hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--draws K]

A step is one pass of the whole hot path over one batch of synthetic input:
for each hidden linear layer of the workload, the reward scan (a4), the
noise-regenerating draw reduction (a1 + a5) and the weight estimate G_W (a6);
for the LM head, the clean logits (a2, tcgen05), the fused perturbed cross
entropy and its draw reduction over all vocabulary chunks (a1 + a3 + a5) and
the head's G_W (a6).  The synthetic costs c that stand in for the perturbed
forward of the hidden layers are produced once, before timing (harness).

Metric: draws x tokens per second summed over the layers of one step,
value = the draws x tokens of all ranks / max-over-ranks step time.  With
N > 1 GPUs the step is split one of three ways (--shard):
  sequences (default): every rank processes its own batch of whole sequences
    (weak scaling, data parallel), its tokens placed after the previous
    ranks' in the global batch (noise token_begin); the weight estimates are
    summed over ranks by one NCCL all-reduce per step;
  draws: every rank runs a range of the K draws of the same batch (strong
    scaling); the partial weight estimates are summed by the all-reduce;
  vocab: the hidden layers as in `draws`, the LM head split by vocabulary
    chunk (each rank all K draws of a range of chunk passes); its disjoint
    G_W rows are gathered (strong scaling).

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from activation_perturbation_es_b200 import inputs as I  # noqa: E402

DEFAULT_WORKLOAD = I.SCALED.name
METRIC = "Dust draws×tokens/s per layer step"
UNIT = "draws×tokens/s"

# Algorithmic work per element of the ALU-bound kernels, in lane issue slots:
# the noise specification's operations, each in its cheapest sm_100 instruction
# form (one warp instruction issues per scheduler per clock, so a lane gets one
# slot per clock).  Counted per Philox call (4 elements, 2 Box-Muller pairs):
#   Philox4x32-10: 10 rounds x (2 wide 32x32->64 products + 2 three-input xors),
#     less the draw-independent product and xor of round 1              = 38
#   radius uniforms: 2 shift-and-insert + 1 packed subtraction          =  3
#   ln: 2 x 4 integer (exponent split, magic float) + 15 packed fp32
#     (4(m-1), m+1, quotient correction 3, square, Horner 5, product, magic,
#     2 fma) + 2 reciprocal estimates                                   = 25
#   sqrt: 2 clamps + 2 reciprocal-sqrt estimates + 4 packed             =  8
#   angle: 2 x 2 fraction bits + 4 packed + 2 x 2 odd-octant select     = 12
#   sin / cos Horner: 11 packed                                         = 11
#   octant swap and signs: 2 x 7                                        = 14
# (packed: one __ffma2_rn / __fadd2_rn / __fmul2_rn for the same fp32 op on
# both pairs).  Consumers: the hidden reduction adds r rho and two fma (3
# packed) and the load of r (1) = 4; the head adds a = rho cos / rho sin (2),
# the expm1 series and the sum (10), the fma into g (2) and the load of p (1)
# = 15.  Not counted (so the bound stays an upper bound): loop control, the
# head's per-draw warp reduction and log1p.
SLOTS_A5 = (111 + 4) / 4               # 28.75 per Gaussian
SLOTS_HEAD = (111 + 15) / 4            # 31.5 per perturbed logit
LANES_PER_SM = 128                     # 4 schedulers x 32 lanes

# The same work on the datapath that binds both ALU kernels, the FMA-heavy one:
# a packed fp32 instruction holds it (and FMA-lite) for 2 cycles, a 32x32->64
# product holds it for 4 (ncu's active-cycle and instruction counters fit these
# costs).  Per Philox call, with every product the specification needs, less
# those that no draw changes: 18 products in the reduction (round 1's quad
# product is draw-invariant, its draw product steps by an add), 18 1/8 in the
# head (the draw product is shared by a lane's 8 quads); packed operations:
# 34 in the generator, 3 in the reduction's consumer and 14 in the head's.
HEAVY_A5 = (18 * 4 + (34 + 3) * 2) / 4          # 36.5 heavy cycles per Gaussian
HEAVY_HEAD = (18.125 * 4 + (34 + 14) * 2) / 4   # 42.125 per perturbed logit


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(I.WORKLOADS))
    p.add_argument("--draws", type=int, default=0, help="override the workload's K")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--shard", choices=["sequences", "draws", "vocab"], default="sequences",
                   help="how N > 1 ranks split the step (see above); at N = 1 every split is the whole step")
    p.add_argument("--fused", action="store_true",
                   help="hidden layers with d_in a multiple of 64 up to 512 run the draw reduction and the weight "
                        "estimate as one kernel (dust_layer_estimate_weight_grad)")
    return p.parse_args()


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def load_peaks():
    """Roofline denominators: MEASURED_PEAKS.json where it holds a positive
    number for a field, else the fallback; `source` says which fields were
    measured."""
    peaks = dict(FALLBACK_PEAKS)
    measured = []
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        d = {}
    if not isinstance(d, dict):
        d = {}
    for key in FALLBACK_PEAKS:
        v = d.get(key)
        if key == "bf16_tflops_sustained" and v is None:
            v = d.get("bf16_tflops")
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            peaks[key] = float(v)
            measured.append(key)
    peaks["measured_keys"] = measured
    peaks["source"] = ("measured" if len(measured) == len(FALLBACK_PEAKS) else
                       "fallback" if not measured else "measured: " + ", ".join(measured) + "; fallback: others")
    return peaks


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_backend():
    """NCCL, one rank per GPU; DUST_BENCH_DIST_BACKEND=gloo runs the same
    multi-rank flow with host-side collectives, which lets ranks share a GPU
    (no kernel of this library waits on another rank)."""
    b = os.environ.get("DUST_BENCH_DIST_BACKEND", "nccl")
    if b not in ("nccl", "gloo"):
        sys.exit(f"bench: DUST_BENCH_DIST_BACKEND must be nccl or gloo, not {b!r}")
    return b


def dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if dist_backend() == "gloo":
            torch.cuda.set_device(local % torch.cuda.device_count())
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
        else:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch.distributed as dist
    if world > 1:
        dist.barrier()


def max_over_ranks(x, world):
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cpu" if dist.get_backend() == "gloo" else "cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ the workload as both arms name it
def parallelism(shard, world):
    return {"sequences": f"dp{world}", "draws": f"draws{world}", "vocab": f"draws{world}+head_vocab{world}"}[shard]


def workload_config(w, K, world, shard, fused):
    """The `config` object of the line, the same for this library's arm and the
    reference arm: the workload, its population and how N ranks split it."""
    return {"workload": w.name, "tokens_per_rank": w.T, "n_seq": w.n_seq, "seq_len": w.seq_len,
            "draws": K, "sigma": w.sigma, "gamma_hidden": w.gamma,
            "hidden": [[h.d_in, h.d_out] for h in w.hidden],
            "head": {"d": w.head_d, "V": w.V, "Vc": w.Vc} if w.V else None,
            "parallelism": parallelism(shard, world), "shard": shard,
            "dist_backend": dist_backend() if world > 1 else None,
            "l2": l2_statement(w, K),
            "fused_estimate_wgrad": bool(fused)}


L2_BYTES = 126 * 2**20


def step_bytes(w, K):
    """Bytes one step streams through HBM on one rank: each hidden layer's costs
    (read by the scan, rewards written and read), layer input and g (fp32 and
    bf16); the head's logits, g and operands."""
    b = 0
    for h in w.hidden:
        b += 3 * 4 * K * w.T + 2 * w.T * h.d_in + 6 * w.T * h.d_out
    if w.V:
        b += 4 * w.T * w.V + 6 * w.T * w.V + 2 * (w.T + w.V) * w.head_d
    return b


def l2_statement(w, K):
    mb = step_bytes(w, K) / 2**20
    if step_bytes(w, K) > L2_BYTES:
        return f"inputs larger than L2 ({mb:.0f} MB per step against 126 MB); no flush"
    return (f"inputs smaller than L2 ({mb:.1f} MB per step against 126 MB): a warm-L2 small case, not a "
            f"configuration for headline numbers")


# ------------------------------------------------------------------ the step
class Step:
    """Device-resident buffers and the sequence of C-ABI calls of one step on
    this rank: its sequences (shard 'sequences'), its draws ('draws') or, for
    the head, its vocabulary chunks ('vocab')."""

    def __init__(self, w: I.Workload, K: int, rank: int, world: int, fused: bool = False, shard: str = "sequences"):
        import torch
        from activation_perturbation_es_b200 import dust, dp
        self.torch, self.dust, self.dp, self.w, self.K, self.world = torch, dust, dp, w, K, world
        self.shard = shard
        dev = torch.device("cuda", torch.cuda.current_device())
        self.dev = dev
        bf = torch.bfloat16
        T = w.T
        by_seq = self.shard == "sequences"
        data_off = rank * 7919 if by_seq else 0          # each rank's own batch, or one batch for all
        tok0 = rank * T if by_seq else 0                 # global index of this rank's first token
        d0, nd = (0, K) if by_seq else dp.draw_range(K, world, rank)
        self.draws = nd
        self.off = torch.from_numpy(I.uniform_offsets(w.n_seq, w.seq_len)).to(dev)
        self.hidden = []
        self.host = {}          # pinned host copies of every per-step input (for e2e)
        for hl in w.hidden:
            li = I.layer_inputs(w, hl, seed_offset=data_off)
            nz = dust.Noise(w.seed, hl.layer, d0, nd, K, w.sigma, token_begin=tok0)
            u = torch.from_numpy(li["u"]).to(dev)
            c = dust.synth_costs(u, nz, w.eps_scale)          # harness: stands in for the perturbed forward
            del u
            X = torch.from_numpy(li["X"]).to(dev, bf)
            L = {"hl": hl, "nz": nz, "c": c, "X": X,
                 "fused": fused and hl.d_in % 64 == 0 and 64 <= hl.d_in <= 512,
                 "r": torch.empty_like(c),
                 "g": torch.empty(T, hl.d_out, dtype=torch.float32, device=dev),
                 "g16": torch.empty(T, hl.d_out, dtype=bf, device=dev),
                 "G": torch.empty(hl.d_out, hl.d_in, dtype=torch.float32, device=dev)}
            self.hidden.append(L)
        self.head = None
        if w.V:
            hi = I.head_inputs(w, seed_offset=data_off)
            W = I.head_inputs(w)["W"]                        # the head's weights are shared by all ranks
            n_chunks = w.V // w.Vc
            if self.shard == "vocab":
                cb, cc = dp.chunk_range(n_chunks, world, rank)
                hd0, hnd = 0, K
            else:
                cb, cc = 0, n_chunks
                hd0, hnd = d0, nd
            Vr = cc * w.Vc
            nz = dust.Noise(w.seed, w.head_layer, hd0, hnd, K, w.sigma, token_begin=tok0)
            self.head = {"nz": nz, "X": torch.from_numpy(hi["X"]).to(dev, bf),
                         "W": torch.from_numpy(W).to(dev, bf),
                         "y": torch.from_numpy(hi["y"]).to(dev),
                         "chunks": (cb, cc), "rows": [dp.chunk_range(n_chunks, world, r)[1] * w.Vc
                                                      for r in range(world)] if self.shard == "vocab" else None,
                         "Z": torch.empty(T, w.V, dtype=torch.float32, device=dev),
                         "g": torch.empty(T, max(Vr, 1), dtype=torch.float32, device=dev),
                         "g16": torch.empty(T, max(Vr, 1), dtype=bf, device=dev),
                         "G": torch.empty(max(Vr, 1), w.head_d, dtype=torch.float32, device=dev)}
            self.head["draws"] = hnd
            self.head["Vr"] = Vr
        torch.cuda.synchronize()
        self.stage_names = []
        for L in self.hidden:
            n = L["hl"].name
            self.stage_names += [f"{n}:scan"] + ([f"{n}:fused_estimate_wgrad"] if L["fused"]
                                                 else [f"{n}:estimate", f"{n}:weight_grad"])
        if self.head:
            self.stage_names += ["head:logits", "head:ce_estimate", "head:weight_grad"]
        self.events = None
        self.G_head_all = None

    def units(self):
        """Draws x tokens of one step summed over the layers, on this rank."""
        u = self.draws * self.w.T * len(self.hidden)
        if self.head:
            # a vocabulary-chunk shard runs all K draws on a fraction Vr/V of the head's chunks
            u += self.head["draws"] * self.w.T * self.head["Vr"] / self.w.V
        return u

    def total_units(self):
        """Draws x tokens of one step over all ranks: every rank's own batch
        (sequences), or the one batch's K draws of every layer (draws, vocab)."""
        per_batch = self.K * self.w.T * (len(self.hidden) + (1 if self.head else 0))
        return per_batch * self.world if self.shard == "sequences" else per_batch

    def scaling(self):
        return "weak" if self.shard == "sequences" else "strong"

    def parallelism(self):
        return parallelism(self.shard, self.world)

    def make_events(self, n_steps):
        ev = self.torch.cuda.Event
        self.events = [[ev(enable_timing=True) for _ in range(len(self.stage_names) + 1)] for _ in range(n_steps)]

    def run(self, step_idx=None):
        dust = self.dust
        evs = self.events[step_idx] if step_idx is not None else None
        i = 0

        def mark():
            nonlocal i
            if evs is not None:
                evs[i].record()
            i += 1

        for L in self.hidden:
            hl = L["hl"]
            mark()
            dust.reward_scan(L["c"], self.off, self.w.gamma, out=L["r"])
            mark()
            self._estimate(L)
            if not L["fused"]:
                mark()
                dust.weight_grad(L["g16"], L["X"], G_W=L["G"])
        if self.head:
            H = self.head
            mark()
            dust.logits(H["X"], H["W"], Z=H["Z"])
            mark()
            self._head(H)
            mark()
            if H["Vr"]:
                dust.weight_grad(H["g16"], H["X"], G_W=H["G"])
        mark()
        if self.world > 1:
            self.allreduce()

    def run_overlapped(self, ready):
        """The step's call sequence with layer j's compute waiting on ready[j]."""
        dust, cur = self.dust, self.torch.cuda.current_stream()
        j = 0
        for L in self.hidden:
            cur.wait_event(ready[j])
            j += 1
            dust.reward_scan(L["c"], self.off, self.w.gamma, out=L["r"])
            self._estimate(L)
            if not L["fused"]:
                dust.weight_grad(L["g16"], L["X"], G_W=L["G"])
        if self.head:
            H = self.head
            cur.wait_event(ready[j])
            dust.logits(H["X"], H["W"], Z=H["Z"])
            self._head(H)
            if H["Vr"]:
                dust.weight_grad(H["g16"], H["X"], G_W=H["G"])
        if self.world > 1:
            self.allreduce()

    def _head(self, H):
        """Row statistics + this rank's chunk passes (a3 + a5) on the cached logits of a2."""
        cb, cc = H["chunks"]
        if cc:
            self.dust.head_step(H["y"], self.w.Vc, H["nz"], Z=H["Z"], g_hat=H["g"], g_hat_bf16=H["g16"],
                                chunk_begin=cb, chunk_count=cc)

    def _estimate(self, L):
        """The draw reduction; fused with the weight estimate when L is eligible."""
        hl = L["hl"]
        if L["fused"]:
            self.dust.layer_estimate_weight_grad(L["r"], True, self.off, self.w.gamma, L["nz"], L["X"], hl.d_out,
                                                 G_W=L["G"])
        else:
            self.dust.layer_estimate(L["r"], True, self.off, self.w.gamma, L["nz"], hl.d_out, g_hat=L["g"],
                                     g_hat_bf16=L["g16"])

    def allreduce(self):
        """The step's exchange: the weight estimates summed over ranks; with the
        head split by vocabulary chunk, its disjoint G_W rows gathered instead."""
        dp = self.dp
        by_vocab = self.head is not None and self.head["rows"] is not None
        dp.allreduce_sum_([L["G"] for L in self.hidden] + ([self.head["G"]] if self.head and not by_vocab else []))
        if by_vocab:
            H = self.head
            self.G_head_all = dp.allgather_rows(H["G"][:H["Vr"]], H["rows"])

    def stage_times(self, n_steps):
        """Mean ms per stage over the timed steps."""
        out = np.zeros(len(self.stage_names))
        for s in range(n_steps):
            e = self.events[s]
            for k in range(len(self.stage_names)):
                out[k] += e[k].elapsed_time(e[k + 1])
        return out / n_steps


def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    import torch
    world, rank, local = dist_setup(args)
    w = I.WORKLOADS[args.workload]
    K = args.draws or w.K
    peaks = load_peaks()
    step = Step(w, K, rank, world, fused=args.fused, shard=args.shard)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    step.make_events(args.steps)
    gpu_id = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for s in range(args.steps):
            step.run(s)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_total = max_over_ranks(t0.elapsed_time(t1), world)
    ms_step = ms_total / args.steps
    value = step.total_units() / (ms_step / 1e3)
    stages = step.stage_times(args.steps)
    clocks = clk.summary()

    ceiling = noise_ceiling(step, K)
    kernels = kernel_report(step, stages, peaks, clocks, ceiling)
    dominant = max((k for k in kernels if not k.get("idle")), key=lambda k: k["ms"])
    e2e = None if args.no_e2e else e2e_run(step, args, world)
    # every tcgen05 / fused kernel records a run-out bounded wait in its workspace's status word:
    # read them all back, so that an aborted kernel cannot pass for a fast one
    from activation_perturbation_es_b200 import dust
    try:
        status = dust.poll_all()
    except dust.DustError as e:
        status = f"error: {e}"
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, K)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": step.scaling(),
            "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded)",
            "config": workload_config(w, K, world, args.shard, args.fused),
            "arithmetic": "f32 noise, cross entropy and reductions; bf16 GEMM operands with f32 accumulation in "
                          "TMEM (tcgen05)",
            "roofline": {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
            | {"kernel": dominant["name"], "clock_mhz_for_peak": dominant.get("clock_mhz_for_peak"),
               "peak_source": dominant.get("peak_source"),
               "fma_heavy_pipe": dominant.get("fma_heavy_pipe"),
               "noise_ceiling_frac": dominant.get("noise_ceiling_frac")},
            "noise_ceiling": ceiling,
            "kernels": kernels,
            "layers": layer_report(step, stages),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step(step) * args.steps,
            "clocks": clocks,
            "status": status,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if status != "ok":
        sys.exit(f"bench: device status word set ({status}): the timed kernels did not all complete")


def launches_per_step(step):
    """Kernels of this library launched per step (counted from the call sequence)."""
    n = 0
    for L in step.hidden:
        n += 1                                   # reward scan
        if L["fused"]:
            n += 2                               # fused reduction + weight GEMM, split reduction
            continue
        n += 1                                   # draw reduction
        n += 1 if step.dust.lib().dust_weight_grad_workspace(step.w.T, L["hl"].d_in, L["hl"].d_out, 1, 1) <= 256 else 2
    if step.head:
        n += 1                                   # logits GEMM
        Vr = step.head["Vr"]
        if Vr:
            n += 2                               # row stats + chunk passes
            n += 1 if step.dust.lib().dust_weight_grad_workspace(step.w.T, step.w.head_d, Vr, 1, 1) <= 256 else 2
    return n


def load_traffic():
    """ncu DRAM bytes per unit from profiles/traffic.txt, for kernels whose
    source files ('+'-joined, hashed in order) are unchanged since the capture
    (sha1 prefix match); else absent.  A kernel may have several lines, one per
    unit its traffic grows with (e.g. r per draw x token, g per token x
    channel); returns {kernel: [(bytes_per_unit, unit), ...]}."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    out = {}
    if not os.path.exists(path):
        return out
    for ln in open(path):
        if ln.startswith("#") or not ln.strip():
            continue
        kernel, per_unit, unit, src, sha = ln.split()
        h = hashlib.sha1()
        try:
            for f in src.split("+"):          # the kernel's file and the headers it inlines
                h.update(open(os.path.join(ROOT, f), "rb").read())
        except OSError:
            continue
        cur = h.hexdigest()[:len(sha)]
        if cur == sha:
            out.setdefault(kernel, []).append((float(per_unit), unit))
    return out


def traffic_bytes(terms, K, T, d_out):
    """Per-launch DRAM bytes from per-unit terms (None when a term's unit is unknown)."""
    counts = {"draw_x_token": float(K) * T, "token_x_out_channel": float(T) * d_out,
              "token_x_vocab": float(T) * d_out}
    if not terms or any(u not in counts for _, u in terms):
        return None
    return sum(b * counts[u] for b, u in terms)


def layer_report(step, stages):
    """The metric per layer step: draws x tokens over the layer's own stages (a hidden layer: scan, reduction and
    weight estimate; the head: logits, its chunk passes and weight estimate), on this rank."""
    per = {}
    for name, ms in zip(step.stage_names, stages):
        layer = name.split(":")[0]
        per[layer] = per.get(layer, 0.0) + float(ms)
    out = []
    for layer, ms in per.items():
        draws = step.head["draws"] if layer == "head" else step.draws
        units = draws * step.w.T * (step.head["Vr"] / step.w.V if layer == "head" else 1)
        out.append({"layer": layer, "ms": ms, "draws_x_tokens_per_s": units / (ms / 1e3) if ms > 0 else None})
    return out


def noise_ceiling(step, K):
    """The generator's empirical ceiling on this GPU: dust_noise_sum (every
    Gaussian regenerated and consumed by one fma, nothing read from HBM) on the
    step's widest noise shape, min(K, 256) draws, timed with CUDA events after
    3 warm-up launches.  It overwrites that layer's g buffer, outside the timed
    region."""
    import torch
    dust, w = step.dust, step.w
    if step.hidden:
        L = max(step.hidden, key=lambda L: L["hl"].d_out)
        out, d, layer = L["g"], L["hl"].d_out, L["hl"].layer
    elif step.head and step.head["Vr"]:
        out, d, layer = step.head["g"], step.head["Vr"], w.head_layer
    else:
        return None
    kc = min(K, 256)
    nz = dust.Noise(w.seed, layer, 0, kc, kc, w.sigma)
    for _ in range(3):
        dust.noise_sum(nz, w.T, d, out=out)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 3
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n):
        dust.noise_sum(nz, w.T, d, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    return {"kernel": "noise_sum_kernel", "gaussians_per_s": kc * w.T * d / (ms / 1e3), "ms": ms,
            "draws": kc, "tokens": w.T, "channels": d,
            "what": "the noise generator alone, each Gaussian consumed by one fma; the ALU-bound kernels' "
                    "noise_ceiling_frac is their elements/s over this"}


def peak_source(peaks, key, what):
    if key in peaks.get("measured_keys", ()):
        return f"of measured: MEASURED_PEAKS.json {key} ({what})"
    return f"of fallback: {FALLBACK_PEAKS[key]:g} from the profiling recipe ({what}); MEASURED_PEAKS.json had none"


def kernel_report(step, stages, peaks, clocks, ceiling=None):
    w, T = step.w, step.w.T
    f_peak = peaks["sm_max_mhz"]
    alu_peak = 148 * LANES_PER_SM * f_peak * 1e6 / 1e12          # T lane-slots/s
    out = []
    names = step.stage_names
    traffic = load_traffic()
    for name, ms in zip(names, stages):
        layer, kind = name.split(":")
        rec = {"name": name, "ms": float(ms)}
        # this rank's share: its draws, and for the head its vocabulary range
        if layer == "head":
            d_in, d_out, K = w.head_d, (w.V if kind == "logits" else step.head["Vr"]), step.head["draws"]
        else:
            hl = next(h for h in w.hidden if h.name == layer)
            d_in, d_out, K = hl.d_in, hl.d_out, step.draws
        if d_out == 0 or ms <= 0:
            rec["idle"] = True                   # a rank with no head chunks
            out.append(rec)
            continue
        if kind == "scan":
            byts = 8.0 * K * T
            ach = byts / (ms / 1e3) / 1e9
            rec |= {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes": byts,
                    "peak_source": peak_source(peaks, "hbm_gbs", "copy bandwidth")}
        elif kind == "fused_estimate_wgrad":
            # ALU-bound like the reduction it contains; the GEMM's flops ride on the tensor pipe alongside
            slots = float(K) * T * d_out * SLOTS_A5
            ach = slots / (ms / 1e3) / 1e12
            f_peak = peaks["sm_max_mhz"]
            rec |= {"bound": "alu", "achieved": ach, "peak": alu_peak, "unit": "T lane-slots/s",
                    "frac": ach / alu_peak, "traffic": None, "algorithmic_slots": slots,
                    "slots_per_element": SLOTS_A5, "clock_mhz_for_peak": f_peak,
                    "gaussians_per_s": float(K) * T * d_out / (ms / 1e3),
                    "gemm_tflops": 2.0 * T * d_in * d_out / (ms / 1e3) / 1e12,
                    "peak_source": "148 SMs x 4 schedulers x 32 lanes x max SM clock"}
            if ceiling:
                rec["noise_ceiling_frac"] = rec["gaussians_per_s"] / ceiling["gaussians_per_s"]
        elif kind in ("weight_grad", "logits"):
            fl = 2.0 * T * d_in * d_out
            ach = fl / (ms / 1e3) / 1e12
            rec |= {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": ach / peaks["bf16_tflops"], "traffic": None, "algorithmic_flops": fl,
                    "peak_source": peak_source(peaks, "bf16_tflops",
                                               "cuBLAS bf16 GEMM, burst (each GEMM runs under a millisecond "
                                               "between ALU-bound kernels, at full clock)")}
        else:
            slots_el = SLOTS_HEAD if layer == "head" else SLOTS_A5
            slots = float(K) * T * d_out * slots_el
            ach = slots / (ms / 1e3) / 1e12
            tkey = "head_chunk_kernel" if layer == "head" else "layer_estimate"
            tr = traffic_bytes(traffic.get(tkey), K, T, d_out)
            # the bytes the step must move: the head reads Z (4 B per logit) and writes g in fp32 and bf16
            # (6 B); the reduction reads r (4 B per draw x token) and writes g in fp32 and bf16
            alg_bytes = 10.0 * T * d_out if layer == "head" else 4.0 * K * T + 6.0 * T * d_out
            rec |= {"bound": "alu", "achieved": ach, "peak": alu_peak, "unit": "T lane-slots/s",
                    "frac": ach / alu_peak, "traffic": tr,
                    "traffic_source": "profiles/traffic.txt (ncu capture, each term scaled by its own unit count)"
                    if tr else None,
                    "algorithmic_bytes": alg_bytes,
                    "traffic_over_algorithmic": tr / alg_bytes if tr else None,
                    "algorithmic_slots": slots,
                    "slots_per_element": slots_el, "clock_mhz_for_peak": f_peak,
                    "gaussians_per_s": float(K) * T * d_out / (ms / 1e3),
                    "peak_source": "148 SMs x 4 schedulers x 32 lanes x max SM clock (one issue slot per lane "
                                   "per clock); work = the specification's operations in their cheapest sm_100 "
                                   "instruction forms"}
            if ceiling:
                # elements (Gaussians of the reduction, perturbed logits of the head) per second over the
                # generator's own ceiling on this GPU
                rec["noise_ceiling_frac"] = rec["gaussians_per_s"] / ceiling["gaussians_per_s"]
            # the binding datapath's view of the same kernel: the specification's FMA-heavy cycles
            # against one cycle per lane per scheduler; the issue-slot fraction above cannot exceed
            # slots_per_element / heavy_cycles_per_element on sm_100
            heavy_el = HEAVY_HEAD if layer == "head" else HEAVY_A5
            rec["fma_heavy_pipe"] = {
                "cycles_per_element": heavy_el,
                "frac": float(K) * T * d_out * heavy_el / (ms / 1e3) / 1e12 / alu_peak,
                "issue_slot_frac_cap": slots_el / heavy_el}
            # and HBM's: the bytes the kernel must move over its time, against the copy bandwidth
            # (small by construction: the noise is regenerated, never read)
            gbs = alg_bytes / (ms / 1e3) / 1e9
            rec["hbm"] = {"achieved_gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
                          "peak_source": peak_source(peaks, "hbm_gbs", "copy bandwidth")}
        out.append(rec)
    return out


# ------------------------------------------------------------------ end to end
def e2e_run(step, args, world):
    """Same metric through the public API with host buffers: every step copies its
    inputs from pinned host memory and reads the weight estimates back, inside
    the timed region.  The device inputs are double-buffered: while step i
    computes on one set, a copy stream fills the other with step i + 1's inputs
    (once step i - 1 has finished reading it), and each layer's compute waits on
    an event recorded after its own inputs have landed."""
    import torch
    # per layer, in compute order: [(container, key, pinned host copy)]
    groups = []
    for L in step.hidden:
        groups.append([(L, "c", L["c"].cpu().pin_memory()), (L, "X", L["X"].cpu().pin_memory())])
    if step.head:
        groups.append([(step.head, k, step.head[k].cpu().pin_memory()) for k in ("X", "W", "y")])
    # two device sets of the inputs: the step's own tensors and a second copy of each
    sets = [[[cont[key] for cont, key, _ in g] for g in groups],
            [[torch.empty_like(cont[key]) for cont, key, _ in g] for g in groups]]
    outs = [L["G"] for L in step.hidden] + ([step.head["G"]] if step.head else [])
    outs_h = [o.cpu().pin_memory() for o in outs]
    h2d = sum(h.numel() * h.element_size() for g in groups for _, _, h in g)
    d2h = sum(o.numel() * o.element_size() for o in outs_h)
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    freed = [torch.cuda.Event(), torch.cuda.Event()]     # set k no longer read by the compute stream
    for ev in freed:
        ev.record(compute)

    def bind(k):
        for g, devs in zip(groups, sets[k]):
            for (cont, key, _), d in zip(g, devs):
                cont[key] = d

    def copy_in(k):
        copy.wait_event(freed[k])
        ready = []
        with torch.cuda.stream(copy):
            for g, devs in zip(groups, sets[k]):
                for (_, _, host), d in zip(g, devs):
                    d.copy_(host, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy)
                ready.append(ev)
        return ready

    def run(n):
        copy.wait_stream(compute)                          # nothing is copied before the region starts
        ready = copy_in(0)
        for i in range(n):
            nxt = copy_in((i + 1) % 2) if i + 1 < n else None
            bind(i % 2)
            step.run_overlapped(ready)
            freed[i % 2].record(compute)
            for o, oh in zip(outs, outs_h):
                oh.copy_(o, non_blocking=True)
            ready = nxt

    run(2)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, min(args.steps, 3))
    barrier(world)
    torch.cuda.synchronize()
    t0.record(compute)
    run(n)
    t1.record(compute)
    torch.cuda.synchronize()
    barrier(world)
    bind(0)
    del sets
    ms = max_over_ranks(t0.elapsed_time(t1), world) / n
    return {"value": step.total_units() / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": n,
            "copies": "pinned host -> device on a copy stream into double-buffered inputs: step i + 1's copies "
                      "overlap step i's compute, layer by layer"}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(w: I.Workload, K: int, n_tok: int):
    """Times the CPU oracle on a bounded sample of one step: for every layer, the
    error estimate of n_tok tokens over all K draws and all output channels (and,
    for hidden layers, their rewards from c).  Returns (seconds, draws x tokens
    processed, extrapolated seconds for the full step)."""
    import oracle
    rs = np.random.Generator(np.random.PCG64(0))
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    toks = np.sort(rs.choice(w.T, n_tok, replace=False)).astype(np.int32)
    t_sample, units, t_full = 0.0, 0, 0.0
    for hl in w.hidden:
        # costs for the sampled tokens' sequences only (the rest of c is never read)
        c = np.zeros((K, w.T), np.float32)
        c[:, toks] = I.normal((K, n_tok), w.sigma, seed=hl.layer)
        t = time.perf_counter()
        oracle.layer_estimate(c, False, hl.d_out, off, w.gamma, w.seed, hl.layer, 0, K, w.sigma, toks)
        dt = time.perf_counter() - t
        t_sample += dt
        units += K * n_tok
        t_full += dt * w.T / n_tok
    if w.V:
        Z = I.normal((n_tok, w.V), 1.0, seed=99)
        y = I.targets(n_tok, w.V, seed=98)
        t = time.perf_counter()
        oracle.head_step(Z, y, toks, w.Vc, w.seed, w.head_layer, 0, K, K, w.sigma, want_c=False)
        dt = time.perf_counter() - t
        t_sample += dt
        units += K * n_tok
        t_full += dt * w.T / n_tok
    return t_sample, units, t_full


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


CPU_SAMPLE_SECONDS = 15.0


def cpu_baseline(w, K):
    """The oracle on a bounded sample sized for about CPU_SAMPLE_SECONDS of host
    work: a probe of one token per host thread, then a multiple of the thread
    count (the oracle runs tokens in parallel) scaled to the target."""
    cores = cpu_cores()
    n0 = max(1, min(w.T, cores))
    t0, _, _ = oracle_sample(w, K, n0)
    n_tok = int(n0 * CPU_SAMPLE_SECONDS / max(t0, 1e-3))
    n_tok = max(n0, min(w.T, 4096, (n_tok // cores) * cores))
    t_s, units, t_full = oracle_sample(w, K, n_tok)
    n_layers = len(w.hidden) + (1 if w.V else 0)
    return {"value": n_layers * K * w.T / t_full, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_tok} sampled tokens per layer x all {K} draws x all channels "
                      f"({len(w.hidden)} hidden layers + head), {t_s:.1f} s, extrapolated linearly in tokens",
            "sample_seconds": t_s}


def reference_arm(args):
    """The CPU oracle as the reference arm: each step is a bounded sample of the
    workload timed on the host cores; other ranks exit without work."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = I.WORKLOADS[args.workload]
    K = args.draws or w.K
    cores = cpu_cores()
    n_tok = max(1, min(128, cores))          # one sampled token per host thread and layer
    for _ in range(args.warmup):
        oracle_sample(w, K, max(1, cores // 4))
    t_s, t_full, units = 0.0, 0.0, 0
    for _ in range(args.steps):
        a, u, f = oracle_sample(w, K, n_tok)
        t_s += a
        units += u
        t_full += f
    n_layers = len(w.hidden) + (1 if w.V else 0)
    value = n_layers * K * w.T * args.steps / t_full
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_full / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic", "config": workload_config(w, K, world, args.shard, args.fused),
            "arithmetic": "the oracle: float64 accumulation, binary32 noise",
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": cores,
                             "sample": f"{n_tok} tokens per layer per step, all draws and channels, "
                                       f"extrapolated linearly in tokens"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
