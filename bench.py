"""Benchmark of the block-sparse attention hot path (forward + backward).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload NAME] [--dropout RATE [--dropout-seed S]]
                [--mask-queries]

One step = one forward + backward pass of the whole hot path over one batch
of the named synthetic workload (default: BigBird-large attention layer at
L=4096: B=4, H=16, block 64, d=64, r=3, bf16).  For N > 1 (torchrun) every
rank runs its own batch (weak scaling: batches are independent, there is no
collective in the data path); the timed region is bracketed by a barrier and
a synchronize on both sides and the slowest rank's device time is reported.

Rank 0 prints one JSON line.  `value` is tokens/s over all ranks with inputs
resident in HBM, timed with CUDA events; between timed steps the L2 is
flushed by writing a 256 MiB buffer outside the timed events.  `e2e` is the
same metric through the public API with pinned host buffers: host->device
copies of the inputs (and the random table build), the two calls, and
device->host copies of all results inside the timed region.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_bwd_b200 import synth  # noqa: E402

METRIC = ("block-sparse attn fwd+bwd tokens/s and attended TFLOP/s at "
          "L=4096 (% bf16 TC peak)")
DEFAULT_WORKLOAD = "large_train_l4096"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}

# DRAM bytes per launch from one ncu capture, keyed by kernel name: (bytes,
# sha256 prefix of the kernel's source file and the shared headers when
# captured, that file, the workload captured).  Another workload or a
# changed source reports null.
NCU_TRAFFIC = {
    # profiles/tc_kernels_large_train_l4096.md (BigBird-large step, one
    # launch each, captured on the sources these hashes describe)
    "tc_fwd": (120852736 + 16990208, "e1206fd0b08f0603", "tc_fwd.cu",
               "large_train_l4096"),
    "tc_dq": (200619264 + 23349248, "9cad32704d22b2fb", "tc_bwd.cu",
              "large_train_l4096"),
    "tc_dkdv": (178125568 + 40513792, "9cad32704d22b2fb", "tc_bwd.cu",
                "large_train_l4096"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=10)
    # Seeded attention dropout on the attended probabilities (rate in [0, 1);
    # 0, the default, is the plain operation the headline line times).
    ap.add_argument("--dropout", type=float, default=0.0)
    ap.add_argument("--dropout-seed", type=int, default=0)
    # With dropout: draw the keep decisions in every pass instead of having
    # the forward store them for the backward (the default).
    ap.add_argument("--redraw-dropout", action="store_true")
    # With a masked workload: the key mask also zeroes the output rows of
    # padding tokens (off by default).
    ap.add_argument("--mask-queries", action="store_true")
    # Profiling runs (ncu) only: leave out the end-to-end and CPU legs.
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    # Leave out the sub-records (the other workloads and the sweep, timed
    # after the headline on rank 0).
    ap.add_argument("--skip-sub", action="store_true")
    # Time only the layer's projections (BigBird-large widths); for profiling.
    ap.add_argument("--proj-only", action="store_true")
    # Sweep mode: one line per (L, block, r) point of the length / block /
    # random-count sweep (B*L = 32768 tokens, H = 12), then the linear-in-L
    # check; not the headline line.
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--sweep-steps", type=int, default=20)
    return ap.parse_args()


def workload(name):
    if name in synth.WORKLOADS:
        return dict(synth.WORKLOADS[name])
    if name == "base_train_l4096":
        # The BigBird-base layer's padded batch through a training step,
        # with the key mask also masking the query side.
        cfg = dict(synth.WORKLOADS["base_fwd_l4096"])
        cfg["passes"] = "fwd+bwd"
        cfg["mask_queries"] = 1
        return cfg
    if name.startswith("sweep_"):  # sweep_L_bs_r
        _, L, bs, r = name.split("_")
        return synth.sweep_point(int(L), int(bs), int(r))
    raise SystemExit(f"unknown workload {name}")


def pairs_per_head(nb, table_h):
    """Attended (query block, key block) pairs of one head: nb for each of
    the two global rows, and for middle rows the size of the set
    {0, nb-1, i-1, i, i+1} U rand(i)."""
    total = 0
    for i in range(nb):
        if i == 0 or i == nb - 1:
            total += nb
        else:
            s = {0, nb - 1, i - 1, i, i + 1}
            s.update(int(j) for j in table_h[i] if 0 <= j < nb)
            total += len(s)
    return total


def valid_key_fraction(nb, bs, table, key_mask):
    """Share of the pattern's attended (query, key) products whose key is
    not masked: per batch row b, each attended block pair counts the valid
    keys of its key block instead of bs.  1.0 without a mask."""
    if key_mask is None:
        return 1.0
    km = key_mask.numpy().astype(bool)
    B = km.shape[0]
    valid = km.reshape(B, nb, bs).sum(axis=2)  # [B, nb] valid keys per block
    full = got = 0
    for h in range(table.shape[0]):
        for i in range(nb):
            if i == 0 or i == nb - 1:
                blocks = range(nb)
            else:
                s = {0, nb - 1, i - 1, i, i + 1}
                s.update(int(j) for j in table[h, i] if 0 <= j < nb)
                blocks = sorted(s)
            for j in blocks:
                full += B * bs
                got += int(valid[:, j].sum())
    return got / full


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_hash(path):
    """Hash of a kernel source and the headers every kernel includes, so a
    recorded ncu figure stops applying once any of them changes."""
    csrc = os.path.dirname(path)
    h = hashlib.sha256()
    for p in [path] + [os.path.join(csrc, n) for n in
                       ("tc_common.cuh", "sm100.cuh", "common.cuh",
                        "dropout.cuh")]:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}",
                 f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0],
                                                   "%Y/%m/%d %H:%M:%S"))
                    rows.append((ts, float(parts[2]), float(parts[3]),
                                 parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = [r for r in rows if t0 - 1 <= r[0] <= t1 + 1] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[k] for r in inside
                          for k, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


def smi_id(local):
    """nvidia-smi --id for this rank's device (UUID survives remapping by
    CUDA_VISIBLE_DEVICES)."""
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


def init_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if args.impl == "reference":
            return world, rank, local  # rank 0 alone runs the CPU oracle
        torch.cuda.set_device(local)
        dist.init_process_group("nccl",
                                timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value, world, device=None):
    """Largest `value` over all ranks (the slowest rank's time); identity on
    one rank.  Works with the nccl (CUDA tensors) or gloo (CPU) backend."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank, steps, max_total_ms, world):
    """Whole-job throughput: tokens of all ranks over the slowest rank's
    device time (weak scaling: every rank runs its own batch)."""
    return tokens_per_rank * world * steps / (max_total_ms / 1e3)


def algorithmic(cfg, pairs_total, keep_bits=False):
    """Algorithmic FLOPs and bytes per launch of each kernel kind.
    keep_bits: the forward stores one dropout keep bit per attended element
    and the two backward passes read them."""
    B, H, L, d, bs = cfg["B"], cfg["H"], cfg["L"], cfg["d"], cfg["block_size"]
    e = 2 if cfg["dtype"] == "bf16" else 4
    rows = B * H * L
    elems = rows * d
    unit = pairs_total * bs * bs * d  # one bs x bs x d contraction per pair
    kb = pairs_total * bs * bs // 8 if keep_bits else 0
    return {
        "fwd": (4 * unit, 4 * elems * e + 4 * rows + kb),
        "bwd_pre": (0, 2 * elems * e + 4 * rows),
        "csr_build": (0, 0),
        "dq": (6 * unit, 5 * elems * e + 8 * rows + kb),
        "dkdv": (8 * unit, 6 * elems * e + 8 * rows + kb),
    }


KERNEL_KIND = {"simt_fwd": "fwd", "tc_fwd": "fwd", "simt_dq": "dq",
               "tc_dq": "dq", "simt_dkdv": "dkdv", "tc_dkdv": "dkdv",
               "bwd_pre": "bwd_pre", "csr_build": "csr_build"}


def kernel_kind(name):
    """Which algorithmic figure a launch name counts against (None for the
    small merge kernels, which have no figure of their own)."""
    return KERNEL_KIND.get(name)


def kernel_bound(name):
    if name.startswith("simt_"):
        return "alu"      # fp32 FFMA on the CUDA cores
    if name.startswith("tc_"):
        return "tensor"   # tcgen05 contractions
    return "hbm"


def run_ours(args, world, rank, local):
    from block_sparse_long_bwd_b200 import binding as bb

    cfg = workload(args.workload)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    backward = cfg["passes"] == "fwd+bwd"
    dt = synth.torch_dtype(cfg["dtype"])
    B, H, L, bs, r = cfg["B"], cfg["H"], cfg["L"], cfg["block_size"], cfg["r"]
    nb = L // bs

    inp = synth.make_inputs(cfg, with_grad=backward)
    att = bb.Attention(B, H, L, bs, r, dt, d=cfg["d"], seed=synth.TABLE_SEED,
                       device=dev, dropout=args.dropout,
                       dropout_seed=args.dropout_seed,
                       mask_queries=int(args.mask_queries or cfg.get("mask_queries", 0)),
                       keep_dropout_bits=not args.redraw_dropout)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    g = inp["dout"].to(dev) if backward else None
    km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    n_fwd = bb.bb_attn_launch_count(att.desc, 0)
    n_bwd = bb.bb_attn_launch_count(att.desc, 1) if backward else 0
    names = ([bb.bb_attn_launch_name(att.desc, 0, i) for i in range(n_fwd)]
             + [bb.bb_attn_launch_name(att.desc, 1, i) for i in range(n_bwd)])
    stream = torch.cuda.current_stream()

    def step(ev_f=None, ev_b=None):
        att.forward(q, k, v, km, out=out, lse=lse, stream=stream, events=ev_f)
        if backward:
            att.backward(q, k, v, out, lse, g, km, dq=dq, dk=dk, dv=dv,
                         stream=stream, events=ev_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = bb.bb_attn_check_status(att.ws_fwd)
    if st != 0:
        raise SystemExit(f"forward status {bb.bb_status_str(st)}")

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)  # creates the underlying CUDA event
        return evs

    K = args.steps
    evf = [new_events(n_fwd + 1) for _ in range(K)]
    evb = [new_events(n_bwd + 1) for _ in range(K)] if backward else None
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(smi_id(local))
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0 = time.time()
    for s in range(K):
        flush.fill_(s & 0xFF)  # outside the step's events: evicts L2
        step(evf[s], evb[s] if backward else None)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(t0, t1)
    # Beside the cold-L2 headline: the same steps back to back without the
    # flush (inputs partly L2-resident), device time per step.
    warm_steps = min(K, 50)
    w0 = torch.cuda.Event(enable_timing=True)
    w1 = torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for s in range(warm_steps):
        step(None, None)
    w1.record(stream)
    w1.synchronize()
    warm_ms = max_over_ranks(w0.elapsed_time(w1), world, dev) / warm_steps

    per_kernel = {n: [] for n in names}
    step_ms = []
    for s in range(K):
        tot = 0.0
        evs = [(evf[s], names[:n_fwd])]
        if backward:
            evs.append((evb[s], names[n_fwd:]))
        for ev, nm in evs:
            for i, n in enumerate(nm):
                t = ev[i].elapsed_time(ev[i + 1])
                per_kernel[n].append(t)
            tot += ev[0].elapsed_time(ev[-1])
        step_ms.append(tot)
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / K
    value = aggregate_tokens_per_s(B * L, K, total_ms, world)

    # Attended FLOPs over the pattern's pairs (masked keys included).
    pairs = sum(pairs_per_head(nb, att.table_host[h].numpy())
                for h in range(H)) * B
    alg = algorithmic(cfg, pairs, keep_bits=att.dropout_bits is not None
                      and cfg["dtype"] == "bf16")
    vkf = valid_key_fraction(nb, bs, att.table_host.numpy(), inp["key_mask"])
    fwd_flops = 4 * pairs * bs * bs * cfg["d"]
    bwd_flops = 10 * pairs * bs * bs * cfg["d"] if backward else 0
    avg = {n: sum(v_) / len(v_) for n, v_ in per_kernel.items()}
    # Device time per step of each launch name: a name launched more than
    # once per step (the dK/dV pass at long lengths) is rated over the sum.
    step_t = {n: sum(v_) / K for n, v_ in per_kernel.items()}
    share = {n: sum(per_kernel[n]) / sum(step_ms) for n in names}
    dom = max(names, key=lambda n: sum(per_kernel[n]))
    peaks, peak_src = load_peaks()
    fl, by = alg.get(kernel_kind(dom), (0, 0))
    dur_s = step_t[dom] / 1e3
    bound = kernel_bound(dom)
    if bound == "tensor":
        unit, achieved = "TFLOP/s", fl / dur_s / 1e12
        peak, how = peaks["bf16_tflops"], "bf16 dense, burst"
    elif bound == "alu":
        unit, achieved = "TFLOP/s", fl / dur_s / 1e12
        # fp32 FFMA: 148 SMs x 128 lanes x 2 FLOP per clock at max SM clock.
        peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        how = "fp32 FFMA, derived from unit counts and max clock"
    else:
        unit, achieved = "GB/s", by / dur_s / 1e9
        peak, how = peaks["hbm_gbs"], "HBM copy"
    traffic = None
    tr = NCU_TRAFFIC.get(dom)
    if (tr is not None and args.workload == tr[3] and not args.dropout and
            not args.mask_queries and
            tr[1] == src_hash(os.path.join(ROOT, "block_sparse_long_bwd_b200",
                                           "csrc", tr[2]))):
        traffic = tr[0]
    # NVIDIA's dense datasheet figures, for context beside the measured peak.
    datasheet = {"TFLOP/s": 2250.0, "GB/s": 7700.0}.get(unit)
    roofline = {"bound": bound, "achieved": round(achieved, 2),
                "peak": round(peak, 1), "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "kernel": dom, "peak_source": f"{peak_src}: {how}",
                "frac_of_datasheet": (round(achieved / datasheet, 4)
                                      if datasheet and bound != "alu" else None)}
    kernels = {n: {"avg_ms": round(avg[n], 5), "share": round(share[n], 4),
                   "launches": len(per_kernel[n]),
                   "tflops": (round(alg[kernel_kind(n)][0] / (step_t[n] / 1e3)
                                    / 1e12, 2)
                              if alg.get(kernel_kind(n), (0, 0))[0] else None),
                   "gbs": (round(alg[kernel_kind(n)][1] / (step_t[n] / 1e3)
                                 / 1e9, 1)
                           if alg.get(kernel_kind(n), (0, 0))[1] else None)}
               for n in names}

    e2e = None if args.skip_e2e else run_e2e(args, cfg, att, inp, dev,
                                             backward, world)
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "warm_ms_per_step": round(warm_ms, 5),  # no L2 flush between steps
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg["dtype"],
        "data": "synthetic (seeded N(0,1) inputs, no dataset)",
        "config": {"workload": args.workload, "B": B, "H": H, "L": L,
                   "block_size": bs, "d": cfg["d"], "r": r,
                   "mask": cfg["mask"], "passes": cfg["passes"],
                   "dropout": args.dropout,
                   "dropout_keep_bits": ("stored by the forward"
                                         if att.dropout_bits is not None
                                         else "drawn in every pass")
                   if args.dropout else None,
                   "mask_queries": bool(args.mask_queries or cfg.get("mask_queries", 0)),
                   "global_batch": B * world, "seq_len": L,
                   "parallelism": f"replicas x{world} (independent batches)",
                   "l2": "flushed between steps (256 MiB write, untimed)"},
        "attended_tflops": {
            "fwd": round(fwd_flops * world / (sum(sum(per_kernel[n]) for n in names[:n_fwd]) / K / 1e3) / 1e12, 2),
            "fwd_bwd": round((fwd_flops + bwd_flops) * world / (ms_per_step / 1e3) / 1e12, 2),
            "convention": "4*bs^2*d per attended block pair fwd, 10*bs^2*d bwd",
            "pairs": pairs,
            # the same rates counting only products with an unmasked key
            "valid_key_fraction": round(vkf, 4),
            "fwd_valid_keys": round(vkf * fwd_flops * world / (sum(sum(per_kernel[n]) for n in names[:n_fwd]) / K / 1e3) / 1e12, 2)},
        "roofline": roofline,
        "kernels": kernels,
        "gpu_launches": K * (n_fwd + n_bwd),
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and not args.skip_sub and args.workload == DEFAULT_WORKLOAD:
        result["sub"] = sub_records(dev, peaks)
    if rank == 0:
        result["cpu_baseline"] = None if args.skip_cpu else cpu_baseline(
            cfg, att.table_host.numpy(), backward, budget_s=12.0,
            dropout=(args.dropout, args.dropout_seed),
            mask_queries=args.mask_queries)
        print(json.dumps(result), flush=True)


def run_e2e(args, cfg, att, inp, dev, backward, world):
    """Same metric through the public API from pinned host buffers, as a
    streaming user would run it: every step builds its random table on the
    host, copies its inputs host->device, runs the forward (+ backward) and
    copies all results device->host; the copies of step s+1 (in) and s-1
    (out) run on their own streams while step s computes (inputs, outputs
    and the pinned table double-buffered; events order the buffers)."""
    from block_sparse_long_bwd_b200 import binding as bb

    B, H, L, bs, r = cfg["B"], cfg["H"], cfg["L"], cfg["block_size"], cfg["r"]
    nb = L // bs
    names = ["q", "k", "v"] + (["dout"] if backward else [])
    host = {n: inp[n].pin_memory() for n in names}
    km_h = None if inp["key_mask"] is None else inp["key_mask"].pin_memory()
    outs = ["out", "lse"] + (["dq", "dk", "dv"] if backward else [])

    def dev_outs():
        o = {"out": torch.empty_like(host["q"], device=dev),
             "lse": torch.empty((B, H, L), dtype=torch.float32, device=dev)}
        if backward:
            for n in ("dq", "dk", "dv"):
                o[n] = torch.empty_like(host["q"], device=dev)
        return o

    din = [{n: torch.empty_like(host[n], device=dev) for n in names}
           for _ in range(2)]
    km_d = [None if km_h is None else torch.empty_like(km_h, device=dev)
            for _ in range(2)]
    tab_d = [torch.empty((H, nb, r), dtype=torch.int32, device=dev)
             for _ in range(2)]
    tab_h = [torch.empty((H, nb, r), dtype=torch.int32).pin_memory()
             for _ in range(2)]
    dout = [dev_outs() for _ in range(2)]
    res_h = {n: torch.empty_like(t, device="cpu").pin_memory()
             for n, t in dout[0].items()}
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    h2d += 0 if km_h is None else km_h.numel()
    h2d += tab_d[0].numel() * 4
    d2h = sum(t.numel() * t.element_size() for t in res_h.values())
    used = [False, False]

    def copy_in(s):
        i = s & 1
        if used[i]:
            ev_in[i].synchronize()       # tab_h[i]'s last copy has left
        tab_h[i].copy_(bb.bb_rand_attn_build(synth.TABLE_SEED, H, nb, r))
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(ev_comp[i])  # step s-2 no longer reads din[i]
            tab_d[i].copy_(tab_h[i], non_blocking=True)
            for n in names:
                din[i][n].copy_(host[n], non_blocking=True)
            if km_h is not None:
                km_d[i].copy_(km_h, non_blocking=True)
            ev_in[i].record(s_in)

    def compute(s):
        i = s & 1
        comp.wait_event(ev_in[i])
        if used[i]:
            comp.wait_event(ev_out[i])   # step s-2's results have been read
        x, o = din[i], dout[i]
        bb.bb_attn_fwd(att.desc, x["q"], x["k"], x["v"], km_d[i], tab_d[i],
                       o["out"], o["lse"], att.ws_fwd, comp)
        if backward:
            bb.bb_attn_bwd(att.desc, x["q"], x["k"], x["v"], o["out"], o["lse"],
                           x["dout"], km_d[i], tab_d[i], o["dq"], o["dk"],
                           o["dv"], att.ws_bwd, comp)
        ev_comp[i].record(comp)

    def copy_out(s):
        i = s & 1
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[i])
            for n in outs:
                res_h[n].copy_(dout[i][n], non_blocking=True)
            ev_out[i].record(s_out)
        used[i] = True

    def run(n):
        copy_in(0)
        for s in range(n):
            if s + 1 < n:
                copy_in(s + 1)
            compute(s)
            copy_out(s)
        torch.cuda.synchronize(dev)

    run(3)
    used[0] = used[1] = False
    n = max(2, args.e2e_steps)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    run(n)
    el = max_over_ranks(time.perf_counter() - t0, world, dev)
    return {"value": round(B * L * world * n / el, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n,
            "timing": "host wall clock over n pipelined steps (copies of "
                      "step s+1 in and s-1 out overlap the compute of s)"}


def cpu_baseline(cfg, table, backward, budget_s=12.0, max_slices=None,
                 dropout=(0.0, 0), mask_queries=False):
    """The fp64 oracle, as it stands, on (b, h) slices of the workload until
    the time budget is spent; scaled to tokens/s of the whole workload
    (each slice is 1/(B*H) of it).  dropout: (rate, seed) of the timed
    call."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()),
                    default=1)
    except Exception:
        cores = len(os.sched_getaffinity(0))
    B, H, L, bs = cfg["B"], cfg["H"], cfg["L"], cfg["block_size"]
    f = lambda x, h: x[:, h:h + 1].double().numpy()
    done, t_used = 0, 0.0
    # (b, h) slices in order, repeated if the whole workload takes less than
    # the budget, until the budget is spent.
    while t_used < budget_s and not (max_slices and done >= max_slices):
        for b in range(B):
            inp = synth.make_inputs(cfg, with_grad=backward,
                                    batch_slice=slice(b, b + 1))
            km = None if inp["key_mask"] is None else inp["key_mask"].numpy()
            for h in range(H):
                drop = (oracle.Dropout(dropout[0], dropout[1], b0=b, h0=h)
                        if dropout[0] else None)
                qm = km if mask_queries else None
                t0 = time.perf_counter()
                oracle.forward(f(inp["q"], h), f(inp["k"], h), f(inp["v"], h),
                               km, table[h:h + 1], bs, dropout=drop,
                               query_mask=qm)
                if backward:
                    oracle.backward(f(inp["q"], h), f(inp["k"], h),
                                    f(inp["v"], h), f(inp["dout"], h), km,
                                    table[h:h + 1], bs, dropout=drop,
                                    query_mask=qm)
                t_used += time.perf_counter() - t0
                done += 1
                if t_used >= budget_s or (max_slices and done >= max_slices):
                    break
            if t_used >= budget_s or (max_slices and done >= max_slices):
                break
    value = (L / H) * done / t_used  # B*L tokens per B*H slices
    return {"value": round(value, 2), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{done} (b,h) slice(s) at full L={L} (each 1/{B * H} "
                      f"of the workload), {'fwd+bwd' if backward else 'fwd'}, "
                      f"{t_used:.1f} s of oracle time"}


def run_reference(args, world, rank):
    """The oracle (the only reference implementation for this method) timed
    on the host cores, one (b, h) slice of the workload per step."""
    if rank != 0:
        return
    import oracle
    cfg = workload(args.workload)
    backward = cfg["passes"] == "fwd+bwd"
    B, H, L, bs, r = cfg["B"], cfg["H"], cfg["L"], cfg["block_size"], cfg["r"]
    table = oracle.rand_table(synth.TABLE_SEED, H, L // bs, r)
    inp = synth.make_inputs(cfg, with_grad=backward, batch_slice=slice(0, 1))
    km = None if inp["key_mask"] is None else inp["key_mask"].numpy()
    f = lambda x, h: x[:, h:h + 1].double().numpy()

    def step(s):
        h = s % H
        drop = (oracle.Dropout(args.dropout, args.dropout_seed, b0=0, h0=h)
                if args.dropout else None)
        qm = km if (args.mask_queries or cfg.get("mask_queries", 0)) else None
        oracle.forward(f(inp["q"], h), f(inp["k"], h), f(inp["v"], h), km,
                       table[h:h + 1], bs, dropout=drop, query_mask=qm)
        if backward:
            oracle.backward(f(inp["q"], h), f(inp["k"], h), f(inp["v"], h),
                            f(inp["dout"], h), km, table[h:h + 1], bs,
                            dropout=drop, query_mask=qm)

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(s)
    el = time.perf_counter() - t0
    value = (L / H) * args.steps / el
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()),
                    default=1)
    except Exception:
        cores = len(os.sched_getaffinity(0))
    sample = (f"one (b,h) slice of b=0 per step at full L={L}, "
              f"{'fwd+bwd' if backward else 'fwd'}; scaled by B*H={B * H}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 2),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) inputs)",
        "config": {"workload": args.workload, "B": B, "H": H, "L": L,
                   "block_size": bs, "d": cfg["d"], "r": r,
                   "dropout": args.dropout,
                   "mask_queries": bool(args.mask_queries or cfg.get("mask_queries", 0)),
                   "global_batch": B, "seq_len": L},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s",
                         "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def time_sweep_point(L, bs, r, steps, dev, flush, peaks):
    """fwd+bwd of one sweep point, device-timed (CUDA events around each
    step on the launching stream, L2 flushed between steps)."""
    from block_sparse_long_bwd_b200 import binding as bb

    cfg = synth.sweep_point(L, bs, r)
    B, H = cfg["B"], cfg["H"]
    inp = synth.make_inputs(cfg)
    att = bb.Attention(B, H, L, bs, r, torch.bfloat16, device=dev)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
    out = torch.empty_like(q)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    stream = torch.cuda.current_stream(dev)

    def step():
        att.forward(q, k, v, None, out=out, lse=lse, stream=stream)
        att.backward(q, k, v, out, lse, g, None, dq=dq, dk=dk, dv=dv,
                     stream=stream)

    for _ in range(3):
        step()
    tot = 0.0
    for s_ in range(steps):
        flush.fill_(s_ & 0xFF)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    ms = tot / steps
    pairs = sum(pairs_per_head(L // bs, att.table_host[h].numpy())
                for h in range(H)) * B
    # FLOPs by the FlashAttention convention: 4 (fwd) + 10 (bwd) bs^2 d per
    # attended pair.
    counted = (4 + 10) * pairs * bs * bs * cfg["d"]
    names = [bb.bb_attn_launch_name(att.desc, 0, i)
             for i in range(bb.bb_attn_launch_count(att.desc, 0))]
    return {"L": L, "block_size": bs, "r": r, "B": B,
            "ms": round(ms, 4),
            "tokens_per_s": round(B * L / (ms / 1e3), 1),
            "attended_tflops": round(counted / (ms / 1e3) / 1e12, 2),
            "frac_of_peak": round(counted / (ms / 1e3) / 1e12
                                  / peaks["bf16_tflops"], 4),
            "path": "tensor" if any(n.startswith("tc_") for n in names)
                    else "cuda-core"}


def linear_in_L(rows):
    """At fixed (block, r): tokens/s over L within +-15 % of its median."""
    checks = []
    for bs in synth.SWEEP_BS:
        for r in synth.SWEEP_R:
            tp = [x["tokens_per_s"] for x in rows
                  if x["block_size"] == bs and x["r"] == r]
            if not tp:
                continue
            med = statistics.median(tp)
            dev_ = max(abs(t / med - 1) for t in tp)
            checks.append({"block_size": bs, "r": r,
                           "max_dev_from_median": round(dev_, 3),
                           "linear_in_L": dev_ <= 0.15})
    return checks


def run_sweep(args):
    """fwd+bwd tokens/s and attended TFLOP/s per sweep point, one JSON line
    each, then the linear-in-L check."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, _ = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows = []
    for bs in synth.SWEEP_BS:
        for r in synth.SWEEP_R:
            for L in synth.SWEEP_L:
                row = time_sweep_point(L, bs, r, args.sweep_steps, dev, flush,
                                       peaks)
                rows.append(row)
                print(json.dumps(row), flush=True)
                torch.cuda.empty_cache()
    print(json.dumps({"sweep_linear_in_L": linear_in_L(rows)}), flush=True)


def time_workload(name, steps, dev, flush):
    """Device time per step of a named workload (its own passes: forward
    only for the BigBird-base layer), per launch and in total, with the
    attended FLOP rates; L2 flushed between steps."""
    from block_sparse_long_bwd_b200 import binding as bb

    cfg = workload(name)
    backward = cfg["passes"] == "fwd+bwd"
    B, H, L, bs, r = cfg["B"], cfg["H"], cfg["L"], cfg["block_size"], cfg["r"]
    inp = synth.make_inputs(cfg, with_grad=backward)
    att = bb.Attention(B, H, L, bs, r, synth.torch_dtype(cfg["dtype"]),
                       d=cfg["d"], device=dev, mask_queries=cfg.get("mask_queries", 0))
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    g = inp["dout"].to(dev) if backward else None
    km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    n_fwd = bb.bb_attn_launch_count(att.desc, 0)
    n_bwd = bb.bb_attn_launch_count(att.desc, 1) if backward else 0
    names = ([bb.bb_attn_launch_name(att.desc, 0, i) for i in range(n_fwd)]
             + [bb.bb_attn_launch_name(att.desc, 1, i) for i in range(n_bwd)])
    stream = torch.cuda.current_stream(dev)

    def events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)
        return evs

    def step(ev_f=None, ev_b=None):
        att.forward(q, k, v, km, out=out, lse=lse, stream=stream, events=ev_f)
        if backward:
            att.backward(q, k, v, out, lse, g, km, dq=dq, dk=dk, dv=dv,
                         stream=stream, events=ev_b)

    for _ in range(3):
        step()
    evf = [events(n_fwd + 1) for _ in range(steps)]
    evb = [events(n_bwd + 1) for _ in range(steps)] if backward else None
    torch.cuda.synchronize(dev)
    for s_ in range(steps):
        flush.fill_(s_ & 0xFF)
        step(evf[s_], evb[s_] if backward else None)
    torch.cuda.synchronize(dev)
    per = {n: 0.0 for n in names}
    fwd_ms = tot = 0.0
    for s_ in range(steps):
        for i, n in enumerate(names[:n_fwd]):
            per[n] += evf[s_][i].elapsed_time(evf[s_][i + 1])
        fwd_ms += evf[s_][0].elapsed_time(evf[s_][-1])
        tot += evf[s_][0].elapsed_time(evf[s_][-1])
        if backward:
            for i, n in enumerate(names[n_fwd:]):
                per[n] += evb[s_][i].elapsed_time(evb[s_][i + 1])
            tot += evb[s_][0].elapsed_time(evb[s_][-1])
    ms = tot / steps
    fwd_ms /= steps
    pairs = sum(pairs_per_head(L // bs, att.table_host[h].numpy())
                for h in range(H)) * B
    unit = pairs * bs * bs * cfg["d"]
    vkf = valid_key_fraction(L // bs, bs, att.table_host.numpy(),
                             inp["key_mask"])
    rec = {"workload": name, "passes": cfg["passes"], "steps": steps,
           "ms_per_step": round(ms, 5),
           "tokens_per_s": round(B * L / (ms / 1e3), 1),
           "attended_tflops_fwd": round(4 * unit / (fwd_ms / 1e3) / 1e12, 2),
           "valid_key_fraction": round(vkf, 4),
           "kernels_ms": {n: round(per[n] / steps, 5) for n in names}}
    if backward:
        rec["attended_tflops_fwd_bwd"] = round(14 * unit / (ms / 1e3) / 1e12, 2)
    if "tc_fwd" in per:
        rec["tc_fwd_tflops"] = round(4 * unit / (per["tc_fwd"] / steps / 1e3)
                                     / 1e12, 2)
    return rec


def time_projections(name, B, L, hidden, H, steps, dev, flush, peaks):
    """The fused Q/K/V projection and the output projection of a layer
    (x [B, L, hidden] -> q, k, v [B, H, L, 64]; o -> out [B, L, hidden]),
    device-timed with CUDA events, L2 flushed between steps; beside them the
    plain torch (cuBLAS) matmul of the same shapes, without the layout
    change, for context."""
    from block_sparse_long_bwd_b200 import binding as bb

    inp = synth.make_proj_inputs(B, L, hidden, H, seed=41)
    t = {k_: v_.to(dev) for k_, v_ in inp.items()}
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    D = 64 * H
    q = torch.empty((B, H, L, 64), dtype=torch.bfloat16, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    out = torch.empty((B, L, hidden), dtype=torch.bfloat16, device=dev)
    x2 = t["x"].view(B * L, hidden)
    o2 = q.permute(0, 2, 1, 3).reshape(B * L, D).contiguous()
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(3):
            fn()
        tot = 0.0
        for s_ in range(steps):
            flush.fill_(s_ & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / steps

    ms_qkv = timed(lambda: bb.bb_qkv_proj(t["x"], t["w_qkv"], t["b_qkv"], H, ws, q, k, v,
                                          stream=stream))
    ms_out = timed(lambda: bb.bb_out_proj(q, t["w_o"], t["b_o"], ws, out, stream=stream))
    ms_qkv_ref = timed(lambda: torch.addmm(t["b_qkv"].to(torch.bfloat16), x2, t["w_qkv"].t()))
    ms_out_ref = timed(lambda: torch.addmm(t["b_o"].to(torch.bfloat16), o2, t["w_o"].t()))
    st = bb.bb_attn_check_status(ws)
    fl_qkv = 2.0 * B * L * 3 * D * hidden
    fl_out = 2.0 * B * L * hidden * D
    tf = lambda fl, ms: round(fl / (ms / 1e3) / 1e12, 2)
    return {"workload": name, "B": B, "L": L, "hidden": hidden, "H": H, "status": st,
            "qkv_ms": round(ms_qkv, 5), "qkv_tflops": tf(fl_qkv, ms_qkv),
            "qkv_frac_of_peak": round(fl_qkv / (ms_qkv / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
            "out_ms": round(ms_out, 5), "out_tflops": tf(fl_out, ms_out),
            "out_frac_of_peak": round(fl_out / (ms_out / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
            "torch_matmul_same_shapes_ms": {"qkv": round(ms_qkv_ref, 5),
                                            "out": round(ms_out_ref, 5)}}


def sub_records(dev, peaks, sweep_steps=5):
    """The other workloads and the sweep, timed in the same run after the
    headline: the BigBird-base forward (its padded batch), the same batch
    through a training step with the query-side mask, the 16K pattern
    (fwd+bwd), the layer's projections at the BigBird-large and -base
    widths, and every sweep point with the linear-in-L verdict."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    subs = {n: time_workload(n, 10, dev, flush)
            for n in ("base_fwd_l4096", "base_train_l4096", "long_l16384")}
    subs["projections"] = [
        time_projections("bigbird_large_layer_l4096", 4, 4096, 1024, 16, 10, dev, flush, peaks),
        time_projections("bigbird_base_layer_l4096", 8, 4096, 768, 12, 10, dev, flush, peaks)]
    rows = []
    for bs in synth.SWEEP_BS:
        for r in synth.SWEEP_R:
            for L in synth.SWEEP_L:
                rows.append(time_sweep_point(L, bs, r, sweep_steps, dev, flush,
                                             peaks))
                torch.cuda.empty_cache()
    subs["sweep"] = {"steps_per_point": sweep_steps,
                     "points": [{k_: x[k_] for k_ in ("L", "block_size", "r",
                                                      "ms", "tokens_per_s",
                                                      "attended_tflops")}
                                for x in rows],
                     "linear_in_L": linear_in_L(rows)}
    return subs


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
        return
    if args.proj_only:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        peaks, _ = load_peaks()
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        print(json.dumps(time_projections("bigbird_large_layer_l4096", 4, 4096, 1024, 16,
                                          max(1, args.steps), dev, flush, peaks)), flush=True)
        return
    world, rank, local = init_dist(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
