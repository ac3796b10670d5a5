#!/usr/bin/env python
"""Throughput of the LAPLEX hot path on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sym2p24|small|phased_head|gram_image|gram_image_full|sym1e9]
                    [--n N]  (large-side size override, for profiling captures of a smaller case)

A step is one training pass of the operator on one batch: sort the anchors,
forward, backward (all gradients), and for N > 1 GPUs the all-reduce of the
anchor gradient over the data-parallel ranks (each rank owns its own batch of
vectors; the anchors are shared parameters).  The default workload is the
symmetric operator at n = 2^24 anchors, U[0, 0.05 n], B = 16 vectors.  Inputs
are seeded synthetic draws (structured_trainable_laplace_b200.inputs); every
per-step input is larger than the 126 MB L2, so no flush is needed between steps.

The line carries: value (elements/s = n * B * ranks / step time, train mode with
the re-sort), infer (cached sort), e2e (the same through host buffers, copies
included), the dominant kernel's roofline from live CUDA-event timings, clocks
sampled during the timed region, and the fp64 oracle's CPU time on a bounded
sample of the same workload.  --impl reference times that oracle alone.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from structured_trainable_laplace_b200 import inputs  # noqa: E402

METRIC = "LAPLEX matvec elements/s (fwd+bwd)"
UNIT = "elements/s"
NOMINAL_HBM_GBS = 8000.0
WARM_MOVE = 0.01          # anchor update of the warm-start line: a fifth of the mean spacing
WARM_MAX_N = 1 << 26      # the warm-start line runs on workloads up to this size
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ workloads

def make_workload(name: str, rank: int, n: int | None = None):
    """Inputs of the named workload; anchors (parameters) identical on every rank,
    vectors drawn per rank.  n overrides the large-side size of the symmetric,
    phased-head and Gram workloads (same recipe otherwise), for profiling captures
    of a smaller case."""
    gen = {
        "sym2p24": lambda s: inputs.sym_2p24_b16(s, n=n or (1 << 24)),
        "small": lambda s: inputs.sym_small_ties(s),
        "sym1e9": lambda s: inputs.sym_extreme(s, n=n or 10 ** 9),
        "phased_head": lambda s: inputs.phased_head_2p22(s, n=n or (1 << 22)),
        "gram_image": lambda s: inputs.gram_image(s, n=n or 3 * 1024 * 1024),
        "gram_image_full": lambda s: _full_gram(inputs.gram_image(s, n=n or 3 * 1024 * 1024)),
    }[name]
    w = gen(rank)
    if rank != 0:
        w0 = gen(0)
        for key in ("a", "b", "phi", "psi", "D"):
            if key in w0:
                w.arrays[key] = w0[key]
    return w


def _full_gram(w):
    """The Gram workload stepped with every gradient (gv, ga, gb, gD)."""
    w.op = "gram_full"
    w.name = w.name + "_full_backward"
    return w


def elements(w) -> int:
    """Units of the metric: scanned length x batch (the large side for rectangular ops)."""
    return w.n * w.B


def compulsory_bytes(w) -> int:
    """Each input read once and each output written once, per step (train mode), in
    the ABI's layout.  Intermediate sorted anchors and permutations count once as
    written and once as read by each consumer call."""
    n, B, k = w.n, w.B, w.k
    if w.op == "sym":
        sort = 4 * n + 8 * n
        fwd = 8 * n + 4 * n * B + 4 * n * B
        bwd = 8 * n + 8 * n * B + 4 * n * B + 4 * n
        return sort + fwd + bwd
    if w.op == "phased_transpose":
        sort = 12 * n + 12 * k
        fwd = 12 * n + 4 * n * B + 4 * k * B
        bwd = 12 * n + 4 * n * B + 4 * k * B + 4 * n * B + 8 * n + 8 * k
        return sort + fwd + bwd
    if w.op == "gram":
        sort = 12 * n + 12 * k
        fwd = 8 * n + 4 * n * B + 4 * n * B + 4 * k
        bwd = 8 * n + 4 * n * B + 4 * k
        return sort + fwd + bwd
    if w.op == "gram_full":
        sort = 12 * n + 12 * k
        fwd = 8 * n + 4 * n * B + 4 * n * B + 4 * k
        bwd = 8 * n + 8 * n * B + 4 * n * B + 4 * n + 8 * k  # v, g in; gv, ga out; gb, gD
        return sort + fwd + bwd
    raise ValueError(w.op)


# Algorithmic bytes of each kernel per training step, two ways:
#   method  the bytes of the method's own data the kernel must move (sorted anchors,
#           permutation, the input and output vectors and gradients), each counted
#           where the path reads or writes it -- the unit of the roofline fraction;
#   design  the bytes the kernel moves in this design, including its intermediates
#           (the sorted tile-major copies of the symmetric path, the radix passes'
#           key and value arrays, the bucketed single-channel outputs).
# Per step, so that kernels launched several times per step (the aggregate pass on
# x and on g, the radix passes of both sorts of a rectangular operator) are summed
# over their launches.
def _sort_bytes(m: int):
    """(method, design) per step of the radix kernels sorting m anchors (up to 8192
    the counting sort runs instead)."""
    if m <= 8192:
        return {"sort_small": (12 * m, 12 * m)}
    # hist reads a; pass 0 reads a and writes key+value, passes 1-3 read and write
    # key+value (the last writes a_sorted and perm)
    return {"radix_hist": (4 * m, 4 * m), "radix_pass": (8 * m, (12 + 3 * 16) * m)}


def _merge(*tables):
    out = {}
    for t in tables:
        for key, (m, d) in t.items():
            pm, pd = out.get(key, (0, 0))
            out[key] = (pm + m, pd + d)
    return out


def kernel_bytes_per_step(kernel: str, w):
    """(method bytes, design bytes) that `kernel` moves per training step, or None."""
    n, B, k = w.n, w.B, w.k
    if w.op == "sym":
        bucketed = B == 1 and n > (1 << 24)
        table = {
            # x (forward) and g (backward) gathered through the permutation; the
            # design also writes their sorted copies
            "sym_agg": (2 * (8 + 4 * B) * n, 2 * (8 + 8 * B) * n),
        }
        if bucketed:
            # the sweeps write sorted-order outputs; the permutation is read and the
            # outputs y, gx, ga written in original order by the bucketed unpermute
            table.update({
                "sym_fwd": (4 * n, (4 + 8 * B) * n),
                "sym_bwd": (4 * n, (4 + 12 * B + 4) * n),
                "unpermute_split": (3 * 4 * n, 3 * 2 * 16 * n),
                "unpermute_place": (3 * 4 * n, 3 * 12 * n),
            })
        else:
            table.update({
                "sym_fwd": ((8 + 4 * B) * n, (8 + 8 * B) * n),               # + the sorted copy of x read
                "sym_bwd": ((8 + 4 * B + 4) * n, (8 + 12 * B + 4) * n),      # + sorted x and g read
            })
        table = _merge(table, _sort_bytes(n))
        return table.get(kernel)
    if w.op == "phased_transpose":
        table = _merge({
            "large_accum": ((12 + 4 * B) * n, (12 + 4 * B) * n),              # s, perm, phi, x rows
            "large_expand_grad": ((12 + 8 * B + 8) * n, (12 + 8 * B + 8) * n),  # + gx rows, ga, gphi
        }, _sort_bytes(n), _sort_bytes(k))
        return table.get(kernel)
    if w.op == "gram":
        table = _merge({
            "large_accum": ((8 + 8 * B) * n, (8 + 8 * B) * n),    # paired pass: s, perm, v and g rows
            "large_expand": ((8 + 4 * B) * n, (8 + 4 * B) * n),   # y rows
        }, _sort_bytes(n), _sort_bytes(k))
        return table.get(kernel)
    if w.op == "gram_full":
        table = _merge({
            # A^T v (B channels, the apply) and the paired A^T v, A^T g (backward)
            "large_accum": ((8 + 4 * B + 8 + 8 * B) * n, (8 + 4 * B + 8 + 8 * B) * n),
            "large_expand": (2 * (8 + 4 * B) * n, 2 * (8 + 4 * B) * n),  # y and gv rows
            # the two accumulating anchor-gradient passes: upstream rows, ga (read back by the second)
            "large_accum_grad": ((2 * (8 + 4 * B + 4) + 4) * n, (2 * (8 + 4 * B + 4) + 4) * n),
        }, _sort_bytes(n), _sort_bytes(k))
        return table.get(kernel)
    return None


# ------------------------------------------------------------------ the step

class Step:
    """Device buffers and one training step of the workload through the binding."""

    def __init__(self, L, w, device, torch, tensors=None):
        self.L, self.w, self.torch = L, w, torch
        self.dev = device
        self.t = tensors if tensors is not None else \
            {key: torch.from_numpy(np.ascontiguousarray(v)).to(device) for key, v in w.arrays.items()}
        self.saved = None
        if w.op == "sym":
            self.saved = L.saved_buffer("sym", w.n, 1, w.B, device)
        elif w.op == "phased_transpose":
            self.saved = L.saved_buffer("phased_transpose", w.n, w.k, w.B, device)
        self.sorted = None

    def sort(self):
        """Sort the anchor sets.  The two sets of a rectangular operator are
        independent: b is sorted on a side stream while a is sorted on the current
        one (stream-ordered calls, joined by an event before the products), so the
        small, launch-latency-bound sort of b overlaps the large sort of a."""
        L, t, torch = self.L, self.t, self.torch
        if "b" not in t:
            self.sorted = (L.sort_anchors(t["a"]), None)
            return
        cur = torch.cuda.current_stream(self.dev)
        if getattr(self, "side", None) is None:
            self.side = torch.cuda.Stream(self.dev)
        self.side.wait_stream(cur)
        with torch.cuda.stream(self.side):
            sb = L.sort_anchors(t["b"])
        sa = L.sort_anchors(t["a"])
        cur.wait_stream(self.side)
        for x in sb:
            x.record_stream(cur)
        self.sorted = (sa, sb)

    def compute(self):
        """Forward + backward from the current sorted anchors; returns the output tensors."""
        L, t, w = self.L, self.t, self.w
        (sa, pa), sb = self.sorted[0], self.sorted[1]
        if w.op == "sym":
            y = L.apply_sym(sa, pa, t["x"], saved=self.saved)
            gr = L.backward("sym", sa, pa, t["x"], t["g"], saved=self.saved, need=("gx", "ga"))
            return {"y": y, "gx": gr["gx"], "ga": gr["ga"]}
        if w.op == "phased_transpose":
            z = L.apply_phased(sa, pa, t["phi"], sb[0], sb[1], t["psi"], t["x"], transpose=True, saved=self.saved)
            gr = L.backward("phased_transpose", sa, pa, t["x"], t["h"], b_sorted=sb[0], perm_b=sb[1], phi=t["phi"],
                            psi=t["psi"], saved=self.saved)
            return {"z": z, **gr}
        if w.op == "gram":
            y, gD = L.gram_apply(sa, pa, sb[0], sb[1], t["D"], t["v"], g=t["g"])
            return {"y": y, "gD": gD}
        if w.op == "gram_full":
            y = L.gram_apply(sa, pa, sb[0], sb[1], t["D"], t["v"])
            gr = L.gram_backward(sa, pa, sb[0], sb[1], t["D"], t["v"], t["g"])
            return {"y": y, **gr}
        raise ValueError(w.op)


def sample_clocks(stop_path: str, out_path: str):
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    try:
        return subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200"],
                                stdout=open(out_path, "w"), stderr=subprocess.DEVNULL)
    except (OSError, FileNotFoundError):
        return None


def summarize_clocks(path: str, gpu_index: int) -> dict:
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    try:
        for line in open(path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or not f[0].isdigit() or int(f[0]) != gpu_index:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
    except OSError:
        pass
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
            "samples": len(sm)}


# the source file that defines each timed kernel (its launches are named by these prefixes)
KERNEL_SOURCE = (("sym_", "sym.cu"), ("radix_", "sort.cu"), ("sort_small", "sort.cu"), ("unpermute_", "sort.cu"),
                 ("resort_", "resort.cu"), ("large_", "rect.cu"), ("side_", "rect.cu"), ("finish", "rect.cu"),
                 ("gram_", "rect.cu"))


def _code_only(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace collapsed (string
    literals kept), so that editing a comment leaves the hash unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_hash(kernel: str) -> str:
    """Hash of the code (comments removed) of the kernel's own .cu file and every
    shared header it can include."""
    csrc = os.path.join(ROOT, "structured_trainable_laplace_b200", "csrc")
    own = next((f for pre, f in KERNEL_SOURCE if kernel.startswith(pre)), None)
    files = sorted(glob.glob(os.path.join(csrc, "*.cuh")) + glob.glob(os.path.join(csrc, "*.h")) +
                   glob.glob(os.path.join(ROOT, "include", "*.h")))
    files += [os.path.join(csrc, own)] if own else sorted(glob.glob(os.path.join(csrc, "*.cu")))
    h = hashlib.sha256()
    for p in files:
        h.update(_code_only(open(p, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current sources of that kernel (a line `traffic <kernel> <workload> <bytes> <hash>`)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = source_hash(kernel)
    for line in open(path):
        f = line.split()
        if len(f) == 5 and f[0] == "traffic" and f[1] == kernel and f[2] == workload and f[4] == cur:
            return float(f[3])
    return None


def measured_peak():
    try:
        j = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(j["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ CPU oracle

def oracle_inputs(w, n_s: int):
    """A draw of n_s rows of the workload's recipe for the oracle (seed 123)."""
    if w.op == "sym":
        return inputs.symmetric(n_s, w.B, seed=123, spacing=0.05)
    if w.op == "phased_transpose":
        return inputs.phased_head(n_s, w.k, w.B, seed=123)
    return inputs.gram(n_s, max(1, int(round(w.k * n_s / w.n))), w.B, seed=123)


def oracle_pass(w, ws):
    """One step of the fp64 oracle (sort + forward + backward, as the GPU step) on
    the draw ws.  Returns (elements, seconds)."""
    import oracle
    t0 = time.perf_counter()
    if w.op == "sym":
        oracle.sym_apply(ws["a"], ws["x"])
        oracle.sym_backward(ws["a"], ws["x"], ws["g"])
    elif w.op == "phased_transpose":
        oracle.rect_apply(ws["a"], ws["b"], ws["x"], ws["phi"], ws["psi"], transpose=True)
        oracle.rect_backward(ws["a"], ws["b"], ws["x"], ws["h"], ws["phi"], ws["psi"], transpose=True)
    else:
        oracle.gram_apply(ws["a"], ws["b"], ws["D"], ws["v"])
        if w.op == "gram_full":
            oracle.gram_backward(ws["a"], ws["b"], ws["D"], ws["v"], ws["g"])
        else:
            oracle.gram_backward_D(ws["a"], ws["b"], ws["v"], ws["g"])
    return ws.n * w.B, time.perf_counter() - t0


def oracle_sample_size(w, budget_s: float) -> int:
    """Rows of the oracle sample that take about budget_s: grown from 2^14 until a
    pass takes a tenth of the budget, then scaled in proportion to the time (the
    oracle's cost is close to linear in n); at most the workload's own n."""
    n_s = 1 << 14
    while True:
        _, dt = oracle_pass(w, oracle_inputs(w, n_s))
        if n_s >= w.n:
            return w.n
        if dt >= 0.1 * budget_s:
            return int(min(w.n, max(n_s, n_s * budget_s / dt)))
        n_s = min(w.n, n_s * 4)


def oracle_sample(w, budget_s: float):
    """The oracle's throughput on a bounded sample of about budget_s.  Returns
    (elements/s, description)."""
    n_s = oracle_sample_size(w, budget_s)
    units, dt = oracle_pass(w, oracle_inputs(w, n_s))
    return units / dt, f"{w.op} n={n_s} B={w.B} (same recipe, seed 123), sort+fwd+bwd in fp64, {dt:.2f} s timed"


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------ measurement

# the other workloads measured inside the default run (nested under "configs")
NESTED = ("small", "phased_head", "gram_image", "gram_image_full", "sym1e9")


def config_of(w, args_workload: str, world: int) -> dict:
    """The line's config (the reference arm prints the same one)."""
    return {"workload": args_workload, "op": w.op, "n": w.n, "k": w.k, "B": w.B, "mode": "train (re-sort)",
            "l2": "per-step inputs > 126 MB L2, no flush" if w.n * w.B * 4 > (126 << 20)
            else "inputs fit in the 126 MB L2 (latency-bound size), no flush",
            "parallelism": f"dp{world}" if world > 1 else "1 GPU"}


def roofline_of(prof: dict, w, steps: int, workload: str, peak_gbs: float, peak_kind: str):
    """Roofline of the kernel with the largest share of the step: the method's bytes
    (and the design's) per launch over its average CUDA-event launch time."""
    if not prof:
        return None
    name, (cnt, tot_ms) = max(prof.items(), key=lambda kv: kv[1][1])
    per_step = kernel_bytes_per_step(name, w)
    if per_step is None:
        return {"kernel": name, "bound": "hbm", "achieved": None, "peak": peak_gbs, "unit": "GB/s", "frac": None,
                "traffic": None, "note": "no byte count for this kernel"}
    launches_per_step = cnt / steps
    avg_ms = tot_ms / cnt
    m_pl, d_pl = per_step[0] / launches_per_step, per_step[1] / launches_per_step
    ach = m_pl / (avg_ms * 1e-3) / 1e9
    dach = d_pl / (avg_ms * 1e-3) / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": peak_gbs, "unit": "GB/s",
            "frac": round(ach / peak_gbs, 4), "traffic": recorded_traffic(name, workload),
            "algorithmic_bytes_per_launch": int(m_pl), "bytes": "the method's own data (sorted anchors, "
            "permutation, input and output vectors and gradients) per launch",
            "design_bytes_per_launch": int(d_pl), "design_achieved": round(dach, 1),
            "design_frac": round(dach / peak_gbs, 4), "avg_launch_ms": round(avg_ms, 5),
            "launches_per_step": launches_per_step, "peak_source": peak_kind}


def measure_workload(L, st, w, workload: str, device, torch, steps: int, warmup: int, timed, peak):
    """Train (re-sort) and cached-sort timings, the per-kernel profile and the
    dominant kernel's roofline of one workload; peak device memory of its step."""
    from structured_trainable_laplace_b200 import dp

    def train_step():
        st.sort()
        return dp.allreduce_param_grads(st.compute())

    for _ in range(warmup):
        train_step()
    L.check()
    ms_train = timed(train_step, steps)
    L.check()
    st.sort()
    ms_infer = timed(lambda: dp.allreduce_param_grads(st.compute()), steps)
    L.profile_enable(True)
    ms_prof = timed(train_step, steps)
    prof = L.profile_report()
    L.profile_enable(False)
    L.check()
    comp = compulsory_bytes(w)
    return {
        "ms_per_step": round(ms_train, 4), "value": round(elements(w) / (ms_train * 1e-3), 1),
        "infer": {"ms_per_step": round(ms_infer, 4), "value": round(elements(w) / (ms_infer * 1e-3), 1)},
        "hbm": {"compulsory_bytes_per_step": comp, "achieved_gbs": round(comp / (ms_train * 1e-3) / 1e9, 1),
                "frac_of_measured": round(comp / (ms_train * 1e-3) / 1e9 / peak[0], 4),
                "frac_of_8tbs": round(comp / (ms_train * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4)},
        "roofline": roofline_of(prof, w, steps, workload, peak[0], peak[1]),
        "kernels": {k: {"launches_per_step": v[0] / steps, "ms_per_step": round(v[1] / steps, 5)}
                    for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])},
        "profiled_ms_per_step": round(ms_prof, 4),
        "gpu_launches": int(sum(v[0] for v in prof.values())),
    }, train_step


def nested_config(L, name: str, device, torch, timed, peak, steps: int) -> dict:
    """One of the other workloads, measured inside the default run: the same
    train / cached-sort / per-kernel measurement as the headline, with the peak
    device memory of its step (the inputs, outputs, sorted anchors, saved state and
    workspace).  The n = 10^9 inputs are drawn on the device (torch's seeded
    generator, the same distributions as the host recipe); the others come from the
    host recipe.  No end-to-end leg: the headline carries it."""
    gc = __import__("gc")
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(device)
    base = torch.cuda.memory_allocated(device)
    if name == "sym1e9":
        w, tensors = inputs.device_symmetric(10 ** 9, 1, device, seed=0, name="sym_n1000000000_b1")
        st = Step(L, w, device, torch, tensors)
        how = "drawn on the device (torch generator, seed 0): a ~ U[0, 0.05 n], x, g ~ N(0, 1)"
    else:
        w = make_workload(name, 0)
        st = Step(L, w, device, torch)
        how = "host recipe (structured_trainable_laplace_b200.inputs, seed 0)"
    res, _ = measure_workload(L, st, w, name, device, torch, steps, 3, timed, peak)
    res["peak_mem_gb"] = round((torch.cuda.max_memory_allocated(device) - base) / 1e9, 2)
    res["hbm_gb"] = 180
    res["config"] = config_of(w, name, 1)
    res["inputs"] = how
    res["steps"] = steps
    del st
    gc.collect()
    L.release_workspace()
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="sym2p24",
                    choices=["sym2p24", "small", "phased_head", "gram_image", "gram_image_full", "sym1e9"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU time")
    ap.add_argument("--n", type=int, default=None, help="large-side anchors (profiling captures of a smaller case)")
    ap.add_argument("--configs", default="auto", choices=["auto", "none"],
                    help="auto: the default single-GPU run also measures the other workloads (nested)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, world, rank)

    import torch
    import torch.distributed as dist
    from structured_trainable_laplace_b200 import dp, laplex as L

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    L.lib()  # fails loudly if the library is missing

    w = make_workload(args.workload, rank, args.n)
    st = Step(L, w, device, torch)
    stream = torch.cuda.current_stream(device)

    def train_step():
        st.sort()
        return dp.allreduce_param_grads(st.compute())

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    def timed(fn, steps):
        barrier()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        barrier()
        ms = e0.elapsed_time(e1) / steps
        if world > 1:
            tt = torch.tensor([ms], device=device)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ms = float(tt.item())
        return ms

    peak = measured_peak()
    for _ in range(args.warmup):
        train_step()
    L.check()

    # headline: train mode (re-sort every step), clocks sampled meanwhile
    clk_path = os.path.join("/tmp", f"laplex_clocks_{os.getpid()}.csv")
    proc = sample_clocks(None, clk_path)
    time.sleep(0.3)
    ms_train = timed(train_step, args.steps)
    time.sleep(0.2)
    if proc is not None:
        proc.terminate()
        proc.wait()
    clocks = summarize_clocks(clk_path, local)
    L.check()

    # cached sort, per-kernel profile and roofline (the same train steps again)
    head, _ = measure_workload(L, st, w, args.workload, device, torch, args.steps, 1, timed, peak)
    peak_mem = torch.cuda.max_memory_allocated(device) / 1e9  # the device-resident step

    # the same train step captured once as a CUDA graph and replayed: every call of
    # the step is stream-ordered and never synchronises, so all its launches go in
    # the graph and the host's per-launch cost leaves the timed region (one GPU:
    # a graph holding NCCL calls is not built here)
    graph = None
    if world == 1:
        # warm-up and capture on one stream, whose scratch (one more workspace) is
        # released afterwards
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            for _ in range(3):
                train_step()  # the capture stream's workspace at its full size
        stream.wait_stream(cap)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            train_step()
        ms_graph = timed(g.replay, args.steps)
        L.check()
        graph = {"value": round(elements(w) / (ms_graph * 1e-3), 1), "ms_per_step": round(ms_graph, 4),
                 "what": "the train step (sort, forward, backward) replayed as one CUDA graph"}
        del g
        L.release_workspace(cap)
        torch.cuda.synchronize(device)
        st.sort()

    # training with a warm-start re-sort: the anchors alternate between two sets
    # one update apart (a and a + WARM_MOVE * N(0, 1)); each step re-sorts from the
    # previous step's permutation, then runs the same forward + backward
    warm = None
    if w.op == "sym" and w.n <= WARM_MAX_N:
        anchors = [st.t["a"], torch.from_numpy(inputs.moved(w.arrays["a"], WARM_MOVE, seed=1)).to(device)]
        path = torch.zeros(1, dtype=torch.int32, device=device)
        paths = []
        state = {"k": 0, "perm": L.sort_anchors(anchors[0])[1]}

        def resort_only():
            state["k"] += 1
            sa, pa = L.resort_anchors(anchors[state["k"] % 2], state["perm"], path)
            state["perm"] = pa
            return sa, pa

        def warm_step():
            st.sorted = (resort_only(), None)
            return dp.allreduce_param_grads(st.compute())

        for _ in range(3):
            warm_step()
            paths.append(int(path.item()))
        L.check()
        ms_warm = timed(warm_step, args.steps)
        ms_resort = timed(resort_only, args.steps)
        L.check()
        warm = {"value": round(elements(w) * world / (ms_warm * 1e-3), 1), "ms_per_step": round(ms_warm, 4),
                "resort_ms": round(ms_resort, 4), "full_sort_ms": None,
                "move": f"anchors alternate between a and a + {WARM_MOVE} * N(0, 1) (mean spacing 0.05)",
                "paths_seen": sorted({L.RESORT_PATHS[q] for q in paths})}
        warm["full_sort_ms"] = round(timed(lambda: L.sort_anchors(anchors[0]), args.steps), 4)
        del anchors
        st.sort()

    torch.cuda.reset_peak_memory_stats(device)  # the end-to-end leg's own peak below

    # end to end through host buffers: every step copies its inputs from pinned host
    # memory to the device, runs, and copies its results back.  The steps are
    # pipelined: step k's inputs go up on one copy stream (into one of two device
    # input sets) while step k-1 computes and step k-1's results come down on a
    # second copy stream, so the two copy directions and the compute overlap.
    host_in = {key: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for key, v in w.arrays.items()}
    outs = train_step()
    host_out = {key: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for key, v in outs.items()}
    del outs
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    bufs = [st.t, {key: torch.empty_like(v) for key, v in st.t.items()}]
    free = [None, None]  # event: the last compute reading input set i has finished

    def e2e_steps(steps):
        for k in range(steps):
            b = k % 2
            with torch.cuda.stream(s_in):
                if free[b] is not None:
                    s_in.wait_event(free[b])
                for key, v in host_in.items():
                    bufs[b][key].copy_(v, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            st.t = bufs[b]
            out = train_step()
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            free[b] = ev_c
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c)
                for key, v in out.items():
                    host_out[key].copy_(v, non_blocking=True)
                    v.record_stream(s_out)
        done = torch.cuda.Event()
        done.record(s_out)
        stream.wait_event(done)

    e2e_steps(2)
    n_e2e = max(2, min(10, args.steps // 2))
    ms_e2e = timed(lambda: e2e_steps(n_e2e), 1) / n_e2e
    st.t = bufs[0]
    peak_mem_e2e = torch.cuda.max_memory_allocated(device) / 1e9  # + a second input set

    units = elements(w) * world
    value = units / (ms_train * 1e-3)
    comp = compulsory_bytes(w)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_train, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; anchors shared, vectors per rank)",
        "config": config_of(w, args.workload, world),
        "infer": {"value": round(units / (head["infer"]["ms_per_step"] * 1e-3), 1),
                  "ms_per_step": head["infer"]["ms_per_step"]},
        "hbm": {"compulsory_bytes_per_step": comp, "achieved_gbs": round(comp / (ms_train * 1e-3) / 1e9, 1),
                "frac_of_measured": round(comp / (ms_train * 1e-3) / 1e9 / peak[0], 4),
                "frac_of_8tbs": round(comp / (ms_train * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4)},
        "e2e": {"value": round(units / (ms_e2e * 1e-3), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "schedule": "copies of step k+1 and k-1 overlap step k", "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 4)},
        "roofline": head["roofline"],
        "train_warm_start": warm,
        "train_graph": graph,
        "kernels": head["kernels"],
        "profiled_ms_per_step": head["profiled_ms_per_step"],
        "gpu_launches": head["gpu_launches"],
        "clocks": clocks,
        "peak_mem_gb": round(peak_mem, 2),
        "peak_mem_e2e_gb": round(peak_mem_e2e, 2),
    }
    del bufs, host_in, host_out, st
    L.release_workspace()
    if rank == 0 and world == 1:
        v, desc = oracle_sample(w, args.cpu_budget)
        result["cpu_baseline"] = {"value": round(v, 1), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                                  "cpu": cpu_model()}
    if world == 1 and args.configs == "auto" and args.workload == "sym2p24" and args.n is None:
        result["configs"] = {}
        for name in NESTED:
            try:
                result["configs"][name] = nested_config(L, name, device, torch, timed, peak,
                                                        steps=5 if name == "sym1e9" else 20)
            except Exception as e:  # recorded in the line, not fatal to the headline
                result["configs"][name] = {"error": f"{type(e).__name__}: {e}"[:300]}
                L.release_workspace()
                torch.cuda.empty_cache()
        result["configs_note"] = ("the other workloads, measured in this run after the headline: train "
                                  "(re-sort) and cached-sort steps, per-kernel CUDA-event profile, the dominant "
                                  "kernel's roofline, peak device memory of the step against 180 GB; no "
                                  "end-to-end leg for these (the headline carries it)")
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


def reference_arm(args, world, rank):
    """The fp64 oracle, as it stands, on the host cores; rank 0 only.  Each step is
    one oracle pass (sort + forward + backward) over a fixed bounded sample of the
    workload, sized once so that the warm-up and timed steps together take about
    two minutes; ms_per_step is the measured time of one such step."""
    if rank != 0:
        return
    w = make_workload(args.workload, 0, args.n)
    per_step_s = min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup))
    n_s = oracle_sample_size(w, per_step_s)
    ws = oracle_inputs(w, n_s)
    for _ in range(args.warmup):
        oracle_pass(w, ws)
    units, secs = 0, 0.0
    for _ in range(args.steps):
        u, dt = oracle_pass(w, ws)
        units += u
        secs += dt
    v = units / secs
    ms = secs / args.steps * 1e3
    desc = (f"{w.op} n={n_s} B={w.B} per step (a bounded sample of the n={w.n} workload, same recipe, seed 123); "
            f"{args.steps} timed steps took {secs:.2f} s of fp64 sort+fwd+bwd")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.workload, world),
        "sample": {"n": n_s, "B": w.B, "elements_per_step": n_s * w.B, "timed_s": round(secs, 3)},
        "cpu_baseline": {"value": round(v, 1), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                         "cpu": cpu_model()},
        "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    main()
