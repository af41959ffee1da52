#!/usr/bin/env python
"""Throughput of the fused edge-conditioned tensor-product convolution on B200.

One step = one pass of the hot path over the NequIP-like workload (1,536 atoms, 46,080
directed edges, 32x(0e,1o,2e) -> 32x(0e,1e,1o,2e,2o), SH lmax 2, uvu, all 15 paths):
forward (tp_conv_fwd), the stable sender transpose (tp_csr_transpose) and backward with
gradients for node features and edge weights (tp_conv_bwd), all through the C ABI.
Inputs are resident in HBM; R seeded copies rotate so that one step's inputs are never
left in L2 by the previous steps (R x input bytes > 2 x L2).

Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import ctypes as C
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "edges/sec for fused TP conv fwd/fwd+bwd on 1 B200; % of HBM/FLOP roofline"
WORKLOADS = {
    "c1": "tiny correctness graph: 24 nodes x 8 incoming edges (192 edges), 4x0e+4x1o -> 4x0e+4x1o, SH lmax 1, "
          "uvu, 4 paths; forward only (a latency: the graph is far too small to load the GPU)",
    "c2": "NequIP-like: 1,536 atoms, 46,080 directed edges, 32x0e+32x1o+32x2e -> "
          "32x0e+32x1e+32x1o+32x2e+32x2o, SH lmax 2, uvu, 15 paths; step = fwd + transpose + bwd(gx, gw)",
    "c3": "SevenNet/MACE-like l=3: 4,096 atoms, ~163k edges, 64x(0e,1o,2e,3o), SH lmax 3, uvu, 34 paths; "
          "step = fwd + transpose + bwd(gx, gw)",
    "c5": "skewed degree 3-120: 8,192 atoms, ~295k edges, 32x(0e,1o,2e,3o), SH lmax 3, uvu, 34 paths; "
          "step = fwd + transpose + bwd(gx, gw, gvec) + dbwd(g_gy, g_x, g_w, g_vec)",
    "c4": "large streaming uvw: 100,000 atoms, ~3.0M edges, 128x(0e,1o,2e) -> 128x(0e,1e,1o,2e,2o), SH lmax 2, "
          "per-path 128x128 mixing, 15 paths; step = fwd + transpose + bwd(gx, gs, gW)",
    "c2-layer": "interaction layer on the c2 graph (1,536 atoms, 46,080 edges): linear 32x(0e,1o,2e) -> same, "
                "convolution (c2 paths), linear with coefficient 1/average degree -> 32x0e+64x0e+32x1o+32x2e, gate "
                "-> 32x(0e,1o,2e); step = that forward + transpose + the backward to x, both linear weights and "
                "the edge weights",
    "c2-gaunt": "spherical-grid (Gaunt) convolution on the c2 graph (1,536 atoms, 46,080 edges): 32x0e+32x1o+32x2e "
                "-> same, edge filter degrees 0..2 with per-degree radial weights, 28-point grid; step = fwd + "
                "transpose + bwd(gx, gw)",
    "c2-radial": "c2 with the radial projection fused in (1,536 atoms, 46,080 edges, c2 irreps and paths): the "
                 "edge weights formed in the kernels from the radial network's last hidden layer h[E, 64] and its "
                 "output layer W_r[64, 480]; step = fwd + transpose + bwd(gx, gh, gW_r)",
    "c3-radial": "c3 with the radial projection fused in (4,096 atoms, ~163k edges, c3 irreps and paths): h[E, 64], "
                 "W_r[64, 2176]; step = fwd + transpose + bwd(gx, gh, gW_r)",
    "c4-layer": "interaction layer on the c4 graph (100,000 atoms, ~3.0M edges): linear 128x(0e,1o,2e) -> same, uvw "
                "convolution (c4 paths, 128x128 mixing), linear with coefficient 1/average degree -> "
                "128x0e+256x0e+128x1o+128x2e, gate -> 128x(0e,1o,2e); step = that forward + transpose + the backward "
                "to x, both linear weights, the edge scalars and the mixing weights",
}


def layer_shapes(mul):
    """Gate input of the layer (scalars, gates for the two gated blocks, gated) and the gate's split."""
    return (f"{mul}x0e+{2 * mul}x0e+{mul}x1o+{mul}x2e", (f"{mul}x0e", f"{2 * mul}x0e", f"{mul}x1o+{mul}x2e"))


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c2", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the records of the other configurations measured after the headline")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--n-atoms", type=int, default=None,
                    help="same-density replica with fewer atoms (profiling small cases)")
    ap.add_argument("--order", default="random", choices=["random", "cell"],
                    help="atom labels in generation order (random) or relabelled by spatial cell")
    return ap.parse_args()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (device time is taken as the slowest rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(edges_per_replica: int, steps: int, world: int, elapsed_max_s: float) -> float:
    """Whole-job edges/s: every rank processes its own replica of the workload (weak scaling)."""
    return world * steps * edges_per_replica / elapsed_max_s


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ------------------------------------------------------------------------------------------
# Algorithmic counts (bytes a perfect kernel must move; stated in the design notes)
# ------------------------------------------------------------------------------------------

def fwd_bytes(N, E, in_dim, out_dim, nw):
    return E * (4 + 12 + 4 * nw) + 4 * N * (in_dim + out_dim) + 4 * (N + 1)


def dbwd_bytes(N, E, in_dim, out_dim, nw):
    # src/perm/colptr + vec, ggvec read, g_vec write; w, ggw read, g_w write; x, ggx, gy read,
    # g_x, g_gy write
    return E * (48 + 12 * nw) + 4 * N * (3 * in_dim + 2 * out_dim)


def uvw_bwd_flops(spec, E):
    """Useful fp32 flops of the uvw sender pass per call: per edge and output channel, the
    coupling Z_p = C (Y x gy) (2 nnz_p + 2 d2 d3 for the outer products, shared per (l2, l3)),
    the state update B_p += s_p Z_p and the scalar gradient gs_p += <xt_p, Z_p> (2 d1 each)."""
    from equivariant_tensor_product_b200.csrc.codegen import cg_nonzeros
    mul = int(spec.irreps_out.split("x")[0])
    ls_in = [int(b.split("x")[1][0]) for b in spec.irreps_in.split("+")]
    ls_sh = [int(b.split("x")[1][0]) for b in spec.irreps_sh.split("+")]
    ls_out = [int(b.split("x")[1][0]) for b in spec.irreps_out.split("+")]
    per = 0
    pairs = set()
    for (a, b, o) in spec.paths:
        l1, l2, l3 = ls_in[a], ls_sh[b], ls_out[o]
        per += 2 * len(cg_nonzeros(l1, l2, l3)) + 4 * (2 * l1 + 1)
        pairs.add((b, o))
    per += sum(2 * (2 * ls_sh[b] + 1) * (2 * ls_out[o] + 1) for (b, o) in pairs)
    return E * mul * per


def _ls(irreps):
    return [int(b.split("x")[1][:-1]) for b in irreps.split("+")]


def _cg_terms(spec):
    """Per path (l1, l2, l3, nnz) and, for the outer products the generated bodies share, the
    number of distinct index pairs used per block pair: (in, sh) -> (m1, m2) for the couplings
    C(x, Y); (sh, out) -> (m2, m3) for the transposed ones; (in, out) -> (m1, m3) for the
    direction gradient.  Pairs of an l2 = 0 block cost nothing (Y_0 = 1)."""
    from equivariant_tensor_product_b200.csrc.codegen import cg_nonzeros
    li, lsh, lo = _ls(spec.irreps_in), _ls(spec.irreps_sh), _ls(spec.irreps_out)
    paths, u_xy, u_yg, u_xg = [], {}, {}, {}
    for a, b, o in spec.paths:
        nz = cg_nonzeros(li[a], lsh[b], lo[o])
        paths.append((li[a], lsh[b], lo[o], len(nz)))
        if lsh[b] > 0:
            u_xy.setdefault((a, b), set()).update((i, j) for i, j, k, c in nz)
            u_yg.setdefault((b, o), set()).update((j, k) for i, j, k, c in nz)
            u_xg.setdefault((a, o), set()).update((i, k) for i, j, k, c in nz)
    n = lambda u: sum(len(v) for v in u.values())
    return paths, n(u_xy), n(u_yg), n(u_xg)


def fwd_flops(spec, E):
    """Useful fp32 flops of the uvu forward, per edge and channel: one product per shared
    (m1, m2) pair, then per path and m3 a chain over its CG non-zeros (2 flops each) and the
    weighted accumulation (2 per m3; the first product of a chain saves one, counted as 2 nnz
    + d3 in total)."""
    paths, uxy, _, _ = _cg_terms(spec)
    mul = int(spec.irreps_in.split("x")[0])
    return E * mul * (uxy + sum(2 * nnz + (2 * l3 + 1) for _, _, l3, nnz in paths))


def bwd_flops(spec, E, gvec):
    """uvu backward (gx, gw[, gvec]) per edge and channel: products per shared (m2, m3) pair;
    per path the chains z_m1 = sum C Y gy (2 nnz - d1), gx += w z (2 d1) and gw = <x, z>
    (2 d1 - 1); with gvec, products per shared (m1, m3) pair and per path with l2 > 0 the
    chains q_m2 = sum C x gy (2 nnz - d2) and gY += w q (2 d2).  The per-edge (not per-channel)
    direction-gradient epilogue is not counted."""
    paths, _, uyg, uxg = _cg_terms(spec)
    mul = int(spec.irreps_in.split("x")[0])
    per = uyg + sum(2 * nnz + 3 * (2 * l1 + 1) - 1 for l1, _, _, nnz in paths)
    if gvec:
        per += uxg + sum(2 * nnz + (2 * l2 + 1) for _, l2, _, nnz in paths if l2 > 0)
    return E * mul * per


def dbwd_flops(spec, E):
    """uvu double backward per edge and channel, term by term:
      g_gy: per shared (m1, m2) pair q = x Y (1) and h = ggx Y + x Y' (3); per path two chains
            over the non-zeros (t = C q, u = C h: 4 nnz - 2 d3) and acc += ggw t + w u (4 d3);
      g_x, g_w: per shared (m2, m3) pair r = Y gy and r' = Y' gy (2); per path z = C r and
            z' = C r' (4 nnz - 2 d1), g_x += ggw z + w z' (4 d1), g_w = <ggx, z> + <x, z'> (4 d1);
      g_vec: per shared (m1, m3) pair s = x gy and s' = ggx gy (2); per path with l2 > 0 the
            chains qa = C s and qb = C s' (4 nnz - 2 d2), G1 += ggw qa + w qb (4 d2), G2 += w qa
            (2 d2).
    Y' = dY[ggvec] and the per-edge SH derivative terms are per edge, not per channel, and are
    not counted."""
    paths, uxy, uyg, uxg = _cg_terms(spec)
    mul = int(spec.irreps_in.split("x")[0])
    per = 4 * uxy + 2 * uyg + 2 * uxg
    for l1, l2, l3, nnz in paths:
        per += 4 * nnz + 2 * (2 * l3 + 1)
        per += 4 * nnz + 6 * (2 * l1 + 1)
        if l2 > 0:
            per += 4 * nnz + 4 * (2 * l2 + 1)
    return E * mul * per


def uvw_fwd_cg_flops(spec, E):
    """CUDA-core flops of the uvw edge pass per edge and channel: as the uvu forward with the
    per-path scalar s[e, p] in place of w (the mixing runs on the tensor cores)."""
    return fwd_flops(spec, E)


def uvw_gemm_flops(spec, N, bwd):
    """Mixing contractions: forward 2 N sum_p d3 mul_in mul_out; backward three of the same
    size (x W, B W^T and x^T B, the last two with d1 in place of d3)."""
    li, lo = _ls(spec.irreps_in), _ls(spec.irreps_out)
    mi, mo = int(spec.irreps_in.split("x")[0]), int(spec.irreps_out.split("x")[0])
    if bwd:
        return 3 * 2 * N * sum((2 * li[a] + 1) * mi * mo for a, b, o in spec.paths)
    return 2 * N * sum((2 * lo[o] + 1) * mi * mo for a, b, o in spec.paths)


def bwd_bytes(N, E, in_dim, out_dim, nw, gvec):
    # perm + vec + w read + gw write (+ gvec write); x read, gy read, gx write; colptr + rowptr
    return E * (4 + 12 + 8 * nw + (12 if gvec else 0)) + 4 * N * (2 * in_dim + out_dim) + 8 * (N + 1)


# ------------------------------------------------------------------------------------------
# Clocks (NVML reads only; nothing is changed)
# ------------------------------------------------------------------------------------------

class ClockSampler:
    def __init__(self, index: int, period=0.05):
        self.samples, self.reasons = [], set()
        self.period = period
        self.ok = False
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # noqa: BLE001
            self.err = str(exc)
        self._stop = threading.Event()

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:  # noqa: BLE001
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        names = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}
        for bit, n in names.items():
            if r & bit:
                self.reasons.add(n)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def max_mhz_or(self, default: float) -> float:
        return float(self.max_mhz) if self.ok else default

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------
# CPU side: the float64 oracle on a bounded sample
# ------------------------------------------------------------------------------------------

def oracle_sample(d, n_rows, seed):
    """fwd on the edges into n_rows receivers, bwd on the edges leaving n_rows senders."""
    from oracle import OraclePlan, backward, forward
    spec = d["spec"]
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
    N = len(d["rowptr"]) - 1
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(N, size=min(n_rows, N), replace=False))
    rp = np.asarray(d["rowptr"], dtype=np.int64)
    eids = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in rows])
    rpf = np.concatenate([[0], np.cumsum(rp[rows + 1] - rp[rows])])
    mask = np.isin(d["src"], rows)
    eb = np.nonzero(mask)[0]
    rpb = np.concatenate([[0], np.cumsum(np.bincount(d["dst"][eb], minlength=N))])
    uvw = spec.mode == "uvw"
    wf = dict(s=d["s"][eids], W=d["W"]) if uvw else dict(w=d["w"][eids])
    wb = dict(s=d["s"][eb], W=d["W"]) if uvw else dict(w=d["w"][eb])
    t0 = time.perf_counter()
    forward(op, rpf, d["src"][eids], d["x"], d["vec"][eids], **wf)
    t1 = time.perf_counter()
    backward(op, rpb, d["src"][eb], d["x"], d["vec"][eb], d["gy"], **wb)
    t2 = time.perf_counter()
    return len(eids), t1 - t0, len(eb), t2 - t1


def cpu_edges_per_s(ef, tf, eb, tb):
    return 1.0 / (tf / ef + tb / eb)


def run_reference(args, rank):
    if rank != 0:
        return 0
    import synth
    from oracle.conv import set_threads
    cores = set_threads()
    if args.workload.endswith("-layer"):
        return run_reference_layer(args, cores)
    if args.workload == "c2-gaunt":
        return run_reference_gaunt(args, cores)
    if args.workload.endswith("-radial"):
        return run_reference_radial(args, cores)
    d = synth.make_inputs(args.workload)
    oracle_sample(d, 4, seed=0)                      # CG tables cached outside the timing
    ef, tf, eb, tb = oracle_sample(d, 16, seed=1)
    per_row = (tf + tb) / 16
    # size each step so the whole run stays near a minute of host time
    rows_per_step = int(max(2, min(256, 60.0 / max(1, args.steps + args.warmup) / per_row)))
    for k in range(args.warmup):
        oracle_sample(d, rows_per_step, seed=k)
    tot_e, tot_t = 0.0, 0.0
    per = []
    for k in range(args.steps):
        ef, tf, eb, tb = oracle_sample(d, rows_per_step, seed=1000 + k)
        per.append(cpu_edges_per_s(ef, tf, eb, tb))
        tot_t += tf + tb
        tot_e += 1.0 / (tf / ef + tb / eb) * (tf + tb)
    value = tot_e / tot_t
    sample = (f"{rows_per_step} random receivers (fwd on their incoming edges) and {rows_per_step} random "
              f"senders (bwd on their outgoing edges) per step, float64")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "name": args.workload, "N": len(d["rowptr"]) - 1,
                       "E": len(d["src"]), "order": "generation order (random)", "parallelism": "single"},
            "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------
# GPU side
# ------------------------------------------------------------------------------------------

SPEC_OF_WORKLOAD = {"c1": "l1_c1", "c2": "full_l2", "c3": "full_l3", "c4": "full_l2", "c5": "full_l3",
                    "c2-layer": "full_l2", "c4-layer": "full_l2", "c2-radial": "full_l2", "c3-radial": "full_l3"}


def kernel_source_hash(kernel="", workload="c2"):
    """Hash of the sources a kernel is built from: the edge-kernel templates and the generated
    body of the workload's path list (uvw: also its GEMM), or the transpose's own file."""
    csrc = os.path.join(ROOT, "equivariant_tensor_product_b200", "csrc")
    if kernel.startswith("k_radix") or kernel.startswith("k_colptr"):
        files = [os.path.join(csrc, "csr.cu")]
    else:
        files = [os.path.join(csrc, "tp_kernels.cuh")]
        if kernel.startswith("k_rad_"):
            files += [os.path.join(csrc, f) for f in ("radial.cuh", "radial.cu", "radial_spec.cu")]
        if "uvw" in kernel or "gemm" in kernel:
            files += [os.path.join(csrc, "tp_uvw.cuh"), os.path.join(csrc, "tp_mma.cuh")]
        spec = SPEC_OF_WORKLOAD.get(workload)
        gen = os.path.join(csrc, "gen", f"spec_{spec}.h")
        if spec and not os.path.exists(gen):
            sys.path.insert(0, csrc)
            import codegen
            sys.path.pop(0)
            codegen.main(os.path.join(csrc, "gen"))
        if spec:
            files.append(gen)
    h = hashlib.sha256()
    for f in files:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if the kernels are unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        rec = json.load(open(path))
        e = rec.get(workload, {}).get(kernel)
        if e and e.get("source_hash") == kernel_source_hash(kernel, workload):
            return e["dram_bytes_per_launch"]
    except Exception:  # noqa: BLE001
        return None
    return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p.get("hbm_gbs", 6650.0), p.get("bf16_tflops", 1590.0), "of measured"
    return 6650.0, 1590.0, "of fallback"


def tc_peak_3xtf32(bf16_tflops):
    """fp32 work through 3xTF32 on tcgen05: the TF32 rate (the measured bf16 peak times the
    nominal TF32 / bf16 ratio, 1.1 / 2.25 PFLOP/s) divided by the three MMAs per product."""
    return bf16_tflops * (1.1 / 2.25) / 3.0


def pass_roofline(ms, nbytes, flops, hbm_gbs, fp32_tflops, gemm_flops=0.0, tc_tflops=None):
    """Roofline of one call: the slowest of its algorithmic bytes at the HBM peak, its CUDA-core
    flops at the fp32 FMA peak and its tensor-core flops at the 3xTF32 peak; frac = that time
    over the measured time."""
    t = {"hbm": nbytes / (hbm_gbs * 1e9), "alu": flops / (fp32_tflops * 1e12)}
    if gemm_flops and tc_tflops:
        t["tensor"] = gemm_flops / (tc_tflops * 1e12)
    bound = max(t, key=t.get)
    sec = ms * 1e-3
    out = {"ms": ms, "bound": bound, "roofline_ms": 1e3 * t[bound], "frac": t[bound] / sec,
           "algorithmic_bytes": nbytes, "cuda_core_flops": flops, "achieved_GBps": nbytes / sec / 1e9,
           "achieved_fp32_TFLOPs": flops / sec / 1e12, "hbm_frac": t["hbm"] / sec, "alu_frac": t["alu"] / sec}
    if "tensor" in t:
        out.update({"tensor_flops": gemm_flops, "tensor_frac": t["tensor"] / sec})
    return out


def prepare_workload(tp, lib, torch, dev, name, n_atoms=None, order="random", rank=0):
    """Inputs of one convolution workload resident in HBM (R rotating seeded copies, together
    more than 2.5 x L2), its output buffers and workspaces, and the C-ABI argument tuples of
    one step: forward, the transpose on a side stream, backward (and double backward)."""
    import types
    import synth
    spec = synth.CONFIGS[name]
    with_dbwd = "dbwd" in spec.passes
    d = synth.make_inputs(name, n_atoms, with_gg=with_dbwd, seed=spec.seed + 7919 * rank)
    if order == "cell":
        d = synth.cell_sorted(d)
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
    N, E = len(d["rowptr"]) - 1, len(d["src"])
    in_dim, out_dim, nw = plan.in_dim, plan.out_dim, plan.n_edge_weights
    want_gvec = with_dbwd or name == "c5"
    uvw = spec.mode == "uvw"
    wkey = "s" if uvw else "w"
    keys = ["rowptr", "src", "x", "vec", wkey, "gy"] + (["W"] if uvw else [])
    copy_bytes = sum(d[k].nbytes for k in keys)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(2, math.ceil(2.5 * l2 / copy_bytes))
    copies = []
    for r in range(R):
        src_d = d
        if r:
            rng = np.random.default_rng(spec.seed + 31 * r + 7919 * rank)
            src_d = dict(d)
            src_d["x"] = rng.standard_normal(d["x"].shape, dtype=np.float32)
            src_d["gy"] = rng.standard_normal(d["gy"].shape, dtype=np.float32)
            src_d[wkey] = (d[wkey] * rng.uniform(0.5, 1.5, size=(1, d[wkey].shape[1]))).astype(np.float32)
        copies.append({k: torch.as_tensor(np.ascontiguousarray(src_d[k])).to(dev) for k in keys})
    y = torch.empty(N, out_dim, device=dev)
    gx = torch.empty(N, in_dim, device=dev)
    gw = torch.empty(E, nw, device=dev)
    gvec = torch.empty(E, 3, device=dev) if want_gvec else None
    # one transpose per input copy: the transpose of step k runs on a side stream while the
    # forward of step k runs on the main stream (they are independent); the backward waits
    colptrs = [torch.empty(N + 1, dtype=torch.int32, device=dev) for _ in range(R)]
    perms = [torch.empty(E, dtype=torch.int32, device=dev) for _ in range(R)]
    gW = torch.empty(plan.n_shared_weights, device=dev) if uvw else None
    ws_bytes = max(tp.tp_workspace_size(plan, N, E, tp.TP_OP_BWD), tp.tp_workspace_size(plan, N, E, tp.TP_OP_FWD),
                   tp.tp_workspace_size(plan, N, E, tp.TP_OP_DBWD) if with_dbwd else 0)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_t_bytes = max(256, tp.tp_csr_transpose_workspace_size(N, E))
    ws_t = torch.empty(ws_t_bytes, dtype=torch.uint8, device=dev)      # side-stream transpose scratch
    # the transpose's side stream runs at a higher priority, so that its few small kernels get
    # SM slots as the forward's CTAs retire instead of queueing behind all of them
    stream, side = torch.cuda.Stream(dev), torch.cuda.Stream(dev, priority=-1)
    sh, sh_side = stream.cuda_stream, side.cuda_stream
    h = plan.handle
    P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None
    argsets = []
    for r, cp in enumerate(copies):
        Wp = P(cp["W"]) if uvw else None
        argsets.append((
            (h, N, E, P(cp["rowptr"]), P(cp["src"]), P(cp["x"]), P(cp["vec"]), P(cp[wkey]), Wp, P(y), P(ws), ws_bytes,
             sh),
            (N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(ws_t), ws_t_bytes, sh_side),
            (h, N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(cp["x"]), P(cp["vec"]),
             P(cp[wkey]), Wp, P(cp["gy"]), P(gx), P(gw), P(gvec), P(gW), P(ws), ws_bytes, sh),
        ))
    dargs, dbuf = None, {}
    if with_dbwd:   # second-order upstream gradients, one set shared by the copies (each > L2)
        dbuf = {k: torch.as_tensor(np.ascontiguousarray(d[k])).to(dev) for k in ("ggx", "ggw", "ggvec")}
        dbuf.update(g_gy=torch.empty(N, out_dim, device=dev), g_x=torch.empty(N, in_dim, device=dev),
                    g_w=torch.empty(E, nw, device=dev), g_vec=torch.empty(E, 3, device=dev))
        dargs = [(h, N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(cp["x"]), P(cp["vec"]),
                  P(cp[wkey]), None, P(cp["gy"]), P(dbuf["ggx"]), P(dbuf["ggw"]), P(dbuf["ggvec"]),
                  P(dbuf["g_gy"]), P(dbuf["g_x"]), P(dbuf["g_w"]), P(dbuf["g_vec"]), P(ws), ws_bytes, sh)
                 for r, cp in enumerate(copies)]
    return types.SimpleNamespace(
        name=name, spec=spec, d=d, plan=plan, N=N, E=E, in_dim=in_dim, out_dim=out_dim, nw=nw, uvw=uvw, wkey=wkey,
        keys=keys, with_dbwd=with_dbwd, want_gvec=want_gvec, copy_bytes=copy_bytes, l2=l2, R=R, copies=copies,
        y=y, gx=gx, gw=gw, gvec=gvec, gW=gW, colptrs=colptrs, perms=perms, ws=ws, ws_bytes=ws_bytes, ws_t=ws_t,
        ws_t_bytes=ws_t_bytes, stream=stream, side=side, argsets=argsets, dargs=dargs, dbuf=dbuf, P=P,
        tr_done=[torch.cuda.Event() for _ in range(R)], bwd_done=[torch.cuda.Event() for _ in range(R)],
        order=order, dev=dev)


def eager_step(w, lib, k, ev=None):
    """One step through the C ABI: transpose (side stream), forward, backward (+ dbwd)."""
    r = k % w.R
    a_f, a_t, a_b = w.argsets[r]
    w.side.wait_event(w.bwd_done[r])          # the backward that last read this copy is done
    if ev is not None:
        ev[4].record(w.side)
    st = lib.tp_csr_transpose(*a_t)
    if ev is not None:
        ev[5].record(w.side)
    w.tr_done[r].record(w.side)
    if ev is not None:
        ev[0].record(w.stream)
    st |= lib.tp_conv_fwd(*a_f)
    if ev is not None:
        ev[1].record(w.stream)
    w.stream.wait_event(w.tr_done[r])
    if ev is not None:
        ev[2].record(w.stream)
    st |= lib.tp_conv_bwd(*a_b)
    if ev is not None:
        ev[3].record(w.stream)
    if w.with_dbwd:
        st |= lib.tp_conv_dbwd(*w.dargs[r])
        if ev is not None:
            ev[6].record(w.stream)
    w.bwd_done[r].record(w.stream)
    if st:
        raise RuntimeError(lib.tp_last_error_message().decode())


def time_eager(w, lib, torch, steps, warmup, local, world):
    """Eager steps with an event pair around every call: per-call mean times and the step time."""
    import torch.distributed as dist
    for k in range(warmup):
        eager_step(w, lib, k)
    torch.cuda.synchronize(w.dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(w.dev)
    free0 = torch.cuda.mem_get_info(w.dev)[0]
    n0 = lib.tp_launch_count()
    with ClockSampler(local) as clk:
        start.record(w.stream)
        for k in range(steps):
            eager_step(w, lib, k, evs[k])
        stop.record(w.stream)
        torch.cuda.synchronize(w.dev)
    launches = lib.tp_launch_count() - n0
    free1 = torch.cuda.mem_get_info(w.dev)[0]
    if world > 1:
        dist.barrier()
    km = {"fwd": statistics.mean(e[0].elapsed_time(e[1]) for e in evs),
          "transpose": statistics.mean(e[4].elapsed_time(e[5]) for e in evs),
          "bwd": statistics.mean(e[2].elapsed_time(e[3]) for e in evs)}
    if w.with_dbwd:
        km["dbwd"] = statistics.mean(e[3].elapsed_time(e[6]) for e in evs)
    return start.elapsed_time(stop) / 1e3, km, launches, clk, free0 - free1


def time_graphs(w, lib, torch, steps, warmup, local, world):
    """The same steps captured as one CUDA graph per input copy (transpose forked onto the side
    stream and joined before the backward) and replayed: removes the host launch path from
    between the kernels.  Returns (elapsed_s, launches, clk, note); elapsed None if capture
    failed."""
    import torch.distributed as dist
    graphs = []
    try:
        n_cap = lib.tp_launch_count()
        for r in range(w.R):
            g = torch.cuda.CUDAGraph()
            fork, join = torch.cuda.Event(), torch.cuda.Event()
            a_f, a_t, a_b = w.argsets[r]
            with torch.cuda.graph(g, stream=w.stream, capture_error_mode="thread_local"):
                fork.record(w.stream)
                w.side.wait_event(fork)
                st = lib.tp_csr_transpose(*a_t)
                join.record(w.side)
                st |= lib.tp_conv_fwd(*a_f)
                w.stream.wait_event(join)
                st |= lib.tp_conv_bwd(*a_b)
                if w.with_dbwd:
                    st |= lib.tp_conv_dbwd(*w.dargs[r])
            if st:
                raise RuntimeError(lib.tp_last_error_message().decode())
            graphs.append(g)
        per_step = (lib.tp_launch_count() - n_cap) // w.R
    except Exception as exc:  # noqa: BLE001
        return None, 0, None, f"capture failed: {exc}"[:200]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(w.stream):
        for k in range(warmup):
            graphs[k % w.R].replay()
    torch.cuda.synchronize(w.dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(w.dev)
    with ClockSampler(local) as clk:
        start.record(w.stream)
        with torch.cuda.stream(w.stream):
            for k in range(steps):
                graphs[k % w.R].replay()
        stop.record(w.stream)
        torch.cuda.synchronize(w.dev)
    if world > 1:
        dist.barrier()
    elapsed = start.elapsed_time(stop) / 1e3
    graphs.clear()   # no graph outlives the process group
    return elapsed, per_step * steps, clk, None


def pass_rooflines(w, km, hbm, fp32_peak, tc_peak):
    """Per-call rooflines of a workload: bytes and CUDA-core flops from the algorithmic counts
    above (and the mixing GEMMs for uvw)."""
    N, E, spec = w.N, w.E, w.spec
    out = {}
    if w.uvw:
        fb = fwd_bytes(N, E, w.in_dim, w.out_dim, w.nw) + 4 * w.plan.n_shared_weights
        bb = bwd_bytes(N, E, w.in_dim, w.out_dim, w.nw, w.want_gvec) + 8 * w.plan.n_shared_weights
        out["fwd"] = pass_roofline(km["fwd"], fb, uvw_fwd_cg_flops(spec, E), hbm, fp32_peak,
                                   uvw_gemm_flops(spec, N, False), tc_peak)
        out["bwd"] = pass_roofline(km["bwd"], bb, uvw_bwd_flops(spec, E), hbm, fp32_peak,
                                   uvw_gemm_flops(spec, N, True), tc_peak)
    else:
        out["fwd"] = pass_roofline(km["fwd"], fwd_bytes(N, E, w.in_dim, w.out_dim, w.nw), fwd_flops(spec, E), hbm,
                                   fp32_peak)
        out["bwd"] = pass_roofline(km["bwd"], bwd_bytes(N, E, w.in_dim, w.out_dim, w.nw, w.want_gvec),
                                   bwd_flops(spec, E, w.want_gvec), hbm, fp32_peak)
        if w.with_dbwd:
            out["dbwd"] = pass_roofline(km["dbwd"], dbwd_bytes(N, E, w.in_dim, w.out_dim, w.nw), dbwd_flops(spec, E),
                                        hbm, fp32_peak)
    return out


KERNEL_OF_PASS = {("uvu", "fwd"): "k_fwd_uvu", ("uvu", "bwd"): "k_bwd_uvu",
                  ("uvu", "dbwd"): "k_dbwd_recv + k_dbwd_send",
                  ("uvw", "fwd"): "tp_conv_fwd (uvw: k_uvw_edge_staged, mixing GEMMs)",
                  ("uvw", "bwd"): "tp_conv_bwd (uvw: k_uvw_send, x W / B W^T / x^T B GEMMs)"}


def config_record(tp, lib, torch, dev, name, steps, warmup, local, hbm, fp32_peak, tc_peak, order="random"):
    """A compact measured record of one workload in the same run: per-call times and rooflines
    (eager loop) and the step time (CUDA-graph replay)."""
    w = prepare_workload(tp, lib, torch, dev, name, order=order)
    el, km, _, clk_e, _ = time_eager(w, lib, torch, steps, warmup, local, 1)
    eg, _, clk_g, note = time_graphs(w, lib, torch, steps, warmup, local, 1)
    ms = 1e3 * (eg if eg is not None else el) / steps
    rec = {"workload": WORKLOADS[name], "N": w.N, "E": w.E, "order": "cell-sorted" if order == "cell" else
           "generation order (random)", "steps": steps, "ms_per_step": ms, "edges_per_s": w.E / (ms * 1e-3),
           "launch": "cuda_graph" if eg is not None else "eager", "eager_ms_per_step": 1e3 * el / steps,
           "kernel_ms": km, "passes": pass_rooflines(w, km, hbm, fp32_peak, tc_peak),
           "clocks": (clk_g or clk_e).summary()}
    if note:
        rec["graph_note"] = note
    del w
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return rec


def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from equivariant_tensor_product_b200 import build as tpbuild
    tpbuild.build()
    import equivariant_tensor_product_b200 as tp
    lib = tp.load()

    w = prepare_workload(tp, lib, torch, dev, args.workload, args.n_atoms, args.order, rank)
    N, E, spec, uvw = w.N, w.E, w.spec, w.uvw
    elapsed, km, launches, clk, free_drop = time_eager(w, lib, torch, args.steps, args.warmup, local, world)
    elapsed_max = max_over_ranks(elapsed, world, dev)
    eager_ms_per_step = 1e3 * elapsed_max / args.steps
    launch_mode, graph_note = "eager", None
    eg, lg, clk_g, graph_note = time_graphs(w, lib, torch, args.steps, args.warmup, local, world)
    if eg is not None:
        elapsed = eg
        elapsed_max = max_over_ranks(eg, world, dev)
        launches, clk, launch_mode = lg, clk_g, "cuda_graph"

    # End to end through the same calls: every step copies its inputs from pinned host memory
    # and its results back.  Two device buffer sets let the copies overlap: the inputs of step
    # k+1 go up and the results of step k-1 come down (each on its own copy stream) while step
    # k computes; nothing is skipped or cached between steps.
    e2e_value, h2d, d2h = run_e2e(w, lib, torch, args.e2e_steps, world)

    if rank == 0:
        hbm, bf16, peak_note = measured_peaks()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        fp32_peak = 2 * 128 * sms * clk.max_mhz_or(1965.0) * 1e6 / 1e12
        tc_peak = tc_peak_3xtf32(bf16)
        passes = pass_rooflines(w, km, hbm, fp32_peak, tc_peak)
        dom = max(passes, key=lambda k: passes[k]["ms"])
        dp = passes[dom]
        kname = KERNEL_OF_PASS[(spec.mode, dom)]
        if dp["bound"] == "hbm":
            roof = {"bound": "hbm", "kernel": kname, "achieved": dp["achieved_GBps"], "peak": hbm, "unit": "GB/s",
                    "frac": dp["achieved_GBps"] / hbm, "peak_note": peak_note,
                    "traffic": traffic_from_profile(kname, args.workload),
                    "algorithmic_bytes_per_launch": dp["algorithmic_bytes"]}
        elif dp["bound"] == "alu":
            roof = {"bound": "alu", "kernel": kname, "achieved": dp["achieved_fp32_TFLOPs"], "peak": fp32_peak,
                    "unit": "TFLOP/s", "frac": dp["achieved_fp32_TFLOPs"] / fp32_peak,
                    "peak_note": "fp32 FMA peak: 2 flop x 128 lanes x SMs x max SM clock; flops counted from the "
                                 "term lists of bench.py (fwd_flops, bwd_flops, dbwd_flops, uvw_bwd_flops)",
                    "traffic": traffic_from_profile(kname, args.workload),
                    "algorithmic_flops_per_call": dp["cuda_core_flops"], "hbm_frac": dp["hbm_frac"]}
        else:
            roof = {"bound": "tensor", "kernel": kname, "achieved": dp["tensor_flops"] / (dp["ms"] * 1e-3) / 1e12,
                    "peak": tc_peak, "unit": "TFLOP/s", "frac": dp["tensor_frac"],
                    "peak_note": f"3xTF32 from the measured bf16 peak ({peak_note})", "traffic": None}
        roof.update({"kernel_ms": km, "passes": passes,
                     "step_roofline_frac": sum(p["roofline_ms"] for p in passes.values()) /
                     (1e3 * elapsed / args.steps)})
        cpu = None
        if not args.no_cpu_baseline and not uvw:
            from oracle.conv import set_threads
            cores = set_threads()
            oracle_sample(w.d, 4, seed=0)            # CG tables cached outside the timing
            n_rows = min(N, 1536)
            ef, tf, eb, tb = oracle_sample(w.d, n_rows, seed=3)
            cpu = {"value": cpu_edges_per_s(ef, tf, eb, tb), "unit": "edges/s", "cores": cores, "kind": "oracle",
                   "sample": f"fwd on the {ef} edges into {n_rows} receivers + bwd on the {eb} edges leaving "
                             f"{n_rows} senders of the same workload (rank 0's copy), float64 torch CPU, "
                             f"{tf + tb:.1f} s"}
        value = replica_throughput(E, args.steps, world, elapsed_max)
        line = {
            "metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * elapsed_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "name": args.workload, "N": N, "E": E,
                       "order": "cell-sorted" if args.order == "cell" else "generation order (random)",
                       "launch": launch_mode, "eager_ms_per_step": eager_ms_per_step,
                       **({"graph_note": graph_note} if graph_note else {}),
                       "l2": f"{w.R} rotating input copies of {w.copy_bytes / 1e6:.1f} MB (> 2x L2 of "
                             f"{w.l2 / 1e6:.0f} MB)", "parallelism": "replicas" if world > 1 else "single"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "edges/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": args.e2e_steps,
                    "pipeline": "two device buffer sets; the H2D copy of step k+1 and the D2H copy of step k-1 "
                                "overlap step k on their own streams"},
            "gpu_launches": int(launches), "clocks": clk.summary(),
            "memory": {"workspace_bytes": w.ws_bytes, "transpose_workspace_bytes": w.ws_t_bytes,
                       "edge_sized_float_scratch_bytes": 0,
                       "device_free_bytes_lost_during_timed_steps": int(free_drop),
                       "note": "the library allocates nothing: every buffer, workspaces included, is the caller's; "
                               "the workspaces hold int32 graph indices (and, for uvw, node- and weight-sized "
                               "state), never an edge x feature float tensor"},
            "library": tp.tp_version(),
        }
        if world == 1 and not args.no_per_config and args.workload == "c2" and args.n_atoms is None:
            # the other configurations measured in the same run (compact records)
            del w
            torch.cuda.empty_cache()
            per = {}
            for name, st, wu in (("c3", 100, 5), ("c5", 30, 3), ("c4", 10, 3)):
                per[name] = config_record(tp, lib, torch, dev, name, st, wu, local, hbm, fp32_peak, tc_peak)
            for name, st, wu in (("c3", 100, 5), ("c4", 10, 3)):
                per[name + "-cell"] = config_record(tp, lib, torch, dev, name, st, wu, local, hbm, fp32_peak,
                                                    tc_peak, order="cell")
            per["c2-radial"] = radial_record(tp, lib, torch, dev, local, "c2", 30, 3, hbm, fp32_peak)
            line["per_config"] = per
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(w, lib, torch, e2e_steps, world):
    """End-to-end leg: the same calls with the inputs copied up from pinned host memory and every
    output copied back inside the timed region, pipelined over two device buffer sets."""
    dev, P, N, E = w.dev, w.P, w.N, w.E
    stream, side = w.stream, w.side
    sh, sh_side = stream.cuda_stream, side.cuda_stream
    h = w.plan.handle
    wkey, uvw = w.wkey, w.uvw
    e2e_keys = w.keys + (["ggx", "ggw", "ggvec"] if w.with_dbwd else [])
    host_in = {k: torch.as_tensor(np.ascontiguousarray(w.d[k])).pin_memory() for k in e2e_keys}
    outs = (w.y, w.gx, w.gw) + ((w.gvec,) if w.want_gvec else ()) + ((w.gW,) if uvw else ()) + \
        (tuple(w.dbuf[k] for k in ("g_gy", "g_x", "g_w", "g_vec")) if w.with_dbwd else ())
    host_out = [torch.empty(t_.shape, dtype=t_.dtype).pin_memory() for t_ in outs]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = []
    for b in range(2):
        dv = {k: torch.empty_like(host_in[k], device=dev) for k in e2e_keys}
        ob = [torch.empty_like(t_) for t_ in outs]
        o = dict(zip(["y", "gx", "gw"] + (["gvec"] if w.want_gvec else []) + (["gW"] if uvw else []) +
                     (["g_gy", "g_x", "g_w", "g_vec"] if w.with_dbwd else []), ob))
        cpb = torch.empty(N + 1, dtype=torch.int32, device=dev)
        pmb = torch.empty(E, dtype=torch.int32, device=dev)
        Wd = P(dv["W"]) if uvw else None
        fa = (h, N, E, P(dv["rowptr"]), P(dv["src"]), P(dv["x"]), P(dv["vec"]), P(dv[wkey]), Wd, P(o["y"]), P(w.ws),
              w.ws_bytes, sh)
        ta = (N, E, P(dv["rowptr"]), P(dv["src"]), P(cpb), P(pmb), P(w.ws_t), w.ws_t_bytes, sh_side)
        ba = (h, N, E, P(dv["rowptr"]), P(dv["src"]), P(cpb), P(pmb), P(dv["x"]), P(dv["vec"]), P(dv[wkey]), Wd,
              P(dv["gy"]), P(o["gx"]), P(o["gw"]), P(o.get("gvec")), P(o.get("gW")), P(w.ws), w.ws_bytes, sh)
        da = None
        if w.with_dbwd:
            da = (h, N, E, P(dv["rowptr"]), P(dv["src"]), P(cpb), P(pmb), P(dv["x"]), P(dv["vec"]), P(dv[wkey]), None,
                  P(dv["gy"]), P(dv["ggx"]), P(dv["ggw"]), P(dv["ggvec"]), P(o["g_gy"]), P(o["g_x"]), P(o["g_w"]),
                  P(o["g_vec"]), P(w.ws), w.ws_bytes, sh)
        sets.append((dv, ob, fa, ta, ba, da))
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    tr2_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(k):
        b = k % 2
        dv, ob, fa, ta, ba, da = sets[b]
        s_h2d.wait_event(comp_done[b])            # buffer set b is free once step k-2 has computed
        with torch.cuda.stream(s_h2d):
            for key in e2e_keys:
                dv[key].copy_(host_in[key], non_blocking=True)
        h2d_done[b].record(s_h2d)
        side.wait_event(h2d_done[b])
        st = lib.tp_csr_transpose(*ta)
        tr2_done[b].record(side)
        stream.wait_event(h2d_done[b])
        stream.wait_event(d2h_done[b])            # step k-2's results are out of set b
        st |= lib.tp_conv_fwd(*fa)
        stream.wait_event(tr2_done[b])
        st |= lib.tp_conv_bwd(*ba)
        if w.with_dbwd:
            st |= lib.tp_conv_dbwd(*da)
        comp_done[b].record(stream)
        if st:
            raise RuntimeError(lib.tp_last_error_message().decode())
        s_d2h.wait_event(comp_done[b])
        with torch.cuda.stream(s_d2h):
            for ho, t_ in zip(host_out, ob):
                ho.copy_(t_, non_blocking=True)
        d2h_done[b].record(s_d2h)

    for k in range(3):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_stream(stream)
    s_d2h.wait_stream(stream)
    side.wait_stream(stream)
    for k in range(e2e_steps):
        e2e_step(k)
    stream.wait_stream(s_d2h)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = e0.elapsed_time(e1) / 1e3
    value = replica_throughput(E, e2e_steps, world, max_over_ranks(e2e_s, world, dev))
    h2d = sum(host_in[k].numel() * host_in[k].element_size() for k in e2e_keys)
    d2h = sum(t_.numel() * t_.element_size() for t_ in host_out)
    return value, h2d, d2h


def linear_flops(ir_in, ir_out, N):
    """2 N sum_k (2l+1) mul_in mul_out over the linear map's instructions (same (l, parity) pairs)."""
    def terms(s):
        return [(int(t.split("x")[0]), int(t.split("x")[1][:-1]), t[-1]) for t in s.split("+")]
    return 2 * N * sum((2 * li + 1) * mi * mo for mi, li, pi in terms(ir_in) for mo, lo, po in terms(ir_out)
                       if (li, pi) == (lo, po))


def layer_node_bytes(lin, N, bwd):
    """Algorithmic bytes of one linear call: fwd reads x and W, writes y; bwd reads x, W and gy,
    writes gx and gW."""
    if bwd:
        return 4 * N * (2 * lin.in_dim + lin.out_dim) + 8 * lin.n_weights
    return 4 * N * (lin.in_dim + lin.out_dim) + 4 * lin.n_weights


def oracle_layer_sample(d, n_rows, seed, W1, W2, g_out):
    """The interaction layer in float64 on the host: the node-side operators on every node and
    the convolution on the edges into / out of n_rows sampled rows (as oracle_sample)."""
    from oracle.block import GateSpec, gate, gate_backward, linear, linear_backward
    spec = d["spec"]
    ir = spec.irreps_in
    mid, gate_args = layer_shapes(int(ir.split("x")[0]))
    gs = GateSpec(*gate_args)
    N = len(d["rowptr"]) - 1
    E = len(d["src"])
    t0 = time.perf_counter()
    h1 = linear(ir, ir, d["x"], W1).numpy()
    t1 = time.perf_counter()
    dd = dict(d)
    dd["x"] = h1.astype(np.float32)
    ef, tf, eb, tb = oracle_sample(dd, n_rows, seed)
    t2 = time.perf_counter()
    y = d["gy"]        # a node array of the convolution's output width (the sampled conv gives no full y)
    h2 = linear(spec.irreps_out, mid, y, W2)
    gate(gs, h2)
    g_h2 = gate_backward(gs, h2, g_out)
    linear_backward(spec.irreps_out, mid, y, W2, g_h2)
    linear_backward(ir, ir, d["x"], W1, np.asarray(d["x"]))
    t3 = time.perf_counter()
    node_t = (t1 - t0) + (t3 - t2)
    return 1.0 / (tf / ef + tb / eb + node_t / E), ef, eb, tf + tb + node_t


def layer_weights(spec, N, n_w1, n_w2, out_dim, rank=0):
    """Seeded weights of the two linear maps (N(0, 1/fan-in)) and the upstream gradient."""
    mul = int(spec.irreps_in.split("x")[0])
    rng = np.random.default_rng(spec.seed + 17 + 7919 * rank)
    W1 = (rng.standard_normal(n_w1) / math.sqrt(mul)).astype(np.float32)
    W2 = (rng.standard_normal(n_w2) / math.sqrt(mul)).astype(np.float32)
    g_out = rng.standard_normal((N, out_dim), dtype=np.float32)
    return W1, W2, g_out


def run_reference_gaunt(args, cores):
    """The float64 oracle of the Gaunt convolution on sampled receivers of the c2 graph."""
    import synth
    from oracle.gaunt import GauntPlan, gaunt_backward, gaunt_forward
    d = synth.make_inputs("c2")
    N = len(d["rowptr"]) - 1
    op = GauntPlan(*GAUNT_SPEC)
    rng = np.random.default_rng(1029)
    x = rng.standard_normal((N, op.in_dim))
    rp = np.asarray(d["rowptr"], dtype=np.int64)

    def sample(n_rows, seed):
        rows = np.sort(np.random.default_rng(seed).choice(N, size=n_rows, replace=False))
        eids = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in rows])
        rpf = np.concatenate([[0], np.cumsum(rp[rows + 1] - rp[rows])])
        w = rng.standard_normal((len(eids), op.nw))
        gy = rng.standard_normal((n_rows, op.out_dim))
        t0 = time.perf_counter()
        gaunt_forward(op, rpf, d["src"][eids], x, d["vec"][eids], w)
        gaunt_backward(op, rpf, d["src"][eids], x, d["vec"][eids], w, gy)
        return len(eids), time.perf_counter() - t0

    sample(4, 0)
    e, t = sample(16, 1)
    rows = int(max(2, min(512, 16 * 60.0 / max(1, args.steps + args.warmup) / max(t, 1e-3))))
    for k in range(args.warmup):
        sample(rows, 100 + k)
    tot_e = tot_t = 0.0
    for k in range(args.steps):
        e, t = sample(rows, 1000 + k)
        tot_e += e
        tot_t += t
    value = tot_e / tot_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS["c2-gaunt"], "name": "c2-gaunt", "N": N, "E": len(d["src"]),
                       "parallelism": "single"},
            "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle",
                             "sample": f"fwd + bwd on the edges into {rows} random receivers per step, float64"},
            "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference_layer(args, cores):
    import synth
    from oracle.block import GateSpec, linear_weight_count
    base = args.workload.split("-")[0]
    spec = synth.CONFIGS[base]
    d = synth.make_inputs(base)
    N = len(d["rowptr"]) - 1
    mid, gate_args = layer_shapes(int(spec.irreps_in.split("x")[0]))
    W1, W2, g_out = layer_weights(spec, N, linear_weight_count(spec.irreps_in, spec.irreps_in),
                                  linear_weight_count(spec.irreps_out, mid), GateSpec(*gate_args).out_dim)
    oracle_sample(d, 4, seed=0)
    v, ef, eb, t = oracle_layer_sample(d, 16, 1, W1, W2, g_out)
    rows = int(max(2, min(256, 16 * 60.0 / max(1, args.steps + args.warmup) / t)))
    for k in range(args.warmup):
        oracle_layer_sample(d, rows, k, W1, W2, g_out)
    vals, tot = [], 0.0
    for k in range(args.steps):
        v, ef, eb, t = oracle_layer_sample(d, rows, 1000 + k, W1, W2, g_out)
        vals.append(v)
        tot += t
    value = statistics.median(vals)
    sample = (f"per step: linears and gate (fwd + bwd) on all {N} nodes, conv fwd into and bwd out of {rows} "
              f"sampled rows, float64")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "name": args.workload},
            "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_layer(args, rank, world, local):
    """One interaction layer per step: linear -> convolution -> linear -> gate, then the
    backward of all four to x, both linear weights and the edge weights, every call through
    the C ABI on one capturable stream (the transpose on a side stream)."""
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from equivariant_tensor_product_b200 import build as tpbuild
    tpbuild.build()
    import equivariant_tensor_product_b200 as tp
    import synth
    lib = tp.load()

    base = args.workload.split("-")[0]
    spec = synth.CONFIGS[base]
    d = synth.make_inputs(base, args.n_atoms, seed=spec.seed + 7919 * rank)
    if args.order == "cell":
        d = synth.cell_sorted(d)
    N, E = len(d["rowptr"]) - 1, len(d["src"])
    uvw = spec.mode == "uvw"
    wkey = "s" if uvw else "w"
    mid, gate_args = layer_shapes(int(spec.irreps_in.split("x")[0]))
    # the 1/average-degree scale of the aggregated messages rides on the next linear map's
    # coefficients (it commutes with the map), which keeps the convolution on its
    # unit-coefficient compiled instances
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
    n2 = tp.Linear(spec.irreps_out, mid).n_instructions
    lin1 = tp.Linear(spec.irreps_in, spec.irreps_in)
    lin2 = tp.Linear(spec.irreps_out, mid, coeff=[N / max(E, 1)] * n2)
    gate = tp.Gate(*gate_args)
    W1, W2, d["g_out"] = layer_weights(spec, N, lin1.n_weights, lin2.n_weights, gate.out_dim, rank)
    in_dim, out_dim, nw = plan.in_dim, plan.out_dim, plan.n_edge_weights

    keys = ["rowptr", "src", "x", "vec", wkey, "g_out"] + (["W"] if uvw else [])
    copy_bytes = sum(d[k].nbytes for k in keys)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(2, math.ceil(2.5 * l2 / copy_bytes))
    copies = []
    for r in range(R):
        src_d = d
        if r:
            rr = np.random.default_rng(spec.seed + 31 * r + 7919 * rank)
            src_d = dict(d)
            src_d["x"] = rr.standard_normal(d["x"].shape, dtype=np.float32)
            src_d["g_out"] = rr.standard_normal(d["g_out"].shape, dtype=np.float32)
            src_d[wkey] = (d[wkey] * rr.uniform(0.5, 1.5, size=(1, nw))).astype(np.float32)
        copies.append({k: torch.as_tensor(np.ascontiguousarray(src_d[k])).to(dev) for k in keys})
    W1d, W2d = torch.as_tensor(W1).to(dev), torch.as_tensor(W2).to(dev)
    f32 = lambda *shape: torch.empty(*shape, device=dev)
    h1, y, h2, out = f32(N, in_dim), f32(N, out_dim), f32(N, lin2.out_dim), f32(N, gate.out_dim)
    g_h2, g_y, g_h1, gx, gw = f32(N, lin2.out_dim), f32(N, out_dim), f32(N, in_dim), f32(N, in_dim), f32(E, nw)
    gW1, gW2 = f32(lin1.n_weights), f32(lin2.n_weights)
    gWc = f32(plan.n_shared_weights) if uvw else None
    colptrs = [torch.empty(N + 1, dtype=torch.int32, device=dev) for _ in range(R)]
    perms = [torch.empty(E, dtype=torch.int32, device=dev) for _ in range(R)]
    ws_bytes = max(tp.tp_workspace_size(plan, N, E, tp.TP_OP_BWD), tp.tp_workspace_size(plan, N, E, tp.TP_OP_FWD))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    wl_bytes = max(tp.tp_linear_workspace_size(lin, N, op) for lin in (lin1, lin2) for op in (0, 1))
    wl = torch.empty(wl_bytes, dtype=torch.uint8, device=dev)
    wt_bytes = max(256, tp.tp_csr_transpose_workspace_size(N, E))
    wt = torch.empty(wt_bytes, dtype=torch.uint8, device=dev)      # side-stream transpose scratch
    stream, side = torch.cuda.Stream(dev), torch.cuda.Stream(dev, priority=-1)   # transpose: high priority
    sh, sh_side = stream.cuda_stream, side.cuda_stream
    P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None
    lf, lb, gf, gb = lib.tp_linear_fwd, lib.tp_linear_bwd, lib.tp_gate_fwd, lib.tp_gate_bwd
    cf, cb, tr_f = lib.tp_conv_fwd, lib.tp_conv_bwd, lib.tp_csr_transpose

    def op_list(cp, colptr, perm):
        return [
            ("linear_in fwd", lf, (lin1.handle, N, P(cp["x"]), P(W1d), P(h1), 0, P(wl), wl_bytes, sh)),
            ("conv fwd", cf, (plan.handle, N, E, P(cp["rowptr"]), P(cp["src"]), P(h1), P(cp["vec"]), P(cp[wkey]),
                              P(cp.get("W")), P(y), P(ws), ws_bytes, sh)),
            ("linear_out fwd", lf, (lin2.handle, N, P(y), P(W2d), P(h2), 0, P(wl), wl_bytes, sh)),
            ("gate fwd", gf, (gate.handle, N, P(h2), P(out), sh)),
            ("gate bwd", gb, (gate.handle, N, P(h2), P(cp["g_out"]), P(g_h2), sh)),
            ("linear_out bwd", lb, (lin2.handle, N, P(y), P(W2d), P(g_h2), P(g_y), P(gW2), P(wl), wl_bytes, sh)),
            ("conv bwd", cb, (plan.handle, N, E, P(cp["rowptr"]), P(cp["src"]), P(colptr), P(perm), P(h1),
                              P(cp["vec"]), P(cp[wkey]), P(cp.get("W")), P(g_y), P(g_h1), P(gw), None, P(gWc),
                              P(ws), ws_bytes, sh)),
            ("linear_in bwd", lb, (lin1.handle, N, P(cp["x"]), P(W1d), P(g_h1), P(gx), P(gW1), P(wl), wl_bytes, sh)),
        ]

    ops = [op_list(cp, colptrs[r], perms[r]) for r, cp in enumerate(copies)]
    targs = [(N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(wt), wt_bytes, sh_side)
             for r, cp in enumerate(copies)]
    names = [o[0] for o in ops[0]]
    conv_bwd_at = names.index("conv bwd")
    tr_done = [torch.cuda.Event() for _ in range(R)]
    step_done = [torch.cuda.Event() for _ in range(R)]

    def step(k, ev=None):
        r = k % R
        side.wait_event(step_done[r])
        st = tr_f(*targs[r])
        tr_done[r].record(side)
        for i, (_, fn, a) in enumerate(ops[r]):
            if i == conv_bwd_at:
                stream.wait_event(tr_done[r])
            if ev is not None:
                ev[i].record(stream)
            st |= fn(*a)
        if ev is not None:
            ev[len(names)].record(stream)
        step_done[r].record(stream)
        if st:
            raise RuntimeError(lib.tp_last_error_message().decode())

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    n0 = lib.tp_launch_count()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for k in range(args.steps):
        step(k, evs[k])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    per_step_launches = (lib.tp_launch_count() - n0) // max(args.steps, 1)
    eager_ms = start.elapsed_time(stop) / args.steps
    op_ms = {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, nm in enumerate(names)}

    # the same steps as CUDA graphs (one per input copy) for the step throughput
    graphs, launch_mode, graph_note = [], "eager", None
    try:
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            fork, join = torch.cuda.Event(), torch.cuda.Event()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                fork.record(stream)
                side.wait_event(fork)
                st = tr_f(*targs[r])
                join.record(side)
                for i, (_, fn, a) in enumerate(ops[r]):
                    if i == conv_bwd_at:
                        stream.wait_event(join)
                    st |= fn(*a)
            if st:
                raise RuntimeError(lib.tp_last_error_message().decode())
            graphs.append(g)
    except Exception as exc:  # noqa: BLE001
        graphs, graph_note = [], f"capture failed: {exc}"[:200]
    if world > 1:
        dist.barrier()
    with ClockSampler(local) as clk:
        if graphs:
            with torch.cuda.stream(stream):
                for k in range(args.warmup):
                    graphs[k % R].replay()
            torch.cuda.synchronize(dev)
            start.record(stream)
            with torch.cuda.stream(stream):
                for k in range(args.steps):
                    graphs[k % R].replay()
            stop.record(stream)
            launch_mode = "cuda_graph"
        else:
            start.record(stream)
            for k in range(args.steps):
                step(k)
            stop.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_max = max_over_ranks(start.elapsed_time(stop) / 1e3, world, dev)

    # end to end through the same calls from pinned host memory, one step after the other:
    # inputs up, the layer forward and backward, the gradients and the output down
    host_in = {k: torch.as_tensor(np.ascontiguousarray(d[k])).pin_memory() for k in keys}
    dv = {k: torch.empty_like(host_in[k], device=dev) for k in keys}
    outs = (out, gx, gw, gW1, gW2) + ((gWc,) if uvw else ())
    host_out = [torch.empty(t_.shape, dtype=t_.dtype).pin_memory() for t_ in outs]
    e_ops = op_list(dv, colptrs[0], perms[0])
    e_tr = (N, E, P(dv["rowptr"]), P(dv["src"]), P(colptrs[0]), P(perms[0]), P(wt), wt_bytes, sh)

    def e2e_step():
        with torch.cuda.stream(stream):
            for k_ in keys:
                dv[k_].copy_(host_in[k_], non_blocking=True)
        st = tr_f(*e_tr)
        for _, fn, a in e_ops:
            st |= fn(*a)
        if st:
            raise RuntimeError(lib.tp_last_error_message().decode())
        with torch.cuda.stream(stream):
            for ho, t_ in zip(host_out, outs):
                ho.copy_(t_, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value = replica_throughput(E, args.e2e_steps, world, max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev))
    h2d = sum(t_.numel() * t_.element_size() for t_ in host_in.values())
    d2h = sum(t_.numel() * t_.element_size() for t_ in host_out)

    if rank == 0:
        hbm, _, peak_note = measured_peaks()
        alg = {"linear_in fwd": layer_node_bytes(lin1, N, False), "conv fwd": fwd_bytes(N, E, in_dim, out_dim, nw),
               "linear_out fwd": layer_node_bytes(lin2, N, False),
               "gate fwd": 4 * N * (gate.in_dim + gate.out_dim),
               "gate bwd": 4 * N * (2 * gate.in_dim + gate.out_dim),
               "linear_out bwd": layer_node_bytes(lin2, N, True),
               "conv bwd": bwd_bytes(N, E, in_dim, out_dim, nw, False),
               "linear_in bwd": layer_node_bytes(lin1, N, True)}
        fl1, fl2 = linear_flops(spec.irreps_in, spec.irreps_in, N), linear_flops(spec.irreps_out, mid, N)
        flops = {"linear_in fwd": fl1, "linear_out fwd": fl2, "linear_out bwd": 2 * fl2, "linear_in bwd": 2 * fl1}
        kname = max(op_ms, key=op_ms.get)
        step_s = elapsed_max / args.steps
        ops = {nm: {"ms": op_ms[nm], "algorithmic_bytes": alg[nm],
                    "hbm_frac": alg[nm] / (op_ms[nm] * 1e-3) / 1e9 / hbm,
                    **({"flops": flops[nm], "tflops": flops[nm] / (op_ms[nm] * 1e-3) / 1e12} if nm in flops else {})}
               for nm in names}
        if uvw and kname.startswith("conv"):
            # the uvw convolution is bound by the fp32 pipe (its per-edge CG work), as in the c4 line
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            peak = 2 * 128 * sms * clk.max_mhz_or(1965.0) * 1e6 / 1e12
            fl = uvw_bwd_flops(spec, E) * (1.0 if kname == "conv bwd" else 0.5)
            achieved = fl / (op_ms[kname] * 1e-3) / 1e12
            roof = {"bound": "alu", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "peak_note": "fp32 FMA peak from the unit counts and max clock",
                    "traffic": None, "algorithmic_flops_per_call": fl, "ops": ops,
                    "step_roofline_frac": (sum(alg.values()) / (hbm * 1e9)) / step_s}
        else:
            achieved = alg[kname] / (op_ms[kname] * 1e-3) / 1e9
            roof = {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "peak_note": peak_note, "traffic": traffic_from_profile(kname, args.workload),
                    "algorithmic_bytes_per_launch": alg[kname], "ops": ops,
                    "step_roofline_frac": (sum(alg.values()) / (hbm * 1e9)) / step_s}
        cpu = None
        if not args.no_cpu_baseline:
            from oracle.conv import set_threads
            cores = set_threads()
            oracle_sample(d, 4, seed=0)
            n_rows = min(N, 64 if uvw else 1536)
            v, ef, eb, t = oracle_layer_sample(d, n_rows, 3, W1, W2, d["g_out"])
            cpu = {"value": v, "unit": "edges/s", "cores": cores, "kind": "oracle",
                   "sample": f"linears and gate (fwd + bwd) on all {N} nodes; conv fwd on the {ef} edges into and "
                             f"bwd on the {eb} edges out of {n_rows} sampled rows; float64, {t:.1f} s"}
        line = {
            "metric": METRIC, "value": replica_throughput(E, args.steps, world, elapsed_max), "unit": "edges/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * step_s,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "name": args.workload, "N": N, "E": E,
                       "order": "cell-sorted" if args.order == "cell" else "generation order (random)",
                       "launch": launch_mode, "eager_ms_per_step": eager_ms,
                       **({"graph_note": graph_note} if graph_note else {}),
                       "l2": f"{R} rotating input copies of {copy_bytes / 1e6:.1f} MB (> 2x L2 of {l2 / 1e6:.0f} MB)",
                       "parallelism": "replicas" if world > 1 else "single"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "edges/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": args.e2e_steps, "pipeline": "sequential on one stream"},
            "gpu_launches": int(per_step_launches * args.steps), "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    graphs.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_latency(args, rank, world, local):
    """Forward-only workloads too small to load the GPU (c1): per-call latency through the C
    ABI (CUDA events around each call, median), and the same call replayed as a CUDA graph."""
    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from equivariant_tensor_product_b200 import build as tpbuild
    tpbuild.build()
    import equivariant_tensor_product_b200 as tp
    import synth
    lib = tp.load()
    spec = synth.CONFIGS[args.workload]
    d = synth.make_inputs(args.workload, args.n_atoms, seed=spec.seed + 7919 * rank)
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
    N, E = len(d["rowptr"]) - 1, len(d["src"])
    g = {k: torch.as_tensor(np.ascontiguousarray(d[k])).to(dev) for k in ("rowptr", "src", "x", "vec", "w")}
    y = torch.empty(N, plan.out_dim, device=dev)
    stream = torch.cuda.Stream(dev)
    P = lambda t: C.c_void_p(t.data_ptr())
    a = (plan.handle, N, E, P(g["rowptr"]), P(g["src"]), P(g["x"]), P(g["vec"]), P(g["w"]), None, P(y), None, 0,
         stream.cuda_stream)
    for _ in range(args.warmup):
        lib.tp_conv_fwd(*a)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        for e0, e1 in evs:
            e0.record(stream)
            if lib.tp_conv_fwd(*a):
                raise RuntimeError(lib.tp_last_error_message().decode())
            e1.record(stream)
        torch.cuda.synchronize(dev)
    lat_ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=stream, capture_error_mode="thread_local"):
        lib.tp_conv_fwd(*a)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            gr.replay()
        start.record(stream)
        for _ in range(args.steps):
            gr.replay()
        stop.record(stream)
    torch.cuda.synchronize(dev)
    graph_ms = start.elapsed_time(stop) / args.steps
    # end to end: inputs up, forward, y down, each call
    host = {k: torch.as_tensor(np.ascontiguousarray(d[k])).pin_memory() for k in ("rowptr", "src", "x", "vec", "w")}
    hy = torch.empty(y.shape).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for k in host:
                g[k].copy_(host[k], non_blocking=True)
            lib.tp_conv_fwd(*a)
            hy.copy_(y, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / max(args.e2e_steps, 1)
    if rank == 0:
        line = {"metric": METRIC, "value": E / (graph_ms * 1e-3), "unit": "edges/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": graph_ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOADS[args.workload], "name": args.workload, "N": N, "E": E,
                           "launch": "cuda_graph", "eager_latency_us_median": 1e3 * lat_ms,
                           "graph_latency_us": 1e3 * graph_ms, "parallelism": "single"},
                "roofline": {"bound": "latency", "note": "192 edges: launch latency, no roofline applies"},
                "cpu_baseline": None,
                "e2e": {"value": E / (e2e_ms * 1e-3), "unit": "edges/s",
                        "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host.values()),
                        "d2h_bytes_per_step": hy.numel() * 4, "steps": args.e2e_steps},
                "gpu_launches": args.steps, "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    return 0


GAUNT_SPEC = ("32x0e+32x1o+32x2e", 2, "32x0e+32x1o+32x2e")


def gaunt_counts(N, E, mul, ng, d_in, d_out, lmax_sh, need_gvec=False):
    """Algorithmic bytes and flops of the Gaunt convolution (fwd, bwd).  Bytes: the operator's
    inputs and outputs (as fwd_bytes / bwd_bytes, w being (lmax_sh + 1) x mul per edge; the
    node grids are workspace, not counted).  Flops of the grid method (an FMA is 2), per edge,
    channel and grid point: the filter sum_l w_l (2l+1) P_l(t) as a polynomial of degree
    lmax_sh in t = r_hat . r_g by Horner's rule (2 lmax_sh) and the product-accumulate (2);
    per edge the dot products t (2 per point, shared by the channels); per node and channel
    the transforms to and from the grid (2 ng d_in and 2 ng d_out).  The backward (gx, gw):
    the grid transforms of x and gy, the filter, the accumulation of gF (2), h = F Gq (1) and
    the weight moments sum h t^n, n <= lmax_sh (2 lmax_sh + 1); with need_gvec also the
    direction terms (the derivative of the filter, 2 lmax_sh - 1, and four accumulations, 8)."""
    nw = (lmax_sh + 1) * mul
    fb = E * (4 + 12 + 4 * nw) + 4 * N * (d_in + d_out) + 4 * (N + 1)
    bb = E * (4 + 12 + 8 * nw + (12 if need_gvec else 0)) + 4 * N * (2 * d_in + d_out) + 8 * (N + 1)
    per_edge_geo = 2 * ng
    ff = E * (mul * ng * (2 * lmax_sh + 2) + per_edge_geo) + N * mul * 2 * ng * (d_in + d_out)
    per_point_b = (2 * lmax_sh + 2) + 1 + (2 * lmax_sh + 1) + ((2 * lmax_sh - 1 + 8) if need_gvec and lmax_sh else 0)
    bf = E * (mul * ng * per_point_b + per_edge_geo) + N * mul * 2 * ng * (2 * d_in + d_out)
    return fb, bb, ff, bf


def radial_counts(spec, N, E, H):
    """Algorithmic bytes and CUDA-core flops of the fused-radial forward and backward.
    Forward: per edge src + vec + the hidden row (4 H), node rows x and y, rowptr, W_r once;
    flops = the uvu forward's (fwd_flops) + the projection 2 H nw per edge.  Backward (gx, gh,
    gW_r): per edge perm + vec + h read + gh write (8 H), x read, gy read, gx write, colptr +
    rowptr, W_r read and gW_r write; flops = the uvu backward's (bwd_flops, no gvec) + three
    H x nw products per edge (the projection, gh = gw W_r^T, gW_r += h^T gw)."""
    import synth
    nw = sum(int(spec.irreps_in.split("+")[a].split("x")[0]) for a, b, o in spec.paths)
    in_dim, out_dim = synth.irreps_dim(spec.irreps_in), synth.irreps_dim(spec.irreps_out)
    fb = E * (4 + 12 + 4 * H) + 4 * N * (in_dim + out_dim) + 4 * (N + 1) + 4 * H * nw
    bb = E * (4 + 12 + 8 * H) + 4 * N * (2 * in_dim + out_dim) + 8 * (N + 1) + 8 * H * nw
    ff = fwd_flops(spec, E) + 2 * E * H * nw
    bf = bwd_flops(spec, E, False) + 3 * 2 * E * H * nw
    return fb, bb, ff, bf, nw


class RadialRun:
    """Inputs, buffers and one eager step of the fused-radial workload: forward, the transpose
    on a higher-priority side stream, backward (gx, gh, gW_r), R rotating input copies (together
    > 2.5 x L2) so that no step starts with its inputs in L2."""

    def __init__(self, tp, lib, torch, dev, base, n_atoms=None, rank=0):
        import synth
        spec = synth.CONFIGS[base]
        d = synth.make_inputs(base, n_atoms, seed=spec.seed + 7919 * rank)
        h0, Wr0 = synth.radial_hidden(d)
        N, E, H = len(d["rowptr"]) - 1, len(d["src"]), h0.shape[1]
        plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
        rng = np.random.default_rng(spec.seed + 31 + 7919 * rank)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        copy_bytes = 4 * (N * (plan.in_dim + plan.out_dim) + E * (H + 4)) + 4 * (N + 1)
        R = max(2, math.ceil(2.5 * l2 / copy_bytes))
        copies = []
        for r in range(R):
            cp = {"rowptr": d["rowptr"], "src": d["src"], "vec": d["vec"],
                  "x": d["x"] if r == 0 else rng.standard_normal((N, plan.in_dim), dtype=np.float32),
                  "h": h0 if r == 0 else np.ascontiguousarray(h0[rng.permutation(E)]),
                  "gy": rng.standard_normal((N, plan.out_dim), dtype=np.float32)}
            copies.append({k: torch.as_tensor(np.ascontiguousarray(v)).to(dev) for k, v in cp.items()})
        Wr = torch.as_tensor(Wr0).to(dev)
        self.y = torch.empty(N, plan.out_dim, device=dev)
        self.gx = torch.empty(N, plan.in_dim, device=dev)
        self.gh = torch.empty(E, H, device=dev)
        self.gWr = torch.empty_like(Wr)
        wsf = torch.empty(max(256, tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_FWD)), dtype=torch.uint8,
                          device=dev)
        wsb = torch.empty(tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_BWD), dtype=torch.uint8, device=dev)
        wst_bytes = max(256, tp.tp_csr_transpose_workspace_size(N, E))
        wst = torch.empty(wst_bytes, dtype=torch.uint8, device=dev)
        colptrs = [torch.empty(N + 1, dtype=torch.int32, device=dev) for _ in range(R)]
        perms = [torch.empty(E, dtype=torch.int32, device=dev) for _ in range(R)]
        self.stream, self.side = torch.cuda.Stream(dev), torch.cuda.Stream(dev, priority=-1)
        sh, sh_side = self.stream.cuda_stream, self.side.cuda_stream
        P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None
        self.lib = lib
        self.fns = (lib.tp_conv_fwd_radial, lib.tp_csr_transpose, lib.tp_conv_bwd_radial)
        self.args_r = []
        for r, cp in enumerate(copies):
            self.args_r.append(((plan.handle, N, E, H, P(cp["rowptr"]), P(cp["src"]), P(cp["x"]), P(cp["vec"]),
                                 P(cp["h"]), P(Wr), P(self.y), P(wsf), wsf.numel(), sh),
                                (N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(wst), wst_bytes,
                                 sh_side),
                                (plan.handle, N, E, H, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]),
                                 P(cp["x"]), P(cp["vec"]), P(cp["h"]), P(Wr), P(cp["gy"]), P(self.gx), P(self.gh),
                                 P(self.gWr), None, P(wsb), wsb.numel(), sh)))
        self.tr_done = [torch.cuda.Event() for _ in range(R)]
        self.bwd_done = [torch.cuda.Event() for _ in range(R)]
        self.spec, self.d, self.h0, self.Wr0, self.plan = spec, d, h0, Wr0, plan
        self.N, self.E, self.H, self.R, self.copies = N, E, H, R, copies
        self.copy_bytes, self.l2, self.ws_bytes = copy_bytes, l2, wsb.numel()

    def step(self, k, ev=None):
        r = k % self.R
        a_f, a_t, a_b = self.args_r[r]
        ff_, tf_, bf_ = self.fns
        self.side.wait_event(self.bwd_done[r])
        st = tf_(*a_t)
        self.tr_done[r].record(self.side)
        if ev is not None:
            ev[0].record(self.stream)
        st |= ff_(*a_f)
        if ev is not None:
            ev[1].record(self.stream)
        self.stream.wait_event(self.tr_done[r])
        if ev is not None:
            ev[2].record(self.stream)
        st |= bf_(*a_b)
        if ev is not None:
            ev[3].record(self.stream)
        self.bwd_done[r].record(self.stream)
        if st:
            raise RuntimeError(self.lib.tp_last_error_message().decode())


def radial_record(tp, lib, torch, dev, local, base, steps, warmup, hbm, fp32_peak):
    """Compact measured record of the fused-radial workload in the same run as the headline."""
    rr = RadialRun(tp, lib, torch, dev, base)
    for k in range(warmup):
        rr.step(k)
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        start.record(rr.stream)
        for k in range(steps):
            rr.step(k, evs[k])
        stop.record(rr.stream)
        torch.cuda.synchronize(dev)
    ms = start.elapsed_time(stop) / steps
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    fb, bb, fl_f, fl_b, nw = radial_counts(rr.spec, rr.N, rr.E, rr.H)
    rec = {"workload": WORKLOADS[base + "-radial"], "N": rr.N, "E": rr.E, "H": rr.H, "steps": steps,
           "ms_per_step": ms, "edges_per_s": rr.E / (ms * 1e-3), "launch": "eager",
           "kernel_ms": {"fwd": fwd_ms, "bwd": bwd_ms},
           "passes": {"fwd": pass_roofline(fwd_ms, fb, fl_f, hbm, fp32_peak),
                      "bwd": pass_roofline(bwd_ms, bb, fl_b, hbm, fp32_peak)},
           "edge_weight_bytes_not_materialised": 4 * rr.E * nw, "clocks": clk.summary()}
    del rr
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return rec


def run_radial(args, rank, world, local):
    """The convolution with the radial projection fused in (tp_conv_fwd_radial / bwd_radial):
    forward, the transpose on a side stream, backward (gx, gh, gW_r), timed as the other
    workloads are (rotating inputs > 2 x L2, CUDA events, end to end with host copies)."""
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from equivariant_tensor_product_b200 import build as tpbuild
    tpbuild.build()
    import equivariant_tensor_product_b200 as tp
    base = args.workload.split("-")[0]
    lib = tp.load()
    rr = RadialRun(tp, lib, torch, dev, base, args.n_atoms, rank)
    spec, d, h0, Wr0, plan = rr.spec, rr.d, rr.h0, rr.Wr0, rr.plan
    N, E, H, R, copies = rr.N, rr.E, rr.H, rr.R, rr.copies
    copy_bytes, l2 = rr.copy_bytes, rr.l2
    y, gx, gh, gWr = rr.y, rr.gx, rr.gh, rr.gWr
    stream, side = rr.stream, rr.side
    step = rr.step

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    n0 = lib.tp_launch_count()
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            step(k, evs[k])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    launches = lib.tp_launch_count() - n0
    elapsed_max = max_over_ranks(start.elapsed_time(stop) / 1e3, world, dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    # end to end: inputs up from pinned memory, outputs down, every step (sequential copies)
    host = {k: torch.as_tensor(np.ascontiguousarray(v.cpu().numpy())).pin_memory() for k, v in copies[0].items()}
    hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (y, gx, gh, gWr)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for k in range(args.e2e_steps):
            for key in host:
                copies[0][key].copy_(host[key], non_blocking=True)
            side.wait_stream(stream)
            step(0)
            stream.wait_stream(side)
            for ho, t in zip(hout, (y, gx, gh, gWr)):
                ho.copy_(t, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    if rank == 0:
        hbm, _, peak_note = measured_peaks()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        fp32_peak = 2 * 128 * sms * clk.max_mhz_or(1965.0) * 1e6 / 1e12
        fb, bb, fl_f, fl_b, nw = radial_counts(spec, N, E, H)
        passes = {"fwd": pass_roofline(fwd_ms, fb, fl_f, hbm, fp32_peak),
                  "bwd": pass_roofline(bwd_ms, bb, fl_b, hbm, fp32_peak)}
        dom = max(passes, key=lambda k: passes[k]["ms"])
        dp = passes[dom]
        kname = {"fwd": "k_rad_fwd", "bwd": "k_rad_send + k_rad_gwr"}[dom]
        if dp["bound"] == "hbm":
            roof = {"bound": "hbm", "kernel": kname, "achieved": dp["achieved_GBps"], "peak": hbm, "unit": "GB/s",
                    "frac": dp["achieved_GBps"] / hbm, "peak_note": peak_note}
        else:
            roof = {"bound": "alu", "kernel": kname, "achieved": dp["achieved_fp32_TFLOPs"], "peak": fp32_peak,
                    "unit": "TFLOP/s", "frac": dp["achieved_fp32_TFLOPs"] / fp32_peak,
                    "peak_note": "fp32 FMA peak; flops by bench.radial_counts"}
        roof.update({"traffic": traffic_from_profile(kname, args.workload), "passes": passes,
                     "kernel_ms": {"fwd": fwd_ms, "bwd": bwd_ms}})
        cpu = None
        if not args.no_cpu_baseline:
            from oracle import OraclePlan
            from oracle.conv import set_threads
            from oracle.radial import backward_radial, forward_radial
            cores = set_threads()
            op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")
            n_rows = 64 if base == "c2" else 16
            rows = np.sort(np.random.default_rng(3).choice(N, size=min(N, n_rows), replace=False))
            rp = np.asarray(d["rowptr"], dtype=np.int64)
            eids = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in rows])
            rpf = np.concatenate([[0], np.cumsum(rp[rows + 1] - rp[rows])])
            gys = copies[0]["gy"].cpu().numpy()
            t0 = time.perf_counter()
            forward_radial(op, rpf, d["src"][eids], d["x"], d["vec"][eids], h0[eids], Wr0)
            backward_radial(op, rpf, d["src"][eids], d["x"], d["vec"][eids], h0[eids], Wr0, gys[rows])
            t1 = time.perf_counter()
            cpu = {"value": len(eids) / (t1 - t0), "unit": "edges/s", "cores": cores, "kind": "oracle",
                   "sample": f"fwd + bwd on the {len(eids)} edges into {len(rows)} random receivers, float64, "
                             f"{t1 - t0:.1f} s"}
        line = {"metric": METRIC, "value": replica_throughput(E, args.steps, world, elapsed_max), "unit": "edges/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * elapsed_max / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOADS[args.workload], "name": args.workload, "N": N, "E": E, "H": H,
                           "n_edge_weights": nw, "launch": "eager",
                           "l2": f"{R} rotating input copies of {copy_bytes / 1e6:.1f} MB (> 2x L2 of {l2 / 1e6:.0f} MB)",
                           "parallelism": "replicas" if world > 1 else "single"},
                "roofline": roof, "cpu_baseline": cpu,
                "e2e": {"value": E * args.e2e_steps / e2e_s, "unit": "edges/s",
                        "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host.values()),
                        "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout),
                        "steps": args.e2e_steps},
                "memory": {"workspace_bytes": rr.ws_bytes, "edge_weight_bytes_not_materialised": 4 * E * nw},
                "gpu_launches": int(launches), "clocks": clk.summary(), "library": tp.tp_version()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_reference_radial(args, cores):
    """The float64 oracle of the fused-radial convolution on sampled receivers of the graph."""
    import synth
    from oracle import OraclePlan
    from oracle.radial import backward_radial, forward_radial
    base = args.workload.split("-")[0]
    spec = synth.CONFIGS[base]
    d = synth.make_inputs(base)
    h, Wr = synth.radial_hidden(d)
    N = len(d["rowptr"]) - 1
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")
    rp = np.asarray(d["rowptr"], dtype=np.int64)

    def sample(n_rows, seed):
        rows = np.sort(np.random.default_rng(seed).choice(N, size=n_rows, replace=False))
        eids = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in rows])
        rpf = np.concatenate([[0], np.cumsum(rp[rows + 1] - rp[rows])])
        t0 = time.perf_counter()
        forward_radial(op, rpf, d["src"][eids], d["x"], d["vec"][eids], h[eids], Wr)
        backward_radial(op, rpf, d["src"][eids], d["x"], d["vec"][eids], h[eids], Wr, d["gy"][rows])
        return len(eids), time.perf_counter() - t0

    sample(4, 0)
    e, t = sample(8, 1)
    rows = int(max(2, min(512, 8 * 60.0 / max(1, args.steps + args.warmup) / max(t, 1e-3))))
    for k in range(args.warmup):
        sample(rows, 100 + k)
    tot_e = tot_t = 0.0
    for k in range(args.steps):
        e, t = sample(rows, 1000 + k)
        tot_e += e
        tot_t += t
    value = tot_e / tot_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "name": args.workload, "N": N, "E": len(d["src"]),
                       "parallelism": "single"},
            "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle",
                             "sample": f"fwd + bwd on the edges into {rows} random receivers per step, float64"},
            "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_gaunt(args, rank, world, local):
    """The spherical-grid (Gaunt) convolution on the c2 graph: forward, the transpose on a
    side stream, backward (gx, gw), through include/tp_gaunt.h, timed as the convolution
    workloads are (rotating inputs > 2 x L2, CUDA graphs, end to end with host copies)."""
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from equivariant_tensor_product_b200 import build as tpbuild
    tpbuild.build()
    import equivariant_tensor_product_b200 as tp
    import synth
    lib = tp.load()
    spec = synth.CONFIGS["c2"]
    d = synth.make_inputs("c2", args.n_atoms, seed=spec.seed + 7919 * rank)
    N, E = len(d["rowptr"]) - 1, len(d["src"])
    g = tp.Gaunt(*GAUNT_SPEC)
    rng = np.random.default_rng(spec.seed + 29 + 7919 * rank)
    mul = int(GAUNT_SPEC[0].split("x")[0])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copy_bytes = 4 * (N * (g.in_dim + g.out_dim) + E * (g.n_edge_weights + 4)) + 4 * (N + 1)
    R = max(2, math.ceil(2.5 * l2 / copy_bytes))
    copies = []
    for r in range(R):
        cp = {"rowptr": d["rowptr"], "src": d["src"], "vec": d["vec"],
              "x": rng.standard_normal((N, g.in_dim), dtype=np.float32),
              "w": rng.standard_normal((E, g.n_edge_weights), dtype=np.float32),
              "gy": rng.standard_normal((N, g.out_dim), dtype=np.float32)}
        copies.append({k: torch.as_tensor(np.ascontiguousarray(v)).to(dev) for k, v in cp.items()})
    y = torch.empty(N, g.out_dim, device=dev)
    gx = torch.empty(N, g.in_dim, device=dev)
    gw = torch.empty(E, g.n_edge_weights, device=dev)
    wsf = torch.empty(tp.tp_gaunt_workspace_size(g, N, E, tp.TP_OP_FWD), dtype=torch.uint8, device=dev)
    wsb = torch.empty(tp.tp_gaunt_workspace_size(g, N, E, tp.TP_OP_BWD), dtype=torch.uint8, device=dev)
    wst_bytes = max(256, tp.tp_csr_transpose_workspace_size(N, E))
    wst = torch.empty(wst_bytes, dtype=torch.uint8, device=dev)
    colptrs = [torch.empty(N + 1, dtype=torch.int32, device=dev) for _ in range(R)]
    perms = [torch.empty(E, dtype=torch.int32, device=dev) for _ in range(R)]
    stream, side = torch.cuda.Stream(dev), torch.cuda.Stream(dev, priority=-1)
    sh, sh_side = stream.cuda_stream, side.cuda_stream
    P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None
    ff_, tf_, bf_ = lib.tp_gaunt_fwd, lib.tp_csr_transpose, lib.tp_gaunt_bwd
    args_r = []
    for r, cp in enumerate(copies):
        args_r.append(((g.handle, N, E, P(cp["rowptr"]), P(cp["src"]), P(cp["x"]), P(cp["vec"]), P(cp["w"]), P(y),
                        P(wsf), wsf.numel(), sh),
                       (N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(wst), wst_bytes, sh_side),
                       (g.handle, N, E, P(cp["rowptr"]), P(cp["src"]), P(colptrs[r]), P(perms[r]), P(cp["x"]),
                        P(cp["vec"]), P(cp["w"]), P(cp["gy"]), P(gx), P(gw), None, P(wsb), wsb.numel(), sh)))
    tr_done = [torch.cuda.Event() for _ in range(R)]
    bwd_done = [torch.cuda.Event() for _ in range(R)]

    def step(k, ev=None):
        r = k % R
        a_f, a_t, a_b = args_r[r]
        side.wait_event(bwd_done[r])
        st = tf_(*a_t)
        tr_done[r].record(side)
        if ev is not None:
            ev[0].record(stream)
        st |= ff_(*a_f)
        if ev is not None:
            ev[1].record(stream)
        stream.wait_event(tr_done[r])
        if ev is not None:
            ev[2].record(stream)
        st |= bf_(*a_b)
        if ev is not None:
            ev[3].record(stream)
        bwd_done[r].record(stream)
        if st:
            raise RuntimeError(lib.tp_last_error_message().decode())

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    n0 = lib.tp_launch_count()
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            step(k, evs[k])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    launches = lib.tp_launch_count() - n0
    elapsed_max = max_over_ranks(start.elapsed_time(stop) / 1e3, world, dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    # end to end: inputs up from pinned memory, outputs down, every step (sequential copies)
    host = {k: torch.as_tensor(np.ascontiguousarray(v.cpu().numpy())).pin_memory() for k, v in copies[0].items()}
    hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (y, gx, gw)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for k in range(args.e2e_steps):
            for key in host:
                copies[0][key].copy_(host[key], non_blocking=True)
            side.wait_stream(stream)
            step(0)
            stream.wait_stream(side)
            for ho, t in zip(hout, (y, gx, gw)):
                ho.copy_(t, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    if rank == 0:
        hbm, _, peak_note = measured_peaks()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        fp32_peak = 2 * 128 * sms * clk.max_mhz_or(1965.0) * 1e6 / 1e12
        d_in = sum(2 * int(t.split("x")[1][:-1]) + 1 for t in GAUNT_SPEC[0].split("+"))
        d_out = sum(2 * int(t.split("x")[1][:-1]) + 1 for t in GAUNT_SPEC[2].split("+"))
        fb, bb, fl_f, fl_b = gaunt_counts(N, E, mul, g.grid_points, d_in, d_out, GAUNT_SPEC[1])
        passes = {"fwd": pass_roofline(fwd_ms, fb, fl_f, hbm, fp32_peak),
                  "bwd": pass_roofline(bwd_ms, bb, fl_b, hbm, fp32_peak)}
        dom = max(passes, key=lambda k: passes[k]["ms"])
        dp = passes[dom]
        kname = {"fwd": "k_gaunt_fwd", "bwd": "k_gaunt_bwd"}[dom]
        if dp["bound"] == "hbm":
            roof = {"bound": "hbm", "kernel": kname, "achieved": dp["achieved_GBps"], "peak": hbm, "unit": "GB/s",
                    "frac": dp["achieved_GBps"] / hbm, "peak_note": peak_note}
        else:
            roof = {"bound": "alu", "kernel": kname, "achieved": dp["achieved_fp32_TFLOPs"], "peak": fp32_peak,
                    "unit": "TFLOP/s", "frac": dp["achieved_fp32_TFLOPs"] / fp32_peak,
                    "peak_note": "fp32 FMA peak; flops of the grid method by bench.gaunt_counts"}
        roof.update({"traffic": traffic_from_profile(kname, "c2-gaunt"), "passes": passes,
                     "kernel_ms": {"fwd": fwd_ms, "bwd": bwd_ms}})
        cpu = None
        if not args.no_cpu_baseline:
            from oracle.conv import set_threads
            from oracle.gaunt import GauntPlan, gaunt_backward, gaunt_forward
            cores = set_threads()
            op = GauntPlan(*GAUNT_SPEC)
            rows = np.sort(np.random.default_rng(3).choice(N, size=min(N, 256), replace=False))
            rp = np.asarray(d["rowptr"], dtype=np.int64)
            eids = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in rows])
            rpf = np.concatenate([[0], np.cumsum(rp[rows + 1] - rp[rows])])
            xs, ws_, gys = (copies[0][k].cpu().numpy() for k in ("x", "w", "gy"))
            t0 = time.perf_counter()
            gaunt_forward(op, rpf, d["src"][eids], xs, d["vec"][eids], ws_[eids])
            gaunt_backward(op, rpf, d["src"][eids], xs, d["vec"][eids], ws_[eids], gys[rows])
            t1 = time.perf_counter()
            cpu = {"value": len(eids) / (t1 - t0), "unit": "edges/s", "cores": cores, "kind": "oracle",
                   "sample": f"fwd + bwd on the {len(eids)} edges into 256 random receivers, float64, {t1 - t0:.1f} s"}
        line = {"metric": METRIC, "value": replica_throughput(E, args.steps, world, elapsed_max), "unit": "edges/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * elapsed_max / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOADS["c2-gaunt"], "name": "c2-gaunt", "N": N, "E": E, "launch": "eager",
                           "grid_points": g.grid_points,
                           "l2": f"{R} rotating input copies of {copy_bytes / 1e6:.1f} MB (> 2x L2 of {l2 / 1e6:.0f} MB)",
                           "parallelism": "replicas" if world > 1 else "single"},
                "roofline": roof, "cpu_baseline": cpu,
                "e2e": {"value": E * args.e2e_steps / e2e_s, "unit": "edges/s",
                        "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host.values()),
                        "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout),
                        "steps": args.e2e_steps},
                "gpu_launches": int(launches), "clocks": clk.summary(), "library": tp.tp_version()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.workload == "c1":
        return run_latency(args, rank, world, local)
    if args.workload == "c2-gaunt":
        return run_gaunt(args, rank, world, local)
    if args.workload.endswith("-radial"):
        return run_radial(args, rank, world, local)
    if args.workload.endswith("-layer"):
        return run_layer(args, rank, world, local)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
