"""Benchmark of the FlashCart hot path on B200.

Headline: edge-convolution forward throughput (edge x channel per second)
on the microbenchmark shape of FlashCart Sec. 6 / App. F -- 1024 nodes,
128 random neighbours each (131,072 edges), 128 channels, rank 3 for
features, direction tensors and outputs, all 23 paths kept separate --
and its fraction of the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one fc_edge_conv call over the whole graph with inputs resident
in HBM.  The 1.54 GB weight tensor is larger than the 126 MB L2, so no L2
flush is needed between steps.  Time is the max over ranks.  --impl reference times the FP64 CPU oracle on a
bounded sample of the same workload (rank 0 only).
Under torchrun the ranks share ONE graph of N x 1024 nodes, cut by receiver
range (cartesian_tensor_products_b200/shard.py): each step all-gathers the
node features over NCCL and convolves the rank's own 1024 receivers.
"""
import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("edge-conv fwd edge·channels/s (1024n×128c×128nb, rank 3) "
          "& % of roofline")
UNIT = "edge*channel/s"
WORKLOAD = "edge_conv_fwd microbench: 1024 nodes x 128 neighbours x 128 channels, rank 3, 23 paths separate"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample", type=int, default=8,
                    help="receivers per oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--rows", default=",".join(ROW_NAMES),
                    help="comma-separated extra rows to time: " + ", ".join(ROW_NAMES))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--grid", action="store_true",
                    help="time forward, VJP and VJP-of-VJP over the edge-convolution benchmark grid "
                         "(1024 nodes; ranks 1-5 x 64/128 neighbours x 64/128/256 channels) and print "
                         "one JSON line with a row per configuration")
    return ap.parse_args()


def algorithmic_bytes(N, E, C, L, P, zrow):
    """Bytes an ideal forward must move: weights, node features once,
    outputs, edge vectors, sender indices, row pointers."""
    xrow = (L + 1) ** 2
    return 4 * (E * P * C + N * xrow * C + N * zrow * C + 3 * E + E + N + 1)


def algorithmic_flops(E, C, L):
    """2 * sum_eta nnz(M_eta) + sum_eta (2 l1 + 1) per edge x channel
    (forming M_eta once per edge is amortised over the channels)."""
    per = {2: 193, 3: 727, 4: 2224}[L]
    return per * E * C


# DRAM bytes (read + write) of one edge_conv_fwd_kernel<3, 128> launch on
# this workload from an ncu capture of the same command, valid only while
# the kernel sources hash to the value it was taken with.
FWD_TRAFFIC = {"sha1": "844ace6b80ea6196f3b17c104747f2bf3eaf8f0a", "bytes": 1594583040 + 48402688}
# the files that define the timed kernel's code (the .cu only dispatches)
FWD_SOURCES = ("cartesian_tensor_products_b200/csrc/fc_edge_conv.cuh",
               "cartesian_tensor_products_b200/csrc/fc_device.cuh",
               "cartesian_tensor_products_b200/csrc/generated/fc_fwd_L3.cuh")


def fwd_sources_sha1():
    import hashlib
    h = hashlib.sha1()
    for rel in FWD_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def fp32_peak_tflops(sm_count, mhz):
    return sm_count * 128 * 2 * mhz * 1e6 / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--id=%s" % self.gpu_id, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}
        sm = [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[2][1:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


def cpu_baseline(wl, n_recv):
    """FP64 oracle on a bounded sample: the first n_recv receivers."""
    from oracle import oracle as O
    L, C, N = wl["lmax"], wl["channels"], wl["n_nodes"]
    m = np.zeros(N, np.uint8)
    m[:n_recv] = 1
    sel = np.nonzero(m[wl["edge_index"][0]])[0]
    t0 = time.perf_counter()
    O.edge_conv(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"], N,
                recv_mask=m)
    dt = time.perf_counter() - t0
    return {"value": len(sel) * C / dt, "unit": UNIT, "cores": O.num_threads(),
            "kind": "oracle",
            "sample": "first %d receivers of the workload (%d edges x %d channels), FP64 dense 3^l oracle" % (
                n_recv, len(sel), C),
            "seconds": dt}


# ---------------------------------------------------------------------------
# multi-rank plumbing (one process per GPU; no collective on the data path)
# ---------------------------------------------------------------------------

def rank_env():
    """(world, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_graph_seed(rank):
    """Each rank runs its own copy of the workload (weak scaling): rank 0 the
    reference graph, the others independent random graphs of the same shape."""
    return 2 if rank == 0 else 2 + 1000 * rank


def reduce_max(value, world, device):
    """Max over ranks of a host float (collective on every rank alike)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_throughput(world, units_per_rank, steps, max_ms):
    """Whole-job units per second: every rank processed units_per_rank per
    step, the job took max_ms (max over ranks) for `steps` steps."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


def composite_bound(peaks, fp32_peak, byts, fp32_fl, tf32_fl, ms, algo_flops):
    """Roofline of a chain of kernels: the largest of HBM time for the
    algorithmic bytes, FP32 time for the SIMT flops and tensor time for the
    TF32 products (tcgen05 TF32 peak = the measured bf16 peak x the nominal
    tf32/bf16 ratio 1.1/2.25; the three-term split counts three products)."""
    tf32_peak = peaks["bf16_tflops"] * 1.1 / 2.25
    t = {"hbm": byts / (peaks["hbm_gbs"] * 1e9), "fp32": fp32_fl / (fp32_peak * 1e12),
         "tf32": tf32_fl / (tf32_peak * 1e12)}
    key = max(t, key=t.get)
    return {"bound": "alu" if key != "hbm" else "hbm", "limit": key,
            "t_roof_us": 1e6 * t[key], "frac": t[key] / (ms * 1e-3),
            "terms_us": {k: 1e6 * v for k, v in t.items()},
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "fp32_tflops": fp32_peak, "tf32_tflops": tf32_peak},
            "algorithmic_flops": algo_flops, "algorithmic_bytes": byts}


def oracle_row(fn, units, unit, sample):
    """The FP64 oracle timed once on a bounded sample of a row's workload
    (host cores of this machine): units processed per second."""
    from oracle import oracle as O
    t0 = time.perf_counter()
    fn()
    dt = time.perf_counter() - t0
    return {"value": units / dt, "unit": unit, "cores": O.num_threads(), "kind": "oracle",
            "sample": sample, "seconds": dt}


def peak_alloc(fn):
    """Device memory the call adds at its peak (torch allocator: outputs and
    workspace the binding allocates; the library itself allocates nothing)."""
    import torch
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    fn()
    torch.cuda.synchronize()
    return torch.cuda.max_memory_allocated() - base


def time_events(fn, steps, warmup, stream, flush=None):
    """Mean device time (ms) of fn over `steps` calls, CUDA events on the
    launching stream; optional L2 flush before every call (not timed)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.mean(times), min(times)


ROW_NAMES = ("edge_conv_vjp_r3", "edge_conv_vvjp_r3", "edge_conv_fwd_r4", "edge_conv_vjp_r4",
             "edge_conv_odd_r3", "ladder", "full_ladder", "block_energy_forces")


def extra_rows(fc, W, dev, stream, peaks, fp32_peak, steps, select=ROW_NAMES):
    """Timed rows of the other hot-path steps (edge-conv VJP, rank 4, ladder,
    one interaction block); `select` names the ones to run."""
    import torch
    unknown = set(select) - set(ROW_NAMES)
    if unknown:
        raise SystemExit("unknown rows: %s" % ", ".join(sorted(unknown)))
    rows = {}
    flush_buf = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MB > L2

    def flush():
        flush_buf.zero_()

    # --- edge-conv VJP, rank 3, microbench graph
    wl = W.microbench_grad(lmax=3)
    L, C, N = 3, 128, wl["n_nodes"]
    E = wl["edge_index"].shape[1]
    P = fc.num_paths(L)
    ei = torch.from_numpy(wl["edge_index"]).to(dev)
    ev = torch.from_numpy(wl["edge_vec"]).to(dev)
    rp = fc.build_rowptr(ei, ev, N)
    if "edge_conv_vjp_r3" in select:
        x = torch.from_numpy(wl["x"]).to(dev)
        w = torch.from_numpy(wl["w"]).to(dev)
        g = torch.from_numpy(wl["g"]).to(dev)
        out = {"x": torch.empty_like(x), "w": torch.empty_like(w),
               "r": torch.empty((E, 3), device=dev)}
        ms, mn = time_events(lambda: fc.edge_conv_vjp(L, rp, ei, ev, x, w, g, out=out),
                             steps, 3, stream)
        zr = fc.out_row(L)
        byt = 4 * (2 * E * P * C + N * zr * C + 2 * N * 16 * C + 3 * E + 3 * E + E + N)
        from oracle import oracle as O
        m4 = np.zeros(N, np.uint8)
        m4[:4] = 1
        em = m4[wl["edge_index"][0]]
        cb = oracle_row(lambda: O.edge_conv_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"],
                                                wl["w"], wl["g"] * m4[:, None], N, edge_mask=em),
                        int(em.sum()) * C, "edge*channel/s",
                        "edges of the first 4 receivers (%d x %d channels), FP64 oracle" % (em.sum(), C))
        rows["edge_conv_vjp_r3"] = {
            "workload": "microbench graph, rank 3, x_bar + w_bar + r_bar",
            "cpu_baseline": cb,
            "peak_alloc_bytes": peak_alloc(lambda: fc.edge_conv_vjp(L, rp, ei, ev, x, w, g)),
            "ms": ms, "ms_min": mn, "edge_channels_per_s": E * C / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": byt / (ms * 1e-3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": byt / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": byt}}
        del out, w, g, x
        torch.cuda.empty_cache()

    if "edge_conv_vvjp_r3" in select:
        # --- VJP-of-VJP, rank 3, microbench graph: all four outputs, all cotangents
        wl = W.microbench_grad(lmax=3)
        cot = W.cotangents(N, E, 3, C, 61, wl["edge_vec"])
        x = torch.from_numpy(wl["x"]).to(dev)
        w = torch.from_numpy(wl["w"]).to(dev)
        g = torch.from_numpy(wl["g"]).to(dev)
        vx = torch.from_numpy(cot["vx"]).to(dev)
        vw = torch.from_numpy(cot["vw"]).to(dev)
        vr = torch.from_numpy(cot["vr"]).to(dev)
        ms, mn = time_events(lambda: fc.edge_conv_vjp_vjp(L, rp, ei, ev, x, w, g, v_x=vx, v_w=vw, v_r=vr),
                             steps, 3, stream)
        zr = fc.out_row(L)
        # w, vw in; w_hat out; x, vx, g in; g_hat, x_hat out (+ zeroing); edges
        byt = 4 * (3 * E * P * C + 2 * N * 16 * C + 2 * N * zr * C + N * 16 * C
                   + 3 * E * 3 + E + N)
        from oracle import oracle as O
        m2 = np.zeros(N, np.uint8)
        m2[:2] = 1
        em = m2[wl["edge_index"][0]]
        cb = oracle_row(lambda: O.edge_conv_vjp_vjp(3, 3, 3, C, wl["edge_index"], wl["edge_vec"], wl["x"],
                                                    wl["w"], wl["g"] * m2[:, None], cot["vx"], cot["vw"],
                                                    cot["vr"], N, edge_mask=em),
                        int(em.sum()) * C, "edge*channel/s",
                        "edges of the first 2 receivers (%d x %d channels), FP64 oracle" % (em.sum(), C))
        rows["edge_conv_vvjp_r3"] = {
            "workload": "microbench graph, rank 3, g_hat + x_hat + w_hat + r_hat from vx, vw, vr",
            "cpu_baseline": cb,
            "peak_alloc_bytes": peak_alloc(lambda: fc.edge_conv_vjp_vjp(L, rp, ei, ev, x, w, g, v_x=vx,
                                                                        v_w=vw, v_r=vr)),
            "ms": ms, "ms_min": mn, "edge_channels_per_s": E * C / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": byt / (ms * 1e-3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": byt / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": byt}}
        del x, w, g, vx, vw, vr
        torch.cuda.empty_cache()

    if "edge_conv_fwd_r4" in select or "edge_conv_vjp_r4" in select:
        # --- rank 4 on the microbench graph, forward and VJP
        wl4 = W.microbench(lmax=4, weight_seed=32)
        L4 = 4
        P4 = fc.num_paths(L4)
        x4 = torch.from_numpy(wl4["x"]).to(dev)
        w4 = torch.from_numpy(wl4["w"]).to(dev)
        if "edge_conv_fwd_r4" in select:
            z4 = torch.empty((N, fc.out_row(L4) * C), device=dev)
            ms4, mn4 = time_events(lambda: fc.edge_conv(L4, rp, ei, ev, x4, w4, out=z4), steps, 3, stream)
            byt4 = 4 * (E * P4 * C + N * 25 * C + N * fc.out_row(L4) * C + 4 * E + N)
            fl4 = algorithmic_flops(E, C, 4)
            rows["edge_conv_fwd_r4"] = {
                "workload": "microbench graph, rank 4 (42 paths), forward",
                "ms": ms4, "ms_min": mn4, "edge_channels_per_s": E * C / (ms4 * 1e-3),
                "roofline": {"bound": "hbm", "achieved": byt4 / (ms4 * 1e-3) / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": byt4 / (ms4 * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "algorithmic_bytes": byt4,
                             "fp32_frac": fl4 / (ms4 * 1e-3) / 1e12 / fp32_peak}}
        if "edge_conv_vjp_r4" in select:
            g4 = torch.randn((N, fc.out_row(L4) * C), device=dev)
            out4 = {"x": torch.empty_like(x4), "w": torch.empty_like(w4),
                    "r": torch.empty((E, 3), device=dev)}
            ms4b, mn4b = time_events(lambda: fc.edge_conv_vjp(L4, rp, ei, ev, x4, w4, g4, out=out4),
                                     steps, 3, stream)
            byt4b = 4 * (2 * E * P4 * C + N * fc.out_row(L4) * C + 2 * N * 25 * C + 7 * E + N)
            rows["edge_conv_vjp_r4"] = {
                "workload": "microbench graph, rank 4, x_bar + w_bar + r_bar",
                "ms": ms4b, "ms_min": mn4b, "edge_channels_per_s": E * C / (ms4b * 1e-3),
                "roofline": {"bound": "hbm", "achieved": byt4b / (ms4b * 1e-3) / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": byt4b / (ms4b * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "algorithmic_bytes": byt4b}}
        z4 = g4 = out4 = None
        del x4, w4
        torch.cuda.empty_cache()

    if "edge_conv_odd_r3" in select:
        # --- odd-J (Levi-Civita) paths, rank 3, microbench graph: forward and VJP
        Po = fc.odd_num_paths(3)
        zro = fc.odd_out_row(3)
        gen = torch.Generator(device=dev)
        gen.manual_seed(77)
        xo = torch.randn(N, 16 * C, device=dev, generator=gen)
        wo = torch.randn(E, Po, C, device=dev, generator=gen) * Po ** -0.5
        go = torch.randn(N, zro * C, device=dev, generator=gen)
        zo = torch.empty((N, zro * C), device=dev)
        mso, mno = time_events(lambda: fc.edge_conv(3, rp, ei, ev, xo, wo, out=zo, odd=True), steps, 3, stream)
        outo = {"x": torch.empty_like(xo), "w": torch.empty_like(wo), "r": torch.empty((E, 3), device=dev)}
        msov, mnov = time_events(lambda: fc.edge_conv_vjp(3, rp, ei, ev, xo, wo, go, out=outo, odd=True),
                                 steps, 3, stream)
        bo = 4 * (E * Po * C + N * 16 * C + N * zro * C + 4 * E + N)
        bov = 4 * (2 * E * Po * C + N * zro * C + 2 * N * 16 * C + 7 * E + N)
        rows["edge_conv_odd_fwd_r3"] = {
            "workload": "microbench graph, rank 3, the %d odd-J (Levi-Civita) paths, forward" % Po,
            "ms": mso, "ms_min": mno, "edge_channels_per_s": E * C / (mso * 1e-3),
            "roofline": {"bound": "hbm", "achieved": bo / (mso * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": bo / (mso * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": bo}}
        rows["edge_conv_odd_vjp_r3"] = {
            "workload": "same odd-J convolution, x_bar + w_bar + r_bar",
            "ms": msov, "ms_min": mnov, "edge_channels_per_s": E * C / (msov * 1e-3),
            "roofline": {"bound": "hbm", "achieved": bov / (msov * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": bov / (msov * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": bov}}
        del xo, wo, go, zo, outo
        torch.cuda.empty_cache()

    if "ladder" in select:
        # --- ladder, 4096 nodes x 128 channels, rank 3, order 4
        lad = W.ladder()
        Ll, Cl, order, Nl = lad["lmax"], lad["channels"], lad["order"], lad["n_nodes"]
        A1 = torch.from_numpy(lad["A1"]).to(dev)
        pw = torch.from_numpy(lad["path_w"]).to(dev)
        mw = torch.from_numpy(lad["mix_w"]).to(dev)
        gz = torch.from_numpy(lad["gz"]).to(dev)
        ws_bytes = max(fc.ladder_workspace_bytes(Ll, Cl, order, Nl),
                       fc.ladder_workspace_bytes(Ll, Cl, order, Nl, vjp=True))
        ws = torch.empty(ws_bytes // 4, device=dev)
        res = {}

        def lad_fwd():
            res["s"], res["z"] = fc.product_ladder(Ll, order, A1, pw, mw, workspace=ws)
        msl, mnl = time_events(lad_fwd, steps, 3, stream, flush=flush)
        states = res["s"]

        def lad_vjp():
            fc.product_ladder_vjp(Ll, order, A1, pw, mw, states, gz, workspace=ws)
        mslb, mnlb = time_events(lad_vjp, steps, 3, stream, flush=flush)
        S = order - 1
        mix_flops = S * 2 * Nl * 16 * Cl * Cl
        tp_flops = S * Nl * Cl * 2 * 751
        plane_b = 4 * Nl * 16 * Cl
        tc = Cl == 128

        def bound(byts, fp32_fl, tf32_fl, ms):
            return composite_bound(peaks, fp32_peak, byts, fp32_fl, tf32_fl, ms, mix_flops + tp_flops)
        from oracle import oracle as O
        ns = 64
        lm = np.zeros(Nl, np.uint8)
        lm[:ns] = 1
        cbf = oracle_row(lambda: O.ladder(Ll, Cl, order, lad["A1"], lad["path_w"], lad["mix_w"], node_mask=lm),
                         ns, "nodes/s", "first %d nodes, FP64 oracle" % ns)
        cbv = oracle_row(lambda: O.ladder_vjp(Ll, Cl, order, lad["A1"], lad["path_w"], lad["mix_w"],
                                              lad["gz"] * lm[:, None], node_mask=lm),
                         ns, "nodes/s", "first %d nodes, FP64 oracle" % ns)
        pa_f = peak_alloc(lambda: fc.product_ladder(Ll, order, A1, pw, mw))
        pa_v = peak_alloc(lambda: fc.product_ladder_vjp(Ll, order, A1, pw, mw, states, gz))
        # forward: A1 read, states written, z written; products FP32; mix TF32 x3 (or FP32)
        fb = plane_b * (1 + S + 1)
        rows["ladder_fwd"] = {
            "nodes_per_s": Nl / (msl * 1e-3), "cpu_baseline": cbf, "peak_alloc_bytes": pa_f,
            "workload": "4096 nodes x 128 channels, rank 3, order 4 (3 products + 3 per-rank 128x128 mixes)",
            "ms": msl, "ms_min": mnl,
            "roofline": bound(fb, tp_flops + (0 if tc else mix_flops), 3 * mix_flops if tc else 0, msl),
            "l2_flush": "256 MB written before every call"}
        # VJP: states and A1 read, gz read, A1_bar written; products 4x (FP32
        # SIMT); two mixes per step, B_bar = A_bar M and M_bar = A_bar^T B, both
        # on the tensor cores at C = 128 (three TF32 products each), else FP32
        vb = plane_b * (1 + S + 1 + 1)
        rows["ladder_vjp"] = {
            "nodes_per_s": Nl / (mslb * 1e-3), "cpu_baseline": cbv, "peak_alloc_bytes": pa_v,
            "workload": "same ladder, A1_bar + path_w_bar + mix_w_bar",
            "ms": mslb, "ms_min": mnlb,
            "roofline": bound(vb, 4 * tp_flops + (0 if tc else 2 * mix_flops),
                              6 * mix_flops if tc else 0, mslb),
            "l2_flush": "256 MB written before every call"}
        del A1, pw, mw, gz, ws, res, states
        torch.cuda.empty_cache()

    if "full_ladder" in select:
        # --- full ladder (path-separated products + per-rank path/channel maps), forward
        Lf, Cf, of, Nf = 3, 128, 4, 4096
        fd = W.full_ladder_inputs(Nf, Lf, Cf, of, 44)
        A = torch.from_numpy(fd["A"]).to(dev)
        W1 = torch.from_numpy(fd["W1"]).to(dev)
        Wq = torch.from_numpy(fd["Wq"]).to(dev)
        wsf = torch.empty(fc.lib().fc_full_ladder_workspace_size(
            ctypes.byref(fc.LadderDesc(Lf, Cf, of)), Nf) // 4, device=dev)
        msf, mnf = time_events(lambda: fc.full_ladder(Lf, of, A, W1, Wq, workspace=wsf), steps, 3, stream,
                               flush=flush)
        P = fc.num_paths(Lf)
        rows_l = Nf * 16
        mix_fl = 2 * rows_l * Cf * Cf + (of - 1) * 2 * Nf * sum(
            (2 * l + 1) * p for l, p in enumerate(W.paths_per_rank(Lf, Lf, Lf))) * Cf * Cf
        tp_fl = (of - 1) * Nf * Cf * 2 * 751
        # A read, order states and z written; products FP32; maps TF32 x3 on the tensor cores
        fbf = 4 * Nf * 16 * Cf * (1 + of + 1)
        from oracle import oracle as O
        ns = 16
        fm = np.zeros(Nf, np.uint8)
        fm[:ns] = 1
        cbff = oracle_row(lambda: O.full_ladder(Lf, Cf, of, fd["A"], fd["W1"], fd["Wq"], node_mask=fm),
                          ns, "nodes/s", "first %d nodes, FP64 oracle" % ns)
        cbfv = oracle_row(lambda: O.full_ladder_vjp(Lf, Cf, of, fd["A"], fd["W1"], fd["Wq"],
                                                    fd["gz"] * fm[:, None], node_mask=fm),
                          ns, "nodes/s", "first %d nodes, FP64 oracle" % ns)
        rows["full_ladder_fwd"] = {
            "nodes_per_s": Nf / (msf * 1e-3), "cpu_baseline": cbff,
            "peak_alloc_bytes": peak_alloc(lambda: fc.full_ladder(Lf, of, A, W1, Wq)),
            "workload": "4096 nodes x 128 channels, rank 3, order 4: path-separated products, "
                        "per-rank (P_l x 128) -> 128 maps on tcgen05 (three-term TF32)",
            "ms": msf, "ms_min": mnf,
            "roofline": composite_bound(peaks, fp32_peak, fbf, tp_fl, 3 * mix_fl, msf, mix_fl + tp_fl),
            "l2_flush": "256 MB written before every call"}
        # VJP: per step the map's weight gradient and the transposed map B_bar,
        # each the forward map's flops, on tcgen05 (three TF32 products each);
        # phi_1's weight gradient on tcgen05 too, its transposed map (A_bar +=
        # p_bar W1) FP32 SIMT; the products recomputed and differentiated
        # (3 x the product flops); A, phi_1..phi_{order-1}, gz read, A_bar
        # written
        st_f, _ = fc.full_ladder(Lf, of, A, W1, Wq, workspace=wsf)
        gzf = torch.from_numpy(fd["gz"]).to(dev)
        wsv = torch.empty(fc.lib().fc_full_ladder_vjp_workspace_size(
            ctypes.byref(fc.LadderDesc(Lf, Cf, of)), Nf) // 4, device=dev)
        msv, mnv = time_events(lambda: fc.full_ladder_vjp(Lf, of, A, W1, Wq, st_f, gzf, workspace=wsv),
                               steps, 3, stream, flush=flush)
        vbf = 4 * Nf * 16 * Cf * (1 + (of - 1) + 1 + 1)
        map1_fl = 2 * rows_l * Cf * Cf
        rows["full_ladder_vjp"] = {
            "nodes_per_s": Nf / (msv * 1e-3), "cpu_baseline": cbfv,
            "peak_alloc_bytes": peak_alloc(lambda: fc.full_ladder_vjp(Lf, of, A, W1, Wq, st_f, gzf)),
            "workload": "same full ladder, A_bar + W1_bar + Wq_bar (B_bar maps and weight "
                        "gradients on tcgen05)",
            "ms": msv, "ms_min": mnv,
            "roofline": composite_bound(peaks, fp32_peak, vbf, map1_fl + 3 * tp_fl,
                                        3 * mix_fl + 3 * (mix_fl - map1_fl), msv, 2 * mix_fl + 3 * tp_fl),
            "l2_flush": "256 MB written before every call"}
        del A, W1, Wq, wsf, wsv, st_f, gzf
        torch.cuda.empty_cache()

    if "block_energy_forces" in select:
        # --- one interaction block on the 1000-atom diamond cell: energy + forces
        dm = W.diamond()
        Nd, Ed = dm["n_nodes"], dm["edge_index"].shape[1]
        dei = torch.from_numpy(dm["edge_index"]).to(dev)
        dev_ = torch.from_numpy(dm["edge_vec"]).to(dev)
        dx = torch.from_numpy(dm["x"]).to(dev)
        dom = torch.from_numpy(dm["omega"]).to(dev)
        dpw = torch.from_numpy(dm["path_w"]).to(dev)
        dmw = torch.from_numpy(dm["mix_w"]).to(dev)
        drp = fc.build_rowptr(dei, dev_, Nd)
        msb, mnb = time_events(lambda: fc.interaction_block(dm["lmax"], dm["order"], drp, dei, dev_, dx,
                                                            dom, dpw, dmw, dm["cutoff"],
                                                            dm["edge_scale"]),
                               steps, 3, stream, flush=flush)
        from oracle import oracle as O
        bm = np.zeros(Nd, np.uint8)
        bm[:2] = 1
        cbb = oracle_row(lambda: O.block_energy_forces(dm["lmax"], dm["channels"], dm["order"],
                                                       dm["edge_index"], dm["edge_vec"], dm["x"],
                                                       dm["omega"], dm["path_w"], dm["mix_w"], Nd,
                                                       dm["cutoff"], dm["edge_scale"], recv_mask=bm),
                         2, "atoms/s", "energies and incoming-edge gradients of the first 2 atoms, "
                         "FP64 oracle")
        rows["block_energy_forces"] = {
            "atoms_per_s": Nd / (msb * 1e-3), "cpu_baseline": cbb,
            "peak_alloc_bytes": peak_alloc(lambda: fc.interaction_block(
                dm["lmax"], dm["order"], drp, dei, dev_, dx, dom, dpw, dmw, dm["cutoff"], dm["edge_scale"])),
            "workload": "1000-atom diamond (5x5x5 cells, a = 3.567 A, 5 A cutoff, %d edges), C=128, rank 3: "
                        "enveloped conv (paths summed) + order-5 ladder + E + ladder VJP + conv VJP + forces" % Ed,
            "ms": msb, "ms_min": mnb, "us_per_atom": 1e3 * msb / Nd,
            "l2_flush": "256 MB written before every call"}
    return rows


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from cartesian_tensor_products_b200 import workloads as W
    wl = W.microbench()
    for _ in range(args.warmup):
        cpu_baseline(wl, 1)
    vals, secs = [], []
    for _ in range(args.steps):
        b = cpu_baseline(wl, args.cpu_sample)
        vals.append(b["value"])
        secs.append(b["seconds"])
    value = statistics.median(vals)
    cb = {"value": value, "unit": UNIT, "cores": b["cores"], "kind": "oracle",
          "sample": b["sample"]}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": b["sample"]},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)

    from __graft_entry__ import build
    build()
    from cartesian_tensor_products_b200 import flashcart as fc
    from cartesian_tensor_products_b200 import workloads as W

    stream = torch.cuda.current_stream()
    sh = None
    if world == 1:
        wl = W.microbench(seed=rank_graph_seed(rank))
        h_ei, h_ev, h_x, h_w = wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"]
        N = N_send = wl["n_nodes"]
    else:
        # one graph of world x 1024 nodes cut by receiver range: this rank's
        # 1024 receivers take their 128 senders from all nodes; the step
        # all-gathers the node features, then convolves the local edges
        from cartesian_tensor_products_b200 import shard
        wl = W.sharded_microbench(rank, world)
        sh = shard.GraphShard(wl["edge_index"], wl["n_nodes"], rank, world, bounds=wl["bounds"])
        h_ei, h_ev, h_x, h_w = sh.edge_index, wl["edge_vec_local"], wl["x_local"], wl["w_local"]
        N, N_send = sh.n_local, wl["n_nodes"]
    L, C = wl["lmax"], wl["channels"]
    E = h_ei.shape[1]
    P = fc.num_paths(L)
    zrow = fc.out_row(L)

    # ---- inputs resident in HBM
    ei = torch.from_numpy(h_ei).to(dev)
    ev = torch.from_numpy(h_ev).to(dev)
    x = torch.from_numpy(h_x).to(dev)
    w = torch.from_numpy(h_w).to(dev)
    rowptr = fc.build_rowptr(ei, ev, N, n_send=N_send)
    z = torch.empty((N, zrow * C), dtype=torch.float32, device=dev)
    x_all = torch.empty((N_send, x.shape[1]), dtype=torch.float32, device=dev) if sh else x
    # receiver row pointer and graph validation, timed on its own (it reads
    # its verdict back, so it synchronises)
    torch.cuda.synchronize()
    csr0 = torch.cuda.Event(enable_timing=True)
    csr1 = torch.cuda.Event(enable_timing=True)
    csr0.record(stream)
    for _ in range(5):
        fc.build_rowptr(ei, ev, N, n_send=N_send)
    csr1.record(stream)
    csr1.synchronize()
    csr_ms = csr0.elapsed_time(csr1) / 5
    conv_peak = peak_alloc(lambda: fc.edge_conv(L, rowptr, ei, ev, x_all, w))
    k_start = torch.cuda.Event(enable_timing=True)
    k_end = torch.cuda.Event(enable_timing=True)
    k_ms = []

    def step(timed=False):
        if sh is not None:
            sh.gather_rows(x, out=x_all)
        if timed:
            k_start.record(stream)
        fc.edge_conv(L, rowptr, ei, ev, x_all, w, out=z)
        if timed:
            k_end.record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(dev)
    gpu_id = str(getattr(props, "uuid", local))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) == 36:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    ev_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        ev_start[i].record(stream)
        step()
        ev_end[i].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    if sh is not None:
        # the convolution kernel alone (the steps above include the all-gather)
        for _ in range(args.steps):
            step(timed=True)
            k_end.synchronize()
            k_ms.append(k_start.elapsed_time(k_end))
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t_all0.elapsed_time(t_all1)
    per = [a.elapsed_time(b) for a, b in zip(ev_start, ev_end)]
    total_ms = reduce_max(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = weak_throughput(world, E * C, args.steps, total_ms)

    # ---- roofline of the (single) kernel of the step
    peaks, peak_kind = load_peaks()
    abytes = algorithmic_bytes(N, E, C, L, P, zrow)
    kern_ms = statistics.mean(k_ms if k_ms else per)
    achieved_gbs = abytes / (kern_ms * 1e-3) / 1e9
    flops = algorithmic_flops(E, C, L)
    sm_count = props.multi_processor_count
    fp32_peak = fp32_peak_tflops(sm_count, peaks.get("sm_max_mhz", 1965.0))
    roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
            "traffic": FWD_TRAFFIC["bytes"] if fwd_sources_sha1() == FWD_TRAFFIC["sha1"] else None,
            "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)",
            "algorithmic_bytes": abytes,
            "fp32": {"achieved_tflops": flops / (kern_ms * 1e-3) / 1e12,
                     "peak_tflops": fp32_peak,
                     "frac": flops / (kern_ms * 1e-3) / 1e12 / fp32_peak,
                     "algorithmic_flops": flops,
                     "peak_source": "148 SM x 128 FP32 lanes x 2 x clocks.max.sm"},
            "t_roof_ms": max(abytes / (peaks["hbm_gbs"] * 1e9),
                             flops / (fp32_peak * 1e12)) * 1e3}
    roof["frac_of_roofline"] = roof["t_roof_ms"] / kern_ms

    # ---- end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        hx = torch.from_numpy(h_x).pin_memory()
        hw = torch.from_numpy(h_w).pin_memory()
        hei = torch.from_numpy(h_ei).pin_memory()
        hev = torch.from_numpy(h_ev).pin_memory()
        hz = torch.empty((N, zrow * C), dtype=torch.float32).pin_memory()
        dx, dw = torch.empty_like(x), torch.empty_like(w)
        dei, dev_ = torch.empty_like(ei), torch.empty_like(ev)
        h2d = sum(t.numel() * t.element_size() for t in (hx, hw, hei, hev))
        d2h = hz.numel() * hz.element_size()

        def e2e_step():
            dx.copy_(hx, non_blocking=True)
            dw.copy_(hw, non_blocking=True)
            dei.copy_(hei, non_blocking=True)
            dev_.copy_(hev, non_blocking=True)
            rp = fc.build_rowptr(dei, dev_, N, n_send=N_send)
            xa = sh.gather_rows(dx, out=x_all) if sh is not None else dx
            fc.edge_conv(L, rp, dei, dev_, xa, dw, out=z)
            hz.copy_(z, non_blocking=True)
        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 5))
        if world > 1:
            dist.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms = a0.elapsed_time(a1)
        e_ms = reduce_max(e_ms, world, dev)
        e2e = {"value": weak_throughput(world, E * C, n_e2e, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": n_e2e, "ms_per_step": e_ms / n_e2e,
               "includes": "H2D of x, w, edge_index, edge_vec; fc_build_rowptr (validates, syncs); "
                           + ("all-gather of x; " if sh is not None else "")
                           + "fc_edge_conv; D2H of z"}

    rows = None
    if world == 1 and not args.no_rows:
        rows = extra_rows(fc, W, dev, stream, peaks, fp32_peak, max(3, min(args.steps, 10)),
                          select=[r for r in args.rows.split(",") if r])

    line = None
    if rank == 0:
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(wl, args.cpu_sample)
            cb.pop("seconds", None)
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": max(args.warmup, 3),
                "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": {"workload": WORKLOAD, "n_nodes": N, "n_edges": E,
                           "channels": C, "lmax": L, "paths": P,
                           "l2_flush": "none: the 1.54 GB weight stream exceeds the 126 MB L2",
                           "per_rank": ("one graph of %d nodes cut by receiver range: per step an "
                                        "NCCL all-gather of the node features, then this rank's "
                                        "1024 receivers (weak scaling)" % N_send) if sh is not None
                           else "the whole graph on one GPU"},
                "roofline": roof, "cpu_baseline": cb, "e2e": e2e,
                "gpu_launches": args.steps, "clocks": clocks, "rows": rows,
                "csr_build_ms": csr_ms, "peak_alloc_bytes": conv_peak,
                "kernel_ms": {"mean": kern_ms, "min": min(per), "max": max(per)}}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_grid(args):
    """The pages' edge-convolution benchmark grid (1024 nodes, 64 or 128
    random neighbours, 64/128/256 channels, ranks 1-5): forward, VJP (x_bar,
    w_bar, r_bar) and VJP-of-VJP (all four outputs, all cotangents) per
    configuration, CUDA events, inputs resident on the device
    (seeded, synthetic; drawn on the device)."""
    import torch
    from cartesian_tensor_products_b200 import flashcart as fc
    from cartesian_tensor_products_b200 import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_kind = load_peaks()
    steps = max(3, min(args.steps, 10))
    props = torch.cuda.get_device_properties(dev)
    gpu_id = str(getattr(props, "uuid", 0))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) == 36:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    out = []
    for k in (64, 128):
        _, ei_np, ev_np = W.random_graph(1024, k, 20.0, 2 + k)
        ei = torch.from_numpy(ei_np).to(dev)
        ev = torch.from_numpy(ev_np).to(dev)
        rp = fc.build_rowptr(ei, ev, 1024)
        E = ei_np.shape[1]
        for L in (1, 2, 3, 4, 5):
            P = fc.num_paths(L)
            for C in (64, 128, 256):
                gen = torch.Generator(device=dev)
                gen.manual_seed(1000 * L + C + k)
                rnd = lambda *shape, s=1.0: torch.randn(*shape, device=dev, generator=gen) * s
                x = rnd(1024, (L + 1) ** 2 * C)
                w = rnd(E, P, C, s=P ** -0.5)
                zr = fc.out_row(L)
                g = rnd(1024, zr * C)
                vx, vw, vr = rnd(1024, (L + 1) ** 2 * C), rnd(E, P, C, s=P ** -0.5), rnd(E, 3)
                z = torch.empty((1024, zr * C), device=dev)
                f_ms, _ = time_events(lambda: fc.edge_conv(L, rp, ei, ev, x, w, out=z), steps, 3, stream)
                v_ms, _ = time_events(lambda: fc.edge_conv_vjp(L, rp, ei, ev, x, w, g), steps, 3, stream)
                # rank 5 runs one launch per path group
                vv_ms, _ = time_events(lambda: fc.edge_conv_vjp_vjp(L, rp, ei, ev, x, w, g, v_x=vx,
                                                                    v_w=vw, v_r=vr), steps, 3, stream)
                fb = algorithmic_bytes(1024, E, C, L, P, zr)
                out.append({"lmax": L, "neighbours": k, "channels": C, "paths": P,
                            "fwd_ms": f_ms, "vjp_ms": v_ms, "vvjp_ms": vv_ms,
                            "fwd_edge_channels_per_s": E * C / (f_ms * 1e-3),
                            "fwd_hbm_frac": fb / (f_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
                del x, w, g, vx, vw, vr, z
                torch.cuda.empty_cache()
    # node-local grid: 4096 nodes, ranks 1-4, orders 2-6, 64/128/256 channels
    lad = []
    for L in (1, 2, 3, 4):
        P = fc.num_paths(L)
        NY = (L + 1) ** 2
        for C in (64, 128, 256):
            for order in (2, 3, 4, 5, 6):
                gen = torch.Generator(device=dev)
                gen.manual_seed(7000 + 100 * L + 10 * order + C)
                A1 = torch.randn(4096, NY * C, device=dev, generator=gen)
                pw = torch.randn(order - 1, P, C, device=dev, generator=gen) * P ** -0.5
                mw = torch.randn(order - 1, L + 1, C, C, device=dev, generator=gen) * C ** -0.5
                gz = torch.randn(4096, NY * C, device=dev, generator=gen)
                res = {}

                def lf():
                    res["s"], res["z"] = fc.product_ladder(L, order, A1, pw, mw)
                f_ms, _ = time_events(lf, steps, 3, stream)
                v_ms, _ = time_events(lambda: fc.product_ladder_vjp(L, order, A1, pw, mw, res["s"], gz),
                                      steps, 3, stream)
                lad.append({"lmax": L, "order": order, "channels": C, "fwd_ms": f_ms, "vjp_ms": v_ms,
                            "mix": ("tcgen05 TF32x3" if C == 128 else
                                    "tcgen05 TF32x3, VJP weight gradient FP32 SIMT" if C == 256 else "FP32 SIMT")})
                del A1, pw, mw, gz, res
                torch.cuda.empty_cache()
    clocks = sampler.stop()
    print(json.dumps({"metric": "edge-conv grid: fwd / VJP / VJP-of-VJP ms per configuration",
                      "clocks": clocks,
                      "unit": "ms", "n_gpus": 1, "dtype": "f32", "data": "synthetic",
                      "peak_source": peak_kind, "steps": steps,
                      "config": {"workload": "1024 nodes, random neighbours in a 20 A box; "
                                             "ranks 1-5 x 64/128 neighbours x 64/128/256 channels"},
                      "grid": out, "ladder_grid": lad}))


def main():
    args = parse()
    if args.grid:
        run_grid(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
