"""Benchmark of the YOCO++ cross-layer KV cache hot path on B200.

One step is one pass of the whole path over one batch of synthetic input:
  1. prefill-size compose/append for self-decoder layers 2..L/2
     (K'_i = lambda(aK1 K_1 + aK2 K_i), V' likewise, written to cache i),
  2. decode-size compose/append of the decoded token for layers 2..L/2,
  3. decode attention of every cross-decoder layer (L/2 of them) over the
     shared cache (K'_{L/2}, V'_{L/2}), each with its own query.
(YOCO++: Enhancing YOCO with KV Residual Connections, section 2 and
section 3; You Only Cache Once, abstract.)

Reported (one JSON line from rank 0):
  value      decode-attention KV-read GB/s: algorithmic KV bytes of all
             cross-decoder layers / their measured time (whole job, all ranks)
  compose_gbs, decode_tok_s, roofline (dominant kernel), e2e (same metric
  through the C ABI with host buffers), clocks, cpu_baseline (the oracle),
  prefill_attention (the causal prefill attention, and the fused composition +
  prefill launch against the two separate launches), and, after the headline
  32 x 8192 workload, the 131072-token and the ragged paged workloads measured
  the same way under "workloads".
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import signal
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn KV-read GB/s (% of B200 HBM peak); compose GB/s; decode tok/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (reported beside the measured copy peak)
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3, help="workload (1..5); 3 = 32 x 8192 throughput decode")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the causal prefill-attention measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--decode-kernel", type=int, default=0, choices=[0, 1, 2],
                    help="score product of the decode kernel: 0 default (= 2), 1 CUDA cores, 2 tcgen05 tensor cores")
    ap.add_argument("--compose-layers", type=int, default=0,
                    help="profiling only: compose just the last N self-decoder layers (0 = all)")
    ap.add_argument("--cross-layers", type=int, default=0,
                    help="profiling only: run just N cross-decoder layers (0 = all)")
    ap.add_argument("--workloads", default=None,
                    help="comma-separated further long-context workloads measured after the headline one, each "
                         "reported under 'workloads' (default: 4,5 with the headline workload 3, else none)")
    return ap.parse_args()


# ---------------------------------------------------------------------------- helpers
def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "compose_append_kernel": ["decode_attention_yocopp_b200/csrc/compose_append.cuh",
                              "decode_attention_yocopp_b200/csrc/common.cuh"],
    "decode_split_kernel": ["decode_attention_yocopp_b200/csrc/decode_attn.cuh",
                            "decode_attention_yocopp_b200/csrc/common.cuh"],
    "decode_tc_kernel": ["decode_attention_yocopp_b200/csrc/decode_attn_tc.cuh",
                         "decode_attention_yocopp_b200/csrc/decode_attn.cuh",
                         "decode_attention_yocopp_b200/csrc/common.cuh"],
    "prefill_tc_kernel": ["decode_attention_yocopp_b200/csrc/prefill_attn_tc.cuh",
                          "decode_attention_yocopp_b200/csrc/common.cuh"],
}


def decode_kernel_name(w, which: int) -> str:
    """The decode kernel the library dispatches for this workload (mirrors the C-ABI rule)."""
    tc = which != 1 and w.dtype == "bf16" and w.d == 128
    return "decode_tc_kernel" if tc else "decode_split_kernel"


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel][workload]
    except Exception:
        return None
    if rec.get("source_hash") != source_hash(KERNEL_SOURCES[kernel]):
        return None
    return rec.get("bytes_per_launch")


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = sorted(float(r[1]) for r in rows)
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": float(rows[0][2]), "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------- distributed
def dist_setup(n):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_workload(cfg: int, rank: int):
    """Weak scaling: every rank serves its own batch of the same shape (its own seed)."""
    import gen
    w = gen.config(cfg)
    if rank:
        w.seed = w.seed + 7919 * rank
    return w


def trim(w, args):
    """Profiling-size step: fewer composed / cross-decoder layers (the shared layer is always kept)."""
    comp = w.composed_layers
    if args.compose_layers:
        comp = comp[-args.compose_layers:]
    cross = w.cross_layers[:args.cross_layers] if args.cross_layers else w.cross_layers
    return comp, cross


# ---------------------------------------------------------------------------- our arm
class Step:
    """Device-resident inputs, caches and outputs of one step of the hot path."""

    def __init__(self, w, comp=None, cross=None):
        import torch
        import gen
        from decode_attention_yocopp_b200.pipeline import SharedKVStack
        self.w = w
        self.tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        comp = comp if comp is not None else w.composed_layers
        self.comp = comp
        self.cross = cross if cross is not None else w.cross_layers
        self.selfl = [1] + comp  # self-decoder layers whose own caches the full decode step reads
        if w.paged:
            self.bt = torch.from_numpy(w.block_table()).cuda()
            self.stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, self.tdt, w.alpha, w.lam,
                                       block_table=self.bt, block_size=w.block_size, num_blocks=w.num_blocks,
                                       cache_layers=[1] + comp)
        else:
            self.stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, self.tdt, w.alpha, w.lam,
                                       capacity=w.max_len, cache_layers=[1] + comp)
        self.lens = torch.tensor(w.lens, dtype=torch.int32, device="cuda")
        self.pos0 = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
        self.posn = torch.clamp(self.lens - 1, min=0)
        self.cu = None if w.uniform else torch.from_numpy(w.cu_prefill.astype("int32")).cuda()
        self.kp = {i: w.device(gen.K_PREFILL, i) for i in [1] + comp}
        self.vp = {i: w.device(gen.V_PREFILL, i) for i in [1] + comp}
        self.kn = {i: w.device(gen.K_NEW, i) for i in [1] + comp}
        self.vn = {i: w.device(gen.V_NEW, i) for i in [1] + comp}
        self.q = {l: w.device(gen.Q, l) for l in self.cross + self.selfl}
        self.out_self = {i: torch.empty((w.batch, w.hq, w.d), dtype=self.tdt, device="cuda") for i in self.selfl}
        self.out = {l: torch.empty((w.batch, w.hq, w.d), dtype=self.tdt, device="cuda") for l in self.cross}
        self.prefill_ntok = w.total_prefill
        self.launches_per_step = 2 * len(comp) + len(self.cross)  # compose x2 per layer, one decode launch per layer

    def setup_fused_contrast(self):
        """Raw caches for the read-time composition contrast: layer 1 (already raw) and a raw
        copy of the shared layer, written at the init alpha (which stores the inputs as they are)."""
        import torch
        from decode_attention_yocopp_b200 import alloc_workspace, make_cache, yocopp_compose_append
        w = self.w
        L2 = w.shared_layer
        k = torch.empty_like(self.stack.k[L2])
        v = torch.empty_like(self.stack.v[L2])
        self.raw_shared = make_cache(k, v, self.bt if w.paged else None)
        init = (0.0, 1.0 / w.lam, 0.0, 1.0 / w.lam)
        if self.cu is None:
            yocopp_compose_append(self.kp[L2], self.vp[L2], self.kp[L2], self.vp[L2], init, w.lam, self.raw_shared,
                                  self.pos0, n_uniform=w.lens[0] - 1, total_new=self.kp[L2].shape[0])
        else:
            yocopp_compose_append(self.kp[L2], self.vp[L2], self.kp[L2], self.vp[L2], init, w.lam, self.raw_shared,
                                  self.pos0, cu_new=self.cu, total_new=self.kp[L2].shape[0])
        yocopp_compose_append(self.kn[L2], self.vn[L2], self.kn[L2], self.vn[L2], init, w.lam, self.raw_shared,
                              self.posn, n_uniform=1, total_new=w.batch)
        self.fused_ws = alloc_workspace(self.raw_shared, w.hq)

    def run_fused(self):
        """Every cross-decoder layer with K', V' composed at read time from two raw caches."""
        from decode_attention_yocopp_b200 import yocopp_decode_attn_fused
        w = self.w
        for l in self.cross:
            yocopp_decode_attn_fused(self.q[l], self.raw_shared, self.stack.desc[1], w.alpha[w.shared_layer], w.lam,
                                     self.lens, self.out[l], self.fused_ws)

    def write_layer1_prefill(self):
        """Layer 1 stores its raw K_1, V_1 (set up once; the composed layers are written every step)."""
        w, s = self.w, self.stack
        if self.cu is None:
            s.write(1, self.kp[1], self.vp[1], self.kp[1], self.vp[1], self.pos0, n_uniform=w.lens[0] - 1)
        else:
            s.write(1, self.kp[1], self.vp[1], self.kp[1], self.vp[1], self.pos0, cu_new=self.cu)

    def run_decode_full(self, ev=None):
        """The attention side of one whole decode step: the decoded token appended to every
        self-decoder layer (layer 1 raw, layers 2..L/2 composed), every self-decoder layer
        attending over its own cache, every cross-decoder layer over the shared cache."""
        w, s = self.w, self.stack
        rec = (lambda k: ev[k].append(_event())) if ev is not None else (lambda k: None)
        rec("a")
        for i in self.selfl:
            s.write(i, self.kn[1], self.vn[1], self.kn[i], self.vn[i], self.posn, n_uniform=1)
        rec("b")
        for i in self.selfl:
            s.self_attend(i, self.q[i], self.lens, self.out_self[i])
        rec("c")
        for l in self.cross:
            s.cross_attend(self.q[l], self.lens, self.out[l])
        rec("d")

    def run(self, ev=None):
        """One step; ev = dict of event lists to record phase boundaries into."""
        w, s = self.w, self.stack
        rec = (lambda k: ev[k].append(_event())) if ev is not None else (lambda k: None)
        rec("t0")
        for i in self.comp:
            if self.cu is None:
                s.write(i, self.kp[1], self.vp[1], self.kp[i], self.vp[i], self.pos0, n_uniform=w.lens[0] - 1)
            else:
                s.write(i, self.kp[1], self.vp[1], self.kp[i], self.vp[i], self.pos0, cu_new=self.cu)
        rec("t1")
        for i in self.comp:
            s.write(i, self.kn[1], self.vn[1], self.kn[i], self.vn[i], self.posn, n_uniform=1)
        rec("t2")
        # the cross-decoder layers back to back (no event between them, so that each launch
        # overlaps the previous one's tail as programmatic dependent launches do in a real step)
        for l in self.cross:
            s.cross_attend(self.q[l], self.lens, self.out[l])
        rec("t3")


def _event():
    import torch
    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def run_ours(args, rank, world, local):
    import torch
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    y.yocopp_set_decode_kernel(args.decode_kernel)
    w = rank_workload(args.config, rank)
    comp_layers, cross_layers = trim(w, args)
    step = Step(w, comp_layers, cross_layers)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    st = y.yocopp_get_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {y.yocopp_status_string(st)}")

    ev = {k: [] for k in ("t0", "t1", "t2", "t3")}
    clocks = Clocks(local) if rank == 0 else None
    if clocks:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    start = _event()
    for _ in range(args.steps):
        step.run(ev)
    stop = _event()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None

    total_ms = start.elapsed_time(stop)
    t_prefill = sum(a.elapsed_time(b) for a, b in zip(ev["t0"], ev["t1"]))
    t_dcomp = sum(a.elapsed_time(b) for a, b in zip(ev["t1"], ev["t2"]))
    t_attn = sum(a.elapsed_time(b) for a, b in zip(ev["t2"], ev["t3"]))
    # average attention launch duration: the cross-decoder layers' span over their count
    per_layer = [t_attn / (args.steps * len(cross_layers))]

    K = args.steps
    kv_bytes_layer = w.kv_bytes()
    kv_bytes = kv_bytes_layer * len(cross_layers) * K
    comp_bytes = w.compose_bytes(w.total_prefill) * len(comp_layers) * K
    # whole job: bytes of all ranks over the slowest rank's time
    t_attn_max = max_over_ranks(t_attn, world)
    t_prefill_max = max_over_ranks(t_prefill, world)
    t_decode_max = max_over_ranks(t_attn + t_dcomp, world)
    total_max = max_over_ranks(total_ms, world)
    kv_all = sum_over_ranks(kv_bytes, world)
    comp_all = sum_over_ranks(comp_bytes, world)
    tok_all = sum_over_ranks(w.batch * K, world)

    # the full attention-side decode step (self-decoder layers included), after the main timing
    step.write_layer1_prefill()
    for _ in range(2):
        step.run_decode_full()
    torch.cuda.synchronize()
    evf = {k: [] for k in "abcd"}
    barrier(world)
    for _ in range(args.steps):
        step.run_decode_full(evf)
    torch.cuda.synchronize()
    t_full = sum(a.elapsed_time(b) for a, b in zip(evf["a"], evf["d"]))
    t_self = sum(a.elapsed_time(b) for a, b in zip(evf["b"], evf["c"]))
    t_full_max = max_over_ranks(t_full, world)
    t_self_max = max_over_ranks(t_self, world)
    # the same decode step captured once in a CUDA graph and replayed
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run_decode_full()
    graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    ga = _event()
    for _ in range(K):
        graph.replay()
    gb = _event()
    torch.cuda.synchronize()
    t_graph_max = max_over_ranks(ga.elapsed_time(gb), world)
    del graph
    self_bytes = sum_over_ranks(w.kv_bytes() * len(step.selfl) * K, world)

    # contrast: the same cross-decoder layers composing K', V' at read time (2x the bytes)
    step.setup_fused_contrast()
    for _ in range(2):
        step.run_fused()
    torch.cuda.synchronize()
    barrier(world)
    fa = _event()
    for _ in range(K):
        step.run_fused()
    fb = _event()
    torch.cuda.synchronize()
    t_fused_max = max_over_ranks(fa.elapsed_time(fb), world)
    del step.raw_shared, step.fused_ws

    prefill = None
    if not args.no_prefill and w.dtype == "bf16" and w.d == 128:
        prefill = run_prefill_attention(args, step, world)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, step, world)
    status = y.yocopp_get_device_status(reset=True)
    if status != 0:
        raise RuntimeError(f"device status after timing: {y.yocopp_status_string(status)}")
    launches = step.launches_per_step * K
    del step
    torch.cuda.empty_cache()

    legs = None
    leg_cfgs = args.workloads if args.workloads is not None else ("4,5" if args.config == 3 else "")
    if leg_cfgs and not (args.compose_layers or args.cross_layers):
        legs = [run_leg(int(c), args, rank, world, local) for c in leg_cfgs.split(",") if c.strip()]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank != 0:
        return None
    peak, peak_kind = hbm_peak()
    value = kv_all / (t_attn_max * 1e-3) / 1e9
    compose_gbs = comp_all / (t_prefill_max * 1e-3) / 1e9
    attn_launch_ms = sum(per_layer) / len(per_layer)
    prefill_launch_ms = t_prefill / (K * len(comp_layers))
    ach_attn = kv_bytes_layer / (attn_launch_ms * 1e-3) / 1e9
    ach_comp = w.compose_bytes(w.total_prefill) / (prefill_launch_ms * 1e-3) / 1e9
    workload = f"{w.name}"
    roof_comp = {"kernel": "compose_append_kernel (prefill size)", "bound": "hbm", "achieved": round(ach_comp, 1),
                 "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(ach_comp / peak, 4),
                 "frac_of_nominal": round(ach_comp / NOMINAL_HBM_GBS, 4),
                 "traffic": ncu_traffic("compose_append_kernel", workload),
                 "algorithmic_bytes_per_launch": w.compose_bytes(w.total_prefill)}
    dk = decode_kernel_name(w, args.decode_kernel)
    roof_attn = {"kernel": f"{dk} (one layer, split + merge)", "bound": "hbm",
                 "achieved": round(ach_attn, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                 "frac": round(ach_attn / peak, 4), "frac_of_nominal": round(ach_attn / NOMINAL_HBM_GBS, 4),
                 "traffic": ncu_traffic(dk, workload),
                 "algorithmic_bytes_per_launch": kv_bytes_layer}
    dominant = roof_comp if t_prefill >= t_attn else roof_attn
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(total_max / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "accumulate": "f32",
        "dtype_note": "caches, q and both tensor-core operands in the storage type; fp32 arithmetic and accumulation",
        "data": "synthetic",
        "config": {"workload": workload, "layers": w.layers, "batch_per_gpu": w.batch, "global_batch": w.batch * world,
                   "context": w.max_len if w.uniform else "ragged", "q_heads": w.hq, "kv_heads": w.hkv,
                   "head_dim": w.d, "paged": w.paged, "parallelism": f"dp{world} (sequences per rank, no exchange)",
                   "l2": "inputs larger than L2 (shared cache and per-step compose streams exceed 126 MB)"},
        "kv_read_frac_of_peak": round(value / world / peak, 4),
        "decode_kernel": decode_kernel_name(w, args.decode_kernel),
        "compose_gbs": round(compose_gbs, 1),
        "compose_frac_of_peak": round(compose_gbs / world / peak, 4),
        "decode_tok_s": round(tok_all / (t_decode_max * 1e-3), 1),
        "decode_compose_us_per_layer": round(1e3 * t_dcomp / (K * len(comp_layers)), 2),
        "decode_full_step": {"tok_s": round(tok_all / (t_full_max * 1e-3), 1),
                             "ms_per_step": round(t_full_max / K, 4),
                             "self_attn_kv_gbs": round(self_bytes / (t_self_max * 1e-3) / 1e9, 1),
                             "cuda_graph_tok_s": round(tok_all / (t_graph_max * 1e-3), 1),
                             "cuda_graph_ms_per_step": round(t_graph_max / K, 4),
                             "what": "decoded token appended to layers 1..L/2, L/2 self-decoder attentions over "
                                     "their own caches, L/2 cross-decoder attentions over the shared cache"},
        "read_time_composition_contrast": {
            "what": "cross-decoder attention composing K', V' from two raw caches while decoding "
                    "(the FusedKV-style alternative); YOCO++ reads one composed cache instead",
            "ms_per_step": round(t_fused_max / K, 4),
            "hbm_read_gbs": round(2 * kv_all / (t_fused_max * 1e-3) / 1e9, 1),
            "slowdown_vs_composed_cache": round(t_fused_max / t_attn_max, 3)},
        "roofline": dominant,
        "prefill_attention": prefill,
        "profiling_trim": bool(args.compose_layers or args.cross_layers),
        "roofline_attention": roof_attn,
        "roofline_compose": roof_comp,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "workloads": legs,
    }
    return line


def run_leg(cfg, args, rank, world, local):
    """A further workload, measured like the headline step (same steps and warm-up,
    CUDA events on the launching stream, max over ranks) with the decode-attention
    and compose rooflines, decode tok/s and the prefill attention beside it."""
    import torch
    import decode_attention_yocopp_b200 as y
    w = rank_workload(cfg, rank)
    step = Step(w)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    st = y.yocopp_get_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"{w.name}: device status after warm-up: {y.yocopp_status_string(st)}")
    ev = {k: [] for k in ("t0", "t1", "t2", "t3")}
    clocks = Clocks(local) if rank == 0 else None
    if clocks:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for _ in range(args.steps):
        step.run(ev)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    K, nc, ncomp = args.steps, len(step.cross), len(step.comp)
    t_prefill = sum(a.elapsed_time(b) for a, b in zip(ev["t0"], ev["t1"]))
    t_dcomp = sum(a.elapsed_time(b) for a, b in zip(ev["t1"], ev["t2"]))
    t_attn = sum(a.elapsed_time(b) for a, b in zip(ev["t2"], ev["t3"]))
    per_layer = [t_attn / (K * nc)]
    t_attn_max = max_over_ranks(t_attn, world)
    t_prefill_max = max_over_ranks(t_prefill, world)
    t_decode_max = max_over_ranks(t_attn + t_dcomp, world)
    kv_all = sum_over_ranks(w.kv_bytes() * nc * K, world)
    comp_all = sum_over_ranks(w.compose_bytes(w.total_prefill) * ncomp * K, world)
    tok_all = sum_over_ranks(w.batch * K, world)
    prefill = None
    if not args.no_prefill and w.dtype == "bf16" and w.d == 128:
        prefill = run_prefill_attention(args, step, world)
    status = y.yocopp_get_device_status(reset=True)
    if status != 0:
        raise RuntimeError(f"{w.name}: device status after timing: {y.yocopp_status_string(status)}")
    del step
    torch.cuda.empty_cache()
    peak, peak_kind = hbm_peak()
    ach_attn = w.kv_bytes() / (sum(per_layer) / len(per_layer) * 1e-3) / 1e9
    ach_comp = w.compose_bytes(w.total_prefill) / (t_prefill / (K * ncomp) * 1e-3) / 1e9
    dk = decode_kernel_name(w, args.decode_kernel)
    return {
        "workload": w.name,
        "config": {"layers": w.layers, "batch_per_gpu": w.batch, "context": w.max_len if w.uniform else "ragged",
                   "total_context": int(sum(w.lens)), "q_heads": w.hq, "kv_heads": w.hkv, "head_dim": w.d,
                   "paged": w.paged, "planted_key": w.planted is not None, "storage": w.dtype},
        "steps": K, "warmup": args.warmup,
        "decode_attention": {"kernel": dk, "kv_read_gbs_job": round(kv_all / (t_attn_max * 1e-3) / 1e9, 1),
                             "achieved_gbs_per_layer": round(ach_attn, 1),
                             "ms_per_layer": round(sum(per_layer) / len(per_layer), 4),
                             "frac": round(ach_attn / peak, 4),
                             "frac_of_nominal": round(ach_attn / NOMINAL_HBM_GBS, 4), "peak": peak,
                             "peak_kind": peak_kind, "traffic": ncu_traffic(dk, w.name),
                             "algorithmic_bytes_per_launch": w.kv_bytes()},
        "compose": {"kernel": "compose_append_kernel (prefill size)",
                    "gbs_job": round(comp_all / (t_prefill_max * 1e-3) / 1e9, 1),
                    "achieved_gbs_per_launch": round(ach_comp, 1),
                    "frac": round(ach_comp / peak, 4),
                    "frac_of_nominal": round(ach_comp / NOMINAL_HBM_GBS, 4), "peak": peak, "peak_kind": peak_kind,
                    "traffic": ncu_traffic("compose_append_kernel", w.name),
                    "algorithmic_bytes_per_launch": w.compose_bytes(w.total_prefill)},
        "decode_tok_s": round(tok_all / (t_decode_max * 1e-3), 1),
        "decode_compose_us_per_layer": round(1e3 * t_dcomp / (K * ncomp), 2),
        "prefill_attention": prefill,
        "clocks": clk,
    }


def tensor_peak():
    """Measured dense bf16 tensor throughput (burst, sustained) in TFLOP/s, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, "fallback"


def causal_pairs(lens) -> int:
    """(query, key) pairs a whole-prompt causal prefill scores: sum over sequences of n (n + 1) / 2."""
    return sum(n * (n + 1) // 2 for n in lens)


def run_prefill_attention(args, step, world):
    """Causal prefill attention of the shared self-decoder layer over its own cache
    (the prefill tokens at positions 0..T-2, already composed by the step), timed
    per launch with CUDA events.  Algorithmic FLOPs: 4 d (2 for q.k, 2 for p v)
    per causal (query, key) pair and query head."""
    import torch
    import gen
    w = step.w
    L = w.shared_layer
    q = w.device(gen.Q_PREFILL, L)
    out = torch.empty_like(q)
    n = w.prefill_lens
    kw = dict(n_uniform=n[0]) if step.cu is None else dict(cu_q=step.cu, max_q=max(n))
    for _ in range(2):
        step.stack.prefill_attend(L, q, out, **kw)
    torch.cuda.synchronize()
    K = max(2, min(args.steps, 5))
    barrier(world)
    marks = [_event()]
    for _ in range(K):
        step.stack.prefill_attend(L, q, out, **kw)
        marks.append(_event())
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in zip(marks[:-1], marks[1:])]
    t_max = max_over_ranks(sum(per), world)
    flops = 4 * w.d * w.hq * causal_pairs(n)
    burst, sustained, kind = tensor_peak()
    ach = flops / (sum(per) / K * 1e-3) / 1e12
    job = sum_over_ranks(flops * K, world) / (t_max * 1e-3) / 1e12
    fused = run_prefill_fused(step, q, out, K, kw, world)
    del q, out
    return {"kernel": "prefill_tc_kernel", "what": "causal attention of one self-decoder layer's prefill tokens "
                                                   "over its own composed cache (bf16, tcgen05 for q.K and P.V)",
            "workload": f"{w.name}: {w.batch} x {n[0] if step.cu is None else 'ragged'} prefill tokens, "
                        f"{w.hq} q / {w.hkv} kv heads, d {w.d}",
            "launches": K, "ms_per_launch": round(sum(per) / K, 4), "tflops_job": round(job, 1),
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": burst, "unit": "TFLOP/s",
                         "frac": round(ach / burst, 4), "peak_kind": f"{kind} bf16 burst",
                         "frac_of_sustained": round(ach / sustained, 4),
                         "algorithmic_flops_per_launch": flops,
                         "traffic": ncu_traffic("prefill_tc_kernel", w.name)},
            "compose_fused": fused}


def run_prefill_fused(step, q, out, K, kw, world):
    """The shared layer's prefill rows composed and attended: two launches
    (yocopp_compose_append, then yocopp_prefill_attn) against one fused launch
    (yocopp_prefill_compose_attn), each timed per pass with CUDA events."""
    import torch
    w, s = step.w, step.stack
    L = w.shared_layer
    pos0 = step.pos0

    def two():
        if step.cu is None:
            s.write(L, step.kp[1], step.vp[1], step.kp[L], step.vp[L], pos0, n_uniform=w.lens[0] - 1)
        else:
            s.write(L, step.kp[1], step.vp[1], step.kp[L], step.vp[L], pos0, cu_new=step.cu)
        s.prefill_attend(L, q, out, pos=pos0, **kw)

    def one():
        s.prefill_write_attend(L, step.kp[1], step.vp[1], step.kp[L], step.vp[L], q, out, pos=pos0, **kw)

    res = {}
    for name, fn in (("two_launches", two), ("fused", one)):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        barrier(world)
        marks = [_event()]
        for _ in range(K):
            fn()
            marks.append(_event())
        torch.cuda.synchronize()
        per = [a.elapsed_time(b) for a, b in zip(marks[:-1], marks[1:])]
        res[name + "_ms"] = round(max_over_ranks(sum(per), world) / K, 4)
    res["fused_speedup"] = round(res["two_launches_ms"] / res["fused_ms"], 4)
    res["what"] = ("composition of the shared layer's prefill rows + their causal attention: "
                   "yocopp_compose_append then yocopp_prefill_attn, against yocopp_prefill_compose_attn")
    return res


def run_e2e(args, step, world):
    """Same metric through the C ABI with host inputs: every step copies its inputs
    from pinned host memory, runs, and reads every layer's output back."""
    import torch
    w = step.w
    comp = step.comp
    # one pinned copy per tensor role; every layer's device input is copied from it
    hk1, hv1 = step.kp[1].cpu().pin_memory(), step.vp[1].cpu().pin_memory()
    hki, hvi = step.kp[comp[-1]].cpu().pin_memory(), step.vp[comp[-1]].cpu().pin_memory()
    hkn = step.kn[1].cpu().pin_memory()
    hq = {l: step.q[l].cpu().pin_memory() for l in step.cross}
    hout = {l: torch.empty(step.out[l].shape, dtype=step.tdt, pin_memory=True) for l in step.cross}
    h2d = 0
    d2h = 0

    def one():
        nonlocal h2d, d2h
        h2d = d2h = 0
        for dst, src in ((step.kp[1], hk1), (step.vp[1], hv1)):
            dst.copy_(src, non_blocking=True)
            h2d += src.numel() * src.element_size()
        for i in comp:
            step.kp[i].copy_(hki, non_blocking=True)
            step.vp[i].copy_(hvi, non_blocking=True)
            h2d += 2 * hki.numel() * hki.element_size()
        for i in [1] + comp:
            step.kn[i].copy_(hkn, non_blocking=True)
            step.vn[i].copy_(hkn, non_blocking=True)
            h2d += 2 * hkn.numel() * hkn.element_size()
        for l in step.cross:
            step.q[l].copy_(hq[l], non_blocking=True)
            h2d += hq[l].numel() * hq[l].element_size()
        step.run()
        for l in step.cross:
            hout[l].copy_(step.out[l], non_blocking=True)
            d2h += hout[l].numel() * hout[l].element_size()

    for _ in range(max(1, min(args.warmup, 2))):
        one()
    torch.cuda.synchronize()
    barrier(world)
    n = max(1, min(args.steps, 3))
    a = _event()
    for _ in range(n):
        one()
    b = _event()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world)
    kv_all = sum_over_ranks(w.kv_bytes() * len(step.cross) * n, world)
    return {"value": round(kv_all / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": round(ms / n, 3),
            "note": "host inputs: one pinned raw K/V pair per role, copied into every layer's device input"}


# ---------------------------------------------------------------------------- oracle (CPU)
def _cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(w, seconds: float, threads: int):
    """Time the oracle on (sequence, kv-head) planes of the workload for about ``seconds``:
    compose of the shared layer's plane from the raw inputs, then attention of one
    cross-decoder layer.  Returns (KV bytes attended, compose bytes, elapsed s, planes)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from oracle import model
    orc = oracle.default()
    planes = [(b, g) for b in range(w.batch) for g in range(w.hkv)]
    L2 = w.shared_layer
    # raw inputs regenerated up front (not timed): the oracle's own work is timed
    pre = {}
    for b, g in planes[: max(1, threads * 2)]:
        pre[b, g] = {(lay, which): model.raw_seq(w, lay, which, b, g) for lay in (1, L2) for which in "KV"}

    def work(bg):
        b, g = bg
        r = pre[b, g]
        a = w.alpha[L2]
        K = orc.round_to(orc.compose(r[1, "K"], r[L2, "K"], a[0], a[1], w.lam, w.dtype), w.dtype)
        V = orc.round_to(orc.compose(r[1, "V"], r[L2, "V"], a[2], a[3], w.lam, w.dtype), w.dtype)
        q = model.query(w, w.cross_layers[0], b)[g * w.group:(g + 1) * w.group]
        orc.attention(q, K, V, w.dtype, 1.0 / math.sqrt(w.d))
        return w.lens[b]

    keys = list(pre)
    done_tok = 0
    done = 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        while time.perf_counter() - t0 < seconds:
            for tok in ex.map(work, keys):
                done_tok += tok
                done += 1
            if time.perf_counter() - t0 > seconds:
                break
    el = time.perf_counter() - t0
    kv = 2 * done_tok * w.d * w.elem_bytes
    comp = 6 * done_tok * w.d * w.elem_bytes
    return kv, comp, el, done


def cpu_baseline(w, seconds):
    threads = _cpu_threads()
    kv, comp, el, n = oracle_sample(w, seconds, threads)
    # the same work on one core, on a shorter sample
    kv1, _, el1, n1 = oracle_sample(w, max(2.0, seconds / 4), 1)
    return {"value": round(kv / el / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} (sequence, kv-head) planes of {w.name}: fp64 compose of the shared layer's plane "
                      f"+ one cross-decoder layer's attention over it, {el:.1f} s",
            "compose_gbs": round(comp / el / 1e9, 4),
            "single_core": {"value": round(kv1 / el1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "sample": f"{n1} planes, {el1:.1f} s"}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = rank_workload(args.config, 0)
    threads = _cpu_threads()
    per_step = max(1.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per_step / 4, threads)
    kv = el = 0.0
    n = 0
    for _ in range(args.steps):
        a, _, e, m = oracle_sample(w, per_step, threads)
        kv += a
        el += e
        n += m
    value = kv / el / 1e9
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * el / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "batch_per_gpu": w.batch, "context": w.max_len if w.uniform else "ragged",
                       "q_heads": w.hq, "kv_heads": w.hkv, "head_dim": w.d, "paged": w.paged},
            "cpu_baseline": {"kind": "oracle", "cores": threads, "value": round(value, 4),
                             "sample": f"{n} (sequence, kv-head) planes over {args.steps} steps"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        line = run_reference(args, rank, world)
    else:
        rank, world, local = dist_setup(args.gpus)
        line = run_ours(args, rank, world, local)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
