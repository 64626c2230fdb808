"""Benchmark of the block-sparse attention path on synthetic video-DiT inputs.

One step = the whole path on one batch: hybrid Top-k ∪ Top-p mask (pool, block
scores, selection), block-sparse attention over the kept tiles, and, for
workloads with the linear branch, the elu+1 state and the alpha blend.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line. `value` is the dense-equivalent attention throughput of a
step, 4*B*H*N^2*d flops over the step time (TFLOP/s, summed over ranks). Inputs
are resident in HBM before timing and each tensor (>= 774 MB) is larger than L2.
Under torchrun every rank runs the full workload on its own GPU (heads are
independent: weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

DEFAULT_WORKLOAD = "wan14b_720p"
METRIC = "sparse_attn_effective_tflops"


# DRAM traffic of one sparse_attn_kernel launch (bf16, blend in the epilogue)
# on the 14B-720p-shaped workload, from an ncu capture of dram__bytes_read.sum
# and dram__bytes_write.sum (one pass) of the bench's own launch; for another
# workload it is scaled by B*H*N*d. `sources_sha` pins the kernel sources the
# counters belong to: once they change, traffic is reported as null until a
# new capture is made.
ATTN_TRAFFIC_CAPTURE = {
    "workload": "wan14b_720p", "dram_bytes_read": 3778778624, "dram_bytes_write": 763836160,
    "sources_sha": "2e7e139c41d0cc61",
    "sources": ("attn_kernel.cu", "sa_device.cuh"),
}


def attn_traffic(wl):
    import hashlib
    cap = ATTN_TRAFFIC_CAPTURE
    h = hashlib.sha256()
    try:
        for f in cap["sources"]:
            with open(os.path.join(ROOT, "block_sparse_attention_softmax_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    if h.hexdigest()[:16] != cap["sources_sha"]:
        return None
    ref = WORKLOADS[cap["workload"]]
    scale = (wl.B * wl.H * wl.N * wl.d) / (ref.B * ref.H * ref.N * ref.d)
    return round((cap["dram_bytes_read"] + cap["dram_bytes_write"]) * scale)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def dense_flops(wl):
    return 4.0 * wl.B * wl.H * wl.N * wl.N * wl.d


def executed_flops(wl, kv_idx, kv_cnt):
    """4*d*sum over kept (q-block, k-block) tiles of valid_q * valid_k."""
    bq, bk, N = wl.bq, wl.bk, wl.N
    cnt = kv_cnt.to(torch.int64)
    valid_q = torch.full((wl.n_qb,), bq, dtype=torch.int64, device=cnt.device)
    valid_q[-1] = N - (wl.n_qb - 1) * bq
    keys = cnt * bk
    last = wl.n_kb - 1
    tail_short = bk - (N - last * bk)
    if tail_short:
        ar = torch.arange(kv_idx.shape[-1], device=cnt.device)
        has_tail = ((kv_idx == last) & (ar < cnt.unsqueeze(-1))).any(-1)
        keys = keys - has_tail.to(torch.int64) * tail_short
    return 4.0 * wl.d * float((keys * valid_q).sum().item())


def run_config(wl, world):
    """The `config` object of both arms' JSON lines (the same keys and values)."""
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d,
            "block": f"{wl.bq}x{wl.bk}", "topk": wl.topk, "topp": wl.topp,
            "linear_branch": wl.linear, "parallelism": f"replica x{world}",
            "l2": (f"inputs larger than L2 (each tensor {wl.B * wl.H * wl.N * wl.d * 2 / 1e6:.0f} MB); no flush"
                   if wl.B * wl.H * wl.N * wl.d * 2 > 126e6 else "inputs smaller than L2; no flush")}


def stats(ms):
    """Median, min, p90 and mean of per-call times (ms)."""
    xs = sorted(ms)
    p90 = xs[min(len(xs) - 1, int(math.ceil(0.9 * len(xs))) - 1)]
    return {"median": round(statistics.median(xs), 4), "min": round(xs[0], 4),
            "p90": round(p90, 4), "mean": round(statistics.mean(xs), 4), "n": len(xs)}


class ClockSampler:
    """SM clock, board power and clock-event reasons sampled every 10 ms during
    the timed region, through NVML read-only queries (nvidia-smi at 200 ms if
    NVML is unavailable). Nothing is set on the GPU."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local, period_s=0.01):
        self.local, self.period = local, period_s
        self.samples = []          # (sm_mhz, power_w, set of reason names)
        self.max_mhz = None
        self.nvml = None
        self.proc = None
        self.stop = threading.Event()
        self.source = None

    def _nvml_handle(self, nv):
        props = torch.cuda.get_device_properties(self.local)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devn = getattr(props, "pci_device_id", 0)
            try:
                return nv.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devn:02x}.0")
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[self.local]) if vis and vis.split(",")[0].isdigit() else self.local
        return nv.nvmlDeviceGetHandleByIndex(idx)

    def _nvml_sample(self):
        nv, h = self.nvml, self.handle
        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        try:
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:
            pw = None
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        return sm, pw, {n for n, c in self.REASONS if bits & getattr(nv, c)}

    def _poll(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self._nvml_sample())
            except Exception:
                return
            self.stop.wait(self.period)

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, self.max_mhz = float(parts[0]), float(parts[1])
                pw = float(parts[2])
            except ValueError:
                continue
            names = [n for n, _ in self.REASONS]
            self.samples.append((sm, pw, {n for n, v in zip(names, parts[4:8]) if v.lower() == "active"}))

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nvml = nv
            self.handle = self._nvml_handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
            self._nvml_sample()          # first query paid before the timed region
            self.source = "nvml 10 ms"
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        except Exception:
            self.nvml = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.local}", f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.t = threading.Thread(target=self._read_smi, daemon=True)
                self.t.start()
                self.source = "nvidia-smi 200 ms"
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.nvml is not None:
            self.t.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": self.source}
        sm = [x[0] for x in self.samples]
        pw = [x[1] for x in self.samples if x[1] is not None]
        reasons = sorted(set().union(*[x[2] for x in self.samples]))
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.max_mhz,
                "power_w_median": round(statistics.median(pw), 1) if pw else None,
                "reasons": reasons, "samples": len(sm), "source": self.source}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our arm
def _event():
    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def _dense_times(sa, q, k, v, bq, o, reps):
    """Per-call ms of our dense attention and of torch SDPA on the same shape."""
    out = {}
    for name, fn in (("ours", lambda: sa.sa_dense_attn_fwd(q, k, v, bq, out=o)),
                     ("sdpa", lambda: torch.nn.functional.scaled_dot_product_attention(q, k, v))):
        try:
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            ev = []
            for _ in range(reps):
                e0 = _event()
                fn()
                ev.append((e0, _event()))
            torch.cuda.synchronize()
            out[name] = stats([x.elapsed_time(y) for x, y in ev])
        except Exception:
            out[name] = None
    return out


def run_ours(args, wl, rank, world, local):
    import block_sparse_attention_softmax_b200 as sa
    lib = sa.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = make_inputs(wl, dev)
    q, k, v, alpha = x["q"], x["k"], x["v"], x["alpha"]
    B, H, N, d = q.shape
    ws_mask = torch.empty(lib.sa_build_mask_workspace_size(B, H, N, d, wl.bq, wl.bk), dtype=torch.uint8, device=dev)
    ws_lin = torch.empty(max(1, lib.sa_linear_workspace_size(B, H, N, d)), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    o_l = torch.empty_like(q) if wl.linear else None

    # our kernels per step: the mask builder's (pooling, then scores and
    # selection, or row statistics, candidate scores, candidate selection and
    # two hand-back launches that return at once when no row was handed back,
    # as the library reports for this shape); with the linear branch, its
    # state, the state's fixed-order reduction and O_l; then the sparse
    # attention, which blends O_l into its output
    launches_per_step = lib.sa_build_mask_launches(B, H, N, d, wl.bq, wl.bk) + 1 + (3 if wl.linear else 0)

    # (start, after mask, after linear branch, after attention) events of each timed step
    marks = []

    def step(record=False):
        if record:
            m0 = _event()
        m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp, workspace=ws_mask)
        if record:
            m1 = _event()
        if wl.linear:
            sa.sa_linear_branch(q, k, v, want_ol=True, workspace=ws_lin, out_ol=o_l)
        if record:
            m2 = _event()
        sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], out=o,
                              o_l=o_l, alpha=alpha if wl.linear else None)
        if record:
            marks.append((m0, m1, m2, _event()))
        return m

    for _ in range(args.warmup):
        m = step()
    torch.cuda.synchronize()
    sa.sa_device_status(dev)
    ex_flops = executed_flops(wl, m["kv_idx"], m["kv_cnt"])
    density = float(m["kv_cnt"].sum().item()) / (B * H * wl.n_qb * wl.n_kb)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(args.steps):
            step(record=True)
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1) / args.steps
    ms_max = max_over_ranks(ms, world, dev)
    mask_t = [a.elapsed_time(b) for a, b, _, _ in marks]
    lin_t = [b.elapsed_time(c) for _, b, c, _ in marks] if wl.linear else []
    attn_t = [c.elapsed_time(e) for _, _, c, e in marks]
    attn_ms, mask_ms = statistics.mean(attn_t), statistics.mean(mask_t)
    lin_ms = statistics.mean(lin_t) if lin_t else None
    sa.sa_device_status(dev)

    # comparison points (not part of the step): dense attention through our
    # kernel and a library dense attention of the same shape (PyTorch SDPA)
    dense = _dense_times(sa, q, k, v, wl.bq, o, 3) if not args.no_dense else {"ours": None, "sdpa": None}

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        ah = alpha.cpu().pin_memory() if alpha is not None else None
        oh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        sa.block_sparse_attention(qh, kh, vh, wl.bq, wl.bk, wl.topk, wl.topp, alpha=ah, out=oh)
        torch.cuda.synchronize()
        reps = max(2, min(args.steps, 5))
        tt0 = time.perf_counter()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            sa.block_sparse_attention(qh, kh, vh, wl.bq, wl.bk, wl.topk, wl.topp, alpha=ah, out=oh)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max(e0.elapsed_time(e1), (time.perf_counter() - tt0) * 1e3) / reps
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh)) + (ah.numel() * 4 if ah is not None else 0)
        e2e = {"value": round(world * dense_flops(wl) / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": q.numel() * 2, "api": "block_sparse_attention (host tensors)"}
        del qh, kh, vh, oh

    hbm, bf16, bf16_s, src = peaks()
    kept = float(m["kv_cnt"].sum().item())
    mask_bytes = int(2 * B * H * N * d * 2 + 4 * kept + 4 * B * H * wl.n_qb)
    achieved = ex_flops / (attn_ms * 1e-3) / 1e12
    d_ours, d_sdpa = dense["ours"], dense["sdpa"]
    result = {
        "metric": METRIC, "value": round(world * dense_flops(wl) / (ms_max * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded video-DiT-shaped Q/K/V)",
        "config": run_config(wl, world),
        "sparse_attn_ms": round(attn_ms, 4), "mask_build_ms": round(mask_ms, 4),
        "linear_branch_ms": None if lin_ms is None else round(lin_ms, 4),
        "blend": "in the sparse attention epilogue" if wl.linear else None,
        "per_call_ms": {"sparse_attn": stats(attn_t), "mask_build": stats(mask_t),
                        "linear_branch": stats(lin_t) if lin_t else None},
        # in call order: NVML's clock reading lags the power controller, so
        # a drop of the SM clock under the power cap part-way through the
        # timed region shows here first
        "sparse_attn_ms_in_order": [round(x, 3) for x in attn_t],
        "dense_attn_ms": None if d_ours is None else d_ours["median"],
        "torch_sdpa_dense_ms": None if d_sdpa is None else d_sdpa["median"],
        "speedup_vs_dense": None if d_ours is None else round(d_ours["median"] / attn_ms, 2),
        "density": round(density, 5), "executed_tflop_per_call": round(ex_flops / 1e12, 4),
        "roofline": {"kernel": "sparse_attn_kernel<128>", "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": bf16, "unit": "TFLOP/s", "frac": round(achieved / bf16, 4),
                     "peak_source": f"{src} bf16 burst", "traffic": attn_traffic(wl),
                     "traffic_unit": "bytes per launch",
                     "traffic_note": "ncu dram read+write of this launch on the 14B-720p workload (scaled by B*H*N*d for others)"},
        "mask_builder_roofline": {"bound": "hbm", "achieved": round(mask_bytes / (mask_ms * 1e-3) / 1e9, 1),
                                  "peak": hbm, "unit": "GB/s", "frac": round(mask_bytes / (mask_ms * 1e-3) / 1e9 / hbm, 4),
                                  "bytes_per_call": mask_bytes,
                                  "bytes_note": "Q and K read once plus the kept kv_idx entries and kv_cnt"},
        "e2e": e2e, "gpu_launches": args.steps * launches_per_step,
        "clocks": clk.summary(),
    }
    return result


PER_WORKLOAD = ("tiny", "wan13b_480p", "sink_skew", "long_245k")


def _times(fn, calls=5, warmup=2):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = []
    for _ in range(calls):
        e0 = _event()
        fn()
        ev.append((e0, _event()))
    torch.cuda.synchronize()
    return stats([x.elapsed_time(y) for x, y in ev])


def measure_backward(sa, wl, dev):
    """The backward of one step on the workload: the sparse attention's dq, dk,
    dv over the step's lists, and with the linear branch its gradients and the
    blend's. Algorithmic flops of the sparse backward: 7 products per kept tile
    (S and dP recomputed for dq and for dk/dv, then dq, dk, dv), 3.5 x the
    forward's 2."""
    x = make_inputs(wl, dev)
    q, k, v, alpha = x["q"], x["k"], x["v"], x["alpha"]
    m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp)
    o, lse = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], want_lse=True)
    dout = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(5), device=dev).to(torch.bfloat16)
    ex = executed_flops(wl, m["kv_idx"], m["kv_cnt"])
    res = {"sparse_attn_bwd_ms": _times(lambda: sa.sa_sparse_attn_bwd(q, k, v, o, lse, dout, wl.bq, wl.bk,
                                                                       m["kv_idx"], m["kv_cnt"]))}
    hbm, bf16, _, src = peaks()
    tf = 3.5 * ex / (res["sparse_attn_bwd_ms"]["median"] * 1e-3) / 1e12
    res.update({"sparse_attn_bwd_exec_tflops": round(tf, 1), "sparse_attn_bwd_frac_of_bf16_peak": round(tf / bf16, 4),
                "flops_note": "3.5 x the forward's executed flops (7 tile products: S, dP twice, dq, dk, dv)"})
    if wl.linear:
        S, z, o_l = sa.sa_linear_branch(q, k, v, want_ol=True)
        res["linear_bwd_ms"] = _times(lambda: sa.sa_linear_bwd(q, k, v, S, z, dout))
        res["blend_bwd_ms"] = _times(lambda: sa.sa_blend_bwd(o, o_l, alpha, dout))
    sa.sa_device_status(dev)
    del x, q, k, v, o, lse, dout, m
    torch.cuda.empty_cache()
    return res


def measure_low_bit_forward(sa, wl, dev):
    """The low-bit forward on the workload: per-head E4M3 quantisation of Q, K
    and V, and the sparse attention on E4M3 operands (with the blend when the
    workload has the linear branch) over the step's lists. Its roofline peak is
    the measured bf16 peak times the nominal fp8 / bf16 ratio of 2."""
    x = make_inputs(wl, dev)
    q, k, v, alpha = x["q"], x["k"], x["v"], x["alpha"]
    m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp)
    ex = executed_flops(wl, m["kv_idx"], m["kv_cnt"])
    q8, qs = sa.sa_quantize_fp8(q)
    k8, ks = sa.sa_quantize_fp8(k)
    v8, vs = sa.sa_quantize_fp8(v)
    quant = _times(lambda: (sa.sa_quantize_fp8(q, out=q8, scale_out=qs), sa.sa_quantize_fp8(k, out=k8, scale_out=ks),
                            sa.sa_quantize_fp8(v, out=v8, scale_out=vs)))
    o_l = alpha_t = None
    if wl.linear:
        _, _, o_l = sa.sa_linear_branch(q, k, v, want_ol=True)
        alpha_t = alpha
    o8 = torch.empty_like(q)
    attn8 = _times(lambda: sa.sa_sparse_attn_fp8_fwd(q8, k8, v8, qs, ks, vs, wl.bq, wl.bk, kv_idx=m["kv_idx"],
                                                     kv_cnt=m["kv_cnt"], out=o8, o_l=o_l, alpha=alpha_t), calls=10)
    o16 = torch.empty_like(q)
    attn16 = _times(lambda: sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"],
                                                  out=o16, o_l=o_l, alpha=alpha_t), calls=10)
    diff = (o8.float() - o16.float()).abs()
    hbm, bf16, _, src = peaks()
    tf = ex / (attn8["median"] * 1e-3) / 1e12
    qbytes = 3 * q.numel() * (2 + 1)             # algorithmic: x read once, codes written (the amax pass reads x again)
    res = {"quantize_qkv_ms": quant, "quantize_gbs": round(qbytes / (quant["median"] * 1e-3) / 1e9, 1),
           "quantize_frac_of_hbm": round(qbytes / (quant["median"] * 1e-3) / 1e9 / hbm, 4),
           "sparse_attn_fp8_ms": attn8, "sparse_attn_bf16_same_calls_ms": attn16,
           "sparse_attn_fp8_exec_tflops": round(tf, 1),
           "sparse_attn_fp8_frac_of_fp8_peak": round(tf / (2 * bf16), 4),
           "peak_note": f"fp8 peak = 2 x the {src} bf16 burst peak ({2 * bf16:.0f} TFLOP/s)",
           "blend": bool(wl.linear),
           "max_abs_diff_vs_bf16_path": round(float(diff.max()), 5),
           "mean_abs_diff_vs_bf16_path": round(float(diff.mean()), 6)}
    sa.sa_device_status(dev)
    del x, q, k, v, q8, k8, v8, o8, o16, m, o_l, diff
    torch.cuda.empty_cache()
    return res


def measure_tile_scoring_and_layouts(sa, dev):
    """Veda's max-pooled heatmap (two tensor-core sweeps of Q K^T over every
    tile: 4 N^2 d flops per head) on the 1.3B-480p shape, all query blocks and
    a 1/8 sample; and the sparse path on per-head 3-D tilings of its latent
    grid (gather, mask, attention, scatter) against the raster order."""
    wl = WORKLOADS["wan13b_480p"]
    x = make_inputs(wl, dev)
    q, k, v = x["q"], x["k"], x["v"]
    hbm, bf16, _, src = peaks()
    heat = torch.empty(wl.B, wl.H, wl.n_qb, wl.n_kb, dtype=torch.float32, device=dev)
    full = _times(lambda: sa.sa_tile_heatmap(q, k, wl.bq, out=heat), calls=3)
    fl = 4.0 * wl.B * wl.H * wl.N * wl.N * wl.d
    rows = torch.arange(0, wl.B * wl.H * wl.n_qb, 8, dtype=torch.int32, device=dev)
    part = _times(lambda: sa.sa_tile_heatmap(q, k, wl.bq, rows=rows, out=heat), calls=3)
    tiles = [(1, 2, 32), (3, 5, 4), (1, 1, 64), (3, 2, 8)] * (wl.H // 4)
    perm = sa.sa_tile_permutation(wl.grid, tiles)
    raster = _times(lambda: sa.block_sparse_attention(q, k, v, wl.bq, wl.bk, wl.topk, wl.topp), calls=5)
    permuted = _times(lambda: sa.block_sparse_attention(q, k, v, wl.bq, wl.bk, wl.topk, wl.topp, perm=perm), calls=5)
    qp, kp = sa.sa_permute_tokens(q, perm), sa.sa_permute_tokens(k, perm)
    dens = float(sa.sa_build_mask(qp, kp, wl.bq, wl.bk, wl.topk, wl.topp)["kv_cnt"].sum()) / (wl.H * wl.n_qb * wl.n_kb)
    sa.sa_device_status(dev)
    del x, q, k, v, heat, qp, kp
    torch.cuda.empty_cache()
    return {"workload": wl.name,
            "tile_heatmap_ms": full, "tile_heatmap_tflops": round(fl / (full["median"] * 1e-3) / 1e12, 1),
            "tile_heatmap_frac_of_bf16_peak": round(fl / (full["median"] * 1e-3) / 1e12 / bf16, 4),
            "tile_heatmap_sampled_1_in_8_ms": part,
            "path_raster_ms": raster, "path_per_head_tilings_ms": permuted,
            "tilings": "per head, cycling (1,2,32), (3,5,4), (1,1,64), (3,2,8) over the 21x30x52 grid",
            "density_per_head_tilings": round(dens, 5)}


def measure_workload(sa, wl, dev, calls, warmup, dense_reps, flush):
    """One workload's step components, each call timed on its own with CUDA
    events (an L2 flush between calls when the inputs fit in L2), with its own
    clock record: mask build, sparse attention (executed-tile TFLOP/s and
    fraction of the bf16 peak), linear + blend when the workload has them, and
    dense attention, ours and torch SDPA."""
    lib = sa.load()
    x = make_inputs(wl, dev)
    q, k, v, alpha = x["q"], x["k"], x["v"], x["alpha"]
    B, H, N, d = q.shape
    ws_mask = torch.empty(lib.sa_build_mask_workspace_size(B, H, N, d, wl.bq, wl.bk), dtype=torch.uint8, device=dev)
    ws_lin = torch.empty(max(1, lib.sa_linear_workspace_size(B, H, N, d)), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    o_l = torch.empty_like(q) if wl.linear else None
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    marks = []
    for i in range(warmup + calls):
        if scratch is not None:
            scratch.fill_(i & 0xFF)
        m0 = _event()
        m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp, workspace=ws_mask)
        m1 = _event()
        if scratch is not None:
            scratch.fill_((i + 1) & 0xFF)
        m4 = m5 = None
        if wl.linear:
            m4 = _event()
            sa.sa_linear_branch(q, k, v, want_ol=True, workspace=ws_lin, out_ol=o_l)
            m5 = _event()
        m2 = _event()
        sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], out=o,
                              o_l=o_l, alpha=alpha if wl.linear else None)
        m3 = _event()
        if i >= warmup:
            marks.append((m0, m1, m2, m3, m4, m5))
        if i == warmup - 1:
            torch.cuda.synchronize()
            clk = ClockSampler(dev.index).__enter__()
    torch.cuda.synchronize()
    clk.__exit__(None, None, None)
    sa.sa_device_status(dev)
    mask_t = [a.elapsed_time(b) for a, b, *_ in marks]
    attn_t = [c.elapsed_time(e) for _, _, c, e, _, _ in marks]
    lin_t = [a.elapsed_time(b) for *_, a, b in marks if a is not None]
    ex = executed_flops(wl, m["kv_idx"], m["kv_cnt"])
    kept = float(m["kv_cnt"].sum().item())
    density = kept / (B * H * wl.n_qb * wl.n_kb)
    hbm, bf16, _, src = peaks()
    mask_bytes = 2 * B * H * N * d * 2 + 4 * kept + 4 * B * H * wl.n_qb
    dense = _dense_times(sa, q, k, v, wl.bq, o, dense_reps) if dense_reps else {"ours": None, "sdpa": None}
    sa.sa_device_status(dev)
    sp, mk = stats(attn_t), stats(mask_t)
    res = {
        "config": {"B": B, "H": H, "N": N, "d": d, "block": f"{wl.bq}x{wl.bk}", "topk": wl.topk,
                   "topp": wl.topp, "linear_branch": wl.linear,
                   "l2": "256 MB flush before each timed call" if flush else "inputs larger than L2; no flush"},
        "density": round(density, 5), "executed_tflop_per_call": round(ex / 1e12, 5),
        "sparse_attn_ms": sp, "mask_build_ms": mk,
        "sparse_exec_tflops": round(ex / (sp["median"] * 1e-3) / 1e12, 1),
        "sparse_frac_of_bf16_peak": round(ex / (sp["median"] * 1e-3) / 1e12 / bf16, 4),
        "mask_gbs": round(mask_bytes / (mk["median"] * 1e-3) / 1e9, 1),
        "mask_frac_of_hbm": round(mask_bytes / (mk["median"] * 1e-3) / 1e9 / hbm, 4),
        "linear_branch_ms": stats(lin_t) if lin_t else None,
        "dense_attn_ms": dense["ours"], "torch_sdpa_dense_ms": dense["sdpa"],
        "speedup_vs_our_dense": None if dense["ours"] is None else round(dense["ours"]["median"] / sp["median"], 2),
        "peaks": f"{src}: bf16 {bf16} TFLOP/s burst, HBM {hbm} GB/s; fractions from medians",
        "clocks": clk.summary(),
    }
    del x, q, k, v, o, o_l, ws_mask, ws_lin, scratch
    torch.cuda.empty_cache()
    return res


def run_per_workload(args, dev):
    import block_sparse_attention_softmax_b200 as sa
    out = {}
    for name in PER_WORKLOAD:
        wl = WORKLOADS[name]
        fits_l2 = wl.B * wl.H * wl.N * wl.d * 2 < (256 << 20)
        reps = 3 if wl.N > 100000 else 5
        out[name] = measure_workload(sa, wl, dev, calls=20, warmup=3, dense_reps=0 if args.no_dense else reps,
                                     flush=fits_l2)
    return out


# ------------------------------------------------------------------ oracle (CPU)
def oracle_step_estimate(wl, x, n_heads, n_blocks=32):
    """Time the fp64 oracle on a bounded sample of one step and scale it up.

    Sample: for each of the first n_heads heads, the whole mask (pool, scores,
    selection), attention on every row of n_blocks query blocks (scaled by
    the head's kept tiles over the sample's), and, with the linear branch, its
    state and output; the per-head mean is scaled by the number of heads.
    Returns (seconds per step, description, threads).
    """
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    t_mask = t_attn = t_attn_sample = t_lin = 0.0
    n_heads = min(n_heads, x["q"].shape[1])
    nb = min(wl.n_qb, n_blocks)
    for h in range(n_heads):
        qh, kh, vh = (oracle.as_f64(x[n][0, h]) for n in ("q", "k", "v"))
        t0 = time.perf_counter()
        ref = oracle.build_mask(qh, kh, wl.bq, wl.bk, wl.topk, wl.topp)
        t_mask += time.perf_counter() - t0
        blocks = rng.choice(wl.n_qb, size=nb, replace=False)
        rows = np.concatenate([np.arange(b * wl.bq, min(wl.N, (b + 1) * wl.bq)) for b in blocks])
        t0 = time.perf_counter()
        oracle.masked_attention(qh, kh, vh, ref["mask"], wl.bq, wl.bk, rows=rows)
        dt = time.perf_counter() - t0
        t_attn_sample += dt
        t_attn += dt * float(ref["mask"].sum()) / max(float(ref["mask"][blocks].sum()), 1.0)
        if wl.linear:
            t0 = time.perf_counter()
            S, z = oracle.linear_state(kh, vh)
            oracle.linear_out(qh, S, z)
            t_lin += time.perf_counter() - t0
    per_head = (t_mask + t_attn + t_lin) / n_heads
    sec = per_head * wl.B * wl.H
    desc = (f"{n_heads} of {wl.B * wl.H} heads: full masks ({t_mask:.2f}s), attention on every row of {nb} "
            f"query blocks per head ({t_attn_sample:.2f}s), scaled by kept tiles to whole heads"
            + (f", linear branch ({t_lin:.2f}s)" if wl.linear else "")
            + "; mean per head scaled by the head count (extrapolated)")
    return sec, desc, cores


def run_reference(args, wl):
    """The oracle as the reference arm: each step is a bounded sample of the workload."""
    x = _head_inputs(wl, REF_HEADS)
    secs = []
    for i in range(args.warmup + args.steps):
        s, desc, cores = oracle_step_estimate(wl, x, REF_HEADS)
        if i >= args.warmup:
            secs.append(s)
    ms = statistics.mean(secs) * 1e3
    val = dense_flops(wl) / (ms * 1e-3) / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded video-DiT-shaped Q/K/V)",
            "config": run_config(wl, int(os.environ.get("WORLD_SIZE", "1"))),
            "extrapolated": True,
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": desc, "extrapolated": True},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


REF_HEADS = 2          # heads per reference-arm step (a few seconds of CPU work each)
CPU_SAMPLE_HEADS = 8     # heads of the cpu_baseline sample (about 10 s of CPU work)


def _head_inputs(wl, n):
    """Inputs of the first n heads only (the oracle sample never reads the others;
    the generator draws head by head, so these equal the full workload's)."""
    from dataclasses import replace
    return make_inputs(replace(wl, H=min(n, wl.H)), "cpu")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per-workload measurements of the other four configurations")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first H heads of the workload (small cases for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = WORKLOADS[args.workload]
    if args.heads > 0:
        from dataclasses import replace
        wl = replace(wl, H=min(args.heads, wl.H))
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        print(json.dumps(run_reference(args, wl)), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    res = run_ours(args, wl, rank, world, local)
    if world == 1 and not args.no_per_workload:
        import block_sparse_attention_softmax_b200 as sa
        dev = torch.device("cuda", local)
        res["backward"] = measure_backward(sa, wl, dev)
        res["low_bit_forward"] = measure_low_bit_forward(sa, wl, dev)
        res["tile_scoring_and_layouts"] = measure_tile_scoring_and_layouts(sa, dev)
        res["per_workload"] = run_per_workload(args, dev)
    if rank == 0:
        if not args.no_cpu_baseline:
            x = _head_inputs(wl, CPU_SAMPLE_HEADS)
            sec, desc, cores = oracle_step_estimate(wl, x, CPU_SAMPLE_HEADS)
            res["cpu_baseline"] = {"value": round(dense_flops(wl) / sec / 1e12, 6), "unit": "TFLOP/s",
                                   "cores": cores, "kind": "oracle", "sample": desc,
                                   "ms_per_step": round(sec * 1e3, 1), "extrapolated": True}
            try:
                from threadpoolctl import threadpool_limits
                with threadpool_limits(1):
                    sec1, _, _ = oracle_step_estimate(wl, x, CPU_SAMPLE_HEADS)
                res["cpu_baseline"]["one_thread"] = {"value": round(dense_flops(wl) / sec1 / 1e12, 6),
                                                     "ms_per_step": round(sec1 * 1e3, 1), "cores": 1}
            except ImportError:
                pass
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
