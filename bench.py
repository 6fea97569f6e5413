"""Benchmark of the N:M sparse linear layer on B200.

One step = one pass of the hot path over one batch of synthetic input:
  activation sparsity (8:16, 16:32, tiny 2:4): prune + window-compress X,
      then the 2:4 sparse GEMM against the offline-lifted weight (optionally
      with the per-token shift and variance corrections around the prune);
  weight sparsity (6:8 sliding windows): lift X online, then the sparse GEMM
      against the offline-decomposed weight;
  hybrid dense + 2:4 weight (decode): gather X by the column permutation and
      one input-split GEMM;
  hybrid GLU MLP (decode): one output-split GEMM for up and gate, the SiLU
      gate, one input-split GEMM for down.
The headline line is the largest single-GPU workload: the Llama-8B down_proj
prefill shape with 16:32 activation sparsity (X [4096 x 14336] N(0, 1) with
0.1% of the channels scaled x20, W [4096 x 14336] N(0, 0.02), bf16, fp32
accumulation, bf16 out).  Every other workload is reported, compactly, under
"workloads" in the same line (fields named by "workloads_fields"); --detail
PATH also writes every workload's full record to PATH.

Timing: CUDA events on the launching stream, W warm-up steps, exactly K timed
steps between barriers + device synchronisation, max over ranks.  Every
workload rotates its inputs (and weights, where they would fit in L2) over
enough device buffers that the bytes touched between two uses of a buffer
exceed 2x L2.  Decode workloads replay the K steps from a CUDA graph.  Clocks
and throttle reasons are polled with NVML during the timed region.

`--impl reference` times the CPU oracle on the host cores instead (a bounded
sample of the headline workload per step).
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "down_proj_16of32_act"
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the
# dominant kernel, from one ncu capture of the kernel as it stands (see
# profiles/); drop an entry whenever that kernel changes.
TRAFFIC = {
    ("down_proj_16of32_act", "k_nm_gemm_2cta<256,1,1>+split2"): 756424704 + 32884480,
    ("up_proj_8of16_act", "k_nm_gemm_2cta<224,2,1>"): 232238080 + 46364672,
    ("hybrid_decode_b8", "k_nm_gemm<16>"): 79020544 + 1609728,
    ("hybrid_decode_b128", "k_nm_gemm_2cta<128,2,1>"): 80018432 + 1831936,
    ("slide_6of8_wt_decode", "k_nm_gemm<16>"): 28556800 + 0,
    ("slide_6of8_wt_prefill", "k_nm_gemm_2cta<224,2,1>"): 81972736 + 17421056,
}
OTHERS = ["up_proj_8of16_act", "up_proj_2of4_act", "up_proj_8of16_act_fp8", "up_proj_8of16_act_xf",
          "slide_6of8_wt_prefill", "slide_6of8_wt_prefill_fp8",
          "slide_6of8_wt_decode", "slide_6of8_wt_decode_fp8",
          "hybrid_decode_b1", "hybrid_decode_b8", "hybrid_decode_b32", "hybrid_decode_b128",
          "spense_mlp_decode_b1", "spense_mlp_decode_b8", "spense_mlp_decode_b32", "spense_mlp_decode_b128",
          "tiny_2of4_act_fp32"]
L2_BYTES = 126 * 1024 * 1024
METRIC = "N:M sparse linear TFLOP/s (dense-equiv)"
REF_TOTAL_S = 150.0


def workload_config(wl, ws: int = 1) -> dict:
    """The workload's `config` dict; both arms print the same one."""
    c = {"workload": wl.name, "T": wl.T, "K": wl.K, "O": wl.O, "N": wl.N, "M": wl.M, "side": wl.side,
         "K_lift": wl.K_lift, "x_dist": wl.x_dist, "w_std": wl.w_std,
         "l2": "rotated buffers, >2x L2 touched between reuses",
         "parallelism": f"replicas x{ws} (no data-path collective)"}
    if wl.fp8:
        c["precision"] = "e4m3 operands"
    if wl.xf:
        c["corrections"] = {1: "D-PTS", 2: "VAR", 3: "D-PTS+VAR"}[wl.xf]
    return c


def sig(v, n: int = 4):
    """v rounded to n significant digits (None stays None)."""
    if v is None:
        return None
    return float(f"{v:.{n}g}")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sust=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


class ClockSampler:
    """Polls NVML (SM clock, throttle reasons) in a thread while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                break
            time.sleep(0.0002)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv is not None:
            self._stop.set()
            self.t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest `value` over all ranks (every rank receives it); the
    identity without a process group.  Timed regions are reported as the
    slowest rank's."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(per_rank_work: float, world_size: int, ms_max: float) -> float:
    """Aggregate throughput of `world_size` replicas that each did
    `per_rank_work` units in a timed region whose slowest rank took ms_max."""
    return world_size * per_rank_work / (ms_max * 1e-3)


# ------------------------------------------------------------ CPU baseline


def cpu_oracle_sample(wl, x, w, budget_s: float, wf=None):
    """Times the oracle (prune + windows + metadata + fp64 GEMM) on whole rows
    of X until about budget_s seconds have passed.  Returns (dense-equiv
    TFLOP/s, rows, seconds, threads).  wf: W widened to fp64 (set-up, not
    timed), computed here when not given."""
    import oracle
    if wf is None:
        wf = oracle.to_f64(w)
    rows_done, t_used = 0, 0.0
    t_prune = 0.0
    chunk = 16
    while t_used < budget_s and rows_done < wl.T:
        xs = np.ascontiguousarray(x[rows_done:rows_done + chunk])
        t0 = time.perf_counter()
        keep = oracle.prune(xs, wl.N, wl.M)
        vals, nib = oracle.compress(xs, keep, wl.M)
        oracle.meta_hw(nib, oracle.lifted_k(wl.K, wl.M))
        t1 = time.perf_counter()
        oracle.linear_f64(oracle.to_f64(xs, keep), wf)
        t2 = time.perf_counter()
        t_prune += t1 - t0
        t_used += t2 - t0
        rows_done += xs.shape[0]
    flops = 2.0 * rows_done * wl.O * wl.K
    cpu_oracle_sample.last_split = {"prune_windows_meta_s": t_prune, "fp64_gemm_s": t_used - t_prune}
    return flops / t_used / 1e12, rows_done, t_used, oracle.num_threads()


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), for the CPU baseline."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def run_reference(args):
    ws, rank, _ = _dist_env()
    if rank != 0:
        return 0
    import oracle
    from semi_structured_sparse_nm_b200 import inputs
    wl, x, w = inputs.make_workload(HEADLINE)
    wf = oracle.to_f64(w)
    # each step is a bounded sample of the workload (whole token rows): the
    # whole run stays within about REF_TOTAL_S seconds of oracle time, and a
    # step's time is the time of the work it did
    step_s = min(args.ref_step_s, max(0.25, REF_TOTAL_S / (args.warmup + args.steps)))
    secs, rows_list = [], []
    for i in range(args.warmup + args.steps):
        tf, r, t, thr = cpu_oracle_sample(wl, x, w, budget_s=step_s, wf=wf)
        if i >= args.warmup:
            secs.append(t)
            rows_list.append(r)
    t_step = float(np.mean(secs))
    value = 2.0 * wl.O * wl.K * float(np.sum(rows_list)) / float(np.sum(secs)) / 1e12
    sample = (f"{int(np.mean(rows_list))} of {wl.T} token rows per step: prune+windows+metadata+fp64 GEMM "
              f"against all of W")
    line = {
        "impl": "reference", "metric": METRIC, "value": sig(value), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sig(t_step * 1e3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, ws),
        "cpu_baseline": {"value": sig(value), "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": sample,
                         "cpu": cpu_model(), "nproc": os.cpu_count()},
        "e2e": {"value": sig(value), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- GPU arm


class Workload:
    """Device state of one workload and its step (two kernels: a prep kernel
    -- prune, lift or gather -- and the GEMM)."""

    def __init__(self, name, dev):
        import torch
        from semi_structured_sparse_nm_b200 import _lib as nm
        from semi_structured_sparse_nm_b200 import inputs
        self.nm, self.torch = nm, torch
        self.wl, x_np, w_np = inputs.make_workload(name, seed=0)
        self.x_np, self.w_np = x_np, w_np
        wl = self.wl
        self.name, self.dev = name, dev
        to_dev = (lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)) if wl.x_dtype == "bf16" \
            else (lambda a: torch.from_numpy(a).to(dev))
        X0, W = to_dev(x_np), to_dev(w_np)
        out_dt = torch.bfloat16 if wl.out_dtype == "bf16" else torch.float32
        self.decode = wl.side == "hybrid" or wl.T <= 128
        if wl.side == "act" and wl.fp8:
            self.Wq = nm.quant_lift_fp8(W, wl.M)                         # offline: per-channel codes, lifted
            self.R = max(2, min(8, int(np.ceil(2 * L2_BYTES / max(X0.numel() * X0.element_size(), 1)))))
            self.X = [X0] + [X0.roll(r, dims=0).contiguous() for r in range(1, self.R)]
            Kl = wl.K_lift
            self.comp = [nm.Fp8Operand(torch.empty((wl.T, Kl // 2), dtype=torch.uint8, device=dev),
                                       torch.empty(wl.T, dtype=torch.float32, device=dev), wl.T, wl.K, wl.N, wl.M,
                                       torch.empty(max(nm.meta_bytes(wl.T, wl.K, wl.M), 16), dtype=torch.uint8,
                                                   device=dev)) for _ in range(2)]
            self.Y = torch.empty((wl.T, wl.O), dtype=out_dt, device=dev)
            self.rows_a, self.rows_b = wl.T, wl.O
            self.prep_name, self.gemm_name = "prune_compress_fp8", "sparse_gemm_fp8"
            self.launches_per_step = 3                               # row scales, prune, GEMM
        elif wl.side == "act" and wl.xf:
            self.Wl = nm.lift(W, wl.M)                                   # offline
            self.wsum = nm.row_sums(W)                                   # offline
            self.R = max(2, min(8, int(np.ceil(2 * L2_BYTES / max(X0.numel() * X0.element_size(), 1)))))
            self.X = [X0] + [X0.roll(r, dims=0).contiguous() for r in range(1, self.R)]
            self.comp = [nm.alloc_xf(wl.T, wl.K, wl.N, wl.M, wl.xf, dev) for _ in range(2)]
            self.Y = torch.empty((wl.T, wl.O), dtype=out_dt, device=dev)
            self.rows_a, self.rows_b = wl.T, wl.O
            self.prep_name, self.gemm_name = "prune_compress_xf", "sparse_gemm_xf"
            # token means (with the shift), prune, factors, GEMM
            self.launches_per_step = 4 if wl.xf & nm.NM_XF_SHIFT else 3
        elif wl.side == "act":
            self.Wl = nm.lift(W, wl.M)                                   # offline
            self.R = max(2, min(8, int(np.ceil(2 * L2_BYTES / max(X0.numel() * X0.element_size(), 1)))))
            self.X = [X0] + [X0.roll(r, dims=0).contiguous() for r in range(1, self.R)]
            self.comp = [nm.alloc_compressed(wl.T, wl.K, wl.N, wl.M, dev) for _ in range(2)]
            self.Y = torch.empty((wl.T, wl.O), dtype=out_dt, device=dev)
            self.rows_a, self.rows_b = wl.T, wl.O
            self.prep_name, self.gemm_name = "prune_compress", "sparse_gemm"
        elif wl.side == "weight" and wl.fp8:
            P = nm.slide_decompose_fp8(W, wl.N, wl.M)                  # offline
            wbytes = P.codes.numel() + P.meta.numel() + P.scale.numel() * 4
            xbytes = X0.numel() * 2
            self.R = max(2, int(np.ceil(2 * L2_BYTES / (wbytes + xbytes))))
            self.P = [P] + [nm.Fp8Operand(P.codes.clone(), P.scale.clone(), wl.O, wl.K, wl.N, wl.M, P.meta.clone())
                            for _ in range(1, self.R)]
            self.X = [X0] + [X0.roll(r, dims=0).contiguous() for r in range(1, self.R)]
            self.Q = [nm.Fp8Operand(torch.empty((wl.T, wl.K_lift), dtype=torch.uint8, device=dev),
                                    torch.empty(wl.T, dtype=torch.float32, device=dev), wl.T, wl.K, 0, wl.M)
                      for _ in range(2)]
            self.Y = torch.empty((wl.T, wl.O), dtype=out_dt, device=dev)
            self.rows_a, self.rows_b = wl.O, wl.T
            self.prep_name, self.gemm_name = "quant_lift_fp8", "sparse_gemm_fp8"
            self.w_bytes = wbytes
        elif wl.side == "weight":
            Wc = nm.slide_decompose(W, wl.N, wl.M)                     # offline
            wbytes = Wc.vals.numel() * 2 + Wc.meta.numel()
            xbytes = X0.numel() * 2
            self.R = max(2, int(np.ceil(2 * L2_BYTES / (wbytes + xbytes))))
            self.Wc = [Wc] + [nm.Compressed(Wc.vals.clone(), Wc.meta.clone(), wl.O, wl.K, wl.N, wl.M)
                              for _ in range(1, self.R)]
            self.X = [X0] + [X0.roll(r, dims=0).contiguous() for r in range(1, self.R)]
            self.Xl = [torch.empty((wl.T, wl.K_lift), dtype=torch.bfloat16, device=dev) for _ in range(2)]
            self.Y = torch.empty((wl.T, wl.O), dtype=out_dt, device=dev)
            self.rows_a, self.rows_b = wl.O, wl.T
            self.prep_name, self.gemm_name = "lift", "sparse_gemm"
            self.w_bytes = wbytes
            # decode shapes: the one-launch form with the lift inside the GEMM
            # (slide_gemm) is timed beside the step (nm_lift, then
            # nm_sparse_gemm; measured faster by about 2 % on B200)
            self.slide_fused = self.decode and nm.slide_gemm_workspace_size(Wc, wl.T) == 0
        elif wl.side == "mlp":
            _, g_np, d_np = inputs.make_mlp_weights(wl, seed=0)
            S = nm.spense_mlp_prepare(W, to_dev(g_np), to_dev(d_np), wl.dense_frac)   # offline
            self.g_np, self.d_np = g_np, d_np
            parts = [S.ug_vals, S.ug_meta, S.ug_dense, S.down_vals, S.down_meta, S.down_dense]
            wbytes = sum(t.numel() * t.element_size() for t in parts if t is not None)
            self.R = max(2, int(np.ceil(2 * L2_BYTES / wbytes)))
            cl = lambda t: None if t is None else t.clone()
            self.S = [S] + [nm.SpenseMlp(S.perm, *[cl(t) for t in parts], S.d, S.I, S.D) for _ in range(1, self.R)]
            self.X = [X0.roll(r, dims=0).contiguous() if r else X0 for r in range(self.R)]
            self.Y = torch.empty((wl.T, wl.K), dtype=out_dt, device=dev)
            self.ws = torch.empty(max(16, nm.spense_mlp_workspace_size(S, wl.T)), dtype=torch.uint8, device=dev)
            self.rows_a, self.rows_b = 2 * wl.O, wl.T
            self.prep_name, self.gemm_name = "none", "spense_mlp"
            self.w_bytes = wbytes
            self.launches_per_step = 3                               # up/gate GEMM, SiLU gate, down GEMM
        else:
            H = nm.hybrid_prepare(W, wl.dense_frac)                      # offline
            wbytes = H.vals_s.numel() * 2 + H.meta_s.numel() + H.W_d.numel() * 2
            self.R = max(2, int(np.ceil(2 * L2_BYTES / wbytes)))
            self.H = [H] + [nm.Hybrid(H.perm.clone(), H.vals_s.clone(), H.meta_s.clone(), H.W_d.clone(),
                                      H.O, H.K, H.K_dense) for _ in range(1, self.R)]
            self.X = [X0.roll(r, dims=0).contiguous() if r else X0 for r in range(self.R)]
            self.Y = torch.empty((wl.T, wl.O), dtype=out_dt, device=dev)
            self.ws = torch.empty(max(16, wl.T * wl.K * 2), dtype=torch.uint8, device=dev)
            self.rows_a, self.rows_b = wl.O, wl.T
            self.prep_name, self.gemm_name = "gather", "hybrid_gemm"
            self.w_bytes = wbytes
        self.launches_per_step = getattr(self, "launches_per_step", 2)
        # scratch of the split last round of SM-pair products (allocated once,
        # outside the timed steps)
        ws_bytes = 0
        if wl.side == "act" and not wl.fp8 and not wl.xf:
            ws_bytes = nm.sparse_gemm_workspace_size(self.comp[0], wl.O, nm.NM_ACT)
        elif wl.side == "weight" and not wl.fp8:
            ws_bytes = max(nm.sparse_gemm_workspace_size(self.Wc[0], wl.T, nm.NM_WEIGHT),
                           nm.slide_gemm_workspace_size(self.Wc[0], wl.T))
        self.ws_sk = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        # prefill 6:8 step: the two-call form (lift, then product), the one
        # launch with the lift inside the GEMM (slide_gemm), or the split
        # window order (the weight packed with each group's even windows
        # first; X sits in the first K columns of its [T][K'] buffer and only
        # the odd windows are lifted, in place), whichever the first timing
        # here finds fastest
        self.use_slide = False
        self.use_split = False
        if wl.side == "weight" and not wl.fp8 and not self.decode:
            Ws = nm.slide_decompose_split(W, wl.N, wl.M)                  # offline
            self.Ws = [Ws] + [nm.Compressed(Ws.vals.clone(), Ws.meta.clone(), wl.O, wl.K, wl.N, wl.M)
                              for _ in range(1, self.R)]
            self.Xw = []
            for r in range(self.R):
                xw = torch.empty((wl.T, wl.K_lift), dtype=torch.bfloat16, device=dev)
                xw[:, :wl.K] = self.X[r]
                self.Xw.append(xw)
            t_two = self._quick_time(self.two_call)
            t_one = self._quick_time(self.slide_step)
            t_split = self._quick_time(self.split_step)
            self.alt_times_us = {"two_call_step_us": t_two * 1e3, "slide_gemm_step_us": t_one * 1e3,
                                 "split_order_step_us": t_split * 1e3}
            best = min(t_two, t_one, t_split)
            self.use_split = t_split == best
            self.use_slide = not self.use_split and t_one == best
            if self.use_slide:
                self.prep_name, self.gemm_name = "none", "slide_gemm"
                self.launches_per_step = 1
            elif self.use_split:
                self.prep_name, self.gemm_name = "lift_odd", "sparse_gemm"
        del W
        torch.cuda.synchronize(dev)

    def _quick_time(self, fn, reps=20):
        torch = self.torch
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(reps):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    # one step; `mark` is called between the prep kernel and the GEMM
    def step(self, i, mark=None):
        nm, wl = self.nm, self.wl
        r = i % self.R
        if wl.side == "act" and wl.fp8:
            c = self.comp[i % 2]
            nm.prune_compress_fp8(self.X[r], wl.N, wl.M, out=c)
            if mark:
                mark()
            nm.sparse_gemm_fp8(c, self.Wq, nm.NM_ACT, self.Y.dtype, out=self.Y)
        elif wl.side == "act" and wl.xf:
            c = self.comp[i % 2]
            nm.prune_compress_xf(self.X[r], wl.N, wl.M, wl.xf, out=c)
            if mark:
                mark()
            nm.sparse_gemm_xf(c, self.Wl, self.wsum, self.Y.dtype, out=self.Y)
        elif wl.side == "act":
            c = self.comp[i % 2]
            nm.prune_compress(self.X[r], wl.N, wl.M, out=c)
            if mark:
                mark()
            nm.sparse_gemm(c, self.Wl, nm.NM_ACT, self.Y.dtype, out=self.Y, ws=self.ws_sk)
        elif wl.side == "weight" and wl.fp8:
            q = self.Q[i % 2]
            nm.quant_lift_fp8(self.X[r], wl.M, out=q)
            if mark:
                mark()
            nm.sparse_gemm_fp8(self.P[r], q, nm.NM_WEIGHT, self.Y.dtype, out=self.Y)
        elif wl.side == "weight":
            if self.use_slide:
                if mark:
                    mark()
                self.slide_step(i)
            elif self.use_split:
                self.split_step(i, mark)
            else:
                self.two_call(i, mark)
        elif wl.side == "mlp":
            if mark:
                mark()
            nm.spense_mlp(self.X[r], self.S[r], out=self.Y, ws=self.ws)
        else:
            if mark:
                mark()
            nm.hybrid_gemm(self.X[r], self.H[r], self.Y.dtype, out=self.Y, ws=self.ws)

    def two_call(self, i, mark=None):
        """The weight-sparse step as two launches: nm_lift, then nm_sparse_gemm."""
        nm, wl = self.nm, self.wl
        r = i % self.R
        xl = self.Xl[i % 2]
        nm.lift(self.X[r], wl.M, out=xl)
        if mark:
            mark()
        nm.sparse_gemm(self.Wc[r], xl, nm.NM_WEIGHT, self.Y.dtype, out=self.Y, ws=self.ws_sk)

    def slide_step(self, i):
        """The weight-sparse step as one launch: slide_gemm lifts X inside the GEMM."""
        r = i % self.R
        self.nm.slide_gemm(self.Wc[r], self.X[r], self.Y.dtype, out=self.Y, ws=self.ws_sk)

    def split_step(self, i, mark=None):
        """The weight-sparse step in the split window order: the odd windows
        lifted in place beside X, then the product."""
        nm, wl = self.nm, self.wl
        r = i % self.R
        d = nm.lift_odd(self.Xw[r], wl.K, wl.M)
        if mark:
            mark()
        nm.sparse_gemm(self.Ws[r], d, nm.NM_WEIGHT, self.Y.dtype, out=self.Y, ws=self.ws_sk)

    def gemm_only(self, i):
        nm, wl = self.nm, self.wl
        r = i % self.R
        if wl.side == "act" and wl.fp8:
            nm.sparse_gemm_fp8(self.comp[0], self.Wq, nm.NM_ACT, self.Y.dtype, out=self.Y)
        elif wl.side == "act" and wl.xf:
            nm.sparse_gemm_xf(self.comp[0], self.Wl, self.wsum, self.Y.dtype, out=self.Y)
        elif wl.side == "act":
            nm.sparse_gemm(self.comp[0], self.Wl, nm.NM_ACT, self.Y.dtype, out=self.Y, ws=self.ws_sk)
        elif wl.side == "weight" and wl.fp8:
            nm.sparse_gemm_fp8(self.P[r], self.Q[0], nm.NM_WEIGHT, self.Y.dtype, out=self.Y)
        elif wl.side == "weight":
            if self.use_slide:
                self.slide_step(i)
            elif self.use_split:
                nm.sparse_gemm(self.Ws[r], self.Xw[0], nm.NM_WEIGHT, self.Y.dtype, out=self.Y, ws=self.ws_sk)
            else:
                nm.sparse_gemm(self.Wc[r], self.Xl[0], nm.NM_WEIGHT, self.Y.dtype, out=self.Y, ws=self.ws_sk)
        elif wl.side == "mlp":
            nm.spense_mlp(self.X[r], self.S[r], out=self.Y, ws=self.ws)
        else:
            nm.hybrid_gemm(self.X[r], self.H[r], self.Y.dtype, out=self.Y, ws=self.ws)

    def algorithmic(self):
        """(dense-equiv flops, sparse-MMA flops, bytes of the GEMM) per step."""
        wl = self.wl
        dense = 2.0 * wl.T * wl.O * wl.K
        if wl.side == "mlp":
            # three projections; bytes: packed weights, x in, y out, the
            # up/gate product written and read, h written and read
            dense = 3.0 * dense
            mma = dense
            byts = (self.w_bytes + 2 * wl.T * wl.K * 2 + 2 * wl.T * 2 * wl.O * 2 + 2 * wl.T * wl.O * 2)
        elif wl.side == "hybrid":
            D = self.H[0].K_dense
            Ks = wl.K - D
            mma = 2.0 * wl.T * wl.O * (Ks + D)          # sparse part counted at its 2:4 rate
            byts = (self.w_bytes + wl.T * wl.K * 2 + wl.T * wl.O * self.Y.element_size())
        elif wl.fp8 and wl.side == "act":
            mma = 2.0 * wl.T * wl.O * wl.K_lift
            byts = (self.rows_a * (wl.K_lift // 2 + 4) + self.nm.meta_bytes(self.rows_a, wl.K, wl.M)
                    + self.rows_b * (wl.K_lift + 4) + wl.T * wl.O * self.Y.element_size())
        elif wl.fp8:
            mma = 2.0 * wl.T * wl.O * wl.K_lift
            byts = self.w_bytes + self.rows_b * (wl.K_lift + 4) + wl.T * wl.O * self.Y.element_size()
        else:
            mma = 2.0 * wl.T * wl.O * wl.K_lift
            sparse_bytes = self.rows_a * wl.K_lift + self.nm.meta_bytes(self.rows_a, wl.K, wl.M)
            byts = sparse_bytes + self.rows_b * wl.K_lift * 2 + wl.T * wl.O * self.Y.element_size()
        return dense, mma, byts


def _count_fixup(wk):
    """A GEMM whose last round was split launches the fixup kernel too."""
    if "+split" in (wk.kernel_name or "") and not getattr(wk, "fixup_counted", False):
        wk.launches_per_step += 1
        wk.fixup_counted = True


def time_workload(wk, steps, warmup, stream, clock=None):
    """Returns (ms per step, ms per prep kernel, ms per GEMM launch)."""
    import torch
    for i in range(warmup):
        wk.step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if wk.decode:
        # replay from CUDA graphs: the host cost of building tensor maps and
        # launching is not part of a device step
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):                      # captured on torch's side stream
            for i in range(steps):
                wk.step(i)
        gg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gg):
            for i in range(steps):
                wk.gemm_only(i)
        g.replay()
        gg.replay()
        torch.cuda.synchronize()
        ctx = clock if clock is not None else _Null()
        with ctx:
            t0.record(stream)
            g.replay()
            t1.record(stream)
            torch.cuda.synchronize()
        step_ms = t0.elapsed_time(t1) / steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gg.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        gemm_ms = e0.elapsed_time(e1) / steps
        prep_ms = max(step_ms - gemm_ms, 0.0)
        wk.kernel_name = wk.nm.last_gemm_kernel()
        _count_fixup(wk)
        del g, gg
        return step_ms, prep_ms, gemm_ms
    # the step as a user runs it: K steps back to back, events only around them
    # (events between the kernels would break their launch chaining)
    ctx = clock if clock is not None else _Null()
    with ctx:
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(steps):
            wk.step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    step_ms = t0.elapsed_time(t1) / steps
    wk.kernel_name = wk.nm.last_gemm_kernel()
    _count_fixup(wk)
    # the same K steps again with an event around each kernel: per-kernel times
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        evs[i][0].record(stream)
        wk.step(i, mark=lambda e=evs[i][1]: e.record(stream))
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    prep_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    gemm_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    wk.instrumented_step_ms = float(np.mean([e[0].elapsed_time(e[2]) for e in evs]))
    return step_ms, prep_ms, gemm_ms


def time_graph(wk, fn, steps=200, warmup=5):
    """ms per call of fn(i) replayed from a CUDA graph of `steps` calls."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del g
    return ms


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_dense(wk, reps=10):
    """In-run dense comparators for a prefill workload: the same unpruned
    product Y = X . W^T on this library's dense tcgen05 kernel, and on cuBLAS
    (torch.matmul) as library context.  Returns (ours_ms, cublas_ms)."""
    import torch
    wl = wk.wl
    dev = wk.dev
    X = torch.from_numpy(wk.x_np).view(torch.bfloat16).to(dev)
    W = torch.from_numpy(wk.w_np).view(torch.bfloat16).to(dev)
    Y = torch.empty((wl.T, wl.O), dtype=torch.bfloat16, device=dev)
    out = []
    for fn in (lambda: wk.nm.dense_gemm(X, W, torch.bfloat16, out=Y), lambda: torch.matmul(X, W.t(), out=Y)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) / reps)
    del X, W, Y
    return out[0], out[1]


def time_dense_fp8(wk, reps=10):
    """cuBLAS 8-bit dense GEMM on the same (unpruned) product as library
    context: X and W quantised per row to E4M3, row-wise scales, bf16 out.
    Returns ms per launch, or None where torch offers no such GEMM."""
    import torch
    wl = wk.wl
    dev = wk.dev
    try:
        X = torch.from_numpy(wk.x_np).view(torch.bfloat16).to(dev).float()
        W = torch.from_numpy(wk.w_np).view(torch.bfloat16).to(dev).float()
        sx = (X.abs().amax(dim=1, keepdim=True) / 448.0).clamp_min(1e-12)
        sw = (W.abs().amax(dim=1, keepdim=True) / 448.0).clamp_min(1e-12)
        Xq = (X / sx).to(torch.float8_e4m3fn)
        Wq = (W / sw).to(torch.float8_e4m3fn)
        del X, W

        def fn():
            return torch._scaled_mm(Xq, Wq.t(), scale_a=sx, scale_b=sw.t(), out_dtype=torch.bfloat16)

        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps
    except Exception:
        return None


def time_dense_mlp(wk, reps=20):
    """The same GLU MLP unpruned, on cuBLAS (torch.matmul) and torch's SiLU,
    replayed from a CUDA graph: library context for the decode MLP.  The
    three dense weights (3 x O x K bf16) exceed 2x L2 by themselves.  Returns
    ms per MLP."""
    import torch
    dev = wk.dev
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)
    Wu, Wg, Wd = bf(wk.w_np), bf(wk.g_np), bf(wk.d_np)
    x = wk.X[0]

    def fn():
        u = torch.matmul(x, Wu.t())
        g = torch.matmul(x, Wg.t())
        return torch.matmul(torch.nn.functional.silu(g) * u, Wd.t())

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        for _ in range(3):
            fn()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g, Wu, Wg, Wd
    return e0.elapsed_time(e1) / reps


def mma_probe():
    """The library's tensor-core rate probe (MMAs from shared memory on every
    SM pair, no loads): the rate the GEMMs' MMA instructions can reach at
    this moment's clocks, in TFLOP/s dense-equivalent, with the SM clock seen
    while it ran (a pure tensor loop can hit the power cap)."""
    import torch
    from semi_structured_sparse_nm_b200 import _lib as nm
    clk = ClockSampler(torch.cuda.current_device())
    with clk:
        out = {"bf16_dense": nm.mma_rate_probe(0), "bf16_sparse": nm.mma_rate_probe(1),
               "e4m3_sparse": nm.mma_rate_probe(2)}
    out["clocks"] = clk.summary()
    return out


def summarize(wk, step_ms, prep_ms, gemm_ms, ws, pk, probe=None):
    dense, mma, byts = wk.algorithmic()
    wl = wk.wl
    kname = getattr(wk, "kernel_name", "") or wk.gemm_name
    traffic = TRAFFIC.get((wl.name, kname))
    out = {
        "value": whole_job_rate(dense, ws, step_ms) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms,
        "tokens_per_s": whole_job_rate(wl.T, ws, step_ms),
        "config": {"T": wl.T, "K": wl.K, "O": wl.O, "N": wl.N, "M": wl.M, "side": wl.side,
                   "K_lift": wl.K_lift, "rotated_buffers": wk.R},
        "kernels": {f"{wk.prep_name}_us": prep_ms * 1e3, f"{wk.gemm_name}_us": gemm_ms * 1e3},
    }
    if wl.xf:
        out["config"]["corrections"] = {1: "shift (D-PTS)", 2: "variance (VAR)", 3: "shift (D-PTS) + variance (VAR)"}[wl.xf]
    if wl.side == "mlp":
        out["config"].update(d=wl.K, I=wl.O, dense_frac=wl.dense_frac, D=wk.S[0].D)
        out["kernels"] = {"spense_mlp_us": step_ms * 1e3,
                          "note": "one MLP = three launches (up/gate output-split GEMM, SiLU gate, "
                                  "down input-split GEMM) replayed from a CUDA graph"}
        cb = time_dense_mlp(wk)
        out["dense_comparator"] = {"cublas_mlp_us": cb * 1e3, "speedup_vs_cublas": cb / step_ms,
                                   "note": "the same MLP unpruned: three cuBLAS GEMMs and torch's SiLU and "
                                           "product, bf16, from a CUDA graph; library context only"}
    if getattr(wk, "instrumented_step_ms", None) is not None:
        out["kernels"]["note"] = ("per-kernel times from a second pass of the same steps with an event around "
                                  "each kernel; that pass's step: %.2f us" % (wk.instrumented_step_ms * 1e3))
    if not wk.decode and wl.fp8:
        c8 = time_dense_fp8(wk)
        out["dense_comparator"] = {
            "cublas_fp8_us": None if c8 is None else c8 * 1e3,
            "sparse_gemm_speedup_vs_cublas_fp8": None if c8 is None else c8 / gemm_ms,
            "note": "same unpruned product, E4M3 operands with per-row scales, bf16 out, cuBLAS "
                    "(torch._scaled_mm); library context only"}
    elif not wk.decode and wl.x_dtype == "bf16":
        ours, cublas = time_dense(wk)
        out["dense_comparator"] = {
            "ours_us": ours * 1e3, "cublas_us": cublas * 1e3,
            "sparse_gemm_speedup_vs_ours": ours / gemm_ms, "step_speedup_vs_ours": ours / step_ms,
            "sparse_gemm_speedup_vs_cublas": cublas / gemm_ms,
            "note": "same unpruned product X . W^T, bf16, fp32 accumulate; cuBLAS is context only"}
    if getattr(wk, "alt_times_us", None):
        out["kernels"]["alternatives"] = wk.alt_times_us
    if getattr(wk, "slide_fused", False):
        out["kernels"]["slide_gemm_step_us"] = time_graph(wk, wk.slide_step) * 1e3
        out["kernels"]["note"] = ("slide_gemm_step_us: the same step as one launch, the lift formed inside the "
                                  "GEMM (slide_gemm), replayed from a CUDA graph")
    if wk.decode:
        achieved = byts / (gemm_ms * 1e-3) / 1e9
        out["roofline"] = {"bound": "hbm", "kernel": kname if wl.side != "mlp" else
                           "spense_mlp (its three launches together)", "achieved": achieved, "peak": pk["hbm"],
                           "unit": "GB/s", "frac": achieved / pk["hbm"], "traffic": traffic,
                           "bytes_per_launch": byts,
                           "peak_note": f"{pk['source']} HBM copy bandwidth"}
    elif wl.fp8:
        peak = 4.0 * pk["bf16"]
        achieved = mma / (gemm_ms * 1e-3) / 1e12
        out["roofline"] = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak,
                           "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                           "flops_per_launch": mma,
                           "peak_note": f"4 x {pk['source']} bf16 burst {pk['bf16']} TFLOP/s (nominal 8-bit / "
                                        f"16-bit ratio 2 x nominal 2:4 sparse ratio 2)"}
        if probe:
            out["roofline"]["probe_tflops"] = probe["e4m3_sparse"]
            out["roofline"]["frac_of_probe"] = achieved / probe["e4m3_sparse"]
    else:
        peak = 2.0 * pk["bf16"]
        achieved = mma / (gemm_ms * 1e-3) / 1e12
        out["roofline"] = {"bound": "tensor", "kernel": kname,
                           "achieved": achieved, "peak": peak,
                           "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                           "flops_per_launch": mma,
                           "peak_note": f"2 x {pk['source']} bf16 burst {pk['bf16']} TFLOP/s "
                                        f"(nominal 2:4 sparse ratio)"}
        if probe:
            out["roofline"]["probe_tflops"] = probe["bf16_sparse"]
            out["roofline"]["frac_of_probe"] = achieved / probe["bf16_sparse"]
    # the compact row printed in the bench line (fields: ROW_FIELDS)
    extra = out["kernels"].get("slide_gemm_step_us")
    out["row"] = [sig(out["value"]), sig(step_ms * 1e3), sig(prep_ms * 1e3, 3), sig(gemm_ms * 1e3),
                  sig(out["roofline"]["frac"], 3), out["roofline"]["bound"][0],
                  None if traffic is None else sig(traffic / byts, 3)]
    if extra is not None:
        out["row"].append(sig(extra, 3))
    return out


# TFLOP/s dense-equivalent; step, prep-kernel and GEMM microseconds; the
# GEMM's roofline fraction and bound (t: tensor, h: HBM); its DRAM traffic
# over its algorithmic bytes (from an ncu capture, null if none); the 6:8
# decode step as one slide_gemm launch
ROW_FIELDS = ["TFLOP/s", "step_us", "prep_us", "gemm_us", "frac", "bound", "traffic/alg", "slide_gemm_us"]


def run_gpu(args):
    import torch
    ws, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from semi_structured_sparse_nm_b200 import _lib as nm
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    pk = _peaks()

    wk = Workload(args.workload, dev)
    if args.profile_steps:
        # plain launches of the step, no graphs and no timing: for profilers;
        # a weight-sparse decode workload also runs the step's one-launch form
        # (slide_gemm) after each step
        for i in range(args.profile_steps):
            wk.step(i)
            if getattr(wk, "slide_fused", False):
                wk.slide_step(i)
        torch.cuda.synchronize()
        status = nm.device_error()
        if rank == 0:
            print(json.dumps({"workload": args.workload, "profile_steps": args.profile_steps,
                              "device_status": status}))
        if dist is not None:
            dist.destroy_process_group()
        return 0 if status == 0 else 1
    if dist is not None:
        dist.barrier()
    clk = ClockSampler(torch.cuda.current_device())
    step_ms, prep_ms, gemm_ms = time_workload(wk, args.steps, args.warmup, stream, clock=clk)
    if dist is not None:
        step_ms = max_over_ranks(step_ms, dist, dev)
        dist.barrier()
    status = nm.device_error()
    probe = mma_probe()
    main = summarize(wk, step_ms, prep_ms, gemm_ms, ws, pk, probe=probe)
    detail = {args.workload: {k: v for k, v in main.items() if k != "row"}}

    # end to end through the public calls: pinned host X in, Y out
    wl = wk.wl
    xh = torch.from_numpy(wk.x_np).view(torch.bfloat16).pin_memory() if wl.x_dtype == "bf16" \
        else torch.from_numpy(wk.x_np).pin_memory()
    yh = torch.empty(tuple(wk.Y.shape), dtype=wk.Y.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    pipelined = wl.side == "act" and not wl.fp8 and not wl.xf and wl.x_dtype == "bf16"
    if pipelined:
        # the library's host-buffer entry point: chunked copies in and out on
        # their own streams, overlapping the prune + GEMM of neighbouring chunks
        hws = nm.act_sparse_linear_host_workspace(wl.T, wl.K, wl.N, wl.M, wl.O, dev)

        def e2e_step(i):
            nm.act_sparse_linear_host(xh, wk.Wl, wl.N, wl.M, yh, ws=hws)
    else:
        def e2e_step(i):
            wk.X[0].copy_(xh, non_blocking=True)
            wk.step(0)
            yh.copy_(wk.Y, non_blocking=True)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    # the host link's own rate for context: a plain pinned copy of the same X
    # into device memory (the end-to-end step cannot beat its copy in)
    xd_probe = torch.empty(tuple(xh.shape), dtype=xh.dtype, device=dev)
    xd_probe.copy_(xh, non_blocking=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(3):
        xd_probe.copy_(xh, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    h2d_gbs = xh.numel() * xh.element_size() * 3 / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del xd_probe
    dense, _, _ = wk.algorithmic()

    rf = main["roofline"]
    roofline = {"bound": rf["bound"], "kernel": rf["kernel"], "achieved": sig(rf["achieved"]), "peak": rf["peak"],
                "unit": rf["unit"], "frac": sig(rf["frac"], 3), "traffic": rf["traffic"],
                "peak_src": ("2x" if wl.side == "act" and not wl.fp8 else "") + f" {pk['source']} bf16 burst"}
    if "flops_per_launch" in rf:
        roofline["flops_per_launch"] = rf["flops_per_launch"]
    if "bytes_per_launch" in rf:
        roofline["bytes_per_launch"] = rf["bytes_per_launch"]
    if "probe_tflops" in rf:
        roofline["frac_of_probe"] = sig(rf["frac_of_probe"], 3)
    dc = main.get("dense_comparator") or {}
    line = {
        "metric": METRIC, "value": sig(main["value"]), "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sig(step_ms), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, ws),
        "tokens_per_s": sig(main["tokens_per_s"]),
        "kernels_us": {k[:-3]: sig(v) for k, v in main["kernels"].items() if k.endswith("_us")},
        "roofline": roofline,
        "e2e": {"value": sig(ws * dense / (e2e_ms * 1e-3) / 1e12), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
                "d2h_bytes_per_step": int(yh.numel() * yh.element_size()),
                "path": "nm_act_sparse_linear_host" if pipelined else "copy in, step, copy out",
                "h2d_copy_GBps": sig(h2d_gbs)},
        "gpu_launches": wk.launches_per_step * args.steps,
        "clocks": clk.summary(),
        "device_status": status,
    }
    if dc.get("ours_us") is not None:
        line["dense_us"] = {"ours": sig(dc["ours_us"]), "cublas": sig(dc["cublas_us"])}
    line["probe_tflops"] = {k: sig(v) for k, v in probe.items() if k != "clocks"}
    del wk
    torch.cuda.empty_cache()

    if not args.only_main:
        rows = {}
        for name in OTHERS:
            if name == args.workload:
                continue
            w2 = Workload(name, dev)
            s_, p_, g_ = time_workload(w2, args.steps, args.warmup, stream)
            full = summarize(w2, s_, p_, g_, 1, pk, probe=probe)
            rows[name] = full.pop("row")
            detail[name] = full
            del w2
            torch.cuda.empty_cache()
        line["workloads_fields"] = ROW_FIELDS
        line["workloads"] = rows
        line["device_status"] = max(status, nm.device_error())

    if rank == 0 and not args.no_cpu_baseline:
        from semi_structured_sparse_nm_b200 import inputs
        wlh, xh_np, wh_np = inputs.make_workload(args.workload)
        if wlh.side == "act":
            tf, rows_done, t, thr = cpu_oracle_sample(wlh, xh_np, wh_np, budget_s=args.cpu_budget_s)
            line["cpu_baseline"] = {"value": sig(tf), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                    "sample": f"{rows_done} of {wlh.T} token rows (prune, windows, metadata, fp64 GEMM), {t:.1f} s",
                                    "cpu": cpu_model()}
            detail["cpu_baseline_split_s"] = getattr(cpu_oracle_sample, "last_split", None)
    if rank == 0:
        if args.detail:
            with open(args.detail, "w") as f:
                json.dump(detail, f, indent=1)
        print(json.dumps(line, separators=(",", ":")), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if line["device_status"] == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--only-main", action="store_true", help="skip the other workloads")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--detail", default="", help="write every workload's full record (JSON) to this path")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="run this many plain steps of --workload and exit (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
