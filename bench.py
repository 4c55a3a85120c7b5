"""Benchmark of the detail-branch attention path (one JSON line on rank 0).

A step is one pass of the whole path over one synthetic input resident in
HBM: reorder+RoPE of detail Q and K, reorder of detail V, RoPE of global Q
and K, the asymmetric local-global attention, and the unorder of the detail
output -- seven launches of this repository's kernels through the C-ABI.

    python bench.py [--gpus N --steps K --warmup W] [--workload 720p]
    python bench.py --impl reference ...   # the fp64 CPU oracle, same metric

Metric: TFLOP/s of unmasked attention FLOPs (4*D per allowed query-key pair
per head) over the whole step; the attention kernel's own TFLOP/s and the
reorder+RoPE kernels' GB/s (one read + one write of detail Q, K, V and global
Q, K) are reported beside it with their fractions of the measured peaks.
Multi-GPU (torchrun): every rank runs its own copy of the workload (weak
scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from video_dit_windowed_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "local-global attn TFLOP/s (unmasked) & % BF16 peak; reorder+RoPE GB/s"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


def tensor_peak(pk, pk_kind, timed_s):
    """The bf16 tensor peak a kernel is held to. MEASURED_PEAKS.json has two:
    a burst figure (cuBLAS GEMMs back to back for well under a second, SM
    clock at its maximum) and a sustained one (the same GEMM looped for
    seconds, clock settled under the power cap). A timed region shorter than
    three seconds runs at the burst clock, so it is held to the burst peak;
    only a longer region is held to the sustained one."""
    if timed_s < 3.0:
        return pk["bf16_tflops"], f"{pk_kind} bf16 burst (timed region {timed_s:.2f} s < 3 s)"
    return (pk["bf16_tflops_sustained"],
            f"{pk_kind} bf16 sustained (timed region {timed_s:.1f} s >= 3 s)")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples every 100 ms from start() to stop(); only the samples
    stamped inside the timed region (window()) are summarised."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def window(self, t0: float, t1: float):
        self.t0, self.t1 = t0, t1

    def stop(self):
        import datetime
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, clk_max = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            if not (getattr(self, "t0", 0) <= ts <= getattr(self, "t1", 1e30)):
                continue
            sm.append(clk)
            mx.append(clk_max)
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the GPU path
# ---------------------------------------------------------------------------
class Path:
    """Device buffers and the C-ABI calls of one step.

    mask "all" (the headline): reorder (+RoPE) detail Q and K, reorder V; RoPE
      of global Q and K; attention (own window + every global key of the
      problem); unorder O_d.
    "aligned": the aligned-proxy-tokens variant. As "all", but global Q, K
      (+RoPE) and V are put in the aligned order (cube by cube of the detail
      grid, any grid ratios), each window sees only its aligned global keys,
      and O_g is unordered too.
    "raster": naive block attention for comparison. RoPE of detail Q and K
      in raster order, no reorder; windows of window_len consecutive raster
      rows (+ every global key); no unorder.
    "dense": full attention for comparison. RoPE of every Q and K into one
      buffer of N+G rows, one attention call in which every row sees every row.
    Windows that the cube does not divide (partial cubes) go through the
    window-offset form of the attention."""

    def __init__(self, w, device, stream, mask="all", batch=1, backward=False):
        from video_dit_windowed_b200 import atlas
        if mask == "dense" and batch != 1:
            raise ValueError("--mask dense runs one problem (batch 1)")
        if backward and mask == "dense":
            raise ValueError("--backward runs the method's masks (all, aligned, raster)")
        self.backward = backward
        if mask in ("raster", "dense") and w.partial:
            raise ValueError(f"--mask {mask} needs a cube that divides the grid")
        self.atlas, self.w, self.dev, self.stream = atlas, w, device, stream
        self.mask, self.B = mask, batch
        self.rd = atlas.make_rope(w.theta, w.split, w.detail_scales)
        self.rg = atlas.make_rope(w.theta, w.split, w.global_scales)
        e = lambda t: torch.empty_like(t)
        N, G, B = w.n_detail, w.n_global, batch
        if mask == "dense":
            # every Q, K and V in one [N+G] buffer, detail rows first
            shp = (N + G, w.heads, w.head_dim)
            self.q_all = torch.empty(shp, dtype=w.torch_dtype, device=device)
            self.k_all, self.v_all = e(self.q_all), e(self.q_all)
            self.o_all = e(self.q_all)
            x = make_inputs(w, device=device)
            self.v_all[:N].copy_(x["v_d"])
            self.v_all[N:].copy_(x["v_g"])
            x["v_d"], x["v_g"] = self.v_all[:N], self.v_all[N:]
            self.x = x
            self.o_raster, self.o_g = self.o_all[:N], self.o_all[N:]
            return
        x = make_inputs(w, device=device, batch=B)
        self.x = x
        self.q_d, self.k_d, self.v_d = e(x["q_d"]), e(x["k_d"]), e(x["v_d"])
        self.q_g, self.k_g = e(x["q_g"]), e(x["k_g"])
        self.o_d, self.o_g = e(x["q_d"]), e(x["q_g"])
        self.o_raster = e(x["q_d"])
        self.win = (atlas.cube_window_offsets(w.grid, w.cube).to(device)
                    if w.partial or mask == "aligned" else None)
        self.gwin = None
        if mask == "aligned":
            self.gwin = atlas.aligned_global_offsets(w.grid, w.cube, w.global_grid).to(device)
            self.v_g = e(x["v_g"])
            self.o_graster = e(x["q_g"])
        self.lse = None
        if backward:
            # output gradients (raster order, as a user hands them in), the
            # forward's LSE, the delta workspace, gradients in the
            # attention's order and in raster order
            from video_dit_windowed_b200.workloads import normal
            self.do = {"d": normal(x["q_d"].shape, 0, w.torch_dtype, 1, device),
                       "g": normal(x["q_g"].shape, 3, w.torch_dtype, 1, device)}
            self.do_att = {"d": e(x["q_d"]), "g": e(x["q_g"])}
            self.lse = torch.empty(B, w.heads, N + G, dtype=torch.float32, device=device)
            self.delta = torch.empty_like(self.lse)
            names = ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")
            self.grad = [e(x[n]) for n in names]
            self.grad_raster = [e(x[n]) for n in names]
            self.rd_t = atlas.transpose_rope(self.rd)
            self.rg_t = atlas.transpose_rope(self.rg)

    def step(self, ev=None):
        """One pass; ``ev`` (5 CUDA events) brackets the phases if given."""
        a, w, s, x, B = self.atlas, self.w, self.stream, self.x, self.B
        rec = (lambda i: ev[i].record(s)) if ev is not None else (lambda i: None)
        N, G = w.n_detail, w.n_global
        if self.mask == "dense":
            rec(0)
            if N:
                a.rope3d(x["q_d"], self.q_all[:N], w.grid, self.rd, stream=s)
                a.rope3d(x["k_d"], self.k_all[:N], w.grid, self.rd, stream=s)
            rec(1)
            a.rope3d(x["q_g"], self.q_all[N:], w.global_grid, self.rg, stream=s)
            a.rope3d(x["k_g"], self.k_all[N:], w.global_grid, self.rg, stream=s)
            rec(2)
            a.local_global_attn(None, None, None, 1, self.q_all, self.k_all, self.v_all, None,
                                self.o_all, None, stream=s)
            rec(3)
            rec(4)
            return
        rec(0)
        if N:
            if self.mask == "raster":
                a.rope3d_batched(x["q_d"], self.q_d, B, w.grid, self.rd, stream=s)
                a.rope3d_batched(x["k_d"], self.k_d, B, w.grid, self.rd, stream=s)
            else:
                a.cube_reorder_batched(x["q_d"], self.q_d, B, w.grid, w.cube, self.rd, stream=s)
                a.cube_reorder_batched(x["k_d"], self.k_d, B, w.grid, w.cube, self.rd, stream=s)
                a.cube_reorder_batched(x["v_d"], self.v_d, B, w.grid, w.cube, None, stream=s)
        rec(1)
        v_g = x["v_g"]
        if G:
            if self.mask == "aligned":
                args = (w.grid, w.cube, w.global_grid)
                a.aligned_global_reorder(x["q_g"], self.q_g, *args, self.rg, B, stream=s)
                a.aligned_global_reorder(x["k_g"], self.k_g, *args, self.rg, B, stream=s)
                a.aligned_global_reorder(x["v_g"], self.v_g, *args, None, B, stream=s)
                v_g = self.v_g
            else:
                a.rope3d_batched(x["q_g"], self.q_g, B, w.global_grid, self.rg, stream=s)
                a.rope3d_batched(x["k_g"], self.k_g, B, w.global_grid, self.rg, stream=s)
        rec(2)
        v_d = x["v_d"] if self.mask == "raster" else self.v_d
        if B == 1 and self.win is None:
            a.local_global_attn(self.q_d, self.k_d, v_d, w.window_len, self.q_g, self.k_g, v_g,
                                self.o_d, self.o_g, self.lse, stream=s)
        else:
            a.local_global_attn_ex(self.q_d, self.k_d, v_d, self.q_g, self.k_g, v_g, self.o_d,
                                   self.o_g, self.lse, batch=B, window_len=w.window_len,
                                   window_offsets=self.win, global_window_offsets=self.gwin,
                                   stream=s)
        rec(3)
        if N and self.mask != "raster":
            a.cube_unorder_batched(self.o_d, self.o_raster, B, w.grid, w.cube, stream=s)
        if self.mask == "aligned" and G:
            a.aligned_global_unorder(self.o_g, self.o_graster, w.grid, w.cube, w.global_grid,
                                     batch=B, stream=s)
        rec(4)
        if self.backward:
            self.step_backward(v_d, v_g, ev)

    def step_backward(self, v_d, v_g, ev=None):
        """Gradients of the step's outputs w.r.t. its raster inputs: dO to the
        attention's order, the attention backward, then the gradients back
        to raster order (the transposed RoPE for dQ and dK)."""
        a, w, s, B = self.atlas, self.w, self.stream, self.B
        rec = (lambda i: ev[i].record(s)) if ev is not None else (lambda i: None)
        N, G, m = w.n_detail, w.n_global, self.mask
        gg, args = w.global_grid, (w.grid, w.cube, w.global_grid)
        do_d, do_g = self.do["d"], self.do["g"]
        if N and m != "raster":
            a.cube_reorder_batched(do_d, self.do_att["d"], B, w.grid, w.cube, stream=s)
            do_d = self.do_att["d"]
        if G and m == "aligned":
            a.aligned_global_reorder(do_g, self.do_att["g"], *args, batch=B, stream=s)
            do_g = self.do_att["g"]
        rec(5)
        g = self.grad
        a.local_global_attn_bwd(self.q_d, self.k_d, v_d, self.o_d, do_d, self.q_g, self.k_g,
                                v_g, self.o_g, do_g, self.lse, *g, self.delta, batch=B,
                                window_len=w.window_len, window_offsets=self.win,
                                global_window_offsets=self.gwin, stream=s)
        rec(6)
        r = self.grad_raster
        if N:
            if m == "raster":
                a.rope3d_batched(g[0], r[0], B, w.grid, self.rd_t, stream=s)
                a.rope3d_batched(g[1], r[1], B, w.grid, self.rd_t, stream=s)
            else:
                a.cube_unorder_rope(g[0], r[0], w.grid, w.cube, self.rd_t, B, stream=s)
                a.cube_unorder_rope(g[1], r[1], w.grid, w.cube, self.rd_t, B, stream=s)
                a.cube_unorder_batched(g[2], r[2], B, w.grid, w.cube, stream=s)
        if G:
            if m == "aligned":
                a.aligned_global_unorder(g[3], r[3], *args, self.rg_t, B, stream=s)
                a.aligned_global_unorder(g[4], r[4], *args, self.rg_t, B, stream=s)
                a.aligned_global_unorder(g[5], r[5], *args, batch=B, stream=s)
            else:
                a.rope3d_batched(g[3], r[3], B, gg, self.rg_t, stream=s)
                a.rope3d_batched(g[4], r[4], B, gg, self.rg_t, stream=s)
        rec(7)

    def outputs(self):
        """Step results in raster order (the tensors a user reads back)."""
        if self.mask == "raster":
            return self.o_d, self.o_g
        if self.mask == "aligned":
            return self.o_raster, self.o_graster
        return self.o_raster, self.o_g

    def gradients(self):
        """Backward results in raster order (dq_d, dk_d, dv_d, dq_g, dk_g, dv_g)."""
        g, r, m = self.grad, self.grad_raster, self.mask
        return [r[0], r[1], g[2] if m == "raster" else r[2], r[3], r[4],
                r[5] if m == "aligned" else g[5]]

    def launches_per_step(self):
        w, m = self.w, self.mask
        nd, ng = bool(w.n_detail), bool(w.n_global)
        if m == "dense":
            return 2 * nd + 2 + 1
        if m == "raster":
            fwd = 2 * nd + 2 * ng + 1
        elif m == "aligned":
            fwd = 3 * nd + 3 * ng + 1 + nd + ng
        else:
            fwd = 3 * nd + 2 * ng + 1 + nd
        if not self.backward:
            return fwd
        # dO reorder(s); delta + dQ + dK/dV kernels; gradients to raster order
        pre = (nd if m != "raster" else 0) + (ng if m == "aligned" else 0)
        post = (2 * nd + (nd if m != "raster" else 0)) + (2 * ng + (ng if m == "aligned" else 0))
        return fwd + pre + 3 + post

    def bwd_flops(self):
        """Tensor-core FLOPs the backward kernels execute: per allowed pair
        6*D in the dQ pass (S, dP, dQ) and 8*D in the dK/dV pass (S, dP, dV,
        dK), i.e. 3.5 times the forward's 4*D."""
        return self.flops() * 14 // 4

    def flops(self):
        return self.B * self.w.unmasked_flops(self.mask)

    def prep_bytes(self):
        """Algorithmic bytes of the reorder/RoPE phase: one read and one
        write of every tensor it touches."""
        w, m = self.w, self.mask
        row = w.heads * w.head_dim * w.elem_bytes
        det = (2 if m in ("raster", "dense") else 3) * w.n_detail
        glob = (3 if m == "aligned" else 2) * w.n_global
        return self.B * 2 * (det + glob) * row

    def unorder_bytes(self):
        w, m = self.w, self.mask
        row = w.heads * w.head_dim * w.elem_bytes
        rows = {"all": w.n_detail, "aligned": w.n_detail + w.n_global}.get(m, 0)
        return self.B * 2 * rows * row

    def attn_bytes(self):
        """Minimum DRAM bytes of one attention launch: Q, K, V read once, O
        written once."""
        w = self.w
        return self.B * 4 * (w.n_detail + w.n_global) * w.heads * w.head_dim * w.elem_bytes

    @staticmethod
    def phase_ms(ev):
        d = {"reorder": ev[0].elapsed_time(ev[1]), "rope_g": ev[1].elapsed_time(ev[2]),
             "attn": ev[2].elapsed_time(ev[3]), "unorder": ev[3].elapsed_time(ev[4])}
        if len(ev) > 5:
            d.update({"bwd_pre": ev[4].elapsed_time(ev[5]), "bwd_attn": ev[5].elapsed_time(ev[6]),
                      "bwd_post": ev[6].elapsed_time(ev[7])})
        return d


class ProjPath:
    """The path with the projections on either side, fused (--proj): QKV
    projection with RoPE and reorder in the GEMM epilogue (detail tokens, and
    the global proxy with a 1x1x1 cube), the attention, and the output
    projection writing rows back to raster order. Model width C =
    heads*head_dim; weights are seeded, random (N(0,1)/sqrt(C)), bf16.
    Also times, for comparison only, the same projections unfused: torch's
    matmul (cuBLAS) then the separate reorder / RoPE / unorder kernels."""

    def __init__(self, w, device, stream):
        from video_dit_windowed_b200 import atlas
        from video_dit_windowed_b200.workloads import normal
        self.atlas, self.w, self.stream = atlas, w, stream
        C = w.heads * w.head_dim
        self.C = C
        N, G = w.n_detail, w.n_global
        bf = torch.bfloat16
        self.x_d = normal((N, C), "q_d", bf, 0, device)
        self.x_g = normal((G, C), "q_g", bf, 0, device)
        self.w_qkv = (normal((3 * C, C), "k_d", torch.float32, 0, device) / C ** 0.5).to(bf)
        self.w_o = (normal((C, C), "v_d", torch.float32, 0, device) / C ** 0.5).to(bf)
        e = lambda rows: torch.empty(rows, w.heads, w.head_dim, dtype=bf, device=device)
        self.q_d, self.k_d, self.v_d = e(N), e(N), e(N)
        self.q_g, self.k_g, self.v_g = e(G), e(G), e(G)
        self.o_d, self.o_g = e(N), e(G)
        self.y_d = torch.empty(N, C, dtype=bf, device=device)
        self.y_g = torch.empty(G, C, dtype=bf, device=device)
        self.rd = atlas.make_rope(w.theta, w.split, w.detail_scales)
        self.rg = atlas.make_rope(w.theta, w.split, w.global_scales)
        self.one = (1, 1, 1)
        self.mask = "all"
        self.backward = False

    def step(self, ev=None):
        a, w, s = self.atlas, self.w, self.stream
        rec = (lambda i: ev[i].record(s)) if ev is not None else (lambda i: None)
        rec(0)
        a.qkv_proj_reorder(self.x_d, self.w_qkv, w.grid, w.cube, self.q_d, self.k_d, self.v_d,
                           self.rd, stream=s)
        rec(1)
        a.qkv_proj_reorder(self.x_g, self.w_qkv, w.global_grid, self.one, self.q_g, self.k_g,
                           self.v_g, self.rg, stream=s)
        rec(2)
        a.local_global_attn(self.q_d, self.k_d, self.v_d, w.window_len, self.q_g, self.k_g,
                            self.v_g, self.o_d, self.o_g, None, stream=s)
        rec(3)
        a.out_proj_unorder(self.o_d, self.w_o, w.grid, w.cube, self.y_d, stream=s)
        a.out_proj_unorder(self.o_g, self.w_o, w.global_grid, self.one, self.y_g, stream=s)
        rec(4)

    def unfused_ms(self, steps):
        """Median time of the same projections unfused (cuBLAS matmul, then
        the separate permutation kernels), QKV and output parts."""
        a, w, s = self.atlas, self.w, self.stream
        C, N = self.C, w.n_detail
        tmp = torch.empty(N, C, dtype=torch.bfloat16, device=self.x_d.device)
        tmp_o = torch.empty(N, w.heads, w.head_dim, dtype=torch.bfloat16, device=tmp.device)
        t_qkv, t_out = [], []
        for i in range(steps + 2):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            with torch.cuda.stream(s):
                ev[0].record(s)
                for j, (dst, rope) in enumerate(((self.q_d, self.rd), (self.k_d, self.rd),
                                                 (self.v_d, None))):
                    torch.matmul(self.x_d, self.w_qkv[j * C:(j + 1) * C].t(), out=tmp)
                    a.cube_reorder(tmp.view(N, w.heads, w.head_dim), dst, w.grid, w.cube, rope,
                                   stream=s)
                ev[1].record(s)
                a.cube_unorder(self.o_d, tmp_o, w.grid, w.cube, stream=s)
                torch.matmul(tmp_o.view(N, C), self.w_o.t(), out=self.y_d)
                ev[2].record(s)
            torch.cuda.synchronize()
            if i >= 2:
                t_qkv.append(ev[0].elapsed_time(ev[1]))
                t_out.append(ev[1].elapsed_time(ev[2]))
        return statistics.median(t_qkv), statistics.median(t_out)

    def flops(self):
        return self.w.unmasked_flops()

    def proj_flops(self):
        """(QKV, output) projection FLOPs: 2*rows*C*3C and 2*rows*C*C."""
        rows = self.w.n_detail + self.w.n_global
        return 2 * rows * self.C * 3 * self.C, 2 * rows * self.C * self.C

    def launches_per_step(self):
        return 5

    phase_ms = staticmethod(lambda ev: {"qkv_d": ev[0].elapsed_time(ev[1]),
                                        "qkv_g": ev[1].elapsed_time(ev[2]),
                                        "attn": ev[2].elapsed_time(ev[3]),
                                        "out": ev[3].elapsed_time(ev[4])})


def attn_kernel_name(w, mask="all"):
    """The attention kernel instance a workload's step launches."""
    if w.dtype != "bf16":
        return f"attn_simt_kernel<{w.head_dim}>"
    narrow = w.partial or mask == "aligned"
    return f"attn_tc_kernel<{w.head_dim}, {'true' if narrow else 'false'}>"


def kernel_source_hash():
    """Hash of the attention kernel's source with comments and whitespace
    removed: a comment edit keeps the stored traffic valid, a code edit does
    not."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "video_dit_windowed_b200", "csrc")
    for name in ("attn_tc.cu", "sm100_ptx.cuh"):
        with open(os.path.join(csrc, name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_traffic(w):
    """Per-launch DRAM bytes of the attention kernel for workload ``w``, from
    the committed ncu summary if it was taken on the current kernel source and
    the same workload geometry (scaled by the head count); else None."""
    path = os.path.join(ROOT, "profiles", "attn_tc_traffic.txt")
    if not os.path.exists(path):
        return None
    d = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#") and "=" in line:
                k, v = line.split("=", 1)
                d[k.strip()] = v.strip()
    if d.get("source_hash") != kernel_source_hash() or d.get("workload") != w.name:
        return None
    per_head = (int(d["dram_read_bytes"]) + int(d["dram_write_bytes"])) / int(d["heads"])
    return per_head * w.heads


# ---------------------------------------------------------------------------
# oracle timing (CPU)
# ---------------------------------------------------------------------------
def oracle_sample_flops(w, n_det_rows, n_glob_rows):
    D = w.head_dim
    return 4 * D * (n_det_rows * (w.window_len + w.n_global) + n_glob_rows * w.n_global)


def time_oracle(w, budget_s=15.0, seed=0):
    """Time the fp64 oracle on a bounded sample of the workload (one head):
    whole windows of detail rows plus 128-row blocks of global rows, added
    until about ``budget_s`` of CPU work. Returns (TFLOP/s, cores, sample)."""
    sys.path.insert(0, ROOT)
    import oracle
    orc = oracle.Oracle()
    cores = orc.max_threads()
    rng = np.random.default_rng(seed)
    D, L, G, N = w.head_dim, w.window_len, w.n_global, w.n_detail
    kg = rng.standard_normal((G, D))
    vg = rng.standard_normal((G, D))
    flops = 0
    t_total = 0.0
    det_rows = glob_rows = 0
    while t_total < budget_s:
        if N:
            k = rng.standard_normal((L, D))
            v = rng.standard_normal((L, D))
            q = rng.standard_normal((L, D))
            ids = np.arange(L, dtype=np.int64)
            t0 = time.perf_counter()
            orc.attention_head(N, L, G, w.softmax_scale, k, v, 0, kg, vg, ids, q, cores)
            t_total += time.perf_counter() - t0
            det_rows += L
        if G:
            q = rng.standard_normal((128, D))
            ids = N + np.arange(128, dtype=np.int64)
            t0 = time.perf_counter()
            orc.attention_head(N, max(L, 1), G, w.softmax_scale, None, None, 0, kg, vg, ids,
                               q, cores)
            t_total += time.perf_counter() - t0
            glob_rows += 128
        if t_total > 2 * budget_s:
            break
    flops = oracle_sample_flops(w, det_rows, glob_rows)
    sample = (f"{det_rows} detail rows (whole windows) + {glob_rows} global rows of one head, "
              f"{t_total:.1f} s of fp64 oracle work")
    return flops / t_total / 1e12, cores, sample, t_total


def time_oracle_aligned(w, budget_s=10.0, seed=0):
    """Time the fp64 oracle of the "aligned proxy tokens only" variant on a
    bounded sample of one head: whole windows of detail rows, picked at
    random, each against its own window and its aligned global keys, then a
    128-row block of global rows, until about ``budget_s`` of work. FLOPs
    count the pairs the mask allows (4*D per pair). Returns (TFLOP/s, cores,
    sample, seconds)."""
    sys.path.insert(0, ROOT)
    import oracle
    orc = oracle.Oracle()
    cores = orc.max_threads()
    rng = np.random.default_rng(seed)
    D, G, N = w.head_dim, w.n_global, w.n_detail
    off = orc.cube_windows(w.grid, w.cube)
    n_win = off.size - 1
    boxes = [w.aligned_boxes(a) for a in range(3)]
    nb = [-(-E // c) for E, c in zip(w.grid, w.cube)]
    kg, vg = rng.standard_normal((G, D)), rng.standard_normal((G, D))
    flops, t, det, glob = 0, 0.0, 0, 0
    for wi in rng.permutation(n_win):
        if t >= budget_s:
            break
        lo, hi = int(off[wi]), int(off[wi + 1])
        n = hi - lo
        k, v, q = (rng.standard_normal((n, D)) for _ in range(3))
        t0 = time.perf_counter()
        orc.attention_head_aligned(w.grid, w.cube, w.global_grid, w.softmax_scale, k, v, lo, kg,
                                   vg, np.arange(lo, hi, dtype=np.int64), q, cores)
        t += time.perf_counter() - t0
        bt, rest = divmod(int(wi), nb[1] * nb[2])
        bh, bw = divmod(rest, nb[2])
        flops += 4 * D * n * (n + boxes[0][bt] * boxes[1][bh] * boxes[2][bw])
        det += n
    if G:
        rows = min(128, G)
        q = rng.standard_normal((rows, D))
        t0 = time.perf_counter()
        orc.attention_head_aligned(w.grid, w.cube, w.global_grid, w.softmax_scale, None, None, 0,
                                   kg, vg, N + np.arange(rows, dtype=np.int64), q, cores)
        t += time.perf_counter() - t0
        flops += 4 * D * rows * G
        glob = rows
    sample = (f"{det} detail rows (whole windows, random) + {glob} global rows of one head, "
              f"aligned mask, {t:.1f} s of fp64 oracle work")
    return flops / t / 1e12, cores, sample, t


def slab_workload(w, mask):
    """One head of the workload cut to its first slab of cubes along time
    (the first ct frames of the detail grid); the global grid stays whole for
    the method's mask and is cut to the frames aligned with the slab for the
    aligned mask."""
    import dataclasses
    grid = (min(w.grid[0], w.cube[0]), w.grid[1], w.grid[2])
    gg = w.global_grid
    if mask == "aligned" and w.n_global:
        gg = (max(1, -(-grid[0] * gg[0] // w.grid[0])), gg[1], gg[2])
    return dataclasses.replace(w, grid=grid, global_grid=gg, heads=1)


def time_oracle_bwd(w, mask="all", seed=0):
    """Time the fp64 oracle's backward (softmax-Jacobian definition: every
    row's statistics, then dQ over query rows and dK, dV over key rows), in
    full, on one head of the workload's first slab of cubes along time
    (slab_workload). FLOPs: 2.5x the forward's allowed-pair FLOPs, the count
    the GPU's training-step line uses. Returns (TFLOP/s, cores, sample, s)."""
    sys.path.insert(0, ROOT)
    import oracle
    orc = oracle.Oracle()
    cores = orc.max_threads()
    rng = np.random.default_rng(seed)
    s = slab_workload(w, mask)
    N, G, D = s.n_detail, s.n_global, s.head_dim
    q_d, k_d, v_d, do_d = (rng.standard_normal((N, 1, D)) for _ in range(4))
    q_g, k_g, v_g, do_g = (rng.standard_normal((G, 1, D)) for _ in range(4))
    t0 = time.perf_counter()
    if mask == "aligned":
        orc.attention_bwd_full_aligned(q_d, k_d, v_d, s.grid, s.cube, q_g, k_g, v_g,
                                       s.global_grid, do_d, do_g, s.softmax_scale, cores)
    else:
        off = orc.cube_windows(s.grid, s.cube) if s.partial else None
        orc.attention_bwd_full(q_d, k_d, v_d, s.window_len, q_g, k_g, v_g, do_d, do_g,
                               s.softmax_scale, cores, win_off=off)
    t = time.perf_counter() - t0
    flops = s.unmasked_flops(mask) * 5 // 2
    sample = (f"one head, detail {s.grid[0]}x{s.grid[1]}x{s.grid[2]} (first slab of cubes), "
              f"global {s.global_grid[0]}x{s.global_grid[1]}x{s.global_grid[2]}, {mask} mask, "
              f"full backward, {t:.1f} s of fp64 oracle work")
    return flops / t / 1e12, cores, sample, t


def time_oracle_proj(w, seed=0):
    """Time the oracle's projections (fp64 matmul composed with its RoPE and
    cube reorder for Q, K, V; its unorder composed with the output matmul)
    on a corner of the workload's grid two cubes wide (ct x ch x 2cw tokens),
    model width heads*head_dim, random weights. FLOPs 2*rows*C*3C + 2*rows*C*C. Returns
    (TFLOP/s, cores, sample, seconds)."""
    sys.path.insert(0, ROOT)
    import oracle
    orc = oracle.Oracle()
    rng = np.random.default_rng(seed)
    grid = (min(w.grid[0], w.cube[0]), min(w.grid[1], w.cube[1]),
            min(w.grid[2], 2 * w.cube[2]))
    rows = grid[0] * grid[1] * grid[2]
    C = w.heads * w.head_dim
    x = rng.standard_normal((rows, C))
    w_qkv = rng.standard_normal((3 * C, C)) / C ** 0.5
    w_o = rng.standard_normal((C, C)) / C ** 0.5
    t0 = time.perf_counter()
    q, _, _ = orc.qkv_proj_reorder(x, w_qkv, grid, w.cube, w.heads, w.head_dim, w.theta,
                                   w.split, w.detail_scales)
    orc.out_proj_unorder(q.reshape(rows, C), w_o, grid, w.cube)
    t = time.perf_counter() - t0
    flops = 2 * rows * C * 3 * C + 2 * rows * C * C
    cores = os.cpu_count() or 1
    sample = (f"detail {grid[0]}x{grid[1]}x{grid[2]} ({rows} rows, two cubes), width "
              f"{C}: QKV projection + RoPE + reorder and unorder + output projection, "
              f"{t:.1f} s (numpy fp64 matmul on up to {cores} threads)")
    return flops / t / 1e12, cores, sample, t


def prep_phase_bytes(w):
    """Algorithmic bytes of one problem's reorder+RoPE phase (bf16 I/O, every
    head), the figure the GPU phase's GB/s counts; used to extrapolate the
    oracle's sampled rate to the whole configuration."""
    row = w.heads * w.head_dim * w.elem_bytes
    return 2 * (3 * w.n_detail + 2 * w.n_global) * row


def time_oracle_prep(w, heads=4):
    """Time the fp64 oracle's reorder + RoPE phase: RoPE then cube reorder of
    detail Q and K, byte reorder of detail V (bf16 rows), RoPE of global Q
    and K, for the first ``heads`` heads. The 720p grid is taken whole; for
    the 4K grids the sample is the first slab of cubes along time (the first
    ct frames: every window of that slab, the same rows, positions and cube
    order as in the full grid), with the whole global grid. Bytes are the
    phase's algorithmic bf16 bytes for the sample (one read and one write of
    each tensor), as the GPU figure counts them. The oracle's RoPE and reorder
    are single-threaded. Returns (GB/s, cores, sample, seconds)."""
    sys.path.insert(0, ROOT)
    import oracle
    orc = oracle.Oracle()
    rng = np.random.default_rng(0)
    D, G = w.head_dim, w.n_global
    grid = w.grid
    if w.n_detail > 200_000:
        grid = (w.cube[0], w.grid[1], w.grid[2])
    N = grid[0] * grid[1] * grid[2] if w.n_detail else 0
    t = 0.0
    for _ in range(2 if N else 0):                  # detail Q, K
        x = rng.standard_normal((N, heads, D))
        t0 = time.perf_counter()
        y = orc.rope3d_grid(x, grid, w.theta, w.split, w.detail_scales)
        orc.cube_reorder(y, grid, w.cube)
        t += time.perf_counter() - t0
    if N:                                           # detail V: a byte permutation
        xb = rng.integers(0, 1 << 16, (N, heads, D), dtype=np.uint16)
        t0 = time.perf_counter()
        orc.cube_reorder(xb, grid, w.cube)
        t += time.perf_counter() - t0
    for _ in range(2 if G else 0):                  # global Q, K
        x = rng.standard_normal((G, heads, D))
        t0 = time.perf_counter()
        orc.rope3d_grid(x, w.global_grid, w.theta, w.split, w.global_scales)
        t += time.perf_counter() - t0
    nbytes = 2 * (3 * N + 2 * G) * heads * D * 2
    where = "whole detail grid" if grid == w.grid else \
        f"detail sub-grid {grid[0]}x{grid[1]}x{grid[2]} (first slab of cubes)"
    sample = (f"{where} + whole global grid, {heads} head(s): {nbytes / 1e6:.0f} MB of bf16 "
              f"I/O, {t:.1f} s of fp64 oracle work")
    return nbytes / t / 1e9, 1, sample, t


# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def config_of(w, world, mask="all", batch=1, backward=False, graph=False, shard="replicas"):
    """The line's config. ``w`` is one rank's workload; with head sharding
    its heads are the rank's share of the problem's."""
    c = {"workload": w.name, "mask": mask, "pass": "forward+backward" if backward else "forward",
         "launch": "cuda graph" if graph else "stream", "detail_grid": list(w.grid), "cube": list(w.cube),
         "global_grid": list(w.global_grid), "n_detail": w.n_detail, "window_len": w.window_len,
         "n_global": w.n_global, "heads": w.heads, "head_dim": w.head_dim,
         "rope_split": list(w.split), "detail_scales": list(w.detail_scales),
         "global_scales": list(w.global_scales), "batch_per_gpu": batch,
         "parallelism": f"{world} independent replicas" if world > 1 else "single GPU"}
    if shard == "heads" and world > 1:
        c["heads"] = w.heads * world
        c["heads_per_gpu"] = w.heads
        c["parallelism"] = f"head-parallel over {world} GPUs (no collective)"
    per_tensor = max(w.n_detail, w.n_global) * w.heads * w.head_dim * w.elem_bytes
    c["l2"] = (f"inputs larger than L2 ({per_tensor / 1e6:.0f} MB per tensor)"
               if per_tensor > 126e6 else "inputs smaller than L2; no flush")
    return c


def run_reference(args, world, rank):
    if rank != 0:
        return
    if args.mask != "all" or args.batch != 1 or args.backward:
        raise SystemExit("the oracle arm times the method's own mask, one problem per step "
                         "(--mask all --batch 1)")
    w = workload(args, world)
    times = []
    # each step a bounded sample: the whole --steps/--warmup run stays near a minute
    budget = max(0.5, min(args.cpu_budget, 60.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        tf, cores, sample, t = time_oracle(w, budget_s=budget, seed=i)
        if i >= args.warmup:
            times.append(tf)
    value = statistics.mean(times)
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
           "scaling": scaling_of(args), "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "impl": "reference",
           "config": config_of(w, world, shard=args.shard),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                            "sample": sample + " per step"},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


def workload(args, world=1):
    """One rank's workload: the named one (with --heads, that many heads);
    with --shard heads, this rank's share of the heads of one problem (heads
    are independent end to end, so the shards need no collective)."""
    import dataclasses
    w = WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    if getattr(args, "shard", "replicas") == "heads" and world > 1:
        if w.heads % world:
            raise SystemExit(f"--shard heads: {w.heads} heads do not split over {world} GPUs")
        w = dataclasses.replace(w, heads=w.heads // world)
    return w


def scaling_of(args):
    """Weak: every rank adds a problem. Strong: the ranks share one problem."""
    return "strong" if getattr(args, "shard", "replicas") == "heads" else "weak"


def run_atlas(args, world, rank, local):
    from video_dit_windowed_b200 import atlas, build
    if not os.path.exists(atlas.LIB_PATH):
        build.build()
    w = workload(args, world)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        mem0 = torch.cuda.memory_allocated(dev)
        path = (ProjPath(w, dev, stream) if args.proj
                else Path(w, dev, stream, args.mask, args.batch, args.backward))
        path_bytes = torch.cuda.memory_allocated(dev) - mem0
    torch.cuda.synchronize(dev)
    for _ in range(args.warmup):
        path.step()
    torch.cuda.synchronize(dev)
    code = atlas.last_device_error(stream)
    if code:
        raise RuntimeError(f"device error word 0x{code:x} after warm-up")

    graph = None
    n_ev = 8 if args.backward else 5
    if args.graph:
        # the whole step as one CUDA graph (the first calls above have cached
        # every table and attribute), replayed once per timed step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            path.step()
        with torch.cuda.stream(stream):
            graph.replay()
        torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)            # let nvidia-smi start sampling before the timed region
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    start.record(stream)
    for i in range(args.steps):
        if graph is not None:
            with torch.cuda.stream(stream):       # replay() launches on the current stream
                graph.replay()
        else:
            path.step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clocks.window(t_wall0, time.time())
    barrier(world)
    clk = clocks.stop()
    elapsed = start.elapsed_time(stop)
    phases = {}
    if graph is not None:
        # phase times from eager steps after the timed region (events inside
        # a graph cannot be timed)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
               for _ in range(min(args.steps, 10))]
        for ev in evs:
            path.step(ev)
        torch.cuda.synchronize(dev)
    for ev in evs:
        for k, v in type(path).phase_ms(ev).items():
            phases.setdefault(k, []).append(v)
    elapsed = max_over_ranks(elapsed, world)
    code = atlas.last_device_error(stream)
    if code:
        raise RuntimeError(f"device error word 0x{code:x} in the timed region")

    if args.proj:
        return report_proj(args, world, rank, path, elapsed, phases, clk)

    # end to end through the C-ABI with host buffers
    e2e = None
    if not args.no_e2e:
        # a second buffer set for the pipelined run, if the device holds two
        twin = None
        free, total = torch.cuda.mem_get_info(dev)
        if path_bytes < 0.8 * free:
            with torch.cuda.stream(stream):
                twin = Path(w, dev, stream, args.mask, args.batch, args.backward)
            torch.cuda.synchronize(dev)
        e2e = run_e2e(path, w, dev, stream, args, world, twin)
        del twin

    if rank != 0:
        return
    pk, pk_kind = peaks()
    ms = elapsed / args.steps
    flops = path.flops()
    # a training step counts the backward at the usual 2.5x the forward
    step_flops = flops * 7 // 2 if args.backward else flops
    value = world * step_flops / (ms * 1e-3) / 1e12
    attn_ms = statistics.median(phases["attn"])
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    rr_ms = statistics.median(phases["reorder"]) + statistics.median(phases["rope_g"])
    rr_gbs = path.prep_bytes() / (rr_ms * 1e-3) / 1e9 if rr_ms > 0 else None
    un_ms = statistics.median(phases["unorder"])
    un_bytes = path.unorder_bytes()
    traffic = measured_traffic(w) if (args.mask, args.batch) == ("all", 1) else None
    peak_tf, peak_kind = tensor_peak(pk, pk_kind, elapsed * 1e-3)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": scaling_of(args), "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, world, args.mask, args.batch, args.backward, args.graph,
                            args.shard),
        "attn_tflops": attn_tf, "attn_ms": attn_ms,
        "attn_frac_of_bf16_peak": {"sustained": attn_tf / pk["bf16_tflops_sustained"],
                                   "burst": attn_tf / pk["bf16_tflops"], "peaks": pk_kind},
        "reorder_rope_gbs": rr_gbs, "reorder_rope_ms": rr_ms,
        "reorder_rope_frac_of_hbm": (rr_gbs / pk["hbm_gbs"]) if rr_gbs else None,
        "unorder_gbs": un_bytes / (un_ms * 1e-3) / 1e9 if un_ms > 0 and un_bytes else None,
        "roofline": {"bound": "tensor", "kernel": attn_kernel_name(w, args.mask),
                     "achieved": attn_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": attn_tf / peak_tf, "peak_kind": peak_kind,
                     "frac_of_sustained": attn_tf / pk["bf16_tflops_sustained"],
                     "traffic": traffic,
                     "algorithmic_bytes": path.attn_bytes()},
        "roofline_reorder_rope": {"bound": "hbm", "achieved": rr_gbs, "peak": pk["hbm_gbs"],
                                  "unit": "GB/s",
                                  "frac": (rr_gbs / pk["hbm_gbs"]) if rr_gbs else None,
                                  "peak_kind": f"{pk_kind} copy"},
        "gpu_launches": path.launches_per_step() * args.steps,
        "clocks": clk,
    }
    if args.backward:
        b_ms = statistics.median(phases["bwd_attn"])
        b_exec = path.bwd_flops() / (b_ms * 1e-3) / 1e12
        out["backward"] = {
            "attn_bwd_ms": b_ms, "pre_ms": statistics.median(phases["bwd_pre"]),
            "post_ms": statistics.median(phases["bwd_post"]),
            "attn_bwd_tflops_executed": b_exec,
            "attn_bwd_tflops_model": flops * 5 / 2 / (b_ms * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "attn_bwd_tc_kernel (dQ + dK/dV, with "
                         "the delta pass in the timed call)", "achieved": b_exec,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": b_exec / peak_tf,
                         "peak_kind": peak_kind}}
    if e2e:
        out["e2e"] = e2e
    if not args.no_cpu_baseline and world == 1 and args.backward and args.mask in ("all",
                                                                                  "aligned"):
        tf, cores, sample, _ = time_oracle_bwd(w, args.mask)
        out["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample, "counts": "backward as 2.5x the forward"}
    if not args.no_cpu_baseline and world == 1 and args.mask == "aligned" and not args.backward:
        tf, cores, sample, _ = time_oracle_aligned(w, budget_s=min(args.cpu_budget, 10.0))
        out["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample,
                               "extrapolated_full_config_s": flops / (tf * 1e12)}
    if not args.no_cpu_baseline and world == 1 and args.mask == "all" and not args.backward:
        tf, cores, sample, _ = time_oracle(w, budget_s=args.cpu_budget)
        out["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample,
                               "extrapolated_full_config_s": flops / (tf * 1e12)}
        gbs, pcores, psample, _ = time_oracle_prep(w, heads=8)
        out["cpu_baseline_reorder_rope"] = {
            "value": gbs, "unit": "GB/s", "cores": pcores, "kind": "oracle", "sample": psample,
            "extrapolated_full_config_s": prep_phase_bytes(w) / (gbs * 1e9)}
    extra = (world == 1 and not args.no_workloads and args.workload == "720p" and
             args.mask == "all" and args.batch == 1 and not args.backward and not args.graph
             and not args.heads)
    if extra:
        # the 4K and long-video grids in the same run, after the 720p buffers
        # are released (the long clip alone holds ~119 GB)
        del path
        out["workloads"] = {}
        for name, k in (("4k", 10), ("4k_long", 5)):
            out["workloads"][name] = run_workload_line(
                args, WORKLOADS[name], dev, stream, max(3, min(args.steps, k)), pk, pk_kind,
                min(args.cpu_budget, 8.0))
    print(json.dumps(out), flush=True)


def run_workload_line(args, w, dev, stream, steps, pk, pk_kind, cpu_budget):
    """One more workload in the same run (the 4K and long-video grids beside
    the 720p headline): the same step, W warm-up and ``steps`` timed steps on
    its own buffers (inputs larger than L2), per-phase CUDA events, clocks
    sampled over its timed region, and the oracle timed on the same grid."""
    torch.cuda.empty_cache()
    with torch.cuda.stream(stream):
        path = Path(w, dev, stream)
    torch.cuda.synchronize(dev)
    for _ in range(max(3, min(args.warmup, 5))):
        path.step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.5)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    start.record(stream)
    for i in range(steps):
        path.step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clocks.window(t_wall0, time.time())
    clk = clocks.stop()
    from video_dit_windowed_b200 import atlas
    code = atlas.last_device_error(stream)
    if code:
        raise RuntimeError(f"device error word 0x{code:x} in the {w.name} timed region")
    elapsed = start.elapsed_time(stop)
    med = lambda k: statistics.median(Path.phase_ms(ev)[k] for ev in evs)
    flops = path.flops()
    attn_ms = med("attn")
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    rr_ms = med("reorder") + med("rope_g")
    rr_gbs = path.prep_bytes() / (rr_ms * 1e-3) / 1e9
    peak_tf, peak_kind = tensor_peak(pk, pk_kind, elapsed * 1e-3)
    ms = elapsed / steps
    line = {
        "value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "steps": steps, "ms_per_step": ms,
        "config": config_of(w, 1),
        "attn_tflops": attn_tf, "attn_ms": attn_ms,
        "roofline": {"bound": "tensor", "kernel": attn_kernel_name(w), "achieved": attn_tf,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": attn_tf / peak_tf,
                     "peak_kind": peak_kind,
                     "frac_of_sustained": attn_tf / pk["bf16_tflops_sustained"],
                     "algorithmic_bytes": path.attn_bytes()},
        "roofline_reorder_rope": {"bound": "hbm", "achieved": rr_gbs, "peak": pk["hbm_gbs"],
                                  "unit": "GB/s", "frac": rr_gbs / pk["hbm_gbs"],
                                  "peak_kind": f"{pk_kind} copy", "ms": rr_ms,
                                  "algorithmic_bytes": path.prep_bytes()},
        "gpu_launches": path.launches_per_step() * steps,
        "clocks": clk,
    }
    del path
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        tf, cores, sample, _ = time_oracle(w, budget_s=cpu_budget)
        line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample,
                                "extrapolated_full_config_s": flops / (tf * 1e12)}
        gbs, pcores, psample, _ = time_oracle_prep(w)
        line["cpu_baseline_reorder_rope"] = {
            "value": gbs, "unit": "GB/s", "cores": pcores, "kind": "oracle", "sample": psample,
            "extrapolated_full_config_s": prep_phase_bytes(w) / (gbs * 1e9)}
    return line


def report_proj(args, world, rank, path, elapsed, phases, clk):
    """JSON line of a --proj run: the whole step's FLOPs (projections +
    attention), the fused projections' TFLOP/s and roofline, and the unfused
    comparison."""
    if rank != 0:
        return
    pk, pk_kind = peaks()
    ms = elapsed / args.steps
    f_qkv, f_out = path.proj_flops()
    f_attn = path.flops()
    med = lambda k: statistics.median(phases[k])
    qkv_ms = med("qkv_d") + med("qkv_g")
    out_ms = med("out")
    proj_tf = (f_qkv + f_out) / ((qkv_ms + out_ms) * 1e-3) / 1e12
    un_qkv, un_out = path.unfused_ms(min(args.steps, 10))
    peak_tf, peak_kind = tensor_peak(pk, pk_kind, elapsed * 1e-3)
    out = {
        "metric": METRIC + " (with fused projections)", "value":
            world * (f_qkv + f_out + f_attn) / (ms * 1e-3) / 1e12, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded inputs, random weights)",
        "config": dict(config_of(path.w, world), model_width=path.C, projections="fused"),
        "qkv_proj_ms": qkv_ms, "out_proj_ms": out_ms, "attn_ms": med("attn"),
        "qkv_proj_tflops": f_qkv / (qkv_ms * 1e-3) / 1e12,
        "out_proj_tflops": f_out / (out_ms * 1e-3) / 1e12,
        "attn_tflops": f_attn / (med("attn") * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "gemm_proj_kernel (QKV + output projections)",
                     "achieved": proj_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": proj_tf / peak_tf, "peak_kind": peak_kind},
        "unfused_detail_ms": {"qkv_cublas_plus_reorder": un_qkv,
                              "unorder_plus_cublas_out": un_out,
                              "fused_qkv_detail": med("qkv_d"), "fused_out_detail_and_global":
                                  out_ms},
        "gpu_launches": path.launches_per_step() * args.steps,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        tf, cores, sample, _ = time_oracle_proj(path.w)
        out["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample, "counts": "projection FLOPs only"}
    print(json.dumps(out), flush=True)


def run_e2e(path, w, dev, stream, args, world, twin=None):
    """The same step through the C-ABI with host buffers: every step uploads
    its inputs from pinned host memory (the six raster tensors; with
    --backward also dO) and downloads its results (O_d and O_g; with
    --backward also the six gradients). With ``twin`` (a second set of device
    buffers) the steps are pipelined: step i+1's upload (one copy stream) and
    step i-1's download (another) overlap step i's compute; each step still
    carries its own copies. Without it the copies and the compute of a step
    run in order on one stream."""
    paths = [path] + ([twin] if twin is not None else [])

    def dev_inputs(p):
        d = dict(p.x)
        if p.backward:
            d.update({"do_d": p.do["d"], "do_g": p.do["g"]})
        return d

    def results(p):
        r = list(p.outputs())
        if p.backward:
            r += p.gradients()
        return r

    ins = [dev_inputs(p) for p in paths]
    res = [results(p) for p in paths]
    host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in ins[0].items()}
    for k in host:
        host[k].copy_(ins[0][k].cpu())
    outs = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in r] for r in res]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs[0])
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    n_sets = len(paths)
    ev = lambda: torch.cuda.Event()
    in_ready = [ev() for _ in range(n_sets)]
    comp_done = [ev() for _ in range(n_sets)]
    out_done = [ev() for _ in range(n_sets)]

    def one(i):
        b = i % n_sets
        if n_sets == 1:
            with torch.cuda.stream(stream):
                for k in host:
                    ins[0][k].copy_(host[k], non_blocking=True)
                paths[0].step()
                for o, t in zip(outs[0], res[0]):
                    o.copy_(t, non_blocking=True)
            return
        with torch.cuda.stream(up):
            if i >= n_sets:
                up.wait_event(comp_done[b])        # set b's inputs are free again
            for k in host:
                ins[b][k].copy_(host[k], non_blocking=True)
            in_ready[b].record(up)
        stream.wait_event(in_ready[b])
        if i >= n_sets:
            stream.wait_event(out_done[b])         # set b's results were read
        paths[b].step()
        comp_done[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[b])
            for o, t in zip(outs[b], res[b]):
                o.copy_(t, non_blocking=True)
            out_done[b].record(down)

    for i in range(min(args.warmup, 3)):
        one(i)
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 10))
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    first = up if n_sets > 1 else stream
    last = down if n_sets > 1 else stream
    t0.record(first)
    for i in range(steps):
        one(i)
    t1.record(last)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    step_flops = path.flops() * 7 // 2 if path.backward else path.flops()
    return {"value": world * step_flops / (ms * 1e-3) / 1e12, "unit": UNIT,
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "pipelined": n_sets > 1}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="atlas", choices=["atlas", "reference"])
    ap.add_argument("--workload", default="720p", choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the 4K and long-video lines the default 720p run adds")
    ap.add_argument("--mask", default="all", choices=["all", "aligned", "raster", "dense"],
                    help="all: the method (every global key); aligned: aligned global keys "
                         "only; raster / dense: comparison modes (naive raster-order blocks, "
                         "full attention)")
    ap.add_argument("--batch", type=int, default=1, help="problems per GPU")
    ap.add_argument("--graph", action="store_true",
                    help="capture the step in a CUDA graph and time its replays (phase times "
                         "come from eager steps after the timed region)")
    ap.add_argument("--proj", action="store_true",
                    help="include the QKV and output projections, fused with the reorder, "
                         "RoPE and unorder (random weights, model width heads*head_dim)")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step: the forward path plus its backward (gradients "
                         "w.r.t. the raster inputs); value counts the backward as 2.5x the "
                         "forward FLOPs")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="with --gpus N: replicas (every rank runs its own problem, weak "
                         "scaling) or heads (the ranks split one problem's heads, strong "
                         "scaling)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads instead of its own "
                         "(smaller cases for profiler captures; reported in config)")
    args = ap.parse_args()
    if args.shard == "heads" and args.proj:
        raise SystemExit("--proj runs replicas only: with the heads split, the output "
                         "projection would need a sum over the ranks")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_atlas(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
