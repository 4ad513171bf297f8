"""Benchmark of the MTA forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mine|reference]

One step = one call of the library over one batch of seeded synthetic input
(mta_attn_fwd for attention workloads, mta_layer_fwd for layer workloads).
Inputs rotate through three resident sets larger than L2 together, so no step
reads its inputs from L2 left by the previous one.  Timing: W untimed warm-up
steps, then K steps bracketed by a barrier and torch.cuda.synchronize(), timed
with CUDA events on the launch stream; the max over ranks is reported.  Rank 0
prints one JSON line.

Multi-GPU (torchrun): the (batch, head-group) units of MTA are independent, so
every rank runs its own copy of the workload (weak scaling, no collective on
the data path); value = all ranks' tokens / max-over-ranks time.

--impl reference times the fp64 CPU oracle (test infrastructure, oracle/) on a
bounded sample of the same workload on the host cores; it is a deliberately
slow baseline, not a target.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from token_attention_b200 import synth  # noqa: E402

METRIC = "MTA fwd tokens/s and TFLOP/s at L=2048 on 1 B200; % of BF16 tensor peak"
METRIC_BWD = "MTA attention backward (mta_attn_bwd) tokens/s on 1 B200"
METRIC_LAYER_BWD = "MTA layer backward (mta_layer_bwd) tokens/s on 1 B200"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "pretrain_d128_L2048"
N_SETS = 3
# B200: 148 SMs x 128 fp32 lanes x 2 flop per FMA at the 1965 MHz max SM clock
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# workload arithmetic (algorithmic counts per step)
# ---------------------------------------------------------------------------

def flops(wl: synth.Workload) -> dict:
    """Algorithmic flops of one step.  Per causal (query, key) pair and head:
    F_std = 4d (Q K^T and A V), F_mta = F_std + 2 c_q c_k + 2 c_h
    (the key-query convolution and the head mix), plus 2 c_q c_k more when the
    convolution also acts after the softmax.  Layer adds 2 B L D 4D
    (QKV and output projections)."""
    P = wl.causal_pairs
    f_std = 4 * wl.d * P
    conv = 2 * wl.c_q * wl.c_k * ((1 if wl.kq_place else 0) + (1 if wl.kq_post else 0)) * P
    mix = (2 * wl.c_h if wl.head_place else 0) * P
    gemm = 2 * wl.B * wl.L * wl.D * 4 * wl.D if wl.layer else 0
    return {"std": f_std + gemm, "mta": f_std + conv + mix + gemm, "conv": conv, "gemm": gemm,
            "attn_std": f_std, "attn_mta": f_std + conv + mix}


def uses_contraction(wl: synth.Workload) -> bool:
    """Whether the library's default path runs the contraction kernel (with its
    prepass) for this workload."""
    return (wl.dtype == "bf16" and wl.d in (64, 96, 128) and wl.kq_place == synth.PRE
            and (wl.c_q, wl.c_k) == (6, 11)
            and (wl.head_place == synth.OFF or wl.c_h == 2))


def kq_kernel_name(wl: synth.Workload) -> str:
    """The contraction kernel the library launches: the CTA-pair form for sequences of
    4096 and more (d = 128, or d = 64 with post-softmax mixing; no post-softmax
    convolution), else the one-CTA form."""
    pair = (wl.L >= 4096 and not wl.kq_post and
            ((wl.d == 128 and wl.head_place in (synth.OFF, synth.POST)) or
             (wl.d == 64 and wl.head_place == synth.POST)))
    return "attn_kq_pair_kernel" if pair else "attn_kq_kernel"


def contraction_tensor_flops(wl: synth.Workload) -> float:
    """Tensor flops the contraction kernel executes per launch: per (batch, head,
    query tile, key tile at or below the diagonal) a 128x128 tile of the
    c_q*d-long contraction (for each source head of the group with pre-softmax
    mixing) and, per V head held (both heads of the group with post-softmax
    mixing), a 128x128xd P V product.  With the post-softmax convolution the
    query tiles hold 123 output rows, the contraction runs in both passes and
    P V becomes c_q row-shifted products with the convolved values."""
    nv = 2 if wl.head_place == synth.POST else 1
    nsrc = 2 if wl.head_place == synth.PRE else 1
    if wl.kq_post:
        nq = -(-wl.L // 123)
        tiles = wl.B * wl.H * sum(min(wl.L - 1, qt * 123 - 5 + 127) // 128 + 1 for qt in range(nq))
        return tiles * 2.0 * 128 * 128 * (2 * nsrc * wl.c_q * wl.d + nv * wl.c_q * wl.d)
    nt = -(-wl.L // 128)
    tiles = wl.B * wl.H * nt * (nt + 1) // 2
    return tiles * 2.0 * 128 * 128 * (nsrc * wl.c_q * wl.d + nv * wl.d)


def uses_direct_tc(wl: synth.Workload) -> bool:
    """Whether the default path runs the direct tensor-core kernel."""
    return (not uses_contraction(wl) and wl.dtype == "bf16" and wl.d in (64, 128)
            and not wl.kq_post and (wl.c_h == 2 or wl.head_place == synth.OFF)
            and (wl.kq_place == synth.OFF or (wl.c_q, wl.c_k) == (6, 11)))


def uses_bwd_tc(wl: synth.Workload) -> bool:
    """Whether the default backward runs on the tensor cores (attn_bwd_tc.cu)."""
    return (wl.dtype == "bf16" and wl.d in (64, 96, 128) and wl.kq_place == synth.PRE
            and (wl.c_q, wl.c_k) == (6, 11)
            and (wl.head_place == synth.OFF or wl.c_h == 2))


def bwd_tc_rows(wl: synth.Workload) -> int:
    """Rows of a query block's S strip in the tensor-core backward (its choice from L)."""
    return 384 if wl.L <= 3072 else 512


def bwd_tc_no(wl: synth.Workload) -> int:
    """Own rows of a query block of the tensor-core backward."""
    return bwd_tc_rows(wl) - (3 if wl.kq_post else 2) * (wl.c_q - 1)


def bwd_tc_launches(wl: synth.Workload) -> int:
    """Kernels of the tensor-core backward per call: per query block the S and dA''
    GEMMs, the convolution / softmax kernel, the adjoint kernel and the dQ, dK and dV
    GEMMs; with the convolution after the softmax four more (its output gradient, its
    adjoint, the mixed weights, the softmax's backward)."""
    return (11 if wl.kq_post else 7) * -(-wl.L // bwd_tc_no(wl))


def bwd_tc_gemm_flops(wl: synth.Workload) -> float:
    """Tensor flops the tensor-core backward's GEMMs execute per call (bf16 MMAs):
    per query block of NO rows (strips of R rows) and keys 0 .. W-1, for every
    head: S (R x W x d), dA'' (RC x W x d), dQ (NO x d x 2W: hi and lo halves),
    dK and dV (W x d x 2R)."""
    R, no = bwd_tc_rows(wl), bwd_tc_no(wl)
    rc = no + (2 if wl.kq_post else 1) * (wl.c_q - 1)
    f = 0.0
    for r0 in range(0, wl.L, no):
        W = min(wl.L, r0 + rc)
        f += 2 * (R + rc) * W * wl.d + 2 * no * wl.d * 2 * W + 2 * 2 * W * wl.d * 2 * R
    return f * wl.B * wl.H


def launches_per_step(wl: synth.Workload) -> int:
    """Kernels of this library one step launches: the attention kernel (and the
    prepass of the contraction kernel); a layer adds the two projection GEMMs,
    and the stand-alone group norm when the attention runs on the CUDA-core
    kernel."""
    kq = uses_contraction(wl)
    tc = uses_direct_tc(wl)
    # the contraction kernel runs after its prepass (and the value prepass with the
    # post-softmax convolution)
    attn = (3 if wl.kq_post else 2) if kq else 1
    if not wl.layer:
        return attn
    return 2 + (attn if (kq or tc) else 2)


def max_over_ranks(ms: float, world: int, device) -> float:
    """The job's time: the largest of the ranks' device-timed milliseconds (an
    all-reduce MAX over the default process group when there is more than one)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank_step: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank processes its own batch each step (weak
    scaling, replicas), divided by the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (ms / 1e3)


def read_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# source files each kernel's code comes from (a committed traffic figure counts only
# while these files are unchanged since its capture)
KERNEL_SOURCES = {
    "attn_kq_kernel": ("attn_kq.cu", "ptx.cuh"),
    "attn_kq_pair_kernel": ("attn_kq_pair.cu", "ptx.cuh"),
    "kq_prep_kernel": ("kq_prep.cu",),
    "vt_prep_kernel": ("kq_prep.cu",),
    "attn_tc_kernel": ("attn_tc.cu", "ptx.cuh"),
    "attn_simt_kernel": ("attn_simt.cu",),
    "attn_bwd_simt_kernel": ("attn_bwd_simt.cu", "bwd_common.cuh"),
    "attn_bwd_post_kernel": ("attn_bwd_post_simt.cu", "bwd_common.cuh"),
    "group_norm_d128_kernel": ("group_norm.cu",),
    "gemm_bf16_nt_kernel": ("gemm_tc.cu", "ptx.cuh"),
}


def source_sha(kernel_key: str) -> str | None:
    """sha1 (16 hex digits) over the source files of a kernel, as committed."""
    import hashlib
    files = KERNEL_SOURCES.get(kernel_key)
    if not files:
        return None
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "token_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def read_traffic(kernel_key: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if one matches this
    workload and was taken from the kernel's current source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f)
    e = t.get(kernel_key, {}).get(workload)
    if e is None or e.get("source_sha") != source_sha(kernel_key):
        return None
    return e.get("bytes_per_launch")


def call_traffic(kernel_keys, workload: str):
    """dram bytes of one call made of several launches (null unless every one is known)."""
    parts = [read_traffic(k, workload) for k in kernel_keys]
    return None if any(x is None for x in parts) else sum(parts)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + f[0].split(".")[1]) if "." in f[0] else 0.0
                rows.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except (ValueError, IndexError):
                continue
        if not rows:
            return None
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.15 <= r[0] <= self.t1 + 0.15]
        use = inside or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "samples_in_window": len(inside)}


# ---------------------------------------------------------------------------
# the library arm
# ---------------------------------------------------------------------------

def make_sets(wl, dev, n_sets, bwd=False, rank=0):
    """n_sets input sets of the workload.  Under N ranks each rank draws its own
    batches (a seed offset per rank): the ranks process different units of the
    same shape, with no exchange between them."""
    import torch

    def to(x, dt):
        t = torch.from_numpy(np.ascontiguousarray(x)).to(dev)
        return t.to(torch.bfloat16) if dt == "bf16" else t

    sets = []
    for s in range(n_sets):
        w = synth.shrink(wl, seed=wl.seed + 100 * s + 100_000 * rank)
        if wl.layer:
            inp = synth.make_layer_inputs(w)
            keys = ("x", "wqkv", "wo", "theta", "w", "gamma", "beta")
            sets.append({k: to(inp[k], "bf16" if k in ("x", "wqkv", "wo") else "f32") for k in keys})
        else:
            inp = synth.make_attn_inputs(w)
            sets.append({k: to(inp[k], wl.dtype if k in "qkv" else "f32")
                         for k in ("q", "k", "v", "theta", "w")})
        sets[-1]["theta_post"] = None
        if inp["theta_post"] is not None:  # pre- and post-softmax kernels stacked once, outside the timed steps
            sets[-1]["theta"] = to(np.stack([inp["theta"], inp["theta_post"]]), "f32")
        if bwd:  # gradient of the output, drawn like the values
            dout = synth.normal(w.seed, 20, (wl.B, wl.L, wl.D) if wl.layer else (wl.B, wl.L, wl.H, wl.d))
            sets[-1]["dout"] = to(synth.round_bf16(dout) if wl.dtype == "bf16" else dout, wl.dtype)
    return sets


def step_fn(wl, mta, sets, ws, outs, stream, bwd=False):
    """Returns f(i, events=None): enqueue step i (input set i % n) on `stream`;
    the library records `events` around the step's kernels (mta_cfg.events)."""
    if bwd and wl.layer:
        def f(i, events=None):
            s = sets[i % len(sets)]
            mta.layer_bwd(s["x"], s["wqkv"], s["theta"], s["w"], s["gamma"], s["beta"], s["wo"], s["dout"],
                          wl.H, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, eps=1e-5,
                          layer=wl.depth, ws=ws, stream=stream, theta_post=s["theta_post"], events=events)
    elif bwd:
        def f(i, events=None):
            s = sets[i % len(sets)]
            mta.attn_bwd(s["q"], s["k"], s["v"], s["theta"], s["w"], s["dout"], wl.c_q, wl.c_k, wl.c_h,
                         wl.kq_place, wl.head_place, ws=ws, stream=stream, grads=outs[i % len(outs)],
                         events=events)
    elif wl.layer:
        def f(i, events=None):
            s = sets[i % len(sets)]
            mta.layer_fwd(s["x"], s["wqkv"], s["theta"], s["w"], s["gamma"], s["beta"], s["wo"],
                          wl.H, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, eps=1e-5,
                          layer=wl.depth, out=outs[i % len(outs)], ws=ws, stream=stream,
                          theta_post=s["theta_post"], events=events)
    else:
        def f(i, events=None):
            s = sets[i % len(sets)]
            mta.attn_fwd(s["q"], s["k"], s["v"], s["theta"], s["w"], wl.c_q, wl.c_k, wl.c_h,
                         wl.kq_place, wl.head_place, out=outs[i % len(outs)], ws=ws, stream=stream,
                         theta_post=s["theta_post"], events=events)
    return f


def step_kernels(wl: synth.Workload, bwd: bool) -> list[str]:
    """Names of the library's kernels one step launches, in launch order (the
    library records a timing event after each; see mta_cfg.events)."""
    bwd_kernel = ("attn_bwd_tc" if uses_bwd_tc(wl) else
                  "attn_bwd_post_kernel" if wl.kq_post else "attn_bwd_simt_kernel")
    if bwd and wl.layer:
        return (["gemm_qkv"] + [k for k in step_kernels(wl, False)[1:-1] if k != "group_norm_kernel"] +
                ["gemm_dy", "group_norm_bwd_kernel", "gemm_dwo", bwd_kernel, "pack_qkv_grad_kernel",
                 "gemm_dx", "gemm_dwqkv"])
    if bwd:
        return [bwd_kernel]
    if uses_contraction(wl):
        attn = ["kq_prep_kernel"] + (["vt_prep_kernel"] if wl.kq_post else []) + [kq_kernel_name(wl)]
    elif uses_direct_tc(wl):
        attn = ["attn_tc_kernel"]
    else:
        attn = ["attn_simt_kernel"] + (["group_norm_kernel"] if wl.layer else [])
    return ["gemm_qkv"] + attn + ["gemm_out"] if wl.layer else attn


def dominant_kernel(wl: synth.Workload, bwd: bool) -> tuple[int, int, str]:
    """(a, b, name): the step's dominant kernel runs between the library's timing
    events a and b of a step (event 0 before the first kernel, event k after the
    k-th; see mta_cfg.events), and its name."""
    if bwd:
        names = step_kernels(wl, True)
        i = next(k for k, n in enumerate(names) if n.startswith("attn_bwd"))
        return i, i + 1, names[i]
    n = launches_per_step(wl) + 1
    if uses_contraction(wl):
        # ... key prepass, (value prepass), attention kernel, (output GEMM)
        k = kq_kernel_name(wl)
        return (n - 3, n - 2, k) if wl.layer else (n - 2, n - 1, k)
    name = "attn_tc_kernel" if uses_direct_tc(wl) else "attn_simt_kernel"
    return (1, 2, name) if wl.layer else (0, 1, name)


def choose_peak(peaks: dict, region_ms: float, clocks) -> tuple[float, str]:
    """The bf16 denominator for the timed region: the sustained figure only for a
    region of a second or more that ran under the power cap, else the burst one."""
    capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    if region_ms >= 1000.0 and capped:
        return peaks["bf16_tflops_sustained"], f"sustained (timed region {region_ms:.0f} ms under sw_power_cap)"
    why = "no power cap" if not capped else "region shorter than 1 s"
    return peaks["bf16_tflops"], f"burst (timed region {region_ms:.1f} ms, {why})"


def run_epilogue(mta, dev, stream, launches=20):
    """The group norm with depth scale as its own kernel (mta_group_norm_scale) on the
    full layer's Y: 8192 tokens x 16 heads x 128 channels bf16 (B*L = 2*4096,
    D = 2048).  Four input/output pairs rotate (4 x 67 MB, above the 126 MB L2), so
    that no launch reads data the previous one left in L2.  Returns achieved
    HBM GB/s on the algorithmic bytes (2 B read + 2 B written per element)."""
    import torch
    T, H, d = 8192, 16, 128
    g = torch.Generator(device="cpu").manual_seed(5)
    xs = [torch.randn((T, H, d), generator=g).to(torch.bfloat16).to(dev) for _ in range(4)]
    ys = [torch.empty_like(xs[0]) for _ in range(4)]
    gamma = (1 + 0.1 * torch.randn(H * d, generator=g)).to(dev)
    beta = (0.1 * torch.randn(H * d, generator=g)).to(dev)
    for i in range(3):
        mta.group_norm_scale(xs[i % 4], gamma, beta, 1e-5, 0.978141, out=ys[i % 4], stream=stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(launches):
            ev[i][0].record(stream)
            mta.group_norm_scale(xs[i % 4], gamma, beta, 1e-5, 0.978141, out=ys[i % 4], stream=stream)
            ev[i][1].record(stream)
    stream.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    nbytes = 2 * T * H * d * 2
    return {"kernel": "group_norm_d128_kernel", "workload": "Y of layer_*_D2048_L4096: 8192 x 16 x 128 bf16",
            "bytes_per_launch": nbytes, "ms_per_launch": ms, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
            "launches": launches, "l2": "4 rotating input/output pairs (268 MB)"}


def run_mine(args, wl, rank, world, local_rank):
    import torch
    from token_attention_b200 import mta
    import ctypes

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    mta.lib()
    stream = torch.cuda.Stream(device=dev)
    sets = make_sets(wl, dev, N_SETS, args.bwd, rank)
    out_shape = (wl.B, wl.L, wl.D) if wl.layer else (wl.B, wl.L, wl.H, wl.d)
    odt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    if args.bwd and wl.layer:  # mta.layer_bwd allocates its gradients
        outs = [None]
    elif args.bwd:  # fp32 gradients of q, k, v, the kernels and the mixing weights
        z = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
        n_th = (1 if wl.kq_place else 0) + (1 if wl.kq_post else 0)
        outs = []
        for _ in range(N_SETS):
            dth = z(n_th, wl.H, wl.c_q, wl.c_k) if n_th else None
            outs.append({"dq": z(*out_shape), "dk": z(*out_shape), "dv": z(*out_shape), "dtheta_all": dth,
                         "dtheta": None, "dtheta_post": None,
                         "dw": z(wl.H // wl.c_h, wl.c_h, wl.c_h) if wl.head_place else None})
    else:
        outs = [torch.empty(out_shape, dtype=odt, device=dev) for _ in range(N_SETS)]
    cfg = mta.make_cfg(wl.B, wl.H, wl.L, wl.d, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                       mta.F32 if wl.dtype == "f32" else mta.BF16, kq_post=int(wl.kq_post))
    if args.bwd:
        nbytes = (mta.lib().mta_layer_bwd_workspace_bytes if wl.layer else mta.lib().mta_attn_bwd_workspace_bytes)(
            ctypes.byref(cfg))
    else:
        nbytes = (mta.lib().mta_layer_workspace_bytes if wl.layer else mta.lib().mta_attn_workspace_bytes)(
            ctypes.byref(cfg))
    ws = mta.workspace(nbytes, dev)
    f = step_fn(wl, mta, sets, ws, outs, stream, args.bwd)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    sampler = ClockSampler(local_rank) if not args.no_clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    warm = max(3, args.warmup)
    with torch.cuda.stream(stream):
        for i in range(warm):
            f(i)
    stream.synchronize()
    # status word of the warm-up calls: no kernel gave up a wait
    cfg.workspace, cfg.workspace_bytes, cfg.stream = ws.data_ptr(), ws.numel(), stream.cuda_stream
    st = mta.lib().mta_sync_status(ctypes.byref(cfg))
    if st != 0:
        raise RuntimeError(f"warm-up status {mta.STATUS.get(st, st)}")

    # the library records n_ev events per step around its kernels (mta_cfg.events);
    # each is recorded once here first, so that torch has created it
    n_ev = len(step_kernels(wl, args.bwd)) + 1
    step_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for evs in step_ev:
            for e in evs:
                e.record(stream)
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_begin()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_begin.record(stream)
        for i in range(args.steps):
            f(warm + i, step_ev[i])
        t_end.record(stream)
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_end()
    total_ms = t_begin.elapsed_time(t_end)
    ka, kb, kname = dominant_kernel(wl, args.bwd)
    kernel_ms = [evs[ka].elapsed_time(evs[kb]) for evs in step_ev]
    names = step_kernels(wl, args.bwd)
    per_kernel = {f"{i}:{n}": statistics.mean(evs[i].elapsed_time(evs[i + 1]) for evs in step_ev)
                  for i, n in enumerate(names) if i + 1 < n_ev}
    step_ms = [evs[0].elapsed_time(evs[-1]) for evs in step_ev]
    st = mta.lib().mta_sync_status(ctypes.byref(cfg))
    if st != 0:
        raise RuntimeError(f"timed-region status {mta.STATUS.get(st, st)}")
    # every call clears the error word, so a wait that ran out in an earlier step shows
    # only as that step's time: at least the 2 s wait bound, hidden in the mean of a
    # long timed region (short profiling runs, whose profiled steps take that long
    # too, are not checked)
    med = statistics.median(step_ms)
    if args.steps >= 20 and max(step_ms) >= 1900.0:
        raise RuntimeError(f"a step took {max(step_ms):.1f} ms against a median of {med:.3f} ms: "
                           "a bounded wait ran out during the timed region")
    clocks = sampler.stop() if sampler else None

    t_max = max_over_ranks(total_ms, world, dev)

    e2e = None
    if not args.no_e2e and not args.bwd:
        e2e = run_e2e(args, wl, mta, sets, ws, stream, dev, barrier, world)
    epi = None
    if not args.no_epilogue and not args.bwd and rank == 0:
        epi = run_epilogue(mta, dev, stream)
    return {"total_ms": t_max, "region_ms": total_ms, "kernel_ms": statistics.mean(kernel_ms),
            "per_kernel_ms": per_kernel,
            "kernel": kname, "kernel_calls_ms": statistics.mean(step_ms), "clocks": clocks, "e2e": e2e,
            "warmup": warm, "epilogue": epi}


def run_e2e(args, wl, mta, sets, ws, stream, dev, barrier, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory to the device, runs the call, and reads
    the result back to pinned host memory.  The steps are pipelined over three
    streams with two buffer slots: step i+1's upload and step i-1's download run
    while step i computes (PCIe is full duplex, and the copy engines are not the
    SMs)."""
    import torch
    names = ("x",) if wl.layer else ("q", "k", "v")
    host_sets = [{n: s[n].cpu().pin_memory() for n in names} for s in sets]
    dev_in = [{n: torch.empty_like(sets[0][n]) for n in names} for _ in range(2)]
    out_shape = (wl.B, wl.L, wl.D) if wl.layer else (wl.B, wl.L, wl.H, wl.d)
    odt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    douts = [torch.empty(out_shape, dtype=odt, device=dev) for _ in range(2)]
    houts = [torch.empty(out_shape, dtype=odt).pin_memory() for _ in range(2)]
    steps = max(3, min(args.steps, args.e2e_steps))
    h2d = sum(host_sets[0][n].numel() * host_sets[0][n].element_size() for n in names)
    d2h = houts[0].numel() * houts[0].element_size()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    in_free = [ev(), ev()]    # the call of slot k has read its inputs
    out_free = [ev(), ev()]   # the download of slot k has read its output
    primed = [False, False]

    def one(i):
        k = i % 2
        hs, s = host_sets[i % len(host_sets)], sets[i % len(sets)]
        in_ready, out_ready = ev(), ev()
        with torch.cuda.stream(up):
            if primed[k]:
                up.wait_event(in_free[k])
            for n in names:
                dev_in[k][n].copy_(hs[n], non_blocking=True)
            in_ready.record(up)
        with torch.cuda.stream(stream):
            stream.wait_event(in_ready)
            if primed[k]:
                stream.wait_event(out_free[k])
            x = dev_in[k]
            if wl.layer:
                mta.layer_fwd(x["x"], s["wqkv"], s["theta"], s["w"], s["gamma"], s["beta"], s["wo"],
                              wl.H, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, layer=wl.depth,
                              out=douts[k], ws=ws, stream=stream, theta_post=s["theta_post"])
            else:
                mta.attn_fwd(x["q"], x["k"], x["v"], s["theta"], s["w"], wl.c_q, wl.c_k, wl.c_h,
                             wl.kq_place, wl.head_place, out=douts[k], ws=ws, stream=stream,
                             theta_post=s["theta_post"])
            in_free[k].record(stream)
            out_ready.record(stream)
        with torch.cuda.stream(down):
            down.wait_event(out_ready)
            houts[k].copy_(douts[k], non_blocking=True)
            out_free[k].record(down)
        primed[k] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    for i in range(steps):
        one(i)
    down.wait_stream(up)
    down.wait_stream(stream)
    b.record(down)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    return {"value": job_tokens_per_s(world, wl.tokens, steps, ms), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": ms / steps, "pipelined": "uploads, calls and downloads on three streams, two slots"}


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(wl, budget_s: float, mode: str):
    """Times the oracle on a bounded sample of the workload.  mode "groups":
    whole head groups at full length; mode "rows": single query rows of one
    head group.  Returns (tokens-equivalent/s, seconds, description)."""
    import oracle as O
    if wl.layer and mode == "bwd_groups":
        # the layer backward's dominant step: the attention backward of whole head
        # groups of batch 0 at full length, on its QKV (computed outside the timing)
        inp = synth.make_layer_inputs(wl)
        D, ch, H = wl.D, wl.c_h, wl.H
        qkv = inp["x"][0].astype(np.float64) @ inp["wqkv"].astype(np.float64).T
        q, k, v = (qkv[:, i * D:(i + 1) * D].reshape(wl.L, H, wl.d) for i in range(3))
        dout = synth.normal(wl.seed, 20, (wl.L, H, wl.d))
        tp = inp["theta_post"]
        done, t0 = 0, time.perf_counter()
        for g in range(H // ch):
            hs = slice(g * ch, (g + 1) * ch)
            grp = lambda x: np.ascontiguousarray(x[:, hs].transpose(1, 0, 2))
            O.mta_attention_group_bwd(grp(q), grp(k), grp(v), inp["theta"][hs], inp["w"][g], np.arange(wl.L),
                                      1 / math.sqrt(wl.d), wl.kq_place, wl.head_place, grp(dout),
                                      None if tp is None else tp[hs])
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        tok = done * ch / H * wl.L
        return tok / dt, dt, (f"attention backward (the layer backward's dominant step) of {done} of {H // ch} "
                              f"head groups of one batch at full length L={wl.L} ({tok:.0f} token-equivalents; "
                              f"the projections' and the norm's gradients are not in the sample)")
    if wl.layer:
        inp = synth.make_layer_inputs(wl)
        rows = [(0, 0)]
        t = time.perf_counter()
        O.mta_layer_rows(inp["x"][:1], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"],
                         inp["beta"], inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, rows,
                         wl.kq_place, wl.head_place, theta_post=inp["theta_post"])
        dt = time.perf_counter() - t
        return 1 / dt, dt, "1 token of the layer (QKV of its batch, attention window, norm, projection)"
    inp = synth.make_attn_inputs(wl)
    q, k, v, th, w = inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"]
    tp = inp["theta_post"]
    ch = wl.c_h
    if mode == "bwd_groups":  # the backward oracle on whole head groups at full length
        n_units = wl.B * (wl.H // ch)
        dout = synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d))
        done, t0 = 0, time.perf_counter()
        for u in range(n_units):
            b, g = divmod(u, wl.H // ch)
            hs = slice(g * ch, (g + 1) * ch)
            grp = lambda x: np.ascontiguousarray(x[b, :, hs].transpose(1, 0, 2))
            O.mta_attention_group_bwd(grp(q), grp(k), grp(v), th[hs], w[g], np.arange(wl.L),
                                      1 / math.sqrt(wl.d), wl.kq_place, wl.head_place, grp(dout),
                                      None if tp is None else tp[hs])
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        tok = done * ch / wl.H * wl.L
        return tok / dt, dt, (f"backward of {done} of {n_units} (batch, head-group) units at full length "
                              f"L={wl.L} ({tok:.0f} token-equivalents)")
    if mode == "groups":
        n_units = wl.B * (wl.H // ch)
        done, t0 = 0, time.perf_counter()
        for u in range(n_units):
            b, g = divmod(u, wl.H // ch)
            hs = slice(g * ch, (g + 1) * ch)
            O.mta_attention_group(np.ascontiguousarray(q[b, :, hs].transpose(1, 0, 2)),
                                  np.ascontiguousarray(k[b, :, hs].transpose(1, 0, 2)),
                                  np.ascontiguousarray(v[b, :, hs].transpose(1, 0, 2)),
                                  th[hs], w[g], np.arange(wl.L), 1 / math.sqrt(wl.d),
                                  wl.kq_place, wl.head_place,
                                  None if tp is None else tp[hs])
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        tok = done * ch / wl.H * wl.L
        return tok / dt, dt, (f"{done} of {n_units} (batch, head-group) units at full length "
                              f"L={wl.L} ({tok:.0f} token-equivalents)")
    # rows of one head group, spread over the sequence
    rng = np.random.default_rng(0)
    done, t0 = 0, time.perf_counter()
    g = 0
    hs = slice(0, ch)
    while True:
        i = int(rng.integers(wl.L))
        O.mta_attention_rows(q[:1, :, hs], k[:1, :, hs], v[:1, :, hs], th[hs], w[g:g + 1], ch,
                             [(0, i)], wl.kq_place, wl.head_place,
                             theta_post=None if tp is None else tp[hs])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    tok = done * ch / wl.H
    return tok / dt, dt, f"{done} single query rows of one head group (uniform positions)"


def run_reference(args, wl, rank):
    if rank != 0:
        return None
    budget_total = 150.0
    nsteps = max(1, args.steps) + max(3, args.warmup)
    per_step = max(0.02, min(2.0, budget_total / nsteps))
    # warm-up steps (untimed), then timed steps
    for _ in range(max(3, args.warmup)):
        oracle_sample(wl, per_step, "rows")
    vals, secs = [], 0.0
    desc = ""
    for _ in range(max(1, args.steps)):
        v, s, desc = oracle_sample(wl, per_step, "rows")
        vals.append(v)
        secs += s
    value = statistics.mean(vals)
    return {"value": value, "seconds": secs, "sample": desc, "cores": blas_threads()}


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline (rank 0, N=1)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-epilogue", action="store_true",
                    help="skip the stand-alone group-norm bandwidth measurement")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (mta_attn_bwd) of an attention workload instead")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.WORKLOADS[args.workload]
    fl = flops(wl)
    config = {"workload": wl.name, "B": wl.B, "H": wl.H, "L": wl.L, "d": wl.d, "c_q": wl.c_q,
              "c_k": wl.c_k, "c_h": wl.c_h, "kq_place": ["off", "pre", "post", "pre_exact"][wl.kq_place],
              "kq_post": bool(wl.kq_post),
              "head_place": ["off", "pre", "post"][wl.head_place],
              "parallelism": f"replicas x{max(world, args.gpus)}" if max(world, args.gpus) > 1 else "single",
              "l2": f"{N_SETS} rotating input sets, each step reads a set not touched by the previous step"}
    if wl.layer:
        config["D"] = wl.D

    if args.impl == "reference":
        r = run_reference(args, wl, rank)
        if r is None:
            return 0
        line = {"impl": "reference", "metric": METRIC, "value": r["value"], "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": max(3, args.warmup),
                "ms_per_step": 1e3 * r["seconds"] / max(1, args.steps), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config,
                "cpu_baseline": {"value": r["value"], "unit": UNIT, "cores": r["cores"],
                                 "kind": "oracle", "sample": r["sample"]},
                "e2e": {"value": r["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_mine(args, wl, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms = res["total_ms"]
    value = job_tokens_per_s(world, wl.tokens, args.steps, ms)
    peaks, peak_src = read_peaks()
    # one time everywhere: the step time is the timed region / steps; the dominant
    # kernel's time is the mean, over the timed steps, of the library's events around it
    s = ms / args.steps / 1e3
    ks = res["kernel_ms"] / 1e3
    kernel = res["kernel"]
    bf16_peak, peak_kind = choose_peak(peaks, res["region_ms"], res["clocks"])
    fp32_src = "148 SMs x 128 FP32 lanes x 2 x 1965 MHz"
    timing = (f"achieved = per_unit x units / {kernel}'s mean duration over the {args.steps} timed "
              f"steps (CUDA events the library records around it on the launch stream)")
    if args.bwd and uses_bwd_tc(wl):
        # the tensor-core backward: its CUDA-core kernels take most of its time; their
        # algorithmic work is the convolution recomputed, its adjoint and the kernel
        # gradient, 3 x 2 c_q c_k fp32 flop per causal pair-head.  The time is the whole
        # backward's (its GEMMs included), so the fraction is a lower bound.
        n_conv = 2 if wl.kq_post else 1
        f_cc = 6 * wl.c_q * wl.c_k * n_conv * wl.causal_pairs
        achieved = f_cc / ks / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_PEAK_TFLOPS, "traffic": None,
                "kernel": kernel, "kernel_ms": ks * 1e3,
                "per_unit": f"F_cc = 6 c_q c_k per convolution = {6 * wl.c_q * wl.c_k * n_conv} fp32 flop per "
                            f"causal pair-head (each convolution recomputed, its adjoint and its kernel "
                            f"gradient on the CUDA cores), x {wl.causal_pairs} "
                            f"pair-heads per call; the time is the whole backward's, its "
                            f"{bwd_tc_launches(wl)} kernels (GEMMs included)",
                "peak_source": fp32_src, "timing": timing,
                "tensor_gemm_tflops": bwd_tc_gemm_flops(wl) / ks / 1e12}
    elif args.bwd:
        # the backward on the CUDA cores: F_bwd = 8d + 4 c_q c_k + 4 c_h fp32 flop per causal
        # pair-head (dS, dQ, dK, dV products; the convolution's adjoint and kernel gradient;
        # the mixing adjoints)
        n_conv = (1 if wl.kq_place else 0) + (1 if wl.kq_post else 0)
        f_bwd = (8 * wl.d + 4 * wl.c_q * wl.c_k * n_conv + (4 * wl.c_h if wl.head_place else 0)) \
            * wl.causal_pairs
        achieved = f_bwd / ks / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_PEAK_TFLOPS, "traffic": read_traffic(kernel, wl.name),
                "kernel": kernel, "kernel_ms": ks * 1e3,
                "per_unit": f"F_bwd = 8d + 4 c_q c_k (per convolution) + 4 c_h = {f_bwd // wl.causal_pairs} fp32 flop per "
                            f"causal pair-head, x {wl.causal_pairs} pair-heads per launch",
                "peak_source": fp32_src, "timing": timing}
    elif uses_contraction(wl):
        # the dominant kernel is attn_kq_kernel (after its prepass, inside the layer between
        # the two projection GEMMs): algorithmic flops F_mta per causal pair-head
        achieved = fl["attn_mta"] / ks / 1e12
        executed = contraction_tensor_flops(wl) / ks / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": achieved / bf16_peak, "traffic": read_traffic(kernel, wl.name),
                "kernel": kernel, "kernel_ms": ks * 1e3,
                "per_unit": f"F_mta = 4d + 2 c_q c_k{' x 2' if wl.kq_post else ''} + 2 c_h = "
                            f"{fl['attn_mta'] // wl.causal_pairs} flop "
                            f"per causal pair-head, x {wl.causal_pairs} pair-heads per launch",
                "executed_tensor_tflops": executed, "executed_frac": executed / bf16_peak,
                "executed_note": "MMA work the kernel issues (the contraction of length c_q*d, P V for "
                                 "the heads held): a design figure, not the roofline",
                "peak_source": f"{peak_src} bf16 {peak_kind}", "timing": timing}
    elif not uses_direct_tc(wl):
        # the CUDA-core kernel: every step in fp32 FMA on the CUDA cores
        achieved = fl["attn_mta"] / ks / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_PEAK_TFLOPS, "traffic": read_traffic(kernel, wl.name),
                "kernel": kernel, "kernel_ms": ks * 1e3,
                "per_unit": f"F_mta = {fl['attn_mta'] // wl.causal_pairs} fp32 flop per causal "
                            f"pair-head (both convolutions), x {wl.causal_pairs} pair-heads per launch",
                "peak_source": fp32_src, "timing": timing}
    else:
        achieved = fl["conv"] / ks / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_PEAK_TFLOPS, "traffic": read_traffic(kernel, wl.name),
                "kernel": kernel, "kernel_ms": ks * 1e3,
                "per_unit": f"2*c_q*c_k = {2 * wl.c_q * wl.c_k} fp32 flop per causal pair-head "
                            f"(key-query convolution), x {wl.causal_pairs} pair-heads per launch",
                "peak_source": fp32_src, "timing": timing}
    # the whole call (every kernel of the step) against the bf16 peak
    call_f = fl["mta"] if not args.bwd else None
    roof["call"] = None if args.bwd else {
        "achieved": call_f / s / 1e12, "frac": call_f / s / 1e12 / bf16_peak, "unit": "TFLOP/s",
        "ms": s * 1e3, "flops": "F_mta per causal pair-head" + (" + 8 B L D^2 projection GEMM flops" if wl.layer else ""),
        "peak": bf16_peak, "peak_source": f"{peak_src} bf16 {peak_kind}"}
    epi = res.get("epilogue")
    if epi is not None:
        epi = dict(epi, peak_gbs=peaks["hbm_gbs"], frac=epi["achieved_gbs"] / peaks["hbm_gbs"],
                   peak_source=f"{peak_src} HBM copy bandwidth",
                   traffic=read_traffic("group_norm_d128_kernel", "layer_Y_T8192_H16_d128"))
    line = {
        "metric": (METRIC_LAYER_BWD if wl.layer else METRIC_BWD) if args.bwd else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps,
        "warmup": res["warmup"], "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic", "config": config,
        "tflops": {"std": fl["std"] / s / 1e12, "mta": fl["mta"] / s / 1e12},
        "pct_bf16_peak": {"std": fl["std"] / s / 1e12 / bf16_peak,
                          "mta": fl["mta"] / s / 1e12 / bf16_peak,
                          "peak_tflops": bf16_peak, "peak_source": f"{peak_src} bf16 {peak_kind}"},
        "roofline": roof, "gpu_launches": args.steps * (len(step_kernels(wl, args.bwd))
                                       + (bwd_tc_launches(wl) - 1 if args.bwd and uses_bwd_tc(wl) else 0)),
        "timed_region_ms": res["region_ms"], "per_kernel_ms": res["per_kernel_ms"],
        "clocks": res["clocks"], "e2e": res["e2e"], "epilogue_group_norm": epi,
    }
    if world == 1 and not args.no_cpu:
        mode = "bwd_groups" if args.bwd else "groups" if not wl.layer else "rows"
        v, secs, desc = oracle_sample(wl, args.cpu_budget, mode)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{desc}; {secs:.1f} s",
                                "note": "the stated CPU baseline: the oracle on whole head groups at full "
                                        "length, its natural unit (the --impl reference arm samples single "
                                        "query rows instead, which recomputes every key's logits per row and "
                                        "so runs several times slower per token)"}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
