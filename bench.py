"""Benchmark of the FP8 MoE quantisation + grouped-GEMM hot path on B200.

One step = one pass of the whole path over the dense Llama3-8B FFN
up-projection workload (one expert group, X [8192, 4096] bf16, W [14336,
4096] bf16): rowwise quantisation of X (one scale per token), rowwise
quantisation of W (one scale per output channel), FP8 scaled grouped GEMM
(fp32 out).  ``value`` is the step's throughput in GEMM-equivalent TFLOP/s
(2*M*N*K per step divided by the whole step time, quantisation included);
the per-kernel figures (quantisation GB/s, GEMM TFLOP/s, fractions of the
measured peaks) sit beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of
the workload (the path has no exchange step; weak scaling); the timed region
is bracketed by a barrier and a device synchronise, and the time is the max
over ranks.  ``--impl reference`` times the CPU oracle (single thread) on a
bounded sample of the same workload, on rank 0 only.
"""
import argparse
import json
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

from quantization_grouped_gemm_b200 import workloads as wl  # noqa: E402

METRIC = "fused FP8 quant GB/s (% HBM peak); FP8 grouped GEMM TFLOP/s (% peak)"
L2_BYTES = 126 * 1024 * 1024


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                     power=float(parts[3]) if parts[3] not in ("", "[N/A]") else 0.0,
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return dict(sm_mhz=statistics.median(r["sm"] for r in loaded),
                    sm_max_mhz=max(r["smax"] for r in loaded), reasons=sorted(reasons),
                    samples=len(loaded))


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, rows_x, rows_w, n_elem, seed=0):
    """Times the oracle on a bounded sample: rowwise quantisation of rows_x rows
    of X and rows_w rows of W, and n_elem GEMM outputs built from them.
    Returns (seconds for the sample, seconds extrapolated to one full step)."""
    import oracle as orc
    m, k = w.x.shape
    n = w.w.shape[1]
    g = np.random.default_rng(seed)
    xr = np.sort(g.choice(m, rows_x, replace=False))
    wr = np.sort(g.choice(n, rows_w, replace=False))
    xb = wl.bf16_bits(w.x)[xr]
    wb = wl.bf16_bits(w.w.reshape(n, k))[wr]
    t0 = time.perf_counter()
    qa, sa, _ = orc.quant_rowwise(xb)
    t1 = time.perf_counter()
    qb, sb, _ = orc.quant_rowwise(wb)
    t2 = time.perf_counter()
    ri = g.integers(0, rows_x, n_elem)
    ci = g.integers(0, rows_w, n_elem)
    orc.gemm_m_jagged_sample(qa, sa, qb[None], sb[None], np.array([rows_x], np.int32), ri, ci)
    t3 = time.perf_counter()
    full = (t1 - t0) * m / rows_x + (t2 - t1) * n / rows_w + (t3 - t2) * (m * n) / n_elem
    return t3 - t0, full, dict(rows_x=rows_x, rows_w=rows_w, gemm_outputs=n_elem)


def host_cores():
    """CPU cores this process may run on (the oracle itself uses one thread)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = wl.llama3_8b_up_proj()
    m, k = w.x.shape
    n = w.w.shape[1]
    flops = 2.0 * m * n * k
    rows_x, rows_w, n_elem = 128, 128, 1500
    for _ in range(args.warmup):
        oracle_sample(w, rows_x, rows_w, n_elem)
    fulls = []
    t_sample = 0.0
    for i in range(args.steps):
        s, full, desc = oracle_sample(w, rows_x, rows_w, n_elem, seed=i + 1)
        t_sample += s
        fulls.append(full)
    t_step = statistics.mean(fulls)
    value = flops / t_step / 1e12
    sample = (f"per step: oracle rowwise quantisation of {rows_x} X rows and {rows_w} W rows, "
              f"{n_elem} fp64 GEMM outputs; time extrapolated to the full step by rows and "
              f"outputs")
    line = dict(metric=METRIC, value=value, unit="TFLOP/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=t_step * 1e3,
                ms_per_step_kind="extrapolated from the timed sample to one full step",
                sample_ms_per_step=t_sample / args.steps * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f32 quantisation / f64 GEMM",
                data="synthetic", impl="reference", config=config_dict(w),
                cpu_baseline=dict(value=value, unit="TFLOP/s", cores=1,
                                  host_cores=host_cores(), kind="oracle", sample=sample,
                                  extrapolated=True),
                e2e=dict(value=value, unit="TFLOP/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))
    print(json.dumps(line))
    return 0


def config_dict(w, Step=None):
    src = w.x if w.x is not None else w.grad_out
    m, k = src.shape
    d = dict(workload=w.name, M=m, K=k, E=w.num_groups, fmt="e4m3fn", gemm_out="fp32")
    if Step is not None and getattr(Step, "STEP", None):
        d.update(N=(w.grad_out if w.grad_out is not None and Step.BACKWARD else w.w).shape[1],
                 step=Step.STEP, fmt=Step.FMT)
        d.update(workload=w.name + "_mxfp8")
        if Step.__name__ == "MxDualCompareStep":
            d.update(K=None, gemm_out=None)
    elif Step is not None and Step.__name__ == "DualCompareStep":
        d.update(K=None, N=w.grad_out.shape[1], gemm_out=None,
                 step=("grad_out quantised for both backward GEMMs: rowwise + padded transposed "
                       "jagged column-wise as two calls, then as one dual-output call"))
    elif w.grad_out is not None and Step is not None and Step.__name__ == "BackwardDwStep":
        d.update(N=w.grad_out.shape[1],
                 step=("jagged column-wise quant + transpose of grad_out and of X, groups "
                       "at 128-token boundaries + contraction-jagged FP8 grouped GEMM (dW)"))
    else:
        d.update(N=w.w.shape[1],
                 step=("rowwise quant X + rowwise quant W (per expert output channel) + "
                       "token-jagged FP8 grouped GEMM"))
    d["l2"] = ("no explicit flush: each step reads and writes more than the 126 MB L2 "
               "(bf16 inputs plus fp32 output)")
    return d


# ----------------------------------------------------------------------------- GPU arm
class ForwardStep:
    """Token-jagged forward: rowwise X, rowwise W viewed [E*N, K] (one scale per
    expert output channel), FP8 grouped GEMM (fp32 out)."""

    def __init__(self, w):
        import quantization_grouped_gemm_b200 as qgg
        self.qgg = qgg
        self.w = w
        m, k = w.x.shape
        e, n = w.w.shape[0], w.w.shape[1]
        self.m, self.n, self.k, self.e = m, n, k, e
        self.x = w.x.cuda()
        self.wt = w.w.reshape(e * n, k).cuda()
        self.off = torch.from_numpy(w.offsets).cuda()
        self.qa = torch.empty((m, k), dtype=torch.uint8, device="cuda")
        self.sa = torch.empty((m,), dtype=torch.float32, device="cuda")
        self.qb = torch.empty((e * n, k), dtype=torch.uint8, device="cuda")
        self.sb = torch.empty((e * n,), dtype=torch.float32, device="cuda")
        self.out = torch.empty((m, n), dtype=torch.float32, device="cuda")
        rows = int(np.asarray(w.offsets)[-1]) if len(w.offsets) else 0
        self.flops = 2.0 * rows * n * k
        self.names = ["quant_rowwise_x", "quant_rowwise_w", "grouped_gemm"]
        self.launches = 3  # this library's kernels per step
        self.bytes = [m * k * 3 + m * 4, e * n * k * 3 + e * n * 4, None]
        self.host_inputs = [(self.x, w.x), (self.wt, w.w.reshape(e * n, k))]
        self.input_bytes = 2 * (m * k + e * n * k)
        self.result = self.out

    def kernels(self):
        q = self.qgg
        e, n, k = self.e, self.n, self.k
        return [
            lambda: q.fp8_quant_rowwise(self.x, q=self.qa, scales=self.sa),
            lambda: q.fp8_quant_rowwise(self.wt, q=self.qb, scales=self.sb),
            lambda: q.fp8_scaled_grouped_gemm(q.M_JAGGED, self.qa, self.sa,
                                              self.qb.view(e, n, k), self.sb.view(e, n),
                                              self.off, out=self.out),
        ]


class BackwardDwStep:
    """Contraction-jagged weight gradient: jagged column-wise quantisation with
    fused transpose of grad_out [M, N] and of X [M, K], then dW_e = dH_e^T X_e."""

    def __init__(self, w):
        import quantization_grouped_gemm_b200 as qgg
        self.qgg = qgg
        self.w = w
        m, k = w.x.shape
        n = w.grad_out.shape[1]
        e = w.num_groups
        self.m, self.n, self.k, self.e = m, n, k, e
        self.g = w.grad_out.cuda()
        self.x = w.x.cuda()
        self.off = torch.from_numpy(w.offsets).cuda()
        # padded transposed codes: every group starts on a 128-token block of
        # the GEMM's copies and is zero-filled to the next one
        ld = (m + 128 * e + 127) // 128 * 128
        self.qg = torch.empty((n, ld), dtype=torch.uint8, device="cuda")
        self.qx = torch.empty((k, ld), dtype=torch.uint8, device="cuda")
        self.sg = torch.empty((e, n), dtype=torch.float32, device="cuda")
        self.sx = torch.empty((e, k), dtype=torch.float32, device="cuda")
        self.wsg = torch.empty(qgg.colwise_workspace_bytes(m, n, e), dtype=torch.uint8,
                               device="cuda")
        self.wsx = torch.empty(qgg.colwise_workspace_bytes(m, k, e), dtype=torch.uint8,
                               device="cuda")
        self.out = torch.empty((e, n, k), dtype=torch.float32, device="cuda")
        self.flops = 2.0 * m * n * k
        self.names = ["quant_colwise_t_grad_out", "quant_colwise_t_x", "grouped_gemm"]
        self.launches = 3
        self.bytes = [m * n * 3 + e * n * 4 + e * 4, m * k * 3 + e * k * 4 + e * 4, None]
        self.host_inputs = [(self.g, w.grad_out), (self.x, w.x)]
        self.input_bytes = 2 * (m * n + m * k)
        self.result = self.out

    def kernels(self):
        q = self.qgg
        T = q.LAYOUT_TRANSPOSED_PADDED
        return [
            lambda: q.fp8_quant_colwise_jagged(self.g, self.off, T, q=self.qg, scales=self.sg,
                                               workspace=self.wsg),
            lambda: q.fp8_quant_colwise_jagged(self.x, self.off, T, q=self.qx, scales=self.sx,
                                               workspace=self.wsx),
            lambda: q.fp8_scaled_grouped_gemm(q.K_JAGGED_PADDED, self.qg, self.sg, self.qx,
                                              self.sx, self.off, m_total=self.m, out=self.out),
        ]


class DualCompareStep:
    """The backward quantisation of grad_out [M, N] for both backward GEMMs:
    the two separate calls (rowwise codes for the input gradient, padded
    transposed jagged column-wise codes for the weight gradient), then the
    dual-output call that writes both from one read.  The step runs all three
    so that each is timed on the same data; the comparison is the sum of the
    first two against the third."""

    def __init__(self, w):
        import quantization_grouped_gemm_b200 as qgg
        self.qgg = qgg
        self.w = w
        m, n = w.grad_out.shape
        e = w.num_groups
        self.m, self.n, self.e = m, n, e
        self.g = w.grad_out.cuda()
        self.off = torch.from_numpy(w.offsets).cuda()
        ld = (m + 128 * e + 127) // 128 * 128
        self.qr = torch.empty((m, n), dtype=torch.uint8, device="cuda")
        self.sr = torch.empty((m,), dtype=torch.float32, device="cuda")
        self.qc = torch.empty((n, ld), dtype=torch.uint8, device="cuda")
        self.sc = torch.empty((e, n), dtype=torch.float32, device="cuda")
        self.qr2 = torch.empty_like(self.qr)
        self.sr2 = torch.empty_like(self.sr)
        self.qc2 = torch.empty_like(self.qc)
        self.sc2 = torch.empty_like(self.sc)
        self.ws = torch.empty(qgg.colwise_workspace_bytes(m, n, e), dtype=torch.uint8,
                              device="cuda")
        self.wsd = torch.empty(qgg.dual_workspace_bytes(m, n, e), dtype=torch.uint8,
                               device="cuda")
        self.flops = 0.0
        self.names = ["quant_rowwise_grad_out", "quant_colwise_t_grad_out", "quant_dual_grad_out"]
        self.launches = 3
        rows = m * n * 3 + m * 4
        cols = m * n * 3 + e * n * 4 + e * 4
        self.bytes = [rows, cols, m * n * 4 + m * 4 + e * n * 4 + e * 4]
        self.host_inputs = [(self.g, w.grad_out)]
        self.input_bytes = 2 * m * n
        self.result = self.qc2

    def kernels(self):
        q = self.qgg
        T = q.LAYOUT_TRANSPOSED_PADDED
        return [
            lambda: q.fp8_quant_rowwise(self.g, q=self.qr, scales=self.sr),
            lambda: q.fp8_quant_colwise_jagged(self.g, self.off, T, q=self.qc, scales=self.sc,
                                               workspace=self.ws),
            lambda: q.fp8_quant_dual_jagged(self.g, self.off, q_row=self.qr2, scales_row=self.sr2,
                                            q_col=self.qc2, scales_col=self.sc2,
                                            workspace=self.wsd),
        ]


class MxForwardStep:
    """MXFP8 token-jagged forward: MX rowwise quantisation of X and of W viewed
    [E*N, K] (one E8M0 scale per 32 elements along K), block-scaled grouped
    GEMM (fp32 out)."""
    STEP = ("MX rowwise quant X + MX rowwise quant W (32-element blocks along K) + "
            "block-scaled token-jagged MXFP8 grouped GEMM")
    FMT = "mxfp8 (e4m3fn elements, E8M0 scales per 32 elements)"
    BACKWARD = False

    def __init__(self, w):
        import quantization_grouped_gemm_b200 as qgg
        self.qgg = qgg
        self.w = w
        m, k = w.x.shape
        e, n = w.w.shape[0], w.w.shape[1]
        self.m, self.n, self.k, self.e = m, n, k, e
        self.x = w.x.cuda()
        self.wt = w.w.reshape(e * n, k).cuda()
        self.off = torch.from_numpy(w.offsets).cuda()
        gk = qgg.mx_scale_groups(k)
        self.qa = torch.empty((m, k), dtype=torch.uint8, device="cuda")
        self.sa = torch.empty((gk, m), dtype=torch.int32, device="cuda")
        self.qb = torch.empty((e * n, k), dtype=torch.uint8, device="cuda")
        self.sb = torch.empty((gk, e * n), dtype=torch.int32, device="cuda")
        self.out = torch.empty((m, n), dtype=torch.float32, device="cuda")
        rows = int(np.asarray(w.offsets)[-1]) if len(w.offsets) else 0
        self.flops = 2.0 * rows * n * k
        self.names = ["mx_quant_rowwise_x", "mx_quant_rowwise_w", "mx_grouped_gemm"]
        self.launches = 3
        self.bytes = [m * k * 3 + m * k // 32, e * n * k * 3 + e * n * k // 32, None]
        self.host_inputs = [(self.x, w.x), (self.wt, w.w.reshape(e * n, k))]
        self.input_bytes = 2 * (m * k + e * n * k)
        self.result = self.out

    def kernels(self):
        q = self.qgg
        e, n = self.e, self.n
        return [
            lambda: q.fp8_mx_quant_rowwise(self.x, q=self.qa, scales=self.sa),
            lambda: q.fp8_mx_quant_rowwise(self.wt, q=self.qb, scales=self.sb),
            lambda: q.fp8_mx_grouped_gemm(q.M_JAGGED, self.qa, self.sa, self.qb.view(e, n, -1),
                                          self.sb, self.off, out=self.out),
        ]


class MxBackwardDwStep:
    """MXFP8 contraction-jagged weight gradient: MX quantisation of grad_out
    [M, N] and of X [M, K] along each group's tokens (32-token blocks),
    transposed into the padded layout, then the block-scaled
    dW_e = dH_e^T X_e."""
    STEP = ("MX quant + transpose of grad_out and of X along each group's tokens "
            "(32-token blocks, groups at 128-token boundaries) + block-scaled "
            "contraction-jagged MXFP8 grouped GEMM (dW)")
    FMT = "mxfp8 (e4m3fn elements, E8M0 scales per 32 tokens)"
    BACKWARD = True

    def __init__(self, w):
        import quantization_grouped_gemm_b200 as qgg
        self.qgg = qgg
        self.w = w
        m, k = w.x.shape
        n = w.grad_out.shape[1]
        e = w.num_groups
        self.m, self.n, self.k, self.e = m, n, k, e
        self.g = w.grad_out.cuda()
        self.x = w.x.cuda()
        self.off = torch.from_numpy(w.offsets).cuda()
        ld = (m + 128 * e + 127) // 128 * 128
        self.qg = torch.empty((n, ld), dtype=torch.uint8, device="cuda")
        self.qx = torch.empty((k, ld), dtype=torch.uint8, device="cuda")
        self.sg = torch.empty((ld // 128, n), dtype=torch.int32, device="cuda")
        self.sx = torch.empty((ld // 128, k), dtype=torch.int32, device="cuda")
        self.out = torch.empty((e, n, k), dtype=torch.float32, device="cuda")
        self.flops = 2.0 * m * n * k
        self.names = ["mx_quant_colwise_t_grad_out", "mx_quant_colwise_t_x", "mx_grouped_gemm"]
        self.launches = 3
        self.bytes = [m * n * 3 + m * n // 32, m * k * 3 + m * k // 32, None]
        self.host_inputs = [(self.g, w.grad_out), (self.x, w.x)]
        self.input_bytes = 2 * (m * n + m * k)
        self.result = self.out

    def kernels(self):
        q = self.qgg
        return [
            lambda: q.fp8_mx_quant_colwise_padded(self.g, self.off, q=self.qg, scales=self.sg),
            lambda: q.fp8_mx_quant_colwise_padded(self.x, self.off, q=self.qx, scales=self.sx),
            lambda: q.fp8_mx_grouped_gemm(q.K_JAGGED_PADDED, self.qg, self.sg, self.qx, self.sx,
                                          self.off, m_total=self.m, out=self.out),
        ]



class MxDualCompareStep:
    """The MXFP8 backward quantisation of grad_out [M, N] for both backward
    GEMMs: the MX rowwise call and the MX padded column-wise call, then the
    dual-output call that writes both from one read."""
    STEP = ("grad_out quantised in MXFP8 for both backward GEMMs: MX rowwise + MX padded "
            "column-wise as two calls, then as one dual-output call")
    FMT = "mxfp8 (e4m3fn elements, E8M0 scales per 32 elements)"
    BACKWARD = True

    def __init__(self, w):
        import quantization_grouped_gemm_b200 as qgg
        self.qgg = qgg
        self.w = w
        m, n = w.grad_out.shape
        e = w.num_groups
        self.m, self.n, self.e = m, n, e
        self.g = w.grad_out.cuda()
        self.off = torch.from_numpy(w.offsets).cuda()
        ld = (m + 128 * e + 127) // 128 * 128
        gn = qgg.mx_scale_groups(n)
        self.qr = torch.empty((m, n), dtype=torch.uint8, device="cuda")
        self.sr = torch.empty((gn, m), dtype=torch.int32, device="cuda")
        self.qc = torch.empty((n, ld), dtype=torch.uint8, device="cuda")
        self.sc = torch.empty((ld // 128, n), dtype=torch.int32, device="cuda")
        self.qr2 = torch.empty_like(self.qr)
        self.sr2 = torch.empty_like(self.sr)
        self.qc2 = torch.empty_like(self.qc)
        self.sc2 = torch.empty_like(self.sc)
        self.flops = 0.0
        self.names = ["mx_quant_rowwise_grad_out", "mx_quant_colwise_t_grad_out",
                      "mx_quant_dual_grad_out"]
        self.launches = 3
        one = m * n * 3 + m * n // 32
        self.bytes = [one, one, m * n * 4 + 2 * (m * n // 32)]
        self.host_inputs = [(self.g, w.grad_out)]
        self.input_bytes = 2 * m * n
        self.result = self.qc2

    def kernels(self):
        q = self.qgg
        return [
            lambda: q.fp8_mx_quant_rowwise(self.g, q=self.qr, scales=self.sr),
            lambda: q.fp8_mx_quant_colwise_padded(self.g, self.off, q=self.qc, scales=self.sc),
            lambda: q.fp8_mx_quant_dual_padded(self.g, self.off, q_row=self.qr2,
                                               scales_row=self.sr2, q_col=self.qc2,
                                               scales_col=self.sc2),
        ]


WORKLOADS = {
    "llama3_8b_up_proj": (lambda: wl.llama3_8b_up_proj(), ForwardStep),
    "tiny_moe": (lambda: wl.tiny_moe(), ForwardStep),
    "deepseek_moe16b_bwd": (lambda: wl.deepseek_moe_16b_backward(), BackwardDwStep),
    "deepseek_moe16b_bwd_dual": (lambda: wl.deepseek_moe_16b_backward(with_x=False),
                                 DualCompareStep),
    "deepseek_v3_fwd": (lambda: wl.deepseek_v3_local_experts(), ForwardStep),
    "llama4_m8192_zipf": (lambda: wl.llama4_sweep(8192, "zipf"), ForwardStep),
    "llama4_m131072_uniform": (lambda: wl.llama4_sweep(131072, "uniform"), ForwardStep),
    "llama3_8b_up_proj_mxfp8": (lambda: wl.llama3_8b_up_proj(), MxForwardStep),
    "deepseek_moe16b_bwd_mxfp8": (lambda: wl.deepseek_moe_16b_backward(), MxBackwardDwStep),
    "deepseek_moe16b_bwd_dual_mxfp8": (lambda: wl.deepseek_moe_16b_backward(with_x=False),
                                       MxDualCompareStep),
}


def time_steps(st, steps, warmup, flush=None):
    """Runs `warmup` untimed steps, then `steps` timed ones with CUDA events on
    the current stream around every kernel call.  `flush` (optional) runs
    between steps, outside the events.  Returns (total ms of the timed region,
    per-kernel mean ms, events)."""
    ks = st.kernels()
    nk = len(ks)

    def step(ev=None):
        for i, f in enumerate(ks):
            if ev is not None:
                ev[i].record()
            f()
        if ev is not None:
            ev[nk].record()

    for _ in range(max(warmup, 3)):
        if flush is not None:
            flush()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(steps):
        if flush is not None:
            flush()
        step(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    k_ms = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i in range(nk)]
    return t_start.elapsed_time(t_end), k_ms, step


def kernel_table(st, k_ms, pk):
    """Per-kernel figures of a step: GB/s and fraction of the HBM peak for the
    quantisations (algorithmic bytes), TFLOP/s and fraction of the FP8 peak for
    the GEMM."""
    fp8_peak = 2.0 * pk["bf16"]
    kern = {}
    for name, b, t in zip(st.names, st.bytes, k_ms):
        if b:
            gbs = b / (t * 1e-3) / 1e9
            kern[name] = dict(us=t * 1e3, gbs=gbs, frac_hbm=gbs / pk["hbm_gbs"],
                              algorithmic_bytes=b)
        else:
            tf = st.flops / (t * 1e-3) / 1e12
            kern[name] = dict(us=t * 1e3, tflops=tf, frac_fp8=tf / fp8_peak, flops=st.flops)
    q = [(b, t) for b, t in zip(st.bytes, k_ms) if b]
    if q:
        q_gbs = sum(b for b, _ in q) / (sum(t for _, t in q) * 1e-3) / 1e9
        kern.update(quant_gbs=q_gbs, quant_frac_hbm=q_gbs / pk["hbm_gbs"])
    return kern


def extra_workload(name, steps, warmup, pk):
    """Times one more workload in the same run: the step's kernels with L2
    flushed between steps (a 256 MB write outside the timed kernels) when its
    inputs fit in L2.  Returns the per-kernel figures; the step time is the sum
    of the kernels' event times."""
    make, Step = WORKLOADS[name]
    w = make()
    st = Step(w)
    small = st.input_bytes < 2 * L2_BYTES
    flush = None
    if small:
        buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        flush = lambda: buf.fill_(1)  # noqa: E731
    _, k_ms, _ = time_steps(st, steps, warmup, flush)
    step_ms = sum(k_ms)
    d = dict(config=config_dict(w, Step), ms_per_step=step_ms,
             gemm_equivalent_tflops=st.flops / (step_ms * 1e-3) / 1e12 if st.flops else None,
             kernels=kernel_table(st, k_ms, pk), gpu_launches_per_step=st.launches,
             l2=("flushed between steps (256 MB write, not timed)" if small else
                 "no flush: the step reads and writes more than the 126 MB L2"))
    tr = TRAFFIC.get(name)
    if tr:
        d["traffic"] = tr
    del st, w
    torch.cuda.empty_cache()
    return d


# Workloads timed in the default run beside the headline one: the tiny MoE
# layer (launch-bound), the DeepSeek-MoE-16B backward weight-gradient step,
# the dual-output comparison, and the MXFP8 forward and weight-gradient steps.
EXTRA_WORKLOADS = ("tiny_moe", "deepseek_moe16b_bwd", "deepseek_moe16b_bwd_dual",
                   "llama3_8b_up_proj_mxfp8", "deepseek_moe16b_bwd_mxfp8",
                   "deepseek_moe16b_bwd_dual_mxfp8")


def run_gpu(args, world, rank, local):
    pk = peaks()
    make, Step = WORKLOADS[args.workload]
    w = make()
    st = Step(w)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        total_ms, k_ms, step = time_steps(st, args.steps, args.warmup)
    barrier(world)
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    clocks = clk.summary()

    # end to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory to the device, runs the step's calls
    # and copies its result back to pinned host memory.  Two sets of device
    # buffers and three streams (upload, compute, download) let step i + 1's
    # upload run while step i computes and downloads (PCIe is full duplex);
    # events order each buffer's reuse.
    sts = [st, Step(w)]
    pinned = [[(d, h.contiguous().pin_memory()) for d, h in t.host_inputs] for t in sts]
    houts = [torch.empty(t.result.shape, dtype=t.result.dtype).pin_memory() for t in sts]
    e2e_steps = max(3, min(args.steps, 6))
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {key: [torch.cuda.Event() for _ in sts] for key in ("up", "comp", "down")}
    calls = [t.kernels() for t in sts]
    first = [True, True]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(up):
            if not first[b]:
                up.wait_event(ev["comp"][b])  # the step two back has read these inputs
            for d, h in pinned[b]:
                d.copy_(h.view(d.shape), non_blocking=True)
            ev["up"][b].record(up)
        comp.wait_event(ev["up"][b])
        if not first[b]:
            comp.wait_event(ev["down"][b])  # the result two back has been read
        for f in calls[b]:
            f()
        ev["comp"][b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev["comp"][b])
            houts[b].copy_(sts[b].result, non_blocking=True)
            ev["down"][b].record(down)
        first[b] = False

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    for b in range(2):
        comp.wait_event(ev["down"][b])
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    hout = houts[0]
    pinned = pinned[0]

    flops = st.flops
    fp8_peak = 2.0 * pk["bf16"]
    kern = kernel_table(st, k_ms, pk)
    kern.update(hbm_peak_gbs=pk["hbm_gbs"], fp8_peak_tflops=fp8_peak)
    if flops:
        # GEMM-equivalent TFLOP/s of the whole step; the roofline is the GEMM's
        value = flops * world / (ms_step * 1e-3) / 1e12
        unit = "TFLOP/s"
        e2e_value = flops * world / (e2e_ms * 1e-3) / 1e12
        gemm_name = next(nm for nm in st.names if nm.endswith("grouped_gemm"))
        gemm_tflops = kern[gemm_name]["tflops"]
        roof = dict(bound="tensor", achieved=gemm_tflops, peak=fp8_peak, unit="TFLOP/s",
                    frac=gemm_tflops / fp8_peak, traffic=TRAFFIC.get(args.workload),
                    peak_note=(f"{pk['source']} bf16 burst {pk['bf16']} TFLOP/s x 2 "
                               "(nominal fp8:bf16 dense ratio)"))
    else:
        # a quantisation-only step: algorithmic GB/s; the roofline is its last kernel's
        qbytes = sum(st.bytes)
        value = qbytes * world / (ms_step * 1e-3) / 1e9
        unit = "GB/s"
        e2e_value = qbytes * world / (e2e_ms * 1e-3) / 1e9
        last = kern[st.names[-1]]
        roof = dict(bound="hbm", achieved=last["gbs"], peak=pk["hbm_gbs"], unit="GB/s",
                    frac=last["frac_hbm"], traffic=TRAFFIC.get(args.workload),
                    peak_note=f"{pk['source']} HBM copy bandwidth")
    line = dict(
        metric=METRIC, value=value, unit=unit, n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="fp8_e4m3", data="synthetic", config=config_dict(w, Step),
        roofline=roof,
        kernels=kern,
        e2e=dict(value=e2e_value, unit=unit,
                 h2d_bytes_per_step=int(sum(h.numel() * h.element_size() for _, h in pinned)),
                 d2h_bytes_per_step=int(hout.numel() * hout.element_size()), ms_per_step=e2e_ms),
        gpu_launches=st.launches * args.steps,
        clocks=clocks,
    )
    del pinned, hout, houts, sts
    if rank == 0 and world == 1 and Step is ForwardStep and not args.no_cpu_baseline:
        _, full, desc = oracle_sample(w, min(8192, st.m), min(8192, st.e * st.n), 120000)
        cpu_v = flops / full / 1e12
        line["cpu_baseline"] = dict(
            value=cpu_v, unit="TFLOP/s", cores=1, host_cores=host_cores(), kind="oracle",
            extrapolated=True,
            sample=(f"oracle (1 thread) rowwise quantisation of {desc['rows_x']} X rows and "
                    f"{desc['rows_w']} W rows plus {desc['gemm_outputs']} fp64 GEMM outputs, "
                    "extrapolated to one full step"))
    if args.workload == "llama3_8b_up_proj" and not args.no_extra:
        # the other workloads the targets name, timed in the same run (not in
        # `value`, which stays the headline workload's)
        del st, w
        torch.cuda.empty_cache()
        line["configs"] = {name: extra_workload(name, args.steps, args.warmup, pk)
                           for name in EXTRA_WORKLOADS}
    if rank == 0:
        print(json.dumps(line))
    return 0


# DRAM bytes per launch of the grouped GEMM from an ncu capture of the same
# command (dram__bytes_read.sum + dram__bytes_write.sum, profiles/); a workload
# is absent until the current kernel has been captured on it.
TRAFFIC = {
    "llama3_8b_up_proj": 161937152 + 426585088,     # grouped_gemm_2sm_kernel<0>
    "llama3_8b_up_proj_mxfp8": 158574592 + 426209536,  # mx_grouped_gemm_kernel<0, 0>
    "deepseek_moe16b_bwd": 389905920 + 683739136,   # grouped_gemm_kernel<1, 0>, padded operands
    "deepseek_moe16b_bwd_mxfp8": 401601792 + 683939072,  # mx_grouped_gemm_kernel<1, 0>
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama3_8b_up_proj", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (skip the extra workloads of the default run)")
    args = ap.parse_args()
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 alone; no process group is needed
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
    world, rank, local = dist_setup(args)
    try:
        if not torch.cuda.is_available():
            raise RuntimeError("bench.py needs a CUDA device for the GPU arm")
        rc = run_gpu(args, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
