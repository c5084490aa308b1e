#!/usr/bin/env python
"""Benchmark of the ternary BitLinear path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (one JSON line on rank 0): effective packed-weight GB/s of the decode
path at N=1 on the BitNet-b1.58-2B-shaped workload -- 30 decoder layers x 7
BitLinear projections (q 2560x2560, k/v 640x2560, o 2560x2560, gate/up
6912x2560, down 2560x6912), every linear fed one token.  One step:

    quant_act_grouped(90 x 2560 and 30 x 6912 activation rows, one launch)
    gemv_grouped(all 210 layers, one launch)

i.e. per-token absmax int8 quantisation of every layer input and the ternary x
int8 GEMV with fused rescale of every projection; the 521 MB of packed weights
exceed the 126 MB L2, so no flush is needed between steps.  The same JSON line
carries the prefill measurement (7B-shaped layer, 7 projections, N=512 tokens,
tensor-core GEMM, int8 TOPS), a dependent per-layer decode chain (the launch
order a real decoder imposes, captured in a CUDA graph), the end-to-end number
through host buffers, the roofline of the dominant kernel and the CPU oracle
baseline.

--impl reference times the CPU oracle (the reference arm of this project) on a
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from ternary_weight_bit_bitlinear_b200 import _lib, api, inputs  # noqa: E402

METRIC = "ternary BitLinear GB/s (% HBM peak) at N=1; int8 TOPS (% peak) at N=512"
DECODE_CFG = 2
PREFILL_CFG = 3
SWEEP_CFG = 4
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
INT8_PER_BF16 = 2.0          # nominal dense int8 : bf16 tensor throughput (4.5 : 2.25 PFLOP/s)
HBM_NOMINAL_GBS = 8000.0     # B200 HBM3e spec figure (context beside the measured copy peak)

# DRAM bytes (read + write) per launch from one ncu capture of each workload's
# dominant kernel (summaries in profiles/).  They describe the kernel source
# they were taken on, identified by a sha256 prefix: once that file changes
# the figure no longer applies and the bench reports null.
NCU_TRAFFIC = {
    "gemv": {"file": "ternary_weight_bit_bitlinear_b200/csrc/gemv.cuh",
             "sha256": "d0ffe60ca94b9a32", "bytes": 522_076_623 + 2_235_136,
             "profile": "profiles/launches_decode_2b.md"},
    "gemv_quant": {"file": "ternary_weight_bit_bitlinear_b200/csrc/gemv_quant.cuh",
                   "sha256": "7f228f2d4b4f408d", "bytes": 523_122_432 + 2_571_093,
                   "profile": "profiles/gemv_quant_2b_decode_stream.md"},
    "gemm": {"file": ["ternary_weight_bit_bitlinear_b200/csrc/gemm.cuh",
                      "ternary_weight_bit_bitlinear_b200/csrc/gemm_pair.cuh"],
             "sha256": "0eb46b29ec660fd4", "bytes": 62_596_096 + 29_230_080,
             "profile": "profiles/gemm_i8_pair_7b_prefill.md"},
}


def ncu_traffic(kernel):
    import hashlib
    ent = NCU_TRAFFIC.get(kernel)
    if not ent:
        return None
    files = ent["file"] if isinstance(ent["file"], list) else [ent["file"]]
    h = hashlib.sha256()
    for name in files:   # the kernel's sources, hashed in order
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != ent["sha256"]:
        return None
    return ent["bytes"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(PEAKS_FALLBACK)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index, interval_ms=50):
        self.gpu, self.interval, self.proc = gpu_index, interval_ms, None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", str(self.interval)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.out.flush()
        self.out.seek(0)
        sm, smax, reasons = [], None, set()
        for line in self.out.read().splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for name, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.out.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- workloads

def input_proj(p):
    """Projection whose seed names the input of projection p (q,k,v share one
    input, gate/up share one)."""
    return 0 if p < 3 else 3 if p == 3 else 4 if p < 6 else 6


class DecodeWorkload:
    """30 layers x 7 projections of the 2B shape, one token per linear."""

    def __init__(self, device, layers=None, cfg=DECODE_CFG):
        wl = inputs.WORKLOADS[cfg]
        self.shape = wl.model
        self.layers = layers or wl.layers
        h, f = self.shape.hidden, self.shape.ffn
        L = self.layers
        self.weights = []            # [layer][proj] -> (packed, alpha, M, K)
        for l in range(L):
            row = []
            for p, (name, M, K) in enumerate(self.shape.projections()):
                W = inputs.latent_weights(M, K, inputs.weight_seed(cfg, l, p), device=device)
                packed, alpha = api.pack_weights(W)
                del W
                row.append((packed, alpha, M, K))
            self.weights.append(row)
        torch.cuda.synchronize()
        # activation inputs: per layer x_qkv, x_o, x_ffn (K = hidden), x_down (K = ffn)
        self.Xh = torch.empty((3 * L, h), device=device)
        self.Xf = torch.empty((L, f), device=device)
        for l in range(L):
            for j, p in enumerate((0, 3, 4)):
                self.Xh[3 * l + j] = inputs.activations(1, h, inputs.act_seed(cfg, l, p),
                                                        device=device)[0]
            self.Xf[l] = inputs.activations(1, f, inputs.act_seed(cfg, l, 6), device=device)[0]
        self.XQh = torch.empty((3 * L, h), dtype=torch.int8, device=device)
        self.XQf = torch.empty((L, f), dtype=torch.int8, device=device)
        self.AMh = torch.empty(3 * L, device=device)
        self.AMf = torch.empty(L, device=device)
        self.XSh = torch.empty(3 * L, dtype=torch.int32, device=device)
        self.XSf = torch.empty(L, dtype=torch.int32, device=device)
        per_layer = sum(M for _, M, _ in self.shape.projections())
        self.Y = torch.empty(L * per_layer, device=device)   # all outputs, one buffer
        self.ys = []
        off = 0
        entries = []
        for l in range(L):
            ys_l = []
            for p, (packed, alpha, M, K) in enumerate(self.weights[l]):
                y = self.Y[off:off + M].view(1, M)
                off += M
                ys_l.append(y)
                entries.append((packed, alpha, M, K) + self._act(l, p) + (y, None))
            self.ys.append(ys_l)
        self.prob = _lib.make_problems(entries)
        self.n_prob = len(entries)
        # the same 210 linears on fp32 inputs for the fused quantise+GEMV kernel;
        # projections that share an input get the same row view, side by side
        fents = [(packed, alpha, M, K, self._x(l, p), self.ys[l][p], None)
                 for l in range(L) for p, (packed, alpha, M, K) in enumerate(self.weights[l])]
        self.fprob = _lib.make_fused_problems(fents)
        # the same weights in TL2-style storage (5 bits per three weights)
        self.tl2 = [[api.tl2_from_packed(packed, K) for (packed, _, _, K) in row]
                    for row in self.weights]
        tents = [(self.tl2[l][p], alpha, M, K, self._act(l, p)[0], self._act(l, p)[1],
                  self.ys[l][p], None)
                 for l in range(L) for p, (_, alpha, M, K) in enumerate(self.weights[l])]
        self.tl2prob = _lib.make_tl2_problems(tents)
        self.tl2_bytes = sum(t.numel() for row in self.tl2 for t in row)
        self.acts = _lib.make_acts([(self.Xh, self.XQh, self.AMh, self.XSh),
                                    (self.Xf, self.XQf, self.AMf, self.XSf)])
        self.packed_bytes = sum(M * K // 4 for row in self.weights for _, _, M, K in row)
        # algorithmic bytes of the grouped GEMV launch: packed weights, the int8
        # activations and alpha/amax/xsum each layer reads, and its fp32 outputs
        self.alg_bytes = sum(M * K // 4 + K + 12 + 4 * M for (_, _, M, K, *_r) in entries)
        # ... and of the fused launch: packed weights, alpha and fp32 outputs per
        # layer, plus every distinct fp32 input once
        self.alg_bytes_fused = (sum(M * K // 4 + 4 + 4 * M for (_, _, M, K, *_r) in entries)
                                + 4 * (self.Xh.numel() + self.Xf.numel()))

    def fused_table(self, Xh, Xf, Y):
        """The fused problem table over given input buffers (shaped like Xh, Xf)
        and output buffer (shaped like Y); same layer order as `fprob`."""
        ents, off = [], 0
        for l in range(self.layers):
            for p, (packed, alpha, M, K) in enumerate(self.weights[l]):
                if p == 6:
                    x = Xf[l:l + 1]
                else:
                    x = Xh[3 * l + (0 if p < 3 else 1 if p == 3 else 2)].view(1, -1)
                ents.append((packed, alpha, M, K, x, Y[off:off + M].view(1, M), None))
                off += M
        return _lib.make_fused_problems(ents)

    def _x(self, l, p):
        """fp32 row view of the input projection p of layer l reads."""
        if p == 6:
            return self.Xf[l:l + 1]
        r = 3 * l + (0 if p < 3 else 1 if p == 3 else 2)
        return self.Xh[r:r + 1]

    def _act(self, l, p):
        """(xq, amax, xsum) row views of the input projection p of layer l reads."""
        if p == 6:
            return (self.XQf[l:l + 1], self.AMf[l:l + 1], self.XSf[l:l + 1])
        r = 3 * l + (0 if p < 3 else 1 if p == 3 else 2)
        return (self.XQh[r:r + 1], self.AMh[r:r + 1], self.XSh[r:r + 1])

    # each call launches exactly one kernel
    def quant(self, s):
        _lib.check(_lib.bitlinear_quant_act_grouped(self.acts, 2, s), "quant_act_grouped")

    def gemv(self, s):
        _lib.check(_lib.bitlinear_gemv_grouped(self.prob, self.n_prob, 1, s), "gemv_grouped")

    def two_step(self, s):
        """Quantiser launch, then the GEMV launch."""
        self.quant(s)
        self.gemv(s)

    def gemv_tl2(self, s):
        """The GEMV launch over the TL2-style copy of the weights."""
        _lib.check(_lib.bitlinear_gemv_tl2_grouped(self.tl2prob, self.n_prob, 1, s),
                   "gemv_tl2_grouped")

    def step(self, s):
        """The decode path: one fused quantise+GEMV launch over all 210 linears."""
        _lib.check(_lib.bitlinear_gemv_quant_grouped(self.fprob, self.n_prob, 1, s),
                   "gemv_quant_grouped")

    def chain_step_fused(self, s):
        """The dependent per-layer order with the fused kernel: four launches
        per layer (q/k/v, o, gate/up, down)."""
        for l in range(self.layers):
            w = self.weights[l]
            for projs in ((0, 1, 2), (3,), (4, 5), (6,)):
                ents = [(w[p][0], w[p][1], w[p][2], w[p][3], self._x(l, p), self.ys[l][p], None)
                        for p in projs]
                arr = _lib.make_fused_problems(ents)
                _lib.check(_lib.bitlinear_gemv_quant_grouped(arr, len(ents), 1, s),
                           "gemv_quant_grouped")

    def chain_step(self, s):
        """The order a real decoder imposes: per layer, quantise an input, then
        run the projections that read it, one group after the other."""
        h, f = self.shape.hidden, self.shape.ffn
        for l in range(self.layers):
            w = self.weights[l]
            for projs in ((0, 1, 2), (3,), (4, 5), (6,)):
                K = w[projs[0]][3]
                if projs[0] == 6:
                    x, xq, am, xs = self.Xf[l:l + 1], *self._act(l, 6)
                else:
                    r = 3 * l + (0 if projs[0] < 3 else 1 if projs[0] == 3 else 2)
                    x, xq, am, xs = self.Xh[r:r + 1], *self._act(l, projs[0])
                _lib.check(_lib.bitlinear_quant_act(x, 1, K, xq, am, xs, s), "quant_act")
                ents = [(w[p][0], w[p][1], w[p][2], K, xq, am, xs, self.ys[l][p], None)
                        for p in projs]
                arr = _lib.make_problems(ents)
                _lib.check(_lib.bitlinear_gemv_grouped(arr, len(ents), 1, s), "gemv_grouped")


class PrefillWorkload:
    """One 7B-shaped layer, 7 projections, N tokens through the tensor-core GEMM."""

    def __init__(self, device, cfg=PREFILL_CFG):
        wl = inputs.WORKLOADS[cfg]
        self.shape = wl.model
        self.N = wl.tokens[0]
        h, f, N = self.shape.hidden, self.shape.ffn, self.N
        self.weights = []
        for p, (name, M, K) in enumerate(self.shape.projections()):
            W = inputs.latent_weights(M, K, inputs.weight_seed(cfg, 0, p), device=device)
            self.weights.append(api.pack_weights(W) + (M, K))
            del W
        self.X = [inputs.activations(N, h, inputs.act_seed(cfg, 0, p), device=device)
                  for p in (0, 3, 4)]
        self.X.append(inputs.activations(N, f, inputs.act_seed(cfg, 0, 6), device=device))
        self.Q = [api.quant_act(x) for x in self.X]
        self.src = [0, 0, 0, 1, 2, 2, 3]       # which input each projection reads
        self.Y = [torch.empty((N, M), device=device) for (_, _, M, _) in self.weights]
        self.flops = sum(2 * M * N * K for (_, _, M, K) in self.weights)
        self._make_problems()

    def _make_problems(self):
        ents = []
        for p, (packed, alpha, M, K) in enumerate(self.weights):
            xq, am, xs = self.Q[self.src[p]]
            ents.append((packed, alpha, M, K, xq, am, xs, self.Y[p], None))
        self.prob = _lib.make_problems(ents)
        self.acts = _lib.make_acts([(x,) + tuple(q) for x, q in zip(self.X, self.Q)])

    def quant_all(self, s):
        """The four distinct layer inputs in one launch."""
        _lib.check(_lib.bitlinear_quant_act_grouped(self.acts, 4, s), "quant_act_grouped")

    def gemm(self, p, s):
        """One projection alone (for the per-projection breakdown)."""
        packed, alpha, M, K = self.weights[p]
        xq, am, xs = self.Q[self.src[p]]
        _lib.check(_lib.bitlinear_gemm(packed, alpha, M, K, xq, am, xs, self.N, self.Y[p],
                                       None, s), "gemm")

    def gemm_all(self, s):
        """All seven projections in one grouped launch."""
        _lib.check(_lib.bitlinear_gemm_grouped(self.prob, 7, self.N, s), "gemm_grouped")


# ----------------------------------------------------------------------------- timing helpers

def events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def flush_l2(buf):
    buf.zero_()


def measure_prefill(dev, s, peaks, K):
    """7B-shaped layer at N=512 on the tensor cores: the seven projections in
    one grouped GEMM launch, timed with events around it; L2 flushed before
    every timed step.  A per-projection breakdown (one launch each) follows."""
    pre = PrefillWorkload(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(3):
        pre.quant_all(s)
        pre.gemm_all(s)
    torch.cuda.synchronize()
    P = max(10, min(200, K // 50))
    gemm_ms, quant_ms = 0.0, 0.0
    for _ in range(P):
        flush_l2(flush)
        e = events(3)
        e[0].record(s)
        pre.quant_all(s)
        e[1].record(s)
        pre.gemm_all(s)
        e[2].record(s)
        torch.cuda.synchronize()
        quant_ms += e[0].elapsed_time(e[1])
        gemm_ms += e[1].elapsed_time(e[2])
    gemm_ms /= P
    quant_ms /= P
    per_proj = [0.0] * 7
    for _ in range(P):
        flush_l2(flush)
        e = events(8)
        e[0].record(s)
        for p in range(7):
            pre.gemm(p, s)
            e[1 + p].record(s)
        torch.cuda.synchronize()
        for p in range(7):
            per_proj[p] += e[p].elapsed_time(e[1 + p])
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
    tops = pre.flops / (gemm_ms * 1e-3) / 1e12
    prefill = {
        "workload": "7B-shaped layer, 7 projections (q,k,v,o 4096x4096; gate/up 11008x4096; "
                    "down 4096x11008), N=512 tokens, one grouped GEMM launch",
        "value": round(tops, 1), "unit": "int8 TOPS",
        "gemm_ms": round(gemm_ms, 4), "quant_ms": round(quant_ms, 4),
        "step_tops_incl_quant": round(pre.flops / ((gemm_ms + quant_ms) * 1e-3) / 1e12, 1),
        "per_projection_ms_separate_launches": [round(v / P, 4) for v in per_proj],
        "roofline": {"bound": "tensor", "kernel": "gemm_i8_pair (CTA pairs, grouped, 7 layers)",
                     "achieved": round(tops, 1), "peak": round(int8_peak, 1),
                     "unit": "TOPS", "frac": round(tops / int8_peak, 4),
                     "peak_note": "int8 peak = measured bf16 burst x nominal int8:bf16 ratio 2 (%s)"
                                  % peaks["source"],
                     "frac_of_nominal_4500": round(tops / 4500.0, 4),
                     "traffic": ncu_traffic("gemm"),
                     "traffic_source": NCU_TRAFFIC["gemm"]["profile"]},
        "l2": "256 MB buffer written between timed steps (flush)",
    }
    del flush
    return prefill


def measure_crossover(dev, s, reps=30):
    """The 8B-shaped batch sweep on one layer (7 projections, one grouped launch
    per path): the CUDA-core GEMV (N <= 16) against the tensor-core GEMM, with
    L2 flushed before every timed launch.  Locates the GEMV -> GEMM crossover."""
    wl = inputs.WORKLOADS[SWEEP_CFG]
    layers = []
    for p, (name, M, K) in enumerate(wl.model.projections()):
        W = inputs.latent_weights(M, K, inputs.weight_seed(SWEEP_CFG, 0, p), device=dev)
        layers.append(api.pack_weights(W) + (M, K))
        del W
    packed_bytes = sum(M * K // 4 for (_, _, M, K) in layers)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    out = {"workload": "8B-shaped layer (q 4096x4096, k/v 1024x4096, o 4096x4096, gate/up "
                       "14336x4096, down 4096x14336), 7 projections per grouped launch",
           "N": [], "gemv_us": [], "gemm_us": [], "gemv_gbs": [], "gemm_tops": []}
    for N in wl.tokens:
        xs = {}
        for p in (0, 3, 4, 6):
            K = wl.model.ffn if p == 6 else wl.model.hidden
            x = inputs.activations(N, K, inputs.act_seed(SWEEP_CFG, 0, p), device=dev,
                                   outlier_frac=wl.outlier_frac)
            xs[p] = api.quant_act(x)
        src = [0, 0, 0, 3, 4, 4, 6]
        ents = []
        for p, (packed, alpha, M, K) in enumerate(layers):
            xq, am, xsum = xs[src[p]]
            ents.append((packed, alpha, M, K, xq, am, xsum,
                         torch.empty((N, M), device=dev), None))
        prob = _lib.make_problems(ents)
        res = {}
        for path, fn in (("gemv", _lib.bitlinear_gemv_grouped), ("gemm", _lib.bitlinear_gemm_grouped)):
            if path == "gemv" and N > api.GEMV_MAX_TOKENS:
                res[path] = None
                continue
            for _ in range(3):
                _lib.check(fn(prob, len(ents), N, s), path)
            tot = 0.0
            for _ in range(reps):
                flush_l2(flush)
                a, b = events(2)
                a.record(s)
                _lib.check(fn(prob, len(ents), N, s), path)
                b.record(s)
                torch.cuda.synchronize()
                tot += a.elapsed_time(b)
            res[path] = tot / reps
        flops = sum(2 * M * N * K for (_, _, M, K) in layers)
        out["N"].append(N)
        out["gemv_us"].append(None if res["gemv"] is None else round(res["gemv"] * 1e3, 2))
        out["gemm_us"].append(round(res["gemm"] * 1e3, 2))
        out["gemv_gbs"].append(None if res["gemv"] is None else
                               round(packed_bytes / (res["gemv"] * 1e-3) / 1e9, 1))
        out["gemm_tops"].append(round(flops / (res["gemm"] * 1e-3) / 1e12, 1))
    faster = [n for n, v, m in zip(out["N"], out["gemv_us"], out["gemm_us"])
              if v is not None and m < v]
    out["gemm_faster_at_N"] = faster
    out["dispatch"] = "api.matmul: GEMV below N = %d, GEMM from there" % api.GEMM_MIN_TOKENS
    del flush
    return out


# ----------------------------------------------------------------------------- ranks

def rank_max(v, dist=None, device="cpu"):
    """The maximum of v over the ranks of the process group (v without one).
    Every rank must call it at the same point."""
    if dist is None:
        return v
    t = torch.tensor([float(v)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def whole_job_gbs(world, bytes_per_rank_step, ms_per_step):
    """Replicas: every rank streams the same bytes per step; the job's rate is
    all ranks' bytes over the slowest rank's step time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks = load_peaks()
    s = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v):
        return rank_max(v, dist, dev)

    if args.only == "prefill":
        print(json.dumps({"partial_run": "prefill", "prefill": measure_prefill(dev, s, peaks,
                                                                              args.steps)}))
        return
    if args.only == "crossover":
        print(json.dumps({"partial_run": "crossover", "crossover": measure_crossover(dev, s)}))
        return
    dec = DecodeWorkload(dev)
    for _ in range(args.warmup):
        dec.step(s)
        dec.two_step(s)
    torch.cuda.synchronize()

    # ---- headline: K timed decode steps, each one fused quantise+GEMV launch
    # over the 210 linears.  Only the ends carry events: an event between two
    # launches would serialise the programmatic dependent launch that lets one
    # step's CTAs start while the previous step's last CTAs finish.
    K = args.steps
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = events(2)
    t0.record(s)
    for i in range(K):
        dec.step(s)
    t1.record(s)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(t0.elapsed_time(t1))

    # ---- the two-step path (quantiser launch, then GEMV launch), same steps
    barrier()
    torch.cuda.synchronize()
    t0, t1 = events(2)
    t0.record(s)
    for i in range(K):
        dec.two_step(s)
    t1.record(s)
    torch.cuda.synchronize()
    barrier()
    two_ms = max_over_ranks(t0.elapsed_time(t1)) / K

    # ---- per-launch breakdown: a second pass with events around every launch
    # (these launches therefore do not overlap)
    K2 = min(K, 4000)
    ev = events(5 * K2)
    for e in ev:              # create every event before the timed pass
        e.record(s)
    torch.cuda.synchronize()
    for i in range(K2):
        e = ev[5 * i:5 * i + 5]
        e[0].record(s)
        dec.step(s)
        e[1].record(s)
        e[2].record(s)
        dec.quant(s)
        e[3].record(s)
        dec.gemv(s)
        e[4].record(s)
    torch.cuda.synchronize()
    per = {"gemv_quant": 0.0, "quant": 0.0, "gemv": 0.0}
    for i in range(K2):
        e = ev[5 * i:5 * i + 5]
        per["gemv_quant"] += e[0].elapsed_time(e[1])
        per["quant"] += e[2].elapsed_time(e[3])
        per["gemv"] += e[3].elapsed_time(e[4])
    per = {k: v / K2 for k, v in per.items()}
    # ---- the TL2-style storage: the GEMV launch alone, events around each
    K3 = min(K2, 2000)
    for _ in range(3):
        dec.gemv_tl2(s)
    ev = events(2 * K3)
    for e in ev:
        e.record(s)
    torch.cuda.synchronize()
    for i in range(K3):
        ev[2 * i].record(s)
        dec.gemv_tl2(s)
        ev[2 * i + 1].record(s)
    torch.cuda.synchronize()
    per["gemv_tl2"] = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K3)) / K3
    del ev
    ms_per_step = total_ms / K
    gbs = whole_job_gbs(world, dec.packed_bytes, ms_per_step)
    fused_gbs = dec.alg_bytes_fused / (per["gemv_quant"] * 1e-3) / 1e9
    gemv_gbs = dec.alg_bytes / (per["gemv"] * 1e-3) / 1e9
    hbm_peak = peaks["hbm_gbs"]
    if args.only == "decode":
        print(json.dumps({"partial_run": "decode", "value": round(gbs, 1), "unit": "GB/s",
                          "tl2_gemv_ms": round(per["gemv_tl2"], 5),
                          "tl2_equiv_gbs": round(dec.packed_bytes / (per["gemv_tl2"] * 1e-3)
                                                 / 1e9, 1),
                          "two_step_gbs": round(dec.packed_bytes / (two_ms * 1e-3) / 1e9, 1),
                          "kernel_ms": per, "gemv_quant_gbs": round(fused_gbs, 1),
                          "gemv_gbs": round(gemv_gbs, 1), "clocks": clk}))
        return

    # ---- dependent per-layer chains, each in one CUDA graph
    def time_graph(fn):
        try:
            gs = torch.cuda.Stream()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(gs):
                fn(gs)          # warm
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=gs):
                fn(gs)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            reps = max(20, K // 50)
            a, b = events(2)
            a.record(s)
            for _ in range(reps):
                g.replay()
            b.record(s)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / reps
            del g
            return ms
        except Exception as exc:  # noqa: BLE001
            return "failed: %s" % exc

    chain_ms = time_graph(dec.chain_step_fused)
    chain2_ms = time_graph(dec.chain_step)

    # ---- end to end through host buffers: every step copies its fp32 inputs
    # host -> device and its outputs device -> host, around one fused launch.
    # Two sets of device buffers let step i's input copy and step i-1's output
    # copy (one copy stream each) run while step i-1 computes.
    hXh = [torch.empty(dec.Xh.shape, pin_memory=True) for _ in range(2)]
    hXf = [torch.empty(dec.Xf.shape, pin_memory=True) for _ in range(2)]
    hY = [torch.empty(dec.Y.shape, pin_memory=True) for _ in range(2)]
    for b in range(2):
        hXh[b].copy_(dec.Xh)
        hXf[b].copy_(dec.Xf)
    dXh = [dec.Xh, torch.empty_like(dec.Xh)]
    dXf = [dec.Xf, torch.empty_like(dec.Xf)]
    dY = [dec.Y, torch.empty_like(dec.Y)]
    tables = [dec.fused_table(dXh[b], dXf[b], dY[b]) for b in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(50, K // 10)

    def e2e_step(i):
        b = i & 1
        up.wait_event(comp_done[b])          # step i-2 has finished reading dX[b]
        with torch.cuda.stream(up):
            dXh[b].copy_(hXh[b], non_blocking=True)
            dXf[b].copy_(hXf[b], non_blocking=True)
        h2d_done[b].record(up)
        s.wait_event(h2d_done[b])
        s.wait_event(d2h_done[b])            # step i-2's outputs have left dY[b]
        _lib.check(_lib.bitlinear_gemv_quant_grouped(tables[b], dec.n_prob, 1, s),
                   "gemv_quant_grouped")
        comp_done[b].record(s)
        down.wait_event(comp_done[b])
        with torch.cuda.stream(down):
            hY[b].copy_(dY[b], non_blocking=True)
        d2h_done[b].record(down)

    for b in range(2):                       # every event recorded once before use
        comp_done[b].record(s)
        d2h_done[b].record(s)
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    a, z = events(2)
    a.record(up)
    for i in range(e2e_steps):
        e2e_step(i)
    z.record(down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(z) / e2e_steps)
    h2d = (dec.Xh.numel() + dec.Xf.numel()) * 4
    d2h = dec.Y.numel() * 4
    del tables

    prefill = measure_prefill(dev, s, peaks, K)
    crossover = measure_crossover(dev, s)

    # ---- CPU oracle baseline (rank 0, N=1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(dec, budget_s=args.cpu_seconds)

    if rank == 0:
        out = {
            "metric": METRIC,
            "value": round(gbs, 1),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "i8",
            "data": "synthetic (seeded N(0,0.02) latent weights, N(0,1) activations)",
            "config": {
                "workload": "BitNet-b1.58-2B-shaped decode: 30 layers x 7 projections, N=1",
                "layers": dec.layers, "tokens": 1,
                "packed_bytes_per_step": dec.packed_bytes,
                "launches_per_step": 1,
                "l2": "no flush: 521 MB of packed weights per step > 126 MB L2",
                "parallelism": "replicas" if world > 1 else "single GPU",
            },
            "pct_of_measured_hbm": round(100 * gbs / world / hbm_peak, 2),
            "pct_of_nominal_hbm_8000": round(100 * gbs / world / HBM_NOMINAL_GBS, 2),
            "roofline": {
                "bound": "hbm",
                "kernel": "gemv_quant (fused quantise + GEMV, grouped, 210 layers, K=2560 and 6912)",
                "achieved": round(fused_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(fused_gbs / hbm_peak, 4),
                "peak_note": "hbm_gbs %s (burst copy)" % peaks["source"],
                "bytes_per_launch": dec.alg_bytes_fused,
                "avg_launch_ms": round(per["gemv_quant"], 5),
                "timing": "events around each launch, second pass of %d steps" % K2,
                "traffic": ncu_traffic("gemv_quant"),
                "traffic_source": NCU_TRAFFIC["gemv_quant"]["profile"],
            },
            "kernel_ms": {k: round(v, 5) for k, v in per.items()},
            "two_step": {
                "what": "the same step as two launches: grouped quantiser, then grouped GEMV",
                "ms_per_step": round(two_ms, 5),
                "gbs": round(whole_job_gbs(world, dec.packed_bytes, two_ms), 1),
                "gemv_roofline": {
                    "achieved": round(gemv_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(gemv_gbs / hbm_peak, 4), "bytes_per_launch": dec.alg_bytes,
                    "avg_launch_ms": round(per["gemv"], 5),
                    "traffic": ncu_traffic("gemv"),
                    "traffic_source": NCU_TRAFFIC["gemv"]["profile"]},
            },
            "tl2_storage": {
                "what": "the GEMV launch over the same 210 layers stored at 5 bits per three "
                        "weights (TL2-style), int8 activations from the quantiser",
                "bytes_per_launch": dec.tl2_bytes,
                "packed_2bit_bytes": dec.packed_bytes,
                "avg_launch_ms": round(per["gemv_tl2"], 5),
                "tl2_bytes_gbs": round(dec.tl2_bytes / (per["gemv_tl2"] * 1e-3) / 1e9, 1),
                "weights_per_s_as_2bit_gbs": round(dec.packed_bytes / (per["gemv_tl2"] * 1e-3)
                                                   / 1e9, 1),
            },
            "decode_chain": {
                "what": "same 210 linears, per-layer dependent launches, one CUDA graph: fused "
                        "(qkv, o, gate/up, down: 4 launches per layer) and two-step (a quantiser "
                        "launch before each: 8 per layer)",
                "ms_per_step": chain_ms if isinstance(chain_ms, str) else round(chain_ms, 4),
                "gbs": None if isinstance(chain_ms, str) else
                round(dec.packed_bytes / (chain_ms * 1e-3) / 1e9, 1),
                "launches_per_step": 4 * dec.layers,
                "two_step_ms_per_step": chain2_ms if isinstance(chain2_ms, str)
                else round(chain2_ms, 4),
                "two_step_launches_per_step": 8 * dec.layers,
            },
            "prefill": prefill,
            "crossover": crossover,
            "e2e": {"value": round(whole_job_gbs(world, dec.packed_bytes, e2e_ms), 1),
                    "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "per step: pinned host -> device copy of the fp32 inputs, one fused "
                           "launch, device -> host copy of the outputs; two buffer sets and "
                           "two copy streams overlap step i's copies with step i-1's launch"},
            "gpu_launches": K,
            "gpu_launches_other_passes": {"two_step": 2 * K, "breakdown": 3 * K2,
                                          "tl2": K3 + 3},
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(out), flush=True)
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_layer_sample(dec, layer):
    """Host copies of one layer for the oracle: codes (unpacked from the
    oracle's own ternarisation of the seeded latent weights) and activations."""
    import oracle
    h = dec.shape.hidden
    items = []
    for p, (name, M, K) in enumerate(dec.shape.projections()):
        W = inputs.latent_weights(M, K, inputs.weight_seed(DECODE_CFG, layer, p),
                                  device="cuda").cpu().numpy()
        alpha = oracle.absmean(W)
        codes = oracle.ternarize(W, alpha)
        del W
        if K == h:
            r = 3 * layer + (0 if p < 3 else 1 if p == 3 else 2)
            x = dec.Xh[r:r + 1].cpu().numpy()
        else:
            x = dec.Xf[layer:layer + 1].cpu().numpy()
        items.append((codes, alpha, x, M * K // 4))
    return items


def _oracle_time(items):
    import oracle
    t0 = time.perf_counter()
    nbytes = 0
    for codes, alpha, x, pb in items:
        q, amax, _ = oracle.quant_act(x)
        acc = oracle.matmul_i32(codes, q)
        oracle.rescale(acc, alpha, amax)
        nbytes += pb
    return nbytes, time.perf_counter() - t0


def cpu_baseline(dec, budget_s=15.0):
    items = _oracle_layer_sample(dec, 0)
    nbytes, secs, reps = 0, 0.0, 0
    while secs < budget_s or reps == 0:
        b, t = _oracle_time(items)
        nbytes += b
        secs += t
        reps += 1
    return {"value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": "layer 0 of the 2B-shaped stream (7 projections, N=1): quant_act + int32 "
                      "triple-loop matmul + rescale, x%d (%.1f s)" % (reps, secs)}


def run_reference(args, rank, world):
    """CPU oracle on bounded samples of the decode workload (rank 0 only)."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    cfg = inputs.WORKLOADS[DECODE_CFG]
    h = cfg.model.hidden
    projs = cfg.model.projections()
    # one step = rows [r0, r0+R) of one projection of layer 0 (rotating), N=1;
    # R sized so that warmup + steps stay within ~90 s of CPU time
    data = []
    for p, (name, M, K) in enumerate(projs):
        W = inputs.latent_weights(M, K, inputs.weight_seed(DECODE_CFG, 0, p)).numpy()
        alpha = oracle.absmean(W)
        codes = oracle.ternarize(W, alpha)
        x = inputs.activations(1, K, inputs.act_seed(DECODE_CFG, 0, input_proj(p))).numpy()
        data.append((codes, alpha, x))
    t0 = time.perf_counter()
    c, a, x = data[0]
    q, amax, _ = oracle.quant_act(x)
    oracle.matmul_i32(c[:256], q)
    rate = 256 * c.shape[1] / max(time.perf_counter() - t0, 1e-6)     # weights per second
    total = max(1, args.steps + args.warmup)
    per_step_w = max(128 * 2560, int(rate * 90.0 / total))
    nbytes, secs = 0, 0.0
    for i in range(args.warmup + args.steps):
        codes, alpha, x = data[i % 7]
        rows = max(1, min(codes.shape[0], per_step_w // codes.shape[1]))
        r0 = (i * 131) % max(1, codes.shape[0] - rows + 1)
        t = time.perf_counter()
        q, amax, _ = oracle.quant_act(x)
        acc = oracle.matmul_i32(np.ascontiguousarray(codes[r0:r0 + rows]), q)
        oracle.rescale(acc, alpha, amax)
        dt = time.perf_counter() - t
        if i >= args.warmup:
            nbytes += rows * codes.shape[1] // 4
            secs += dt
    v = nbytes / secs / 1e9
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(1e3 * secs / max(1, args.steps), 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
           "config": {"workload": "BitNet-b1.58-2B-shaped decode: 30 layers x 7 projections, N=1",
                      "layers": 30, "tokens": 1},
           "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                            "sample": "per step: a row block of one projection of layer 0 "
                                      "(rotating over the 7), quant_act + matmul + rescale"},
           "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "decode", "prefill", "crossover"], default="all",
                    help="profiling runs: time only one part and print a partial line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", args.gpus if args.gpus == 1 else 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
