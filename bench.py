#!/usr/bin/env python
"""Benchmark of the ternary BitLinear path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (one JSON line on rank 0): effective packed-weight GB/s of the decode
path at N = 1 on the 70B-shaped weight stream -- 80 decoder layers x 7
BitLinear projections (q/o 8192x8192, k/v 1024x8192, gate/up 28672x8192, down
8192x28672), 17.11 GB of 2-bit weights resident in HBM, every linear fed one
token.  One step is the fused quantise + GEMV kernel over all 560 linears from
their fp32 inputs, as four grouped calls of 20 layers (one launch each):
per-token absmax int8 quantisation of every layer input, the ternary x int8
product in int32 and the fused rescale, for every projection.  The weights
exceed the 126 MB L2 more than a hundred times over, so no flush is needed.

The same line carries, on the same configuration: the per-launch roofline of
the fused kernel, a sustained leg of at least two seconds of back-to-back
steps with the SM clock sampled, the dependent per-group order a real decoder
imposes (one CUDA graph), an end-to-end number through host buffers, and
prefill at N = 2048 on one layer (int8 tensor cores).  Then the other
configurations: the 2B-shaped 30-layer stream (fused, two-step, per-group
chain, TL2-style storage), the 7B-shaped prefill at N = 512 (int8 TOPS), the
8B-shaped batch sweep that locates the GEMV -> GEMM crossover, and the single
1024x1024 GEMV as a latency.  Last, the CPU oracle timed on this host's cores
(one thread, and one process per core).

--impl reference times the CPU oracle (the reference arm of this project) on a
bounded sample of the same workload, on rank 0 only.
"""
import argparse
import json
import os
import platform
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
HEADLINE_CFG = 5       # 70B-shaped 80-layer stream: the largest single-GPU configuration
STREAM2B_CFG = 2
PREFILL_CFG = 3
SWEEP_CFG = 4
CROSSOVER_COPIES = 4      # 4 x 54.5 MB of packed weights > 126 MB L2
SINGLE_CFG = 1
HEADLINE_LAUNCH_LAYERS = 20   # layers per grouped call of the headline step (4 calls)
SUSTAINED_S = 2.0
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
INT8_PER_BF16 = 2.0          # nominal dense int8 : bf16 tensor throughput (4.5 : 2.25 PFLOP/s)
HBM_NOMINAL_GBS = 8000.0     # B200 HBM3e spec figure (context beside the measured copy peak)

# DRAM bytes (read + write) per launch from one ncu capture of a kernel on a
# named workload.  Each figure belongs to the kernel source it was taken on,
# identified by a sha256 prefix of its files: once they change, the figure no
# longer applies and the bench reports null.
NCU_TRAFFIC = {
    "gemv": {"file": ["ternary_weight_bit_bitlinear_b200/csrc/gemv.cuh"],
             "sha256": "35fa6f20632f142c", "bytes": 522_951_424 + 7_624_960,
             "source": "ncu dram__bytes_read+write, gemv_tile_kernel<1>, 2B stream launch"},
    "gemm": {"file": ["ternary_weight_bit_bitlinear_b200/csrc/gemm.cuh",
                      "ternary_weight_bit_bitlinear_b200/csrc/gemm_pair.cuh"],
             "sha256": "dc825d0a324fa159", "bytes": 62_600_960 + 31_451_648,
             "source": "ncu dram__bytes_read+write, gemm_i8_pair_kernel<5>, 7B prefill N=512"},
    # captured on a 4-layer launch of the 70B stream (DRAM reads 1.003 x the
    # packed bytes, so traffic grows with the layers), x5 to the headline's
    # 20-layer launch
    "gemv_quant": {"file": ["ternary_weight_bit_bitlinear_b200/csrc/gemv_quant.cuh",
                            "ternary_weight_bit_bitlinear_b200/csrc/gemv.cuh",
                            "ternary_weight_bit_bitlinear_b200/csrc/quant_math.cuh"],
                   "sha256": "0c47ba719c21d7ae", "bytes": (859_360_000 + 4_622_336) * 5,
                   "source": "ncu dram__bytes_read+write, gemv_quant_kernel<1>, 4-layer launch of "
                             "the 70B stream, scaled x5 to the 20-layer launch"},
}


def ncu_traffic(kernel):
    import hashlib
    ent = NCU_TRAFFIC.get(kernel)
    if not ent:
        return None
    h = hashlib.sha256()
    for name in ent["file"]:   # the kernel's sources, hashed in order
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
        sm, smax, power, reasons = [], None, [], set()
        for line in self.out.read().splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.out.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "sm_min_mhz": min(sm) if sm else None,
                "power_w": statistics.median(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- timing helpers

def events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def back_to_back_ms(fn, s, steps):
    """Mean ms of `steps` calls of fn(s) issued back to back, events only at the
    two ends (an event between launches would serialise the programmatic
    dependent launch that lets one launch start while the last one drains)."""
    torch.cuda.synchronize()
    a, b = events(2)
    a.record(s)
    for _ in range(steps):
        fn(s)
    b.record(s)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def time_graph(fn, s, reps):
    """Capture fn(stream) in one CUDA graph; mean ms per replay."""
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


FLUSH_BYTES = 256 * 1024 * 1024


def chain_entry(what, packed_bytes, fused_ms, two_ms, hbm_peak):
    """The dependent decode order, timed per group two ways in a CUDA graph:
    the fused quantise + GEMV launch, and the two-step path (a quantiser launch
    for the group's input, then an int8 GEMV launch).  ms_per_step is the
    faster of the two."""
    def rate(t):
        return None if isinstance(t, str) else round(packed_bytes / (t * 1e-3) / 1e9, 1)

    def frac(t):
        return None if isinstance(t, str) else round(packed_bytes / (t * 1e-3) / 1e9 / hbm_peak,
                                                     4)
    ok = [t for t in (fused_ms, two_ms) if not isinstance(t, str)]
    best = min(ok) if ok else fused_ms
    return {"what": what + ", one CUDA graph per step",
            "path": "two-step per group" if best is two_ms else "fused per group",
            "ms_per_step": rounded(best), "gbs": rate(best), "frac_of_measured_hbm": frac(best),
            "fused_per_group": {"what": "one fused quantise + GEMV launch per group",
                                "ms_per_step": rounded(fused_ms), "gbs": rate(fused_ms)},
            "two_step_per_group": {"what": "a quantiser launch, then an int8 GEMV launch, per "
                                           "group", "ms_per_step": rounded(two_ms),
                                   "gbs": rate(two_ms)}}


def flush_buffer(dev):
    """Two 256 MB halves for flush_l2: the first is written, the second read."""
    return torch.empty(2 * FLUSH_BYTES, dtype=torch.uint8, device=dev)


def device_busy(s, us=100):
    """Queue a ~us microsecond spin on stream s, so that the event recorded
    next and the launch after it reach a busy device: the timed region then
    holds the kernel alone, not the host's work to enqueue it."""
    with torch.cuda.stream(s):
        torch.cuda._sleep(int(us * 2000))


def flush_l2(buf):
    """Evict L2 (126 MB) before a timed launch: write 256 MB, then read another
    256 MB so that the written lines go back to HBM here, outside the timed
    region, and the timed kernel's misses evict clean lines only."""
    buf[:FLUSH_BYTES].zero_()
    buf[FLUSH_BYTES:].view(torch.int64).sum()


def rounded(v, nd=4):
    return v if isinstance(v, str) or v is None else round(v, nd)


# ----------------------------------------------------------------------------- workloads

def input_slot(p):
    """Which of a layer's four inputs projection p reads: q/k/v share the
    attention input (0), o reads the attention output (1), gate/up share the
    FFN input (2), down reads the FFN activation (3)."""
    return 0 if p < 3 else 1 if p == 3 else 2 if p < 6 else 3


def input_proj(p):
    """Projection whose seed names the input of projection p."""
    return (0, 3, 4, 6)[input_slot(p)]


GROUPS = ((0, 1, 2), (3,), (4, 5), (6,))   # the dependent order of one decoder layer


class DecodeStream:
    """All layers of one model shape packed on the device, one token per
    linear: weights, fp32 inputs per layer, output buffers and the problem
    tables of every call the benchmark makes."""

    def __init__(self, device, cfg, launch_layers=None, int8_path=False, tl2=False, layers=None):
        wl = inputs.WORKLOADS[cfg]
        self.cfg, self.shape, self.layers = cfg, wl.model, layers or wl.layers
        self.launch_layers = launch_layers or self.layers
        h, f, L = self.shape.hidden, self.shape.ffn, self.layers
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
        # inputs: per layer x_qkv, x_o, x_ffn (width hidden) and x_down (width ffn)
        self.Xh = torch.empty((3 * L, h), device=device)
        self.Xf = torch.empty((L, f), device=device)
        for l in range(L):
            for j, p in enumerate((0, 3, 4)):
                self.Xh[3 * l + j] = inputs.activations(1, h, inputs.act_seed(cfg, l, p),
                                                        device=device)[0]
            self.Xf[l] = inputs.activations(1, f, inputs.act_seed(cfg, l, 6), device=device)[0]
        per_layer = sum(M for _, M, _ in self.shape.projections())
        self.Y = torch.empty(L * per_layer, device=device)   # all outputs, one buffer
        self.ys, off = [], 0
        for l in range(L):
            ys_l = []
            for p, (_, _, M, _) in enumerate(self.weights[l]):
                ys_l.append(self.Y[off:off + M].view(1, M))
                off += M
            self.ys.append(ys_l)
        self.n_prob = 7 * L
        self.calls = self.fused_calls(self.Xh, self.Xf, self.Y)
        self.packed_bytes = sum(M * K // 4 for row in self.weights for _, _, M, K in row)
        # algorithmic bytes of the fused launches: packed weights, alpha and fp32
        # outputs per layer, plus every distinct fp32 input once
        self.alg_bytes_fused = (sum(M * K // 4 + 4 + 4 * M for row in self.weights
                                    for (_, _, M, K) in row)
                                + 4 * (self.Xh.numel() + self.Xf.numel()))
        self.call_bytes = []
        for c0 in range(0, L, self.launch_layers):
            c1 = min(L, c0 + self.launch_layers)
            b = sum(M * K // 4 + 4 + 4 * M for l in range(c0, c1)
                    for (_, _, M, K) in self.weights[l])
            self.call_bytes.append(b + 4 * (3 * h + f) * (c1 - c0))
        if int8_path:
            self._make_int8_path(device)
        if tl2:
            self._make_tl2(device)

    def _x(self, l, p, Xh=None, Xf=None):
        """fp32 row view of the input projection p of layer l reads."""
        Xh = self.Xh if Xh is None else Xh
        Xf = self.Xf if Xf is None else Xf
        slot = input_slot(p)
        if slot == 3:
            return Xf[l:l + 1]
        return Xh[3 * l + slot:3 * l + slot + 1]

    def fused_calls(self, Xh, Xf, Y):
        """Problem tables of the fused step over the given input / output
        buffers: one table per `launch_layers` layers, layers in order,
        projections that share an input side by side."""
        calls = []
        per_layer = sum(M for _, M, _ in self.shape.projections())
        for c0 in range(0, self.layers, self.launch_layers):
            c1 = min(self.layers, c0 + self.launch_layers)
            ents = []
            for l in range(c0, c1):
                off = l * per_layer
                for p, (packed, alpha, M, K) in enumerate(self.weights[l]):
                    ents.append((packed, alpha, M, K, self._x(l, p, Xh, Xf),
                                 Y[off:off + M].view(1, M), None))
                    off += M
            calls.append((_lib.make_fused_problems(ents), len(ents)))
        return calls

    def step(self, s, calls=None):
        """The decode path: the fused quantise + GEMV kernel over every linear."""
        for arr, n in (calls or self.calls):
            _lib.check(_lib.bitlinear_gemv_quant_grouped(arr, n, 1, s), "gemv_quant_grouped")

    def chain_tables(self):
        tabs = []
        for l in range(self.layers):
            w = self.weights[l]
            for projs in GROUPS:
                ents = [(w[p][0], w[p][1], w[p][2], w[p][3], self._x(l, p), self.ys[l][p], None)
                        for p in projs]
                tabs.append((_lib.make_fused_problems(ents), len(ents)))
        return tabs

    def chain_two_tables(self):
        """The dependent order as the two-step path per group: one quantiser
        launch for the group's input, then one int8 GEMV launch over its
        layers."""
        if not hasattr(self, "XQh"):
            self._make_int8_buffers(self.ys[0][0].device)
        tabs = []
        for l in range(self.layers):
            w = self.weights[l]
            for projs in GROUPS:
                xq, am, xs = self._act(l, projs[0])
                acts = _lib.make_acts([(self._x(l, projs[0]), xq, am, xs)])
                ents = [(w[p][0], w[p][1], w[p][2], w[p][3]) + self._act(l, p) +
                        (self.ys[l][p], None) for p in projs]
                tabs.append((acts, _lib.make_problems(ents), len(ents)))
        return tabs

    def chain_two_step(self, s, tabs):
        for acts, prob, n in tabs:
            _lib.check(_lib.bitlinear_quant_act_grouped(acts, 1, s), "quant_act_grouped")
            _lib.check(_lib.bitlinear_gemv_grouped(prob, n, 1, s), "gemv_grouped")

    def chain_step(self, s, tabs):
        """The dependent order of a real decoder: per layer q/k/v, then o, then
        gate/up, then down, each one launch after the other."""
        for arr, n in tabs:
            _lib.check(_lib.bitlinear_gemv_quant_grouped(arr, n, 1, s), "gemv_quant_grouped")

    # ---- the two-step path (quantiser launch, then GEMV launch) and TL2 storage

    def _make_int8_buffers(self, device):
        """int8 copies, amax and sum of q of every distinct input."""
        L, h, f = self.layers, self.shape.hidden, self.shape.ffn
        self.XQh = torch.empty((3 * L, h), dtype=torch.int8, device=device)
        self.XQf = torch.empty((L, f), dtype=torch.int8, device=device)
        self.AMh = torch.empty(3 * L, device=device)
        self.AMf = torch.empty(L, device=device)
        self.XSh = torch.empty(3 * L, dtype=torch.int32, device=device)
        self.XSf = torch.empty(L, dtype=torch.int32, device=device)

    def _make_int8_path(self, device):
        self._make_int8_buffers(device)
        L = self.layers
        ents = []
        for l in range(L):
            for p, (packed, alpha, M, K) in enumerate(self.weights[l]):
                ents.append((packed, alpha, M, K) + self._act(l, p) + (self.ys[l][p], None))
        self.prob = _lib.make_problems(ents)
        self.acts = _lib.make_acts([(self.Xh, self.XQh, self.AMh, self.XSh),
                                    (self.Xf, self.XQf, self.AMf, self.XSf)])
        self.alg_bytes_gemv = sum(M * K // 4 + K + 12 + 4 * M for (_, _, M, K, *_r) in ents)

    def _act(self, l, p):
        slot = input_slot(p)
        if slot == 3:
            return (self.XQf[l:l + 1], self.AMf[l:l + 1], self.XSf[l:l + 1])
        r = 3 * l + slot
        return (self.XQh[r:r + 1], self.AMh[r:r + 1], self.XSh[r:r + 1])

    def quant(self, s):
        _lib.check(_lib.bitlinear_quant_act_grouped(self.acts, 2, s), "quant_act_grouped")

    def gemv(self, s):
        _lib.check(_lib.bitlinear_gemv_grouped(self.prob, self.n_prob, 1, s), "gemv_grouped")

    def two_step(self, s):
        self.quant(s)
        self.gemv(s)

    def _make_tl2(self, device):
        self.tl2 = [[api.tl2_from_packed(packed, K) for (packed, _, _, K) in row]
                    for row in self.weights]
        tents = [(self.tl2[l][p], alpha, M, K, self._act(l, p)[0], self._act(l, p)[1],
                  self.ys[l][p], None)
                 for l in range(self.layers) for p, (_, alpha, M, K) in enumerate(self.weights[l])]
        self.tl2prob = _lib.make_tl2_problems(tents)
        self.tl2_bytes = sum(t.numel() for row in self.tl2 for t in row)

    def gemv_tl2(self, s):
        _lib.check(_lib.bitlinear_gemv_tl2_grouped(self.tl2prob, self.n_prob, 1, s),
                   "gemv_tl2_grouped")


class PrefillLayer:
    """One layer of a model shape, 7 projections, N tokens through the
    tensor-core GEMM (the four distinct inputs quantised in one launch)."""

    def __init__(self, device, cfg, N):
        wl = inputs.WORKLOADS[cfg]
        self.shape, self.N = wl.model, N
        h, f = self.shape.hidden, self.shape.ffn
        self.weights = []
        for p, (name, M, K) in enumerate(self.shape.projections()):
            W = inputs.latent_weights(M, K, inputs.weight_seed(cfg, 0, p), device=device)
            self.weights.append(api.pack_weights(W) + (M, K))
            del W
        self.X = [inputs.activations(N, h, inputs.act_seed(cfg, 0, p), device=device)
                  for p in (0, 3, 4)]
        self.X.append(inputs.activations(N, f, inputs.act_seed(cfg, 0, 6), device=device))
        self.Q = [api.quant_act(x) for x in self.X]
        self.Y = [torch.empty((N, M), device=device) for (_, _, M, _) in self.weights]
        self.flops = sum(2 * M * N * K for (_, _, M, K) in self.weights)
        ents = []
        for p, (packed, alpha, M, K) in enumerate(self.weights):
            xq, am, xs = self.Q[input_slot(p)]
            ents.append((packed, alpha, M, K, xq, am, xs, self.Y[p], None))
        self.prob = _lib.make_problems(ents)
        self.acts = _lib.make_acts([(x,) + tuple(q) for x, q in zip(self.X, self.Q)])

    def quant_all(self, s):
        _lib.check(_lib.bitlinear_quant_act_grouped(self.acts, 4, s), "quant_act_grouped")

    def gemm(self, p, s):
        packed, alpha, M, K = self.weights[p]
        xq, am, xs = self.Q[input_slot(p)]
        _lib.check(_lib.bitlinear_gemm(packed, alpha, M, K, xq, am, xs, self.N, self.Y[p],
                                       None, s), "gemm")

    def gemm_all(self, s):
        _lib.check(_lib.bitlinear_gemm_grouped(self.prob, 7, self.N, s), "gemm_grouped")


# ----------------------------------------------------------------------------- measurements

def soft(fn, *a, **k):
    """Run one secondary measurement; a failure becomes a string in the JSON
    line instead of losing the whole line."""
    try:
        return fn(*a, **k)
    except Exception as exc:  # noqa: BLE001
        torch.cuda.synchronize()
        return "failed: %s" % exc


def measure_prefill(dev, s, peaks, cfg, N, reps, breakdown=True):
    """One layer at N tokens on the tensor cores: the seven projections in one
    grouped GEMM launch, timed with events around it, L2 flushed before every
    timed step (the quantiser launch timed separately)."""
    pre = PrefillLayer(dev, cfg, N)
    flush = flush_buffer(dev)
    for _ in range(3):
        pre.quant_all(s)
        pre.gemm_all(s)
    torch.cuda.synchronize()
    gemm_ms, quant_ms = 0.0, 0.0
    for _ in range(reps):
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
    gemm_ms /= reps
    quant_ms /= reps
    # the step as a user launches it: quantiser then GEMM back to back, one
    # interval (the GEMM's set-up may then overlap the quantiser's tail)
    step_ms = 0.0
    for _ in range(reps):
        flush_l2(flush)
        e = events(2)
        e[0].record(s)
        pre.quant_all(s)
        pre.gemm_all(s)
        e[1].record(s)
        torch.cuda.synchronize()
        step_ms += e[0].elapsed_time(e[1])
    step_ms /= reps
    out = {}
    if breakdown:
        per_proj = [0.0] * 7
        for _ in range(reps):
            flush_l2(flush)
            e = events(8)
            e[0].record(s)
            for p in range(7):
                pre.gemm(p, s)
                e[1 + p].record(s)
            torch.cuda.synchronize()
            for p in range(7):
                per_proj[p] += e[p].elapsed_time(e[1 + p])
        out["per_projection_ms_separate_launches"] = [round(v / reps, 4) for v in per_proj]
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
    tops = pre.flops / (gemm_ms * 1e-3) / 1e12
    sh = pre.shape
    kernel = "gemm_i8_pair_kernel<5> (CTA pairs)" if N > 128 else "gemm_i8_tcgen05_kernel"
    out.update({
        "workload": "%s-shaped layer, 7 projections (q %dx%d, k/v %dx%d, o %dx%d, gate/up %dx%d, "
                    "down %dx%d), N=%d tokens, one grouped GEMM launch"
                    % (sh.name, sh.hidden, sh.hidden, sh.kv_dim, sh.hidden, sh.hidden, sh.hidden,
                       sh.ffn, sh.hidden, sh.hidden, sh.ffn, N),
        "value": round(tops, 1), "unit": "int8 TOPS",
        "gemm_ms": round(gemm_ms, 4), "quant_ms": round(quant_ms, 4),
        "step_ms": round(step_ms, 4),
        "step_tops_incl_quant": round(pre.flops / (step_ms * 1e-3) / 1e12, 1),
        "step_note": "quantiser + GEMM launched back to back, one event interval per step; "
                     "quant_ms and gemm_ms time each launch alone",
        "ops_per_launch": pre.flops,
        "roofline": {"bound": "tensor", "kernel": kernel + ", grouped, 7 layers",
                     "achieved": round(tops, 1), "peak": round(int8_peak, 1),
                     "unit": "TOPS", "frac": round(tops / int8_peak, 4),
                     "peak_note": "int8 peak = bf16 burst peak (%s) x nominal int8:bf16 ratio 2"
                                  % peaks["source"],
                     "frac_of_nominal_4500": round(tops / 4500.0, 4)},
        "l2": "flush before every timed step: 256 MB written, then another 256 MB read "
              "(the written lines go back to HBM before the timed launch)",
    })
    if cfg == PREFILL_CFG:
        out["roofline"]["traffic"] = ncu_traffic("gemm")
        out["roofline"]["traffic_source"] = NCU_TRAFFIC["gemm"]["source"]
    del flush, pre
    torch.cuda.empty_cache()
    return out


def measure_crossover(dev, s, reps=30):
    """The 8B-shaped batch sweep on one layer (7 projections, one grouped launch
    per path): the CUDA-core GEMV (N <= 16) against the tensor-core GEMM.
    Timed launches rotate over CROSSOVER_COPIES copies of the layer's packed
    weights (218 MB > the 126 MB L2), so every launch reads its weights from
    HBM, as a decoder reading layer after layer does, and nothing is written
    to evict L2.  Locates the GEMV -> GEMM crossover."""
    wl = inputs.WORKLOADS[SWEEP_CFG]
    layers = []
    for p, (name, M, K) in enumerate(wl.model.projections()):
        W = inputs.latent_weights(M, K, inputs.weight_seed(SWEEP_CFG, 0, p), device=dev)
        layers.append(api.pack_weights(W) + (M, K))
        del W
    packed_bytes = sum(M * K // 4 for (_, _, M, K) in layers)
    copies = [layers] + [[(packed.clone(), alpha, M, K) for (packed, alpha, M, K) in layers]
                         for _ in range(CROSSOVER_COPIES - 1)]
    out = {"workload": "8B-shaped layer (q 4096x4096, k/v 1024x4096, o 4096x4096, gate/up "
                       "14336x4096, down 4096x14336), 7 projections per grouped launch",
           "N": [], "gemv_us": [], "gemv_quant_us": [], "gemm_us": [], "gemv_gbs": [],
           "gemm_gbs": [], "gemm_tops": [],
           "paths": "gemv: CUDA cores on int8 activations; gemv_quant: CUDA cores from fp32 "
                    "activations, quantiser fused; gemm: tensor cores on int8 activations "
                    "(A in tensor memory up to 32 tokens)"}
    for N in wl.tokens:
        xs, xf = {}, {}
        for p in (0, 3, 4, 6):
            K = wl.model.ffn if p == 6 else wl.model.hidden
            x = inputs.activations(N, K, inputs.act_seed(SWEEP_CFG, 0, p), device=dev,
                                   outlier_frac=wl.outlier_frac)
            xf[p] = x
            xs[p] = api.quant_act(x)
        ys = [torch.empty((N, M), device=dev) for (_, _, M, _) in layers]
        probs, fprobs = [], []
        for cp in copies:
            ents = [(packed, alpha, M, K) + tuple(xs[input_proj(p)]) + (ys[p], None)
                    for p, (packed, alpha, M, K) in enumerate(cp)]
            probs.append(_lib.make_problems(ents))
            fents = [(packed, alpha, M, K, xf[input_proj(p)], ys[p], None)
                     for p, (packed, alpha, M, K) in enumerate(cp)]
            fprobs.append(_lib.make_fused_problems(fents))
        nproj = len(layers)
        res = {}
        for path, fn in (("gemv", lambda c: _lib.bitlinear_gemv_grouped(probs[c], nproj, N, s)),
                         ("gemv_quant",
                          lambda c: _lib.bitlinear_gemv_quant_grouped(fprobs[c], nproj, N, s)),
                         ("gemm", lambda c: _lib.bitlinear_gemm_grouped(probs[c], nproj, N, s))):
            if path != "gemm" and N > api.GEMV_MAX_TOKENS:
                res[path] = None
                continue
            if path == "gemv_quant" and not all(api.gemv_quant_fits(N, K)
                                                for (_, _, _, K) in layers):
                res[path] = None      # the fused kernel's int8 copy of x does not fit
                continue
            for c in range(CROSSOVER_COPIES):
                _lib.check(fn(c), path)
            torch.cuda.synchronize()
            tot = 0.0
            for i in range(reps):
                a, b = events(2)
                device_busy(s)
                a.record(s)
                _lib.check(fn(i % CROSSOVER_COPIES), path)
                b.record(s)
                torch.cuda.synchronize()
                tot += a.elapsed_time(b)
            res[path] = tot / reps
        flops = sum(2 * M * N * K for (_, _, M, K) in layers)
        out["N"].append(N)
        out["gemv_us"].append(None if res["gemv"] is None else round(res["gemv"] * 1e3, 2))
        out["gemv_quant_us"].append(None if res["gemv_quant"] is None else
                                    round(res["gemv_quant"] * 1e3, 2))
        out["gemm_us"].append(round(res["gemm"] * 1e3, 2))
        out["gemv_gbs"].append(None if res["gemv"] is None else
                               round(packed_bytes / (res["gemv"] * 1e-3) / 1e9, 1))
        out["gemm_gbs"].append(round(packed_bytes / (res["gemm"] * 1e-3) / 1e9, 1))
        out["gemm_tops"].append(round(flops / (res["gemm"] * 1e-3) / 1e12, 1))
    faster = [n for n, v, m in zip(out["N"], out["gemv_us"], out["gemm_us"])
              if v is not None and m < v]
    out["gemm_faster_at_N"] = faster
    out["packed_bytes"] = packed_bytes
    out["dispatch"] = "api.matmul: GEMV below N = %d, GEMM from there" % api.GEMM_MIN_TOKENS
    out["l2"] = ("no flush: %d copies of the layer (%.0f MB) visited in turn, so each timed "
                 "launch reads weights that left L2 three launches earlier"
                 % (CROSSOVER_COPIES, CROSSOVER_COPIES * packed_bytes / 1e6))
    del copies
    torch.cuda.empty_cache()
    return out


def measure_single(dev, s, reps=2000):
    """The single 1024x1024 decode GEMV (N = 1, 4 outlier channels) through the
    fused kernel, as a latency: 1024 packed copies (256 MB, twice the L2)
    visited in turn, so every launch reads its weights from HBM."""
    wl = inputs.WORKLOADS[SINGLE_CFG]
    M, K = wl.single
    W = inputs.latent_weights(M, K, inputs.weight_seed(SINGLE_CFG, 0, 0), device=dev)
    packed, alpha = api.pack_weights(W)
    del W
    copies = 1024
    P = packed.repeat(copies, 1).view(copies, M, packed.shape[1])
    x = inputs.activations(1, K, inputs.act_seed(SINGLE_CFG, 0, 0), device=dev,
                           outlier_count=wl.outlier_count)
    y = torch.empty((1, M), device=dev)
    tabs = [_lib.make_fused_problems([(P[i], alpha, M, K, x, y, None)]) for i in range(copies)]

    def launch(i, st):
        _lib.check(_lib.bitlinear_gemv_quant_grouped(tabs[i % copies], 1, 1, st), "single")

    for i in range(copies):
        launch(i, s)
    torch.cuda.synchronize()
    ev = events(2 * reps)
    for e in ev:
        e.record(s)
    torch.cuda.synchronize()
    for i in range(reps):
        ev[2 * i].record(s)
        launch(i, s)
        ev[2 * i + 1].record(s)
    torch.cuda.synchronize()
    lat = sorted(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(reps))
    b2b = back_to_back_ms(lambda st: [launch(i, st) for i in range(copies)], s, 2) / copies
    nbytes = M * K // 4
    out = {"workload": "single 1024x1024 decode GEMV, N=1, fused quantise + GEMV, "
                       "1024 weight copies visited in turn (256 MB > L2)",
           "latency_us_median": round(1e3 * lat[len(lat) // 2], 2),
           "latency_us_p10": round(1e3 * lat[len(lat) // 10], 2),
           "back_to_back_us_per_launch": round(1e3 * b2b, 2),
           "packed_bytes": nbytes,
           "gbs_at_median_latency": round(nbytes / (lat[len(lat) // 2] * 1e-3) / 1e9, 1)}
    del P, tabs
    torch.cuda.empty_cache()
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
    hbm_peak = peaks["hbm_gbs"]
    s = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v):
        return rank_max(v, dist, dev)

    if args.only in ("headline", "chain"):
        # profiling runs: the fused decode step (or the per-group chain) on the
        # first --layers layers of the 70B-shaped stream, nothing else
        dec = DecodeStream(dev, HEADLINE_CFG, launch_layers=HEADLINE_LAUNCH_LAYERS,
                           layers=args.layers)
        if args.only == "headline":
            for _ in range(args.warmup):
                dec.step(s)
            ms = back_to_back_ms(dec.step, s, args.steps)
            print(json.dumps({"partial_run": "headline", "layers": dec.layers,
                              "ms_per_step": round(ms, 5),
                              "gbs": round(dec.packed_bytes / (ms * 1e-3) / 1e9, 1)}))
        else:
            tabs = dec.chain_tables()
            for _ in range(args.warmup):
                dec.chain_step(s, tabs)
            ms = back_to_back_ms(lambda st: dec.chain_step(st, tabs), s, args.steps)
            ttabs = dec.chain_two_tables()
            for _ in range(args.warmup):
                dec.chain_two_step(s, ttabs)
            tms = back_to_back_ms(lambda st: dec.chain_two_step(st, ttabs), s, args.steps)
            print(json.dumps({"partial_run": "chain", "layers": dec.layers,
                              "fused_per_group_ms": round(ms, 5),
                              "fused_per_group_gbs":
                                  round(dec.packed_bytes / (ms * 1e-3) / 1e9, 1),
                              "two_step_per_group_ms": round(tms, 5),
                              "two_step_per_group_gbs":
                                  round(dec.packed_bytes / (tms * 1e-3) / 1e9, 1)}))
        return
    if args.only == "prefill":
        print(json.dumps({"partial_run": "prefill",
                          "prefill": measure_prefill(dev, s, peaks, PREFILL_CFG, 512,
                                                     args.steps)}))
        return
    if args.only == "prefill70":
        print(json.dumps({"partial_run": "prefill70",
                          "prefill_70b": measure_prefill(dev, s, peaks, HEADLINE_CFG, 2048,
                                                         args.steps, breakdown=False)}))
        return
    if args.only == "stream2b":
        print(json.dumps({"partial_run": "stream2b",
                          "stream_2b": measure_stream_2b(dev, s, args.steps, hbm_peak)}))
        return
    if args.only == "crossover":
        print(json.dumps({"partial_run": "crossover", "crossover": measure_crossover(dev, s)}))
        return

    # ================================================================ headline
    dec = DecodeStream(dev, HEADLINE_CFG, launch_layers=HEADLINE_LAUNCH_LAYERS)
    for _ in range(args.warmup):
        dec.step(s)
    torch.cuda.synchronize()

    K = args.steps
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = events(2)
    t0.record(s)
    for _ in range(K):
        dec.step(s)
    t1.record(s)
    torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1))
    ms_per_step = total_ms / K

    # sustained: back-to-back steps for at least SUSTAINED_S seconds, clocks sampled
    sus_steps = max(K, int(SUSTAINED_S / max(ms_per_step * 1e-3, 1e-6)) + 1)
    sclocks = ClockSampler(local_rank, interval_ms=20)
    sclocks.start()
    sus_ms = max_over_ranks(back_to_back_ms(dec.step, s, sus_steps))
    sclk = sclocks.stop()
    clk = clocks.stop()

    # per-launch timing of the fused kernel: events around each grouped call
    K2 = max(5, min(K, 200))
    ncalls = len(dec.calls)
    ev = events(2 * ncalls * K2)
    for e in ev:
        e.record(s)
    torch.cuda.synchronize()
    for i in range(K2):
        for c, (arr, n) in enumerate(dec.calls):
            ev[2 * (i * ncalls + c)].record(s)
            _lib.check(_lib.bitlinear_gemv_quant_grouped(arr, n, 1, s), "gemv_quant_grouped")
            ev[2 * (i * ncalls + c) + 1].record(s)
    torch.cuda.synchronize()
    launch_ms = sum(ev[2 * j].elapsed_time(ev[2 * j + 1]) for j in range(ncalls * K2)) / (
        ncalls * K2)
    del ev
    fused_gbs = dec.alg_bytes_fused / (launch_ms * ncalls * 1e-3) / 1e9

    # dependent per-group order, one CUDA graph
    tabs = dec.chain_tables()
    chain_fused_ms = time_graph(lambda st: dec.chain_step(st, tabs), s, max(10, K // 2))
    ttabs = dec.chain_two_tables()
    chain_two_ms = time_graph(lambda st: dec.chain_two_step(st, ttabs), s, max(10, K // 2))
    del ttabs
    del tabs

    # end to end through host buffers: every step copies its fp32 inputs
    # host -> device and its outputs device -> host around the fused launches.
    # Two sets of device buffers let step i's input copy and step i-1's output
    # copy (one copy stream each) run while step i-1 computes.
    e2e_ms, h2d, d2h = measure_e2e(dec, s, max(30, K))
    e2e_ms = max_over_ranks(e2e_ms)
    gbs = whole_job_gbs(world, dec.packed_bytes, ms_per_step)
    headline = {
        "packed_bytes": dec.packed_bytes, "alg_bytes": dec.alg_bytes_fused,
        "ncalls": ncalls, "launch_ms": launch_ms, "fused_gbs": fused_gbs,
        "sus_steps": sus_steps, "sus_ms": sus_ms, "sclk": sclk, "clk": clk,
        "chain_fused_ms": chain_fused_ms, "chain_two_ms": chain_two_ms,
        "call_bytes": dec.call_bytes,
    }
    del dec
    torch.cuda.empty_cache()

    prefill_70b = soft(measure_prefill, dev, s, peaks, HEADLINE_CFG, 2048, 10, breakdown=False)
    s2 = soft(measure_stream_2b, dev, s, K, hbm_peak)
    prefill = soft(measure_prefill, dev, s, peaks, PREFILL_CFG, 512, max(10, min(200, K // 50)))
    crossover = soft(measure_crossover, dev, s)
    single = soft(measure_single, dev, s)

    # ---- CPU oracle baseline (rank 0, N=1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = soft(cpu_baseline, budget_s=args.cpu_seconds)

    if rank == 0:
        emit(args, world, peaks, headline, ms_per_step, gbs, K, K2, e2e_ms, h2d, d2h,
             prefill_70b, s2, prefill, crossover, single, cpu)
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def measure_stream_2b(dev, s, K, hbm_peak):
    """The 2B-shaped 30-layer stream: fused step, two-step path, per-launch
    rooflines, the dependent per-group chain and the TL2-style storage."""
    d2 = DecodeStream(dev, STREAM2B_CFG, int8_path=True, tl2=True)
    for _ in range(3):
        d2.step(s)
        d2.two_step(s)
        d2.gemv_tl2(s)
    torch.cuda.synchronize()
    k2 = max(K, 20)
    s2 = {
        "workload": "BitNet-b1.58-2B-shaped decode: 30 layers x 7 projections (q/o 2560x2560, "
                    "k/v 640x2560, gate/up 6912x2560, down 2560x6912), N=1, one fused launch",
        "packed_bytes": d2.packed_bytes,
    }
    f_ms = back_to_back_ms(d2.step, s, k2)
    t_ms = back_to_back_ms(d2.two_step, s, k2)
    per = {}
    for name, fn in (("gemv_quant", d2.step), ("quant", d2.quant), ("gemv", d2.gemv),
                     ("gemv_tl2", d2.gemv_tl2)):
        ev = events(2 * k2)
        for e in ev:
            e.record(s)
        torch.cuda.synchronize()
        for i in range(k2):
            ev[2 * i].record(s)
            fn(s)
            ev[2 * i + 1].record(s)
        torch.cuda.synchronize()
        per[name] = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(k2)) / k2
    tabs = d2.chain_tables()
    c2_fused_ms = time_graph(lambda st: d2.chain_step(st, tabs), s, max(20, K))
    ttabs = d2.chain_two_tables()
    c2_two_ms = time_graph(lambda st: d2.chain_two_step(st, ttabs), s, max(20, K))
    del ttabs
    del tabs
    s2.update({
        "ms_per_step": round(f_ms, 5), "gbs": round(d2.packed_bytes / (f_ms * 1e-3) / 1e9, 1),
        "fused_roofline": {"achieved": round(d2.alg_bytes_fused / (per["gemv_quant"] * 1e-3)
                                             / 1e9, 1),
                           "peak": hbm_peak, "unit": "GB/s",
                           "frac": round(d2.alg_bytes_fused / (per["gemv_quant"] * 1e-3) / 1e9
                                         / hbm_peak, 4),
                           "bytes_per_launch": d2.alg_bytes_fused,
                           "avg_launch_ms": round(per["gemv_quant"], 5)},
        "two_step": {"what": "grouped quantiser launch, then grouped GEMV launch",
                     "ms_per_step": round(t_ms, 5),
                     "gbs": round(d2.packed_bytes / (t_ms * 1e-3) / 1e9, 1),
                     "gemv_roofline": {
                         "achieved": round(d2.alg_bytes_gemv / (per["gemv"] * 1e-3) / 1e9, 1),
                         "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(d2.alg_bytes_gemv / (per["gemv"] * 1e-3) / 1e9 / hbm_peak,
                                       4),
                         "bytes_per_launch": d2.alg_bytes_gemv,
                         "avg_launch_ms": round(per["gemv"], 5),
                         "traffic": ncu_traffic("gemv"),
                         "traffic_source": NCU_TRAFFIC["gemv"]["source"]}},
        "quant_launch_ms": round(per["quant"], 5),
        "decode_chain": chain_entry(
            "the 210 linears in the order a decoder imposes: per layer q/k/v, then o, then "
            "gate/up, then down (120 dependent groups)", d2.packed_bytes, c2_fused_ms,
            c2_two_ms, hbm_peak),
        "tl2_storage": {"what": "the GEMV launch over the same 210 layers stored at 5 bits per "
                                "three weights (TL2-style), int8 activations from the quantiser",
                        "bytes_per_launch": d2.tl2_bytes,
                        "avg_launch_ms": round(per["gemv_tl2"], 5),
                        "tl2_bytes_gbs": round(d2.tl2_bytes / (per["gemv_tl2"] * 1e-3) / 1e9, 1),
                        "weights_per_s_as_2bit_gbs": round(d2.packed_bytes /
                                                           (per["gemv_tl2"] * 1e-3) / 1e9, 1)},
    })
    s2["launches"] = 2 * k2 + k2 * 4 + 3 * 3
    del d2
    torch.cuda.empty_cache()
    return s2


def emit(args, world, peaks, h, ms_per_step, gbs, K, K2, e2e_ms, h2d, d2h, prefill_70b, s2,
         prefill, crossover, single, cpu):
    """Print the one JSON line (rank 0)."""
    hbm_peak = peaks["hbm_gbs"]
    sus_gbs = h["packed_bytes"] / (h["sus_ms"] * 1e-3) / 1e9
    chain_entry_70b = chain_entry(
        "the same 560 linears in the order a decoder imposes: per layer q/k/v, then o, then "
        "gate/up, then down (320 dependent groups)", h["packed_bytes"], h["chain_fused_ms"],
        h["chain_two_ms"], hbm_peak)
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
            "workload": "70B-shaped decode weight stream: 80 layers x 7 projections "
                        "(q/o 8192x8192, k/v 1024x8192, gate/up 28672x8192, down "
                        "8192x28672), N=1",
            "layers": 80, "tokens": 1,
            "packed_bytes_per_step": h["packed_bytes"],
            "launches_per_step": h["ncalls"],
            "l2": "no flush: 17.11 GB of packed weights per step > 126 MB L2",
            "parallelism": "replicas" if world > 1 else "single GPU",
        },
        "headline_basis": "value = packed weight bytes per step / back-to-back step time "
                          "(K steps, events at the ends; consecutive launches overlap their "
                          "start-up through programmatic dependent launch). roofline.achieved "
                          "= all bytes the fused kernel must move / its mean launch time, "
                          "events around every launch (no overlap).",
        "pct_of_measured_hbm": round(100 * gbs / world / hbm_peak, 2),
        "pct_of_nominal_hbm_8000": round(100 * gbs / world / HBM_NOMINAL_GBS, 2),
        "roofline": {
            "bound": "hbm",
            "kernel": "gemv_quant (fused quantise + GEMV, grouped, 20 layers = 140 linears "
                      "per launch, K=8192 and 28672)",
            "achieved": round(h["fused_gbs"], 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(h["fused_gbs"] / hbm_peak, 4),
            "peak_note": "hbm_gbs %s (burst copy)" % peaks["source"],
            "bytes_per_launch": round(h["alg_bytes"] / h["ncalls"]),
            "avg_launch_ms": round(h["launch_ms"], 5),
            "timing": "events around each launch, %d steps x %d launches" % (K2, h["ncalls"]),
            "traffic": ncu_traffic("gemv_quant"),
            "traffic_source": NCU_TRAFFIC["gemv_quant"]["source"],
        },
        "sustained": {
            "what": "the headline step back to back for >= %.0f s" % SUSTAINED_S,
            "steps": h["sus_steps"], "ms_per_step": round(h["sus_ms"], 5),
            "gbs": round(sus_gbs, 1), "frac_of_measured_hbm": round(sus_gbs / hbm_peak, 4),
            "peak_note": "against hbm_gbs (burst copy); MEASURED_PEAKS has no sustained "
                         "copy figure",
            "clocks": h["sclk"],
        },
        "decode_chain": chain_entry_70b,
        "e2e": {"value": round(whole_job_gbs(world, h["packed_bytes"], e2e_ms), 1),
                "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "per step: pinned host -> device copy of every fp32 layer input, "
                       "the fused launches, device -> host copy of every output; two buffer "
                       "sets and two copy streams overlap step i's copies with step i-1's "
                       "launches"},
        "prefill_70b": prefill_70b,
        "prefill": prefill,
        "stream_2b": s2,
        "crossover": crossover,
        "single_1024": single,
        "gpu_launches": K * h["ncalls"],
        "gpu_launches_other_passes": {"sustained": h["sus_steps"] * h["ncalls"],
                                      "per_launch_timing": K2 * h["ncalls"],
                                      "stream_2b": s2.get("launches")
                                      if isinstance(s2, dict) else None},
        "clocks": h["clk"],
        "cpu_baseline": cpu,
    }
    print(json.dumps(out), flush=True)


def measure_e2e(dec, s, steps):
    hXh = [torch.empty(dec.Xh.shape, pin_memory=True) for _ in range(2)]
    hXf = [torch.empty(dec.Xf.shape, pin_memory=True) for _ in range(2)]
    hY = [torch.empty(dec.Y.shape, pin_memory=True) for _ in range(2)]
    for b in range(2):
        hXh[b].copy_(dec.Xh)
        hXf[b].copy_(dec.Xf)
    dXh = [dec.Xh, torch.empty_like(dec.Xh)]
    dXf = [dec.Xf, torch.empty_like(dec.Xf)]
    dY = [dec.Y, torch.empty_like(dec.Y)]
    calls = [dec.fused_calls(dXh[b], dXf[b], dY[b]) for b in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i & 1
        up.wait_event(comp_done[b])          # step i-2 has finished reading dX[b]
        with torch.cuda.stream(up):
            dXh[b].copy_(hXh[b], non_blocking=True)
            dXf[b].copy_(hXf[b], non_blocking=True)
        h2d_done[b].record(up)
        s.wait_event(h2d_done[b])
        s.wait_event(d2h_done[b])            # step i-2's outputs have left dY[b]
        dec.step(s, calls[b])
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
    for i in range(steps):
        e2e_step(i)
    z.record(down)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / steps
    h2d = (dec.Xh.numel() + dec.Xf.numel()) * 4
    d2h = dec.Y.numel() * 4
    del calls, dXh[1], dXf[1], dY[1]
    return ms, h2d, d2h


# ----------------------------------------------------------------------------- CPU oracle

def host_info():
    model = platform.processor() or None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def _oracle_sample(rows_per_proj):
    """Oracle inputs for the CPU baseline: layer 0 of the 70B-shaped stream,
    the first `rows_per_proj` rows of each of its 7 projections (alpha from the
    whole latent tensor, as the path defines it), and each projection's
    one-token input.  Latent weights are drawn on the GPU (same generator as
    every other leg) and copied to the host."""
    import oracle
    cfg = HEADLINE_CFG
    shape = inputs.WORKLOADS[cfg].model
    items = []
    for p, (name, M, K) in enumerate(shape.projections()):
        W = inputs.latent_weights(M, K, inputs.weight_seed(cfg, 0, p), device="cuda").cpu().numpy()
        alpha = oracle.absmean(W)
        codes = oracle.ternarize(W[:rows_per_proj], alpha)
        del W
        x = inputs.activations(1, K, inputs.act_seed(cfg, 0, input_proj(p)),
                               device="cuda").cpu().numpy()
        items.append((codes, alpha, x))
    return items


def cpu_baseline(budget_s=15.0, parallel_s=3.0):
    """The oracle as it stands on this host: single-threaded (the oracle is
    plain single-threaded C) for about budget_s seconds, then one oracle
    process per core on disjoint row blocks of a whole projection, each block
    repeated for about parallel_s seconds."""
    import oracle
    from oracle import rowpar
    rows = 1024
    items = _oracle_sample(rows)
    nbytes_rep = sum(c.size // 4 for c, _, _ in items)
    secs, reps = 0.0, 0
    while secs < budget_s or reps == 0:
        t0 = time.perf_counter()
        for codes, alpha, x in items:
            q, amax, _ = oracle.quant_act(x)
            acc = oracle.matmul_i32(codes, q)
            oracle.rescale(acc, alpha, amax)
        secs += time.perf_counter() - t0
        reps += 1
    single = nbytes_rep * reps / secs / 1e9
    info = host_info()
    # all cores: the whole gate projection of layer 0, its rows split over one
    # single-threaded oracle process per core
    workers = info["host_cores"] or 1
    try:
        shape = inputs.WORKLOADS[HEADLINE_CFG].model
        name, M, K = shape.projections()[4]
        W = inputs.latent_weights(M, K, inputs.weight_seed(HEADLINE_CFG, 0, 4),
                                  device="cuda").cpu().numpy()
        alpha = oracle.absmean(W)
        codes = oracle.ternarize(W, alpha)
        del W
        x = inputs.activations(1, K, inputs.act_seed(HEADLINE_CFG, 0, input_proj(4)),
                               device="cuda").cpu().numpy()
        q, amax, _ = oracle.quant_act(x)
        block_bytes = (M // workers + 1) * K / 4
        prep = max(1, int(parallel_s * single * 1e9 / block_bytes))
        dt, workers = rowpar.time_all_cores(codes, q, amax, alpha, reps=prep, workers=workers)
        par = prep * M * K / 4 / dt / 1e9
        par_sample = ("the gate projection of layer 0 (%dx%d, %d packed bytes), N=1, rows split "
                      "over %d single-threaded oracle processes, each block %d times; first "
                      "start to last finish %.2f s" % (M, K, M * K // 4, workers, prep, dt))
        del codes
    except Exception as exc:  # noqa: BLE001
        par, par_sample = "failed: %s" % exc, None
    return {"value": round(single, 4), "unit": "GB/s", "cores": 1, "threads": 1,
            "kind": "oracle",
            "sample": "70B-shaped layer 0, the first %d rows of each of its 7 projections "
                      "(%d packed bytes), N=1: quant_act + int32 triple-loop matmul + "
                      "rescale, x%d (%.1f s), one thread" % (rows, nbytes_rep, reps, secs),
            "all_cores": {"value": par if isinstance(par, str) else round(par, 4),
                          "unit": "GB/s", "processes": workers, "sample": par_sample},
            **info}


def run_reference(args, rank, world):
    """CPU oracle on bounded samples of the headline workload (rank 0 only)."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    cfg = HEADLINE_CFG
    projs = inputs.WORKLOADS[cfg].model.projections()
    # one step = rows [r0, r0+R) of one projection of layer 0 (rotating), N=1;
    # R sized so that warmup + steps stay within ~90 s of CPU time
    data = []
    for p, (name, M, K) in enumerate(projs):
        W = inputs.latent_weights(M, K, inputs.weight_seed(cfg, 0, p)).numpy()
        alpha = oracle.absmean(W)
        codes = oracle.ternarize(W[:2048], alpha)
        del W
        x = inputs.activations(1, K, inputs.act_seed(cfg, 0, input_proj(p))).numpy()
        data.append((codes, alpha, x))
    t0 = time.perf_counter()
    c, a, x = data[0]
    q, amax, _ = oracle.quant_act(x)
    oracle.matmul_i32(c[:256], q)
    rate = 256 * c.shape[1] / max(time.perf_counter() - t0, 1e-6)     # weights per second
    total = max(1, args.steps + args.warmup)
    per_step_w = max(128 * 8192, int(rate * 90.0 / total))
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
           "config": {"workload": "70B-shaped decode weight stream: 80 layers x 7 projections "
                                  "(q/o 8192x8192, k/v 1024x8192, gate/up 28672x8192, down "
                                  "8192x28672), N=1",
                      "layers": 80, "tokens": 1},
           "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": 1, "threads": 1,
                            "kind": "oracle",
                            "sample": "per step: a row block of one projection of layer 0 "
                                      "(rotating over the 7), quant_act + matmul + rescale",
                            **host_info()},
           "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "headline", "chain", "prefill", "prefill70",
                                       "stream2b", "crossover"],
                    default="all",
                    help="profiling runs: time only one part and print a partial line")
    ap.add_argument("--layers", type=int, default=None,
                    help="with --only headline|chain: layers of the 70B-shaped stream (default 80)")
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
