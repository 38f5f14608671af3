#!/usr/bin/env python
"""Benchmark of the rotation-based W4A4 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the online path over one batch of synthetic input:
  rq_rotate_quantize(X)   randomized Hadamard + quantize + pack (HBM-bound)
  rq_w4a4_gemm(Xq, Wq)    quantized GEMM on tcgen05 tensor cores
with the weights rotated and quantized once beforehand (the offline side).
For the KV workload a step is rq_kv_rotate_quantize on K and on V.

The metric is the pair "fused Hadamard+quant GB/s vs HBM peak; W4A4 GEMM TOPS
vs tensor peak": `value` is the fused rotate+quantize throughput in GB/s
(algorithmic bytes / device time), and the `gemm` object carries the GEMM's
TOPS.  Times are CUDA events on the launching stream around K steps run back
to back; the inputs cycle through distinct sets that together exceed the L2
(no flush is needed), the per-kernel figures come from K launches of each
kernel alone over the same inputs, and for N > 1 each rank runs its own batch
(weak scaling, no data-path collective) and the time is the max over ranks.
"""

import argparse
import json
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from rotation_w4a4_quantization_b200 import synthetic as syn  # noqa: E402

METRIC = "fused Hadamard+quant GB/s vs HBM peak; W4A4 GEMM TOPS vs tensor peak"
L2_BYTES = 126 << 20      # B200 L2 (nominal)
RING_MAX = 16
# The default run measures every timed configuration of the metric in one
# invocation: the headline is down_proj (the largest one carrying both halves
# of the metric, rotate+quantize and the W4A4 GEMM); q_proj INT4 (full-width
# rotation), q_proj NVFP4 and the KV4 cache are reported beside it.  The tiny
# 64 x 512 case is a parity case (launch-bound), not a bench line.
DEFAULT_WORKLOAD = "all"
HEADLINE = "down_proj_int4"
ALSO_MEASURED = ("q_proj_int4", "q_proj_nvfp4", "kv4")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=["all"] + sorted(syn.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--y-dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


ROTATE_SOURCES = ("rq_common.cuh", "rq_rotate.cuh")
GEMM_SOURCES = ("rq_common.cuh", "rq_tc.cuh", "rq_gemm.cuh")
ATTN_SOURCES = ("rq_common.cuh", "rq_attn.cuh")
_ROT, _GEM, _ATT = "121dbfcc644440af", "74cfd6dd085e3e33", "80b39046d2c3159b"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch from one
# ncu capture of the kernel (summarised in profiles/), with the fingerprint of
# the sources it was taken on (reported as null once they change).  kv4 and
# kv4_decode were captured at B = 4 and are scaled to the bench's B = 16 (traffic
# grows with the vectors processed); kv4_decode is the partial + combine pair.
TRAFFIC = {
    ("hadamard_quant", "q_proj_int4"): (16818432, _ROT),
    ("hadamard_quant", "down_proj_int4"): (108285440, _ROT),
    ("hadamard_quant", "kv4"): (149308928 * 4, _ROT),
    ("hadamard_quant", "q_proj_nvfp4"): (16851200, _ROT),
    ("hadamard_quant", "q_proj_mxfp4"): (16832000, _ROT),
    ("hadamard_quant", "q_proj_w4a8"): (16817920, _ROT),
    ("hadamard_quant", "q_proj_w8a8"): (16817920, _ROT),
    ("hadamard_quant", "q_proj_nvfp4_b16"): (16850944, _ROT),
    ("hadamard_quant", "q_proj_int4_asym"): (16847360, _ROT),
    ("hadamard_quant", "kv4_decode"): (72226048 * 4, _ATT),
    ("gemm", "q_proj_int4"): (12650496, _GEM),
    ("gemm", "down_proj_int4"): (59438848, _GEM),
    ("gemm", "q_proj_nvfp4"): (14189312, _GEM),
    ("gemm", "q_proj_mxfp4"): (13400064, _GEM),
    ("gemm", "q_proj_w4a8"): (16844544, _GEM),
    ("gemm", "q_proj_w8a8"): (25230592, _GEM),
    ("gemm_bytes", "q_proj_int4"): (21044480, _GEM),
    ("gemm_bytes", "down_proj_int4"): (94283520, _GEM),
}


def code_bytes(fmt, rows, k):
    """Bytes of codes and scales the rotate kernel writes for `rows` rows of K."""
    return {"int4": rows * k // 2 + rows * 4, "nvfp4": rows * k // 2 + rows * (k // 16),
            "mxfp4": rows * k // 2 + rows * (k // 32), "int8": rows * k + rows * 4,
            "int6": rows * k + rows * 4, "int4_asym": rows * k // 2 + rows * (k // 128) * 4}[fmt]


def ring_slots(name):
    """How many distinct input sets the timed steps cycle through so that a set
    is out of L2 when it comes round again: the step's distinct inputs (X and
    the weight codes) times the slot count cover at least twice the L2.  The KV
    workloads' inputs alone are several times the L2."""
    c = syn.WORKLOADS[name]
    if name in ("kv4", "kv4_decode"):
        return 1
    per = c["M"] * c["K"] * 2
    if c["fmt"] != "int4_asym":
        per += code_bytes(c.get("wfmt", c["fmt"]), c["N"], c["K"])
    return int(min(RING_MAX, max(1, -(-2 * L2_BYTES // per))))


def ring_bytes(name):
    c = syn.WORKLOADS[name]
    if name == "kv4":
        return 2 * c["B"] * c["H"] * c["S"] * c["D"] * 2
    if name == "kv4_decode":
        return 2 * c["B"] * c["H"] * c["S"] * 68
    per = c["M"] * c["K"] * 2
    if c["fmt"] != "int4_asym":
        per += code_bytes(c.get("wfmt", c["fmt"]), c["N"], c["K"])
    return ring_slots(name) * per


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank times (every rank takes this collective at
    the same point); the job is as slow as its slowest rank."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().numpy()


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed over the (max) time, per second."""
    return units_per_rank * world / (ms * 1e-3)


def source_fingerprint(files):
    import hashlib
    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "rotation_w4a4_quantization_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def traffic(kind, workload):
    entry = TRAFFIC.get((kind, workload))
    if entry is None:
        return None
    if workload == "kv4_decode":
        files = ATTN_SOURCES
    else:
        files = ROTATE_SOURCES if kind == "hadamard_quant" else GEMM_SOURCES
    return entry[0] if source_fingerprint(files) == entry[1] else None


# --------------------------------------------------------------------------- workload
class Workload:
    """Device-resident inputs and the step function for one workload."""

    def __init__(self, name, rq, device, seed_offset, y_dtype):
        self.name = name
        self.rq = rq
        self.cfg = syn.WORKLOADS[name]
        self.y_dtype = y_dtype
        self.kv = name == "kv4"
        self.kvdec = name == "kv4_decode"
        self.R = 1
        if self.kvdec:
            c = self.cfg
            self.signs = syn.workload_signs(name).to(device)
            k = syn.kv(device=device, which=0, seed_offset=seed_offset)
            self.kcache = rq.kv_rotate_quantize(k, self.signs)
            del k
            v = syn.kv(device=device, which=1, seed_offset=seed_offset)
            self.vcache = rq.kv_rotate_quantize(v, self.signs)
            del v
            g = torch.Generator(device=device)
            g.manual_seed(4000 + c["index"] + seed_offset)
            self.q = torch.randn((c["B"], c["H"], c["D"]), generator=g, device=device).to(torch.bfloat16)
            self.out = torch.empty((c["B"], c["H"], c["D"]), dtype=torch.float32, device=device)
            nws = int(rq.lib.rq_kv4_attention_workspace_bytes(c["B"], c["H"], c["S"]))
            self.attn_ws = torch.empty((nws,), dtype=torch.uint8, device=device)
            bh = c["B"] * c["H"]
            # the whole cache (K and V: 64 B of codes + fp16 scale and zero per token and head), q and o
            self.quant_bytes = bh * c["S"] * 2 * (64 + 4) + bh * c["D"] * (2 + 4)
            self.gemm_ops = 0
            self.h2d_bytes = self.q.numel() * 2
        elif self.kv:
            c = self.cfg
            self.k = syn.kv(device=device, which=0, seed_offset=seed_offset)
            self.v = syn.kv(device=device, which=1, seed_offset=seed_offset)
            self.signs = syn.workload_signs(name).to(device)
            shape = (c["B"], c["H"], c["S"])
            self.outs = [(torch.empty(shape + (64,), dtype=torch.uint8, device=device),
                          torch.empty(shape, dtype=torch.float16, device=device),
                          torch.empty(shape, dtype=torch.float16, device=device)) for _ in range(2)]
            n_vec = 2 * c["B"] * c["H"] * c["S"]
            self.quant_bytes = n_vec * (128 * 2 + 64 + 2 + 2)
            self.gemm_ops = 0
            self.h2d_bytes = 2 * self.k.numel() * 2
        else:
            c = self.cfg
            self.fmt = c["fmt"]
            self.wfmt = c.get("wfmt", self.fmt)
            self.block = c["block"]
            self.R = ring_slots(name)
            # R distinct input sets (activations from their own seeds, copies of the
            # weight codes) and outputs, cycled step to step
            self.xs = [syn.activations(name, device=device, seed_offset=seed_offset * RING_MAX + r)
                       for r in range(self.R)]
            self.x = self.xs[0]
            w = syn.weights(name, device=device)
            self.signs = syn.workload_signs(name).to(device)
            wq = None if self.fmt == "int4_asym" else rq.prepare_weights(w, self.signs, self.block, self.wfmt)
            del w
            self.wqs = [None if wq is None else tuple(None if t is None else t.clone() for t in wq)
                        for _ in range(self.R)]
            self.wq = self.wqs[0]
            # INT4 weights also in the byte layout (the same codes one per byte), for the
            # W4A4 GEMM that reads them without widening
            self.wqs_bytes = None
            if self.fmt == "int4":
                w = syn.weights(name, device=device)
                wb = rq.prepare_weights(w, self.signs, self.block, "int4_bytes")
                del w
                self.wqs_bytes = [tuple(None if t is None else t.clone() for t in wb) for _ in range(self.R)]
            m, k, n = c["M"], c["K"], c["N"]
            self.xq_outs = [rq._alloc_quant_outputs(m, k, rq._fmt(self.fmt), device) for _ in range(self.R)]
            self.xq_out = self.xq_outs[0]
            self.gscales = [torch.empty((1,), dtype=torch.float32, device=device) for _ in range(self.R)]
            self.gscale = self.gscales[0]
            self.ws = torch.empty((16,), dtype=torch.uint8, device=device)
            self.ys = [torch.empty((m, n), dtype=torch.bfloat16 if y_dtype == "bf16" else torch.float32,
                                   device=device) for _ in range(self.R)]
            self.y = self.ys[0]
            self.quant_bytes = m * k * 2 + code_bytes(self.fmt, m, k)
            self.gemm_ops = 2 * m * n * k
            self.h2d_bytes = self.x.numel() * 2
        self.d2h_bytes = 0

    def nvfp4_one_pass(self):
        if self.kv or self.kvdec:
            return False
        # librq quantizes dynamic NVFP4 in one launch when each SM's share of
        # the rows (plus the sign table) fits its 220 KiB of shared memory;
        # otherwise a max launch precedes the quantize launch
        m, k = self.cfg["M"], self.cfg["K"]
        sms = torch.cuda.get_device_properties(self.xs[0].device).multi_processor_count
        rpc = -(-m // sms)
        return rpc * k * 2 + (k // 128) * 256 + 32 <= 220 * 1024

    def quant_launches(self):
        if self.kv or self.kvdec:
            return 2
        if self.fmt == "nvfp4":
            return 1 if self.nvfp4_one_pass() else 2
        return 1

    def quant_kernel(self):
        if self.kvdec:
            return "kv4_attn_partial_kernel + kv4_attn_combine_kernel"
        if self.kv:
            return "rotate_kernel<KV4>"
        if self.fmt == "nvfp4" and self.nvfp4_one_pass():
            return "rotate_nvfp4_resident_kernel"
        mode = {"int8": "INT8, ", "int6": "INT8, ", "int4_asym": "ASYM4, "}.get(self.fmt, "")
        if self.block == 0 and self.cfg["K"] == 4096:
            return "rotate_full4096_kernel<%s>" % ("INT8" if self.fmt in ("int8", "int6") else "INT4")
        return "rotate_kernel<%s%s>" % (mode, "full width" if self.block == 0 else "%d-blocks" % self.block)

    def gemm_launches(self):
        return 0 if (self.kv or self.kvdec or self.fmt == "int4_asym") else 1

    def quant(self, i=0):
        rq = self.rq
        r = i % self.R
        if self.kvdec:
            rq.kv4_decode_attention(self.q, self.kcache, self.vcache, self.signs, out=self.out,
                                    workspace=self.attn_ws)
            return None
        if self.kv:
            rq.kv_rotate_quantize(self.k, self.signs, out=self.outs[0])
            rq.kv_rotate_quantize(self.v, self.signs, out=self.outs[1])
            return None
        return rq.rotate_quantize(self.xs[r], self.signs, self.block, self.fmt, "dynamic", gscale=self.gscales[r],
                                  out=self.xq_outs[r], workspace=self.ws)

    def slot_codes(self, i):
        """The quantized activations of slot i (as the rotate kernel left them)."""
        r = i % self.R
        return self.xq_outs[r] + (self.gscales[r] if self.fmt == "nvfp4" else None,)

    def gemm(self, xq, i=0):
        if self.kv or self.kvdec or self.fmt == "int4_asym":
            return None
        r = i % self.R
        if self.fmt in ("int8", "int6"):
            return self.rq.int_gemm(xq, self.fmt, self.wqs[r], self.wfmt, self.y_dtype, y=self.ys[r])
        return self.rq.w4a4_gemm(xq, self.wqs[r], self.fmt, self.y_dtype, y=self.ys[r])

    def gemm_bytes(self, xq, i=0):
        """The same W4A4 product against the weights' INT4 codes in the byte layout."""
        r = i % self.R
        return self.rq.int_gemm(xq, "int4", self.wqs_bytes[r], "int4_bytes", self.y_dtype, y=self.ys[r])

    def result(self):
        if self.kvdec:
            return self.out
        if getattr(self, "fmt", None) == "int4_asym":
            return self.xq_out[0]
        return self.outs[0][0] if self.kv else self.y


def gemm_kernel_name(wl, two_sm):
    if wl.fmt in ("int8", "int6"):
        return "gemm_int_2sm_ts_kernel<A8, %s>" % ("W8" if wl.wfmt in ("int8", "int6") else "W4")
    if wl.fmt == "int4":
        return "gemm_int_2sm_ts_kernel<A4, W4>" if two_sm else "gemm_int4_kernel"
    return ("gemm_fp4_2sm_kernel" if two_sm else "gemm_fp4_kernel") + "<%s>" % wl.fmt


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    from a background thread every ~2 ms while the timed region runs (read-only;
    nothing is changed on the GPU)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = False
        self._thread = None

    def start(self):
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:  # NVML numbers GPUs physically; find ours by PCI bus id
                pr = torch.cuda.get_device_properties(self.index)
                bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None

    def _run(self):
        nv = self.nv
        while not self._stop:
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS:
                    if r & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def stop(self):
        if self._thread is None:
            return None
        self._stop = True
        self._thread.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------------------- CPU oracle leg
_ORACLE_W = {}


def oracle_sample(name, rows):
    """Time the oracle (as it stands) on `rows` rows of the workload; returns (GB/s, TOPS, seconds, desc, threads)."""
    from oracle import gemm as ogemm, hadamard as ohad, quant as oquant
    c = syn.WORKLOADS[name]
    if name == "kv4_decode":
        # rows = (batch entry, head) pairs over the full sequence length: the
        # cache of one batch entry is built once and attended rows / H times
        from oracle import attention as oattn
        s = syn.workload_signs(name).numpy()
        heads = min(rows, c["H"])
        reps = max(1, rows // heads)
        k = syn.kv(batch=1, heads=heads, which=0).to(torch.float64).numpy()
        v = syn.kv(batch=1, heads=heads, which=1).to(torch.float64).numpy()
        caches = []
        for x in (k, v):
            q4, sh, zh, _, _ = oquant.kv4_vectors(oattn.rotate_heads(x, s).reshape(-1, 128))
            caches += [q4.reshape(x.shape), sh.reshape(x.shape[:-1]), zh.reshape(x.shape[:-1])]
        qv = np.random.default_rng(0).standard_normal((1, heads, 128))
        t0 = time.perf_counter()
        for _ in range(reps):
            oattn.kv4_decode_attention(qv, *caches, s)
        dt = time.perf_counter() - t0
        nbytes = reps * heads * c["S"] * 2 * (64 + 4)
        return nbytes / dt / 1e9, None, dt, "%d x %d heads x %d tokens of the cache" % (reps, heads, c["S"])
    if name == "kv4":
        kv = syn.kv(batch=1, heads=4, seq=rows)
        s = syn.workload_signs(name).numpy()
        x = kv.to(torch.float64).numpy().reshape(-1, 128)
        t0 = time.perf_counter()
        xr = ohad.rotate(x, s, 128)
        q, sh, zh, _, _ = oquant.kv4_vectors(xr)
        oquant.pack_nibbles(q)
        dt = time.perf_counter() - t0
        nbytes = x.shape[0] * (128 * 2 + 64 + 4)
        return nbytes / dt / 1e9, None, dt, "%d head_dim vectors (1 x 4 heads x %d tokens)" % (x.shape[0], rows)
    if c["fmt"] == "int4_asym":
        # the quantizer alone (no GEMM consumes these codes)
        x = syn.activations(name, rows=rows).to(torch.float64).numpy()
        s = syn.workload_signs(name).numpy()
        t0 = time.perf_counter()
        q, _, _, _, _ = oquant.asym_int4_groups(ohad.rotate(x, s, c["block"]))
        oquant.pack_nibbles(q)
        dt = time.perf_counter() - t0
        return ((rows * c["K"] * 2 + code_bytes("int4_asym", rows, c["K"])) / dt / 1e9, None, dt,
                "%d of %d rows of X" % (rows, c["M"]))
    # rows beyond 4096 are timed as repeats of one 4096-row batch (host memory)
    chunk = min(rows, 4096)
    reps = -(-rows // chunk)
    x = syn.activations(name, rows=chunk).to(torch.float64).numpy()
    s = syn.workload_signs(name).numpy()
    k, n = c["K"], c["N"]
    block = c["block"]
    bits = {"int4": 4, "int6": 6, "int8": 8}
    if name not in _ORACLE_W:  # the offline side, once per run (not timed)
        wr = ohad.rotate(syn.weights(name).to(torch.float64).numpy(), s, block)
        if c["fmt"] in ("int8", "int6"):
            _ORACLE_W[name] = oquant.int_sym_rows(wr, bits[c.get("wfmt", c["fmt"])])[:2]
        elif c["fmt"] == "int4":
            _ORACLE_W[name] = oquant.int4_sym_rows(wr)[:2]
        elif c["fmt"] == "nvfp4":
            gw = oquant.nvfp4_global_scale(wr)
            _ORACLE_W[name] = oquant.nvfp4_rows(wr, gw)[:2] + (gw,)
        else:
            _ORACLE_W[name] = oquant.mxfp4_rows(wr)[:2]
        del wr
    if c["fmt"] in ("int8", "int6", "int4"):
        qw, sw = _ORACLE_W[name]
    elif c["fmt"] == "nvfp4":
        ew, sfw, gw = _ORACLE_W[name]
    else:
        ew, sfw = _ORACLE_W[name]
    tq = tg = 0.0
    for _ in range(reps):
        t0 = time.perf_counter()
        xr = ohad.rotate(x, s, block)
        if c["fmt"] in ("int8", "int6"):
            qx, sx, _ = oquant.int_sym_rows(xr, bits[c["fmt"]])
            qx.astype(np.int8)
        elif c["fmt"] == "int4":
            qx, sx, _ = oquant.int4_sym_rows(xr)
            oquant.pack_nibbles(qx)
        elif c["fmt"] == "nvfp4":
            gx = oquant.nvfp4_global_scale(xr)
            ex, sfx, _, _ = oquant.nvfp4_rows(xr, gx)
            oquant.pack_nibbles(ex)
        else:
            ex, sfx, _, _ = oquant.mxfp4_rows(xr)
            oquant.pack_nibbles(ex)
        t1 = time.perf_counter()
        if c["fmt"] in ("int8", "int6"):
            ogemm.int4_y(ogemm.int_acc(qx, qw), sx, sw)
        elif c["fmt"] == "int4":
            ogemm.int4_y(ogemm.int4_acc(qx, qw), sx, sw)
        elif c["fmt"] == "nvfp4":
            ogemm.nvfp4_y(ex, sfx, gx, ew, sfw, gw)
        else:
            ogemm.mxfp4_y(ex, sfx, ew, sfw)
        t2 = time.perf_counter()
        tq += t1 - t0
        tg += t2 - t1
    done = reps * chunk
    nbytes = done * k * 2 + code_bytes(c["fmt"], done, k)
    return (nbytes / tq / 1e9, 2.0 * done * n * k / tg / 1e12, tq + tg,
            "%d rows of X (%d x %d) with the full W" % (done, reps, chunk))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def sample_rows(name):
    """Rows (tokens, vectors, or head-passes for kv4_decode) of the oracle's timed
    sample: about 5-10 s of host work on a 16-core host."""
    return {"tiny_int4": 64, "q_proj_int4": 40960, "down_proj_int4": 16384, "q_proj_nvfp4": 8192, "kv4": 102400,
            "q_proj_mxfp4": 16384, "kv4_decode": 1024, "q_proj_w4a8": 40960, "q_proj_w8a8": 40960,
            "q_proj_nvfp4_b16": 8192, "q_proj_mxfp4_b32": 16384, "q_proj_int4_asym": 16384}[name]


def min_rows(name):
    return {"kv4_decode": 1, "kv4": 64}.get(name, 8)


# --------------------------------------------------------------------------- main
def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from rotation_w4a4_quantization_b200 import rq
    rq.init(local)
    if args.workload == "all":
        # every rank measures the same configurations in the same order
        head = run_workload(HEADLINE, args, rq, dev, dist, world, rank, local, cpu_scale=0.5)
        head["config"] = workload_config(args, HEADLINE)
        head["configs"] = {}
        for name in ALSO_MEASURED:
            sub = run_workload(name, args, rq, dev, dist, world, rank, local, cpu_scale=0.4)
            for key in ("metric", "n_gpus", "warmup", "higher_is_better", "scaling", "vs_baseline", "data"):
                sub.pop(key, None)
            head["configs"][name] = sub
        out = head
    else:
        out = run_workload(args.workload, args, rq, dev, dist, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def product_errors(name, wl, rq, rows=256):
    """Relative product error ||X W^T - Y|| / ||X W^T|| of the library's own Y
    on the first `rows` rows of the workload's X (all N outputs), for the
    rotated arm (the workload's block and signs) and the unrotated arm
    (block = 1, all signs +1: the same quantizers on X and W themselves).
    X W^T is formed in fp64 on the host from the bf16 inputs."""
    c = wl.cfg
    dev = wl.x.device
    x = wl.xs[0][:rows]
    w = syn.weights(name, device=dev)
    y_true = x.double().cpu().numpy() @ w.double().cpu().numpy().T
    ones = torch.ones_like(wl.signs)
    out = {"rows": int(rows), "outputs": int(c["N"]), "reference": "fp64 X.W^T on the host from the bf16 inputs"}
    for arm, block, sg in (("rotated", c["block"], wl.signs), ("unrotated", 1, ones)):
        wq = rq.prepare_weights(w, sg, block, wl.wfmt)
        xq = rq.rotate_quantize(x.contiguous(), sg, block, wl.fmt)
        y = rq.w4a4_gemm(xq, wq, wl.fmt, "f32")
        yh = y.double().cpu().numpy()
        out[arm] = round(float(np.linalg.norm(yh - y_true) / np.linalg.norm(y_true)), 5)
        del wq, xq, y
    out["arms"] = "rotated: block %s with the workload's random signs; unrotated: block 1, signs +1" % (
        "full" if c["block"] == 0 else c["block"])
    return out


def run_workload(name, args, rq, dev, dist, world, rank, local, cpu_scale=1.0):
    """Build one workload, time it, and return its JSON object."""
    wl = Workload(name, rq, dev, seed_offset=rank, y_dtype=args.y_dtype)
    stream = torch.cuda.current_stream(dev)
    K = args.steps

    def step(i):
        wl.gemm(wl.quant(i), i)

    def timed(fn):
        """K launches of fn(i) back to back on the stream, between one pair of
        events; the inputs cycle through the ring (larger than L2 together)."""
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # keep the GPU busy until all K launches are queued (~50 us of host time
        # each at most), so the timed region measures the GPU, not the host
        torch.cuda._sleep(min(100_000 * K, 2_000_000_000))
        a.record(stream)
        for i in range(K):
            fn(i)
        b.record(stream)
        return a, b

    for i in range(max(args.warmup, 3, wl.R)):
        step(i)
    rq.get_device_error()
    torch.cuda.synchronize()

    # the timed region: K steps of the whole path, back to back
    clocks = ClockSampler(local)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed steps " + name)
    ev_step = timed(step)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    # per-kernel averages for the roofline: each kernel alone, K launches the same way
    ev_q = timed(lambda i: wl.quant(i))
    ev_g = timed(lambda i: wl.gemm(wl.slot_codes(i), i)) if wl.gemm_launches() else None
    ev_gb = timed(lambda i: wl.gemm_bytes(wl.slot_codes(i), i)) if getattr(wl, "wqs_bytes", None) else None
    torch.cuda.synchronize()
    clk = clocks.stop()
    rq.get_device_error()
    step_tot = ev_step[0].elapsed_time(ev_step[1])
    q_tot = ev_q[0].elapsed_time(ev_q[1])
    g_tot = ev_g[0].elapsed_time(ev_g[1]) if ev_g is not None else 0.0
    tot = max_over_ranks([step_tot, q_tot, g_tot], dist, dev)
    ms_step = tot[0] / K
    q_mean_ms = tot[1] / K
    g_mean_ms = tot[2] / K

    # end to end through the public API: pinned host input -> device -> path -> host result
    e2e = measure_e2e(wl, rq, dev, stream, K=min(K, 50))
    e2e_ms = max_over_ranks([e2e["ms_per_step"]], dist, dev)[0]
    e2e["value"] = round(job_rate(wl.quant_bytes, world, e2e_ms) / 1e9, 3)
    e2e["ms_per_step"] = round(e2e_ms, 4)

    peaks = load_peaks()
    quant_gbs = job_rate(wl.quant_bytes, world, q_mean_ms) / 1e9
    out = {
        "metric": METRIC,
        "value": round(quant_gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.cfg.get("fmt", "int4"),
        "data": "synthetic (seeded, shaped like the article's Qwen3-8B layer inputs)",
        "config": workload_config(args, name),
        "gpu_launches": K * (wl.quant_launches() + wl.gemm_launches()),
    }
    q_launch_ms = q_mean_ms / wl.quant_launches()
    roof_q = {"bound": "hbm", "achieved": round(wl.quant_bytes / wl.quant_launches() / (q_launch_ms * 1e-3) / 1e9, 1),
              "peak": peaks["hbm"], "unit": "GB/s", "traffic": traffic("hadamard_quant", name),
              "kernel": wl.quant_kernel(),
              "peak_source": peaks["src"]}
    roof_q["frac"] = round(roof_q["achieved"] / roof_q["peak"], 4)
    if wl.gemm_launches():
        ratio = 2.0  # INT8 and FP4 dense tensor peaks are 2x / 4x the bf16 one (nominal ratios)
        if wl.fmt in ("nvfp4", "mxfp4"):
            ratio = 4.0
        tops = job_rate(wl.gemm_ops, world, g_mean_ms) / 1e12
        peak_t = peaks["bf16"] * ratio
        two_sm = wl.cfg["M"] > 128
        roof_g = {"bound": "tensor", "achieved": round(wl.gemm_ops / (g_mean_ms * 1e-3) / 1e12, 1), "peak": peak_t,
                  "unit": "TFLOP/s", "traffic": traffic("gemm", name),
                  "kernel": gemm_kernel_name(wl, two_sm),
                  "peak_source": "%s bf16 x %g (nominal %s/bf16 ratio)" % (peaks["src"], ratio,
                                                                           "int8" if ratio == 2 else "fp4")}
        roof_g["frac"] = round(roof_g["achieved"] / peak_t, 4)
        out["gemm"] = {"value": round(tops, 2), "unit": "TOPS", "ms": round(g_mean_ms, 5),
                       "frac_of_peak": roof_g["frac"]}
        if ev_gb is not None:
            gb_ms = max_over_ranks([ev_gb[0].elapsed_time(ev_gb[1])], dist, dev)[0] / K
            gb_tops = job_rate(wl.gemm_ops, world, gb_ms) / 1e12
            out["gemm_int4_bytes"] = {
                "value": round(gb_tops, 2), "unit": "TOPS", "ms": round(gb_ms, 5),
                "frac_of_peak": round(wl.gemm_ops / (gb_ms * 1e-3) / 1e12 / peak_t, 4),
                "kernel": "gemm_int_2sm_ts_kernel<A4, W8>", "traffic": traffic("gemm_bytes", name),
                "weights": "the same INT4 codes and scales, one code per byte (twice the packed weight memory)"}
        dominant = roof_g if g_mean_ms >= q_mean_ms else roof_q
        out["roofline"] = dominant
        out["roofline_hadamard_quant"] = roof_q
        out["roofline_gemm"] = roof_g
    else:
        out["roofline"] = roof_q
    out["hadamard_quant_ms"] = round(q_mean_ms, 5)
    out["e2e"] = e2e
    out["clocks"] = clk
    if wl.gemm_launches() and wl.fmt in ("int4", "nvfp4"):
        out["product_error"] = product_errors(name, wl, rq)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = max(min_rows(name), int(sample_rows(name) * cpu_scale))
        gbs, tops_cpu, secs, desc = oracle_sample(name, rows)
        out["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                               "sample": desc, "seconds": round(secs, 2), "host_cpus": os.cpu_count()}
        if tops_cpu is not None:
            out["cpu_baseline"]["gemm_tops"] = round(tops_cpu, 5)
    del wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def measure_e2e(wl, rq, dev, stream, K):
    """Same metric through the public API with host buffers: per step, the pinned
    host -> device copy of the step's input, the path, and the device -> host copy
    of its result.  For the matrix workloads the copies run on their own streams
    and are double-buffered (two input and two output slots), so step i's copies
    overlap step i - 1's compute as in a serving loop; the KV workloads' steps
    run in sequence on one stream."""
    def e2e_result(ms, h2d, d2h):
        return {"value": round(wl.quant_bytes / (ms * 1e-3) / 1e9, 3), "unit": "GB/s", "ms_per_step": round(ms, 4),
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    if wl.kv or wl.kvdec:
        if wl.kvdec:
            host_in, dev_in = [wl.q.cpu().pin_memory()], [wl.q]
        else:
            host_in, dev_in = [wl.k.cpu().pin_memory(), wl.v.cpu().pin_memory()], [wl.k, wl.v]
        res = wl.result()
        host_out = torch.empty(res.shape, dtype=res.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = host_out.numel() * host_out.element_size()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(K + 2):
            if i == 2:
                ev0.record(stream)
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            wl.gemm(wl.quant())
            host_out.copy_(wl.result(), non_blocking=True)
        ev1.record(stream)
        torch.cuda.synchronize()
        return e2e_result(ev0.elapsed_time(ev1) / K, h2d, d2h)

    # matrix workloads: slots 0 and 1 of the ring, copies on their own streams
    results = [wl.ys[r] if wl.gemm_launches() else wl.xq_outs[r][0] for r in range(2)]
    host_in = [wl.xs[r].cpu().pin_memory() for r in range(2)]
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in results]
    h2d = host_in[0].numel() * host_in[0].element_size()
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for i in range(K + 2):
        r = i % 2
        if i >= 2:
            s_in.wait_event(ev_done[r])        # step i - 2 has read input slot r
        if i == 2:
            t0.record(s_in)
        with torch.cuda.stream(s_in):
            wl.xs[r].copy_(host_in[r], non_blocking=True)
        ev_in[r].record(s_in)
        stream.wait_event(ev_in[r])
        if i >= 2:
            stream.wait_event(ev_out[r])       # step i - 2's result has left output slot r
        wl.gemm(wl.quant(r), r)
        ev_done[r].record(stream)
        s_out.wait_event(ev_done[r])
        with torch.cuda.stream(s_out):
            host_out[r].copy_(results[r], non_blocking=True)
        ev_out[r].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return e2e_result(t0.elapsed_time(t1) / K, h2d, d2h)


def workload_config(args, name):
    """The `config` object of both arms for workload `name`; with the default
    --workload all, the headline's config also lists the other measured ones."""
    c = dict(syn.WORKLOADS[name])
    c.pop("index", None)
    cfg = {"workload": name}
    cfg.update(c)
    if name not in ("kv4", "kv4_decode"):
        cfg["block"] = "full" if c["block"] == 0 else c["block"]
        cfg["y_dtype"] = args.y_dtype
        cfg["weights"] = "rotated+quantized once before timing (offline side)"
    r = ring_slots(name)
    if r > 1:
        cfg["l2"] = ("inputs larger than L2: %d distinct input sets (activations and weight codes, %d MB) "
                     "cycled step to step, steps back to back, no flush" % (r, ring_bytes(name) // 10**6))
    else:
        cfg["l2"] = ("inputs larger than L2 (%d MB read per step), steps back to back, no flush"
                     % (ring_bytes(name) // 10**6))
    cfg["timing"] = ("K steps between one event pair (max over ranks); per-kernel averages from K launches "
                     "of each kernel alone over the same inputs")
    if args.workload == "all" and name == HEADLINE:
        cfg["also_measured"] = list(ALSO_MEASURED)
    return cfg


def run_reference(args, world, rank):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    K = args.steps
    name = HEADLINE if args.workload == "all" else args.workload
    # each step a bounded sample: about sample_rows() rows in all, split over
    # the K steps, so that the whole run stays within a few minutes
    rows = max(min_rows(name), sample_rows(name) // max(K, 1))
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_sample(name, rows)
    rates, secs = [], 0.0
    for _ in range(K):
        gbs, tops, s, desc = oracle_sample(name, rows)
        rates.append(gbs)
        secs += s
    v = float(len(rates) / np.sum(1.0 / np.array(rates)))  # the rate over all steps' bytes (equal per step)
    out = {
        "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / K, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
        "config": workload_config(args, name),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
