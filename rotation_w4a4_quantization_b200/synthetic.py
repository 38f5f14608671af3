"""Seeded synthetic inputs shaped like the article's layer inputs.

This module only draws random tensors; it holds none of the rotation or
quantization arithmetic.  Both the parity tests (CUDA path vs. the CPU oracle)
and the benchmark take their inputs from here.

The article ("Rotations for 4-Bit Activations: QuaRot, SpinQuant, and
Friends") measures Qwen3-8B q_proj and down_proj inputs: q_proj has outliers in
fixed channels, down_proj spikes a different channel on different tokens
(opening section and section "A rotation changes nothing, and that is the
point").  Those layers are not available, so these stand-ins reproduce the
shapes and the outlier structure:

* ``tiny_int4``      X 64x512 ~ N(0,1), channels {3, 77, 200, 411} x50;
                     W 256x512 ~ N(0, 0.02^2); 128-wide blocks; INT4.
* ``q_proj_int4``    X 2048x4096 ~ N(0,1), 8 fixed channels (a seeded
                     permutation) each scaled by a fixed factor ~ U[20, 60] on
                     every token; W 4096x4096 ~ N(0, 0.02^2); full-width; INT4.
* ``down_proj_int4`` X 4096x12288 ~ N(0,1); on every token one uniformly
                     drawn channel gets + (Laplace(0, 40) + 30);
                     W 4096x12288 ~ N(0, 0.02^2); 128-wide blocks; INT4.
* ``q_proj_nvfp4``   X, W as q_proj_int4; 128-wide blocks; NVFP4.
* ``kv4``            K, V [16, 32, 4096, 128] ~ N(0,1) with 2 fixed dims per
                     head (seeded, shared over batch and sequence) x30;
                     Hadamard over head_dim 128.

Seeds: data 1000 + i, signs 2000 + i, outlier placement 3000 + i, with i the
workload's index (1..5).  ``rows`` / ``batch`` overrides draw a smaller case of
the same recipe (the first rows of the same distribution, not of the same
tensor).
"""

import torch

WORKLOADS = {
    "tiny_int4": dict(index=1, M=64, K=512, N=256, block=128, fmt="int4"),
    "q_proj_int4": dict(index=2, M=2048, K=4096, N=4096, block=0, fmt="int4"),
    "down_proj_int4": dict(index=3, M=4096, K=12288, N=4096, block=128, fmt="int4"),
    "q_proj_nvfp4": dict(index=4, M=2048, K=4096, N=4096, block=128, fmt="nvfp4"),
    "kv4": dict(index=5, B=16, H=32, S=4096, D=128),
    "q_proj_mxfp4": dict(index=6, M=2048, K=4096, N=4096, block=128, fmt="mxfp4"),
    # a decode step over the kv4 workload's cache (written once by the KV4 kernel)
    "kv4_decode": dict(index=7, B=16, H=32, S=4096, D=128),
    # 8-bit activations: W4A8 (4-bit weights) and W8A8, q_proj shapes and recipe
    "q_proj_w4a8": dict(index=8, M=2048, K=4096, N=4096, block=0, fmt="int8", wfmt="int4"),
    "q_proj_w8a8": dict(index=9, M=2048, K=4096, N=4096, block=0, fmt="int8", wfmt="int8"),
    # format-sized block rotations: one block per NVFP4 (16) or MXFP4 (32) scale group
    "q_proj_nvfp4_b16": dict(index=10, M=2048, K=4096, N=4096, block=16, fmt="nvfp4"),
    "q_proj_mxfp4_b32": dict(index=11, M=2048, K=4096, N=4096, block=32, fmt="mxfp4"),
    # per-group (128) asymmetric INT4 of the activations (quantizer only: no GEMM consumes it)
    "q_proj_int4_asym": dict(index=12, M=2048, K=4096, N=4096, block=128, fmt="int4_asym"),
}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def signs(k, seed, device="cpu"):
    """+-1 int8 vector of length k (one random sign per channel)."""
    g = _gen(seed, device)
    return (torch.randint(0, 2, (k,), generator=g, device=device, dtype=torch.int8) * 2 - 1).to(torch.int8)


def workload_signs(name, device="cpu"):
    w = WORKLOADS[name]
    k = w["D"] if "D" in w else w["K"]
    return signs(k, 2000 + w["index"], device)


def activations(name, rows=None, device="cpu", seed_offset=0):
    """X [rows, K] bf16 for a GEMM workload."""
    w = WORKLOADS[name]
    m = w["M"] if rows is None else rows
    k = w["K"]
    g = _gen(1000 + w["index"] + seed_offset, device)
    x = torch.randn((m, k), generator=g, device=device, dtype=torch.float32)
    if name == "tiny_int4":
        x[:, [3, 77, 200, 411]] *= 50.0
    elif name.startswith("q_proj"):
        gp = _gen(3000 + w["index"], "cpu")
        ch = torch.randperm(k, generator=gp)[:8]
        mult = 20.0 + 40.0 * torch.rand((8,), generator=gp, dtype=torch.float64)
        x[:, ch.to(device)] *= mult.to(device=device, dtype=torch.float32)
    elif name == "down_proj_int4":
        gp = _gen(3000 + w["index"] + seed_offset, device)
        ch = torch.randint(0, k, (m,), generator=gp, device=device)
        u = torch.rand((m,), generator=gp, device=device, dtype=torch.float64) - 0.5
        lap = -40.0 * torch.sign(u) * torch.log1p(-2.0 * u.abs())   # Laplace(0, 40) by inverse CDF
        spike = (lap + 30.0).to(torch.float32)
        x[torch.arange(m, device=device), ch] += spike
    return x.to(torch.bfloat16)


def weights(name, rows=None, device="cpu"):
    """W [N, K] bf16 ~ N(0, 0.02^2)."""
    w = WORKLOADS[name]
    n = w["N"] if rows is None else rows
    g = _gen(1500 + w["index"], device)
    return (0.02 * torch.randn((n, w["K"]), generator=g, device=device, dtype=torch.float32)).to(torch.bfloat16)


def kv(batch=None, heads=None, seq=None, device="cpu", which=0, seed_offset=0):
    """K (which=0) or V (which=1) [B, H, S, 128] bf16 with 2 outlier dims per head x30."""
    w = WORKLOADS["kv4"]
    b = w["B"] if batch is None else batch
    h = w["H"] if heads is None else heads
    s = w["S"] if seq is None else seq
    d = w["D"]
    g = _gen(1000 + w["index"] + 17 * which + seed_offset, device)
    t = torch.randn((b, h, s, d), generator=g, device=device, dtype=torch.float32)
    gp = _gen(3000 + w["index"] + 17 * which, "cpu")
    mult = torch.ones((h, d), dtype=torch.float32)
    for hh in range(h):
        dims = torch.randperm(d, generator=gp)[:2]
        mult[hh, dims] = 30.0
    t *= mult.to(device)[None, :, None, :]
    return t.to(torch.bfloat16)


def stated_recipe():
    """One line per workload, for reports."""
    return {k: dict(v) for k, v in WORKLOADS.items()}


__all__ = ["WORKLOADS", "signs", "workload_signs", "activations", "weights", "kv", "stated_recipe"]
