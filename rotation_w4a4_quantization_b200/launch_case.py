"""Launch one kernel of a synthetic workload a few times, for a profiler capture.

    python -m rotation_w4a4_quantization_b200.launch_case rotate <workload> [reps]
    python -m rotation_w4a4_quantization_b200.launch_case gemm <workload> [reps]
    python -m rotation_w4a4_quantization_b200.launch_case gemm_bytes <workload> [reps]
    python -m rotation_w4a4_quantization_b200.launch_case attention kv4_decode [reps]

Each call builds the workload's inputs on cuda:0 (the rotations' inputs are
made by the package's own kernels where a cache or codes are needed) and
launches the named step `reps` times, so that a capture can skip the first
launch (`-s 1 -c 1`).  `gemm_bytes` is the INT4 workloads' GEMM with the
weights' codes stored one per byte (RQ_INT4_BYTES).  The KV4 cases use a quarter of the batch (B = 4): each
tensor is then still above the 126 MB L2 but the capture stays small.
"""

import sys

import torch

from . import rq
from . import synthetic as syn


def main(argv):
    kind, name = argv[0], argv[1]
    reps = int(argv[2]) if len(argv) > 2 else 3
    rq.init(0)
    c = syn.WORKLOADS[name]
    s = syn.workload_signs(name).cuda()
    if kind == "rotate" and name == "kv4":
        kv = syn.kv(batch=4, heads=c["H"], seq=c["S"], device="cuda")
        for _ in range(reps):
            rq.kv_rotate_quantize(kv, s)
    elif kind == "rotate":
        x = syn.activations(name, device="cuda")
        for _ in range(reps):
            rq.rotate_quantize(x, s, c["block"], c["fmt"])
    elif kind == "gemm":
        x = syn.activations(name, device="cuda")
        w = syn.weights(name, device="cuda")
        wfmt = c.get("wfmt", c["fmt"])
        wq = rq.prepare_weights(w, s, c["block"], wfmt)
        xq = rq.rotate_quantize(x, s, c["block"], c["fmt"])
        y = torch.empty((c["M"], c["N"]), dtype=torch.bfloat16, device="cuda")
        for _ in range(reps):
            if c["fmt"] in ("int8", "int6"):
                rq.int_gemm(xq, c["fmt"], wq, wfmt, "bf16", y=y)
            else:
                rq.w4a4_gemm(xq, wq, c["fmt"], "bf16", y=y)
    elif kind == "gemm_bytes":
        x = syn.activations(name, device="cuda")
        w = syn.weights(name, device="cuda")
        wq = rq.prepare_weights(w, s, c["block"], "int4_bytes")
        xq = rq.rotate_quantize(x, s, c["block"], "int4")
        y = torch.empty((c["M"], c["N"]), dtype=torch.bfloat16, device="cuda")
        for _ in range(reps):
            rq.int_gemm(xq, "int4", wq, "int4_bytes", "bf16", y=y)
    elif kind == "attention":
        kc = rq.kv_rotate_quantize(syn.kv(batch=4, device="cuda", which=0), s)
        vc = rq.kv_rotate_quantize(syn.kv(batch=4, device="cuda", which=1), s)
        g = torch.Generator(device="cuda")
        g.manual_seed(4000 + c["index"])
        q = torch.randn((4, c["H"], c["D"]), generator=g, device="cuda").to(torch.bfloat16)
        for _ in range(reps):
            rq.kv4_decode_attention(q, kc, vc, s)
    else:
        raise SystemExit("unknown kind %r" % kind)
    torch.cuda.synchronize()
    rq.get_device_error()
    print("ok", kind, name)


if __name__ == "__main__":
    main(sys.argv[1:])
