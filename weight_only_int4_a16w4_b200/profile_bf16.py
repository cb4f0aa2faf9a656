"""Time the dequant variant with bf16 activations next to the fp16 one.

    python -m weight_only_int4_a16w4_b200.profile_bf16 [workload ...]

For each named workload (default: decode_m1 decode_m16 prefill moe_e8) the
fp16 dequant call and the bf16 dequant call on the same shapes, each the mean
of a CUDA graph of repeated calls between two events on the capture stream
(weights re-read from HBM every call: they exceed L2 except at decode_m1,
where consecutive calls alternate between two weight copies).  Prints us per
call, the weight-stream rate (packed bytes / time) and the dense rate
(2 M N K / time).  Inputs are the seeded synthetic workloads of ``inputs``
(bf16: the same distributions encoded as bf16).
"""
import sys

import numpy as np


def _graph_us(torch, fns, reps):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for f in fns:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                for f in fns:
                    f()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (reps * len(fns))


def _bf16(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def main(argv):
    import torch

    import weight_only_int4_a16w4_b200 as w4
    from inputs import make_workload, workload

    names = argv or ["decode_m1", "decode_m16", "prefill", "moe_e8"]
    print("| workload | fp16 dequant us | bf16 dequant us | bf16 GB/s (weights) | bf16 TFLOP/s |")
    print("|---|---|---|---|---|")
    for name in names:
        wl = workload(name)
        row = []
        for act in ("fp16", "bf16"):
            c = make_workload(name, act=act)
            op = w4.OP_DEQUANT_BF16 if act == "bf16" else w4.OP_DEQUANT
            up = (lambda a: _bf16(torch, a)) if act == "bf16" else (lambda a: torch.from_numpy(a).cuda())
            ydt = torch.bfloat16 if act == "bf16" else torch.float16
            x = up(c.x)
            copies = 2 if name == "decode_m1" else 1
            wp = [[w4.repack(torch.from_numpy(p).cuda(), c.K, c.N) for p in c.wp] for _ in range(copies)]
            sc = [up(s) for s in c.scale]
            y = torch.empty((c.M, c.N), dtype=ydt, device="cuda")
            ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g, E=c.E)
            if c.E > 1:
                off = torch.from_numpy(c.offsets).cuda()
                fns = [lambda wpi=wpi: w4.w4a16_grouped_matmul(op, x, wpi, sc, off, c.E, c.M, c.K, c.N, c.g, y, ws)
                       for wpi in wp]
            else:
                fn = w4.w4a16_dequant_matmul_bf16 if act == "bf16" else w4.w4a16_dequant_matmul
                fns = [lambda wpi=wpi: fn(x, wpi[0], sc[0], c.M, c.K, c.N, c.g, y, ws) for wpi in wp]
            reps = 200 if c.M * c.N * c.K < (1 << 36) else 10
            row.append(_graph_us(torch, fns, reps))
            if w4.w4a16_read_status(ws):
                raise SystemExit("device status set")
        us = row[1]
        wbytes = wl.E * wl.K * wl.N / 2
        flops = 2.0 * wl.M * wl.N * wl.K
        print(f"| {name} | {row[0]:.2f} | {us:.2f} | {wbytes / us / 1e3:.0f} | {flops / us / 1e6:.1f} |")


if __name__ == "__main__":
    main(sys.argv[1:])
