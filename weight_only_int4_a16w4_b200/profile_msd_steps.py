"""Time MSD with 2, 3 and 4 unfold steps on the workloads.

    python -m weight_only_int4_a16w4_b200.profile_msd_steps [workload ...]

For each named workload (default: decode_m1 decode_m16 prefill moe_e8) the
MSD call with S = 2, 3 and 4 digit planes, each the mean of a CUDA graph of
repeated calls between two events on the capture stream (decode_m1 alternates
two weight copies so that the weights come from HBM).  Prints us per call
and the useful rate 2 M N K / time.  Inputs are the seeded synthetic
workloads of ``inputs``.
"""
import sys

from weight_only_int4_a16w4_b200.profile_bf16 import _graph_us

OPS = {2: 3, 3: 0, 4: 4}      # steps -> W4A16_OP_* code


def main(argv):
    import torch

    import weight_only_int4_a16w4_b200 as w4
    from inputs import make_workload, workload

    names = argv or ["decode_m1", "decode_m16", "prefill", "moe_e8"]
    print("| workload | S=2 us | S=3 us | S=4 us | S=2 / S=3 / S=4 TFLOP/s (2MNK) |")
    print("|---|---|---|---|---|")
    for name in names:
        wl = workload(name)
        c = make_workload(name)
        x = torch.from_numpy(c.x).cuda()
        copies = 2 if name == "decode_m1" else 1
        wp = [[w4.repack(torch.from_numpy(p).cuda(), c.K, c.N) for p in c.wp] for _ in range(copies)]
        sc = [torch.from_numpy(s).cuda() for s in c.scale]
        y = torch.empty((c.M, c.N), dtype=torch.float16, device="cuda")
        off = torch.from_numpy(c.offsets).cuda() if c.E > 1 else None
        us = []
        for S in (2, 3, 4):
            op = OPS[S]
            ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g, E=c.E)
            if c.E > 1:
                fns = [lambda wpi=wpi, op=op, ws=ws: w4.w4a16_grouped_matmul(op, x, wpi, sc, off, c.E, c.M, c.K, c.N,
                                                                             c.g, y, ws) for wpi in wp]
            else:
                fns = [lambda wpi=wpi, S=S, ws=ws: w4.w4a16_msd_matmul_steps(S, x, wpi[0], sc[0], c.M, c.K, c.N, c.g,
                                                                             y, ws) for wpi in wp]
            reps = 200 if c.M * c.N * c.K < (1 << 36) else 10
            us.append(_graph_us(torch, fns, reps))
            if w4.w4a16_read_status(ws):
                raise SystemExit("device status set")
        fl = 2.0 * wl.M * wl.N * wl.K
        rates = " / ".join(f"{fl / u / 1e6:.1f}" for u in us)
        print(f"| {name} | {us[0]:.2f} | {us[1]:.2f} | {us[2]:.2f} | {rates} |")


if __name__ == "__main__":
    main(sys.argv[1:])
