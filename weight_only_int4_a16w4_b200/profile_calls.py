"""A few calls of each variant on one of the seeded workloads, for profilers.

    python -m weight_only_int4_a16w4_b200.profile_calls [workload] [calls] [variant ...]

Runs `calls` matmuls of each variant in turn (default 4 each; variants msd,
dequant, bf16, msd2, msd4; default msd then dequant) on the workload's
inputs, rotating over `calls` copies of the packed weights, and checks the
device status word.  Every launch is the library's own.  bf16 uses the same
distributions encoded as bf16; msd2 / msd4 are MSD with 2 / 4 unfold steps.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    import torch
    import weight_only_int4_a16w4_b200 as w4
    from inputs import make_workload
    name = argv[0] if argv else "decode_m1"
    calls = int(argv[1]) if len(argv) > 1 else 4
    variants = argv[2:] or ["msd", "dequant"]
    c = make_workload(name)
    if c.E != 1:
        raise SystemExit("profile_calls runs the dense workloads")
    wl = torch.from_numpy(c.wp[0]).cuda()
    wp = [w4.repack(wl, c.K, c.N) for _ in range(calls)]
    for v in variants:
        if v == "bf16":
            cb = make_workload(name, act="bf16")
            x = torch.from_numpy(cb.x.view("int16")).cuda().view(torch.bfloat16)
            sc = torch.from_numpy(cb.scale[0].view("int16")).cuda().view(torch.bfloat16)
            y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
        else:
            x = torch.from_numpy(c.x).cuda()
            sc = torch.from_numpy(c.scale[0]).cuda()
            y = torch.empty((c.M, c.N), dtype=torch.float16, device="cuda")
        op = {"msd": w4.OP_MSD, "dequant": w4.OP_DEQUANT, "bf16": w4.OP_DEQUANT_BF16,
              "msd2": w4.OP_MSD_2STEP, "msd4": w4.OP_MSD_4STEP}[v]
        ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g)
        for i in range(calls):
            if v in ("msd2", "msd4"):
                w4.w4a16_msd_matmul_steps(2 if v == "msd2" else 4, x, wp[i], sc, c.M, c.K, c.N, c.g, y, ws)
            else:
                fn = {"msd": w4.w4a16_msd_matmul, "dequant": w4.w4a16_dequant_matmul,
                      "bf16": w4.w4a16_dequant_matmul_bf16}[v]
                fn(x, wp[i], sc, c.M, c.K, c.N, c.g, y, ws)
        torch.cuda.synchronize()
        if w4.w4a16_read_status(ws) != 0:
            raise SystemExit("device wait timed out")
    print("ok")


if __name__ == "__main__":
    main()
