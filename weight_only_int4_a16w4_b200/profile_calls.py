"""A few calls of each variant on one of the seeded workloads, for profilers.

    python -m weight_only_int4_a16w4_b200.profile_calls [workload] [calls]

Runs `calls` MSD matmuls, then `calls` dequant matmuls (default 4 each) on
the workload's inputs, rotating over `calls` copies of the packed weights,
and checks the device status word.  Every launch is the library's own.
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
    c = make_workload(name)
    if c.E != 1:
        raise SystemExit("profile_calls runs the dense workloads")
    x = torch.from_numpy(c.x).cuda()
    sc = torch.from_numpy(c.scale[0]).cuda()
    wl = torch.from_numpy(c.wp[0]).cuda()
    wp = [w4.repack(wl, c.K, c.N) for _ in range(calls)]
    y = torch.empty((c.M, c.N), dtype=torch.float16, device="cuda")
    for op in (w4.OP_MSD, w4.OP_DEQUANT):
        ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g)
        fn = w4.w4a16_msd_matmul if op == w4.OP_MSD else w4.w4a16_dequant_matmul
        for i in range(calls):
            fn(x, wp[i], sc, c.M, c.K, c.N, c.g, y, ws)
        torch.cuda.synchronize()
        if w4.w4a16_read_status(ws) != 0:
            raise SystemExit("device wait timed out")
    print("ok")


if __name__ == "__main__":
    main()
