"""Time the routing prep of the grouped form on the GPU.

    python -m weight_only_int4_a16w4_b200.profile_moe [T] [E] [K] [N] [topk ...]

For the grouped workload's shape (default T=4096 tokens, E=8 experts,
K=4096, N=14336, g=128) and each topk: the expert grouping, the row gather,
the gate-weighted un-permute, and the whole routed matmul next to the plain
grouped matmul on pre-sorted rows (both variants).  Every number is the mean
of a CUDA graph of repeated calls between two events on the capture stream.
Inputs are seeded and synthetic: router ids uniform over the experts, gate
weights uniform in [0, 1), x ~ N(0, 1) fp16, weights uniform int4.
"""
import sys

import numpy as np


def _graph_us(torch, fn, reps):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                fn()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def main(argv):
    import torch

    import weight_only_int4_a16w4_b200 as w4
    from inputs import draw_scale, draw_w, draw_x, pack_int4

    args = [int(a) for a in argv]
    T, E, K, N = (args + [4096, 8, 4096, 14336][len(args):])[:4]
    topks = args[4:] or [1, 2]
    g = 128
    rng = np.random.Generator(np.random.PCG64(20260))
    x = torch.from_numpy(draw_x(rng, T, K)).cuda()
    wp = [w4.repack(torch.from_numpy(pack_int4(draw_w(rng, K, N))).cuda(), K, N) for _ in range(E)]
    sc = [torch.from_numpy(draw_scale(rng, K // g, N)).cuda() for _ in range(E)]
    print(f"routing prep, T={T} E={E} K={K} N={N} g={g} (us per call)")
    print("| topk | align | gather | combine | routed MSD | grouped MSD | routed dequant | grouped dequant |")
    print("|---|---|---|---|---|---|---|---|")
    for topk in topks:
        rows = T * topk
        ids = torch.from_numpy(rng.integers(0, E, (T, topk)).astype(np.int32)).cuda()
        wts = torch.from_numpy(rng.uniform(0, 1, (T, topk)).astype(np.float32)).cuda()
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        st = torch.empty(rows, dtype=torch.int32, device="cuda")
        inv = torch.empty(rows, dtype=torch.int32, device="cuda")
        hdr = torch.zeros(256, dtype=torch.uint8, device="cuda")
        xs = torch.empty((rows, K), dtype=torch.float16, device="cuda")
        ys = torch.zeros((rows, N), dtype=torch.float16, device="cuda")
        y = torch.empty((T, N), dtype=torch.float16, device="cuda")
        t_align = _graph_us(torch, lambda: w4.w4a16_moe_align(ids, T, topk, E, offsets, st, inv, hdr), 50)
        t_gather = _graph_us(torch, lambda: w4.w4a16_moe_gather(x, st, rows, K, xs), 20)
        t_comb = _graph_us(torch, lambda: w4.w4a16_moe_combine(ys, inv, wts, T, topk, N, y), 20)
        res = []
        for op in (w4.OP_MSD, w4.OP_DEQUANT):
            ws = torch.zeros(w4.w4a16_moe_workspace_size(op, T, topk, K, N, g, E), dtype=torch.uint8, device="cuda")
            gws = w4.alloc_workspace(op, rows, K, N, g, E=E)
            routed = _graph_us(torch, lambda: w4.w4a16_moe_matmul(op, x, ids, wts, wp, sc, E, T, topk, K, N, g, y,
                                                                  ws), 5)
            grouped = _graph_us(torch, lambda: w4.w4a16_grouped_matmul(op, xs, wp, sc, offsets, E, rows, K, N, g,
                                                                       ys, gws), 5)
            if w4.w4a16_read_status(ws) or w4.w4a16_read_status(gws):
                raise SystemExit("device status set")
            res += [routed, grouped]
        print(f"| {topk} | {t_align:.2f} | {t_gather:.2f} | {t_comb:.2f} | {res[0]:.1f} | {res[1]:.1f} | "
              f"{res[2]:.1f} | {res[3]:.1f} |")


if __name__ == "__main__":
    main(sys.argv[1:])
