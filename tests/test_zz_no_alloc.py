"""The allocation-free MSD entry point, for callers that cannot obtain device
scratch memory (for example a plug-in inside a host program whose memory pool
owns the whole GPU, or a latency-critical path that cannot afford cudaMalloc's
implicit synchronisation).  Its scratch is an array the library keeps in
device memory.  Through the C ABI this checks, on two calls in a row, that
its result is bit-identical to the workspace-taking entry point's (the same
kernels on the same inputs, so any difference -- a stale digit from the
previous call, a timed-out wait leaving rows unwritten -- shows) and within
the MSD tolerance of the CPU oracle, and that it refuses problems whose
scratch would not fit.

This file is collected last on purpose: the array is shared process-wide,
and the test must pass both on its own and after every other test.
"""
import numpy as np
import pytest

import oracle
from inputs import make_case

pytestmark = pytest.mark.gpu

MSD_REL, MSD_ABS = 2e-3, 1e-3


def _run_pair(w4, torch, c, dev):
    """(no-alloc result, workspace-entry result) for one case, both fp16."""
    x, wp, sc = dev
    y_ref = torch.full((c.M, c.N), float("nan"), dtype=torch.float16, device="cuda")
    ws = w4.alloc_workspace(w4.OP_MSD, c.M, c.K, c.N, c.g)
    w4.w4a16_msd_matmul(x, wp, sc, c.M, c.K, c.N, c.g, y_ref, ws)
    y = torch.full((c.M, c.N), float("nan"), dtype=torch.float16, device="cuda")
    w4.w4a16_msd_matmul_noalloc(x, wp, sc, c.M, c.K, c.N, c.g, y)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return y.cpu().numpy(), y_ref.cpu().numpy()


@pytest.mark.parametrize("M,K,N,g", [(1, 4096, 4096, 128), (16, 2048, 1536, 64), (40, 512, 264, 128)])
def test_noalloc_matches_workspace_entry_and_oracle_twice(cuda_lib, M, K, N, g):
    import torch
    w4 = cuda_lib
    for call in range(2):                       # two calls in a row share the array
        c = make_case(M, K, N, g, seed=9000 + 17 * call + M)
        dev = (torch.from_numpy(c.x).cuda(), w4.repack(torch.from_numpy(c.wp[0]).cuda(), K, N),
               torch.from_numpy(c.scale[0]).cuda())
        y, y_ref = _run_pair(w4, torch, c, dev)
        assert np.all(np.isfinite(y.astype(np.float64))), f"call {call}: unwritten or non-finite outputs"
        assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16)), \
            f"call {call}: {int((y.view(np.uint16) != y_ref.view(np.uint16)).sum())} outputs differ from the " \
            "workspace entry point"
        # sampled columns of the oracle (every row, a spread of columns incl. the last)
        cols = np.unique(np.concatenate([np.arange(0, N, max(1, N // 24)), [N - 1]]))
        ref = oracle.msd(c.x, c.wp[0][:, cols], c.scale[0][:, cols], g)
        tol = MSD_REL * np.abs(ref).max() + MSD_ABS
        err = np.abs(y[:, cols].astype(np.float64) - ref).max()
        assert err <= tol, f"call {call}: max error {err:.3e} against the oracle > {tol:.3e}"


def test_noalloc_rejects_oversized_problem(cuda_lib):
    w4 = cuda_lib
    fake = 1 << 40                              # never dereferenced: the size check comes first
    need = w4.w4a16_workspace_size(w4.OP_MSD, 4096, 4096, 4096, 128)
    assert need > w4.NOALLOC_SCRATCH_BYTES
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_msd_matmul_noalloc(fake, fake, fake, 4096, 4096, 4096, 128, fake, stream=0)
    assert e.value.code == 3                    # W4A16_ERR_WORKSPACE
