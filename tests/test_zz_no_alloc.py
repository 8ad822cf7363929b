"""sparse_attn_plan_noalloc: the plan call for callers that cannot allocate device
memory (a runtime that reserves its whole budget up front, a plugin whose host
owns the allocator, a latency-critical path that must not call cudaMalloc).

Called through the C ABI and compared with sparse_attn_plan (which takes a
caller-allocated workspace) on two calls in a row with different inputs: the
masks, counts, kept lists and tile pairs must be identical (same kernels, same
arithmetic, deterministic pairing). Kept in its own
file, collected last."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from free_block_sparse_mean_b200 import _lib
    from free_block_sparse_mean_b200 import workloads as wl
    from free_block_sparse_mean_b200._lib import SaShape


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(B, H, Nb, tiles, dev):
    return (torch.empty((B, H, Nb, Nb), dtype=torch.uint8, device=dev),
            torch.empty((B, H, Nb), dtype=torch.int32, device=dev),
            torch.full((B, H, Nb, Nb), -1, dtype=torch.int32, device=dev),
            torch.empty((2 * tiles,), dtype=torch.int32, device=dev))


def test_noalloc_plan_matches_workspace_plan_twice():
    lib = _lib.load()
    dev = torch.device("cuda:0")
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    # Nb = 47 and 18 (64-block score tiles), 313 and 3125 blocks, all within the fixed
    # scratch; at Nb = 3125 the two calls compute and select the score strips in
    # different batch counts (the workspace holds 40 strips, the fixed scratch about
    # 14), which must not change any output
    cases = [(1, 4, 3000, 128, False, 0.95, 1), (2, 3, 1100, 64, True, 0.9, 2),
             (1, 2, 20000, 64, False, 0.9, 3), (1, 2, 200000, 64, False, 0.95, 4)]
    for B, H, N, d, causal, tau, seed in cases:
        q, k, _ = wl.random_qkv(B, H, N, d, seed=seed, device=dev, scale_qk=2.0)
        s = SaShape(B, H, N, d, 64)
        Nb = -(-N // 64)
        tiles = int(lib.sparse_attn_num_tiles(s))
        scale = d ** -0.5
        ref = _outputs(B, H, Nb, tiles, dev)
        ws_bytes = int(lib.sparse_attn_plan_workspace_size(s))
        ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
        st = lib.sparse_attn_plan(_p(q), _p(k), s, tau, scale, int(causal), *(_p(t) for t in ref),
                                  _p(ws), ws_bytes, stream)
        assert st == 0, lib.sparse_attn_status_string(st)
        got = _outputs(B, H, Nb, tiles, dev)
        st = lib.sparse_attn_plan_noalloc(_p(q), _p(k), s, tau, scale, int(causal), *(_p(t) for t in got),
                                          stream)
        assert st == 0, lib.sparse_attn_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0])                       # mask
        assert torch.equal(got[1], ref[1])                       # count
        ri, gi = ref[2].reshape(-1, Nb).cpu().numpy(), got[2].reshape(-1, Nb).cpu().numpy()
        for r, c in enumerate(ref[1].reshape(-1).cpu().numpy()):
            np.testing.assert_array_equal(gi[r, :c], ri[r, :c])        # ascending kept lists
        assert torch.equal(got[3], ref[3])                       # tile pairs (deterministic)


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib.load()
    dev = torch.device("cuda:0")
    q = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device=dev)
    out = _outputs(1, 1, 1, 1, dev)
    big = SaShape(1, 40, 75600, 128, 64)     # needs about 50 MB of scratch > 32 MiB
    st = lib.sparse_attn_plan_noalloc(_p(q), _p(q), big, 0.9, 0.1, 0, *(_p(t) for t in out), None)
    assert st == 3                          # SA_ERR_WORKSPACE, nothing launched
