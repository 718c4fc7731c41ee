"""dllm_mask_compact_noalloc: the compaction entry point for callers that cannot allocate.

Some callers cannot give the library a workspace: an engine whose memory planner owns all
of HBM and forbids side allocations, or a plugin that must not call cudaMalloc because it
can synchronise the whole device.  dllm_mask_compact_noalloc keeps its scratch (the
per-tile mask counts) in a fixed static device array instead.  Its output must be exactly
that of dllm_mask_compact, call after call, although every call reuses the same scratch.
"""
import ctypes

import pytest
import torch

from mask_only_logits_b200 import _abi, build


def _compact_both(dl, M):
    """Run the allocation-free entry point and the workspace one on the same mask."""
    B, L = M.shape
    n = B * L
    outs = []
    for noalloc in (True, False):
        row_idx = torch.full((n,), -3, dtype=torch.int32, device="cuda")
        seq_off = torch.full((B + 1,), -3, dtype=torch.int32, device="cuda")
        count = torch.full((4,), -3, dtype=torch.int32, device="cuda")
        if noalloc:
            dl.mask_compact_noalloc(M, row_idx, seq_off, count)
        else:
            ws = torch.empty(dl.workspace_bytes(B, L, 64, 1), dtype=torch.uint8, device="cuda")
            dl.mask_compact(M, row_idx, seq_off, count, ws)
        assert dl.get_status() == 0
        outs.append((row_idx, seq_off, count))
    return outs


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_only_logits_b200 as dl
    g = torch.Generator(device="cuda").manual_seed(0)
    # first call: the largest input the fixed scratch allows (every scratch slot in use);
    # second call: a small ragged input, so slots written by the first call stay stale
    masks = [
        (torch.rand(2, 1 << 26, generator=g, device="cuda") < 0.01).to(torch.uint8),
        (torch.rand(3, 7001, generator=g, device="cuda") < 0.4).to(torch.uint8),
    ]
    assert masks[0].numel() == 16384 * 8192
    for M in masks:
        (r0, s0, c0), (r1, s1, c1) = _compact_both(dl, M)
        # integer outputs: bit-exact, including the untouched entries past count
        assert int(c0[0]) == int(c1[0]) == int((M != 0).sum())
        assert torch.equal(s0, s1)
        assert torch.equal(r0, r1)


def test_noalloc_rejects_oversize_before_launch():
    """Sizes beyond the fixed scratch fail with DLLM_ERR_SCRATCH (-9) on the host; no GPU
    work is enqueued, so this runs without a GPU too."""
    build.build()
    lib = _abi.load()
    a = ctypes.c_void_p(1 << 20)             # aligned fake addresses: never dereferenced
    nul = ctypes.c_void_p(None)
    assert lib.dllm_mask_compact_noalloc(a, 2, (1 << 26) + 1, a, a, a, nul) == -9
    assert lib.dllm_mask_compact_noalloc(a, 16385, 8192, a, a, a, nul) == -9
    assert lib.dllm_status_string(-9) == \
        b"B*L exceeds the fixed scratch of the allocation-free entry point"
    assert lib.dllm_mask_compact_noalloc(nul, 2, 16, a, a, a, nul) == -1
    assert lib.dllm_mask_compact_noalloc(a, 0, 16, a, a, a, nul) == -3
