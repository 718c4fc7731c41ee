"""The virtual-memory arena and workspaces sized for a known masked count, on the GPU.

* An Arena maps, grows and shrinks its backing in whole chunks at one fixed address; the
  device's free memory follows the mapped size.
* Decode steps whose workspace lives in an arena mapped for each step's own masked count
  (Mosaic page, Fig. 4: reserved memory against the theoretical peak) select exactly what
  steps on the full fixed workspace select, across a mask-ratio sweep that shrinks and
  grows the mapping, and through host inputs.
* A workspace sized for fewer rows than the mask holds computes the rows it can hold,
  reports DLLM_ERR_CAPACITY and writes nothing past its end (a guard region checks it).
"""
import numpy as np
import pytest
import torch

import workloads as WL

pytestmark = pytest.mark.gpu

MiB = 1 << 20


@pytest.fixture(scope="module")
def dl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_only_logits_b200 as m
    return m


def test_arena_maps_grows_and_shrinks(dl):
    # load the torch kernels used below first: a kernel module loaded lazily on its first
    # launch takes device memory of its own and would show up in the free-memory deltas
    w = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    w.fill_(0x5A)
    w[-4096:] = 3
    assert int(w[12345]) == 0x5A
    del w
    a = dl.Arena(512 * MiB)
    try:
        chunk = a.chunk
        assert chunk >= 2 * MiB and chunk % (2 * MiB) == 0
        assert a.reserved >= 512 * MiB and a.mapped == 0 and a.ptr % 256 == 0
        base = a.ptr
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        assert a.map(100 * MiB + 1) == -(-(100 * MiB + 1) // chunk) * chunk
        free1, _ = torch.cuda.mem_get_info()
        assert abs((free0 - free1) - a.mapped) <= 8 * MiB, (free0 - free1, a.mapped)
        t = a.tensor()
        assert t.numel() == a.mapped and t.data_ptr() == base and t.is_cuda
        t.fill_(0x5A)
        t[-1] = 7
        torch.cuda.synchronize()
        assert int(t[12345]) == 0x5A and int(t[-1]) == 7
        # shrink: the first chunks keep their contents and the address is unchanged
        a.map(10 * MiB)
        assert a.mapped == -(-10 * MiB // chunk) * chunk and a.ptr == base
        assert int(a.tensor()[12345]) == 0x5A
        # the released chunks are back on the device's free list
        free2, _ = torch.cuda.mem_get_info()
        assert abs((free0 - free2) - a.mapped) <= 8 * MiB, (free0 - free2, a.mapped)
        # grow again past the old end: the device footprint is the mapped total (nothing
        # leaks across a shrink)
        a.map(300 * MiB)
        v = a.tensor()
        v[-4096:] = 3
        torch.cuda.synchronize()
        assert int(v[-1]) == 3 and int(v[12345]) == 0x5A
        free4, _ = torch.cuda.mem_get_info()
        assert abs((free0 - free4) - a.mapped) <= 8 * MiB, (free0 - free4, a.mapped)
        with pytest.raises(dl.DllmError):
            a.map(a.reserved + 1)                        # past the reservation: refused
        assert a.mapped == -(-300 * MiB // chunk) * chunk
        a.map(0)
        assert a.mapped == 0
    finally:
        a.close()
    torch.cuda.synchronize()
    free3, _ = torch.cuda.mem_get_info()
    assert free3 >= free0 - 8 * MiB                      # all of it back once closed


def _inputs(cfg, seed):
    inp = WL.make_inputs(cfg, seed=seed)
    return inp, inp["H"].cuda(), inp["M"].cuda(), inp["W"].cuda()


def _same(a, b, keys=("tok", "conf", "lse")):
    c = int(a["count"][0])
    assert c == int(b["count"][0])
    for key in keys:
        assert torch.equal(a[key][:c], b[key][:c]), key
    assert torch.equal(a["row_idx"][:c], b["row_idx"][:c])
    assert torch.equal(a["idx"], b["idx"]) and torch.equal(a["n_sel"], b["n_sel"])


def test_steps_in_an_arena_sized_per_step_match_fixed_workspace(dl):
    """A mask-ratio sweep (0.9, 0.1, 0.5, 0.9, 0.3) through one arena: each step maps the
    workspace for its own masked count, shrinking and growing the backing, and selects
    exactly what a step on the full fixed workspace selects."""
    base = WL.custom_config(1, 16384, 512, 8192, 32, r=0.9)
    plain = dl.DecodeStep(base.B, base.L, base.d, base.V, base.k)
    st = dl.DecodeStep(base.B, base.L, base.d, base.V, base.k, arena=True)
    full = dl.workspace_bytes(base.B, base.L, base.d, base.V)
    try:
        W = None
        for i, r in enumerate((0.9, 0.1, 0.5, 0.9, 0.3)):
            cfg = WL.custom_config(1, 16384, 512, 8192, 32, r=r)
            inp, H, M, W_i = _inputs(cfg, seed=5)          # same W and H, nested masks
            W = W_i if W is None else W
            count = int(inp["M"].sum())
            ref = {k: v.clone() for k, v in plain.run(H, M, W).items()}
            out = st.run(H, M, W, max_rows=count)
            assert dl.get_status() == 0
            _same(out, ref)
            need = dl.workspace_bytes_rows(cfg.B, cfg.L, cfg.d, cfg.V, count)
            assert need <= st.arena.mapped < need + st.arena.chunk
            assert dl.workspace_rows(cfg.B, cfg.L, cfg.d, cfg.V, st.arena.mapped) >= count
            if r < 0.9:
                assert st.arena.mapped < 0.75 * full
    finally:
        st.arena.close()


@pytest.mark.parametrize("name", ["cfg0", "cfg1", "cfg4_block"])
def test_workload_steps_through_an_arena(dl, name):
    cfg = WL.CONFIGS[name]
    inp, H, M, W = _inputs(cfg, seed=0)
    lo = None if inp["win_lo"] is None else torch.from_numpy(inp["win_lo"]).cuda()
    hi = None if inp["win_hi"] is None else torch.from_numpy(inp["win_hi"]).cuda()
    blk = cfg.block_only
    plain = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    ref = {k: v.clone() for k, v in plain.run(H, M, W, lo, hi, block_only=blk).items()}
    st = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, arena=True)
    try:
        out = st.run(H, M, W, lo, hi, block_only=blk)          # masked count read from M
        assert dl.get_status() == 0
        _same(out, ref)
        # the same step from pinned host inputs (count taken on the host)
        sel = st.run_host(inp["H"].pin_memory(), inp["M"].pin_memory(), W, lo, hi,
                          block_only=blk)
        assert dl.get_status() == 0
        assert torch.equal(sel["idx"], ref["idx"].cpu())
        assert torch.equal(sel["n_sel"], ref["n_sel"].cpu())
        with pytest.raises(RuntimeError):
            st.capture(H, M, W, lo, hi, blk)
    finally:
        st.arena.close()


def test_workspace_smaller_than_the_mask_reports_capacity(dl):
    """A workspace sized for 100 rows fewer than the mask holds: the step computes the rows
    that fit, reports DLLM_ERR_CAPACITY, and writes nothing past ws_bytes."""
    cfg = WL.custom_config(1, 4096, 256, 3000, 8, r=0.5)
    inp, H, M, W = _inputs(cfg, seed=3)
    count = int(inp["M"].sum())
    plain = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    ref = {k: v.clone() for k, v in plain.run(H, M, W).items()}
    assert dl.get_status() == 0
    small = dl.workspace_bytes_rows(cfg.B, cfg.L, cfg.d, cfg.V, count - 100)
    cap = dl.workspace_rows(cfg.B, cfg.L, cfg.d, cfg.V, small)
    assert count - 100 <= cap < count
    guard = 1 << 20
    buf = torch.full((small + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    n = cfg.B * cfg.L
    i32 = dict(dtype=torch.int32, device="cuda")
    tok, row_idx, cnt = torch.full((n,), -1, **i32), torch.empty(n, **i32), torch.empty(4, **i32)
    conf = torch.full((n,), -1.0, device="cuda")
    lse = torch.full((n,), -1.0, device="cuda")
    seq_off = torch.empty(cfg.B + 1, **i32)
    dl.masked_logits(H, M, W, tok, conf, lse, row_idx, seq_off, cnt, buf[:small])
    assert dl.get_status() == -11                          # DLLM_ERR_CAPACITY
    assert bool((buf[small:] == 0xA5).all())               # nothing written past ws_bytes
    assert int(cnt[0]) == count
    assert torch.equal(row_idx[:count], ref["row_idx"][:count])
    # the rows that fit are computed (the schedule differs, so up to fp32 rounding order)
    assert torch.equal(tok[:cap], ref["tok"][:cap])
    np.testing.assert_allclose(lse[:cap].cpu().numpy(), ref["lse"][:cap].cpu().numpy(), rtol=1e-5)
    np.testing.assert_allclose(conf[:cap].cpu().numpy(), ref["conf"][:cap].cpu().numpy(), rtol=1e-4)
    assert bool((tok[cap:] == -1).all())                   # the rest untouched
    # a workspace too small for even one row is refused before any launch
    with pytest.raises(dl.DllmError):
        dl.masked_logits(H, M, W, tok, conf, lse, row_idx, seq_off, cnt, buf[:64])
