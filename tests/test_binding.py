"""The Python binding's marshalling on a machine without a GPU, against a fake library: every
wrapper passes as many arguments as the C prototype declares, and refuses a buffer smaller
than the call may touch (the library sees only pointers, so a short tensor would otherwise
let a kernel run past its end) before anything is launched."""
import pytest
import torch

import mask_only_logits_b200 as dl
from mask_only_logits_b200 import _abi
from mask_only_logits_b200.sharded import PartialLayout

B, L, d, V, k = 2, 40, 64, 100, 4
N = B * L
S = 0                                               # explicit stream: no CUDA call needed


class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name not in _abi.PROTOTYPES:
            raise AttributeError(name)

        def call(*args):
            assert len(args) == len(_abi.PROTOTYPES[name][1]), (name, len(args))
            if name == "dllm_workspace_bytes":             # sizing, not a library call to log
                return 4096
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(dl, "lib", lambda: lib)
    monkeypatch.setattr(dl, "_on_device", lambda t, host_ok: True)
    return lib


def i32(n):
    return torch.zeros(n, dtype=torch.int32)


def f32(n):
    return torch.zeros(n, dtype=torch.float32)


def bufs():
    return dict(H=torch.zeros(N, d, dtype=torch.bfloat16), M=torch.zeros(B, L, dtype=torch.uint8),
                W=torch.zeros(V, d, dtype=torch.bfloat16), tok=i32(N), conf=f32(N), lse=f32(N),
                ent=f32(N), mar=f32(N), row_idx=i32(N), seq_off=i32(B + 1), count=i32(4),
                idx=i32(B * k), n_sel=i32(B), tok_sel=i32(B * k), conf_sel=f32(B * k),
                lo=i32(B), hi=i32(B), ws=torch.zeros(64, dtype=torch.uint8))


CALLS = {
    "mask_compact": lambda b: dl.mask_compact(b["M"], b["row_idx"], b["seq_off"], b["count"], b["ws"], S),
    "mask_compact_window": lambda b: dl.mask_compact(b["M"], b["row_idx"], b["seq_off"], b["count"],
                                                     b["ws"], S, b["lo"], b["hi"]),
    "mask_compact_noalloc": lambda b: dl.mask_compact_noalloc(b["M"], b["row_idx"], b["seq_off"],
                                                              b["count"], S),
    "masked_logits": lambda b: dl.masked_logits(b["H"], b["M"], b["W"], b["tok"], b["conf"], b["lse"],
                                                b["row_idx"], b["seq_off"], b["count"], b["ws"], S),
    "masked_logits_ex": lambda b: dl.masked_logits_ex(
        b["H"], b["M"], b["W"], 3, b["tok"], b["conf"], b["lse"], b["ent"], b["mar"], b["row_idx"],
        b["seq_off"], b["count"], b["ws"], S),
    "masked_logits_window": lambda b: dl.masked_logits_ex(
        b["H"], b["M"], b["W"], 3, b["tok"], b["conf"], b["lse"], b["ent"], b["mar"], b["row_idx"],
        b["seq_off"], b["count"], b["ws"], S, b["lo"], b["hi"]),
    "prepare_rows": lambda b: dl.prepare_rows(b["H"], b["M"], d, V, b["row_idx"], b["seq_off"],
                                              b["count"], b["ws"], S, b["lo"], b["hi"]),
    "masked_logits_prepared": lambda b: dl.masked_logits_prepared(
        b["W"], B, L, 3, b["tok"], b["conf"], b["lse"], b["ent"], b["mar"], b["count"], b["ws"], S),
    "select_unmask": lambda b: dl.select_unmask(b["conf"], b["row_idx"], b["seq_off"], B, L, k,
                                                b["idx"], b["n_sel"], b["lo"], b["hi"], b["tok"],
                                                b["tok_sel"], b["conf_sel"], S),
    "select_unmask_ex": lambda b: dl.select_unmask_ex(b["conf"], b["row_idx"], b["seq_off"], B, L, k,
                                                      0.5, 1, b["idx"], b["n_sel"], False, b["lo"],
                                                      b["hi"], b["tok"], b["tok_sel"], b["conf_sel"], S),
    "decode_step": lambda b: dl.decode_step(b["H"], b["M"], b["W"], k, b["tok"], b["conf"], b["lse"],
                                            b["row_idx"], b["seq_off"], b["count"], b["idx"],
                                            b["n_sel"], b["ws"], b["lo"], b["hi"], b["tok_sel"],
                                            b["conf_sel"], S),
    "decode_block_step": lambda b: dl.decode_step(b["H"], b["M"], b["W"], k, b["tok"], b["conf"],
                                                  b["lse"], b["row_idx"], b["seq_off"], b["count"],
                                                  b["idx"], b["n_sel"], b["ws"], b["lo"], b["hi"],
                                                  b["tok_sel"], b["conf_sel"], S, block_only=True),
    "debug_lmhead_logits": lambda b: dl.debug_lmhead_logits(b["H"], b["M"], b["W"], f32(N * V),
                                                            b["row_idx"], b["seq_off"], b["count"],
                                                            b["ws"], S),
}

# buffers each call must check, with the size it needs
NEEDS = {
    "mask_compact": ["row_idx", "seq_off"],
    "mask_compact_window": ["row_idx", "seq_off", "lo", "hi"],
    "mask_compact_noalloc": ["row_idx", "seq_off"],
    "masked_logits": ["H", "tok", "conf", "lse", "row_idx", "seq_off"],
    "masked_logits_ex": ["H", "tok", "conf", "lse", "ent", "mar", "row_idx", "seq_off"],
    "masked_logits_window": ["H", "tok", "conf", "lse", "ent", "mar", "row_idx", "seq_off", "lo", "hi"],
    "prepare_rows": ["H", "row_idx", "seq_off", "lo", "hi"],
    "masked_logits_prepared": ["tok", "conf", "lse", "ent", "mar"],
    "select_unmask": ["seq_off", "idx", "n_sel", "tok_sel", "conf_sel", "lo", "hi"],
    "select_unmask_ex": ["seq_off", "idx", "n_sel", "tok_sel", "conf_sel", "lo", "hi"],
    "decode_step": ["H", "tok", "conf", "lse", "row_idx", "seq_off", "idx", "n_sel", "tok_sel",
                    "conf_sel", "lo", "hi"],
    "decode_block_step": ["H", "tok", "conf", "lse", "row_idx", "seq_off", "idx", "n_sel",
                          "tok_sel", "conf_sel", "lo", "hi"],
    "debug_lmhead_logits": ["H", "row_idx", "seq_off"],
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_wrapper_arity_and_sizes(fake, name):
    CALLS[name](bufs())                               # every buffer large enough: one C call
    assert len(fake.calls) == 1
    for key in NEEDS[name]:
        b = bufs()
        t = b[key]
        b[key] = t.reshape(-1)[:-1]                   # one element short
        with pytest.raises(ValueError, match="needs at least"):
            CALLS[name](b)
    assert len(fake.calls) == 1                       # nothing reached the library


def test_vocab_partials_and_merge_sizes(fake):
    """Per-shard partials take B*L entries per field; the merge reads n_split strided splits,
    which the gathered layout's field views cover exactly."""
    world = 3
    lay = PartialLayout(N, extended=True)
    local, gathered = lay.empty(None, "cpu"), lay.empty(world, "cpu")
    b = bufs()
    lf, gf = lay.fields_of(local), lay.fields_of(gathered)
    dl.masked_partials(b["H"], b["M"], b["W"][:50], 0, 3, lf["m"], lf["s"], lf["a"], lf["t"],
                       lf["m2"], b["row_idx"], b["seq_off"], b["count"], b["ws"], S)
    dl.lse_merge(gf["m"], gf["s"], gf["a"], gf["t"], gf["m2"], lay.split_stride, world, b["count"],
                 N, 3, b["tok"], b["conf"], b["lse"], b["ent"], b["mar"], S)
    assert fake.calls == ["dllm_masked_partials", "dllm_lse_merge"]
    with pytest.raises(ValueError, match="part_m: needs at least"):
        dl.masked_partials(b["H"], b["M"], b["W"][:50], 0, 0, f32(N - 1), lf["s"], lf["a"], None,
                           None, b["row_idx"], b["seq_off"], b["count"], b["ws"], S)
    short = gathered.reshape(-1)[:(world - 1) * lay.split_stride + N - 1]
    with pytest.raises(ValueError, match="part_m: needs at least"):
        dl.lse_merge(short, gf["s"], gf["a"], None, None, lay.split_stride, world, b["count"], N, 0,
                     b["tok"], b["conf"], b["lse"], stream=S)
    with pytest.raises(ValueError, match="tok: needs at least"):
        dl.lse_merge(gf["m"], gf["s"], gf["a"], None, None, lay.split_stride, world, b["count"], N,
                     0, i32(N - 1), b["conf"], b["lse"], stream=S)
    # the gathered views reach the last rank's field
    for v in (gf["m"], gf["s"], gf["a"], gf["t"], gf["m2"]):
        assert v.numel() >= (world - 1) * lay.split_stride + lay.n_cap


def test_debug_merge_sizes(fake):
    pm, ps, pa = f32(6), f32(6), i32(6)
    dl.debug_lse_merge(pm.view(2, 3), ps, pa, i32(3), f32(3), f32(3), S)
    with pytest.raises(ValueError, match="part_s: needs at least"):
        dl.debug_lse_merge(pm.view(2, 3), f32(5), pa, i32(3), f32(3), f32(3), S)
    with pytest.raises(ValueError, match="lse: needs at least"):
        dl.debug_lse_merge(pm.view(2, 3), ps, pa, i32(3), f32(3), f32(2), S)


def test_cpu_tensors_are_refused_without_the_fake(monkeypatch):
    """Without the stand-in device check, an ordinary CPU tensor is refused by name."""
    monkeypatch.setattr(dl, "lib", lambda: FakeLib())
    b = bufs()
    with pytest.raises(ValueError, match="M: expected a CUDA tensor"):
        dl.mask_compact(torch.zeros(B, L, dtype=torch.uint8), b["row_idx"], b["seq_off"],
                        b["count"], b["ws"], S)


@pytest.mark.parametrize("Bq,kq", [(1, 1), (3, 5), (8, 4), (2, 1024), (7, 3)])
def test_decode_step_selection_layout(Bq, kq):
    """The packed selection buffer (one copy brings a step's selection to the host): four
    parts idx, n_sel, tok_sel, conf_sel, each starting 16-byte aligned, disjoint, with the
    shapes and dtypes of the selection outputs; host-side byte counts of the end-to-end
    path."""
    st = dl.DecodeStep(Bq, 64, 64, 100, kq, device="cpu")
    views = [st.idx, st.n_sel, st.tok_sel, st.conf_sel]
    assert [v.shape for v in views] == [(Bq, kq), (Bq,), (Bq, kq), (Bq, kq)]
    assert [v.dtype for v in views] == [torch.int32, torch.int32, torch.int32, torch.float32]
    base = st.sel_buf.data_ptr()
    spans = []
    for v in views:
        off = v.data_ptr() - base
        assert off % 16 == 0
        spans.append((off, off + v.numel() * 4))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))          # disjoint
    assert spans[-1][1] <= st.sel_buf.numel() * 4
    # writing through the views lands in the one buffer the host copies back
    st.sel_buf.zero_()
    st.conf_sel.fill_(0.5)
    assert int((st.sel_buf.view(torch.float32) == 0.5).sum()) == Bq * kq
    assert st.d2h_bytes() == st.sel_buf.numel() * 4
    # only the mask and the masked rows of H cross the bus
    assert st.h2d_bytes_zero_copy(10) == Bq * 64 + 2 * 10 * 64


def test_decode_step_validates_policy_and_shapes():
    with pytest.raises(ValueError, match="policy"):
        dl.DecodeStep(1, 64, 64, 100, 4, device="cpu", policy="random")
    with pytest.raises(ValueError, match="k must be"):
        dl.DecodeStep(1, 64, 64, 100, dl.MAX_K + 1, device="cpu")
    with pytest.raises(ValueError, match="invalid shapes"):
        dl.DecodeStep(1, 64, 100, 100, 4, device="cpu")              # d not a multiple of 64


class _FakeStream:
    def __init__(self, log, name):
        self.log, self.name, self.cuda_stream = log, name, 0

    def wait_stream(self, other):
        self.log.append(("wait_stream", self.name, other.name))

    def wait_event(self, ev):
        self.log.append(("wait", self.name, ev.ident))


class _FakeEvent:
    count = 0

    def __init__(self, log):
        _FakeEvent.count += 1
        self.log, self.ident = log, _FakeEvent.count

    def record(self, stream):
        self.log.append(("record", stream.name, self.ident))


@pytest.mark.parametrize("policy,threshold", [("confidence", None), ("entropy", 7.0)])
def test_overlapped_loop_call_order(fake, monkeypatch, policy, threshold):
    """run_overlapped on fake streams and events: per step one staging call on the staging
    stream, then the GEMM and the selection on the compute stream after the staging
    event; from the third step on, the staging of step i waits for the event recorded
    after step i-2's selection (the workspace it is about to overwrite)."""
    import contextlib
    log = []
    fake.calls = log                                   # library calls go to the same log
    comp, prep = _FakeStream(log, "s"), _FakeStream(log, "ps")
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _FakeEvent(log))
    monkeypatch.setattr(torch.cuda, "stream", lambda st: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: comp)
    st = dl.DecodeStep(B, L, d, V, k, device="cpu", policy=policy, threshold=threshold)
    b = bufs()
    n_steps = 5
    sel_out = [torch.empty_like(st.sel_buf) for _ in range(n_steps)]
    st.run_overlapped([(b["H"], b["M"])] * n_steps, b["W"], stream=comp, prep_stream=prep,
                      sel_out=sel_out)
    calls = [e for e in log if isinstance(e, str)]
    sel_name = "dllm_select_unmask" if policy == "confidence" and threshold is None \
        else "dllm_select_unmask_ex"
    assert calls == ["dllm_prepare_rows", "dllm_masked_logits_prepared", sel_name] * n_steps
    assert log[0] == ("wait_stream", "ps", "s")
    # walk the log: per step, the events recorded and waited on
    step = -1
    used_ev, prepped_ev = {}, {}
    pending_wait = []
    for e in log[1:]:
        if e == "dllm_prepare_rows":
            step += 1
            if step >= 2:                              # waited for step-2's used event
                assert ("ps", used_ev[step - 2]) in pending_wait, step
            pending_wait = []
        elif isinstance(e, tuple) and e[0] == "wait":
            pending_wait.append((e[1], e[2]))
        elif isinstance(e, tuple) and e[0] == "record" and e[1] == "ps":
            prepped_ev[step] = e[2]
        elif e == "dllm_masked_logits_prepared":
            assert ("s", prepped_ev[step]) in pending_wait       # GEMM after its staging
        elif isinstance(e, tuple) and e[0] == "record" and e[1] == "s":
            used_ev[step] = e[2]
    assert step == n_steps - 1 and len(used_ev) == n_steps
    # consecutive steps alternate workspaces: the staging events of steps i and i+2 are the
    # same two events, re-recorded
    assert prepped_ev[0] == prepped_ev[2] != prepped_ev[1] == prepped_ev[3]


def test_overlapped_loop_waits_for_each_lazy_batch(fake, monkeypatch):
    """Batches from a generator: the current stream when the call starts is waited for once,
    and each batch's staging waits for an event recorded on the current stream at the moment
    that batch was yielded (a list's batches are taken as ready at the call)."""
    import contextlib
    log = []
    fake.calls = log
    comp, prep, cur = _FakeStream(log, "s"), _FakeStream(log, "ps"), _FakeStream(log, "cur")
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _FakeEvent(log))
    monkeypatch.setattr(torch.cuda, "stream", lambda st: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: cur)
    st = dl.DecodeStep(B, L, d, V, k, device="cpu")
    b = bufs()
    n_steps = 4

    def gen():
        for i in range(n_steps):
            log.append(("yield", i))
            yield b["H"], b["M"]

    st.run_overlapped(gen(), b["W"], stream=comp, prep_stream=prep)
    assert log[:2] == [("wait_stream", "ps", "s"), ("wait_stream", "ps", "cur")]
    for i in range(n_steps):
        y = log.index(("yield", i))
        p = [j for j, e in enumerate(log) if e == "dllm_prepare_rows"][i]
        between = log[y:p]
        rec = [e for e in between if isinstance(e, tuple) and e[0] == "record" and e[1] == "cur"]
        assert len(rec) == 1, (i, between)
        assert ("wait", "ps", rec[0][2]) in between, (i, between)
    # a list: no per-batch event on the current stream
    log.clear()
    st.run_overlapped([(b["H"], b["M"])] * n_steps, b["W"], stream=comp, prep_stream=prep)
    assert not [e for e in log if isinstance(e, tuple) and e[0] == "record" and e[1] == "cur"]


def test_overlapped_loop_checks_each_batch(fake, monkeypatch):
    import contextlib
    log = []
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _FakeEvent(log))
    monkeypatch.setattr(torch.cuda, "stream", lambda st: contextlib.nullcontext())
    st = dl.DecodeStep(B, L, d, V, k, device="cpu")
    b = bufs()
    comp, prep = _FakeStream(log, "s"), _FakeStream(log, "ps")
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: comp)
    bad_M = torch.zeros(L, B, dtype=torch.uint8)                   # transposed
    with pytest.raises(ValueError, match="M: expected shape"):
        st.run_overlapped([(b["H"], b["M"]), (b["H"], bad_M)], b["W"], stream=comp, prep_stream=prep)
    with pytest.raises(ValueError, match="H: needs at least"):
        st.run_overlapped([(b["H"][:-1], b["M"])], b["W"], stream=comp, prep_stream=prep)


@pytest.mark.parametrize("policy,threshold,block_only,expected", [
    ("confidence", None, False, ["dllm_decode_step"]),
    ("confidence", None, True, ["dllm_decode_block_step"]),
    ("confidence", 0.5, False, ["dllm_masked_logits_ex", "dllm_select_unmask_ex"]),
    ("entropy", None, False, ["dllm_masked_logits_ex", "dllm_select_unmask_ex"]),
    ("margin", 0.1, True, ["dllm_masked_logits_window", "dllm_select_unmask_ex"]),
])
def test_decode_step_run_calls(fake, policy, threshold, block_only, expected):
    """DecodeStep.run: the plain confidence top-k is one library call (the whole step);
    every other policy is the extended logits call and the threshold selection; block-only
    steps take the windowed entry points."""
    st = dl.DecodeStep(B, L, d, V, k, device="cpu", policy=policy, threshold=threshold)
    b = bufs()
    st.run(b["H"], b["M"], b["W"], b["lo"], b["hi"], S, block_only=block_only)
    assert fake.calls == expected


def test_vocab_sharded_step_one_rank_calls(fake):
    """One-rank vocabulary-parallel step: partials on the whole vocabulary, the merge (no
    collective), the selection."""
    from mask_only_logits_b200.sharded import VocabShardedStep
    vs = VocabShardedStep(B, L, d, V, k, device="cpu")
    b = bufs()
    out = vs.run(b["H"], b["M"], b["W"], stream=S)
    assert fake.calls == ["dllm_masked_partials", "dllm_lse_merge", "dllm_select_unmask"]
    assert out["idx"].shape == (B, k)
    with pytest.raises(ValueError, match="W_shard"):
        vs.run(b["H"], b["M"], b["W"][:-1], stream=S)


@pytest.mark.parametrize("n_cap,extended,world", [(1, False, 1), (7, False, 3), (130, True, 4),
                                                  (4096, True, 2)])
def test_partial_layout_addresses(n_cap, extended, world):
    """Packed partials: each rank's local fields, gathered in rank order, are found by the
    merge at (field view start) + j * split_stride for rank j, with every field's start
    16-byte aligned; the gathered views cover every entry read."""
    lay = PartialLayout(n_cap, extended)
    names = ("m", "s", "a", "t", "m2")[:lay.fields]
    locals_ = []
    for j in range(world):
        loc = lay.empty(None, "cpu")
        f = lay.fields_of(loc)
        for q, name in enumerate(names):
            vals = torch.arange(n_cap, dtype=torch.int32) + 1000 * q + 100000 * j
            if name == "a":
                f[name][:n_cap] = vals
            else:
                f[name][:n_cap] = vals.float()
        locals_.append(loc)
    gathered = torch.stack(locals_)                  # what the all-gather produces
    gf = lay.fields_of(gathered)
    for q, name in enumerate(names):
        v = gf[name]
        assert (v.data_ptr() - gathered.data_ptr()) % 16 == 0
        assert v.numel() >= (world - 1) * lay.split_stride + n_cap
        for j in range(world):
            got = v[j * lay.split_stride: j * lay.split_stride + n_cap]
            want = torch.arange(n_cap, dtype=torch.int32) + 1000 * q + 100000 * j
            assert torch.equal(got if name == "a" else got.to(torch.int32), want)


def test_decode_step_refuses_a_w_of_another_shape(fake, monkeypatch):
    import contextlib
    log = []
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _FakeEvent(log))
    monkeypatch.setattr(torch.cuda, "stream", lambda st: contextlib.nullcontext())
    st = dl.DecodeStep(B, L, d, V, k, device="cpu")
    b = bufs()
    W_bad = torch.zeros(V + 1, d, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="W: expected shape"):
        st.run(b["H"], b["M"], W_bad, stream=S)
    with pytest.raises(ValueError, match="W: expected shape"):
        st.run_overlapped([(b["H"], b["M"])], W_bad, stream=_FakeStream(log, "s"),
                          prep_stream=_FakeStream(log, "ps"))
    assert fake.calls == []
