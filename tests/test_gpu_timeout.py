"""Failure detection on the GPU without a fault: a copy of the library built with
DLLM_FAULT_SKIP_STAGE leaves one shared-memory stage of the GEMM's pipeline unarmed, so the
MMA issuer's bounded wait on it runs out (limit 1 s).  The kernel must unwind (every role
sees the abort flag, issued MMAs drain, TMEM is freed), the host must read DLLM_ERR_TIMEOUT
from dllm_get_status, and the CUDA context must stay usable: the regular library then
computes a correct step in the same process.  Nothing here traps, faults or hangs a GPU."""
import ctypes
import time

import numpy as np
import pytest
import torch

import gpu_util as GU
import oracle.oracle as O
import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def injected():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import os
    from mask_only_logits_b200 import _abi, build
    # built next to libdllm.so (in the package directory, never committed)
    out = os.path.join(build.PKG_DIR, "libdllm_fault_skip_stage.so")
    build.build(extra_flags=["-DDLLM_FAULT_SKIP_STAGE=1"], out=out)
    return _abi.load_from(out)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("variant", [1, 2], ids=["single", "pair"])
def test_unarmed_stage_times_out_and_context_survives(injected, variant):
    import mask_only_logits_b200 as dl
    inp = WL.make_inputs(WL.CONFIGS["cfg0"], seed=0)
    cfg = inp["cfg"]
    dev = GU.to_device(inp)
    n = cfg.B * cfg.L
    i32 = dict(dtype=torch.int32, device="cuda")
    tok, row_idx, count = torch.empty(n, **i32), torch.empty(n, **i32), torch.empty(4, **i32)
    conf, lse = torch.empty(n, device="cuda"), torch.empty(n, device="cuda")
    seq_off = torch.empty(cfg.B + 1, **i32)
    ws = torch.empty(injected.dllm_workspace_bytes(cfg.B, cfg.L, cfg.d, cfg.V), dtype=torch.uint8,
                     device="cuda")
    assert injected.dllm_debug_set_gemm_variant(variant) == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.perf_counter()
    st = injected.dllm_masked_logits(_p(dev["H"]), _p(dev["M"]), _p(dev["W"]), cfg.B, cfg.L, cfg.d,
                                     cfg.V, _p(tok), _p(conf), _p(lse), _p(row_idx), _p(seq_off),
                                     _p(count), _p(ws), ws.numel(), stream)
    assert st == 0                                       # the launch itself is valid
    status = injected.dllm_get_status(stream)            # synchronises, then reads the word
    elapsed = time.perf_counter() - t0
    assert status == -6, status                          # DLLM_ERR_TIMEOUT
    assert elapsed < 30.0
    assert injected.dllm_get_status(stream) == 0         # reading cleared it
    # the context is intact: the regular library computes a correct step right after
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    out = step.run(dev["H"], dev["M"], dev["W"])
    assert dl.get_status() == 0
    c = int(out["count"][0])
    Hb, Wb, M = GU.inputs_bits(inp)
    ref = O.oracle_rows(Hb, Wb, M)
    GU.check_rows(out["tok"][:c].cpu().numpy(), out["conf"][:c].cpu().numpy(),
                  out["lse"][:c].cpu().numpy(), ref, np.arange(c), "after-timeout")
