"""Mask-only logits + confidence unmasking for diffusion-LLM decoding on B200 (sm_100a).

Python face of the C ABI in ``include/dllm.h``.  Every step of the path runs in the
library's CUDA kernels; this module only turns torch tensors into pointers and picks the
current CUDA stream.  PyTorch supplies device memory and streams.  There is no CPU
fallback: if ``libdllm.so`` is missing, loading fails loudly.

Low-level calls (same names and arguments as the C ABI, tensors instead of pointers):
``workspace_bytes``, ``mask_compact``, ``masked_logits``, ``select_unmask``,
``decode_step``, ``get_status``, and for a vocabulary-parallel LM head ``masked_partials``
and ``lse_merge``.  ``DecodeStep`` owns the buffers of one shape and runs a whole step on
device tensors (``run``) or on host tensors with the copies included (``run_host``,
``run_host_pipeline``); ``sharded.VocabShardedStep`` runs it with W split over ranks.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi

__all__ = [
    "DllmError", "lib", "version", "workspace_bytes", "workspace_bytes_rows", "workspace_rows",
    "Arena", "mask_compact", "mask_compact_noalloc",
    "masked_logits", "masked_logits_ex", "select_unmask_ex", "STAT_ENTROPY", "STAT_MARGIN",
    "masked_partials", "lse_merge", "prepare_rows", "masked_logits_prepared",
    "select_unmask", "decode_step", "get_status", "debug_lmhead_logits", "debug_lse_merge",
    "debug_set_gemm_variant",
    "prof_begin", "prof_end", "DecodeStep", "MAX_K",
]

MAX_K = 1024
STAT_ENTROPY = 1
STAT_MARGIN = 2

STATUS = {0: "DLLM_OK", -1: "DLLM_ERR_NULL", -2: "DLLM_ERR_ALIGN", -3: "DLLM_ERR_SHAPE",
          -4: "DLLM_ERR_WORKSPACE", -5: "DLLM_ERR_CUDA", -6: "DLLM_ERR_TIMEOUT",
          -7: "DLLM_ERR_DEVICE", -8: "DLLM_ERR_BOUNDS", -9: "DLLM_ERR_SCRATCH",
          -10: "DLLM_ERR_MEMORY", -11: "DLLM_ERR_CAPACITY"}


class DllmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().dllm_status_string(status).decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def lib() -> ctypes.CDLL:
    return _abi.load()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DllmError(status, where)


def _on_device(t: torch.Tensor, host_ok: bool) -> bool:
    """Whether the library's kernels can read t: device memory, or (host_ok) page-locked
    host memory."""
    return t.is_cuda or (host_ok and t.is_pinned())


def _ptr(t: torch.Tensor | None, dtype: torch.dtype | None = None, name: str = "",
         host_ok: bool = False, n: int = 0) -> ctypes.c_void_p:
    """Device pointer of a tensor of at least n elements; with host_ok, a page-locked CPU
    tensor is also accepted (the library reads it over the bus; only the step inputs H and
    M allow this).  The library sees only pointers, so the sizes are checked here: a short
    buffer is refused before any launch could run past its end."""
    if t is None:
        return ctypes.c_void_p(None)
    if t.numel() < n:
        raise ValueError(f"{name}: needs at least {n} elements, got {t.numel()}")
    if not _on_device(t, host_ok):
        raise ValueError(f"{name}: expected a CUDA tensor" +
                         (" or a page-locked (pinned) CPU tensor" if host_ok else ""))
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def version() -> int:
    return int(lib().dllm_version())


def workspace_bytes(B: int, L: int, d: int, V: int) -> int:
    return int(lib().dllm_workspace_bytes(B, L, d, V))


def workspace_bytes_rows(B: int, L: int, d: int, V: int, max_rows: int) -> int:
    """Workspace bytes for steps with at most max_rows masked rows (0 if invalid)."""
    return int(lib().dllm_workspace_bytes_rows(B, L, d, V, max_rows))


def workspace_rows(B: int, L: int, d: int, V: int, ws_bytes: int) -> int:
    """Masked-row capacity of a workspace of ws_bytes (B*L for the full size, 0 if too small)."""
    return int(lib().dllm_workspace_rows(B, L, d, V, ws_bytes))


class _DeviceBytes:
    """A device byte range exposed through __cuda_array_interface__, so that torch can view
    it as a uint8 tensor without copying or allocating."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = dict(shape=(nbytes,), typestr="|u1", data=(ptr, False),
                                             version=3, strides=None)


class Arena:
    """Device memory behind one fixed virtual address range, backed on demand (the C ABI's
    dllm_arena: the Mosaic page's memory manager with virtual memory mapping).

    ``map(nbytes)`` backs [0, nbytes) (whole chunks) with physical memory and releases the
    chunks past it; the address never moves.  ``tensor()`` is a uint8 view of the mapped
    prefix, usable as a step's workspace.  Shrinking synchronises the device first."""

    def __init__(self, reserve_bytes: int, chunk_bytes: int = 0, device=None):
        if device is not None:
            d = torch.device(device)
            torch.cuda.set_device(d.index if d.index is not None else torch.cuda.current_device())
        self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        _check(lib().dllm_arena_create(reserve_bytes, chunk_bytes, ctypes.byref(h)),
               "dllm_arena_create")
        self._h = h
        self._view = None

    @property
    def ptr(self) -> int:
        return int(lib().dllm_arena_ptr(self._h) or 0)

    @property
    def reserved(self) -> int:
        return int(lib().dllm_arena_reserved(self._h))

    @property
    def mapped(self) -> int:
        return int(lib().dllm_arena_mapped(self._h))

    @property
    def chunk(self) -> int:
        return int(lib().dllm_arena_chunk(self._h))

    def map(self, nbytes: int) -> int:
        """Back [0, nbytes) with physical memory (whole chunks); returns the mapped size."""
        if self._h is None:
            raise RuntimeError("arena closed")
        self._view = None
        _check(lib().dllm_arena_map(self._h, nbytes), "dllm_arena_map")
        return self.mapped

    def tensor(self) -> torch.Tensor:
        """uint8 view of the mapped prefix (valid until the next map() or close())."""
        if self._view is None:
            n = self.mapped
            if n == 0:
                raise RuntimeError("nothing is mapped")
            self._view = torch.as_tensor(_DeviceBytes(self.ptr, n), device=self.device)
        return self._view

    def close(self) -> None:
        if self._h is not None:
            self._view = None
            _check(lib().dllm_arena_destroy(self._h), "dllm_arena_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass


def mask_compact(M, row_idx, seq_off, count, ws, stream=None, win_lo=None, win_hi=None) -> None:
    """Compaction of the masked positions of M; with windows (device int32 [B] each), of
    the masked positions l of sequence b with win_lo[b] <= l < win_hi[b] only."""
    B, L = M.shape
    if win_lo is None and win_hi is None:
        _check(lib().dllm_mask_compact(_ptr(M, torch.uint8, "M"), B, L,
                                       _ptr(row_idx, torch.int32, "row_idx", n=B * L),
                                       _ptr(seq_off, torch.int32, "seq_off", n=B + 1),
                                       _ptr(count, torch.int32, "count", n=1), _ptr(ws, None, "ws"),
                                       ws.numel() * ws.element_size(), _stream(stream)),
               "dllm_mask_compact")
        return
    _check(lib().dllm_mask_compact_window(_ptr(M, torch.uint8, "M"), B, L,
                                          _ptr(win_lo, torch.int32, "win_lo", n=B),
                                          _ptr(win_hi, torch.int32, "win_hi", n=B),
                                          _ptr(row_idx, torch.int32, "row_idx", n=B * L),
                                          _ptr(seq_off, torch.int32, "seq_off", n=B + 1),
                                          _ptr(count, torch.int32, "count", n=1), _ptr(ws, None, "ws"),
                                          ws.numel() * ws.element_size(), _stream(stream)),
           "dllm_mask_compact_window")


def mask_compact_noalloc(M, row_idx, seq_off, count, stream=None) -> None:
    """mask_compact for callers that cannot allocate device memory: no workspace; the
    library's fixed static scratch is used instead (B*L <= 134,217,728; calls that overlap
    on the GPU race on that scratch)."""
    B, L = M.shape
    _check(lib().dllm_mask_compact_noalloc(_ptr(M, torch.uint8, "M"), B, L,
                                           _ptr(row_idx, torch.int32, "row_idx", n=B * L),
                                           _ptr(seq_off, torch.int32, "seq_off", n=B + 1),
                                           _ptr(count, torch.int32, "count", n=1), _stream(stream)),
           "dllm_mask_compact_noalloc")


def masked_logits(H, M, W, tok, conf, lse, row_idx, seq_off, count, ws, stream=None) -> None:
    B, L = M.shape
    V, d = W.shape
    n = B * L
    _check(lib().dllm_masked_logits(
        _ptr(H, torch.bfloat16, "H", True, n * d), _ptr(M, torch.uint8, "M", True),
        _ptr(W, torch.bfloat16, "W"),
        B, L, d, V, _ptr(tok, torch.int32, "tok", n=n), _ptr(conf, torch.float32, "conf", n=n),
        _ptr(lse, torch.float32, "lse", n=n), _ptr(row_idx, torch.int32, "row_idx", n=n),
        _ptr(seq_off, torch.int32, "seq_off", n=B + 1), _ptr(count, torch.int32, "count", n=1),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
        "dllm_masked_logits")


def masked_logits_ex(H, M, W, stats, tok, conf, lse, entropy, margin, row_idx, seq_off, count,
                     ws, stream=None, win_lo=None, win_hi=None) -> None:
    """masked_logits plus the softmax entropy and/or top-2 probability margin per masked row
    (stats: bitwise OR of STAT_ENTROPY and STAT_MARGIN; pass None for outputs not asked for).
    With windows (device int32 [B] each), only the masked rows inside each sequence's window
    [win_lo[b], win_hi[b]) get logits (current-block-only decoding)."""
    B, L = M.shape
    V, d = W.shape
    n = B * L
    common = (_ptr(tok, torch.int32, "tok", n=n), _ptr(conf, torch.float32, "conf", n=n),
              _ptr(lse, torch.float32, "lse", n=n), _ptr(entropy, torch.float32, "entropy", n=n),
              _ptr(margin, torch.float32, "margin", n=n),
              _ptr(row_idx, torch.int32, "row_idx", n=n),
              _ptr(seq_off, torch.int32, "seq_off", n=B + 1), _ptr(count, torch.int32, "count", n=1),
              _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream))
    ins = (_ptr(H, torch.bfloat16, "H", True, n * d), _ptr(M, torch.uint8, "M", True),
           _ptr(W, torch.bfloat16, "W"), B, L, d, V)
    if win_lo is None and win_hi is None:
        _check(lib().dllm_masked_logits_ex(*ins, stats, *common), "dllm_masked_logits_ex")
    else:
        _check(lib().dllm_masked_logits_window(*ins, _ptr(win_lo, torch.int32, "win_lo", n=B),
                                               _ptr(win_hi, torch.int32, "win_hi", n=B), stats,
                                               *common), "dllm_masked_logits_window")


def prepare_rows(H, M, d, V, row_idx, seq_off, count, ws, stream=None, win_lo=None,
                 win_hi=None) -> None:
    """First half of masked_logits: compaction of M (in the windows, if given) and the gather
    of the masked rows of H into ``ws``.  H and M may be page-locked CPU tensors (read over
    the bus: only the mask and the masked rows move)."""
    B, L = M.shape
    _check(lib().dllm_prepare_rows(*_step_inputs(H, M, B, L, d), B, L, d, V,
                                   *_prepare_tail(B, L, row_idx, seq_off, count, ws, win_lo, win_hi),
                                   _stream(stream)), "dllm_prepare_rows")


def _step_inputs(H, M, B: int, L: int, d: int) -> tuple:
    """Pointers of a step's H [B*L, d] and M [B, L] (device or page-locked host memory)."""
    if tuple(M.shape) != (B, L):
        raise ValueError(f"M: expected shape ({B}, {L}), got {tuple(M.shape)}")
    return _ptr(H, torch.bfloat16, "H", True, B * L * d), _ptr(M, torch.uint8, "M", True)


def _prepare_tail(B, L, row_idx, seq_off, count, ws, win_lo, win_hi) -> tuple:
    """Arguments of dllm_prepare_rows after (H, M, B, L, d, V), without the stream."""
    return (_ptr(win_lo, torch.int32, "win_lo", n=B), _ptr(win_hi, torch.int32, "win_hi", n=B),
            _ptr(row_idx, torch.int32, "row_idx", n=B * L),
            _ptr(seq_off, torch.int32, "seq_off", n=B + 1), _ptr(count, torch.int32, "count", n=1),
            _ptr(ws, None, "ws"), ws.numel() * ws.element_size())


def masked_logits_prepared(W, B, L, stats, tok, conf, lse, entropy, margin, count, ws,
                           stream=None) -> None:
    """Second half of masked_logits: the GEMM and its statistics on rows prepared in ``ws``."""
    _check(lib().dllm_masked_logits_prepared(
        *_prepared_args(W, B, L, stats, tok, conf, lse, entropy, margin, count, ws),
        _stream(stream)), "dllm_masked_logits_prepared")


def _prepared_args(W, B, L, stats, tok, conf, lse, entropy, margin, count, ws) -> tuple:
    """Arguments of dllm_masked_logits_prepared, without the stream."""
    V, d = W.shape
    n = B * L
    return (_ptr(W, torch.bfloat16, "W"), B, L, d, V, stats, _ptr(tok, torch.int32, "tok", n=n),
            _ptr(conf, torch.float32, "conf", n=n), _ptr(lse, torch.float32, "lse", n=n),
            _ptr(entropy, torch.float32, "entropy", n=n),
            _ptr(margin, torch.float32, "margin", n=n), _ptr(count, torch.int32, "count", n=1),
            _ptr(ws, None, "ws"), ws.numel() * ws.element_size())


def masked_partials(H, M, W_shard, v_offset, stats, part_m, part_s, part_a, part_t, part_m2,
                    row_idx, seq_off, count, ws, stream=None, win_lo=None, win_hi=None) -> None:
    """One vocabulary shard of a vocabulary-parallel LM head (W_shard = rows v_offset ..
    v_offset + V_shard - 1 of W): per masked row, the softmax partial (max, sum of exp,
    global argmax; plus t and second max when stats != 0) over the shard's vocabulary."""
    B, L = M.shape
    V_shard, d = W_shard.shape
    n = B * L
    _check(lib().dllm_masked_partials(
        _ptr(H, torch.bfloat16, "H", True, n * d), _ptr(M, torch.uint8, "M", True),
        _ptr(W_shard, torch.bfloat16, "W_shard"), B, L, d, V_shard, int(v_offset),
        _ptr(win_lo, torch.int32, "win_lo", n=B), _ptr(win_hi, torch.int32, "win_hi", n=B), stats,
        _ptr(part_m, torch.float32, "part_m", n=n), _ptr(part_s, torch.float32, "part_s", n=n),
        _ptr(part_a, torch.int32, "part_a", n=n), _ptr(part_t, torch.float32, "part_t", n=n),
        _ptr(part_m2, torch.float32, "part_m2", n=n), _ptr(row_idx, torch.int32, "row_idx", n=n),
        _ptr(seq_off, torch.int32, "seq_off", n=B + 1), _ptr(count, torch.int32, "count", n=1),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
        "dllm_masked_partials")


def lse_merge(part_m, part_s, part_a, part_t, part_m2, split_stride, n_split, count, n_cap,
              stats, tok, conf, lse, entropy=None, margin=None, stream=None) -> None:
    """Merge per-shard partials (split j of row i at j * split_stride + i) into tok, conf,
    lse (and entropy / margin) for rows below the device-side count."""
    np_ = max(0, (int(n_split) - 1) * int(split_stride) + int(n_cap))   # partial entries read
    _check(lib().dllm_lse_merge(
        _ptr(part_m, torch.float32, "part_m", n=np_), _ptr(part_s, torch.float32, "part_s", n=np_),
        _ptr(part_a, torch.int32, "part_a", n=np_), _ptr(part_t, torch.float32, "part_t", n=np_),
        _ptr(part_m2, torch.float32, "part_m2", n=np_), int(split_stride), int(n_split),
        _ptr(count, torch.int32, "count", n=1), int(n_cap), stats,
        _ptr(tok, torch.int32, "tok", n=n_cap),
        _ptr(conf, torch.float32, "conf", n=n_cap), _ptr(lse, torch.float32, "lse", n=n_cap),
        _ptr(entropy, torch.float32, "entropy", n=n_cap),
        _ptr(margin, torch.float32, "margin", n=n_cap),
        _stream(stream)), "dllm_lse_merge")


def select_unmask_ex(score, row_idx, seq_off, B, L, k, threshold, min_sel, idx, n_sel,
                     ascending=False, win_lo=None, win_hi=None, tok=None, tok_sel=None,
                     score_sel=None, stream=None) -> None:
    """Threshold-based selection: per sequence min(k, max(min(min_sel, n), #qualifying))
    best candidates; qualifying = score >= threshold (<= with ascending=True)."""
    _check(lib().dllm_select_unmask_ex(
        *_select_ex_args(score, row_idx, seq_off, B, L, k, threshold, min_sel, idx, n_sel,
                         ascending, win_lo, win_hi, tok, tok_sel, score_sel),
        _stream(stream)), "dllm_select_unmask_ex")


def _select_ex_args(score, row_idx, seq_off, B, L, k, threshold, min_sel, idx, n_sel,
                    ascending, win_lo, win_hi, tok, tok_sel, score_sel) -> tuple:
    """Arguments of dllm_select_unmask_ex, without the stream.  The per-row inputs are read
    below the device-side seq_off[B] only (callers may pass exactly that many entries), so
    only the [B+1], [B] and [B, k] buffers are size-checked."""
    nk = B * k
    return (_ptr(score, torch.float32, "score"), _ptr(row_idx, torch.int32, "row_idx"),
            _ptr(seq_off, torch.int32, "seq_off", n=B + 1), B, L, k, float(threshold), min_sel,
            1 if ascending else 0, _ptr(win_lo, torch.int32, "win_lo", n=B),
            _ptr(win_hi, torch.int32, "win_hi", n=B), _ptr(tok, torch.int32, "tok"),
            _ptr(idx, torch.int32, "idx", n=nk), _ptr(n_sel, torch.int32, "n_sel", n=B),
            _ptr(tok_sel, torch.int32, "tok_sel", n=nk),
            _ptr(score_sel, torch.float32, "score_sel", n=nk))


def select_unmask(conf, row_idx, seq_off, B, L, k, idx, n_sel, win_lo=None, win_hi=None,
                  tok=None, tok_sel=None, conf_sel=None, stream=None) -> None:
    _check(lib().dllm_select_unmask(
        *_select_args(conf, row_idx, seq_off, B, L, k, idx, n_sel, win_lo, win_hi, tok, tok_sel,
                      conf_sel), _stream(stream)), "dllm_select_unmask")


def _select_args(conf, row_idx, seq_off, B, L, k, idx, n_sel, win_lo, win_hi, tok, tok_sel,
                 conf_sel) -> tuple:
    """Arguments of dllm_select_unmask, without the stream (sizes checked as in
    _select_ex_args)."""
    nk = B * k
    return (_ptr(conf, torch.float32, "conf"), _ptr(row_idx, torch.int32, "row_idx"),
            _ptr(seq_off, torch.int32, "seq_off", n=B + 1), B, L, k,
            _ptr(win_lo, torch.int32, "win_lo", n=B), _ptr(win_hi, torch.int32, "win_hi", n=B),
            _ptr(tok, torch.int32, "tok"),
            _ptr(idx, torch.int32, "idx", n=nk), _ptr(n_sel, torch.int32, "n_sel", n=B),
            _ptr(tok_sel, torch.int32, "tok_sel", n=nk),
            _ptr(conf_sel, torch.float32, "conf_sel", n=nk))


def decode_step(H, M, W, k, tok, conf, lse, row_idx, seq_off, count, idx, n_sel, ws,
                win_lo=None, win_hi=None, tok_sel=None, conf_sel=None, stream=None,
                block_only=False) -> None:
    """The whole step.  With block_only=True (windows required) logits are computed for the
    masked rows inside the windows only (dllm_decode_block_step); the selection is the same."""
    B, L = M.shape
    V, d = W.shape
    fn, name = ((lib().dllm_decode_block_step, "dllm_decode_block_step") if block_only
                else (lib().dllm_decode_step, "dllm_decode_step"))
    n, nk = B * L, B * k
    _check(fn(
        _ptr(H, torch.bfloat16, "H", True, n * d), _ptr(M, torch.uint8, "M", True),
        _ptr(W, torch.bfloat16, "W"),
        B, L, d, V, k, _ptr(win_lo, torch.int32, "win_lo", n=B),
        _ptr(win_hi, torch.int32, "win_hi", n=B),
        _ptr(tok, torch.int32, "tok", n=n), _ptr(conf, torch.float32, "conf", n=n),
        _ptr(lse, torch.float32, "lse", n=n), _ptr(row_idx, torch.int32, "row_idx", n=n),
        _ptr(seq_off, torch.int32, "seq_off", n=B + 1), _ptr(count, torch.int32, "count", n=1),
        _ptr(idx, torch.int32, "idx", n=nk), _ptr(n_sel, torch.int32, "n_sel", n=B),
        _ptr(tok_sel, torch.int32, "tok_sel", n=nk),
        _ptr(conf_sel, torch.float32, "conf_sel", n=nk),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)), name)


def get_status(stream=None) -> int:
    return int(lib().dllm_get_status(_stream(stream)))


def debug_lmhead_logits(H, M, W, logits_out, row_idx, seq_off, count, ws, stream=None) -> None:
    B, L = M.shape
    V, d = W.shape
    n = B * L
    _check(lib().dllm_debug_lmhead_logits(
        _ptr(H, torch.bfloat16, "H", n=n * d), _ptr(M, torch.uint8, "M"),
        _ptr(W, torch.bfloat16, "W"),
        B, L, d, V, _ptr(logits_out, torch.float32, "logits_out", n=n * V),
        _ptr(row_idx, torch.int32, "row_idx", n=n), _ptr(seq_off, torch.int32, "seq_off", n=B + 1),
        _ptr(count, torch.int32, "count", n=1), _ptr(ws, None, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)), "dllm_debug_lmhead_logits")


def debug_lse_merge(part_m, part_s, part_a, tok, conf, lse, stream=None) -> None:
    n_split, n_rows = part_m.shape
    np_ = n_split * n_rows
    _check(lib().dllm_debug_lse_merge(
        _ptr(part_m, torch.float32, "part_m"), _ptr(part_s, torch.float32, "part_s", n=np_),
        _ptr(part_a, torch.int32, "part_a", n=np_), n_rows, n_split,
        _ptr(tok, torch.int32, "tok", n=n_rows),
        _ptr(conf, torch.float32, "conf", n=n_rows), _ptr(lse, torch.float32, "lse", n=n_rows),
        _stream(stream)),
        "dllm_debug_lse_merge")


def debug_set_gemm_variant(cta_group: int) -> None:
    """Test hook: 2 = paired-SM GEMM, 1 = single-SM GEMM, 0 = default (chosen on the device
    from the masked count: single SMs for at most 128 rows, pairs above)."""
    _check(lib().dllm_debug_set_gemm_variant(cta_group), "dllm_debug_set_gemm_variant")


def prof_begin() -> None:
    _check(lib().dllm_prof_begin(), "dllm_prof_begin")


def prof_end() -> tuple[float, int, int]:
    ms = ctypes.c_double(0.0)
    g = ctypes.c_int32(0)
    kcount = ctypes.c_int32(0)
    _check(lib().dllm_prof_end(ctypes.byref(ms), ctypes.byref(g), ctypes.byref(kcount)),
           "dllm_prof_end")
    return ms.value, g.value, kcount.value


POLICIES = ("confidence", "entropy", "margin")


class DecodeStep:
    """Buffers for one decode-step shape (B, L, d, V, k) on one device, and the step itself.

    ``policy`` picks the score the positions to unmask are ranked by: "confidence" (largest
    softmax probability, higher is better), "entropy" (of the row's softmax, lower is
    better) or "margin" (top-1 minus top-2 probability, higher is better).  With
    ``threshold`` set, every candidate whose score is at least as good as the threshold is
    unmasked, at most k and at least min(min_sel, candidates) per sequence; without it, the k
    best.  ``conf_sel`` then holds the policy's score of each selected position.

    Outputs are views into buffers owned by this object; their first ``count`` entries are
    valid (``count`` stays on the device unless read).
    """

    def __init__(self, B: int, L: int, d: int, V: int, k: int, device="cuda",
                 policy: str = "confidence", threshold: float | None = None, min_sel: int = 1,
                 arena: bool = False, arena_chunk: int = 0):
        if k < 1 or k > MAX_K:
            raise ValueError(f"k must be in [1, {MAX_K}]")
        if policy not in POLICIES:
            raise ValueError(f"policy must be one of {POLICIES}")
        self.B, self.L, self.d, self.V, self.k = B, L, d, V, k
        self.policy, self.threshold, self.min_sel = policy, threshold, min_sel
        self.stats = {"confidence": 0, "entropy": STAT_ENTROPY, "margin": STAT_MARGIN}[policy]
        self.device = torch.device(device)
        n = B * L
        i32 = dict(dtype=torch.int32, device=self.device)
        self.tok = torch.empty(n, **i32)
        self.conf = torch.empty(n, dtype=torch.float32, device=self.device)
        self.lse = torch.empty(n, dtype=torch.float32, device=self.device)
        self.entropy = torch.empty(n, dtype=torch.float32, device=self.device) \
            if policy == "entropy" else None
        self.margin = torch.empty(n, dtype=torch.float32, device=self.device) \
            if policy == "margin" else None
        self.row_idx = torch.empty(n, **i32)
        self.seq_off = torch.empty(B + 1, **i32)
        self.count = torch.empty(4, **i32)          # 16 bytes: keeps the next buffer aligned
        # the selection outputs share one buffer (each part starts 16-byte aligned), so that
        # one copy brings a step's whole selection back to the host
        self._sel_parts = [B * k, B, B * k, B * k]            # idx, n_sel, tok_sel, conf_sel
        self._sel_off = [0]
        for n_part in self._sel_parts:
            self._sel_off.append(self._sel_off[-1] + (n_part + 3) // 4 * 4)
        self.sel_buf = torch.empty(self._sel_off[-1], **i32)
        self.idx, self.n_sel, self.tok_sel, self.conf_sel = self._sel_views(self.sel_buf)
        nbytes = workspace_bytes(B, L, d, V)
        if nbytes == 0:
            raise ValueError("invalid shapes (d must be a positive multiple of 64)")
        # arena=True: the workspace lives in an Arena whose mapping follows each step's
        # masked count (``run(..., max_rows=...)``) instead of the worst case over all masks
        self.arena = Arena(nbytes, arena_chunk, self.device) if arena else None
        self.ws = None if arena else torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self._host = None

    def size_for_rows(self, max_rows: int) -> int:
        """Arena mode: map the workspace a step with at most max_rows masked rows needs
        (growing or shrinking the arena's backing); returns the bytes that step needs."""
        if self.arena is None:
            raise RuntimeError("size_for_rows needs DecodeStep(..., arena=True)")
        need = workspace_bytes_rows(self.B, self.L, self.d, self.V, max(1, int(max_rows)))
        if self.ws is None or self.arena.mapped != -(-need // self.arena.chunk) * self.arena.chunk:
            self.arena.map(need)
        self.ws = self.arena.tensor()
        return need

    def _rows_of(self, M, win_lo, win_hi, block_only) -> int:
        """Masked rows a step on M computes (a device mask is read back: a synchronisation)."""
        m = M != 0
        if block_only:
            pos = torch.arange(self.L, device=M.device)[None, :]
            m = m & (pos >= win_lo.to(M.device)[:, None]) & (pos < win_hi.to(M.device)[:, None])
        return int(m.sum())

    def _sel_views(self, buf):
        """idx [B, k], n_sel [B], tok_sel [B, k] (int32) and conf_sel [B, k] (float32) views
        of a selection buffer laid out like ``sel_buf`` (device or host)."""
        B, k = self.B, self.k
        o = self._sel_off
        return (buf[o[0]:o[0] + B * k].view(B, k), buf[o[1]:o[1] + B],
                buf[o[2]:o[2] + B * k].view(B, k),
                buf[o[3]:o[3] + B * k].view(torch.float32).view(B, k))

    def _check_W(self, W) -> None:
        """W must be this step's [V, d] projection: the staging and the GEMM halves of a step
        take their shapes from this object and from W respectively."""
        if tuple(W.shape) != (self.V, self.d):
            raise ValueError(f"W: expected shape ({self.V}, {self.d}), got {tuple(W.shape)}")

    def _plain(self) -> bool:
        return self.policy == "confidence" and self.threshold is None

    def _select_call(self, row_idx, seq_off, win_lo, win_hi) -> tuple:
        """(C entry point, its arguments without the stream, name) of the selection of this
        step's policy on the scores the logits call leaves."""
        if self._plain():
            return (lib().dllm_select_unmask,
                    _select_args(self.conf, row_idx, seq_off, self.B, self.L, self.k, self.idx,
                                 self.n_sel, win_lo, win_hi, self.tok, self.tok_sel,
                                 self.conf_sel), "dllm_select_unmask")
        score = {"confidence": self.conf, "entropy": self.entropy, "margin": self.margin}[self.policy]
        ascending = self.policy == "entropy"
        tau = self.threshold
        if tau is None:                                  # plain top-k of this score
            tau = float("inf") if ascending else float("-inf")
        return (lib().dllm_select_unmask_ex,
                _select_ex_args(score, row_idx, seq_off, self.B, self.L, self.k, tau,
                                self.min_sel, self.idx, self.n_sel, ascending, win_lo, win_hi,
                                self.tok, self.tok_sel, self.conf_sel), "dllm_select_unmask_ex")

    def _select(self, row_idx, seq_off, win_lo, win_hi, stream) -> None:
        """The selection of this step's policy on the scores the logits call left."""
        fn, args, name = self._select_call(row_idx, seq_off, win_lo, win_hi)
        _check(fn(*args, _stream(stream)), name)

    def _outputs(self) -> dict:
        out = dict(tok=self.tok, conf=self.conf, lse=self.lse, row_idx=self.row_idx,
                   seq_off=self.seq_off, count=self.count[:1], idx=self.idx, n_sel=self.n_sel,
                   tok_sel=self.tok_sel, conf_sel=self.conf_sel)
        if self.entropy is not None:
            out["entropy"] = self.entropy
        if self.margin is not None:
            out["margin"] = self.margin
        return out

    def run(self, H, M, W, win_lo=None, win_hi=None, stream=None, block_only=False,
            max_rows: int | None = None) -> dict:
        """One step on device tensors.  block_only=True (windows required): logits for the
        masked rows inside the windows only; tok/conf/lse/row_idx then cover those rows.
        Arena mode: the workspace is mapped for max_rows masked rows first (a decoding loop
        knows its masked count; if max_rows is None it is counted from M)."""
        self._check_W(W)
        if self.arena is not None:
            self.size_for_rows(self._rows_of(M, win_lo, win_hi, block_only)
                               if max_rows is None else max_rows)
        if self._plain():
            decode_step(H, M, W, self.k, self.tok, self.conf, self.lse, self.row_idx,
                        self.seq_off, self.count, self.idx, self.n_sel, self.ws, win_lo, win_hi,
                        self.tok_sel, self.conf_sel, stream, block_only)
        else:
            masked_logits_ex(H, M, W, self.stats, self.tok, self.conf, self.lse, self.entropy,
                             self.margin, self.row_idx, self.seq_off, self.count, self.ws,
                             stream, *((win_lo, win_hi) if block_only else (None, None)))
            self._select(self.row_idx, self.seq_off, win_lo, win_hi, stream)
        return self._outputs()

    # -- end-to-end from host memory ---------------------------------------------------------
    def capture(self, H, M, W, win_lo=None, win_hi=None, block_only=False):
        """Capture one step on these device tensors into a CUDA graph.  ``replay()`` then
        reruns the whole step (every kernel, with the programmatic-launch edges between them)
        on whatever those tensors hold at replay time, for one launch of CPU work; the
        outputs are this object's buffers as after ``run``.  Tensors must keep their
        addresses while the graph is used."""
        if self.arena is not None:
            # a graph would keep the workspace size of capture time while the arena's mapping
            # follows later masks
            raise RuntimeError("capture() needs a fixed workspace: use arena=False")
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            for _ in range(2):                   # one-time device set-up happens outside capture
                self.run(H, M, W, win_lo, win_hi, side, block_only)
        torch.cuda.current_stream(self.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            self.run(H, M, W, win_lo, win_hi, None, block_only)
        self._graph = graph
        return graph

    def replay(self, stream=None) -> dict:
        """Rerun the captured step (``capture`` first) on the current (or given) stream."""
        if getattr(self, "_graph", None) is None:
            raise RuntimeError("capture() a step first")
        if stream is None:
            self._graph.replay()
        else:
            with torch.cuda.stream(stream):
                self._graph.replay()
        return self._outputs()

    def _host_buffers(self):
        if self._host is None:
            B, L, d = self.B, self.L, self.d
            self._host = dict(
                H=torch.empty(B * L, d, dtype=torch.bfloat16, device=self.device),
                M=torch.empty(B, L, dtype=torch.uint8, device=self.device),
                sel=torch.empty(self.sel_buf.numel(), dtype=torch.int32, pin_memory=True))
        return self._host

    def run_host(self, H_host, M_host, W, win_lo=None, win_hi=None, stream=None,
                 block_only=False) -> dict:
        """One step from host H and M: copy them in, run, copy the selection back.

        W (the resident vocabulary projection) and the windows are device tensors.  Returns
        host tensors idx, n_sel, tok_sel, conf_sel; synchronises the stream.
        """
        hb = self._host_buffers()
        s = stream if stream is not None else torch.cuda.current_stream()
        rows = (self._rows_of(M_host, win_lo, win_hi, block_only)   # counted on the host
                if self.arena is not None else None)
        with torch.cuda.stream(s):
            hb["H"].copy_(H_host, non_blocking=True)
            hb["M"].copy_(M_host, non_blocking=True)
            self.run(hb["H"], hb["M"], W, win_lo, win_hi, s, block_only, max_rows=rows)
            hb["sel"].copy_(self.sel_buf, non_blocking=True)
        s.synchronize()
        return dict(zip(("idx", "n_sel", "tok_sel", "conf_sel"), self._sel_views(hb["sel"])))

    def _double(self) -> dict:
        """Two sets of (workspace, row_idx, seq_off, count): this object's own and a second
        one, so that staging of one step can run while the previous step computes."""
        if self.arena is not None:
            raise RuntimeError("the overlapped loops keep two fixed workspaces; with arena=True "
                               "run steps one at a time (run, run_host)")
        if getattr(self, "_dbl", None) is None:
            i32 = dict(dtype=torch.int32, device=self.device)
            self._dbl = dict(ws=[self.ws, torch.empty_like(self.ws)],
                             row_idx=[self.row_idx, torch.empty(self.B * self.L, **i32)],
                             seq_off=[self.seq_off, torch.empty(self.B + 1, **i32)],
                             count=[self.count, torch.empty(4, **i32)])
        return self._dbl

    def run_host_pipeline(self, batches, W, win_lo=None, win_hi=None, stream=None,
                          prep_stream=None, block_only=False):
        """Decode steps over host batches [(H_host, M_host), ...] in page-locked host memory,
        with the input staging of step i+1 overlapping step i.

        Staging (``prepare_rows``: compaction of the mask and the gather of only the masked
        rows of H, both read straight from host memory over the bus) runs on a second
        stream into one of two workspaces, while the compute stream runs the previous
        step's GEMM and selection on the other (``masked_logits_prepared``,
        ``select_unmask``) and copies the selection back to page-locked host memory.
        Yields, per step, host tensors idx, n_sel, tok_sel, conf_sel (valid until the next
        iteration).  Each batch's H_host and M_host must stay valid and unchanged until its
        step has been yielded.
        """
        self._check_W(W)
        B, L, d, V = self.B, self.L, self.d, self.V
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        ps = prep_stream if prep_stream is not None else torch.cuda.Stream(self.device)
        if getattr(self, "_pipe", None) is None:
            self._pipe = dict(
                self._double(),
                out_buf=[torch.empty(self.sel_buf.numel(), dtype=torch.int32, pin_memory=True)
                         for _ in range(2)],
                copy_stream=torch.cuda.Stream(self.device))
            self._pipe["out"] = [dict(zip(("idx", "n_sel", "tok_sel", "conf_sel"),
                                          self._sel_views(b))) for b in self._pipe["out_buf"]]
        pb = self._pipe
        cs = pb["copy_stream"]
        prepped = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        selected = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        pw = (win_lo, win_hi) if block_only else (None, None)
        # every argument but each batch's H and M, validated and marshalled once per call
        lb = lib()
        prep_tail = [_prepare_tail(B, L, pb["row_idx"][b], pb["seq_off"][b], pb["count"][b],
                                   pb["ws"][b], *pw) for b in range(2)]
        gemm = [_prepared_args(W, B, L, self.stats, self.tok, self.conf, self.lse, self.entropy,
                               self.margin, pb["count"][b], pb["ws"][b]) for b in range(2)]
        sel = [self._select_call(pb["row_idx"][b], pb["seq_off"][b], win_lo, win_hi)
               for b in range(2)]
        s_h, ps_h = _stream(s), _stream(ps)

        def prep(i, Hh, Mh):
            if not (Hh.is_pinned() and Mh.is_pinned()):
                raise ValueError("host batches must be page-locked (pinned) CPU tensors")
            b = i & 1
            if i >= 2:
                ps.wait_event(used[b])               # step i-2 no longer reads this workspace
            _check(lb.dllm_prepare_rows(*_step_inputs(Hh, Mh, B, L, d), B, L, d, V,
                                        *prep_tail[b], ps_h), "dllm_prepare_rows")
            prepped[b].record(ps)

        def compute(i):
            b = i & 1
            s.wait_event(prepped[b])
            _check(lb.dllm_masked_logits_prepared(*gemm[b], s_h), "dllm_masked_logits_prepared")
            if i >= 1:
                s.wait_event(done[(i - 1) & 1])      # step i-1's selection has been copied out
            fn, args, name = sel[b]
            _check(fn(*args, s_h), name)
            used[b].record(s)
            selected[b].record(s)
            # the selection goes back on the copy stream: the next step's GEMM does not wait
            with torch.cuda.stream(cs):
                cs.wait_event(selected[b])
                pb["out_buf"][b].copy_(self.sel_buf, non_blocking=True)
                done[b].record(cs)

        it = iter(batches)
        cur = next(it, None)
        if cur is None:
            return
        prep(0, *cur)
        i = 0
        pending = None
        while True:
            nxt = next(it, None)
            if nxt is not None:
                prep(i + 1, *nxt)                    # overlaps the compute of step i
            compute(i)
            if pending is not None:
                done[pending].synchronize()
                yield pb["out"][pending]
            pending = i & 1
            if nxt is None:
                break
            i += 1
        done[pending].synchronize()
        yield pb["out"][pending]

    def run_overlapped(self, batches, W, win_lo=None, win_hi=None, stream=None,
                       prep_stream=None, block_only=False, sel_out=None) -> dict:
        """Whole steps over device-resident batches [(H, M), ...] (or pinned host ones), each
        step's staging (compaction and gather, ``prepare_rows``) on a second stream during
        the previous step's GEMM, with no host synchronisation: the throughput loop of a
        serving process whose inputs are already on the GPU.  sel_out, if given, is a list
        (one per batch) of int32 device buffers shaped like ``sel_buf`` that receive each
        step's packed selection; otherwise only the last step's outputs remain (this
        object's buffers).

        Every argument but each batch's H and M is validated and turned into pointers once
        per call, so a step costs the host three library calls and four event operations:
        short steps stay bound by the device, not by Python.

        Readiness of the inputs: a list or tuple of batches must be written before the call,
        on ``stream`` or on the current stream (the staging stream waits for both once).
        Any other iterable is taken as produced lazily: each batch is waited for on the
        current stream at the moment it is yielded, so a generator may write a batch on the
        current stream just before yielding it.  When that stream is ``stream`` itself, each
        staging then also waits for the previous step's GEMM (correct, without overlap)."""
        self._check_W(W)
        B, L, d, V = self.B, self.L, self.d, self.V
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        ps = prep_stream if prep_stream is not None else torch.cuda.Stream(self.device)
        ob = self._double()
        lb = lib()
        pw = (win_lo, win_hi) if block_only else (None, None)
        prep = [_prepare_tail(B, L, ob["row_idx"][b], ob["seq_off"][b], ob["count"][b],
                              ob["ws"][b], *pw) for b in range(2)]
        gemm = [_prepared_args(W, B, L, self.stats, self.tok, self.conf, self.lse, self.entropy,
                               self.margin, ob["count"][b], ob["ws"][b]) for b in range(2)]
        sel = [self._select_call(ob["row_idx"][b], ob["seq_off"][b], win_lo, win_hi)
               for b in range(2)]
        s_h, ps_h = _stream(s), _stream(ps)
        prepped = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        cur = torch.cuda.current_stream(self.device)
        ps.wait_stream(s)                            # inputs written before the call are ready
        if cur != s:
            ps.wait_stream(cur)
        lazy = not isinstance(batches, (list, tuple))
        last = 0
        for i, (H, M) in enumerate(batches):
            b = i & 1
            if lazy:                                 # written on the current stream as yielded
                ready = torch.cuda.Event()
                ready.record(torch.cuda.current_stream(self.device))
                ps.wait_event(ready)
            if i >= 2:
                ps.wait_event(used[b])               # step i-2 no longer reads this workspace
            _check(lb.dllm_prepare_rows(*_step_inputs(H, M, B, L, d), B, L, d, V, *prep[b], ps_h),
                   "dllm_prepare_rows")
            prepped[b].record(ps)
            s.wait_event(prepped[b])
            _check(lb.dllm_masked_logits_prepared(*gemm[b], s_h), "dllm_masked_logits_prepared")
            fn, args, name = sel[b]
            _check(fn(*args, s_h), name)
            used[b].record(s)
            if sel_out is not None:
                with torch.cuda.stream(s):
                    sel_out[i].copy_(self.sel_buf, non_blocking=True)
            last = b
        if last == 1:                                # leave the last step's compaction in place
            with torch.cuda.stream(s):
                self.row_idx.copy_(ob["row_idx"][1])
                self.seq_off.copy_(ob["seq_off"][1])
                self.count.copy_(ob["count"][1])
        return self._outputs()

    def h2d_bytes_zero_copy(self, count: int) -> int:
        """Bytes one pipelined step reads from host memory: the mask and the masked rows."""
        return self.B * self.L + count * self.d * 2

    def h2d_bytes(self) -> int:
        return self.B * self.L * self.d * 2 + self.B * self.L

    def d2h_bytes(self) -> int:
        return self.sel_buf.numel() * 4
