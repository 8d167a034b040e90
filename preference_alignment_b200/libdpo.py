"""ctypes binding of libdpo (include/dpo.h): argument marshalling only.

Every step of the DPO head path runs in the CUDA library; this module turns
Python arguments into the C ABI's plain pointers and sizes. Device buffers may
be given as torch tensors (their data_ptr() is passed) or as integer device
addresses; host row-length arrays as numpy int32 arrays. The names follow the C
entry points without the `dpo_` prefix.

The module refuses to run without the compiled library: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libdpo.so")

# dpo_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BAD_TARGET, ERR_WORKSPACE = range(7)
# dpo_dtype
BF16, F32, F16 = 0, 1, 2
# dpo_layout
PAIRS_HALVES, PAIRS_ADJACENT = 0, 1

LAYOUTS = {"halves": PAIRS_HALVES, "adjacent": PAIRS_ADJACENT}
DTYPES = {"bf16": BF16, "f32": F32, "f16": F16}


class DpoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Batch(ctypes.Structure):
    _fields_ = [
        ("R", ctypes.c_int32), ("L", ctypes.c_int32), ("d", ctypes.c_int32), ("V", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("H", ctypes.c_void_p), ("W", ctypes.c_void_p), ("tokens", ctypes.c_void_p),
        ("prompt_len", ctypes.c_void_p), ("completion_len", ctypes.c_void_p),
    ]


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdpo.so (built in-tree by preference_alignment_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libdpo.so is not built ({path}); run "
                           "`python -m preference_alignment_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i32, u32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint32, ctypes.c_float
    bp = ctypes.POINTER(Batch)
    szp = ctypes.POINTER(ctypes.c_size_t)
    lib.dpo_workspace_size.argtypes = [bp, szp, szp, szp]
    lib.dpo_seq_logprobs.argtypes = [bp, ctypes.c_int, vp, vp, vp, vp, sz, vp]
    lib.dpo_loss.argtypes = [i32, i32, vp, vp, f32, f32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.dpo_backward.argtypes = [bp, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp]
    lib.dpo_check.argtypes = [vp]
    lib.dpo_set_wait_budget_ms.argtypes = [u32]
    lib.dpo_set_wait_budget_ms.restype = u32
    lib.dpo_status_string.argtypes = [ctypes.c_int]
    lib.dpo_status_string.restype = ctypes.c_char_p
    lib.dpo_version.restype = i32
    for name in ("dpo_workspace_size", "dpo_seq_logprobs", "dpo_loss", "dpo_backward", "dpo_check"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


# element types a buffer argument may have (bf16 data may also arrive as its 16-bit pattern)
_KINDS = {"f32": ("float32",), "i32": ("int32",), "f16": ("float16",),
          "bf16": ("bfloat16", "int16", "uint16")}


def _ptr(x, kind: Optional[str] = None) -> Optional[int]:
    """Device/host address of a torch tensor, numpy array or raw integer; None -> NULL.
    The C ABI reads dense row-major arrays of the element type its header names, so a
    strided view (a transpose, a column slice) or a tensor of another element type
    (`kind`: "f32", "i32", "bf16") is refused rather than passed on; a raw integer
    address is taken as it is."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        name = str(x.dtype).replace("torch.", "")
        ptr = x.data_ptr()
        dense = x.numel() == 0 or x.is_contiguous()
        shape = tuple(x.shape)
    elif isinstance(x, np.ndarray):
        name = x.dtype.name
        ptr = x.ctypes.data
        dense = bool(x.flags["C_CONTIGUOUS"])
        shape = x.shape
    else:
        raise TypeError(f"cannot take the address of {type(x)}")
    if not dense:
        raise ValueError(f"buffer of shape {shape} is not contiguous")
    if kind is not None and name not in _KINDS[kind]:
        raise TypeError(f"expected a {kind} buffer, got {name} (shape {shape})")
    return ptr


def _stream(s) -> Optional[int]:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str):
    if status != OK:
        raise DpoError(status, where)


def status_string(status: int) -> str:
    return load().dpo_status_string(int(status)).decode()


def version() -> int:
    return load().dpo_version()


def set_wait_budget_ms(ms: int) -> int:
    return load().dpo_set_wait_budget_ms(int(ms))


_HW_KIND = {BF16: "bf16", F32: "f32", F16: "f16"}


class BatchArgs:
    """A dpo_batch plus the Python objects its pointers refer to (kept alive)."""

    def __init__(self, H, W, tokens, prompt_len, completion_len, R=None, L=None, d=None, V=None,
                 dtype="bf16"):
        self.prompt_len = np.ascontiguousarray(prompt_len, dtype=np.int32)
        self.completion_len = np.ascontiguousarray(completion_len, dtype=np.int32)
        shapeH = tuple(H.shape) if hasattr(H, "shape") else None
        shapeW = tuple(W.shape) if hasattr(W, "shape") else None
        R = R if R is not None else shapeH[0]
        L = L if L is not None else shapeH[1]
        d = d if d is not None else shapeH[2]
        V = V if V is not None else shapeW[0]
        self.keep = (H, W, tokens)
        self.dtype = DTYPES.get(dtype, dtype) if isinstance(dtype, str) else int(dtype)
        self.c = Batch(int(R), int(L), int(d), int(V), self.dtype,
                       _ptr(H, _HW_KIND.get(self.dtype)), _ptr(W, _HW_KIND.get(self.dtype)),
                       _ptr(tokens, "i32"), self.prompt_len.ctypes.data,
                       self.completion_len.ctypes.data)

    @property
    def n_scored(self) -> int:
        return int(self.completion_len.sum())


def workspace_size(batch: BatchArgs):
    """(fwd_bytes, bwd_bytes, bwd_min_bytes) for this batch."""
    f, b, m = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().dpo_workspace_size(ctypes.byref(batch.c), ctypes.byref(f), ctypes.byref(b),
                                     ctypes.byref(m)), "dpo_workspace_size")
    return f.value, b.value, m.value


def _nbytes(ws, ws_bytes):
    if ws_bytes is not None:
        return int(ws_bytes)
    if hasattr(ws, "numel"):
        return ws.numel() * ws.element_size()
    raise ValueError("ws_bytes is required for a raw workspace address")


def seq_logprobs(batch: BatchArgs, want_grad: bool, seq_logp, tok_logp, lse_state, ws,
                 ws_bytes=None, stream=None):
    _check(load().dpo_seq_logprobs(ctypes.byref(batch.c), 1 if want_grad else 0,
                                   _ptr(seq_logp, "f32"), _ptr(tok_logp, "f32"),
                                   _ptr(lse_state, "f32"), _ptr(ws), _nbytes(ws, ws_bytes),
                                   _stream(stream)), "dpo_seq_logprobs")


def loss(B: int, layout, pol, ref, beta: float, grad_scale: float, loss_out, accuracy=None,
         margins=None, chosen_rewards=None, rejected_rewards=None, weights=None, row_coef=None,
         stream=None):
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    _check(load().dpo_loss(int(B), lay, _ptr(pol, "f32"), _ptr(ref, "f32"), float(beta),
                           float(grad_scale), _ptr(loss_out, "f32"), _ptr(accuracy, "f32"),
                           _ptr(margins, "f32"), _ptr(chosen_rewards, "f32"),
                           _ptr(rejected_rewards, "f32"), _ptr(weights, "f32"),
                           _ptr(row_coef, "f32"), _stream(stream)),
           "dpo_loss")


class LossOptions(ctypes.Structure):
    _fields_ = [("normalize", ctypes.c_int32), ("nll_weight", ctypes.c_float),
                ("completion_len", ctypes.c_void_p), ("pairs_total", ctypes.c_int32),
                ("nll_tokens_total", ctypes.c_int64), ("reference_free", ctypes.c_int32)]


def loss_ex(B: int, layout, pol, ref, beta: float, grad_scale: float, loss_out, accuracy=None,
            margins=None, chosen_rewards=None, rejected_rewards=None, weights=None, row_coef=None,
            nll=None, normalize=False, nll_weight=0.0, completion_len=None, pairs_total=0,
            nll_tokens_total=0, reference_free=False, stream=None):
    """dpo_loss_ex: length-normalised and/or SFT-NLL variants (completion_len: device int32 [2B]);
    pairs_total / nll_tokens_total > 0 make the outputs this rank's share of a data-parallel
    batch of that many pairs / chosen tokens; reference_free reads the reference sums as 0
    (ref is then not read and may be None)."""
    lib = load()
    fn = lib.dpo_loss_ex
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.c_int32, ctypes.c_int32, vp, vp, ctypes.c_float, ctypes.c_float,
                   ctypes.POINTER(LossOptions), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    opt = LossOptions(1 if normalize else 0, float(nll_weight), _ptr(completion_len, "i32"),
                      int(pairs_total), int(nll_tokens_total), 1 if reference_free else 0)
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    _check(fn(int(B), lay, _ptr(pol, "f32"), _ptr(ref, "f32"), float(beta), float(grad_scale),
              ctypes.byref(opt), _ptr(loss_out, "f32"), _ptr(accuracy, "f32"), _ptr(margins, "f32"),
              _ptr(chosen_rewards, "f32"), _ptr(rejected_rewards, "f32"), _ptr(weights, "f32"),
              _ptr(row_coef, "f32"), _ptr(nll, "f32"), _stream(stream)),
           "dpo_loss_ex")


def backward(batch: BatchArgs, lse_state, row_coef, dH, dW, accumulate_dW: bool, ws,
             ws_bytes=None, stream=None):
    _check(load().dpo_backward(ctypes.byref(batch.c), _ptr(lse_state, "f32"),
                               _ptr(row_coef, "f32"), _ptr(dH, "f32"), _ptr(dW, "f32"),
                               1 if accumulate_dW else 0, _ptr(ws),
                               _nbytes(ws, ws_bytes), _stream(stream)), "dpo_backward")


def backward_dw(batch: BatchArgs, v_begin: int, v_end: int, dW, accumulate_dW: bool, ws,
                ws_bytes=None, max_sms: int = 0, stream=None):
    """dpo_backward_dw: rows [v_begin, v_end) of dW from the dz a preceding
    backward(dW=None) left in the workspace ws (max_sms > 0 caps the SMs it uses)."""
    lib = load()
    fn = lib.dpo_backward_dw
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.c_int32, ctypes.c_int32, vp, ctypes.c_int,
                   ctypes.c_int32, vp, ctypes.c_size_t, vp]
    fn.restype = ctypes.c_int
    _check(fn(ctypes.byref(batch.c), int(v_begin), int(v_end), _ptr(dW, "f32"),
              1 if accumulate_dW else 0, int(max_sms), _ptr(ws), _nbytes(ws, ws_bytes),
              _stream(stream)), "dpo_backward_dw")


def backward_dh(batch: BatchArgs, dH, ws, ws_bytes=None, max_sms: int = 0, stream=None):
    """dpo_backward_dh: dH (fully written) from the dz a preceding backward(dW=None) left in ws."""
    lib = load()
    fn = lib.dpo_backward_dh
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(Batch), vp, ctypes.c_int32, vp, ctypes.c_size_t, vp]
    fn.restype = ctypes.c_int
    _check(fn(ctypes.byref(batch.c), _ptr(dH, "f32"), int(max_sms), _ptr(ws), _nbytes(ws, ws_bytes),
              _stream(stream)), "dpo_backward_dh")


MAX_SCATTER_RANKS = 8


class DwScatter(ctypes.Structure):
    _fields_ = [("n_ranks", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("rows_per_rank", ctypes.c_int32),
                ("recv", ctypes.c_void_p * MAX_SCATTER_RANKS)]


def backward_dw_scatter(batch: BatchArgs, n_ranks: int, rank: int, rows_per_rank: int, recv, ws,
                        ws_bytes=None, max_sms: int = 0, stream=None):
    """dpo_backward_dw_scatter: this rank's dW contribution, each row stored into its owner's
    receive buffer (recv: one device address or tensor per rank, as this process maps it)."""
    lib = load()
    fn = lib.dpo_backward_dw_scatter
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.POINTER(DwScatter), ctypes.c_int32, vp,
                   ctypes.c_size_t, vp]
    fn.restype = ctypes.c_int
    ptrs = [_ptr(r, "f32") for r in recv]
    if len(ptrs) != n_ranks or n_ranks > MAX_SCATTER_RANKS:
        raise ValueError("recv needs one buffer per rank (at most 8 ranks)")
    x = DwScatter(int(n_ranks), int(rank), int(rows_per_rank),
                  (ctypes.c_void_p * MAX_SCATTER_RANKS)(*(ptrs + [None] * (MAX_SCATTER_RANKS - n_ranks))))
    _check(fn(ctypes.byref(batch.c), ctypes.byref(x), int(max_sms), _ptr(ws), _nbytes(ws, ws_bytes),
              _stream(stream)), "dpo_backward_dw_scatter")


def dw_reduce_slots(recv, n_slots: int, rows: int, d: int, dW_shard, accumulate: bool = False,
                    stream=None):
    """dpo_dw_reduce_slots: dW_shard (+)= the sum of recv's n_slots slots, in slot order."""
    lib = load()
    fn = lib.dpo_dw_reduce_slots
    vp = ctypes.c_void_p
    fn.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, ctypes.c_int, vp]
    fn.restype = ctypes.c_int
    _check(fn(_ptr(recv, "f32"), int(n_slots), int(rows), int(d), _ptr(dW_shard, "f32"),
              1 if accumulate else 0,
              _stream(stream)), "dpo_dw_reduce_slots")


class IpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


def ipc_export(ptr):
    """dpo_ipc_export: (64-byte handle as bytes, byte offset) of the allocation holding ptr."""
    lib = load()
    fn = lib.dpo_ipc_export
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(IpcHandle), ctypes.POINTER(ctypes.c_size_t)]
    fn.restype = ctypes.c_int
    h, off = IpcHandle(), ctypes.c_size_t()
    _check(fn(_ptr(ptr), ctypes.byref(h), ctypes.byref(off)), "dpo_ipc_export")
    return bytes(h.bytes), off.value


def ipc_import(handle: bytes) -> int:
    """dpo_ipc_import: map another process's exported allocation; returns its base address."""
    lib = load()
    fn = lib.dpo_ipc_import
    fn.argtypes = [ctypes.POINTER(IpcHandle), ctypes.POINTER(ctypes.c_void_p)]
    fn.restype = ctypes.c_int
    h = IpcHandle((ctypes.c_ubyte * 64)(*handle))
    base = ctypes.c_void_p()
    _check(fn(ctypes.byref(h), ctypes.byref(base)), "dpo_ipc_import")
    return base.value


def ipc_close(base: int):
    lib = load()
    fn = lib.dpo_ipc_close
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(base), "dpo_ipc_close")


class VocabShard(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_int32), ("total", ctypes.c_int32)]


def shard_logprob_parts(batch: BatchArgs, offset: int, total: int, shard_lse, shard_zy, ws,
                        ws_bytes=None, stream=None):
    """dpo_shard_logprob_parts: per-position (lse, target logit or -inf) over one shard's rows."""
    lib = load()
    fn = lib.dpo_shard_logprob_parts
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.POINTER(VocabShard), vp, vp, vp, ctypes.c_size_t, vp]
    fn.restype = ctypes.c_int
    sh = VocabShard(int(offset), int(total))
    _check(fn(ctypes.byref(batch.c), ctypes.byref(sh), _ptr(shard_lse, "f32"),
              _ptr(shard_zy, "f32"), _ptr(ws),
              _nbytes(ws, ws_bytes), _stream(stream)), "dpo_shard_logprob_parts")


def shard_combine(batch: BatchArgs, total: int, n_shards: int, shard_lse, shard_zy, seq_logp,
                  tok_logp, lse_state, ws, ws_bytes=None, stream=None):
    """dpo_shard_combine: merge gathered [n_shards, Nc] parts into sums, log-probs and lse."""
    lib = load()
    fn = lib.dpo_shard_combine
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, vp, vp,
                   ctypes.c_size_t, vp]
    fn.restype = ctypes.c_int
    _check(fn(ctypes.byref(batch.c), int(total), int(n_shards), _ptr(shard_lse, "f32"),
              _ptr(shard_zy, "f32"), _ptr(seq_logp, "f32"), _ptr(tok_logp, "f32"),
              _ptr(lse_state, "f32"), _ptr(ws), _nbytes(ws, ws_bytes),
              _stream(stream)), "dpo_shard_combine")


def shard_backward(batch: BatchArgs, offset: int, total: int, lse_state, row_coef, dH_part,
                   dW_shard, accumulate_dW: bool, ws, ws_bytes=None, stream=None):
    """dpo_shard_backward: this shard's dW rows and a partial dH (summed over shards = dH)."""
    lib = load()
    fn = lib.dpo_shard_backward
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.POINTER(VocabShard), vp, vp, vp, vp, ctypes.c_int,
                   vp, ctypes.c_size_t, vp]
    fn.restype = ctypes.c_int
    sh = VocabShard(int(offset), int(total))
    _check(fn(ctypes.byref(batch.c), ctypes.byref(sh), _ptr(lse_state, "f32"),
              _ptr(row_coef, "f32"), _ptr(dH_part, "f32"), _ptr(dW_shard, "f32"),
              1 if accumulate_dW else 0, _ptr(ws),
              _nbytes(ws, ws_bytes), _stream(stream)), "dpo_shard_backward")


def logits_mean(batch: BatchArgs, layout, means, ws, ws_bytes=None, stream=None):
    """dpo_logits_mean: means (device float32 [2]) = mean logit of the chosen rows and of the
    rejected rows over every position and vocabulary entry."""
    lib = load()
    fn = lib.dpo_logits_mean
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_size_t, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    _check(fn(ctypes.byref(batch.c), lay, _ptr(means, "f32"), _ptr(ws), _nbytes(ws, ws_bytes),
              _stream(stream)), "dpo_logits_mean")


def selftest_wait_timeout(budget_ms: int, stream=None):
    """Launch the bounded-wait self-test (records DPO_ERR_TIMEOUT after budget_ms)."""
    lib = load()
    fn = lib.dpo_selftest_wait_timeout
    fn.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(int(budget_ms), _stream(stream)), "dpo_selftest_wait_timeout")


def fingerprint(data, nbytes, out, stream=None):
    """dpo_fingerprint: 64-bit order-independent hash of a device buffer into out (device uint64)."""
    lib = load()
    fn = lib.dpo_fingerprint
    fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(_ptr(data), int(nbytes), _ptr(out), _stream(stream)), "dpo_fingerprint")


def set_gemm_variant(variant: int) -> int:
    """Mask per GEMM k (forward, dz, dH, dW): bit k runs it on the single-CTA kernel, bit 4 + k
    gives the CTA-pair kernel the static tile schedule instead of tiles claimed in raster order;
    bit 8 keeps dH from being split over the vocabulary (set it before sizing workspaces)."""
    lib = load()
    fn = lib.dpo_set_gemm_variant
    fn.argtypes = [ctypes.c_int32]
    fn.restype = ctypes.c_int32
    return fn(int(variant))


def check(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return load().dpo_check(_stream(stream))


def seq_logprobs_noalloc(batch: BatchArgs, want_grad: bool, seq_logp, tok_logp, lse_state,
                         stream=None):
    """dpo_seq_logprobs_noalloc: the forward with the library's built-in scratch.

    For callers that may not allocate device memory (no workspace argument). The
    batch's forward workspace must fit NOALLOC_SCRATCH_BYTES; calls that overlap on
    the GPU share the scratch and must be serialised.
    """
    lib = load()
    fn = lib.dpo_seq_logprobs_noalloc
    fn.argtypes = [ctypes.POINTER(Batch), ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(ctypes.byref(batch.c), 1 if want_grad else 0, _ptr(seq_logp, "f32"),
              _ptr(tok_logp, "f32"), _ptr(lse_state, "f32"), _stream(stream)),
           "dpo_seq_logprobs_noalloc")


NOALLOC_SCRATCH_BYTES = 32 << 20
