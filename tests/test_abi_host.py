"""The C ABI on a machine without a GPU: the library loads, exports every entry
point include/dpo.h declares, and rejects bad arguments on the host before any
CUDA call (errors leave outputs untouched and need no device)."""
import ctypes
import os
import re

import numpy as np
import pytest

from preference_alignment_b200 import build as B
from preference_alignment_b200 import libdpo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dpo.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return libdpo.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dpo_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("dpo_workspace_size", "dpo_seq_logprobs", "dpo_loss", "dpo_backward", "dpo_check",
              "dpo_status_string", "dpo_version", "dpo_set_wait_budget_ms"):
        assert n in names
    text = open(HEADER).read()
    assert "torch" not in re.sub(r"/\*.*?\*/", "", text, flags=re.S).lower()
    assert 'extern "C"' in text


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} is declared in dpo.h but not exported"


def test_status_strings_and_version(lib):
    for code in range(7):
        assert libdpo.status_string(code)
    assert libdpo.status_string(99) == "unknown status"
    assert libdpo.version() == 300


FAKE = 0x10000  # never dereferenced: every call below fails its host checks first


def _batch(R=4, L=32, d=64, V=100, dtype="bf16", P=None, C=None, H=FAKE, W=FAKE, tokens=FAKE):
    P = np.full(R, 4, np.int32) if P is None else np.asarray(P, np.int32)
    C = np.full(R, 10, np.int32) if C is None else np.asarray(C, np.int32)
    return libdpo.BatchArgs(H, W, tokens, P, C, R=R, L=L, d=d, V=V, dtype=dtype)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype="f16"), libdpo.ERR_UNSUPPORTED),          # fp16 refused
    (dict(dtype=7), libdpo.ERR_INVALID_ARG),
    (dict(d=60), libdpo.ERR_UNSUPPORTED),                  # d must be a multiple of 8
    (dict(R=0), libdpo.ERR_INVALID_ARG),
    (dict(L=1), libdpo.ERR_INVALID_ARG),
    (dict(V=0), libdpo.ERR_INVALID_ARG),
    (dict(V=(1 << 24) + 1), libdpo.ERR_INVALID_ARG),
    (dict(P=[0, 4, 4, 4]), libdpo.ERR_INVALID_ARG),        # no predictor for the first token
    (dict(C=[-1, 10, 10, 10]), libdpo.ERR_INVALID_ARG),
    (dict(P=[20, 4, 4, 4], C=[13, 10, 10, 10]), libdpo.ERR_INVALID_ARG),  # P + C > L
    (dict(H=FAKE + 8), libdpo.ERR_INVALID_ARG),            # H not 16-byte aligned
    (dict(W=0), libdpo.ERR_INVALID_ARG),                   # null W
])
def test_workspace_size_rejects(lib, kw, code):
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.workspace_size(_batch(**kw))
    assert e.value.status == code


def test_workspace_sizes_are_consistent(lib):
    f1, b1, m1 = libdpo.workspace_size(_batch())
    assert f1 % 256 == 0 and b1 % 256 == 0 and m1 % 256 == 0
    assert m1 <= b1
    # more scored positions never need less
    f2, b2, m2 = libdpo.workspace_size(_batch(C=[20, 20, 20, 20]))
    assert f2 >= f1 and b2 >= b1
    # the backward workspace grows with Nc * V (the bf16 dz chunk), the forward with Nc * d
    f3, b3, _ = libdpo.workspace_size(_batch(V=10000))
    assert b3 - b1 >= 40 * (10000 - 100) * 2 * 0.99
    # an empty batch still gets a valid, small workspace
    f0, b0, m0 = libdpo.workspace_size(_batch(C=[0, 0, 0, 0]))
    assert 0 < f0 <= f1 and 0 < m0 <= b0


def test_calls_fail_on_the_host_and_leave_outputs_alone(lib):
    out = np.full(4, 7.0, np.float32)      # host array: must never be written
    b = _batch(P=[0, 4, 4, 4])
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.seq_logprobs(b, False, out, None, None, FAKE, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    b = _batch()
    with pytest.raises(libdpo.DpoError) as e:   # no workspace
        libdpo.seq_logprobs(b, False, out, None, None, 0, ws_bytes=0)
    assert e.value.status == libdpo.ERR_WORKSPACE
    with pytest.raises(libdpo.DpoError) as e:   # misaligned workspace
        libdpo.seq_logprobs(b, False, out, None, None, FAKE + 16, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_WORKSPACE
    with pytest.raises(libdpo.DpoError) as e:   # want_grad without lse_state
        libdpo.seq_logprobs(b, True, out, None, None, FAKE, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    with pytest.raises(libdpo.DpoError) as e:   # backward without row coefficients
        libdpo.backward(b, FAKE, None, None, FAKE, False, FAKE, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    with pytest.raises(libdpo.DpoError) as e:   # dW not 16-byte aligned
        libdpo.backward(b, FAKE, FAKE, None, FAKE + 4, False, FAKE, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    with pytest.raises(libdpo.DpoError) as e:   # dH not 16-byte aligned
        libdpo.backward(b, FAKE, FAKE, FAKE + 8, FAKE, False, FAKE, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    bl = _batch(L=128, C=[100, 100, 100, 100])    # 400 scored positions: chunked below bwd
    _, bwl, mnl = libdpo.workspace_size(bl)
    assert mnl < bwl
    with pytest.raises(libdpo.DpoError) as e:   # dW deferred, but dz would not stay whole
        libdpo.backward(bl, FAKE, FAKE, None, None, False, FAKE, ws_bytes=mnl)
    assert e.value.status == libdpo.ERR_WORKSPACE
    f, bw, mn = libdpo.workspace_size(b)
    with pytest.raises(libdpo.DpoError) as e:   # backward workspace below the minimum
        libdpo.backward(b, FAKE, FAKE, None, FAKE, False, FAKE, ws_bytes=mn - 256)
    assert e.value.status == libdpo.ERR_WORKSPACE
    assert np.all(out == 7.0)


@pytest.mark.parametrize("args", [
    dict(B=0), dict(layout=2), dict(beta=0.0), dict(beta=-1.0), dict(beta=float("nan")),
    dict(grad_scale=float("inf")), dict(pol=None), dict(loss_out=None),
])
def test_loss_rejects(lib, args):
    a = dict(B=2, layout="halves", pol=FAKE, ref=FAKE, beta=0.1, grad_scale=1.0, loss_out=FAKE)
    a.update(args)
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.loss(a["B"], a["layout"], a["pol"], a["ref"], a["beta"], a["grad_scale"],
                    a["loss_out"])
    assert e.value.status == libdpo.ERR_INVALID_ARG


@pytest.mark.parametrize("v0,v1,dW,max_sms,ws,code", [
    (4, 96, FAKE, 0, 1 << 30, libdpo.ERR_INVALID_ARG),     # v_begin not a multiple of 8
    (0, 101, FAKE, 0, 1 << 30, libdpo.ERR_INVALID_ARG),    # past V
    (16, 8, FAKE, 0, 1 << 30, libdpo.ERR_INVALID_ARG),     # empty-reversed range
    (0, 90, FAKE, 0, 1 << 30, libdpo.ERR_INVALID_ARG),     # v_end neither 8k nor V
    (0, 100, None, 0, 1 << 30, libdpo.ERR_INVALID_ARG),    # no dW
    (0, 100, FAKE, -1, 1 << 30, libdpo.ERR_INVALID_ARG),   # negative SM budget
    (0, 100, FAKE, 0, 0, libdpo.ERR_WORKSPACE),            # no workspace
])
def test_backward_dw_rejects(lib, v0, v1, dW, max_sms, ws, code):
    b = _batch()
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.backward_dw(b, v0, v1, dW, False, FAKE if ws else 0, ws_bytes=ws, max_sms=max_sms)
    assert e.value.status == code


def test_backward_dh_and_dw_need_the_whole_dz(lib):
    b = _batch(L=128, C=[100, 100, 100, 100])
    _, bw, mn = libdpo.workspace_size(b)
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.backward_dw(b, 0, 100, FAKE, False, FAKE, ws_bytes=mn)
    assert e.value.status == libdpo.ERR_WORKSPACE
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.backward_dh(b, FAKE, FAKE, ws_bytes=bw - 256)
    assert e.value.status == libdpo.ERR_WORKSPACE
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.backward_dh(b, None, FAKE, ws_bytes=bw)
    assert e.value.status == libdpo.ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(pairs_total=1), dict(pairs_total=-3),
                                dict(nll_tokens_total=-1)])
def test_loss_ex_rejects_bad_data_parallel_counts(lib, kw):
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.loss_ex(2, "halves", FAKE, FAKE, 0.1, 1.0, FAKE, **kw)
    assert e.value.status == libdpo.ERR_INVALID_ARG


def test_noalloc_refuses_oversized_batches_on_the_host(lib):
    b = _batch(R=2, L=4096, d=4096, V=1000, P=[1, 1], C=[4095, 4095])
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.seq_logprobs_noalloc(b, False, FAKE, None, None)
    assert e.value.status == libdpo.ERR_WORKSPACE


def test_wait_budget_roundtrip(lib):
    old = libdpo.set_wait_budget_ms(1234)
    assert libdpo.set_wait_budget_ms(old) == 1234


@pytest.mark.parametrize("kw", [dict(normalize=True), dict(nll_weight=0.5),
                                dict(nll_weight=-1.0, completion_len=FAKE),
                                dict(nll_weight=float("nan"), completion_len=FAKE)])
def test_loss_ex_rejects_bad_options(lib, kw):
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.loss_ex(2, "halves", FAKE, FAKE, 0.1, 1.0, FAKE, **kw)
    assert e.value.status == libdpo.ERR_INVALID_ARG


def test_loss_needs_a_reference_unless_reference_free(lib):
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.loss_ex(2, "halves", FAKE, None, 0.1, 1.0, FAKE)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.loss(2, "halves", FAKE, None, 0.1, 1.0, FAKE)
    assert e.value.status == libdpo.ERR_INVALID_ARG


def test_loss_ex_rejects_a_reference_free_flag_other_than_0_or_1(lib):
    fn = lib.dpo_loss_ex
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.c_int32, ctypes.c_int32, vp, vp, ctypes.c_float, ctypes.c_float,
                   ctypes.POINTER(libdpo.LossOptions), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    opt = libdpo.LossOptions(0, 0.0, None, 0, 0, 2)
    assert fn(2, 0, FAKE, None, 0.1, 1.0, ctypes.byref(opt), FAKE, None, None, None, None, None,
              None, None, None) == libdpo.ERR_INVALID_ARG


@pytest.mark.parametrize("kw,layout,means,ws,code", [
    (dict(R=3, P=[4, 4, 4], C=[10, 10, 10]), "halves", FAKE, FAKE, libdpo.ERR_INVALID_ARG),  # odd R
    (dict(), 5, FAKE, FAKE, libdpo.ERR_INVALID_ARG),                                     # layout
    (dict(), "halves", None, FAKE, libdpo.ERR_INVALID_ARG),                              # no output
    (dict(dtype="f16"), "halves", FAKE, FAKE, libdpo.ERR_UNSUPPORTED),
    (dict(), "halves", FAKE, FAKE + 16, libdpo.ERR_WORKSPACE),                           # misaligned
    (dict(), "halves", FAKE, None, libdpo.ERR_WORKSPACE),
])
def test_logits_mean_rejects(lib, kw, layout, means, ws, code):
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.logits_mean(_batch(**kw), layout, means, ws, ws_bytes=1 << 30)
    assert e.value.status == code


def test_forward_workspace_covers_the_logits_mean(lib):
    # d = 65536 with a single scored position: the column-sum partials set the size
    f, _, _ = libdpo.workspace_size(_batch(R=2, L=4, d=65536, V=16, P=[1, 1], C=[1, 0]))
    slabs, groups = 65536 // 256, 65536 // 32
    assert f >= (3 * (1024 // slabs) * 65536 + 2 * groups) * 8


@pytest.mark.parametrize("offset,total,code", [
    (-1, 100, libdpo.ERR_INVALID_ARG),
    (1, 100, libdpo.ERR_INVALID_ARG),            # offset + V = 101 > total
    (0, (1 << 24) + 1, libdpo.ERR_INVALID_ARG),
    (0, 0, libdpo.ERR_INVALID_ARG),
])
def test_shard_calls_reject_windows_outside_the_head(lib, offset, total, code):
    b = _batch(V=100)
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.shard_logprob_parts(b, offset, total, FAKE, FAKE, FAKE, ws_bytes=1 << 30)
    assert e.value.status == code
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.shard_backward(b, offset, total, FAKE, FAKE, None, FAKE, False, FAKE,
                              ws_bytes=1 << 30)
    assert e.value.status == code


def test_shard_calls_reject_missing_outputs_and_workspace(lib):
    b = _batch(V=100)
    for lse, zy in ((None, FAKE), (FAKE, None)):
        with pytest.raises(libdpo.DpoError) as e:
            libdpo.shard_logprob_parts(b, 0, 300, lse, zy, FAKE, ws_bytes=1 << 30)
        assert e.value.status == libdpo.ERR_INVALID_ARG
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.shard_logprob_parts(b, 0, 300, FAKE, FAKE, FAKE + 16, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_WORKSPACE
    for total, n, seq in ((99, 1, FAKE), (300, 0, FAKE), (300, 2, None), ((1 << 24) + 1, 2, FAKE)):
        with pytest.raises(libdpo.DpoError) as e:
            libdpo.shard_combine(b, total, n, FAKE, FAKE, seq, None, None, FAKE, ws_bytes=1 << 30)
        assert e.value.status == libdpo.ERR_INVALID_ARG


@pytest.mark.parametrize("R,L,d,V", [(16, 512, 2048, 32000), (8, 2048, 4096, 128256),
                                     (4, 4096, 2048, 151936), (4, 300, 128, 700),
                                     (2, 900, 256, 70001), (2, 8, 8, 1 << 24)])
def test_dh_split_plan_matches_the_bench_launch_count(lib, R, L, d, V):
    """The backward workspace holds split-K partial sums exactly when the library splits
    dH over the vocabulary (compared with the diagnostic bit that turns the split off),
    and bench.py's launch count restates the same plan."""
    import bench
    P = np.full(R, 1, np.int32)
    C = np.full(R, L - 1, np.int32)
    b = _batch(R=R, L=L, d=d, V=V, P=P, C=C)
    _, bw_split, _ = libdpo.workspace_size(b)
    old = libdpo.set_gemm_variant(256)
    try:
        _, bw_plain, _ = libdpo.workspace_size(b)
    finally:
        libdpo.set_gemm_variant(old)
    nc = int(C.sum())
    split = bw_split > bw_plain
    assert (bench.dh_parts(nc, d, V) > 1) == split        # one split launch + its reduce
    if split:                                             # >= one part's fp32 partial sums
        assert bw_split - bw_plain >= nc * d * 4


@pytest.mark.parametrize("n_ranks,rank,per,recv,code", [
    (0, 0, 50, FAKE, libdpo.ERR_INVALID_ARG),        # no ranks
    (9, 0, 10, FAKE, libdpo.ERR_INVALID_ARG),        # beyond DPO_MAX_SCATTER_RANKS
    (2, 2, 50, FAKE, libdpo.ERR_INVALID_ARG),        # rank out of range
    (2, -1, 50, FAKE, libdpo.ERR_INVALID_ARG),
    (3, 0, 50, FAKE, libdpo.ERR_INVALID_ARG),        # the last rank would own no row (V 100)
    (2, 0, 0, FAKE, libdpo.ERR_INVALID_ARG),         # no rows per rank
    (2, 0, 50, FAKE + 4, libdpo.ERR_INVALID_ARG),    # a misaligned receive buffer
    (2, 0, 50, 0, libdpo.ERR_INVALID_ARG),           # a missing receive buffer
])
def test_backward_dw_scatter_rejects(lib, n_ranks, rank, per, recv, code):
    """The library's own checks, through the raw call (all 8 buffer slots filled)."""
    import ctypes
    b = _batch()
    x = libdpo.DwScatter(n_ranks, rank, per)
    for i in range(libdpo.MAX_SCATTER_RANKS):
        x.recv[i] = recv
    st = lib.dpo_backward_dw_scatter(ctypes.byref(b.c), ctypes.byref(x), 0, FAKE, 1 << 30, None)
    assert st == code


def test_backward_dw_scatter_refuses_fp32_and_small_workspaces(lib):
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.backward_dw_scatter(_batch(dtype="f32"), 1, 0, 100, [FAKE], FAKE, ws_bytes=1 << 30)
    assert e.value.status == libdpo.ERR_UNSUPPORTED
    b = _batch(L=128, C=[100, 100, 100, 100])
    _, bw, mn = libdpo.workspace_size(b)
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.backward_dw_scatter(b, 1, 0, 100, [FAKE], FAKE, ws_bytes=mn)
    assert e.value.status == libdpo.ERR_WORKSPACE


@pytest.mark.parametrize("kw", [dict(n_slots=0), dict(n_slots=9), dict(d=12), dict(rows=-1),
                                dict(recv=FAKE + 4), dict(out=None)])
def test_dw_reduce_slots_rejects(lib, kw):
    a = dict(recv=FAKE, n_slots=2, rows=10, d=64, out=FAKE)
    a.update(kw)
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.dw_reduce_slots(a["recv"], a["n_slots"], a["rows"], a["d"], a["out"])
    assert e.value.status == libdpo.ERR_INVALID_ARG


def test_ipc_calls_fail_cleanly_without_device_memory(lib):
    with pytest.raises(libdpo.DpoError):
        libdpo.ipc_export(FAKE)                      # not device memory of this process
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.ipc_close(0)
    assert e.value.status == libdpo.ERR_INVALID_ARG


def test_binding_refuses_strided_views(lib):
    """The C ABI reads dense arrays: a transposed or column-sliced device buffer is refused
    by the binding instead of being passed as the address of its first element (host row
    tables are copied to dense int32 arrays by BatchArgs)."""
    import torch
    dense = torch.zeros(2, 4)
    with pytest.raises(ValueError):
        libdpo.loss(2, "halves", dense.t(), FAKE, 0.1, 1.0, FAKE)
    with pytest.raises(ValueError):
        libdpo.loss(2, "halves", FAKE, FAKE, 0.1, 1.0, FAKE, margins=torch.zeros(2, 2)[:, 0])


def test_binding_refuses_buffers_of_another_element_type(lib):
    """Outputs the header declares fp32 refuse fp64 tensors, tokens refuse int64, and the
    bf16 batch refuses fp32 weights, before any call into the library."""
    import torch
    with pytest.raises(TypeError):
        libdpo.loss(2, "halves", FAKE, FAKE, 0.1, 1.0, torch.zeros(1, dtype=torch.float64))
    with pytest.raises(TypeError):
        libdpo.BatchArgs(FAKE, FAKE, torch.zeros(4, 8, dtype=torch.int64), np.ones(4, np.int32),
                         np.ones(4, np.int32), R=4, L=8, d=8, V=8)
    with pytest.raises(TypeError):
        libdpo.BatchArgs(FAKE, torch.zeros(8, 8), FAKE, np.ones(4, np.int32), np.ones(4, np.int32),
                         R=4, L=8, d=8, V=8, dtype="bf16")
    b = libdpo.BatchArgs(FAKE, torch.zeros(8, 8, dtype=torch.bfloat16), FAKE, np.ones(4, np.int32),
                         np.ones(4, np.int32), R=4, L=8, d=8, V=8, dtype="bf16")
    assert b.c.V == 8
