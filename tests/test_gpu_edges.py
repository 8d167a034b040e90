"""Edge cases of the CUDA path against the oracle: extreme and ragged shapes,
argument combinations, and replay of the whole step from a captured CUDA graph."""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import (DeviceWorkload, TOL_GRAD, TOL_LOSS, TOL_TOK, assert_seq_close, np64,
                         rel_frob)

pytestmark = pytest.mark.gpu


def _fwd_bwd_check(w, coef_seed=0, bwd=True):
    import torch
    dw = DeviceWorkload(w)
    H = WL.widen(w.H, w.dtype)
    W = WL.widen(w.W, w.dtype)
    o = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    seq, tok, lse = dw.forward(dw.W, want_grad=True)
    assert libdpo.check() == libdpo.OK
    assert np.abs(np64(tok) - o["tok_logp"]).max() <= TOL_TOK
    assert_seq_close(np64(seq), o["seq_logp"])
    if not bwd:
        return
    coef = np.random.default_rng(coef_seed).normal(0, 0.05, size=w.R).astype(np.float32)
    dH, dW = dw.backward(lse, torch.from_numpy(coef).cuda())
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, coef.astype(np.float64))
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


def test_more_rows_than_one_row_table_launch():
    # R = 1100 > 1024 rows: the row table is uploaded by two launches
    w = WL.make_custom(R=1100, L=10, d=64, V=300, dtype="bf16", seed=61, prompt_range=(1, 6))
    _fwd_bwd_check(w)


def test_vocab_not_a_multiple_of_8():
    # the bf16 dz rows are padded to 1008 columns; the padding must never be read as data
    w = WL.make_custom(R=4, L=200, d=128, V=1001, dtype="bf16", seed=62, prompt_range=(1, 80))
    _fwd_bwd_check(w)


def test_smallest_hidden_size():
    w = WL.make_custom(R=4, L=60, d=8, V=500, dtype="bf16", seed=63, prompt_range=(1, 30))
    _fwd_bwd_check(w)


def test_large_vocab_small_hidden():
    w = WL.make_custom(R=2, L=150, d=64, V=70001, dtype="bf16", seed=64, prompt_range=(1, 40))
    _fwd_bwd_check(w)


def test_scored_positions_exact_multiple_of_tile():
    # Nc = 512 = two 256-row pair tiles, no ragged tail
    w = WL.make_custom(R=4, L=200, d=64, V=300, dtype="bf16", seed=65, prompt_range=(1, 5))
    w.prompt_len[:] = 40
    w.completion_len[:] = 128
    assert w.n_scored == 512
    _fwd_bwd_check(w)


def test_some_rows_empty():
    w = WL.make_custom(R=6, L=120, d=64, V=400, dtype="bf16", seed=66, prompt_range=(1, 50))
    w.completion_len[[1, 4]] = 0
    _fwd_bwd_check(w)


def test_backward_without_dH():
    import torch
    w = WL.make_custom(R=4, L=150, d=128, V=600, dtype="bf16", seed=67, prompt_range=(1, 50))
    dw = DeviceWorkload(w)
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.linspace(-0.1, 0.1, 4, device="cuda")
    _, dW1 = dw.backward(lse, coef)
    _, dW2 = dw.backward(lse, coef, want_dH=False)
    assert libdpo.check() == libdpo.OK
    assert np.array_equal(np64(dW1), np64(dW2))


def test_adjacent_layout_bf16_end_to_end():
    w = WL.make_custom(R=8, L=160, d=256, V=900, dtype="bf16", seed=68, layout="adjacent",
                       prompt_range=(1, 60), ref_std=0.05)
    dw = DeviceWorkload(w)
    H = WL.widen(w.H, "bf16")
    op = O.seq_logprobs(H, WL.widen(w.W, "bf16"), w.tokens, w.prompt_len, w.completion_len)
    orf = O.seq_logprobs(H, WL.widen(w.W_ref, "bf16"), w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, "adjacent")
    pol, _, _ = dw.forward(dw.W, want_grad=False)
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    out = dw.loss(pol, ref)
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS
    np.testing.assert_allclose(np64(out["weights"]), ol["weights"], atol=1e-4)


def test_whole_step_replays_from_a_cuda_graph():
    """The four calls of a step are captured into one CUDA graph and replayed; the replay
    gives the same outputs as the direct calls (all are deterministic)."""
    import torch
    w = WL.make_custom(R=8, L=300, d=256, V=1500, dtype="bf16", seed=69, prompt_range=(1, 100))
    dw = DeviceWorkload(w)
    bp, br = dw.batch(dw.W), dw.batch(dw.W_ref)
    f, b, _ = libdpo.workspace_size(bp)
    ws = torch.empty(max(f, b), dtype=torch.uint8, device="cuda")
    R, B = w.R, w.R // 2
    pol, ref = torch.empty(R, device="cuda"), torch.empty(R, device="cuda")
    lse = torch.empty(w.n_scored, device="cuda")
    outs = [torch.empty(n, device="cuda") for n in (1, 1, B, B, B, B, R)]
    dH = torch.empty(R, w.L, w.d, device="cuda")
    dW = torch.empty(w.V, w.d, device="cuda")

    def step(stream):
        libdpo.seq_logprobs(bp, True, pol, None, lse, ws, stream=stream)
        libdpo.seq_logprobs(br, False, ref, None, None, ws, stream=stream)
        libdpo.loss(B, w.layout, pol, ref, w.beta, 1.0, *outs, stream=stream)
        libdpo.backward(bp, lse, outs[6], dH, dW, False, ws, stream=stream)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step(s.cuda_stream)                      # direct run (also sets up the kernels)
    s.synchronize()
    direct = [t.clone() for t in (pol, ref, lse, *outs, dH, dW)]
    for t in (pol, ref, lse, *outs, dH, dW):
        t.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s.cuda_stream)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert libdpo.check() == libdpo.OK
    for a, b in zip(direct, (pol, ref, lse, *outs, dH, dW)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("shape", [(6, 300, 256, 1000, 2), (8, 200, 200, 777, 3), (2, 700, 128, 2048, 4)])
def test_single_cta_gemm_kernel(shape):
    """The single-CTA GEMM (the fallback when CTA pairs cannot be co-scheduled) stays correct."""
    R, L, d, V, seed = shape
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype="bf16", seed=seed, prompt_range=(1, L // 3),
                       full_rows=1)
    old = libdpo.set_gemm_variant(15)
    try:
        _fwd_bwd_check(w)
    finally:
        libdpo.set_gemm_variant(old)


def test_gemm_variants_agree():
    """Single-CTA and CTA-pair kernels, and dH with or without split-K (0x100), agree
    within rounding; the pair kernel's two tile schedules (claimed in raster order, or
    static round-robin: 0xF0) compute every tile the same way, so they agree bit for bit."""
    import torch
    w = WL.make_custom(R=4, L=400, d=256, V=1500, dtype="bf16", seed=91, prompt_range=(1, 100))
    dw = DeviceWorkload(w)
    outs = []
    for v in (0, 15, 5, 0x100, 0xF0, 0x50):
        old = libdpo.set_gemm_variant(v)
        try:
            seq, tok, lse = dw.forward(dw.W, want_grad=True)
            dH, dW = dw.backward(lse, torch.linspace(-0.1, 0.1, 4, device="cuda"))
        finally:
            libdpo.set_gemm_variant(old)
        assert libdpo.check() == libdpo.OK
        outs.append((np64(tok), np64(dH), np64(dW)))
    for o in outs[1:4]:
        assert np.abs(outs[0][0] - o[0]).max() <= 1e-4
        assert rel_frob(outs[0][1], o[1]) <= 1e-3
        assert rel_frob(outs[0][2], o[2]) <= 1e-3
    for o in outs[4:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(a, b)


@pytest.mark.parametrize("R,L,d,V,seed", [
    (2, 8, 8, 1 << 24, 101),      # the largest vocabulary the boundary accepts (65,536 vocab tiles)
    (2, 8, 65536, 64, 102),       # the largest hidden size (1,024 K blocks per tile)
    (65535, 2, 8, 16, 103),       # the most rows (64 row-table launches, one position each)
])
def test_maximum_sizes(R, L, d, V, seed):
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype="bf16", seed=seed, prompt_range=(1, 1),
                       min_completion=1)
    _fwd_bwd_check(w)


@pytest.mark.parametrize("R,L,d,V,seed", [
    (4, 600, 512, 5000, 111),      # 10 output tiles: dH split into K parts
    (2, 900, 256, 70001, 112),     # long vocabulary, few tiles: one split launch, ragged K
])
def test_split_k_dh_against_the_oracle(R, L, d, V, seed):
    """Shapes whose dH GEMM has too few output tiles to fill the GPU run it as K parts
    of one launch (the workspace holds their fp32 partial sums); the parts are added in
    a fixed order, so dH equals the oracle's within tolerance and repeats bit for bit."""
    import torch
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype="bf16", seed=seed, prompt_range=(1, L // 3),
                       full_rows=1)
    dw = DeviceWorkload(w)
    _, bwd, _ = libdpo.workspace_size(dw.batch())
    nc = w.n_scored
    assert bwd >= nc * ((V + 7) // 8 * 8 * 2 + d * 4)      # dz rows + at least one part
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.from_numpy(np.random.default_rng(seed).normal(0, 0.05, R).astype(np.float32)).cuda()
    dH1, dW1 = dw.backward(lse, coef)
    dH2, dW2 = dw.backward(lse, coef)
    assert libdpo.check() == libdpo.OK
    assert torch.equal(dH1, dH2) and torch.equal(dW1, dW2)
    Hd = WL.widen(w.H, "bf16")
    oH, oW = O.backward(Hd, WL.widen(w.W, "bf16"), w.tokens, w.prompt_len, w.completion_len,
                        coef.double().cpu().numpy())
    assert rel_frob(np64(dH1), oH) <= TOL_GRAD
    assert rel_frob(np64(dW1), oW) <= TOL_GRAD


def test_split_k_dh_in_a_chunked_backward():
    """A workspace smaller than the whole batch's runs the backward in token chunks; with
    dH split over K each chunk's partial sums sit after its dz rows. The result equals the
    one-chunk backward within rounding (the dW chunks add in a different order)."""
    import torch
    w = WL.make_custom(R=4, L=600, d=512, V=5000, dtype="bf16", seed=113, prompt_range=(1, 200),
                       full_rows=1)
    dw = DeviceWorkload(w)
    b = dw.batch()
    _, full, mn = libdpo.workspace_size(b)
    row = (full - mn) // max(1, w.n_scored - 128)          # bytes per position (dz + parts)
    small = mn + 2 * 128 * row                             # 384 positions per chunk
    assert row > ((w.V + 7) // 8 * 8) * 2 and small < full
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.from_numpy(np.random.default_rng(113).normal(0, 0.05, w.R).astype(np.float32)).cuda()
    dH1, dW1 = dw.backward(lse, coef)
    dH2, dW2 = dw.backward(lse, coef, ws_bytes=small)
    assert libdpo.check() == libdpo.OK
    assert rel_frob(np64(dH2), np64(dH1)) < 1e-6
    assert rel_frob(np64(dW2), np64(dW1)) < 1e-5


def test_workspace_contents_do_not_matter():
    """The GEMMs' tile claim counter and every table live in the workspace; each call
    writes what it reads (the counter is zeroed before each launch), so a workspace full
    of garbage gives the same bits as a fresh one."""
    import torch
    w = WL.make_custom(R=6, L=300, d=256, V=3000, dtype="bf16", seed=114, prompt_range=(1, 100),
                       full_rows=2)
    dw = DeviceWorkload(w)
    b = dw.batch()
    fwd, bwd, _ = libdpo.workspace_size(b)
    n = max(fwd, bwd)
    coef = torch.linspace(-0.1, 0.2, w.R, device="cuda")
    outs = []
    for fill in (0x00, 0x7F, 0xFF):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        seq = torch.empty(w.R, device="cuda")
        lse = torch.empty(w.n_scored, device="cuda")
        libdpo.seq_logprobs(b, True, seq, None, lse, ws)
        dH = torch.empty(w.R, w.L, w.d, device="cuda")
        dW = torch.empty(w.V, w.d, device="cuda")
        ws.fill_(fill)
        libdpo.backward(b, lse, coef, dH, dW, False, ws)
        assert libdpo.check() == libdpo.OK
        outs.append((seq, lse, dH, dW))
    for o in outs[1:]:
        for a, c in zip(outs[0], o):
            assert torch.equal(a, c)
