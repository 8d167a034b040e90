"""The backward in phases (dpo_backward with dW = NULL, then dpo_backward_dw by
blocks of vocabulary rows and dpo_backward_dh), the data-parallel caller's route:
bit-identical to the one-call backward whatever the blocks and the SM budget, and
within tolerance of the oracle."""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import dp as DP
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, TOL_GRAD, np64, rel_frob

pytestmark = pytest.mark.gpu

CASES = [
    # R, L, d, V, dtype, prompt range, seed
    (6, 300, 256, 1000, "bf16", (1, 200), 81),        # ragged vocabulary tail
    (4, 600, 512, 70000, "bf16", (1, 300), 82),       # dH in vocabulary chunks
    (4, 40, 64, 300, "f32", (1, 20), 83),             # fp32 route
]


@pytest.mark.parametrize("R,L,d,V,dtype,pr,seed", CASES)
def test_phased_backward_equals_one_call(R, L, d, V, dtype, pr, seed):
    import torch
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype=dtype, seed=seed, prompt_range=pr, full_rows=1)
    dw = DeviceWorkload(w)
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.from_numpy(np.random.default_rng(seed).normal(0, 0.05, w.R).astype(np.float32)).cuda()
    dH1, dW1 = dw.backward(lse, coef)
    b = dw.batch()
    _, bwd, _ = libdpo.workspace_size(b)
    ws = dw.workspace(bwd)
    for n_buckets, max_sms in ((1, 0), (3, 40), (8, 132)):
        dH2 = torch.full_like(dH1, float("nan"))
        dW2 = torch.full_like(dW1, float("nan"))
        libdpo.backward(b, lse, coef, None, None, False, ws)
        for v0, v1 in DP.vocab_buckets(w.V, n_buckets, align=8):
            libdpo.backward_dw(b, v0, v1, dW2, False, ws, max_sms=max_sms)
        libdpo.backward_dh(b, dH2, ws, max_sms=max_sms)
        assert libdpo.check() == libdpo.OK
        assert torch.equal(dW2, dW1)
        assert torch.equal(dH2, dH1)
    # accumulation over a block: dW += the same rows again gives twice the rows
    libdpo.backward(b, lse, coef, None, None, False, ws)
    libdpo.backward_dw(b, 0, min(w.V, 256), dW2, True, ws)
    assert libdpo.check() == libdpo.OK
    r = min(w.V, 256)
    assert torch.allclose(dW2[:r], 2 * dW1[:r], rtol=1e-6, atol=1e-12)
    assert torch.equal(dW2[r:], dW1[r:])
    # and the values against the oracle
    Hd = WL.widen(w.H, w.dtype)
    oH, oW = O.backward(Hd, WL.widen(w.W, w.dtype), w.tokens, w.prompt_len, w.completion_len,
                        coef.double().cpu().numpy())
    assert rel_frob(np64(dH1), oH) <= TOL_GRAD
    assert rel_frob(np64(dW1), oW) <= TOL_GRAD


def test_backward_exchange_on_one_rank_equals_one_call():
    """dp.backward_exchange on a single-rank gloo group (gloo reduces CUDA tensors
    through host staging; the all-reduce of one rank is the identity): the same bits
    as the one-call backward."""
    import socket
    import torch
    import torch.distributed as dist
    w = WL.make_custom(R=4, L=400, d=256, V=3000, dtype="bf16", seed=84, prompt_range=(1, 200),
                       full_rows=1)
    dw = DeviceWorkload(w)
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.from_numpy(np.random.default_rng(84).normal(0, 0.05, w.R).astype(np.float32)).cuda()
    dH1, dW1 = dw.backward(lse, coef)
    b = dw.batch()
    _, bwd, _ = libdpo.workspace_size(b)
    ws = dw.workspace(bwd)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        dW2 = torch.full_like(dW1, float("nan"))
        dH2 = torch.full_like(dH1, float("nan"))
        works = DP.backward_exchange(b, lse, coef, dH2, dW2, ws, n_buckets=4, max_sms=100)
        DP.finish(works)
        torch.cuda.synchronize()
        assert libdpo.check() == libdpo.OK
        assert torch.equal(dW2, dW1)
        assert torch.equal(dH2, dH1)
    finally:
        dist.destroy_process_group()
