"""Offline reference scoring on the GPU: the weight fingerprint, and scores stored
once, reloaded under checked metadata and used in the loss."""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import artifact as A
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, TOL_LOSS, np64

pytestmark = pytest.mark.gpu

M64 = (1 << 64) - 1


def _mix(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def fingerprint_reference(buf: bytes) -> int:
    """The same hash, written independently with Python integers."""
    n = len(buf)
    padded = buf + b"\0" * ((-n) % 16)
    s = 0
    for i in range(len(padded) // 16):
        lo = int.from_bytes(padded[16 * i:16 * i + 8], "little")
        hi = int.from_bytes(padded[16 * i + 8:16 * i + 16], "little")
        s = (s + _mix((_mix(lo ^ _mix(2 * i + 1)) + hi + 0x9E3779B97F4A7C15 * (i + 1)) & M64)) & M64
    return _mix(s ^ n)


def _gpu_fp(t, nbytes):
    import torch
    out = torch.zeros(1, dtype=torch.int64, device="cuda")
    libdpo.fingerprint(t, nbytes, out)
    return int(out.item()) & M64


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 4096 + 7, 300001])
def test_fingerprint_matches_an_independent_evaluation(n):
    import torch
    rng = np.random.default_rng(n)
    data = rng.integers(0, 256, size=max(n, 1), dtype=np.uint8)[:n]
    t = torch.zeros(max(n, 16), dtype=torch.uint8, device="cuda")
    t[:n] = torch.from_numpy(data).cuda()
    assert _gpu_fp(t, n) == fingerprint_reference(data.tobytes())


def test_fingerprint_is_stable_and_sensitive():
    import torch
    w = torch.randn(4096, 1024, device="cuda").to(torch.bfloat16)
    nb = w.numel() * 2
    a, b = _gpu_fp(w, nb), _gpu_fp(w, nb)
    assert a == b
    w2 = w.clone()
    w2.view(-1)[123457] += 1.0
    assert _gpu_fp(w2, nb) != a


def test_offline_scores_roundtrip_into_the_loss(tmp_path):
    import torch
    w = WL.make_custom(R=8, L=200, d=128, V=900, dtype="bf16", seed=81, prompt_range=(1, 60),
                       ref_std=0.05)
    dw = DeviceWorkload(w)
    # scoring run: reference sums without grad state, stored with the weights' fingerprint
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    fp = _gpu_fp(dw.W_ref, w.V * w.d * 2)
    meta = A.metadata(w.d, w.V, w.L, "bf16", fp, libdpo.version(), dataset="synthetic-81")
    A.save(str(tmp_path), np64(ref), w.layout, meta)
    # training run: the expected metadata is rebuilt from the weights it holds
    expect = A.metadata(w.d, w.V, w.L, "bf16", _gpu_fp(dw.W_ref, w.V * w.d * 2), libdpo.version(),
                        dataset="synthetic-81")
    ref_loaded = torch.from_numpy(A.load(str(tmp_path), expect, layout=w.layout).astype(np.float32)).cuda()
    pol, _, _ = dw.forward(dw.W, want_grad=False)
    out = dw.loss(pol, ref_loaded)
    H = WL.widen(w.H, "bf16")
    op = O.seq_logprobs(H, WL.widen(w.W, "bf16"), w.tokens, w.prompt_len, w.completion_len)
    orf = O.seq_logprobs(H, WL.widen(w.W_ref, "bf16"), w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, w.layout)
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS
    # other weights: the fingerprint differs and the artifact is refused
    expect_other = dict(expect, weights_fingerprint=f"{_gpu_fp(dw.W, w.V * w.d * 2):016x}")
    with pytest.raises(A.ArtifactMismatch):
        A.load(str(tmp_path), expect_other, layout=w.layout)
