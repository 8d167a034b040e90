"""Shared test harness: runs the CUDA path through the C ABI on seeded workloads.

Only marshalling lives here (device copies of the generator's arrays, buffers,
calls through preference_alignment_b200.libdpo). Expected values come from the
oracle, never from this module.
"""
from __future__ import annotations

import numpy as np

from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL


def torch_mod():
    import torch
    return torch


def to_device(arr, dtype, dev="cuda"):
    torch = torch_mod()
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(dev)


class DeviceWorkload:
    """Device copies of a workload and helpers to call every entry point."""

    def __init__(self, w: WL.Workload, dev="cuda"):
        torch = torch_mod()
        self.w = w
        self.H = to_device(w.H, w.dtype, dev)
        self.W = to_device(w.W, w.dtype, dev)
        self.W_ref = to_device(w.W_ref, w.dtype, dev) if w.W_ref is not None else None
        self.tokens = torch.from_numpy(np.ascontiguousarray(w.tokens, np.int32)).to(dev)
        self.dev = dev

    def batch(self, W=None, prompt_len=None, completion_len=None, tokens=None):
        w = self.w
        return libdpo.BatchArgs(self.H, self.W if W is None else W,
                                self.tokens if tokens is None else tokens,
                                w.prompt_len if prompt_len is None else prompt_len,
                                w.completion_len if completion_len is None else completion_len,
                                dtype=w.dtype)

    def workspace(self, nbytes):
        torch = torch_mod()
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=self.dev)

    def forward(self, W=None, want_grad=True, with_tok=True, batch=None):
        torch = torch_mod()
        b = batch if batch is not None else self.batch(W)
        fwd, _, _ = libdpo.workspace_size(b)
        ws = self.workspace(fwd)
        R, L = self.w.R, self.w.L
        seq = torch.full((R,), float("nan"), device=self.dev)
        tok = torch.full((R, L), float("nan"), device=self.dev) if with_tok else None
        lse = torch.full((max(b.n_scored, 1),), float("nan"), device=self.dev) if want_grad else None
        libdpo.seq_logprobs(b, want_grad, seq, tok, lse, ws)
        return seq, tok, lse

    def loss(self, pol, ref, beta=None, grad_scale=1.0, layout=None):
        torch = torch_mod()
        B = self.w.R // 2
        out = {k: torch.full((n,), float("nan"), device=self.dev) for k, n in
               [("loss", 1), ("accuracy", 1), ("margins", B), ("chosen_rewards", B),
                ("rejected_rewards", B), ("weights", B), ("row_coef", 2 * B)]}
        libdpo.loss(B, layout or self.w.layout, pol, ref, self.w.beta if beta is None else beta,
                    grad_scale, out["loss"], out["accuracy"], out["margins"], out["chosen_rewards"],
                    out["rejected_rewards"], out["weights"], out["row_coef"])
        return out

    def backward(self, lse, row_coef, W=None, ws_bytes=None, accumulate=False, dW=None, want_dH=True,
                 batch=None):
        torch = torch_mod()
        b = batch if batch is not None else self.batch(W)
        _, bwd, _ = libdpo.workspace_size(b)
        ws = self.workspace(bwd if ws_bytes is None else ws_bytes)
        w = self.w
        dH = torch.full((w.R, w.L, w.d), float("nan"), device=self.dev) if want_dH else None
        if dW is None:
            dW = torch.full((w.V, w.d), float("nan"), device=self.dev)
        libdpo.backward(b, lse, row_coef, dH, dW, accumulate, ws, ws_bytes=ws.numel())
        return dH, dW


def np64(t):
    return t.detach().double().cpu().numpy()


def rel_frob(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# Tolerances of the path (per-token log-prob, sequence sums, loss, gradients).
TOL_TOK = 2e-3
TOL_SEQ_ABS = 5e-2
TOL_SEQ_REL = 1e-4
TOL_LOSS = 1e-4
TOL_GRAD = 1e-2


def assert_seq_close(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    assert np.all(err <= TOL_SEQ_ABS), f"seq abs err {err.max()}"
    assert np.all(err <= TOL_SEQ_REL * np.maximum(np.abs(ref), 1.0)), \
        f"seq rel err {(err / np.maximum(np.abs(ref), 1.0)).max()}"
