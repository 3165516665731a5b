"""Seeded synthetic inputs for the gated delta rule.

This module only draws random numbers and lays them out; it holds none of the method's arithmetic.
Both the CUDA path's callers and the CPU oracle's callers read the tensors it returns, so the two
sides always see the same rounded values.

Recipe (the workloads of the chunked-prefill and decode benchmarks of this library):

* q, k ~ N(0, 1), then L2-normalised per (token, head) in fp32 (norm clamped at 1e-12), then rounded
  to the storage dtype (fp32 or bf16).  The gated delta rule expects normalised q and k.
* v ~ N(0, 1), rounded to the storage dtype.
* beta = sigmoid(N(0, 1)) in fp32.
* g (log of the gate alpha = exp(g)), fp32, one of
  - ``"uniform"``:  g ~ U[-0.5, 0)
  - ``"softplus"``: g = -softplus(N(0, 1)) * 0.1
* initial states (optional) ~ N(0, std^2) in fp32, layout ``[N, H, dv, dk]``.

All draws come from one ``torch.Generator`` seeded with ``seed`` on the target device, in the order
q, k, v, g, beta, state.  Tensors are created directly on ``device``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_prefill_inputs", "make_decode_inputs", "make_verify_inputs",
           "cu_seqlens_of"]


@dataclass(frozen=True)
class Workload:
    name: str
    lengths: List[int] = field(default_factory=list)
    H: int = 32
    dk: int = 128
    dv: int = 128
    dtype: str = "bf16"
    gate: str = "softplus"
    state_std: Optional[float] = None
    seed: int = 0
    decode_batch: int = 0
    decode_steps: int = 0

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))


# The five benchmark workloads of the method (chunked prefill with C = 32, and the decode step).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", [128], H=2, dk=64, dv=64, dtype="fp32", gate="uniform"),
    "prefill_4k": Workload("prefill_4k", [4096]),
    "varlen_resume": Workload("varlen_resume", [8192, 3000, 517, 13000], state_std=0.05),
    "long_128k": Workload("long_128k", [131072]),
    "decode_b64": Workload("decode_b64", [], dtype="bf16", gate="uniform", state_std=0.05,
                           decode_batch=64, decode_steps=1000),
    # speculative verify: 4 drafted tokens for each of 64 sequences, the decode_b64 distributions
    "verify_b64_k4": Workload("verify_b64_k4", [], dtype="bf16", gate="uniform", state_std=0.05,
                              decode_batch=64, decode_steps=4),
    # tree verify: 8 drafted tokens per sequence in the best-first tree of best_first_parents(8)
    "verify_tree_b64_k8": Workload("verify_tree_b64_k8", [], dtype="bf16", gate="uniform", state_std=0.05,
                                   decode_batch=64, decode_steps=8),
}


def best_first_parents(Tk):
    """Parent of each of Tk drafted tokens in a best-first draft tree: a main chain through the first
    half of the tokens, the rest branching off main-chain tokens (token t under main token
    (7 t) mod (Tk / 2)), and the last token a second child of the committed state (-1) when Tk > 2.
    Every parent precedes its child."""
    main = max(1, Tk // 2)
    row = []
    for t in range(Tk):
        if t == 0 or (t == Tk - 1 and Tk > 2):
            row.append(-1)
        elif t < main:
            row.append(t - 1)
        else:
            row.append((7 * t) % main)
    return row


def _torch_dtype(name: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def cu_seqlens_of(lengths, device="cpu") -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _gate(gen, shape, gate, device):
    if gate == "uniform":
        return -0.5 * torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    if gate == "softplus":
        z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        return -torch.nn.functional.softplus(z) * 0.1
    if gate == "zero":
        return torch.zeros(shape, device=device, dtype=torch.float32)
    raise ValueError(gate)


def make_prefill_inputs(lengths, H, dk, dv, dtype="bf16", gate="softplus", seed=0,
                        state_std=None, device="cpu"):
    """Inputs of one packed prefill call.  Returns a dict of tensors on ``device``:
    q, k ``[T, H, dk]``; v ``[T, H, dv]`` (storage dtype); g, beta ``[T, H]`` fp32;
    cu_seqlens int32 ``[N + 1]``; state_in ``[N, H, dv, dk]`` fp32 or None."""
    T = int(sum(lengths))
    N = len(lengths)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    dt = _torch_dtype(dtype)
    q = _l2n(torch.randn((T, H, dk), generator=gen, device=device)).to(dt)
    k = _l2n(torch.randn((T, H, dk), generator=gen, device=device)).to(dt)
    v = torch.randn((T, H, dv), generator=gen, device=device).to(dt)
    g = _gate(gen, (T, H), gate, device)
    beta = torch.sigmoid(torch.randn((T, H), generator=gen, device=device))
    state = None
    if state_std is not None:
        state = torch.randn((N, H, dv, dk), generator=gen, device=device) * float(state_std)
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu_seqlens_of(lengths, device),
                state_in=state)


def make_decode_inputs(B, H, dk, dv, steps, dtype="bf16", gate="uniform", seed=0, state_std=0.05,
                       device="cpu"):
    """Inputs of a chain of ``steps`` decode steps over ``B`` sequences.

    Returns q, k ``[steps, B, H, dk]``, v ``[steps, B, H, dv]``, g, beta ``[steps, B, H]`` and the
    initial state ``[B, H, dv, dk]``.  Step ``s`` draws fresh inputs (one generator, drawn in step
    order), so the chain is not a repetition of one token."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    dt = _torch_dtype(dtype)
    state = torch.randn((B, H, dv, dk), generator=gen, device=device) * float(state_std)
    q = _l2n(torch.randn((steps, B, H, dk), generator=gen, device=device)).to(dt)
    k = _l2n(torch.randn((steps, B, H, dk), generator=gen, device=device)).to(dt)
    v = torch.randn((steps, B, H, dv), generator=gen, device=device).to(dt)
    g = _gate(gen, (steps, B, H), gate, device)
    beta = torch.sigmoid(torch.randn((steps, B, H), generator=gen, device=device))
    return dict(q=q, k=k, v=v, g=g, beta=beta, state=state)


def make_verify_inputs(B, H, dk, dv, Tk, dtype="bf16", gate="uniform", seed=0, state_std=0.05, device="cpu"):
    """Inputs of one multi-token verify: ``Tk`` drafted tokens for each of ``B`` sequences, laid out
    ``[B, Tk, H, d]`` / ``[B, Tk, H]``, drawn as ``make_decode_inputs`` draws a chain of Tk steps."""
    d = make_decode_inputs(B, H, dk, dv, Tk, dtype=dtype, gate=gate, seed=seed, state_std=state_std, device=device)
    out = {n: d[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}
    out["state"] = d["state"]
    return out


def workload_inputs(name: str, device="cpu", seed=None):
    """Prefill inputs of one named workload (see ``WORKLOADS``)."""
    w = WORKLOADS[name]
    return make_prefill_inputs(w.lengths, w.H, w.dk, w.dv, w.dtype, w.gate,
                               w.seed if seed is None else seed, w.state_std, device)
