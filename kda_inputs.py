"""Seeded synthetic inputs for the KDA recurrence, shared by the tests, the smoke check and the
benchmark.

This module only draws random numbers in the shapes, dtypes and distributions of the workloads;
it holds none of the recurrence's arithmetic and imports neither the library nor the oracle.

Common recipe (every workload): q, k ~ N(0, 1) L2-normalised per (token, head) over d_k in fp32,
then rounded to bf16; v ~ N(0, 1) bf16; decay logits a bf16; beta fp32 [T, H]; gate logits
~ N(0, 1) bf16; A_log fp32 [H]; states fp32.  Tensors are drawn on the requested device from a
generator seeded with the workload's seed, in a fixed order, token block by token block, so the
same seed and device always give the same bits.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

_BLOCK_TOKENS = 1 << 16  # draw large tensors in token blocks to bound temporary memory


@dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple
    H: int
    d_k: int
    d_v: int
    a_mean: float = 0.0
    a_std: float = 1.0
    A_log: str = "zero"            # "zero" | "uniform"   (U(-1, 1) per head)
    beta: str = "sigmoid_normal"   # "sigmoid_normal" | "uniform_0.9_1"
    init_state: str = "none"       # "none" (zeros, passed as NULL) | "normal_0.02"
    gate: bool = True
    final_state: bool = True
    seed: int = 0
    note: str = ""

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def varlen_lengths(n: int = 64, lo: int = 512, hi: int = 32768, seed: int = 0) -> tuple:
    """Sequence lengths ~ U{lo..hi}, drawn on the CPU so they do not depend on the device."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


# The five workloads of the benchmark family (named by what they are, with their sizes).
PR1_REF = Workload("pr1_ref_B1_H2_T256_d64", (256,), 2, 64, 64, A_log="zero",
                   init_state="none", note="B=1 H=2 T=256 d=64, chunk 64 / tile 16, seed 0")
PREFILL_8K = Workload("prefill_B1_H32_T8192_d128", (8192,), 32, 128, 128, A_log="uniform",
                      init_state="normal_0.02",
                      note="B=1 H=32 T=8192 d=128, A_h~U(-1,1), S0~N(0,0.02)")
SATURATED = Workload("saturated_B2_H32_T16384_d128", (16384, 16384), 32, 128, 128, a_mean=8.0,
                     beta="uniform_0.9_1", note="a~N(8,1): g ~ -5 in every channel")
NOFADE = SATURATED.replace(name="nofade_B2_H32_T16384_d128", a_mean=-8.0, seed=1,
                           note="a~N(-8,1): g ~ 0 (no fade)")
VARLEN = Workload("varlen_64seq_U512_32768_H64_d128", varlen_lengths(), 64, 128, 128,
                  init_state="normal_0.02", note="64 sequences, lengths ~U{512..32768}")
LONG_1M = Workload("long_B1_H32_T1048576_d128", (1 << 20,), 32, 128, 128,
                   note="B=1 H=32 T=1,048,576 d=128, zero initial state")

WORKLOADS = {w.name: w for w in (PR1_REF, PREFILL_8K, SATURATED, NOFADE, VARLEN, LONG_1M)}


@dataclass(frozen=True)
class DecodeWorkload:
    name: str = "decode_N256_H64_d128_512steps"
    N: int = 256
    H: int = 64
    d_k: int = 128
    d_v: int = 128
    steps: int = 512
    seed: int = 0


DECODE = DecodeWorkload()


@dataclasses.dataclass(frozen=True)
class SpecWorkload:
    """Speculative decode: K proposed tokens per sequence per round, then an accepted prefix.

    The shapes are the decode configuration's (256 sequences x 64 heads, 128 x 128 states); K = 4
    proposals per round, and each sequence accepts a prefix of length ~ U{0..K} (the pages give no
    acceptance rate; uniform is the plainest stand-in)."""
    name: str = "spec_N256_H64_d128_K4"
    N: int = 256
    H: int = 64
    d_k: int = 128
    d_v: int = 128
    K: int = 4
    rounds: int = 64
    seed: int = 0


SPEC = SpecWorkload()


def _gen(device, seed):
    return torch.Generator(device=torch.device(device)).manual_seed(int(seed))


def _unit_rows(T, H, d, gen, device):
    out = torch.empty((T, H, d), dtype=torch.bfloat16, device=device)
    for s in range(0, T, _BLOCK_TOKENS):
        e = min(T, s + _BLOCK_TOKENS)
        x = torch.randn((e - s, H, d), generator=gen, device=device, dtype=torch.float32)
        x = x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)
        out[s:e] = x.to(torch.bfloat16)
    return out


def _normal_rows(T, H, d, gen, device, mean=0.0, std=1.0):
    out = torch.empty((T, H, d), dtype=torch.bfloat16, device=device)
    for s in range(0, T, _BLOCK_TOKENS):
        e = min(T, s + _BLOCK_TOKENS)
        x = torch.randn((e - s, H, d), generator=gen, device=device, dtype=torch.float32)
        out[s:e] = (x * std + mean).to(torch.bfloat16)
    return out


def _beta(T, H, kind, gen, device):
    if kind == "sigmoid_normal":
        return torch.sigmoid(torch.randn((T, H), generator=gen, device=device))
    if kind == "uniform_0.9_1":
        return 0.9 + 0.1 * torch.rand((T, H), generator=gen, device=device)
    raise ValueError(kind)


def make_inputs(w: Workload, device="cpu") -> dict:
    """Draw every input of workload ``w`` on ``device``.

    Returns q, k, a [T, H, d_k] bf16; v, gate [T, H, d_v] bf16 (gate None if disabled);
    beta [T, H] fp32; A_log [H] fp32; cu_seqlens [N+1] int32; initial_state fp32
    [N, H, d_k, d_v] or None; plus the workload itself under "workload".
    """
    g = _gen(device, w.seed)
    T, H = w.total_tokens, w.H
    q = _unit_rows(T, H, w.d_k, g, device)
    k = _unit_rows(T, H, w.d_k, g, device)
    v = _normal_rows(T, H, w.d_v, g, device)
    a = _normal_rows(T, H, w.d_k, g, device, mean=w.a_mean, std=w.a_std)
    beta = _beta(T, H, w.beta, g, device)
    gate = _normal_rows(T, H, w.d_v, g, device) if w.gate else None
    if w.A_log == "uniform":
        A_log = torch.rand((H,), generator=g, device=device) * 2.0 - 1.0
    else:
        A_log = torch.zeros((H,), device=device)
    S0 = None
    if w.init_state == "normal_0.02":
        S0 = torch.randn((w.num_seqs, H, w.d_k, w.d_v), generator=g, device=device) * 0.02
    cu = [0]
    for L in w.seqlens:
        cu.append(cu[-1] + int(L))
    cu_seqlens = torch.tensor(cu, dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, a=a, beta=beta, gate=gate, A_log=A_log, cu_seqlens=cu_seqlens,
                initial_state=S0, workload=w)


def make_decode_inputs(w: DecodeWorkload, device="cpu", steps: int | None = None) -> dict:
    """Per-step decode inputs [steps, N, H, d] and the starting states [N, H, d_k, d_v].

    Inputs follow the common recipe with a ~ N(0, 1), A_h = 0 and beta = sigmoid(N(0, 1));
    states ~ N(0, 0.02).
    """
    steps = w.steps if steps is None else steps
    g = _gen(device, w.seed)
    N, H = w.N, w.H
    state = torch.randn((N, H, w.d_k, w.d_v), generator=g, device=device) * 0.02
    q = _unit_rows(steps * N, H, w.d_k, g, device).view(steps, N, H, w.d_k)
    k = _unit_rows(steps * N, H, w.d_k, g, device).view(steps, N, H, w.d_k)
    v = _normal_rows(steps * N, H, w.d_v, g, device).view(steps, N, H, w.d_v)
    a = _normal_rows(steps * N, H, w.d_k, g, device).view(steps, N, H, w.d_k)
    beta = _beta(steps * N, H, "sigmoid_normal", g, device).view(steps, N, H)
    gate = _normal_rows(steps * N, H, w.d_v, g, device).view(steps, N, H, w.d_v)
    A_log = torch.zeros((H,), device=device)
    return dict(q=q, k=k, v=v, a=a, beta=beta, gate=gate, A_log=A_log, state=state, workload=w)


def make_spec_inputs(w: SpecWorkload, device="cpu", rounds: int | None = None) -> dict:
    """Per-round inputs [rounds, N, K, H, d], accepted counts [rounds, N] (int32, U{0..K}) and the
    starting states [N, H, d_k, d_v]; inputs follow the decode recipe."""
    rounds = w.rounds if rounds is None else rounds
    g = _gen(device, w.seed)
    N, H, K = w.N, w.H, w.K
    rows = rounds * N * K
    state = torch.randn((N, H, w.d_k, w.d_v), generator=g, device=device) * 0.02
    q = _unit_rows(rows, H, w.d_k, g, device).view(rounds, N, K, H, w.d_k)
    k = _unit_rows(rows, H, w.d_k, g, device).view(rounds, N, K, H, w.d_k)
    v = _normal_rows(rows, H, w.d_v, g, device).view(rounds, N, K, H, w.d_v)
    a = _normal_rows(rows, H, w.d_k, g, device).view(rounds, N, K, H, w.d_k)
    beta = _beta(rows, H, "sigmoid_normal", g, device).view(rounds, N, K, H)
    gate = _normal_rows(rows, H, w.d_v, g, device).view(rounds, N, K, H, w.d_v)
    accepted = torch.randint(0, K + 1, (rounds, N), generator=g, device=device, dtype=torch.int32)
    A_log = torch.zeros((H,), device=device)
    return dict(q=q, k=k, v=v, a=a, beta=beta, gate=gate, A_log=A_log, state=state, accepted=accepted,
                workload=w)
