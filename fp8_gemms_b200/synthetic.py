"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no scaling, casting or GEMM).  Both sides receive the same
bf16 bits from here.

Recipe:
  * every tensor has its own CPU ``torch.Generator`` seeded with
    ``seed * 1009 + index`` (index = position of the tensor in its workload),
    so any one tensor can be regenerated without drawing the others;
  * the same recipe can draw on a CUDA device instead (``device=``), with a
    CUDA generator seeded the same way: same distributions and seeds, other
    values.  The benchmark uses it for workloads too large to draw on the host
    in reasonable time (the 28-layer stack); the parity tests use host draws;
  * values are drawn in fp32 and rounded to bf16 (round to nearest even);
  * "N(0, s)" means standard deviation s; "t3" means a standard Student-t with
    3 degrees of freedom, Z / sqrt(chi2_3 / 3), not rescaled.

The shapes are those of the little-lm 3.8B model (decomputer.nl, "Het trainen
van een 3.8B LLM tot 0.384 CORE voor $998", "Appendix: De configuratie":
hidden_size 3072, intermediate_size 12288, 24 query / 8 KV heads of 128,
vocab 50,257 padded to 50,304).  Weights follow the N(0, 0.02) linear init
named in section "Wat niet werkte" (Nanochat-stijl initialisatie bullet);
activations N(0, 1) or t3; incoming gradients N(0, 1e-3).  They stand in for
the real run's activations, which depend on its data and trained weights.
"""
from dataclasses import dataclass, field

import torch

D_MODEL = 3072
D_FF = 12288
N_LAYERS = 28
N_Q_HEADS, N_KV_HEADS, HEAD_DIM = 24, 8, 128
VOCAB, VOCAB_PADDED = 50257, 50304


def _gen(seed: int, index: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1009 + index)
    return g


def normal_bf16(shape, std: float, seed: int, index: int, device="cpu") -> torch.Tensor:
    x = torch.randn(*shape, generator=_gen(seed, index, device), dtype=torch.float32,
                    device=device)
    return (x * std).to(torch.bfloat16)


def student_t3_bf16(shape, seed: int, index: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, index, device)
    z = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    c = torch.randn(3, *shape, generator=g, dtype=torch.float32, device=device).square().sum(0)
    return (z / torch.sqrt(c / 3.0)).to(torch.bfloat16)


def draw(spec, seed: int, index: int, device="cpu") -> torch.Tensor:
    shape, dist = spec
    kind, param = dist
    if kind == "normal":
        return normal_bf16(shape, param, seed, index, device)
    if kind == "t3":
        return student_t3_bf16(shape, seed, index, device)
    raise ValueError(kind)


@dataclass
class MlpWorkload:
    """relu^2 MLP block: X [M x d], W_up [f x d], W_down [d x f], dY [M x d]."""
    name: str
    M: int
    d: int
    f: int
    backward: bool
    x_dist: tuple = ("normal", 1.0)
    seed: int = 0

    def tensors(self, device="cpu"):
        x = draw(((self.M, self.d), self.x_dist), self.seed, 0, device)
        wu = draw(((self.f, self.d), ("normal", 0.02)), self.seed, 1, device)
        wd = draw(((self.d, self.f), ("normal", 0.02)), self.seed, 2, device)
        out = dict(X=x, W_up=wu, W_down=wd)
        if self.backward:
            out["dY"] = draw(((self.M, self.d), ("normal", 1e-3)), self.seed, 3, device)
        return out

    @property
    def flops(self) -> int:
        n = 6 if self.backward else 2
        return n * 2 * self.M * self.d * self.f


@dataclass
class LinearWorkload:
    """A set of plain linears Y = X W^T run fwd + dgrad + wgrad."""
    name: str
    M: int
    linears: list = field(default_factory=list)  # (name, out_features, in_features)
    x_dist: tuple = ("normal", 1.0)
    seed: int = 0

    def tensors(self, i: int, device="cpu"):
        lname, n_out, n_in = self.linears[i]
        base = 4 * i
        return dict(
            name=lname,
            X=draw(((self.M, n_in), self.x_dist), self.seed, base + 0, device),
            W=draw(((n_out, n_in), ("normal", 0.02)), self.seed, base + 1, device),
            dY=draw(((self.M, n_out), ("normal", 1e-3)), self.seed, base + 2, device),
        )

    @property
    def flops(self) -> int:
        return sum(3 * 2 * self.M * o * k for _, o, k in self.linears)


ATTN_LINEARS = [
    ("q", N_Q_HEADS * HEAD_DIM, D_MODEL),
    ("k", N_KV_HEADS * HEAD_DIM, D_MODEL),
    ("v", N_KV_HEADS * HEAD_DIM, D_MODEL),
    ("o", D_MODEL, N_Q_HEADS * HEAD_DIM),
]

TINY_MLP = MlpWorkload("tiny relu2 MLP fwd+bwd M=256 d=256 f=1024", 256, 256, 1024, True)
MLP_FWD = MlpWorkload("relu2 MLP fwd M=16384 d=3072 f=12288", 16384, D_MODEL, D_FF, False)
MLP_FWD_BWD = MlpWorkload("relu2 MLP fwd+dgrad+wgrad M=16384 d=3072 f=12288", 16384,
                          D_MODEL, D_FF, True)
ATTN_HEAD = LinearWorkload("attention projections + LM head fwd+dgrad+wgrad M=8192", 8192,
                           ATTN_LINEARS + [("lm_head", VOCAB_PADDED, D_MODEL)])


def stack_layer(layer: int, M: int = 16384):
    """Layer `layer` of the 28-layer stack: attention linears + relu^2 MLP,
    t3 activations, each layer with its own seeds."""
    seed = 1000 + layer
    return (LinearWorkload(f"stack layer {layer} attention linears", M, ATTN_LINEARS,
                           ("t3", None), seed),
            MlpWorkload(f"stack layer {layer} relu2 MLP", M, D_MODEL, D_FF, True,
                        ("t3", None), seed))


def bits_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bits (a view, no arithmetic)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
