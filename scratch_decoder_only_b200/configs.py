"""The five workloads the library is built and measured on.

Sizes follow the pages: the tiny byte-level model uses RustGPT's sizes
("RustGPT", section "Technical implementation": embedding 128, hidden 256,
max sequence 80, 3 blocks, lr 5e-4, clip 5.0); the packed model is
LucilleAI's SFT class ("LucilleAI", "Real measured numbers": seq 512 with
packing); the 30M byte model is Smallem's ("Smallem", "Ce qu'est un modele
de langage": 257 byte tokens, a 30M-parameter network); GPT-2 small mirrors
Feste ("Feste", "Model Architecture mirrors GPT-2": 12 blocks, 768 = 12 x 64).
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict


@dataclass(frozen=True)
class ModelConfig:
    vocab: int
    vocab_padded: int
    d_model: int
    n_heads: int
    d_mlp: int
    n_layers: int
    max_seq: int
    max_batch: int
    tied: bool = False
    precision: str = "fp32"          # "fp32", "bf16" or "fp16"
    loss_scaling: bool = False       # dynamic loss scale
    init_loss_scale: float = 1.0
    ln_eps: float = 1e-5
    init_std: float = 0.02
    arch: str = "gpt2"               # "gpt2" or "llama" (RMSNorm, rotary positions, grouped K/V heads, SwiGLU)
    n_kv_heads: int = 0              # llama: key / value heads (0: n_heads)
    rope_base: float = 10000.0       # llama: rotary base

    @property
    def head_dim(self) -> int:
        return self.d_model // self.n_heads

    def num_params(self) -> int:
        C, F, Vp = self.d_model, self.d_mlp, self.vocab_padded
        if self.arch == "llama":
            kv = (self.n_kv_heads or self.n_heads) * self.head_dim
            per_layer = C * (C + 2 * kv) + C * C + 3 * F * C + 2 * C
            n = Vp * C + self.n_layers * per_layer + C
        else:
            per_layer = 4 * C * C + 2 * F * C + 9 * C + F
            n = Vp * C + self.max_seq * C + self.n_layers * per_layer + 2 * C
        if not self.tied:
            n += Vp * C
        return n

    def as_dict(self):
        return asdict(self)


@dataclass(frozen=True)
class AdamWConfig:
    lr: float
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01
    clip_norm: float = 1.0


@dataclass(frozen=True)
class Workload:
    name: str
    model: ModelConfig
    batch: int
    seq: int
    adamw: AdamWConfig
    data_seed: int
    init_seed: int = 42
    packed: bool = False
    steps: int = 1
    extra: dict = field(default_factory=dict)


TINY_BYTE = Workload(
    name="tiny-byte-v257-c128-l3-t80-b4-fp32",
    model=ModelConfig(vocab=257, vocab_padded=257, d_model=128, n_heads=8, d_mlp=256,
                      n_layers=3, max_seq=80, max_batch=4, precision="fp32"),
    batch=4, seq=80,
    adamw=AdamWConfig(lr=5e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, clip_norm=5.0),
    data_seed=101,
)

PACKED_SMALL = Workload(
    name="packed-v8000-c192-l4-t512-b8-bf16",
    model=ModelConfig(vocab=8000, vocab_padded=8000, d_model=192, n_heads=6, d_mlp=768,
                      n_layers=4, max_seq=512, max_batch=8, precision="bf16",
                      loss_scaling=True, init_loss_scale=2.0 ** 15),
    batch=8, seq=512,
    adamw=AdamWConfig(lr=1e-4, clip_norm=1.0),
    data_seed=102, packed=True,
)

BYTE_30M = Workload(
    name="byte30m-v257-c512-l8-t1024-b32-bf16",
    model=ModelConfig(vocab=257, vocab_padded=257, d_model=512, n_heads=8, d_mlp=2048,
                      n_layers=8, max_seq=1024, max_batch=32, precision="bf16"),
    batch=32, seq=1024,
    adamw=AdamWConfig(lr=3e-4, clip_norm=1.0),
    data_seed=103, steps=20,
)

GPT2_124M = Workload(
    name="gpt2-124m-v50257p50304-c768-l12-t1024-b16-bf16",
    model=ModelConfig(vocab=50257, vocab_padded=50304, d_model=768, n_heads=12, d_mlp=3072,
                      n_layers=12, max_seq=1024, max_batch=16, tied=True, precision="bf16"),
    batch=16, seq=1024,
    adamw=AdamWConfig(lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, clip_norm=1.0),
    data_seed=104, steps=50,
)

GPT2_DECODE = Workload(
    name="gpt2-124m-greedy-decode-prompt128-new384",
    model=ModelConfig(vocab=50257, vocab_padded=50304, d_model=768, n_heads=12, d_mlp=3072,
                      n_layers=12, max_seq=1024, max_batch=32, tied=True, precision="bf16"),
    batch=32, seq=512,
    adamw=AdamWConfig(lr=6e-4),
    data_seed=105, extra={"prompt_len": 128, "n_new": 384, "batches": (1, 32)},
)

WORKLOADS = {w.name: w for w in (TINY_BYTE, PACKED_SMALL, BYTE_30M, GPT2_124M, GPT2_DECODE)}
