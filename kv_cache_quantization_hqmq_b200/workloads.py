"""Seeded synthetic KV-cache workloads.

This module only draws random numbers: it holds none of the HQMQ arithmetic,
and it is the one module that both the product-side tests/bench and the
oracle-side checks use, so that both see the same input bytes.

The shapes are those of the models the HQMQ pages evaluate or quote
(Llama-3-8B and -70B GQA caches, an outlier-heavy Qwen-class GQA cache, a
dense-MHA 7B cache).  No weights or datasets exist here, so the K/V values are
drawn from the distributions named per workload:

* ``normal``            i.i.d. N(0, 1)
* ``student_t3``        Student-t(3); a fixed fraction of channels per
                        (layer, head, role) multiplied by a constant
* ``lognormal_scale``   N(0, 1) times a per-(layer, head, role, channel)
                        scale drawn from LogNormal(0, 0.5)
* ``normal_channels``   N(0, 1); a fixed fraction of channels per
                        (layer, head, role) multiplied by a constant

Seeds: input values seed 0, codebook seed 1, outlier-channel choice seed 2;
each (layer, role) call draws from its own generator seeded from these.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

ROLE_K, ROLE_V = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    heads: int            # KV heads per layer
    head_dim: int
    batch: int
    tokens: int
    dtype: str            # "f32" or "bf16"
    S: int                # secondary codebook size
    med3: bool            # run the median-multiplier outlier step
    values: str
    C: float = 3.0
    channel_frac: float = 0.0
    channel_scale: float = 1.0
    input_seed: int = 0
    codebook_seed: int = 1
    channel_seed: int = 2
    q_heads: int = 0      # query heads per layer (GQA); 0 = heads (MHA)
    query_seed: int = 3
    note: str = field(default="", compare=False)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self):
        return 4 if self.dtype == "f32" else 2

    @property
    def call_shape(self):
        """[B, H, T, D] of one (layer, role) call."""
        return (self.batch, self.heads, self.tokens, self.head_dim)

    @property
    def call_elems(self):
        B, H, T, D = self.call_shape
        return B * H * T * D

    @property
    def n_calls(self):
        return self.layers * 2

    @property
    def cache_bytes(self):
        """Bytes of the whole K+V cache in its input dtype."""
        return self.n_calls * self.call_elems * self.elem_bytes

    @property
    def n_groups(self):
        """Codebook groups: one per (layer, role, head)."""
        return self.layers * 2 * self.heads

    @property
    def n_q_heads(self):
        return self.q_heads if self.q_heads > 0 else self.heads

    def n_outlier_channels(self):
        if self.channel_frac <= 0:
            return 0
        return max(1, int(round(self.channel_frac * self.head_dim)))

    def with_(self, **kw):
        d = {k: getattr(self, k) for k in self.__dataclass_fields__}
        d.update(kw)
        return Workload(**d)


def group0(layer: int, role: int, heads: int) -> int:
    """First codebook group of call (layer, role); group of head h is group0 + h."""
    return (layer * 2 + role) * heads


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 1, 256, "f32", 8, False, "normal",
                     note="1 layer x 1 KV head x 128, 256 tokens, fp32 N(0,1), S=8, no Med3x"),
    "llama3_8b": Workload("llama3_8b", 32, 8, 128, 1, 8192, "bf16", 8, False, "normal",
                          q_heads=32,
                          note="Llama-3-8B GQA cache, 8192 tokens, bf16 N(0,1), S=8"),
    "qwen_outlier": Workload("qwen_outlier", 28, 4, 128, 1, 32768, "bf16", 32, True, "student_t3",
                             channel_frac=0.02, channel_scale=50.0, q_heads=28,
                             note="Qwen-class GQA cache, 32768 tokens, bf16 t(3), 2% channels x50, "
                                  "Med3x C=3, S=32"),
    "mha7b_s8": Workload("mha7b_s8", 32, 32, 128, 8, 4096, "bf16", 8, True, "lognormal_scale",
                         note="dense-MHA 7B cache, batch 8 x 4096 tokens, LogNormal(0,0.5) channel "
                              "scales, Med3x, S=8"),
    "mha7b_s32": Workload("mha7b_s32", 32, 32, 128, 8, 4096, "bf16", 32, True, "lognormal_scale",
                          note="dense-MHA 7B cache, batch 8 x 4096 tokens, LogNormal(0,0.5) channel "
                               "scales, Med3x, S=32"),
    "llama3_70b_128k": Workload("llama3_70b_128k", 80, 8, 128, 1, 131072, "bf16", 32, True,
                                "normal_channels", channel_frac=0.01, channel_scale=30.0,
                                q_heads=64,
                                note="Llama-3-70B GQA cache, 131072 tokens (42.95 GB K+V bf16), "
                                     "1% channels x30, Med3x C=3, S=32, layer by layer"),
    # one layer (K and V) of the Llama-3-70B 128k cache: the same calls and
    # kernels at 537 MB, small enough for a full ncu capture
    "llama3_70b_128k_1layer": Workload("llama3_70b_128k_1layer", 1, 8, 128, 1, 131072, "bf16", 32,
                                       True, "normal_channels", channel_frac=0.01,
                                       channel_scale=30.0, q_heads=64,
                                       note="one layer of the Llama-3-70B 128k cache (profiling)"),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _call_seed(base: int, layer: int, role: int) -> int:
    return base * 1_000_003 + layer * 2 + role + 1


def make_call_input(w: Workload, layer: int, role: int, device="cpu",
                    tokens: int | None = None, batch: int | None = None) -> torch.Tensor:
    """The [B, H, T, D] K (role 0) or V (role 1) tensor of one layer, in the
    workload dtype, drawn on `device`.  `tokens`/`batch` override the sequence
    length / batch (same distribution, smaller tensor) for quick parity cases."""
    B = w.batch if batch is None else batch
    T = w.tokens if tokens is None else tokens
    H, D = w.heads, w.head_dim
    g = _gen(device, _call_seed(w.input_seed, layer, role))
    shape = (B, H, T, D)
    if w.values in ("normal", "normal_channels", "lognormal_scale"):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    elif w.values == "student_t3":
        z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        chi = torch.zeros(shape, device=device, dtype=torch.float32)
        for _ in range(3):
            e = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            chi.addcmul_(e, e)
        x = z / torch.sqrt(chi / 3.0)
        del chi
    else:
        raise ValueError(w.values)
    if w.values == "lognormal_scale":
        gs = _gen(device, _call_seed(w.channel_seed, layer, role))
        scale = torch.exp(0.5 * torch.randn((1, H, 1, D), generator=gs, device=device,
                                            dtype=torch.float32))
        x.mul_(scale)
    n_ch = w.n_outlier_channels()
    if n_ch:
        gc = torch.Generator(device="cpu")
        gc.manual_seed(_call_seed(w.channel_seed, layer, role))
        mult = torch.ones((1, H, 1, D), dtype=torch.float32)
        for h in range(H):
            ch = torch.randperm(D, generator=gc)[:n_ch]
            mult[0, h, 0, ch] = w.channel_scale
        x.mul_(mult.to(device))
    return x.to(w.torch_dtype).contiguous()


def make_query(w: Workload, layer: int, device="cpu", batch: int | None = None,
               step: int = 0) -> torch.Tensor:
    """The bf16 [B, Hq, D] query of one decode step of one layer: N(0, 1)
    (the pages give no query statistics; a trained model's queries are not
    available here)."""
    B = w.batch if batch is None else batch
    g = _gen(device, _call_seed(w.query_seed, layer, 0) + 7919 * step)
    q = torch.randn((B, w.n_q_heads, w.head_dim), generator=g, device=device,
                    dtype=torch.float32)
    return q.to(torch.bfloat16).contiguous()


def as_numpy_bits(x: torch.Tensor):
    """Host numpy view of a tensor: bf16 as uint16 bit patterns, fp32 as float32."""
    t = x.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)
