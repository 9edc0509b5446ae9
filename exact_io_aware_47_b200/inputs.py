"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and casts them; it holds none of the
attention arithmetic.  Both the CUDA path's tests and the CPU oracle's tests
take their inputs from here.

Recipe (one generator per workload, ``torch.Generator(device).manual_seed(seed)``;
large workloads are drawn on the GPU, where torch's counter-based generator is
fast, small ones on the CPU; the two devices give different draws, and a test
always hands both the kernel and the oracle the same tensors):

1. ragged workload only: valid key lengths ``seqlens[b]`` drawn uniformly
   from {1, ..., N} (``torch.randint``);
2. Q, K, V, then dO, each an iid N(0, 1) float32 draw of shape [B, H, N, d];
3. ragged workload only: K row j multiplied by (1 + 3 j / N) in float32, so
   that the running row max keeps growing across K tiles;
4. each tensor cast round-to-nearest-even to the workload's 16-bit dtype.

Packed variable-length inputs (``make_inputs_varlen``): sequence lengths
drawn uniformly from {1, ..., max_len} (``torch.randint``) unless given,
``cu_seqlens`` their running sum from 0, then Q, K, V, dO each an iid N(0, 1)
float32 draw of shape [H, T, d] (T = total length), cast as in step 4.

The pages name no dataset or benchmark suite; these shapes stand in for the
workloads they discuss (n = 8192 fp16 sizing, 32k context, short training
shapes, padded batches).
"""

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_inputs_shape", "PackedWorkload",
           "PACKED_WORKLOADS", "make_inputs_varlen", "make_inputs_packed", "window_block_mask",
           "BLOCKSPARSE_WORKLOADS"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtypes: tuple            # 16-bit dtypes the kernels run in
    ragged: bool = False     # key-padding with drawn valid lengths
    draw_dtype: str = "f32"  # inputs drawn in float32, then cast
    description: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 64, False, (torch.bfloat16, torch.float16),
                     description="B1 H1 N128 d64, fp32 draws cast to bf16 and fp16, non-causal"),
    "small": Workload("small", 4, 16, 1024, 64, True, (torch.bfloat16,),
                      description="B4 H16 N1024 d64 bf16 causal (short training shape)"),
    "mid": Workload("mid", 2, 32, 8192, 128, True, (torch.bfloat16, torch.float16),
                    description="B2 H32 N8192 d128 causal, bf16 and fp16"),
    "long": Workload("long", 1, 32, 32768, 128, True, (torch.bfloat16,),
                     description="B1 H32 N32768 d128 bf16 causal (no NxN buffer)"),
    "ragged": Workload("ragged", 8, 16, 4099, 128, False, (torch.bfloat16,), ragged=True,
                       description="B8 H16 N4099 d128 bf16, key padding with seqlens ~ U{1..N}, "
                                   "K row j scaled by (1 + 3j/N)"),
}


def make_inputs_shape(B, H, N, d, dtype, seed=0, ragged=False, with_do=True,
                      seqlens=None, device="cpu"):
    """Draw q, k, v (and dO) of shape [B, H, N, d] on ``device``.

    Returns a dict with 16-bit tensors ``q, k, v, do`` and ``seqlens``
    (int32 [B] or None).  ``ragged`` draws seqlens and grows K along the
    sequence as in the module docstring; an explicit ``seqlens`` sequence
    overrides the drawn one.
    """
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    sl = None
    if ragged:
        sl = torch.randint(1, N + 1, (B,), generator=g, dtype=torch.int64,
                           device=device).to(torch.int32)
    if seqlens is not None:
        sl = torch.as_tensor(seqlens, dtype=torch.int32).to(device)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    k = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    v = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    do = torch.randn(shape, generator=g, dtype=torch.float32, device=device) if with_do else None
    if ragged:
        grow = 1.0 + 3.0 * torch.arange(N, dtype=torch.float32, device=device) / N
        k = k * grow[None, None, :, None]
    out = {"q": q.to(dtype), "k": k.to(dtype), "v": v.to(dtype),
           "do": do.to(dtype) if do is not None else None, "seqlens": sl}
    return out


def make_inputs(name, dtype=None, seed=0, with_do=True, device="cpu"):
    """Inputs of a named workload (``WORKLOADS``) in ``dtype`` (default: its first)."""
    w = WORKLOADS[name]
    dt = dtype if dtype is not None else w.dtypes[0]
    return make_inputs_shape(w.B, w.H, w.N, w.d, dt, seed=seed, ragged=w.ragged,
                             with_do=with_do, device=device)


@dataclass(frozen=True)
class PackedWorkload:
    name: str
    B: int          # sequences
    H: int
    max_len: int    # lengths ~ U{1, ..., max_len}
    d: int
    causal: bool
    dtype: torch.dtype
    description: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


PACKED_WORKLOADS = {
    "varlen": PackedWorkload("varlen", 8, 16, 4099, 128, False, torch.bfloat16,
                             description="8 packed sequences, lengths ~ U{1..4099}, H16 d128 bf16, "
                                         "non-causal (the padded batch without its padding)"),
}


def make_inputs_varlen(B, H, max_len, d, dtype, seed=0, lengths=None, with_do=True,
                       device="cpu"):
    """Draw a packed batch: q, k, v (and dO) [H, T, d], ``cu_seqlens`` int32
    [B + 1] and the host list ``lengths``; ``max_seqlen`` is max(lengths, 1)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    if lengths is None:
        ln = torch.randint(1, max_len + 1, (B,), generator=g, dtype=torch.int64, device=device)
        lengths = [int(x) for x in ln.cpu()]
    lengths = [int(x) for x in lengths]
    if len(lengths) != B or min(lengths) < 0:
        raise ValueError("lengths must be B non-negative integers")
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    T = cu[-1]
    shape = (H, T, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    k = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    v = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    do = torch.randn(shape, generator=g, dtype=torch.float32, device=device) if with_do else None
    return {"q": q.to(dtype), "k": k.to(dtype), "v": v.to(dtype),
            "do": do.to(dtype) if do is not None else None,
            "cu_seqlens": torch.tensor(cu, dtype=torch.int32, device=device),
            "lengths": lengths, "max_seqlen": max(max(lengths), 1)}


def make_inputs_packed(name, seed=0, with_do=True, device="cpu"):
    """Inputs of a named packed workload (``PACKED_WORKLOADS``)."""
    w = PACKED_WORKLOADS[name]
    return make_inputs_varlen(w.B, w.H, w.max_len, w.d, w.dtype, seed=seed, with_do=with_do,
                              device=device)


def window_block_mask(n_tiles, window, n_global=0):
    """Boolean [n_tiles, n_tiles] tile mask: query tile i sees key tiles
    i - window + 1 .. i (a sliding window) and the first ``n_global`` key
    tiles."""
    i = torch.arange(n_tiles)[:, None]
    j = torch.arange(n_tiles)[None, :]
    return ((i - j >= 0) & (i - j < window)) | (j < n_global)


# Block-sparse workloads: a dense workload's inputs plus a tile mask.
BLOCKSPARSE_WORKLOADS = {
    "sparse": dict(kind="sparse", base="mid", window=8, n_global=1,
                   description="B2 H32 N8192 d128 bf16 causal, 8-tile (1024-key) sliding window "
                               "plus the first key tile, 128 x 128 tiles"),
    # dropout on the probabilities (the mask is regenerated from seed and
    # position inside both kernels)
    "dropout": dict(kind="dropout", base="mid", p_drop=0.1, seed=0x5EED,
                    description="B2 H32 N8192 d128 bf16 causal with dropout p = 0.1 on the "
                                "probabilities"),
}

# 8-bit inputs: the dense workload's bf16 draws, quantised to e4m3 with one
# descale per 128-row tile by the library itself (forward only)
E4M3_WORKLOADS = {
    "fp8": dict(base="mid",
                description="B2 H32 N8192 d128 causal, bf16 draws quantised to e4m3 with one "
                            "descale per 128-row tile, forward only"),
}
