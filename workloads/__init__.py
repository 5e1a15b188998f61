"""Seeded synthetic inputs for the CSA lightning-indexer top-k step.

This module only draws random numbers and stores them in the input formats
(bfloat16, fp32, E4M3 bytes with a per-key fp32 scale).  It holds none of the
indexer's arithmetic; both the CUDA path's tests and the CPU oracle consume
what it returns.

Shapes follow "StreamIndex: Memory-Bounded Compressed Sparse Attention via
Streaming Top-k", abstract (H_I = 64 indexer heads, compression m = 4,
V4-Flash-shaped synthetic inputs, S up to 262,144), and the decode setting of
the Multi-layer Indexer blog post (2048 selected entries per query, long
context).  Value distributions:

* ``integer``: q, k uniform on {-4..4}/4 (exact in bf16), w uniform on
  {+-1/4, +-1/2, +-1} -- every product and partial sum of the score is exact
  in fp32, so a correct GPU result equals the oracle bit for bit;
* ``normal``: q, k ~ N(0, 1) rounded to bf16 (round-to-nearest-even),
  w ~ N(0, 1/H_I) in fp32;
* FP8 keys: k ~ N(0, 1) in fp32, per-key scale = max_j |k[s, j]| / 448,
  bytes = E4M3(k / scale) with round-to-nearest-even (torch's
  ``float8_e4m3fn`` cast).  The effective key is scale * E4M3 value.  With
  integer values the bytes encode 4*k (integers in [-4, 4], exact in E4M3)
  and every scale is 1/4, so the effective keys equal the integer recipe's.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    T: int
    H: int
    d: int
    m: int
    topk: int
    causal: bool = True
    key_fp8: bool = False
    gated: bool = False
    values: str = "normal"  # "normal" | "integer"
    q_pieces: int = 0       # E4M3 keys: query pieces on the tensor core (0/2 exact split, 1 one rounding)
    num_splits: int = 0     # key-range splits per query block (0 = the library's choice)
    seed: int = 0
    note: str = ""

    @property
    def q_offset(self) -> int:
        """Absolute position of query row 0 (bottom-right alignment)."""
        return max(0, self.T * self.m - self.S)

    def visible(self, i: int) -> int:
        """Number of keys query row i may see (the causal rule, closed form)."""
        if not self.causal:
            return self.T
        t = i + self.q_offset
        return max(0, min(self.T, (t + 1) // self.m))

    def visible_pairs(self) -> int:
        """Sum over all queries of the visible key count."""
        if not self.causal:
            return self.B * self.S * self.T
        total = 0
        # closed form over the clipped ramp, evaluated piecewise
        for i in range(self.S):
            total += self.visible(i)
        return total * self.B

    def flops(self) -> int:
        """Algorithmic tensor flops: visible pairs x 2 x H_I x d."""
        return self.visible_pairs() * 2 * self.H * self.d

    def input_bytes(self) -> int:
        kb = self.B * self.T * self.d * (1 if self.key_fp8 else 2)
        ks = self.B * self.T * 4 if self.key_fp8 else 0
        return self.B * self.S * self.H * self.d * 2 + self.B * self.S * self.H * 4 + kb + ks

    def output_bytes(self) -> int:
        return self.B * self.S * self.topk * 8

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Workload("tiny", B=1, S=1024, T=256, H=4, d=32, m=4, topk=16,
                     values="integer", seed=101,
                     note="integer-valued, bit-exact check"),
    "dsa_prefill": Workload("dsa_prefill", B=1, S=8192, T=8192, H=64, d=128, m=1,
                            topk=2048, seed=102, note="DSA-style uncompressed prefill"),
    "v4flash_prefill": Workload("v4flash_prefill", B=1, S=65536, T=16384, H=64, d=128,
                                m=4, topk=2048, seed=103,
                                note="V4-Flash-shaped prefill"),
    "long_prefill_fp8": Workload("long_prefill_fp8", B=1, S=262144, T=65536, H=64,
                                 d=128, m=4, topk=2048, key_fp8=True, seed=104,
                                 note="long prefill, FP8 keys"),
    "long_prefill_fp8_gated": Workload("long_prefill_fp8_gated", B=1, S=262144, T=65536,
                                       H=64, d=128, m=4, topk=2048, key_fp8=True,
                                       gated=True, seed=104,
                                       note="long prefill, FP8 keys, sigmoid gate"),
    "decode_fp8": Workload("decode_fp8", B=32, S=64, T=131072, H=64, d=128, m=4,
                           topk=2048, key_fp8=True, seed=105,
                           note="batched decode window of 64 queries at context 524288"),
    "decode1_fp8": Workload("decode1_fp8", B=32, S=1, T=131072, H=64, d=128, m=4,
                            topk=2048, key_fp8=True, seed=106,
                            note="one query per sequence at context 524288 (HBM-bound)"),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _integer_quarters(shape, g, device):
    return torch.randint(-4, 5, shape, generator=g, device=device).to(torch.float32) / 4.0


def _weights_pow2(shape, g, device):
    mag = torch.tensor([0.25, 0.5, 1.0], device=device)
    pick = torch.randint(0, 3, shape, generator=g, device=device)
    sign = torch.randint(0, 2, shape, generator=g, device=device).to(torch.float32) * 2 - 1
    return mag[pick] * sign


def quantize_e4m3(k32: torch.Tensor):
    """Per-key E4M3 storage of fp32 keys: returns (bytes uint8 [...,d], scale fp32 [...])."""
    amax = k32.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    k8 = (k32 / scale.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return k8.view(torch.uint8), scale.to(torch.float32)


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None, chunk_rows: int = 1 << 22):
    """Draw the inputs of workload ``wl`` on ``device`` (CPU or CUDA generator).

    Draw order: q, k, w.  Large tensors are drawn in row chunks so that the
    fp32 staging buffer stays small; the chunking is part of the recipe (the
    same seed, device and chunk size give the same bytes).
    Returns a dict with ``q`` (bf16 [B,S,H,d]), ``w`` (fp32 [B,S,H]), ``k``
    (bf16 [B,T,d] or uint8 E4M3 bytes [B,T,d]) and ``k_scale`` (fp32 [B,T] or
    None).
    """
    seed = wl.seed if seed is None else seed
    g = _gen(device, seed)
    B, S, T, H, d = wl.B, wl.S, wl.T, wl.H, wl.d

    q = torch.empty((B * S * H, d), dtype=torch.bfloat16, device=device)
    for r0 in range(0, q.shape[0], chunk_rows):
        r1 = min(q.shape[0], r0 + chunk_rows)
        if wl.values == "integer":
            q[r0:r1] = _integer_quarters((r1 - r0, d), g, device).to(torch.bfloat16)
        else:
            q[r0:r1] = torch.randn((r1 - r0, d), generator=g, device=device).to(torch.bfloat16)
    q = q.view(B, S, H, d)

    if wl.values == "integer":
        k32 = _integer_quarters((B, T, d), g, device)
    else:
        k32 = torch.randn((B, T, d), generator=g, device=device)
    if wl.key_fp8 and wl.values == "integer":
        # 4*k is an integer in [-4, 4]: exact in E4M3, scale 1/4 exact in fp32
        k = (k32 * 4.0).to(torch.float8_e4m3fn).view(torch.uint8)
        k_scale = torch.full((B, T), 0.25, dtype=torch.float32, device=device)
    elif wl.key_fp8:
        k, k_scale = quantize_e4m3(k32)
    else:
        k, k_scale = k32.to(torch.bfloat16), None
    del k32

    if wl.values == "integer":
        w = _weights_pow2((B, S, H), g, device)
    else:
        w = torch.randn((B, S, H), generator=g, device=device) * (1.0 / H) ** 0.5
    return {"q": q.contiguous(), "w": w.contiguous(), "k": k.contiguous(),
            "k_scale": None if k_scale is None else k_scale.contiguous()}


def as_numpy_bits(inputs):
    """The inputs as the raw numpy arrays the oracle reads (q/k as bit patterns)."""
    q = inputs["q"].detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
    w = inputs["w"].detach().cpu().contiguous().numpy()
    k = inputs["k"].detach().cpu().contiguous()
    if k.dtype == torch.bfloat16:
        k = k.view(torch.int16).numpy().view("uint16")
    else:
        k = k.numpy()
    ks = inputs["k_scale"]
    ks = None if ks is None else ks.detach().cpu().contiguous().numpy()
    return q, w, k, ks
