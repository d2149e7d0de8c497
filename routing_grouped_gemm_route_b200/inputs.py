"""Seeded synthetic inputs for the routed MoE layer workloads.

This module only draws random numbers and names workload shapes; it holds none of
the layer's arithmetic, so both the CUDA path and the CPU oracle may use it.

The shapes follow the workloads of the Olmo-core 3 write-ups ("Ai2'nin raporladığı
sayılar" on the deniz.in page: an expert pool grown from 8 to 128 experts with four
experts per token at a fixed active size; "Três números, três denominadores" on the
bigchange.ai page: headline rows measured under random routing, and an MXFP8 row).
The pages print no layer sizes; d_model, d_ff and T are the workload definitions
this library is measured on:

==================  =====  ====  ===  ==  ====  =======  =========================
name                T      d     E    k   d_ff  storage  routing logits
==================  =====  ====  ===  ==  ====  =======  =========================
tiny_fp32           512    128   8    2   256   fp32     x . Wr, Wr ~ N(0, 0.02)
e8_bf16             8192   2048  8    4   1024  bf16     iid N(0, 1) fp32
e128_bf16           16384  2048  128  4   1024  bf16     iid N(0, 1) fp32
e128_skew_bf16      16384  2048  128  4   1024  bf16     N(0,1) + Zipf(1.2) bias
e128_mxfp8_large    32768  4096  128  8   1536  bf16 IO  iid N(0, 1) fp32
==================  =====  ====  ===  ==  ====  =======  =========================

Values are never constant: the pages report that kernel time depends on the input
values, not only on shapes ("दस्तावेज़ीकृत निष्कर्ष" on the unite.ai page), so every
tensor is drawn from N(0, 1) (activations, upstream gradients, logits) or
N(0, 0.02) (weights).
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    d_ff: int
    dtype: str          # "fp32", "bf16" or "mxfp8" (grouped-GEMM operand precision)
    router: bool        # True: logits = x . Wr on the device; False: logits are injected
    skew: bool          # Zipf-skewed expert bias added to the injected logits
    seed: int = 0
    shared: bool = False  # one shared expert (an extra W13/W2 slice, applied to every token)

    @property
    def R(self) -> int:
        """Routed rows T*k."""
        return self.T * self.k

    @property
    def storage(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 512, 128, 8, 2, 256, "fp32", router=True, skew=False),
    "e8_bf16": Workload("e8_bf16", 8192, 2048, 8, 4, 1024, "bf16", router=False, skew=False),
    "e128_bf16": Workload("e128_bf16", 16384, 2048, 128, 4, 1024, "bf16", router=False, skew=False),
    "e128_skew_bf16": Workload("e128_skew_bf16", 16384, 2048, 128, 4, 1024, "bf16",
                               router=False, skew=True),
    "e128_mxfp8_large": Workload("e128_mxfp8_large", 32768, 4096, 128, 8, 1536, "mxfp8",
                                 router=False, skew=False),
}


def zipf_bias(E: int, generator: torch.Generator, s: float = 1.2, scale: float = 1.5) -> torch.Tensor:
    """Per-expert logit bias b_e = scale*log(1/rank_e**s) over a seeded permutation of ranks 1..E.

    Computed in fp64, returned as fp32 (the precision of the logits it is added to).
    """
    ranks = torch.randperm(E, generator=generator, device="cpu").to(torch.float64) + 1.0
    b = scale * (-s * torch.log(ranks))
    return b.to(torch.float32)


def make_inputs(w: Workload, device: str | torch.device = "cpu", seed: int | None = None) -> dict:
    """Draw one seeded batch of layer inputs for workload ``w`` on ``device``.

    Returns a dict of tensors: x [T,d], W13 [E,2*d_ff,d] (rows 0..d_ff-1 gate W1, then up W3),
    W2 [E,d,d_ff], dy [T,d] (upstream gradient), and either Wr [d,E] (router on) or
    logits [T,E] fp32 (injected random routing).  Activations and weights are in the
    workload's storage dtype; logits are always fp32.  With a shared expert W13 and W2
    have E+1 slices, the last drawn after everything else (so the rest is unchanged).
    """
    device = torch.device(device)
    s = w.seed if seed is None else seed
    g = torch.Generator(device=device)
    g.manual_seed(s)
    st = w.storage

    def normal(shape, std=1.0):
        t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t.to(st)

    out = {}
    out["x"] = normal((w.T, w.d))
    out["W13"] = normal((w.E, 2 * w.d_ff, w.d), 0.02)
    out["W2"] = normal((w.E, w.d, w.d_ff), 0.02)
    if w.router:
        out["Wr"] = normal((w.d, w.E), 0.02)
        out["logits"] = None
    else:
        out["Wr"] = None
        logits = torch.randn(w.T, w.E, generator=g, device=device, dtype=torch.float32)
        if w.skew:
            gb = torch.Generator(device="cpu")
            gb.manual_seed(s + 7919)
            logits += zipf_bias(w.E, gb).to(device)
        out["logits"] = logits
    out["dy"] = normal((w.T, w.d))
    if w.shared:
        out["W13"] = torch.cat([out["W13"], normal((1, 2 * w.d_ff, w.d), 0.02)])
        out["W2"] = torch.cat([out["W2"], normal((1, w.d, w.d_ff), 0.02)])
    return out


def random_logits(T: int, E: int, seed: int, device="cpu", skew: bool = False) -> torch.Tensor:
    """iid N(0,1) fp32 routing logits (plus the Zipf bias when ``skew``)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    L = torch.randn(T, E, generator=g, device=device, dtype=torch.float32)
    if skew:
        gb = torch.Generator(device="cpu")
        gb.manual_seed(seed + 7919)
        L += zipf_bias(E, gb).to(device)
    return L


def normal_tensor(shape, seed: int, std: float = 1.0, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """Seeded N(0, std) tensor cast to ``dtype``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


__all__ = ["Workload", "WORKLOADS", "make_inputs", "zipf_bias", "random_logits", "normal_tensor"]
