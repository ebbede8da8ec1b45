"""Seeded synthetic inputs for the fused MoE layer forward.

This module draws the inputs of a layer and nothing else: token activations
``x``, router weights ``Wg``, the routing-skew bias ``log p``, and the expert
weights.  It holds none of the layer's arithmetic, so both the CUDA path and
the CPU oracle can take their inputs from it.

Recipe (Decoding the Skew, abstract: routing distributions are produced by
Dirichlet-based reverse modelling; the shapes follow the five layer
configurations named by the workload table of the same study):

* every weight is an fp32 draw from N(0, 1/d) (N(0, 1/f) for the down
  projection W2 and Ws2), rounded to bf16 with round-to-nearest-even;
* ``Wg`` ~ N(0, 1/d);
* ``x`` ~ N(0, 1/d) for the tiny layer (as its description states) and
  N(0, 1) elsewhere;
* one routing distribution ``p ~ Dirichlet(alpha * 1_E)`` per (layer, alpha,
  seed), shared by every token; the bias handed to the router is ``log p``
  (fp32).  ``p`` is drawn in log space (Gamma(alpha) as Gamma(alpha+1) times
  U^(1/alpha), Marsaglia and Tsang 2000), so tiny alpha never yields log 0.

Each tensor has its own generator, seeded from (seed, tensor name), so a
tensor does not depend on which other tensors were drawn before it.  On CPU
the draws use torch's CPU generator; on CUDA they use torch's CUDA generator
(different values, same distribution), which lets the multi-gigabyte layers be
drawn on the device in seconds.
"""

from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Dict, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape and routing skew of one MoE layer forward."""

    name: str
    T: int            # tokens
    d: int            # model dim
    f: int            # per-expert FFN dim
    E: int            # routed experts
    k: int            # experts per token
    alpha: float      # Dirichlet concentration of the routing distribution
    f_shared: int = 0 # FFN dim of the always-on shared expert (0 = none)
    x_std: Optional[float] = None  # None -> 1.0

    @property
    def P(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)


# The five layer families of the workload table, at their default T / alpha.
TINY = LayerShape("tiny", T=64, d=256, f=512, E=8, k=2, alpha=1.0, x_std=1.0 / math.sqrt(256))
DECODE64 = LayerShape("decode64", T=32, d=2048, f=1024, E=64, k=8, alpha=1.0)
MIXTRAL = LayerShape("mixtral", T=256, d=4096, f=14336, E=8, k=2, alpha=1.0)
DEEPSEEK_V3 = LayerShape("deepseek_v3", T=1024, d=7168, f=2048, E=256, k=8, alpha=0.5, f_shared=2048)
KIMI_K2 = LayerShape("kimi_k2", T=256, d=7168, f=2048, E=384, k=8, alpha=0.02)

FAMILIES = {s.name: s for s in (TINY, DECODE64, MIXTRAL, DEEPSEEK_V3, KIMI_K2)}

# The sweep points each family is specified at.
SWEEP = {
    "tiny": [dict(T=64, alpha=1.0)],
    "decode64": [dict(T=32, alpha=a) for a in (0.1, 1.0, 10.0)],
    "mixtral": [dict(T=t, alpha=1.0) for t in (1, 16, 256, 4096)],
    "deepseek_v3": [dict(T=t, alpha=a) for t in (64, 1024, 16384) for a in (0.05, 0.5, 5.0)],
    "kimi_k2": [dict(T=t, alpha=0.02) for t in (8, 256, 8192)],
}


def shape(name: str, **kw) -> LayerShape:
    return FAMILIES[name].with_(**kw)


def _seed_for(seed: int, tag: str) -> int:
    return (int(seed) * 0x9E3779B1 + zlib.crc32(tag.encode())) & 0x7FFF_FFFF_FFFF


def _normal_bf16(shape_, std: float, seed: int, tag: str, device) -> torch.Tensor:
    """fp32 N(0, std^2) draws rounded to bf16 (RNE), drawn in slabs to bound memory."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(_seed_for(seed, tag))
    out = torch.empty(shape_, dtype=torch.bfloat16, device=dev)
    flat = out.view(-1) if out.numel() else out
    slab = 1 << 26
    n = flat.numel()
    for s in range(0, n, slab):
        e = min(n, s + slab)
        tmp = torch.randn(e - s, generator=gen, dtype=torch.float32, device=dev)
        tmp.mul_(std)
        flat[s:e].copy_(tmp)  # fp32 -> bf16 copy rounds to nearest even
    return out


def dirichlet_log_p(E: int, alpha: float, seed: int) -> np.ndarray:
    """log p for p ~ Dirichlet(alpha * 1_E), drawn in log space (float64)."""
    rng = np.random.default_rng([int(seed), zlib.crc32(b"dirichlet")])
    g = rng.standard_gamma(alpha + 1.0, size=E)        # Gamma(alpha + 1) > 0
    u = 1.0 - rng.random(E)                            # U in (0, 1]
    log_x = np.log(g) + np.log(u) / alpha              # log Gamma(alpha)
    m = log_x.max()
    return log_x - (m + np.log(np.exp(log_x - m).sum()))


def make_inputs(s: LayerShape, seed: int = 0, device="cpu",
                weights: bool = True) -> Dict[str, torch.Tensor]:
    """Draw every input of layer ``s``; bf16 tensors in nn.Linear (K-major) storage.

    x [T,d], Wg [E,d], bias [E] fp32 (= log p), W1/W3 [E,f,d], W2 [E,d,f],
    and, when ``s.f_shared`` > 0, Ws1/Ws3 [f_shared,d] and Ws2 [d,f_shared].
    """
    x_std = 1.0 if s.x_std is None else s.x_std
    inp: Dict[str, torch.Tensor] = {}
    inp["x"] = _normal_bf16((s.T, s.d), x_std, seed, "x", device)
    inp["Wg"] = _normal_bf16((s.E, s.d), 1.0 / math.sqrt(s.d), seed, "Wg", device)
    log_p = dirichlet_log_p(s.E, s.alpha, seed)
    inp["bias"] = torch.from_numpy(log_p.astype(np.float32)).to(device)
    if weights:
        inp.update(make_weights(s, seed, device))
    return inp


def make_weights(s: LayerShape, seed: int = 0, device="cpu") -> Dict[str, torch.Tensor]:
    w: Dict[str, torch.Tensor] = {}
    w["W1"] = _normal_bf16((s.E, s.f, s.d), 1.0 / math.sqrt(s.d), seed, "W1", device)
    w["W3"] = _normal_bf16((s.E, s.f, s.d), 1.0 / math.sqrt(s.d), seed, "W3", device)
    w["W2"] = _normal_bf16((s.E, s.d, s.f), 1.0 / math.sqrt(s.f), seed, "W2", device)
    w.update(make_shared_weights(s, seed, device))
    return w


def make_expert_weights(s: LayerShape, seed: int, e: int, device="cpu") -> Dict[str, torch.Tensor]:
    """One routed expert's W1[e] [f,d], W3[e] [f,d], W2[e] [d,f], each drawn from a
    generator of its own (seeded from (seed, name, e)): the same distribution as
    ``make_weights``, different values.  Lets a host-side sample of a very large
    layer draw only the experts its tokens use."""
    return {
        "W1": _normal_bf16((s.f, s.d), 1.0 / math.sqrt(s.d), seed, f"W1/{e}", device),
        "W3": _normal_bf16((s.f, s.d), 1.0 / math.sqrt(s.d), seed, f"W3/{e}", device),
        "W2": _normal_bf16((s.d, s.f), 1.0 / math.sqrt(s.f), seed, f"W2/{e}", device),
    }


def make_shared_weights(s: LayerShape, seed: int = 0, device="cpu") -> Dict[str, torch.Tensor]:
    """The shared expert's Ws1/Ws3 [f_shared,d] and Ws2 [d,f_shared] (as ``make_weights`` draws them)."""
    fs = s.f_shared
    if not fs:
        return {}
    return {
        "Ws1": _normal_bf16((fs, s.d), 1.0 / math.sqrt(s.d), seed, "Ws1", device),
        "Ws3": _normal_bf16((fs, s.d), 1.0 / math.sqrt(s.d), seed, "Ws3", device),
        "Ws2": _normal_bf16((s.d, fs), 1.0 / math.sqrt(fs), seed, "Ws2", device),
    }


def random_logits(T: int, E: int, seed: int, ties: bool = False, device="cpu") -> torch.Tensor:
    """fp32 router logits for top-k tests; ``ties`` quantises them so equal values are common."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(_seed_for(seed, "logits"))
    L = torch.randn(T, E, generator=gen, dtype=torch.float32, device=device)
    if ties:
        L = torch.round(L * 2.0) / 2.0
    return L


def random_routing(T: int, E: int, k: int, alpha: float, seed: int) -> torch.Tensor:
    """topk_idx [T,k] int32 with k distinct experts per token drawn under a Dirichlet skew."""
    rng = np.random.default_rng([int(seed), zlib.crc32(b"routing")])
    log_p = dirichlet_log_p(E, alpha, seed)
    # Gumbel top-k draws k distinct experts per token with probabilities ~ p.
    u = rng.random((T, E)) * (1.0 - 2e-16) + 1e-16   # U in (0, 1)
    gumbel = -np.log(-np.log(u))
    keys = log_p[None, :] + gumbel
    idx = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    return torch.from_numpy(idx.astype(np.int32))


def random_gates(T: int, k: int, seed: int) -> torch.Tensor:
    """Positive fp32 gate weights [T,k] summing to 1 per token."""
    rng = np.random.default_rng([int(seed), zlib.crc32(b"gates")])
    w = rng.random((T, k)) + 0.05
    w = w / w.sum(axis=1, keepdims=True)
    return torch.from_numpy(w.astype(np.float32))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """A bf16 tensor's raw bit patterns as a host uint16 numpy array (no copy for CPU tensors)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
