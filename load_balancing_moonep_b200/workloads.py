"""Seeded synthetic inputs for the MoonEP hot path.

This module draws router outputs, hidden states and gradients.  It holds
none of the planning, permute or reduction arithmetic: both the CUDA library
and the CPU oracle consume what it produces, and it imports neither.

Routing recipe (the pages measure on a maxvio sweep and ship no data set;
"MoonEP article" below is "Moonshot AI Open-Sources MoonEP: A Perfectly
Balanced Expert Parallelism Library for MoE Training"):

* logits ``z[t, e] = N(0, 1) + alpha * b_e`` with a Zipf-rank bias
  ``b_e = -s * ln(rho(e))`` for a seeded permutation ``rho`` of ``1..E``
  (``rho`` = identity for the adversarial variant that puts all hot experts
  on rank 0);
* top-K: the K largest logits of each token, largest first -- this fixes the
  k order;
* combine weights: softmax over the K selected logits, in float64, rounded
  to float32;
* ``alpha`` is bisected until the realised ``maxvio = max_e T_e / T_bar - 1``
  (MoonEP article, "The problem MoonEP targets"; ``T_bar = S*K*R/E`` as in
  the article's explainer, maxvio tab) is within ``tol`` of the target;
* ``maxvio = 0`` is the constructed balanced routing: pair ``p = t*K + k``
  picks expert ``p mod E``;
* the ``hot`` kind (decode shape) adds ``delta`` to one seeded expert
  instead of the Zipf bias and bisects ``delta``;
* hidden states, upstream gradients and expert outputs are N(0, 1) rounded
  to bf16 (round-to-nearest-even by torch); replica gradients are fp32
  N(0, 1e-3).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    R: int
    E: int
    K: int
    S: int
    H: int
    B: int
    kind: str = "zipf"          # "zipf" | "hot"
    zipf_s: float = 1.0
    maxvio: float = 1.0         # default target
    sweep: tuple = ()           # maxvio points measured by the benchmark
    H_ffn: int = 0              # expert FFN width H' (replica gradient shape)
    n_proj: int = 3             # gate, up, down

    @property
    def L(self) -> int:
        return self.E // self.R

    @property
    def C(self) -> int:
        return self.S * self.K

    @property
    def tokens(self) -> int:
        return self.R * self.S

    @property
    def pairs(self) -> int:
        return self.R * self.S * self.K

    @property
    def t_bar(self) -> float:
        return self.S * self.K * self.R / self.E

    @property
    def grad_elems(self) -> int:
        """Elements of one expert's weight gradient (gate + up + down)."""
        return self.n_proj * self.H * self.H_ffn

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # Tiny: the small case the oracle finishes in well under a second.
    "tiny": Workload("tiny", R=4, E=16, K=2, S=256, H=128, B=2, zipf_s=1.2, maxvio=1.0,
                     sweep=(0.0, 1.0)),
    "mid": Workload("mid", R=8, E=64, K=6, S=2048, H=2048, B=4, zipf_s=1.0, maxvio=1.0,
                    sweep=(0.0, 0.5, 1.0, 2.0, 3.0)),
    # Large training shape; the backward config shares its routing.
    "large": Workload("large", R=32, E=384, K=8, S=4096, H=7168, B=12, zipf_s=1.0, maxvio=1.0,
                      sweep=(0.0, 0.5, 1.0, 2.0, 3.0), H_ffn=2048),
    # The pages' own sweep: EP=8 at maxvio 0.2, 1, 10, 20 (expert count not
    # stated there; 256 experts, top-8 makes maxvio 20 reachable).
    "ep8": Workload("ep8", R=8, E=256, K=8, S=4096, H=7168, B=4, zipf_s=1.0, maxvio=1.0,
                    sweep=(0.2, 1.0, 10.0, 20.0)),
    # Decode: one hot expert, extreme skew, latency bound.
    "decode": Workload("decode", R=64, E=384, K=8, S=128, H=7168, B=4, kind="hot", maxvio=5.0,
                       sweep=(5.0, 10.0, 13.4, 20.0)),
}


def maxvio_of_counts(T, R: int, S: int, K: int, E: int) -> float:
    """maxvio = max_e T_e / T_bar - 1 with T_bar = S*K*R/E."""
    T = np.asarray(T, dtype=np.float64)
    t_bar = S * K * R / E
    return float(T.max() / t_bar - 1.0)


def hottest_expert_count(maxvio: float, S: int, K: int, R: int, E: int) -> int:
    """Tokens on the hottest expert at a given maxvio: round((1 + maxvio) * T_bar).
    (The MoonEP article's explainer tabulates this for maxvio 0.2, 1, 10, 20.)"""
    return int(round((1.0 + maxvio) * (S * K * R / E)))


def _counts(topk: torch.Tensor, E: int) -> np.ndarray:
    return torch.bincount(topk.reshape(-1).long(), minlength=E).cpu().numpy()


@dataclass
class Routing:
    topk_idx: torch.Tensor      # int32 [R*S, K]
    weights: torch.Tensor       # float32 [R*S, K]
    maxvio: float               # realised
    target: float
    knob: float                 # alpha (zipf) or delta (hot)


def _topk_weights(z: torch.Tensor, K: int):
    vals, idx = torch.topk(z, K, dim=1, largest=True, sorted=True)
    w = torch.softmax(vals.double(), dim=1).float()
    return idx.to(torch.int32).contiguous(), w.contiguous()


def balanced_routing(wl: Workload, seed: int = 0, device="cpu") -> Routing:
    """Pair p = t*K + k picks expert p mod E: every T_e is floor or ceil of T_bar."""
    R, S, K, E = wl.R, wl.S, wl.K, wl.E
    p = torch.arange(R * S * K, device=device, dtype=torch.int64)
    topk = (p % E).to(torch.int32).reshape(R * S, K).contiguous()
    g = torch.Generator(device=device).manual_seed(seed)
    z = torch.randn(R * S, K, generator=g, device=device, dtype=torch.float32)
    z, _ = torch.sort(z, dim=1, descending=True)
    w = torch.softmax(z.double(), dim=1).float().contiguous()
    mv = maxvio_of_counts(_counts(topk, E), R, S, K, E)
    return Routing(topk, w, mv, 0.0, 0.0)


def routing(wl: Workload, maxvio: float | None = None, seed: int = 0, device="cpu",
            adversarial: bool = False, tol: float = 0.02, max_iter: int = 48) -> Routing:
    """Top-K routing whose realised maxvio is within ``tol`` of ``maxvio``."""
    target = wl.maxvio if maxvio is None else float(maxvio)
    if target <= 0.0:
        return balanced_routing(wl, seed, device)
    R, S, K, E = wl.R, wl.S, wl.K, wl.E
    g = torch.Generator(device=device).manual_seed(seed)
    noise = torch.randn(R * S, E, generator=g, device=device, dtype=torch.float32)
    rng = np.random.default_rng(seed)
    if wl.kind == "hot":
        hot = int(rng.integers(E))
        bias = torch.zeros(E, device=device, dtype=torch.float32)
        bias[hot] = 1.0
    else:
        rho = np.arange(1, E + 1) if adversarial else rng.permutation(E) + 1
        bias = torch.tensor(-wl.zipf_s * np.log(rho), device=device, dtype=torch.float32)

    def at(knob: float):
        idx, w = _topk_weights(noise + knob * bias, K)
        return idx, w, maxvio_of_counts(_counts(idx, E), R, S, K, E)

    lo, hi = 0.0, 1.0
    idx, w, mv = at(hi)
    while mv < target and hi < 1e6:
        lo, hi = hi, hi * 2.0
        idx, w, mv = at(hi)
    best = (abs(mv - target), hi, idx, w, mv)
    for _ in range(max_iter):
        if best[0] <= tol:
            break
        mid = 0.5 * (lo + hi)
        idx, w, mv = at(mid)
        if abs(mv - target) < best[0]:
            best = (abs(mv - target), mid, idx, w, mv)
        if mv < target:
            lo = mid
        else:
            hi = mid
    _, knob, idx, w, mv = best
    return Routing(idx, w, mv, target, knob)


def bf16_normal(shape, seed: int, device="cpu", std: float = 1.0,
                chunk_elems: int = 1 << 28) -> torch.Tensor:
    """N(0, std^2) rounded to bf16, drawn in chunks to bound temporaries."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    g = torch.Generator(device=device).manual_seed(seed)
    for s in range(0, flat.numel(), chunk_elems):
        e = min(flat.numel(), s + chunk_elems)
        flat[s:e] = (torch.randn(e - s, generator=g, device=device) * std).to(torch.bfloat16)
    return out


def f32_normal(shape, seed: int, device="cpu", std: float = 1.0,
               chunk_elems: int = 1 << 28) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.float32, device=device)
    flat = out.view(-1)
    g = torch.Generator(device=device).manual_seed(seed)
    for s in range(0, flat.numel(), chunk_elems):
        e = min(flat.numel(), s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=g, device=device) * std
    return out


def over_budget_routing(wl: Workload, seed: int = 0, device="cpu") -> Routing:
    """One empty rank among R - 1 evenly overloaded ones: rank 0's experts get
    no tokens and every other rank's load is C * R / (R - 1) (rounded), so
    each of the R - 1 ranks sheds its excess to rank 0, which water-filling
    turns into R - 1 replicas on rank 0 (more than a budget B < R - 1).
    A rank's first expert carries the rank's rounding remainder; the others
    share the rest evenly.  Each token's K experts are distinct (pair slots
    are dealt expert-sorted with stride R*S, longer than any expert's run),
    and tokens are shuffled."""
    R, S, K, E, L = wl.R, wl.S, wl.K, wl.E, wl.L
    C = S * K
    T = np.zeros(E, np.int64)
    load = np.full(R - 1, (R * C) // (R - 1), np.int64)
    load[: (R * C) % (R - 1)] += 1
    for r in range(1, R):
        q = load[r - 1] // L
        T[r * L:(r + 1) * L] = q
        T[r * L] += load[r - 1] - q * L
    assert T.sum() == R * C and T.max() <= R * S
    ids = np.repeat(np.arange(E, dtype=np.int32), T)
    topk = ids.reshape(K, R * S).T.copy()
    rng = np.random.default_rng(seed)
    topk = topk[rng.permutation(R * S)]
    g = torch.Generator(device="cpu").manual_seed(seed)
    z, _ = torch.sort(torch.randn(R * S, K, generator=g), dim=1, descending=True)
    w = torch.softmax(z.double(), dim=1).float().contiguous()
    mv = maxvio_of_counts(T, R, S, K, E)
    return Routing(torch.from_numpy(np.ascontiguousarray(topk)).to(device), w.to(device), mv, mv, 0.0)


def hidden_states(wl: Workload, seed: int = 1, device="cpu") -> torch.Tensor:
    return bf16_normal((wl.tokens, wl.H), seed, device)


def bits(t: torch.Tensor) -> np.ndarray:
    """A bf16 tensor's bit patterns as a host uint16 array (no copy of values)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


__all__ = [
    "Workload", "WORKLOADS", "Routing", "routing", "balanced_routing", "over_budget_routing",
    "maxvio_of_counts",
    "hottest_expert_count", "bf16_normal", "f32_normal", "hidden_states", "bits", "from_bits",
]
