"""Seeded synthetic workloads shaped like the autoregressive-video KV caches.

Data model (the same for keys and values, each branch with its own draws):
    x_t = c_{z_t} + U g_t + noise * eps_t,  z_t ~ Uniform{0..C-1},
    c_j ~ N(0, I_J),  U a random J x rank orthonormal basis,
    g_t ~ N(0, I_rank),  eps_t ~ N(0, I_J),
optionally with a fraction of tokens multiplied by 8 (outliers).  Queries are
N(0, 1)/sqrt(d).  Stored values are rounded to the workload's storage dtype
(bf16, or fp32 for the tiny case) before anyone uses them, so every consumer
sees identical numbers.

Codec parameters stand in for fitted ones (fitting needs real video models):
the decoder D (J x r) has orthonormal columns, either random ("random") or
spanning the data's low-rank factor plus random extra columns ("span"); it is
rounded to the storage dtype and the encoder is exactly its transpose.

Only random draws happen here; nothing in this module assigns, projects,
quantises, decodes or attends.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    d: int
    T: int          # history tokens (time order, oldest first)
    T_full: int     # most recent history tokens routed to full-dim attention
    Tq: int         # query-chunk tokens (= current-chunk tokens)
    C: int          # centers per K/V codebook
    r: int          # joint rank
    rank: int       # rank of the data's low-rank factor
    seed: int
    fp32: bool = False
    decoder: str = "span"
    noise: float = 0.05
    outlier_frac: float = 0.0
    outlier_mult: float = 8.0
    layers: int = 1
    chunk: int = 4680

    @property
    def J(self) -> int:
        return self.H * self.d

    @property
    def T_low(self) -> int:
        return self.T - self.T_full

    @property
    def dtype(self) -> torch.dtype:
        return torch.float32 if self.fp32 else torch.bfloat16

    @property
    def scale_dtype(self) -> torch.dtype:
        return torch.float32 if self.fp32 else torch.float16

    def layer_seed(self, layer: int) -> int:
        return self.seed if self.layers == 1 else self.seed + layer

    def describe(self) -> str:
        mode = "full-dim" if self.T_low == 0 else "mixed-dim"
        return (f"{self.name}: {mode}, H={self.H} d={self.d} (J={self.J}), T={self.T} "
                f"(T_full={self.T_full}, T_low={self.T_low}), Tq={self.Tq}, C={self.C}, r={self.r}"
                + (f", x{self.layers} layers" if self.layers > 1 else ""))


WORKLOADS = {
    # tiny, fp32 throughout: full-dim decode-attention + current chunk merge
    "tiny": Workload("tiny", H=2, d=16, T=256, T_full=256, Tq=64, C=8, r=8, rank=6,
                     seed=0, fp32=True, decoder="random", chunk=64),
    # one layer, full-dim over 3 history chunks
    "full": Workload("full", H=12, d=128, T=14040, T_full=14040, Tq=4680, C=64, r=192,
                     rank=160, seed=1),
    # same shapes, most recent chunk full-dim, two older chunks low-dim
    "mixed": Workload("mixed", H=12, d=128, T=14040, T_full=4680, Tq=4680, C=64, r=192,
                      rank=160, seed=2),
    # long rollout: 20 chunks, last 2 full-dim, 1% x8 outlier tokens
    "long": Workload("long", H=24, d=128, T=93600, T_full=9360, Tq=4680, C=256, r=384,
                     rank=320, seed=3, outlier_frac=0.01),
    # 30-layer step: encode previous chunk, mixed attend (last chunk full), merge
    "step30": Workload("step30", H=12, d=128, T=46800, T_full=4680, Tq=4680, C=64, r=192,
                       rank=160, seed=4000, layers=30),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _round(x: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    """Round to the storage dtype (round-to-nearest-even, torch's cast)."""
    return x.to(dtype)


def make_codec(w: Workload, g: torch.Generator, device) -> dict:
    """Centers [C, J], decoder D [J, r], encoder E [r, J] (storage dtype) and the
    generator-private basis U [J, rank] (fp32)."""
    J, r, C, rank = w.J, w.r, w.C, w.rank
    centers = _round(torch.randn(C, J, generator=g, device=device), w.dtype)
    U = torch.linalg.qr(torch.randn(J, rank, generator=g, device=device, dtype=torch.float64))[0]
    if w.decoder == "random":
        basis = torch.randn(J, r, generator=g, device=device, dtype=torch.float64)
    else:
        assert r >= rank
        extra = torch.randn(J, r - rank, generator=g, device=device, dtype=torch.float64)
        basis = torch.cat([U, extra], dim=1)
    D = _round(torch.linalg.qr(basis)[0], w.dtype).contiguous()
    E = D.t().contiguous()
    return {"centers": centers.contiguous(), "D": D, "E": E, "U": U.to(torch.float32)}


def make_tokens(w: Workload, codec: dict, n: int, g: torch.Generator, device,
                block: int = 8192) -> tuple[torch.Tensor, torch.Tensor]:
    """n tokens [n, J] in the storage dtype, and their generating labels [n]."""
    J, C, rank = w.J, w.C, w.rank
    labels = torch.randint(0, C, (n,), generator=g, device=device)
    out = torch.empty(n, J, dtype=w.dtype, device=device)
    cen = codec["centers"].to(torch.float32)
    U = codec["U"]
    for s in range(0, n, block):
        e = min(n, s + block)
        gg = torch.randn(e - s, rank, generator=g, device=device)
        eps = torch.randn(e - s, J, generator=g, device=device)
        x = cen[labels[s:e]] + gg @ U.t() + w.noise * eps
        out[s:e] = _round(x, w.dtype)
    if w.outlier_frac > 0 and n > 0:
        k = int(round(w.outlier_frac * n))
        idx = torch.randperm(n, generator=g, device=device)[:k]
        out[idx] = _round(out[idx].to(torch.float32) * w.outlier_mult, w.dtype)
    return out, labels


def make_problem(w: Workload, layer: int = 0, device="cpu") -> dict:
    """One layer's inputs: codecs for K and V, raw history K/V [T, J], the
    current chunk's K/V [Tq, J] and queries [Tq, H, d]; all in storage dtype."""
    g = _gen(w.layer_seed(layer), device)
    ck = make_codec(w, g, device)
    cv = make_codec(w, g, device)
    hk, lk = make_tokens(w, ck, w.T, g, device)
    hv, lv = make_tokens(w, cv, w.T, g, device)
    kc, _ = make_tokens(w, ck, w.Tq, g, device)
    vc, _ = make_tokens(w, cv, w.Tq, g, device)
    q = _round(torch.randn(w.Tq, w.H, w.d, generator=g, device=device) / math.sqrt(w.d), w.dtype)
    return {
        "codec_k": ck, "codec_v": cv,
        "hist_k": hk, "hist_v": hv, "labels_k": lk, "labels_v": lv,
        "k_cur": kc.view(w.Tq, w.H, w.d), "v_cur": vc.view(w.Tq, w.H, w.d),
        "q": q.contiguous(),
    }


def scaled(w: Workload, **kw) -> Workload:
    """A smaller copy of a workload (for parity cases that the oracle finishes
    in seconds): same codec structure, other sizes."""
    return dataclasses.replace(w, **kw)


def make_lowdim_maps(w: Workload, seed: int, device="cpu") -> dict:
    """Maps for heads at a reduced attention dimension: U and W [H, d, d],
    each head a random orthonormal basis (QR of a Gaussian draw) rounded to
    the storage dtype.  Any orthonormal map is a valid input (the deployed
    maps are learned); which columns a head uses is the caller's d_h."""
    g = _gen(seed, device)

    def one():
        m = torch.randn(w.H, w.d, w.d, generator=g, device=device, dtype=torch.float64)
        return _round(torch.linalg.qr(m)[0], w.dtype).contiguous()
    return {"U": one(), "W": one()}
