"""Seeded synthetic inputs for HiLS attention (the only module both the oracle
side and the CUDA side use).

It holds no arithmetic of the method: it only draws tensors.  The recipe:

* q, k, v and the landmark queries q'_c are i.i.d. N(0, 1), drawn in float32
  by a seeded ``torch.Generator`` and cast to bf16 (round to nearest even)
  for bf16 workloads;
* Q-Cal workloads add hidden states h ~ N(0, 1) of width ``d_model`` and
  W_down [r, d_model], W_up [H_q*d, r] ~ N(0, 0.02^2);
* "needles": for each query head h a query position i and an earlier key
  position j are drawn and k[h // G, j] is overwritten with
  4 * q[h, i] / |q[h, i]| (computed from the stored, already rounded q, then
  rounded to the storage type), so that the needle's chunk carries one dominant
  logit for that query.  Collisions on j are redrawn.

Small workloads are drawn on the CPU; large ones (``device='cuda'``) are drawn
by the CUDA generator of torch with the same seed, which is deterministic for
a given seed and device.  The oracle always receives host copies of exactly the
tensors the CUDA path receives.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int  # prefill length, or decode cache length L
    Hq: int
    Hkv: int
    d: int
    S: int
    W: int
    K: int
    M: int = 4
    dtype: str = "bf16"  # "f32" | "bf16"
    decode: bool = False
    needles_per_head: int = 0
    needle_gap: tuple[int, int] | None = None  # (lo, hi) of i - j, else uniform over i's candidate region
    d_model: int = 0  # Q-Cal hidden width (0 = no Q-Cal)
    qcal_rank: int = 0
    seed_index: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def C(self) -> int:
        return self.N // self.S

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def seed(self) -> int:
        return SEED_BASE + self.seed_index

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads, in order.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, N=512, Hq=4, Hkv=1, d=64, S=32, W=64, K=4, M=4, dtype="f32",
                         seed_index=0),
    "prefill_8k": Workload("prefill_8k", B=1, N=8192, Hq=32, Hkv=8, d=128, S=64, W=512, K=16, M=4,
                           needles_per_head=8, needle_gap=(2048, 6144), seed_index=1),
    "prefill_128k": Workload("prefill_128k", B=1, N=131072, Hq=32, Hkv=8, d=128, S=64, W=512, K=32, M=4,
                             needles_per_head=64, seed_index=2),
    "decode_512k": Workload("decode_512k", B=16, N=524288, Hq=32, Hkv=8, d=128, S=64, W=512, K=32,
                            decode=True, seed_index=3),
    "prefill_512k_qcal": Workload("prefill_512k_qcal", B=1, N=524288, Hq=32, Hkv=8, d=128, S=64, W=1024, K=64,
                                  M=4, needles_per_head=256, d_model=4096, qcal_rank=64, seed_index=4),
}


def _randn(shape, gen, device, dtype, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _generator(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _plant_needles(w: Workload, q: torch.Tensor, k: torch.Tensor, gen_cpu: torch.Generator) -> list:
    """Overwrite keys with normalised copies of earlier-drawn queries (see module doc)."""
    if w.needles_per_head <= 0:
        return []
    nw = w.W // w.S
    used = set()
    needles = []
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // w.G
            placed = 0
            tries = 0
            while placed < w.needles_per_head and tries < 100 * w.needles_per_head:
                tries += 1
                if w.needle_gap is not None:
                    lo, hi = w.needle_gap
                    j = int(torch.randint(0, w.N - lo, (1,), generator=gen_cpu))
                    i = j + int(torch.randint(lo, hi + 1, (1,), generator=gen_cpu))
                    if i >= w.N:
                        continue
                else:
                    first = (nw + 1) * w.S  # smallest i that has a candidate chunk
                    if first >= w.N:
                        break
                    i = int(torch.randint(first, w.N, (1,), generator=gen_cpu))
                    region = (i // w.S - nw + 1) * w.S
                    j = int(torch.randint(0, region, (1,), generator=gen_cpu))
                if (b, g, j) in used:
                    continue
                used.add((b, g, j))
                qi = q[b, h, i].float()
                k[b, g, j] = (4.0 * qi / qi.norm()).to(k.dtype)
                needles.append((b, h, i, j))
                placed += 1
    return needles


def prefill_inputs(w: Workload, device: str = "cpu") -> dict:
    """q [B,Hq,N,d], k/v [B,Hkv,N,d], q_lmk [B,Hq,C,d] (+ h, w_down, w_up for Q-Cal)."""
    gen = _generator(w.seed, device)
    dt = w.torch_dtype
    q = _randn((w.B, w.Hq, w.N, w.d), gen, device, dt)
    k = _randn((w.B, w.Hkv, w.N, w.d), gen, device, dt)
    v = _randn((w.B, w.Hkv, w.N, w.d), gen, device, dt)
    q_lmk = _randn((w.B, w.Hq, w.C, w.d), gen, device, dt)
    out = dict(q=q, k=k, v=v, q_lmk=q_lmk)
    if w.d_model:
        out["h"] = _randn((w.B, w.N, w.d_model), gen, device, dt)
        out["w_down"] = _randn((w.qcal_rank, w.d_model), gen, device, dt, std=0.02)
        out["w_up"] = _randn((w.Hq * w.d, w.qcal_rank), gen, device, dt, std=0.02)
    out["needles"] = _plant_needles(w, q, k, _generator(w.seed + 7919, "cpu"))
    return out


def decode_inputs(w: Workload, device: str = "cpu") -> dict:
    """q [B,Hq,d] (the token at position L-1), k/v cache [B,Hkv,L,d], q_lmk [B,Hq,C,d]."""
    gen = _generator(w.seed, device)
    dt = w.torch_dtype
    q = _randn((w.B, w.Hq, w.d), gen, device, dt)
    k = _randn((w.B, w.Hkv, w.N, w.d), gen, device, dt)
    v = _randn((w.B, w.Hkv, w.N, w.d), gen, device, dt)
    q_lmk = _randn((w.B, w.Hq, w.C, w.d), gen, device, dt)
    return dict(q=q, k=k, v=v, q_lmk=q_lmk, needles=[])
