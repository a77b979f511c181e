"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

This module is shared by the tests, the benchmark and the oracle checks. It
draws queries, key/value caches and hyperplanes; it never hashes, scores,
selects or attends. It imports neither the CUDA binding nor the oracle.

The shapes follow the decode workloads the SOCKET and HATA pages evaluate on
(Llama-3.2-1B, Llama-3.1-8B and Qwen3-30B long-context decode; HATA-style
hard hashing); the public benchmarks they use (LongBench, RULER) are not
available, so seeded Gaussian caches with the structure listed per workload
stand in for them:

* ``outlier_channels``: per KV head, that many seeded channels of both K and V
  are multiplied by ``outlier_scale`` (before rounding to bf16);
* ``lognormal_sigma``: value rows are v_i = exp(sigma * xi_i) * u_i with
  xi_i ~ N(0, 1) per key and u_i ~ N(0, I), i.e. heavy-tailed value norms;
* ``needles``: per (batch, kv-head) pair, that many keys at seeded distinct
  positions are replaced by 3 * sqrt(d) * q_hat_h + eps, eps ~ N(0, I), where
  q_hat_h is the unit query of head h = kvh * G + (j mod G) -- a key that points
  along the query with a typical key norm (the needle-in-a-haystack idea of
  the HGA page, gist.science/ja/paper/2606.30709, section 4 "結果").

Draw order (one torch.Generator per workload, on the target device): Q, R,
then for each batch element K[b], V[b] (and xi[b]), then outlier channels,
needle positions and needle noise.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    L: int          # hash tables (0 for the hard-hash variant)
    P: int          # hyperplanes per table (0 for the hard-hash variant)
    tau: float      # soft-assignment temperature (0 for the hard-hash variant)
    k: int          # keys kept per (batch, kv-head) pair
    kv_dtype: str   # "f32" or "bf16"
    seed: int
    needles: int = 0
    outlier_channels: int = 0
    outlier_scale: float = 8.0
    lognormal_sigma: float = 0.0
    hata: bool = False

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def pairs(self) -> int:
        return self.B * self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_kv_dtype(self) -> torch.dtype:
        return torch.float32 if self.kv_dtype == "f32" else torch.bfloat16

    def describe(self) -> dict:
        return dataclasses.asdict(self)


def _k_from_sparsity(N: int, sparsity: int) -> int:
    return N // sparsity


# The five decode workloads. k = floor(N / sparsity) (102400 / 33 -> 3103).
TINY_F32 = Workload("tiny_f32", B=1, Hq=1, Hkv=1, d=128, N=4096, L=8, P=4, tau=0.5, k=128,
                    kv_dtype="f32", seed=1000, needles=4)
LLAMA_1B = Workload("llama3.2-1b_n32k", B=1, Hq=32, Hkv=8, d=64, N=32768, L=32, P=8, tau=0.3,
                    k=_k_from_sparsity(32768, 33), kv_dtype="bf16", seed=2000, outlier_channels=4)
LLAMA_8B = Workload("llama3.1-8b_n100k", B=4, Hq=32, Hkv=8, d=128, N=102400, L=32, P=8, tau=0.3,
                    k=_k_from_sparsity(102400, 33), kv_dtype="bf16", seed=3000, needles=16,
                    outlier_channels=4)
QWEN3_30B = Workload("qwen3-30b_n140k", B=8, Hq=32, Hkv=4, d=128, N=143360, L=48, P=8, tau=0.2,
                     k=_k_from_sparsity(143360, 50), kv_dtype="bf16", seed=4000, lognormal_sigma=0.5)
HATA_16 = Workload("hata_n256k", B=16, Hq=32, Hkv=8, d=128, N=262144, L=0, P=0, tau=0.0, k=2048,
                   kv_dtype="bf16", seed=5000, hata=True)

WORKLOADS = {w.name: w for w in (TINY_F32, LLAMA_1B, LLAMA_8B, QWEN3_30B, HATA_16)}


def shrink(w: Workload, **changes) -> Workload:
    """A smaller variant of a workload (for tests): same structure, new sizes."""
    return dataclasses.replace(w, **changes)


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def make_inputs(w: Workload, device="cpu", ncap: int | None = None) -> dict:
    """Draw one decode step's inputs for workload ``w`` on ``device``.

    Returns a dict with
      Q  [B, Hq, d]        (kv dtype),
      K, V [B, Hkv, Ncap, d] (kv dtype; rows >= N are zero),
      R  [L*P, d] bf16     (SOCKET) or R128 [128, d] bf16 (hard-hash variant),
      needle_pos [B, Hkv, needles] int64 (may be empty),
      outlier_ch [Hkv, outlier_channels] int64 (may be empty).
    Ncap defaults to N rounded up to a multiple of 32.
    """
    device = torch.device(device)
    ncap = round_up(w.N, 32) if ncap is None else ncap
    if ncap < w.N or ncap % 32:
        raise ValueError("Ncap must be >= N and a multiple of 32")
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_kv_dtype

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    Q = randn(w.B, w.Hq, w.d).to(dt)
    nproj = 128 if w.hata else w.L * w.P
    R = randn(nproj, w.d).to(torch.bfloat16)

    K = torch.zeros(w.B, w.Hkv, ncap, w.d, dtype=dt, device=device)
    V = torch.zeros(w.B, w.Hkv, ncap, w.d, dtype=dt, device=device)
    Kf = []
    Vf = []
    for b in range(w.B):
        kb = randn(w.Hkv, w.N, w.d)
        vb = randn(w.Hkv, w.N, w.d)
        if w.lognormal_sigma > 0:
            xi = randn(w.Hkv, w.N, 1)
            vb = vb * torch.exp(w.lognormal_sigma * xi)
        Kf.append(kb)
        Vf.append(vb)

    outlier_ch = torch.empty(w.Hkv, w.outlier_channels, dtype=torch.int64, device=device)
    for h in range(w.Hkv):
        if w.outlier_channels:
            outlier_ch[h] = torch.randperm(w.d, generator=gen, device=device)[:w.outlier_channels]
    for b in range(w.B):
        for h in range(w.Hkv):
            if w.outlier_channels:
                Kf[b][h][:, outlier_ch[h]] *= w.outlier_scale
                Vf[b][h][:, outlier_ch[h]] *= w.outlier_scale

    needle_pos = torch.empty(w.B, w.Hkv, w.needles, dtype=torch.int64, device=device)
    if w.needles:
        for b in range(w.B):
            for h in range(w.Hkv):
                needle_pos[b, h] = torch.randperm(w.N, generator=gen, device=device)[:w.needles]
        qf = Q.float()
        for b in range(w.B):
            for h in range(w.Hkv):
                noise = randn(w.needles, w.d)
                for j in range(w.needles):
                    qh = qf[b, h * w.G + (j % w.G)]
                    q_hat = qh / qh.norm()
                    Kf[b][h][needle_pos[b, h, j]] = 3.0 * math.sqrt(w.d) * q_hat + noise[j]

    for b in range(w.B):
        K[b, :, :w.N] = Kf[b].to(dt)
        V[b, :, :w.N] = Vf[b].to(dt)
    out = {"Q": Q, "K": K, "V": V, "needle_pos": needle_pos, "outlier_ch": outlier_ch}
    out["R128" if w.hata else "R"] = R
    return out
