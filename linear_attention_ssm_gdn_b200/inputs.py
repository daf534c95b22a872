"""Seeded synthetic inputs for the GDN hot path (CPU tensors).

This module only draws and rounds random numbers in the shapes and value
distributions of the five workloads; it holds none of the method's
arithmetic.  The CUDA path and the oracle both read the tensors it returns
(the oracle widens the very same bf16/f32 values to f64).

Distributions (per workload description):
  q, k, v  ~ N(0, 1), q and k L2-normalised per (token, head) in f32, then
           rounded to bf16;
  g        = log-sigmoid(N(2, 1))  (so g <= 0), f32;
  beta     = sigmoid(N(0, 1)), f32;
  h0       ~ N(0, 0.02) (0.02 is the standard deviation), f32, or zeros;
  BA front end: x ~ N(0,1) bf16 [M, K], W_ba ~ N(0, 0.02) bf16 [2 nv, K],
           A_log ~ U(-1, 1), dt_bias ~ N(0, 0.1), both f32 [nv].
Every workload draws from one torch CPU generator seeded with its index.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

CHUNK = 64


def _normal(gen, shape, std=1.0, mean=0.0):
    return torch.randn(shape, generator=gen, dtype=torch.float32) * std + mean


def _l2norm_bf16(x: torch.Tensor) -> torch.Tensor:
    """Unit-norm each last-dim row in f32, then round to bf16 (input recipe)."""
    n = torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-6)
    return (x / n).to(torch.bfloat16)


@dataclass
class PrefillInputs:
    q: torch.Tensor          # bf16 [T, H_k, d_k]
    k: torch.Tensor          # bf16 [T, H_k, d_k]
    v: torch.Tensor          # bf16 [T, H_v, d_v]
    g: torch.Tensor | None   # f32 [T, H_v]  (None when the BA front end produces it)
    beta: torch.Tensor | None
    cu_seqlens: torch.Tensor  # int32 [N + 1]
    h0: torch.Tensor          # f32 [N, H_v, d_k, d_v]
    H_k: int
    H_v: int
    d_k: int
    d_v: int
    scale: float = 1.0

    @property
    def total_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)


@dataclass
class BAInputs:
    x: torch.Tensor        # bf16 [M, K]
    w: torch.Tensor        # bf16 [2 nv, K]
    a_log: torch.Tensor    # f32 [nv]
    dt_bias: torch.Tensor  # f32 [nv]
    nv: int
    vheads_per_group: int


@dataclass
class VerifyInputs:
    pool: torch.Tensor      # f32 [slots, H_v, d_k, d_v]  the state pool
    slots: torch.Tensor     # int64 [batch]  pool slot of sequence b (h_table[b])
    q: torch.Tensor         # bf16 [batch*K, H_k, d_k]
    k: torch.Tensor
    v: torch.Tensor         # bf16 [batch*K, H_v, d_v]
    g: torch.Tensor         # f32 [batch*K, H_v] (values rounded to bf16)
    beta: torch.Tensor
    na: torch.Tensor        # int32 [batch] in 0..K
    batch: int
    K: int
    H_k: int
    H_v: int
    d_k: int
    d_v: int
    scale: float = 1.0


def prefill_inputs(seqlens, H_k, H_v, d_k, d_v, seed, h0_std=None, gates=True,
                   gen=None) -> PrefillInputs:
    """q/k/v/g/beta/h0 for packed sequences of the given lengths."""
    gen = torch.Generator().manual_seed(seed) if gen is None else gen
    seqlens = [int(s) for s in seqlens]
    T = sum(seqlens)
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    q = _l2norm_bf16(_normal(gen, (T, H_k, d_k)))
    k = _l2norm_bf16(_normal(gen, (T, H_k, d_k)))
    v = _normal(gen, (T, H_v, d_v)).to(torch.bfloat16)
    g = beta = None
    if gates:
        g = torch.nn.functional.logsigmoid(_normal(gen, (T, H_v), 1.0, 2.0))
        beta = torch.sigmoid(_normal(gen, (T, H_v)))
    if h0_std is None:
        h0 = torch.zeros(len(seqlens), H_v, d_k, d_v, dtype=torch.float32)
    else:
        h0 = _normal(gen, (len(seqlens), H_v, d_k, d_v), h0_std)
    return PrefillInputs(q, k, v, g, beta, cu, h0, H_k, H_v, d_k, d_v)


def ba_inputs(M, K, nv, vheads_per_group, seed, gen=None) -> BAInputs:
    gen = torch.Generator().manual_seed(seed) if gen is None else gen
    x = _normal(gen, (M, K)).to(torch.bfloat16)
    w = _normal(gen, (2 * nv, K), 0.02).to(torch.bfloat16)
    a_log = torch.rand((nv,), generator=gen, dtype=torch.float32) * 2.0 - 1.0
    dt_bias = _normal(gen, (nv,), 0.1)
    return BAInputs(x, w, a_log, dt_bias, nv, vheads_per_group)


def verify_inputs(batch, K, H_k, H_v, d_k, d_v, slots_total, seed) -> VerifyInputs:
    gen = torch.Generator().manual_seed(seed)
    pool = _normal(gen, (slots_total, H_v, d_k, d_v), 0.02)
    slots = torch.randperm(slots_total, generator=gen)[:batch]
    R = batch * K
    q = _l2norm_bf16(_normal(gen, (R, H_k, d_k)))
    k = _l2norm_bf16(_normal(gen, (R, H_k, d_k)))
    v = _normal(gen, (R, H_v, d_v)).to(torch.bfloat16)
    g = torch.nn.functional.logsigmoid(_normal(gen, (R, H_v), 1.0, 2.0))
    g = g.to(torch.bfloat16).to(torch.float32)
    beta = torch.sigmoid(_normal(gen, (R, H_v))).to(torch.bfloat16).to(torch.float32)
    na = torch.randint(0, K + 1, (batch,), generator=gen, dtype=torch.int32)
    return VerifyInputs(pool, slots, q, k, v, g, beta, na, batch, K, H_k, H_v, d_k, d_v)


# ---------------------------------------------------------------------------
# The five named workloads
# ---------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    index: int
    prefill: PrefillInputs | None = None
    ba: BAInputs | None = None
    verify: VerifyInputs | None = None
    meta: dict = field(default_factory=dict)


WORKLOAD_NAMES = {
    0: "gdn-prefill-tiny: T=256 H_k=H_v=2 d=64",
    1: "gdn-prefill-single: T=4096 H_k=16 H_v=32 d=128",
    2: "gdn-prefill-ba: M=4576 K=5120 H_k=16 H_v=48 d=128",
    3: "gdn-prefill-varlen: 8 seqs in [512,8192] H_k=16 H_v=48 d=128",
    4: "gdn-verify-fold: batch=64 K=4 H_k=16 H_v=48 d=128",
}


def varlen_lengths(seed: int = 3, n: int = 8, lo: int = 512, hi: int = 8192):
    gen = torch.Generator().manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]


def workload(index: int) -> Workload:
    """Inputs of workload `index` (0..4), drawn with seed = index."""
    if index == 0:
        p = prefill_inputs([256], 2, 2, 64, 64, seed=0, h0_std=None)
        return Workload(WORKLOAD_NAMES[0], 0, prefill=p)
    if index == 1:
        p = prefill_inputs([4096], 16, 32, 128, 128, seed=1, h0_std=0.02)
        return Workload(WORKLOAD_NAMES[1], 1, prefill=p)
    if index == 2:
        gen = torch.Generator().manual_seed(2)
        ba = ba_inputs(4576, 5120, 48, 3, seed=2, gen=gen)
        p = prefill_inputs([4576], 16, 48, 128, 128, seed=2, h0_std=None, gates=False, gen=gen)
        return Workload(WORKLOAD_NAMES[2], 2, prefill=p, ba=ba)
    if index == 3:
        lens = varlen_lengths(3)
        p = prefill_inputs(lens, 16, 48, 128, 128, seed=3, h0_std=0.02)
        return Workload(WORKLOAD_NAMES[3], 3, prefill=p, meta={"seqlens": lens})
    if index == 4:
        vi = verify_inputs(64, 4, 16, 48, 128, 128, slots_total=128, seed=4)
        return Workload(WORKLOAD_NAMES[4], 4, verify=vi)
    raise ValueError(f"no workload {index}")
