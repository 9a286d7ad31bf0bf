"""Seeded synthetic workloads for the CSA/HCA attention step.

This module only draws random inputs of the right shapes and distributions;
it holds none of the method's arithmetic and imports neither the CUDA binding
nor the oracle, so both sides can be fed the same bits.

Shapes follow the V4 hyper-parameters printed on "DeepSeek-V4-Pro - Model
techniques map" (table "Checked in its code": 128 query heads of dim 512 with
one KV head, sliding window 128, indexer 64 heads x 128 dims, top-k 1024,
compress ratios 4 and 128).

Distributions (the recipe; every tensor has its own seed ``seed*1000 + id``
and, for per-sequence tensors, ``+ 100000*(b+1)``):
  * streams A, B, queries q, indexer queries q_I, indexer keys K_I and the
    directly drawn compressed KV rows: bf16 from N(0,1) (fp32 draw, RNE cast);
  * pooling logits [2m][d] (the positional bias): fp32 N(0,1);
  * input-dependent compression weights Z_a, Z_b [T][d]: bf16 from N(0,1);
  * indexer head weights w: fp32 U(0,1);
  * the FP4 workload scales ``key_outliers`` fixed indexer-key channels by 8
    (ceil(1% of 128) = 2 channels, chosen by a seeded permutation).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

# tensor ids for seeding
_ID_A, _ID_B, _ID_LOGITS, _ID_Q, _ID_QI, _ID_W, _ID_KI, _ID_KV, _ID_OUTLIER, _ID_ZA, _ID_ZB = range(1, 12)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    T: int              # context length; decode queries sit at position T-1
    m: int              # compression ratio
    H: int = 128        # query heads
    D: int = 512        # head dim == KV dim == latent stream width
    H_I: int = 64       # indexer heads
    d_I: int = 128      # indexer head dim
    k: int = 1024       # top-k
    W: int = 128        # sliding window
    nq: int = 1         # queries per sequence
    q_pos0: Optional[int] = None   # first query position (default T - nq)
    eps: float = 1e-6
    hca: bool = False
    fp4: bool = False
    key_outliers: int = 0          # indexer-key channels scaled x8
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T // self.m

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def q_positions(self) -> torch.Tensor:
        p0 = self.T - self.nq if self.q_pos0 is None else self.q_pos0
        pos = torch.arange(p0, p0 + self.nq, dtype=torch.int32)
        return pos.unsqueeze(0).expand(self.batch, self.nq).contiguous()

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five synthetic configurations.
TINY = Workload("tiny_csa_decode", batch=1, T=2048, m=4, H=8, D=64, H_I=4, d_I=32, k=64, W=16)
CSA_DECODE = Workload("csa_decode_128k", batch=8, T=131072, m=4)
CSA_PREFILL = Workload("csa_prefill_64k", batch=1, T=65536, m=4, nq=4096, q_pos0=61440)
HCA_DECODE = Workload("hca_decode_1m", batch=32, T=1048576, m=128, hca=True)
FP4_DECODE = Workload("fp4_index_decode_1m", batch=4, T=1048576, m=4, fp4=True, key_outliers=2)

ALL = (TINY, CSA_DECODE, CSA_PREFILL, HCA_DECODE, FP4_DECODE)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _seed(wl: Workload, tid: int, b: Optional[int] = None) -> int:
    s = wl.seed * 1000 + tid
    if b is not None:
        s += 100000 * (b + 1)
    return s


def normal_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def uniform_f32(shape, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


def stream(wl: Workload, which: str, b: int, device="cpu", T: Optional[int] = None) -> torch.Tensor:
    """Latent KV stream 'A' or 'B' of sequence b: [T][D] bf16."""
    tid = _ID_A if which == "A" else _ID_B
    return normal_bf16((wl.T if T is None else T, wl.D), _seed(wl, tid, b), device)


def compression_weights(wl: Workload, which: str, b: int, device="cpu", T: Optional[int] = None) -> torch.Tensor:
    """Compression-weight rows 'Za' or 'Zb' of sequence b: [T][D] bf16."""
    tid = _ID_ZA if which == "Za" else _ID_ZB
    return normal_bf16((wl.T if T is None else T, wl.D), _seed(wl, tid, b), device)


def streams(wl: Workload, device="cpu"):
    A = torch.stack([stream(wl, "A", b, device) for b in range(wl.batch)])
    B = torch.stack([stream(wl, "B", b, device) for b in range(wl.batch)])
    return A, B


def pool_logits(wl: Workload, device="cpu") -> torch.Tensor:
    g = _gen(device, _seed(wl, _ID_LOGITS))
    return torch.randn((2 * wl.m, wl.D), generator=g, device=device, dtype=torch.float32)


def queries(wl: Workload, device="cpu") -> torch.Tensor:
    """Attention queries [batch][nq][H][D] bf16."""
    return torch.stack([normal_bf16((wl.nq, wl.H, wl.D), _seed(wl, _ID_Q, b), device)
                        for b in range(wl.batch)])


def index_queries(wl: Workload, device="cpu") -> torch.Tensor:
    """Indexer queries [batch][nq][H_I][d_I] bf16."""
    return torch.stack([normal_bf16((wl.nq, wl.H_I, wl.d_I), _seed(wl, _ID_QI, b), device)
                        for b in range(wl.batch)])


def index_weights(wl: Workload, device="cpu") -> torch.Tensor:
    """Indexer head weights [batch][nq][H_I] fp32 ~ U(0,1)."""
    return torch.stack([uniform_f32((wl.nq, wl.H_I), _seed(wl, _ID_W, b), device)
                        for b in range(wl.batch)])


def outlier_channels(wl: Workload) -> torch.Tensor:
    g = _gen("cpu", _seed(wl, _ID_OUTLIER))
    return torch.randperm(wl.d_I, generator=g)[: wl.key_outliers].sort().values


def index_keys(wl: Workload, device="cpu", b: Optional[int] = None) -> torch.Tensor:
    """Compressed indexer keys [batch][N][d_I] bf16 (or [N][d_I] for one sequence)."""
    def one(bb):
        k = normal_bf16((wl.N, wl.d_I), _seed(wl, _ID_KI, bb), device)
        if wl.key_outliers:
            ch = outlier_channels(wl).to(device)
            k[:, ch] = k[:, ch] * 8   # power-of-two scale: exact in bf16
        return k
    if b is not None:
        return one(b)
    return torch.stack([one(bb) for bb in range(wl.batch)])


def direct_kv(wl: Workload, device="cpu", b: Optional[int] = None) -> torch.Tensor:
    """Compressed KV rows drawn directly, [batch][N][D] bf16 N(0,1)."""
    if b is not None:
        return normal_bf16((wl.N, wl.D), _seed(wl, _ID_KV, b), device)
    return torch.stack([normal_bf16((wl.N, wl.D), _seed(wl, _ID_KV, bb), device)
                        for bb in range(wl.batch)])


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def by_name(name: str) -> Workload:
    for wl in ALL:
        if wl.name == name:
            return wl
    raise KeyError(name)
