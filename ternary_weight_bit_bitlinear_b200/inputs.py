"""Seeded synthetic inputs shaped like the pages' ternary models.

This module only draws random numbers and describes shapes.  It holds none of
the method's arithmetic (no quantisation, packing or matmul), so both the CUDA
path's tests and the CPU oracle may take their inputs from it.

Recipe (applies to every test, the smoke check and the benchmark):
  * latent weights W[M,K] ~ N(0, 0.02^2), fp32, one torch generator per matrix
    seeded with 1000*config + 16*layer + projection_index;
  * activations x[N,K] ~ N(0, 1), fp32, seeded with the same number + 500;
    a set of outlier channels (columns of x) is multiplied by 10.

The model shapes stand in for the 700M-100B ternary models of the Bitnet.cpp
reading notes (section 2.2, model sizes) and the BitNet b1.58 2B release named
in the CPU deployment notes; no dataset or trained weight is involved.
"""
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class ModelShape:
    name: str
    hidden: int
    ffn: int
    kv_dim: int       # width of the k and v projections (heads_kv * head_dim)

    def projections(self):
        """(name, M, K) of the seven BitLinear layers of one decoder layer,
        weights stored [M=out_features, K=in_features]."""
        h, f, kv = self.hidden, self.ffn, self.kv_dim
        return [("q", h, h), ("k", kv, h), ("v", kv, h), ("o", h, h),
                ("gate", f, h), ("up", f, h), ("down", h, f)]

    def weights_per_layer(self):
        return sum(M * K for _, M, K in self.projections())


# hidden, FFN, KV width (= kv_heads * head_dim)
MODEL_2B = ModelShape("bitnet-b1.58-2B", 2560, 6912, 640)     # 20 heads / 5 KV, head 128
MODEL_7B = ModelShape("7B", 4096, 11008, 4096)                # MHA 32 heads
MODEL_8B = ModelShape("8B", 4096, 14336, 1024)                # GQA 32 / 8
MODEL_70B = ModelShape("70B", 8192, 28672, 1024)              # GQA 64 / 8


@dataclass(frozen=True)
class Workload:
    """One benchmark / parity configuration."""
    index: int
    name: str
    model: ModelShape = None
    layers: int = 1
    tokens: tuple = (1,)
    single: tuple = None          # (M, K) for the single-matrix case
    outlier_frac: float = 0.0
    outlier_count: int = 0


WORKLOADS = {
    1: Workload(1, "single 1024x1024 decode GEMV", single=(1024, 1024), tokens=(1,),
                outlier_count=4),
    2: Workload(2, "2B-shaped decode, 30 layers streamed", model=MODEL_2B, layers=30,
                tokens=(1,)),
    3: Workload(3, "7B-shaped prefill, 7 projections", model=MODEL_7B, layers=1,
                tokens=(512,)),
    4: Workload(4, "8B-shaped batch sweep", model=MODEL_8B, layers=16,
                tokens=(1, 2, 4, 8, 16, 32, 64, 128), outlier_frac=0.01),
    5: Workload(5, "70B-shaped weight stream, 80 layers", model=MODEL_70B, layers=80,
                tokens=(1, 2048)),
}

OUTLIER_SCALE = 10.0


def weight_seed(config: int, layer: int, proj: int) -> int:
    return 1000 * config + 16 * layer + proj


def act_seed(config: int, layer: int, proj: int) -> int:
    return weight_seed(config, layer, proj) + 500


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def latent_weights(M: int, K: int, seed: int, device="cpu", std: float = 0.02):
    """fp32 W[M,K] ~ N(0, std^2)."""
    g = _gen(seed, device)
    w = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    return w.mul_(std)


def outlier_channels(K: int, seed: int, count: int = 0, frac: float = 0.0):
    """Sorted channel indices that carry outliers (drawn on the CPU)."""
    n = count if count else int(round(frac * K))
    if n <= 0:
        return torch.empty(0, dtype=torch.long)
    g = _gen(seed + 77, "cpu")
    return torch.randperm(K, generator=g)[:n].sort().values


def activations(N: int, K: int, seed: int, device="cpu", outlier_count: int = 0,
                outlier_frac: float = 0.0):
    """fp32 x[N,K] ~ N(0,1) with outlier channels scaled by OUTLIER_SCALE."""
    g = _gen(seed, device)
    x = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    idx = outlier_channels(K, seed, outlier_count, outlier_frac)
    if idx.numel():
        x[:, idx.to(x.device)] *= OUTLIER_SCALE
    return x
