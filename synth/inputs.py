"""Workload definitions and seeded generators for the NVFP4 MoE expert-FFN.

Shapes are DeepSeek-style MoE FFN shapes (hidden 7168, intermediate 2048, 256 experts,
top-8), matching the pages' model (DSV4 NVFP4 MegaMoE); no trained weights are used.

Seeds and order (torch generators):
  logits : seed                    (CPU)
  x      : seed + 1                (CPU), drawn in float32 then rounded to bf16
  W1[e]  : 1000 * seed + e         (N(0, 0.02) in float32, rounded to bf16, on the requested device)
  W2[e]  : 1000 * seed + 500 + e
For the E=256 workloads the weights are drawn on the GPU (6+ GB of float32 would take minutes
on the host); a check that needs an expert's floats on the host copies them back.
"""

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    logits: str          # "normal" | "uniform" | "zipf_gumbel"
    x_outliers: bool = False
    seed: int = 0
    renormalize: bool = True
    gs_h: float = 1.0    # static global scale of the intermediate h (calibrated per shape)

    @property
    def slots(self):
        return self.T * self.k

    def flops(self):
        """Algorithmic FLOPs: 2 * slots * (H * 2I + I * H); padding rows do not count."""
        return 2 * self.slots * (self.H * 2 * self.I + self.I * self.H)


@dataclass(frozen=True)
class SweepConfig:
    name: str
    E: int
    K: int
    N: int
    m_max: int
    seed: int = 0


@dataclass(frozen=True)
class DenseConfig:
    """A dense NVFP4 linear out = RMSNorm(x) W^T (M x K activations, N x K weight): the MoE
    shared expert's gate/up projection, hidden 7168 -> 2 * 2048."""
    name: str
    M: int
    N: int
    K: int
    norm: bool = True
    eps: float = 1e-6
    seed: int = 0

    def flops(self):
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class SharedConfig:
    """The MoE shared expert on every token: RMSNorm(x) -> L1 (2I x H) + SwiGLU -> L2 (H x I)."""
    name: str
    M: int
    H: int
    I: int
    eps: float = 1e-6
    gs_h: float = 1.0
    seed: int = 0

    def flops(self):
        return 2 * self.M * self.H * 2 * self.I + 2 * self.M * self.I * self.H


CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, H=256, I=128, E=8, k=2, logits="normal", gs_h=64.0),
    "decode": MoEConfig("decode", T=16, H=7168, I=2048, E=256, k=8, logits="uniform"),
    "mid": MoEConfig("mid", T=512, H=7168, I=2048, E=256, k=8, logits="zipf_gumbel", x_outliers=True),
    "prefill": MoEConfig("prefill", T=8192, H=7168, I=2048, E=256, k=8, logits="uniform"),
    "sweep": SweepConfig("sweep", E=32, K=7168, N=4096, m_max=4096),
    "dense_decode": DenseConfig("dense_decode", M=16, N=4096, K=7168),
    "dense_prefill": DenseConfig("dense_prefill", M=8192, N=4096, K=7168),
    "shared_decode": SharedConfig("shared_decode", M=16, H=7168, I=2048),
    "shared_prefill": SharedConfig("shared_prefill", M=8192, H=7168, I=2048),
}


def gen_logits(cfg):
    """Router logits float32 (T, E) on the CPU.

    normal      N(0, 1)
    uniform     U(0, 1) i.i.d. (near-uniform expert load)
    zipf_gumbel log p_pi(e) + Gumbel(0, 1), p proportional to rank^-1.2 over a seeded
                permutation pi, so top-k samples experts without replacement by p; 8 seeded
                experts are set to -inf (they receive no tokens: empty experts).
    """
    g = torch.Generator().manual_seed(cfg.seed)
    T, E = cfg.T, cfg.E
    if cfg.logits == "normal":
        return torch.randn(T, E, generator=g, dtype=torch.float32)
    if cfg.logits == "uniform":
        return torch.rand(T, E, generator=g, dtype=torch.float32)
    if cfg.logits == "zipf_gumbel":
        perm = torch.randperm(E, generator=g)
        rank = torch.empty(E, dtype=torch.float64)
        rank[perm] = torch.arange(1, E + 1, dtype=torch.float64)
        logp = (-1.2 * torch.log(rank)).to(torch.float32)
        u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_(1e-12, 1 - 1e-12)
        gumbel = (-torch.log(-torch.log(u))).to(torch.float32)
        lg = logp[None, :] + gumbel
        masked = torch.randperm(E, generator=g)[:8]
        lg[:, masked] = float("-inf")
        return lg
    raise ValueError(cfg.logits)


def gen_x(cfg, T=None, H=None):
    """Activations bf16 (T, H) on the CPU: N(0, 1); with outliers, a seeded 1% of the elements
    are multiplied by 50."""
    T = cfg.T if T is None else T
    H = cfg.H if H is None else H
    g = torch.Generator().manual_seed(cfg.seed + 1)
    x = torch.randn(T, H, generator=g, dtype=torch.float32)
    if cfg.x_outliers:
        mask = torch.rand(T, H, generator=g) < 0.01
        x = torch.where(mask, x * 50.0, x)
    return x.to(torch.bfloat16)


def gen_weight_expert(seed, which, e, N, K, device="cpu", std=0.02):
    """bf16 (N, K) weight of expert e (drawn in float32, rounded to bf16 like model weights):
    which=1 for W1 (2I x H, gate rows then up rows), 2 for W2 (H x I)."""
    s = 1000 * seed + (0 if which == 1 else 500) + e
    g = torch.Generator(device=device).manual_seed(s)
    w = torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * std
    return w.to(torch.bfloat16)


def gen_sweep(cfg, device="cpu"):
    """Group sizes M_g ~ U{0..m_max} (seeded) for the standalone grouped-GEMM sweep, plus
    generators for A (N(0,1)) and B (N(0,0.02)) rows."""
    g = torch.Generator().manual_seed(cfg.seed)
    m = torch.randint(0, cfg.m_max + 1, (cfg.E,), generator=g)
    return m.tolist()


def gen_sweep_a(cfg, rows, device="cpu"):
    g = torch.Generator(device=device).manual_seed(cfg.seed + 7)
    return torch.randn(rows, cfg.K, generator=g, dtype=torch.float32, device=device)


def gen_dense(cfg, device="cpu"):
    """Inputs of a dense workload: x bf16 (M, K) N(0, 1) (seed + 11), gamma bf16 (K,)
    1 + 0.1 N(0, 1) (seed + 12), W bf16 (N, K) N(0, 0.02) (seed + 13, on `device`)."""
    g = torch.Generator().manual_seed(cfg.seed + 11)
    x = torch.randn(cfg.M, cfg.K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    g = torch.Generator().manual_seed(cfg.seed + 12)
    gamma = (1.0 + 0.1 * torch.randn(cfg.K, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    g = torch.Generator(device=device).manual_seed(cfg.seed + 13)
    w = (torch.randn(cfg.N, cfg.K, generator=g, dtype=torch.float32, device=device) * 0.02)
    return x, gamma, w.to(torch.bfloat16)


def gen_shared(cfg, device="cpu"):
    """Inputs of a shared-expert workload: x bf16 (M, H) N(0, 1) (seed + 21), gamma bf16 (H,)
    1 + 0.1 N(0, 1) (seed + 22); W1 (2I x H, gate rows then up rows) and W2 (H x I) bf16
    N(0, 0.02) from seeds seed + 23 and seed + 24 (on `device`)."""
    g = torch.Generator().manual_seed(cfg.seed + 21)
    x = torch.randn(cfg.M, cfg.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    g = torch.Generator().manual_seed(cfg.seed + 22)
    gamma = (1.0 + 0.1 * torch.randn(cfg.H, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    g = torch.Generator(device=device).manual_seed(cfg.seed + 23)
    w1 = torch.randn(2 * cfg.I, cfg.H, generator=g, dtype=torch.float32, device=device) * 0.02
    g = torch.Generator(device=device).manual_seed(cfg.seed + 24)
    w2 = torch.randn(cfg.H, cfg.I, generator=g, dtype=torch.float32, device=device) * 0.02
    return x, gamma, w1.to(torch.bfloat16), w2.to(torch.bfloat16)
