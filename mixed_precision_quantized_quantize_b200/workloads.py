"""Seeded synthetic inputs for the hybrid W4A4 + outlier linear layer.

This module only draws numbers: it holds none of the layer's arithmetic
(no scales, codes, packing or products), so that the CUDA path and the CPU
oracle can both be fed from it without sharing any of the method.

The layer shapes stand in for the Llama projections that the QUIK and Atom
pages evaluate on (QUIK abstract: LLaMA / OPT / Falcon; Atom summary:
Llama 7B-65B); their trained weights and datasets are not used.  Values:

* activations X ~ N(0, 1), except for ``k_o`` outlier channels (the last
  ``k_o`` entries of a seeded random permutation of the K input channels),
  which are multiplied by ``outlier_mult``; with ``student_t`` the outlier
  channels draw from a Student-t with 3 degrees of freedom instead of N(0,1)
  before the multiplication (heavy tails);
* weights W ~ N(0, w_std^2); bias ~ N(0, 0.01^2) when present;
* with an RMS norm in front of the layer (``rmsnorm``), X is the hidden state
  before the norm: the activations above with every token row multiplied by
  2^u, u ~ U(-2, 3) (tokens of different magnitude), and the norm weight is
  gamma = |1 + 0.25 N(0, 1)| clamped to [0.02, 4]; eps = 1e-5.

Everything is drawn on the CPU in fp32 from ``torch.Generator`` streams with
fixed seeds and then rounded to fp16.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

# One seed per independent stream.
SEED_X, SEED_W, SEED_PERM, SEED_BIAS, SEED_T, SEED_NORM = 0, 1, 2, 3, 4, 5
NORM_EPS = 1e-5


@dataclass(frozen=True)
class LayerConfig:
    name: str
    M: int
    N: int
    K: int
    k_o: int
    group: int = 0              # 0: per-token / per-channel scales; 128: groups of 128
    outlier_int8: bool = False  # False: FP16 outlier block (QUIK); True: INT8 (Atom)
    outlier_mult: float = 30.0
    student_t: bool = False
    w_std: float = 0.02
    bias: bool = False
    act_bits: int = 4           # 4: INT4 activations (W4A4); 8: INT8 activations (W4A8)
    weight_bits: int = 4        # 4: INT4 weights; 8: INT8 weights (W8A8)
    rmsnorm: bool = False       # X is the hidden state before an RMS norm folded into the layer
    sparse24: bool = False      # W pruned to 2:4 (two kept INT4 codes per group of four)
    description: str = field(default="", compare=False)

    @property
    def K_i(self) -> int:
        return self.K - self.k_o

    @property
    def ops(self) -> int:
        """Multiply-adds x 2 over the full K (INT4 part and outliers)."""
        return 2 * self.M * self.N * self.K

    @property
    def gemm_bytes(self) -> int:
        """Bytes the GEMM must move at least once: packed codes (half a byte
        each), the outlier blocks, the fp32 scales, the fp16 output and bias."""
        groups = self.K_i // 128 if self.group else 1
        ob = 1 if self.outlier_int8 else 2
        if self.sparse24:  # kept codes (K_i / 4 bytes) and position pairs (K_i / 8) per W row
            b = self.M * self.act_bits * self.K_i // 8 + self.N * (self.K_i // 4 + self.K_i // 8)
        else:
            b = (self.M * self.act_bits + self.N * self.weight_bits) * self.K_i // 8  # Xq, Wq
        b += (self.M + self.N) * self.k_o * ob           # Xo, Wo
        b += (self.M + self.N) * groups * 4              # sx, sw
        if self.outlier_int8 and self.k_o:
            b += (self.M + self.N) * 4                   # sxo, swo
        b += self.M * self.N * 2                         # Y
        if self.bias:
            b += self.N * 2
        return b


    @property
    def quant_bytes(self) -> int:
        """Bytes the activation quantiser must move: the fp16 row read once,
        the codes, outlier block and scales written."""
        groups = self.K_i // 128 if self.group else 1
        b = self.M * self.K * 2                                      # X
        b += self.M * self.act_bits * self.K_i // 8                  # Xq
        b += self.M * self.k_o * (1 if self.outlier_int8 else 2)     # Xo
        b += self.M * groups * 4                                     # sx
        if self.outlier_int8 and self.k_o:
            b += self.M * 4                                          # sxo
        return b


# The five layer workloads (the third has three token counts).
CONFIGS = {
    "tiny_16x256x256": LayerConfig(
        "tiny_16x256x256", M=16, N=256, K=256, k_o=32, outlier_mult=20.0, bias=True,
        description="tiny hybrid linear, FP16 outliers, bias"),
    "llama7b_attn_2048x4096x4096": LayerConfig(
        "llama7b_attn_2048x4096x4096", M=2048, N=4096, K=4096, k_o=128, student_t=True,
        description="Llama-7B attention projection, 128 FP16 outliers (Student-t x30)"),
    "llama7b_up_16x11008x4096": LayerConfig(
        "llama7b_up_16x11008x4096", M=16, N=11008, K=4096, k_o=128,
        description="Llama-7B MLP up-projection, 16 tokens"),
    "llama7b_up_256x11008x4096": LayerConfig(
        "llama7b_up_256x11008x4096", M=256, N=11008, K=4096, k_o=128,
        description="Llama-7B MLP up-projection, 256 tokens"),
    "llama7b_up_2048x11008x4096": LayerConfig(
        "llama7b_up_2048x11008x4096", M=2048, N=11008, K=4096, k_o=128,
        description="Llama-7B MLP up-projection, 2048 tokens"),
    "llama65b_mlp_grouped_1024x22016x8192": LayerConfig(
        "llama65b_mlp_grouped_1024x22016x8192", M=1024, N=22016, K=8192, k_o=128, group=128,
        outlier_int8=True, w_std=0.015,
        description="Atom-style grouped W4A4 (group 128), INT8 outliers, Llama-65B MLP"),
    "llama7b_attn_w4a8_2048x4096x4096": LayerConfig(
        "llama7b_attn_w4a8_2048x4096x4096", M=2048, N=4096, K=4096, k_o=128, student_t=True,
        act_bits=8,
        description="the attention projection with INT8 activations (W4A8, QQQ), 128 FP16 outliers"),
    "llama7b_attn_w8a8_2048x4096x4096": LayerConfig(
        "llama7b_attn_w8a8_2048x4096x4096", M=2048, N=4096, K=4096, k_o=128, student_t=True,
        act_bits=8, weight_bits=8,
        description="the attention projection as W8A8 (the INT8 baseline), 128 FP16 outliers"),
    "llama7b_attn_rmsnorm_2048x4096x4096": LayerConfig(
        "llama7b_attn_rmsnorm_2048x4096x4096", M=2048, N=4096, K=4096, k_o=128, student_t=True,
        rmsnorm=True,
        description="the attention projection behind its RMS norm (norm folded into the quantiser)"),
    "llama7b_up_sparse24_16x11008x4096": LayerConfig(
        "llama7b_up_sparse24_16x11008x4096", M=16, N=11008, K=4096, k_o=128, sparse24=True,
        description="the MLP up-projection, 16 tokens, with 2:4-sparse INT4 weights"),
    "llama7b_attn_sparse24_2048x4096x4096": LayerConfig(
        "llama7b_attn_sparse24_2048x4096x4096", M=2048, N=4096, K=4096, k_o=128, student_t=True,
        sparse24=True,
        description="the attention projection with 2:4-sparse INT4 weights"),
    "llama7b_down_fused_4096x4096x11008": LayerConfig(
        "llama7b_down_fused_4096x4096x11008", M=4096, N=4096, K=11008, k_o=256,
        outlier_mult=50.0, bias=True,
        description="Llama-7B down-projection, quantize + GEMM together, 256 FP16 outliers, bias"),
}

# The workload the benchmark times at one GPU.
BENCH_CONFIG = "llama7b_attn_2048x4096x4096"


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def make_perm(K: int, seed: int = SEED_PERM) -> torch.Tensor:
    """Seeded random permutation of the K input channels (int32)."""
    return torch.randperm(K, generator=_gen(seed)).to(torch.int32)


def student_t3(shape, seed: int = SEED_T) -> torch.Tensor:
    """Student-t (3 degrees of freedom) from its definition Z / sqrt(chi2_3 / 3)."""
    g = _gen(seed)
    z = torch.randn(shape, generator=g)
    chi2 = torch.randn((3,) + tuple(shape), generator=g).square().sum(0)
    return z / torch.sqrt(chi2 / 3.0)


def make_activations(M: int, K: int, perm: torch.Tensor, k_o: int, outlier_mult: float,
                     student_t: bool = False, seed: int = SEED_X,
                     t_seed: int = SEED_T) -> torch.Tensor:
    """X fp16 [M, K]; the channels perm[K-k_o:] are the outliers."""
    x = torch.randn((M, K), generator=_gen(seed))
    if k_o > 0:
        cols = perm[K - k_o:].long()
        base = student_t3((M, k_o), t_seed) if student_t else x[:, cols]
        x[:, cols] = base * outlier_mult
    return x.to(torch.float16)


def token_magnitudes(M: int, seed: int = SEED_NORM) -> torch.Tensor:
    """Per-token factors 2^u, u ~ U(-2, 3), fp32 [M, 1]."""
    u = torch.rand((M, 1), generator=_gen(seed + 100)) * 5.0 - 2.0
    return torch.exp2(u)


def make_hidden(M: int, K: int, perm: torch.Tensor, k_o: int, outlier_mult: float,
                student_t: bool = False, seed: int = SEED_X, t_seed: int = SEED_T,
                norm_seed: int = SEED_NORM) -> torch.Tensor:
    """The hidden state before an RMS norm, fp16 [M, K]: the activations of
    make_activations (drawn in fp32) times a per-token magnitude."""
    x = torch.randn((M, K), generator=_gen(seed))
    if k_o > 0:
        cols = perm[K - k_o:].long()
        base = student_t3((M, k_o), t_seed) if student_t else x[:, cols]
        x[:, cols] = base * outlier_mult
    return (x * token_magnitudes(M, norm_seed)).to(torch.float16)


def make_norm_weight(K: int, seed: int = SEED_NORM) -> torch.Tensor:
    """RMS-norm weight gamma fp16 [K]: |1 + 0.25 N(0, 1)| clamped to [0.02, 4]."""
    g = (1.0 + 0.25 * torch.randn((K,), generator=_gen(seed))).abs().clamp(0.02, 4.0)
    return g.to(torch.float16)


def make_weights(N: int, K: int, w_std: float, seed: int = SEED_W) -> torch.Tensor:
    return (torch.randn((N, K), generator=_gen(seed)) * w_std).to(torch.float16)


def make_bias(N: int, seed: int = SEED_BIAS) -> torch.Tensor:
    return (torch.randn((N,), generator=_gen(seed)) * 0.01).to(torch.float16)


def make_layer(cfg: LayerConfig, M: int | None = None, seed_offset: int = 0):
    """All inputs of one layer call: dict(X, W, perm, bias) as CPU tensors
    (plus gamma and eps of the RMS norm when ``cfg.rmsnorm``).

    ``M`` overrides the token count (same weights); ``seed_offset`` shifts every
    stream so that tests can draw several independent cases of one shape.
    """
    M = cfg.M if M is None else M
    so = seed_offset
    perm = make_perm(cfg.K, SEED_PERM + so)
    if cfg.rmsnorm:
        X = make_hidden(M, cfg.K, perm, cfg.k_o, cfg.outlier_mult, cfg.student_t,
                        SEED_X + so, SEED_T + so, SEED_NORM + so)
    else:
        X = make_activations(M, cfg.K, perm, cfg.k_o, cfg.outlier_mult, cfg.student_t,
                             SEED_X + so, SEED_T + so)
    W = make_weights(cfg.N, cfg.K, cfg.w_std, SEED_W + so)
    bias = make_bias(cfg.N, SEED_BIAS + so) if cfg.bias else None
    d = dict(X=X, W=W, perm=perm, bias=bias)
    if cfg.rmsnorm:
        d.update(gamma=make_norm_weight(cfg.K, SEED_NORM + so), eps=NORM_EPS)
    return d


def custom_config(M: int, N: int, K: int, k_o: int, group: int = 0, outlier_int8: bool = False,
                  bias: bool = True, outlier_mult: float = 30.0, student_t: bool = False,
                  w_std: float = 0.02, act_bits: int = 4, weight_bits: int = 4,
                  rmsnorm: bool = False) -> LayerConfig:
    return LayerConfig(f"custom_{M}x{N}x{K}_ko{k_o}_g{group}_{'i8' if outlier_int8 else 'f16'}"
                       f"_w{weight_bits}a{act_bits}{'_rms' if rmsnorm else ''}",
                       M=M, N=N, K=K, k_o=k_o, group=group, outlier_int8=outlier_int8,
                       outlier_mult=outlier_mult, student_t=student_t, w_std=w_std, bias=bias,
                       act_bits=act_bits, weight_bits=weight_bits, rmsnorm=rmsnorm)
