"""Seeded synthetic inputs for the quantized linear layer.

This module holds no arithmetic of the method: it only draws random tensors
(activations with outlier channels, weights, bias, the per-layer bit mask of
the block chain) and rounds them to bf16.  Both the CUDA path and the CPU
oracle consume exactly these bf16 bytes.

The shapes stand in for the video diffusion transformers the pages study
(HunyuanVideo-13B and Wan2.1-14B linears, QuantSparse "Resumen técnico" §1 and
§4; DVD-Quant §4): trained weights and real activations are not available, so
activations are N(0, 1) with a few channels scaled up as outliers (the
extreme values the Hadamard rotation spreads, DVD-Quant §2.B), weights are
N(0, sigma_w) and bias N(0, 0.01).

Draw order for one layer (a single CPU ``torch.Generator`` seeded once):
  1. activations float32 randn(M, K);
  2. outlier channels: the first round(p*K) entries of randperm(K), those
     columns multiplied by the outlier factor;
  3. weights randn(N, K) * sigma_w;
  4. bias randn(N) * 0.01.
For the block chain the 4-entry layer mask rand(4) < 0.25 (True = 8-bit) is
drawn first; then qkv, out and up draw steps 1-4 in turn, and down draws only
steps 3-4 (its input is GELU of the up output).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    seed: int
    bits: int
    M: int
    K: int
    N: int
    outlier_frac: float
    outlier_factor: float
    sigma_w: float
    alpha: float
    bits_x: int = 0  # activation code width; 0 = the same as `bits` (the weights')

    @property
    def act_bits(self) -> int:
        return self.bits_x or self.bits

    @property
    def n_outliers(self) -> int:
        return int(round(self.outlier_frac * self.K))

    @property
    def ops(self) -> int:
        """Integer multiply-adds counted as 2 ops: 2*M*N*K."""
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class ChainConfig:
    name: str
    seed: int
    M: int
    layers: tuple = field(default_factory=tuple)  # (name, K, N)
    outlier_frac: float = 0.01
    outlier_factor: float = 50.0
    sigma_w: float = 0.02
    alpha: float = 1.0
    p8: float = 0.25


TINY = LayerConfig("w4a4_tiny_M256_K512_N512", 0, 4, 256, 512, 512, 0.01, 20.0, 0.02, 1.0)
HY_QKV = LayerConfig("w4a4_hunyuan_qkv_M8192_K3072_N9216", 1, 4, 8192, 3072, 9216, 0.01, 50.0, 0.02, 1.0)
WAN_FFN = LayerConfig("w4a4_wan14b_ffn_up_M32760_K5120_N13824", 2, 4, 32760, 5120, 13824, 0.005, 100.0, 0.015, 0.9)
WAN_FFN_W8 = LayerConfig("w8a8_wan14b_ffn_up_M32760_K5120_N13824", 3, 8, 32760, 5120, 13824, 0.005, 100.0, 0.015, 1.0)
WAN_CHAIN = ChainConfig(
    "wan14b_block_chain_M32760", 4, 32760,
    (("qkv", 5120, 15360), ("out", 5120, 5120), ("ffn_up", 5120, 13824), ("ffn_down", 13824, 5120)),
)

# Mixed widths at the same FFN shape: QuantSparse's W4A8 and DVD-Quant's W4A6
# (both "Resumen técnico" §4).
WAN_FFN_W4A8 = LayerConfig("w4a8_wan14b_ffn_up_M32760_K5120_N13824", 5, 4, 32760, 5120, 13824, 0.005, 100.0, 0.015, 1.0, 8)
WAN_FFN_W4A6 = LayerConfig("w4a6_wan14b_ffn_up_M32760_K5120_N13824", 6, 4, 32760, 5120, 13824, 0.005, 100.0, 0.015, 0.9, 6)

LAYER_CONFIGS = (TINY, HY_QKV, WAN_FFN, WAN_FFN_W8)
MIXED_CONFIGS = (WAN_FFN_W4A8, WAN_FFN_W4A6)


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def _activations(g: torch.Generator, M: int, K: int, frac: float, factor: float) -> torch.Tensor:
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    n_out = int(round(frac * K))
    cols = torch.randperm(K, generator=g)[:n_out]
    if n_out:
        x[:, cols] *= factor
    return x


def make_layer(cfg: LayerConfig, M: int | None = None) -> dict:
    """bf16 CPU tensors x [M,K], w [N,K], bias [N] for one layer config.

    ``M`` overrides the token count (the draw order is unchanged, so the
    weights and bias do not depend on it).
    """
    M = cfg.M if M is None else M
    g = torch.Generator(device="cpu").manual_seed(cfg.seed)
    x = _activations(g, M, cfg.K, cfg.outlier_frac, cfg.outlier_factor)
    w = torch.randn(cfg.N, cfg.K, generator=g, dtype=torch.float32) * cfg.sigma_w
    b = torch.randn(cfg.N, generator=g, dtype=torch.float32) * 0.01
    return {"x": _bf16(x), "w": _bf16(w), "bias": _bf16(b), "bits": cfg.bits, "alpha": cfg.alpha}


def make_shape(seed: int, M: int, K: int, N: int, bits: int, alpha: float = 1.0,
               outlier_frac: float = 0.01, outlier_factor: float = 20.0,
               sigma_w: float = 0.02, bits_x: int = 0) -> dict:
    """Same recipe at an arbitrary shape (parity cases and edge shapes)."""
    cfg = LayerConfig("custom", seed, bits, M, K, N, outlier_frac, outlier_factor, sigma_w, alpha,
                      bits_x)
    return make_layer(cfg)


def make_chain(cfg: ChainConfig = WAN_CHAIN, M: int | None = None) -> dict:
    """Per-layer bits mask and bf16 tensors of the block chain.

    Returns {"bits": [4|8]*4, "layers": [{name, K, N, x (None for down), w, bias}]}.
    """
    M = cfg.M if M is None else M
    g = torch.Generator(device="cpu").manual_seed(cfg.seed)
    mask = torch.rand(4, generator=g) < cfg.p8
    bits = [8 if bool(m) else 4 for m in mask]
    layers = []
    for i, (name, K, N) in enumerate(cfg.layers):
        if i < 3:
            x = _bf16(_activations(g, M, K, cfg.outlier_frac, cfg.outlier_factor))
        else:
            x = None
        w = _bf16(torch.randn(N, K, generator=g, dtype=torch.float32) * cfg.sigma_w)
        b = _bf16(torch.randn(N, generator=g, dtype=torch.float32) * 0.01)
        layers.append({"name": name, "K": K, "N": N, "x": x, "w": w, "bias": b, "bits": bits[i]})
    return {"bits": bits, "layers": layers, "alpha": cfg.alpha}


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 CPU tensor (what the oracle consumes)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


SALIENT_FRACTION = 1 / 16


def salient_rows(M: int, seed: int, frac: float = SALIENT_FRACTION) -> list[int]:
    """Stand-in for the salient tokens of SemanticDialect's activation
    decomposition (chosen there from attention scores of a trained model):
    round(frac * M) distinct rows drawn by a generator of their own (seed +
    7919, so the layer's tensors are unchanged), in increasing order."""
    g = torch.Generator(device="cpu").manual_seed(seed + 7919)
    n = max(1, round(frac * M))
    return sorted(torch.randperm(M, generator=g)[:n].tolist())
