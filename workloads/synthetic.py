"""Seeded synthetic workloads for the ConvRot W8A8 / W4A8 linear.

The shapes are those of the decoder projections that the model cards quantise
("MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)", file table,
"Quantized" row: attention, gated-DeltaNet projections, MLP; and
"Qwen3-VL-8B-Heretic-1.3.0 - INT8 ConvRot", "Precision layout": q/k/v/o and
gate/up/down).  No trained weights or calibration text are available, so the
values are drawn from seeded distributions:

* activations: N(0,1) (or 0.5 * Student-t with 3 degrees of freedom) with a
  seeded set of outlier channels multiplied by a constant factor, which is the
  activation-outlier structure that the "Why ConvRot" section of
  "Qwen3.5 INT8 ConvRot Text Encoders for ComfyUI" says the rotation suppresses;
* weights: N(0, 0.02^2);
* RMSNorm weights: N(0, 0.1^2) (the norm multiplies by 1 + w).

Seeds: 0 for activations, 1 for weights, 2 for the outlier-channel choice,
3 for the norm weight.  A layer index offsets the weight seed so that every
layer of a multi-layer workload gets its own weights.

Every generator returns a torch tensor (bf16 unless stated) on the requested
device.  The CPU path uses ``torch.Generator`` so that the oracle and the GPU
path see identical bits; large bench workloads may be drawn on the GPU with a
CUDA generator instead (same seeds, different stream of numbers).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import torch

SEED_X = 0
SEED_W = 1
SEED_OUTLIER = 2
SEED_NORM = 3


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_channels(K: int, count: int, seed: int = SEED_OUTLIER) -> torch.Tensor:
    """Indices of ``count`` distinct outlier channels out of K (CPU, int64)."""
    if count <= 0:
        return torch.zeros(0, dtype=torch.int64)
    perm = torch.randperm(K, generator=_gen(seed, "cpu"))
    return perm[:count].sort().values


def activations(M: int, K: int, *, dist: str = "normal", outlier_count: int = 0,
                outlier_scale: float = 20.0, seed: int = SEED_X,
                outlier_seed: int = SEED_OUTLIER, device="cpu",
                dtype=torch.bfloat16) -> torch.Tensor:
    """Token activations x [M, K].

    dist = "normal": N(0,1).  dist = "student_t3": 0.5 * t with 3 degrees of
    freedom, drawn as z / sqrt((z1^2 + z2^2 + z3^2) / 3) from four normals.
    The chosen outlier channels are multiplied by ``outlier_scale``; the value
    is drawn and scaled in fp32 and rounded once to ``dtype``.
    """
    g = _gen(seed, device)
    if dist == "normal":
        x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    elif dist == "student_t3":
        z = torch.randn(4, M, K, generator=g, device=device, dtype=torch.float32)
        chi2 = (z[1] * z[1] + z[2] * z[2] + z[3] * z[3]) / 3.0
        x = 0.5 * z[0] / torch.sqrt(chi2.clamp_min(1e-12))
    else:
        raise ValueError(f"unknown activation distribution {dist!r}")
    if outlier_count > 0:
        ch = outlier_channels(K, outlier_count, outlier_seed).to(device)
        x[:, ch] *= outlier_scale
    return x.to(dtype)


def weight(N: int, K: int, *, std: float = 0.02, seed: int = SEED_W, layer: int = 0,
           device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """nn.Linear weight W [N, K] (out, in) ~ N(0, std^2)."""
    g = _gen(seed + 1000 * layer, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std
    return w.to(dtype)


def norm_weight(K: int, *, std: float = 0.1, seed: int = SEED_NORM, device="cpu") -> torch.Tensor:
    """RMSNorm weight w [K] in fp32 (the norm applies 1 + w)."""
    g = _gen(seed, device)
    return torch.randn(K, generator=g, device=device, dtype=torch.float32) * std


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    N: int   # out features
    K: int   # in features


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: a set of linears applied to M tokens."""
    name: str
    M: int
    linears: Tuple[Linear, ...]
    dist: str = "normal"
    outlier_frac: float = 0.0
    outlier_count: int = 0
    outlier_scale: float = 20.0
    norm: bool = False          # RMSNorm with folded SmoothQuant scale before the linear
    weight_bits: int = 8        # 8 = int8 codes, 4 = packed signed 4-bit codes
    layers: int = 1
    # MLP block down(SiLU(gate(x)) * up(x)): linears[0] is the fused gate/up
    # projection (N = 2 I rows, gate and up interleaved), linears[1] down_proj,
    # whose input is the block's intermediate H instead of fresh activations
    mlp: bool = False
    # weight-only path: rotated bf16 activations (no quantisation) and the bf16
    # tensor-core GEMM over the int8 weight codes
    weight_only: bool = False

    def n_outliers(self, K: int) -> int:
        if self.outlier_count:
            return self.outlier_count
        return int(round(self.outlier_frac * K))

    def ops(self) -> int:
        """Integer multiply-add work, counted as 2 ops per multiply-accumulate."""
        return self.layers * sum(2 * self.M * l.N * l.K for l in self.linears)

    def weight_bytes(self) -> int:
        per = 1 if self.weight_bits == 8 else 0.5
        return int(self.layers * sum(l.N * l.K * per for l in self.linears))


_DECODER = (
    Linear("q_proj", 4096, 4096),
    Linear("k_proj", 1024, 4096),
    Linear("v_proj", 1024, 4096),
    Linear("o_proj", 4096, 4096),
    Linear("gate_proj", 12288, 4096),
    Linear("up_proj", 12288, 4096),
    Linear("down_proj", 4096, 12288),
)

WORKLOADS = {
    # one small linear: two Hadamard groups, four outlier channels x20
    "single_linear_m32": Workload("single_linear_m32", 32, (Linear("linear", 256, 512),),
                                  outlier_count=4, outlier_scale=20.0),
    # down-proj shaped linear behind an RMSNorm with folded SmoothQuant scales
    "down_proj_m512": Workload("down_proj_m512", 512, (Linear("down_proj", 4096, 12288),),
                               dist="student_t3", outlier_frac=0.01, outlier_scale=30.0,
                               norm=True),
    # the seven projections of one decoder layer (hidden 4096, intermediate 12288)
    "decoder_layer_m2048": Workload("decoder_layer_m2048", 2048, _DECODER,
                                    outlier_frac=0.005, outlier_scale=20.0),
    # fused gate+up token sweep
    **{f"gate_up_m{m}": Workload(f"gate_up_m{m}", m, (Linear("gate_up", 24576, 4096),),
                                 outlier_frac=0.01, outlier_scale=20.0)
       for m in (1, 16, 128, 1024, 8192)},
    # fused projection sets: q/k/v of the decoder layer as one GEMM behind the
    # input RMSNorm (N = 4096 + 1024 + 1024), and a gated-DeltaNet-style input
    # projection with its small-N companion (N = 12288 + 64; illustrative
    # widths, the cards give none)
    "attn_qkv_m2048": Workload("attn_qkv_m2048", 2048, (Linear("qkv_proj", 6144, 4096),),
                               outlier_frac=0.005, outlier_scale=20.0, norm=True),
    "gdn_in_proj_m2048": Workload("gdn_in_proj_m2048", 2048, (Linear("in_proj_qkvz_ba", 12352, 4096),),
                                  outlier_frac=0.005, outlier_scale=20.0, norm=True),
    # weight-only path on the fused gate/up shape: decode (weight-stream bound,
    # int8 weights are half the bytes of bf16) and prefill (bf16 tensor rate)
    **{f"weight_only_gate_up_m{m}": Workload(f"weight_only_gate_up_m{m}", m,
                                             (Linear("gate_up", 24576, 4096),),
                                             outlier_frac=0.01, outlier_scale=20.0, weight_only=True)
       for m in (16, 2048)},
    # the decoder layer's MLP block as one chain: RMSNorm + rotate-quantise,
    # gate/up GEMM with the SiLU(gate) * up epilogue, rotate-quantise of H,
    # down_proj; SmoothQuant folded into the norm and into up_proj's rows
    "mlp_block_m2048": Workload("mlp_block_m2048", 2048,
                                (Linear("gate_up", 24576, 4096), Linear("down_proj", 4096, 12288)),
                                outlier_frac=0.005, outlier_scale=20.0, norm=True, mlp=True),
    # int4-weight variant over 36 decoder layers
    "w4a8_36_layers_m4096": Workload("w4a8_36_layers_m4096", 4096, _DECODER,
                                     outlier_frac=0.01, outlier_scale=20.0,
                                     weight_bits=4, layers=36),
}


def mlp_weights(w: Workload, device="cpu"):
    """(Wg [I, H], Wu [I, H], Wd [H, I]) bf16 of an MLP-block workload, seeds
    SEED_W, SEED_W + 1 and SEED_W + 2."""
    gu, down = w.linears
    I, H = gu.N // 2, gu.K
    return (weight(I, H, seed=SEED_W, device=device), weight(I, H, seed=SEED_W + 1, device=device),
            weight(H, I, seed=SEED_W + 2, device=device))


def workload_inputs(w: Workload, lin: Linear, *, M: Optional[int] = None, layer: int = 0,
                    device="cpu"):
    """(x [M,K] bf16, W [N,K] bf16, norm weight [K] fp32 or None) for one linear."""
    m = w.M if M is None else M
    x = activations(m, lin.K, dist=w.dist, outlier_count=w.n_outliers(lin.K),
                    outlier_scale=w.outlier_scale, device=device)
    W = weight(lin.N, lin.K, layer=layer, device=device)
    nw = norm_weight(lin.K, device=device) if w.norm else None
    return x, W, nw
