"""Seeded synthetic inputs shaped like the pages' models.

This module only draws random numbers: it holds none of the method's
arithmetic (no quantiser, no packing, no dot product), so both the CUDA path
and the oracle may use it.

Generator: numpy ``default_rng(seed)`` (PCG64), ``standard_normal`` in fp64,
scaled, then cast to fp32.  Outliers: after the normals, the same generator
draws ``random(shape)``; entries below ``p`` are multiplied by ``factor``.
bf16 activations are the fp32 draw rounded to nearest-even by torch.

Seeds: ``1000*config + 10*matrix + {0: weights, 1: activations}``, except the
single ternary linear, which uses seed 0 for its weights and 1 for its
activations.

Workloads (page and section the shapes come from):

* ``single_ternary`` -- one 192->768 ternary linear, M=256, fp32 out
  ("Extreme DQT with an FP4 Optimizer", Model Overview: d=192, d_ff=768).
* ``atomic_stack`` -- 6 layers of QKV 256->768, O 256->256, FFN 256->1024->256
  plus a 256->4096 head, ternary, M in {1, 256}, bf16 out ("Atomic-1Bit"
  README, Quick Start config: 256d, 6 layers, 4 heads, vocab 4096).
* ``impeto_binary`` -- 8 layers of Q 192->192, K 192->96, V 192->96,
  O 192->192, gate 192->768, up 192->768, down 768->192 plus a 192->2048 head,
  binary, M=16384, fp32 out ("Extreme DQT with an FP4 Optimizer", Model
  Overview and DDReGLU).
* ``t4nt_int4`` -- 1280->3584 and 3584->1280, 4-bit, M in {1, 8, 256, 8192},
  bf16 out ("T4NT-0.5B" model card, Architecture table).
* ``ternary_4b`` -- 2560->9728 and 9728->2560, ternary, bf16 activations with
  0.5% x10 outliers, M in {1, 16, 128, 1024, 8192}, bf16 out (4B-class
  ternary shapes from the "Low-Precision Formats" topic list).

Workloads of the prologue and binary variants (same page sources for the
shapes; "M8.8 - Native Binary and Ternary Transformers" for the variants):

* ``ternary_4b_rmsnorm`` -- ``ternary_4b`` behind an RMSNorm with a gain
  vector (0x02E, 0x03; b1.58 and T4NT use RMSNorm).
* ``bitnet_v1_binary`` -- the Impeto stack shapes with BitNet v1 centred
  binary codes and one scale per tensor (0x02B, 0x02E).
* ``onebit_4096`` -- 4096->4096 sign codes with OneBit's input and output
  value vectors (0x06A; d = 4096 is the page's ledger example of 0x06C),
  M in {1, 16, 4096}.
* ``h_bitlinear_4b`` -- the 4B-class FFN down projection 9728->2560 and an
  attention output 2560->2560 as H-BitLinear (0x07C): RMSNorm with gain, then
  a Hadamard rotation in blocks of 512 before the codes, M in {1, 16, 1024,
  8192}.

Gain vectors are 1 + 0.1 N(0,1); OneBit value vectors are exp(0.3 N(0,1))
(input side) and 0.02 exp(0.3 N(0,1)) (output side), all fp32.  Their seeds
add 2 (gain or input vector) and 3 (output vector) to the matrix's weight
seed.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

TERNARY2, BINARY1, INT4 = 0, 1, 2
F32, BF16 = 0, 1


@dataclass(frozen=True)
class Matrix:
    name: str
    K: int  # input features
    N: int  # output features


@dataclass(frozen=True)
class Workload:
    name: str
    index: int  # position in the table below, used in seeds
    fmt: int
    matrices: tuple
    Ms: tuple
    x_dtype: int
    y_dtype: int
    w_std: float = 0.02
    outlier_p: float = 0.01
    outlier_factor: float = 8.0
    notes: str = ""
    extra: dict = field(default_factory=dict)
    # activation prologue: RMSNorm (with a gain vector), Hadamard block size
    norm: bool = False
    hadamard: int = 0
    # weight quantiser variant: "default", "centred" (BitNet v1) or "onebit"
    # (sign codes with value vectors)
    quantizer: str = "default"


def _atomic_stack():
    mats = []
    for layer in range(6):
        mats += [Matrix(f"L{layer}.qkv", 256, 768), Matrix(f"L{layer}.o", 256, 256),
                 Matrix(f"L{layer}.ffn_up", 256, 1024), Matrix(f"L{layer}.ffn_down", 1024, 256)]
    mats.append(Matrix("head", 256, 4096))
    return tuple(mats)


def _impeto_binary():
    mats = []
    for layer in range(8):
        mats += [Matrix(f"L{layer}.q", 192, 192), Matrix(f"L{layer}.k", 192, 96),
                 Matrix(f"L{layer}.v", 192, 96), Matrix(f"L{layer}.o", 192, 192),
                 Matrix(f"L{layer}.gate", 192, 768), Matrix(f"L{layer}.up", 192, 768),
                 Matrix(f"L{layer}.down", 768, 192)]
    mats.append(Matrix("head", 192, 2048))
    return tuple(mats)


WORKLOADS = {
    "single_ternary": Workload("single_ternary", 1, TERNARY2, (Matrix("ffn_up", 192, 768),),
                               (256,), F32, F32),
    "atomic_stack": Workload("atomic_stack", 2, TERNARY2, _atomic_stack(), (1, 256), F32, BF16),
    "impeto_binary": Workload("impeto_binary", 3, BINARY1, _impeto_binary(), (16384,), F32, F32),
    "t4nt_int4": Workload("t4nt_int4", 4, INT4,
                          (Matrix("ffn_up", 1280, 3584), Matrix("ffn_down", 3584, 1280)),
                          (1, 8, 256, 8192), F32, BF16),
    "ternary_4b": Workload("ternary_4b", 5, TERNARY2,
                           (Matrix("ffn_up", 2560, 9728), Matrix("ffn_down", 9728, 2560)),
                           (1, 16, 128, 1024, 8192), BF16, BF16,
                           outlier_p=0.005, outlier_factor=10.0),
}


WORKLOADS.update({
    "ternary_4b_rmsnorm": Workload("ternary_4b_rmsnorm", 6, TERNARY2,
                                   (Matrix("ffn_up", 2560, 9728), Matrix("ffn_down", 9728, 2560)),
                                   (1, 16, 128, 1024, 8192), BF16, BF16, outlier_p=0.005, outlier_factor=10.0,
                                   norm=True),
    "bitnet_v1_binary": Workload("bitnet_v1_binary", 7, BINARY1, _impeto_binary(), (16384,), F32, F32,
                                 quantizer="centred"),
    "onebit_4096": Workload("onebit_4096", 8, BINARY1, (Matrix("proj", 4096, 4096),), (1, 16, 4096), F32, BF16,
                            quantizer="onebit"),
    "h_bitlinear_4b": Workload("h_bitlinear_4b", 9, TERNARY2,
                               (Matrix("ffn_down", 9728, 2560), Matrix("attn_out", 2560, 2560)),
                               (1, 16, 1024, 8192), BF16, BF16, outlier_p=0.005, outlier_factor=10.0,
                               norm=True, hadamard=512),
})


def weight_seed(wl: Workload, matrix_index: int) -> int:
    if wl.index == 1:
        return 0
    return 1000 * wl.index + 10 * matrix_index


def act_seed(wl: Workload, matrix_index: int) -> int:
    if wl.index == 1:
        return 1
    return 1000 * wl.index + 10 * matrix_index + 1


def normal_weights(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """fp32 [N, K] weights drawn N(0, std)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, K)) * std).astype(np.float32)


def normal_activations(seed: int, M: int, K: int, outlier_p: float = 0.01,
                       outlier_factor: float = 8.0) -> np.ndarray:
    """fp32 [M, K] activations N(0, 1) with a fraction ``outlier_p`` scaled
    by ``outlier_factor``."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    if outlier_p > 0:
        mask = rng.random((M, K)) < outlier_p
        x = np.where(mask, x * outlier_factor, x)
    return x.astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), nearest-even, via torch."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def workload_weights(wl: Workload, matrix_index: int) -> np.ndarray:
    m = wl.matrices[matrix_index]
    return normal_weights(weight_seed(wl, matrix_index), m.N, m.K, wl.w_std)


def workload_activations(wl: Workload, matrix_index: int, M: int):
    """Activations for one matrix at M tokens: fp32 array, or uint16 bf16 bits
    when the workload's activations are bf16."""
    m = wl.matrices[matrix_index]
    x = normal_activations(act_seed(wl, matrix_index), M, m.K, wl.outlier_p, wl.outlier_factor)
    if wl.x_dtype == BF16:
        return to_bf16_bits(x)
    return x


def gain_vector(seed: int, K: int) -> np.ndarray:
    """fp32 [K] gains 1 + 0.1 N(0,1) (an RMSNorm gain)."""
    rng = np.random.default_rng(seed)
    return (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)


def value_vector(seed: int, n: int, scale: float) -> np.ndarray:
    """fp32 [n] positive values scale * exp(0.3 N(0,1)) (a OneBit value vector)."""
    rng = np.random.default_rng(seed)
    return (scale * np.exp(0.3 * rng.standard_normal(n))).astype(np.float32)


def workload_gain(wl: Workload, matrix_index: int):
    """The activation-side vector of a matrix: the RMSNorm gain, OneBit's
    input value vector, or None."""
    m = wl.matrices[matrix_index]
    if wl.quantizer == "onebit":
        return value_vector(weight_seed(wl, matrix_index) + 2, m.K, 1.0)
    if wl.norm:
        return gain_vector(weight_seed(wl, matrix_index) + 2, m.K)
    return None


def workload_output_vector(wl: Workload, matrix_index: int):
    """OneBit's output value vector of a matrix (its per-row weight scale), or None."""
    if wl.quantizer != "onebit":
        return None
    return value_vector(weight_seed(wl, matrix_index) + 3, wl.matrices[matrix_index].N, 0.02)
