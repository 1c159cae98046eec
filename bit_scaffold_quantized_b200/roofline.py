"""Algorithmic byte model of the DF-SSM decode step (host logic, no GPU).

Bytes a decode step must move at minimum: every weight read once, every state
element read once and written once, plus the step's inputs and outputs.  The
component sizes follow the model-size breakdown of "Density Field State Space
Models" (Section 3.3, Table 1): scaffold 1 bit per weight, LoRA int8, the rest
fp16/fp32.  Per-row scaffold scales (fp16) and per-row LoRA scales are counted
too.  These are the numerators of the roofline fractions the benchmark reports.
"""
from __future__ import annotations

from .synth import Dims


def proj_weight_bytes(rows: int, cols: int, rank: int) -> int:
    bits = rows * cols // 8
    alpha = 2 * rows
    lora = rank * cols + rows * rank + 2 * rank + 2 * rows if rank > 0 else 0
    return bits + alpha + lora


def layer_weight_bytes(d: Dims) -> int:
    C = d.conv_dim
    other = (2 * d.d_model            # pre-norm weight fp16
             + 2 * C * d.d_conv + 2 * C  # conv weight + bias fp16
             + 3 * 4 * d.nheads       # dt_bias, A_log, D fp32
             + 2 * d.d_inner)         # gated-norm weight fp16
    return (proj_weight_bytes(d.in_rows, d.d_model, d.rank)
            + proj_weight_bytes(d.d_model, d.d_inner, d.rank) + other)


def layer_state_bytes(d: Dims) -> int:
    """fp32 conv state + SSM state (fp32, or fp16 when d.ssm_state_dtype == 1) of all
    batch rows, read once and written once."""
    ssm_es = 2 if getattr(d, "ssm_state_dtype", 0) == 1 else 4
    per_row = 4 * (d.d_conv - 1) * d.conv_dim + ssm_es * d.nheads * d.headdim * d.d_state
    return 2 * d.batch * per_row


def layer_step_bytes(d: Dims) -> int:
    """One layer step: weights + state r/w + fp32 residual in and out."""
    return layer_weight_bytes(d) + layer_state_bytes(d) + 2 * 4 * d.batch * d.d_model


def model_token_bytes(d: Dims, n_layer: int, vocab: int, head: str = "fp16") -> int:
    """One greedy token for all batch rows: embedding rows, all layers, final norm,
    tied LM head (fp16, or int8 codes + an fp32 scale per row), token ids in and out."""
    if head == "int8":
        emb_row, head_bytes = d.d_model + 4, vocab * (d.d_model + 4)
    else:
        emb_row, head_bytes = 2 * d.d_model, 2 * vocab * d.d_model
    return (d.batch * emb_row
            + n_layer * (layer_weight_bytes(d) + layer_state_bytes(d))
            + 2 * d.d_model
            + head_bytes
            + 2 * 4 * d.batch)


def proj_bytes(rows: int, cols: int, rank: int, batch: int) -> int:
    """Isolated projection: weights once, fp16 activations in, fp32 outputs out."""
    return proj_weight_bytes(rows, cols, rank) + 2 * batch * cols + 4 * batch * rows


def proj_flops(rows: int, cols: int, rank: int, batch: int) -> int:
    """Multiply-adds x2 of scaffold plus both LoRA stages."""
    return 2 * batch * (rows * cols + rank * cols + rows * rank)
