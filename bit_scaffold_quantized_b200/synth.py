"""Seeded synthetic inputs for the DF-SSM decode step.

This module only draws random numbers in a fixed, documented order and lays them
out in the shapes the decode step consumes.  It holds none of the method's
arithmetic (no packing, no quantisation, no norm, no projection), so both the
CUDA path and the CPU oracle can consume what it produces without sharing any
computation.

Value distributions follow the workload descriptions of the DF-SSM decode
benchmarks ("Density Field State Space Models", Section 4.3 and Table 1 for the
model shape; Appendix B for d_state = 128 at 1.3B):

  sign words        uniform uint32 (each sign bit Bernoulli 0.5)
  alpha (row scale) fp16 U(0.01, 0.05)
  A_q, B_q          int8 uniform on [-127, 127]
  sA, sB            fp16 constant 1e-3
  A_log             fp32 U(0, ln 16)
  dt_bias           fp32 N(0, 0.1)
  D                 fp32 N(1, 0.1)
  conv w, b         fp16 U(-0.5, 0.5)   (Conv1d default bound 1/sqrt(fan_in=4))
  norm weights      fp16 N(1, 0.1)
  embedding         fp16 N(0, 0.02)
  layer inputs      fp16 N(0, 1), carried as fp32 residual
  states            zero
  token ids         uniform on [0, vocab)
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np


@dataclass(frozen=True)
class Dims:
    """Shape of one Mamba-2 layer with DF-SSM projections."""
    batch: int
    d_model: int
    d_inner: int
    nheads: int
    headdim: int
    d_state: int
    ngroups: int = 1
    d_conv: int = 4
    rank: int = 0
    ssm_state_dtype: int = 0      # SSM state storage: 0 fp32, 1 fp16
    df_chunk_codec: int = 0       # prompt pass: density-field codec between scan chunks

    @property
    def in_rows(self) -> int:
        """in_proj output width for the [z | x | B | C | dt] split."""
        return 2 * self.d_inner + 2 * self.ngroups * self.d_state + self.nheads

    @property
    def conv_dim(self) -> int:
        return self.d_inner + 2 * self.ngroups * self.d_state

    def with_batch(self, batch: int) -> "Dims":
        return replace(self, batch=batch)


# Workloads, named by what they are.
LAYER_SMALL = Dims(batch=1, d_model=256, d_inner=512, nheads=8, headdim=64,
                   d_state=16, rank=8)
LAYER_1P3B = Dims(batch=1, d_model=2048, d_inner=4096, nheads=64, headdim=64,
                  d_state=128, rank=32)
VOCAB_1P3B = 50280
N_LAYER_1P3B = 48

WORKLOADS: Dict[str, dict] = {
    # one small layer, batch 1, 16 decode steps
    "layer_d256_b1_16steps": dict(dims=LAYER_SMALL, steps=16, seed=0),
    # one Mamba-2-1.3B-shaped layer, batch 1, 256 decode steps
    "layer_d2048_b1_256steps": dict(dims=LAYER_1P3B, steps=256, seed=1),
    # 48-layer 1.3B-shaped model, batch 1, greedy decode of 512 tokens from a 1-token prompt
    "model_48x2048_v50280_b1_greedy512": dict(dims=LAYER_1P3B, n_layer=N_LAYER_1P3B,
                                              vocab=VOCAB_1P3B, steps=512, seed=2),
    # same model at batch 16 and 64, 256 steps, random token ids
    "model_48x2048_v50280_b16_256steps": dict(dims=LAYER_1P3B.with_batch(16), n_layer=N_LAYER_1P3B,
                                              vocab=VOCAB_1P3B, steps=256, seed=3),
    "model_48x2048_v50280_b64_256steps": dict(dims=LAYER_1P3B.with_batch(64), n_layer=N_LAYER_1P3B,
                                              vocab=VOCAB_1P3B, steps=256, seed=3),
}

# Isolated projection sweep: (d_in, d_out) x rank x batch
PROJ_SWEEP_SHAPES = [(2048, 8512), (4096, 2048)]
PROJ_SWEEP_RANKS = [16, 32, 64]
PROJ_SWEEP_BATCHES = [1, 4, 16, 64, 256]
PROJ_SWEEP_SEED = 4


@dataclass
class ProjWeights:
    rows: int               # d_out
    cols: int               # d_in
    bits: np.ndarray        # uint32 [rows, cols // 32], bit j of word w <-> column 32w + j
    alpha: np.ndarray       # float16 [rows]
    A: Optional[np.ndarray]   # int8 [rank, cols]
    sA: Optional[np.ndarray]  # float16 [rank]
    B: Optional[np.ndarray]   # int8 [rows, rank]
    sB: Optional[np.ndarray]  # float16 [rows]

    @property
    def rank(self) -> int:
        return 0 if self.A is None else int(self.A.shape[0])


@dataclass
class LayerWeights:
    prenorm_w: np.ndarray   # float16 [d_model]
    inp: ProjWeights        # d_model -> in_rows
    conv_w: np.ndarray      # float16 [conv_dim, d_conv]; column d_conv-1 multiplies the newest input
    conv_b: np.ndarray      # float16 [conv_dim]
    dt_bias: np.ndarray     # float32 [nheads]
    A_log: np.ndarray       # float32 [nheads]
    D: np.ndarray           # float32 [nheads]
    gnorm_w: np.ndarray     # float16 [d_inner]
    out: ProjWeights        # d_inner -> d_model


@dataclass
class LayerState:
    conv: np.ndarray        # float32 [batch, d_conv-1, conv_dim], index 0 oldest
    ssm: np.ndarray         # float32 [batch, nheads, headdim, d_state]


@dataclass
class Model:
    dims: Dims
    vocab: int
    embed: np.ndarray       # float16 [vocab, d_model] (tied LM head)
    normf_w: np.ndarray     # float16 [d_model]
    layers: List[LayerWeights] = field(default_factory=list)


def _f16(a) -> np.ndarray:
    return np.asarray(a).astype(np.float16)


def gen_proj(rng: np.random.Generator, rows: int, cols: int, rank: int) -> ProjWeights:
    """Draw order: sign words, alpha, A_q, B_q (scales are constants)."""
    assert cols % 32 == 0
    bits = rng.integers(0, 2 ** 32, size=(rows, cols // 32), dtype=np.uint64).astype(np.uint32)
    alpha = _f16(rng.uniform(0.01, 0.05, size=rows))
    if rank > 0:
        A = rng.integers(-127, 128, size=(rank, cols), dtype=np.int16).astype(np.int8)
        B = rng.integers(-127, 128, size=(rows, rank), dtype=np.int16).astype(np.int8)
        sA = np.full(rank, 1e-3, dtype=np.float16)
        sB = np.full(rows, 1e-3, dtype=np.float16)
    else:
        A = B = sA = sB = None
    return ProjWeights(rows, cols, bits, alpha, A, sA, B, sB)


def gen_layer(rng: np.random.Generator, d: Dims) -> LayerWeights:
    """Draw order: prenorm_w, in_proj, conv_w, conv_b, dt_bias, A_log, D, gnorm_w, out_proj."""
    prenorm_w = _f16(rng.normal(1.0, 0.1, size=d.d_model))
    inp = gen_proj(rng, d.in_rows, d.d_model, d.rank)
    conv_w = _f16(rng.uniform(-0.5, 0.5, size=(d.conv_dim, d.d_conv)))
    conv_b = _f16(rng.uniform(-0.5, 0.5, size=d.conv_dim))
    dt_bias = rng.normal(0.0, 0.1, size=d.nheads).astype(np.float32)
    A_log = rng.uniform(0.0, np.log(16.0), size=d.nheads).astype(np.float32)
    D = rng.normal(1.0, 0.1, size=d.nheads).astype(np.float32)
    gnorm_w = _f16(rng.normal(1.0, 0.1, size=d.d_inner))
    out = gen_proj(rng, d.d_model, d.d_inner, d.rank)
    return LayerWeights(prenorm_w, inp, conv_w, conv_b, dt_bias, A_log, D, gnorm_w, out)


def zero_state(d: Dims) -> LayerState:
    return LayerState(
        conv=np.zeros((d.batch, d.d_conv - 1, d.conv_dim), dtype=np.float32),
        ssm=np.zeros((d.batch, d.nheads, d.headdim, d.d_state),
                     dtype=np.float16 if d.ssm_state_dtype == 1 else np.float32),
    )


def gen_layer_inputs(rng: np.random.Generator, d: Dims, steps: int) -> np.ndarray:
    """fp16 N(0,1) residual inputs, one [batch, d_model] slab per decode step, as fp32."""
    return _f16(rng.normal(0.0, 1.0, size=(steps, d.batch, d.d_model))).astype(np.float32)


def gen_model(rng: np.random.Generator, d: Dims, n_layer: int, vocab: int) -> Model:
    """Draw order: embedding, final norm weight, then layers 0..n_layer-1."""
    embed = _f16(rng.normal(0.0, 0.02, size=(vocab, d.d_model)))
    normf_w = _f16(rng.normal(1.0, 0.1, size=d.d_model))
    layers = [gen_layer(rng, d) for _ in range(n_layer)]
    return Model(d, vocab, embed, normf_w, layers)


def silent_model(rng: np.random.Generator, d: Dims, n_layer: int, vocab: int) -> Model:
    """gen_model with three changes: every layer's out_proj scales (alpha and, with a
    LoRA, sB) are zero; the embedding rows are signed permutations of one fp16 vector,
    so every row has exactly the same norm and two rows are parallel only if equal;
    the final-norm weight is the constant 1.5."""
    m = gen_model(rng, d, n_layer, vocab)
    u = _f16(rng.normal(0.0, 0.05, size=d.d_model))
    rows = rng.permuted(np.tile(u, (vocab, 1)), axis=1)
    signs = rng.integers(0, 2, size=(vocab, d.d_model), dtype=np.int8) * 2 - 1
    m.embed = (rows * signs.astype(np.float16)).astype(np.float16)
    m.normf_w = np.full(d.d_model, 1.5, dtype=np.float16)
    for lw in m.layers:
        lw.out.alpha[:] = 0
        if lw.out.sB is not None:
            lw.out.sB[:] = 0
    return m


def gen_tokens(rng: np.random.Generator, batch: int, vocab: int) -> np.ndarray:
    return rng.integers(0, vocab, size=batch, dtype=np.int64).astype(np.int32)


def layer_workload(name: str, steps: Optional[int] = None, batch: Optional[int] = None):
    """(dims, weights, state, inputs) for a single-layer workload."""
    w = WORKLOADS[name]
    d = w["dims"] if batch is None else w["dims"].with_batch(batch)
    rng = np.random.default_rng(w["seed"])
    lw = gen_layer(rng, d)
    xs = gen_layer_inputs(rng, d, w["steps"] if steps is None else steps)
    return d, lw, zero_state(d), xs


def model_workload(name: str, n_layer: Optional[int] = None):
    """(model, prompt tokens) for a model workload."""
    w = WORKLOADS[name]
    d = w["dims"]
    rng = np.random.default_rng(w["seed"])
    m = gen_model(rng, d, w["n_layer"] if n_layer is None else n_layer, w["vocab"])
    tok = gen_tokens(rng, d.batch, w["vocab"])
    return m, tok


def proj_workload(d_in: int, d_out: int, rank: int, batch: int, seed: int = PROJ_SWEEP_SEED):
    """(weights, fp16 activations [batch, d_in]) for one projection sweep point."""
    rng = np.random.default_rng([seed, d_in, d_out, rank, batch])
    p = gen_proj(rng, d_out, d_in, rank)
    x = _f16(rng.normal(0.0, 1.0, size=(batch, d_in)))
    return p, x
