"""CPU oracle for the DF-SSM decode step -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy restatement of what one DF-SSM Mamba-2
decode step computes.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does.  It shares no code with the CUDA library and imports nothing from it.

Arithmetic is fp64 except where the method fixes a storage format or where a
floating-point value decides an integer:
  * activations entering a projection are stored as fp16;
  * SSM state, conv state, the residual stream and the gated value y*silu(z)
    are stored as fp32 (the SSM state in fp16 when the given state array is fp16:
    the fp64 update rounded once);
  * the int8 activation quantiser takes its decision in fp32 (scale = amax/127
    as an IEEE fp32 divide, code = round-half-even of x/scale in fp32), the
    precision the kernel uses, so both sides take the same integer decision;
  * the low-rank stage-1 product A_q . x_q is exact integer arithmetic.

Sources ("Density Field State Space Models", C. Shinde):
  Eq. 3 (Section 3.2)   y = W_scaffold x + W_A (W_B x): frozen scaffold plus low-rank correction
  Section 3.3           LoRA matrices int8 with per-channel scales
  Table 1               scaffold stored 1-bit packed
  Section 4.1           bits expanded on the fly; conv step is a stateful shift register;
                        SSM step is a stateful recurrence; preallocated persistent state
  Appendix B, Table 12  h = A h + (x dt) (x) B; d_state = 128 at 1.3B; norm(y * silu(z))
  Section 2, Appendix B the chunked (SSD) form of the scan over a prompt, block_len 64:
                        the prompt pass (conv_seq, ssd_scan, layer_prefill, model_prefill)
  Section 3.4, App. D   the density-field state representation (df_field_size, df_encode,
                        df_decode, df_roundtrip) and its use at chunk boundaries (DF-SSD)
Where the pages are silent (the [z|x|B|C|dt] split, softplus, eps, conv tap order,
activation quantiser, the per-row scaffold scale alpha) the standard Mamba-2
block and the decode-step description this package implements fix the reading;
every such reading is listed in the design notes.

Parity pins: every function here is checked by tests/test_oracle_pins.py
against brute force, closed forms, library routines and the pages' own numbers.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

EPS = 1e-5          # RMSNorm epsilon (pages silent; Mamba-2 default)
TILE_ROWS = 16      # tiled sign-word layout: 16 rows ...
TILE_COLS = 256     # ... by 256 columns per 512-byte tile


# --------------------------------------------------------------------------
# 1-bit scaffold storage (Table 1: "1-bit packed"; Section 4.1: expanded on the fly)
# --------------------------------------------------------------------------

def pack_signs(w: np.ndarray) -> np.ndarray:
    """Dense [rows, cols] -> uint32 [rows, cols/32]; bit j of word k is column 32k+j.

    bit = 1 encodes +1 and is taken where w >= 0 (so -0.0 packs to +1); any
    other value (negative, NaN) packs to 0, which encodes -1.
    """
    w = np.asarray(w)
    rows, cols = w.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    b = (w >= 0).astype(np.uint64).reshape(rows, cols // 32, 32)
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return (b * weights).sum(axis=-1).astype(np.uint32)


def unpack_signs(bits: np.ndarray, cols: int) -> np.ndarray:
    """uint32 [rows, cols/32] -> int8 [rows, cols] of +1 (bit set) / -1 (bit clear)."""
    bits = np.asarray(bits, dtype=np.uint32)
    rows = bits.shape[0]
    shifts = np.arange(32, dtype=np.uint32)
    b = ((bits[:, :, None] >> shifts) & np.uint32(1)).reshape(rows, cols)
    return (2 * b.astype(np.int8) - 1).astype(np.int8)


def tiled_bit_position(row, col, cols: int):
    """(word index, bit index) of weight (row, col) in the tiled sign-word layout.

    Works elementwise on integers or integer arrays.  The tiled layout is a
    bijective permutation of the row-major bits into 16-row x 256-column tiles of
    128 words (32 lanes x 4 words), built for m16n8k32 int8 tensor-core products.
    A tile's 256 columns are 8 products of 32 columns, s = 0..7.  Register q of the
    A fragment of product s, for every lane, is bits s, s + 8, s + 16, s + 24 of the
    lane's word q (byte i = bit s + 8 i).  A register is therefore one mask of word
    q, or a shift and a mask.  The columns of products 2m and 2m + 1 are interleaved
    so that lane t finds its B-fragment bytes for both at 16 consecutive columns,
    64 m + 16 t .. 64 m + 16 t + 15.
    Within a tile:
      r16 = row % 16, c = col % 256, m = c // 64, p = c % 64,
      t = p // 16, e = (p % 16) // 8, h = (p % 8) // 4, i = p % 4,
      lane = (r16 % 8) * 4 + t,  q = r16 // 8 + 2 * h,  s = 2 * m + e,
      bit = s + 8 * i,
      word = ((row // 16) * (cols // 256) + col // 256) * 128 + lane * 4 + q.
    For product s the fragment's column 4t + i (+16 when q >= 2) is therefore
    column 64 m + 16 t + 8 e + i (+4) of the tile.
    """
    row = np.asarray(row, dtype=np.int64)
    col = np.asarray(col, dtype=np.int64)
    r16 = row % TILE_ROWS
    c = col % TILE_COLS
    m = c // 64
    p = c % 64
    t = p // 16
    e = (p % 16) // 8
    h = (p % 8) // 4
    i = p % 4
    lane = (r16 % 8) * 4 + t
    q = r16 // 8 + 2 * h
    s = 2 * m + e
    bit = s + 8 * i
    word = ((row // TILE_ROWS) * (cols // TILE_COLS) + col // TILE_COLS) * 128 + lane * 4 + q
    return word, bit


def padded_rows(rows: int) -> int:
    return -(-rows // TILE_ROWS) * TILE_ROWS


def tile_signs(bits_rowmajor: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Row-major sign words -> tiled sign words (rows padded to 16 with clear bits)."""
    if cols % TILE_COLS:
        raise ValueError("cols must be a multiple of 256 for the tiled layout")
    s = unpack_signs(bits_rowmajor, cols)
    out = np.zeros(padded_rows(rows) * cols // 32, dtype=np.uint64)
    r_idx, c_idx = np.nonzero(s > 0)
    wd, bt = tiled_bit_position(r_idx, c_idx, cols)
    np.bitwise_or.at(out, wd, np.uint64(1) << bt.astype(np.uint64))
    return out.astype(np.uint32)


# --------------------------------------------------------------------------
# int8 low-rank correction (Eq. 3; Section 3.3 "int8 with per-channel scaling")
# --------------------------------------------------------------------------

def quantize_act(x16: np.ndarray):
    """Per-row symmetric int8 quantisation of fp16 activations, decided in fp32.

    amax = max|x| (exact in fp32); scale sx = amax / 127 (IEEE fp32 divide);
    code = clamp(round_half_even(x / sx), -127, 127) with x / sx an fp32 divide.
    A zero row gives codes 0 and sx = 1.  Returns (int8 codes, fp32 scales [rows]).
    """
    xf = np.asarray(x16, dtype=np.float16).astype(np.float32)
    amax = np.max(np.abs(xf), axis=-1)
    safe = np.where(amax > 0, amax, np.float32(127.0)).astype(np.float32)
    sx = (safe / np.float32(127.0)).astype(np.float32)
    q = np.rint((xf / sx[..., None]).astype(np.float32))
    q = np.clip(q, -127, 127)
    q = np.where(amax[..., None] > 0, q, 0)
    return q.astype(np.int8), sx


def lora_stage1(A: np.ndarray, xq: np.ndarray) -> np.ndarray:
    """acc[b, j] = sum_k A[j, k] * xq[b, k], exact in int64, checked to fit int32."""
    acc = xq.astype(np.int64) @ A.astype(np.int64).T
    if acc.size and (acc.max() >= 2 ** 31 or acc.min() < -(2 ** 31)):
        raise OverflowError("int8 x int8 partial exceeds int32")
    return acc


@dataclass
class ProjTrace:
    y: np.ndarray                       # fp64 [B, rows]
    xq: Optional[np.ndarray] = None     # int8 [B, cols]
    sx: Optional[np.ndarray] = None     # fp32 [B]
    acc: Optional[np.ndarray] = None    # int64 [B, rank]
    u: Optional[np.ndarray] = None      # fp64 [B, rank]


def project(x16: np.ndarray, p) -> ProjTrace:
    """One DF-SSM projection (Eq. 3 with the per-row scaffold scale alpha):

        y[o] = alpha[o] * sum_k s[o,k] x[k]  +  sB[o] * sum_j B_q[o,j] u[j],
        u[j] = acc[j] * sA[j] * sx,  acc = A_q . x_q.

    The LoRA multiplier of Eq. 3 is folded into the scales (taken as 1).
    """
    x = np.asarray(x16, dtype=np.float16).astype(np.float64)
    S = unpack_signs(p.bits, p.cols).astype(np.float64)
    y = p.alpha.astype(np.float64) * (x @ S.T)
    if p.A is None or p.A.shape[0] == 0:
        return ProjTrace(y=y)
    xq, sx = quantize_act(x16)
    acc = lora_stage1(p.A, xq)
    u = acc.astype(np.float64) * p.sA.astype(np.float64) * sx.astype(np.float64)[:, None]
    y = y + p.sB.astype(np.float64) * (u @ p.B.astype(np.float64).T)
    return ProjTrace(y=y, xq=xq, sx=sx, acc=acc, u=u)


# --------------------------------------------------------------------------
# Mamba-2 block pieces
# --------------------------------------------------------------------------

def rmsnorm(v: np.ndarray, w: np.ndarray, eps: float = EPS) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return v * r * np.asarray(w, dtype=np.float64)


def silu(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def softplus(v: np.ndarray) -> np.ndarray:
    """log(1 + e^v), returned as v itself above 20."""
    v = np.asarray(v, dtype=np.float64)
    return np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))


def conv_step(conv_state: np.ndarray, xBC: np.ndarray, w: np.ndarray, b: np.ndarray):
    """Causal depthwise conv1d step as a shift register (Section 4.1).

    conv_state [B, W-1, C] holds the previous W-1 inputs, oldest first; the window
    is [state..., xBC]; tap j multiplies window entry j (tap W-1 the newest input).
    Output silu(bias + sum_j w[:, j] * window[j]); the state shifts by one.
    Returns (xc fp64 [B, C], new state fp32).
    """
    cs = np.asarray(conv_state, dtype=np.float64)
    xBC = np.asarray(xBC, dtype=np.float64)
    win = np.concatenate([cs, xBC[:, None, :]], axis=1)           # [B, W, C]
    wt = np.asarray(w, dtype=np.float64).T                         # [W, C]
    pre = np.asarray(b, dtype=np.float64) + np.sum(wt[None] * win, axis=1)
    new_state = win[:, 1:, :].astype(np.float32)
    return silu(pre), new_state


def ssm_step(h: np.ndarray, x: np.ndarray, Bv: np.ndarray, Cv: np.ndarray,
             dt_raw: np.ndarray, dt_bias: np.ndarray, A_log: np.ndarray, D: np.ndarray,
             state_dtype=np.float32):
    """Selective-SSM state update for one token (Appendix B, corrected form).

    h [B, H, P, N], x [B, H, P], Bv/Cv [B, N] (one group), dt_raw [B, H].
      dt = softplus(dt_raw + dt_bias),  A = -exp(A_log),  dA = exp(dt * A)
      h' = dA * h + (x * dt) (outer) B
      y  = sum_n C[n] h'[.., n] + D * x
    Returns (y fp64 [B, H, P], h' rounded once from fp64 to the state's storage
    type: fp32, or fp16 for the half-precision state of the survey's next items).
    """
    h = np.asarray(h, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    dt = softplus(np.asarray(dt_raw, dtype=np.float64) + np.asarray(dt_bias, dtype=np.float64))
    A = -np.exp(np.asarray(A_log, dtype=np.float64))
    dA = np.exp(dt * A)                                            # [B, H]
    xdt = x * dt[:, :, None]                                       # [B, H, P]
    hn = dA[:, :, None, None] * h + xdt[:, :, :, None] * np.asarray(Bv, dtype=np.float64)[:, None, None, :]
    y = np.einsum("bhpn,bn->bhp", hn, np.asarray(Cv, dtype=np.float64))
    y = y + np.asarray(D, dtype=np.float64)[None, :, None] * x
    return y, hn.astype(state_dtype)


def gated_rmsnorm(y: np.ndarray, z: np.ndarray, w: np.ndarray, eps: float = EPS) -> np.ndarray:
    """norm(y * silu(z)) -- gate first, then RMSNorm over the whole d_inner (Appendix B)."""
    g = np.asarray(y, dtype=np.float64) * silu(z)
    return rmsnorm(g, w, eps)


def ssd_scan(h0: np.ndarray, x: np.ndarray, Bm: np.ndarray, Cm: np.ndarray, dt_raw: np.ndarray,
             dt_bias: np.ndarray, A_log: np.ndarray, D: np.ndarray, chunk: int = 64, df: bool = False):
    """Selective-SSM over a whole prompt of T tokens in the chunked (state space
    duality, "SSD") form of Mamba-2, which the pages name (Section 2) and use with
    block_len = 64 (Appendix B, DF-SSD).  One group.

    h0 [B, H, P, N] state before the prompt, x [B, T, H, P], Bm/Cm [B, T, N],
    dt_raw [B, T, H].  Per token dt = softplus(dt_raw + dt_bias), a = dt * A with
    A = -exp(A_log).  Within a chunk starting at c0, cs[t] = sum_{r=c0..t} a_r, so
    prod_{r=s+1..t} dA_r = exp(cs[t] - cs[s]):
      y_t = sum_{s=c0..t} (C_t . B_s) exp(cs[t] - cs[s]) dt_s x_s       (within the chunk)
          + exp(cs[t]) C_t . h_prev                                      (from the carried state)
          + D x_t,
      h_next = exp(cs[end]) h_prev + sum_s exp(cs[end] - cs[s]) dt_s x_s (outer) B_s.
    This is the recurrence h_t = dA_t h_{t-1} + (x_t dt_t) (outer) B_t, y_t = C_t . h_t
    + D x_t unrolled over a chunk, in fp64 throughout (no rounding of the state
    between tokens).  With df (DF-SSD, Section 3.4 / Appendix D) the state carried
    from one chunk to the next passes through the density-field encoding and readout
    (df_roundtrip); the state after the last chunk is returned as computed.
    Returns (y fp64 [B, T, H, P], final state fp64 [B, H, P, N])."""
    x = np.asarray(x, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    Cm = np.asarray(Cm, dtype=np.float64)
    dt = softplus(np.asarray(dt_raw, dtype=np.float64) + np.asarray(dt_bias, dtype=np.float64))
    A = -np.exp(np.asarray(A_log, dtype=np.float64))
    a = dt * A                                                      # [B, T, H]
    T = x.shape[1]
    h = np.asarray(h0, dtype=np.float64).copy()
    y = np.zeros(x.shape)
    for c0 in range(0, T, chunk):
        c1 = min(c0 + chunk, T)
        cs = np.cumsum(a[:, c0:c1], axis=1)                         # [B, L, H]
        L = c1 - c0
        # decay from s+1 to t, only where s <= t (the upper triangle would overflow exp)
        low = np.tril(np.ones((L, L), dtype=bool))[None, :, :, None]
        seg = np.exp(np.where(low, cs[:, :, None, :] - cs[:, None, :, :], -np.inf))   # [B, t, s, H]
        CB = np.einsum("btn,bsn->bts", Cm[:, c0:c1], Bm[:, c0:c1])   # [B, t, s]
        xdt = x[:, c0:c1] * dt[:, c0:c1, :, None]                   # [B, L, H, P]
        y[:, c0:c1] = np.einsum("bts,btsh,bshp->bthp", CB, seg, xdt)
        y[:, c0:c1] += np.exp(cs)[..., None] * np.einsum("btn,bhpn->bthp", Cm[:, c0:c1], h)
        tail = np.exp(cs[:, -1:, :] - cs)                           # [B, L, H]: decay from s+1 to the end
        h = np.exp(cs[:, -1, :])[:, :, None, None] * h + np.einsum("bsh,bshp,bsn->bhpn", tail, xdt, Bm[:, c0:c1])
        if df and c1 < T:
            h = df_roundtrip(h)
    y += np.asarray(D, dtype=np.float64)[None, None, :, None] * x
    return y, h


# --------------------------------------------------------------------------
# Density-field state representation (Section 3.4, Appendix D)
# --------------------------------------------------------------------------
# Reading of the pages (Section 3.4: a K x K binary field with K^2 ~ 4 d_state, mean
# +- 3 sigma normalisation to [0, 1], first-order sigma-delta with an 8-bit
# accumulator, threshold 0.5, popcount readout; Appendix D: K = 23 at d_state 128):
#   * one field per state row (the d_state values of one head row); K is the smallest
#     integer with K^2 >= 4 d_state, each value owns 4 consecutive cells (raster
#     order), the K^2 - 4 d_state spare cells stay 0;
#   * mu and sigma are the row's mean and population standard deviation (fp64 sums
#     left to right); the field keeps lo = mu - 3 sigma and span = 6 sigma as fp32;
#   * the 8-bit input of value i is q_i = rint(255 clip((h_i - lo) / span, 0, 1))
#     (q = 128 when span is 0);
#   * the sigma-delta error e (signed 8-bit, 0 at the row's first cell, carried from
#     value to value) gives cell = [e + q >= 128] (0.5 of full scale) and
#     e <- e + q - 255 cell;
#   * the readout is lo + span popcount / 4 over the value's cells (fp64).

DF_CELLS = 4     # cells per state value


def df_field_size(n: int) -> int:
    """K of the K x K field of a row of n state values: the least K with K^2 >= 4 n."""
    K = 1
    while K * K < DF_CELLS * n:
        K += 1
    return K


def df_encode(row: np.ndarray):
    """Encode one state row (n values).  Returns (cells uint8 [K*K], lo fp32, span fp32)."""
    h = np.asarray(row, dtype=np.float64)
    n = h.shape[0]
    total = 0.0
    for v in h:                       # left to right
        total = total + v
    mu = total / n
    ss = 0.0
    for v in h:
        d = v - mu
        ss = ss + d * d
    sigma = np.sqrt(ss / n)
    lo = np.float32(mu - 3.0 * sigma)
    span = np.float32(6.0 * sigma)
    K = df_field_size(n)
    cells = np.zeros(K * K, dtype=np.uint8)
    e = 0
    for i in range(n):
        if span == 0:
            q = 128
        else:
            t = (h[i] - np.float64(lo)) / np.float64(span)
            q = int(np.rint(255.0 * min(1.0, max(0.0, t))))
        for j in range(DF_CELLS):
            s_ = e + q
            bit = 1 if s_ >= 128 else 0
            e = s_ - 255 * bit
            cells[DF_CELLS * i + j] = bit
    return cells, lo, span


def df_decode(cells: np.ndarray, lo, span, n: int) -> np.ndarray:
    """Readout of a field: value i = lo + span * (ones among its cells) / 4 (fp64)."""
    c = np.asarray(cells, dtype=np.int64)[:DF_CELLS * n].reshape(n, DF_CELLS)
    d = c.sum(axis=1) / float(DF_CELLS)
    return np.float64(lo) + d * np.float64(span)


def df_roundtrip(h: np.ndarray) -> np.ndarray:
    """Encode and read out every row (last axis) of a state array; fp64 result."""
    h = np.asarray(h, dtype=np.float64)
    flat = h.reshape(-1, h.shape[-1])
    out = np.empty_like(flat)
    for r in range(flat.shape[0]):
        cells, lo, span = df_encode(flat[r])
        out[r] = df_decode(cells, lo, span, flat.shape[1])
    return out.reshape(h.shape)


def conv_seq(conv_state: np.ndarray, xBC: np.ndarray, w: np.ndarray, b: np.ndarray):
    """Causal depthwise conv1d over a whole prompt (Section 4.1's conv step, applied to
    T tokens at once, as the prompt pass of a Mamba-2 layer does).

    conv_state [B, W-1, C] holds the W-1 inputs before the prompt, oldest first;
    xBC [B, T, C] are the prompt's inputs.  Over the concatenation s = [state, xBC],
    output t is silu(bias + sum_j w[:, j] * s[t + j]) (tap W-1 multiplies token t's own
    input); the new state is the last W-1 entries of s, stored as fp32.  Inputs inside
    the prompt enter the window at full precision.  Returns (xc fp64 [B, T, C], new
    state fp32 [B, W-1, C])."""
    cs = np.asarray(conv_state, dtype=np.float64)
    x = np.asarray(xBC, dtype=np.float64)
    W = cs.shape[1] + 1
    T = x.shape[1]
    seq = np.concatenate([cs, x], axis=1)                          # [B, W-1+T, C]
    wt = np.asarray(w, dtype=np.float64)                            # [C, W]
    pre = np.broadcast_to(np.asarray(b, dtype=np.float64), x.shape).copy()
    for j in range(W):
        pre += wt[:, j][None, None, :] * seq[:, j:j + T, :]
    return silu(pre), seq[:, T:T + W - 1, :].astype(np.float32)


@dataclass
class LayerTrace:
    res: np.ndarray          # fp32 [B, D] residual after the layer
    conv: np.ndarray         # fp32 new conv state
    ssm: np.ndarray          # fp32 new SSM state
    x_in: np.ndarray         # fp16 [B, D] pre-norm output (in_proj activation)
    proj_in: ProjTrace
    zxbcdt: np.ndarray       # fp64 [B, in_rows]
    xc: np.ndarray           # fp64 [B, conv_dim] conv output
    y: np.ndarray            # fp64 [B, d_inner] SSM output (before gate)
    g: np.ndarray            # [B, d_inner] gated value y * silu(z), stored as fp32 (held in fp64)
    x_out: np.ndarray        # fp16 [B, d_inner] gated-norm output (out_proj activation)
    proj_out: ProjTrace


def check_layer_shapes(d, lw, st) -> None:
    """Argument validation; a d_state or head mismatch is an error (Appendix B, Table 12)."""
    conv_dim = d.d_inner + 2 * d.ngroups * d.d_state
    in_rows = 2 * d.d_inner + 2 * d.ngroups * d.d_state + d.nheads
    if d.nheads * d.headdim != d.d_inner:
        raise ValueError("d_inner must equal nheads * headdim")
    if lw.inp.rows != in_rows or lw.inp.cols != d.d_model:
        raise ValueError(f"in_proj shape {lw.inp.rows}x{lw.inp.cols} does not match dims ({in_rows}x{d.d_model})")
    if lw.out.rows != d.d_model or lw.out.cols != d.d_inner:
        raise ValueError("out_proj shape does not match dims")
    if st.ssm.shape != (d.batch, d.nheads, d.headdim, d.d_state):
        raise ValueError(f"ssm state shape {st.ssm.shape} does not match dims")
    if st.conv.shape != (d.batch, d.d_conv - 1, conv_dim):
        raise ValueError("conv state shape does not match dims")
    if lw.conv_w.shape != (conv_dim, d.d_conv):
        raise ValueError("conv weight shape does not match dims")


def layer_step(res: np.ndarray, lw, st, d) -> LayerTrace:
    """One decode token through one DF-SSM Mamba-2 layer (residual add included)."""
    check_layer_shapes(d, lw, st)
    E, N, G, H, P = d.d_inner, d.d_state, d.ngroups, d.nheads, d.headdim
    C = E + 2 * G * N
    res = np.asarray(res, dtype=np.float32)
    x_in = rmsnorm(res, lw.prenorm_w).astype(np.float16)
    pin = project(x_in, lw.inp)
    zxbcdt = pin.y
    z = zxbcdt[:, :E]
    xBC = zxbcdt[:, E:E + C]
    dt_raw = zxbcdt[:, E + C:]
    xc, conv_new = conv_step(st.conv, xBC, lw.conv_w, lw.conv_b)
    xs = xc[:, :E].reshape(d.batch, H, P)
    Bg = xc[:, E:E + G * N].reshape(d.batch, G, N)
    Cg = xc[:, E + G * N:].reshape(d.batch, G, N)
    heads_per_group = H // G
    y = np.zeros((d.batch, H, P))
    ssm_new = np.zeros_like(st.ssm)
    for gi in range(G):
        hs = slice(gi * heads_per_group, (gi + 1) * heads_per_group)
        y[:, hs], ssm_new[:, hs] = ssm_step(st.ssm[:, hs], xs[:, hs], Bg[:, gi], Cg[:, gi],
                                            dt_raw[:, hs], lw.dt_bias[hs], lw.A_log[hs], lw.D[hs],
                                            state_dtype=st.ssm.dtype)
    y = y.reshape(d.batch, E)
    # the gated value is an activation between two kernels and is stored as fp32,
    # like the residual stream; the gated RMSNorm reads the stored values
    g = (y * silu(z)).astype(np.float32).astype(np.float64)
    gw = g.reshape(d.batch, G, E // G)
    xo = rmsnorm(gw, lw.gnorm_w.reshape(G, E // G)).reshape(d.batch, E)
    x_out = xo.astype(np.float16)
    pout = project(x_out, lw.out)
    res_new = (res.astype(np.float64) + pout.y).astype(np.float32)
    return LayerTrace(res_new, conv_new, ssm_new, x_in, pin, zxbcdt, xc, y, g, x_out, pout)


@dataclass
class PrefillTrace:
    res: np.ndarray          # fp32 [B, T, D] residual after the layer, every prompt token
    conv: np.ndarray         # fp32 conv state after the prompt
    ssm: np.ndarray          # SSM state after the prompt (the fp64 final state rounded once)
    x_in: np.ndarray         # fp16 [B, T, D]
    zxbcdt: np.ndarray       # fp64 [B, T, in_rows]
    xc: np.ndarray           # fp64 [B, T, conv_dim]
    y: np.ndarray            # fp64 [B, T, d_inner]
    g: np.ndarray            # [B, T, d_inner] gated value, stored as fp32 (held in fp64)
    x_out: np.ndarray        # fp16 [B, T, d_inner]


def layer_prefill(res: np.ndarray, lw, st, d, chunk: int = 64, df: bool = False) -> PrefillTrace:
    """A whole prompt of T tokens through one layer in one pass (the prompt step
    before decode): the projections over all B*T token rows, the causal conv over the
    sequence (conv_seq), the selective SSM as the chunked SSD scan (ssd_scan, Section
    2; block_len 64, Appendix B), gate, gated RMSNorm and out_proj per token.  Each
    token row goes through the same per-token arithmetic as layer_step; the SSM state
    is carried in fp64 through the prompt and stored once at the end.
    res fp32 [B, T, D].  df: the density-field state codec at the chunk boundaries of
    the scan (ssd_scan).  Returns the per-token residuals and the states after the
    prompt."""
    check_layer_shapes(d, lw, st)
    E, N, G, H, P = d.d_inner, d.d_state, d.ngroups, d.nheads, d.headdim
    C = E + 2 * G * N
    if G != 1:
        raise ValueError("layer_prefill follows one group")
    res = np.asarray(res, dtype=np.float32)
    Bsz, T, Dm = res.shape
    if T < 1:
        raise ValueError("a prompt has at least one token")
    x_in = rmsnorm(res, lw.prenorm_w).astype(np.float16)
    zx = project(x_in.reshape(Bsz * T, Dm), lw.inp).y.reshape(Bsz, T, -1)
    z = zx[..., :E]
    xc, conv_new = conv_seq(st.conv, zx[..., E:E + C], lw.conv_w, lw.conv_b)
    xs = xc[..., :E].reshape(Bsz, T, H, P)
    y, hT = ssd_scan(st.ssm, xs, xc[..., E:E + N], xc[..., E + N:E + 2 * N], zx[..., E + C:],
                     lw.dt_bias, lw.A_log, lw.D, chunk=chunk, df=df)
    y = y.reshape(Bsz, T, E)
    g = (y * silu(z)).astype(np.float32).astype(np.float64)
    x_out = rmsnorm(g, lw.gnorm_w).astype(np.float16)
    out = project(x_out.reshape(Bsz * T, E), lw.out).y.reshape(Bsz, T, Dm)
    res_new = (res.astype(np.float64) + out).astype(np.float32)
    return PrefillTrace(res_new, conv_new, hT.astype(st.ssm.dtype), x_in, zx, xc, y, g, x_out)


@dataclass
class State:
    conv: np.ndarray         # fp32 [B, W-1, conv_dim]
    ssm: np.ndarray          # fp32 [B, H, P, N]


@dataclass
class ModelTrace:
    logits: np.ndarray       # fp64 [B, vocab]
    tokens: np.ndarray       # int32 [B]
    res: np.ndarray          # fp32 [B, D] residual entering the final norm
    states: list             # [State] per layer, fp32


def quantize_embedding(embed16: np.ndarray):
    """Per-row int8 quantisation of the tied embedding / LM-head matrix (Section 3.3:
    the embedding is quantised to int8 per row; Table 1: embedding + LM head int8).
    The pages do not give the quantiser; this reading uses the activations' symmetric
    one: scale = max|row| / 127 and code = round-half-even(e / scale) clamped to
    [-127, 127], both decided in fp32; an all-zero row gets codes 0 and scale 1.
    Returns (int8 codes [V, D], fp32 scales [V])."""
    return quantize_act(embed16)


def model_prefill(tokens: np.ndarray, m, states, chunk: int = 64, df: bool = False) -> ModelTrace:
    """A whole prompt tokens [B, T] through the model in one pass (layer_prefill per
    layer), then the final RMSNorm, tied LM head and greedy argmax of the LAST prompt
    token.  Returns the logits and token of that position, the last token's residual
    and every layer's state after the prompt."""
    d = m.dims
    tok = np.asarray(tokens, dtype=np.int64)
    res = m.embed[tok].astype(np.float32)                            # [B, T, D]
    new_states = []
    for lw, st in zip(m.layers, states):
        t = layer_prefill(res, lw, st, d, chunk=chunk, df=df)
        res = t.res
        new_states.append(State(t.conv, t.ssm))
    last = res[:, -1, :]
    xf = rmsnorm(last, m.normf_w)
    logits = xf @ m.embed.astype(np.float64).T
    return ModelTrace(logits, np.argmax(logits, axis=-1).astype(np.int32), last, new_states)


def model_step(tokens: np.ndarray, m, states, emb_q=None) -> ModelTrace:
    """One greedy decode token for the whole model: embedding gather, all layers,
    final RMSNorm, tied LM head (logits = E . norm(res)), argmax with the lowest
    token id winning ties.

    emb_q = (codes, scales) from quantize_embedding selects the int8 embedding: the
    gathered row is scale * code (an fp32 product) and logit v is
    scale_v * sum_k code[v, k] * norm(res)[k]."""
    d = m.dims
    tok = np.asarray(tokens, dtype=np.int64)
    if emb_q is None:
        res = m.embed[tok].astype(np.float32)
    else:
        q, sc = emb_q
        res = (sc[tok].astype(np.float32)[:, None] * q[tok].astype(np.float32)).astype(np.float32)
    new_states = []
    for lw, st in zip(m.layers, states):
        t = layer_step(res, lw, st, d)
        res = t.res
        new_states.append(State(t.conv, t.ssm))
    xf = rmsnorm(res, m.normf_w)
    if emb_q is None:
        logits = xf @ m.embed.astype(np.float64).T
    else:
        q, sc = emb_q
        logits = (xf @ q.astype(np.float64).T) * sc.astype(np.float64)[None, :]
    toks = np.argmax(logits, axis=-1).astype(np.int32)
    return ModelTrace(logits, toks, res, new_states)
