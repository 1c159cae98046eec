"""Pins for the CPU oracle: each check ties an oracle function to something other
than itself -- brute force on tiny inputs, closed forms, invariants, library
routines (np.convolve, np.logaddexp) and numbers printed in "Density Field State
Space Models" (Table 1, Appendix B).  A plausible slip anywhere in the oracle
(a dropped term, a wrong sign or index, a transposed operand) fails one of these.
"""
import json
import math
from dataclasses import replace
import os

import numpy as np
import pytest

from oracle import dfssm_oracle as O
from bit_scaffold_quantized_b200 import synth as S
from bit_scaffold_quantized_b200 import roofline as R

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _proj_from_dense(rng, S0, rank, alpha=None):
    rows, cols = S0.shape
    p = S.gen_proj(rng, rows, cols, rank)
    p.bits = O.pack_signs(S0.astype(np.float32))
    if alpha is not None:
        p.alpha = alpha.astype(np.float16)
    return p


# ---------------------------------------------------------------- packing

def test_pack_single_bit_position():
    # bit j of word k <-> column 32k + j; +1 <-> bit set
    w = -np.ones((3, 96), dtype=np.float32)
    w[1, 37] = 1.0
    bits = O.pack_signs(w)
    expect = np.zeros((3, 3), dtype=np.uint32)
    expect[1, 1] = 1 << 5
    assert np.array_equal(bits, expect)


def test_pack_zero_negzero_nan():
    w = np.array([[0.0, -0.0, np.nan, -1e-30] + [1.0] * 28], dtype=np.float32)
    b = int(O.pack_signs(w)[0, 0])
    assert b & 1 == 1 and (b >> 1) & 1 == 1      # 0.0 and -0.0 -> +1
    assert (b >> 2) & 1 == 0 and (b >> 3) & 1 == 0  # NaN, negative -> -1


def test_pack_unpack_roundtrip_bruteforce():
    rng = np.random.default_rng(10)
    w = rng.normal(size=(7, 64)).astype(np.float32)
    bits = O.pack_signs(w)
    s = O.unpack_signs(bits, 64)
    for r in range(7):
        for c in range(64):
            assert s[r, c] == (1 if w[r, c] >= 0 else -1)
    assert np.array_equal(O.pack_signs(s.astype(np.float32)), bits)


def test_tiled_layout_is_bijection():
    rows, cols = 32, 512
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    wd, bt = O.tiled_bit_position(r.ravel(), c.ravel(), cols)
    flat = wd * 32 + bt
    assert flat.min() == 0 and flat.max() == rows * cols - 1
    assert len(np.unique(flat)) == rows * cols


def test_tiled_layout_matches_mma_fragment_table():
    """Independent check against the m16n8k32 .s8 A-fragment table of the PTX ISA:
    lane = 4*groupID + threadID_in_group; register 0 holds (g, 4t..4t+3), register 1
    (g+8, 4t..4t+3), register 2 (g, 16+4t..), register 3 (g+8, 16+4t..).  Register q
    of product s is (word_q >> s) & 0x01010101; byte i of it is the sign bit of the
    fragment's column 4t+i (+16 for q >= 2), which the layout places at tile column
    64 (s // 2) + 16 t + 8 (s % 2) + i (+4 for q >= 2).  The B fragment of lane t
    (columns 4t..4t+3 and 16+4t..16+4t+3 of the product) is then the 8 bytes at
    64 (s // 2) + 16 t + 8 (s % 2): products 2m and 2m+1 read 16 consecutive bytes."""
    rng = np.random.default_rng(11)
    rows, cols = 16, 256
    dense = rng.choice([-1.0, 1.0], size=(rows, cols)).astype(np.float32)
    tiled = O.tile_signs(O.pack_signs(dense), rows, cols)
    frag_pos = {0: (0, 0), 1: (8, 0), 2: (0, 16), 3: (8, 16)}   # reg q -> (row offset, col offset)
    seen = np.zeros((rows, cols), dtype=int)
    for lane in range(32):
        g, t = lane // 4, lane % 4
        for s in range(8):
            for q in range(4):
                reg = (int(tiled[lane * 4 + q]) >> s) & 0x01010101
                ro, co = frag_pos[q]
                for i in range(4):
                    bit = (reg >> (8 * i)) & 0xFF
                    assert bit in (0, 1)
                    kcol = co + 4 * t + i                            # fragment column 0..31
                    col = 64 * (s // 2) + 16 * t + 8 * (s % 2) + 4 * (co // 16) + i
                    # the same fragment column of the B operand (lane t: b0 = 4t..4t+3,
                    # b1 = 16+4t..) sits at byte 8 * (s % 2) + 4 * (co // 16) + i of the
                    # lane's 16 bytes from 64 (s // 2) + 16 t
                    assert col == 64 * (s // 2) + 16 * t + (8 * (s % 2) + 4 * (kcol // 16) + kcol % 4)
                    assert (1.0 if bit else -1.0) == dense[g + ro, col]
                    seen[g + ro, col] += 1
    assert np.all(seen == 1)


def test_tiled_rows_padded():
    rows, cols = 24, 256
    dense = np.ones((rows, cols), dtype=np.float32)
    tiled = O.tile_signs(O.pack_signs(dense), rows, cols)
    assert tiled.size == 32 * cols // 32
    # padded rows 24..31 are clear
    r, c = np.meshgrid(np.arange(24, 32), np.arange(cols), indexing="ij")
    wd, bt = O.tiled_bit_position(r.ravel(), c.ravel(), cols)
    assert all(((int(tiled[w]) >> int(b)) & 1) == 0 for w, b in zip(wd, bt))


# ---------------------------------------------------------------- scaffold

def test_scaffold_matches_dense_source_matrix():
    """Pack a known dense +/-1 matrix; the oracle projection must equal alpha * (S0 x)
    computed from the original dense matrix (not from the unpacked bits)."""
    rng = np.random.default_rng(12)
    for rows, cols, batch in [(40, 64, 1), (33, 96, 3), (17, 32, 2)]:
        S0 = rng.choice([-1, 1], size=(rows, cols))
        alpha = rng.uniform(0.01, 0.05, size=rows).astype(np.float16)
        p = _proj_from_dense(rng, S0, 0, alpha)
        x = rng.normal(size=(batch, cols)).astype(np.float16)
        y = O.project(x, p).y
        ref = np.zeros((batch, rows))
        for b in range(batch):
            for o in range(rows):
                acc = 0.0
                for k in range(cols):
                    acc += float(S0[o, k]) * float(x[b, k])
                ref[b, o] = float(alpha[o]) * acc
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("sign", [1, -1])
def test_all_same_sign_gives_alpha_sum(sign):
    rng = np.random.default_rng(13)
    rows, cols = 24, 128
    p = _proj_from_dense(rng, np.full((rows, cols), sign), 0)
    x = rng.normal(size=(2, cols)).astype(np.float16)
    y = O.project(x, p).y
    closed = sign * p.alpha.astype(np.float64)[None, :] * x.astype(np.float64).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(y, closed, rtol=1e-13)


# ---------------------------------------------------------------- low-rank correction

def test_rank0_equals_zero_B_bit_identical():
    rng = np.random.default_rng(14)
    p = S.gen_proj(rng, 48, 256, 8)
    x = rng.normal(size=(3, 256)).astype(np.float16)
    p0 = S.ProjWeights(p.rows, p.cols, p.bits, p.alpha, None, None, None, None)
    pz = S.ProjWeights(p.rows, p.cols, p.bits, p.alpha, p.A, p.sA, np.zeros_like(p.B), p.sB)
    assert np.array_equal(O.project(x, p0).y, O.project(x, pz).y)
    assert not np.array_equal(O.project(x, p0).y, O.project(x, p).y)


def test_lora_bruteforce_integer_and_fp():
    rng = np.random.default_rng(15)
    rows, cols, rank, batch = 9, 64, 4, 2
    p = S.gen_proj(rng, rows, cols, rank)
    p.sA = rng.uniform(5e-4, 2e-3, size=rank).astype(np.float16)
    p.sB = rng.uniform(5e-4, 2e-3, size=rows).astype(np.float16)
    x = rng.normal(size=(batch, cols)).astype(np.float16)
    tr = O.project(x, p)
    S0 = O.unpack_signs(p.bits, cols)
    for b in range(batch):
        q = [int(v) for v in tr.xq[b]]
        for j in range(rank):
            acc = 0
            for k in range(cols):
                acc += int(p.A[j, k]) * q[k]
            assert acc == int(tr.acc[b, j])
        u = [int(tr.acc[b, j]) * float(p.sA[j]) * float(tr.sx[b]) for j in range(rank)]
        for o in range(rows):
            scaf = sum(int(S0[o, k]) * float(x[b, k]) for k in range(cols)) * float(p.alpha[o])
            lo = sum(int(p.B[o, j]) * u[j] for j in range(rank)) * float(p.sB[o])
            assert abs(tr.y[b, o] - (scaf + lo)) <= 1e-12 * max(1.0, abs(scaf + lo))


def test_identity_like_A_picks_codes():
    rng = np.random.default_rng(16)
    cols, rank = 128, 8
    p = S.gen_proj(rng, 16, cols, rank)
    picks = rng.choice(cols, size=rank, replace=False)
    A = np.zeros((rank, cols), dtype=np.int8)
    A[np.arange(rank), picks] = 1
    A[3, picks[3]] = -1
    x = rng.normal(size=(1, cols)).astype(np.float16)
    xq, _ = O.quantize_act(x)
    acc = O.lora_stage1(A, xq)
    expect = xq[0, picks].astype(np.int64)
    expect[3] = -expect[3]
    assert np.array_equal(acc[0], expect)


def test_lora_worst_case_fits_int32():
    A = np.full((1, 4096), 127, dtype=np.int8)
    xq = np.full((1, 4096), -127, dtype=np.int8)
    assert int(O.lora_stage1(A, xq)[0, 0]) == -4096 * 127 * 127
    A2 = np.full((1, 2 ** 18), 127, dtype=np.int8)
    with pytest.raises(OverflowError):
        O.lora_stage1(A2, np.full((1, 2 ** 18), 127, dtype=np.int8))


# ---------------------------------------------------------------- quantiser

def test_quantize_ties_half_even_and_extremes():
    x = np.array([[127.0, 2.5, 3.5, -2.5, -127.0, 0.5, 1.5, 0.0]], dtype=np.float16)
    q, sx = O.quantize_act(x)
    assert sx[0] == np.float32(1.0)
    assert q.tolist() == [[127, 2, 4, -2, -127, 0, 2, 0]]


def test_quantize_zero_row_and_bounds():
    rng = np.random.default_rng(17)
    x = rng.normal(size=(4, 512)).astype(np.float16)
    x[2] = 0
    q, sx = O.quantize_act(x)
    assert np.all(q[2] == 0) and sx[2] == 1.0
    for r in (0, 1, 3):
        i = int(np.argmax(np.abs(x[r].astype(np.float32))))
        assert abs(int(q[r, i])) == 127 and np.sign(q[r, i]) == np.sign(x[r, i])
        err = np.abs(x[r].astype(np.float64) - q[r].astype(np.float64) * float(sx[r]))
        assert err.max() <= 0.5 * float(sx[r]) * (1 + 1e-6)
        assert np.all(np.abs(q[r]) <= 127)


# ---------------------------------------------------------------- conv step

def test_conv_step_matches_np_convolve():
    rng = np.random.default_rng(18)
    T, Cc, W = 11, 5, 4
    u = rng.normal(size=(T, Cc))
    w = rng.uniform(-0.5, 0.5, size=(Cc, W)).astype(np.float16)
    b = rng.uniform(-0.5, 0.5, size=Cc).astype(np.float16)
    st = np.zeros((1, W - 1, Cc), dtype=np.float32)
    outs = []
    for t in range(T):
        y, st = O.conv_step(st, u[t:t + 1].astype(np.float32), w, b)
        outs.append(y[0])
    outs = np.array(outs)
    u32 = u.astype(np.float32).astype(np.float64)
    for c in range(Cc):
        pre = np.convolve(u32[:, c], w[c, ::-1].astype(np.float64))[:T] + float(b[c])
        np.testing.assert_allclose(outs[:, c], pre / (1 + np.exp(-pre)), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_conv_one_hot_tap_delays(tap):
    T, W = 9, 4
    u = np.arange(1, T + 1, dtype=np.float32)[:, None] * 0.25
    w = np.zeros((1, W), dtype=np.float16)
    w[0, tap] = 1
    st = np.zeros((1, W - 1, 1), dtype=np.float32)
    for t in range(T):
        y, st = O.conv_step(st, u[t:t + 1], w, np.zeros(1, np.float16))
        src = t - (W - 1 - tap)
        v = float(u[src, 0]) if src >= 0 else 0.0
        assert y[0, 0] == pytest.approx(v / (1 + np.exp(-v)), rel=1e-14, abs=0)


# ---------------------------------------------------------------- SSM step

def _ssm_args(rng, Bb=2, H=3, P=4, N=5):
    h = rng.normal(size=(Bb, H, P, N)).astype(np.float32)
    x = rng.normal(size=(Bb, H, P))
    Bv = rng.normal(size=(Bb, N))
    Cv = rng.normal(size=(Bb, N))
    dt_raw = rng.normal(size=(Bb, H))
    dt_bias = rng.normal(0, 0.1, size=H).astype(np.float32)
    A_log = rng.uniform(0, np.log(16), size=H).astype(np.float32)
    D = rng.normal(1, 0.1, size=H).astype(np.float32)
    return h, x, Bv, Cv, dt_raw, dt_bias, A_log, D


def test_softplus_library():
    v = np.linspace(-30, 20, 1001)
    np.testing.assert_allclose(O.softplus(v), np.logaddexp(0.0, v), rtol=1e-15, atol=1e-300)
    big = np.linspace(20.001, 60, 101)       # above the threshold: identity, off by < e^-20
    assert np.array_equal(O.softplus(big), big)
    assert np.max(np.abs(np.logaddexp(0.0, big) - big)) < np.exp(-20.0)
    assert O.softplus(np.array([-1e4]))[0] == 0.0


def test_ssm_bruteforce_scalar_loops():
    rng = np.random.default_rng(19)
    h, x, Bv, Cv, dt_raw, dt_bias, A_log, D = _ssm_args(rng)
    y, hn = O.ssm_step(h, x, Bv, Cv, dt_raw, dt_bias, A_log, D)
    import math
    Bb, H, P, N = h.shape
    for b in range(Bb):
        for hh in range(H):
            v = float(dt_raw[b, hh]) + float(dt_bias[hh])
            dt = math.log1p(math.exp(v))
            dA = math.exp(-dt * math.exp(float(A_log[hh])))
            for p in range(P):
                yy = 0.0
                for n in range(N):
                    hv = dA * float(h[b, hh, p, n]) + dt * float(x[b, hh, p]) * float(Bv[b, n])
                    assert hn[b, hh, p, n] == np.float32(hv)
                    yy += float(Cv[b, n]) * hv
                yy += float(D[hh]) * float(x[b, hh, p])
                assert y[b, hh, p] == pytest.approx(yy, rel=1e-12, abs=1e-12)


def test_ssm_dt_zero_leaves_state():
    rng = np.random.default_rng(20)
    h, x, Bv, Cv, dt_raw, dt_bias, A_log, D = _ssm_args(rng)
    dt_bias[:] = -1e4
    y, hn = O.ssm_step(h, x, Bv, Cv, dt_raw, dt_bias, A_log, D)
    assert np.array_equal(hn, h)
    np.testing.assert_allclose(y, np.einsum("bhpn,bn->bhp", h.astype(np.float64), Cv) + D[None, :, None] * x,
                               rtol=1e-13)


def test_ssm_recurrence_equals_unrolled_closed_form():
    rng = np.random.default_rng(21)
    T = 7
    h0, _, _, _, _, dt_bias, A_log, D = _ssm_args(rng, Bb=1)
    h0 = h0.astype(np.float64)
    xs = rng.normal(size=(T, 1, 3, 4))
    Bs = rng.normal(size=(T, 1, 5))
    Cs = rng.normal(size=(T, 1, 5))
    dts = rng.normal(size=(T, 1, 3))
    # fp64 recurrence (state kept in fp64 by re-deriving from the oracle's formula pieces)
    h = h0.copy()
    dAs, dtv = [], []
    for t in range(T):
        dt = O.softplus(dts[t] + dt_bias)
        dA = np.exp(dt * -np.exp(A_log.astype(np.float64)))
        dAs.append(dA)
        dtv.append(dt)
        y, hn = O.ssm_step(h.astype(np.float32), xs[t], Bs[t], Cs[t], dts[t], dt_bias, A_log, D)
        # oracle's own step (fp32 storage) must track the fp64 recurrence closely
        h = dA[:, :, None, None] * h + (xs[t] * dt[:, :, None])[..., None] * Bs[t][:, None, None, :]
        np.testing.assert_allclose(hn, h, rtol=1e-5, atol=1e-6)
    closed = np.prod(dAs, axis=0)[:, :, None, None] * h0
    for t in range(T):
        decay = np.ones_like(dAs[0])
        for s in range(t + 1, T):
            decay = decay * dAs[s]
        closed = closed + decay[:, :, None, None] * (xs[t] * dtv[t][:, :, None])[..., None] * Bs[t][:, None, None, :]
    np.testing.assert_allclose(h, closed, rtol=1e-12, atol=1e-12)


def test_ssm_no_decay_is_running_sum():
    rng = np.random.default_rng(22)
    h, x, Bv, Cv, dt_raw, dt_bias, A_log, D = _ssm_args(rng)
    A_log[:] = -80.0   # A = -exp(-80): dt*A rounds exp() to exactly 1
    h[:] = 0
    acc = np.zeros(h.shape)
    for t in range(3):
        _, h = O.ssm_step(h, x, Bv, Cv, dt_raw, dt_bias, A_log, D)
        dt = np.logaddexp(0.0, dt_raw + dt_bias)
        acc = acc + (x * dt[:, :, None])[..., None] * Bv[:, None, None, :]
        np.testing.assert_allclose(h, acc, rtol=1e-5, atol=1e-6)


def test_appendixB_dt_scaling_matters():
    fix = json.load(open(os.path.join(GOLDEN, "appendixB_block_fixes.json")))
    assert "dt" in fix["fixes"][0]["correct"]
    rng = np.random.default_rng(23)
    h, x, Bv, Cv, dt_raw, dt_bias, A_log, D = _ssm_args(rng)
    _, hn = O.ssm_step(h, x, Bv, Cv, dt_raw, dt_bias, A_log, D)
    dt = np.logaddexp(0.0, dt_raw + dt_bias)
    dA = np.exp(-dt * np.exp(A_log))
    buggy = dA[:, :, None, None] * h + x[..., None] * Bv[:, None, None, :]
    assert np.max(np.abs(hn - buggy)) > 1e-2


# ---------------------------------------------------------------- gated norm

def test_gate_then_norm_order_and_unit_rms():
    fix = json.load(open(os.path.join(GOLDEN, "appendixB_block_fixes.json")))
    assert fix["fixes"][2]["correct"] == "norm(y * silu(z))"
    rng = np.random.default_rng(24)
    y = rng.normal(size=(2, 64))
    z = rng.normal(size=(2, 64))
    w = np.ones(64, dtype=np.float16)
    got = O.gated_rmsnorm(y, z, w)
    np.testing.assert_allclose(np.mean(got ** 2, axis=-1), 1.0, rtol=1e-4)
    g = y * (z / (1 + np.exp(-z)))
    np.testing.assert_allclose(got, g / np.sqrt(np.mean(g ** 2, axis=-1, keepdims=True) + O.EPS), rtol=1e-13)
    wrong = O.rmsnorm(y, w) * (z / (1 + np.exp(-z)))
    assert np.max(np.abs(got - wrong)) > 0.1


# ---------------------------------------------------------------- layer / model

def _small_layer(seed=25, batch=2):
    d = S.LAYER_SMALL.with_batch(batch)
    rng = np.random.default_rng(seed)
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    st.conv[:] = rng.normal(size=st.conv.shape)
    st.ssm[:] = rng.normal(size=st.ssm.shape)
    res = rng.normal(size=(batch, d.d_model)).astype(np.float32)
    return d, lw, st, res


def test_appendixB_d_state_mismatch_rejected():
    d, lw, st, res = _small_layer()
    bad = S.Dims(batch=d.batch, d_model=d.d_model, d_inner=d.d_inner, nheads=d.nheads,
                 headdim=d.headdim, d_state=d.d_state // 2, rank=d.rank)
    with pytest.raises(ValueError):
        O.layer_step(res, lw, st, bad)


def test_layer_identity_when_out_proj_is_zero():
    d, lw, st, res = _small_layer()
    lw.out.alpha[:] = 0
    lw.out.A = lw.out.B = lw.out.sA = lw.out.sB = None
    t = O.layer_step(res, lw, st, d)
    assert np.array_equal(t.res, res)


def test_layer_conv_state_shift_and_dt_zero():
    d, lw, st, res = _small_layer()
    lw.dt_bias[:] = -1e4
    t = O.layer_step(res, lw, st, d)
    assert np.array_equal(t.conv[:, :2], st.conv[:, 1:])
    E, C = d.d_inner, d.conv_dim
    assert np.array_equal(t.conv[:, 2], t.zxbcdt[:, E:E + C].astype(np.float32))
    assert np.array_equal(t.ssm, st.ssm)


def test_layer_pieces_compose():
    """The layer's intermediates agree with the pinned pieces applied one at a time."""
    d, lw, st, res = _small_layer()
    t = O.layer_step(res, lw, st, d)
    E, C, N = d.d_inner, d.conv_dim, d.d_state
    x_in = O.rmsnorm(res, lw.prenorm_w).astype(np.float16)
    assert np.array_equal(x_in, t.x_in)
    assert np.array_equal(O.project(x_in, lw.inp).y, t.zxbcdt)
    xc, _ = O.conv_step(st.conv, t.zxbcdt[:, E:E + C], lw.conv_w, lw.conv_b)
    y, _ = O.ssm_step(st.ssm, xc[:, :E].reshape(d.batch, d.nheads, d.headdim), xc[:, E:E + N],
                      xc[:, E + N:], t.zxbcdt[:, E + C:], lw.dt_bias, lw.A_log, lw.D)
    np.testing.assert_array_equal(y.reshape(d.batch, E), t.y)
    g32 = (t.y * O.silu(t.zxbcdt[:, :E])).astype(np.float32)
    assert np.array_equal(t.g, g32.astype(np.float64))
    xo = O.rmsnorm(g32, lw.gnorm_w).astype(np.float16)
    assert np.array_equal(xo, t.x_out)


def test_model_argmax_lowest_id_on_ties_and_embedding():
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(26)
    m = S.gen_model(rng, d, 0, 40)
    m.embed[7] = m.embed[3]
    m.embed[3] *= 8
    m.embed[7] = m.embed[3]
    tr = O.model_step(np.array([3, 7], dtype=np.int32), m, [])
    assert np.array_equal(tr.res, m.embed[[3, 7]].astype(np.float32))
    assert tr.tokens.tolist() == [3, 3]


@pytest.mark.parametrize("chunk", [1, 3, 8, 64])
def test_ssd_chunked_scan_equals_token_recurrence(chunk):
    """The chunked SSD form over a prompt equals the token-by-token recurrence
    (ssm_step with the state carried in fp64) for every chunk length, including a
    ragged last chunk and a nonzero starting state."""
    rng = np.random.default_rng(29)
    Bsz, T, H, P, N = 2, 20, 3, 4, 8
    h0 = rng.normal(size=(Bsz, H, P, N))
    x = rng.normal(size=(Bsz, T, H, P))
    Bm, Cm = rng.normal(size=(Bsz, T, N)), rng.normal(size=(Bsz, T, N))
    dt_raw = rng.normal(size=(Bsz, T, H))
    dt_bias = rng.normal(0, 0.1, size=H).astype(np.float32)
    A_log = rng.uniform(0, np.log(16), size=H).astype(np.float32)
    D = rng.normal(1, 0.1, size=H).astype(np.float32)
    y, hT = O.ssd_scan(h0, x, Bm, Cm, dt_raw, dt_bias, A_log, D, chunk=chunk)
    h = h0.copy()
    for t in range(T):
        yt, h = O.ssm_step(h, x[:, t], Bm[:, t], Cm[:, t], dt_raw[:, t], dt_bias, A_log, D,
                           state_dtype=np.float64)
        assert np.max(np.abs(y[:, t] - yt)) <= 1e-12 * max(1.0, np.max(np.abs(yt)))
    assert np.max(np.abs(hT - h)) <= 1e-12 * max(1.0, np.max(np.abs(h)))


def test_ssm_fp16_state_is_the_fp64_update_rounded_once():
    """Half-precision state storage: the new state is the fp64 update h' rounded once
    to fp16 (checked per element against a plain loop), y is computed from the
    unrounded h' exactly as with fp32 storage, and a layer step whose state is fp16
    keeps it fp16."""
    rng = np.random.default_rng(28)
    Bsz, H, P, N = 2, 3, 4, 8
    h = rng.normal(size=(Bsz, H, P, N)).astype(np.float16)
    x = rng.normal(size=(Bsz, H, P))
    Bv, Cv = rng.normal(size=(Bsz, N)), rng.normal(size=(Bsz, N))
    dt_raw = rng.normal(size=(Bsz, H))
    dt_bias = rng.normal(0, 0.1, size=H).astype(np.float32)
    A_log = rng.uniform(0, np.log(16), size=H).astype(np.float32)
    D = rng.normal(1, 0.1, size=H).astype(np.float32)
    y16, h16 = O.ssm_step(h, x, Bv, Cv, dt_raw, dt_bias, A_log, D, state_dtype=np.float16)
    y32, h32 = O.ssm_step(h, x, Bv, Cv, dt_raw, dt_bias, A_log, D)
    assert h16.dtype == np.float16 and h32.dtype == np.float32
    assert np.array_equal(y16, y32)
    for b in range(Bsz):
        for hh in range(H):
            dt = float(np.log1p(np.exp(float(dt_raw[b, hh]) + float(dt_bias[hh]))))
            dA = np.exp(-dt * np.exp(float(A_log[hh])))
            for p in range(P):
                for n in range(N):
                    v = dA * float(h[b, hh, p, n]) + (float(x[b, hh, p]) * dt) * float(Bv[b, n])
                    assert h16[b, hh, p, n] == np.float16(v)
    d = S.Dims(batch=2, d_model=256, d_inner=512, nheads=8, headdim=64, d_state=16, rank=8, ssm_state_dtype=1)
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    assert st.ssm.dtype == np.float16
    t = O.layer_step(S.gen_layer_inputs(rng, d, 1)[0], lw, st, d)
    assert t.ssm.dtype == np.float16 and t.conv.dtype == np.float32


def test_int8_embedding_rows_and_logits_brute_force():
    """Section 3.3 int8 per-row embedding: the gathered row is scale * code in fp32,
    and the logits of the tied head are scale_v * (codes . norm(res)); checked
    element by element against a plain loop, plus the quantiser's bound and the
    zero-row case."""
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(27)
    m = S.gen_model(rng, d, 0, 24)
    m.embed[5] = 0
    q, sc = O.quantize_embedding(m.embed)
    assert q.dtype == np.int8 and sc.dtype == np.float32 and sc[5] == 1.0 and np.all(q[5] == 0)
    for v in (0, 9, 23):
        e = m.embed[v].astype(np.float64)
        i = int(np.argmax(np.abs(e)))
        assert abs(int(q[v, i])) == 127
        assert np.max(np.abs(e - q[v].astype(np.float64) * float(sc[v]))) <= 0.5 * float(sc[v]) * (1 + 1e-6)
    toks = np.array([9, 5], dtype=np.int32)
    tr = O.model_step(toks, m, [], emb_q=(q, sc))
    for b, t in enumerate(toks):
        for k in (0, 17, 255):
            assert tr.res[b, k] == np.float32(np.float32(sc[t]) * np.float32(q[t, k]))
    xf = O.rmsnorm(tr.res, m.normf_w)
    for b in range(2):
        for v in (0, 3, 23):
            ref = float(sc[v]) * sum(float(q[v, k]) * xf[b, k] for k in range(d.d_model))
            assert abs(tr.logits[b, v] - ref) <= 1e-12 * max(1.0, abs(ref))
    assert tr.tokens.tolist() == np.argmax(tr.logits, axis=-1).tolist()


# ---------------------------------------------------------------- byte model vs Table 1

def test_byte_model_head_and_state_variants():
    """int8 head: 1 byte per element plus a 4-byte scale per row (embedding row and
    head); fp16 SSM state: 2 bytes per state element, conv state unchanged."""
    d = S.LAYER_1P3B
    V, L = S.VOCAB_1P3B, 48
    f16 = R.model_token_bytes(d, L, V)
    i8 = R.model_token_bytes(d, L, V, head="int8")
    assert f16 - i8 == (2 * d.d_model - (d.d_model + 4)) + V * (2 * d.d_model - (d.d_model + 4))
    d16 = replace(d, ssm_state_dtype=1)
    ssm = d.nheads * d.headdim * d.d_state
    assert R.layer_state_bytes(d) - R.layer_state_bytes(d16) == 2 * d.batch * 2 * ssm
    assert f16 == 597_628_936


def test_table1_sizes_from_shapes():
    t1 = json.load(open(os.path.join(GOLDEN, "table1_model_size.json")))
    d = S.LAYER_1P3B
    n = t1["n_layer"]
    scaffold = n * (d.in_rows * d.d_model + d.d_model * d.d_inner) // 8
    assert abs(scaffold / 1e6 - t1["scaffold_1bit_MB"]) < 0.5
    emb = S.VOCAB_1P3B * d.d_model
    assert abs(emb / 1e6 - t1["embedding_lm_head_int8_MB"]) < 0.5
    r = t1["lora_rank"]
    lora = n * r * (d.d_model + d.in_rows + d.d_inner + d.d_model)
    assert abs(lora / 1e6 - t1["lora_int8_r16_MB"]) < 1.0
    # the byte model counts the same scaffold and LoRA bytes
    d16 = S.Dims(1, 2048, 4096, 64, 64, 128, rank=r)
    bits_only = R.proj_weight_bytes(d16.in_rows, 2048, 0) - 2 * d16.in_rows \
        + R.proj_weight_bytes(2048, 4096, 0) - 2 * 2048
    assert n * bits_only == scaffold


def test_decode_token_bytes_1p3b():
    d = S.LAYER_1P3B
    assert R.layer_weight_bytes(d) == 3_861_120
    assert R.layer_state_bytes(d) == 4_298_752
    tok = R.model_token_bytes(d, 48, S.VOCAB_1P3B)
    assert abs(tok / 1e6 - 597.6) < 0.1


# ---------------------------------------------------------------- layer wiring, by hand

def _scalar_rmsnorm(v, w, eps=1e-5):
    ms = sum(float(a) * float(a) for a in v) / len(v)
    r = 1.0 / math.sqrt(ms + eps)
    return [float(a) * r * float(b) for a, b in zip(v, w)]


def _scalar_silu(v):
    return v / (1.0 + math.exp(-v))


def test_rmsnorm_weight_is_applied_per_element():
    """RMSNorm with a non-unit, non-uniform weight against a scalar loop: a dropped,
    inverted or reversed weight fails."""
    rng = np.random.default_rng(30)
    v = rng.normal(size=(3, 40))
    w = rng.uniform(0.25, 3.0, size=40).astype(np.float16)
    got = O.rmsnorm(v, w)
    for b in range(3):
        ref = _scalar_rmsnorm(v[b], w)
        for k in range(40):
            assert got[b, k] == pytest.approx(ref[k], rel=1e-13, abs=0)
    assert np.max(np.abs(got - O.rmsnorm(v, np.ones(40)))) > 0.1
    assert np.max(np.abs(got - O.rmsnorm(v, 1.0 / w.astype(np.float64)))) > 0.1


def test_final_norm_weight_and_tied_head_by_hand():
    """Model with no layers: logits[b, v] = sum_k E[v, k] * rmsnorm(E[tok_b])[k] * wf[k],
    written out as scalar loops with a non-uniform final norm weight."""
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(31)
    m = S.gen_model(rng, d, 0, 12)
    m.normf_w = rng.uniform(0.2, 2.5, size=d.d_model).astype(np.float16)
    toks = np.array([4, 9], dtype=np.int32)
    tr = O.model_step(toks, m, [])
    for b, t in enumerate(toks):
        xn = _scalar_rmsnorm(m.embed[t].astype(np.float32), m.normf_w)
        for v in range(12):
            ref = sum(float(m.embed[v, k]) * xn[k] for k in range(d.d_model))
            assert tr.logits[b, v] == pytest.approx(ref, rel=1e-12, abs=1e-15)
    m.normf_w = np.ones(d.d_model, dtype=np.float16)
    assert np.max(np.abs(O.model_step(toks, m, []).logits - tr.logits)) > 1e-3


def _hand_layer(seed):
    """A hand-sized layer: d_model 32, two heads of headdim 16 (d_inner 32), d_state 2,
    rank 0, random signs and non-uniform weights, nonzero conv and SSM state."""
    d = S.Dims(batch=1, d_model=32, d_inner=32, nheads=2, headdim=16, d_state=2, rank=0)
    rng = np.random.default_rng(seed)
    lw = S.gen_layer(rng, d)
    lw.prenorm_w = rng.uniform(0.3, 2.0, size=32).astype(np.float16)
    lw.gnorm_w = rng.uniform(0.3, 2.0, size=32).astype(np.float16)
    lw.inp.alpha = rng.uniform(0.05, 0.6, size=d.in_rows).astype(np.float16)
    lw.out.alpha = rng.uniform(0.05, 0.6, size=32).astype(np.float16)
    lw.dt_bias = np.array([0.3, -0.4], dtype=np.float32)
    lw.A_log = np.array([0.2, 1.1], dtype=np.float32)
    lw.D = np.array([0.7, 1.3], dtype=np.float32)
    st = S.zero_state(d)
    st.conv[:] = rng.normal(size=st.conv.shape)
    st.ssm[:] = rng.normal(size=st.ssm.shape)
    res = rng.normal(size=(1, 32)).astype(np.float32)
    return d, lw, st, res


def _hand_layer_expected(d, lw, st, res):
    """The layer written out with scalar loops and explicit index ranges.

    in_proj rows, Mamba-2 order: z = [0, E), x = [E, 2E), B = [2E, 2E+N),
    C = [2E+N, 2E+2N), dt_raw = [2E+2N, 2E+2N+H).  The conv runs over x, B and C
    (window = three stored inputs, oldest first, then the new one; tap 3 = newest).
    State update h' = dA h + (x dt) B[n]; read-out y = sum_n C[n] h'[n] + D x.
    Gate z: g = y silu(z), stored fp32; xo = fp16(rmsnorm(g) w_g); res += out_proj(xo).
    """
    E, N, H, P, Dm = d.d_inner, d.d_state, d.nheads, d.headdim, d.d_model
    r = [float(v) for v in res[0]]
    x_in = [float(np.float16(v)) for v in _scalar_rmsnorm(r, lw.prenorm_w)]
    sin = O.unpack_signs(lw.inp.bits, Dm)
    zx = [float(lw.inp.alpha[o]) * sum(int(sin[o, k]) * x_in[k] for k in range(Dm)) for o in range(d.in_rows)]
    z = zx[0:E]
    xBC = zx[E:2 * E + 2 * N]
    dt_raw = zx[2 * E + 2 * N:2 * E + 2 * N + H]
    xc, conv_new = [], []
    for c in range(E + 2 * N):
        win = [float(st.conv[0, 0, c]), float(st.conv[0, 1, c]), float(st.conv[0, 2, c]), xBC[c]]
        pre = float(lw.conv_b[c]) + sum(float(lw.conv_w[c, j]) * win[j] for j in range(4))
        xc.append(_scalar_silu(pre))
        conv_new.append(win[1:])
    xs, Bv, Cv = xc[0:E], xc[E:E + N], xc[E + N:E + 2 * N]
    y = [0.0] * E
    hnew = np.zeros((H, P, N))
    for h in range(H):
        v = dt_raw[h] + float(lw.dt_bias[h])
        dt = v if v > 20 else math.log1p(math.exp(v))
        dA = math.exp(dt * -math.exp(float(lw.A_log[h])))
        for p in range(P):
            e = h * P + p
            acc = 0.0
            for n in range(N):
                hv = dA * float(st.ssm[0, h, p, n]) + (xs[e] * dt) * Bv[n]
                hnew[h, p, n] = hv
                acc += Cv[n] * hv
            y[e] = acc + float(lw.D[h]) * xs[e]
    g = [float(np.float32(y[e] * _scalar_silu(z[e]))) for e in range(E)]
    xo = [float(np.float16(v)) for v in _scalar_rmsnorm(g, lw.gnorm_w)]
    sout = O.unpack_signs(lw.out.bits, E)
    res_new = [float(np.float32(r[o] + float(lw.out.alpha[o]) * sum(int(sout[o, k]) * xo[k] for k in range(E))))
               for o in range(Dm)]
    return dict(x_in=x_in, zx=zx, xc=xc, conv=conv_new, y=y, ssm=hnew, g=g, xo=xo, res=res_new)


@pytest.mark.parametrize("seed", [32, 33])
def test_layer_wiring_by_hand(seed):
    """Every intermediate of one layer step against the scalar-loop restatement above:
    a B <-> C swap, x used as the gate instead of z, a wrong dt slice, a dropped or
    misplaced norm weight, or a wrong conv window each change these values."""
    d, lw, st, res = _hand_layer(seed)
    t = O.layer_step(res, lw, st, d)
    ex = _hand_layer_expected(d, lw, st, res)
    close = dict(rel=1e-11, abs=1e-12)
    assert [float(v) for v in t.x_in[0]] == ex["x_in"]
    for o in range(d.in_rows):
        assert t.zxbcdt[0, o] == pytest.approx(ex["zx"][o], **close)
    for c in range(len(ex["xc"])):
        assert t.xc[0, c] == pytest.approx(ex["xc"][c], **close)
        for j in range(3):
            assert float(t.conv[0, j, c]) == pytest.approx(float(np.float32(ex["conv"][c][j])), rel=1e-6)
    for e in range(d.d_inner):
        assert t.y[0, e] == pytest.approx(ex["y"][e], **close)
        assert t.g[0, e] == pytest.approx(ex["g"][e], rel=1e-6, abs=1e-9)
    np.testing.assert_allclose(t.ssm[0].astype(np.float64), ex["ssm"], rtol=1e-6, atol=1e-7)
    assert [float(v) for v in t.x_out[0]] == ex["xo"]
    np.testing.assert_allclose(t.res[0].astype(np.float64), ex["res"], rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------- prompt pass (prefill)

def test_conv_seq_matches_np_convolve_and_steps():
    """The sequence conv against np.convolve per channel (zero initial state) and
    against token-by-token conv_step with a nonzero initial state (inputs exactly
    representable in fp32, so the step's fp32 state storage rounds nothing)."""
    rng = np.random.default_rng(40)
    T, Cc, W = 13, 6, 4
    u = rng.normal(size=(1, T, Cc)).astype(np.float32).astype(np.float64)
    w = rng.uniform(-0.5, 0.5, size=(Cc, W)).astype(np.float16)
    b = rng.uniform(-0.5, 0.5, size=Cc).astype(np.float16)
    xc, st = O.conv_seq(np.zeros((1, W - 1, Cc), np.float32), u, w, b)
    for c in range(Cc):
        pre = np.convolve(u[0, :, c], w[c, ::-1].astype(np.float64))[:T] + float(b[c])
        np.testing.assert_allclose(xc[0, :, c], pre / (1 + np.exp(-pre)), rtol=1e-12, atol=1e-14)
    assert np.array_equal(st[0], u[0, T - 3:].astype(np.float32))
    st0 = rng.normal(size=(2, W - 1, Cc)).astype(np.float32)
    u2 = rng.normal(size=(2, T, Cc)).astype(np.float32).astype(np.float64)
    xs, sN = O.conv_seq(st0, u2, w, b)
    s = st0
    for t in range(T):
        y, s = O.conv_step(s, u2[:, t], w, b)
        np.testing.assert_allclose(xs[:, t], y, rtol=1e-13, atol=1e-15)
    assert np.array_equal(sN, s)
    # a one-token prompt is exactly one conv step
    y1, s1 = O.conv_seq(st0, u2[:, :1], w, b)
    ys, ss = O.conv_step(st0, u2[:, 0], w, b)
    assert np.array_equal(y1[:, 0], ys) and np.array_equal(s1, ss)


def _prefill_layer(seed, T, batch=2, rank=8):
    d = S.Dims(batch=batch, d_model=256, d_inner=512, nheads=8, headdim=64, d_state=16, rank=rank)
    rng = np.random.default_rng(seed)
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    st.conv[:] = rng.normal(size=st.conv.shape)
    st.ssm[:] = rng.normal(size=st.ssm.shape)
    res = rng.normal(size=(batch, T, d.d_model)).astype(np.float16).astype(np.float32)
    return d, lw, st, res


def test_layer_prefill_one_token_is_one_layer_step():
    d, lw, st, res = _prefill_layer(41, 1)
    p = O.layer_prefill(res, lw, st, d)
    t = O.layer_step(res[:, 0], lw, st, d)
    assert np.array_equal(p.res[:, 0], t.res)
    assert np.array_equal(p.conv, t.conv) and np.array_equal(p.ssm, t.ssm)
    assert np.array_equal(p.x_out[:, 0], t.x_out)


@pytest.mark.parametrize("T,chunk", [(5, 64), (9, 4), (20, 8)])
def test_layer_prefill_tracks_token_steps(T, chunk):
    """A prompt in one pass against T layer steps: the only difference is where the
    states are rounded (fp32 after every token step, once after the prompt), so the
    two agree to fp32 rounding, far inside the 2e-3 bar; the chunk length does not
    matter beyond rounding."""
    d, lw, st, res = _prefill_layer(42 + T, T)
    p = O.layer_prefill(res, lw, st, d, chunk=chunk)
    s = st
    for t in range(T):
        tr = O.layer_step(res[:, t], lw, s, d)
        s = O.State(tr.conv, tr.ssm)
        assert np.max(np.abs(p.res[:, t] - tr.res)) <= 1e-4 * max(1.0, np.max(np.abs(tr.res)))
    np.testing.assert_allclose(p.ssm, s.ssm, rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(p.conv, s.conv, rtol=1e-6, atol=1e-6)


def test_model_prefill_last_logits_track_token_steps():
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(43)
    m = S.gen_model(rng, d, 2, 300)
    toks = rng.integers(0, 300, size=(2, 7)).astype(np.int32)
    p = O.model_prefill(toks, m, [O.State(*(lambda z: (z.conv, z.ssm))(S.zero_state(d))) for _ in m.layers])
    states = [O.State(*(lambda z: (z.conv, z.ssm))(S.zero_state(d))) for _ in m.layers]
    for t in range(7):
        tr = O.model_step(toks[:, t], m, states)
        states = tr.states
    rms = np.sqrt(np.mean(tr.logits ** 2))
    assert np.max(np.abs(p.logits - tr.logits)) <= 1e-4 * rms
    for a, b in zip(p.states, states):
        np.testing.assert_allclose(a.ssm, b.ssm, rtol=1e-4, atol=1e-5)
    with pytest.raises(ValueError):
        O.layer_prefill(np.zeros((2, 0, d.d_model), np.float32), m.layers[0], S.zero_state(d), d)


def test_silent_layers_greedy_decode_repeats_the_token():
    """Closed form over several greedy tokens through a layer stack.  With every
    out_proj scaled to zero, each layer returns its input residual unchanged (the
    residual add of Section 4.1), so the final residual is the token's embedding row.
    With equal-norm rows and a constant final-norm weight c, Cauchy-Schwarz makes the
    token's own row the strict argmax of the tied head, with logit
    c |e|^2 / sqrt(|e|^2 / D + eps).  A dropped residual, a wrong row gathered or a
    transposed head fails this; the layers' states must still move."""
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(47)
    m = S.silent_model(rng, d, 3, 64)
    assert len(np.unique(m.embed, axis=0)) == 64
    norms = np.sum(m.embed.astype(np.float64) ** 2, axis=1)
    assert np.all(norms == norms[0])
    states = [O.State(*(lambda z: (z.conv, z.ssm))(S.zero_state(d))) for _ in m.layers]
    toks = np.array([5, 41], dtype=np.int32)
    e2 = float(norms[0])
    own = 1.5 * e2 / math.sqrt(e2 / d.d_model + O.EPS)
    for _ in range(5):
        tr = O.model_step(toks, m, states)
        assert np.array_equal(tr.res, m.embed[toks].astype(np.float32))
        assert tr.tokens.tolist() == toks.tolist()
        for b, t in enumerate(toks):
            assert tr.logits[b, t] == pytest.approx(own, rel=1e-12)
            assert np.max(np.delete(tr.logits[b], t)) < 0.5 * own
        states = tr.states
    assert all(np.max(np.abs(s.ssm)) > 0 for s in states)


def test_batch_rows_are_independent():
    """A batch is its rows run one at a time: each sequence keeps its own conv and SSM
    state (Section 4.1), and activations are normalised and quantised per row
    (Section 3.3).  Rows of different magnitudes and random states; a reduction over
    the wrong axis or a per-tensor quantiser scale mixes rows and fails this.  BLAS
    may sum a batch and a single row in different orders, so fp values agree to 1e-12
    and tokens and integer codes exactly."""
    d = S.LAYER_SMALL.with_batch(3)
    rng = np.random.default_rng(53)
    m = S.gen_model(rng, d, 2, 200)
    toks = np.array([5, 17, 123], dtype=np.int32)
    m.embed[17] = (m.embed[17].astype(np.float32) * 4).astype(np.float16)
    z = S.zero_state(d)
    states = [O.State(rng.normal(size=z.conv.shape).astype(z.conv.dtype),
                      rng.normal(0, 0.5, size=z.ssm.shape).astype(z.ssm.dtype)) for _ in m.layers]
    m1 = replace(m, dims=d.with_batch(1))
    single = [[O.State(st.conv[b:b + 1].copy(), st.ssm[b:b + 1].copy()) for st in states] for b in range(3)]
    tok = toks.copy()
    tok1 = [toks[b:b + 1].copy() for b in range(3)]
    for _ in range(3):
        tr = O.model_step(tok, m, states)
        for b in range(3):
            t1 = O.model_step(tok1[b], m1, single[b])
            assert tr.tokens[b] == t1.tokens[0]
            scale = np.max(np.abs(t1.logits))
            assert np.max(np.abs(tr.logits[b] - t1.logits[0])) <= 1e-12 * scale
            for l in range(len(m.layers)):
                np.testing.assert_allclose(tr.states[l].ssm[b], t1.states[l].ssm[0], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(tr.states[l].conv[b], t1.states[l].conv[0], rtol=1e-12, atol=1e-12)
            single[b] = t1.states
            tok1[b] = t1.tokens
        states = tr.states
        tok = tr.tokens
    x16 = (rng.normal(size=(3, 64)) * np.array([[0.01], [1.0], [30.0]])).astype(np.float16)
    q, sx = O.quantize_act(x16)
    for b in range(3):
        q1, sx1 = O.quantize_act(x16[b:b + 1])
        assert np.array_equal(q[b], q1[0]) and sx[b] == sx1[0]


def test_ssd_scan_strong_decay_stays_finite():
    """A strongly decaying head over a 64-token chunk (cumulative log-decay near -10^3):
    the scan must stay finite and equal the token recurrence (the state forgets its
    start, the output follows the last tokens)."""
    rng = np.random.default_rng(44)
    Bsz, T, H, P, N = 1, 64, 2, 3, 4
    h0 = rng.normal(size=(Bsz, H, P, N))
    x = rng.normal(size=(Bsz, T, H, P))
    Bm, Cm = rng.normal(size=(Bsz, T, N)), rng.normal(size=(Bsz, T, N))
    dt_raw = np.full((Bsz, T, H), 3.0)
    dt_bias = np.zeros(H, dtype=np.float32)
    A_log = np.array([np.log(16.0), 0.0], dtype=np.float32)
    D = np.ones(H, dtype=np.float32)
    y, hT = O.ssd_scan(h0, x, Bm, Cm, dt_raw, dt_bias, A_log, D, chunk=64)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(hT))
    h = h0.copy()
    for t in range(T):
        yt, h = O.ssm_step(h, x[:, t], Bm[:, t], Cm[:, t], dt_raw[:, t], dt_bias, A_log, D, state_dtype=np.float64)
        assert np.max(np.abs(y[:, t] - yt)) <= 1e-10 * max(1.0, np.max(np.abs(yt)))
    assert np.max(np.abs(hT - h)) <= 1e-10 * max(1.0, np.max(np.abs(h)))


# ---------------------------------------------------------------- density-field state codec

def test_df_field_size_matches_appendix_d():
    """Appendix D: K = 23 for d_state = 128 (field 23 x 23 = 529); Section 3.4: K^2 ~ 4 d_state."""
    assert O.df_field_size(128) == 23
    for n in range(1, 300):
        K = O.df_field_size(n)
        assert K * K >= 4 * n > (K - 1) * (K - 1)


def test_df_worked_example():
    """A two-value row worked by hand (tests/golden/df_codec_worked_example.json)."""
    g = json.load(open(os.path.join(GOLDEN, "df_codec_worked_example.json")))
    cells, lo, span = O.df_encode(np.array(g["row"]))
    assert O.df_field_size(len(g["row"])) == g["K"]
    assert cells.tolist() == g["cells"]
    assert float(lo) == g["lo"] and float(span) == g["span"]
    assert O.df_decode(cells, lo, span, 2).tolist() == g["decoded"]


def test_df_constant_row_is_exact():
    """A constant row has sigma 0: the readout is the value itself."""
    for c in (0.0, 1.5, -3.25, np.float32(0.1)):
        row = np.full(128, np.float64(np.float32(c)))
        assert np.array_equal(O.df_roundtrip(row), row)


def test_df_total_density_tracks_the_input():
    """First-order error feedback keeps the field's total density within half a cell
    of the normalised input's (plus the 8-bit rounding): the ones over the row, B,
    satisfy |B - 4 sum v| <= 0.5 + 4 n / 510.  Without the feedback (each cell
    rounded alone) the error grows with n."""
    rng = np.random.default_rng(11)
    for n in (16, 128):
        for _ in range(20):
            row = rng.normal(0.0, rng.uniform(0.1, 3.0), size=n) + rng.normal()
            cells, lo, span = O.df_encode(row)
            v = np.clip((row - np.float64(lo)) / np.float64(span), 0.0, 1.0)
            B = int(cells.sum())
            assert abs(B - 4 * v.sum()) <= 0.5 + 4 * n / 510.0 + 1e-9
            assert cells[4 * n:].sum() == 0          # spare cells stay empty


def test_df_readout_levels_and_clipping():
    """Every readout is lo + span k/4 (k = 0..4); values beyond mean +- 3 sigma clip
    to the field's ends."""
    rng = np.random.default_rng(12)
    row = rng.normal(size=128)
    row[5], row[77] = 50.0, -50.0                    # far outside mean +- 3 sigma
    cells, lo, span = O.df_encode(row)
    out = O.df_decode(cells, lo, span, 128)
    k = (out - np.float64(lo)) / np.float64(span) * 4
    assert np.allclose(k, np.rint(k), atol=1e-9) and k.min() >= 0 and k.max() <= 4
    assert out[5] == np.float64(lo) + np.float64(span) and out[77] == np.float64(lo)


def test_ssd_scan_df_only_at_interior_chunk_boundaries():
    """DF-SSD: with one chunk there is no interior boundary (identical to the plain
    scan); with two, the second chunk starts from the codec's readout of the first
    chunk's state."""
    rng = np.random.default_rng(13)
    B_, T, H, P, N = 1, 12, 2, 3, 4
    h0 = rng.normal(size=(B_, H, P, N))
    x = rng.normal(size=(B_, T, H, P))
    Bm, Cm = rng.normal(size=(B_, T, N)), rng.normal(size=(B_, T, N))
    dt_raw = rng.normal(size=(B_, T, H))
    dtb, Al, D = rng.normal(size=H), rng.uniform(0, 2, size=H), rng.normal(size=H)
    y1, h1 = O.ssd_scan(h0, x, Bm, Cm, dt_raw, dtb, Al, D, chunk=T, df=True)
    y0, h0_ = O.ssd_scan(h0, x, Bm, Cm, dt_raw, dtb, Al, D, chunk=T, df=False)
    assert np.array_equal(y1, y0) and np.array_equal(h1, h0_)
    ya, ha = O.ssd_scan(h0, x[:, :6], Bm[:, :6], Cm[:, :6], dt_raw[:, :6], dtb, Al, D, chunk=6)
    yb, hb = O.ssd_scan(O.df_roundtrip(ha), x[:, 6:], Bm[:, 6:], Cm[:, 6:], dt_raw[:, 6:], dtb, Al, D, chunk=6)
    y2, h2 = O.ssd_scan(h0, x, Bm, Cm, dt_raw, dtb, Al, D, chunk=6, df=True)
    assert np.allclose(y2, np.concatenate([ya, yb], axis=1), rtol=1e-12, atol=1e-12)
    assert np.allclose(h2, hb, rtol=1e-12, atol=1e-12)
