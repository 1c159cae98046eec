"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same
seeded inputs.  Bit-exact for packing and for the int8 x int8 -> int32 low-rank
partials; max relative error <= 2e-3 for fp outputs and states."""
import time

import numpy as np
import pytest
import torch
from dataclasses import replace

from oracle import dfssm_oracle as O
from bit_scaffold_quantized_b200 import synth as S
from bit_scaffold_quantized_b200 import dfssm as F
from tests._util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
FAITHFUL = 1e-6   # observed-agreement bound for fp32 outputs of an exact/fp64 pipeline


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    F.lib()


def _sync():
    torch.cuda.synchronize()


# ---------------------------------------------------------------- packing

@pytest.mark.parametrize("rows,cols", [(64, 512), (1064, 256), (8512, 2048)])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_pack_bit_exact(rows, cols, dtype):
    rng = np.random.default_rng(rows * 7 + cols)
    w = rng.normal(size=(rows, cols)).astype(dtype)
    w.flat[rng.choice(w.size, 64, replace=False)] = 0.0
    w.flat[rng.choice(w.size, 64, replace=False)] = -0.0
    wt = torch.from_numpy(w).to(DEV)
    for layout in (F.LAYOUT_ROWMAJOR, F.LAYOUT_TILED):
        out = torch.full((F.packed_words(rows, cols, layout),), -1, dtype=torch.int32, device=DEV)
        F.pack_weights(wt, rows, cols, layout, out)
        _sync()
        got = to_np(out).view(np.uint32)
        ref = O.pack_signs(w)
        if layout == F.LAYOUT_TILED:
            ref = O.tile_signs(ref, rows, cols)
        assert np.array_equal(got, ref.ravel())


@pytest.mark.parametrize("rows,cols", [(16, 256), (40, 512), (1064, 256), (2048, 4096)])
def test_repack_bit_exact(rows, cols):
    rng = np.random.default_rng(rows + cols)
    bits = rng.integers(0, 2 ** 32, size=(rows, cols // 32), dtype=np.uint64).astype(np.uint32)
    src = torch.from_numpy(bits.view(np.int32)).to(DEV)
    out = torch.full((F.packed_words(rows, cols, F.LAYOUT_TILED),), -1, dtype=torch.int32, device=DEV)
    F.repack_bits(src, rows, cols, out)
    _sync()
    assert np.array_equal(to_np(out).view(np.uint32), O.tile_signs(bits, rows, cols))


# ---------------------------------------------------------------- projection (Eq. 3)

def _proj_case(p, x, rank):
    dp = F.DeviceProj.from_host(p)
    xt = torch.from_numpy(x).to(DEV)
    y = torch.full((x.shape[0], p.rows), np.nan, dtype=torch.float32, device=DEV)
    ws = F.proj_workspace(p.rows, p.cols, rank, x.shape[0])
    F.proj_forward(dp, rank, xt, y, ws)
    _sync()
    L = F.proj_workspace_layout(p.rows, p.cols, rank, x.shape[0])
    ref = O.project(x, p)
    e = rel_err(to_np(y), ref.y)
    assert e <= TOL, e
    assert e <= FAITHFUL, e      # exact scaffold + fp64 epilogue: only the final fp32 rounding differs
    B = x.shape[0]
    _check_digits(to_np(F.ws_view(ws, L.xd_in, torch.int8, (B, 6, p.cols))),
                  to_np(F.ws_view(ws, L.xdsum_in, torch.int32, (B, 6))), x)
    if rank:
        xq = to_np(F.ws_view(ws, L.xq_in, torch.int8, (B, p.cols)))
        sx = to_np(F.ws_view(ws, L.sx_in, torch.float32, (B,)))
        acc = to_np(F.ws_view(ws, L.acc_in, torch.int32, (B, rank)))
        assert np.array_equal(xq, ref.xq)
        assert np.array_equal(sx, ref.sx)
        assert np.array_equal(acc.astype(np.int64), ref.acc)
    return to_np(y), ref


def _check_digits(xd, xdsum, x16):
    """Digit planes are an exact balanced base-256 representation of x * 2^24."""
    X = (x16.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    rec = np.zeros_like(X)
    for dd in range(5, -1, -1):
        rec = rec * 256 + xd[:, dd, :].astype(np.int64)
    assert np.array_equal(rec, X)
    assert np.array_equal(xdsum.astype(np.int64), xd.astype(np.int64).sum(axis=2))


@pytest.mark.parametrize("d_in,d_out", S.PROJ_SWEEP_SHAPES)
@pytest.mark.parametrize("rank", S.PROJ_SWEEP_RANKS)
@pytest.mark.parametrize("batch", S.PROJ_SWEEP_BATCHES)
def test_proj_sweep_parity(d_in, d_out, rank, batch):
    p, x = S.proj_workload(d_in, d_out, rank, batch)
    _proj_case(p, x, rank)


@pytest.mark.parametrize("rows,cols,rank,batch", [(1064, 256, 8, 3), (40, 512, 0, 9), (17, 256, 4, 1),
                                                   (8512, 2048, 32, 13)])
def test_proj_ragged_and_rank0(rows, cols, rank, batch):
    rng = np.random.default_rng(rows + cols + rank + batch)
    p = S.gen_proj(rng, rows, cols, rank)
    x = rng.normal(size=(batch, cols)).astype(np.float16)
    if batch > 1:
        x[1] = 0          # all-zero activation row: codes 0, scale 1
    _proj_case(p, x, rank)


def test_proj_all_plus_one_gives_alpha_sum():
    rng = np.random.default_rng(5)
    p = S.gen_proj(rng, 48, 512, 0)
    p.bits[:] = 0xFFFFFFFF
    x = rng.normal(size=(2, 512)).astype(np.float16)
    y, _ = _proj_case(p, x, 0)
    closed = p.alpha.astype(np.float64)[None] * x.astype(np.float64).sum(1, keepdims=True)
    assert rel_err(y, closed) <= 1e-5


def test_proj_rank0_bit_identical_to_zero_B():
    rng = np.random.default_rng(6)
    p = S.gen_proj(rng, 256, 1024, 16)
    x = rng.normal(size=(1, 1024)).astype(np.float16)
    p0 = S.ProjWeights(p.rows, p.cols, p.bits, p.alpha, None, None, None, None)
    pz = S.ProjWeights(p.rows, p.cols, p.bits, p.alpha, p.A, p.sA, np.zeros_like(p.B), p.sB)
    y0, _ = _proj_case(p0, x, 0)
    yz, _ = _proj_case(pz, x, 16)
    assert np.array_equal(y0, yz)


# ---------------------------------------------------------------- layer step

# small shape the batch-1 persistent kernel accepts (nheads and d_state multiples of 16)
LAYER_SMALL_P = S.Dims(batch=1, d_model=256, d_inner=512, nheads=16, headdim=32, d_state=16, rank=8)


class LayerRun:
    def __init__(self, d, lw, st):
        self.d = d
        self.dw = F.DeviceLayer.from_host(lw)
        self.ds = F.DeviceState.from_host(st)
        self.ws = F.workspace(d)
        self.L = F.workspace_layout(d)

    def step(self, res_np):
        res = torch.from_numpy(np.ascontiguousarray(res_np)).to(DEV)
        F.layer_step(self.d, self.dw, self.ds, res, self.ws)
        _sync()
        assert int(self.view("status", torch.int32, (1,))[0]) == 0
        return to_np(res)

    def view(self, name, dtype, shape):
        return to_np(F.ws_view(self.ws, getattr(self.L, name), dtype, shape))


def _check_layer_step(run, lw, d, ost, res_in):
    got = run.step(res_in)
    t = O.layer_step(res_in, lw, ost, d)
    B, D, E = d.batch, d.d_model, d.d_inner
    errs = {
        "res": rel_err(got, t.res),
        "conv": rel_err(to_np(run.ds.conv), t.conv),
        "ssm": rel_err(to_np(run.ds.ssm), t.ssm),
        "zxbcdt": rel_err(run.view("zxbcdt", torch.float64, (B, d.in_rows)), t.zxbcdt),
        "xc": rel_err(run.view("xc", torch.float64, (B, d.conv_dim)), t.xc),
        "g": rel_err(run.view("g", torch.float32, (B, E)), t.g),
    }
    bad = {k: v for k, v in errs.items() if v > TOL}
    assert not bad, bad
    loose = {k: v for k, v in errs.items() if v > FAITHFUL}
    assert not loose, loose
    # fp16 activations entering the projections: identical to the oracle's
    assert np.array_equal(run.view("x_in", torch.float16, (B, D)), t.x_in)
    assert np.array_equal(run.view("x_out", torch.float16, (B, E)), t.x_out)
    if d.rank:
        # int8 codes, scales and int8 x int8 -> int32 partials: bit-exact
        for pre, tr in (("in", t.proj_in), ("out", t.proj_out)):
            K = D if pre == "in" else E
            assert np.array_equal(run.view(f"xq_{pre}", torch.int8, (B, K)), tr.xq)
            assert np.array_equal(run.view(f"sx_{pre}", torch.float32, (B,)), tr.sx)
            assert np.array_equal(run.view(f"acc_{pre}", torch.int32, (B, d.rank)).astype(np.int64), tr.acc)
    _check_digits(run.view("xd_in", torch.int8, (B, 6, D)), run.view("xdsum_in", torch.int32, (B, 6)), t.x_in)
    return t


@pytest.mark.parametrize("name,steps", [("layer_d256_b1_16steps", 16), ("layer_d2048_b1_256steps", 48)])
def test_layer_step_parity(name, steps):
    d, lw, st, xs = S.layer_workload(name, steps=steps)
    run = LayerRun(d, lw, st)
    ost = st
    for t in range(steps):
        tr = _check_layer_step(run, lw, d, ost, xs[t])
        ost = O.State(tr.conv, tr.ssm)


def test_layer_step_persistent_small_parity():
    rng = np.random.default_rng(40)
    d = LAYER_SMALL_P
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    xs = S.gen_layer_inputs(rng, d, 12)
    assert F.launches_per_decode_step(d, 1, 1000) == 1      # takes the persistent kernel
    run = LayerRun(d, lw, st)
    ost = st
    for t in range(12):
        tr = _check_layer_step(run, lw, d, ost, xs[t])
        ost = O.State(tr.conv, tr.ssm)


@pytest.mark.parametrize("batch", [9, 16])
def test_layer_step_batched_parity(batch):
    d, lw, st, xs = S.layer_workload("layer_d256_b1_16steps", steps=4, batch=batch)
    run = LayerRun(d, lw, st)
    ost = st
    for t in range(4):
        tr = _check_layer_step(run, lw, d, ost, xs[t])
        ost = O.State(tr.conv, tr.ssm)


def test_layer_step_1p3b_batched_parity():
    """The 1.3B layer at batch 3: cluster prologue at K = 2048 and 4096 with rank 32,
    4-row projection tiles with a ragged batch tile, streaming SSM with N = 128."""
    d, lw, st, xs = S.layer_workload("layer_d2048_b1_256steps", steps=2, batch=3)
    run = LayerRun(d, lw, st)
    ost = st
    for t in range(2):
        tr = _check_layer_step(run, lw, d, ost, xs[t])
        ost = O.State(tr.conv, tr.ssm)


@pytest.mark.parametrize("headdim,d_state,rank", [(64, 256, 8), (128, 128, 0)])
def test_layer_step_large_state_items_parity(headdim, d_state, rank):
    """(batch, head) state items too large for two shared-memory buffers take the
    one-block-per-item SSM kernel (d_state 256 also takes its two-chunk form);
    rank 0 runs the prologue without LoRA rows."""
    d = S.Dims(batch=2, d_model=256, d_inner=512, nheads=512 // headdim, headdim=headdim, d_state=d_state,
               rank=rank)
    rng = np.random.default_rng(41 + headdim)
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    xs = S.gen_layer_inputs(rng, d, 3)
    run = LayerRun(d, lw, st)
    ost = st
    for t in range(3):
        tr = _check_layer_step(run, lw, d, ost, xs[t])
        ost = O.State(tr.conv, tr.ssm)


@pytest.mark.parametrize("name,batch", [("layer_d256_b1_16steps", 3), ("layer_d2048_b1_256steps", 2)])
def test_layer_step_fp16_state_parity(name, batch):
    """Half-precision SSM state (streaming kernel, fp64 update rounded once to fp16);
    the oracle stores the same rounding, so states compare exactly up to rounding-order
    differences far below an fp16 ulp."""
    d, lw, st, xs = S.layer_workload(name, steps=3, batch=batch)
    d = replace(d, ssm_state_dtype=1)
    st = S.zero_state(d)
    assert st.ssm.dtype == np.float16
    run = LayerRun(d, lw, st)
    ost = st
    for t in range(3):
        tr = _check_layer_step(run, lw, d, ost, xs[t])
        assert tr.ssm.dtype == np.float16 and run.ds.ssm.dtype == torch.float16
        assert np.array_equal(to_np(run.ds.ssm), tr.ssm)
        ost = O.State(tr.conv, tr.ssm)


def test_model_decode_fp16_state_parity():
    """Batch-1 model with fp16 state takes the multi-launch path and matches the oracle."""
    d = replace(LAYER_SMALL_P, ssm_state_dtype=1)
    rng = np.random.default_rng(37)
    m = S.gen_model(rng, d, 3, 1000)
    assert F.launches_per_decode_step(d, 3, 1000) > 1
    _teacher_forced(m, S.gen_tokens(rng, 1, 1000), 4)


def test_layer_dt_zero_leaves_ssm_state():
    d, lw, st, xs = S.layer_workload("layer_d256_b1_16steps", steps=2)
    lw.dt_bias[:] = -1e4
    rng = np.random.default_rng(3)
    st.ssm[:] = rng.normal(size=st.ssm.shape)
    run = LayerRun(d, lw, st)
    run.step(xs[0])
    assert np.array_equal(to_np(run.ds.ssm), st.ssm)


def test_layer_graph_replay_matches_eager():
    d, lw, st, xs = S.layer_workload("layer_d2048_b1_256steps", steps=6)
    eager = LayerRun(d, lw, st)
    outs = [eager.step(xs[t]) for t in range(6)]
    g_run = LayerRun(d, lw, st)
    res = torch.zeros((d.batch, d.d_model), dtype=torch.float32, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        res.copy_(torch.from_numpy(xs[0]).to(DEV))
        F.layer_step(d, g_run.dw, g_run.ds, res, g_run.ws)    # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    _sync()
    # restore state, then capture one step and replay it
    g_run.ds.conv.zero_(); g_run.ds.ssm.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        F.layer_step(d, g_run.dw, g_run.ds, res, g_run.ws)
    for t in range(6):
        res.copy_(torch.from_numpy(xs[t]).to(DEV))
        graph.replay()
        _sync()
        assert np.array_equal(to_np(res), outs[t])
    assert np.array_equal(to_np(g_run.ds.ssm), to_np(eager.ds.ssm))


def test_state_checkpoint_resume_bit_identical():
    d, lw, st, xs = S.layer_workload("layer_d256_b1_16steps", steps=8)
    run = LayerRun(d, lw, st)
    for t in range(4):
        run.step(xs[t])
    saved = (run.ds.conv.clone(), run.ds.ssm.clone())
    first = [run.step(xs[t]) for t in range(4, 8)]
    run.ds.conv.copy_(saved[0]); run.ds.ssm.copy_(saved[1])
    again = [run.step(xs[t]) for t in range(4, 8)]
    for a, b in zip(first, again):
        assert np.array_equal(a, b)


# ---------------------------------------------------------------- model decode

def _teacher_forced(m, tok0, steps, n_check_tokens=True, head="fp16", all_layers=False):
    d = m.dims
    dm = F.DeviceModel.from_host(m, head=head)
    emb_q = None
    if head == "int8":
        emb_q = O.quantize_embedding(m.embed)
        # the device quantiser takes the oracle's integer decisions
        assert np.array_equal(to_np(dm.embed_q), emb_q[0])
        assert np.array_equal(to_np(dm.embed_scale), emb_q[1])
    states = [F.DeviceState.zeros(d) for _ in m.layers]
    call = F.ModelCall(dm, states)
    ws = F.workspace(d, len(m.layers), m.vocab)
    L = F.workspace_layout(d, len(m.layers), m.vocab)
    tok_in = torch.from_numpy(tok0.astype(np.int32)).to(DEV)
    tok_out = torch.zeros(d.batch, dtype=torch.int32, device=DEV)
    logits = torch.zeros((d.batch, m.vocab), dtype=torch.float32, device=DEV)
    ost = [S.zero_state(d) for _ in m.layers]
    ost = [O.State(s.conv, s.ssm) for s in ost]
    tok = tok0.astype(np.int32)
    for t in range(steps):
        tok_in.copy_(torch.from_numpy(tok).to(DEV))
        call(tok_in, tok_out, ws, logits)
        _sync()
        assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) == 0
        tr = O.model_step(tok, m, ost, emb_q=emb_q)
        e = rel_err(to_np(logits), tr.logits)
        assert e <= TOL, (t, e)
        for l in (range(len(m.layers)) if all_layers else (0, len(m.layers) - 1)):
            assert rel_err(to_np(states[l].ssm), tr.states[l].ssm) <= TOL, (t, l)
            assert rel_err(to_np(states[l].conv), tr.states[l].conv) <= TOL, (t, l)
        got = to_np(tok_out)
        gl = to_np(logits)
        assert np.array_equal(got, np.argmax(gl, axis=-1))          # argmax of its own logits
        for b in range(d.batch):
            if got[b] != tr.tokens[b]:
                top = np.sort(tr.logits[b])[-2:]
                assert top[1] - top[0] <= 4 * TOL * np.sqrt(np.mean(tr.logits[b] ** 2))
        ost = tr.states
        tok = tr.tokens


def test_model_decode_small_persistent_parity():
    rng = np.random.default_rng(31)
    m = S.gen_model(rng, LAYER_SMALL_P, 3, 1000)
    assert F.launches_per_decode_step(LAYER_SMALL_P, 3, 1000) == 1
    _teacher_forced(m, S.gen_tokens(rng, 1, 1000), 6)


def test_model_decode_small_parity():
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(30)
    m = S.gen_model(rng, d, 3, 1000)
    _teacher_forced(m, S.gen_tokens(rng, 2, 1000), 6)


def test_model_decode_batched_tc_head_parity():
    """Batch 12: the tensor-core LM head with 16 batch rows per block (a ragged second
    n-tile) and a vocabulary whose last 16-row tile is half empty."""
    d = S.LAYER_SMALL.with_batch(12)
    rng = np.random.default_rng(34)
    m = S.gen_model(rng, d, 3, 1000)
    _teacher_forced(m, S.gen_tokens(rng, 12, 1000), 4)


def test_quantize_rows_int8_bit_exact():
    """Per-row int8 quantiser (Section 3.3) against the oracle: zero row, exact
    half-way codes, the largest fp16, subnormals, and random rows."""
    rng = np.random.default_rng(35)
    w = rng.normal(0.0, 0.02, size=(37, 512)).astype(np.float16)
    w[3] = 0
    w[4, :4] = [127.0, 2.5, -3.5, 0.5]          # scale 1: codes 127, 2, -4, 0 (half-even)
    w[4, 4:] = 0
    w[5, 0], w[5, 1] = np.float16(65504.0), np.float16(-65504.0)
    w[6] = np.float16(2.0 ** -24) * rng.integers(-3, 4, size=512)
    q, sc = F.quantize_rows_int8(torch.from_numpy(w).to(DEV))
    _sync()
    rq, rs = O.quantize_embedding(w)
    assert np.array_equal(to_np(q), rq)
    assert np.array_equal(to_np(sc), rs)
    assert to_np(q)[4, :4].tolist() == [127, 2, -4, 0]


@pytest.mark.parametrize("case", ["persistent_b1", "multi_b2", "multi_b12"])
def test_model_decode_int8_head_parity(case):
    """The int8 per-row embedding / tied LM head on both paths and all head kernels."""
    rng = np.random.default_rng(36)
    if case == "persistent_b1":
        d = LAYER_SMALL_P
    else:
        d = S.LAYER_SMALL.with_batch(2 if case == "multi_b2" else 12)
    m = S.gen_model(rng, d, 3, 1000)
    assert (F.launches_per_decode_step(d, 3, 1000) == 1) == (case == "persistent_b1")
    _teacher_forced(m, S.gen_tokens(rng, d.batch, 1000), 4, head="int8")


def test_model_decode_1p3b_int8_head_parity():
    m, tok = S.model_workload("model_48x2048_v50280_b1_greedy512")
    assert F.launches_per_decode_step(m.dims, len(m.layers), m.vocab) == 1
    _teacher_forced(m, tok, 2, head="int8")


def test_model_decode_1p3b_parity():
    """The benchmark's own launch configuration (48 layers, batch 1, the single-launch
    token kernel) over 8 teacher-forced tokens, every layer's SSM and conv state
    compared after every token."""
    m, tok = S.model_workload("model_48x2048_v50280_b1_greedy512")
    # the benchmark shape must take the single-launch persistent kernel
    assert F.launches_per_decode_step(m.dims, len(m.layers), m.vocab) == 1
    _teacher_forced(m, tok, 8, all_layers=True)


def test_model_decode_silent_layers_repeat_token_1p3b():
    """A property that holds at any size, checked at the benchmark's shape and in its
    launch configuration (the single-launch token kernel) without running the oracle.
    Every out_proj is scaled to zero, the embedding rows have equal norms and the
    final-norm weight is a constant c.  The residual therefore stays the token's
    embedding row through the 48 layers.  The tied head's argmax is the token itself,
    with logit c |e|^2 / sqrt(|e|^2 / D + eps), so greedy decode repeats it.  The SSM
    states still move."""
    rng = np.random.default_rng(61)
    d = S.LAYER_1P3B
    m = S.silent_model(rng, d, S.N_LAYER_1P3B, S.VOCAB_1P3B)
    assert F.launches_per_decode_step(d, len(m.layers), m.vocab) == 1
    dm = F.DeviceModel.from_host(m)
    states = [F.DeviceState.zeros(d) for _ in m.layers]
    call = F.ModelCall(dm, states)
    ws = F.workspace(d, len(m.layers), m.vocab)
    L = F.workspace_layout(d, len(m.layers), m.vocab)
    t0 = 31337
    tok = torch.tensor([t0], dtype=torch.int32, device=DEV)
    logits = torch.zeros((1, m.vocab), dtype=torch.float32, device=DEV)
    e2 = float(np.sum(m.embed[t0].astype(np.float64) ** 2))
    own = 1.5 * e2 / np.sqrt(e2 / d.d_model + O.EPS)
    for _ in range(6):
        call(tok, tok, ws, logits)
        _sync()
        assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) == 0
        assert int(to_np(tok)[0]) == t0
        gl = to_np(logits)[0]
        assert gl[t0] == pytest.approx(own, rel=1e-5)
        assert np.max(np.delete(gl, t0)) < 0.5 * own
    assert all(float(np.max(np.abs(to_np(s.ssm)))) > 0 for s in states)


@pytest.mark.parametrize("batch", [16, 64])
def test_model_decode_silent_layers_repeat_tokens_48x2048_batched(batch):
    """The silent-layers closed form at the batched decode workloads' full shape (48
    layers, d_model 2048, vocab 50280) on the multi-launch path, no oracle run: every
    batch row must repeat its own token, and every row's own-token logit is the same
    c |e|^2 / sqrt(|e|^2 / D + eps) (all embedding rows have one norm)."""
    rng = np.random.default_rng(62)
    d = S.LAYER_1P3B.with_batch(batch)
    m = S.silent_model(rng, d, S.N_LAYER_1P3B, S.VOCAB_1P3B)
    assert F.launches_per_decode_step(d, len(m.layers), m.vocab) > 1
    dm = F.DeviceModel.from_host(m)
    states = [F.DeviceState.zeros(d) for _ in m.layers]
    call = F.ModelCall(dm, states)
    ws = F.workspace(d, len(m.layers), m.vocab)
    L = F.workspace_layout(d, len(m.layers), m.vocab)
    t0 = rng.choice(m.vocab, size=batch, replace=False).astype(np.int32)
    tok_in = torch.from_numpy(t0).to(DEV)
    tok_out = torch.zeros(batch, dtype=torch.int32, device=DEV)
    logits = torch.zeros((batch, m.vocab), dtype=torch.float32, device=DEV)
    e2 = float(np.sum(m.embed[0].astype(np.float64) ** 2))
    own = 1.5 * e2 / np.sqrt(e2 / d.d_model + O.EPS)
    rows = np.arange(batch)
    for _ in range(3):
        call(tok_in, tok_out, ws, logits)
        _sync()
        assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) == 0
        assert np.array_equal(to_np(tok_out), t0)
        gl = to_np(logits).copy()
        np.testing.assert_allclose(gl[rows, t0], own, rtol=1e-5)
        gl[rows, t0] = -np.inf
        assert np.max(gl) < 0.5 * own
        tok_in.copy_(tok_out)
    assert all(float(np.max(np.abs(to_np(s.ssm)))) > 0 for s in states)


def test_model_decode_1p3b_b16_parity():
    """The batched decode workload at its own shape ("Density Field State Space
    Models", Section 4.3, Table 2: batched decode): 48 layers, d_model 2048, batch 16,
    random token ids as the prompt, the multi-launch path with the 16-row tensor-core
    LM head; every layer's state after every step."""
    m, tok = S.model_workload("model_48x2048_v50280_b16_256steps")
    assert m.dims.batch == 16
    assert F.launches_per_decode_step(m.dims, len(m.layers), m.vocab) == 1 + 5 * 48 + 2
    _teacher_forced(m, tok, 2, all_layers=True)


def test_model_decode_1p3b_b64_parity():
    """Batch 64 at the 1.3B layer shape and the full vocabulary (the batch-64 decode
    workload's kernels: the 2 x 16-row tensor-core LM head, the streamed SSM grid over
    64 x 64 items), with 4 of its 48 layers to keep the oracle's time bounded."""
    w = S.WORKLOADS["model_48x2048_v50280_b64_256steps"]
    rng = np.random.default_rng(w["seed"])
    m = S.gen_model(rng, w["dims"], 4, w["vocab"])
    tok = S.gen_tokens(rng, 64, w["vocab"])
    _teacher_forced(m, tok, 2, all_layers=True)


def test_bounded_wait_runs_out_and_is_reported():
    """Failure detection without a GPU fault: the workspace's test hooks make CTA 0
    withhold its layer-0 residual words and bound every wait at 4096 polls.  The next
    layer's gather runs out: the call returns promptly with status value 4 (the
    residual gather) and the abort flag set, every CTA having left the token; a later
    call on the same workspace refuses to run (status value 1); a fresh workspace and
    state decode oracle-exact again."""
    rng = np.random.default_rng(37)
    m = S.gen_model(rng, LAYER_SMALL_P, 3, 1000)
    d = m.dims
    assert F.launches_per_decode_step(d, 3, 1000) == 1
    dm = F.DeviceModel.from_host(m)
    states = [F.DeviceState.zeros(d) for _ in m.layers]
    call = F.ModelCall(dm, states)
    ws = F.workspace(d, 3, 1000)
    L = F.workspace_layout(d, 3, 1000)
    ctl = F.ws_view(ws, L.control, torch.int32, (4,))
    ctl[2] = 1
    ctl[3] = 4096
    tok = torch.from_numpy(S.gen_tokens(rng, 1, 1000)).to(DEV)
    out = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.time()
    call(tok, out, ws, None)
    _sync()
    assert time.time() - t0 < 60
    status = int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0])
    assert status & 4, status
    assert int(to_np(ctl)[1]) == 1
    ctl[2] = 0
    ctl[3] = 0
    call(tok, out, ws, None)
    _sync()
    assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) & 1
    _teacher_forced(m, S.gen_tokens(rng, 1, 1000), 2)


@pytest.fixture
def tc_path(monkeypatch):
    """Batched projections on the tcgen05 kernel (k_proj_tc) for the test's calls."""
    monkeypatch.setenv("DFSSM_PROJ_PATH", "tc")


@pytest.mark.parametrize("d_in,d_out,rank,batch", [(2048, 8512, 32, 16), (4096, 2048, 32, 64), (256, 1064, 8, 40),
                                                   (2048, 8512, 64, 256), (256, 48, 0, 3), (1024, 48, 16, 5),
                                                   (8192, 256, 128, 33)])
def test_proj_tcgen05_parity(tc_path, d_in, d_out, rank, batch):
    """The tcgen05 tile kernel against the oracle: int8 codes / partials bit-exact, the
    projection to fp32 rounding; ragged M tiles (1064, 48 rows) and batch groups (40,
    33 rows), K split over clusters of 2, 4 and 8 CTAs (8512 rows at batch 16, 2048 at
    64, 48 rows at K 1024, 256 rows at K 8192), LoRA ranks 0 to 128."""
    if rank:
        p, x = S.proj_workload(d_in, d_out, rank, batch)
    else:
        rng = np.random.default_rng(7)
        p = S.gen_proj(rng, d_out, d_in, 0)
        x = rng.normal(size=(batch, d_in)).astype(np.float16)
    _proj_case(p, x, rank)


@pytest.fixture
def mma_path(monkeypatch):
    """Batched projections on the mma.sync kernel (k_proj) for the test's calls."""
    monkeypatch.setenv("DFSSM_PROJ_PATH", "mma")


@pytest.mark.parametrize("d_in,d_out,rank,batch", [(2048, 8512, 32, 64), (4096, 2048, 64, 16)])
def test_proj_mma_forced_parity(mma_path, d_in, d_out, rank, batch):
    """The mma.sync kernel at batches where tcgen05 is the default."""
    p, x = S.proj_workload(d_in, d_out, rank, batch)
    _proj_case(p, x, rank)


def test_model_decode_mma_batched_parity(mma_path):
    """A 2-layer 1.3B-shaped model at batch 16 with every projection on k_proj."""
    w = S.WORKLOADS["model_48x2048_v50280_b16_256steps"]
    rng = np.random.default_rng(w["seed"] + 1)
    m = S.gen_model(rng, w["dims"], 2, w["vocab"])
    _teacher_forced(m, S.gen_tokens(rng, 16, w["vocab"]), 2, all_layers=True)


def test_model_decode_tcgen05_batched_parity(tc_path):
    """A 3-layer small model at batch 12 and a 2-layer 1.3B-shaped one at batch 16,
    decoded with every projection on the tcgen05 kernel."""
    d = S.LAYER_SMALL.with_batch(12)
    rng = np.random.default_rng(38)
    m = S.gen_model(rng, d, 3, 1000)
    _teacher_forced(m, S.gen_tokens(rng, 12, 1000), 3)
    w = S.WORKLOADS["model_48x2048_v50280_b16_256steps"]
    rng = np.random.default_rng(w["seed"])
    m = S.gen_model(rng, w["dims"], 2, w["vocab"])
    _teacher_forced(m, S.gen_tokens(rng, 16, w["vocab"]), 2, all_layers=True)
