"""GPU parity of the prompt pass (prefill) against the oracle: one layer and the
whole model over prompts of T tokens (chunk boundaries of the 64-token scan at T =
63, 64, 65 and a multi-chunk T = 200), through the C ABI; the states it leaves are
then decoded from, and compared with, the oracle's token steps."""
import numpy as np
import pytest
import torch

from oracle import dfssm_oracle as O
from bit_scaffold_quantized_b200 import synth as S
from bit_scaffold_quantized_b200 import dfssm as F
from tests._util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    F.lib()


def _layer_case(d, T, seed, nonzero_state=True):
    rng = np.random.default_rng(seed)
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    if nonzero_state:
        st.conv[:] = rng.normal(size=st.conv.shape)
        st.ssm[:] = rng.normal(size=st.ssm.shape).astype(st.ssm.dtype)
    res = S.gen_layer_inputs(rng, d, T).transpose(1, 0, 2).copy()      # [B, T, D]
    return lw, st, res


def _run_layer_prefill(d, T, lw, st, res):
    dw = F.DeviceLayer.from_host(lw)
    ds = F.DeviceState.from_host(st)
    r = torch.from_numpy(res.copy()).to(DEV)
    ws = F.prefill_workspace(d, T)
    L = F.prefill_workspace_layout(d, T)
    F.layer_prefill(d, T, dw, ds, r, ws)
    torch.cuda.synchronize()
    assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) == 0
    return to_np(r), ds, ws, L


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_layer_prefill_parity(T):
    d = S.LAYER_SMALL.with_batch(2)
    lw, st, res = _layer_case(d, T, 50 + T)
    got, ds, ws, L = _run_layer_prefill(d, T, lw, st, res)
    tr = O.layer_prefill(res, lw, O.State(st.conv, st.ssm), d)
    BT, D, E = d.batch * T, d.d_model, d.d_inner
    assert np.array_equal(to_np(F.ws_view(ws, L.x_in, torch.float16, (BT, D))), tr.x_in.reshape(BT, D))
    errs = {
        "res": rel_err(got, tr.res),
        "conv": rel_err(to_np(ds.conv), tr.conv),
        "ssm": rel_err(to_np(ds.ssm), tr.ssm),
        "zxbcdt": rel_err(to_np(F.ws_view(ws, L.zxbcdt, torch.float64, (BT, d.in_rows))), tr.zxbcdt.reshape(BT, -1)),
        "xc": rel_err(to_np(F.ws_view(ws, L.xc, torch.float64, (BT, d.conv_dim))), tr.xc.reshape(BT, -1)),
        "g": rel_err(to_np(F.ws_view(ws, L.g, torch.float32, (BT, E))), tr.g.reshape(BT, E)),
    }
    assert max(errs.values()) <= TOL, errs
    # the projection's integer work is exact: the in_proj output agrees to fp64 rounding
    assert errs["zxbcdt"] <= 1e-12 and errs["xc"] <= 1e-12, errs
    # and the prompt pass tracks T decode steps of the oracle (states rounded per token)
    s = O.State(st.conv, st.ssm)
    for t in range(T):
        step = O.layer_step(res[:, t], lw, s, d)
        s = O.State(step.conv, step.ssm)
        assert rel_err(got[:, t], step.res) <= TOL, t
    assert rel_err(to_np(ds.ssm), s.ssm) <= TOL
    assert rel_err(to_np(ds.conv), s.conv) <= TOL


def test_layer_prefill_1p3b_shape_two_chunks():
    """The 1.3B layer shape (64 heads x 64, d_state 128, rank 32) over 65 tokens."""
    d = S.LAYER_1P3B
    T = 65
    lw, st, res = _layer_case(d, T, 60)
    got, ds, ws, L = _run_layer_prefill(d, T, lw, st, res)
    tr = O.layer_prefill(res, lw, O.State(st.conv, st.ssm), d)
    assert rel_err(got, tr.res) <= TOL
    assert rel_err(to_np(ds.ssm), tr.ssm) <= TOL
    assert rel_err(to_np(ds.conv), tr.conv) <= TOL


def test_layer_prefill_fp16_state():
    d = S.Dims(batch=2, d_model=256, d_inner=512, nheads=8, headdim=64, d_state=16, rank=8, ssm_state_dtype=1)
    T = 70
    lw, st, res = _layer_case(d, T, 61)
    got, ds, ws, L = _run_layer_prefill(d, T, lw, st, res)
    tr = O.layer_prefill(res, lw, O.State(st.conv, st.ssm), d)
    assert ds.ssm.dtype == torch.float16
    assert rel_err(got, tr.res) <= TOL and rel_err(to_np(ds.ssm), tr.ssm) <= TOL


def test_prefill_rejects_empty_prompt():
    d = S.LAYER_SMALL.with_batch(1)
    assert F.lib().dfssm_prefill_workspace_bytes(F.C.byref(F.cdims(d)), 0, 0, 0) == 0
    lw, st, res = _layer_case(d, 2, 62)
    dw, ds = F.DeviceLayer.from_host(lw), F.DeviceState.from_host(st)
    r = torch.from_numpy(res).to(DEV)
    ws = F.prefill_workspace(d, 2)
    with pytest.raises(F.DfssmError) as e:
        F.layer_prefill(d, 0, dw, ds, r, ws)
    assert e.value.code == F.ERR_INVALID_ARG


def test_model_prefill_then_decode():
    """A 2-layer model over a 70-token prompt (batch 2): last-token logits, greedy token
    and every layer's state against the oracle's prompt pass; then two decode tokens
    from the prefilled state against the oracle's token steps (teacher-forced)."""
    d = S.LAYER_SMALL.with_batch(2)
    rng = np.random.default_rng(63)
    m = S.gen_model(rng, d, 2, 1000)
    T = 70
    toks = rng.integers(0, 1000, size=(2, T)).astype(np.int32)
    dm = F.DeviceModel.from_host(m)
    states = [F.DeviceState.zeros(d) for _ in m.layers]
    ws = F.prefill_workspace(d, T, 2, 1000)
    L = F.prefill_workspace_layout(d, T, 2, 1000)
    tok_out = torch.zeros(2, dtype=torch.int32, device=DEV)
    logits = torch.zeros((2, 1000), dtype=torch.float32, device=DEV)
    F.model_prefill(dm, states, torch.from_numpy(toks).to(DEV), tok_out, ws, logits)
    torch.cuda.synchronize()
    assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) == 0
    ost = [O.State(*(lambda z: (z.conv, z.ssm))(S.zero_state(d))) for _ in m.layers]
    tr = O.model_prefill(toks, m, ost)
    assert rel_err(to_np(logits), tr.logits) <= TOL
    gl = to_np(logits)
    assert np.array_equal(to_np(tok_out), np.argmax(gl, axis=-1))
    for a, b in zip(states, tr.states):
        assert rel_err(to_np(a.ssm), b.ssm) <= TOL and rel_err(to_np(a.conv), b.conv) <= TOL
    # decode from the prompt's state
    call = F.ModelCall(dm, states)
    dws = F.workspace(d, 2, 1000)
    tok = tr.tokens.astype(np.int32)
    ost = tr.states
    for _ in range(2):
        tin = torch.from_numpy(tok).to(DEV)
        call(tin, tok_out, dws, logits)
        torch.cuda.synchronize()
        step = O.model_step(tok, m, ost)
        assert rel_err(to_np(logits), step.logits) <= TOL
        ost, tok = step.states, step.tokens
