"""GPU parity of the density-field state codec ("Density Field State Space Models",
Section 3.4 and Appendix D) against the oracle: the fields (cells, lo, span) are
bit-exact and so is the fp32 readout; the prompt pass with the codec at its chunk
boundaries (DF-SSD) matches the oracle's."""
from dataclasses import replace

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


def _rows(n, seed):
    """Rows of every kind the codec meets: scaled and shifted normals, constants,
    zeros, rows with far outliers, a two-level row."""
    rng = np.random.default_rng(seed)
    rows = [rng.normal(rng.normal(), rng.uniform(0.01, 5.0), size=n) for _ in range(200)]
    rows += [np.full(n, c) for c in (0.0, 1.0, -2.5, 3e-5)]
    for _ in range(20):
        r = rng.normal(size=n)
        r[rng.integers(n)] = 100.0 * rng.choice([-1, 1])
        rows.append(r)
    rows.append(np.where(np.arange(n) % 2 == 0, -1.0, 1.0))
    return np.asarray(rows, dtype=np.float32)


@pytest.mark.parametrize("n", [128, 16, 7, 1])
def test_df_encode_decode_parity(n):
    rows = _rows(n, 70 + n)
    R = rows.shape[0]
    W = F.df_field_words(n)
    K = O.df_field_size(n)
    assert W == (K * K + 31) // 32
    x = torch.from_numpy(rows).to(DEV)
    cells = torch.zeros((R, W), dtype=torch.int32, device=DEV)
    lo = torch.zeros(R, dtype=torch.float32, device=DEV)
    span = torch.zeros(R, dtype=torch.float32, device=DEV)
    out = torch.zeros_like(x)
    F.df_encode(x, cells, lo, span, out)
    back = torch.zeros_like(x)
    F.df_decode(cells, lo, span, back)
    torch.cuda.synchronize()
    words = to_np(cells).view(np.uint32)
    bits = ((words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(R, -1)[:, :K * K]
    lo_g, span_g, out_g, back_g = to_np(lo), to_np(span), to_np(out), to_np(back)
    for r in range(R):
        c, l, s = O.df_encode(rows[r].astype(np.float64))
        assert np.array_equal(bits[r], c), r
        assert lo_g[r] == l and span_g[r] == s, r
        ref = O.df_decode(c, l, s, n).astype(np.float32)
        assert np.array_equal(out_g[r], ref) and np.array_equal(back_g[r], ref), r


def _prefill(d, T, lw, st, res):
    dw = F.DeviceLayer.from_host(lw)
    ds = F.DeviceState.from_host(st)
    r = torch.from_numpy(res.copy()).to(DEV)
    ws = F.prefill_workspace(d, T)
    L = F.prefill_workspace_layout(d, T)
    F.layer_prefill(d, T, dw, ds, r, ws)
    torch.cuda.synchronize()
    assert int(to_np(F.ws_view(ws, L.status, torch.int32, (1,)))[0]) == 0
    return to_np(r), ds, ws, L


def _layer_case(d, T, seed):
    rng = np.random.default_rng(seed)
    lw = S.gen_layer(rng, d)
    st = S.zero_state(d)
    st.conv[:] = rng.normal(size=st.conv.shape)
    st.ssm[:] = rng.normal(size=st.ssm.shape).astype(st.ssm.dtype)
    res = S.gen_layer_inputs(rng, d, T).transpose(1, 0, 2).copy()
    return lw, st, res


@pytest.mark.parametrize("T", [64, 65, 200])
def test_layer_prefill_df_parity(T):
    """DF-SSD through the C ABI: no codec at T = 64 (one chunk), one boundary at 65,
    three at 200; the per-token residuals, g and the final states match the oracle's
    layer_prefill(df=True), and from 65 on differ from the exact scan."""
    d = S.LAYER_SMALL.with_batch(2)
    dd = replace(d, df_chunk_codec=1)
    lw, st, res = _layer_case(d, T, 90 + T)
    got, ds, ws, L = _prefill(dd, T, lw, st, res)
    tr = O.layer_prefill(res, lw, O.State(st.conv, st.ssm), d, df=True)
    BT, E = d.batch * T, d.d_inner
    errs = {
        "res": rel_err(got, tr.res),
        "ssm": rel_err(to_np(ds.ssm), tr.ssm),
        "conv": rel_err(to_np(ds.conv), tr.conv),
        "g": rel_err(to_np(F.ws_view(ws, L.g, torch.float32, (BT, E))), tr.g.reshape(BT, E)),
    }
    assert max(errs.values()) <= TOL, errs
    plain = O.layer_prefill(res, lw, O.State(st.conv, st.ssm), d, df=False)
    if T > 64:
        assert rel_err(tr.res, plain.res) > 1e-4
    else:
        assert np.array_equal(tr.res, plain.res)


def test_layer_prefill_df_1p3b_shape():
    """The 1.3B layer shape (d_state 128: K = 23) over 65 tokens with the codec."""
    d = S.LAYER_1P3B
    T = 65
    dd = replace(d, df_chunk_codec=1)
    lw, st, res = _layer_case(d, T, 95)
    got, ds, ws, L = _prefill(dd, T, lw, st, res)
    tr = O.layer_prefill(res, lw, O.State(st.conv, st.ssm), d, df=True)
    assert rel_err(got, tr.res) <= TOL
    assert rel_err(to_np(ds.ssm), tr.ssm) <= TOL


def test_df_flag_is_validated():
    d = S.LAYER_SMALL.with_batch(1)
    dd = replace(d, df_chunk_codec=2)
    with pytest.raises(F.DfssmError):
        F.prefill_workspace_layout(dd, 4)
        lw, st, res = _layer_case(d, 4, 3)
        _prefill(dd, 4, lw, st, res)
