"""dfssm_proj_forward_noalloc: the projection for callers that cannot call
cudaMalloc (no allocator of their own, or no device-wide synchronisation allowed),
running on the library's built-in scratch array instead of a caller workspace.

Checked through the C ABI against dfssm_proj_forward on the same inputs, for two
calls in a row (the second reuses the scratch the first left behind), plus the
size check.  This file sorts last so a run that stops at the first failure has
already run every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

from bit_scaffold_quantized_b200 import dfssm as F
from bit_scaffold_quantized_b200 import synth as S
from tests._util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu


def _with_workspace(dp, rank, x):
    y = torch.full((x.shape[0], dp.rows), np.nan, dtype=torch.float32, device="cuda")
    ws = F.proj_workspace(dp.rows, dp.cols, rank, x.shape[0])
    F.proj_forward(dp, rank, x, y, ws)
    return y


def test_noalloc_matches_workspace_entry_two_calls():
    assert torch.cuda.is_available()
    L = F.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for d_in, d_out, rank, batch in [(2048, 8512, 32, 4), (4096, 2048, 16, 1)]:
        p, x = S.proj_workload(d_in, d_out, rank, batch)
        dp = F.DeviceProj.from_host(p)
        xt = torch.from_numpy(x).cuda()
        y_ref = _with_workspace(dp, rank, xt)
        y = torch.full_like(y_ref, np.nan)
        cp = dp.c()
        rc = L.dfssm_proj_forward_noalloc(C.byref(cp), rank, batch, xt.data_ptr(), y.data_ptr(), stream)
        assert rc == 0, F.last_error()
        torch.cuda.synchronize()
        assert rel_err(to_np(y), to_np(y_ref)) <= TOL
        assert np.array_equal(to_np(y), to_np(y_ref))


def test_noalloc_rejects_oversize():
    L = F.lib()
    fake = 1 << 20                     # never dereferenced: the size check fails first
    p = F.CProj(8512, 8192, fake, fake, fake, fake, fake, fake)
    rc = L.dfssm_proj_forward_noalloc(C.byref(p), 64, 256, fake, fake, None)
    assert rc == F.ERR_WORKSPACE_TOO_SMALL
    assert "scratch" in F.last_error()
