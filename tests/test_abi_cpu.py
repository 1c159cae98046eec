"""C-ABI checks that need no GPU: the library builds, loads and exports every entry
point include/dfssm.h declares, and host-side validation rejects bad arguments
before anything is enqueued."""
import ctypes as C
import os
import re
import subprocess

import pytest

from bit_scaffold_quantized_b200 import dfssm as F
from bit_scaffold_quantized_b200 import synth as S
from bit_scaffold_quantized_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    hdr = open(os.path.join(ROOT, "include", "dfssm.h")).read()
    return sorted(set(re.findall(r"DFSSM_API[^;(]*?\b(dfssm_\w+)\s*\(", hdr)))


def test_library_builds_and_loads():
    build.build()
    L = F.lib()
    assert L.dfssm_version() == 210


def test_phase_timers_absent_from_the_product_build():
    buf = (C.c_uint64 * 64)()
    assert F.lib().dfssm_phase_timers(buf, 64, 1) == F.ERR_NOT_BUILT
    assert "DFSSM_PHASE_TIMERS" in F.last_error()


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", F.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (dfssm_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(names) == set(F.EXPORTS)
    # nothing else leaks from the library besides the ABI
    assert exported == set(names)


def test_packed_words_and_workspace_sizes():
    assert F.packed_words(8512, 2048, F.LAYOUT_ROWMAJOR) == 8512 * 64
    assert F.packed_words(1064, 256, F.LAYOUT_TILED) == 1072 * 8      # rows padded to 16
    assert F.packed_words(16, 100, F.LAYOUT_TILED) == 0
    d = S.LAYER_1P3B
    L = F.workspace_layout(d)
    assert L.total_bytes > 0 and L.res == 2 ** 64 - 1
    Lm = F.workspace_layout(d, 48, S.VOCAB_1P3B)
    assert Lm.res != 2 ** 64 - 1 and Lm.total_bytes > L.total_bytes
    for f in ("x_in", "xq_in", "acc_in", "zxbcdt", "g", "x_out"):
        assert getattr(L, f) % 256 == 0


FAKE = 1 << 20   # aligned, never dereferenced: validation fails before any launch


def _layer_structs(d, **over):
    def proj(rows, cols):
        return F.CProj(rows, cols, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    w = F.CLayerWeights(FAKE, proj(d.in_rows, d.d_model), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                        proj(d.d_model, d.d_inner))
    for k, v in over.items():
        setattr(w, k, v)
    return w, F.CLayerState(FAKE, FAKE)


def _call_layer(d, w, s, res=FAKE, ws=FAKE, nbytes=1 << 30):
    cd = F.cdims(d)
    return F.lib().dfssm_layer_step(C.byref(cd), C.byref(w), C.byref(s), res, ws, nbytes, None)


def test_layer_step_rejects_bad_arguments():
    d = S.LAYER_SMALL
    w, s = _layer_structs(d)
    assert F.lib().dfssm_layer_step(None, C.byref(w), C.byref(s), FAKE, FAKE, 1, None) == F.ERR_INVALID_ARG
    bad = S.Dims(1, 256, 512, 8, 64, 16, ngroups=2, rank=8)
    assert _call_layer(bad, w, s) == F.ERR_UNSUPPORTED_SHAPE
    assert "ngroups" in F.last_error()
    assert _call_layer(S.Dims(1, 300, 512, 8, 64, 16, rank=8), w, s) == F.ERR_UNSUPPORTED_SHAPE
    assert _call_layer(S.Dims(1, 256, 512, 8, 60, 16, rank=8), w, s) == F.ERR_UNSUPPORTED_SHAPE
    assert _call_layer(d, w, s, res=FAKE + 4) == F.ERR_MISALIGNED
    assert _call_layer(d, w, s, res=0) == F.ERR_INVALID_ARG
    assert _call_layer(d, w, s, nbytes=16) == F.ERR_WORKSPACE_TOO_SMALL
    w2, s2 = _layer_structs(d, conv_w=0)
    assert _call_layer(d, w2, s2) == F.ERR_INVALID_ARG
    w3, s3 = _layer_structs(d)
    w3.inp.A = 0
    assert _call_layer(d, w3, s3) == F.ERR_INVALID_ARG and "LoRA" in F.last_error()


def test_d_state_mismatch_is_rejected():
    """Appendix B, Table 12: a wrong d_state assumption must not run silently."""
    d = S.LAYER_1P3B
    w, s = _layer_structs(d)
    wrong = S.Dims(1, 2048, 4096, 64, 64, 64, rank=32)   # weights built for d_state 128
    assert _call_layer(wrong, w, s) == F.ERR_UNSUPPORTED_SHAPE
    assert "d_state" in F.last_error()


def test_pack_and_proj_reject_bad_arguments():
    L = F.lib()
    assert L.dfssm_pack_weights(FAKE, 0, 16, 100, F.LAYOUT_TILED, FAKE, None) == F.ERR_UNSUPPORTED_SHAPE
    assert L.dfssm_pack_weights(FAKE, 7, 16, 256, F.LAYOUT_TILED, FAKE, None) == F.ERR_INVALID_ARG
    assert L.dfssm_pack_weights(FAKE + 2, 0, 16, 256, F.LAYOUT_TILED, FAKE, None) == F.ERR_MISALIGNED
    p = F.CProj(64, 256, FAKE, FAKE, 0, 0, 0, 0)
    assert L.dfssm_proj_forward(C.byref(p), 8, 1, FAKE, FAKE, FAKE, 1 << 20, None) == F.ERR_INVALID_ARG
    assert L.dfssm_proj_forward(C.byref(p), 6, 1, FAKE, FAKE, FAKE, 1 << 20, None) == F.ERR_UNSUPPORTED_SHAPE
    assert L.dfssm_proj_forward(C.byref(p), 0, 1, FAKE, FAKE, FAKE, 8, None) == F.ERR_WORKSPACE_TOO_SMALL


def test_model_decode_rejects_bad_arguments():
    d = S.LAYER_SMALL
    w, s = _layer_structs(d)
    cd = F.cdims(d)
    L = F.lib()
    ws_ = (F.CLayerWeights * 1)(w)
    ss_ = (F.CLayerState * 1)(s)
    args = [C.byref(cd), 1, 100, FAKE, ws_, ss_, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None]
    bad = list(args); bad[1] = 0
    assert L.dfssm_model_decode(*bad) == F.ERR_INVALID_ARG
    bad = list(args); bad[1] = 65
    assert L.dfssm_model_decode(*bad) == F.ERR_INVALID_ARG
    bad = list(args); bad[9] = FAKE + 8
    assert L.dfssm_model_decode(*bad) == F.ERR_MISALIGNED
    bad = list(args); bad[11] = 64
    assert L.dfssm_model_decode(*bad) == F.ERR_WORKSPACE_TOO_SMALL


def test_int8_head_and_state_dtype_reject_bad_arguments():
    from dataclasses import replace
    d = S.LAYER_SMALL
    w, s = _layer_structs(d)
    cd = F.cdims(d)
    L = F.lib()
    ws_ = (F.CLayerWeights * 1)(w)
    ss_ = (F.CLayerState * 1)(s)
    args = [C.byref(cd), 1, 100, FAKE, FAKE, ws_, ss_, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None]
    bad = list(args); bad[3] = None                 # int8 codes NULL
    assert L.dfssm_model_decode_q8(*bad) == F.ERR_INVALID_ARG
    bad = list(args); bad[4] = FAKE + 4             # scales misaligned
    assert L.dfssm_model_decode_q8(*bad) == F.ERR_MISALIGNED
    bad = list(args); bad[12] = 64
    assert L.dfssm_model_decode_q8(*bad) == F.ERR_WORKSPACE_TOO_SMALL
    # SSM state storage type must be 0 (fp32) or 1 (fp16)
    cd_bad = F.cdims(replace(d, ssm_state_dtype=2))
    assert L.dfssm_layer_step(C.byref(cd_bad), C.byref(w), C.byref(s), FAKE, FAKE, 1 << 30, None) == \
        F.ERR_INVALID_ARG
    assert "ssm_state_dtype" in F.last_error()
    # the row quantiser
    assert L.dfssm_quantize_rows_int8(FAKE, 0, 16, FAKE, FAKE, None) == F.ERR_INVALID_ARG
    assert L.dfssm_quantize_rows_int8(FAKE, 4, 16, FAKE + 1, FAKE, None) == F.ERR_MISALIGNED
    assert L.dfssm_quantize_rows_int8(None, 4, 16, FAKE, FAKE, None) == F.ERR_INVALID_ARG
