"""Thin ctypes binding over libdfssm.so (C ABI in include/dfssm.h).

Argument marshalling only: PyTorch provides device memory and the stream; every
step of the decode path runs in the library's CUDA kernels.  There is no CPU or
PyTorch fallback -- if the library cannot be loaded, importing the entry points
raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# DFSSM_VARIANT=phases loads the build with the token kernel's phase timers
# (libdfssm_phases.so, see build.py); DFSSM_LIBRARY names any other build of the
# same library by path; the default is the product build.
VARIANT = os.environ.get("DFSSM_VARIANT", "")
LIB_PATH = os.environ.get("DFSSM_LIBRARY") or os.path.join(
    _PKG, "libdfssm_phases.so" if VARIANT == "phases" else "libdfssm.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_MISALIGNED = -3
ERR_WORKSPACE_TOO_SMALL = -4
ERR_CUDA = -5
ERR_DEVICE = -6
ERR_NOT_BUILT = -7
DTYPE_F16, DTYPE_F32 = 0, 1
LAYOUT_ROWMAJOR, LAYOUT_TILED = 0, 1

EXPORTS = [
    "dfssm_packed_words", "dfssm_pack_weights", "dfssm_repack_bits",
    "dfssm_proj_workspace_bytes", "dfssm_proj_forward", "dfssm_proj_forward_noalloc",
    "dfssm_proj_workspace_layout",
    "dfssm_workspace_bytes", "dfssm_workspace_layout", "dfssm_layer_step",
    "dfssm_model_decode", "dfssm_model_decode_launches", "dfssm_last_error", "dfssm_version",
    "dfssm_model_decode_q8", "dfssm_quantize_rows_int8", "dfssm_phase_timers",
    "dfssm_prefill_workspace_bytes", "dfssm_prefill_workspace_layout", "dfssm_layer_prefill",
    "dfssm_model_prefill", "dfssm_df_field_words", "dfssm_df_encode", "dfssm_df_decode",
]


class DfssmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"dfssm error {code}: {msg}")
        self.code = code


class CDims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in
                ("batch", "d_model", "d_inner", "nheads", "headdim", "d_state", "ngroups", "d_conv", "rank",
                 "ssm_state_dtype", "df_chunk_codec")]


class CProj(C.Structure):
    _fields_ = [("rows", C.c_int32), ("cols", C.c_int32), ("bits", C.c_void_p), ("alpha", C.c_void_p),
                ("A", C.c_void_p), ("sA", C.c_void_p), ("B", C.c_void_p), ("sB", C.c_void_p)]


class CLayerWeights(C.Structure):
    _fields_ = [("prenorm_w", C.c_void_p), ("inp", CProj), ("conv_w", C.c_void_p), ("conv_b", C.c_void_p),
                ("dt_bias", C.c_void_p), ("A_log", C.c_void_p), ("D", C.c_void_p), ("gnorm_w", C.c_void_p),
                ("out", CProj)]


class CLayerState(C.Structure):
    _fields_ = [("conv_state", C.c_void_p), ("ssm_state", C.c_void_p)]


class CWsLayout(C.Structure):
    _fields_ = [(n, C.c_size_t) for n in
                ("total_bytes", "status", "x_in", "xq_in", "sx_in", "acc_in", "u_in", "xd_in", "xdsum_in",
                 "zxbcdt", "xc", "g", "x_out", "xq_out", "sx_out", "acc_out", "u_out", "xd_out", "xdsum_out",
                 "res", "scratch", "control")]


_lib = None


def lib() -> C.CDLL:
    """Load libdfssm.so (building it first if the sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        from . import build
        build.build(variant=VARIANT)
    L = C.CDLL(LIB_PATH)
    vp, i, sz = C.c_void_p, C.c_int, C.c_size_t
    L.dfssm_packed_words.argtypes = [i, i, i]
    L.dfssm_packed_words.restype = sz
    L.dfssm_pack_weights.argtypes = [vp, i, i, i, i, vp, vp]
    L.dfssm_repack_bits.argtypes = [vp, i, i, vp, vp]
    L.dfssm_proj_workspace_bytes.argtypes = [i, i, i, i]
    L.dfssm_proj_workspace_bytes.restype = sz
    L.dfssm_proj_workspace_layout.argtypes = [i, i, i, i, C.POINTER(CWsLayout)]
    L.dfssm_proj_forward.argtypes = [C.POINTER(CProj), i, i, vp, vp, vp, sz, vp]
    L.dfssm_proj_forward_noalloc.argtypes = [C.POINTER(CProj), i, i, vp, vp, vp]
    L.dfssm_workspace_bytes.argtypes = [C.POINTER(CDims), i, i]
    L.dfssm_workspace_bytes.restype = sz
    L.dfssm_workspace_layout.argtypes = [C.POINTER(CDims), i, i, C.POINTER(CWsLayout)]
    L.dfssm_layer_step.argtypes = [C.POINTER(CDims), C.POINTER(CLayerWeights), C.POINTER(CLayerState),
                                   vp, vp, sz, vp]
    L.dfssm_model_decode.argtypes = [C.POINTER(CDims), i, i, vp, C.POINTER(CLayerWeights),
                                     C.POINTER(CLayerState), vp, vp, vp, vp, vp, sz, vp]
    L.dfssm_model_decode_launches.argtypes = [C.POINTER(CDims), i, i]
    L.dfssm_model_decode_q8.argtypes = [C.POINTER(CDims), i, i, vp, vp, C.POINTER(CLayerWeights),
                                        C.POINTER(CLayerState), vp, vp, vp, vp, vp, sz, vp]
    L.dfssm_quantize_rows_int8.argtypes = [vp, i, i, vp, vp, vp]
    L.dfssm_phase_timers.argtypes = [vp, i, i]
    L.dfssm_prefill_workspace_bytes.argtypes = [C.POINTER(CDims), i, i, i]
    L.dfssm_prefill_workspace_bytes.restype = sz
    L.dfssm_prefill_workspace_layout.argtypes = [C.POINTER(CDims), i, i, i, C.POINTER(CWsLayout)]
    L.dfssm_layer_prefill.argtypes = [C.POINTER(CDims), i, C.POINTER(CLayerWeights), C.POINTER(CLayerState),
                                      vp, vp, sz, vp]
    L.dfssm_model_prefill.argtypes = [C.POINTER(CDims), i, i, vp, C.POINTER(CLayerWeights),
                                      C.POINTER(CLayerState), vp, i, vp, vp, vp, vp, sz, vp]
    L.dfssm_df_field_words.argtypes = [i]
    L.dfssm_df_encode.argtypes = [vp, i, i, vp, vp, vp, vp, vp]
    L.dfssm_df_decode.argtypes = [vp, vp, vp, i, i, vp, vp]
    L.dfssm_last_error.restype = C.c_char_p
    L.dfssm_version.restype = C.c_int
    for name in EXPORTS:
        getattr(L, name)
    _lib = L
    return L


def last_error() -> str:
    return lib().dfssm_last_error().decode()


def _check(rc: int) -> None:
    if rc != OK:
        raise DfssmError(rc, last_error())


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def cdims(d) -> CDims:
    return CDims(d.batch, d.d_model, d.d_inner, d.nheads, d.headdim, d.d_state, d.ngroups, d.d_conv, d.rank,
                 getattr(d, "ssm_state_dtype", 0), getattr(d, "df_chunk_codec", 0))


# ------------------------------------------------------------------ host -> device

def _dev(a: np.ndarray, device):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).to(device)


@dataclass
class DeviceProj:
    rows: int
    cols: int
    bits: object          # torch int32 (tiled sign words)
    alpha: object
    A: object = None
    sA: object = None
    B: object = None
    sB: object = None

    @classmethod
    def from_host(cls, p, device="cuda", stream=None) -> "DeviceProj":
        """Upload a synth.ProjWeights; its row-major sign words are permuted into the
        tiled layout on the device by dfssm_repack_bits."""
        import torch
        rm = _dev(p.bits, device)
        tiled = torch.empty(packed_words(p.rows, p.cols, LAYOUT_TILED), dtype=torch.int32, device=device)
        repack_bits(rm, p.rows, p.cols, tiled, stream)
        out = cls(p.rows, p.cols, tiled, _dev(p.alpha, device))
        if p.A is not None:
            out.A, out.sA, out.B, out.sB = (_dev(p.A, device), _dev(p.sA, device), _dev(p.B, device),
                                            _dev(p.sB, device))
        return out

    def c(self) -> CProj:
        return CProj(self.rows, self.cols, _ptr(self.bits), _ptr(self.alpha), _ptr(self.A), _ptr(self.sA),
                     _ptr(self.B), _ptr(self.sB))


@dataclass
class DeviceLayer:
    prenorm_w: object
    inp: DeviceProj
    conv_w: object
    conv_b: object
    dt_bias: object
    A_log: object
    D: object
    gnorm_w: object
    out: DeviceProj

    @classmethod
    def from_host(cls, lw, device="cuda", stream=None) -> "DeviceLayer":
        return cls(_dev(lw.prenorm_w, device), DeviceProj.from_host(lw.inp, device, stream),
                   _dev(lw.conv_w, device), _dev(lw.conv_b, device), _dev(lw.dt_bias, device),
                   _dev(lw.A_log, device), _dev(lw.D, device), _dev(lw.gnorm_w, device),
                   DeviceProj.from_host(lw.out, device, stream))

    def c(self) -> CLayerWeights:
        return CLayerWeights(_ptr(self.prenorm_w), self.inp.c(), _ptr(self.conv_w), _ptr(self.conv_b),
                             _ptr(self.dt_bias), _ptr(self.A_log), _ptr(self.D), _ptr(self.gnorm_w),
                             self.out.c())


@dataclass
class DeviceState:
    conv: object   # fp32 [B, W-1, conv_dim]
    ssm: object    # [B, H, P, N], fp32 or fp16 (d.ssm_state_dtype == 1)

    @classmethod
    def zeros(cls, d, device="cuda") -> "DeviceState":
        import torch
        sdt = torch.float16 if getattr(d, "ssm_state_dtype", 0) == 1 else torch.float32
        return cls(torch.zeros((d.batch, d.d_conv - 1, d.conv_dim), dtype=torch.float32, device=device),
                   torch.zeros((d.batch, d.nheads, d.headdim, d.d_state), dtype=sdt, device=device))

    @classmethod
    def from_host(cls, st, device="cuda") -> "DeviceState":
        return cls(_dev(st.conv, device), _dev(st.ssm, device))

    def c(self) -> CLayerState:
        return CLayerState(_ptr(self.conv), _ptr(self.ssm))


@dataclass
class DeviceModel:
    dims: object
    vocab: int
    embed: object                  # fp16 [vocab][d_model]
    normf_w: object
    layers: List[DeviceLayer]
    embed_q: object = None         # head="int8": int8 codes [vocab][d_model] ...
    embed_scale: object = None     # ... and fp32 row scales [vocab]

    @classmethod
    def from_host(cls, m, device="cuda", stream=None, head: str = "fp16") -> "DeviceModel":
        """head="int8" quantises the tied embedding per row on the device
        (dfssm_quantize_rows_int8) and decodes through dfssm_model_decode_q8."""
        if head not in ("fp16", "int8"):
            raise ValueError("head must be 'fp16' or 'int8'")
        dm = cls(m.dims, m.vocab, _dev(m.embed, device), _dev(m.normf_w, device),
                 [DeviceLayer.from_host(lw, device, stream) for lw in m.layers])
        if head == "int8":
            dm.embed_q, dm.embed_scale = quantize_rows_int8(dm.embed, stream)
        return dm


# ------------------------------------------------------------------ entry points

def quantize_rows_int8(w16, stream=None):
    """Per-row int8 codes and fp32 scales of a device fp16 matrix (dfssm_quantize_rows_int8)."""
    import torch
    rows, cols = w16.shape
    q = torch.empty((rows, cols), dtype=torch.int8, device=w16.device)
    sc = torch.empty((rows,), dtype=torch.float32, device=w16.device)
    _check(lib().dfssm_quantize_rows_int8(_ptr(w16), rows, cols, _ptr(q), _ptr(sc), _stream(stream)))
    return q, sc


def packed_words(rows: int, cols: int, layout: int) -> int:
    return int(lib().dfssm_packed_words(rows, cols, layout))


def pack_weights(w, rows: int, cols: int, layout: int, bits, stream=None) -> None:
    import torch
    dtype = DTYPE_F16 if w.dtype == torch.float16 else DTYPE_F32
    _check(lib().dfssm_pack_weights(_ptr(w), dtype, rows, cols, layout, _ptr(bits), _stream(stream)))


def repack_bits(rowmajor, rows: int, cols: int, tiled, stream=None) -> None:
    _check(lib().dfssm_repack_bits(_ptr(rowmajor), rows, cols, _ptr(tiled), _stream(stream)))


def proj_workspace_layout(rows: int, cols: int, rank: int, batch: int) -> CWsLayout:
    L = CWsLayout()
    _check(lib().dfssm_proj_workspace_layout(rows, cols, rank, batch, C.byref(L)))
    return L


def proj_forward(p: DeviceProj, rank: int, x, y, ws, stream=None) -> None:
    cp = p.c()
    _check(lib().dfssm_proj_forward(C.byref(cp), rank, x.shape[0], _ptr(x), _ptr(y), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)))


def proj_forward_noalloc(p: DeviceProj, rank: int, x, y, stream=None) -> None:
    """dfssm_proj_forward without a caller workspace (library-owned 4 MiB scratch)."""
    cp = p.c()
    _check(lib().dfssm_proj_forward_noalloc(C.byref(cp), rank, x.shape[0], _ptr(x), _ptr(y), _stream(stream)))


def workspace_layout(d, n_layer: int = 0, vocab: int = 0) -> CWsLayout:
    L = CWsLayout()
    cd = cdims(d)
    _check(lib().dfssm_workspace_layout(C.byref(cd), n_layer, vocab, C.byref(L)))
    return L


def workspace(d, n_layer: int = 0, vocab: int = 0, device="cuda"):
    """Zero-filled workspace tensor of the size the call needs."""
    import torch
    return torch.zeros(workspace_layout(d, n_layer, vocab).total_bytes, dtype=torch.uint8, device=device)


def proj_workspace(rows: int, cols: int, rank: int, batch: int, device="cuda"):
    import torch
    return torch.zeros(proj_workspace_layout(rows, cols, rank, batch).total_bytes, dtype=torch.uint8,
                       device=device)


def layer_step(d, w: DeviceLayer, s: DeviceState, residual, ws, stream=None) -> None:
    cd, cw, cs = cdims(d), w.c(), s.c()
    _check(lib().dfssm_layer_step(C.byref(cd), C.byref(cw), C.byref(cs), _ptr(residual), _ptr(ws),
                                  ws.numel(), _stream(stream)))


class ModelCall:
    """Prepared arguments of dfssm_model_decode for one (model, states) pair."""

    def __init__(self, m: DeviceModel, states: Sequence[DeviceState]):
        n = len(m.layers)
        self.m = m
        self.states = list(states)
        self.cd = cdims(m.dims)
        self.cw = (CLayerWeights * n)(*[lw.c() for lw in m.layers])
        self.cs = (CLayerState * n)(*[s.c() for s in self.states])

    def __call__(self, tok_in, tok_out, ws, logits=None, stream=None) -> None:
        m = self.m
        if m.embed_q is not None:
            _check(lib().dfssm_model_decode_q8(C.byref(self.cd), len(m.layers), m.vocab, _ptr(m.embed_q),
                                               _ptr(m.embed_scale), self.cw, self.cs, _ptr(m.normf_w),
                                               _ptr(tok_in), _ptr(tok_out), _ptr(logits), _ptr(ws), ws.numel(),
                                               _stream(stream)))
            return
        _check(lib().dfssm_model_decode(C.byref(self.cd), len(m.layers), m.vocab, _ptr(m.embed), self.cw,
                                        self.cs, _ptr(m.normf_w), _ptr(tok_in), _ptr(tok_out), _ptr(logits),
                                        _ptr(ws), ws.numel(), _stream(stream)))


def launches_per_decode_step(d, n_layer: int, vocab: int = 50280) -> int:
    cd = cdims(d)
    return int(lib().dfssm_model_decode_launches(C.byref(cd), n_layer, vocab))


def model_decode(m: DeviceModel, states, tok_in, tok_out, ws, logits=None, stream=None) -> None:
    ModelCall(m, states)(tok_in, tok_out, ws, logits, stream)


def ws_view(ws, offset: int, dtype, shape):
    """Typed view of a workspace region (for reading intermediates back)."""
    import torch
    n = int(np.prod(shape))
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return ws[offset:offset + nbytes].view(dtype).view(*shape)


# ------------------------------------------------------------------ prompt pass

def prefill_workspace_layout(d, T: int, n_layer: int = 0, vocab: int = 0) -> CWsLayout:
    L = CWsLayout()
    cd = cdims(d)
    _check(lib().dfssm_prefill_workspace_layout(C.byref(cd), T, n_layer, vocab, C.byref(L)))
    return L


def prefill_workspace(d, T: int, n_layer: int = 0, vocab: int = 0, device="cuda"):
    import torch
    return torch.zeros(prefill_workspace_layout(d, T, n_layer, vocab).total_bytes, dtype=torch.uint8,
                       device=device)


def layer_prefill(d, T: int, w: DeviceLayer, s: DeviceState, residual, ws, stream=None) -> None:
    """One layer over a prompt: residual fp32 [batch, T, d_model] in/out (dfssm_layer_prefill)."""
    cd, cw, cs = cdims(d), w.c(), s.c()
    _check(lib().dfssm_layer_prefill(C.byref(cd), T, C.byref(cw), C.byref(cs), _ptr(residual), _ptr(ws),
                                     ws.numel(), _stream(stream)))


def model_prefill(m: DeviceModel, states: Sequence[DeviceState], tokens, tok_out, ws, logits=None,
                  stream=None) -> None:
    """The model over prompts tokens int32 [batch, T] (dfssm_model_prefill): states
    updated in place, logits / greedy token of the last prompt token."""
    n = len(m.layers)
    cd = cdims(m.dims)
    cw = (CLayerWeights * n)(*[lw.c() for lw in m.layers])
    cs = (CLayerState * n)(*[s.c() for s in states])
    _check(lib().dfssm_model_prefill(C.byref(cd), n, m.vocab, _ptr(m.embed), cw, cs, _ptr(m.normf_w),
                                     int(tokens.shape[1]), _ptr(tokens), _ptr(tok_out), _ptr(logits), _ptr(ws),
                                     ws.numel(), _stream(stream)))


# ------------------------------------------------------------------ density-field state codec

def df_field_words(d_state: int) -> int:
    """32-bit words of one state row's density field (K x K cells, K^2 >= 4 d_state)."""
    n = int(lib().dfssm_df_field_words(C.c_int(d_state)))
    if n < 0:
        _check(n)
    return n


def df_encode(rows, cells, lo, span, rows_out=None, stream=None) -> None:
    """rows fp32 [R, n] (device) -> cells int32 [R, df_field_words(n)], lo, span fp32 [R];
    rows_out (fp32 [R, n], may be rows itself) receives the readout."""
    R, n = rows.shape
    _check(lib().dfssm_df_encode(_ptr(rows), C.c_int(R), C.c_int(n), _ptr(cells), _ptr(lo), _ptr(span),
                                 _ptr(rows_out) if rows_out is not None else None, _stream(stream)))


def df_decode(cells, lo, span, rows, stream=None) -> None:
    """Readout of fields written by df_encode into rows fp32 [R, n]."""
    R, n = rows.shape
    _check(lib().dfssm_df_decode(_ptr(cells), _ptr(lo), _ptr(span), C.c_int(R), C.c_int(n), _ptr(rows),
                                 _stream(stream)))
