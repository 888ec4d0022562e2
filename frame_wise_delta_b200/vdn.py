"""Python binding of libvdn (ctypes; argument marshalling only).

Every function has the name of its C entry point in include/vdn.h, takes
torch CUDA tensors (or None where the C call accepts NULL), passes their
device pointers and the current torch stream, and raises VdnError on any
status other than VDN_OK. All arithmetic happens in the library's kernels;
there is no fallback: if libvdn.so is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvdn.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "vdn.h")

VDN_OK, VDN_ERR_INVALID, VDN_ERR_UNSUPPORTED, VDN_ERR_CUDA, VDN_ERR_NUMERIC = range(5)
VDN_F32, VDN_BF16 = 0, 1
VDN_INFO_TIMEOUT = -1
_DTYPES = {"f32": VDN_F32, "bf16": VDN_BF16, VDN_F32: VDN_F32, VDN_BF16: VDN_BF16}
TORCH_DTYPE = {VDN_F32: torch.float32, VDN_BF16: torch.bfloat16}


class VdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class vdn_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "T", "U", "dk", "dv", "n_text", "chunk", "anchors", "in_dtype", "out_dtype",
                 "beta_per_token", "decay_bridge")]

    @property
    def C(self) -> int:
        return -(-self.T // self.chunk) if self.T > 0 else 0


def make_shape(B, H, T, U, d, n_text, chunk=5, anchors=0, in_dtype="bf16", out_dtype=None,
               beta_per_token=False, decay_bridge=False) -> vdn_shape:
    in_dt = _DTYPES[in_dtype]
    out_dt = in_dt if out_dtype is None else _DTYPES[out_dtype]
    return vdn_shape(B, H, T, U, d, d, n_text, chunk, anchors, in_dt, out_dt, int(bool(beta_per_token)),
                     int(bool(decay_bridge)))


def shape_for(w, B=None, H=None) -> vdn_shape:
    """Shape of a synth.Workload (optionally with other batch/head counts)."""
    return make_shape(w.B if B is None else B, w.H if H is None else H, w.T, w.U, w.d, w.n_text,
                      w.chunk, w.anchors, w.dtype, beta_per_token=w.beta_per_token,
                      decay_bridge=getattr(w, "decay_bridge", False))


class vdn_out_gate(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("norm_weight", ctypes.c_void_p), ("eps", ctypes.c_float)]


def out_gate(gate, norm_weight, eps=1e-6):
    """The readout epilogue's arguments: gate logits [B,H,T,U,dv] (input dtype),
    RMSNorm weights [H,dv] float32, eps. Returns a vdn_out_gate (keep the
    tensors alive while it is in use)."""
    return vdn_out_gate(_ptr(gate), _ptr(norm_weight), float(eps))


def _og(og):
    return None if og is None else ctypes.cast(ctypes.pointer(og), _P)


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "vdn_frame_grams": [_P, _P, _P, _P, _P, _P, _P, _P],
    "vdn_frame_factor": [_P, _P, _P, _P, _P, _P, _P, _P],
    "vdn_chunk_compose": [_P, _P, _P, _P, _P, _P, _P, _P],
    "vdn_scan_fwd": [_P, _P, _P, _P, _P, _P],
    "vdn_scan_bwd": [_P, _P, _P, _P, _P, _P],
    "vdn_scan_bidir": [_P, _P, _P, _P, _P, _P, _P, _P, _P],
    "vdn_chunk_readout": [_P, _P, _P, _P, _P, _P, _P],
    "vdn_text_state": [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P],
    "vdn_forward": [_P] * 13 + [ctypes.c_size_t, _P, _P, _P, _P],
    "vdn_frame_invert": [_P, _P, _P, _P, _P],
    "vdn_text_state_noalloc": [_P, _P, _P, _P, _P, _P, _P],
    "vdn_forward_pipelined": [_P] * 13 + [ctypes.c_size_t, _P, ctypes.c_int32, _P, _P, _P, _P],
    "vdn_chunk_readout_gated": [_P] * 8,
    "vdn_chunk_readout_bridged": [_P] * 9,
    "vdn_selftest_wait": [_P, _P],
    "vdn_stream_segment": [_P] * 6 + [ctypes.c_longlong] + [_P] * 5 + [ctypes.c_size_t, _P, _P],
    "vdn_stream_segment_bridged": [_P] * 6 + [ctypes.c_longlong] + [_P] * 7 + [ctypes.c_size_t, _P, _P],
}


def lib() -> ctypes.CDLL:
    """Load libvdn.so (built in-tree by frame_wise_delta_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise VdnError(VDN_ERR_CUDA, f"{LIB_PATH} is missing; build it with "
                                         "`python -m frame_wise_delta_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        for name in ("vdn_text_state_workspace_bytes", "vdn_forward_workspace_bytes",
                     "vdn_stream_workspace_bytes"):
            fn = getattr(L, name)
            fn.argtypes = [_P]
            fn.restype = ctypes.c_size_t
        L.vdn_status_string.argtypes = [ctypes.c_int]
        L.vdn_status_string.restype = ctypes.c_char_p
        L.vdn_last_error.argtypes = []
        L.vdn_last_error.restype = ctypes.c_char_p
        L.vdn_version.argtypes = []
        L.vdn_version.restype = ctypes.c_int32
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Every function name that include/vdn.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vdn_\w+)\s*\(", text)))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise VdnError(VDN_ERR_INVALID, "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise VdnError(VDN_ERR_INVALID, "tensor is not contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != VDN_OK:
        L = lib()
        name = L.vdn_status_string(status).decode()
        msg = L.vdn_last_error().decode()
        raise VdnError(status, f"{name}: {msg}")


def _shp(s: vdn_shape):
    return ctypes.cast(ctypes.pointer(s), _P)


def vdn_frame_grams(s, K, V, beta, A, Bm, info=None, stream=None):
    _check(lib().vdn_frame_grams(_shp(s), _ptr(K), _ptr(V), _ptr(beta), _ptr(A), _ptr(Bm), _ptr(info),
                                 _stream(stream)))


def vdn_frame_factor(s, A, Bm, alpha, M, J, info, stream=None):
    _check(lib().vdn_frame_factor(_shp(s), _ptr(A), _ptr(Bm), _ptr(alpha), _ptr(M), _ptr(J), _ptr(info),
                                  _stream(stream)))


def vdn_frame_invert(s, A, W, info, stream=None):
    _check(lib().vdn_frame_invert(_shp(s), _ptr(A), _ptr(W), _ptr(info), _stream(stream)))


def vdn_chunk_compose(s, M, J, Mf, Jf, Mb, Jb, stream=None):
    _check(lib().vdn_chunk_compose(_shp(s), _ptr(M), _ptr(J), _ptr(Mf), _ptr(Jf), _ptr(Mb), _ptr(Jb),
                                   _stream(stream)))


def vdn_scan_fwd(s, Mf, Jf, S_T, F, stream=None):
    _check(lib().vdn_scan_fwd(_shp(s), _ptr(Mf), _ptr(Jf), _ptr(S_T), _ptr(F), _stream(stream)))


def vdn_scan_bwd(s, Mb, Jb, S_T, G, stream=None):
    _check(lib().vdn_scan_bwd(_shp(s), _ptr(Mb), _ptr(Jb), _ptr(S_T), _ptr(G), _stream(stream)))


def vdn_scan_bidir(s, Mf, Jf, Mb, Jb, S_T, F, G, stream=None):
    _check(lib().vdn_scan_bidir(_shp(s), _ptr(Mf), _ptr(Jf), _ptr(Mb), _ptr(Jb), _ptr(S_T), _ptr(F),
                                _ptr(G), _stream(stream)))


def vdn_chunk_readout(s, Q, F, G, O, info=None, stream=None):
    _check(lib().vdn_chunk_readout(_shp(s), _ptr(Q), _ptr(F), _ptr(G), _ptr(O), _ptr(info),
                                   _stream(stream)))


def vdn_text_state_workspace_bytes(s) -> int:
    return int(lib().vdn_text_state_workspace_bytes(_shp(s)))


def vdn_text_state(s, Kx, Vx, beta_x, S_T, workspace, info, stream=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().vdn_text_state(_shp(s), _ptr(Kx), _ptr(Vx), _ptr(beta_x), _ptr(S_T), _ptr(workspace),
                                nbytes, _ptr(info), _stream(stream)))


def vdn_text_state_noalloc(s, Kx, Vx, beta_x, S_T, info, stream=None):
    """vdn_text_state with the library's fixed device scratch instead of a workspace."""
    _check(lib().vdn_text_state_noalloc(_shp(s), _ptr(Kx), _ptr(Vx), _ptr(beta_x), _ptr(S_T), _ptr(info),
                                        _stream(stream)))


def vdn_forward_workspace_bytes(s) -> int:
    return int(lib().vdn_forward_workspace_bytes(_shp(s)))


def vdn_forward(s, Q, K, V, beta, alpha, Kx, Vx, beta_x, O, F, G, workspace, info, events=None,
                stream=None, og=None):
    """events: None or 7 torch.cuda.Event (enable_timing, already recorded once so
    that their CUDA handles exist) recorded by the library between the stages.
    og: None or an out_gate(...) for the gated RMSNorm readout epilogue."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    ev = None
    if events is not None:
        handles = [e.cuda_event if e is not None else None for e in events]
        if any(e is not None and not h for e, h in zip(events, handles)):
            raise VdnError(VDN_ERR_INVALID, "stage events must have been recorded once (no CUDA handle yet)")
        arr = (ctypes.c_void_p * 7)(*handles)
        ev = ctypes.cast(arr, ctypes.c_void_p)
    _check(lib().vdn_forward(_shp(s), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(alpha), _ptr(Kx),
                             _ptr(Vx), _ptr(beta_x), _ptr(O), _ptr(F), _ptr(G), _ptr(workspace), nbytes,
                             _ptr(info), ev, _og(og), _stream(stream)))


def pipeline_events(groups: int):
    """The 8 + groups timing events vdn_forward_pipelined records (created
    here by torch and recorded once so that their CUDA handles exist)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8 + groups)]
    for e in evs:
        e.record()
    return evs


def vdn_forward_pipelined(s, Q, K, V, beta, alpha, Kx, Vx, beta_x, O, F, G, workspace, info, groups, aux,
                          events, stream=None, og=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    handles = [e.cuda_event for e in events]
    if len(handles) < 8 + groups or not all(handles):
        raise VdnError(VDN_ERR_INVALID, "need 8 + groups recorded events")
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _check(lib().vdn_forward_pipelined(_shp(s), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(alpha), _ptr(Kx),
                                       _ptr(Vx), _ptr(beta_x), _ptr(O), _ptr(F), _ptr(G), _ptr(workspace),
                                       nbytes, _ptr(info), int(groups), _stream(aux),
                                       ctypes.cast(arr, ctypes.c_void_p), _og(og), _stream(stream)))


def vdn_chunk_readout_gated(s, Q, F, G, og, O, info=None, stream=None):
    _check(lib().vdn_chunk_readout_gated(_shp(s), _ptr(Q), _ptr(F), _ptr(G), _og(og), _ptr(O), _ptr(info),
                                         _stream(stream)))


def vdn_chunk_readout_bridged(s, Q, F, G, alpha, og, O, info=None, stream=None):
    """The chunk readout through the decay bridge (shape.decay_bridge = 1); og may be None."""
    _check(lib().vdn_chunk_readout_bridged(_shp(s), _ptr(Q), _ptr(F), _ptr(G), _ptr(alpha), _og(og), _ptr(O),
                                           _ptr(info), _stream(stream)))


def vdn_stream_workspace_bytes(s) -> int:
    return int(lib().vdn_stream_workspace_bytes(_shp(s)))


def vdn_stream_segment(s, Q, K, V, beta, alpha, frame0, S_prev, S_in, O, F, workspace, info, stream=None):
    """One segment of a live stream through the forward memory only (see vdn.h)."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().vdn_stream_segment(_shp(s), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(alpha), int(frame0),
                                    _ptr(S_prev), _ptr(S_in), _ptr(O), _ptr(F), _ptr(workspace), nbytes,
                                    _ptr(info), _stream(stream)))


def vdn_stream_segment_bridged(s, Q, K, V, beta, alpha, frame0, S_prev, S_in, alpha_prev, O, F, alpha_tail,
                               workspace, info, stream=None):
    """One stream segment read through the decay bridge (see vdn.h); alpha_prev
    None for the stream's first segment, alpha_tail None when not needed."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().vdn_stream_segment_bridged(_shp(s), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(alpha),
                                            int(frame0), _ptr(S_prev), _ptr(S_in), _ptr(alpha_prev), _ptr(O),
                                            _ptr(F), _ptr(alpha_tail), _ptr(workspace), nbytes, _ptr(info),
                                            _stream(stream)))


def vdn_selftest_wait(info, stream=None):
    """Self-test of the bounded pipeline waits (see vdn.h): *info becomes VDN_INFO_TIMEOUT."""
    _check(lib().vdn_selftest_wait(_ptr(info), _stream(stream)))


def vdn_status_string(status: int) -> str:
    return lib().vdn_status_string(status).decode()


def vdn_last_error() -> str:
    return lib().vdn_last_error().decode()


def vdn_version() -> int:
    return int(lib().vdn_version())


# ------------------------------------------------------------------ helpers
def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte-aligned uint8 device buffer of at least nbytes bytes."""
    return torch.empty(max(1, nbytes), dtype=torch.uint8, device=device)


class Stream:
    """A live stream read through the forward memory: call with each segment's
    frames (whole chunks except the last); the carried states (the forward
    states before the last two chunks) start as the text state S^T."""

    def __init__(self, s: vdn_shape, S_T: torch.Tensor, device="cuda"):
        self.s = s
        self.ws = workspace(vdn_stream_workspace_bytes(s), device)
        self.info = torch.zeros(1, dtype=torch.int32, device=device)
        self.O = torch.empty((s.B, s.H, s.T, s.U, s.dv), dtype=TORCH_DTYPE[s.out_dtype], device=device)
        self.F = torch.empty((s.B, s.H, s.C + 1, s.dv, s.dk), dtype=torch.float32, device=device)
        self.S_prev = S_T.clone()
        self.S_in = S_T.clone()
        self.frame0 = 0
        # with the decay bridge: the last chunk's decay product, carried too
        self.alpha_tail = (torch.ones((s.B, s.H, s.dk), dtype=torch.float32, device=device)
                           if s.decay_bridge else None)

    def __call__(self, Q, K, V, beta, alpha, stream=None):
        if self.s.decay_bridge:
            prev = None if self.frame0 == 0 else self.alpha_tail.clone()
            vdn_stream_segment_bridged(self.s, Q, K, V, beta, alpha, self.frame0, self.S_prev, self.S_in, prev,
                                       self.O, self.F, self.alpha_tail, self.ws, self.info, stream)
        else:
            vdn_stream_segment(self.s, Q, K, V, beta, alpha, self.frame0, self.S_prev, self.S_in, self.O,
                               self.F, self.ws, self.info, stream)
        C = self.s.C
        if C > 0:
            self.S_prev.copy_(self.F[:, :, C - 1])
            self.S_in.copy_(self.F[:, :, C])
        self.frame0 += self.s.T
        return self.O


class Forward:
    """Preallocated buffers for repeated vdn_forward calls on one shape."""

    def __init__(self, s: vdn_shape, device="cuda", keep_states=True):
        self.s = s
        BH = s.B * s.H
        C = s.C
        self.ws = workspace(vdn_forward_workspace_bytes(s), device)
        self.info = torch.zeros(1, dtype=torch.int32, device=device)
        out_dt = TORCH_DTYPE[s.out_dtype]
        self.O = torch.empty((s.B, s.H, s.T, s.U, s.dv), dtype=out_dt, device=device)
        self.F = self.G = None
        if keep_states:
            self.F = torch.empty((s.B, s.H, C + 1, s.dv, s.dk), dtype=torch.float32, device=device)
            self.G = torch.empty_like(self.F)
        del BH

    def __call__(self, Q, K, V, beta, alpha, Kx, Vx, beta_x, events=None, stream=None, og=None):
        vdn_forward(self.s, Q, K, V, beta, alpha, Kx, Vx, beta_x, self.O, self.F, self.G, self.ws,
                    self.info, events, stream, og)
        return self.O


class PipelinedForward(Forward):
    """vdn_forward_pipelined with its own auxiliary stream and events."""

    def __init__(self, s: vdn_shape, groups: int = 3, device="cuda", keep_states=True):
        super().__init__(s, device, keep_states)
        self.groups = groups
        self.aux = torch.cuda.Stream(device=device)
        self.events = pipeline_events(groups)

    def __call__(self, Q, K, V, beta, alpha, Kx, Vx, beta_x, events=None, stream=None, og=None):
        vdn_forward_pipelined(self.s, Q, K, V, beta, alpha, Kx, Vx, beta_x, self.O, self.F, self.G, self.ws,
                              self.info, self.groups, self.aux, self.events, stream, og)
        return self.O
