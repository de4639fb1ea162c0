"""Python binding of libtq (TurboQuant-style online vector quantization on B200).

Argument marshalling only: every call goes straight to the C ABI declared in
include/tq.h, and every step of the computation runs in the library's CUDA kernels
(host-only steps: codebook and state creation). PyTorch tensors are accepted for
device buffers and streams; plain integers (device addresses) work too.

The library must be built first (``python vector_quantization_tq_b200/build.py`` or
``__graft_entry__.build()``); importing this package without it raises ImportError.
There is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

__all__ = [
    "TQError", "lib", "LIB_PATH", "HEADER_PATH", "declared_symbols",
    "MSE", "PROD", "ROT_DENSE", "ROT_RHT", "F32", "BF16",
    "build_codebook", "draw_gaussian", "draw_signs", "haar_rotation",
    "State", "quantize_workspace", "quantize_mse", "quantize_prod", "dequant", "score_workspace", "score",
    "attend_workspace", "attend_decode", "attend_decode_noalloc", "ip_stats", "search_workspace", "search_topk",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "tq.h")

MSE, PROD = 0, 1
ROT_DENSE, ROT_RHT = 0, 1
F32, BF16 = 0, 1
FIELD_CENTROIDS, FIELD_BOUNDS, FIELD_PI, FIELD_SIGNS, FIELD_S = 0, 1, 2, 3, 4
STATUS = {0: "TQ_OK", 1: "TQ_EINVAL", 2: "TQ_EUNSUPPORTED", 3: "TQ_ENOMEM", 4: "TQ_ECUDA", 5: "TQ_EDEVICE"}


class TQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_lib.tq_status_string(status).decode()})"
                         + (f", cudaError {_lib.tq_last_cuda_error()}" if status == 4 else ""))


class Params(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("b", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("rot", ctypes.c_int32), ("mat_dtype", ctypes.c_int32), ("device", ctypes.c_int32),
                ("seed_pi", ctypes.c_uint64), ("seed_s", ctypes.c_uint64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtq.so is not built at {LIB_PATH}; run `python vector_quantization_tq_b200/build.py`")
    return ctypes.CDLL(LIB_PATH, mode=ctypes.RTLD_GLOBAL)


class Planes(ctypes.Structure):
    """Device planes of one channel group (tq_planes): codes, qjl, norms, rnorms."""
    _fields_ = [("codes", ctypes.c_void_p), ("qjl", ctypes.c_void_p), ("norms", ctypes.c_void_p),
                ("rnorms", ctypes.c_void_p)]


_lib = _load()
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_DP = ctypes.POINTER(ctypes.c_double)

_SIGS = {
    "tq_status_string": (ctypes.c_char_p, [_I]),
    "tq_last_cuda_error": (_I, []),
    "tq_version": (_I, []),
    "tq_device_status": (_I, [_I]),
    "tq_check_error_path": (_I, [_I, ctypes.c_uint32]),
    "tq_build_codebook": (_I, [_I, _I, _DP, _DP, _DP]),
    "tq_draw_gaussian": (_I, [ctypes.c_uint64, _SZ, _DP]),
    "tq_draw_signs": (_I, [ctypes.c_uint64, _SZ, _P]),
    "tq_haar_rotation": (_I, [_I, _DP, _DP]),
    "tq_state_create": (_I, [ctypes.POINTER(Params), _DP, _P, _DP, ctypes.POINTER(_P)]),
    "tq_state_destroy": (_I, [_P]),
    "tq_state_params": (_I, [_P, ctypes.POINTER(Params)]),
    "tq_state_codebook_info": (_I, [_P, ctypes.POINTER(_I), _DP]),
    "tq_state_copy": (_I, [_P, _I, _DP, _SZ]),
    "tq_state_export": (_I, [_P, _P, ctypes.POINTER(_SZ)]),
    "tq_state_import": (_I, [_P, _SZ, _I, ctypes.POINTER(_P)]),
    "tq_code_layout": (_I, [_P, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]),
    "tq_quantize_workspace": (_I, [_P, _I, _I64, _I64, ctypes.POINTER(_SZ)]),
    "tq_quantize_mse": (_I, [_P, _P, _I, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "tq_quantize_prod": (_I, [_P, _P, _I, _I64, _I64, _P, _P, _P, _P, _P, _SZ, _P]),
    "tq_dequant": (_I, [_P, _P, _P, _P, _P, _I64, _P, _P]),
    "tq_score_workspace": (_I, [_P, _I64, _I64, ctypes.POINTER(_SZ)]),
    "tq_score": (_I, [_P, _P, _I, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "tq_attend_workspace": (_I, [_P, _P, _I, _I64, ctypes.POINTER(_SZ)]),
    "tq_attend_decode": (_I, [_P, _P, _P, _I, _I, _I64, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _SZ, _P]),
    "tq_attend_decode_noalloc": (_I, [_P, _P, _P, _I, _I, _I64, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P]),
    "tq_ip_stats": (_I, [_P, _P, _I64, _I, _P, _I64, _P, _P, _I]),
    "tq_search_workspace": (_I, [_P, _I64, _I64, _I, ctypes.POINTER(_SZ)]),
    "tq_search_topk": (_I, [_P, _P, _I, _I64, _P, _P, _P, _P, _I64, _I, _P, _P, _P, _SZ, _P]),
    "tq_attend_decode_grouped": (_I, [_P, _P, _P, _I, _I, _I, _I64, _I64, _P, _P, _P, _P, _P, _P, ctypes.c_float,
                                      _P, _P, _SZ, _P]),
    "tq_attend_append_decode": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _I, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                     ctypes.c_float, _P, _P, _SZ, _P]),
    "tq_entropy_table": (_I, [_P, _P, _P, _DP]),
    "tq_entropy_max_bytes": (_I, [_P, _I64, ctypes.POINTER(_SZ)]),
    "tq_entropy_workspace": (_I, [_P, _I64, ctypes.POINTER(_SZ)]),
    "tq_entropy_encode": (_I, [_P, _P, _I64, _P, _P, _SZ, _P, _SZ, _P]),
    "tq_entropy_decode": (_I, [_P, _P, _P, _I64, _P, _P]),
    "tq_split_create": (_I, [_P, _P, _P, _I, ctypes.POINTER(_P)]),
    "tq_split_destroy": (None, [_P]),
    "tq_split_quantize": (_I, [_P, _P, _I, _I64, _I64, ctypes.POINTER(Planes), ctypes.POINTER(Planes), _P]),
    "tq_split_dequant": (_I, [_P, ctypes.POINTER(Planes), ctypes.POINTER(Planes), _I64, _P, _P]),
    "tq_split_score_workspace": (_I, [_P, _I, _I64, _I64, ctypes.POINTER(_SZ)]),
    "tq_split_score": (_I, [_P, _P, _I, _I64, _I64, ctypes.POINTER(Planes), ctypes.POINTER(Planes), _I64, _P, _P,
                            _SZ, _P]),
    "tq_split_attend_workspace": (_I, [_P, _P, _I, _I64, ctypes.POINTER(_SZ)]),
    "tq_split_attend_decode": (_I, [_P, _P, _P, _I, _I, _I64, ctypes.POINTER(Planes), ctypes.POINTER(Planes),
                                    ctypes.POINTER(Planes), ctypes.POINTER(Planes), ctypes.c_float, _P, _P, _SZ,
                                    _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib():
    return _lib


def device_status(device: int = 0):
    """Synchronise `device`; raise TQError(TQ_EDEVICE) if a kernel recorded an error."""
    _check(_lib.tq_device_status(device), "tq_device_status")


def declared_symbols(header: str = HEADER_PATH):
    """Names of the functions declared in include/tq.h."""
    with open(header) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def _check(rc: int, what: str):
    if rc != 0:
        raise TQError(rc, what)


def _ptr(t):
    """Device (or host) address of a tensor / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available() and torch.cuda.is_initialized():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _dp(a):
    return a.ctypes.data_as(_DP) if a is not None else None


# ---- host-only calls -------------------------------------------------------------------

def build_codebook(d: int, b: int):
    """(centroids[2^b], boundaries[2^b-1], D_mse) from the library's host codebook builder."""
    c = np.zeros(1 << b)
    t = np.zeros(max(1, (1 << b) - 1))
    D = ctypes.c_double()
    _check(_lib.tq_build_codebook(d, b, _dp(c), _dp(t), ctypes.byref(D)), "tq_build_codebook")
    return c, t[: (1 << b) - 1], D.value


def draw_gaussian(seed: int, count: int) -> np.ndarray:
    out = np.zeros(count)
    _check(_lib.tq_draw_gaussian(seed, count, _dp(out)), "tq_draw_gaussian")
    return out


def draw_signs(seed: int, count: int) -> np.ndarray:
    out = np.zeros(count, dtype=np.int8)
    _check(_lib.tq_draw_signs(seed, count, out.ctypes.data), "tq_draw_signs")
    return out


def haar_rotation(g: np.ndarray) -> np.ndarray:
    g = np.ascontiguousarray(g, dtype=np.float64)
    d = g.shape[0]
    out = np.zeros((d, d))
    _check(_lib.tq_haar_rotation(d, _dp(g), _dp(out)), "tq_haar_rotation")
    return out


# ---- states ----------------------------------------------------------------------------

class State:
    """A quantizer state (codebook, rotation, QJL matrix) held by libtq on one device."""

    def __init__(self, d: int, b: int, mode: int = MSE, rot: int = ROT_DENSE, mat_dtype: int = F32,
                 device: int = 0, seed_pi: int = 0, seed_s: int = 1, gauss_pi=None, signs=None, s=None,
                 _handle=None):
        self._h = _P()
        if _handle is not None:
            self._h = _handle
        else:
            p = Params(d, b, mode, rot, mat_dtype, device, seed_pi, seed_s)
            g = None if gauss_pi is None else np.ascontiguousarray(gauss_pi, dtype=np.float64)
            sg = None if signs is None else np.ascontiguousarray(signs, dtype=np.int8)
            sm = None if s is None else np.ascontiguousarray(s, dtype=np.float64)
            _check(_lib.tq_state_create(ctypes.byref(p), _dp(g), None if sg is None else sg.ctypes.data,
                                        _dp(sm), ctypes.byref(self._h)), "tq_state_create")
        p = Params()
        _check(_lib.tq_state_params(self._h, ctypes.byref(p)), "tq_state_params")
        self.params = p
        bm, dm = _I(), ctypes.c_double()
        _check(_lib.tq_state_codebook_info(self._h, ctypes.byref(bm), ctypes.byref(dm)), "tq_state_codebook_info")
        self.b_mse, self.dmse = bm.value, dm.value
        cb, qb = _SZ(), _SZ()
        _check(_lib.tq_code_layout(self._h, ctypes.byref(cb), ctypes.byref(qb)), "tq_code_layout")
        self.code_bytes, self.qjl_bytes = cb.value, qb.value

    @property
    def handle(self):
        return self._h

    @property
    def d(self):
        return self.params.d

    @property
    def mode(self):
        return self.params.mode

    def copy(self, field: int) -> np.ndarray:
        d, L = self.params.d, 1 << self.b_mse
        size = {FIELD_CENTROIDS: L, FIELD_BOUNDS: max(0, L - 1), FIELD_PI: d * d, FIELD_SIGNS: d, FIELD_S: d * d}[field]
        out = np.zeros(max(1, size))
        _check(_lib.tq_state_copy(self._h, field, _dp(out), out.size), "tq_state_copy")
        out = out[:size]
        return out.reshape(d, d) if field in (FIELD_PI, FIELD_S) else out

    def export(self) -> bytes:
        n = _SZ()
        _check(_lib.tq_state_export(self._h, None, ctypes.byref(n)), "tq_state_export")
        buf = ctypes.create_string_buffer(n.value)
        _check(_lib.tq_state_export(self._h, buf, ctypes.byref(n)), "tq_state_export")
        return buf.raw[: n.value]

    @classmethod
    def from_bytes(cls, blob: bytes, device: int = -1) -> "State":
        h = _P()
        buf = ctypes.create_string_buffer(blob, len(blob))
        _check(_lib.tq_state_import(buf, len(blob), device, ctypes.byref(h)), "tq_state_import")
        return cls(0, 0, _handle=h)

    def close(self):
        if self._h:
            _lib.tq_state_destroy(self._h)
            self._h = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # allocation helpers (torch device tensors; plumbing only)
    def empty_planes(self, n: int, device=None):
        import torch
        dev = device if device is not None else torch.device("cuda", self.params.device)
        codes = torch.empty((n, self.code_bytes), dtype=torch.uint8, device=dev)
        norms = torch.empty(n, dtype=torch.float32, device=dev)
        if self.mode == PROD:
            qjl = torch.empty((n, self.qjl_bytes), dtype=torch.uint8, device=dev)
            rnorms = torch.empty(n, dtype=torch.float32, device=dev)
            return codes, qjl, norms, rnorms
        return codes, None, norms, None


# ---- device calls ----------------------------------------------------------------------

def _ws(workspace, nbytes, device):
    """(pointer, size) of a caller workspace; a torch buffer of `nbytes` is made when none is given.

    The library itself never allocates device memory: this is the binding's plumbing, the
    same as allocating the output planes."""
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    if nbytes == 0:
        return None, 0
    import torch
    return torch.empty(nbytes, dtype=torch.uint8, device=torch.device("cuda", device)), nbytes


def quantize_workspace(st: State, n: int, dtype: int, ld=None) -> int:
    out = _SZ()
    _check(_lib.tq_quantize_workspace(st.handle, dtype, n, st.d if ld is None else ld, ctypes.byref(out)),
           "tq_quantize_workspace")
    return out.value


def quantize_mse(st: State, x, codes, norms, stream=None, n=None, ld=None, dtype=None, workspace=None):
    n = x.shape[0] if n is None else n
    ld = x.stride(0) if ld is None else ld
    dt = _dtype_code(x) if dtype is None else dtype
    ws, wsb = _ws(workspace, quantize_workspace(st, n, dt, ld) if workspace is None else 0, st.params.device)
    _check(_lib.tq_quantize_mse(st.handle, _ptr(x), dt, n, ld, _ptr(codes), _ptr(norms), _ptr(ws), wsb,
                                _stream(stream)), "tq_quantize_mse")


def quantize_prod(st: State, x, codes, qjl, norms, rnorms, stream=None, n=None, ld=None, dtype=None,
                  workspace=None):
    n = x.shape[0] if n is None else n
    ld = x.stride(0) if ld is None else ld
    dt = _dtype_code(x) if dtype is None else dtype
    ws, wsb = _ws(workspace, quantize_workspace(st, n, dt, ld) if workspace is None else 0, st.params.device)
    _check(_lib.tq_quantize_prod(st.handle, _ptr(x), dt, n, ld, _ptr(codes), _ptr(qjl), _ptr(norms),
                                 _ptr(rnorms), _ptr(ws), wsb, _stream(stream)), "tq_quantize_prod")


def dequant(st: State, codes, qjl, norms, rnorms, out, stream=None, n=None):
    n = norms.shape[0] if n is None else n
    _check(_lib.tq_dequant(st.handle, _ptr(codes), _ptr(qjl), _ptr(norms), _ptr(rnorms), n, _ptr(out),
                           _stream(stream)), "tq_dequant")


def score_workspace(st: State, groups: int, nq: int) -> int:
    out = _SZ()
    _check(_lib.tq_score_workspace(st.handle, groups, nq, ctypes.byref(out)), "tq_score_workspace")
    return out.value


def score(st: State, q, codes, qjl, norms, rnorms, scores, groups: int = 1, nq=None, n=None, stream=None,
          workspace=None):
    """scores[g][i][k] = estimate of <q[g][i], x[g][k]>; q is [groups*nq, d] or [groups, nq, d]."""
    nq = (q.shape[-2] if q.dim() == 3 else q.shape[0] // groups) if nq is None else nq
    n = norms.shape[-1] if n is None else n
    if norms.dim() == 1 and n == norms.shape[0] and groups > 1:
        n = norms.shape[0] // groups
    ws, wsb = _ws(workspace, score_workspace(st, groups, nq) if workspace is None else 0, st.params.device)
    _check(_lib.tq_score(st.handle, _ptr(q), _dtype_code(q), groups, nq, _ptr(codes), _ptr(qjl), _ptr(norms),
                         _ptr(rnorms), n, _ptr(scores), _ptr(ws), wsb, _stream(stream)), "tq_score")


def attend_workspace(ks: State, vs: State, H: int, T: int) -> int:
    n = _SZ()
    _check(_lib.tq_attend_workspace(ks.handle, vs.handle, H, T, ctypes.byref(n)), "tq_attend_workspace")
    return n.value


def attend_decode(ks: State, vs: State, q, kcodes, kqjl, knorms, krnorms, vcodes, vnorms, scale: float, out,
                  workspace, ws_bytes=None, H=None, T=None, stream=None):
    H = q.shape[0] if H is None else H
    T = knorms.numel() // H if T is None else T
    ws_bytes = (workspace.numel() * workspace.element_size() if workspace is not None else 0) \
        if ws_bytes is None else ws_bytes
    _check(_lib.tq_attend_decode(ks.handle, vs.handle, _ptr(q), _dtype_code(q), H, T, _ptr(kcodes), _ptr(kqjl),
                                 _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), float(scale), _ptr(out),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "tq_attend_decode")


def attend_decode_grouped(ks: State, vs: State, q, G: int, T: int, Tcap: int, kcodes, kqjl, knorms, krnorms, vcodes,
                          vnorms, scale: float, out, workspace, ws_bytes=None, stream=None):
    """H = q.shape[0] query heads, G per KV head; planes [H/G][Tcap], the first T rows valid."""
    H = q.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.tq_attend_decode_grouped(ks.handle, vs.handle, _ptr(q), _dtype_code(q), H, G, T, Tcap, _ptr(kcodes),
                                         _ptr(kqjl), _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms),
                                         float(scale), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
           "tq_attend_decode_grouped")


def attend_append_decode(ks: State, vs: State, q, G: int, k_new, v_new, T: int, Tcap: int, kcodes, kqjl, knorms,
                         krnorms, vcodes, vnorms, scale: float, out, workspace, ws_bytes=None, stream=None):
    """Encode k_new / v_new [H/G][d] into row T of each KV head's planes, then attend over T + 1 tokens."""
    H = q.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.tq_attend_append_decode(ks.handle, vs.handle, _ptr(q), _dtype_code(q), H, G, _ptr(k_new),
                                        _ptr(v_new), _dtype_code(k_new), T, Tcap, _ptr(kcodes), _ptr(kqjl),
                                        _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), float(scale),
                                        _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
           "tq_attend_append_decode")


def attend_decode_noalloc(ks: State, vs: State, q, kcodes, kqjl, knorms, krnorms, vcodes, vnorms, scale: float,
                          out, H=None, T=None, stream=None):
    """tq_attend_decode with the library's fixed device scratch instead of a workspace.

    For callers that cannot allocate device memory (runtimes whose own pool owns all device
    memory, latency-critical loops that must not allocate). Calls that overlap on the GPU
    share the library's fixed scratch and race; see tq.h.
    """
    H = q.shape[0] if H is None else H
    T = knorms.numel() // H if T is None else T
    _check(_lib.tq_attend_decode_noalloc(ks.handle, vs.handle, _ptr(q), _dtype_code(q), H, T, _ptr(kcodes),
                                         _ptr(kqjl), _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms),
                                         float(scale), _ptr(out), _stream(stream)), "tq_attend_decode_noalloc")


def ip_stats(x, xt, q, out, device: int = 0, stream=None):
    """Six fp64 sums (see tq.h) of reconstruction and inner-product errors into `out` (device)."""
    n, d = x.shape
    _check(_lib.tq_ip_stats(_ptr(x), _ptr(xt), n, d, _ptr(q), q.shape[0], _ptr(out), _stream(stream), device),
           "tq_ip_stats")


def search_workspace(st: State, nq: int, n: int, k: int) -> int:
    out = _SZ()
    _check(_lib.tq_search_workspace(st.handle, nq, n, k, ctypes.byref(out)), "tq_search_workspace")
    return out.value


def search_topk(st: State, q, codes, qjl, norms, rnorms, k: int, idx, vals, workspace, ws_bytes=None,
                stream=None):
    nq, n = q.shape[0], norms.shape[0]
    ws_bytes = (workspace.numel() * workspace.element_size() if workspace is not None else 0) \
        if ws_bytes is None else ws_bytes
    _check(_lib.tq_search_topk(st.handle, _ptr(q), _dtype_code(q), nq, _ptr(codes), _ptr(qjl), _ptr(norms),
                               _ptr(rnorms), n, k, _ptr(idx), _ptr(vals), _ptr(workspace), ws_bytes,
                               _stream(stream)), "tq_search_topk")


# ---- outlier-channel split ----------------------------------------------------------------

def _planes(pl):
    codes, qjl, norms, rnorms = pl
    return Planes(_ptr(codes), _ptr(qjl), _ptr(norms), _ptr(rnorms))


class Split:
    """The channels `channels` (ascending) quantized by `outer`, the rest by `inner`."""

    def __init__(self, outer: State, inner: State, channels):
        ch = np.ascontiguousarray(channels, dtype=np.int32)
        self.outer, self.inner = outer, inner
        self.channels = ch
        self.d = outer.d + inner.d
        self._h = _P()
        _check(_lib.tq_split_create(outer.handle, inner.handle, ch.ctypes.data, len(ch), ctypes.byref(self._h)),
               "tq_split_create")

    @property
    def handle(self):
        return self._h

    def empty_planes(self, n: int, device=None):
        """((codes, qjl, norms, rnorms) of the outer group, same of the inner group)."""
        return self.outer.empty_planes(n, device), self.inner.empty_planes(n, device)

    def close(self):
        if self._h:
            _lib.tq_split_destroy(self._h)
            self._h = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def split_quantize(sp: Split, x, outer_planes, inner_planes, stream=None, n=None, ld=None):
    n = x.shape[0] if n is None else n
    ld = x.stride(0) if ld is None else ld
    po, pi = _planes(outer_planes), _planes(inner_planes)
    _check(_lib.tq_split_quantize(sp.handle, _ptr(x), _dtype_code(x), n, ld, ctypes.byref(po), ctypes.byref(pi),
                                  _stream(stream)), "tq_split_quantize")


def split_dequant(sp: Split, outer_planes, inner_planes, out, stream=None, n=None):
    n = out.shape[0] if n is None else n
    po, pi = _planes(outer_planes), _planes(inner_planes)
    _check(_lib.tq_split_dequant(sp.handle, ctypes.byref(po), ctypes.byref(pi), n, _ptr(out), _stream(stream)),
           "tq_split_dequant")


def split_score_workspace(sp: Split, qdtype: int, groups: int, nq: int) -> int:
    out = _SZ()
    _check(_lib.tq_split_score_workspace(sp.handle, qdtype, groups, nq, ctypes.byref(out)), "tq_split_score_workspace")
    return out.value


def split_score(sp: Split, q, outer_planes, inner_planes, scores, groups: int = 1, nq=None, n=None, stream=None,
                workspace=None):
    nq = (q.shape[-2] if q.dim() == 3 else q.shape[0] // groups) if nq is None else nq
    norms = outer_planes[2]
    n = norms.shape[-1] if n is None else n
    if norms.dim() == 1 and n == norms.shape[0] and groups > 1:
        n = norms.shape[0] // groups
    po, pi = _planes(outer_planes), _planes(inner_planes)
    ws, wsb = _ws(workspace, split_score_workspace(sp, _dtype_code(q), groups, nq) if workspace is None else 0,
                  sp.outer.params.device)
    _check(_lib.tq_split_score(sp.handle, _ptr(q), _dtype_code(q), groups, nq, ctypes.byref(po), ctypes.byref(pi),
                               n, _ptr(scores), _ptr(ws), wsb, _stream(stream)), "tq_split_score")


def split_attend_workspace(ks: Split, vs: Split, H: int, T: int) -> int:
    n = _SZ()
    _check(_lib.tq_split_attend_workspace(ks.handle, vs.handle, H, T, ctypes.byref(n)), "tq_split_attend_workspace")
    return n.value


def split_attend_decode(ks: Split, vs: Split, q, k_planes, v_planes, scale: float, out, workspace, ws_bytes=None,
                        H=None, T=None, stream=None):
    """k_planes / v_planes: (outer planes, inner planes) as from Split.empty_planes."""
    H = q.shape[0] if H is None else H
    T = k_planes[0][2].numel() // H if T is None else T
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    ko, ki = _planes(k_planes[0]), _planes(k_planes[1])
    vo, vi = _planes(v_planes[0]), _planes(v_planes[1])
    _check(_lib.tq_split_attend_decode(ks.handle, vs.handle, _ptr(q), _dtype_code(q), H, T, ctypes.byref(ko),
                                       ctypes.byref(ki), ctypes.byref(vo), ctypes.byref(vi), float(scale), _ptr(out),
                                       _ptr(workspace), ws_bytes, _stream(stream)), "tq_split_attend_decode")


# ---- prefix coding of the indices ---------------------------------------------------------

def entropy_table(st: State):
    """(lengths[2^b_mse], canonical codewords[2^b_mse], mean bits per coordinate)."""
    L = 1 << st.b_mse
    ln = np.zeros(L, dtype=np.int32)
    w = np.zeros(L, dtype=np.uint32)
    mean = ctypes.c_double()
    _check(_lib.tq_entropy_table(st.handle, ln.ctypes.data, w.ctypes.data, ctypes.byref(mean)), "tq_entropy_table")
    return ln, w, mean.value


def entropy_max_bytes(st: State, n: int) -> int:
    b = _SZ()
    _check(_lib.tq_entropy_max_bytes(st.handle, n, ctypes.byref(b)), "tq_entropy_max_bytes")
    return b.value


def entropy_workspace(st: State, n: int) -> int:
    b = _SZ()
    _check(_lib.tq_entropy_workspace(st.handle, n, ctypes.byref(b)), "tq_entropy_workspace")
    return b.value


def entropy_encode(st: State, codes, offsets, stream, workspace, n=None, cuda_stream=None):
    """codes [n][code_bytes] -> offsets [n + 1] (int64) and the prefix-coded stream (uint8)."""
    n = codes.shape[0] if n is None else n
    _check(_lib.tq_entropy_encode(st.handle, _ptr(codes), n, _ptr(offsets), _ptr(stream), stream.numel(),
                                  _ptr(workspace), workspace.numel(), _stream(cuda_stream)), "tq_entropy_encode")


def entropy_decode(st: State, stream, offsets, codes, n=None, cuda_stream=None):
    n = codes.shape[0] if n is None else n
    _check(_lib.tq_entropy_decode(st.handle, _ptr(stream), _ptr(offsets), n, _ptr(codes), _stream(cuda_stream)),
           "tq_entropy_decode")
