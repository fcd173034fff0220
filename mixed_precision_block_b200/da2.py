"""ctypes binding of libda2.so — argument marshalling only.

Every entry point of ``include/da2.h`` is exposed under the same name.  Tensors
are passed by device pointer; the stream defaults to torch's current stream on
the tensors' device.  PyTorch provides memory and streams and nothing else:
every step of the attention path runs in the library's CUDA kernels.  Importing
this module raises if the library has not been built (``python -m
mixed_precision_block_b200.build``); there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libda2.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m mixed_precision_block_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

DA2_OK, DA2_ERR_ARG, DA2_ERR_UNSUPPORTED, DA2_ERR_WORKSPACE, DA2_ERR_CUDA, DA2_ERR_TIMEOUT = range(6)

VIEWS = ["PERM", "Q_AVG", "K_AVG", "Q_MAX", "K_MAX", "Q_I8", "K_I8", "Q_S8", "K_S8",
         "Q_F4", "K_F4", "Q_SF4", "K_SF4", "V_I8", "V_S8", "V_F4", "V_SF4", "V_G4",
         "SCORES", "MAP", "LISTS", "COUNTS", "STATUS"]
EXPORTS = ["da2_plan", "da2_prepare", "da2_draft_rank", "da2_rank_from_scores", "da2_attention",
           "da2_dense_attention", "da2_dense_check_status", "da2_attention_wait_test",
           "da2_attention_occupancy", "da2_debug_view",
           "da2_rank_noalloc", "da2_check_status", "da2_host_bytes", "da2_forward_host", "da2_status_string"]
NOALLOC_MAX_HEADS = 64  # DA2_NOALLOC_MAX_HEADS


class Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("Hh", ctypes.c_int),
                ("Ww", ctypes.c_int), ("d", ctypes.c_int), ("rh", ctypes.c_int), ("rw", ctypes.c_int),
                ("lam", ctypes.c_float), ("budget_pct", ctypes.c_float * 4)]

    @classmethod
    def make(cls, B, H, T, Hh, Ww, d, lam, budget, rh=8, rw=8):
        return cls(B, H, T, Hh, Ww, d, rh, rw, lam, (ctypes.c_float * 4)(*budget))

    @classmethod
    def from_workload(cls, wl, **kw):
        f = dict(B=wl.B, H=wl.H, T=wl.T, Hh=wl.Hh, Ww=wl.Ww, d=wl.d, lam=wl.lam,
                 budget=tuple(wl.budget), rh=wl.rh, rw=wl.rw)
        f.update(kw)
        return cls.make(**f)


class PlanInfo(ctypes.Structure):
    _fields_ = [("pairs_per_head", ctypes.c_longlong), ("n16", ctypes.c_longlong),
                ("n8", ctypes.c_longlong), ("n4", ctypes.c_longlong), ("nskip", ctypes.c_longlong),
                ("nb", ctypes.c_int), ("nry", ctypes.c_int), ("nrx", ctypes.c_int), ("N", ctypes.c_int),
                ("Np", ctypes.c_int), ("ws_bytes", ctypes.c_size_t)]


_P = ctypes.POINTER(Problem)
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_lib.da2_plan.argtypes = [_P, ctypes.POINTER(PlanInfo)]
_lib.da2_prepare.argtypes = [_P, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.da2_draft_rank.argtypes = [_P, _vp, _sz, _vp]
_lib.da2_rank_from_scores.argtypes = [_P, _vp, _vp, _sz, _vp]
_lib.da2_attention.argtypes = [_P, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
_lib.da2_dense_attention.argtypes = [ctypes.c_int] * 4 + [_vp] * 5
_lib.da2_dense_check_status.argtypes = [_vp]
_lib.da2_attention_wait_test.argtypes = [_P, _vp, _vp, _vp, _vp, _sz, _vp, ctypes.c_int, ctypes.c_uint, _vp]
_lib.da2_attention_occupancy.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
_lib.da2_debug_view.argtypes = [_P, _vp, ctypes.c_int, ctypes.POINTER(_vp), ctypes.POINTER(_sz)]
_lib.da2_rank_noalloc.argtypes = [_P, _vp, _vp, _vp, _vp, _vp]
_lib.da2_check_status.argtypes = [_P, _vp, _sz, _vp]
_lib.da2_host_bytes.argtypes = [_P, ctypes.c_int, ctypes.POINTER(_sz)]
_lib.da2_forward_host.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _sz, ctypes.c_int, _vp]
_lib.da2_status_string.argtypes = [ctypes.c_int]
_lib.da2_status_string.restype = ctypes.c_char_p
for _f in EXPORTS[:-1]:
    getattr(_lib, _f).restype = ctypes.c_int


class Da2Error(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn}: {da2_status_string(code)} ({code})")
        self.code = code


def _check(fn, code):
    if code != DA2_OK:
        raise Da2Error(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, t):
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def da2_status_string(code: int) -> str:
    return _lib.da2_status_string(code).decode()


def da2_plan(p: Problem) -> PlanInfo:
    info = PlanInfo()
    _check("da2_plan", _lib.da2_plan(ctypes.byref(p), ctypes.byref(info)))
    return info


def workspace(p: Problem, device="cuda") -> torch.Tensor:
    """Caller-owned workspace (a uint8 device tensor) for problem ``p``."""
    ws = torch.empty(da2_plan(p).ws_bytes, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def da2_prepare(p, q, k, v, ws, stream=None):
    _check("da2_prepare", _lib.da2_prepare(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(ws),
                                           ws.numel(), _stream(stream, ws)))


def da2_draft_rank(p, ws, stream=None):
    _check("da2_draft_rank", _lib.da2_draft_rank(ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream, ws)))


def da2_rank_from_scores(p, scores, ws, stream=None):
    _check("da2_rank_from_scores", _lib.da2_rank_from_scores(ctypes.byref(p), _ptr(scores), _ptr(ws),
                                                             ws.numel(), _stream(stream, ws)))


def da2_rank_noalloc(p, scores, prec_map, lists, counts, stream=None):
    """Ranking + assignment without a workspace, for callers that cannot
    allocate device memory at call time; its scratch is a fixed array inside
    the library (at most NOALLOC_MAX_HEADS batch x head pairs).  Outputs go to
    the caller's uint8 map, int16/uint16 lists and int32 counts tensors."""
    _check("da2_rank_noalloc", _lib.da2_rank_noalloc(ctypes.byref(p), _ptr(scores), _ptr(prec_map),
                                                     _ptr(lists), _ptr(counts), _stream(stream, scores)))


def da2_attention(p, q, k, v, ws, out, stream=None):
    _check("da2_attention", _lib.da2_attention(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(ws),
                                               ws.numel(), _ptr(out), _stream(stream, ws)))


def da2_check_status(p, ws, stream=None):
    """Synchronise `stream` and return the status of the last attention on `ws`
    (0, or DA2_ERR_TIMEOUT = 5 if a bounded wait in the kernel expired)."""
    return _lib.da2_check_status(ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream, ws))


def da2_host_bytes(p, heads_per_chunk):
    n = _sz()
    _check("da2_host_bytes", _lib.da2_host_bytes(ctypes.byref(p), int(heads_per_chunk), ctypes.byref(n)))
    return n.value


def host_buffer(p, heads_per_chunk, device="cuda") -> torch.Tensor:
    """Caller-owned device buffer (uint8) for `da2_forward_host`."""
    buf = torch.empty(da2_host_bytes(p, heads_per_chunk), dtype=torch.uint8, device=device)
    assert buf.data_ptr() % 256 == 0
    return buf


def da2_forward_host(p, q, k, v, out, dev, heads_per_chunk, stream=None):
    """The whole call on host (ideally pinned) bf16 tensors: chunks of
    `heads_per_chunk` (batch, head) slices, copies overlapped with kernels;
    returns once `out` holds the result."""
    for t in (q, k, v, out):
        if t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("da2_forward_host takes contiguous bf16 host tensors")
    _check("da2_forward_host", _lib.da2_forward_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                     _ptr(dev), dev.numel(), int(heads_per_chunk),
                                                     _stream(stream, dev)))
    return out


def da2_dense_attention(q, k, v, out, stream=None):
    B, H, N, d = q.shape
    _check("da2_dense_attention", _lib.da2_dense_attention(B, H, N, d, _ptr(q), _ptr(k), _ptr(v),
                                                           _ptr(out), _stream(stream, q)))


def da2_dense_check_status(stream=None):
    """Synchronise `stream` and return the dense calls' status (0, or
    DA2_ERR_TIMEOUT = 5 if a bounded wait in a dense kernel expired)."""
    return _lib.da2_dense_check_status(_vp(stream if isinstance(stream, int) else
                                           (stream.cuda_stream if stream is not None
                                            else torch.cuda.current_stream().cuda_stream)))


def da2_attention_wait_test(p, q, k, v, ws, out, withheld_cta, wait_polls, stream=None):
    """Failure-path test hook: da2_attention with every wait bounded by
    `wait_polls` polls and CTA `withheld_cta` never issuing its first key
    load.  Returns the call's status code (the kernel's own outcome is read
    with da2_check_status)."""
    return _lib.da2_attention_wait_test(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(ws), ws.numel(),
                                        _ptr(out), int(withheld_cta), int(wait_polls), _stream(stream, ws))


def da2_attention_occupancy(d, dense=False):
    """CTAs of the attention kernel (head dimension d) that one SM holds at once."""
    n = ctypes.c_int()
    _check("da2_attention_occupancy", _lib.da2_attention_occupancy(int(d), 1 if dense else 0, ctypes.byref(n)))
    return n.value


def da2_debug_view(p, ws, which):
    """(device address, bytes) of one workspace intermediate."""
    idx = VIEWS.index(which) if isinstance(which, str) else int(which)
    ptr, nbytes = _vp(), _sz()
    _check("da2_debug_view", _lib.da2_debug_view(ctypes.byref(p), _ptr(ws), idx, ctypes.byref(ptr),
                                                 ctypes.byref(nbytes)))
    return ptr.value, nbytes.value


def view(p, ws, which) -> torch.Tensor:
    """A typed, shaped torch view of one workspace intermediate (no copy)."""
    info = da2_plan(p)
    addr, nbytes = da2_debug_view(p, ws, which)
    off = addr - ws.data_ptr()
    raw = ws[off:off + nbytes]
    BH, nb, d = p.B * p.H, info.nb, p.d
    spec = {
        "PERM": (torch.int32, (nb, 64)),
        "Q_AVG": (torch.float32, (BH, nb, d)), "K_AVG": (torch.float32, (BH, nb, d)),
        "Q_MAX": (torch.float32, (BH, nb, d)), "K_MAX": (torch.float32, (BH, nb, d)),
        "Q_I8": (torch.int8, (BH, nb, 64, d)), "K_I8": (torch.int8, (BH, nb, 64, d)),
        "Q_S8": (torch.float32, (BH, nb)), "K_S8": (torch.float32, (BH, nb)),
        "Q_F4": (torch.uint8, (BH, nb, 64, d // 2)), "K_F4": (torch.uint8, (BH, nb, 64, d // 2)),
        "Q_SF4": (torch.uint8, (BH, nb, d // 64, 32, 16)), "K_SF4": (torch.uint8, (BH, nb, d // 64, 32, 16)),
        "V_I8": (torch.bfloat16, (BH, nb, 64, d)), "V_S8": (torch.float32, (BH, d)),
        "V_F4": (torch.uint8, (BH, nb, d, 32)), "V_SF4": (torch.uint8, (BH, nb, 32, 16)),
        "V_G4": (torch.float32, (BH, d)),
        "SCORES": (torch.float32, (BH, nb, nb)), "MAP": (torch.uint8, (BH, nb, nb)),
        "LISTS": (torch.int16, (BH, nb, nb)), "COUNTS": (torch.int32, (BH, nb, 4)),
        "STATUS": (torch.int32, (64,)),
    }[which if isinstance(which, str) else VIEWS[which]]
    return raw.view(spec[0]).view(spec[1])


def attention(p, q, k, v, ws, out, stream=None):
    """One DraftAttention2 call: prepare → draft/rank → attention, on one stream."""
    da2_prepare(p, q, k, v, ws, stream)
    da2_draft_rank(p, ws, stream)
    da2_attention(p, q, k, v, ws, out, stream)
    return out
