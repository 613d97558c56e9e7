"""ctypes binding of libcta (include/cta.h): argument marshalling only.

Every step of the computation runs in the CUDA kernels of ``libcta.so``; this
module only turns torch tensors into pointers and sizes, allocates outputs and
the workspace with torch (device memory is plumbing), and checks return
codes.  There is no fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcta.so")

CTA_F32, CTA_BF16 = 0, 1
CTA_OK = 0
CTA_DEV_NONFINITE = 0x1
CTA_DEV_INTERNAL = 0x2
CTA_DEV_TIMEOUT = 0x4

# Entry points declared in include/cta.h; the CPU test checks each is exported.
EXPORTED = ("cta_opts_init", "cta_workspace_size", "cta_certified_topk_attn", "cta_dense_attn",
            "cta_status_string", "cta_version", "cta_certified_topk_attn_noalloc")
CTA_ERR_TOO_LARGE = -7
NOALLOC_SCRATCH_BYTES = 32 << 20


class cta_opts(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("m", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("reserved0", ctypes.c_int32),
        ("stream", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("err_out", ctypes.c_void_p),
        ("kl_out", ctypes.c_void_p),
        ("status_dev", ctypes.c_void_p),
        ("phase_events", ctypes.c_void_p),
        ("gap_out", ctypes.c_void_p),
    ]


class CtaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where} failed: {cta_status_string(code)} (status {code})")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load libcta.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libcta.so is not built at {LIB_PATH}; run __graft_entry__.build()")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.cta_opts_init.argtypes = [ctypes.POINTER(cta_opts)]
        lib.cta_opts_init.restype = None
        lib.cta_workspace_size.argtypes = [i64, i32, i32, i32, ctypes.POINTER(cta_opts)]
        lib.cta_workspace_size.restype = ctypes.c_size_t
        lib.cta_certified_topk_attn.argtypes = [vp, vp, vp, i64, i32, i32, i32, dbl, vp, vp, vp, vp,
                                                ctypes.POINTER(cta_opts)]
        lib.cta_certified_topk_attn.restype = i32
        lib.cta_certified_topk_attn_noalloc.argtypes = lib.cta_certified_topk_attn.argtypes
        lib.cta_certified_topk_attn_noalloc.restype = i32
        lib.cta_dense_attn.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, ctypes.POINTER(cta_opts)]
        lib.cta_dense_attn.restype = i32
        lib.cta_status_string.argtypes = [i32]
        lib.cta_status_string.restype = ctypes.c_char_p
        lib.cta_version.argtypes = []
        lib.cta_version.restype = i32
        _lib = lib
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CTA_F32
    if t.dtype == torch.bfloat16:
        return CTA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; libcta takes float32 or bfloat16")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def cta_status_string(code: int) -> str:
    return load().cta_status_string(int(code)).decode()


def cta_version() -> int:
    return int(load().cta_version())


def make_opts(*, batch=1, m=1, dtype=CTA_BF16, stream=None, workspace=None, err_out=None,
              kl_out=None, status_dev=None, phase_events=None, gap_out=None) -> cta_opts:
    o = cta_opts()
    load().cta_opts_init(ctypes.byref(o))
    o.batch, o.m, o.dtype = int(batch), int(m), int(dtype)
    o.stream = stream
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    o.err_out = None if err_out is None else err_out.data_ptr()
    o.kl_out = None if kl_out is None else kl_out.data_ptr()
    o.status_dev = None if status_dev is None else status_dev.data_ptr()
    o.phase_events = phase_events
    o.gap_out = None if gap_out is None else gap_out.data_ptr()
    return o


def cta_workspace_size(n: int, d: int, n_heads: int, n_kv_heads: int, *, batch=1, m=1,
                       dtype=CTA_BF16) -> int:
    o = make_opts(batch=batch, m=m, dtype=dtype)
    return int(load().cta_workspace_size(int(n), int(d), int(n_heads), int(n_kv_heads),
                                         ctypes.byref(o)))


def _shape(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor):
    if q.dim() != 4 or K.dim() != 4 or V.dim() != 4:
        raise ValueError("q is [batch, n_heads, m, d]; K, V are [batch, n_kv_heads, n, d]")
    batch, n_heads, m, d = q.shape
    kb, n_kv_heads, n, kd = K.shape
    if kb != batch or kd != d or tuple(V.shape) != tuple(K.shape):
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, K {tuple(K.shape)}, V {tuple(V.shape)}")
    for t in (q, K, V):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError("q, K, V must be contiguous CUDA tensors of one dtype")
    return batch, n_heads, m, d, n_kv_heads, n


def cta_certified_topk_attn(q, K, V, eps, *, out=None, k_out=None, idx_out=None, tv_out=None,
                            err_out=None, kl_out=None, want_err=True, want_kl=True,
                            gap_out=None, want_gap=False, workspace=None, status_dev=None,
                            stream=None, phase_events=None):
    """Certified Top-k attention through libcta.

    Returns a dict of device tensors: ``out`` [batch, n_heads, m, d],
    ``k`` [batch, n_heads, m] int32, ``idx`` [batch, n_heads, m, n] int32
    (entries [0, k) of each row are the kept keys, ascending), ``tv``, ``err``,
    ``kl`` and ``gap`` (the single-gap certificate) [batch, n_heads, m] fp32
    (``err``/``kl``/``gap`` None when not wanted).
    """
    batch, n_heads, m, d, n_kv_heads, n = _shape(q, K, V)
    dev = q.device
    rows = (batch, n_heads, m)
    out = torch.empty_like(q) if out is None else out
    k_out = torch.empty(rows, dtype=torch.int32, device=dev) if k_out is None else k_out
    idx_out = torch.empty((*rows, n), dtype=torch.int32, device=dev) if idx_out is None else idx_out
    tv_out = torch.empty(rows, dtype=torch.float32, device=dev) if tv_out is None else tv_out
    if want_err and err_out is None:
        err_out = torch.empty(rows, dtype=torch.float32, device=dev)
    if want_kl and kl_out is None:
        kl_out = torch.empty(rows, dtype=torch.float32, device=dev)
    if want_gap and gap_out is None:
        gap_out = torch.empty(rows, dtype=torch.float32, device=dev)
    code = _dtype_code(q)
    if workspace is None:
        nbytes = cta_workspace_size(n, d, n_heads, n_kv_heads, batch=batch, m=m, dtype=code)
        if nbytes == 0:
            raise CtaError(-2, "cta_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    o = make_opts(batch=batch, m=m, dtype=code, stream=_stream_handle(stream), workspace=workspace,
                  err_out=err_out if want_err else None, kl_out=kl_out if want_kl else None,
                  status_dev=status_dev, phase_events=phase_events,
                  gap_out=gap_out if want_gap else None)
    rc = load().cta_certified_topk_attn(_ptr(q), _ptr(K), _ptr(V), n, d, n_heads, n_kv_heads,
                                        float(eps), _ptr(out), _ptr(k_out), _ptr(idx_out),
                                        _ptr(tv_out), ctypes.byref(o))
    if rc != CTA_OK:
        raise CtaError(rc, "cta_certified_topk_attn")
    return {"out": out, "k": k_out, "idx": idx_out, "tv": tv_out,
            "err": err_out if want_err else None, "kl": kl_out if want_kl else None,
            "gap": gap_out if want_gap else None}


def cta_dense_attn(q, K, V, *, out=None, stream=None):
    """Dense softmax attention over all keys (reference output), via libcta."""
    batch, n_heads, m, d, n_kv_heads, n = _shape(q, K, V)
    out = torch.empty_like(q) if out is None else out
    o = make_opts(batch=batch, m=m, dtype=_dtype_code(q), stream=_stream_handle(stream))
    rc = load().cta_dense_attn(_ptr(q), _ptr(K), _ptr(V), n, d, n_heads, n_kv_heads, _ptr(out),
                               ctypes.byref(o))
    if rc != CTA_OK:
        raise CtaError(rc, "cta_dense_attn")
    return out


def cta_certified_topk_attn_noalloc(q, K, V, eps, *, out, k_out, idx_out, tv_out, err_out=None,
                                    kl_out=None, status_dev=None, stream=None):
    """The no-allocation entry point: the library's own fixed scratch replaces
    the workspace.  Every output must be passed in (this wrapper allocates
    nothing either).  Returns the same dict of (the caller's) tensors as
    cta_certified_topk_attn.  See include/cta.h for its limits and ordering
    rules."""
    batch, n_heads, m, d, n_kv_heads, n = _shape(q, K, V)
    o = make_opts(batch=batch, m=m, dtype=_dtype_code(q), stream=_stream_handle(stream),
                  err_out=err_out, kl_out=kl_out, status_dev=status_dev)
    rc = load().cta_certified_topk_attn_noalloc(_ptr(q), _ptr(K), _ptr(V), n, d, n_heads,
                                                n_kv_heads, float(eps), _ptr(out), _ptr(k_out),
                                                _ptr(idx_out), _ptr(tv_out), ctypes.byref(o))
    if rc != CTA_OK:
        raise CtaError(rc, "cta_certified_topk_attn_noalloc")
    return {"out": out, "k": k_out, "idx": idx_out, "tv": tv_out, "err": err_out, "kl": kl_out}
