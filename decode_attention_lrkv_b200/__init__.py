"""Low-rank compressed-KV decode attention for NVIDIA B200 (sm_100a).

A thin Python binding over the C ABI of ``liblrkv.so`` (declared in
``include/lrkv.h``).  It only marshals arguments: PyTorch supplies device
memory and the stream, every step of the computation runs in the library's
CUDA kernels, and there is no CPU fallback -- importing works without a
GPU, but every compute call needs the built library and a CUDA device.

Entry points (same names as the C ABI):
    lrkv_workspace_size(dims) -> int
    lrkv_compress(dims, cache, k_new, v_new, tau, t_new_b=None, err_out=None, ws=...)
    lrkv_decode_attn(dims, cache, q, out, ws=...)
    lrkv_decode_attn_noalloc(dims, cache, q, out)   (scratch held by the library)
    lrkv_append_decode_attn(dims, cache, k_new, v_new, tau, q, out, t_new_b=None, err_out=None, ws=...)
    lrkv_fit_workspace_size(dims, n_rows) -> int
    lrkv_fit_basis(dims, X, r, ...) -> (U [Hkv,d,r] bf16, eigenvalues [Hkv,d] fp32)
    lrkv_rank_for_budget(eigvals, budget) -> int32 ranks   (host call)
    lrkv_oja_workspace_size(dims, n_rows, r) -> int
    lrkv_oja_update(dims, X, U, eta, U_out=None)   (online basis update, U fp32 in place)
    lrkv_status_str(code) -> str
plus ``LayerCache`` (allocates one layer's buffers with torch) and
``make_workspace``.
"""
import ctypes
import os
from dataclasses import dataclass

import torch

from . import accounting  # noqa: F401  (host-side byte accounting)

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblrkv.so")

LRKV_OK = 0
LRKV_ERR_INVALID_ARG = 1
STATUS_NAMES = {0: "LRKV_OK", 1: "LRKV_ERR_INVALID_ARG", 2: "LRKV_ERR_UNSUPPORTED",
                3: "LRKV_ERR_ALIGNMENT", 4: "LRKV_ERR_CUDA"}
DEV_FULL_OVERFLOW = 0x1
DEV_SEQ_OVERFLOW = 0x2
DEV_BAD_COUNT = 0x4
DEV_WAIT_TIMEOUT = 0x8


class LrkvError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({lrkv_status_str(code)})")


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "d", "r_k", "r_v", "T_cap", "F_cap",
                                               "coef_bits")]


class _Cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "U_k", "U_v", "coef_k", "coef_v", "route_mask", "full_idx", "full_k", "full_v",
        "full_cnt", "seq_len", "dev_status", "U_kq", "mu_k", "scale_k", "scale_v")]


_lib = None


def load_library(path=None):
    """Load liblrkv.so (built in-tree).  Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m decode_attention_lrkv_b200.build`")
    lib = ctypes.CDLL(p)
    P = ctypes.c_void_p
    lib.lrkv_workspace_size.argtypes = [ctypes.POINTER(_Dims)]
    lib.lrkv_workspace_size.restype = ctypes.c_size_t
    lib.lrkv_compress.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Cache), P, P,
                                  ctypes.c_int32, P, ctypes.c_float, P, P, ctypes.c_size_t, P]
    lib.lrkv_compress.restype = ctypes.c_int
    lib.lrkv_decode_attn.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Cache), P, P, P,
                                     ctypes.c_size_t, P]
    lib.lrkv_decode_attn.restype = ctypes.c_int
    lib.lrkv_decode_attn_noalloc.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Cache), P, P, P]
    lib.lrkv_decode_attn_noalloc.restype = ctypes.c_int
    lib.lrkv_append_decode_attn.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Cache), P, P, P,
                                            ctypes.c_float, P, P, P, P, ctypes.c_size_t, P]
    lib.lrkv_append_decode_attn.restype = ctypes.c_int
    lib.lrkv_fit_workspace_size.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int32]
    lib.lrkv_fit_workspace_size.restype = ctypes.c_size_t
    lib.lrkv_fit_basis.argtypes = [ctypes.POINTER(_Dims), P, ctypes.c_int32, ctypes.c_int32, P, P, P,
                                   ctypes.c_size_t, P]
    lib.lrkv_fit_basis.restype = ctypes.c_int
    lib.lrkv_oja_workspace_size.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int32, ctypes.c_int32]
    lib.lrkv_oja_workspace_size.restype = ctypes.c_size_t
    lib.lrkv_oja_update.argtypes = [ctypes.POINTER(_Dims), P, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.c_float, P, P, P, ctypes.c_size_t, P]
    lib.lrkv_oja_update.restype = ctypes.c_int
    lib.lrkv_rank_for_budget.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_double, P]
    lib.lrkv_rank_for_budget.restype = ctypes.c_int
    lib.lrkv_status_str.argtypes = [ctypes.c_int]
    lib.lrkv_status_str.restype = ctypes.c_char_p
    if path is None:
        _lib = lib
    return lib


@dataclass(frozen=True)
class Dims:
    B: int
    Hq: int
    Hkv: int
    d: int
    r_k: int
    r_v: int
    T_cap: int
    F_cap: int
    coef_bits: int = 0     # stored coefficients: 0/16 bf16, 8 int8 codes, 4 int4 codes

    @property
    def g(self):
        return self.Hq // self.Hkv

    @property
    def bits(self):
        return 16 if self.coef_bits == 0 else self.coef_bits

    def c(self):
        return _Dims(self.B, self.Hq, self.Hkv, self.d, self.r_k, self.r_v, self.T_cap, self.F_cap,
                     self.coef_bits)


class LayerCache:
    """One layer of compressed cache as torch tensors, in the C ABI's layout.

    bf16 tensors: U_k [Hkv,d,r_k], U_v [Hkv,d,r_v], coef_k [B,Hkv,T_cap,r_k],
    coef_v [B,Hkv,T_cap,r_v] (quantised caches: uint8 code bytes [B,Hkv,T_cap,r*bits/8]
    with fp32 scale_k/scale_v [B,Hkv,T_cap]), full_k/full_v [B,Hkv,F_cap,d];
    int32: route_mask [B,Hkv,T_cap/32] (bit patterns), full_idx [B,Hkv,F_cap],
    full_cnt [B,Hkv], seq_len [B]; dev_status int32 [4] (word 0 used).
    """
    FIELDS = ("U_k", "U_v", "coef_k", "coef_v", "route_mask", "full_idx", "full_k", "full_v",
              "full_cnt", "seq_len", "dev_status", "U_kq", "mu_k", "scale_k", "scale_v")

    def __init__(self, dims, U_k, U_v, device="cuda", U_kq=None, mu_k=None):
        D = dims
        self.dims = D
        z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device=device)
        self.U_k = U_k.to(device=device, dtype=torch.bfloat16).contiguous()
        self.U_v = U_v.to(device=device, dtype=torch.bfloat16).contiguous()
        assert tuple(self.U_k.shape) == (D.Hkv, D.d, D.r_k) and tuple(self.U_v.shape) == (D.Hkv, D.d, D.r_v)
        # attention-aware key basis (optional): query-side basis and key mean
        self.U_kq = None if U_kq is None else U_kq.to(device=device, dtype=torch.bfloat16).contiguous()
        self.mu_k = None if mu_k is None else mu_k.to(device=device, dtype=torch.float32).contiguous()
        assert self.U_kq is None or tuple(self.U_kq.shape) == (D.Hkv, D.d, D.r_k)
        assert self.mu_k is None or tuple(self.mu_k.shape) == (D.Hkv, D.d)
        if D.bits == 16:
            self.coef_k = z(D.B, D.Hkv, D.T_cap, D.r_k)
            self.coef_v = z(D.B, D.Hkv, D.T_cap, D.r_v)
            self.scale_k = self.scale_v = None
        else:   # integer codes (bytes; 4-bit codes two per byte) and per-row scales
            self.coef_k = z(D.B, D.Hkv, D.T_cap, D.r_k * D.bits // 8, dt=torch.uint8)
            self.coef_v = z(D.B, D.Hkv, D.T_cap, D.r_v * D.bits // 8, dt=torch.uint8)
            self.scale_k = z(D.B, D.Hkv, D.T_cap, dt=torch.float32)
            self.scale_v = z(D.B, D.Hkv, D.T_cap, dt=torch.float32)
        self.route_mask = z(D.B, D.Hkv, D.T_cap // 32, dt=torch.int32)
        self.full_idx = z(D.B, D.Hkv, max(D.F_cap, 1), dt=torch.int32)
        self.full_k = z(D.B, D.Hkv, max(D.F_cap, 1), D.d)
        self.full_v = z(D.B, D.Hkv, max(D.F_cap, 1), D.d)
        self.full_cnt = z(D.B, D.Hkv, dt=torch.int32)
        self.seq_len = z(D.B, dt=torch.int32)
        self.dev_status = z(4, dt=torch.int32)

    def c(self):
        return _Cache(*[None if getattr(self, f) is None else getattr(self, f).data_ptr()
                        for f in self.FIELDS])

    def nbytes(self):
        return sum(getattr(self, f).numel() * getattr(self, f).element_size() for f in self.FIELDS
                   if getattr(self, f) is not None)


def lrkv_rank_for_budget(eigvals, budget, check=True):
    """Smallest rank per head whose discarded eigenvalue mass is within `budget`
    of the total (host call; see include/lrkv.h).

    eigvals: [n_heads, d] fp32 on the host or the device (copied to the host),
    as returned by lrkv_fit_basis.  Returns an int32 tensor [n_heads] (CPU)."""
    lam = eigvals.detach().to("cpu", torch.float32).contiguous()
    if lam.dim() == 1:
        lam = lam.unsqueeze(0)
    r = torch.zeros(lam.shape[0], dtype=torch.int32)
    code = load_library().lrkv_rank_for_budget(lam.data_ptr(), int(lam.shape[0]), int(lam.shape[1]),
                                               float(budget), r.data_ptr())
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_rank_for_budget")
    return r


def lrkv_status_str(code):
    return load_library().lrkv_status_str(int(code)).decode()


def lrkv_workspace_size(dims):
    return int(load_library().lrkv_workspace_size(ctypes.byref(dims.c())))


def make_workspace(dims, device="cuda"):
    """A zero-filled workspace tensor of lrkv_workspace_size(dims) bytes."""
    n = lrkv_workspace_size(dims)
    if n == 0:
        raise ValueError(f"invalid dims {dims}")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def lrkv_compress(dims, cache, k_new, v_new, tau, t_new_b=None, err_out=None, ws=None,
                  stream=None, check=True):
    """Append k_new/v_new [B,t_new,Hkv,d] (bf16, device) to ``cache``; see include/lrkv.h."""
    lib = load_library()
    t_new = int(k_new.shape[1])
    code = lib.lrkv_compress(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(k_new),
                             _ptr(v_new), t_new, _ptr(t_new_b), float(tau), _ptr(err_out),
                             _ptr(ws), 0 if ws is None else ws.numel(), _stream_ptr(stream))
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_compress")
    return code


def lrkv_decode_attn(dims, cache, q, out, ws=None, stream=None, check=True):
    """out [B,Hq,d] fp32 <- decode attention of q [B,Hq,d] (bf16) over ``cache``."""
    lib = load_library()
    code = lib.lrkv_decode_attn(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(q), _ptr(out),
                                _ptr(ws), 0 if ws is None else ws.numel(), _stream_ptr(stream))
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_decode_attn")
    return code


def lrkv_decode_attn_noalloc(dims, cache, q, out, stream=None, check=True):
    """lrkv_decode_attn with the library's own device scratch instead of a workspace."""
    lib = load_library()
    code = lib.lrkv_decode_attn_noalloc(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(q),
                                        _ptr(out), _stream_ptr(stream))
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_decode_attn_noalloc")
    return code


def lrkv_append_decode_attn(dims, cache, k_new, v_new, tau, q, out, t_new_b=None, err_out=None,
                            ws=None, stream=None, check=True):
    """Append one token per row (k_new/v_new [B,1,Hkv,d] bf16) and attend with q, in one launch."""
    lib = load_library()
    assert int(k_new.shape[1]) == 1, "one new token per row"
    code = lib.lrkv_append_decode_attn(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(k_new),
                                       _ptr(v_new), _ptr(t_new_b), float(tau), _ptr(err_out),
                                       _ptr(q), _ptr(out), _ptr(ws), 0 if ws is None else ws.numel(),
                                       _stream_ptr(stream))
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_append_decode_attn")
    return code


def lrkv_oja_workspace_size(dims, n_rows, r):
    return int(load_library().lrkv_oja_workspace_size(ctypes.byref(dims.c()), int(n_rows), int(r)))


def lrkv_oja_update(dims, X, U, eta, U_out=None, ws=None, stream=None, check=True):
    """One Oja step of every kv head's basis U [Hkv, d, r] (fp32, updated in place)
    from rows X [..., Hkv, d] (bf16, device); U_out (optional bf16) receives the
    rounded basis.  See include/lrkv.h."""
    lib = load_library()
    n_rows = X.numel() // (dims.Hkv * dims.d)
    r = int(U.shape[-1])
    if ws is None:
        ws = torch.empty(max(lrkv_oja_workspace_size(dims, n_rows, r), 16), dtype=torch.uint8,
                         device=X.device)
    code = lib.lrkv_oja_update(ctypes.byref(dims.c()), _ptr(X), int(n_rows), r, float(eta), _ptr(U),
                               _ptr(U_out), _ptr(ws), ws.numel(), _stream_ptr(stream))
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_oja_update")
    return U_out


def lrkv_fit_workspace_size(dims, n_rows):
    return int(load_library().lrkv_fit_workspace_size(ctypes.byref(dims.c()), int(n_rows)))


def lrkv_fit_basis(dims, X, r, U_out=None, eigvals_out=None, ws=None, stream=None, check=True):
    """StaticPCA basis of every kv head from calibration rows X [..., Hkv, d] (bf16, device).

    Returns (U [Hkv, d, r] bf16, eigenvalues [Hkv, d] fp32 descending); see include/lrkv.h."""
    lib = load_library()
    n_rows = X.numel() // (dims.Hkv * dims.d)
    dev = X.device
    if U_out is None:
        U_out = torch.empty(dims.Hkv, dims.d, r, dtype=torch.bfloat16, device=dev)
    if eigvals_out is None:
        eigvals_out = torch.empty(dims.Hkv, dims.d, dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(lrkv_fit_workspace_size(dims, n_rows), 16), dtype=torch.uint8, device=dev)
    code = lib.lrkv_fit_basis(ctypes.byref(dims.c()), _ptr(X), int(n_rows), int(r), _ptr(U_out),
                              _ptr(eigvals_out), _ptr(ws), ws.numel(), _stream_ptr(stream))
    if check and code != LRKV_OK:
        raise LrkvError(code, "lrkv_fit_basis")
    return U_out, eigvals_out
