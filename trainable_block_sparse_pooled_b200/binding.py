"""ctypes binding of libspa2.so (C ABI in include/spa2.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. The functions keep the C names (``spa2_block_mask`` ...) and take
device pointers as Python ints; ``Spa2`` below adds torch-tensor conveniences
(buffer allocation through torch, the current CUDA stream) for tests, the
bench and users. There is no fallback: if the library is missing or a call
fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import math
import os
import re
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libspa2.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "spa2.h")

(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_WORKSPACE, ERR_DEVICE_BOUNDS,
 ERR_RANGE) = range(8)
OP_MASK, OP_FWD, OP_BWD, OP_SELECT = range(4)
DTYPE_BF16, DTYPE_F32 = 0, 1
BQ, BKV = 128, 64


class Spa2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} (status {code})")
        self.code = code


class spa2_mask(ctypes.Structure):
    _fields_ = [
        ("row_cnt", ctypes.c_void_p),
        ("row_idx", ctypes.c_void_p),
        ("col_cnt", ctypes.c_void_p),
        ("col_idx", ctypes.c_void_p),
        ("pbar", ctypes.c_void_p),
        ("bitmap", ctypes.c_void_p),
    ]


_lib = None

_SIGS = {
    "spa2_abi_version": (ctypes.c_int, []),
    "spa2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "spa2_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 7),
    "spa2_block_mask": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 6
                        + [ctypes.c_float, ctypes.c_float, ctypes.POINTER(spa2_mask), ctypes.c_void_p,
                           ctypes.c_size_t, ctypes.c_void_p]),
    "spa2_block_mask_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 6
                                + [ctypes.c_float, ctypes.c_float, ctypes.POINTER(spa2_mask), ctypes.c_void_p,
                                   ctypes.c_void_p]),
    "spa2_select_blocks": (ctypes.c_int, [ctypes.c_void_p] + [ctypes.c_int] * 4
                           + [ctypes.c_float, ctypes.c_float, ctypes.POINTER(spa2_mask), ctypes.c_void_p,
                              ctypes.c_size_t, ctypes.c_void_p]),
    "spa2_sparse_attn_fwd": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6
                             + [ctypes.POINTER(spa2_mask), ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "spa2_sparse_attn_bwd": (ctypes.c_int, [ctypes.c_void_p] * 7 + [ctypes.c_int] * 6
                             + [ctypes.POINTER(spa2_mask), ctypes.c_float] + [ctypes.c_void_p] * 3
                             + [ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "spa2_stream_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "spa2_debug_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_longlong]),
    "spa2_debug_timeout_probe": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "spa2_timing_enable": (ctypes.c_int, [ctypes.c_int]),
    "spa2_kernel_count": (ctypes.c_int, []),
    "spa2_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
    "spa2_timing_read": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]),
}


def header_symbols(path: str = HEADER) -> list[str]:
    """Names of every function the C header declares."""
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spa2_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load libspa2.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m trainable_block_sparse_pooled_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().spa2_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != OK:
        raise Spa2Error(code, what)


# ---- C-named wrappers (raw pointers as ints) --------------------------------
def spa2_abi_version() -> int:
    return lib().spa2_abi_version()


def spa2_workspace_bytes(op, B, H, N, d, bq=BQ, bkv=BKV) -> int:
    return lib().spa2_workspace_bytes(op, B, H, N, d, bq, bkv)


def spa2_block_mask(q, k, B, H, N, d, bq, bkv, k_frac, p_frac, mask: spa2_mask, ws, ws_bytes, stream) -> int:
    return lib().spa2_block_mask(q, k, B, H, N, d, bq, bkv, k_frac, p_frac, ctypes.byref(mask), ws, ws_bytes,
                                 stream)


def spa2_block_mask_noalloc(q, k, B, H, N, d, bq, bkv, k_frac, p_frac, mask: spa2_mask, status, stream) -> int:
    return lib().spa2_block_mask_noalloc(q, k, B, H, N, d, bq, bkv, k_frac, p_frac, ctypes.byref(mask), status,
                                         stream)


def spa2_select_blocks(pbar, B, H, Tm, Tn, k_frac, p_frac, mask: spa2_mask, ws, ws_bytes, stream) -> int:
    return lib().spa2_select_blocks(pbar, B, H, Tm, Tn, k_frac, p_frac, ctypes.byref(mask), ws, ws_bytes, stream)


def spa2_sparse_attn_fwd(q, k, v, B, H, N, d, bq, bkv, mask: spa2_mask, scale, o, o_lo, lse, ws, ws_bytes,
                         stream) -> int:
    return lib().spa2_sparse_attn_fwd(q, k, v, B, H, N, d, bq, bkv, ctypes.byref(mask), scale, o, o_lo, lse, ws,
                                      ws_bytes, stream)


def spa2_sparse_attn_bwd(q, k, v, o, o_lo, lse, dout, B, H, N, d, bq, bkv, mask: spa2_mask, scale, dq, dk, dv,
                         grad_dtype, ws, ws_bytes, stream) -> int:
    return lib().spa2_sparse_attn_bwd(q, k, v, o, o_lo, lse, dout, B, H, N, d, bq, bkv, ctypes.byref(mask), scale,
                                      dq, dk, dv, grad_dtype, ws, ws_bytes, stream)


def spa2_stream_status(ws, stream) -> int:
    return lib().spa2_stream_status(ws, stream)


def spa2_debug_set_wait_limit_ns(limit: int) -> int:
    return lib().spa2_debug_set_wait_limit_ns(int(limit))


def spa2_debug_timeout_probe(ws, ws_bytes, stream) -> int:
    return lib().spa2_debug_timeout_probe(ws, ws_bytes, stream)


def spa2_timing_enable(on: bool) -> int:
    return lib().spa2_timing_enable(1 if on else 0)


def spa2_kernel_count() -> int:
    return lib().spa2_kernel_count()


def spa2_kernel_name(kernel_id: int) -> str:
    return lib().spa2_kernel_name(int(kernel_id)).decode()


def spa2_timing_read() -> dict:
    """{kernel name: (launches, summed event ms)} since the last read (kernels
    with no launch omitted); waits for the recorded events."""
    n = spa2_kernel_count()
    launches = (ctypes.c_int * n)()
    ms = (ctypes.c_double * n)()
    _check(lib().spa2_timing_read(n, launches, ms), "spa2_timing_read")
    return {spa2_kernel_name(i): (launches[i], ms[i]) for i in range(n) if launches[i]}


# ---- torch conveniences -------------------------------------------------------
@dataclass
class Mask:
    """Device buffers of one block mask (torch tensors) and its C view."""
    row_cnt: "object"
    row_idx: "object"
    col_cnt: "object"
    col_idx: "object"
    pbar: "object" = None
    bitmap: "object" = None

    def c(self) -> spa2_mask:
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        return spa2_mask(p(self.row_cnt), p(self.row_idx), p(self.col_cnt), p(self.col_idx), p(self.pbar),
                         p(self.bitmap))

    def kept_blocks(self) -> int:
        return int(self.row_cnt.sum().item())


def block_counts(N: int, bq: int = BQ, bkv: int = BKV) -> tuple[int, int]:
    return math.ceil(N / bq), math.ceil(N / bkv)


def _stream(torch):
    return torch.cuda.current_stream().cuda_stream


class Spa2:
    """Torch-tensor front end of the C ABI for one problem shape.

    Buffers (mask, workspaces, outputs) are allocated through torch by the
    caller side of the ABI; the library itself never allocates.
    """

    def __init__(self, B, H, N, d, device="cuda", with_pbar=False, with_bitmap=False, bq=BQ, bkv=BKV):
        import torch
        self.torch = torch
        self.B, self.H, self.N, self.d = B, H, N, d
        self.bq, self.bkv = bq, bkv
        self.Tm, self.Tn = block_counts(N, bq, bkv)
        self.device = device
        L = lib()
        self.ws_bytes = {op: L.spa2_workspace_bytes(op, B, H, N, d, bq, bkv) for op in (OP_MASK, OP_FWD, OP_BWD)}
        if min(self.ws_bytes.values()) == 0:
            raise Spa2Error(ERR_UNSUPPORTED, f"shape B={B} H={H} N={N} d={d} bq={bq} bkv={bkv}")
        # zero-filled so that the status word of an op never run reads as OK
        self.ws = {op: torch.zeros(n, dtype=torch.uint8, device=device) for op, n in self.ws_bytes.items()}
        self.with_pbar, self.with_bitmap = with_pbar, with_bitmap

    def new_mask(self) -> Mask:
        t, B, H, Tm, Tn = self.torch, self.B, self.H, self.Tm, self.Tn
        i32 = dict(dtype=t.int32, device=self.device)
        return Mask(t.empty(B, H, Tm, **i32), t.empty(B, H, Tm, Tn, **i32), t.empty(B, H, Tn, **i32),
                    t.empty(B, H, Tn, Tm, **i32),
                    t.empty(B, H, Tm, Tn, dtype=t.float32, device=self.device) if self.with_pbar else None,
                    t.empty(B, H, Tm, Tn, dtype=t.uint8, device=self.device) if self.with_bitmap else None)

    def block_mask(self, q, k, k_frac, p_frac, mask: Mask | None = None) -> Mask:
        mask = mask or self.new_mask()
        cm = mask.c()
        ws = self.ws[OP_MASK]
        _check(spa2_block_mask(q.data_ptr(), k.data_ptr(), self.B, self.H, self.N, self.d, self.bq, self.bkv,
                               float(k_frac),
                               float(p_frac), cm, ws.data_ptr(), ws.numel(), _stream(self.torch)), "spa2_block_mask")
        return mask

    def fwd(self, q, k, v, mask: Mask, scale=0.0, o=None, lse=None, o_lo=None, want_o_lo=True):
        """O (bf16), LSE (fp32) and, if wanted, O's bf16 residual for the backward."""
        t = self.torch
        o = t.empty_like(q) if o is None else o
        if want_o_lo and o_lo is None:
            o_lo = t.empty_like(q)
        lse = t.empty(self.B, self.H, self.N, dtype=t.float32, device=q.device) if lse is None else lse
        cm = mask.c()
        ws = self.ws[OP_FWD]
        _check(spa2_sparse_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), self.B, self.H, self.N, self.d, self.bq,
                                    self.bkv, cm, float(scale), o.data_ptr(), None if o_lo is None else o_lo.data_ptr(),
                                    lse.data_ptr(), ws.data_ptr(), ws.numel(), _stream(t)), "spa2_sparse_attn_fwd")
        self.o_lo = o_lo
        return o, lse

    def bwd(self, q, k, v, o, lse, dout, mask: Mask, scale=0.0, dq=None, dk=None, dv=None, o_lo="auto",
            grad_dtype=DTYPE_F32):
        """dQ, dK, dV (fp32 by default; grad_dtype=DTYPE_BF16 for bf16)."""
        t = self.torch
        gt = t.float32 if grad_dtype == DTYPE_F32 else t.bfloat16
        dq = t.empty(q.shape, dtype=gt, device=q.device) if dq is None else dq
        dk = t.empty(k.shape, dtype=gt, device=q.device) if dk is None else dk
        dv = t.empty(v.shape, dtype=gt, device=q.device) if dv is None else dv
        if isinstance(o_lo, str):
            o_lo = getattr(self, "o_lo", None)
        cm = mask.c()
        ws = self.ws[OP_BWD]
        _check(spa2_sparse_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                    None if o_lo is None else o_lo.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                                    self.B, self.H, self.N, self.d, self.bq, self.bkv, cm, float(scale), dq.data_ptr(),
                                    dk.data_ptr(), dv.data_ptr(), int(grad_dtype), ws.data_ptr(), ws.numel(),
                                    _stream(t)), "spa2_sparse_attn_bwd")
        return dq, dk, dv

    def check(self, op=None):
        """Synchronise and raise if a device-side error was recorded."""
        for o in ([op] if op is not None else list(self.ws)):
            _check(spa2_stream_status(self.ws[o].data_ptr(), _stream(self.torch)), f"device status (op {o})")


def select_blocks(pbar, k_frac, p_frac, with_csc=True, with_bitmap=True) -> Mask:
    """Selection alone on a given P-bar [B, H, T_m, T_n] fp32 CUDA tensor."""
    import torch
    B, H, Tm, Tn = pbar.shape
    i32 = dict(dtype=torch.int32, device=pbar.device)
    m = Mask(torch.empty(B, H, Tm, **i32), torch.empty(B, H, Tm, Tn, **i32),
             torch.empty(B, H, Tn, **i32) if with_csc else None,
             torch.empty(B, H, Tn, Tm, **i32) if with_csc else None, None,
             torch.empty(B, H, Tm, Tn, dtype=torch.uint8, device=pbar.device) if with_bitmap else None)
    n = lib().spa2_workspace_bytes(OP_SELECT, B, H, Tm, Tn, 0, 0)
    ws = torch.empty(n, dtype=torch.uint8, device=pbar.device)
    cm = m.c()
    s = torch.cuda.current_stream().cuda_stream
    pbar = pbar.contiguous()
    _check(spa2_select_blocks(pbar.data_ptr(), B, H, Tm, Tn, float(k_frac), float(p_frac), cm,
                              ws.data_ptr(), n, s), "spa2_select_blocks")
    _check(spa2_stream_status(ws.data_ptr(), s), "spa2_select_blocks device status")
    return m
