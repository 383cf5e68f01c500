"""Python binding of the sm_100a QLoRA linear-layer library (libqlora_nf4.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels; this module allocates outputs and workspace with torch, passes raw
device pointers and the current CUDA stream through the C ABI declared in
include/qlora_nf4.h, and turns status codes into exceptions. Importing the
package loads the shared library and fails loudly if it has not been built.

Layouts (see the C header): W0 [n, k] fp32; x [M, k] bf16; A [r, k] bf16;
B [n, r] bf16; h [M, n] bf16; dY [M, n] bf16; dX [M, k]; dA [r, k];
dB [n, r] (bf16).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libqlora_nf4.so")

# status codes (mirror of nf4_status)
NF4_OK = 0
NF4_ERR_INVALID_ARG = 1
NF4_ERR_UNSUPPORTED_SHAPE = 2
NF4_ERR_ALIGNMENT = 3
NF4_ERR_NONFINITE = 4
NF4_ERR_TIMEOUT = 5
NF4_ERR_CUDA = 6
NF4_ERR_WORKSPACE = 7

BLOCK_SIZE = 64
DQ_GROUP = 256


class NF4Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = ""
        if code == NF4_ERR_CUDA:
            detail = ": " + lib.nf4_last_cuda_error().decode(errors="replace")
        super().__init__(f"{where}: {status_string(code)} (status {code}){detail}")


class NF4WeightStruct(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64),
        ("k", ctypes.c_int64),
        ("block_size", ctypes.c_int32),
        ("double_quant", ctypes.c_int32),
        ("codes", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("absmax_q8", ctypes.c_void_p),
        ("absmax_c", ctypes.c_void_p),
    ]


class NF4KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m bit_nf4_quantized_05_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    u64 = ctypes.c_uint64
    W = ctypes.POINTER(NF4WeightStruct)
    sig = {
        "nf4_quantize": ([vp, W, vp], ctypes.c_int),
        "nf4_quantize_typed": ([vp, i32, W, vp], ctypes.c_int),
        "nf4_dequantize": ([W, vp, i32, vp], ctypes.c_int),
        "qlora_fwd_workspace_bytes": ([i64, i64, i64, i32], sz),
        "qlora_linear_fwd": ([W, vp, i64, vp, vp, i32, f32, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_linear_fwd_noalloc": ([W, vp, i64, vp, vp, i32, f32, vp, vp, vp], ctypes.c_int),
        "qlora_bwd_workspace_bytes": ([i64, i64, i64, i32], sz),
        "qlora_linear_bwd": ([W, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp],
                             ctypes.c_int),
        "qlora_linear_bwd_f32grad": ([W, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp],
                                     ctypes.c_int),
        "qlora_linear_fwd_dropout": ([W, vp, i64, vp, vp, i32, f32, f32, vp, vp, vp, vp, sz, vp],
                                     ctypes.c_int),
        "qlora_bwd_dropout_workspace_bytes": ([i64, i64, i64, i32], sz),
        "nf4_debug_flag_wait": ([i32, i64], ctypes.c_int),
        "nf4_last_cuda_error": ([], ctypes.c_char_p),
        "qlora_linear_fwd_dropout_philox": ([W, vp, i64, vp, vp, i32, f32, f32, u64, u64, vp, vp, vp,
                                             sz, vp], ctypes.c_int),
        "qlora_linear_bwd_dropout_philox": ([W, vp, i64, vp, vp, i32, f32, f32, u64, u64, vp, vp, vp,
                                             vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_linear_bwd_dropout": ([W, vp, i64, vp, vp, i32, f32, f32, vp, vp, vp, vp, vp, vp, vp,
                                      sz, vp], ctypes.c_int),
        "qlora_merge": ([W, vp, vp, i32, f32, vp, i32, vp], ctypes.c_int),
        "qlora_multi_lora_fwd": ([W, vp, i64, vp, vp, i32, i32, ctypes.POINTER(f32), vp, vp, vp, sz,
                                  vp], ctypes.c_int),
        "nf4_device_status": ([vp], ctypes.c_int),
        "nf4_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "nf4_profiling": ([i32], ctypes.c_int),
        "nf4_profile_read": ([ctypes.POINTER(NF4KernelTime), i32], ctypes.c_int32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


def status_string(code: int) -> str:
    return lib.nf4_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != NF4_OK:
        raise NF4Error(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts: torch.Tensor):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (the library has no CPU path)")


# The C entry points take raw pointers and the sizes below; they cannot see a
# tensor's extent, so every tensor is checked here against the shape the call
# implies before its pointer is passed on.
def _check_t(name: str, t: torch.Tensor, shape, dtype, device) -> None:
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the weight on {device}")


def _layer_args(qw: "QuantizedWeight", x: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                rank_cols: Optional[int] = None) -> Tuple[int, int]:
    """(M, r) of x [M, k], A [r, k] and B [n, r] (B [n, rank_cols] when given)."""
    if x.dim() != 2 or A.dim() != 2:
        raise ValueError("x and A must be 2-D")
    M, r = x.shape[0], A.shape[0]
    _check_t("x", x, (M, qw.k), torch.bfloat16, qw.device)
    _check_t("A", A, (r, qw.k), torch.bfloat16, qw.device)
    _check_t("B", B, (qw.n, r if rank_cols is None else rank_cols), torch.bfloat16, qw.device)
    return M, r


def _check_ws(ws: Optional[torch.Tensor], device) -> None:
    if ws is not None:
        if ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous() or ws.device != device:
            raise ValueError("workspace must be a contiguous 1-D uint8 tensor on the weight's device")


def _check_keep(keep: torch.Tensor, M: int, k: int, device) -> None:
    _check_t("keep", keep, (M * k // 8,), torch.uint8, device)


def _check_bwd(qw: "QuantizedWeight", M: int, r: int, dY: torch.Tensor, u: Optional[torch.Tensor],
               outs: Optional[tuple], workspace: Optional[torch.Tensor]) -> None:
    _check_t("dY", dY, (M, qw.n), torch.bfloat16, qw.device)
    if u is not None:
        _check_t("u", u, (M, r), torch.float32, qw.device)
    if outs is not None:
        dX, dA, dB = outs
        if dX is not None:
            _check_t("dX", dX, (M, qw.k), torch.bfloat16, qw.device)
        gdt = dA.dtype if dA.dtype in (torch.bfloat16, torch.float32) else torch.bfloat16
        _check_t("dA", dA, (r, qw.k), gdt, qw.device)
        _check_t("dB", dB, (qw.n, r), gdt, qw.device)
    _check_ws(workspace, qw.device)


@dataclass
class QuantizedWeight:
    """A frozen NF4 weight: device tensors owned by this object."""
    n: int
    k: int
    double_quant: bool
    codes: torch.Tensor                  # uint8 [n*k/2]
    absmax: torch.Tensor                 # fp32 [n*k/block_size]
    absmax_q8: Optional[torch.Tensor]    # uint8 [n*k/block_size]
    absmax_c: Optional[torch.Tensor]     # fp32 [ceil(n*k/block_size/256)]
    block_size: int = BLOCK_SIZE         # 64 or 128 elements per block

    def struct(self) -> NF4WeightStruct:
        self._check_arrays()
        return NF4WeightStruct(self.n, self.k, self.block_size, int(self.double_quant),
                               self.codes.data_ptr(), self.absmax.data_ptr(),
                               self.absmax_q8.data_ptr() if self.absmax_q8 is not None else None,
                               self.absmax_c.data_ptr() if self.absmax_c is not None else None)

    @property
    def device(self) -> torch.device:
        return self.codes.device

    def _check_arrays(self) -> None:
        """The arrays hold at least the entries the C library reads or writes."""
        if self.block_size not in (64, 128):
            raise ValueError("block_size must be 64 or 128")
        nb = self.n * self.k // self.block_size
        need = [("codes", self.codes, torch.uint8, self.n * self.k // 2),
                ("absmax", self.absmax, torch.float32, nb)]
        if self.double_quant:
            need += [("absmax_q8", self.absmax_q8, torch.uint8, nb),
                     ("absmax_c", self.absmax_c, torch.float32, (nb + 255) // 256)]
        for name, t, dtype, count in need:
            if t is None:
                raise ValueError(f"{name} is required")
            if t.dtype != dtype or not t.is_contiguous() or t.numel() < count or t.device != self.device:
                raise ValueError(f"{name}: expected a contiguous {dtype} tensor of at least {count} "
                                 f"entries on {self.device}")

    @staticmethod
    def empty(n: int, k: int, double_quant: bool, device, block_size: int = BLOCK_SIZE) -> "QuantizedWeight":
        if block_size not in (64, 128):
            raise ValueError("block_size must be 64 or 128")
        nb = n * k // block_size
        ng = (nb + DQ_GROUP - 1) // DQ_GROUP
        dev = torch.device(device)
        return QuantizedWeight(
            n, k, double_quant,
            torch.empty(n * k // 2, dtype=torch.uint8, device=dev),
            torch.empty(max(nb, 1), dtype=torch.float32, device=dev),
            torch.empty(max(nb, 1), dtype=torch.uint8, device=dev) if double_quant else None,
            torch.empty(max(ng, 1), dtype=torch.float32, device=dev) if double_quant else None,
            block_size)


_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}   # nf4_dtype


def nf4_quantize(W0: torch.Tensor, double_quant: bool = True,
                 out: Optional[QuantizedWeight] = None, block_size: int = BLOCK_SIZE) -> QuantizedWeight:
    """Blockwise NF4 quantisation of a [n, k] fp32, bf16 or fp16 CUDA tensor in
    blocks of 64 or 128 elements."""
    _need_cuda(W0)
    if W0.dtype not in _DTYPES or W0.dim() != 2 or not W0.is_contiguous():
        raise ValueError("W0 must be a contiguous 2-D float32, bfloat16 or float16 tensor")
    n, k = W0.shape
    if out is not None and ((out.n, out.k) != (n, k) or bool(out.double_quant) != bool(double_quant)
                            or out.device != W0.device):
        raise ValueError("out must be a weight of W0's shape, double-quant flag and device")
    qw = out if out is not None else QuantizedWeight.empty(n, k, double_quant, W0.device, block_size)
    s = qw.struct()
    if W0.dtype == torch.float32:
        _check(lib.nf4_quantize(_ptr(W0), ctypes.byref(s), _stream(W0.device)), "nf4_quantize")
    else:
        _check(lib.nf4_quantize_typed(_ptr(W0), _DTYPES[W0.dtype], ctypes.byref(s), _stream(W0.device)),
               "nf4_quantize_typed")
    return qw


def nf4_dequantize(qw: QuantizedWeight, bf16: bool = True) -> torch.Tensor:
    out = torch.empty(qw.n, qw.k, dtype=torch.bfloat16 if bf16 else torch.float32, device=qw.device)
    s = qw.struct()
    _check(lib.nf4_dequantize(ctypes.byref(s), _ptr(out), int(bf16), _stream(qw.device)),
           "nf4_dequantize")
    return out


def fwd_workspace_bytes(M: int, n: int, k: int, r: int) -> int:
    return int(lib.qlora_fwd_workspace_bytes(M, n, k, r))


def bwd_workspace_bytes(M: int, n: int, k: int, r: int) -> int:
    return int(lib.qlora_bwd_workspace_bytes(M, n, k, r))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def qlora_linear_fwd(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     alpha: float, save_u: bool = True, h: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, u: Optional[torch.Tensor] = None
                     ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """h = x W~^T + (alpha/r)(x A^T) B^T; also returns u = x A^T (fp32) if save_u."""
    M, r = _layer_args(qw, x, A, B)
    if h is not None:
        _check_t("h", h, (M, qw.n), torch.bfloat16, qw.device)
    if u is not None:
        _check_t("u", u, (M, r), torch.float32, qw.device)
    _check_ws(workspace, qw.device)
    _need_cuda(x, A, B)
    if h is None:
        h = torch.empty(M, qw.n, dtype=torch.bfloat16, device=x.device)
    if u is None and save_u:
        u = torch.empty(M, r, dtype=torch.float32, device=x.device)
    nbytes = fwd_workspace_bytes(M, qw.n, qw.k, r)
    ws = workspace if workspace is not None else _workspace(nbytes, x.device)
    s = qw.struct()
    _check(lib.qlora_linear_fwd(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                _ptr(h), _ptr(u), _ptr(ws), ws.numel(), _stream(x.device)),
           "qlora_linear_fwd")
    return h, u


def qlora_linear_fwd_noalloc(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor,
                             B: torch.Tensor, alpha: float, save_u: bool = True,
                             h: Optional[torch.Tensor] = None, u: Optional[torch.Tensor] = None
                             ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The forward without a workspace argument: the library uses its own fixed
    4 MiB device scratch, for callers that cannot allocate device memory while
    they run (see the C header for the token limit). Pass preallocated `h` and
    `u` to make the call itself allocation-free."""
    M, r = _layer_args(qw, x, A, B)
    if h is not None:
        _check_t("h", h, (M, qw.n), torch.bfloat16, qw.device)
    if u is not None:
        _check_t("u", u, (M, r), torch.float32, qw.device)
    _need_cuda(x, A, B)
    if h is None:
        h = torch.empty(M, qw.n, dtype=torch.bfloat16, device=x.device)
    if u is None and save_u:
        u = torch.empty(M, r, dtype=torch.float32, device=x.device)
    s = qw.struct()
    _check(lib.qlora_linear_fwd_noalloc(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r,
                                        float(alpha), _ptr(h), _ptr(u), _stream(x.device)),
           "qlora_linear_fwd_noalloc")
    return h, u


def qlora_linear_bwd(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     alpha: float, dY: torch.Tensor, u: Optional[torch.Tensor] = None,
                     need_dX: bool = True, workspace: Optional[torch.Tensor] = None,
                     outs: Optional[tuple] = None, grad_dtype: torch.dtype = torch.bfloat16):
    """(dX, dA, dB) of the layer; dX is None when need_dX is False. The adapter
    gradients are bf16 (qlora_linear_bwd) or fp32 (qlora_linear_bwd_f32grad):
    the dtype of the given outs, else grad_dtype."""
    M, r = _layer_args(qw, x, A, B)
    _check_bwd(qw, M, r, dY, u, outs, workspace)
    _need_cuda(x, A, B, dY)
    if outs is not None:
        dX, dA, dB = outs
    else:
        if grad_dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("adapter gradients are bf16 or fp32")
        dX = torch.empty(M, qw.k, dtype=torch.bfloat16, device=x.device) if need_dX else None
        dA = torch.empty(r, qw.k, dtype=grad_dtype, device=x.device)
        dB = torch.empty(qw.n, r, dtype=grad_dtype, device=x.device)
    nbytes = bwd_workspace_bytes(M, qw.n, qw.k, r)
    ws = workspace if workspace is not None else _workspace(nbytes, x.device)
    s = qw.struct()
    fn, name = ((lib.qlora_linear_bwd_f32grad, "qlora_linear_bwd_f32grad") if dA.dtype == torch.float32
                else (lib.qlora_linear_bwd, "qlora_linear_bwd"))
    _check(fn(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha), _ptr(dY), _ptr(u),
              _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream(x.device)), name)
    return dX, dA, dB


def qlora_multi_lora_fwd(qw: QuantizedWeight, x: torch.Tensor, A_all: torch.Tensor,
                         B_all: torch.Tensor, r: int, alphas, adapter_of_token: torch.Tensor,
                         h: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """h[m] = x[m] W~^T + (alphas[a]/r)(x[m] A_a^T) B_a^T with a = adapter_of_token[m]
    (int32 CUDA tensor; values outside [0, len(alphas)) mean no adapter). A_all stacks
    the adapters' A as [n_adapters * r, k], B_all their B as [n, n_adapters * r]."""
    n_ad = len(alphas)
    if n_ad < 1 or A_all.dim() != 2 or A_all.shape[0] != n_ad * r:
        raise ValueError("A_all must stack len(alphas) adapters of rank r: [len(alphas) * r, k]")
    M, _ = _layer_args(qw, x, A_all, B_all)
    _check_t("adapter_of_token", adapter_of_token, (M,), torch.int32, qw.device)
    if h is not None:
        _check_t("h", h, (M, qw.n), torch.bfloat16, qw.device)
    _check_ws(workspace, qw.device)
    _need_cuda(x, A_all, B_all, adapter_of_token)
    if h is None:
        h = torch.empty(M, qw.n, dtype=torch.bfloat16, device=x.device)
    nbytes = fwd_workspace_bytes(M, qw.n, qw.k, n_ad * r)
    ws = workspace if workspace is not None else _workspace(nbytes, x.device)
    al = (ctypes.c_float * n_ad)(*[float(a) for a in alphas])
    s = qw.struct()
    _check(lib.qlora_multi_lora_fwd(ctypes.byref(s), _ptr(x), M, _ptr(A_all), _ptr(B_all), int(r),
                                    n_ad, al, _ptr(adapter_of_token), _ptr(h), _ptr(ws), ws.numel(),
                                    _stream(x.device)), "qlora_multi_lora_fwd")
    return h


def qlora_merge(qw: QuantizedWeight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                bf16: bool = True, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """W~ + (alpha/r) B A as a [n, k] tensor (bf16, or fp32 for re-quantisation):
    the adapters folded into the dequantised frozen weight."""
    if A.dim() != 2:
        raise ValueError("A must be 2-D")
    r = A.shape[0]
    _check_t("A", A, (r, qw.k), torch.bfloat16, qw.device)
    _check_t("B", B, (qw.n, r), torch.bfloat16, qw.device)
    if out is not None:
        _check_t("out", out, (qw.n, qw.k), torch.bfloat16 if bf16 else torch.float32, qw.device)
    _need_cuda(A, B)
    if out is None:
        out = torch.empty(qw.n, qw.k, dtype=torch.bfloat16 if bf16 else torch.float32,
                          device=qw.device)
    s = qw.struct()
    _check(lib.qlora_merge(ctypes.byref(s), _ptr(A), _ptr(B), r, float(alpha), _ptr(out),
                           int(bf16), _stream(qw.device)), "qlora_merge")
    return out


def pack_keep(keep: torch.Tensor) -> torch.Tensor:
    """Device bit mask (uint8, bit e & 7 of byte e >> 3, e = m * k + kk) of a boolean
    [M, k] CUDA tensor of kept elements."""
    b = keep.reshape(-1, 8).to(torch.uint8)
    w = torch.tensor([1, 2, 4, 8, 16, 32, 64, 128], dtype=torch.uint8, device=keep.device)
    return (b * w).sum(dim=1, dtype=torch.int32).to(torch.uint8).contiguous()


def qlora_linear_fwd_dropout(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor,
                             B: torch.Tensor, alpha: float, p: float, keep: torch.Tensor,
                             save_u: bool = True, h: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None):
    """Forward with LoRA dropout; keep is the packed bit mask over x (see pack_keep).
    Returns (h, u) with u = (keep . x) A^T."""
    M, r = _layer_args(qw, x, A, B)
    _check_keep(keep, M, qw.k, qw.device)
    if h is not None:
        _check_t("h", h, (M, qw.n), torch.bfloat16, qw.device)
    _check_ws(workspace, qw.device)
    _need_cuda(x, A, B, keep)
    if h is None:
        h = torch.empty(M, qw.n, dtype=torch.bfloat16, device=x.device)
    u = torch.empty(M, r, dtype=torch.float32, device=x.device) if save_u else None
    ws = workspace if workspace is not None else _workspace(fwd_workspace_bytes(M, qw.n, qw.k, r), x.device)
    s = qw.struct()
    _check(lib.qlora_linear_fwd_dropout(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                        float(p), _ptr(keep), _ptr(h), _ptr(u), _ptr(ws), ws.numel(),
                                        _stream(x.device)), "qlora_linear_fwd_dropout")
    return h, u


def qlora_linear_bwd_dropout(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor,
                             B: torch.Tensor, alpha: float, p: float, keep: torch.Tensor,
                             dY: torch.Tensor, u: Optional[torch.Tensor] = None,
                             need_dX: bool = True, workspace: Optional[torch.Tensor] = None,
                             outs: Optional[tuple] = None):
    """(dX, dA, dB) with LoRA dropout (the mask of the forward)."""
    M, r = _layer_args(qw, x, A, B)
    _check_keep(keep, M, qw.k, qw.device)
    _check_bwd(qw, M, r, dY, u, outs, workspace)
    _need_cuda(x, A, B, dY, keep)
    if outs is not None:
        dX, dA, dB = outs
        if dA.dtype != torch.bfloat16:
            raise ValueError("the dropout backward writes bf16 adapter gradients")
    else:
        dX = torch.empty(M, qw.k, dtype=torch.bfloat16, device=x.device) if need_dX else None
        dA = torch.empty(r, qw.k, dtype=torch.bfloat16, device=x.device)
        dB = torch.empty(qw.n, r, dtype=torch.bfloat16, device=x.device)
    nbytes = int(lib.qlora_bwd_dropout_workspace_bytes(M, qw.n, qw.k, r))
    ws = workspace if workspace is not None else _workspace(nbytes, x.device)
    s = qw.struct()
    _check(lib.qlora_linear_bwd_dropout(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                        float(p), _ptr(keep), _ptr(dY), _ptr(u), _ptr(dX), _ptr(dA),
                                        _ptr(dB), _ptr(ws), ws.numel(), _stream(x.device)),
           "qlora_linear_bwd_dropout")
    return dX, dA, dB


def qlora_linear_fwd_dropout_philox(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor,
                                    B: torch.Tensor, alpha: float, p: float, seed: int,
                                    offset: int, save_u: bool = True,
                                    h: Optional[torch.Tensor] = None,
                                    workspace: Optional[torch.Tensor] = None):
    """Forward with LoRA dropout whose mask the kernels draw from Philox4x32-10
    at (seed, offset). Returns (h, u) with u = (keep . x) A^T."""
    M, r = _layer_args(qw, x, A, B)
    if h is not None:
        _check_t("h", h, (M, qw.n), torch.bfloat16, qw.device)
    _check_ws(workspace, qw.device)
    _need_cuda(x, A, B)
    if h is None:
        h = torch.empty(M, qw.n, dtype=torch.bfloat16, device=x.device)
    u = torch.empty(M, r, dtype=torch.float32, device=x.device) if save_u else None
    ws = workspace if workspace is not None else _workspace(fwd_workspace_bytes(M, qw.n, qw.k, r), x.device)
    s = qw.struct()
    _check(lib.qlora_linear_fwd_dropout_philox(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r,
                                               float(alpha), float(p), int(seed) & (2 ** 64 - 1),
                                               int(offset) & (2 ** 64 - 1), _ptr(h), _ptr(u), _ptr(ws),
                                               ws.numel(), _stream(x.device)),
           "qlora_linear_fwd_dropout_philox")
    return h, u


def qlora_linear_bwd_dropout_philox(qw: QuantizedWeight, x: torch.Tensor, A: torch.Tensor,
                                    B: torch.Tensor, alpha: float, p: float, seed: int,
                                    offset: int, dY: torch.Tensor,
                                    u: Optional[torch.Tensor] = None, need_dX: bool = True,
                                    workspace: Optional[torch.Tensor] = None,
                                    outs: Optional[tuple] = None):
    """(dX, dA, dB) with LoRA dropout, the mask regenerated from the forward's
    (p, seed, offset)."""
    M, r = _layer_args(qw, x, A, B)
    _check_bwd(qw, M, r, dY, u, outs, workspace)
    _need_cuda(x, A, B, dY)
    if outs is not None:
        dX, dA, dB = outs
        if dA.dtype != torch.bfloat16:
            raise ValueError("the dropout backward writes bf16 adapter gradients")
    else:
        dX = torch.empty(M, qw.k, dtype=torch.bfloat16, device=x.device) if need_dX else None
        dA = torch.empty(r, qw.k, dtype=torch.bfloat16, device=x.device)
        dB = torch.empty(qw.n, r, dtype=torch.bfloat16, device=x.device)
    nbytes = int(lib.qlora_bwd_dropout_workspace_bytes(M, qw.n, qw.k, r))
    ws = workspace if workspace is not None else _workspace(nbytes, x.device)
    s = qw.struct()
    _check(lib.qlora_linear_bwd_dropout_philox(ctypes.byref(s), _ptr(x), M, _ptr(A), _ptr(B), r,
                                               float(alpha), float(p), int(seed) & (2 ** 64 - 1),
                                               int(offset) & (2 ** 64 - 1), _ptr(dY), _ptr(u),
                                               _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(),
                                               _stream(x.device)),
           "qlora_linear_bwd_dropout_philox")
    return dX, dA, dB


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    dev = torch.device("cuda" if device is None else device)
    return int(lib.nf4_device_status(_stream(dev)))


def profiling(enable: bool) -> None:
    """Enable (and clear) or disable per-kernel event timing inside the library."""
    _check(lib.nf4_profiling(int(enable)), "nf4_profiling")


def profile_read() -> dict:
    """{kernel kind: (launches, total milliseconds)} for the launches recorded
    since profiling was last enabled (synchronises the recorded events)."""
    buf = (NF4KernelTime * 32)()
    n = lib.nf4_profile_read(buf, 32)
    if n < 0:
        raise NF4Error(NF4_ERR_CUDA, "nf4_profile_read")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(n)}
