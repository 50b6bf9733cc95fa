"""NVFP4 block-scaled GEMM for NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/nvfp4_gemm.h``
(``libnvfp4gemm.so``): it checks tensor shapes and dtypes, passes raw device
pointers and the current CUDA stream, and raises on a non-OK status.  Every
step of the computation runs in the library's CUDA kernels; PyTorch is used
only for device memory and streams.  There is no CPU fallback: if the library
is missing, importing the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4gemm.so")

STATUS = {
    0: "NVFP4_OK",
    1: "NVFP4_ERR_INVALID_ARG",
    2: "NVFP4_ERR_UNSUPPORTED_SHAPE",
    3: "NVFP4_ERR_UNSUPPORTED_DEVICE",
    4: "NVFP4_ERR_CUDA",
    5: "NVFP4_ERR_TIMEOUT",
    6: "NVFP4_ERR_NO_MEMORY",
}

# Every symbol include/nvfp4_gemm.h declares.
EXPORTS = (
    "nvfp4_gemm", "nvfp4_gemm_ex", "nvfp4_grouped_gemm", "nvfp4_quantize", "nvfp4_swizzle_scales",
    "nvfp4_swizzled_scale_bytes", "nvfp4_get_device_error", "nvfp4_status_string",
    "nvfp4_debug_wait_timeout", "nvfp4_version", "nvfp4_kernel_launches",
    "nvfp4_gemm_noalloc", "nvfp4_fp4_peak_probe", "nvfp4_quantize_scaled", "nvfp4_gemm_bf16a",
    "nvfp4_gemm_sparse24", "nvfp4_gemm_mxfp4",
)


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnvfp4gemm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m nvfp4_block_scaled_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.nvfp4_gemm.argtypes = [P, P, P, P, f32, P, i32, i32, i32, P]
        L.nvfp4_gemm_ex.argtypes = [P, P, P, P, f32, P, i32, i32, i32, ctypes.c_uint, P]
        L.nvfp4_grouped_gemm.argtypes = [P, P, P, P, P, P, i32, P, i32, i32, i32, P]
        L.nvfp4_quantize.argtypes = [P, i32, i32, P, P, P, P]
        L.nvfp4_swizzle_scales.argtypes = [P, i32, i32, P, P]
        L.nvfp4_swizzled_scale_bytes.argtypes = [i32, i32]
        L.nvfp4_swizzled_scale_bytes.restype = ctypes.c_size_t
        L.nvfp4_get_device_error.argtypes = [P]
        L.nvfp4_status_string.argtypes = [i32]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_debug_wait_timeout.argtypes = [ctypes.c_uint64, P]
        for name in ("nvfp4_gemm", "nvfp4_gemm_ex", "nvfp4_grouped_gemm", "nvfp4_quantize", "nvfp4_swizzle_scales",
                     "nvfp4_get_device_error", "nvfp4_debug_wait_timeout"):
            getattr(L, name).restype = i32
        L.nvfp4_version.restype = i32
        L.nvfp4_kernel_launches.restype = ctypes.c_ulonglong
        L.nvfp4_gemm_noalloc.argtypes = [P, P, P, P, f32, P, i32, i32, i32, P]
        L.nvfp4_gemm_noalloc.restype = i32
        L.nvfp4_fp4_peak_probe.argtypes = [i32, ctypes.c_longlong, ctypes.POINTER(i32), P]
        L.nvfp4_fp4_peak_probe.restype = i32
        L.nvfp4_quantize_scaled.argtypes = [P, i32, i32, i32, f32, P, P, P]
        L.nvfp4_quantize_scaled.restype = i32
        L.nvfp4_gemm_bf16a.argtypes = [P, f32, P, P, f32, P, i32, i32, i32, P]
        L.nvfp4_gemm_bf16a.restype = i32
        L.nvfp4_gemm_sparse24.argtypes = [P, P, P, P, P, f32, P, i32, i32, i32, ctypes.c_uint, P]
        L.nvfp4_gemm_sparse24.restype = i32
        L.nvfp4_gemm_mxfp4.argtypes = [P, P, P, P, f32, P, i32, i32, i32, ctypes.c_uint, P]
        L.nvfp4_gemm_mxfp4.restype = i32
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise Nvfp4Error(status, where)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def packed_k(a: torch.Tensor) -> int:
    """K of a packed E2M1 tensor [rows, K/2]."""
    return a.shape[-1] * 2


B_CONSTANT = 1


def gemm(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor, sB: torch.Tensor, alpha: float,
         out: torch.Tensor | None = None, stream=None, b_constant: bool = False) -> torch.Tensor:
    """D[M,N] (bf16) = alpha * (A * sA) @ (B * sB)^T.

    A uint8 [M, K/2], sA uint8 [M, K/16], B uint8 [N, K/2], sB uint8 [N, K/16].
    K is given by the packed operands: both must hold K/2 bytes per row
    (a mismatch is reported here rather than as a kernel error).
    b_constant: B and sB are not written by earlier work still running on the
    stream (weights); lets the kernel start loading them early.
    """
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A and B must be 2-D packed E2M1 tensors [rows, K/2]")
    M, N, K = A.shape[0], B.shape[0], packed_k(A)
    if packed_k(B) != K:
        raise ValueError(f"K mismatch: A holds K={K} (shape {tuple(A.shape)}), B holds K={packed_k(B)} "
                         f"(shape {tuple(B.shape)}); both operands are [rows, K/2] bytes")
    _need(A, "A", torch.uint8, (M, K // 2))
    _need(B, "B", torch.uint8, (N, K // 2))
    _need(sA, "sA", torch.uint8, (M, K // 16))
    _need(sB, "sB", torch.uint8, (N, K // 16))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _need(out, "out", torch.bfloat16, (M, N))
    if b_constant:
        _check(lib().nvfp4_gemm_ex(A.data_ptr(), sA.data_ptr(), B.data_ptr(), sB.data_ptr(), float(alpha),
                                   out.data_ptr(), M, N, K, B_CONSTANT, _stream(stream)), "nvfp4_gemm_ex")
    else:
        _check(lib().nvfp4_gemm(A.data_ptr(), sA.data_ptr(), B.data_ptr(), sB.data_ptr(), float(alpha),
                                out.data_ptr(), M, N, K, _stream(stream)), "nvfp4_gemm")
    return out


NOALLOC_SCRATCH_BYTES = 8 << 20   # static device scratch of nvfp4_gemm_noalloc


def gemm_noalloc(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor, sB: torch.Tensor, alpha: float,
                 out: torch.Tensor, stream=None) -> torch.Tensor:
    """Same as gemm(), through nvfp4_gemm_noalloc: the library allocates no
    device memory (its scale scratch is a fixed static device array), so the
    output tensor must be supplied.  Calls whose GPU work overlaps race on
    that shared scratch; keep them serialised."""
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A and B must be 2-D packed E2M1 tensors [rows, K/2]")
    M, N, K = A.shape[0], B.shape[0], packed_k(A)
    if packed_k(B) != K:
        raise ValueError(f"K mismatch: A holds K={K}, B holds K={packed_k(B)}")
    _need(A, "A", torch.uint8, (M, K // 2))
    _need(B, "B", torch.uint8, (N, K // 2))
    _need(sA, "sA", torch.uint8, (M, K // 16))
    _need(sB, "sB", torch.uint8, (N, K // 16))
    _need(out, "out", torch.bfloat16, (M, N))
    _check(lib().nvfp4_gemm_noalloc(A.data_ptr(), sA.data_ptr(), B.data_ptr(), sB.data_ptr(), float(alpha),
                                    out.data_ptr(), M, N, K, _stream(stream)), "nvfp4_gemm_noalloc")
    return out


def gemm_sparse24(A: torch.Tensor, sA: torch.Tensor, Bv: torch.Tensor, Bm: torch.Tensor, sB: torch.Tensor,
                  alpha: float, out: torch.Tensor | None = None, stream=None,
                  b_constant: bool = False) -> torch.Tensor:
    """D[M,N] (bf16) = alpha * (A * sA) @ (B * sB)^T with 2:4-sparse weights.

    A uint8 [M, K/2], sA uint8 [M, K/16]; B as kept bytes Bv uint8 [N, K/4],
    position nibbles Bm uint8 [N, K/16] and scales sB uint8 [N, K/16] (layout
    in nvfp4_gemm.h, nvfp4_gemm_sparse24)."""
    if A.dim() != 2 or Bv.dim() != 2:
        raise ValueError("A must be [M, K/2] packed codes and Bv [N, K/4] kept bytes")
    M, N, K = A.shape[0], Bv.shape[0], packed_k(A)
    if Bv.shape[1] * 4 != K:
        raise ValueError(f"K mismatch: A holds K={K} (shape {tuple(A.shape)}), Bv holds K={Bv.shape[1] * 4} "
                         f"(shape {tuple(Bv.shape)}); Bv is [N, K/4]")
    _need(A, "A", torch.uint8, (M, K // 2))
    _need(sA, "sA", torch.uint8, (M, K // 16))
    _need(Bv, "Bv", torch.uint8, (N, K // 4))
    _need(Bm, "Bm", torch.uint8, (N, K // 16))
    _need(sB, "sB", torch.uint8, (N, K // 16))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _need(out, "out", torch.bfloat16, (M, N))
    _check(lib().nvfp4_gemm_sparse24(A.data_ptr(), sA.data_ptr(), Bv.data_ptr(), Bm.data_ptr(), sB.data_ptr(),
                                     float(alpha), out.data_ptr(), M, N, K, B_CONSTANT if b_constant else 0,
                                     _stream(stream)), "nvfp4_gemm_sparse24")
    return out


def gemm_mxfp4(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor, sB: torch.Tensor, alpha: float,
               out: torch.Tensor | None = None, stream=None, b_constant: bool = False) -> torch.Tensor:
    """D[M,N] (bf16) = alpha * (A * sA) @ (B * sB)^T in MXFP4: uint8 codes
    A [M, K/2], B [N, K/2] as for gemm(), E8M0 scales sA [M, K/32],
    sB [N, K/32] (one per 32 values, 2^(byte - 127))."""
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A and B must be 2-D packed E2M1 tensors [rows, K/2]")
    M, N, K = A.shape[0], B.shape[0], packed_k(A)
    if packed_k(B) != K:
        raise ValueError(f"K mismatch: A holds K={K}, B holds K={packed_k(B)}")
    _need(A, "A", torch.uint8, (M, K // 2))
    _need(B, "B", torch.uint8, (N, K // 2))
    _need(sA, "sA", torch.uint8, (M, K // 32))
    _need(sB, "sB", torch.uint8, (N, K // 32))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _need(out, "out", torch.bfloat16, (M, N))
    _check(lib().nvfp4_gemm_mxfp4(A.data_ptr(), sA.data_ptr(), B.data_ptr(), sB.data_ptr(), float(alpha),
                                  out.data_ptr(), M, N, K, B_CONSTANT if b_constant else 0, _stream(stream)),
           "nvfp4_gemm_mxfp4")
    return out


def grouped_gemm(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor, sB: torch.Tensor, alpha: torch.Tensor,
                 row_offsets: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Grouped GEMM: rows [off[g], off[g+1]) of A times B[g]^T, scaled by alpha[g].

    A uint8 [M_total, K/2], sA [M_total, K/16], B uint8 [G, N, K/2],
    sB [G, N, K/16], alpha fp32 [G], row_offsets int32 [G+1] (all CUDA).
    """
    if A.dim() != 2 or B.dim() != 3:
        raise ValueError("A must be [M_total, K/2] and B [G, N, K/2]")
    Mt, (G, N, _), K = A.shape[0], B.shape, packed_k(A)
    if B.shape[2] * 2 != K:
        raise ValueError(f"K mismatch: A holds K={K}, B holds K={B.shape[2] * 2}")
    _need(A, "A", torch.uint8, (Mt, K // 2))
    _need(sA, "sA", torch.uint8, (Mt, K // 16))
    _need(B, "B", torch.uint8, (G, N, K // 2))
    _need(sB, "sB", torch.uint8, (G, N, K // 16))
    _need(alpha, "alpha", torch.float32, (G,))
    _need(row_offsets, "row_offsets", torch.int32, (G + 1,))
    if out is None:
        out = torch.empty((Mt, N), dtype=torch.bfloat16, device=A.device)
    _need(out, "out", torch.bfloat16, (Mt, N))
    _check(lib().nvfp4_grouped_gemm(A.data_ptr(), sA.data_ptr(), B.data_ptr(), sB.data_ptr(), alpha.data_ptr(),
                                    row_offsets.data_ptr(), G, out.data_ptr(), Mt, N, K, _stream(stream)),
           "nvfp4_grouped_gemm")
    return out


def gemm_bf16a(A: torch.Tensor, gA: float, B: torch.Tensor, sB: torch.Tensor, alpha: float,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """D = the NVFP4 GEMM of BF16 activations A [M, K] (quantized inside the
    call with global scale gA) and weights B [N, K/2], sB [N, K/16]."""
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A must be [M, K] BF16 and B [N, K/2]")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] * 2 != K:
        raise ValueError(f"K mismatch: A holds K={K}, B holds K={B.shape[1] * 2}")
    _need(A, "A", torch.bfloat16, (M, K))
    _need(B, "B", torch.uint8, (N, K // 2))
    _need(sB, "sB", torch.uint8, (N, K // 16))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _need(out, "out", torch.bfloat16, (M, N))
    _check(lib().nvfp4_gemm_bf16a(A.data_ptr(), float(gA), B.data_ptr(), sB.data_ptr(), float(alpha), out.data_ptr(),
                                  M, N, K, _stream(stream)), "nvfp4_gemm_bf16a")
    return out


def quantize_scaled(X: torch.Tensor, g: float, stream=None):
    """fp32 or BF16 [rows, K] (CUDA) with a given global scale g ->
    (codes uint8 [rows, K/2], scales uint8 [rows, K/16]) in one launch."""
    if X.dim() != 2:
        raise ValueError("X must be 2-D [rows, K]")
    if X.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"X must be float32 or bfloat16, got {X.dtype}")
    rows, K = X.shape
    _need(X, "X", X.dtype, (rows, K))
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=X.device)
    scales = torch.empty((rows, K // 16), dtype=torch.uint8, device=X.device)
    _check(lib().nvfp4_quantize_scaled(X.data_ptr(), 1 if X.dtype == torch.bfloat16 else 0, rows, K, float(g),
                                       codes.data_ptr(), scales.data_ptr(), _stream(stream)),
           "nvfp4_quantize_scaled")
    return codes, scales


def fp4_peak_probe(pair: bool, steps: int, stream=None) -> int:
    """Launch the dense-FP4 calibration kernel (nvfp4_fp4_peak_probe) on
    `stream`; returns the number of CTAs.  The launch performs
    steps x CTAs x 2 x 128 x 256 x 64 FLOPs; time it with CUDA events."""
    ctas = ctypes.c_int(0)
    _check(lib().nvfp4_fp4_peak_probe(1 if pair else 0, int(steps), ctypes.byref(ctas), _stream(stream)),
           "nvfp4_fp4_peak_probe")
    return ctas.value


FP4_PEAK_FLOPS_PER_STEP = 2 * 128 * 256 * 64   # per CTA and step, both forms


def quantize(X: torch.Tensor, stream=None):
    """fp32 [rows, K] (CUDA) -> (codes uint8 [rows, K/2], scales uint8 [rows, K/16], g fp32 [1])."""
    if X.dim() != 2:
        raise ValueError("X must be 2-D [rows, K]")
    rows, K = X.shape
    _need(X, "X", torch.float32, (rows, K))
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=X.device)
    scales = torch.empty((rows, K // 16), dtype=torch.uint8, device=X.device)
    g = torch.empty((1,), dtype=torch.float32, device=X.device)
    _check(lib().nvfp4_quantize(X.data_ptr(), rows, K, codes.data_ptr(), scales.data_ptr(), g.data_ptr(),
                                _stream(stream)), "nvfp4_quantize")
    return codes, scales, g


def swizzled_scale_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_swizzled_scale_bytes(rows, K))


def swizzle_scales(s: torch.Tensor, K: int, stream=None) -> torch.Tensor:
    """Row-major E4M3 scales [rows, K/16] -> tensor-core atom layout (flat uint8)."""
    rows = s.shape[0]
    _need(s, "s", torch.uint8, (rows, K // 16))
    out = torch.empty((swizzled_scale_bytes(rows, K),), dtype=torch.uint8, device=s.device)
    _check(lib().nvfp4_swizzle_scales(s.data_ptr(), rows, K, out.data_ptr(), _stream(stream)),
           "nvfp4_swizzle_scales")
    return out


def get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(lib().nvfp4_get_device_error(_stream(stream)))


def debug_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(lib().nvfp4_debug_wait_timeout(int(timeout_ns), _stream(stream)), "nvfp4_debug_wait_timeout")


def kernel_launches() -> int:
    """Kernels the library has enqueued (or captured) in this process."""
    return int(lib().nvfp4_kernel_launches())


def version() -> int:
    return int(lib().nvfp4_version())
