"""B200 (sm_100a) W4A4 NVFP4 linear layer: Python binding of ``libw4a4.so``.

Every function here marshals arguments (tensor pointers, sizes, the current
CUDA stream) into the C ABI declared in ``include/w4a4.h`` and raises on a
non-zero status.  All arithmetic runs in the CUDA kernels of the shared
library; there is no CPU or PyTorch fallback: if the library is missing the
import of any wrapper raises.

PyTorch is used only for device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

import math

import torch

__all__ = [
    "lib", "W4A4Error", "nvfp4_sf_bytes", "nvfp4_quant_workspace_bytes", "w4a4_workspace_bytes",
    "nvfp4_quantize_act", "nvfp4_pack_weight", "w4a4_gemm", "w4a4_linear", "w4a4_device_status",
    "w4a4_status_string", "EPI_NONE", "EPI_GELU_TANH", "SRC_BF16", "SRC_F32",
    "QuantizedActivation", "PackedWeight", "quantize_act", "pack_weight", "linear", "gemm",
    "new_workspace", "nvfp4_sf_to_rowmajor", "sf_rowmajor", "w4a4_set_wait_bound",
    "nvfp4_quantize_act_noalloc", "nvfp4_quantize_act_with_amax", "w4a4_gemm_next_amax", "w4a4_gemm_swiglu",
    "gemm_swiglu", "w4a4_gemm_quantize_next", "gemm_quantize_next", "w4a4_gemm_rope", "gemm_rope",
    "fp8_quant_workspace_bytes", "fp8_quantize", "attention_fp8", "Fp8Tensor", "quantize_fp8", "attention",
    "w4a4_fp4_mma_rate", "w4a4_last_error", "MAX_K",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libw4a4.so")

EPI_NONE, EPI_GELU_TANH = 0, 1
SRC_BF16, SRC_F32 = 0, 1
MAX_K = 1 << 20  # W4A4_MAX_K: the widest K (activation or weight columns) the entry points accept

_c = ctypes
_P = _c.c_void_p
_I64 = _c.c_int64
_SIG = {
    "nvfp4_sf_bytes": (_c.c_size_t, [_I64, _I64]),
    "nvfp4_quant_workspace_bytes": (_c.c_size_t, [_I64, _I64, _c.c_int]),
    "w4a4_workspace_bytes": (_c.c_size_t, [_I64, _I64, _I64, _c.c_int]),
    "nvfp4_quantize_act": (_c.c_int, [_P, _I64, _I64, _I64, _P, _P, _c.c_int, _P, _P, _P, _P, _P, _P,
                                      _c.c_size_t, _P]),
    "nvfp4_quantize_act_with_amax": (_c.c_int, [_P, _I64, _I64, _I64, _P, _P, _c.c_int, _P, _P, _P, _P, _P,
                                                _P, _P, _c.c_size_t, _P]),
    "nvfp4_pack_weight": (_c.c_int, [_P, _c.c_int, _I64, _I64, _I64, _P, _P, _P, _P, _c.c_size_t, _P]),
    "w4a4_gemm": (_c.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _c.c_int, _P, _c.c_int,
                             _P, _I64, _P]),
    "w4a4_gemm_next_amax": (_c.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _c.c_int, _P,
                                       _c.c_int, _P, _I64, _P, _P, _P]),
    "w4a4_gemm_swiglu": (_c.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _c.c_int, _P, _I64, _P, _I64,
                                    _P, _I64, _P, _P, _P]),
    "w4a4_gemm_rope": (_c.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _c.c_int, _P, _I64, _I64, _P,
                                  _I64, _I64, _P, _I64, _P, _I64, _P, _P, _P]),
    "fp8_quant_workspace_bytes": (_c.c_size_t, [_I64, _I64]),
    "w4a4_fp4_mma_rate": (_c.c_int, [_c.c_int, _c.c_int, _P, _P]),
    "fp8_quantize": (_c.c_int, [_P, _I64, _I64, _I64, _c.c_int, _P, _I64, _P, _P, _c.c_size_t, _P]),
    "attention_fp8": (_c.c_int, [_P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I64, _P, _P, _P, _c.c_float, _P, _I64,
                                 _P]),
    "w4a4_gemm_quantize_next": (_c.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _c.c_int, _P,
                                           _c.c_int, _I64, _P, _I64, _P, _I64, _P, _P, _P, _I64, _P, _I64, _I64,
                                           _P, _P]),
    "w4a4_linear": (_c.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _c.c_int, _P, _c.c_int, _P,
                               _P, _c.c_size_t, _P]),
    "nvfp4_quantize_act_noalloc": (_c.c_int, [_P, _I64, _I64, _I64, _P, _P, _c.c_int, _P, _P, _P, _P, _P, _P]),
    "w4a4_device_status": (_c.c_int, [_c.POINTER(_c.c_int), _c.c_int]),
    "w4a4_last_error": (_c.c_int, []),
    "w4a4_set_wait_bound": (_c.c_int, [_I64]),
    "nvfp4_sf_to_rowmajor": (_c.c_int, [_P, _I64, _I64, _P, _P]),
    "w4a4_status_string": (_c.c_char_p, [_c.c_int]),
}

_lib = None


class W4A4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed with status {status}: {w4a4_status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded shared library (built by ``build.py``); raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_diffusion_transformer_nvfp4_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIG.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(fn: str, st: int):
    if st != 0:
        raise W4A4Error(fn, st)


# ------------------------------------------------------------------ raw ABI

def nvfp4_sf_bytes(rows: int, K: int) -> int:
    return lib().nvfp4_sf_bytes(rows, K)


def nvfp4_quant_workspace_bytes(M: int, K: int, r: int) -> int:
    return lib().nvfp4_quant_workspace_bytes(M, K, r)


def w4a4_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return lib().w4a4_workspace_bytes(M, N, K, r)


def w4a4_status_string(status: int) -> str:
    return lib().w4a4_status_string(status).decode()


def nvfp4_quantize_act(X, M, K, ldx, inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, workspace, stream=None):
    _check("nvfp4_quantize_act", lib().nvfp4_quantize_act(
        _ptr(X), M, K, ldx, _ptr(inv_s), _ptr(L1t), r, _ptr(t_w), _ptr(Xq), _ptr(Xsf), _ptr(t_x),
        _ptr(U), _ptr(workspace), workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream(stream)))


def nvfp4_quantize_act_with_amax(X, M, K, ldx, inv_s, L1t, r, t_w, amax, Xq, Xsf, t_x, U, workspace,
                                 stream=None):
    _check("nvfp4_quantize_act_with_amax", lib().nvfp4_quantize_act_with_amax(
        _ptr(X), M, K, ldx, _ptr(inv_s), _ptr(L1t), r, _ptr(t_w), _ptr(amax), _ptr(Xq), _ptr(Xsf), _ptr(t_x),
        _ptr(U), _ptr(workspace), workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream(stream)))


def nvfp4_pack_weight(R, src_dtype, N, K, ldr, Wq, Wsf, t_w, workspace, stream=None):
    _check("nvfp4_pack_weight", lib().nvfp4_pack_weight(
        _ptr(R), src_dtype, N, K, ldr, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0, _stream(stream)))


def w4a4_gemm(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy, stream=None):
    _check("w4a4_gemm", lib().w4a4_gemm(
        _ptr(Xq), _ptr(Xsf), _ptr(t_x), _ptr(U), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(L2t), r,
        _ptr(bias), epilogue, _ptr(Y), ldy, _stream(stream)))


def w4a4_gemm_next_amax(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy, next_inv_s,
                        next_amax, stream=None):
    _check("w4a4_gemm_next_amax", lib().w4a4_gemm_next_amax(
        _ptr(Xq), _ptr(Xsf), _ptr(t_x), _ptr(U), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(L2t), r,
        _ptr(bias), epilogue, _ptr(Y), ldy, _ptr(next_inv_s), _ptr(next_amax), _stream(stream)))


def w4a4_gemm_swiglu(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, n_plain, Y, ldy, H, ldh, next_inv_s,
                     next_amax, stream=None):
    _check("w4a4_gemm_swiglu", lib().w4a4_gemm_swiglu(
        _ptr(Xq), _ptr(Xsf), _ptr(t_x), _ptr(U), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(L2t), r,
        _ptr(bias), n_plain, _ptr(Y), ldy, _ptr(H), ldh, _ptr(next_inv_s), _ptr(next_amax), _stream(stream)))


def w4a4_gemm_rope(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, n_rope, d_head, rope, ld_rope, n_plain, Y,
                   ldy, H, ldh, next_inv_s, next_amax, stream=None):
    _check("w4a4_gemm_rope", lib().w4a4_gemm_rope(
        _ptr(Xq), _ptr(Xsf), _ptr(t_x), _ptr(U), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(L2t), r,
        _ptr(bias), n_rope, d_head, _ptr(rope), ld_rope, n_plain, _ptr(Y), ldy, _ptr(H), ldh, _ptr(next_inv_s),
        _ptr(next_amax), _stream(stream)))


def w4a4_last_error() -> int:
    """The sticky device status (no device synchronisation: synchronise the
    streams of interest first)."""
    return lib().w4a4_last_error()


def w4a4_fp4_mma_rate(iters, pair, cycles, stream=None):
    _check("w4a4_fp4_mma_rate", lib().w4a4_fp4_mma_rate(int(iters), int(pair), _ptr(cycles), _stream(stream)))


def fp8_quant_workspace_bytes(rows, cols) -> int:
    return lib().fp8_quant_workspace_bytes(rows, cols)


def fp8_quantize(X, rows, cols, ldx, transpose, out, ldo, scale, workspace, stream=None):
    _check("fp8_quantize", lib().fp8_quantize(
        _ptr(X), rows, cols, ldx, int(transpose), _ptr(out), ldo, _ptr(scale), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))


def attention_fp8(Q8, K8, Vt8, batch, S, heads, ldq, ldk, ldvt, s_q, s_k, s_v, softmax_scale, O, ldo, stream=None):
    _check("attention_fp8", lib().attention_fp8(
        _ptr(Q8), _ptr(K8), _ptr(Vt8), batch, S, heads, ldq, ldk, ldvt, _ptr(s_q), _ptr(s_k), _ptr(s_v),
        float(softmax_scale), _ptr(O), ldo, _stream(stream)))


def w4a4_gemm_quantize_next(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, n_plain, Y, ldy, H,
                            ldh, next_inv_s, next_t, next_q, next_ldq, next_sf, next_K, next_col, next_amax,
                            stream=None):
    _check("w4a4_gemm_quantize_next", lib().w4a4_gemm_quantize_next(
        _ptr(Xq), _ptr(Xsf), _ptr(t_x), _ptr(U), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(L2t), r,
        _ptr(bias), epilogue, n_plain, _ptr(Y), ldy, _ptr(H), ldh, _ptr(next_inv_s), _ptr(next_t), _ptr(next_q),
        next_ldq, _ptr(next_sf), next_K, next_col, _ptr(next_amax), _stream(stream)))


def w4a4_linear(X, M, N, K, Wq, Wsf, t_w, inv_s, L1t, L2t, r, bias, epilogue, Y, workspace, stream=None):
    _check("w4a4_linear", lib().w4a4_linear(
        _ptr(X), M, N, K, _ptr(Wq), _ptr(Wsf), _ptr(t_w), _ptr(inv_s), _ptr(L1t), _ptr(L2t), r, _ptr(bias),
        epilogue, _ptr(Y), _ptr(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0, _stream(stream)))


def nvfp4_sf_to_rowmajor(sf_atoms, rows, K, sf_rowmajor, stream=None):
    _check("nvfp4_sf_to_rowmajor", lib().nvfp4_sf_to_rowmajor(
        _ptr(sf_atoms), rows, K, _ptr(sf_rowmajor), _stream(stream)))


def sf_rowmajor(sf_atoms: torch.Tensor, rows: int, K: int, stream=None) -> torch.Tensor:
    """The scale bytes of an SF-atom buffer as a row-major [rows, K/16] uint8 tensor."""
    out = torch.empty(rows, K // 16, dtype=torch.uint8, device=sf_atoms.device)
    nvfp4_sf_to_rowmajor(sf_atoms, rows, K, out, stream)
    return out


def w4a4_set_wait_bound(cycles: int = 0) -> None:
    """Device-side waits give up after ``cycles`` SM clock cycles (0: the default)."""
    _check("w4a4_set_wait_bound", lib().w4a4_set_wait_bound(cycles))


def nvfp4_quantize_act_noalloc(X, M, K, ldx, inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, stream=None):
    _check("nvfp4_quantize_act_noalloc", lib().nvfp4_quantize_act_noalloc(
        _ptr(X), M, K, ldx, _ptr(inv_s), _ptr(L1t), r, _ptr(t_w), _ptr(Xq), _ptr(Xsf), _ptr(t_x), _ptr(U),
        _stream(stream)))


def w4a4_device_status(reset: bool = False) -> int:
    v = ctypes.c_int(0)
    _check("w4a4_device_status", lib().w4a4_device_status(ctypes.byref(v), 1 if reset else 0))
    return v.value


# ------------------------------------------------------------------ tensor-level helpers
# These allocate outputs with torch (device memory is the caller's business in
# the C ABI) and call the raw wrappers above.

def _u8(n, device):
    return torch.empty(n, dtype=torch.uint8, device=device)


def new_workspace(nbytes, device):
    """A workspace for the entry points that take one, zeroed once: the
    library's synchronisation words start from zeros and every call leaves
    them valid for the next (zero it again only after a device error)."""
    return torch.zeros(max(16, nbytes), dtype=torch.uint8, device=device)


class QuantizedActivation:
    """Outputs of nvfp4_quantize_act: codes, SF atoms, tensor scale, low-rank U."""

    def __init__(self, Xq, Xsf, t_x, U, M, K, r):
        self.Xq, self.Xsf, self.t_x, self.U = Xq, Xsf, t_x, U
        self.M, self.K, self.r = M, K, r


class PackedWeight:
    """A prepared W4A4 linear: NVFP4 residual weight plus its side inputs."""

    def __init__(self, Wq, Wsf, t_w, N, K, inv_s=None, L1t=None, L2t=None, bias=None):
        self.Wq, self.Wsf, self.t_w = Wq, Wsf, t_w
        self.N, self.K = N, K
        self.inv_s, self.L1t, self.L2t, self.bias = inv_s, L1t, L2t, bias
        self.r = 0 if L1t is None else int(L1t.shape[0])

    def rows(self, r0: int, r1: int) -> "PackedWeight":
        """Views of output channels [r0, r1) (r0 a multiple of 128): the same
        activation quantisation (smoothing, L1t, t_w) serves both parts of a
        fused projection."""
        if r0 % 128 or not (0 <= r0 < r1 <= self.N):
            raise ValueError("row slice must start on a 128-row boundary")
        atom_row = (self.K // 64) * 512
        sf0 = (r0 // 128) * atom_row
        sf1 = -(-r1 // 128) * atom_row
        return PackedWeight(self.Wq[r0:r1], self.Wsf[sf0:sf1], self.t_w, r1 - r0, self.K, self.inv_s,
                            self.L1t, None if self.L2t is None else self.L2t[r0:r1],
                            None if self.bias is None else self.bias[r0:r1])


def quantize_act(X: torch.Tensor, inv_s=None, L1t=None, t_w=None, stream=None, amax=None,
                 workspace=None) -> QuantizedActivation:
    """NVFP4 activation quantisation; ``amax`` (fp32 device scalar, e.g. from
    ``gemm(..., next_amax=...)``) supplies the tensor amax instead of measuring it.
    ``workspace``: a uint8 device tensor from ``new_workspace`` of at least
    ``nvfp4_quant_workspace_bytes(M, K, r)`` bytes, reused across calls (a
    fresh one is made when None)."""
    M, K = X.shape
    r = 0 if L1t is None else int(L1t.shape[0])
    dev = X.device
    Xq = _u8(M * K // 2, dev).view(M, K // 2)
    Xsf = _u8(nvfp4_sf_bytes(M, K), dev)
    t_x = torch.empty(1, dtype=torch.float32, device=dev)
    U = torch.empty(M, 2 * r, dtype=torch.bfloat16, device=dev) if r else None
    ws = new_workspace(nvfp4_quant_workspace_bytes(M, K, r), dev) if workspace is None else workspace
    if amax is None:
        nvfp4_quantize_act(X, M, K, X.stride(0), inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, ws, stream)
    else:
        nvfp4_quantize_act_with_amax(X, M, K, X.stride(0), inv_s, L1t, r, t_w, amax, Xq, Xsf, t_x, U, ws, stream)
    return QuantizedActivation(Xq, Xsf, t_x, U, M, K, r)


def pack_weight(R: torch.Tensor, inv_s=None, L1t=None, L2t=None, bias=None, stream=None) -> PackedWeight:
    N, K = R.shape
    dev = R.device
    src = SRC_F32 if R.dtype == torch.float32 else SRC_BF16
    Wq = _u8(N * K // 2, dev).view(N, K // 2)
    Wsf = _u8(nvfp4_sf_bytes(N, K), dev)
    t_w = torch.empty(1, dtype=torch.float32, device=dev)
    ws = new_workspace(nvfp4_quant_workspace_bytes(N, K, 0), dev)
    nvfp4_pack_weight(R, src, N, K, R.stride(0), Wq, Wsf, t_w, ws, stream)
    return PackedWeight(Wq, Wsf, t_w, N, K, inv_s, L1t, L2t, bias)


def gemm(qa: QuantizedActivation, w: PackedWeight, epilogue: int = EPI_NONE, Y=None, stream=None,
         next_inv_s=None, next_amax=None):
    """Y = the fused W4A4 GEMM.  With ``next_amax`` (fp32 device scalar holding
    a non-negative value, normally 0) it also max-es in the tensor amax
    max |fl(Y * next_inv_s)| that the next layer's quantiser needs."""
    if Y is None:
        Y = torch.empty(qa.M, w.N, dtype=torch.bfloat16, device=qa.Xq.device)
    if next_amax is None:
        w4a4_gemm(qa.Xq, qa.Xsf, qa.t_x, qa.U, qa.M, w.N, w.K, w.Wq, w.Wsf, w.t_w, w.L2t, w.r, w.bias,
                  epilogue, Y, Y.stride(0), stream)
    else:
        w4a4_gemm_next_amax(qa.Xq, qa.Xsf, qa.t_x, qa.U, qa.M, w.N, w.K, w.Wq, w.Wsf, w.t_w, w.L2t, w.r, w.bias,
                            epilogue, Y, Y.stride(0), next_inv_s, next_amax, stream)
    return Y


def gemm_swiglu(qa: QuantizedActivation, w: PackedWeight, n_plain: int, Y=None, H=None, stream=None,
                next_inv_s=None, next_amax=None):
    """The fused projection with the SwiGLU epilogue: the first ``n_plain``
    packed weight rows give Y [M, n_plain]; the rest, gate/up pairs in the
    order of ``prep.swiglu_row_order``, give H = silu(gate) * up [M, (N -
    n_plain) / 2].  Returns (Y, H)."""
    n_h = (w.N - n_plain) // 2
    dev = qa.Xq.device
    if Y is None and n_plain > 0:
        Y = torch.empty(qa.M, n_plain, dtype=torch.bfloat16, device=dev)
    if H is None:
        H = torch.empty(qa.M, n_h, dtype=torch.bfloat16, device=dev)
    w4a4_gemm_swiglu(qa.Xq, qa.Xsf, qa.t_x, qa.U, qa.M, w.N, w.K, w.Wq, w.Wsf, w.t_w, w.L2t, w.r, w.bias, n_plain,
                     Y, Y.stride(0) if Y is not None else 0, H, H.stride(0), next_inv_s, next_amax, stream)
    return Y, H


def gemm_rope(qa: QuantizedActivation, w: PackedWeight, rope, n_rope: int, d_head: int, n_plain=None, Y=None,
              H=None, stream=None, next_inv_s=None, next_amax=None):
    """The fused projection with the rotary embedding on its first ``n_rope``
    outputs (heads of ``d_head`` features; ``rope`` fp32 [M, >= d_head], per
    token the (cos, sin) of each feature pair, interleaved) and, with
    ``n_plain`` < N, the SwiGLU epilogue on the rest as in ``gemm_swiglu``.
    Returns (Y, H); H is None without SwiGLU outputs."""
    dev = qa.Xq.device
    n_plain = w.N if n_plain is None else n_plain
    if Y is None:
        Y = torch.empty(qa.M, n_plain, dtype=torch.bfloat16, device=dev)
    if H is None and n_plain < w.N:
        H = torch.empty(qa.M, (w.N - n_plain) // 2, dtype=torch.bfloat16, device=dev)
    w4a4_gemm_rope(qa.Xq, qa.Xsf, qa.t_x, qa.U, qa.M, w.N, w.K, w.Wq, w.Wsf, w.t_w, w.L2t, w.r, w.bias, n_rope,
                   d_head, rope, rope.stride(0), n_plain, Y, Y.stride(0), H, 0 if H is None else H.stride(0),
                   next_inv_s, next_amax, stream)
    return Y, H


class Fp8Tensor:
    """E4M3 codes of a bf16 tensor and its fp32 scale (row-major, or
    transposed when ``transposed``)."""

    def __init__(self, codes, scale, rows, cols, transposed):
        self.codes, self.scale, self.rows, self.cols, self.transposed = codes, scale, rows, cols, transposed


def quantize_fp8(X, transpose: bool = False, out=None, workspace=None, stream=None) -> Fp8Tensor:
    """Per-tensor E4M3 quantisation of a bf16 [rows, cols] view (row stride
    X.stride(0)); transposed codes [cols, rows] with ``transpose``."""
    rows, cols = X.shape
    dev = X.device
    if out is None:
        out = torch.empty((cols, rows) if transpose else (rows, cols), dtype=torch.uint8, device=dev)
    scale = torch.empty(1, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(fp8_quant_workspace_bytes(rows, cols), 16), dtype=torch.uint8, device=dev)
    fp8_quantize(X, rows, cols, X.stride(0), transpose, out, out.stride(0), scale, workspace, stream)
    return Fp8Tensor(out, scale, rows, cols, transpose)


def attention(q: Fp8Tensor, k: Fp8Tensor, vt: Fp8Tensor, heads: int, batch: int = 1, O=None, softmax_scale=None,
              stream=None):
    """FP8 attention over ``batch`` sequences of q.rows / batch tokens, heads
    of 128 features; q, k row-major codes [tokens, heads*128], vt the values'
    transposed codes [heads*128, tokens].  Returns bf16 O [tokens, heads*128]."""
    S = q.rows // batch
    if O is None:
        O = torch.empty(q.rows, heads * 128, dtype=torch.bfloat16, device=q.codes.device)
    c = 1.0 / math.sqrt(128.0) if softmax_scale is None else softmax_scale
    attention_fp8(q.codes, k.codes, vt.codes, batch, S, heads, q.codes.stride(0), k.codes.stride(0),
                  vt.codes.stride(0), q.scale, k.scale, vt.scale, c, O, O.stride(0), stream)
    return O


def gemm_quantize_next(qa: QuantizedActivation, w: PackedWeight, next_t, next_inv_s=None, epilogue: int = EPI_NONE,
                       n_plain=None, store_outputs: bool = True, next_K=None, next_col: int = 0, next_q=None,
                       next_sf=None, next_amax=None, stream=None):
    """The GEMM whose epilogue also writes the next layer's NVFP4 codes and
    scale bytes of its final outputs (Y, or H with ``n_plain`` < N) under
    the given tensor scale ``next_t``.  Returns (Y, H, next_q, next_sf);
    Y / H are None when not stored."""
    dev = qa.Xq.device
    n_plain = w.N if n_plain is None else n_plain
    n_out = w.N if n_plain == w.N else (w.N - n_plain) // 2
    next_K = n_out if next_K is None else next_K
    Y = H = None
    if n_plain == w.N:
        if store_outputs:
            Y = torch.empty(qa.M, w.N, dtype=torch.bfloat16, device=dev)
    else:
        if n_plain:
            Y = torch.empty(qa.M, n_plain, dtype=torch.bfloat16, device=dev)
        if store_outputs:
            H = torch.empty(qa.M, n_out, dtype=torch.bfloat16, device=dev)
    if next_q is None:
        next_q = torch.zeros(qa.M, next_K // 2, dtype=torch.uint8, device=dev)
    if next_sf is None:
        next_sf = torch.zeros(nvfp4_sf_bytes(qa.M, next_K), dtype=torch.uint8, device=dev)
    w4a4_gemm_quantize_next(qa.Xq, qa.Xsf, qa.t_x, qa.U, qa.M, w.N, w.K, w.Wq, w.Wsf, w.t_w, w.L2t, w.r, w.bias,
                            epilogue, n_plain, Y, 0 if Y is None else Y.stride(0), H, 0 if H is None else H.stride(0),
                            next_inv_s, next_t, next_q, next_q.stride(0), next_sf, next_K, next_col, next_amax,
                            stream)
    return Y, H, next_q, next_sf


def linear(X: torch.Tensor, w: PackedWeight, epilogue: int = EPI_NONE, Y=None, workspace=None, stream=None):
    M, K = X.shape
    if Y is None:
        Y = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = new_workspace(w4a4_workspace_bytes(M, w.N, K, w.r), X.device)
    w4a4_linear(X, M, w.N, K, w.Wq, w.Wsf, w.t_w, w.inv_s, w.L1t, w.L2t, w.r, w.bias, epilogue, Y,
                workspace, stream)
    return Y
