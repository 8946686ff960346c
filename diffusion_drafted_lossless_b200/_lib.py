"""ctypes binding of libuno.so (include/uno.h). Argument marshalling only.

Each function has the C entry point's name and takes torch tensors (device memory) where
the C ABI takes device pointers; it checks shapes/dtypes enough to build the call, passes
`torch.cuda.current_stream()` unless a stream is given, and raises UnoError on any status
other than UNO_OK. All computation happens in the library's CUDA kernels: there is no
fallback path, and a missing or unloadable libuno.so is an error.
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libuno.so"

UNO_OK, UNO_ERR_INVALID_ARG, UNO_ERR_UNSUPPORTED, UNO_ERR_CUDA, UNO_ERR_TIMEOUT, UNO_ERR_WORKSPACE = range(6)
UNO_BF16, UNO_F32 = 0, 1

EXPORTED = (
    "uno_status_string", "uno_last_error_string", "uno_version", "uno_read_device_status",
    "uno_gated_lora_linear_workspace_size", "uno_gated_lora_linear",
    "uno_block_verify_workspace_size", "uno_block_verify_min_workspace_size", "uno_block_verify",
    "uno_block_verify_noalloc",
    "uno_tv_loss_workspace_size", "uno_tv_loss", "uno_block_noise",
)


class UnoError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_status_name(status)}: {detail}")


_lib = None
_vp, _sz, _i64, _i32, _f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int32, ctypes.c_float


def load(path: str | os.PathLike | None = None) -> ctypes.CDLL:
    """Load libuno.so (build it first with `python -m diffusion_drafted_lossless_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    p = Path(path) if path else LIB_PATH
    if not p.exists():
        raise RuntimeError(f"{p} is missing: build it with `python -m diffusion_drafted_lossless_b200.build` "
                           "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(str(p))
    lib.uno_status_string.restype = ctypes.c_char_p
    lib.uno_status_string.argtypes = [ctypes.c_int]
    lib.uno_last_error_string.restype = ctypes.c_char_p
    lib.uno_version.restype = ctypes.c_int
    lib.uno_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.uno_gated_lora_linear_workspace_size.restype = _sz
    lib.uno_gated_lora_linear_workspace_size.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int]
    lib.uno_gated_lora_linear.argtypes = [_vp, _vp, _vp, _vp, _vp, _f32, _i64, _i64, _i64, _i64, ctypes.c_int,
                                          _vp, _vp, _sz, _vp]
    lib.uno_block_verify_workspace_size.restype = _sz
    lib.uno_block_verify_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _f32, ctypes.c_int]
    lib.uno_block_verify_min_workspace_size.restype = _sz
    lib.uno_block_verify_min_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _f32, ctypes.c_int]
    lib.uno_block_verify.argtypes = [_vp, _vp, ctypes.c_int, _i32, _i32, _i32, _f32, _i32, _f32,
                                     _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.uno_block_verify_noalloc.argtypes = [_vp, _vp, ctypes.c_int, _i32, _i32, _i32, _f32, _i32, _f32,
                                             _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.uno_block_verify_noalloc.restype = ctypes.c_int
    lib.uno_tv_loss_workspace_size.restype = _sz
    lib.uno_tv_loss_workspace_size.argtypes = [_i64, _i64, ctypes.c_int]
    lib.uno_tv_loss.argtypes = [_vp, _vp, ctypes.c_int, _i64, _i64, _vp, _f32, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.uno_block_noise.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]
    lib.uno_block_noise.restype = ctypes.c_int
    for fn in ("uno_gated_lora_linear", "uno_block_verify", "uno_tv_loss"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.uno_read_device_status.restype = ctypes.c_int
    _lib = lib
    return lib


def _status_name(s: int) -> str:
    return load().uno_status_string(int(s)).decode()


def _check(status: int) -> None:
    if status != UNO_OK:
        raise UnoError(status, load().uno_last_error_string().decode())


def _ptr(t):
    """Device address of a tensor argument (None passes NULL). The C ABI takes row-major
    contiguous device memory, so anything else is refused here rather than misread there."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous CUDA tensors "
                         f"(got {type(t).__name__}{'' if not isinstance(t, torch.Tensor) else f' on {t.device}, contiguous={t.is_contiguous()}'})")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return UNO_BF16
    if t.dtype == torch.float32:
        return UNO_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def uno_version() -> int:
    return int(load().uno_version())


def uno_read_device_status() -> int:
    code = ctypes.c_uint32(0)
    _check(load().uno_read_device_status(ctypes.byref(code)))
    return int(code.value)


# ---------------------------------------------------------------------------------------
def uno_gated_lora_linear_workspace_size(M, d_in, d_out, rank, dtype=UNO_BF16) -> int:
    return int(load().uno_gated_lora_linear_workspace_size(M, d_in, d_out, rank, dtype))


def uno_gated_lora_linear(x, w0, lora_a, lora_b, row_gate, scale, y, workspace=None, stream=None):
    """y = x w0^T + scale * diag(row_gate) (x lora_a^T) lora_b^T  (see include/uno.h)."""
    M, d_in = x.shape
    d_out, rank = w0.shape[0], lora_a.shape[0]
    code = _dtype_code(x)
    ws, nb = _workspace(uno_gated_lora_linear_workspace_size(M, d_in, d_out, rank, code), x.device, workspace)
    _check(load().uno_gated_lora_linear(_ptr(x), _ptr(w0), _ptr(lora_a), _ptr(lora_b), _ptr(row_gate),
                                        float(scale), M, d_in, d_out, rank, code, _ptr(y), _ptr(ws), nb,
                                        _stream(stream)))
    return y


# ---------------------------------------------------------------------------------------
def uno_block_verify_workspace_size(B, K, V, top_k, top_p, dtype=UNO_BF16) -> int:
    return int(load().uno_block_verify_workspace_size(B, K, V, top_k, top_p, dtype))


def uno_block_verify_min_workspace_size(B, K, V, top_k, top_p, dtype=UNO_BF16) -> int:
    return int(load().uno_block_verify_min_workspace_size(B, K, V, top_k, top_p, dtype))


def uno_block_verify(verifier_logits, drafter_logits, temperature, top_k, top_p, uniforms,
                     out_tokens, out_count, out_next_token=None, out_p_tok=None, out_q_tok=None, out_tv=None,
                     draft_tokens=None, pos0_tokens=None, workspace=None, stream=None):
    """Lossless block verify over [B, K, V] logits (see include/uno.h)."""
    B, K, V = verifier_logits.shape
    code = _dtype_code(verifier_logits)
    ws, nb = _workspace(uno_block_verify_workspace_size(B, K, V, top_k, top_p, code),
                        verifier_logits.device, workspace)
    _check(load().uno_block_verify(
        _ptr(verifier_logits), _ptr(drafter_logits), code, B, K, V, float(temperature), int(top_k), float(top_p),
        _ptr(draft_tokens), _ptr(pos0_tokens), _ptr(uniforms), _ptr(out_tokens), _ptr(out_count),
        _ptr(out_next_token), _ptr(out_p_tok), _ptr(out_q_tok), _ptr(out_tv), _ptr(ws), nb, _stream(stream)))


def uno_block_verify_noalloc(verifier_logits, drafter_logits, temperature, top_k, top_p, uniforms,
                             out_tokens, out_count, out_next_token=None, out_p_tok=None, out_q_tok=None,
                             out_tv=None, draft_tokens=None, pos0_tokens=None, stream=None):
    """uno_block_verify with the library's fixed scratch array instead of a workspace, for
    callers that cannot allocate device memory (see include/uno.h)."""
    B, K, V = verifier_logits.shape
    code = _dtype_code(verifier_logits)
    _check(load().uno_block_verify_noalloc(
        _ptr(verifier_logits), _ptr(drafter_logits), code, B, K, V, float(temperature), int(top_k), float(top_p),
        _ptr(draft_tokens), _ptr(pos0_tokens), _ptr(uniforms), _ptr(out_tokens), _ptr(out_count),
        _ptr(out_next_token), _ptr(out_p_tok), _ptr(out_q_tok), _ptr(out_tv), _stream(stream)))


# ---------------------------------------------------------------------------------------
def uno_tv_loss_workspace_size(N, V, dtype=UNO_BF16) -> int:
    return int(load().uno_tv_loss_workspace_size(N, V, dtype))


def uno_tv_loss(teacher_logits, student_logits, out_tv, out_mean, grad_student=None, response_mask=None,
                grad_scale=1.0, workspace=None, stream=None):
    """TV self-distillation loss and gradient over [N, V] logits (see include/uno.h)."""
    N, V = teacher_logits.shape
    code = _dtype_code(teacher_logits)
    ws, nb = _workspace(uno_tv_loss_workspace_size(N, V, code), teacher_logits.device, workspace)
    _check(load().uno_tv_loss(_ptr(teacher_logits), _ptr(student_logits), code, N, V, _ptr(response_mask),
                              float(grad_scale), _ptr(out_tv), _ptr(out_mean), _ptr(grad_student), _ptr(ws), nb,
                              _stream(stream)))


# ---------------------------------------------------------------------------------------
def uno_block_noise(clean_tokens, uniforms, V, noised_tokens, row_gate=None, stream=None):
    """Block-noised copy, noise mode random_uniform: position 0 kept, draft positions
    min(V - 1, floor(u V)); optional row gate (see include/uno.h)."""
    B, K = clean_tokens.shape
    _check(load().uno_block_noise(_ptr(clean_tokens), _ptr(uniforms), B, K, int(V), _ptr(noised_tokens),
                                  _ptr(row_gate), _stream(stream)))
    return noised_tokens
