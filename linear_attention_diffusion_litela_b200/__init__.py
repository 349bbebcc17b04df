"""LiteLA forward (Sana's ReLU linear self-attention) on B200: Python binding of liblitela.

This module only marshals arguments to the C ABI of liblitela.so (include/litela.h); every
step of the computation runs in the library's CUDA kernels.  torch supplies device memory
and the current stream.  There is no fallback: if the library is missing or the tensors are
not on a CUDA device, the calls raise.

    from linear_attention_diffusion_litela_b200 import lite_la_fwd
    out = lite_la_fwd(qkv, H=70)          # qkv: bf16 CUDA tensor [B, N, 3*H*32]
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "LiteLAError", "lib", "lib_path", "lite_la_fwd", "lite_la_block_causal_fwd", "lite_la_bwd",
    "lite_la_fwd_oproj", "lite_la_out_proj",
    "lite_la_workspace_bytes", "lite_la_release_workspace", "lite_la_forward_form",
    "lite_la_set_paired_min_chunk", "STATUS", "EXPORTED_SYMBOLS",
]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG_DIR, "liblitela.so")

STATUS = {
    0: "LITELA_OK",
    1: "LITELA_ERR_INVALID_ARGUMENT",
    2: "LITELA_ERR_UNSUPPORTED",
    3: "LITELA_ERR_OUT_OF_MEMORY",
    4: "LITELA_ERR_CUDA",
    5: "LITELA_ERR_DEVICE_TIMEOUT",
}

# name -> (restype, argtypes); mirrors include/litela.h
_c_int, _c_float, _vp, _c_size = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_SIGNATURES = {
    "lite_la_fwd": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _vp]),
    "lite_la_block_causal_fwd": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_fwd_f32out": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _vp]),
    "lite_la_block_causal_fwd_f32out": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_fwd_events": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _vp, _vp]),
    "lite_la_block_causal_fwd_events": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int,
                                                 _vp, _vp]),
    "lite_la_block_causal_fwd_carry": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp, _vp, _vp]),
    "lite_la_block_causal_fwd_carry_f32out": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp, _vp, _vp]),
    "lite_la_device_status": (_c_int, [_vp]),
    "lite_la_selftest_timeout": (_c_int, [_vp]),
    "lite_la_state_fwd": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "lite_la_status_string": (ctypes.c_char_p, [_c_int]),
    "lite_la_last_error": (ctypes.c_char_p, []),
    "lite_la_release_workspace": (_c_int, []),
    "lite_la_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "lite_la_fwd_noalloc": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _vp]),
    "lite_la_kernels_per_call": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "lite_la_bwd_kernels_per_call": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "lite_la_forward_form": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "lite_la_set_paired_min_chunk": (_c_int, [_c_int]),
    "lite_la_elu1_fwd": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_elu1_fwd_f32out": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_elu1_fwd_events": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp, _vp]),
    "lite_la_bwd": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _vp]),
    "lite_la_block_causal_bwd": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_bwd_f32out": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _vp]),
    "lite_la_block_causal_bwd_f32out": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int,
                                                 _vp]),
    "lite_la_bwd_events": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp, _vp]),
    "lite_la_bwd_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "lite_la_fwd_save_state": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_bwd_from_state": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_fwd_oproj": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "lite_la_fwd_oproj_events": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                          _c_int, _vp, _vp]),
    "lite_la_out_proj": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp]),
}
EXPORTED_SYMBOLS = tuple(_SIGNATURES)

_lib = None
_lock = threading.Lock()


class LiteLAError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__("%s: %s" % (STATUS.get(status, status), message))


def lib() -> ctypes.CDLL:
    """The loaded liblitela.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(lib_path):
                raise ImportError("liblitela.so is not built; run "
                                  "`python -m linear_attention_diffusion_litela_b200.build`")
            h = ctypes.CDLL(lib_path)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(h, name)
                fn.restype, fn.argtypes = res, args
            _lib = h
    return _lib


ffma_lib_path = os.path.join(_PKG_DIR, "liblitela_ffma_peak.so")
_ffma_lib = None


def ffma_peak_lib() -> ctypes.CDLL:
    """The benchmark's fp32 FMA-peak microbenchmark (include/litela_ffma_peak.h)."""
    global _ffma_lib
    with _lock:
        if _ffma_lib is None:
            if not os.path.exists(ffma_lib_path):
                raise ImportError("liblitela_ffma_peak.so is not built; run "
                                  "`python -m linear_attention_diffusion_litela_b200.build`")
            h = ctypes.CDLL(ffma_lib_path)
            h.litela_ffma_flops.restype = ctypes.c_longlong
            h.litela_ffma_flops.argtypes = [_c_int, _c_int, ctypes.c_longlong]
            h.litela_ffma_launch.restype = _c_int
            h.litela_ffma_launch.argtypes = [_vp, _c_int, _c_int, ctypes.c_longlong, _vp]
            _ffma_lib = h
    return _ffma_lib


def _check(status: int) -> None:
    if status != 0:
        msg = lib().lite_la_last_error().decode(errors="replace")
        raise LiteLAError(status, msg)


def _torch():
    import torch
    return torch


def _prepare(qkv, H: int, d: int, out, out_dtype):
    torch = _torch()
    if not isinstance(qkv, torch.Tensor) or not qkv.is_cuda:
        raise TypeError("qkv must be a CUDA tensor")
    if qkv.dtype != torch.bfloat16 or qkv.dim() != 3 or not qkv.is_contiguous():
        raise TypeError("qkv must be a contiguous bf16 tensor [B, N, 3*H*d]")
    B, N, W = qkv.shape
    if W != 3 * H * d:
        raise ValueError("qkv last dim %d != 3*H*d = %d" % (W, 3 * H * d))
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=qkv.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or not out.is_contiguous() \
            or tuple(out.shape) != (B, N, H * d) or out.device != qkv.device:
        raise TypeError("out must be a contiguous bf16/fp32 tensor [B, N, H*d] on qkv's device")
    return B, N, out


def _stream_handle(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def lite_la_fwd(qkv, H: int, d: int = 32, eps: float = 1e-15, out=None, out_dtype=None, stream=None):
    """Non-causal LiteLA forward; returns out [B, N, H*d] (bf16 unless out/out_dtype say fp32)."""
    torch = _torch()
    B, N, out = _prepare(qkv, H, d, out, out_dtype or torch.bfloat16)
    fn = lib().lite_la_fwd if out.dtype == torch.bfloat16 else lib().lite_la_fwd_f32out
    with torch.cuda.device(qkv.device):
        _check(fn(qkv.data_ptr(), out.data_ptr(), B, N, H, d, eps, _stream_handle(stream, qkv.device)))
    return out


def lite_la_block_causal_fwd(qkv, H: int, tokens_per_block: int, d: int = 32, eps: float = 1e-15,
                             out=None, out_dtype=None, stream=None):
    """Block-causal LiteLA forward (a query in block b sees blocks 0..b); returns out."""
    torch = _torch()
    B, N, out = _prepare(qkv, H, d, out, out_dtype or torch.bfloat16)
    fn = lib().lite_la_block_causal_fwd if out.dtype == torch.bfloat16 else lib().lite_la_block_causal_fwd_f32out
    with torch.cuda.device(qkv.device):
        _check(fn(qkv.data_ptr(), out.data_ptr(), B, N, H, d, eps, int(tokens_per_block),
                  _stream_handle(stream, qkv.device)))
    return out


def lite_la_block_causal_fwd_carry(qkv, H: int, tokens_per_block: int, state_in=None, state_out=None,
                                   d: int = 32, eps: float = 1e-15, out=None, out_dtype=None, stream=None):
    """Block-causal LiteLA of one chunk with the state of earlier chunks carried in (state_in,
    fp32 [B, H, d+1, d] or None) and the state after this chunk written to state_out (allocated
    when None; may be state_in).  Returns (out, state_out)."""
    torch = _torch()
    B, N, out = _prepare(qkv, H, d, out, out_dtype or torch.bfloat16)
    shape = (B, H, d + 1, d)
    for t in (state_in,):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous()
                              or t.device != qkv.device):
            raise TypeError("state_in must be a contiguous fp32 tensor [B, H, d+1, d] on qkv's device")
    if state_out is None:
        state_out = torch.empty(shape, dtype=torch.float32, device=qkv.device)
    elif state_out.dtype != torch.float32 or tuple(state_out.shape) != shape or not state_out.is_contiguous():
        raise TypeError("state_out must be a contiguous fp32 tensor [B, H, d+1, d]")
    fn = lib().lite_la_block_causal_fwd_carry if out.dtype == torch.bfloat16 else lib().lite_la_block_causal_fwd_carry_f32out
    with torch.cuda.device(qkv.device):
        _check(fn(qkv.data_ptr(), out.data_ptr(), B, N, H, d, eps, int(tokens_per_block),
                  None if state_in is None else state_in.data_ptr(), state_out.data_ptr(),
                  _stream_handle(stream, qkv.device)))
    return out, state_out


def lite_la_state_fwd(qkv, H: int, tokens_per_block: int = 0, d: int = 32, out=None, stream=None):
    """Per-(batch, head, block) inclusive prefix states, fp32 [B, H, nblk, d+1, d]."""
    torch = _torch()
    if not isinstance(qkv, torch.Tensor) or not qkv.is_cuda or qkv.dtype != torch.bfloat16 \
            or qkv.dim() != 3 or not qkv.is_contiguous():
        raise TypeError("qkv must be a contiguous bf16 CUDA tensor [B, N, 3*H*d]")
    B, N, W = qkv.shape
    if W != 3 * H * d:
        raise ValueError("qkv last dim %d != 3*H*d = %d" % (W, 3 * H * d))
    T = tokens_per_block if 0 < tokens_per_block < N else N
    nblk = -(-N // T) if N > 0 else 0
    if out is None:
        out = torch.empty((B, H, nblk, d + 1, d), dtype=torch.float32, device=qkv.device)
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != (B, H, nblk, d + 1, d):
        raise TypeError("out must be a contiguous fp32 tensor [B, H, nblk, d+1, d]")
    with torch.cuda.device(qkv.device):
        _check(lib().lite_la_state_fwd(qkv.data_ptr(), out.data_ptr(), B, N, H, d, int(tokens_per_block),
                                       _stream_handle(stream, qkv.device)))
    return out


def lite_la_elu1_fwd(qkv, H: int, tokens_per_block: int = 0, d: int = 32, clamp_min: float = 1e-6, out=None,
                     out_dtype=None, stream=None):
    """The ELU+1 variant (phi = ELU + 1, phi(q) / sqrt(d), denominator clamped at clamp_min);
    block-causal when tokens_per_block > 0.  Returns out [B, N, H*d]."""
    torch = _torch()
    B, N, out = _prepare(qkv, H, d, out, out_dtype or torch.bfloat16)
    fn = lib().lite_la_elu1_fwd if out.dtype == torch.bfloat16 else lib().lite_la_elu1_fwd_f32out
    with torch.cuda.device(qkv.device):
        _check(fn(qkv.data_ptr(), out.data_ptr(), B, N, H, d, clamp_min, int(tokens_per_block),
                  _stream_handle(stream, qkv.device)))
    return out


def lite_la_bwd(qkv, dout, H: int, tokens_per_block: int = 0, d: int = 32, eps: float = 1e-15, dqkv=None,
                out_dtype=None, stream=None):
    """Gradients (dq | dk | dv, in qkv's layout [B, N, 3*H*d]) of sum(dout * out) for the LiteLA
    forward of qkv (block-causal when tokens_per_block > 0).  dout: bf16 [B, N, H*d]; the
    result is bf16 unless dqkv/out_dtype say fp32."""
    torch = _torch()
    B, N, _ = _prepare(qkv, H, d, dout, torch.bfloat16)
    if dout.dtype != torch.bfloat16:
        raise TypeError("dout must be a contiguous bf16 tensor [B, N, H*d]")
    if dqkv is None:
        dqkv = torch.empty((B, N, 3 * H * d), dtype=out_dtype or torch.bfloat16, device=qkv.device)
    if dqkv.dtype not in (torch.bfloat16, torch.float32) or not dqkv.is_contiguous() \
            or tuple(dqkv.shape) != (B, N, 3 * H * d) or dqkv.device != qkv.device:
        raise TypeError("dqkv must be a contiguous bf16/fp32 tensor [B, N, 3*H*d] on qkv's device")
    f32 = dqkv.dtype == torch.float32
    sh = _stream_handle(stream, qkv.device)
    with torch.cuda.device(qkv.device):
        if tokens_per_block > 0:
            fn = lib().lite_la_block_causal_bwd_f32out if f32 else lib().lite_la_block_causal_bwd
            _check(fn(qkv.data_ptr(), dout.data_ptr(), dqkv.data_ptr(), B, N, H, d, eps, int(tokens_per_block), sh))
        else:
            fn = lib().lite_la_bwd_f32out if f32 else lib().lite_la_bwd
            _check(fn(qkv.data_ptr(), dout.data_ptr(), dqkv.data_ptr(), B, N, H, d, eps, sh))
    return dqkv


def lite_la_fwd_save_state(qkv, H: int, tokens_per_block: int = 0, d: int = 32, eps: float = 1e-15, stream=None):
    """Forward (bf16 out) that also returns the states its queries use, fp32 [B, H, nblk, d+1, d],
    for lite_la_bwd_from_state.  Returns (out, states)."""
    torch = _torch()
    B, N, out = _prepare(qkv, H, d, None, torch.bfloat16)
    T = tokens_per_block if 0 < tokens_per_block < N else N
    nblk = -(-N // T) if N > 0 else 0
    states = torch.empty((B, H, nblk, d + 1, d), dtype=torch.float32, device=qkv.device)
    with torch.cuda.device(qkv.device):
        _check(lib().lite_la_fwd_save_state(qkv.data_ptr(), out.data_ptr(), states.data_ptr(), B, N, H, d, eps,
                                            int(tokens_per_block), _stream_handle(stream, qkv.device)))
    return out, states


def lite_la_bwd_from_state(qkv, dout, states, H: int, tokens_per_block: int = 0, d: int = 32, eps: float = 1e-15,
                           stream=None):
    """lite_la_bwd (bf16 dqkv) given the forward's states from lite_la_fwd_save_state."""
    torch = _torch()
    B, N, _ = _prepare(qkv, H, d, dout, torch.bfloat16)
    if dout.dtype != torch.bfloat16:
        raise TypeError("dout must be a contiguous bf16 tensor [B, N, H*d]")
    if states.dtype != torch.float32 or not states.is_contiguous() or states.device != qkv.device:
        raise TypeError("states must be a contiguous fp32 tensor on qkv's device")
    dqkv = torch.empty((B, N, 3 * H * d), dtype=torch.bfloat16, device=qkv.device)
    with torch.cuda.device(qkv.device):
        _check(lib().lite_la_bwd_from_state(qkv.data_ptr(), dout.data_ptr(), states.data_ptr(), dqkv.data_ptr(), B, N,
                                            H, d, eps, int(tokens_per_block), _stream_handle(stream, qkv.device)))
    return dqkv


_AUTOGRAD_FN = None


def _autograd_fn():
    """The torch.autograd.Function behind lite_la (built on first use: torch is imported lazily)."""
    global _AUTOGRAD_FN
    if _AUTOGRAD_FN is None:
        torch = _torch()

        class LiteLAFunction(torch.autograd.Function):
            @staticmethod
            def forward(ctx, qkv, H, tokens_per_block, d, eps):
                out, states = lite_la_fwd_save_state(qkv, H, tokens_per_block, d, eps)
                ctx.save_for_backward(qkv, states)
                ctx.args = (H, tokens_per_block, d, eps)
                return out

            @staticmethod
            def backward(ctx, grad_out):
                qkv, states = ctx.saved_tensors
                H, tokens_per_block, d, eps = ctx.args
                if grad_out.dtype != torch.bfloat16 or not grad_out.is_contiguous():
                    grad_out = grad_out.to(torch.bfloat16).contiguous()
                dqkv = lite_la_bwd_from_state(qkv, grad_out, states, H, tokens_per_block, d, eps)
                return dqkv, None, None, None, None

        _AUTOGRAD_FN = LiteLAFunction
    return _AUTOGRAD_FN


def lite_la(qkv, H: int, tokens_per_block: int = 0, d: int = 32, eps: float = 1e-15):
    """LiteLA forward (block-causal when tokens_per_block > 0) that torch autograd can
    differentiate: returns out bf16 [B, N, H*d].  The forward keeps the fp32 states its queries
    use (lite_la_fwd_save_state); the backward hands them with the incoming gradient (as bf16)
    to lite_la_bwd_from_state and returns d(qkv) in qkv's layout."""
    return _autograd_fn().apply(qkv, H, int(tokens_per_block), d, eps)


def lite_la_workspace_bytes(B: int, N: int, H: int, d: int = 32, tokens_per_block: int = 0) -> int:
    return int(lib().lite_la_workspace_bytes(B, N, H, d, tokens_per_block))


# forms of a forward call (lite_la_forward_form)
FORMS = {0: "three_kernel", 1: "fused", 2: "fused_paired", 3: "fused_causal", 4: "fused_paired_causal"}


def lite_la_forward_form(B: int, N: int, H: int, d: int = 32, tokens_per_block: int = 0) -> str:
    """Which kernel form a forward call with these arguments takes on the current device."""
    f = int(lib().lite_la_forward_form(B, N, H, d, tokens_per_block))
    if f < 0:
        raise ValueError("empty or invalid problem")
    return FORMS[f]


def lite_la_set_paired_min_chunk(tokens: int) -> int:
    """Sets the chunk length (the block size of block-causal calls) from which calls take a paired
    fused form (tokens <= 0: the default); returns the previous value."""
    return int(lib().lite_la_set_paired_min_chunk(int(tokens)))


def _check_weight(w, bias, C_in, device):
    torch = _torch()
    if not isinstance(w, torch.Tensor) or w.dtype != torch.bfloat16 or w.dim() != 2 or not w.is_contiguous() \
            or w.shape[1] != C_in or w.device != device:
        raise TypeError("w_o must be a contiguous bf16 tensor [C_out, %d] on the input's device" % C_in)
    if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (w.shape[0],)
                             or not bias.is_contiguous() or bias.device != device):
        raise TypeError("bias must be a contiguous fp32 tensor [C_out] on the input's device")
    return int(w.shape[0])


def _proj_out(out, B, N, C_out, device):
    torch = _torch()
    if out is None:
        return torch.empty((B, N, C_out), dtype=torch.bfloat16, device=device)
    if out.dtype != torch.bfloat16 or not out.is_contiguous() or tuple(out.shape) != (B, N, C_out) \
            or out.device != device:
        raise TypeError("out must be a contiguous bf16 tensor [B, N, C_out] on the input's device")
    return out


def lite_la_fwd_oproj(qkv, H: int, w_o, bias=None, tokens_per_block: int = 0, d: int = 32, eps: float = 1e-15,
                      out=None, stream=None):
    """LiteLA followed by the output projection, y = LiteLA(qkv) w_o^T (+ bias), in one pass
    whose apply runs inside the projection GEMM (LiteLA's output never goes to memory).
    w_o: bf16 [C_out, H*d]; bias: fp32 [C_out] or None; returns y bf16 [B, N, C_out]."""
    torch = _torch()
    if not isinstance(qkv, torch.Tensor) or not qkv.is_cuda or qkv.dtype != torch.bfloat16 or qkv.dim() != 3 \
            or not qkv.is_contiguous() or qkv.shape[2] != 3 * H * d:
        raise TypeError("qkv must be a contiguous bf16 CUDA tensor [B, N, 3*H*d]")
    B, N = int(qkv.shape[0]), int(qkv.shape[1])
    C_out = _check_weight(w_o, bias, H * d, qkv.device)
    out = _proj_out(out, B, N, C_out, qkv.device)
    with torch.cuda.device(qkv.device):
        _check(lib().lite_la_fwd_oproj(qkv.data_ptr(), w_o.data_ptr(), bias.data_ptr() if bias is not None else None,
                                       out.data_ptr(), B, N, H, d, C_out, eps, int(tokens_per_block),
                                       _stream_handle(stream, qkv.device)))
    return out


def lite_la_out_proj(x, w_o, bias=None, out=None, stream=None):
    """The projection alone, y = x w_o^T (+ bias), on a bf16 [B, N, C_in] input (e.g.
    lite_la_fwd's output: the unfused chain), with the same GEMM kernel."""
    torch = _torch()
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 3 \
            or not x.is_contiguous():
        raise TypeError("x must be a contiguous bf16 CUDA tensor [B, N, C_in]")
    B, N, C_in = x.shape
    C_out = _check_weight(w_o, bias, C_in, x.device)
    out = _proj_out(out, B, N, C_out, x.device)
    with torch.cuda.device(x.device):
        _check(lib().lite_la_out_proj(x.data_ptr(), w_o.data_ptr(), bias.data_ptr() if bias is not None else None,
                                      out.data_ptr(), B, N, C_in, C_out, _stream_handle(stream, x.device)))
    return out


def lite_la_device_status(stream=None) -> None:
    """Synchronises the stream and raises LiteLAError if a kernel reported a timed-out wait."""
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    _check(lib().lite_la_device_status(ctypes.c_void_p(s.cuda_stream)))


def lite_la_release_workspace() -> None:
    _check(lib().lite_la_release_workspace())
