"""FLARE++ token-mixer forward for NVIDIA B200 (sm_100a).

Python binding of ``libflarepp.so`` (C ABI declared in ``include/flarepp.h``).
The functions here only marshal torch CUDA tensors into pointers and sizes
and call the library with the same names; every step of the computation runs
in the library's CUDA kernels.  There is no fallback: if the library is not
built, or a tensor is not on a CUDA device, the call raises.

    seed encode     Q_dyn = softmax_N(Q~ K^T) V
    routing encode  Z     = softmax_N(Q_dyn K^T) V
    decode          Y     = softmax_M(K Q_dyn^T) Z          (scale 1 throughout)

Layouts: seeds / fixed queries [H, M, D]; K, V, Y [B, H, N, D]; Q_dyn, Z
[B, H, M, D]; contiguous; dtype torch.bfloat16 (tensor cores) or
torch.float32 (CUDA cores).
"""
from __future__ import annotations

import ctypes
import os
import re

__all__ = [
    "FlareError",
    "lib",
    "flare_encode",
    "flare_decode",
    "flarepp_mix",
    "flarepp_mix_debug",
    "flare_encode_workspace_size",
    "flare_encode_lse",
    "flare_encode_lse_workspace_size",
    "flare_lse_combine",
    "flarepp_mix_backward",
    "flarepp_mix_backward_workspace_size",
    "flarepp_mix_save",
    "flarepp_mix_backward_saved",
    "flarepp_saved_bytes",
    "flarepp_mix_backward_shard",
    "flarepp_workspace_size",
    "flarepp_mix_host",
    "flare_communication_matrix",
    "flare_check_status",
    "flare_last_launch_count",
    "flare_cuda_error_string",
    "flare_set_split_override",
    "flare_encode_splits",
    "flare_set_launch_overlap",
    "flare_set_wait_limit_ms",
    "flare_profile_begin",
    "flare_profile_end",
    "LIB_PATH",
    "HEADER_PATH",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflarepp.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "flarepp.h")

F32, BF16, BF16_F32OUT = 0, 1, 2
CUDA_ERROR = 3  # FLARE_ERR_CUDA
_c_int, _c_i64, _c_size, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
_SIZES = [_c_int, _c_int, _c_i64, _c_int, _c_int, _c_int]  # B, H, N, M, D, dtype

_SIGNATURES = {
    "flare_encode_workspace_size": (_c_size, _SIZES),
    "flarepp_workspace_size": (_c_size, _SIZES),
    "flare_encode": (_c_int, [_vp, _c_int, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flare_decode": (_c_int, [_vp, _vp, _c_int, _vp, _vp, *_SIZES, _vp]),
    "flare_encode_lse_workspace_size": (_c_size, _SIZES),
    "flarepp_mix_backward_workspace_size": (_c_size, _SIZES),
    "flarepp_mix_backward": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flarepp_saved_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "flarepp_mix_save": (_c_int, [_vp, _vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flarepp_mix_backward_saved": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flarepp_backward_shard_exchange_floats": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "flarepp_backward_shard_workspace_size": (_c_size, _SIZES),
    "flarepp_mix_backward_shard": (_c_int, [_c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, *_SIZES, _vp,
                                            _c_size, _vp]),
    "flare_encode_lse": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flare_lse_combine": (_c_int, [_vp, _vp, _c_int, _c_i64, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                   _vp]),
    "flarepp_mix": (_c_int, [_vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flarepp_mix_debug": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flare_check_status": (_c_int, [_vp, ctypes.POINTER(_c_int)]),
    "flare_status_string": (ctypes.c_char_p, [_c_int]),
    "flare_last_launch_count": (_c_int, []),
    "flare_cuda_error_string": (ctypes.c_char_p, []),
    "flarepp_mix_host_workspace_size": (_c_size, _SIZES),
    "flarepp_mix_host": (_c_int, [_vp, _vp, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flare_communication_workspace_size": (_c_size, _SIZES),
    "flare_communication_matrix": (_c_int, [_vp, _c_int, _vp, _vp, *_SIZES, _vp, _c_size, _vp]),
    "flare_set_split_override": (_c_int, [_c_int]),
    "flare_encode_splits": (_c_int, [_c_int, _c_int, ctypes.c_int64]),
    "flare_set_launch_overlap": (_c_int, [_c_int]),
    "flare_selftest_wait_timeout": (_c_int, [_c_int, _vp]),
    "flare_set_wait_limit_ms": (_c_int, [_c_int]),
    "flare_profile_begin": (_c_int, [_c_int]),
    "flare_profile_end": (_c_int, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_c_int), _c_int]),
}

KERNEL_NAMES = {1: "encode_tc", 2: "lse_merge", 3: "decode_tc", 4: "encode_f32", 5: "decode_f32",
                6: "bwd_token_stats", 7: "bwd_latent", 8: "bwd_reduce", 9: "bwd_token_grad", 10: "comm_tc",
                11: "comm_reduce"}

_lib = None


class FlareError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {lib().flare_status_string(status).decode()} (status {status})"
        if status == CUDA_ERROR:
            msg += f": {lib().flare_cuda_error_string().decode()}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded ``libflarepp.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m rank_latent_attention_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


def header_functions() -> list[str]:
    """Names of the functions ``include/flarepp.h`` declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(flare\w*)\s*\(", text, flags=re.M)


# ---------------------------------------------------------------- marshalling
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _ptr(t, name: str, dtype):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise FlareError(rc, where)


def _ws(workspace):
    if workspace is None:
        return None, 0
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def flare_encode_workspace_size(B, H, N, M, D, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if "bfloat16" in str(dtype) else F32)
    return lib().flare_encode_workspace_size(B, H, N, M, D, code)


def flarepp_workspace_size(B, H, N, M, D, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if "bfloat16" in str(dtype) else F32)
    return lib().flarepp_workspace_size(B, H, N, M, D, code)


def flare_encode(Q, K, V, Z=None, *, workspace=None, stream=None):
    """FLARE encode Z = softmax_N(Q K^T) V.  Q is [H,M,D] (shared) or [B,H,M,D]."""
    torch = _torch()
    B, H, N, D = K.shape
    q_batched = 1 if Q.dim() == 4 else 0
    M = Q.shape[-2]
    if Z is None:
        Z = torch.empty((B, H, M, D), dtype=K.dtype, device=K.device)
    ws, wsb = _ws(workspace)
    _check(lib().flare_encode(_ptr(Q, "Q", K.dtype), q_batched, _ptr(K, "K", K.dtype), _ptr(V, "V", K.dtype),
                              _ptr(Z, "Z", K.dtype), B, H, N, M, D, _dtype_code(K), ws, wsb, _stream(stream)),
           "flare_encode")
    return Z


def flare_decode(K, Q, Z, Y=None, *, stream=None):
    """FLARE decode Y = softmax_M(K Q^T) Z.  Q is [H,M,D] (shared) or [B,H,M,D]."""
    torch = _torch()
    B, H, N, D = K.shape
    q_batched = 1 if Q.dim() == 4 else 0
    M = Q.shape[-2]
    if Y is None:
        Y = torch.empty_like(K)
    _check(lib().flare_decode(_ptr(K, "K", K.dtype), _ptr(Q, "Q", K.dtype), q_batched, _ptr(Z, "Z", K.dtype),
                              _ptr(Y, "Y", K.dtype), B, H, N, M, D, _dtype_code(K), _stream(stream)),
           "flare_decode")
    return Y


def flare_encode_lse_workspace_size(B, H, N, M, D, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if "bfloat16" in str(dtype) else F32)
    return lib().flare_encode_lse_workspace_size(B, H, N, M, D, code)


def flare_encode_lse(Q, K, V, O=None, lse=None, *, workspace=None, stream=None):
    """One token shard's encode: O = softmax over the shard's tokens of Q K^T,
    times V (fp32 [B,H,M,D]), and lse = log-sum-exp of those logits (fp32
    [B,H,M], natural log).  K and V may hold no tokens (N = 0): O = 0 and
    lse = -inf.  Returns (O, lse)."""
    torch = _torch()
    B, H, N, D = K.shape
    q_batched = 1 if Q.dim() == 4 else 0
    M = Q.shape[-2]
    if O is None:
        O = torch.empty((B, H, M, D), dtype=torch.float32, device=Q.device)
    if lse is None:
        lse = torch.empty((B, H, M), dtype=torch.float32, device=Q.device)
    kv = (None, None) if N == 0 else (_ptr(K, "K", K.dtype), _ptr(V, "V", K.dtype))
    ws, wsb = _ws(workspace)
    _check(lib().flare_encode_lse(_ptr(Q, "Q", K.dtype), q_batched, kv[0], kv[1], _ptr(O, "O", torch.float32),
                                  _ptr(lse, "lse", torch.float32), B, H, N, M, D, _dtype_code(K), ws, wsb,
                                  _stream(stream)),
           "flare_encode_lse")
    return O, lse


def flare_lse_combine(O_parts, lse_parts, out=None, lse_out=None, *, dtype=None, shape=None, part_stride=0,
                      stream=None):
    """Exact combination of R token shards' (O, lse): out = sum_r
    exp(lse_r - L) O_r with L = log sum_r exp(lse_r).

    Dense form: O_parts [R,B,H,M,D] and lse_parts [R,B,H,M] fp32.  Strided
    form (``part_stride`` > 0, ``shape`` = (R, B, H, M, D)): O_parts and
    lse_parts are flat fp32 tensors whose shard r starts ``r * part_stride``
    floats in.  ``out`` [B,H,M,D] has ``dtype`` (default: out's, else
    bfloat16); ``lse_out`` [B,H,M] fp32 is written when given."""
    torch = _torch()
    R, B, H, M, D = shape if shape is not None else O_parts.shape
    if out is None:
        out = torch.empty((B, H, M, D), dtype=dtype or torch.bfloat16, device=O_parts.device)
    _check(lib().flare_lse_combine(_ptr(O_parts, "O_parts", torch.float32), _ptr(lse_parts, "lse_parts", torch.float32),
                                   R, part_stride, _ptr(out, "out", out.dtype),
                                   _ptr(lse_out, "lse_out", torch.float32), B, H, M, D, _dtype_code(out),
                                   _stream(stream)),
           "flare_lse_combine")
    return out


def flarepp_mix_backward_workspace_size(B, H, N, M, D, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if "bfloat16" in str(dtype) else F32)
    return lib().flarepp_mix_backward_workspace_size(B, H, N, M, D, code)


def flarepp_mix_backward(seeds, K, V, dY, d_seeds=None, dK=None, dV=None, *, workspace=None, stream=None):
    """Gradients (d_seeds [H,M,D], dK, dV [B,H,N,D]) of sum(dY * Y) for
    Y = flarepp_mix(seeds, K, V); all tensors share K's dtype."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[-2]
    if d_seeds is None:
        d_seeds = torch.empty_like(seeds)
    if dK is None:
        dK = torch.empty_like(K)
    if dV is None:
        dV = torch.empty_like(V)
    ws, wsb = _ws(workspace)
    dt = K.dtype
    _check(lib().flarepp_mix_backward(_ptr(seeds, "seeds", dt), _ptr(K, "K", dt), _ptr(V, "V", dt),
                                      _ptr(dY, "dY", dt), _ptr(d_seeds, "d_seeds", dt), _ptr(dK, "dK", dt),
                                      _ptr(dV, "dV", dt), B, H, N, M, D, _dtype_code(K), ws, wsb,
                                      _stream(stream)),
           "flarepp_mix_backward")
    return d_seeds, dK, dV


def flarepp_saved_bytes(B, H, M, D, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (BF16 if "bfloat16" in str(dtype) else F32)
    return lib().flarepp_saved_bytes(B, H, M, D, code)


def flarepp_mix_save(seeds, K, V, Y=None, saved=None, *, workspace=None, stream=None):
    """flarepp_mix that also keeps the backward's state (Q_dyn, Z and the two
    encodes' log-sum-exps) in `saved`, a uint8 CUDA tensor of
    flarepp_saved_bytes bytes.  Returns (Y, saved)."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[-2]
    if Y is None:
        Y = torch.empty_like(K)
    if saved is None:
        saved = torch.empty(flarepp_saved_bytes(B, H, M, D, K.dtype), dtype=torch.uint8, device=K.device)
    ws, wsb = _ws(workspace)
    dt = K.dtype
    _check(lib().flarepp_mix_save(_ptr(seeds, "seeds", dt), _ptr(K, "K", dt), _ptr(V, "V", dt), _ptr(Y, "Y", dt),
                                  _ptr(saved, "saved", torch.uint8), B, H, N, M, D, _dtype_code(K), ws, wsb,
                                  _stream(stream)),
           "flarepp_mix_save")
    return Y, saved


def flarepp_mix_backward_saved(seeds, K, V, dY, saved, d_seeds=None, dK=None, dV=None, *, workspace=None,
                               stream=None):
    """flarepp_mix_backward reading Q_dyn, Z and the log-sum-exps that
    flarepp_mix_save kept instead of recomputing the two encodes."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[-2]
    d_seeds = torch.empty_like(seeds) if d_seeds is None else d_seeds
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    ws, wsb = _ws(workspace)
    dt = K.dtype
    _check(lib().flarepp_mix_backward_saved(_ptr(seeds, "seeds", dt), _ptr(K, "K", dt), _ptr(V, "V", dt),
                                            _ptr(dY, "dY", dt), _ptr(saved, "saved", torch.uint8),
                                            _ptr(d_seeds, "d_seeds", dt), _ptr(dK, "dK", dt), _ptr(dV, "dV", dt),
                                            B, H, N, M, D, _dtype_code(K), ws, wsb, _stream(stream)),
           "flarepp_mix_backward_saved")
    return d_seeds, dK, dV


def flarepp_mix_backward_shard(phase, seeds, K, V, dY, saved, exchange, d_seeds, dK, dV, workspace, *,
                               stream=None):
    """One phase (0-3) of the token-sharded backward for this rank's tokens
    K, V, dY [B,H,N_r,D] (N_r may be 0).  `saved` is the whole cloud's state
    (uint8, flarepp_mix_save's layout), `exchange` an fp32 buffer the caller
    sums over the ranks between phases, `workspace` a uint8 buffer kept for
    all four phases.  d_seeds is written in phase 3, dK and dV too."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[-2]
    dt = seeds.dtype
    kv = (None,) * 5 if N == 0 else (_ptr(K, "K", dt), _ptr(V, "V", dt), _ptr(dY, "dY", dt), _ptr(dK, "dK", dt),
                                     _ptr(dV, "dV", dt))
    _check(lib().flarepp_mix_backward_shard(phase, _ptr(seeds, "seeds", dt), kv[0], kv[1], kv[2],
                                            _ptr(saved, "saved", torch.uint8), _ptr(exchange, "exchange", torch.float32),
                                            _ptr(d_seeds, "d_seeds", dt), kv[3], kv[4], B, H, N, M, D,
                                            _dtype_code(seeds), ctypes.c_void_p(workspace.data_ptr()),
                                            workspace.numel(), _stream(stream)),
           "flarepp_mix_backward_shard")


def flarepp_mix_host(seeds, K, V, Y=None, *, out_dtype=None, workspace=None, stream=None):
    """flarepp_mix with seeds, K, V and Y in host memory (CPU tensors; pin
    them for asynchronous copies).  The library streams the heads through
    the GPU, overlapping copies in, compute and copies out; Y is complete
    once `stream` (default: the current CUDA stream) has completed."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[-2]
    code, ydt = _mix_mode(K, out_dtype)
    for name, t in (("seeds", seeds), ("K", K), ("V", V)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
    if Y is None:
        Y = torch.empty((B, H, N, D), dtype=ydt, pin_memory=K.is_pinned())
    if Y.device.type != "cpu" or not Y.is_contiguous() or Y.dtype != ydt:
        raise ValueError("Y must be a contiguous CPU tensor of the output dtype")
    ws, wsb = _ws(workspace)
    _check(lib().flarepp_mix_host(seeds.data_ptr(), K.data_ptr(), V.data_ptr(), Y.data_ptr(), B, H, N, M, D, code,
                                  ws, wsb, _stream(stream)), "flarepp_mix_host")
    return Y


def flare_communication_matrix(Q, K, C=None, *, out_dtype=None, workspace=None, stream=None):
    """C = softmax_N(Q K^T) softmax_M(K Q^T) per head: [B,H,M,M], row-stochastic.

    Its eigenvalues are the nonzero eigenvalues of the rank-M token-to-token
    communication matrix W = W_dec W_enc; the library forms C (the O(M^2 N)
    part) and leaves the O(M^3) eigen-solve of the small M x M matrices to the
    caller.  Q is [H,M,D] (shared) or [B,H,M,D] (e.g. FLARE++'s routing
    queries Q_dyn).  out_dtype=torch.float32 with bf16 inputs returns C in
    fp32 (FLARE_BF16_F32OUT)."""
    torch = _torch()
    B, H, N, D = K.shape
    q_batched = 1 if Q.dim() == 4 else 0
    M = Q.shape[-2]
    code, odt = _mix_mode(K, out_dtype)
    if C is None:
        C = torch.empty((B, H, M, M), dtype=odt, device=K.device)
    ws, wsb = _ws(workspace)
    _check(lib().flare_communication_matrix(_ptr(Q, "Q", K.dtype), q_batched, _ptr(K, "K", K.dtype),
                                            _ptr(C, "C", odt), B, H, N, M, D, code, ws, wsb,
                                            _stream(stream)), "flare_communication_matrix")
    return C


def _mix_mode(K, out_dtype):
    """(dtype code, output torch dtype): bf16 K with out_dtype=float32 selects the fp32-output mode."""
    torch = _torch()
    if out_dtype is None or out_dtype == K.dtype:
        return _dtype_code(K), K.dtype
    if K.dtype == torch.bfloat16 and out_dtype == torch.float32:
        return BF16_F32OUT, torch.float32
    raise TypeError(f"unsupported input/output dtypes {K.dtype} -> {out_dtype}")


def flarepp_mix(seeds, K, V, Y=None, *, out_dtype=None, workspace=None, stream=None):
    """FLARE++ mixer forward: seeds [H,M,D], K/V [B,H,N,D] -> Y [B,H,N,D].

    out_dtype=torch.float32 with bf16 inputs selects the split-precision,
    fp32-output mode (FLARE_BF16_F32OUT)."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[1]
    code, odt = _mix_mode(K, out_dtype)
    if Y is None:
        Y = torch.empty(K.shape, dtype=odt, device=K.device)
    ws, wsb = _ws(workspace)
    _check(lib().flarepp_mix(_ptr(seeds, "seeds", K.dtype), _ptr(K, "K", K.dtype), _ptr(V, "V", K.dtype),
                             _ptr(Y, "Y", odt), B, H, N, M, D, code, ws, wsb, _stream(stream)),
           "flarepp_mix")
    return Y


def flarepp_mix_debug(seeds, K, V, *, Y=None, Q_dyn=None, Z=None, out_dtype=None, workspace=None, stream=None):
    """As flarepp_mix, also returning the intermediates: (Y, Q_dyn, Z)
    (allocated unless given)."""
    torch = _torch()
    B, H, N, D = K.shape
    M = seeds.shape[1]
    code, odt = _mix_mode(K, out_dtype)
    Y = torch.empty(K.shape, dtype=odt, device=K.device) if Y is None else Y
    Qd = torch.empty((B, H, M, D), dtype=odt, device=K.device) if Q_dyn is None else Q_dyn
    Z = torch.empty_like(Qd) if Z is None else Z
    ws, wsb = _ws(workspace)
    _check(lib().flarepp_mix_debug(_ptr(seeds, "seeds", K.dtype), _ptr(K, "K", K.dtype), _ptr(V, "V", K.dtype),
                                   _ptr(Y, "Y", odt), _ptr(Qd, "Q_dyn", odt), _ptr(Z, "Z", odt),
                                   B, H, N, M, D, code, ws, wsb, _stream(stream)),
           "flarepp_mix_debug")
    return Y, Qd, Z


def flare_check_status(stream=None) -> tuple[int, int]:
    """Synchronise the stream and return (status, site) of the device status word (cleared)."""
    site = ctypes.c_int(0)
    rc = lib().flare_check_status(_stream(stream), ctypes.byref(site))
    return rc, site.value


def flare_last_launch_count() -> int:
    return lib().flare_last_launch_count()


def flare_set_split_override(splits: int) -> int:
    return lib().flare_set_split_override(splits)


def flare_encode_splits(B: int, H: int, N: int) -> int:
    """CTAs per head of the tensor-core encode for B x H heads of N tokens (1: no merge follows)."""
    return lib().flare_encode_splits(B, H, N)


def flare_set_launch_overlap(mode: int) -> int:
    """1: the mixer's later kernels overlap their predecessors' tails; 0: never; -1: by size (default)."""
    return lib().flare_set_launch_overlap(mode)


def flare_set_wait_limit_ms(ms: int) -> int:
    return lib().flare_set_wait_limit_ms(ms)


def flare_profile_begin(max_launches: int) -> None:
    _check(lib().flare_profile_begin(max_launches), "flare_profile_begin")


def flare_profile_end(max_records: int = 1 << 16) -> list[tuple[str, float]]:
    """[(kernel name, ms)] for the launches recorded since flare_profile_begin."""
    ms = (ctypes.c_float * max_records)()
    kinds = (_c_int * max_records)()
    n = lib().flare_profile_end(ms, kinds, max_records)
    if n < 0:
        raise FlareError(-n, "flare_profile_end")
    return [(KERNEL_NAMES.get(kinds[i], str(kinds[i])), float(ms[i])) for i in range(n)]
