"""B200 (sm_100a) FAVOR attention forward pass: Python binding of libfavor.so.

The binding only marshals arguments. Every step of the computation runs in the CUDA kernels
of ``libfavor.so``, and PyTorch supplies device memory and streams. There is no CPU fallback:
if the library is missing or a call fails, an exception is raised.

Entry points mirror the C ABI in include/favor.h:
    favor_attention, favor_attention_chunked, favor_attention_f32, favor_orf_omega,
    favor_attention_host, favor_sync_status, favor_status_string, favor_workspace_bytes,
    favor_selftest_timeout, favor_selftest_sincos, favor_attention_f32_noalloc,
    favor_noalloc_scratch_bytes,
    favor_decode_state_bytes, favor_decode_init, favor_decode_step, favor_orf_omega_seeded,
    favor_orf_gaussians_seeded, favor_philox4x64, favor_attention_backward_f32
"""
from __future__ import annotations

import ctypes
import os

FAVOR_TRIG = 0
FAVOR_RELU = 1
STATUS = {
    0: "FAVOR_OK", -1: "FAVOR_ERR_NULL", -2: "FAVOR_ERR_ALIGN", -3: "FAVOR_ERR_SHAPE",
    -4: "FAVOR_ERR_KIND", -5: "FAVOR_ERR_UNSUPPORTED", -6: "FAVOR_ERR_CUDA",
    -7: "FAVOR_ERR_TIMEOUT", -8: "FAVOR_ERR_DEVICE",
}
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfavor.so")

_vp, _i, _ll, _sz, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_uint64
_SIGS = {
    "favor_attention": (_i, [_vp] * 5 + [_i] * 7 + [_vp]),
    "favor_attention_chunked": (_i, [_vp] * 5 + [_i] * 8 + [_vp]),
    "favor_attention_f32": (_i, [_vp] * 5 + [_i] * 7 + [_vp]),
    "favor_orf_omega": (_i, [_vp] * 3 + [_i] * 4 + [_vp]),
    "favor_attention_host": (_i, [_vp] * 5 + [_i] * 8 + [_vp]),
    "favor_sync_status": (_i, [_vp]),
    "favor_status_string": (ctypes.c_char_p, [_i]),
    "favor_selftest_timeout": (_i, [_ll, _vp]),
    "favor_selftest_sincos": (_i, [_vp] * 3 + [_i, _vp]),
    "favor_workspace_bytes": (_sz, [_i] * 7),
    "favor_attention_f32_noalloc": (_i, [_vp] * 5 + [_i] * 7 + [_vp]),
    "favor_noalloc_scratch_bytes": (_sz, []),
    "favor_decode_state_bytes": (_sz, [_i] * 5),
    "favor_decode_init": (_i, [_vp] + [_i] * 5 + [_vp]),
    "favor_decode_step": (_i, [_vp] * 6 + [_i] * 5 + [_vp]),
    "favor_orf_omega_seeded": (_i, [_u64, _vp] + [_i] * 4 + [_vp]),
    "favor_orf_gaussians_seeded": (_i, [_u64, _vp, _vp] + [_i] * 3 + [_vp]),
    "favor_philox4x64": (_i, [_u64, _u64, _u64, _vp, _vp]),
    "favor_attention_backward_f32": (_i, [_vp] * 8 + [_i] * 7 + [_vp]),
}
_LIB = None


class FavorError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({favor_status_string(code)})")


def lib() -> ctypes.CDLL:
    """Load libfavor.so (built in-tree). Raises ImportError if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m linear_kernelized_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _LIB = L
    return _LIB


def favor_status_string(code: int) -> str:
    return lib().favor_status_string(int(code)).decode()


def _check(rc: int, where: str):
    if rc != 0:
        raise FavorError(rc, where)


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check_qkv(q, k, v, omega, dtype):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("omega", omega)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share the shape [B, H, L, d]")
    B, H, L, d = q.shape
    if omega.dim() != 3 or omega.shape[0] != H or omega.shape[2] != d:
        raise ValueError("omega must have shape [H, M, d]")
    return B, H, L, d, omega.shape[1]


def _check_out(out, like, name="out"):
    """An output tensor must match `like` in shape, dtype and device, and be contiguous: the C
    layer sees only a pointer and writes B*H*L*d elements through it."""
    import torch
    if not isinstance(out, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if out.shape != like.shape or out.dtype != like.dtype or out.device != like.device:
        raise ValueError(f"{name} must have shape {tuple(like.shape)}, dtype {like.dtype} and device "
                         f"{like.device}; got {tuple(out.shape)}, {out.dtype}, {out.device}")
    if not out.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def favor_attention(q, k, v, omega, out=None, feature_kind=FAVOR_TRIG, causal=False, chunk=0,
                    stream=None):
    """bf16 FAVOR forward. q, k, v: [B,H,L,d]; omega: [H,M,d]. Tensor-core kernels for the shapes
    they cover; other shapes up to d = 128, M = 512 run the fp32 CUDA-core kernels on widened
    copies (favor_attention in include/favor.h)."""
    import torch
    B, H, L, d, M = _check_qkv(q, k, v, omega, torch.bfloat16)
    if out is None:
        out = torch.empty_like(q)
    _check_out(out, q)
    rc = lib().favor_attention_chunked(q.data_ptr(), k.data_ptr(), v.data_ptr(), omega.data_ptr(),
                                       out.data_ptr(), B, H, L, d, M, int(feature_kind), int(causal),
                                       int(chunk), _stream(stream))
    _check(rc, "favor_attention")
    return out


def favor_attention_chunked(q, k, v, omega, out=None, feature_kind=FAVOR_TRIG, causal=False,
                            chunk=0, stream=None):
    return favor_attention(q, k, v, omega, out, feature_kind, causal, chunk, stream)


def favor_attention_f32(q, k, v, omega, out=None, feature_kind=FAVOR_TRIG, causal=False,
                        stream=None):
    """fp32 FAVOR forward on the accuracy path."""
    import torch
    B, H, L, d, M = _check_qkv(q, k, v, omega, torch.float32)
    if out is None:
        out = torch.empty_like(q)
    _check_out(out, q)
    rc = lib().favor_attention_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), omega.data_ptr(),
                                   out.data_ptr(), B, H, L, d, M, int(feature_kind), int(causal),
                                   _stream(stream))
    _check(rc, "favor_attention_f32")
    return out


def _check_omega_out(out, H, M, d):
    import torch
    if not isinstance(out, torch.Tensor) or not out.is_cuda or not out.is_contiguous():
        raise TypeError("out must be a contiguous CUDA tensor")
    if tuple(out.shape) != (H, M, d) or out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError(f"out must have shape {(H, M, d)} and dtype float32 or bfloat16")


def favor_orf_omega(gauss_blocks, gauss_norms, M, dtype=None, out=None, stream=None):
    """Build ORF Omega [H, M, d] on the device from fp64 Gaussian draws (see include/favor.h)."""
    import torch
    dtype = dtype or torch.bfloat16
    H, nb, d, d2 = gauss_blocks.shape
    if d != d2 or gauss_norms.shape != (H, M, d) or nb != -(-M // d):
        raise ValueError("gauss_blocks must be [H, ceil(M/d), d, d] and gauss_norms [H, M, d]")
    for t in (gauss_blocks, gauss_norms):
        if t.dtype != torch.float64 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("Gaussian draws must be contiguous float64 CUDA tensors")
    if out is None:
        out = torch.empty((H, M, d), dtype=dtype, device=gauss_blocks.device)
    _check_omega_out(out, H, M, d)
    code = {torch.float32: 0, torch.bfloat16: 1}[out.dtype]
    rc = lib().favor_orf_omega(gauss_blocks.data_ptr(), gauss_norms.data_ptr(), out.data_ptr(), H, M,
                               d, code, _stream(stream))
    _check(rc, "favor_orf_omega")
    return out


def favor_attention_host(q, k, v, omega, out, feature_kind=FAVOR_TRIG, causal=False, stream=None):
    """Host-buffer entry: q, k, v, omega, out are CPU tensors (pinned for async copies)."""
    import torch
    for t in (q, k, v, omega, out):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
            raise TypeError("favor_attention_host takes contiguous CPU tensors")
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("favor_attention_host takes float32 or bfloat16 tensors")
    code = {torch.float32: 0, torch.bfloat16: 1}[q.dtype]
    if q.dim() != 4:
        raise ValueError("q must have shape [B, H, L, d]")
    B, H, L, d = q.shape
    for name, t in (("k", k), ("v", v), ("out", out)):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape {tuple(q.shape)} and dtype {q.dtype}")
    if omega.dim() != 3 or omega.shape[0] != H or omega.shape[2] != d or omega.dtype != q.dtype:
        raise ValueError("omega must have shape [H, M, d] and q's dtype")
    M = omega.shape[1]
    rc = lib().favor_attention_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), omega.data_ptr(),
                                    out.data_ptr(), B, H, L, d, M, int(feature_kind), int(causal),
                                    code, _stream(stream))
    _check(rc, "favor_attention_host")
    return out


def favor_sync_status(stream=None) -> int:
    return lib().favor_sync_status(_stream(stream))


def favor_workspace_bytes(B, H, L, d, M, feature_kind=FAVOR_TRIG, causal=False) -> int:
    return lib().favor_workspace_bytes(B, H, L, d, M, int(feature_kind), int(causal))


def favor_selftest_timeout(limit_cycles: int, stream=None) -> int:
    return lib().favor_selftest_timeout(int(limit_cycles), _stream(stream))


def favor_selftest_sincos(u, stream=None):
    """FMA-pipe (sin(u), cos(u)) of a contiguous float32 CUDA tensor, as two new tensors."""
    import torch
    if u.dtype != torch.float32 or not u.is_cuda or not u.is_contiguous():
        raise ValueError("u must be a contiguous float32 CUDA tensor")
    s, c = torch.empty_like(u), torch.empty_like(u)
    rc = lib().favor_selftest_sincos(u.data_ptr(), s.data_ptr(), c.data_ptr(), u.numel(), _stream(stream))
    if rc != 0:
        raise FavorError(rc, "favor_selftest_sincos")
    return s, c


def favor_attention_f32_noalloc(q, k, v, omega, out=None, feature_kind=FAVOR_TRIG, causal=False,
                                stream=None):
    """fp32 forward with its workspace in the library's static device array (no allocation by
    the library; `out` is allocated here only if not given). Calls that overlap in time race on
    the shared workspace: see include/favor.h."""
    import torch
    B, H, L, d, M = _check_qkv(q, k, v, omega, torch.float32)
    if out is None:
        out = torch.empty_like(q)
    _check_out(out, q)
    rc = lib().favor_attention_f32_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), omega.data_ptr(),
                                           out.data_ptr(), B, H, L, d, M, int(feature_kind), int(causal),
                                           _stream(stream))
    _check(rc, "favor_attention_f32_noalloc")
    return out


def favor_noalloc_scratch_bytes() -> int:
    return lib().favor_noalloc_scratch_bytes()


# ---------------------------------------------------------------- causal decode (carried state)
def favor_decode_state_bytes(B, H, d, M, feature_kind=FAVOR_TRIG) -> int:
    return lib().favor_decode_state_bytes(B, H, d, M, int(feature_kind))


def favor_decode_init(state, B, H, d, M, feature_kind=FAVOR_TRIG, stream=None):
    """Set `state` (a CUDA tensor of favor_decode_state_bytes bytes) to the empty state."""
    rc = lib().favor_decode_init(state.data_ptr(), B, H, d, M, int(feature_kind), _stream(stream))
    _check(rc, "favor_decode_init")
    return state


def favor_decode_new_state(B, H, d, M, feature_kind=FAVOR_TRIG, device="cuda", stream=None):
    """Allocate (with torch) and initialise an empty decode state: a flat float32 tensor."""
    import torch
    n = favor_decode_state_bytes(B, H, d, M, feature_kind)
    if n == 0:
        raise FavorError(-5, "favor_decode_state_bytes")
    state = torch.empty(n // 4, dtype=torch.float32, device=device)
    return favor_decode_init(state, B, H, d, M, feature_kind, stream)


def favor_decode_state_views(state, B, H, d, M, feature_kind=FAVOR_TRIG):
    """Views (S [B*H, F, d], z [B*H, F], c [B*H]) of a decode state, per include/favor.h."""
    F = 2 * M if feature_kind == FAVOR_TRIG else M
    BH = B * H
    S = state[:BH * F * d].view(BH, F, d)
    z = state[BH * F * d:BH * F * (d + 1)].view(BH, F)
    c = state[BH * F * (d + 1):BH * F * (d + 1) + BH]
    return S, z, c


def favor_decode_step(q, k, v, omega, state, out=None, feature_kind=FAVOR_TRIG, stream=None):
    """One causal decode step. q, k, v: [B, H, d] bf16 (one token per head); omega: [H, M, d]
    bf16; state: from favor_decode_new_state, updated in place. Returns out [B, H, d] bf16."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("omega", omega)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share the shape [B, H, d]")
    B, H, d = q.shape
    if omega.dim() != 3 or omega.shape[0] != H or omega.shape[2] != d:
        raise ValueError("omega must have shape [H, M, d]")
    M = omega.shape[1]
    need = favor_decode_state_bytes(B, H, d, M, feature_kind)
    if not state.is_cuda or state.numel() * state.element_size() < need:
        raise ValueError(f"state must be a CUDA tensor of at least {need} bytes")
    if out is None:
        out = torch.empty_like(q)
    _check_out(out, q)
    rc = lib().favor_decode_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), omega.data_ptr(),
                                 state.data_ptr(), out.data_ptr(), B, H, d, M, int(feature_kind),
                                 _stream(stream))
    _check(rc, "favor_decode_step")
    return out


# ---------------------------------------------------------------- ORF redrawn from a seed
def favor_orf_omega_seeded(seed, H, M, d, dtype=None, out=None, device="cuda", stream=None):
    """ORF Omega [H, M, d] drawn on the device from `seed` (Philox4x64-10; see include/favor.h)."""
    import torch
    dtype = dtype or torch.bfloat16
    if out is None:
        out = torch.empty((H, M, d), dtype=dtype, device=device)
    _check_omega_out(out, H, M, d)
    code = {torch.float32: 0, torch.bfloat16: 1}[out.dtype]
    rc = lib().favor_orf_omega_seeded(int(seed) & (2**64 - 1), out.data_ptr(), H, M, d, code, _stream(stream))
    _check(rc, "favor_orf_omega_seeded")
    return out


def favor_orf_gaussians_seeded(seed, H, M, d, device="cuda", stream=None):
    """The draws behind favor_orf_omega_seeded: (G [H, ceil(M/d), d, d], R [H, M, d]) float64."""
    import torch
    nb = -(-M // d)
    G = torch.empty((H, nb, d, d), dtype=torch.float64, device=device)
    R = torch.empty((H, M, d), dtype=torch.float64, device=device)
    rc = lib().favor_orf_gaussians_seeded(int(seed) & (2**64 - 1), G.data_ptr(), R.data_ptr(), H, M, d,
                                          _stream(stream))
    _check(rc, "favor_orf_gaussians_seeded")
    return G, R


def favor_philox4x64(key, first_counter, n_blocks, device="cuda", stream=None):
    """Raw Philox4x64-10 blocks: an int64 tensor [n_blocks, 4] holding the uint64 words' bits."""
    import torch
    out = torch.empty((n_blocks, 4), dtype=torch.int64, device=device)
    rc = lib().favor_philox4x64(int(key) & (2**64 - 1), int(first_counter) & (2**64 - 1), int(n_blocks),
                                out.data_ptr(), _stream(stream))
    _check(rc, "favor_philox4x64")
    return out


# ---------------------------------------------------------------- backward
def favor_attention_backward_f32(q, k, v, omega, dout, feature_kind=FAVOR_TRIG, causal=False, stream=None):
    """fp32 gradients (dq, dk, dv) of sum(dout * out) for out = favor_attention_f32(q, k, v, omega)."""
    import torch
    B, H, L, d, M = _check_qkv(q, k, v, omega, torch.float32)
    if dout.shape != q.shape or dout.dtype != torch.float32 or not dout.is_cuda or not dout.is_contiguous():
        raise ValueError("dout must be a contiguous float32 CUDA tensor shaped like q")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = lib().favor_attention_backward_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), omega.data_ptr(),
                                            dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                            B, H, L, d, M, int(feature_kind), int(causal), _stream(stream))
    _check(rc, "favor_attention_backward_f32")
    return dq, dk, dv
