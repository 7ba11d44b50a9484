"""The C ABI without a GPU: the library loads, exports every function include/favor.h declares,
and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import linear_kernelized_attention_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(favor_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 9, names
    lib = ctypes.CDLL(F.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    for n in _declared():
        assert hasattr(F, n), n


def test_status_strings():
    for code in range(-8, 1):
        s = F.favor_status_string(code)
        assert s and "unknown" not in s
    assert "unknown" in F.favor_status_string(-99)


def _call(**over):
    a = dict(q=16, k=32, v=48, om=64, out=80, B=1, H=1, L=8, d=64, M=64, kind=0, causal=0)
    a.update(over)
    vp = ctypes.c_void_p
    return F.lib().favor_attention(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["om"]), vp(a["out"]),
                                   a["B"], a["H"], a["L"], a["d"], a["M"], a["kind"], a["causal"], None)


@pytest.mark.parametrize("over,code", [
    ({"q": 0}, -1), ({"out": 0}, -1),
    ({"k": 33}, -2), ({"om": 8}, -2),
    ({"L": 0}, -3), ({"B": -1}, -3), ({"M": 0}, -3), ({"d": 0}, -3),
    ({"kind": 2}, -4), ({"kind": -1}, -4),
])
def test_host_validation_rejects_before_any_cuda_call(over, code):
    # fake, never-dereferenced pointers: validation fails first, so nothing touches a device
    assert _call(**over) == code


def test_f32_and_orf_validation():
    vp = ctypes.c_void_p
    L = F.lib()
    assert L.favor_attention_f32(None, vp(16), vp(16), vp(16), vp(16), 1, 1, 1, 1, 1, 0, 0, None) == -1
    assert L.favor_attention_f32(vp(16), vp(16), vp(16), vp(16), vp(16), 1, 1, 1, 1, 1, 5, 0, None) == -4
    assert L.favor_orf_omega(None, vp(16), vp(16), 1, 1, 1, 0, None) == -1
    assert L.favor_orf_omega(vp(16), vp(24), vp(16), 1, 1, 1, 0, None) == -2
    assert L.favor_orf_omega(vp(16), vp(16), vp(16), 0, 1, 1, 0, None) == -3
    assert L.favor_attention_chunked(vp(16), vp(16), vp(16), vp(16), vp(16), 1, 1, 8, 64, 64, 0, 1, 7, None) in (-5, -8, -6)


def test_workspace_bytes_is_host_only():
    assert F.favor_workspace_bytes(1, 1, 1, 64, 64, 0, False) >= 0
    assert F.favor_workspace_bytes(0, 1, 1, 64, 64, 0, False) == 0
    # bidirectional: at least one fp32 partial state per (head, 128-angle block) and one state
    # image per head; causal takes none
    B, H, L, d, M = 4, 8, 4096, 64, 256
    ws = F.favor_workspace_bytes(B, H, L, d, M, 0, False)
    assert ws >= B * H * 2 * (d + 1) * 256 * 4 + B * H * 2 * 256 * (d + 16) * 2
    assert F.favor_workspace_bytes(B, H, L, d, M, 1, False) > 0
    assert F.favor_workspace_bytes(B, H, L, d, M, 0, True) == 0
    # shapes the tensor-core kernels leave out take the CUDA-core route: fp32 copies of q, k, v,
    # the output and Omega, plus the fp32 path's chunk states
    for (dd, MM, causal) in [(48, M, False), (d, 272, False), (128, M, True), (128, M, False)]:
        n = B * H * L * dd
        assert F.favor_workspace_bytes(B, H, L, dd, MM, 0, causal) >= 4 * 4 * n + 4 * H * MM * dd
    # beyond every kernel: none
    assert F.favor_workspace_bytes(B, H, L, 136, M, 0, False) == 0
    assert F.favor_workspace_bytes(B, H, L, d, 528, 1, True) == 0


# ------------------------------------------------------------------ decode entry points
@pytest.mark.parametrize("B,H,d,M,kind", [(1, 1, 64, 256, 0), (4, 8, 64, 256, 1), (2, 3, 128, 512, 0),
                                          (1, 2, 16, 1024, 1)])
def test_decode_state_bytes(B, H, d, M, kind):
    F_ = 2 * M if kind == 0 else M
    assert F.favor_decode_state_bytes(B, H, d, M, kind) == 4 * (B * H * F_ * (d + 1) + B * H)


@pytest.mark.parametrize("args", [(1, 1, 48, 64, 0), (1, 1, 64, 513, 0), (1, 1, 64, 1025, 1),
                                  (0, 1, 64, 64, 0), (1, 1, 64, 64, 2)])
def test_decode_state_bytes_unsupported_is_zero(args):
    assert F.favor_decode_state_bytes(*args) == 0


def _dec(**over):
    a = dict(q=16, k=32, v=48, om=64, st=80, out=96, B=1, H=1, d=64, M=64, kind=0)
    a.update(over)
    vp = ctypes.c_void_p
    return F.lib().favor_decode_step(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["om"]), vp(a["st"]),
                                     vp(a["out"]), a["B"], a["H"], a["d"], a["M"], a["kind"], None)


@pytest.mark.parametrize("over,code", [
    ({"q": 0}, -1), ({"st": 0}, -1), ({"out": 0}, -1),
    ({"v": 50}, -2), ({"st": 84}, -2),
    ({"B": 0}, -3), ({"M": -4}, -3), ({"H": 1 << 30}, -3),
    ({"kind": 3}, -4),
    ({"d": 48}, -5), ({"d": 256}, -5), ({"M": 513}, -5), ({"M": 1025, "kind": 1}, -5),
])
def test_decode_validation_rejects_before_any_cuda_call(over, code):
    assert _dec(**over) == code


def test_decode_init_validation():
    vp = ctypes.c_void_p
    assert F.lib().favor_decode_init(vp(0), 1, 1, 64, 64, 0, None) == -1
    assert F.lib().favor_decode_init(vp(20), 1, 1, 64, 64, 0, None) == -2
    assert F.lib().favor_decode_init(vp(32), 1, 1, 64, 64, 5, None) == -4
    assert F.lib().favor_decode_init(vp(32), 1, 1, 40, 64, 0, None) == -5


def test_seeded_orf_validation_rejects_before_any_cuda_call():
    vp, u = ctypes.c_void_p, ctypes.c_uint64
    L = F.lib()
    assert L.favor_orf_omega_seeded(u(1), vp(0), 1, 64, 64, 0, None) == -1
    assert L.favor_orf_omega_seeded(u(1), vp(24), 1, 64, 64, 0, None) == -2
    assert L.favor_orf_omega_seeded(u(1), vp(32), 0, 64, 64, 0, None) == -3
    assert L.favor_orf_omega_seeded(u(1), vp(32), 1, 64, 256, 0, None) == -5
    assert L.favor_orf_omega_seeded(u(1), vp(32), 1, 64, 64, 3, None) == -5
    assert L.favor_orf_gaussians_seeded(u(1), vp(32), vp(0), 1, 64, 64, None) == -1
    assert L.favor_orf_gaussians_seeded(u(1), vp(32), vp(40), 1, 64, 64, None) == -2
    assert L.favor_orf_gaussians_seeded(u(1), vp(32), vp(48), 1, -1, 64, None) == -3
    assert L.favor_philox4x64(u(1), u(0), u(4), vp(0), None) == -1
    assert L.favor_philox4x64(u(1), u(0), u(4), vp(8), None) == -2
    assert L.favor_philox4x64(u(1), u(0), u(0), vp(16), None) == -3


def test_backward_validation_rejects_before_any_cuda_call():
    vp = ctypes.c_void_p
    L = F.lib()

    def call(**over):
        a = dict(q=16, k=32, v=48, om=64, do=80, dq=96, dk=112, dv=128, B=1, H=1, L_=8, d=64, M=64, kind=0)
        a.update(over)
        return L.favor_attention_backward_f32(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["om"]), vp(a["do"]),
                                              vp(a["dq"]), vp(a["dk"]), vp(a["dv"]), a["B"], a["H"], a["L_"],
                                              a["d"], a["M"], a["kind"], 0, None)
    assert call(do=0) == -1 and call(dk=0) == -1
    assert call(dv=136) == -2 and call(q=20) == -2
    assert call(L_=0) == -3
    assert call(kind=2) == -4
    assert call(d=65) == -5 and call(M=513) == -5
