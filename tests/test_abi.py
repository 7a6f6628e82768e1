"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/sattn.h, and rejects bad arguments before any CUDA call."""

import ctypes
import os
import re

import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sattn.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
BF16, FP16, NVFP4, QTOK = 0, 0x100, 1, 0x200


@pytest.fixture(scope="module")
def L():
    sattn_build.build()
    return sattn.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sattn_[a-z_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert set(names) == set(sattn.EXPORTS), names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in range(5):
        assert L.sattn_status_string(code).startswith(b"SATTN_")
    assert b"unknown" in L.sattn_status_string(99)


def test_nvfp4_workspace_layout(L):
    lay = sattn.workspace_layout(1, 12, 32760, 128, mode="nvfp4")
    bh, n, d = 12, 32760, 128
    assert lay["nv"] == 32768 and lay["nblk"] == 256
    assert lay["k8"] - lay["q8"] >= bh * n * d // 2
    assert lay["sk"] - lay["sq"] >= bh * 256 * 2 * 512
    assert lay["mu"] - lay["sv"] >= bh * 256 * 1024
    assert lay["total"] == L.sattn_workspace_bytes(1, 12, 32760, 128, NVFP4)


def test_mxfp4_mode_shares_the_nvfp4_layout(L):
    for shape in ((1, 12, 32760, 128), (2, 3, 300, 64)):
        assert sattn.workspace_layout(*shape, mode="mxfp4") == sattn.workspace_layout(*shape, mode="nvfp4")
    assert L.sattn_workspace_bytes(1, 2, 256, 64, 2) == L.sattn_workspace_bytes(1, 2, 256, 64, NVFP4) > 0
    assert L.sattn_workspace_bytes(1, 2, 256, 64, 2 | 0x200) == 0   # per-token Q is I8QK_F8PV only
    p = ctypes.c_void_p(1 << 20)
    assert L.sattn_quantize(p, p, p, 1, 2, 256, 64, 2 | 0x200, ctypes.c_void_p(1 << 21), 1 << 30,
                            None) == UNSUPPORTED


def test_workspace_bytes_and_layout(L):
    assert L.sattn_workspace_bytes(1, 2, 256, 64, FP16) > 0
    assert L.sattn_workspace_bytes(1, 2, 0, 64, BF16) == 0       # N < 1
    assert L.sattn_workspace_bytes(1, 2, 256, 96, BF16) == 0      # d unsupported
    assert L.sattn_workspace_bytes(1, 2, 256, 64, 7) == 0         # unknown mode
    lay = sattn.workspace_layout(1, 12, 32760, 128)
    assert lay["nblk"] == 256 and lay["nv"] == 32768
    bh, n, d = 12, 32760, 128
    assert lay["k8"] - lay["q8"] >= bh * n * d
    assert lay["sk"] - lay["sq"] >= bh * 256 * 4
    assert lay["total"] >= lay["vmax"] + bh * d * 4
    for key in ("q8", "k8", "vt8", "sq", "sk", "sv", "mu", "ksum"):
        assert lay[key] % 256 == 0, key
    assert lay["total"] == L.sattn_workspace_bytes(1, 12, 32760, 128, BF16)


def test_invalid_arguments_rejected_before_launch(L):
    p = ctypes.c_void_p(1 << 20)          # never dereferenced: validation fails first
    mis = ctypes.c_void_p((1 << 20) + 8)
    ws = ctypes.c_void_p(1 << 21)
    q = L.sattn_quantize
    assert q(p, p, p, 1, 2, 256, 96, BF16, ws, 1 << 30, None) == UNSUPPORTED
    assert q(p, p, p, 1, 2, 0, 64, BF16, ws, 1 << 30, None) == INVALID
    assert q(p, p, p, 0, 2, 256, 64, BF16, ws, 1 << 30, None) == INVALID
    assert q(p, p, p, 1, 2, 256, 64, 5, ws, 1 << 30, None) == INVALID
    assert q(None, p, p, 1, 2, 256, 64, BF16, ws, 1 << 30, None) == INVALID
    assert q(mis, p, p, 1, 2, 256, 64, BF16, ws, 1 << 30, None) == INVALID
    assert q(p, p, p, 1, 2, 256, 64, BF16, None, 1 << 30, None) == WORKSPACE
    assert q(p, p, p, 1, 2, 256, 64, BF16, ctypes.c_void_p((1 << 21) + 16), 1 << 30, None) == WORKSPACE
    assert q(p, p, p, 1, 2, 256, 64, BF16, ws, 16, None) == WORKSPACE
    assert q(p, p, p, 1, 2, 256, 64, NVFP4, ws, 16, None) == WORKSPACE       # rejected before any launch
    assert q(p, p, p, 1, 2, 256, 96, NVFP4, ws, 1 << 30, None) == UNSUPPORTED
    assert q(p, p, p, 1 << 16, 1, 256, 64, BF16, ws, 1 << 40, None) == UNSUPPORTED   # B*H too large
    f = L.sattn_fwd_quantized
    assert f(ws, 1 << 30, None, 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID
    assert f(ws, 16, p, 1, 2, 256, 64, 0, 0.0, BF16, None) == WORKSPACE
    # out overlapping the workspace
    assert f(ws, 1 << 30, ctypes.c_void_p((1 << 21) + 1024), 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID
    g = L.sattn_fwd
    assert g(p, p, p, None, 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID
    assert g(p, p, p, p, 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID      # out aliases q
    assert g(p, p, p, mis, 1, 2, 256, 128, 0, 0.0, 0x800, None) == INVALID   # unknown flag
    assert g(p, p, p, p, 1, 2, 256, 64, 0, 0.0, NVFP4 | 0x400, None) == UNSUPPORTED   # per-token P: I8QK_F8PV only


def test_fwd_host_rejects_bad_arguments_before_any_cuda_call(L):
    p = ctypes.c_void_p(1 << 20)          # host addresses, never dereferenced: validation fails first
    o = ctypes.c_void_p(1 << 40)
    h = L.sattn_fwd_host
    assert h(None, p, p, o, 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID
    assert h(p, p, p, None, 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID
    assert h(p, p, p, p, 1, 2, 256, 64, 0, 0.0, BF16, None) == INVALID      # out aliases q
    assert h(p, p, p, o, 1, 2, 256, 96, 0, 0.0, BF16, None) == UNSUPPORTED
    assert h(p, p, p, o, 1, 2, 0, 64, 0, 0.0, BF16, None) == INVALID
    assert h(p, p, p, o, 1, 2, 256, 64, 0, 0.0, 0x800, None) == INVALID     # unknown flag
    assert h(p, p, p, o, 1, 2, 256, 64, 0, 0.0, NVFP4 | QTOK, None) == UNSUPPORTED
    assert h(p, p, p, o, 1, 2, 256, 64, 0, 0.0, NVFP4 | 0x400, None) == UNSUPPORTED   # per-token P


def test_fwd_host_binding_rejects_device_or_mismatched_tensors():
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sattn.fwd_host(q, q, q[:, :1])
    with pytest.raises(TypeError):
        sattn.fwd_host(q, q, q.half())
    with pytest.raises(ValueError):
        sattn.fwd_host(q, q, q, out=torch.zeros(1, 2, 64, 32, dtype=torch.bfloat16))


def test_lazy_tau_of_binding_matches_header():
    m = re.search(r"#define\s+SATTN_I8F8_LAZY_TAU\s+([0-9.]+)f?", open(HEADER).read())
    assert m and float(m.group(1)) == sattn.I8F8_LAZY_TAU


def test_per_token_q_layout(L):
    blk = sattn.workspace_layout(2, 3, 1000, 128)
    tok = sattn.workspace_layout(2, 3, 1000, 128, q_per_token=True)
    assert tok["sk"] - tok["sq"] >= 6 * 1000 * 4 > blk["sk"] - blk["sq"]
    assert tok["total"] == L.sattn_workspace_bytes(2, 3, 1000, 128, QTOK)
    assert L.sattn_workspace_bytes(2, 3, 1000, 128, NVFP4 | QTOK) == 0
    assert L.sattn_workspace_bytes(2, 3, 1000, 128, 0x800) == 0          # unknown flag
    # per-token P changes the attention, not the quantised operands
    assert L.sattn_workspace_bytes(2, 3, 1000, 128, 0x400) == L.sattn_workspace_bytes(2, 3, 1000, 128, 0)
    assert L.sattn_workspace_bytes(2, 3, 1000, 128, NVFP4 | 0x400) == 0


def test_scores_accessor_validates_before_any_cuda_call(L):
    ws = ctypes.c_void_p(1 << 21)
    out = ctypes.c_void_p(1 << 22)
    f = L.sattn_debug_scores
    f.argtypes = [ctypes.c_void_p, ctypes.c_size_t] + [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_void_p]
    assert f(ws, 16, 1, 2, 256, 64, NVFP4, out, None) == WORKSPACE
    assert f(ws, 1 << 30, 1, 2, 256, 64, 2 | QTOK, out, None) == UNSUPPORTED    # MXFP4 with per-token Q
    assert f(ws, 1 << 30, 1, 2, 256, 64, BF16, None, None) == INVALID
    assert f(ws, 1 << 30, 1, 2, 256, 64, BF16, ctypes.c_void_p((1 << 22) + 4), None) == INVALID
    assert f(ws, 16, 1, 2, 256, 64, BF16, out, None) == WORKSPACE
    assert f(None, 1 << 30, 1, 2, 256, 64, BF16, out, None) == WORKSPACE
    assert f(ws, 1 << 30, 1, 2, 256, 96, BF16, out, None) == UNSUPPORTED


def test_block_sparse_entry_points_validate_before_any_cuda_call(L):
    p = ctypes.c_void_p(1 << 20)
    o = ctypes.c_void_p(1 << 40)
    m = ctypes.c_void_p(1 << 30)
    f = L.sattn_fwd_sparse
    assert f(p, p, p, o, 1, 2, 1000, 128, 0, 0.0, BF16, None, None) == INVALID       # no mask
    assert f(p, p, p, o, 1, 1, 262145, 64, 0, 0.0, BF16, m, None) == UNSUPPORTED     # more than 2048 key tiles
    assert f(p, p, p, o, 1, 2, 1000, 96, 0, 0.0, BF16, m, None) == UNSUPPORTED       # head dim
    g = L.sattn_fwd_quantized_sparse
    assert g(p, 1 << 30, o, 1, 2, 1000, 128, 0, 0.0, BF16, None, None) == INVALID
    assert g(None, 1 << 30, o, 1, 2, 1000, 128, 0, 0.0, BF16, m, None) == WORKSPACE
