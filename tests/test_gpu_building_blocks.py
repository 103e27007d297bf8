"""GPU checks of the building blocks under the attention kernels, each against
a float64 CPU product: the TMA 128-byte swizzle placement and the four
tcgen05 operand forms the kernels use (test-only diagnostics library)."""
import ctypes
import os

import numpy as np
import pytest

from synth import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DIAG = os.path.join(ROOT, "exact_attention_156_b200", "libattn156_diag.so")


@pytest.fixture(scope="module")
def diag():
    lib = ctypes.CDLL(DIAG)
    vp = ctypes.c_void_p
    lib.attn_diag_mma.argtypes = [ctypes.c_int, vp, vp, vp, vp]
    lib.attn_diag_tma.argtypes = [vp, vp, vp]
    return lib


def _bf16_matrix(seed):
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal((128, 128)).astype(np.float32))


def _dev(bits):
    import torch
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _swz(row, col):
    box, chunk = col // 64, (col % 64) // 8
    return box * 16384 + row * 128 + ((chunk ^ (row & 7)) << 4) + (col % 8) * 2


def test_tma_load_uses_the_128_byte_swizzle(diag):
    import torch
    a = _bf16_matrix(1)
    out = torch.zeros(2 * 16384, dtype=torch.uint8, device="cuda")
    assert diag.attn_diag_tma(_dev(a).data_ptr(), out.data_ptr(), None) == 0
    assert diag.attn_diag_error() == 0
    raw = out.cpu().numpy()
    got = np.zeros((128, 128), dtype=np.uint16)
    for r in range(128):
        for c in range(128):
            o = _swz(r, c)
            got[r, c] = raw[o] | (np.uint16(raw[o + 1]) << 8)
    np.testing.assert_array_equal(got, a)


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4, 5, 6, 7])
def test_tcgen05_operand_forms(diag, mode):
    import torch
    a, b = _bf16_matrix(10 + mode), _bf16_matrix(20 + mode)
    A = bf16_bits_to_f32(a).astype(np.float64)
    B = bf16_bits_to_f32(b).astype(np.float64)
    ref = {0: A @ B.T, 1: A @ B, 2: A @ B, 3: A.T @ B}[mode % 4]
    c = torch.zeros(128, 128, dtype=torch.float32, device="cuda")
    assert diag.attn_diag_mma(mode, _dev(a).data_ptr(), _dev(b).data_ptr(), c.data_ptr(), None) == 0
    assert diag.attn_diag_error() == 0
    got = c.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, f"mode {mode}: relative error {err:.3e}"


@pytest.mark.parametrize("mode", [8, 9, 10])
def test_tcgen05_cta_pair_products(diag, mode):
    """One 256 x 128 x 128 product shared by a pair of CTAs (cta_group::2): each CTA
    holds half of A's rows and half of B's rows; mode 10 brings the operands in with
    the pair's TMA loads counted on the even CTA's barrier."""
    import torch
    diag.attn_diag_mma_pair.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p]
    rng = np.random.default_rng(30 + mode)
    a = f32_to_bf16_bits(rng.standard_normal((256, 128)).astype(np.float32))
    b = _bf16_matrix(40 + mode)
    A = bf16_bits_to_f32(a).astype(np.float64)
    B = bf16_bits_to_f32(b).astype(np.float64)
    ref = A @ B if mode == 9 else A @ B.T
    c = torch.zeros(256, 128, dtype=torch.float32, device="cuda")
    assert diag.attn_diag_mma_pair(mode, _dev(a).data_ptr(), _dev(b).data_ptr(), c.data_ptr(), None) == 0
    assert diag.attn_diag_error() == 0
    got = c.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, f"mode {mode}: relative error {err:.3e}"
