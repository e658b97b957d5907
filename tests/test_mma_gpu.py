"""The tensor-core tile (tcgen05 + TMEM) against a host matmul, through the C ABI.

The operand images are built here with the 128-byte swizzle written out
directly: in each 64-column K chunk, row r's eight 16-byte units are stored at
unit index (u XOR r % 8).
"""
import numpy as np
import pytest

from streaming_persistent_sm_b200 import wpk as W


def sw128_image(m16: np.ndarray) -> np.ndarray:
    """[R][K] 16-bit values -> bytes of the chunked, swizzled image."""
    R, K = m16.shape
    assert R % 8 == 0 and K % 64 == 0
    blocks = m16.reshape(R, K // 64, 8, 8)                 # row, chunk, unit, element
    unit = np.arange(8)[None, :] ^ (np.arange(R)[:, None] & 7)
    out = np.empty_like(blocks)
    out[np.arange(R)[:, None], :, unit, :] = blocks.transpose(0, 2, 1, 3)[np.arange(R)[:, None], np.arange(8)[None, :]]
    return np.ascontiguousarray(out.transpose(1, 0, 2, 3)).view(np.uint8).ravel()


def bf16_bits(x: np.ndarray) -> np.ndarray:
    import torch

    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_swizzle_helper_places_units():
    m = np.arange(16 * 64, dtype=np.uint16).reshape(16, 64)
    img = sw128_image(m).view(np.uint16).reshape(16, 64)
    for r in range(16):
        for u in range(8):
            np.testing.assert_array_equal(img[r, (u ^ (r % 8)) * 8:(u ^ (r % 8)) * 8 + 8], m[r, u * 8:u * 8 + 8])


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,two", [(16, 64, False), (48, 512, True), (128, 2048, True), (256, 256, False)])
def test_tcgen05_tile_matches_host(N, K, two):
    import torch

    rng = np.random.default_rng(N * 7 + K)
    a = bf16_bits(rng.standard_normal((128, K)) * 0.02)
    b1 = bf16_bits(rng.standard_normal((N, K)))
    b2 = bf16_bits(rng.standard_normal((N, K)) * 1e-3)
    dev = lambda x: torch.from_numpy(x).cuda()
    A, B1, B2 = dev(sw128_image(a)), dev(sw128_image(b1)), dev(sw128_image(b2))
    D = torch.zeros((128, N), dtype=torch.float32, device="cuda")
    W.wpk_debug_gemm(A.data_ptr(), B1.data_ptr(), B2.data_ptr() if two else 0, D.data_ptr(), K // 64, N, True,
                     torch.cuda.current_stream().cuda_stream)
    ref = bits_to_f64(a) @ (bits_to_f64(b1) + (bits_to_f64(b2) if two else 0)).T
    got = D.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err
