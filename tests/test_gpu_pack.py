"""The packed expert-weight layout: 128 x 64 tiles with the 128-byte swizzle."""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu


def tiled_index(n, k, k_blocks):
    """Element index of (row n, column k) in the tiled layout, written out
    from the layout's definition: tile (n // 128, k // 64) in row-block-major
    order, 128 rows of 64 elements per tile, the 16-byte chunk c of row r
    stored at chunk c XOR (r mod 8)."""
    blk = (n // 128) * k_blocks + (k // 64)
    r, c = n % 128, k % 64
    return blk * 8192 + r * 64 + (((c // 8) ^ (r % 8)) * 8) + (c % 8)


@pytest.mark.parametrize("E,d,f", [(2, 128, 256), (3, 80, 48), (1, 192, 64)])
def test_pack_layout(E, d, f):
    dv = dev()
    W1 = synth.normal_bf16((E, d, f), 1, synth.STREAM_W1, 1.0, dv)
    W3 = synth.normal_bf16((E, d, f), 1, synth.STREAM_W3, 1.0, dv)
    W2 = synth.normal_bf16((E, f, d), 1, synth.STREAM_W2, 1.0, dv)
    dims = abi.Dims(4, d, f, E, 1)
    W13p, W2p = abi.pack_weights(dims, W1, W3, W2)
    torch.cuda.synchronize()
    p13 = W13p.view(torch.int16).cpu().numpy()
    p2 = W2p.view(torch.int16).cpu().numpy()
    w1 = W1.view(torch.int16).cpu().numpy()
    w3 = W3.view(torch.int16).cpu().numpy()
    w2 = W2.view(torch.int16).cpu().numpy()
    kb13, nb13 = (d + 63) // 64, (2 * f + 127) // 128
    kb2, nb2 = (f + 63) // 64, (d + 127) // 128
    assert p13.size == E * nb13 * kb13 * 8192 and p2.size == E * nb2 * kb2 * 8192
    seen13 = np.zeros(p13.size, dtype=bool)
    seen2 = np.zeros(p2.size, dtype=bool)
    for e in range(E):
        base = e * nb13 * kb13 * 8192
        for n in range(2 * f):
            b, j = divmod(n, 32)
            src = w1 if j < 16 else w3
            col = 16 * b + (j % 16)
            ks = np.arange(d)
            ii = base + np.array([tiled_index(n, k, kb13) for k in ks])
            assert np.array_equal(p13[ii], src[e, ks, col])
            seen13[ii] = True
        base = e * nb2 * kb2 * 8192
        for n in range(d):
            ks = np.arange(f)
            ii = base + np.array([tiled_index(n, k, kb2) for k in ks])
            assert np.array_equal(p2[ii], w2[e, ks, n])
            seen2[ii] = True
    assert np.all(p13[~seen13] == 0) and np.all(p2[~seen2] == 0)   # padding is zero
