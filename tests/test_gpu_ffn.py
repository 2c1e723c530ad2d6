"""Expert FFN parity: the grouped tcgen05 GEMMs against the fp64 oracle FFN.

Shapes cover both tile orientations (weight rows on the MMA M side for small
groups, token rows for large ones), empty groups, groups smaller than one
tile, ragged tails, split reductions and the packed-weight layout.
"""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O
from tests.gpu_util import Y_MAX_ABS, Y_MIRROR_MAX_ABS, Y_MIRROR_REL_L2, Y_REL_L2, assert_close_y, dev, f64

pytestmark = pytest.mark.gpu


def _run(T, d, f, E, K, skew=0.0, seed=11, w_std=0.05):
    dv = dev()
    wts = None if skew == 0 else torch.tensor([(r + 1.0) ** -skew for r in range(E)])
    idx = synth.distinct_choices(T, E, K, seed=seed, weights=wts).to(dv)
    x = synth.normal_bf16((T, d), seed, synth.STREAM_X, 1.0, dv)
    W1 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W1, w_std, dv)
    W3 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W3, w_std, dv)
    W2 = synth.normal_bf16((E, f, d), seed, synth.STREAM_W2, w_std, dv)
    dims = abi.Dims(T, d, f, E, K)
    ws = abi.alloc_workspace(dims)
    W13p, W2p = abi.pack_weights(dims, W1, W3, W2)
    i32 = dict(dtype=torch.int32, device=dv)
    A = T * K
    counts, kept, offsets = torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32)
    inv, src = torch.empty(T, K, **i32), torch.empty(A, **i32)
    xp = torch.zeros(A, d, dtype=torch.bfloat16, device=dv)
    abi.moe_permute(dims, idx, x, counts, kept, offsets, inv, src, xp, None, ws)
    h = torch.zeros(A, f, dtype=torch.bfloat16, device=dv)
    yp = torch.zeros(A, d, dtype=torch.float32, device=dv)
    abi.moe_expert_ffn(dims, xp, offsets, W13p, W2p, h, yp, ws)
    torch.cuda.synchronize()
    st, detail = abi.moe_get_device_status(ws)
    assert st == abi.MOE_OK, f"device wait ran out (code {detail})"
    # oracle: its own dispatch of the same idx, then the FFN per expert
    o = O.dispatch(idx.cpu().numpy(), E, None)
    x64 = f64(x)
    W1h, W3h, W2h = f64(W1), f64(W3), f64(W2)
    off, srco = o["offsets"], o["src"]
    Y = np.zeros((A, d))
    Yr = np.zeros((A, d))
    H = np.zeros((A, f))
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        Xe = x64[srco[r0:r1]]
        g, u = Xe @ W1h[e], Xe @ W3h[e]
        H[r0:r1] = O.silu(g) * u
        Y[r0:r1] = O.swiglu_ffn(Xe, W1h[e], W3h[e], W2h[e])
        Yr[r0:r1] = O.swiglu_ffn(Xe, W1h[e], W3h[e], W2h[e], h_round=O.bf16_round)
    return dict(h=f64(h), yp=f64(yp), H=H, Y=Y, Yr=Yr, n=int(off[-1]), offsets=off)


@pytest.mark.parametrize("T,d,f,E,K,skew", [
    (64, 128, 256, 8, 2, 0.0),        # small groups: weight-major tiles
    (256, 512, 512, 8, 2, 0.0),       # decode-like CTA pairs, no split
    (300, 256, 192, 16, 4, 1.0),      # ragged, some groups tiny
    (2000, 256, 320, 4, 2, 0.0),      # large groups: token-major tiles, ragged m tail
    (1500, 384, 704, 12, 3, 1.5),     # skewed: empty groups possible
    (130, 128, 128, 1, 1, 0.0),       # single expert = dense FFN
    (2100, 512, 256, 4, 2, 0.0),      # mean group >= 1024 rows, widths x256: CTA-pair tiles, ragged tail
    (6200, 256, 384, 6, 1, 1.5),      # CTA-pair tiles with skewed groups (the smallest may be tiny)
    (256, 256, 1024, 8, 2, 1.5),      # decode-like CTA pairs, 4-way split, one group > 128 rows (token-major)
    (256, 256, 1408, 8, 2, 0.0),      # decode-like CTA pairs, 6-way split of 22 k-blocks (4, 4, 4, 4, 4, 2)
    (256, 384, 1536, 8, 2, 1.5),      # single-CTA, 4-way split, one group > 128 rows (token-major)
    (256, 128, 1024, 8, 2, 0.0),      # single-CTA, 8-way split
    (512, 512, 512, 16, 4, 1.5),      # CTA pairs, both tile queues: skewed groups above and below 128 rows
    (256, 512, 1664, 8, 2, 1.5),      # CTA pairs, both queues, down split of 26 k-blocks as 7,7,7,5 (odd two-k-block tails)
    (40, 256, 1024, 8, 2, 0.0),       # CTA pairs, groups under 16 rows, 4-way split
    (600, 256, 256, 16, 4, 1.2),      # CTA pairs, weight- and token-major groups in one launch
    (512, 256, 2560, 64, 4, 0.0),     # CTA pairs, gate/up tiles of two 256-row weight sub-tiles, 8-way split
    (1024, 1024, 1024, 256, 8, 1.1),  # CTA pairs, two weight sub-tiles in both phases, skewed small groups
    (2000, 256, 256, 1, 1, 0.0),      # one expert (dense FFN) on CTA-pair token-major tiles, ragged tail
    (1, 256, 512, 8, 2, 0.0),         # a single token: two one-row groups on CTA-pair weight-major tiles
    (1024, 256, 512, 16, 4, 1.2),     # CTA pairs, both queues: 128-row pair tiles for the last chunks of groups of 321-893 rows
    (1024, 256, 512, 8, 2, 1.5),      # CTA pairs, both queues: 128-row last chunks of 17 and 43 rows
    # mid-sized groups: single-CTA token-major tiles with ragged 128-row tails
    (3000, 256, 384, 12, 2, 0.5),
    (4000, 512, 256, 8, 1, 1.2),      # skewed: groups from tens to ~1500 rows
    (700, 256, 768, 2, 1, 0.0),
    # CTA-pair token-major tiles: exact 256-row tiles, and skewed groups with one under a tile
    (2048, 256, 256, 2, 1, 0.0),
    (5000, 256, 256, 2, 1, 0.0),
    (9000, 256, 512, 4, 1, 1.0),
])
def test_expert_ffn_vs_oracle(T, d, f, E, K, skew):
    # weight scale shrinks with the width so |y| stays O(1), the scale the
    # max-abs bound was derived for
    r = _run(T, d, f, E, K, skew, w_std=0.05 * min(1.0, (256.0 / d) ** 0.5))
    n = r["n"]
    # H: bf16 rounding of an fp32 value close to the fp64 one
    Hg, H = r["h"][:n], r["H"][:n]
    assert np.all(np.abs(Hg - H) <= np.abs(H) * 2.0 ** -8 + 1e-4)
    assert_close_y(r["yp"][:n], r["Y"][:n], Y_MAX_ABS, Y_REL_L2, "y_perm")
    assert_close_y(r["yp"][:n], r["Yr"][:n], Y_MIRROR_MAX_ABS, Y_MIRROR_REL_L2, "y_perm (H rounded)")


# Explicit group sizes on the edges of the epilogue's and the tiles' cases:
# 32-row slabs that are exactly full (staged TMA stores) or not (direct
# stores), last chunks of 1, 33, 44 and 128 rows, groups of 129 and 257 rows,
# empty groups; each case checks that the kernel it means to reach is the one
# launched.
@pytest.mark.parametrize("d,f,sizes,kernel", [
    # single-CTA token-major tiles (mean group 500 rows): slabs of 128, 160 (the last exactly 32), 33, 1, 118 rows
    (256, 384, [128, 160, 0, 33, 1, 2678], "grouped_gemm_kernel"),
    # CTA pairs with weight-major tiles enabled: 128-row last chunks of 1, 128 and 44 rows, a 129-row group
    (256, 256, [257, 384, 129, 0, 31, 128, 300, 100], "grouped_gemm_2sm_kernel"),
    # CTA pairs, groups of >= 1024 rows on average: 256-row last chunks of 33 and 127 rows
    (256, 256, [1057, 2175], "grouped_gemm_2sm_kernel"),
    # CTA pairs with a 4-way split of the down projection and one 300-row group (256 + a 44-row chunk)
    (256, 1024, [300, 40, 40, 40, 40, 40, 40, 40], "grouped_gemm_2sm_kernel"),
])
def test_expert_ffn_explicit_groups(d, f, sizes, kernel):
    dv = dev()
    E, T = len(sizes), sum(sizes)
    dims = abi.Dims(T, d, f, E, 1)
    assert abi.moe_ffn_kernel(dims) == kernel
    seed = 21
    w_std = 0.05 * min(1.0, (256.0 / d) ** 0.5)
    xp = synth.normal_bf16((T, d), seed, synth.STREAM_X, 1.0, dv)
    W1 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W1, w_std, dv)
    W3 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W3, w_std, dv)
    W2 = synth.normal_bf16((E, f, d), seed, synth.STREAM_W2, w_std, dv)
    W13p, W2p = abi.pack_weights(dims, W1, W3, W2)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    offsets = torch.from_numpy(off).to(dv)
    ws = abi.alloc_workspace(dims)
    h = torch.zeros(T, f, dtype=torch.bfloat16, device=dv)
    yp = torch.zeros(T, d, dtype=torch.float32, device=dv)
    abi.moe_expert_ffn(dims, xp, offsets, W13p, W2p, h, yp, ws)
    torch.cuda.synchronize()
    st, detail = abi.moe_get_device_status(ws)
    assert st == abi.MOE_OK, f"device wait ran out (code {detail})"
    x64, W1h, W3h, W2h = f64(xp), f64(W1), f64(W3), f64(W2)
    Y, Yr = np.zeros((T, d)), np.zeros((T, d))
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 > r0:
            Y[r0:r1] = O.swiglu_ffn(x64[r0:r1], W1h[e], W3h[e], W2h[e])
            Yr[r0:r1] = O.swiglu_ffn(x64[r0:r1], W1h[e], W3h[e], W2h[e], h_round=O.bf16_round)
    assert_close_y(f64(yp), Y, Y_MAX_ABS, Y_REL_L2, "y_perm")
    assert_close_y(f64(yp), Yr, Y_MIRROR_MAX_ABS, Y_MIRROR_REL_L2, "y_perm (H rounded)")
