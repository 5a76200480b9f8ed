"""GPU parity of csa_quantize_mxfp4: packed E2M1 codes and E8M0 block scales
bit-exact against the oracle (both sides decide every code exactly)."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
from oracle.formats import E2M1_GRID, mxfp4_quantize

pytestmark = pytest.mark.gpu


def _gpu(x):
    rows, cols = x.shape
    xd = torch.from_numpy(x).cuda()
    codes = torch.full((rows, cols // 2), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((rows, cols // 32), 0xAB, dtype=torch.uint8, device="cuda")
    csa.quantize_mxfp4(xd, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _compare(x):
    gc, gs = _gpu(x)
    rc, rs = mxfp4_quantize(x)
    bad = np.argwhere(gs != rs)
    assert bad.size == 0, f"scales differ at {bad[:5].tolist()}"
    bad = np.argwhere(gc != rc)
    assert bad.size == 0, f"codes differ at {bad[:5].tolist()}: gpu {gc[tuple(bad[0])]:#x} oracle {rc[tuple(bad[0])]:#x}"


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 96), (300, 64), (4096, 256)])
def test_random_wide_range(rows, cols):
    rng = np.random.default_rng(rows * 1000 + cols)
    x = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-60, 60, (rows, cols // 32)).repeat(32, axis=1))
    _compare(x.astype(np.float32))


def test_ties_zeros_and_extremes():
    """Exact ties of the E2M1 grid after scaling, -0, zero blocks, subnormal
    and near-overflow blocks, saturation between 6 and 8."""
    g = np.asarray(E2M1_GRID)
    mids = (g[:-1] + g[1:]) / 2
    rows = []
    for X in (-127, -20, -1, 0, 3, 100, 125):
        blk = np.zeros(32)
        blk[0] = 7.5                        # max: floor(log2 7.5) = 2 -> this block's X
        blk[1:8] = mids
        blk[8:15] = -mids
        blk[15:23] = g
        blk[23] = -0.0
        blk[24] = 6.9
        blk[25] = -7.9
        blk[26:32] = [0.1, -0.1, 0.26, -0.24, 5.0, -3.5]
        rows.append(blk * 2.0 ** X)
    zero = np.zeros(32)
    neg0 = -np.zeros(32)
    sub = np.full(32, 1e-42) * np.sign(np.arange(32) - 15.5)
    x = np.stack(rows + [zero, neg0, sub]).astype(np.float32)
    x = np.concatenate([x, x[::-1]], axis=1)   # 64 columns, two blocks per row
    _compare(x)


def test_rows_zero_is_noop():
    x = torch.empty((0, 64), device="cuda")
    codes = torch.empty((0, 32), dtype=torch.uint8, device="cuda")
    scales = torch.empty((0, 2), dtype=torch.uint8, device="cuda")
    csa.quantize_mxfp4(x, codes, scales)
    torch.cuda.synchronize()
