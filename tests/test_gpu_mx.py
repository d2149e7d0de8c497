"""MXFP8 quantiser on the GPU (moe_mx_quantize) against the oracle's OCP MX quantiser:
E4M3 codes and E8M0 scale bytes must be bit-exact, rowwise and colwise, with ragged
segments (partial 32-row blocks, empty segments)."""
import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib

pytestmark = pytest.mark.gpu


def unchunk_rowwise(sf, seg_off, C):
    """Per-segment [cnt, C/32] scale bytes from the chunked layout."""
    out = []
    tile = 0
    for e in range(len(seg_off) - 1):
        cnt = seg_off[e + 1] - seg_off[e]
        p = np.arange(cnt)[:, None]
        b = np.arange(C // 32)[None, :]
        chunk = (tile + p // 128) * (C // 128) + b // 4
        idx = chunk * 512 + 16 * (p % 32) + 4 * ((p % 128) // 32) + b % 4
        out.append(sf[idx])
        tile += (cnt + 127) // 128
    return out


def unchunk_colwise(sf, seg_off, C):
    """Per-segment [ceil(cnt/32), C] scale bytes from the chunked layout."""
    out = []
    tile = 0
    for e in range(len(seg_off) - 1):
        cnt = seg_off[e + 1] - seg_off[e]
        p0 = 32 * np.arange((cnt + 31) // 32)[:, None]
        c = np.arange(C)[None, :]
        chunk = (tile + p0 // 128) * (C // 128) + c // 128
        idx = chunk * 512 + 16 * (c % 32) + 4 * ((c % 128) // 32) + (p0 % 128) // 32
        out.append(sf[idx])
        tile += (cnt + 127) // 128
    return out


def make_x(R, C, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(R, C, generator=g) * torch.exp(torch.randn(R, 1, generator=g) * 3)
    x[::17] = 0.0                                    # all-zero rows (all-zero row blocks)
    x[3, 5] = -0.0
    if R > 40:
        x[40, :64] = 1e30                            # huge values: large shared exponent
        x[41, 7] = 1e-30                             # tiny value in a normal block
    x[:, 127] *= 300.0                               # values that saturate after scaling
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("C", [128, 384])
@pytest.mark.parametrize("colwise", [False, True])
@pytest.mark.parametrize("counts", [[300], [128, 0, 77, 256, 1, 33], [0, 0, 500], [40] * 9])
def test_mx_quantize_bit_exact(cuda_lib, counts, colwise, C):
    seg_off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    R = int(seg_off[-1])
    E = len(counts)
    x = make_x(R, C, seed=R + E)
    codes = torch.full((R, C), 0xAB, dtype=torch.uint8, device="cuda")
    nsf = lib.moe_mx_scale_bytes(R, C, E)
    sf = torch.full((nsf,), 0xCD, dtype=torch.uint8, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    lib.moe_mx_quantize(x.cuda(), torch.tensor(seg_off, dtype=torch.int32, device="cuda"), colwise,
                        codes, sf, ws)
    torch.cuda.synchronize()
    got_codes = codes.cpu().numpy()
    got_sf = sf.cpu().numpy()
    X = x.double().numpy()
    unchunk = unchunk_colwise if colwise else unchunk_rowwise
    got_sfs = unchunk(got_sf, seg_off, C)
    for e in range(E):
        r0, r1 = seg_off[e], seg_off[e + 1]
        if r1 == r0:
            continue
        ref_codes, ref_sf, _ = oracle.mx_quantize(X[r0:r1], axis=0 if colwise else 1)
        assert np.array_equal(got_codes[r0:r1], ref_codes), ("codes", e)
        assert np.array_equal(got_sfs[e], ref_sf), ("scales", e)
    if colwise:
        # slots of each segment's last chunk past its last 32-row block hold 0 (2^-127)
        tile = 0
        for e in range(E):
            cnt = int(seg_off[e + 1] - seg_off[e])
            if cnt:
                last = (cnt - 1) // 32
                c = np.arange(C)
                chunk = (tile + last // 4) * (C // 128) + c // 128
                for b in range(last % 4 + 1, 4):
                    idx = chunk * 512 + 16 * (c % 32) + 4 * ((c % 128) // 32) + b
                    assert np.all(got_sf[idx] == 0), ("pad", e, b)
            tile += (cnt + 127) // 128


def test_mx_quantize_rejects_bad_shapes(cuda_lib):
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    x = torch.zeros(10, 100, dtype=torch.bfloat16, device="cuda")       # cols % 128 != 0
    off = torch.tensor([0, 10], dtype=torch.int32, device="cuda")
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.MoEError) as ei:
        lib.moe_mx_quantize(x, off, False, buf, buf, ws)
    assert ei.value.status == lib.MOE_EINVAL
