"""The 8-bit shared cache on the GPU.  Quantisation codes and scales are
compared with the oracle's bit for bit (both sides decide them in fp32 with
IEEE division and round-half-even); decode over the 8-bit cache is compared
with the oracle's decode over the dequantised values, at the bf16 bar."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.util import assert_close

pytestmark = pytest.mark.gpu
BF, F32 = torch.bfloat16, torch.float32


def _unpack(rows_u8, Hkv, D):
    """uint8 cache rows -> (codes int8 [rows, Hkv, D], scales float32 [rows, Hkv])."""
    a = rows_u8.cpu().numpy()
    codes = a[:, :Hkv * D].view(np.int8).reshape(-1, Hkv, D)
    scales = np.ascontiguousarray(a[:, Hkv * D:Hkv * D + 4 * Hkv]).view(np.float32).reshape(-1, Hkv)
    return codes, scales


@pytest.mark.parametrize("dtype,Hkv,D", [(BF, 8, 128), (BF, 1, 128), (F32, 2, 64), (BF, 4, 64)])
def test_quantize_matches_oracle_bit_for_bit(cuda_lib, dtype, Hkv, D):
    n = 300
    k = wl.normal((n, Hkv, D), 2500 + D, dtype)
    v = wl.normal((n, Hkv, D), 2501 + D, dtype) * 7.0
    k[5, 0] = 0                       # an all-zero head row: scale 0, codes 0
    v[9, -1, 3] = 1000.0              # one large value dominating its row
    kq, vq = cuda_lib.kv_quantize_i8(k.cuda(), v.cuda())
    for name, x, rows in (("k", k, kq), ("v", v, vq)):
        codes, scales = _unpack(rows, Hkv, D)
        rc, rs = oracle.quantize_kv_i8(x)
        np.testing.assert_array_equal(codes, rc, err_msg=f"{name} codes")
        np.testing.assert_array_equal(scales.view(np.uint32), rs.view(np.uint32), err_msg=f"{name} scales")


def test_quantize_scatter_touches_only_addressed_rows(cuda_lib):
    Hkv, D, rows = 8, 128, 64
    k = wl.normal((4, Hkv, D), 2600, BF).cuda()
    v = wl.normal((4, Hkv, D), 2601, BF).cuda()
    rb = cuda_lib.kv_i8_row_bytes(Hkv, D)
    kq = torch.full((rows, rb), 0xA5, dtype=torch.uint8, device="cuda")
    vq = torch.full((rows, rb), 0x5A, dtype=torch.uint8, device="cuda")
    dst = torch.tensor([3, 40, 17, 63], dtype=torch.int64, device="cuda")
    cuda_lib.kv_quantize_i8(k, v, kq, vq, dst_rows=dst)
    dense_k, dense_v = cuda_lib.kv_quantize_i8(k, v)
    untouched = sorted(set(range(rows)) - {3, 40, 17, 63})
    assert bool((kq[untouched] == 0xA5).all()) and bool((vq[untouched] == 0x5A).all())
    for i, r in enumerate([3, 40, 17, 63]):
        assert torch.equal(kq[r], dense_k[i]) and torch.equal(vq[r], dense_v[i])


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 1), (8, 2), (16, 2), (4, 4)])
def test_decode_i8_matches_oracle_on_dequantised_cache(cuda_lib, Hq, Hkv):
    D = 128
    lens = [1, 17, 300, 1000, 2051, 128]
    B = len(lens)
    starts = np.cumsum([0] + [l + 5 for l in lens[:-1]])
    rows = int(starts[-1] + lens[-1] + 3)
    k = wl.normal((rows, Hkv, D), 2700, BF)
    v = wl.normal((rows, Hkv, D), 2701, BF)
    q = wl.normal((B, Hq, D), 2702, BF)
    kq, vq = cuda_lib.kv_quantize_i8(k.cuda(), v.cuda())
    ss = torch.tensor(starts, dtype=torch.int64, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = cuda_lib.cross_decode_i8(q.cuda(), kq, vq, Hkv, ss, sl, max(lens), want_lse=True)
    ck, sk = oracle.quantize_kv_i8(k)
    cv, sv = oracle.quantize_kv_i8(v)
    ro, rlse = oracle.cross_decode(q, oracle.dequantize_kv_i8(ck, sk), oracle.dequantize_kv_i8(cv, sv), starts, lens)
    assert_close(o, ro, BF, "o")
    assert_close(lse, rlse, BF, "lse", max_abs=1e-3, rel_l2=1e-4)


def test_decode_i8_long_ragged_close_to_bf16(cuda_lib):
    # 64K-token sequences: the 8-bit path matches the oracle on its own cache,
    # and the quantisation moves the output only slightly from the bf16 path
    Hq, Hkv, D = 32, 8, 128
    lens = [65536, 40000, 70001]
    B = len(lens)
    starts = np.cumsum([0] + lens[:-1])
    rows = int(sum(lens))
    k = wl.normal((rows, Hkv, D), 2800, BF, "cuda")
    v = wl.normal((rows, Hkv, D), 2801, BF, "cuda")
    q = wl.normal((B, Hq, D), 2802, BF)
    kq, vq = cuda_lib.kv_quantize_i8(k, v)
    ss = torch.tensor(starts, dtype=torch.int64, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o8 = cuda_lib.cross_decode_i8(q.cuda(), kq, vq, Hkv, ss, sl, max(lens))
    o16 = cuda_lib.cross_decode(q.cuda(), k, v, ss, sl, max(lens))
    ck, sk = _unpack(kq, Hkv, D)
    cv, sv = _unpack(vq, Hkv, D)
    ro, _ = oracle.cross_decode(q, oracle.dequantize_kv_i8(ck, sk), oracle.dequantize_kv_i8(cv, sv), starts, lens)
    assert_close(o8, ro, BF, "o (8-bit cache)")
    assert_close(o8, o16.float().cpu().numpy(), BF, "8-bit vs bf16 cache", max_abs=2e-2, rel_l2=5e-2)
