"""GPU parity of the cache-entry encoders against the oracle (bit-exact)."""
import numpy as np
import pytest

from oracle import quant as oq
from oracle import codecs as oc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _rows(seed, n, scales=(1e-3, 1.0, 7.0, 300.0, 1e4)):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 512)).astype(np.float32)
    x *= rng.choice(scales, size=(n, 1)).astype(np.float32)
    # special rows: zeros, signed zeros, tiny subnormals, saturation, ties
    x[0] = 0.0
    x[1] = -0.0
    x[2, :] = np.float32(1e-40)
    x[3, :] = np.float32(1e30)
    x[4, ::2] = 1.0
    x[4, 1::2] = -0.25
    x[5, :16] = np.float32([6, 3, -1.5, 0.25] + [0.75] * 12)
    x[6] = np.float32(2.0 ** -130)
    return x


def _encode(csa, x, fmt, dtype=torch.float32, dim=512):
    src = torch.from_numpy(x).to("cuda").to(dtype)
    nb = {csa.CSA_FMT_FP4_E2M1_E4M3X16: 288, csa.CSA_FMT_FP8_E4M3_UE8M0X32: 528}.get(fmt, dim)
    dst = torch.full((x.shape[0], nb), 0xAB, dtype=torch.uint8, device="cuda")
    csa.csa_quant_kv(src, fmt, dst)
    torch.cuda.synchronize()
    return dst.cpu().numpy()


def test_fp4_entries_bit_exact(csa):
    x = _rows(1, 3000)
    got = _encode(csa, x, csa.CSA_FMT_FP4_E2M1_E4M3X16)
    assert np.array_equal(got, oq.fp4_quant_rows(x))


def test_fp4_entries_from_bf16_bit_exact(csa):
    x = _rows(2, 1000)
    xb = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = _encode(csa, xb, csa.CSA_FMT_FP4_E2M1_E4M3X16, dtype=torch.bfloat16)
    assert np.array_equal(got, oq.fp4_quant_rows(xb))


def test_fp8_window_entries_bit_exact(csa):
    x = _rows(3, 3000, scales=(1e-30, 1e-3, 1.0, 50.0, 1e5, 1e30))
    got = _encode(csa, x, csa.CSA_FMT_FP8_E4M3_UE8M0X32)
    assert np.array_equal(got, oq.fp8_window_quant_rows(x))


def test_plain_e4m3_cast_bit_exact(csa):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((777, 64)) * rng.choice([1e-3, 1, 100, 1e4], size=(777, 1))).astype(np.float32)
    got = _encode(csa, x, csa.CSA_FMT_FP8_E4M3_PLAIN, dim=64)
    assert np.array_equal(got, oq.e4m3_cast(x))


def _rounding_patterns():
    """fp32 bit patterns covering every rounding decision of E4M3 / E2M1:
    all signs and exponents, every value of the top 11 mantissa bits, and low
    bits at the boundaries (0, 1, half-1, half, half+1, all ones)."""
    sign = np.array([0, 1], dtype=np.uint32) << 31
    exp = np.arange(256, dtype=np.uint32) << 23
    hi = np.arange(2048, dtype=np.uint32) << 12
    lo = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], dtype=np.uint32)
    pat = (sign[:, None, None, None] | exp[None, :, None, None] | hi[None, None, :, None]
           | lo[None, None, None, :]).reshape(-1)
    f = pat.view(np.float32)
    return f[np.isfinite(f)]


def test_e4m3_encode_all_rounding_patterns(csa):
    x = _rounding_patterns()
    n = (x.size // 64) * 64
    x = x[:n].reshape(-1, 64)
    got = _encode(csa, x, csa.CSA_FMT_FP8_E4M3_PLAIN, dim=64)
    assert np.array_equal(got, oc.e4m3_encode(x).reshape(got.shape))


def test_e2m1_encode_all_rounding_patterns(csa):
    """Blocks whose amax is exactly 6 get scale 1.0, so the element codes are
    E2M1(x) of the raw values: covers every |x| <= 6 rounding pattern."""
    x = _rounding_patterns()
    x = x[np.abs(x) <= 6.0]
    n = (x.size // 15) * 15
    blocks = x[:n].reshape(-1, 15)
    rows = np.concatenate([np.full((blocks.shape[0], 1), 6.0, np.float32), blocks], axis=1).reshape(-1)
    m = (rows.size // 512) * 512
    rows = rows[:m].reshape(-1, 512)
    got = _encode(csa, rows, csa.CSA_FMT_FP4_E2M1_E4M3X16)
    assert np.all(got[:, 256:] == 0x38)       # every scale is exactly 1.0
    assert np.array_equal(got, oq.fp4_quant_rows(rows))


def test_strided_rows_and_zero_rows(csa):
    x = _rows(5, 64)
    src = torch.from_numpy(x).cuda()
    dst = torch.zeros((64, 2, 288), dtype=torch.uint8, device="cuda")   # every other 288-B slot
    csa.csa_quant_kv(src, csa.CSA_FMT_FP4_E2M1_E4M3X16, dst[:, 0], dst_row_stride=576)
    csa.csa_quant_kv(src, csa.CSA_FMT_FP4_E2M1_E4M3X16, dst[:, 1], n_rows=0, dst_row_stride=576)
    torch.cuda.synchronize()
    d = dst.cpu().numpy()
    assert np.array_equal(d[:, 0], oq.fp4_quant_rows(x))
    assert np.all(d[:, 1] == 0)
