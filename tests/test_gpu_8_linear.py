"""INT8-weight / BF16-compute linear layer through the C ABI against the oracle (reading in nomas.h and
oracle/linear.py; fluxbbs.com "单卡 4090 怎么做到的", first technique).  Codes, scales and dequantised
weights are compared bit for bit; y = x W^T element by element within the fp32 accumulation bound
(2 K 2^-23 sum_k |x||w|, allowing for any summation order and truncating adds), on ragged shapes that
span several tiles and on the DiT's QKV and FFN-down shapes (sampled rows); bf16 outputs additionally
within one bf16 rounding."""
import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200 import _nomas as N
from int8_kv_cache_action_b200.runtime import Int8Linear
from oracle import linear as ol

pytestmark = pytest.mark.gpu


def _weights(n, k, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(n, k, generator=g) * 0.02
    w[:: max(1, n // 7)] *= 30.0                      # some loud rows
    w[1 % n, : min(k, 5)] = 0.0
    return w.to(torch.bfloat16)


def _acts(m, k, seed):
    return torch.randn(m, k, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)


def _ref(x, lin, rows=None):
    codes, scales = lin.codes.cpu().numpy(), lin.scales.cpu().numpy()
    xf = x.float().numpy()
    return ol.linear(xf, codes, scales, rows), ol.abs_product_sum(xf, codes, scales, rows)


@pytest.mark.parametrize("n,k", [(1, 8), (7, 24), (300, 136), (513, 2048)])
def test_quantise_and_dequantise_bit_exact(n, k):
    w = _weights(n, k, 1)
    lin = Int8Linear.from_weights(w.cuda())
    q, s = ol.quantize_weights(w.float().numpy())
    assert np.array_equal(lin.codes.cpu().numpy(), q)
    assert np.array_equal(lin.scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    deq = lin.dequantized().float().cpu().numpy()
    assert np.array_equal(deq.view(np.uint32), ol.dequantize_bf16(q, s).view(np.uint32))


@pytest.mark.parametrize("m,n,k", [(1, 1, 8), (5, 300, 136), (200, 513, 264), (257, 256, 2048), (131, 1000, 72)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_linear_within_the_accumulation_bound(m, n, k, out_dtype):
    x = _acts(m, k, 2)
    lin = Int8Linear.from_weights(_weights(n, k, 3).cuda())
    y = lin(x.cuda(), out_dtype=out_dtype).float().cpu().numpy().astype(np.float64)
    assert lin.status() == N.NOMAS_OK
    ref, mag = _ref(x, lin)
    bound = 2.0 * k * 2.0 ** -23 * mag + 1e-30
    if out_dtype == torch.bfloat16:
        bound = bound + 2.0 ** -8 * np.abs(ref)
    err = np.abs(y - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    assert np.sum(err) <= 1e-2 * np.sum(np.abs(ref)) + 1e-30


@pytest.mark.parametrize("m,n,k", [(27680, 6144, 2048), (27680, 2048, 8192)])
def test_dit_shapes_sampled_rows(m, n, k):
    # QKV projection of a production segment (26400 video + 1280 text tokens, hidden 2048) and the FFN's
    # down projection (8192 -> 2048); rows sampled across the M tiles, the last one included
    x = _acts(m, k, 4)
    lin = Int8Linear.from_weights(_weights(n, k, 5).cuda())
    y = lin(x.cuda(), out_dtype=torch.float32)
    assert lin.status() == N.NOMAS_OK
    rows = np.array(sorted(set(np.random.default_rng(6).integers(0, m, 24).tolist()) | {0, m - 1}))
    ref, mag = _ref(x, lin, rows)
    got = y[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 * k * 2.0 ** -23 * mag)


def test_strided_input_and_output():
    m, n, k = 130, 260, 96
    xb = _acts(m, 2 * k, 7)
    x = xb[:, :k]                                     # row pitch 2K
    lin = Int8Linear.from_weights(_weights(n, k, 8).cuda())
    ybuf = torch.full((m, n + 44), 7.0, dtype=torch.float32, device="cuda")
    out = ybuf[:, :n]                                 # row pitch N + 44
    xd = xb.cuda()[:, :k]
    lin(xd, out=out)
    assert lin.status() == N.NOMAS_OK
    ref, mag = _ref(x.contiguous(), lin)
    assert np.all(np.abs(out.cpu().numpy() - ref) <= 2.0 * k * 2.0 ** -23 * mag)
    assert torch.all(ybuf[:, n:] == 7.0)              # nothing written past each row's N columns


def test_argument_errors_return_before_any_launch():
    lin = Int8Linear.from_weights(_weights(16, 32, 9).cuda())
    x = _acts(4, 32, 10).cuda()
    y = torch.empty(4, 16, device="cuda")
    st = lin.status_word.data_ptr()
    ws = lin.workspace.data_ptr()
    args = dict(x=x.data_ptr(), m=4, k_in=32, ldx=32, codes=lin.codes.data_ptr(), scales=lin.scales.data_ptr(),
                n_out=16, y=y.data_ptr(), ldy=16, y_dtype=N.NOMAS_DTYPE_F32, workspace=ws, status=st)

    def call(**kw):
        a = dict(args, **kw)
        return N.nomas_w8a16_linear(a["x"], a["m"], a["k_in"], a["ldx"], a["codes"], a["scales"], a["n_out"],
                                    a["y"], a["ldy"], a["y_dtype"], a["workspace"], a["status"])
    assert call() == N.NOMAS_OK
    assert call(k_in=30, ldx=30) == N.NOMAS_EINVAL          # K not a multiple of 8
    assert call(ldx=16) == N.NOMAS_EINVAL                   # pitch below K
    assert call(m=0) == N.NOMAS_EINVAL
    assert call(x=x.data_ptr() + 2) == N.NOMAS_EINVAL       # misaligned
    assert call(y_dtype=5) == N.NOMAS_EINVAL
    assert call(status=0) == N.NOMAS_EINVAL
    torch.cuda.synchronize()
    assert lin.status() == N.NOMAS_OK


def test_forced_wait_limit_reports_timeout_and_the_next_call_is_exact():
    m, n, k = 300, 512, 512
    x = _acts(m, k, 11).cuda()
    lin = Int8Linear.from_weights(_weights(n, k, 12).cuda())
    ref = lin(x, out_dtype=torch.float32).clone()
    assert lin.status() == N.NOMAS_OK
    prev = N.nomas_set_wait_limit_ns(0)
    try:
        lin(x, out_dtype=torch.float32)
        torch.cuda.synchronize()
        st = lin.status()
    finally:
        N.nomas_set_wait_limit_ns(prev)
    assert st == N.NOMAS_ETIMEOUT
    again = lin(x, out_dtype=torch.float32)
    assert lin.status() == N.NOMAS_OK
    assert torch.equal(again, ref)
