"""GPU parity of nvfp4_amax (the amax values of Eq. 1 from one read of the
tensor: plain, rotated rows, rotated columns) and of NVFP4_AMAX_PROVIDED
(quantize from those values instead of an amax pass of its own).

The amax values must equal the oracle's bit for bit (Four Over Six §2.1
Eq. 1; rotated values as the rotating modes quantize them), and every output
of a quantize call with NVFP4_AMAX_PROVIDED must equal the same call's
two-pass result byte for byte: the alpha of Eq. 1 follows from the same amax
by the same division.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu

ROW, COL, B2D, GEMM, RHT, HEADROOM = 0x1, 0x2, 0x4, 0x20, 0x40, 0x200
RTN, FOUR_SIX, RHT_SR, MS_EDEN, RHT_SR_HW = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import api as _api
    return _api


def _bits(t):
    return t.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("shape", [(256, 1024), (48, 144), (80, 272), (1040, 1552), (8192, 4096)])
@pytest.mark.parametrize("seed", [0, 77])
def test_amax_values_match_the_oracle(api, shape, seed):
    R, C = shape
    x = synthetic.normal_with_channel_outliers(R, C, seed=R + C + seed)
    bits = synthetic.bf16_bits(x)
    a = api.nvfp4_amax(x.cuda(), ROW | COL | RHT, seed=seed)
    torch.cuda.synchronize()
    got = a.cpu().numpy()
    assert got[0] == np.float32(oracle.amax(bits, 0, False, seed))
    assert got[1] == np.float32(oracle.amax(bits, 0, True, seed))
    assert got[2] == np.float32(oracle.amax(bits, 1, True, seed))
    # the orientations not asked for stay 0; without rotation only the plain value
    b = api.nvfp4_amax(x.cuda(), COL | RHT, seed=seed)
    c = api.nvfp4_amax(x.cuda(), 0)
    torch.cuda.synchronize()
    assert b.cpu().numpy()[1] == 0.0 and b.cpu().numpy()[2] == got[2] and b.cpu().numpy()[0] == got[0]
    assert np.array_equal(c.cpu().numpy(), np.array([got[0], 0.0, 0.0], np.float32))


def test_amax_nonfinite_sets_status_and_marker(api):
    x = torch.randn(64, 128, dtype=torch.bfloat16, device="cuda")
    x[5, 7] = float("nan")
    for flags in (0, ROW | RHT, COL | RHT, ROW | COL | RHT):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        a = api.nvfp4_amax(x, flags, seed=3, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == -4, flags
        assert _bits(a)[0] == 0xFFFFFFFF


def test_amax_empty_tensor_clears_the_output(api):
    out = torch.full((3,), 7.0, dtype=torch.float32, device="cuda")
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    api.nvfp4_amax(x, ROW | RHT, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), np.zeros(3, np.float32))


def _same(q, p, flags):
    for side, bit in (("row", ROW), ("col", COL)):
        if not flags & bit:
            continue
        for k in ("codes", "scales", "alpha"):
            assert torch.equal(getattr(q, f"{k}_{side}"), getattr(p, f"{k}_{side}")), (side, k)
    assert torch.equal(q.amax, p.amax)


CASES = [(FOUR_SIX, ROW | GEMM), (FOUR_SIX, ROW | B2D | GEMM), (RTN, ROW | COL), (RTN, COL | RHT | GEMM),
         (MS_EDEN, ROW | COL | GEMM), (RHT_SR, ROW | COL), (RHT_SR_HW, ROW | COL), (FOUR_SIX, ROW | RHT | HEADROOM),
         (FOUR_SIX, ROW | COL | B2D)]


@pytest.mark.parametrize("mode,flags", CASES)
@pytest.mark.parametrize("shape", [(256, 1024), (1024, 4096)])
def test_amax_provided_equals_the_two_pass_call(api, mode, flags, shape):
    R, C = shape
    x = synthetic.laplace_with_spikes(R, C, seed=R + mode).cuda()
    seed, sid = 21, 2
    p = api.nvfp4_quantize(x, mode, flags, seed=seed, stream_id=sid)
    rot = bool(flags & RHT) or mode in (RHT_SR, MS_EDEN, RHT_SR_HW)
    rot = rot and not flags & B2D
    a = api.nvfp4_amax(x, (ROW | COL | RHT) if rot else 0, seed=seed)
    q = api.nvfp4_quantize(x, mode, flags, seed=seed, stream_id=sid, amax=a)
    torch.cuda.synchronize()
    _same(q, p, flags)


def test_linear_step_with_shared_amax_passes(api):
    # the 8B-shaped forward operands and rotated backward partners from one
    # amax pass per tensor, against the two-pass calls
    layer = synthetic.layer(1024, 512, 1536, seed=9)
    seed = 4000
    for name, t in (("x", layer["x"]), ("w", layer["w"])):
        t = t.cuda()
        a = api.nvfp4_amax(t, COL | RHT, seed=seed)
        fwd_flags = ROW | GEMM | (B2D if name == "w" else 0)
        _same(api.nvfp4_quantize(t, FOUR_SIX, fwd_flags, amax=a), api.nvfp4_quantize(t, FOUR_SIX, fwd_flags),
              fwd_flags)
        bwd = COL | RHT | GEMM
        _same(api.nvfp4_quantize(t, RTN, bwd, seed=seed, stream_id=1, amax=a),
              api.nvfp4_quantize(t, RTN, bwd, seed=seed, stream_id=1), bwd)
