"""macaq_linear_fixed_scratch (no device allocation) against macaq_linear, through the C ABI.

Each case runs the fixed-scratch call twice in a row; both results must match the existing entry
point within the GEMM tolerance (1e-5 of sum|terms| per element), and the bf16 output must be the
round-to-nearest-even cast of the fp32 one. The file is collected last so that it also runs after
every other test has used the library on the device; it passes on its own as well."""
import ctypes

import numpy as np
import pytest
import torch

import w4a4_mxfp4_quantized_b200 as mq
from sfutil import swizzle

pytestmark = pytest.mark.gpu
RTOL = 1e-5
FIXED_SCRATCH_BYTES = 8 << 20   # MACAQ_FIXED_SCRATCH_BYTES
E2M1_ABS = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=torch.float64)


def operands(seed, M, N, K):
    rng = np.random.default_rng(seed)
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    Asf = rng.integers(112, 140, (M, K // 32), dtype=np.uint8)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Wsf = rng.integers(112, 140, (N, K // 32), dtype=np.uint8)
    return Aq, Asf, Wq, Wsf


def abs_dequant(q, sf):
    """|value| of every element: low nibble first, one 2^(e - 127) scale per 32 elements."""
    q = torch.from_numpy(q).long()
    codes = torch.stack([q & 0xF, q >> 4], dim=-1).reshape(q.shape[0], -1)
    mag = E2M1_ABS[codes & 7]
    scale = torch.pow(2.0, torch.from_numpy(sf).double() - 127.0)
    return (mag.reshape(q.shape[0], -1, 32) * scale[..., None]).reshape(q.shape[0], -1)


def fixed_scratch_call(dA, dAsf, dW, dWsf, Y, M, N, K, out_dtype):
    return mq.lib().macaq_linear_fixed_scratch(
        mq.A_QUANTIZED, dA.data_ptr(), dAsf.data_ptr(), None, M, N, K, 32, dW.data_ptr(), dWsf.data_ptr(),
        Y.data_ptr(), out_dtype, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K", [
    (1, 14336, 4096),     # skinny, whole tiles
    (16, 4096, 4096),     # skinny, split tiles reduced through the scratch
    (5, 1024, 5120),      # skinny, split tiles
    (128, 512, 1024),
    (77, 384, 1280),      # K % 256 != 0: general kernel, no scratch
    (300, 256, 512),      # M > 128: general kernel, no scratch
])
def test_fixed_scratch_matches_linear(M, N, K):
    Aq, Asf, Wq, Wsf = operands(M * 13 + N + K, M, N, K)
    dA, dW = torch.from_numpy(Aq).cuda(), torch.from_numpy(Wq).cuda()
    dAsf, dWsf = torch.from_numpy(swizzle(Asf, K)).cuda(), torch.from_numpy(swizzle(Wsf, K)).cuda()
    ref = mq.linear(dA, dAsf, dW, dWsf, out_dtype=mq.OUT_F32)
    torch.cuda.synchronize()
    T = (abs_dequant(Aq, Asf).cuda() @ abs_dequant(Wq, Wsf).cuda().T)
    bound = RTOL * T + 1e-30
    for _ in range(2):
        y32 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        y16 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert fixed_scratch_call(dA, dAsf, dW, dWsf, y32, M, N, K, mq.OUT_F32) == 0
        assert fixed_scratch_call(dA, dAsf, dW, dWsf, y16, M, N, K, mq.OUT_BF16) == 0
        torch.cuda.synchronize()
        assert mq.device_status() == 0
        err = (y32.double() - ref.double()).abs()
        assert bool((err <= bound).all()), f"max rel err {float((err / (T + 1e-30)).max()):.3g}"
        assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


def test_fixed_scratch_rejects_plans_beyond_its_size():
    """A skinny plan that needs more scratch than the fixed area is refused before any launch."""
    M = 128
    shape = None
    for N in (1024, 4096, 8192, 16384):           # partial tiles grow with tiles x pieces x M
        for K in (16384, 32768, 65536, 131072):
            if mq.workspace_bytes(M, N, K) > FIXED_SCRATCH_BYTES:
                shape = (N, K)
                break
        if shape:
            break
    assert shape is not None, "no shape found whose skinny plan exceeds the fixed scratch"
    N, K = shape
    dA = torch.zeros(M, K // 2, dtype=torch.uint8, device="cuda")
    dAsf = torch.zeros(mq.sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    dW = torch.zeros(N, K // 2, dtype=torch.uint8, device="cuda")
    dWsf = torch.zeros(mq.sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    Y = torch.full((M, N), 3.0, dtype=torch.float32, device="cuda")
    status = fixed_scratch_call(dA, dAsf, dW, dWsf, Y, M, N, K, mq.OUT_F32)
    torch.cuda.synchronize()
    assert mq.status_str(status) == "MACAQ_ERR_WORKSPACE"
    assert bool((Y == 3.0).all()), "a refused call must not write Y"


def test_fixed_scratch_after_a_timeout_needs_no_clean_up():
    """A split-tile call whose pipeline waits run out (1 ns limit) reports MACAQ_ERR_TIMEOUT and may
    leave per-tile counters behind in the fixed scratch; the next call clears the counters it uses,
    so it matches macaq_linear again without any clean-up by the caller."""
    M, N, K = 16, 4096, 4096
    Aq, Asf, Wq, Wsf = operands(77, M, N, K)
    dA, dW = torch.from_numpy(Aq).cuda(), torch.from_numpy(Wq).cuda()
    dAsf, dWsf = torch.from_numpy(swizzle(Asf, K)).cuda(), torch.from_numpy(swizzle(Wsf, K)).cuda()
    ref = mq.linear(dA, dAsf, dW, dWsf, out_dtype=mq.OUT_F32)
    torch.cuda.synchronize()
    mq.device_status(reset=True)
    y32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    try:
        mq.set_wait_limit_ns(1)
        assert fixed_scratch_call(dA, dAsf, dW, dWsf, y32, M, N, K, mq.OUT_F32) == 0
        torch.cuda.synchronize()
    finally:
        mq.set_wait_limit_ns(0)
    assert mq.device_status(reset=True) == 6
    T = (abs_dequant(Aq, Asf).cuda() @ abs_dequant(Wq, Wsf).cuda().T)
    for _ in range(2):
        y32.fill_(float("nan"))
        assert fixed_scratch_call(dA, dAsf, dW, dWsf, y32, M, N, K, mq.OUT_F32) == 0
        torch.cuda.synchronize()
        assert mq.device_status() == 0
        assert bool(((y32.double() - ref.double()).abs() <= RTOL * T + 1e-30).all())
