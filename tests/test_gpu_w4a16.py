"""GPU parity of the weight-only (W4A16) decode mode.

macaq_act_transform: bf16 bits equal to the oracle's act_transform_bf16 (bit for bit), every block size,
with and without s. macaq_linear_w4a16: the fp32 output within 1e-5 of sum|terms| of the oracle's
float64 weight-only layer (the same bf16 activations times the exact dequantized weights) on every
output, and the bf16 output equal to the round-to-nearest-even cast of the fp32 output; both the
whole-tile and the split-tile plans, ragged M, extreme weight scales (E8M0 from 1 to 252) and every
code, and the Llama-3-8B decode shapes.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import Guarded, swizzle

pytestmark = pytest.mark.gpu
RTOL = 1e-5


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
@pytest.mark.parametrize("M,K", [(1, 256), (17, 1152), (300, 4096)])
def test_act_transform_matches_oracle(M, K, b):
    c = inputs.dense_case(2000 + M + K + b, M, K, 1, n_outliers=3, outlier_factor=40.0, draw_w=False)
    for with_s in (True, False):
        inv = (np.float32(1.0) / c.s.numpy()).astype(np.float32) if with_s else None
        ref = oracle.act_transform_bf16(c.X, inv, b)
        out = Guarded(M * K * 2, dtype=torch.bfloat16, shape=(M, K))
        mq.act_transform(c.X.cuda(), None if inv is None else torch.from_numpy(inv).cuda(), b, Xt=out.t)
        torch.cuda.synchronize()
        assert out.intact()
        np.testing.assert_array_equal(out.t.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def run_w4a16(X, inv, b, Wq, Wsf, out_dtype):
    M, N = X.shape[0], Wq.shape[0]
    dt = torch.float32 if out_dtype == mq.OUT_F32 else torch.bfloat16
    Y = Guarded(M * N * (4 if out_dtype == mq.OUT_F32 else 2), dtype=dt, shape=(M, N))
    mq.linear_w4a16(X.cuda(), None if inv is None else torch.from_numpy(inv).cuda(), Wq, Wsf, had_block=b,
                    out_dtype=out_dtype, Y=Y.t)
    torch.cuda.synchronize()
    assert Y.intact(), "write outside Y"
    assert mq.device_status() == 0
    return Y.t


def check(X, inv, b, Wq_np, Wsf_np, repeats=1):
    """Wq_np, Wsf_np: codes [N, K/2] and row-major scales [N, K/32] given to both sides."""
    K = Wq_np.shape[1] * 2
    Wq, Wsf = torch.from_numpy(Wq_np).cuda(), torch.from_numpy(swizzle(Wsf_np, K)).cuda()
    Y, T = oracle.w4a16_linear(X, inv, b, Wq_np, Wsf_np)
    for _ in range(repeats):
        y32 = run_w4a16(X, inv, b, Wq, Wsf, mq.OUT_F32)
        y16 = run_w4a16(X, inv, b, Wq, Wsf, mq.OUT_BF16)
        err = np.abs(y32.double().cpu().numpy() - Y)
        bad = np.argwhere(err > RTOL * T + 1e-30)
        assert bad.size == 0, f"{len(bad)} outputs off, worst rel {np.max(err / (T + 1e-30)):.3g} at {bad[:3].tolist()}"
        assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (3, 1024, 1024), (16, 14336 // 4, 4096), (17, 512, 2048),
                                   (64, 1024, 5120), (64, 768, 1536)])
def test_random_codes(M, N, K):
    rng = np.random.default_rng(M + N + K)
    c = inputs.dense_case(3000 + M + N + K, M, K, 1, n_outliers=2, outlier_factor=30.0, draw_w=False)
    inv = (np.float32(1.0) / c.s.numpy()).astype(np.float32)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Wsf = rng.integers(112, 140, (N, K // 32), dtype=np.uint8)
    check(c.X, inv, 32, Wq, Wsf, repeats=2)   # twice on one workspace: split counters reset themselves


def test_larger_batches_are_refused():
    X = torch.zeros(65, 256, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(256, 128, dtype=torch.uint8, device="cuda")
    Wsf = torch.zeros(mq.sf_bytes(256, 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(mq.MacaqError, match="MACAQ_ERR_SHAPE"):
        mq.linear_w4a16(X, None, Wq, Wsf, had_block=1, workspace=torch.zeros(1 << 20, dtype=torch.uint8, device="cuda"))


def test_extreme_scales_and_every_code():
    M, N, K = 4, 256, 512
    Wq = np.tile(np.arange(256, dtype=np.uint8), (N, K // 2 // 256 + 1))[:, :K // 2].copy()
    Wsf = np.full((N, K // 32), 127, np.uint8)
    Wsf[:, 0] = 1          # 2^-126: values down to the smallest normal bf16 / 2 (a subnormal)
    Wsf[:, 1] = 252        # 2^125: values up to 6 * 2^125, the largest the mode takes
    X = torch.zeros(M, K, dtype=torch.float32)
    X[:, :32] = 1.0e-3     # group 0 (2^-126): products below the smallest normal fp32
    X[:, 32:64] = 1.0e-30  # group 1 (2^125): keeps its products finite in fp32
    X[:, 64:] = torch.randn(M, K - 64, generator=torch.Generator().manual_seed(3))
    check(X.to(torch.bfloat16), None, 1, Wq, Wsf)


@pytest.mark.parametrize("M", [1, 16])
def test_llama3_8b_up_decode(M):
    c = inputs.llama3_8b_up(M)
    Wq, Wsf, inv = oracle.prep_weights(c.W, c.s, 32)
    check(c.X, inv, 32, Wq, Wsf)
