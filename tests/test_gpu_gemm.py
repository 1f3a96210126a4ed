"""GPU parity of the W4A4 block-scaled GEMM (dense and grouped).

The fp32 output must match the oracle's float64 sum to within 1e-5 of sum|terms| per element
(the accumulation order is free); the bf16 output must equal the round-to-nearest-even cast of
the fp32 output bit for bit. Inputs are either seeded random codes and scales (all 16 codes and a
spread of scales, independent of the quantizer) or the full pipeline from bf16 X and W, in which
case each side quantizes with its own code."""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import Guarded, grouped_sf_rows, sf_index, swizzle

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def random_operands(seed, M, N, K, E=None):
    rng = np.random.default_rng(seed)
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    Asf = rng.integers(112, 140, (M, K // 32), dtype=np.uint8)
    shape_w = (N, K // 2) if E is None else (E, N, K // 2)
    Wq = rng.integers(0, 256, shape_w, dtype=np.uint8)
    Wsf = rng.integers(112, 140, shape_w[:-1] + (K // 32,), dtype=np.uint8)
    return Aq, Asf, Wq, Wsf


def run_linear(Aq, Asf_tiled, Wq, Wsf_tiled, M, N, out_dtype, use_workspace=True):
    Y = Guarded(M * N * (4 if out_dtype == mq.OUT_F32 else 2),
                dtype=torch.float32 if out_dtype == mq.OUT_F32 else torch.bfloat16, shape=(M, N))
    mq.linear(Aq, Asf_tiled, Wq, Wsf_tiled, out_dtype=out_dtype, Y=Y.t, use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert Y.intact(), "write outside Y"
    assert mq.device_status() == 0
    return Y.t


def assert_close(y_gpu, Y, T, rows=None):
    y = y_gpu.double().cpu().numpy()
    if rows is not None:
        y = y[rows]
    err = np.abs(y - Y)
    bound = RTOL * T + 1e-30
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} outputs off, worst rel {np.max(err / (T + 1e-30)):.3g} at {bad[:3].tolist()}"


def check_dense(Aq, Asf, Wq, Wsf, rows=None, use_workspace=True):
    M, N, K = Aq.shape[0], Wq.shape[0], Aq.shape[1] * 2
    dA = torch.from_numpy(Aq).cuda()
    dW = torch.from_numpy(Wq).cuda()
    dAsf = torch.from_numpy(swizzle(Asf, K)).cuda()
    dWsf = torch.from_numpy(swizzle(Wsf, K)).cuda()
    y32 = run_linear(dA, dAsf, dW, dWsf, M, N, mq.OUT_F32, use_workspace)
    y16 = run_linear(dA, dAsf, dW, dWsf, M, N, mq.OUT_BF16, use_workspace)
    Y, T = oracle.linear(Aq, Asf, Wq, Wsf, rows=rows)
    assert_close(y32, Y, T, rows)
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [
    (16, 256, 256), (1, 128, 128), (3, 384, 384), (17, 256, 768), (128, 256, 512),
    (129, 512, 512), (300, 128, 1024), (256, 768, 4096), (64, 1024, 5120),
    (300, 256, 384), (513, 512, 1280), (1024, 1024, 2048),
])
def test_random_codes(M, N, K):
    check_dense(*random_operands(M * 7 + N + K, M, N, K))


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (16, 256, 256), (77, 384, 1280), (128, 512, 2048)])
def test_general_kernel_at_small_m(M, N, K):
    """Without a workspace, small M runs the general (non-skinny) kernel: same results."""
    check_dense(*random_operands(M * 5 + N + K, M, N, K), use_workspace=False)


@pytest.mark.parametrize("M,N,K", [(1, 256, 4096), (5, 1024, 5120), (16, 14336 // 4, 4096), (128, 512, 1024)])
def test_skinny_split_tiles(M, N, K):
    """Skinny kernel with tiles split over several CTAs (partial sums reduced through the workspace),
    called repeatedly on one workspace: the per-tile counters must reset themselves."""
    ops = random_operands(M * 3 + N + K, M, N, K)
    for _ in range(3):
        check_dense(*ops)
    ws = mq._workspace(torch.device("cuda"), 0)
    assert int(ws[:mq.WORKSPACE_COUNTER_BYTES].count_nonzero()) == 0


def test_skinny_shared_workspace_across_shapes():
    """Calls of different shapes share one workspace: each call must leave the counter region zero so
    that the next call's counters start at zero, whatever it left in the scratch behind them."""
    for M, N, K in [(1, 7168, 4096), (1, 14336, 2048), (3, 256, 4096), (1, 14336, 4096), (16, 1024, 5120)]:
        check_dense(*random_operands(M + N + K, M, N, K), rows=np.array([0, M - 1]))
        ws = mq._workspace(torch.device("cuda"), 0)
        assert int(ws[:mq.WORKSPACE_COUNTER_BYTES].count_nonzero()) == 0, (M, N, K)


def test_extreme_scales_and_codes():
    """Every code against every code, and scales near both ends of the fp32 product range."""
    M, N, K = 16, 256, 256
    Aq = np.tile(np.arange(256, dtype=np.uint8), (M, K // 2 // 256 + 1))[:, :K // 2].copy()
    Wq = np.roll(np.tile(np.arange(256, dtype=np.uint8), (N, 1))[:, :K // 2], 3, axis=1).copy()
    Asf = np.full((M, K // 32), 127, np.uint8)
    Wsf = np.full((N, K // 32), 127, np.uint8)
    Asf[1] = 160          # 2^33: products up to 2^96 * 36 stay finite in fp32
    Wsf[:, 1] = 60        # 2^-67
    Asf[2, 3] = 0         # the smallest scale, 2^-127
    Wsf[5] = 190          # 2^63
    Asf[5] = 10           # 2^-117
    check_dense(Aq, Asf, Wq, Wsf)


def pipeline(c, b=32):
    """Each side quantizes with its own code; returns GPU operands and oracle operands."""
    s = c.s
    oWq, oWsf, oinv = oracle.prep_weights(c.W, s, b)
    oXq, oXsf = oracle.act_quant(c.X, oinv, b)
    gWq, gWsf, ginv = mq.prep_weights(c.W.cuda(), s.cuda(), b)
    gXq, gXsf = mq.act_quant(c.X.cuda(), ginv, b)
    return (gXq, gXsf, gWq, gWsf), (oXq, oXsf, oWq, oWsf)


def test_tiny_workload_pipeline():
    c = inputs.tiny()
    (gXq, gXsf, gWq, gWsf), (oXq, oXsf, oWq, oWsf) = pipeline(c)
    M, N = c.X.shape[0], c.W.shape[0]
    y32 = run_linear(gXq, gXsf, gWq, gWsf, M, N, mq.OUT_F32)
    y16 = run_linear(gXq, gXsf, gWq, gWsf, M, N, mq.OUT_BF16)
    Y, T = oracle.linear(oXq, oXsf, oWq, oWsf)
    assert_close(y32, Y, T)
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    ref = c.X.double() @ c.W.double().T
    rel = (y32.double().cpu() - ref).norm() / ref.norm()
    assert rel < 0.6


@pytest.mark.parametrize("M", inputs.LLAMA3_8B_M)
def test_llama3_8b_up_sampled(M):
    c = inputs.llama3_8b_up(M)
    (gXq, gXsf, gWq, gWsf), (oXq, oXsf, oWq, oWsf) = pipeline(c)
    N = c.W.shape[0]
    y32 = run_linear(gXq, gXsf, gWq, gWsf, M, N, mq.OUT_F32)
    y16 = run_linear(gXq, gXsf, gWq, gWsf, M, N, mq.OUT_BF16)
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    if M <= 512:
        rows = np.arange(M)
    else:  # 256 random rows plus both edge rows of every 128-row tile
        rng = np.random.default_rng(M)
        rows = np.unique(np.concatenate([np.arange(0, M, 128), np.arange(127, M, 128),
                                         rng.choice(M, 256, replace=False)]))
    Y, T = oracle.linear_matmul(oXq, oXsf, oWq, oWsf, rows=rows)
    assert_close(y32, Y, T, rows)


@pytest.mark.parametrize("M,N,K", [(2048, 14336, 4096), (640, 2816, 1536)])
def test_random_codes_every_output_many_rounds(M, N, K):
    """Every output of a shape with more tiles than 2-SM pairs (2048 x 14336: 448 tiles of 256 x 256
    over 74 pairs, 7 persistent rounds; 640 x 2816: 33 tiles with a ragged last row tile), random
    codes and scales, checked against the float64 oracle over the whole matrix."""
    Aq, Asf, Wq, Wsf = random_operands(M + N + K, M, N, K)
    dA, dW = torch.from_numpy(Aq).cuda(), torch.from_numpy(Wq).cuda()
    dAsf, dWsf = torch.from_numpy(swizzle(Asf, K)).cuda(), torch.from_numpy(swizzle(Wsf, K)).cuda()
    y32 = run_linear(dA, dAsf, dW, dWsf, M, N, mq.OUT_F32)
    y16 = run_linear(dA, dAsf, dW, dWsf, M, N, mq.OUT_BF16)
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    Y, T = oracle.linear_matmul(Aq, Asf, Wq, Wsf)
    assert_close(y32, Y, T)


# ------------------------------------------------------------------------------------- grouped
def run_grouped(Aq, Asf_t, offsets, Wq, Wsf_t, out_dtype):
    M = Aq.shape[0]
    E, N, _ = Wq.shape
    dt = torch.float32 if out_dtype == mq.OUT_F32 else torch.bfloat16
    Y = Guarded(M * N * (4 if out_dtype == mq.OUT_F32 else 2), dtype=dt, shape=(M, N))
    Y.t.zero_()
    off_d = torch.tensor(np.asarray(offsets, np.int32), device="cuda")
    mq.grouped_linear(Aq, Asf_t, off_d, Wq, Wsf_t, out_dtype=out_dtype, Y=Y.t)
    torch.cuda.synchronize()
    assert Y.intact()
    assert mq.device_status() == 0
    return Y.t


def grouped_tiled_sf(Asf, offsets, K):
    rows = grouped_sf_rows(offsets)
    E = len(offsets) - 1
    buf = np.zeros(mq.grouped_sf_bytes(Asf.shape[0], E, K), np.uint8)
    buf[sf_index(rows, K)] = Asf
    return buf


_PAIR_SIZES = [0, 513, 7, 256, 255, 900, 128, 1, 0, 640, 384, 129, 1000, 2, 300, 17, 760, 64, 3, 222]


@pytest.mark.parametrize("offsets,N,K", [
    ([0, 5, 5, 140, 141, 141, 300], 256, 256),
    ([0, 0, 1, 129, 257, 257], 128, 384),
    ([0, 64, 64, 64, 200], 512, 1024),
    # at least 256 rows per expert on average, N and K multiples of 256: the 2-SM grouped form, with
    # empty experts, one-row experts, odd tile counts (a pair's second half past its expert) and
    # partial tiles
    ([0, 0, 300, 429, 1429, 1430, 2130], 512, 512),
    ([0, 1024, 1024, 2500], 768, 768),
    ([0] + list(np.cumsum(_PAIR_SIZES)), 256, 1024),
])
def test_grouped_random_codes(offsets, N, K):
    """Every output of the grouped GEMM against the oracle (fp32 within 1e-5 of sum|terms|, bf16 the
    rounded fp32), on random codes and scales."""
    E = len(offsets) - 1
    M = offsets[-1]
    Aq, Asf, Wq, Wsf = random_operands(E * 11 + K, M, N, K, E=E)
    dWsf = torch.from_numpy(np.stack([swizzle(Wsf[e], K) for e in range(E)])).cuda()
    dAsf = torch.from_numpy(grouped_tiled_sf(Asf, offsets, K)).cuda()
    dA, dW = torch.from_numpy(Aq).cuda(), torch.from_numpy(Wq).cuda()
    y32 = run_grouped(dA, dAsf, offsets, dW, dWsf, mq.OUT_F32)
    y16 = run_grouped(dA, dAsf, offsets, dW, dWsf, mq.OUT_BF16)
    Y, T = oracle.grouped_linear(Aq, Asf, offsets, Wq, Wsf)
    assert_close(y32, Y, T)
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


@pytest.mark.parametrize("T", [64])
def test_moe_pipeline_sampled(T):
    c = inputs.moe_30b_a3b(T, "gate_up")
    E, N, K = c.W.shape
    off = c.offsets.numpy()
    oinv = [None] * E
    oWq = np.empty((E, N, K // 2), np.uint8)
    oWsf = np.empty((E, N, K // 32), np.uint8)
    gWq = torch.empty(E, N, K // 2, dtype=torch.uint8, device="cuda")
    gWsf = torch.empty(E, mq.sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    ginv = torch.empty(E, K, dtype=torch.float32, device="cuda")
    Wd = c.W.cuda()
    sd = c.s.cuda()
    for e in range(E):
        oWq[e], oWsf[e], oinv[e] = oracle.prep_weights(c.W[e], c.s[e], 32)
        mq.prep_weights(Wd[e], sd[e], 32, Wq=gWq[e], Wsf=gWsf[e], inv_s=ginv[e])
    oinv = np.stack(oinv)
    oXq, oXsf = oracle.act_quant(c.X, oinv, 32, offsets=off)
    off_d = c.offsets.cuda()
    gXq, gXsf = mq.act_quant(c.X.cuda(), ginv, 32, group_offsets=off_d)
    y32 = run_grouped(gXq, gXsf, off, gWq, gWsf, mq.OUT_F32)
    rng = np.random.default_rng(T)
    rows = np.unique(np.concatenate([[0, off[-1] - 1], rng.integers(0, off[-1], 24)]))
    Y, Tt = oracle.grouped_linear(oXq, oXsf, off, oWq, oWsf, rows=rows)
    assert_close(y32, Y, Tt, rows)


# ------------------------------------------------------------------------------------- failure
def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait limit of 1 ns makes the GEMM's first pipeline wait run out: the kernel must return,
    report MACAQ_ERR_TIMEOUT through the status word, and leave the context usable."""
    M, N, K = 256, 512, 2048
    Aq, Asf, Wq, Wsf = random_operands(3, M, N, K)
    dA, dW = torch.from_numpy(Aq).cuda(), torch.from_numpy(Wq).cuda()
    dAsf, dWsf = torch.from_numpy(swizzle(Asf, K)).cuda(), torch.from_numpy(swizzle(Wsf, K)).cuda()
    mq.device_status(reset=True)
    try:
        mq.set_wait_limit_ns(1)
        mq.linear(dA, dAsf, dW, dWsf, out_dtype=mq.OUT_F32)
        torch.cuda.synchronize()
    finally:
        mq.set_wait_limit_ns(0)
    assert mq.device_status(reset=True) == 6
    assert mq.device_status() == 0
    check_dense(Aq, Asf, Wq, Wsf, rows=np.array([0, 100, 255]))
