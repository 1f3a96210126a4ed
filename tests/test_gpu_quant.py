"""GPU parity of the transform + MXFP4 quantizer (activations and weight preparation).

Bit-exact against the CPU oracle: every FP4 code byte and every E8M0 scale (after undoing the
documented tiling), padding rows of the tiled SF zero, canary zones around every output intact."""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import Guarded, grouped_padding_rows, grouped_sf_rows, sf_index, unswizzle

pytestmark = pytest.mark.gpu


def gpu_act_quant(X, inv_s, b, offsets=None):
    M, K = X.shape
    E = 0 if offsets is None else len(offsets) - 1
    n_sf = mq.grouped_sf_bytes(M, E, K) if offsets is not None else mq.sf_bytes(M, K)
    q = Guarded(M * K // 2, shape=(M, K // 2))
    sf = Guarded(max(n_sf, 16))
    off_d = None if offsets is None else torch.tensor(np.asarray(offsets, np.int32), device="cuda")
    inv_d = None if inv_s is None else torch.as_tensor(np.ascontiguousarray(inv_s)).cuda()
    mq.act_quant(X.cuda(), inv_d, b, group_offsets=off_d, Xq=q.t, Xsf=sf.t)
    torch.cuda.synchronize()
    assert q.intact() and sf.intact(), "write outside the output buffers"
    assert mq.device_status() == 0
    return q.t.cpu().numpy(), sf.t.cpu().numpy()


def check_act(X, inv_s, b, offsets=None):
    M, K = X.shape
    oq, osf = oracle.act_quant(X, inv_s, b, offsets=offsets)
    gq, gsf = gpu_act_quant(X, inv_s, b, offsets)
    bad = np.argwhere(gq != oq)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    if offsets is None:
        np.testing.assert_array_equal(unswizzle(gsf, M, K), osf)
        pad = np.arange(M, (M + 127) // 128 * 128)
    else:
        np.testing.assert_array_equal(unswizzle(gsf, M, K, grouped_sf_rows(offsets)), osf)
        pad = grouped_padding_rows(offsets)
    if pad.size:
        assert np.all(gsf[sf_index(pad, K)] == 0), "padding rows of the SF must be zero"


def test_tiny_workload():
    c = inputs.tiny()
    inv_s = np.float32(1.0) / c.s.numpy()
    check_act(c.X, inv_s, 32)


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
@pytest.mark.parametrize("with_scale", [True, False])
def test_hadamard_blocks(b, with_scale):
    c = inputs.dense_case(77 + b, 37, 512, 1, n_outliers=5, outlier_factor=40.0, draw_w=False)
    inv_s = np.float32(1.0) / c.s.numpy() if with_scale else None
    check_act(c.X, inv_s, b)


@pytest.mark.parametrize("M", [1, 3, 17, 129, 300])
@pytest.mark.parametrize("K", [128, 384, 768])
def test_ragged_rows(M, K):
    c = inputs.dense_case(500 + M + K, M, K, 1, n_outliers=2, outlier_factor=30.0, draw_w=False)
    check_act(c.X, np.float32(1.0) / c.s.numpy(), 32)


def test_exact_ties_zeros_and_signed_zero():
    """Hand-built groups whose scaled values sit exactly on E2M1 rounding ties (b = 1, no scale)."""
    K = 128
    X = torch.zeros(6, K, dtype=torch.float32)
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -2.5, -5.0, 7.0, -7.0, -0.1, 6.0]
    for r, e in enumerate([-3, 0, 5, 40]):
        X[r, :len(ties)] = torch.tensor(ties) * 2.0 ** e
        X[r, 31] = 4.0 * 2.0 ** e               # fixes the group's scale at E = 127 + e
        X[r, 32:64] = 2.0 ** (e - 130)          # a group far below its neighbours
    X[4] = 0.0                                   # all-zero row: E = 0, codes 0
    X[5] = -0.0                                  # negative zeros keep their sign bit
    X[5, 100] = 1e-39                            # subnormal-only group
    check_act(X.to(torch.bfloat16), None, 1)


def test_llama3_8b_up_full_act_quant():
    for M in inputs.LLAMA3_8B_M:
        c = inputs.llama3_8b_up(M, draw_w=False)
        check_act(c.X, np.float32(1.0) / c.s.numpy(), 32)


@pytest.mark.parametrize("b", [16, 64, 128])
def test_llama3_8b_up_block_sweep(b):
    c = inputs.llama3_8b_up(128, had_block=b, draw_w=False)
    check_act(c.X, np.float32(1.0) / c.s.numpy(), b)


def test_grouped_small_with_empty_experts():
    g = torch.Generator().manual_seed(9)
    K, E = 256, 6
    offsets = [0, 5, 5, 140, 141, 141, 300]        # experts 1 and 4 empty, one spans two tiles
    X = torch.randn(300, K, generator=g).to(torch.bfloat16)
    inv_s = (1.0 / torch.exp(torch.rand(E, K, generator=g) * 2.77 - 0.69)).to(torch.float32).numpy()
    check_act(X, inv_s, 32, offsets)


@pytest.mark.parametrize("T", [64, 1024])
@pytest.mark.parametrize("proj", ["gate_up", "down"])
def test_moe_grouped_act_quant(T, proj):
    c = inputs.moe_30b_a3b(T, proj, draw_w=False)
    inv_s = (np.float32(1.0) / c.s.numpy()).astype(np.float32)
    check_act(c.X, inv_s, 32, c.offsets.numpy())


def _check_prep(W, s, b):
    N, K = W.shape
    oq, osf, oinv = oracle.prep_weights(W, s, b)
    q = Guarded(N * K // 2, shape=(N, K // 2))
    sf = Guarded(mq.sf_bytes(N, K))
    inv = Guarded(K * 4, dtype=torch.float32) if s is not None else None
    mq.prep_weights(W.cuda(), None if s is None else s.cuda(), b, Wq=q.t, Wsf=sf.t,
                    inv_s=None if inv is None else inv.t)
    torch.cuda.synchronize()
    assert q.intact() and sf.intact() and (inv is None or inv.intact())
    np.testing.assert_array_equal(q.t.cpu().numpy(), oq)
    np.testing.assert_array_equal(unswizzle(sf.t.cpu().numpy(), N, K), osf)
    if s is not None:
        np.testing.assert_array_equal(inv.t.cpu().numpy().view(np.uint32), oinv.view(np.uint32))


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
def test_prep_weights_blocks(b):
    c = inputs.dense_case(900 + b, 1, 512, 384, w_std=0.02)
    _check_prep(c.W, c.s, b)
    _check_prep(c.W, None, b)


def test_prep_weights_llama3_8b_up():
    c = inputs.llama3_8b_up(1)
    _check_prep(c.W, c.s, 32)


def test_repeated_runs_stay_bit_exact():
    """Many tiles per CTA and a congested load queue: stage reuse must never let a TMA refill a
    shared-memory stage before every lane has read it (five repeats of two such workloads)."""
    c = inputs.llama3_8b_up(1)
    oq, osf, _ = oracle.prep_weights(c.W, c.s, 32)
    Wd, sd = c.W.cuda(), c.s.cuda()
    m = inputs.moe_30b_a3b(1024, "gate_up", draw_w=False)
    inv = (np.float32(1.0) / m.s.numpy()).astype(np.float32)
    mq_ref, _ = oracle.act_quant(m.X, inv, 32, offsets=m.offsets.numpy())
    Xd, invd, offd = m.X.cuda(), torch.from_numpy(inv).cuda(), m.offsets.cuda()
    for _ in range(5):
        gq, _, _ = mq.prep_weights(Wd, sd, 32)
        xq, _ = mq.act_quant(Xd, invd, 32, group_offsets=offd)
        torch.cuda.synchronize()
        assert np.array_equal(gq.cpu().numpy(), oq)
        assert np.array_equal(xq.cpu().numpy(), mq_ref)
