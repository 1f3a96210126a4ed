"""GPU parity of the mixture-of-experts routing glue: the gathering activation quantizer (dispatch)
and the weighted top-k combine.

Gather: output row m quantizes X[row_index[m]]; codes and scales must equal the oracle's act_quant of
the gathered copy bit for bit, and equal macaq_act_quant on that copy. Combine: the fp32 weighted sum
in the fixed order is one defined value, so fp32 and bf16 outputs must equal the oracle's bit for bit.
Inputs are the MoE 30B-A3B routing (128 experts, top-8, Zipf popularity) and seeded synthetic rows.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import Guarded, grouped_padding_rows, grouped_sf_rows, sf_index, tile_bases, unswizzle

pytestmark = pytest.mark.gpu


def gather_gpu(X, idx, inv, b, offsets=None):
    M, K = idx.numel(), X.shape[1]
    E = 0 if offsets is None else len(offsets) - 1
    n_sf = mq.grouped_sf_bytes(M, E, K) if offsets is not None else mq.sf_bytes(M, K)
    q = Guarded(max(M * K // 2, 16))
    sf = Guarded(max(n_sf, 16))
    off_d = None if offsets is None else torch.tensor(np.asarray(offsets, np.int32), device="cuda")
    inv_d = None if inv is None else torch.as_tensor(np.ascontiguousarray(inv)).cuda()
    mq.act_quant_gather(X.cuda(), idx.to(torch.int32).cuda(), inv_d, b, group_offsets=off_d,
                        Xq=q.t[:M * K // 2].view(M, K // 2), Xsf=sf.t)
    torch.cuda.synchronize()
    assert q.intact() and sf.intact(), "write outside the output buffers"
    assert mq.device_status() == 0
    return q.t[:M * K // 2].cpu().numpy().reshape(M, K // 2), sf.t.cpu().numpy()


@pytest.mark.parametrize("T", [64, 1024])
def test_gather_dispatch_moe_gate_up(T):
    """MoE 30B-A3B gate/up input: the quantizer reads token rows through the routing's row index."""
    c = inputs.moe_30b_a3b(T, "gate_up", draw_w=False)
    off = c.offsets.numpy()
    inv = (np.float32(1.0) / c.s.numpy()).astype(np.float32)
    oq, osf = oracle.act_quant(c.X_tok[c.routing.token], inv, 32, offsets=off)
    gq, gsf = gather_gpu(c.X_tok, c.routing.token, inv, 32, off)
    np.testing.assert_array_equal(gq, oq)
    K = c.X.shape[1]
    np.testing.assert_array_equal(unswizzle(gsf, off[-1], K, grouped_sf_rows(off)), osf)
    pad = grouped_padding_rows(off)
    assert np.all(gsf[sf_index(pad, K)] == 0)
    # the same bytes as quantizing the materialised expert-sorted copy
    pq, psf = mq.act_quant(c.X.cuda(), torch.from_numpy(inv).cuda(), 32, group_offsets=c.offsets.cuda())
    np.testing.assert_array_equal(pq.cpu().numpy(), gq)
    used = int(tile_bases(off)[-1]) * 128 * (K // 32)   # the tiles the experts own; the rest of the bound is unused
    np.testing.assert_array_equal(psf.cpu().numpy()[:used], gsf[:used])


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
@pytest.mark.parametrize("K", [768, 2048])
def test_gather_dense_blocks_and_clamping(b, K):
    """Dense gather (no groups) with repeated, unordered and out-of-range indices (clamped into X)."""
    g = torch.Generator().manual_seed(700 + b + K)
    x_rows, M = 37, 300
    X = (torch.randn(x_rows, K, generator=g) * torch.exp(torch.randn(K, generator=g))).to(torch.bfloat16)
    idx = torch.randint(0, x_rows, (M,), generator=g)
    idx[:4] = torch.tensor([-5, x_rows, x_rows + 100, 0])
    inv = (1.0 / torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69)).to(torch.float32).numpy()
    clamped = idx.clamp(0, x_rows - 1)
    oq, osf = oracle.act_quant(X[clamped], inv, b)
    gq, gsf = gather_gpu(X, idx, inv, b)
    np.testing.assert_array_equal(gq, oq)
    np.testing.assert_array_equal(unswizzle(gsf, M, K), osf)


def test_gather_empty_and_single_row():
    X = torch.randn(5, 256).to(torch.bfloat16)
    q, sf = gather_gpu(X, torch.tensor([3], dtype=torch.int32), None, 32)
    oq, osf = oracle.act_quant(X[[3]], None, 32)
    np.testing.assert_array_equal(q, oq)
    np.testing.assert_array_equal(unswizzle(sf, 1, 256), osf)
    Xq, Xsf = mq.act_quant_gather(X.cuda(), torch.zeros(0, dtype=torch.int32, device="cuda"), None, 32)
    torch.cuda.synchronize()
    assert Xq.shape == (0, 128)


@pytest.mark.parametrize("T", [64, 1024, 8192])
def test_combine_moe_30b_a3b(T):
    """Weighted top-8 combine of a synthetic down-projection output [8T, 2048] back to token order."""
    c = inputs.moe_30b_a3b(T, "down", draw_w=False)
    r = c.routing
    rows, N = int(c.offsets[-1]), 2048
    g = torch.Generator().manual_seed(T)
    Y = torch.randn(rows, N, generator=g).to(torch.bfloat16)
    ref = oracle.moe_combine(Y, r.pos.numpy(), r.weights.numpy())
    Yd, pd, wd = Y.cuda(), r.pos.cuda(), r.weights.cuda()
    o32 = Guarded(T * N * 4, dtype=torch.float32, shape=(T, N))
    o16 = Guarded(T * N * 2, dtype=torch.bfloat16, shape=(T, N))
    mq.moe_combine(Yd, pd, wd, out_dtype=mq.OUT_F32, out=o32.t)
    mq.moe_combine(Yd, pd, wd, out_dtype=mq.OUT_BF16, out=o16.t)
    torch.cuda.synchronize()
    assert o32.intact() and o16.intact()
    np.testing.assert_array_equal(o32.t.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    np.testing.assert_array_equal(o16.t.cpu().view(torch.int16).numpy().view(np.uint16), oracle.bf16_rne(ref))


def test_combine_dropped_choices_and_odd_topk():
    g = torch.Generator().manual_seed(5)
    rows, N, T, topk = 50, 64, 33, 11
    Y = torch.randn(rows, N, generator=g).to(torch.bfloat16)
    pos = torch.randint(0, rows, (T, topk), generator=g).to(torch.int32)
    pos[::3, 4] = -1
    pos[1, 10] = rows
    w = torch.randn(T, topk, generator=g).to(torch.float32)
    ref = oracle.moe_combine(Y, pos.numpy(), w.numpy())
    got = mq.moe_combine(Y.cuda(), pos.cuda(), w.cuda(), out_dtype=mq.OUT_F32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy().view(np.uint32), ref.view(np.uint32))
