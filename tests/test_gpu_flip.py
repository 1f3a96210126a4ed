"""GPU parity of Flip-Refinement (macaq_flip_refine): the refined codes and the per-row move counts
must equal the oracle's bit for bit. The Hessian is X'^T X' / M of seeded calibration rows X
transformed as the activations are (oracle transform, float64 product, rounded to fp32 once), the
same array on both sides. Shapes cover every rows-per-CTA variant (K up to 2048, 4096, 8192 and
16384), every Hadamard block size, with and without s, and one and two sweeps."""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import unswizzle

pytestmark = pytest.mark.gpu


def case(seed, N, K, b, with_s, M=256):
    c = inputs.dense_case(seed, M, K, N, w_std=0.02, n_outliers=max(1, K // 256), outlier_factor=20.0)
    s = c.s if with_s else None
    inv = None if s is None else (np.float32(1.0) / s.numpy()).astype(np.float32)
    Xt = oracle.transform_rows(c.X, inv, b, absorb=False).astype(np.float64)
    H = (Xt.T @ Xt / M).astype(np.float32)
    return c.W, s, H


@pytest.mark.parametrize("N,K,b,sweeps,with_s,checked", [
    (128, 256, 32, 1, True, 128), (256, 1024, 64, 2, True, 256), (128, 2048, 128, 1, False, 128),
    (128, 4096, 32, 2, True, 128), (128, 8192, 16, 1, True, 16), (128, 16384, 1, 1, False, 4),
])
def test_flip_refine_matches_oracle(N, K, b, sweeps, with_s, checked):
    """Rows are refined independently, so for the largest K the oracle (O(K^2) per row) checks the
    first `checked` rows of the GPU's result."""
    W, s, H = case(N + K + b, N, K, b, with_s)
    oWq, oWsf, _ = oracle.prep_weights(W[:checked], s, b)
    ref_q, ref_flips = oracle.flip_refine(W[:checked], s, b, H, sweeps, oWq, oWsf)
    gWq, gWsf, _ = mq.prep_weights(W.cuda(), None if s is None else s.cuda(), b)
    np.testing.assert_array_equal(gWq.cpu().numpy()[:checked], oWq)
    np.testing.assert_array_equal(unswizzle(gWsf.cpu().numpy(), checked, K), oWsf)
    flips = mq.flip_refine(W.cuda(), None if s is None else s.cuda(), torch.from_numpy(H).cuda(), gWq, gWsf,
                           had_block=b, sweeps=sweeps)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    np.testing.assert_array_equal(flips.cpu().numpy()[:checked], ref_flips)
    np.testing.assert_array_equal(gWq.cpu().numpy()[:checked], ref_q)
    assert int(ref_flips.sum()) > 0, "the case moves no code: it would not test the updates"


def test_flip_refine_no_op_cases():
    """sweeps = 0 and a diagonal Hessian leave the prepared codes untouched."""
    W, s, H = case(7, 128, 512, 32, True)
    gWq, gWsf, _ = mq.prep_weights(W.cuda(), s.cuda(), 32)
    before = gWq.clone()
    mq.flip_refine(W.cuda(), s.cuda(), torch.from_numpy(H).cuda(), gWq, gWsf, had_block=32, sweeps=0)
    D = torch.diag(torch.from_numpy(np.diag(H).copy())).cuda()
    flips = mq.flip_refine(W.cuda(), s.cuda(), D, gWq, gWsf, had_block=32, sweeps=2)
    torch.cuda.synchronize()
    assert torch.equal(gWq, before)
    assert int(flips.sum()) == 0
