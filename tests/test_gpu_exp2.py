"""The document pass's polynomial base-2 exponential (FMA pipe) against the
hardware ex2 instruction and against float64, over the range the softmax
feeds it (scaled scores minus a possibly stale maximum: at most +8)."""
import numpy as np
import pytest
import torch

from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_poly_exp2_error_bound():
    m = gu.pp()
    x = torch.cat([torch.linspace(-130.0, 9.0, 1 << 20), torch.tensor([0.0, -0.0, 1.0, -1.0,
                                                                      8.0, -126.0, -125.5])])
    x = x.to(torch.float32).cuda().contiguous()
    yp, yh = m.debug_exp2(x)
    torch.cuda.synchronize()
    xd = x.cpu().double().numpy()
    ref = np.exp2(xd)
    yp, yh = yp.cpu().double().numpy(), yh.cpu().double().numpy()
    assert np.all(np.isfinite(yp)) and np.all(yp >= 0)
    normal = xd >= -125.0
    rel = np.abs(yp[normal] - ref[normal]) / ref[normal]
    assert rel.max() < 1e-4, rel.max()
    # hardware ex2 agrees with float64 far below bf16 resolution as well
    relh = np.abs(yh[normal] - ref[normal]) / ref[normal]
    assert relh.max() < 1e-5
    # the deep negative tail is (near) zero, as masked scores require
    tail = xd < -125.0
    assert np.all(yp[tail] <= 2.0 ** -124)
    # -inf (a masked score) maps to (near) zero on both paths
    z = torch.tensor([-float("inf"), -float("inf")], dtype=torch.float32, device="cuda")
    zp, zh = m.debug_exp2(z)
    assert float(zh.max()) == 0.0 and float(zp.max()) <= 2.0 ** -124
