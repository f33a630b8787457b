"""The polynomial 2^x that the attention kernel uses for a quarter of its
exponentials, checked against the float64 exponential and its stated bound."""
import numpy as np
import pytest
import torch

from chunk_causal_wavefront_b200 import wf as W

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-126.0, 64.0, 1_000_001), rng.uniform(-126, 10, 1_000_000),
                        np.arange(-126, 65, dtype=np.float64), [0.5, -0.5, 1e-7, -1e-7]])
    x = x.astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    yt = torch.empty_like(xt)
    st = W.wf_debug_exp2_poly(xt.data_ptr(), yt.data_ptr(), xt.numel(),
                              torch.cuda.current_stream().cuda_stream)
    assert st == W.WF_OK
    torch.cuda.synchronize()
    y = yt.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 7.6e-5, rel.max()


def test_exp2_poly_underflow_and_masked():
    x = np.array([-126.5, -127.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    xt = torch.from_numpy(x).cuda()
    yt = torch.full_like(xt, 7.0)
    assert W.wf_debug_exp2_poly(xt.data_ptr(), yt.data_ptr(), xt.numel(),
                                torch.cuda.current_stream().cuda_stream) == W.WF_OK
    torch.cuda.synchronize()
    assert (yt.cpu().numpy() == 0.0).all()
