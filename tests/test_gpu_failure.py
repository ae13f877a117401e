"""Failure detection on the GPU without a fault: every device spin-wait of the
library has a time limit, after which the kernel records a timeout in the
device error word and returns.  Here a wait that nothing can satisfy runs
out under a 20 ms limit; the host reads NVFP4SK_ERR_TIMEOUT with the wait's
site, and the same context then runs a normal op correctly."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda, to_dev
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives(oracle):
    cuda()
    nv.device_status()                                      # clear
    old = nv.get_option(nv.OPT_TIMEOUT_NS)
    try:
        nv.set_option(nv.OPT_TIMEOUT_NS, 20_000_000)        # 20 ms
        L = nv.load()
        assert L.nvfp4sk_debug_wait_timeout(torch.cuda.current_stream().cuda_stream) == 0
        rc, site = nv.device_status()
        assert (rc, site) == (-6, 900)
        assert b"ran out" in L.nvfp4sk_last_error()
    finally:
        nv.set_option(nv.OPT_TIMEOUT_NS, old)
    # the context is intact: a quantisation after the timeout is bit-exact
    x = inputs.activation_bf16(95, 0, 16, 2048)
    codes, scales, g = nv.quantize(to_dev(x))
    w_codes, w_scales, w_g = oracle.quantize(x.float().numpy())
    assert np.array_equal(codes.cpu().numpy(), w_codes)
    assert np.array_equal(scales.cpu().numpy(), w_scales)
    assert nv.device_status()[0] == 0
