"""Failure detection on the device: a bounded pipeline wait that runs out.

The quantizer's producer waits a bounded time for a free stage.  Test support
lowers that one limit far below a stage's compute time, so the wait gives up
during an ordinary call; nothing faults and no wait is endless: the producer
stops issuing, lets its issued loads land (the drain keeps the normal bound),
and the compute warps see the abort flag and leave their loop.  The host then
reads UFP4_ERR_DEVICE_TIMEOUT once from ufp4_check_device_status, and with
the limit restored the next call is clean and matches the oracle."""
import numpy as np
import torch

import oracle
from fp4_quantized_gemms_b200 import ufp4
from fp4_quantized_gemms_b200 import workloads as wl
from tests.gpu_util import assert_quant_equal, needs_gpu, oracle_cfg, to_dev

pytestmark = needs_gpu


def test_quantizer_wait_timeout_is_reported_once_then_calls_recover():
    # 8192 x 4096 along the columns: 2048 work units, several per CTA, so the
    # producer must wait for stages to come free.
    X = wl.normal(8192, 4096, 1.0, 7)
    x = to_dev(X)
    cfg = ufp4.QuantConfig(grid=ufp4.GRID_E1M2, rounding=ufp4.ROUND_SR, sr_seed=1234, hadamard_n=16,
                           block=16, scale_fmt=ufp4.SCALE_FP32)
    assert ufp4.check_device_status() == ufp4.OK
    ref = ufp4.rht_quantize(x, ufp4.ALONG_COLS, cfg)
    assert ufp4.check_device_status() == ufp4.OK
    q = ufp4.empty_qtensor(8192, 4096, cfg)
    try:
        ufp4.set_quantize_wait_limit_for_tests(1)
        ufp4.rht_quantize(x, ufp4.ALONG_COLS, cfg, out=q)      # launches fine, gives up on the device
        assert ufp4.check_device_status() == ufp4.ERR_DEVICE_TIMEOUT
        assert ufp4.check_device_status() == ufp4.OK            # reported once, then cleared
    finally:
        ufp4.set_quantize_wait_limit_for_tests(0)
    ufp4.rht_quantize(x, ufp4.ALONG_COLS, cfg, out=q)
    assert ufp4.check_device_status() == ufp4.OK
    assert torch.equal(q.codes, ref.codes) and torch.equal(q.scales, ref.scales)
    rows = [0, 1, 255, 4096, 8191]
    oc = oracle_cfg(cfg)
    refs = [oracle.quantize(X, ufp4.ALONG_COLS, oc, r0=r, nr=1) for r in rows]
    want = refs[0]
    want.codes = np.concatenate([r.codes for r in refs])
    want.scales = np.concatenate([r.scales for r in refs])
    assert_quant_equal(q, want, rows)
