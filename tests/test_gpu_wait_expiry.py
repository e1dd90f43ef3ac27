"""The bounded-wait path every kernel uses on its mbarriers: a wait on a
barrier that nothing completes gives up after its cycle budget, the device
error word reports TQ_ERR_TIMEOUT at tq_sync_check (once; the word is
cleared), and the context keeps running kernels afterwards."""
import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import assert_close_rel

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_bounded_wait_expiry_reports_timeout_and_context_survives():
    tq.tq_sync_check()  # start from a clear error word
    tq.tq_check_wait_expiry(1 << 22)  # about 2 ms of polling, then give up
    with pytest.raises(tq.TQError, match="TIMEOUT"):
        tq.tq_sync_check()
    tq.tq_sync_check()  # reported once, then cleared
    # kernels still run and still match the oracle
    dr = synth.method_draws(128, 128, 3, stream=2)
    ora = o.Quantizer(128, 3, prod=False, draws=dr)
    lib = tq.TQParams(128, 3, tq.MODE_MSE, tq.ROT_HADAMARD, signs=dr["signs"])
    x = synth.gaussian_vectors(256, 128, seed=5, dtype="float16", device=DEV)
    codes, norms = tq.tq_encode_mse(lib, x)
    torch.cuda.synchronize()
    tq.tq_sync_check()
    e = ora.encode(x.float().cpu().numpy().astype(np.float64))
    assert_close_rel(norms.cpu().numpy(), e["norms"], 1e-30, what="norms")
