"""Failure detection without a GPU fault: a pipeline wait that runs out of
time is reported through the device error word, the context stays usable,
and a later call works.  The wait that expires is the same bounded mbarrier
wait every kernel of the library uses, given a 1 ms limit."""

import pytest
import torch

from gpu_helpers import TOL, max_err, run_gpu, run_oracle
from mixed_precision_attention_tm_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives():
    assert ops.get_device_error() == ops.TM_OK
    ops.selftest_wait_timeout(1_000_000)          # 1 ms
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_ERR_TIMEOUT
    assert ops.get_device_error() == ops.TM_OK    # reading clears it
    w = inputs.tiny(seed=3, p=0.5)
    out, m, _ = run_gpu(w)
    assert max_err(out, run_oracle(w, m.numpy().view("uint32"))) <= TOL


def test_sequence_longer_than_max_seqlen_is_reported():
    cu = torch.tensor([0, 300, 700], dtype=torch.int32)
    q = inputs.randn_f16((700, 2, 128), 1).cuda()
    k = inputs.randn_f16((700, 1, 128), 2).cuda()
    v = inputs.randn_f16((700, 1, 128), 3).cuda()
    ops.attn_fwd(q, k, v, causal=True, cu_seqlens=cu.cuda(), max_seqlen=256)   # second sequence has 400
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_ERR_INVALID_ARG
    assert ops.get_device_error() == ops.TM_OK
