"""Failure detection on the GPU without a fault: one bounded device-side wait
is made to run out (an mbarrier nothing arrives on); the host reads the
timeout through sagesla_sync_status, the flag clears, and the context keeps
working (a normal call afterwards still matches the oracle's mask)."""
import pytest
import torch

from tests._util import compare_masks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sg():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as s
    assert torch.cuda.is_available()
    return s


def test_expired_wait_is_reported_and_cleared(sg):
    st = torch.cuda.current_stream()
    assert sg.sync_status(st) == 0
    sg.sagesla_watchdog_selftest(1000, stream=st)
    assert sg.sync_status(st) == -5  # SAGESLA_ERR_DEVICE_TIMEOUT
    assert sg.sync_status(st) == 0   # read once, then cleared


def test_context_usable_after_expired_wait(sg):
    from oracle import oracle as orc
    from sparse_bit_attention_smoothing_b200.inputs import TINY, make_workload
    sg.sagesla_watchdog_selftest(100)
    assert sg.sync_status() == -5
    q, k, v, _ = make_workload(TINY)
    m = sg.sagesla_get_mask(q.cuda(), k.cuda(), block=TINY.block, topk=TINY.topk)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    BH = TINY.B * TINY.H
    qf, kf = q.reshape(BH, TINY.N, 128), k.reshape(BH, TINY.N, 128)
    ref = orc.mask(qf, kf, TINY.block, TINY.topk)
    nb = ref["idx"].shape[1]
    s64 = orc.block_scores_f64(qf, kf, TINY.block)
    got = m["idx"].cpu().numpy().reshape(BH * nb, -1)
    eq, near = compare_masks(got, ref["idx"].reshape(BH * nb, -1), s64.reshape(BH * nb, nb), m["k"])
    assert eq + near == BH * nb
