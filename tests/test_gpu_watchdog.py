"""Failure detection on the GPU without a fault.  (1) A bounded wait on an
mbarrier nothing arrives on runs out; the host reads the timeout through
sagesla_sync_status, the flag clears, and the context keeps working (a normal
call afterwards still matches the oracle's mask).  (2) The real sparse flash
kernel, on one CTA with a low probe limit, has one key-tile copy omitted:
its own wait gives up, the CTA winds down, the host reads -5 once, and the
next call is bit-identical to the one before."""
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


def _stall_case():
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    # 2 heads x 16 query blocks (a 40-token tail), k = 4 of 16 key blocks, so
    # one CTA's first pipeline walks 16 query blocks x 2 steps = 32 steps
    q, k, v, _ = make_inputs(1, 2, 1000, 128, seed=21, outliers=True)
    return q.cuda(), k.cuda(), v.cuda()


def test_one_cta_flash_matches_the_persistent_grid(sg):
    """grid = 1: one CTA serves all 32 query blocks through both of its
    pipelines; every query block is computed by the same code in the same
    order, so the output is bit-identical to the normal launch."""
    q, k, v = _stall_case()
    ref = sg.sagesla_attn(q, k, v, None, block=64, topk=0.25)
    one = sg.sagesla_debug_flash_stall(q, k, v, topk=0.25, grid=1, stall_step=-1)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    assert torch.equal(one, ref)


@pytest.mark.parametrize("stall_step", [0, 5, 31])
def test_stalled_flash_pipeline_times_out_and_recovers(sg, stall_step):
    """The K producer omits the copies of one step: the MMA issuer's bounded
    wait on that stage gives up, every role of the CTA stops at its next
    wait, copies and MMAs in flight drain, TMEM is freed and the kernel
    returns.  The host sees the timeout once; the next call is exact."""
    import time
    q, k, v = _stall_case()
    ref = sg.sagesla_attn(q, k, v, None, block=64, topk=0.25)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    t0 = time.perf_counter()
    sg.sagesla_debug_flash_stall(q, k, v, topk=0.25, grid=1, stall_step=stall_step, spin_limit=1 << 14)
    rc = sg.sync_status()
    print(f"stall at step {stall_step}: status {rc} after {1e3 * (time.perf_counter() - t0):.1f} ms")
    assert rc == -5           # SAGESLA_ERR_DEVICE_TIMEOUT
    assert sg.sync_status() == 0
    again = sg.sagesla_attn(q, k, v, None, block=64, topk=0.25)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    assert torch.equal(again, ref)
