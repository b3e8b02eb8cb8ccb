"""A planned decode launch trusts nothing in its workspace that it has not
checked on the device.

The work plan (items, per-sequence lengths and partition counts, merge
counters) lives in caller-owned memory, and a workspace can lose its plan
without the library knowing: freed and handed out again by an allocator,
overwritten by other work, or zeroed.  Every plan carries a stamp that the
launches given it must find in the header; every entry a launch uses is
bounds-checked before it indexes the block table, the partials or the
output ("PagedAttention", e-fortepiano.pl wiki mirror, "Descripció": the
block table is the only indirection the method needs, and every access stays
inside the sequence's own blocks).  A launch that cannot trust the plan
raises PA_DEVERR_PLAN and skips the work; the context stays usable and a new
plan runs normally.

Plan header layout (offset 0 of the workspace): num_pairs, num_items,
work_counter, done_counter (int32 each), stamp (uint64, bytes 16-23),
poisoned (int32, bytes 24-27); the per-sequence arrays start at byte 256.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_478_b200 as pa
from paged_kv_cache_478_b200 import synthetic as syn
from tests.gpu_cases import assert_parity, dev, workspace_for

pytestmark = pytest.mark.gpu

LENS = [40, 300, 17, 129, 1000, 1, 64, 513]
PS = 64  # several partitions per long sequence, so merges run


def _case(group):
    """Group 1 runs the CUDA-core kernel, groups 2 and 4 the tensor-core one."""
    H = 4
    case = syn.decode_case(7, LENS, heads=H, head_dim=128, dtype=np.float16)
    rng = np.random.default_rng(8)
    case["q"] = rng.standard_normal((len(LENS), H * group, 128)).astype(np.float16)
    NB, H, BS, D = case["k_pool"].shape
    pool = pa.pa_pool_create(NB, BS, H, D, torch.float16)
    if group > 1:
        pa.pa_pool_set_query_heads(pool, H * group)
    t = dict(pool=pool, q=dev(case["q"]), kp=dev(case["k_pool"]), vp=dev(case["v_pool"]),
             bt=dev(case["block_tables"]), cl=dev(case["context_lens"]))
    t["ws"] = workspace_for(pool, len(LENS), t["bt"].shape[1], partition_size=PS)
    ref = oracle.decode_attention(case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                                  case["context_lens"], case["scale"])
    return case, t, ref


def _plan(case, t):
    pa.pa_decode_plan(t["pool"], t["cl"], t["bt"].shape[1], t["ws"], partition_size=PS)


def _run(case, t, out):
    pa.pa_decode_attention_planned(t["pool"], t["q"], t["kp"], t["vp"], t["bt"], case["scale"],
                                   out, t["ws"], partition_size=PS)
    return pa.pa_device_errors()


def _replan_and_check(case, t, ref):
    """After a refused launch the context is usable and a new plan runs."""
    _plan(case, t)
    out = torch.empty_like(t["q"])
    assert _run(case, t, out) == 0
    assert_parity(out, ref, "after a new plan")


@pytest.mark.parametrize("group", [1, 2, 4])
def test_a_workspace_that_lost_its_plan_is_refused(group):
    case, t, ref = _case(group)
    _plan(case, t)
    torch.cuda.synchronize()
    t["ws"].zero_()  # the host still records a plan at this address; the memory no longer holds it
    out = torch.full_like(t["q"], 7.0)
    assert _run(case, t, out) == pa.PA_DEVERR_PLAN
    assert bool((out == 7.0).all()), "a refused launch wrote its output"
    assert not bool(t["ws"].any()), "a refused launch wrote into the workspace"
    _replan_and_check(case, t, ref)


@pytest.mark.parametrize("group", [1, 2, 4])
@pytest.mark.parametrize("byte", [0x7F, 0xFF])
def test_damaged_plan_entries_are_skipped(group, byte):
    """Header intact, every per-sequence entry replaced: 0x7f7f7f7f and -1
    both name no sequence, so every item is skipped and nothing is written."""
    case, t, ref = _case(group)
    _plan(case, t)
    torch.cuda.synchronize()
    t["ws"][256:].fill_(byte)
    out = torch.full_like(t["q"], 7.0)
    assert _run(case, t, out) == pa.PA_DEVERR_PLAN
    assert bool((out == 7.0).all())
    _replan_and_check(case, t, ref)


@pytest.mark.parametrize("group", [1, 2, 4])
def test_random_plan_entries_stay_in_bounds(group):
    """Header intact, the rest random: whatever entries pass the checks index
    only inside the caller's buffers (the result is then meaningless, which
    the error bit reports)."""
    case, t, ref = _case(group)
    _plan(case, t)
    torch.cuda.synchronize()
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    body = t["ws"][256:]
    body.copy_(torch.randint(0, 256, body.shape, dtype=torch.uint8, device="cuda", generator=g))
    out = torch.empty_like(t["q"])
    flags = _run(case, t, out)
    assert flags & pa.PA_DEVERR_PLAN
    assert flags & ~pa.PA_DEVERR_PLAN == 0  # the block tables themselves were never at fault
    _replan_and_check(case, t, ref)


@pytest.mark.parametrize("group", [1, 2, 4])
def test_a_poisoned_plan_is_refused_until_rewritten(group):
    """A launch that gives up on a wait marks its plan, since the merge
    counters may then be stale.  Set the mark by hand: the next launch on the
    plan is refused, and pa_decode_plan clears it."""
    case, t, ref = _case(group)
    _plan(case, t)
    torch.cuda.synchronize()
    t["ws"][24:28].copy_(torch.tensor([1, 0, 0, 0], dtype=torch.uint8))
    out = torch.full_like(t["q"], 7.0)
    assert _run(case, t, out) == pa.PA_DEVERR_PLAN
    assert bool((out == 7.0).all())
    _replan_and_check(case, t, ref)


def test_a_plan_left_by_an_earlier_call_does_not_pass_for_a_new_one():
    """Two plans at the same address: launches run only on the newest."""
    case, t, ref = _case(1)
    _plan(case, t)
    torch.cuda.synchronize()
    old = t["ws"].clone()
    _plan(case, t)  # a new stamp
    torch.cuda.synchronize()
    t["ws"].copy_(old)  # the memory now holds the earlier plan
    out = torch.full_like(t["q"], 7.0)
    assert _run(case, t, out) == pa.PA_DEVERR_PLAN
    assert bool((out == 7.0).all())
    _replan_and_check(case, t, ref)
