"""pa_decode_attention_static: decode attention that allocates nothing.

Some callers may not call cudaMalloc: plugins hosted by a runtime that owns
all device memory through its own pool, and latency-bound loops that cannot
pay cudaMalloc's implicit device synchronisation.  For them the library keeps
the plan and split-K partials in a static device buffer of 32 MiB per GPU.
These tests call the entry point through the C ABI twice in a row (different
workloads, so the second call starts from the first call's leftovers).  Each
result must be bit-identical to pa_decode_attention given a caller workspace
(same plan, same kernels, same merge order, so any leftover from the first
call would show), and must match the fp64 oracle within the parity gate the
other GPU tests use.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_478_b200 as pa
from paged_kv_cache_478_b200 import synthetic as syn
from tests.gpu_cases import assert_parity, dev, workspace_for


def _inputs(case):
    NB, H, BS, D = case["k_pool"].shape
    pool = pa.pa_pool_create(NB, BS, H, D, torch.float16)
    return (pool, dev(case["q"]), dev(case["k_pool"]), dev(case["v_pool"]),
            dev(case["block_tables"]), dev(case["context_lens"]))


def _with_workspace(case, pool, q, kp, vp, bt, cl, partition_size):
    out = torch.empty_like(q)
    ws = workspace_for(pool, q.shape[0], bt.shape[1], 0, partition_size)
    pa.pa_decode_attention(pool, q, kp, vp, bt, cl, case["scale"], out, ws,
                           partition_size=partition_size)
    return out


@pytest.mark.gpu
def test_static_scratch_matches_caller_workspace_on_two_calls_in_a_row():
    cases = [(syn.single_layer_case(seed=21, num_seqs=48), 0),
             (syn.decode_case(22, [1, 17, 300, 2048, 777, 0, 64], 8, 128, np.float16,
                              max_blocks=128), 64)]
    prepared = []
    for case, ps in cases:
        args = _inputs(case)
        want = _with_workspace(case, *args, ps)
        prepared.append((case, ps, args, want))
    torch.cuda.synchronize()
    outs = []
    for case, ps, (pool, q, kp, vp, bt, cl), _ in prepared:  # two calls in a row
        got = torch.empty_like(q)
        pa.pa_decode_attention_static(pool, q, kp, vp, bt, cl, case["scale"], got,
                                      partition_size=ps)
        outs.append(got)
    assert pa.pa_device_errors() == 0
    for i, (got, (case, _, _, want)) in enumerate(zip(outs, prepared)):
        assert torch.equal(got, want), f"call {i}: static buffer differs from a caller workspace"
        ref = oracle.decode_attention(case["q"], case["k_pool"], case["v_pool"],
                                      case["block_tables"], case["context_lens"], case["scale"])
        assert_parity(got, ref, f"static call {i} against the oracle")


def test_an_empty_batch_is_a_no_op_like_the_workspace_call():
    """No sequences: both entry points check the pool and launch nothing
    (host-side, so this runs without a GPU)."""
    pool = pa.pa_pool_create(8, 16, 2, 64, pa.PA_F16)
    p = ctypes.c_void_p(256)
    st = pa.lib().pa_decode_attention_static(ctypes.byref(pool), p, p, p, p, 0, p, 0, 0,
                                             ctypes.c_float(0.1), p, 0, None)
    assert st == pa.PA_OK
    st = pa.lib().pa_decode_attention(ctypes.byref(pool), p, p, p, p, 0, p, 0, 0,
                                      ctypes.c_float(0.1), p, None, 0, 0, None)
    assert st == pa.PA_OK


def test_sizes_beyond_the_static_buffer_are_rejected():
    """Host-side check: nothing is launched, so this runs without a GPU."""
    pool = pa.pa_pool_create(100000, 16, 32, 128, pa.PA_F16)
    need = pa.pa_decode_workspace_bytes(pool, 4096, 128, 0, 16)
    assert need > pa.STATIC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    st = pa.lib().pa_decode_attention_static(ctypes.byref(pool), p, p, p, p, 128, p, 4096, 0,
                                             ctypes.c_float(0.1), p, 16, None)
    assert st == 6  # PA_ERR_WORKSPACE
    msg = pa.lib().pa_last_error().decode()
    assert "static" in msg and str(pa.STATIC_SCRATCH_BYTES) in msg
