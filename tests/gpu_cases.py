"""Shared plumbing for the GPU parity tests: device copies, the parity gate,
and one-call wrappers that run the CUDA path and the oracle on the same
seeded inputs.  The CUDA side goes through the C ABI only; the oracle side
through oracle/ only."""
import numpy as np
import torch

import oracle
import paged_kv_cache_478_b200 as pa

ATOL, RTOL = 2e-3, 1e-2  # parity gate for fp16/bf16/fp32 outputs against the fp64 oracle

TORCH_DTYPE = {np.dtype(np.float32): torch.float32, np.dtype(np.float16): torch.float16}


def dev(a):
    if a.dtype == np.int32:
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def bits(a):
    """Raw bit patterns of a numpy or torch array, for exact comparisons."""
    if isinstance(a, torch.Tensor):
        a = host(a.contiguous().view(torch.int16 if a.element_size() == 2 else torch.int32))
    else:
        a = a.view(np.int16 if a.itemsize == 2 else np.int32)
    return a


def assert_parity(gpu, ref, what=""):
    g = gpu.detach().float().cpu().numpy().astype(np.float64) if isinstance(gpu, torch.Tensor) else gpu
    ok = np.abs(g - ref) <= ATOL + RTOL * np.abs(ref)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        err = np.max(np.abs(g - ref))
        raise AssertionError(f"{what}: {int((~ok).sum())} elements outside the gate, max|err| "
                             f"{err:.3e}, first {idx.tolist()}")
    return float(np.max(np.abs(g - ref))) if g.size else 0.0


def workspace_for(pool, num_seqs, max_blocks, max_context_len=0, partition_size=0):
    n = pa.pa_decode_workspace_bytes(pool, num_seqs, max_blocks, max_context_len, partition_size)
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def gpu_append_and_decode(case, partition_size=0, max_context_len=0, check_errors=True):
    """CUDA path on a decode_case: reshape_and_cache of the new token (slots
    from the library's host helper), then decode attention.  Returns
    (out, k_pool, v_pool) as device tensors."""
    q = dev(case["q"])
    kp, vp = dev(case["k_pool"]), dev(case["v_pool"])
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    NB, H, BS, D = case["k_pool"].shape
    pool = pa.pa_pool_create(NB, BS, H, D, q.dtype)
    slots = dev(pa.pa_decode_slots(case["block_tables"], case["context_lens"]))
    pa.pa_reshape_and_cache(pool, dev(case["k_new"]), dev(case["v_new"]), slots, kp, vp)
    out = torch.empty_like(q)
    ws = workspace_for(pool, q.shape[0], bt.shape[1], max_context_len, partition_size)
    pa.pa_decode_attention(pool, q, kp, vp, bt, cl, case["scale"], out, ws,
                           max_context_len=max_context_len, partition_size=partition_size)
    if check_errors:
        assert pa.pa_device_errors() == 0
    return out, kp, vp


def oracle_append_and_decode(case):
    """Oracle on the same case: host reshape_and_cache (slots from the
    oracle's own slot_of) then fp64 attention.  Returns (out, k_pool, v_pool)."""
    kp, vp = case["k_pool"].copy(), case["v_pool"].copy()
    slots = np.array([oracle.slot_of_c(case["block_tables"][s], int(L) - 1) if L > 0 else -1
                      for s, L in enumerate(case["context_lens"])], dtype=np.int32)
    oracle.reshape_and_cache(case["k_new"], case["v_new"], slots, kp, vp)
    out = oracle.decode_attention(case["q"], kp, vp, case["block_tables"], case["context_lens"],
                                  case["scale"])
    return out, kp, vp
