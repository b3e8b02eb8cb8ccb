"""CUDA path against the fp64 oracle on the same seeded inputs.

Parity gate for attention outputs: |gpu - oracle| <= 2e-3 + 1e-2 |oracle|,
elementwise.  Pools after reshape_and_cache / copy_blocks, block tables,
slots and copy pairs must be bit-exact.  The paging invariants of
"PagedAttention" (wiki mirror, "Descripció" and "Formulació matemàtica";
7minutos.es sections 2-3) are checked bit for bit on the GPU: physical
placement, shared versus private prefix, copy-on-write isolation.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_478_b200 as pa
from paged_kv_cache_478_b200 import synthetic as syn
from tests.gpu_cases import (assert_parity, bits, dev, gpu_append_and_decode, host,
                             oracle_append_and_decode, workspace_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if torch.cuda.is_available():
        pa.pa_device_errors()
    yield


# ---- configuration 1: tiny, fp32, head_dim 64 --------------------------------------

@pytest.mark.parametrize("partition_size", [0, 16, 32, 48, 4096])
def test_tiny_config(partition_size):
    case = syn.tiny_case(seed=0)
    out, kp, vp = gpu_append_and_decode(case, partition_size=partition_size)
    ref, kref, vref = oracle_append_and_decode(case)
    assert np.array_equal(bits(kp), bits(kref)) and np.array_equal(bits(vp), bits(vref))
    err = assert_parity(out, ref, "tiny")
    assert err < 1e-5  # fp32 data: error is rounding-level


# ---- configuration 2: one GPT-style layer --------------------------------------------

def test_single_layer_config():
    case = syn.single_layer_case(seed=0)
    out, kp, vp = gpu_append_and_decode(case)
    ref, kref, vref = oracle_append_and_decode(case)
    assert np.array_equal(bits(kp), bits(kref)) and np.array_equal(bits(vp), bits(vref))
    assert_parity(out, ref, "single layer")


# ---- lengths, dtypes, head counts ----------------------------------------------------

EDGE_LENGTHS = [0, 1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257, 511, 512, 513, 777, 1024, 2048]


def _bf16_case(case):
    """Round a float32 case to bfloat16; the oracle reads the bit patterns."""
    out = dict(case)
    for k in ("q", "k_new", "v_new", "k_pool", "v_pool"):
        t = torch.from_numpy(case[k]).to(torch.bfloat16)
        out[k + "_t"] = t
        out[k] = t.view(torch.int16).numpy().view(np.uint16)
    return out


@pytest.mark.parametrize("dtype,head_dim", [(np.float16, 128), (np.float16, 64),
                                            (np.float32, 128), (np.float32, 64),
                                            ("bf16", 128), ("bf16", 64)])
@pytest.mark.parametrize("partition_size", [0, 64])
def test_edge_lengths(dtype, head_dim, partition_size):
    heads = 6  # not a multiple of the 4 heads a CTA serves
    base_dtype = np.float32 if dtype == "bf16" else dtype
    case = syn.decode_case(11, EDGE_LENGTHS, heads, head_dim, base_dtype, max_blocks=130)
    if dtype == "bf16":
        case = _bf16_case(case)
        q = case["q_t"].cuda()
        kp, vp = case["k_pool_t"].cuda(), case["v_pool_t"].cuda()
        k_new, v_new = case["k_new_t"].cuda(), case["v_new_t"].cuda()
    else:
        q, kp, vp = dev(case["q"]), dev(case["k_pool"]), dev(case["v_pool"])
        k_new, v_new = dev(case["k_new"]), dev(case["v_new"])
    NB = kp.shape[0]
    pool = pa.pa_pool_create(NB, 16, heads, head_dim, q.dtype)
    slots = dev(pa.pa_decode_slots(case["block_tables"], case["context_lens"]))
    pa.pa_reshape_and_cache(pool, k_new, v_new, slots, kp, vp)
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    out = torch.empty_like(q)
    ws = workspace_for(pool, q.shape[0], bt.shape[1], 0, partition_size)
    pa.pa_decode_attention(pool, q, kp, vp, bt, cl, case["scale"], out, ws,
                           partition_size=partition_size)
    assert pa.pa_device_errors() == 0
    ref, kref, vref = oracle_append_and_decode_any(case, dtype)
    assert np.array_equal(bits(kp), bits(kref)) and np.array_equal(bits(vp), bits(vref))
    assert_parity(out, ref, f"edge {dtype} D={head_dim}")
    # the empty sequence gives zeros; length one gives its V exactly
    o = out.float().cpu().numpy()
    assert np.array_equal(o[0], np.zeros_like(o[0]))
    assert np.array_equal(bits(out[1]), bits(v_new[1]))


def oracle_append_and_decode_any(case, dtype):
    if dtype != "bf16":
        return oracle_append_and_decode(case)
    kp, vp = case["k_pool"].copy(), case["v_pool"].copy()
    slots = np.array([oracle.slot_of_c(case["block_tables"][s], int(L) - 1) if L > 0 else -1
                      for s, L in enumerate(case["context_lens"])], dtype=np.int32)
    oracle.reshape_and_cache(case["k_new"], case["v_new"], slots, kp, vp)
    out = oracle.decode_attention(case["q"], kp, vp, case["block_tables"], case["context_lens"],
                                  case["scale"], dtype=oracle.BF16)
    return out, kp, vp


# ---- the kernel reads nothing outside the valid tokens ---------------------------------

def test_nan_outside_valid_tokens_is_never_read():
    lens = [1, 7, 16, 17, 100, 300]
    case = syn.decode_case(5, lens, 4, 128, np.float16, pool_fill="nan", num_pool_blocks=64,
                           max_blocks=32)
    # the cached tokens (all but the new one) get finite values through the oracle's scatter
    rng = np.random.default_rng(9)
    for s, L in enumerate(lens):
        prev = np.array([oracle.slot_of_c(case["block_tables"][s], t) for t in range(L - 1)],
                        dtype=np.int32)
        kn = rng.standard_normal((len(prev), 4, 128)).astype(np.float16)
        vn = rng.standard_normal((len(prev), 4, 128)).astype(np.float16)
        oracle.reshape_and_cache(kn, vn, prev, case["k_pool"], case["v_pool"])
    bt = case["block_tables"].copy()
    bt[bt < 0] = 2 ** 30  # entries past the last block are garbage and must not be read
    case["block_tables"] = bt
    out, _, _ = gpu_append_and_decode(case, partition_size=32)
    ref, _, _ = oracle_append_and_decode(case)
    assert np.isfinite(ref).all()
    assert torch.isfinite(out).all()
    assert_parity(out, ref, "nan-poisoned pool")


# ---- invariances, bit for bit -------------------------------------------------------------

def _logical_case(seed, lens, heads=8, head_dim=128):
    """Same logical K/V per sequence, laid out under two different placements."""
    rng = np.random.default_rng(seed)
    K = [rng.standard_normal((L, heads, head_dim)).astype(np.float16) for L in lens]
    V = [rng.standard_normal((L, heads, head_dim)).astype(np.float16) for L in lens]
    q = rng.standard_normal((len(lens), heads, head_dim)).astype(np.float16)
    return q, K, V


def _place(q, K, V, perm_seed, nb):
    """Scatter the logical tokens into a pool through the oracle's scatter,
    with block ids from a seeded permutation."""
    lens = [k.shape[0] for k in K]
    heads, D = q.shape[1], q.shape[2]
    need = [math.ceil(L / 16) for L in lens]
    perm = np.random.default_rng(perm_seed).permutation(nb).astype(np.int32)
    bt = np.full((len(lens), max(need)), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(need):
        bt[s, :n] = perm[pos:pos + n]
        pos += n
    kp = np.zeros((nb, heads, 16, D), dtype=np.float16)
    vp = np.zeros_like(kp)
    for s, L in enumerate(lens):
        slots = np.array([oracle.slot_of_c(bt[s], t) for t in range(L)], dtype=np.int32)
        oracle.reshape_and_cache(K[s], V[s], slots, kp, vp)
    return kp, vp, bt, np.array(lens, dtype=np.int32)


def _decode(q, kp, vp, bt, cl, partition_size=0):
    pool = pa.pa_pool_create(kp.shape[0], 16, q.shape[1], q.shape[2], torch.float16)
    qd, kd, vd, btd, cld = dev(q), dev(kp), dev(vp), dev(bt), dev(cl)
    out = torch.empty_like(qd)
    ws = workspace_for(pool, q.shape[0], bt.shape[1], 0, partition_size)
    pa.pa_decode_attention(pool, qd, kd, vd, btd, cld, 1 / math.sqrt(q.shape[2]), out, ws,
                           partition_size=partition_size)
    assert pa.pa_device_errors() == 0
    return out


@pytest.mark.parametrize("partition_size", [0, 16, 128])
def test_placement_invariance_is_bit_exact(partition_size):
    lens = [1, 16, 33, 200, 511, 1300]
    q, K, V = _logical_case(1, lens)
    nb = sum(math.ceil(L / 16) for L in lens) + 17
    a = _decode(q, *_place(q, K, V, 0, nb), partition_size)
    b = _decode(q, *_place(q, K, V, 1, nb), partition_size)
    assert torch.equal(a, b)
    ref = oracle.decode_attention(q, *_place(q, K, V, 0, nb), 1 / math.sqrt(128))
    assert_parity(a, ref, "placement")


def test_run_to_run_bit_stable_and_partitions_agree():
    case = syn.single_layer_case(seed=3, num_seqs=16)
    ref, _, _ = oracle_append_and_decode(case)
    outs = {}
    for ps in (0, 16, 64, 512, 2048):
        o1, _, _ = gpu_append_and_decode(case, partition_size=ps)
        o2, _, _ = gpu_append_and_decode(case, partition_size=ps)
        assert torch.equal(o1, o2), f"partition {ps} not bit-stable"
        assert_parity(o1, ref, f"partition {ps}")
        outs[ps] = o1


# ---- device-side bounds checks -----------------------------------------------------------

def test_bad_block_id_is_flagged_not_read():
    case = syn.decode_case(2, [40, 20], 4, 64, np.float16, num_pool_blocks=8)
    case["block_tables"][0, 1] = 1000  # outside the 8-block pool
    out, _, _ = gpu_append_and_decode(case, check_errors=False)
    flags = pa.pa_device_errors()
    assert flags & pa.PA_DEVERR_BLOCK_ID


def test_context_len_above_the_bound_is_flagged():
    case = syn.decode_case(2, [40, 20], 4, 64, np.float16, num_pool_blocks=8, max_blocks=3)
    q, kp, vp = dev(case["q"]), dev(case["k_pool"]), dev(case["v_pool"])
    bt = dev(case["block_tables"])
    cl = dev(np.array([40, 49], dtype=np.int32))  # 49 > 3 blocks * 16
    pool = pa.pa_pool_create(8, 16, 4, 64, torch.float16)
    out = torch.empty_like(q)
    ws = workspace_for(pool, 2, 3)
    pa.pa_decode_attention(pool, q, kp, vp, bt, cl, 0.125, out, ws)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN
    # a max_context_len below the real length is flagged too
    ws = workspace_for(pool, 2, 3, max_context_len=32)
    pa.pa_decode_attention(pool, q, kp, vp, bt, dev(case["context_lens"]), 0.125, out, ws,
                           max_context_len=32)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN


def test_reshape_and_cache_slots():
    H, D = 4, 128
    kp = torch.zeros((6, H, 16, D), dtype=torch.float16, device="cuda")
    vp = torch.zeros_like(kp)
    pool = pa.pa_pool_create(6, 16, H, D, torch.float16)
    rng = np.random.default_rng(0)
    kn = rng.standard_normal((5, H, D)).astype(np.float16)
    vn = rng.standard_normal((5, H, D)).astype(np.float16)
    slots = np.array([17, -1, 95, 0, 40], dtype=np.int32)
    pa.pa_reshape_and_cache(pool, dev(kn), dev(vn), dev(slots), kp, vp)
    assert pa.pa_device_errors() == 0
    kref = np.zeros((6, H, 16, D), dtype=np.float16)
    vref = np.zeros_like(kref)
    oracle.reshape_and_cache(kn, vn, slots, kref, vref)
    assert np.array_equal(bits(kp), bits(kref)) and np.array_equal(bits(vp), bits(vref))
    pa.pa_reshape_and_cache(pool, dev(kn[:1]), dev(vn[:1]), dev(np.array([96], np.int32)), kp, vp)
    assert pa.pa_device_errors() & pa.PA_DEVERR_SLOT
    assert np.array_equal(bits(kp), bits(kref))  # the bad slot wrote nothing


def test_copy_blocks_bit_exact_and_bad_pair_flagged():
    rng = np.random.default_rng(4)
    kh = rng.standard_normal((12, 32, 16, 128)).astype(np.float16)
    vh = rng.standard_normal((12, 32, 16, 128)).astype(np.float16)
    kp, vp = dev(kh), dev(vh)
    pool = pa.pa_pool_create(12, 16, 32, 128, torch.float16)
    pairs = np.array([[3, 10], [0, 11], [7, 1]], dtype=np.int32)
    pa.pa_copy_blocks(pool, kp, vp, dev(pairs))
    assert pa.pa_device_errors() == 0
    oracle.copy_blocks(kh, vh, pairs)
    assert np.array_equal(bits(kp), bits(kh)) and np.array_equal(bits(vp), bits(vh))
    pa.pa_copy_blocks(pool, kp, vp, dev(np.array([[2, 12]], dtype=np.int32)))
    assert pa.pa_device_errors() & pa.PA_DEVERR_PAIR
    assert np.array_equal(bits(kp), bits(kh))


def test_wait_limit_reports_a_timeout_and_the_context_survives():
    pa.pa_selftest_wait_timeout()
    flags = pa.pa_device_errors()
    assert flags & pa.PA_DEVERR_TIMEOUT
    # the context is still usable afterwards
    case = syn.tiny_case(seed=1)
    out, _, _ = gpu_append_and_decode(case)
    ref, _, _ = oracle_append_and_decode(case)
    assert_parity(out, ref, "after timeout")


def test_planned_call_refuses_arguments_that_differ_from_the_plan():
    """A planned call reads the work items, partial slots and merge counters the
    plan laid out; with other partition or length bounds it is refused on the
    host instead of running on a layout it does not match."""
    case = syn.decode_case(5, [40, 300, 17, 129], heads=2, head_dim=64, dtype=np.float16)
    NB, H, BS, D = case["k_pool"].shape
    pool = pa.pa_pool_create(NB, BS, H, D, torch.float16)
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    kp, vp, q = dev(case["k_pool"]), dev(case["v_pool"]), dev(case["q"])
    ws = workspace_for(pool, 4, bt.shape[1], partition_size=32)  # large enough for both
    out = torch.empty_like(q)
    pa.pa_decode_plan(pool, cl, bt.shape[1], ws, partition_size=128)
    with pytest.raises(pa.PagedAttnError, match="differ"):
        pa.pa_decode_attention_planned(pool, q, kp, vp, bt, case["scale"], out, ws,
                                       partition_size=32)
    with pytest.raises(pa.PagedAttnError, match="differ"):
        pa.pa_decode_attention_planned(pool, q, kp, vp, bt, case["scale"], out, ws,
                                       max_context_len=160, partition_size=128)
    pa.pa_decode_attention_planned(pool, q, kp, vp, bt, case["scale"], out, ws, partition_size=128)
    assert pa.pa_device_errors() == 0
    ref = oracle.decode_attention(case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                                  case["context_lens"], case["scale"])
    assert_parity(out, ref, "planned call matching its plan")


def test_plan_once_run_many_layers_matches_single_calls():
    """One plan serves several layers that share lengths and tables."""
    case = syn.single_layer_case(seed=4, num_seqs=24)
    NB, H, BS, D = case["k_pool"].shape
    pool = pa.pa_pool_create(NB, BS, H, D, torch.float16)
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    ws = workspace_for(pool, 24, bt.shape[1])
    rng = np.random.default_rng(2)
    layers = []
    for _ in range(3):
        kp = torch.from_numpy(rng.standard_normal(case["k_pool"].shape).astype(np.float16)).cuda()
        vp = torch.from_numpy(rng.standard_normal(case["k_pool"].shape).astype(np.float16)).cuda()
        q = torch.from_numpy(rng.standard_normal(case["q"].shape).astype(np.float16)).cuda()
        layers.append((q, kp, vp))
    pa.pa_decode_plan(pool, cl, bt.shape[1], ws)
    planned = []
    for q, kp, vp in layers:
        out = torch.empty_like(q)
        pa.pa_decode_attention_planned(pool, q, kp, vp, bt, case["scale"], out, ws)
        planned.append(out)
    assert pa.pa_device_errors() == 0
    for (q, kp, vp), got in zip(layers, planned):
        out = torch.empty_like(q)
        ws2 = workspace_for(pool, 24, bt.shape[1])
        pa.pa_decode_attention(pool, q, kp, vp, bt, cl, case["scale"], out, ws2)
        assert torch.equal(out, got)
        ref = oracle.decode_attention(host(q), host(kp), host(vp), case["block_tables"],
                                      case["context_lens"], case["scale"])
        assert_parity(got, ref, "planned layer")


# ---- fused append + attend ------------------------------------------------------------

@pytest.mark.parametrize("dtype,head_dim,partition_size", [(np.float16, 128, 0), (np.float16, 64, 32),
                                                           (np.float32, 128, 16), (np.float32, 64, 0)])
def test_fused_append_equals_cache_then_decode(dtype, head_dim, partition_size):
    """One launch that writes the new token and attends must leave the same
    pool bits and produce the same output bits as reshape_and_cache followed
    by decode, and match the oracle."""
    lens = [0, 1, 2, 16, 17, 32, 33, 255, 256, 257, 1000, 2048, 5]
    case = syn.decode_case(31, lens, 6, head_dim, dtype, max_blocks=130)
    ref_out, ref_k, ref_v = gpu_append_and_decode(case, partition_size=partition_size)
    q, kp, vp = dev(case["q"]), dev(case["k_pool"]), dev(case["v_pool"])
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    NB = kp.shape[0]
    pool = pa.pa_pool_create(NB, 16, 6, head_dim, q.dtype)
    out = torch.empty_like(q)
    ws = workspace_for(pool, len(lens), bt.shape[1], 0, partition_size)
    pa.pa_decode_append_attention(pool, q, dev(case["k_new"]), dev(case["v_new"]), kp, vp, bt, cl,
                                  case["scale"], out, ws, partition_size=partition_size)
    assert pa.pa_device_errors() == 0
    assert torch.equal(bits_t(kp), bits_t(ref_k)) and torch.equal(bits_t(vp), bits_t(ref_v))
    assert torch.equal(out, ref_out)
    want, _, _ = oracle_append_and_decode(case)
    assert_parity(out, want, "fused append")


def bits_t(t):
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


def test_fused_append_planned_over_layers():
    case = syn.single_layer_case(seed=8, num_seqs=32)
    NB, H, BS, D = case["k_pool"].shape
    pool = pa.pa_pool_create(NB, BS, H, D, torch.float16)
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    ws = workspace_for(pool, 32, bt.shape[1])
    pa.pa_decode_plan(pool, cl, bt.shape[1], ws)
    rng = np.random.default_rng(12)
    for layer in range(3):
        kp_h = rng.standard_normal(case["k_pool"].shape).astype(np.float16)
        vp_h = rng.standard_normal(case["k_pool"].shape).astype(np.float16)
        q_h = rng.standard_normal(case["q"].shape).astype(np.float16)
        kn_h = rng.standard_normal(case["q"].shape).astype(np.float16)
        vn_h = rng.standard_normal(case["q"].shape).astype(np.float16)
        kp, vp, q = dev(kp_h), dev(vp_h), dev(q_h)
        out = torch.empty_like(q)
        pa.pa_decode_append_attention_planned(pool, q, dev(kn_h), dev(vn_h), kp, vp, bt,
                                              case["scale"], out, ws)
        assert pa.pa_device_errors() == 0
        layer_case = dict(case, k_pool=kp_h, v_pool=vp_h, q=q_h, k_new=kn_h, v_new=vn_h)
        want, wk, wv = oracle_append_and_decode(layer_case)
        assert np.array_equal(bits(kp), bits(wk)) and np.array_equal(bits(vp), bits(wv))
        assert_parity(out, want, f"fused planned layer {layer}")


# ---- grouped-query attention ------------------------------------------------------------

@pytest.mark.parametrize("group", [2, 4, 8])
@pytest.mark.parametrize("dtype,head_dim", [(np.float16, 128), (np.float32, 64)])
def test_gqa_matches_oracle_and_replicated_mha(group, dtype, head_dim):
    """Query head h reads KV head h // group.  The result must match the
    oracle and be bit-identical to MHA over a pool whose KV heads are
    repeated group times (same arithmetic per query head)."""
    kv_heads = 3
    lens = [1, 15, 16, 17, 300, 513, 1024, 2048, 0]
    case = syn.decode_case(41, lens, kv_heads, head_dim, dtype, max_blocks=130)
    rng = np.random.default_rng(42)
    qg = rng.standard_normal((len(lens), kv_heads * group, head_dim)).astype(dtype)
    NB = case["k_pool"].shape[0]
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    kp, vp = dev(case["k_pool"]), dev(case["v_pool"])
    pool = pa.pa_pool_create(NB, 16, kv_heads, head_dim, TORCH[dtype])
    pa.pa_pool_set_query_heads(pool, kv_heads * group)
    out = torch.empty((len(lens), kv_heads * group, head_dim), dtype=TORCH[dtype], device="cuda")
    ws = workspace_for(pool, len(lens), bt.shape[1])
    q = dev(qg)
    pa.pa_decode_attention(pool, q, kp, vp, bt, cl, case["scale"], out, ws)
    assert pa.pa_device_errors() == 0
    ref = oracle.decode_attention(qg, case["k_pool"], case["v_pool"], case["block_tables"],
                                  case["context_lens"], case["scale"])
    assert_parity(out, ref, f"gqa x{group}")
    # MHA over repeated KV heads
    kr = np.ascontiguousarray(np.repeat(case["k_pool"], group, axis=1))
    vr = np.ascontiguousarray(np.repeat(case["v_pool"], group, axis=1))
    pool_r = pa.pa_pool_create(NB, 16, kv_heads * group, head_dim, TORCH[dtype])
    out_r = torch.empty_like(out)
    ws_r = workspace_for(pool_r, len(lens), bt.shape[1])
    pa.pa_decode_attention(pool_r, q, dev(kr), dev(vr), bt, cl, case["scale"], out_r, ws_r)
    assert pa.pa_device_errors() == 0
    if dtype == np.float32:
        assert torch.equal(out, out_r)  # same CUDA-core arithmetic per query head
    else:
        # fp16 groups run on tensor cores (P rounded to fp16 before P.V): same gate
        assert_parity(out, out_r.double().cpu().numpy(), f"gqa x{group} vs repeated-KV MHA")


@pytest.mark.parametrize("group", [2, 4, 8])
def test_gqa_fused_append(group):
    kv_heads = 2
    lens = [3, 16, 17, 600, 1, 2048]
    case = syn.decode_case(43, lens, kv_heads, 128, np.float16, max_blocks=130)
    rng = np.random.default_rng(44)
    qg = rng.standard_normal((len(lens), kv_heads * group, 128)).astype(np.float16)
    NB = case["k_pool"].shape[0]
    pool = pa.pa_pool_create(NB, 16, kv_heads, 128, torch.float16)
    pa.pa_pool_set_query_heads(pool, kv_heads * group)
    kp, vp = dev(case["k_pool"]), dev(case["v_pool"])
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    out = torch.empty((len(lens), kv_heads * group, 128), dtype=torch.float16, device="cuda")
    ws = workspace_for(pool, len(lens), bt.shape[1])
    pa.pa_decode_append_attention(pool, dev(qg), dev(case["k_new"]), dev(case["v_new"]), kp, vp,
                                  bt, cl, case["scale"], out, ws)
    assert pa.pa_device_errors() == 0
    want_case = dict(case, q=qg)
    kh, vh = case["k_pool"].copy(), case["v_pool"].copy()
    slots = np.array([oracle.slot_of_c(case["block_tables"][s], int(L) - 1)
                      for s, L in enumerate(lens)], dtype=np.int32)
    oracle.reshape_and_cache(case["k_new"], case["v_new"], slots, kh, vh)
    ref = oracle.decode_attention(qg, kh, vh, case["block_tables"], case["context_lens"],
                                  case["scale"])
    assert np.array_equal(bits(kp), bits(kh)) and np.array_equal(bits(vp), bits(vh))
    assert_parity(out, ref, f"gqa fused x{group}")


TORCH = {np.float16: torch.float16, np.float32: torch.float32}


@pytest.mark.parametrize("group", [2, 4, 8])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_gqa_tensor_core_path_ragged_and_poisoned(group, head_dim):
    """bf16 groups on the tensor-core path: lengths 0, 1 and ragged blocks,
    NaN in every pool slot outside the cached tokens, several partition sizes."""
    kv_heads = 3
    lens = [0, 1, 2, 15, 16, 17, 100, 257, 1000]
    case = syn.decode_case(51, lens, kv_heads, head_dim, np.float32, pool_fill="nan",
                           num_pool_blocks=128, max_blocks=64)
    rng = np.random.default_rng(52)
    for s_, L in enumerate(lens):
        slots = np.array([oracle.slot_of_c(case["block_tables"][s_], t) for t in range(L)],
                         dtype=np.int32)
        kn = rng.standard_normal((L, kv_heads, head_dim)).astype(np.float32)
        vn = rng.standard_normal((L, kv_heads, head_dim)).astype(np.float32)
        oracle.reshape_and_cache(kn, vn, slots, case["k_pool"], case["v_pool"])
    qf = rng.standard_normal((len(lens), kv_heads * group, head_dim)).astype(np.float32)
    kt = torch.from_numpy(case["k_pool"]).to(torch.bfloat16)
    vt = torch.from_numpy(case["v_pool"]).to(torch.bfloat16)
    qt = torch.from_numpy(qf).to(torch.bfloat16)
    kb, vb, qb = (x.view(torch.int16).numpy().view(np.uint16) for x in (kt, vt, qt))
    ref = oracle.decode_attention(qb, kb, vb, case["block_tables"], case["context_lens"],
                                  case["scale"], dtype=oracle.BF16)
    pool = pa.pa_pool_create(128, 16, kv_heads, head_dim, torch.bfloat16)
    pa.pa_pool_set_query_heads(pool, kv_heads * group)
    bt, cl = dev(case["block_tables"]), dev(case["context_lens"])
    for ps in (0, 16, 96):
        out = torch.empty((len(lens), kv_heads * group, head_dim), dtype=torch.bfloat16,
                          device="cuda")
        ws = workspace_for(pool, len(lens), bt.shape[1], 0, ps)
        pa.pa_decode_attention(pool, qt.cuda(), kt.cuda(), vt.cuda(), bt, cl, case["scale"], out,
                               ws, partition_size=ps)
        assert pa.pa_device_errors() == 0
        assert torch.isfinite(out.float()).all()
        assert_parity(out, ref, f"gqa bf16 x{group} D={head_dim} ps={ps}")
