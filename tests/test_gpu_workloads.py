"""The three larger workloads through the C ABI against the oracle.

  * shared prefix + copy-on-write: 128 sequences share a 1000-token system
    prefix (63 blocks, the last one partial); each appends a suffix of 1 to
    512 tokens, which copies the partial block on the first divergent write
    ("Atención paginada en modelos de lenguaje grandes (LLM)", 7minutos.es,
    section 3; "PagedAttention" wiki mirror, "Descripció");
  * long context split-K: 8 sequences x 32768 tokens, partitions of 512;
  * the full 32-layer decode step at the pages' scale (200 requests, 32 x 32
    x 128 fp16), checked on sampled layers and sequences, in the launch
    configuration the benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_478_b200 as pa
from paged_kv_cache_478_b200 import synthetic as syn
from tests.gpu_cases import assert_parity, bits, dev, host, workspace_for

pytestmark = pytest.mark.gpu

BS = 16


def _gpu_shared_prefix(case, nb, private_prefix=False):
    """Product side: C++ block manager + reshape_and_cache + copy_blocks +
    decode.  With private_prefix every sequence gets its own copy of the
    prefix instead of sharing it."""
    S, H, D = case["q"].shape
    P = case["prefix_len"]
    bm = pa.BlockManager(nb)
    maxb = math.ceil((P + 512) / BS)
    tables = np.full((S, maxb), -1, dtype=np.int32)
    kp = torch.zeros((nb, H, BS, D), dtype=torch.float16, device="cuda")
    vp = torch.zeros_like(kp)
    pool = pa.pa_pool_create(nb, BS, H, D, torch.float16)
    lens = np.zeros(S, dtype=np.int32)
    kpre, vpre = dev(case["k_prefix"]), dev(case["v_prefix"])
    if private_prefix:
        for s in range(S):
            lens[s], slots, _ = bm.append_tokens(tables[s], 0, P)
            pa.pa_reshape_and_cache(pool, kpre, vpre, dev(slots), kp, vp)
    else:
        lens[0], slots, _ = bm.append_tokens(tables[0], 0, P)
        for s in range(1, S):
            bm.fork_table(tables[0], math.ceil(P / BS), tables[s])
            lens[s] = P
        pa.pa_reshape_and_cache(pool, kpre, vpre, dev(slots), kp, vp)
    all_slots, all_pairs = [], []
    for s in range(S):
        lens[s], slots, pairs = bm.append_tokens(tables[s], int(lens[s]),
                                                 int(case["suffix_lens"][s]))
        all_slots.append(slots)
        all_pairs.append(pairs)
    pairs = np.concatenate(all_pairs).reshape(-1, 2).astype(np.int32)
    if len(pairs):
        pa.pa_copy_blocks(pool, kp, vp, dev(pairs))
    pa.pa_reshape_and_cache(pool, dev(np.concatenate(case["k_suffix"])),
                            dev(np.concatenate(case["v_suffix"])),
                            dev(np.concatenate(all_slots)), kp, vp)
    q = dev(case["q"])
    out = torch.empty_like(q)
    ws = workspace_for(pool, S, maxb)
    pa.pa_decode_attention(pool, q, kp, vp, dev(tables), dev(lens), case["scale"], out, ws)
    assert pa.pa_device_errors() == 0
    return dict(out=out, kp=kp, vp=vp, tables=tables, lens=lens, pairs=pairs, bm=bm, pool=pool,
                ws=ws, slots=all_slots)


def _oracle_shared_prefix(case, nb):
    """Oracle side: page-pool model + host scatter/copy + fp64 attention."""
    S, H, D = case["q"].shape
    P = case["prefix_len"]
    pp = oracle.PagePool(nb)
    reqs = [oracle.PagedRequest(pp) for _ in range(S)]
    kp = np.zeros((nb, H, BS, D), dtype=np.float16)
    vp = np.zeros_like(kp)
    slots = np.array([reqs[0].generate_token()[0] for _ in range(P)], dtype=np.int32)
    for s in range(1, S):
        reqs[s].share_prefix_of(reqs[0])
    oracle.reshape_and_cache(case["k_prefix"], case["v_prefix"], slots, kp, vp)
    all_slots, pairs = [], []
    for s in range(S):
        for _ in range(int(case["suffix_lens"][s])):
            slot, cow = reqs[s].generate_token()
            all_slots.append(slot)
            if cow is not None:
                pairs.append(cow)
    pairs = np.array(pairs, dtype=np.int32).reshape(-1, 2)
    oracle.copy_blocks(kp, vp, pairs)
    oracle.reshape_and_cache(np.concatenate(case["k_suffix"]), np.concatenate(case["v_suffix"]),
                             np.array(all_slots, dtype=np.int32), kp, vp)
    maxb = math.ceil((P + 512) / BS)
    tables = np.full((S, maxb), -1, dtype=np.int32)
    for s, r in enumerate(reqs):
        tables[s, :len(r.block_table)] = r.block_table
    lens = np.array([r.num_tokens for r in reqs], dtype=np.int32)
    out = oracle.decode_attention(case["q"], kp, vp, tables, lens, case["scale"])
    return dict(out=out, kp=kp, vp=vp, tables=tables, lens=lens, pairs=pairs)


def test_shared_prefix_copy_on_write():
    case = syn.shared_prefix_case(seed=0)
    S = 128
    nb = 63 + S + sum(math.ceil(int(n) / BS) for n in case["suffix_lens"])
    g = _gpu_shared_prefix(case, nb)
    r = _oracle_shared_prefix(case, nb)
    # block management: identical tables, lengths and copy pairs
    assert np.array_equal(g["tables"], r["tables"])
    assert np.array_equal(g["lens"], r["lens"])
    assert np.array_equal(g["pairs"], r["pairs"])
    assert len(g["pairs"]) == S - 1  # the last holder writes block 62 in place
    assert all(p[0] == 62 for p in g["pairs"])
    # device state after copy_blocks + reshape_and_cache: bit-exact
    assert np.array_equal(bits(g["kp"]), bits(r["kp"]))
    assert np.array_equal(bits(g["vp"]), bits(r["vp"]))
    assert_parity(g["out"], r["out"], "shared prefix")

    # shared prefix == private copies of the prefix, bit for bit
    nb2 = S * 64 + S + sum(math.ceil(int(n) / BS) for n in case["suffix_lens"])
    priv = _gpu_shared_prefix(case, nb2, private_prefix=True)
    assert torch.equal(priv["out"], g["out"])

    # copy-on-write leaves every other sequence's output unchanged: fork
    # sequence 10 (its blocks become shared) and let the fork write one token
    bm, pool, tables, lens = g["bm"], g["pool"], g["tables"], g["lens"]
    fork = np.full(tables.shape[1], -1, dtype=np.int32)
    n10 = math.ceil(int(lens[10]) / BS)
    bm.fork_table(tables[10], n10, fork)
    L_fork, slots, pairs = bm.append_tokens(fork, int(lens[10]), 1)
    if int(lens[10]) % BS:
        assert len(pairs) == 1 and bm.refcount(int(tables[10][n10 - 1])) == 1
        pa.pa_copy_blocks(pool, g["kp"], g["vp"], dev(pairs))
    rng = np.random.default_rng(1)
    kn = rng.standard_normal((1, 32, 128)).astype(np.float16)
    pa.pa_reshape_and_cache(pool, dev(kn), dev(kn), dev(slots), g["kp"], g["vp"])
    tables2 = np.vstack([tables, fork[None]])
    lens2 = np.append(lens, L_fork).astype(np.int32)
    q2 = torch.cat([dev(case["q"]), dev(case["q"][10:11])])
    out2 = torch.empty_like(q2)
    ws2 = workspace_for(pool, S + 1, tables.shape[1])
    pa.pa_decode_attention(pool, q2, g["kp"], g["vp"], dev(tables2), dev(lens2), case["scale"],
                           out2, ws2)
    assert pa.pa_device_errors() == 0
    assert torch.equal(out2[:S], g["out"])


def test_long_context_split_k():
    S, H, D, CTX = 8, 32, 128, 32768
    lens, tables, nb = syn.long_context_tables(seed=0, num_seqs=S, context=CTX)
    kp = torch.empty((nb, H, BS, D), dtype=torch.float16, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 101)
    syn.fill_normal_device(vp, 102)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((S, H, D)).astype(np.float16)
    kn = rng.standard_normal((S, H, D)).astype(np.float16)
    vn = rng.standard_normal((S, H, D)).astype(np.float16)
    sample = [0, 5]
    kh, vh = host(kp), host(vp)  # oracle inputs: the pools as drawn, before any kernel
    pool = pa.pa_pool_create(nb, BS, H, D, torch.float16)
    slots = pa.pa_decode_slots(tables, lens)
    pa.pa_reshape_and_cache(pool, dev(kn), dev(vn), dev(slots), kp, vp)
    out = torch.empty((S, H, D), dtype=torch.float16, device="cuda")
    ws = workspace_for(pool, S, tables.shape[1], 0, 512)
    pa.pa_decode_attention(pool, dev(q), kp, vp, dev(tables), dev(lens), 1 / math.sqrt(D), out, ws,
                           partition_size=512)
    assert pa.pa_device_errors() == 0
    oslots = np.array([oracle.slot_of_c(tables[s], CTX - 1) for s in range(S)], dtype=np.int32)
    oracle.reshape_and_cache(kn, vn, oslots, kh, vh)
    only = np.zeros(S, dtype=np.int32)
    only[sample] = lens[sample]
    ref = oracle.decode_attention(q, kh, vh, tables, only, 1 / math.sqrt(D))
    assert_parity(out[sample], ref[sample], "long context")
    # the new tokens landed where the oracle put them
    for s in range(S):
        b, o = divmod(int(oslots[s]), BS)
        assert np.array_equal(bits(kp[b, :, o]), bits(kn[s]))


@pytest.mark.parametrize("path", ["fused-planned", "separate"])
def test_full_decode_step_sampled(path):
    """200 requests x 32 layers x 32 heads x 128 fp16, one block-id space for
    every layer (lengths min(2048, 1 + Exponential(500)), seed 0).

    path "fused-planned" is the call sequence the benchmark times, launched
    the same way: pa_decode_plan once for the step, then per layer one
    pa_decode_append_attention_planned (the new token's reshape_and_cache and
    the attention in one launch) with the automatic partition size (512
    tokens at this batch) on the persistent grid, the plan reused by all 32
    layers.  path "separate" runs pa_reshape_and_cache then
    pa_decode_attention per layer.

    For layers 0 and 31: both whole pools after the call are bit-identical to
    the oracle's reshape_and_cache applied to host copies taken before it
    ("Atención paginada en modelos de lenguaje grandes (LLM)", 7minutos.es,
    section 2: the new token goes into the sequence's tail page), and the
    outputs of nine sequences, the longest (split into partitions) among
    them, match the oracle ("PagedAttention" wiki mirror, "Formulació
    matemàtica")."""
    S, H, D, LAYERS = 200, 32, 128, 32
    lens = syn.full_step_lengths(seed=0, num_seqs=S)
    tables, nb = syn.full_step_tables(0, lens)
    pool = pa.pa_pool_create(nb, BS, H, D, torch.float16)
    slots = dev(pa.pa_decode_slots(tables, lens))
    btd, cld = dev(tables), dev(lens)
    ws = workspace_for(pool, S, tables.shape[1])
    rng = np.random.default_rng(0)
    sample_layers = [0, LAYERS - 1]
    longest = int(np.argmax(lens))
    assert lens[longest] > 512  # split into several partitions
    sample_seqs = sorted(set(rng.choice(S, 8, replace=False).tolist()) | {longest})
    oslots = np.array([oracle.slot_of_c(tables[s], int(lens[s]) - 1) for s in range(S)],
                      dtype=np.int32)
    scale = 1 / math.sqrt(D)
    fused = path == "fused-planned"
    if fused:
        pa.pa_decode_plan(pool, cld, tables.shape[1], ws)
    checked = 0
    for layer in range(LAYERS):
        kp = torch.empty((nb, H, BS, D), dtype=torch.float16, device="cuda")
        vp = torch.empty_like(kp)
        syn.fill_normal_device(kp, 1000 + 2 * layer)
        syn.fill_normal_device(vp, 1001 + 2 * layer)
        q = torch.empty((S, H, D), dtype=torch.float16, device="cuda")
        kn, vn = torch.empty_like(q), torch.empty_like(q)
        for t, sd in ((q, 3000), (kn, 4000), (vn, 5000)):
            syn.fill_normal_device(t, sd + layer)
        if layer in sample_layers:
            kh, vh = host(kp), host(vp)
        out = torch.empty_like(q)
        if fused:
            pa.pa_decode_append_attention_planned(pool, q, kn, vn, kp, vp, btd, scale, out, ws)
        else:
            pa.pa_reshape_and_cache(pool, kn, vn, slots, kp, vp)
            pa.pa_decode_attention(pool, q, kp, vp, btd, cld, scale, out, ws)
        assert pa.pa_device_errors() == 0
        if layer in sample_layers:
            oracle.reshape_and_cache(host(kn), host(vn), oslots, kh, vh)
            assert np.array_equal(bits(kp), bits(kh)), f"layer {layer}: K pool"
            assert np.array_equal(bits(vp), bits(vh)), f"layer {layer}: V pool"
            only = np.zeros(S, dtype=np.int32)
            only[sample_seqs] = lens[sample_seqs]
            ref = oracle.decode_attention(host(q), kh, vh, tables, only, scale)
            assert_parity(out[sample_seqs], ref[sample_seqs], f"{path}, layer {layer}")
            checked += 1
            del kh, vh
        del kp, vp
    assert checked == len(sample_layers)


def _groups_to_device(g):
    d = dict(g)
    for k in ("offsets", "members", "blocks"):
        d[k] = dev(np.ascontiguousarray(g[k], dtype=np.int32))
    return d


def test_shared_prefix_path_on_the_forked_prompt():
    """The tensor-core shared-prefix path on the 128-way shared system prompt:
    the same answer as the oracle and as the plain decode path."""
    case = syn.shared_prefix_case(seed=2)
    S = 128
    nb = 63 + S + sum(math.ceil(int(n) / BS) for n in case["suffix_lens"])
    g = _gpu_shared_prefix(case, nb)
    r = _oracle_shared_prefix(case, nb)
    groups = pa.pa_find_shared_prefixes(g["tables"], g["lens"])
    assert groups["num_groups"] == 1 and groups["blocks"].tolist() == [62]
    pool = g["pool"]
    q = dev(case["q"])
    out = torch.empty_like(q)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(
        pool, S, g["tables"].shape[1], groups["max_shared_blocks"]), dtype=torch.uint8,
        device="cuda")
    pa.pa_decode_attention_shared_prefix(pool, q, g["kp"], g["vp"], dev(g["tables"]),
                                         dev(g["lens"]), _groups_to_device(groups),
                                         case["scale"], out, ws)
    assert pa.pa_device_errors() == 0
    assert_parity(out, r["out"], "shared-prefix path")
    assert_parity(out, g["out"].double().cpu().numpy(), "shared-prefix vs plain path")


@pytest.mark.parametrize("dtype,group", [("f16", 1), ("bf16", 2), ("bf16", 4), ("f16", 8)])
def test_shared_prefix_groups_with_gqa_and_a_bad_member(dtype, group):
    rng = np.random.default_rng(60 + group)
    H, D = 2, 128
    HQ = H * group
    # group A: sequences 0-4 share 20 blocks; group B: 5-7 share 3 blocks; 8-9 alone
    lens = np.array([400, 333, 321, 700, 1024, 60, 49, 64, 17, 250], dtype=np.int32)
    nb = 400
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((10, 64), -1, dtype=np.int32)
    pos = 0
    shared_a = perm[pos:pos + 20]; pos += 20
    shared_b = perm[pos:pos + 3]; pos += 3
    for s, L in enumerate(lens):
        n = math.ceil(int(L) / 16)
        pre = shared_a if s < 5 else (shared_b if s < 8 else np.zeros(0, np.int32))
        tables[s, :len(pre)] = pre
        tables[s, len(pre):n] = perm[pos:pos + n - len(pre)]
        pos += n - len(pre)
    groups = pa.pa_find_shared_prefixes(tables, lens)
    assert groups["num_groups"] == 2
    assert groups["blocks"].tolist() == [20, 3]
    # plant a member that does not hold the group's blocks: it must be reported
    # and still get the right answer on its own
    groups["members"] = np.concatenate([groups["members"][:5], [9], groups["members"][5:]])
    groups["offsets"] = np.array([0, 6, 9], dtype=np.int32)
    groups["max_group_size"] = 6
    shape = (nb, H, BS, D)
    kh = rng.standard_normal(shape).astype(np.float32)
    vh = rng.standard_normal(shape).astype(np.float32)
    qh = rng.standard_normal((10, HQ, D)).astype(np.float32)
    if dtype == "bf16":
        tdt = torch.bfloat16
        kt, vt, qt = (torch.from_numpy(x).to(tdt) for x in (kh, vh, qh))
        kb, vb, qb = (x.view(torch.int16).numpy().view(np.uint16) for x in (kt, vt, qt))
        ref = oracle.decode_attention(qb, kb, vb, tables, lens, 1 / math.sqrt(D), dtype=oracle.BF16)
    else:
        tdt = torch.float16
        kt, vt, qt = (torch.from_numpy(x.astype(np.float16)) for x in (kh, vh, qh))
        ref = oracle.decode_attention(qt.numpy(), kt.numpy(), vt.numpy(), tables, lens,
                                      1 / math.sqrt(D))
    pool = pa.pa_pool_create(nb, BS, H, D, tdt)
    pa.pa_pool_set_query_heads(pool, HQ)
    q = qt.cuda()
    out = torch.empty_like(q)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(pool, 10, 64, 20),
                     dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention_shared_prefix(pool, q, kt.cuda(), vt.cuda(), dev(tables), dev(lens),
                                         _groups_to_device(groups), 1 / math.sqrt(D), out, ws)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN  # the planted member
    assert_parity(out, ref, f"shared prefix {dtype} G={group}")


@pytest.mark.parametrize("group", [1, 2, 4])
def test_shared_prefix_partials_are_read_after_their_kernel(group):
    """The decode launch may overlap the shared-prefix kernel before it and
    reads that kernel's partials only once it has completed.  A long shared
    prefix (125 blocks) with a few own tokens per sequence makes every merge
    come early, while the shared-prefix kernel may still run; the workspace is
    poisoned with NaN before each call, so an early read would show."""
    rng = np.random.default_rng(70 + group)
    S, H, D, PB = 64, 8, 128, 125
    HQ = H * group
    lens = (PB * BS + rng.integers(1, 17, S)).astype(np.int32)
    nb = PB + S
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((S, PB + 1), -1, dtype=np.int32)
    tables[:, :PB] = perm[:PB]
    tables[:, PB] = perm[PB:]
    groups = pa.pa_find_shared_prefixes(tables, lens)
    assert groups["num_groups"] == 1 and groups["blocks"].tolist() == [PB]
    kh = rng.standard_normal((nb, H, BS, D)).astype(np.float16)
    vh = rng.standard_normal((nb, H, BS, D)).astype(np.float16)
    qh = rng.standard_normal((S, HQ, D)).astype(np.float16)
    scale = 1 / math.sqrt(D)
    ref = oracle.decode_attention(qh, kh, vh, tables, lens, scale)
    pool = pa.pa_pool_create(nb, BS, H, D, torch.float16)
    pa.pa_pool_set_query_heads(pool, HQ)
    kp, vp, q = dev(kh), dev(vh), dev(qh)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(
        pool, S, PB + 1, groups["max_shared_blocks"]), dtype=torch.uint8, device="cuda")
    gd = _groups_to_device(groups)
    for _ in range(3):
        ws.fill_(0xFF)  # every fp32 partial reads as NaN until written
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_attention_shared_prefix(pool, q, kp, vp, dev(tables), dev(lens), gd, scale,
                                             out, ws)
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert_parity(out, ref, f"shared prefix read after its kernel, G={group}")


def test_shared_prefix_group_larger_than_max_group_size():
    """A group with more members than max_group_size (the launch covers that
    many) is reported, and its members still get the right answer alone."""
    rng = np.random.default_rng(61)
    H, D = 2, 128
    lens = np.array([400, 333, 321, 700, 1024, 250], dtype=np.int32)
    nb = 300
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((6, 64), -1, dtype=np.int32)
    shared = perm[:20]
    pos = 20
    for s, L in enumerate(lens):
        n = math.ceil(int(L) / 16)
        pre = shared if s < 5 else np.zeros(0, np.int32)
        tables[s, :len(pre)] = pre
        tables[s, len(pre):n] = perm[pos:pos + n - len(pre)]
        pos += n - len(pre)
    groups = pa.pa_find_shared_prefixes(tables, lens)
    assert groups["num_groups"] == 1 and groups["offsets"].tolist() == [0, 5]
    groups["max_group_size"] = 3  # the group has 5 members
    shape = (nb, H, BS, D)
    kt = torch.from_numpy(rng.standard_normal(shape).astype(np.float16))
    vt = torch.from_numpy(rng.standard_normal(shape).astype(np.float16))
    qt = torch.from_numpy(rng.standard_normal((6, H, D)).astype(np.float16))
    ref = oracle.decode_attention(qt.numpy(), kt.numpy(), vt.numpy(), tables, lens,
                                  1 / math.sqrt(D))
    pool = pa.pa_pool_create(nb, BS, H, D, torch.float16)
    q = qt.cuda()
    out = torch.empty_like(q)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(pool, 6, 64, 20),
                     dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention_shared_prefix(pool, q, kt.cuda(), vt.cuda(), dev(tables), dev(lens),
                                         _groups_to_device(groups), 1 / math.sqrt(D), out, ws)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN
    assert_parity(out, ref, "oversized group attends alone")


def test_shared_prefix_offsets_past_the_members_array():
    """group_offsets is device data: offsets beyond the members array reject
    the group (reported) without reading past the array."""
    rng = np.random.default_rng(62)
    H, D = 2, 128
    lens = np.array([400, 333, 321, 700, 1024], dtype=np.int32)
    nb = 300
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((5, 64), -1, dtype=np.int32)
    pos = 20
    for s, L in enumerate(lens):
        n = math.ceil(int(L) / 16)
        tables[s, :20] = perm[:20]
        tables[s, 20:n] = perm[pos:pos + n - 20]
        pos += n - 20
    groups = pa.pa_find_shared_prefixes(tables, lens)
    assert groups["offsets"].tolist() == [0, 5]
    groups["members"] = groups["members"][:3]  # offsets say 5 members, the array holds 3
    shape = (nb, H, BS, D)
    kt = torch.from_numpy(rng.standard_normal(shape).astype(np.float16))
    vt = torch.from_numpy(rng.standard_normal(shape).astype(np.float16))
    qt = torch.from_numpy(rng.standard_normal((5, H, D)).astype(np.float16))
    ref = oracle.decode_attention(qt.numpy(), kt.numpy(), vt.numpy(), tables, lens,
                                  1 / math.sqrt(D))
    pool = pa.pa_pool_create(nb, BS, H, D, torch.float16)
    q = qt.cuda()
    out = torch.empty_like(q)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(pool, 5, 64, 20),
                     dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention_shared_prefix(pool, q, kt.cuda(), vt.cuda(), dev(tables), dev(lens),
                                         _groups_to_device(groups), 1 / math.sqrt(D), out, ws)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN
    assert_parity(out, ref, "a rejected group's members attend alone")
