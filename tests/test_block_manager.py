"""The C++ block manager (pa_alloc_*, pa_append_tokens) against the page-pool
oracle: the worked examples of "Atención paginada en modelos de lenguaje
grandes (LLM)" (7minutos.es, sections 2 and 3) and random operation
sequences, compared exactly (block tables, slots, copy pairs, refcounts)."""
import json
import os

import numpy as np
import pytest

import oracle
import paged_kv_cache_478_b200 as pa

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "page_pool_worked_examples.json")))


def test_five_requests_worked_example():
    g = GOLDEN["five_requests"]
    bm = pa.BlockManager(g["pool_pages"])
    tables = []
    for n in g["tokens"]:
        t = np.full(200, -1, dtype=np.int32)
        L, slots, pairs = bm.append_tokens(t, 0, n)
        assert L == n and len(pairs) == 0
        tables.append(t[: (n + 15) // 16].copy())
    assert [len(t) for t in tables] == g["pages"]
    assert bm.num_free() == g["pool_pages"] - sum(g["pages"])
    freed = sorted(tables[g["freed_request"]])
    bm.release_table(tables[g["freed_request"]], len(freed))
    assert [bm.alloc() for _ in freed] == freed


def test_shared_prompt_and_cow_worked_example():
    g = GOLDEN["shared_prompt"]
    bm = pa.BlockManager(512)
    owner = np.full(64, -1, dtype=np.int32)
    L, _, _ = bm.append_tokens(owner, 0, g["prompt_tokens"])
    n = (L + 15) // 16
    assert n == g["prompt_pages"]
    users = []
    for _ in range(g["users"]):
        t = np.full(64, -1, dtype=np.int32)
        bm.fork_table(owner, n, t)
        users.append(t)
    assert all(bm.refcount(int(b)) == g["refcount_after_share"] for b in owner[:n])
    r = users[g["cow_request"]]
    L2, slots, pairs = bm.append_tokens(r, L, 1)
    assert pairs.tolist() == [[g["cow_src_page"], g["cow_new_page"]]]
    assert bm.refcount(g["cow_src_page"]) == g["refcount_src_after_cow"]
    assert slots[0] == g["cow_new_page"] * 16 + g["prompt_tokens"] % 16
    assert L2 == L + 1


def test_errors():
    bm = pa.BlockManager(2)
    bm.alloc()
    bm.alloc()
    with pytest.raises(pa.PagedAttnError) as e:
        bm.alloc()
    assert e.value.status == pa.PA_ERR_NO_FREE_BLOCKS
    bm.free(0)
    with pytest.raises(pa.PagedAttnError):
        bm.free(0)          # double free
    with pytest.raises(pa.PagedAttnError):
        bm.share(0)         # not allocated
    with pytest.raises(pa.PagedAttnError):
        bm.refcount(7)      # outside the pool
    t = np.full(1, -1, dtype=np.int32)
    bm2 = pa.BlockManager(8)
    with pytest.raises(pa.PagedAttnError):
        bm2.append_tokens(t, 0, 17)  # table has room for one block only


@pytest.mark.parametrize("seed", range(5))
def test_random_operations_match_the_oracle(seed):
    """Random appends, forks (prefix sharing) and releases on both managers;
    every block table, slot, copy pair and refcount must agree exactly."""
    rng = np.random.default_rng(seed)
    NB, MAXB = 96, 40
    bm = pa.BlockManager(NB)
    pool = oracle.PagePool(NB)
    seqs = []  # (table np, length, oracle request)
    for step in range(400):
        op = rng.integers(0, 10)
        if op < 6 and seqs:
            i = int(rng.integers(0, len(seqs)))
            t, L, req = seqs[i]
            n = int(rng.integers(1, 20))
            if (L + n + 15) // 16 > MAXB:
                continue
            try:
                want = [req.generate_token() for _ in range(n)]
                ok = True
            except oracle.PoolExhausted:
                ok = False
            if not ok:
                with pytest.raises(pa.PagedAttnError):
                    bm.append_tokens(t, L, n)
                return  # both exhausted: states diverge by design from here
            L2, slots, pairs = bm.append_tokens(t, L, n)
            assert L2 == req.num_tokens
            assert slots.tolist() == [w[0] for w in want]
            assert [tuple(p) for p in pairs.tolist()] == [w[1] for w in want if w[1] is not None]
            seqs[i] = (t, L2, req)
        elif op < 8:
            t = np.full(MAXB, -1, dtype=np.int32)
            req = oracle.PagedRequest(pool)
            if seqs and rng.integers(0, 2):
                j = int(rng.integers(0, len(seqs)))
                st, sL, sreq = seqs[j]
                req.share_prefix_of(sreq)
                bm.fork_table(st, (sL + 15) // 16, t)
                seqs.append((t, sL, req))
            else:
                seqs.append((t, 0, req))
        elif seqs:
            i = int(rng.integers(0, len(seqs)))
            t, L, req = seqs.pop(i)
            req.release()
            bm.release_table(t, (L + 15) // 16)
        for t, L, req in seqs:
            nb = (L + 15) // 16
            assert t[:nb].tolist() == req.block_table
        assert bm.num_free() == pool.num_free()
        for b in range(NB):
            assert bm.refcount(b) == pool.refcount[b]


def test_decode_slots_matches_the_oracle():
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 300, size=30).astype(np.int32)
    tables = np.full((30, 19), -1, dtype=np.int32)
    perm = rng.permutation(30 * 19).astype(np.int32)
    pos = 0
    for s, L in enumerate(lens):
        n = (L + 15) // 16
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    got = pa.pa_decode_slots(tables, lens)
    want = [oracle.slot_of_c(tables[s], int(L) - 1) for s, L in enumerate(lens)]
    assert got.tolist() == want
    lens[4] = 0
    assert pa.pa_decode_slots(tables, lens)[4] == -1


def _prefix_tables():
    """128 sequences share a 1000-token prefix (63 blocks), then each adds a
    suffix; the first divergent write copies block 62 for all but the last."""
    rng = np.random.default_rng(5)
    bm = pa.BlockManager(4096)
    S, P = 128, 1000
    tables = np.full((S, 95), -1, dtype=np.int32)
    lens = np.zeros(S, dtype=np.int32)
    lens[0], _, _ = bm.append_tokens(tables[0], 0, P)
    for s in range(1, S):
        bm.fork_table(tables[0], 63, tables[s])
        lens[s] = P
    for s in range(S):
        lens[s], _, _ = bm.append_tokens(tables[s], int(lens[s]), int(rng.integers(1, 513)))
    return tables, lens


def test_find_shared_prefixes_on_a_forked_prompt():
    tables, lens = _prefix_tables()
    g = pa.pa_find_shared_prefixes(tables, lens)
    assert g["num_groups"] == 1 and g["max_group_size"] == 128
    assert g["blocks"].tolist() == [62]        # block 62 was copied on write by 127 holders
    assert g["members"].tolist() == list(range(128))
    assert g["offsets"].tolist() == [0, 128]


def test_find_shared_prefixes_hand_cases():
    t = np.full((6, 6), -1, dtype=np.int32)
    t[0, :5] = [7, 8, 9, 10, 11]
    t[1, :5] = [7, 8, 9, 20, 21]   # shares 3 blocks with 0
    t[2, :4] = [30, 31, 32, 33]    # alone
    t[3, :3] = [40, 41, 42]
    t[4, :3] = [40, 41, 50]        # shares 2 with 3
    t[5, :2] = [7, 8]              # shares 2 with 0 and 1, but only 1 full block
    lens = np.array([80, 80, 64, 48, 48, 20], dtype=np.int32)
    g = pa.pa_find_shared_prefixes(t, lens)
    # 5 has one full block (20 tokens), so the {0, 1, 5} group shares 1 block
    assert g["num_groups"] == 2
    assert g["members"].tolist() == [0, 1, 5, 3, 4]
    assert g["blocks"].tolist() == [1, 2]
    g2 = pa.pa_find_shared_prefixes(t, lens, min_shared_blocks=2)
    # 5 no longer qualifies (one full block), so 0 and 1 share 3 blocks
    assert g2["members"].tolist() == [0, 1, 3, 4]
    assert g2["blocks"].tolist() == [3, 2]
    assert g2["max_group_size"] == 2 and g2["max_shared_blocks"] == 3
