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
