"""Pins the block-manager oracle to the numbers the pages print.

The worked examples come from "Atención paginada en modelos de lenguaje
grandes (LLM)" (7minutos.es), sections 1 to 4; the fixture file cites each.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import PagePool, PagedRequest

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "page_pool_worked_examples.json")))


def test_bytes_per_token():
    g = GOLDEN["kv_cost"]
    assert oracle.kv_bytes_per_token(g["layers"], g["heads"], g["head_dim"],
                                     g["elem_bytes"]) == g["bytes_per_token"]


def test_naive_allocator_numbers():
    g = GOLDEN["naive_allocator"]
    per_token = GOLDEN["kv_cost"]["bytes_per_token"]
    mib = 1 << 20
    assert g["max_seq_len"] * per_token == g["reserved_mb"] * mib
    assert g["avg_response"] * per_token == g["used_mb"] * mib
    assert round(100 * g["used_mb"] / g["reserved_mb"], 1) == g["utilisation_pct_1dp"]
    assert g["reserved_mb"] - g["used_mb"] == g["idle_mb"]
    # 100 users x 774 MB idle is "75 GB" (GiB, rounded down)
    assert int(g["users"] * g["idle_mb"] / 1024) == g["idle_gb_approx"]


def _run_five_requests():
    g = GOLDEN["five_requests"]
    pool = PagePool(g["pool_pages"], g["page_size"])
    reqs = [PagedRequest(pool) for _ in g["tokens"]]
    for r, n in zip(reqs, g["tokens"]):
        for _ in range(n):
            r.generate_token()
    return g, pool, reqs


def test_five_requests_pages_and_utilisation():
    g, pool, reqs = _run_five_requests()
    assert [len(r.block_table) for r in reqs] == g["pages"]
    used = sum(g["pages"])
    assert round(100 * used / g["pool_pages"], 1) == g["pool_utilisation_pct_1dp"]
    assert pool.num_free() == g["pool_pages"] - used
    # every page id is distinct across requests
    ids = [p for r in reqs for p in r.block_table]
    assert len(set(ids)) == len(ids)


def test_freed_pages_are_reused_immediately():
    g, pool, reqs = _run_five_requests()
    victim = reqs[g["freed_request"]]
    freed = sorted(victim.block_table)
    assert len(freed) == g["freed_pages_count"]
    victim.release()
    assert pool.num_free() == g["pool_pages"] - sum(g["pages"]) + len(freed)
    # freed pages are the lowest free ids, so the next allocations take exactly them
    again = [pool.allocate() for _ in range(len(freed))]
    assert again == freed


def test_shared_prompt_and_copy_on_write():
    g = GOLDEN["shared_prompt"]
    pool = PagePool(512)
    owner = PagedRequest(pool)
    for _ in range(g["prompt_tokens"]):
        owner.generate_token()
    assert len(owner.block_table) == g["prompt_pages"]
    users = [PagedRequest(pool) for _ in range(g["users"])]
    free_before = pool.num_free()
    for u in users:
        u.share_prefix_of(owner)
    assert pool.num_free() == free_before  # sharing allocates nothing
    assert all(pool.refcount[p] == g["refcount_after_share"] for p in owner.block_table)
    assert g["users"] * g["prompt_pages"] == g["naive_pages"]
    assert len({p for u in users for p in u.block_table}) == g["shared_pages"]
    per_token = GOLDEN["kv_cost"]["bytes_per_token"]
    saved = (g["naive_pages"] - g["shared_pages"]) * 16 * per_token
    assert saved == g["saved_mb"] * (1 << 20)
    # the third user writes its first own token: its last shared page is copied
    r = users[g["cow_request"]]
    slot, cow = r.generate_token()
    assert cow == (g["cow_src_page"], g["cow_new_page"])
    assert r.block_table[-1] == g["cow_new_page"]
    assert pool.refcount[g["cow_src_page"]] == g["refcount_src_after_cow"]
    assert pool.refcount[g["cow_new_page"]] == 1
    # the token lands in the private copy at the offset after the 200 prompt tokens
    assert slot == g["cow_new_page"] * 16 + g["prompt_tokens"] % 16
    # the other holders still point at the original page
    for i, u in enumerate(users):
        if i != g["cow_request"]:
            assert u.block_table[-1] == g["cow_src_page"]


def test_last_holder_writes_in_place():
    pool = PagePool(8)
    a = PagedRequest(pool)
    for _ in range(5):
        a.generate_token()
    b = PagedRequest(pool)
    b.share_prefix_of(a)
    _, cow = b.generate_token()  # shared: copies
    assert cow == (0, 1)
    _, cow = a.generate_token()  # a is now the only holder of page 0
    assert cow is None and a.block_table == [0]
    assert pool.refcount[0] == 1


def test_pool_exhaustion_and_double_free():
    pool = PagePool(2)
    pool.allocate()
    pool.allocate()
    with pytest.raises(oracle.PoolExhausted):
        pool.allocate()
    pool.free(0)
    with pytest.raises(ValueError):
        pool.free(0)


def test_utilisation_sweep():
    g = GOLDEN["utilisation_sweep"]
    rng = np.random.default_rng(0)
    for n in g["batch_sizes"]:
        naive, paged = [], []
        for _ in range(20):
            t = np.clip(rng.normal(g["mean"], g["std"], size=n), g["clip_lo"], g["clip_hi"])
            t = np.round(t).astype(int)
            naive.append(oracle.naive_utilisation(t, g["clip_hi"]))
            paged.append(oracle.paged_utilisation(t))
        # clipping at 200 lifts the mean a little above 500, so about 24-26 %
        assert abs(100 * np.mean(naive) - g["naive_pct_approx"]) < 2.5
        assert abs(100 * np.mean(paged) - g["paged_pct_approx"]) < 1.0
