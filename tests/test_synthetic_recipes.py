"""The seeded input recipes produce the workloads their descriptions state:
lengths, sizes and placements (the generators hold none of the method's
arithmetic; this pins them so that the figures quoted for each workload --
cached tokens, pool blocks -- stay the generator's)."""
import math

import numpy as np

from paged_kv_cache_478_b200 import synthetic as syn

BS = 16


def _check_tables(tables, lens, num_blocks, exact):
    """Each sequence's first ceil(L/16) entries are distinct pool ids, the rest
    are -1; with `exact` the ids used are exactly the pool."""
    used = []
    for s, L in enumerate(lens):
        n = math.ceil(int(L) / BS)
        assert np.all(tables[s, n:] == -1)
        used.extend(tables[s, :n].tolist())
    assert len(set(used)) == len(used)
    assert min(used) >= 0 and max(used) < num_blocks
    if exact:
        assert sorted(used) == list(range(num_blocks))


def test_tiny_case():
    c = syn.tiny_case(0)
    assert c["context_lens"].tolist() == [1, 15, 16, 33]
    assert c["k_pool"].shape == (16, 2, BS, 64) and c["k_pool"].dtype == np.float32
    assert c["scale"] == 1 / 8
    _check_tables(c["block_tables"], c["context_lens"], 16, exact=False)


def test_single_layer_lengths():
    lens = syn.single_layer_lengths(0)
    assert lens.shape == (64,) and lens.min() >= 1 and lens.max() <= 2048
    assert int(lens.sum()) == 66850


def test_full_step_workload():
    lens = syn.full_step_lengths(0)
    assert lens.shape == (200,) and lens.min() >= 1 and lens.max() <= 2048
    assert int(lens.sum()) == 111857
    tables, nb = syn.full_step_tables(0, lens)
    assert nb == 7092 and tables.shape == (200, 128)
    _check_tables(tables, lens, nb, exact=True)
    # 512 KB of K and V per token over 32 layers x 32 heads x 128 fp16
    assert int(lens.sum()) * 32 * 32 * 128 * 2 * 2 == 58645282816


def test_long_context_workload():
    lens, tables, nb = syn.long_context_tables(0)
    assert lens.tolist() == [32768] * 8 and nb == 16384 and tables.shape == (8, 2048)
    _check_tables(tables, lens, nb, exact=True)


def test_shared_prefix_case():
    c = syn.shared_prefix_case(0, heads=2, head_dim=16)
    assert c["prefix_len"] == 1000 and math.ceil(1000 / BS) == 63
    suf = c["suffix_lens"]
    assert suf.shape == (128,) and suf.min() >= 1 and suf.max() <= 512
    assert c["k_prefix"].shape == (1000, 2, 16) and c["k_prefix"].dtype == np.float16
    assert [k.shape[0] for k in c["k_suffix"]] == suf.tolist()
    assert c["q"].shape == (128, 2, 16)
