"""Pins the fp64 attention oracle to things other than itself.

Each pin comes from the mathematics of decode attention or from a library
routine, never from the oracle's own formula:
  - torch's scaled_dot_product_attention in fp64 on contiguous K/V (the
    paged result must equal the contiguous one: "PagedAttention" wiki
    mirror, "Formulació matemàtica", blockwise computation);
  - closed forms: one cached token returns its V exactly; a zero query or a
    zero scale gives the mean of V; constant V rows give that constant; a
    duplicated token counts twice; a hand-worked two-token example;
  - invariances: physical block placement, logical token order;
  - IEEE binary16 / bfloat16 decoding against numpy / torch.
The mutation test plants plausible mistakes in a copy of the oracle's C
source and checks that these pins catch every one.
"""
import ctypes
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle

BS = 16


def paged_from_contiguous(rng, K, V, num_pool_blocks=None, fill=np.nan):
    """Scatter per-sequence contiguous K/V (lists of [L, H, D]) into a pool
    at random physical blocks.  Independent of the oracle's gather code."""
    lens = [k.shape[0] for k in K]
    need = [math.ceil(n / BS) for n in lens]
    H, D = K[0].shape[1], K[0].shape[2]
    nb = num_pool_blocks or max(1, sum(need))
    perm = rng.permutation(nb)
    kp = np.full((nb, H, BS, D), fill, dtype=K[0].dtype)
    vp = np.full((nb, H, BS, D), fill, dtype=V[0].dtype)
    tables = np.full((len(K), max(1, max(need))), -1, dtype=np.int32)
    pos = 0
    for s, (k, v) in enumerate(zip(K, V)):
        for j in range(need[s]):
            blk = perm[pos]
            pos += 1
            tables[s, j] = blk
            rows = slice(j * BS, min((j + 1) * BS, k.shape[0]))
            n = rows.stop - rows.start
            kp[blk, :, :n, :] = np.transpose(k[rows], (1, 0, 2))
            vp[blk, :, :n, :] = np.transpose(v[rows], (1, 0, 2))
    return kp, vp, tables, np.array(lens, dtype=np.int32)


def sdpa_reference(q, K, V, scale):
    """torch SDPA in fp64, one sequence at a time on contiguous arrays."""
    outs = []
    for s in range(q.shape[0]):
        qs = torch.from_numpy(q[s].astype(np.float64))[:, None, :]        # [H,1,D]
        ks = torch.from_numpy(K[s].astype(np.float64)).transpose(0, 1)    # [H,L,D]
        vs = torch.from_numpy(V[s].astype(np.float64)).transpose(0, 1)
        o = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, scale=scale)
        outs.append(o[:, 0, :].numpy())
    return np.stack(outs)


def random_problem(seed, lens, H=3, D=8, dtype=np.float32):
    rng = np.random.default_rng(seed)
    K = [rng.standard_normal((n, H, D)).astype(dtype) for n in lens]
    V = [rng.standard_normal((n, H, D)).astype(dtype) for n in lens]
    q = rng.standard_normal((len(lens), H, D)).astype(dtype)
    return rng, q, K, V


# ---- library routine --------------------------------------------------------------

@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_matches_torch_sdpa(dtype):
    lens = [1, 5, 16, 17, 40, 33]
    rng, q, K, V = random_problem(1, lens, H=3, D=8, dtype=dtype)
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V, num_pool_blocks=20)
    scale = 0.37
    got = oracle.decode_attention(q, kp, vp, tables, cl, scale)
    ref = sdpa_reference(q, K, V, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_matches_torch_sdpa_gqa():
    """4 query heads over 2 KV heads: query head h reads KV head h // 2."""
    lens = [3, 18, 31]
    rng, q, K, V = random_problem(2, lens, H=2, D=8)
    q4 = rng.standard_normal((len(lens), 4, 8)).astype(np.float32)
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    got = oracle.decode_attention(q4, kp, vp, tables, cl, 0.5)
    Krep = [np.repeat(k, 2, axis=1) for k in K]
    Vrep = [np.repeat(v, 2, axis=1) for v in V]
    ref = sdpa_reference(q4, Krep, Vrep, 0.5)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---- closed forms -----------------------------------------------------------------

def test_length_one_returns_v_exactly():
    rng, q, K, V = random_problem(3, [1, 1, 1], H=2, D=8, dtype=np.float16)
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V, num_pool_blocks=7)
    got = oracle.decode_attention(q, kp, vp, tables, cl, 0.125)
    want = np.stack([v[0] for v in V]).astype(np.float64)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("mode", ["zero_q", "zero_scale"])
def test_uniform_weights_give_mean_of_v(mode):
    rng, q, K, V = random_problem(4, [7, 16, 29], H=2, D=8)
    if mode == "zero_q":
        q[:] = 0
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    got = oracle.decode_attention(q, kp, vp, tables, cl, 0.0 if mode == "zero_scale" else 0.3)
    want = np.stack([v.astype(np.float64).mean(axis=0) for v in V])
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_constant_v_rows_give_the_constant():
    rng, q, K, V = random_problem(5, [9, 40], H=2, D=8)
    c = rng.standard_normal((2, 8)).astype(np.float32)
    V = [np.broadcast_to(c, v.shape).copy() for v in V]
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    got = oracle.decode_attention(q, kp, vp, tables, cl, 0.9)
    for s in range(2):
        np.testing.assert_allclose(got[s], c.astype(np.float64), rtol=1e-13, atol=1e-13)


def test_duplicated_token_counts_twice():
    rng = np.random.default_rng(6)
    D = 8
    q = rng.standard_normal((1, 1, D)).astype(np.float32)
    a_k, b_k = rng.standard_normal((2, D)).astype(np.float32)
    a_v, b_v = rng.standard_normal((2, D)).astype(np.float32)
    K = [np.stack([a_k, b_k, b_k])[:, None, :]]
    V = [np.stack([a_v, b_v, b_v])[:, None, :]]
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    scale = 0.7
    got = oracle.decode_attention(q, kp, vp, tables, cl, scale)[0, 0]
    qa = scale * float(np.dot(q[0, 0].astype(np.float64), a_k.astype(np.float64)))
    qb = scale * float(np.dot(q[0, 0].astype(np.float64), b_k.astype(np.float64)))
    wa, wb = math.exp(qa), 2.0 * math.exp(qb)
    want = (wa * a_v.astype(np.float64) + wb * b_v.astype(np.float64)) / (wa + wb)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_hand_worked_two_tokens():
    """q=(1,0), k0=(1,0), k1=(0,1), v0=(1,2), v1=(3,4), scale 1:
    weights e and 1, so out = ((e+3)/(e+1), (2e+4)/(e+1))."""
    q = np.array([[[1, 0]]], dtype=np.float32)
    K = [np.array([[[1, 0]], [[0, 1]]], dtype=np.float32)]
    V = [np.array([[[1, 2]], [[3, 4]]], dtype=np.float32)]
    kp, vp, tables, cl = paged_from_contiguous(np.random.default_rng(0), K, V)
    got = oracle.decode_attention(q, kp, vp, tables, cl, 1.0)[0, 0]
    e = math.e
    np.testing.assert_allclose(got, [(e + 3) / (e + 1), (2 * e + 4) / (e + 1)], rtol=1e-15)


def test_dominant_score_selects_its_value():
    rng, q, K, V = random_problem(7, [37], H=1, D=8)
    q[0, 0] = 0
    q[0, 0, 0] = 1
    K[0][:, 0, 0] = 0
    K[0][21, 0, 0] = 60.0  # score 60 above every other: weight ratio e^-60
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    got = oracle.decode_attention(q, kp, vp, tables, cl, 1.0)[0, 0]
    np.testing.assert_allclose(got, V[0][21, 0].astype(np.float64), rtol=1e-20, atol=1e-20)


def test_empty_sequence_gives_zeros():
    rng, q, K, V = random_problem(8, [4], H=1, D=8)
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    cl[:] = 0
    got = oracle.decode_attention(q, kp, vp, tables, cl, 1.0)
    assert np.array_equal(got, np.zeros_like(got))


# ---- invariances ------------------------------------------------------------------

def test_block_placement_is_bit_invariant():
    lens = [3, 16, 45, 64]
    _, q, K, V = random_problem(9, lens, H=2, D=8, dtype=np.float16)
    outs = []
    for placement_seed in range(3):
        kp, vp, tables, cl = paged_from_contiguous(np.random.default_rng(placement_seed), K, V,
                                                   num_pool_blocks=30)
        outs.append(oracle.decode_attention(q, kp, vp, tables, cl, 0.25))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_token_order_invariance():
    lens = [21, 50]
    rng, q, K, V = random_problem(10, lens, H=2, D=8)
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V)
    a = oracle.decode_attention(q, kp, vp, tables, cl, 0.4)
    perms = [rng.permutation(n) for n in lens]
    K2 = [k[p] for k, p in zip(K, perms)]
    V2 = [v[p] for v, p in zip(V, perms)]
    kp2, vp2, tables2, cl2 = paged_from_contiguous(rng, K2, V2)
    b = oracle.decode_attention(q, kp2, vp2, tables2, cl2, 0.4)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def test_unused_slots_and_table_entries_are_never_read():
    """Pool slots past each length are NaN and table entries past the last
    block are garbage ids: the result must stay finite and unchanged."""
    lens = [5, 17, 33]
    rng, q, K, V = random_problem(11, lens, H=2, D=8)
    kp, vp, tables, cl = paged_from_contiguous(rng, K, V, fill=np.nan)
    a = oracle.decode_attention(q, kp, vp, tables, cl, 0.3)
    assert np.isfinite(a).all()
    t2 = tables.copy()
    t2[t2 < 0] = 10 ** 6
    b = oracle.decode_attention(q, kp, vp, t2, cl, 0.3)
    assert np.array_equal(a, b)


# ---- number formats ---------------------------------------------------------------

def test_half_decoding_all_bit_patterns():
    lib = oracle._load()
    bits = np.arange(1 << 16, dtype=np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    got = np.array([lib.oracle_half_to_double(int(b)) for b in bits])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_bf16_decoding_sample():
    lib = oracle._load()
    bits = np.random.default_rng(0).integers(0, 1 << 16, size=4096).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([lib.oracle_bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(t)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], t[~nan])


# ---- cache maintenance ------------------------------------------------------------

def test_reshape_and_cache_hand_example():
    H, D = 2, 4
    kp = np.zeros((3, H, BS, D), dtype=np.float16)
    vp = np.zeros_like(kp)
    k_new = np.arange(3 * H * D, dtype=np.float16).reshape(3, H, D) + 1
    v_new = -k_new
    slots = np.array([17, -1, 47], dtype=np.int32)  # block 1 offset 1; padding; block 2 offset 15
    oracle.reshape_and_cache(k_new, v_new, slots, kp, vp)
    want_k = np.zeros_like(kp)
    want_k[1, :, 1, :] = k_new[0]
    want_k[2, :, 15, :] = k_new[2]
    assert np.array_equal(kp, want_k)
    assert np.array_equal(vp, -want_k)


def test_copy_blocks_matches_numpy():
    rng = np.random.default_rng(12)
    kp = rng.standard_normal((10, 3, BS, 8)).astype(np.float16)
    vp = rng.standard_normal((10, 3, BS, 8)).astype(np.float16)
    pairs = np.array([[2, 7], [0, 9], [5, 1]], dtype=np.int32)
    want_k, want_v = kp.copy(), vp.copy()
    want_k[pairs[:, 1]] = kp[pairs[:, 0]]
    want_v[pairs[:, 1]] = vp[pairs[:, 0]]
    oracle.copy_blocks(kp, vp, pairs)
    assert np.array_equal(kp, want_k) and np.array_equal(vp, want_v)


def test_slot_of():
    row = np.array([5, 2, 9], dtype=np.int32)
    assert oracle.slot_of_c(row, 20) == 2 * 16 + 4
    assert oracle.slot_of_c(row, 0) == 80
    assert oracle.slot_of_c(row, 47) == 9 * 16 + 15
    for pos in range(48):
        assert oracle.slot_of_c(row, pos) == oracle.slot_of(list(row), pos)


# ---- the pins catch planted mistakes ----------------------------------------------

MUTATIONS = {
    "scale_dropped": ("x[t] = scale * acc;", "x[t] = acc;"),
    "k_for_v": ("V[(int64_t)t * head_dim + d] = load_elem(v_pool", "V[(int64_t)t * head_dim + d] = load_elem(k_pool"),
    "offset_off_by_one": ("int64_t off = t % block_size;", "int64_t off = (t + 1) % block_size;"),
    "wrong_kv_head": ("const int32_t kvh = h / group;", "const int32_t kvh = h % group;"),
    "weight_perturbed": ("x[t] = exp(x[t] - m);", "x[t] = exp(x[t] - m) + 1e-3;"),
    "last_token_dropped": ("for (int32_t t = 0; t < L; ++t) acc += x[t]", "for (int32_t t = 0; t < L - 1; ++t) acc += x[t]"),
    "half_exponent_bias": ("expo - 25", "expo - 24"),
}


def _mutated_lib(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attention.c")).read()
    assert old in src, name
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", str(path), "-o", str(so), "-lm"],
                   check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistakes(name, tmp_path, monkeypatch):
    so = _mutated_lib(tmp_path, name, *MUTATIONS[name])
    lib = ctypes.CDLL(so)
    saved = oracle._lib
    oracle._lib = None
    real_build = oracle.build
    monkeypatch.setattr(oracle, "build", lambda force=False: so)
    try:
        pins = [lambda: test_matches_torch_sdpa(np.float16), test_matches_torch_sdpa_gqa,
                test_length_one_returns_v_exactly, test_hand_worked_two_tokens]
        caught = 0
        for pin in pins:
            try:
                pin()
            except AssertionError:
                caught += 1
        assert caught >= 1, f"mutation {name} slipped past every pin"
    finally:
        oracle._lib = saved
        monkeypatch.setattr(oracle, "build", real_build)
    del lib
    shutil.rmtree(tmp_path, ignore_errors=True)
