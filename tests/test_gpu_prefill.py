"""Paged prefill (tcgen05) against the oracle.

Each new query token at position p must equal single-query attention over
tokens 0..p of its sequence ("PagedAttention" wiki mirror, "Formulació
matemàtica": the block-wise computation holds for every query), so the
oracle is the pinned decode oracle run once per query token with
context_len = p + 1 on the same block table."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_478_b200 as pa
from tests.gpu_cases import assert_parity, dev

pytestmark = pytest.mark.gpu


def _case(seed, ctx_new, kv_heads, group, head_dim, dtype, wide_v=0):
    rng = np.random.default_rng(seed)
    S = len(ctx_new)
    lens = np.array([c for c, _ in ctx_new], dtype=np.int32)
    news = np.array([n for _, n in ctx_new], dtype=np.int32)
    need = [math.ceil(int(L) / 16) for L in lens]
    nb = sum(need) + 5
    maxb = max(need)
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((S, maxb), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    shape = (nb, kv_heads, 16, head_dim)
    kf = rng.standard_normal(shape).astype(np.float32)
    vf = rng.standard_normal(shape).astype(np.float32)
    if wide_v:  # values an fp16 V cannot hold, at random places
        at = tuple(rng.integers(0, n, wide_v) for n in shape)
        vf[at] = rng.choice([-1.0, 1.0], wide_v) * rng.uniform(7.0e4, 3.0e5, wide_v)
    T = int(news.sum())
    qf = rng.standard_normal((T, kv_heads * group, head_dim)).astype(np.float32)
    qs = np.concatenate([[0], np.cumsum(news)]).astype(np.int32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    kt, vt, qt = (torch.from_numpy(x).to(tdt) for x in (kf, vf, qf))
    if dtype == "bf16":
        kh, vh, qh = (x.view(torch.int16).numpy().view(np.uint16) for x in (kt, vt, qt))
        odt = oracle.BF16
    else:
        kh, vh, qh = (x.numpy() for x in (kt, vt, qt))
        odt = None
    # oracle: one decode row per query token, context = its position + 1
    rows_t, rows_l = [], []
    for s in range(S):
        for i in range(int(news[s])):
            rows_t.append(tables[s])
            rows_l.append(int(lens[s]) - int(news[s]) + i + 1)
    scale = 1 / math.sqrt(head_dim)
    ref = oracle.decode_attention(qh, kh, vh, np.stack(rows_t), np.array(rows_l, np.int32),
                                  scale, dtype=odt)
    pool = pa.pa_pool_create(nb, 16, kv_heads, head_dim, tdt)
    pa.pa_pool_set_query_heads(pool, kv_heads * group)
    return dict(pool=pool, q=qt.cuda(), k=kt.cuda(), v=vt.cuda(), tables=dev(tables),
                lens=dev(lens), qs=dev(qs), max_new=int(news.max()), ref=ref, scale=scale,
                tables_h=tables)


CASES = [(1, 1), (17, 17), (200, 64), (300, 300), (1000, 129), (128, 128), (2048, 256),
         (700, 1), (45, 13)]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [128, 64])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_prefill_matches_the_oracle(dtype, head_dim, group):
    c = _case(70 + group, CASES, 2, group, head_dim, dtype)
    out = torch.empty_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], c["lens"], c["qs"],
                            c["scale"], out, c["max_new"])
    assert pa.pa_device_errors() == 0
    assert torch.isfinite(out.float()).all()
    assert_parity(out, c["ref"], f"prefill {dtype} D={head_dim} G={group}")


def test_prefill_single_new_token_matches_decode():
    """n = 1 is decode: the two paths agree within the gate."""
    ctx = [(1, 1), (16, 1), (17, 1), (513, 1), (2000, 1)]
    c = _case(80, ctx, 4, 1, 128, "f16")
    out = torch.empty_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], c["lens"], c["qs"],
                            c["scale"], out, 1)
    d_out = torch.empty_like(c["q"])
    ws = torch.empty(pa.pa_decode_workspace_bytes(c["pool"], len(ctx), c["tables"].shape[1]),
                     dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], c["lens"], c["scale"],
                           d_out, ws)
    assert pa.pa_device_errors() == 0
    assert_parity(out, c["ref"], "prefill n=1")
    assert_parity(d_out, c["ref"], "decode")


def test_prefill_rejects_a_context_shorter_than_its_new_tokens():
    c = _case(81, [(40, 20), (30, 10)], 2, 1, 64, "f16")
    bad = torch.tensor([40, 5], dtype=torch.int32, device="cuda")  # 5 < 10 new tokens
    out = torch.zeros_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], bad, c["qs"],
                            c["scale"], out, 20)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN
    assert_parity(out[:20], c["ref"][:20], "the valid sequence still runs")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_ignores_poisoned_rows_past_the_context(dtype):
    """Pool rows past each context and blocks that no table holds are NaN: a
    masked score and a zero weight must never meet them (0 x NaN in P.V)."""
    ctx = [(45, 13), (300, 300), (17, 17), (1000, 129), (200, 64), (64, 64)]
    c = _case(82, ctx, 2, 1, 128, dtype)
    k, v = c["k"], c["v"]
    used = np.zeros(k.shape[0], dtype=bool)
    for s, (L, _) in enumerate(ctx):
        nblk = math.ceil(L / 16)
        blocks = c["tables_h"][s, :nblk]
        used[blocks] = True
        last, rows = int(blocks[-1]), L - (nblk - 1) * 16
        k[last, :, rows:] = float("nan")
        v[last, :, rows:] = float("nan")
    free = torch.from_numpy(np.nonzero(~used)[0]).cuda()
    k[free] = float("nan")
    v[free] = float("nan")
    out = torch.empty_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], k, v, c["tables"], c["lens"], c["qs"], c["scale"],
                            out, c["max_new"])
    assert pa.pa_device_errors() == 0
    assert torch.isfinite(out.float()).all()
    assert_parity(out, c["ref"], f"prefill {dtype} with NaN past the context")


def test_prefill_skips_and_reports_a_sequence_beyond_max_new_tokens():
    """max_new_tokens sizes the launch; a sequence with more new tokens than
    that is reported and left untouched, the others still run."""
    c = _case(83, [(300, 300), (40, 20)], 2, 1, 128, "f16")
    out = torch.zeros_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], c["lens"], c["qs"],
                            c["scale"], out, 256)  # sequence 0 has 300 > 256
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN
    assert torch.count_nonzero(out[:300]) == 0
    assert_parity(out[300:], c["ref"][300:], "the sequence within the bound still runs")


def test_prefill_skips_a_sequence_whose_rows_fall_outside_q():
    """query_start is device data: a sequence whose rows run past the q/out
    rows (num_tokens) is reported and skipped, and nothing outside is read or
    written."""
    c = _case(84, [(64, 32), (40, 20)], 2, 1, 128, "f16")
    bad_qs = torch.tensor([0, 32, 60], dtype=torch.int32, device="cuda")  # 60 > 52 rows
    out = torch.zeros_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], c["lens"], bad_qs,
                            c["scale"], out, 32)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT_LEN
    assert torch.count_nonzero(out[32:]) == 0
    assert_parity(out[:32], c["ref"][:32], "the sequence inside q still runs")


@pytest.mark.parametrize("kv_heads,group", [(32, 1), (8, 4)])
def test_prefill_with_several_items_per_cta(kv_heads, group):
    """fp16 runs one persistent CTA per SM, each walking several 256-query
    items in turn, with the next item's first products overlapping the end of
    the current one.  384 items here (32 query heads x 3 prompts x 4 pairs),
    so every CTA takes two or three; sampled rows against the oracle,
    including the first and last rows of each query tile."""
    ctx = [(1500, 1024), (1100, 1024), (1024, 1000)]
    rng = np.random.default_rng(90 + group)
    S, D = len(ctx), 128
    lens = np.array([c for c, _ in ctx], dtype=np.int32)
    news = np.array([n for _, n in ctx], dtype=np.int32)
    need = [math.ceil(int(L) / 16) for L in lens]
    nb = sum(need) + 3
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((S, max(need)), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    kt = torch.from_numpy(rng.standard_normal((nb, kv_heads, 16, D)).astype(np.float32)).half()
    vt = torch.from_numpy(rng.standard_normal((nb, kv_heads, 16, D)).astype(np.float32)).half()
    T = int(news.sum())
    qt = torch.from_numpy(rng.standard_normal((T, kv_heads * group, D)).astype(np.float32)).half()
    qs = np.concatenate([[0], np.cumsum(news)]).astype(np.int32)
    pool = pa.pa_pool_create(nb, 16, kv_heads, D, torch.float16)
    pa.pa_pool_set_query_heads(pool, kv_heads * group)
    out = torch.empty_like(qt.cuda())
    scale = 1 / math.sqrt(D)
    pa.pa_prefill_attention(pool, qt.cuda(), kt.cuda(), vt.cuda(), dev(tables), dev(lens), dev(qs),
                            scale, out, int(news.max()))
    assert pa.pa_device_errors() == 0
    rows, row_t, row_l = [], [], []
    for s in range(S):
        n = int(news[s])
        pick = {0, 127, 128, 255, 256, 511, 512, n - 1}
        pick |= set(rng.choice(n, 24, replace=False).tolist())
        for i in sorted(p for p in pick if p < n):
            rows.append(int(qs[s]) + i)
            row_t.append(tables[s])
            row_l.append(int(lens[s]) - n + i + 1)
    ref = oracle.decode_attention(qt.numpy()[rows], kt.numpy(), vt.numpy(), np.stack(row_t),
                                  np.array(row_l, np.int32), scale)
    assert_parity(out[rows], ref, f"prefill, several items per CTA, G={group}")


@pytest.mark.parametrize("head_dim,group", [(128, 1), (64, 4)])
def test_prefill_bf16_keeps_v_values_beyond_fp16_range(head_dim, group):
    """bf16 pools hold values no fp16 operand could (|v| up to 3e5 here, at
    random places in many tiles): the products stay in bf16 (P as a high part
    plus residual), so the result matches the oracle and stays finite."""
    c = _case(91 + group, CASES, 2, group, head_dim, "bf16", wide_v=60)
    out = torch.empty_like(c["q"])
    pa.pa_prefill_attention(c["pool"], c["q"], c["k"], c["v"], c["tables"], c["lens"], c["qs"],
                            c["scale"], out, c["max_new"])
    assert pa.pa_device_errors() == 0
    assert torch.isfinite(out.float()).all()
    assert float(np.abs(c["ref"]).max()) > 100.0  # the wide values reach the outputs
    assert_parity(out, c["ref"], f"prefill bf16 wide V D={head_dim} G={group}")
