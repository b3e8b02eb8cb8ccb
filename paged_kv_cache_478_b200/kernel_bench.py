"""Per-kernel timings on synthetic workloads (CUDA events on the launching stream).

    python -m paged_kv_cache_478_b200.kernel_bench prefill [--small | --profile]
    python -m paged_kv_cache_478_b200.kernel_bench gqa [--groups 4,8] [--profile]
    python -m paged_kv_cache_478_b200.kernel_bench shared-prefix [--profile]
    python -m paged_kv_cache_478_b200.kernel_bench long-context [--profile]
    python -m paged_kv_cache_478_b200.kernel_bench single-layer [--profile]
    python -m paged_kv_cache_478_b200.kernel_bench cache-ops [--profile]
    python -m paged_kv_cache_478_b200.kernel_bench decode-dtypes

Each line printed is one JSON object.  These are the measurements behind the
per-kernel tables of the design notes; the headline decode step is bench.py.
`prefill --small` runs three launches of one small case (2 prompts x 2048
tokens) and prints nothing timed: it is the command the profiler captures.
`--profile` does the same for the other workloads: the same inputs, a few
plain launches (no CUDA graph, no timing), so that a profiler capture of
one launch stays small and ends by itself.
"""
from __future__ import annotations

import argparse
import json
import math

import numpy as np
import torch

import paged_kv_cache_478_b200 as pa
from paged_kv_cache_478_b200 import synthetic as syn


def _events_ms(fn, reps: int, warmup: int = 3, flush: torch.Tensor | None = None) -> float:
    """Median milliseconds of fn() over reps, each bracketed by its own pair of
    events on the current stream; with `flush`, L2 is overwritten before every
    rep (outside the events).  All reps are queued before one synchronise, so
    the device never waits on the host between an event pair."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    pairs = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    return float(np.median([e0.elapsed_time(e1) for e0, e1 in pairs]))


def _graph_us(fn, launches: int = 50, reps: int = 20) -> float:
    """Device microseconds per call of a short kernel: `launches` calls are
    captured into one CUDA graph and replayed, so host launch cost (larger
    than these kernels) stays out; median over reps."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(launches):
            fn()
    ms = _events_ms(g.replay, reps)
    del g
    return ms * 1e3 / launches


def _check():
    err = pa.pa_device_errors()
    if err:
        raise RuntimeError(f"device error bits 0x{err:x}")


def _prefill_case(seqs, new_tokens, kv_heads, group, head_dim, dtype, seed=0):
    lens = np.full(seqs, new_tokens, dtype=np.int32)
    need = math.ceil(new_tokens / 16)
    nb = seqs * need
    tables = np.random.default_rng(seed).permutation(nb).astype(np.int32).reshape(seqs, need)
    kp = torch.empty((nb, kv_heads, 16, head_dim), dtype=dtype, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 1)
    syn.fill_normal_device(vp, 2)
    q = torch.empty((seqs * new_tokens, kv_heads * group, head_dim), dtype=dtype, device="cuda")
    syn.fill_normal_device(q, 3)
    qs = torch.arange(0, seqs * new_tokens + 1, new_tokens, dtype=torch.int32, device="cuda")
    pool = pa.pa_pool_create(nb, 16, kv_heads, head_dim, dtype)
    pa.pa_pool_set_query_heads(pool, kv_heads * group)
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    out = torch.empty_like(q)
    scale = 1 / math.sqrt(head_dim)

    def run():
        pa.pa_prefill_attention(pool, q, kp, vp, bt, cl, qs, scale, out, new_tokens)

    # causal attention of fresh prompts: Q.K^T and P.V over the lower triangle
    flops = 4.0 * seqs * kv_heads * group * head_dim * new_tokens * (new_tokens + 1) / 2
    return run, flops


def prefill(small: bool, profile: bool = False):
    if small:
        run, _ = _prefill_case(2, 2048, 32, 1, 128, torch.float16)
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        _check()
        print(json.dumps({"prefill_small_case": "2 x 2048 fp16, 32 heads x 128, 3 launches"}))
        return
    if profile:
        run, _ = _prefill_case(4, 4096, 32, 1, 128, torch.float16)
        _profile_launches(run, "prefill, 4 prompts x 4096 fp16, 32 heads x 128")
        return
    for seqs, n, hk, g, dt in [(4, 4096, 32, 1, torch.float16), (8, 2048, 32, 1, torch.float16),
                               (16, 1024, 8, 4, torch.float16), (8, 2048, 32, 1, torch.bfloat16)]:
        run, flops = _prefill_case(seqs, n, hk, g, 128, dt)
        ms = _events_ms(run, 20)
        _check()
        print(json.dumps({"kernel": "paged_prefill_kernel", "prompts": seqs, "new_tokens": n,
                          "q_heads": hk * g, "kv_heads": hk, "dtype": str(dt).split(".")[-1],
                          "ms": round(ms, 4), "TFLOPs": round(flops / ms / 1e9, 1)}), flush=True)


_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def gqa(partition_size: int = 0, dtype: str = "f16", profile: bool = False, groups=(1, 2, 4, 8)):
    S, HK, D = 200, 8, 128
    dt = _DTYPES[dtype]
    elt = torch.tensor([], dtype=dt).element_size()
    lens = syn.full_step_lengths(0, S)
    tables, nb = syn.full_step_tables(0, lens)
    kp = torch.empty((nb, HK, 16, D), dtype=dt, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 1)
    syn.fill_normal_device(vp, 2)
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    kv_bytes = int(lens.sum()) * HK * D * elt * 2
    for G in groups:
        pool = pa.pa_pool_create(nb, 16, HK, D, dt)
        pa.pa_pool_set_query_heads(pool, HK * G)
        q = torch.randn((S, HK * G, D), dtype=dt, device="cuda")
        kn = torch.randn((S, HK, D), dtype=dt, device="cuda")
        vn = torch.randn_like(kn)
        out = torch.empty_like(q)
        ws = torch.empty(pa.pa_decode_workspace_bytes(pool, S, tables.shape[1], 0, partition_size),
                         dtype=torch.uint8, device="cuda")
        pa.pa_decode_plan(pool, cl, tables.shape[1], ws, partition_size=partition_size)
        run = lambda: pa.pa_decode_append_attention_planned(  # noqa: E731
            pool, q, kn, vn, kp, vp, bt, 1 / math.sqrt(D), out, ws, partition_size=partition_size)
        if profile:
            _profile_launches(run, f"GQA decode, {G} query heads per KV head")
            continue
        ms = _events_ms(run, 50)
        _check()
        print(json.dumps({"kernel": "decode (GQA)", "dtype": dtype, "q_per_kv": G, "kv_heads": HK,
                          "partition_size": partition_size or "auto",
                          "us": round(ms * 1e3, 1), "kv_GBps": round(kv_bytes / ms / 1e6, 1)}),
              flush=True)


def shared_prefix(profile: bool = False):
    H, D, S, P = 32, 128, 128, 1000
    case = syn.shared_prefix_case(0)
    nb = 63 + S + sum(math.ceil(int(n) / 16) for n in case["suffix_lens"])
    bm = pa.BlockManager(nb)
    maxb = math.ceil((P + 512) / 16)
    tables = np.full((S, maxb), -1, dtype=np.int32)
    lens = np.zeros(S, dtype=np.int32)
    lens[0], _, _ = bm.append_tokens(tables[0], 0, P)
    for s in range(1, S):
        bm.fork_table(tables[0], 63, tables[s])
        lens[s] = P
    for s in range(S):
        lens[s], _, _ = bm.append_tokens(tables[s], int(lens[s]), int(case["suffix_lens"][s]))
    kp = torch.empty((nb, H, 16, D), dtype=torch.float16, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 3)
    syn.fill_normal_device(vp, 4)
    pool = pa.pa_pool_create(nb, 16, H, D, torch.float16)
    q = torch.randn((S, H, D), dtype=torch.float16, device="cuda")
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    groups = pa.pa_find_shared_prefixes(tables, lens)
    gd = dict(groups)
    for k in ("offsets", "members", "blocks"):
        gd[k] = torch.from_numpy(groups[k]).cuda()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    used = {int(b) for s in range(S) for b in tables[s, :math.ceil(int(lens[s]) / 16)]}
    unique = len(used) * H * 16 * D * 2 * 2
    logical = int(lens.sum()) * H * D * 2 * 2
    out1, out2 = torch.empty_like(q), torch.empty_like(q)
    ws1 = torch.empty(pa.pa_decode_workspace_bytes(pool, S, maxb), dtype=torch.uint8, device="cuda")
    ws2 = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(pool, S, maxb,
                                                                  groups["max_shared_blocks"]),
                      dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(D)
    plain = lambda: pa.pa_decode_attention(pool, q, kp, vp, bt, cl, scale, out1, ws1)  # noqa: E731
    shared = lambda: pa.pa_decode_attention_shared_prefix(  # noqa: E731
        pool, q, kp, vp, bt, cl, gd, scale, out2, ws2)
    if profile:
        _profile_launches(shared, "shared-prefix path: plan + shared-prefix kernel + decode")
        return
    rows = []
    for l2, fl in (("flushed before every rep", flush), ("warm", None)):
        rows.append(("plain decode", l2, _events_ms(plain, 50, flush=fl)))
        rows.append(("shared-prefix path", l2, _events_ms(shared, 50, flush=fl)))
    _check()
    diff = (out1.float() - out2.float()).abs().max().item()
    for name, l2, ms in rows:
        print(json.dumps({"kernel": name, "sequences": S, "shared_prefix_tokens": P,
                          "us": round(ms * 1e3, 1), "logical_GBps": round(logical / ms / 1e6, 1),
                          "unique_GBps": round(unique / ms / 1e6, 1),
                          "max_abs_diff_vs_plain": diff, "l2": l2}), flush=True)


def _profile_launches(fn, what: str, n: int = 3):
    """n plain launches of fn for a profiler to capture; nothing is timed."""
    for _ in range(n):
        fn()
    torch.cuda.synchronize()
    _check()
    print(json.dumps({"profile_launches": n, "workload": what}), flush=True)


def long_context(partition_size: int = 0, profile: bool = False):
    S, H, D, CTX = 8, 32, 128, 32768
    lens, tables, nb = syn.long_context_tables(0, S, CTX)
    kp = torch.empty((nb, H, 16, D), dtype=torch.float16, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 1)
    syn.fill_normal_device(vp, 2)
    q = torch.randn((S, H, D), dtype=torch.float16, device="cuda")
    kn, vn = torch.randn_like(q), torch.randn_like(q)
    pool = pa.pa_pool_create(nb, 16, H, D, torch.float16)
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    ws = torch.empty(pa.pa_decode_workspace_bytes(pool, S, tables.shape[1], 0, partition_size),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode_plan(pool, cl, tables.shape[1], ws, partition_size=partition_size)
    run = lambda: pa.pa_decode_append_attention_planned(  # noqa: E731
        pool, q, kn, vn, kp, vp, bt, 1 / math.sqrt(D), out, ws, partition_size=partition_size)
    if profile:
        _profile_launches(run, "long context: 8 x 32768 tokens, planned append + attend")
        return
    ms = _events_ms(run, 30)
    _check()
    kv_bytes = int(lens.sum()) * H * D * 2 * 2
    print(json.dumps({"kernel": "decode (long context)", "sequences": S, "context": CTX,
                      "partition_size": partition_size or "auto",
                      "us": round(ms * 1e3, 1), "kv_GBps": round(kv_bytes / ms / 1e6, 1)}))


def single_layer(partition_size: int = 0, profile: bool = False):
    """One layer of 64 sequences, lengths uniform in [1, 2048], 32 heads x 128
    fp16, the pool exactly the used blocks at random places; the new token is
    appended and attended in one launch (about 1.1 GB of K/V, larger than L2)."""
    S, H, D = 64, 32, 128
    lens = syn.single_layer_lengths(0, S)
    tables, nb = syn.full_step_tables(0, lens)
    kp = torch.empty((nb, H, 16, D), dtype=torch.float16, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 1)
    syn.fill_normal_device(vp, 2)
    q = torch.randn((S, H, D), dtype=torch.float16, device="cuda")
    kn, vn = torch.randn_like(q), torch.randn_like(q)
    pool = pa.pa_pool_create(nb, 16, H, D, torch.float16)
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    ws = torch.empty(pa.pa_decode_workspace_bytes(pool, S, tables.shape[1], 0, partition_size),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    run = lambda: pa.pa_decode_append_attention(  # noqa: E731
        pool, q, kn, vn, kp, vp, bt, cl, 1 / math.sqrt(D), out, ws, partition_size=partition_size)
    if profile:
        _profile_launches(run, "single layer: 64 sequences, plan + append + attend")
        return
    ms = _events_ms(run, 50)
    _check()
    kv_bytes = int(lens.sum()) * H * D * 2 * 2
    print(json.dumps({"kernel": "decode (single layer, plan + append + attend)", "sequences": S,
                      "partition_size": partition_size or "auto",
                      "cached_tokens": int(lens.sum()), "us": round(ms * 1e3, 1),
                      "kv_GBps": round(kv_bytes / ms / 1e6, 1)}))


def cache_ops(profile: bool = False):
    """reshape_and_cache and copy_blocks at the sizes of the workloads: one
    decode step's new tokens (200), a long fill (32 768 tokens), and the
    copy-on-write of config 3 (127 block pairs); 32 heads x 128 fp16."""
    H, D = 32, 128
    nb = 4096
    kp = torch.empty((nb, H, 16, D), dtype=torch.float16, device="cuda")
    vp = torch.empty_like(kp)
    syn.fill_normal_device(kp, 1)
    syn.fill_normal_device(vp, 2)
    pool = pa.pa_pool_create(nb, 16, H, D, torch.float16)
    rng = np.random.default_rng(0)
    for T in (200, 32768):
        slots = torch.from_numpy(rng.permutation(nb * 16)[:T].astype(np.int32)).cuda()
        kn = torch.randn((T, H, D), dtype=torch.float16, device="cuda")
        vn = torch.randn_like(kn)
        if profile:
            _profile_launches(lambda: pa.pa_reshape_and_cache(pool, kn, vn, slots, kp, vp),
                              f"reshape_and_cache, {T} tokens", n=1)
            continue
        us = _graph_us(lambda: pa.pa_reshape_and_cache(pool, kn, vn, slots, kp, vp),
                       launches=50 if T <= 1024 else 5)
        _check()
        moved = 2 * 2 * T * H * D * 2  # K and V, read + written
        print(json.dumps({"kernel": "reshape_and_cache", "tokens": T, "us": round(us, 2),
                          "bytes_moved": moved, "GBps": round(moved / us / 1e3, 1)}), flush=True)
    perm = rng.permutation(nb)[:254].astype(np.int32)
    pairs = torch.from_numpy(perm.reshape(127, 2)).cuda()
    if profile:
        _profile_launches(lambda: pa.pa_copy_blocks(pool, kp, vp, pairs), "copy_blocks, 127 pairs",
                          n=1)
        return
    us = _graph_us(lambda: pa.pa_copy_blocks(pool, kp, vp, pairs))
    _check()
    moved = 2 * 2 * 127 * H * 16 * D * 2  # K and V blocks, read + written
    print(json.dumps({"kernel": "copy_blocks", "pairs": 127, "us": round(us, 2), "bytes_moved": moved,
                      "GBps": round(moved / us / 1e3, 1),
                      "l2": "warm: the 32.5 MB of source blocks stay in L2 across replays"}),
          flush=True)


def decode_dtypes():
    """One layer of the full decode step (200 requests, full-step lengths, 32
    heads x 128) for each pool dtype: planned append + attend."""
    S, H, D = 200, 32, 128
    lens = syn.full_step_lengths(0, S)
    tables, nb = syn.full_step_tables(0, lens)
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    for name, dt in _DTYPES.items():
        elt = torch.tensor([], dtype=dt).element_size()
        kp = torch.empty((nb, H, 16, D), dtype=dt, device="cuda")
        vp = torch.empty_like(kp)
        syn.fill_normal_device(kp, 1)
        syn.fill_normal_device(vp, 2)
        q = torch.randn((S, H, D), dtype=dt, device="cuda")
        kn, vn = torch.randn_like(q), torch.randn_like(q)
        out = torch.empty_like(q)
        pool = pa.pa_pool_create(nb, 16, H, D, dt)
        ws = torch.empty(pa.pa_decode_workspace_bytes(pool, S, tables.shape[1]), dtype=torch.uint8,
                         device="cuda")
        pa.pa_decode_plan(pool, cl, tables.shape[1], ws)
        ms = _events_ms(lambda: pa.pa_decode_append_attention_planned(
            pool, q, kn, vn, kp, vp, bt, 1 / math.sqrt(D), out, ws), 30)
        _check()
        kv_bytes = int(lens.sum()) * H * D * elt * 2
        print(json.dumps({"kernel": "decode (one full-step layer)", "dtype": name,
                          "us": round(ms * 1e3, 1), "kv_bytes": kv_bytes,
                          "kv_GBps": round(kv_bytes / ms / 1e6, 1)}), flush=True)
        del kp, vp


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    sub = ap.add_subparsers(dest="what", required=True)
    p = sub.add_parser("prefill")
    p.add_argument("--small", action="store_true", help="3 launches of 2 x 2048 fp16 (profiling)")
    p.add_argument("--profile", action="store_true", help="3 launches of 4 x 4096 fp16 (profiling)")
    p = sub.add_parser("gqa")
    p.add_argument("--partition-size", type=int, default=0, help="0 = automatic")
    p.add_argument("--dtype", choices=sorted(_DTYPES), default="f16")
    p.add_argument("--profile", action="store_true")
    p.add_argument("--groups", default="1,2,4,8", help="query heads per KV head to run")
    p = sub.add_parser("shared-prefix")
    p.add_argument("--profile", action="store_true")
    p = sub.add_parser("long-context")
    p.add_argument("--partition-size", type=int, default=0, help="0 = automatic")
    p.add_argument("--profile", action="store_true")
    p = sub.add_parser("single-layer")
    p.add_argument("--partition-size", type=int, default=0, help="0 = automatic")
    p.add_argument("--profile", action="store_true")
    p = sub.add_parser("cache-ops")
    p.add_argument("--profile", action="store_true")
    sub.add_parser("decode-dtypes")
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("kernel_bench needs a CUDA device")
    torch.manual_seed(0)  # the q tensors drawn below are the same in every run
    if args.what == "prefill":
        prefill(args.small, args.profile)
    elif args.what == "gqa":
        gqa(args.partition_size, args.dtype, args.profile,
            tuple(int(g) for g in args.groups.split(",")))
    elif args.what == "shared-prefix":
        shared_prefix(args.profile)
    elif args.what == "long-context":
        long_context(args.partition_size, args.profile)
    elif args.what == "single-layer":
        single_layer(args.partition_size, args.profile)
    elif args.what == "cache-ops":
        cache_ops(args.profile)
    else:
        decode_dtypes()


if __name__ == "__main__":
    main()
