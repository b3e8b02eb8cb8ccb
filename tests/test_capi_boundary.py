"""The C ABI without a GPU: every symbol include/pagedattn.h declares is
exported by libpagedattn.so, and host-side validation answers with the
documented status codes before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_478_b200 as pa

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pagedattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(pa_[a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["pa_pool_create", "pa_reshape_and_cache", "pa_decode_attention",
                     "pa_copy_blocks", "pa_decode_workspace_bytes", "pa_device_errors",
                     "pa_alloc_create", "pa_cow_block", "pa_append_tokens"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = pa.lib()
    for n in declared_functions():
        assert getattr(lib, n) is not None


def test_pool_create_fills_the_descriptor():
    p = pa.pa_pool_create(100, 16, 32, 128, pa.PA_F16)
    assert (p.num_blocks, p.block_size, p.heads, p.head_dim, p.elem_bytes) == (100, 16, 32, 128, 2)
    assert p.token_stride == 128 and p.head_stride == 16 * 128
    assert p.block_stride == 32 * 16 * 128
    assert p.bytes_per_pool == 100 * 32 * 16 * 128 * 2


@pytest.mark.parametrize("args,status", [
    ((100, 8, 32, 128, pa.PA_F16), 2),        # block_size 8 not built
    ((100, 16, 32, 96, pa.PA_F16), 2),        # head_dim 96 not built
    ((100, 16, 32, 128, 7), 2),               # unknown dtype
    ((0, 16, 32, 128, pa.PA_F16), 1),         # empty pool
    ((1 << 28, 16, 1, 64, pa.PA_F16), 1),     # slots overflow int32
])
def test_pool_create_rejects(args, status):
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_pool_create(*args)
    assert e.value.status == status


def test_workspace_bytes_grows_with_partitions():
    p = pa.pa_pool_create(4096, 16, 32, 128, pa.PA_F16)
    one = pa.pa_decode_workspace_bytes(p, 64, 128, 0, 2048)
    many = pa.pa_decode_workspace_bytes(p, 64, 128, 0, 256)
    assert many > one > 0
    # partials dominate: S * H * P * D * 4 bytes for P = 2048 / 256
    assert many >= 64 * 32 * 8 * 128 * 4
    with pytest.raises(pa.PagedAttnError):
        pa.pa_decode_workspace_bytes(p, 64, 128, 0, 24)  # not a multiple of 16


def test_null_pointers_are_rejected_before_any_cuda_call():
    lib = pa.lib()
    p = pa.pa_pool_create(16, 16, 2, 64, pa.PA_F32)
    st = lib.pa_decode_attention(ctypes.byref(p), None, None, None, None, 1, None, 4, 0,
                                 ctypes.c_float(0.1), None, None, 0, 0, None)
    assert st == 1
    st = lib.pa_reshape_and_cache(ctypes.byref(p), None, None, None, 3, None, None, None)
    assert st == 1
    st = lib.pa_copy_blocks(ctypes.byref(p), None, None, None, 2, None)
    assert st == 1
    # zero-sized calls are no-ops that touch nothing
    assert lib.pa_reshape_and_cache(ctypes.byref(p), None, None, None, 0, None, None, None) == 0
    assert lib.pa_copy_blocks(ctypes.byref(p), None, None, None, 0, None) == 0
    assert lib.pa_decode_attention(ctypes.byref(p), None, None, None, None, 1, None, 0, 0,
                                   ctypes.c_float(0.1), None, None, 0, 0, None) == 0
    assert b"null" in lib.pa_last_error() or lib.pa_last_error() != b""


def test_misaligned_buffers_are_rejected():
    lib = pa.lib()
    p = pa.pa_pool_create(16, 16, 2, 64, pa.PA_F32)
    bad = ctypes.c_void_p(0x1008)
    good = ctypes.c_void_p(0x2000)
    st = lib.pa_reshape_and_cache(ctypes.byref(p), bad, good, good, 1, good, good, None)
    assert st == 1 and b"aligned" in lib.pa_last_error()


def test_status_strings():
    lib = pa.lib()
    assert lib.pa_status_string(0) == b"PA_OK"
    assert lib.pa_status_string(5) == b"PA_ERR_NO_FREE_BLOCKS"


def test_prefill_and_shared_prefix_validate_on_the_host():
    """Both calls reject bad arguments before their first CUDA call."""
    lib = pa.lib()
    f = ctypes.c_float
    ok = ctypes.c_void_p(0x2000)  # aligned, never dereferenced on these paths
    p32 = pa.pa_pool_create(16, 16, 2, 64, pa.PA_F32)
    p16 = pa.pa_pool_create(16, 16, 2, 64, pa.PA_F16)

    def prefill(pool, q=ok, qs=ok, num_seqs=1, num_tokens=8, max_new=8, scale=0.1, out=ok):
        return lib.pa_prefill_attention(ctypes.byref(pool), q, ok, ok, ok, 4, ok, qs, num_seqs,
                                        num_tokens, max_new, 0, f(scale), out, None)

    assert prefill(p32) == 2                      # tensor cores: fp16 / bf16 pools only
    assert prefill(p16, q=None) == 1
    assert prefill(p16, qs=None) == 1
    assert prefill(p16, out=None) == 1
    assert prefill(p16, num_seqs=-1) == 1
    assert prefill(p16, scale=float("nan")) == 1
    assert prefill(p16, q=ctypes.c_void_p(0x2008)) == 1  # misaligned
    assert prefill(p16, q=None, qs=None, out=None, num_tokens=0) == 0  # nothing to do

    def shared(pool, offsets=ok, members=ok, blocks=ok, num_groups=1, ctx=ok):
        return lib.pa_decode_attention_shared_prefix(
            ctypes.byref(pool), ok, ok, ok, ok, 4, ctx, 2, offsets, members, 2, blocks, num_groups,
            2, 2, 0, f(0.1), ok, ok, 1 << 20, 0, None)

    assert shared(p32) == 2                       # the shared blocks go through mma.sync
    assert shared(p16, offsets=None) == 1
    assert shared(p16, members=None) == 1
    assert shared(p16, blocks=None) == 1
    assert shared(p16, ctx=None) == 1
    assert shared(p16, num_groups=-1) == 1
