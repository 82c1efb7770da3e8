"""The C-ABI library: it builds, loads, exports every declared symbol, and
validates arguments on the host before touching the GPU (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import build, pagedkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_library_builds():
    path = build.build()
    assert os.path.exists(path)


def test_every_declared_symbol_is_exported():
    path = build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (pkv_[a-z0-9_]+)\b", out))
    decl = declared_functions()
    assert len(decl) >= 15
    missing = [n for n in decl if n not in exported]
    assert not missing, missing
    L = pkv.lib()
    for n in decl:
        assert hasattr(L, n)


def test_status_strings_and_version():
    assert pagedkv.status_name(0) == "PKV_OK"
    assert pagedkv.status_name(6) == "PKV_ERR_WORKSPACE"
    assert "sm_100a" in pkv.version()


@pytest.mark.parametrize("args,expect", [
    ((256, 32, 8, 128, 40, 16, 0), (640, 1)),       # Llama-3-8B-shaped: one pass
    ((8, 32, 8, 128, 1024, 32, 512), (512, 64)),    # long context: 512-token partitions
    ((8, 32, 8, 128, 1024, 32, -1), (32768, 1)),    # never split
    ((8, 32, 8, 128, 1024, 32, 500), (512, 64)),    # rounded up to a block multiple
    ((4, 8, 8, 64, 13, 16, 0), (208, 1)),           # tiny: one partition covers all
])
def test_decode_plan(args, expect):
    assert pkv.decode_plan(*args) == expect


def test_workspace_bytes():
    # B * Hq * P * (D + 2) floats
    assert pkv.decode_workspace_bytes(8, 32, 8, 128, 1024, 32, 512) == 8 * 32 * 64 * 130 * 4
    assert pkv.decode_workspace_bytes(256, 32, 8, 128, 40, 16, 0) == 0


@pytest.mark.parametrize("shape,status", [
    ((4, 8, 3, 64, 4, 16), pagedkv.ERR_UNSUPPORTED),     # 8 % 3 != 0
    ((4, 32, 2, 64, 4, 16), pagedkv.ERR_UNSUPPORTED),    # group 16 > 8
    ((4, 8, 8, 96, 4, 16), pagedkv.ERR_UNSUPPORTED),     # head_dim 96
    ((4, 8, 8, 64, 4, 8), pagedkv.ERR_UNSUPPORTED),      # block_size 8
    ((4, 8, 8, 64, 0, 16), pagedkv.ERR_INVALID_ARG),     # no table columns
    ((-1, 8, 8, 64, 4, 16), pagedkv.ERR_INVALID_ARG),
])
def test_decode_rejects_shapes_on_host(shape, status):
    B, Hq, Hkv, D, MB, bs = shape
    L = pkv.lib()
    st = L.pkv_paged_attention_decode(None, None, None, None, MB, None, B, Hq, Hkv, D, bs, 100,
                                      1.0, 0, None, 0, None, 1, None)
    assert st == status
    assert L.pkv_last_error()


def test_decode_host_validation_before_any_launch():
    L = pkv.lib()
    # null pointers
    assert L.pkv_paged_attention_decode(None, None, None, None, 4, None, 2, 8, 8, 64, 16, 100,
                                        1.0, 0, None, 0, None, 1, None) == pagedkv.ERR_INVALID_ARG
    # misaligned (never dereferenced: validation fails first)
    fake = 0x1008
    assert L.pkv_paged_attention_decode(fake, fake, fake, fake, 4, fake, 2, 8, 8, 64, 16, 100,
                                        1.0, 0, None, 0, fake, 1, None) == pagedkv.ERR_MISALIGNED
    # split plan without workspace
    a16 = 0x10000
    assert L.pkv_paged_attention_decode(a16, a16, a16, a16, 1024, a16, 8, 32, 8, 128, 32, 10000,
                                        1.0, 512, None, 0, a16, 1, None) == pagedkv.ERR_WORKSPACE
    # non-finite scale, pool too large
    assert L.pkv_paged_attention_decode(a16, a16, a16, a16, 4, a16, 2, 8, 8, 64, 16, 100,
                                        float("nan"), 0, None, 0, a16, 1, None) == pagedkv.ERR_INVALID_ARG
    assert L.pkv_paged_attention_decode(a16, a16, a16, a16, 4, a16, 2, 8, 8, 64, 16, 1 << 28,
                                        1.0, 0, None, 0, a16, 1, None) == pagedkv.ERR_INVALID_ARG
    # empty batch is a no-op
    assert L.pkv_paged_attention_decode(None, None, None, None, 4, None, 0, 8, 8, 64, 16, 100,
                                        1.0, 0, None, 0, None, 1, None) == pagedkv.OK


def test_write_host_validation():
    L = pkv.lib()
    assert L.pkv_kv_cache_write(None, None, None, 0, 8, 64, None, None, 10, 16, 1, None) == pagedkv.OK
    assert L.pkv_kv_cache_write(None, None, None, 3, 8, 64, None, None, 10, 16, 1, None) == pagedkv.ERR_INVALID_ARG
    f = 0x1004
    assert L.pkv_kv_cache_write(f, f, f, 3, 8, 64, f, f, 10, 16, 1, None) == pagedkv.ERR_MISALIGNED
    assert L.pkv_kv_cache_write(None, None, None, -1, 8, 64, None, None, 10, 16, 1, None) == pagedkv.ERR_INVALID_ARG
    assert L.pkv_kv_cache_write(None, None, None, 1, 8, 64, None, None, 10, 16, 7, None) == pagedkv.ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(2, 8, 64, dtype=torch.float16)
    kc = torch.zeros(4, 16, 8, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode(q, kc, kc.clone(), torch.zeros(2, 4, dtype=torch.int32),
                                   torch.ones(2, dtype=torch.int32), 0.125)


def test_cascade_workspace_and_validation():
    L = pkv.lib()
    # prefix records B*Hq*Pp and suffix records B*Hq*Ps, each (m, l, o[D]) floats
    n = L.pkv_decode_cascade_workspace_bytes(256, 32, 8, 128, 125, 16, 8, 16, 0)
    a = lambda x: (x + 255) // 256 * 256
    rp, rs = 256 * 32 * 4, 256 * 32 * 1
    exp = a(rp * 4); exp = a(exp + rp * 4); exp = a(exp + rp * 128 * 4)
    exp = a(exp + rs * 4); exp = a(exp + rs * 4); exp = a(exp + rs * 128 * 4)
    assert n == exp
    assert L.pkv_decode_cascade_workspace_bytes(256, 32, 8, 128, 0, 16, 8, 16, 0) == 0
    assert L.pkv_paged_attention_decode_cascade(None, None, None, None, 4, None, None, 1, 2, None, 4,
                                                None, 2, 8, 8, 64, 16, 100, 1.0, 0, None, 0, None,
                                                1, None) == pagedkv.ERR_INVALID_ARG


def test_prefill_host_validation():
    L = pkv.lib()
    a16 = 0x10000
    # query, num_tokens, query_start, max_query_len, key_cache, value_cache, block_tables,
    # max_blocks, context_lens, batch, Hq, Hkv, D, bs, num_blocks, scale, out, dtype, stream
    def call(q=a16, T=64, qs=a16, mql=32, kc=a16, vc=a16, bt=a16, mb=8, cl=a16, B=2, Hq=8, Hkv=2,
             D=128, bs=16, nb=100, scale=0.125, out=a16, dt=1):
        return L.pkv_paged_attention_prefill(q, T, qs, mql, kc, vc, bt, mb, cl, B, Hq, Hkv, D, bs, nb,
                                             scale, out, dt, None)
    assert call(Hq=32, Hkv=2) == pagedkv.ERR_UNSUPPORTED           # group 16 > 8
    assert call(D=96) == pagedkv.ERR_UNSUPPORTED
    assert call(dt=7) == pagedkv.ERR_INVALID_ARG
    assert call(T=-1) == pagedkv.ERR_INVALID_ARG
    assert call(mql=8 * 16 + 1) == pagedkv.ERR_INVALID_ARG         # > max_blocks * block_size
    assert call(nb=0) == pagedkv.ERR_INVALID_ARG
    assert call(scale=float("inf")) == pagedkv.ERR_INVALID_ARG
    assert call(q=None, qs=None, kc=None, vc=None, bt=None, cl=None, out=None, B=0) == pagedkv.OK
    assert call(T=0, q=None, out=None) == pagedkv.OK                # nothing to do
    assert call(out=None) == pagedkv.ERR_INVALID_ARG
    assert call(q=a16 + 8) == pagedkv.ERR_MISALIGNED


def test_copy_blocks_host_validation():
    L = pkv.lib()
    a16 = 0x10000
    # src_k, src_v, dst_k, dst_v, mapping, num_pairs, src_blocks, dst_blocks, block_bytes, stream
    def call(p=a16, m=a16, n=4, sb=10, db=10, bb=16 * 8 * 128 * 2):
        return L.pkv_copy_blocks(p, p, p, p, m, n, sb, db, bb, None)
    assert call(n=-1) == pagedkv.ERR_INVALID_ARG
    assert call(sb=0) == pagedkv.ERR_INVALID_ARG
    assert call(bb=24) == pagedkv.ERR_UNSUPPORTED                   # not a multiple of 16
    assert call(n=(1 << 30) + 1) == pagedkv.ERR_UNSUPPORTED         # grid of 2 CTAs per pair
    assert call(n=1 << 30) == pagedkv.ERR_UNSUPPORTED               # 2^31 CTAs: one too many
    assert call(n=0, p=None, m=None) == pagedkv.OK
    assert call(m=None) == pagedkv.ERR_INVALID_ARG
    assert call(p=a16 + 8) == pagedkv.ERR_MISALIGNED
    assert call(m=a16 + 4) == pagedkv.ERR_MISALIGNED


def test_hbm_read_probe_host_validation():
    L = pkv.lib()
    a16 = 0x10000
    assert L.pkv_hbm_read_probe(None, 16, a16, 1, None) == pagedkv.ERR_INVALID_ARG
    assert L.pkv_hbm_read_probe(a16, 24, a16, 1, None) == pagedkv.ERR_INVALID_ARG   # not 16-byte units
    assert L.pkv_hbm_read_probe(a16, 16, a16, 0, None) == pagedkv.ERR_INVALID_ARG   # empty grid
    assert L.pkv_hbm_read_probe(a16 + 8, 16, a16, 1, None) == pagedkv.ERR_MISALIGNED
    assert L.pkv_hbm_read_probe(a16, 16, a16 + 2, 1, None) == pagedkv.ERR_MISALIGNED


def test_cascade_plan_choice():
    # 32 groups x 8 kv heads fill the GPU: one pass; 12 x 8 do not: split in 512-token partitions
    assert pkv.decode_cascade_plan(256, 32, 8, 128, 125, 16, 8, 32, 16, 0) == (True, 1)
    assert pkv.decode_cascade_plan(96, 32, 8, 128, 125, 16, 8, 12, 16, 0) == (False, 4)
    assert pkv.decode_cascade_plan(96, 32, 8, 128, 125, 16, 8, 12, 16, -1) == (True, 1)
    assert pkv.decode_cascade_plan(96, 32, 8, 128, 125, 16, 8, 12, 16, 64) == (False, 32)
    assert pkv.decode_cascade_plan(96, 32, 8, 128, 125, 16, 8, 0, 16, -1) == (False, 4)   # no groups
    with pytest.raises(pkv.PagedKVError):
        pkv.decode_cascade_plan(96, 32, 8, 128, 125, 16, 8, 97, 16, 0)                     # > batch


def test_hbm_gather_probe_host_validation():
    L = pkv.lib()
    a16 = 0x10000
    assert L.pkv_hbm_gather_probe(None, 4096, a16, 4, a16, 1, None) == pagedkv.ERR_INVALID_ARG
    assert L.pkv_hbm_gather_probe(a16, 4095, a16, 4, a16, 1, None) == pagedkv.ERR_INVALID_ARG
    assert L.pkv_hbm_gather_probe(a16, 4096, a16, 0, a16, 1, None) == pagedkv.ERR_INVALID_ARG
    assert L.pkv_hbm_gather_probe(a16 + 8, 4096, a16, 4, a16, 1, None) == pagedkv.ERR_MISALIGNED
    assert L.pkv_hbm_gather_probe(a16, 4096, a16 + 2, 4, a16, 1, None) == pagedkv.ERR_MISALIGNED
