"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with:
  * library conversions (numpy float16, torch bfloat16) over every 16-bit code;
  * torch's scaled_dot_product_attention in float64 on a DENSE, contiguous
    layout from which the paged pool was built by scattering whole blocks;
  * closed forms (one-token context, constant keys, hand-worked fixtures in
    tests/golden/, the large-score argmax case);
  * invariants the pages state (physical block placement does not matter;
    shared blocks are read-only; the split form merges back to the unsplit one).
The battery is also run against deliberately mutated copies of the oracle
source (tests/test_oracle.py) to show that plausible mistakes are caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


def codes(x: np.ndarray | torch.Tensor, dtype: str) -> np.ndarray:
    """uint16 storage codes of `x` rounded to `dtype` (torch's RNE cast)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(_TORCH[dtype])
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def values(c: np.ndarray, dtype: str) -> torch.Tensor:
    """float64 values of uint16 codes, decoded by torch (not by the oracle)."""
    t = torch.from_numpy(np.ascontiguousarray(c).view(np.int16)).view(_TORCH[dtype])
    return t.to(torch.float64)


def dense_case(B, Hq, Hkv, D, bs, lens, dtype, seed, pool_extra=5):
    """A paged case built FROM a dense per-sequence layout.

    dense_k/dense_v[b] are [ceil(L_b/bs)*bs, Hkv, D]; the pool gets block i of
    sequence b at a random physical block table[b, i] by whole-block copies
    (numpy reshape + fancy assignment).  Unused pool cells are random too.
    """
    rng = np.random.default_rng(seed)
    nblk = [-(-L // bs) for L in lens]
    NB = sum(nblk) + pool_extra
    MB = max(1, max(nblk) if nblk else 1)
    pool_k = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)
    pool_v = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)
    perm = rng.permutation(NB)
    table = np.full((B, MB), -1, dtype=np.int32)
    dense_k, dense_v = [], []
    cur = 0
    for b in range(B):
        n = nblk[b]
        dk = rng.standard_normal((n * bs, Hkv, D)).astype(np.float32)
        dv = rng.standard_normal((n * bs, Hkv, D)).astype(np.float32)
        ids = perm[cur:cur + n]
        cur += n
        pool_k[ids] = dk.reshape(n, bs, Hkv, D)
        pool_v[ids] = dv.reshape(n, bs, Hkv, D)
        table[b, :n] = ids
        dense_k.append(dk)
        dense_v.append(dv)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    return dict(q=codes(q, dtype), kc=codes(pool_k, dtype), vc=codes(pool_v, dtype),
                table=table, lens=np.array(lens, dtype=np.int32),
                dense_k=[codes(x, dtype) for x in dense_k],
                dense_v=[codes(x, dtype) for x in dense_v], dtype=dtype)


def sdpa_reference(case, scale):
    """torch SDPA (float64) per sequence over the dense layout."""
    dt = case["dtype"]
    q = values(case["q"], dt)
    B, Hq, D = q.shape
    outs = torch.zeros(B, Hq, D, dtype=torch.float64)
    for b in range(B):
        L = int(case["lens"][b])
        if L == 0:
            continue
        k = values(case["dense_k"][b], dt)[:L]          # [L, Hkv, D]
        v = values(case["dense_v"][b], dt)[:L]
        Hkv = k.shape[1]
        k = k.permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)   # [Hq, L, D]
        v = v.permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        o = F.scaled_dot_product_attention(q[b][:, None, :], k, v, scale=scale)
        outs[b] = o[:, 0, :]
    return outs.numpy()


# ---------------------------------------------------------------- pins ----

def pin_decode_f16_exhaustive(orc):
    c = np.arange(65536, dtype=np.uint16)
    mine = orc.decode_array(c, "f16")
    ref = c.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


def pin_decode_bf16_exhaustive(orc):
    c = np.arange(65536, dtype=np.uint16)
    mine = orc.decode_array(c, "bf16")
    ref = values(c, "bf16").numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


DENSE_CASES = [
    # B, Hq, Hkv, D, bs, lens, dtype
    (3, 4, 4, 8, 4, [1, 7, 13], "f16"),
    (4, 8, 2, 16, 16, [16, 17, 40, 64], "bf16"),
    (2, 6, 3, 8, 2, [5, 9], "f16"),
    (2, 4, 1, 64, 16, [33, 3], "bf16"),
]


def pin_dense_sdpa(orc):
    for i, (B, Hq, Hkv, D, bs, lens, dt) in enumerate(DENSE_CASES):
        case = dense_case(B, Hq, Hkv, D, bs, lens, dt, seed=100 + i)
        scale = 1.0 / math.sqrt(D)
        got = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                         case["lens"], scale, dt)
        ref = sdpa_reference(case, scale)
        err = np.abs(got - ref).max()
        assert err < 1e-12, (i, err)


def pin_one_token(orc):
    case = dense_case(3, 4, 2, 16, 4, [1, 1, 1], "bf16", seed=7)
    got = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                     case["lens"], 0.37, "bf16")
    for b in range(3):
        v0 = values(case["dense_v"][b], "bf16")[0].numpy()        # [Hkv, D]
        assert np.array_equal(got[b], np.repeat(v0, 2, axis=0))    # exact


def pin_constant_keys(orc):
    B, Hq, Hkv, D, bs, lens = 2, 2, 1, 8, 4, [11, 6]
    case = dense_case(B, Hq, Hkv, D, bs, lens, "f16", seed=8)
    # every token of every sequence gets the same key -> uniform weights
    same = case["kc"][case["table"][0, 0], 0, 0].copy()
    case["kc"][...] = same
    got = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                     case["lens"], 0.5, "f16")
    for b in range(B):
        v = values(case["dense_v"][b], "f16")[:lens[b], 0].numpy()
        ref = v.mean(axis=0)
        assert np.abs(got[b] - ref[None, :]).max() < 1e-12


def pin_permutation(orc):
    """Moving blocks to other physical ids (and fixing the table) changes nothing, bitwise."""
    case = dense_case(3, 8, 2, 16, 4, [9, 21, 4], "bf16", seed=9, pool_extra=7)
    a = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                   case["lens"], 0.25, "bf16")
    NB = case["kc"].shape[0]
    perm = np.random.default_rng(10).permutation(NB)          # old id -> new id
    kc2 = np.empty_like(case["kc"])
    vc2 = np.empty_like(case["vc"])
    kc2[perm] = case["kc"]
    vc2[perm] = case["vc"]
    t2 = case["table"].copy()
    used = t2 >= 0
    t2[used] = perm[t2[used]]
    b = orc.paged_attention_decode(case["q"], kc2, vc2, t2, case["lens"], 0.25, "bf16")
    assert np.array_equal(a, b)


def pin_gqa_vs_mha(orc):
    """Group G equals MHA over a cache whose kv heads are each repeated G times."""
    G, Hkv = 4, 2
    case = dense_case(2, G * Hkv, Hkv, 8, 4, [10, 3], "f16", seed=11)
    a = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                   case["lens"], 0.3, "f16")
    kc = np.repeat(case["kc"], G, axis=2)
    vc = np.repeat(case["vc"], G, axis=2)
    b = orc.paged_attention_decode(case["q"], kc, vc, case["table"], case["lens"], 0.3, "f16")
    assert np.array_equal(a, b)


def _golden_decode_inputs(fx):
    dt = fx["dtype"]
    nb, bs, Hkv, D = fx["num_blocks"], fx["block_size"], fx["num_kv_heads"], fx["head_dim"]
    kc = np.full((nb, bs, Hkv, D), fx["fill"], dtype=np.float32)
    vc = np.full((nb, bs, Hkv, D), fx["fill"], dtype=np.float32)
    for c in fx["placed"]:
        kc[c["block"], c["offset"], c["kv_head"]] = c["k"]
        vc[c["block"], c["offset"], c["kv_head"]] = c["v"]
    table = np.array([fx["block_table"]], dtype=np.int32)
    lens = np.array([fx["context_len"]], dtype=np.int32)
    q = np.array([fx["query"]], dtype=np.float32)
    return codes(q, dt), codes(kc, dt), codes(vc, dt), table, lens


def golden_fixtures(kind):
    out = []
    for name in sorted(os.listdir(GOLDEN)):
        if name.endswith(".json"):
            fx = json.load(open(os.path.join(GOLDEN, name)))
            if fx["kind"] == kind:
                out.append((name, fx))
    return out


def pin_golden_decode(orc):
    for name, fx in golden_fixtures("decode"):
        q, kc, vc, table, lens = _golden_decode_inputs(fx)
        got = orc.paged_attention_decode(q, kc, vc, table, lens, fx["scale"], fx["dtype"])
        for e in fx["expected"]:
            s = np.array(e["scores"], dtype=np.float64)
            w = np.exp(s - s.max())
            ref = (w[:, None] * np.array(e["values"], dtype=np.float64)).sum(0) / w.sum()
            err = np.abs(got[0, e["head"]] - ref).max()
            assert err < 1e-13, (name, e["head"], err)


def pin_golden_write(orc):
    for name, fx in golden_fixtures("write"):
        dt = fx["dtype"]
        nb, bs, Hkv, D = fx["num_blocks"], fx["block_size"], fx["num_kv_heads"], fx["head_dim"]
        kc = codes(np.full((nb, bs, Hkv, D), fx["canary"], np.float32), dt)
        vc = codes(np.full((nb, bs, Hkv, D), fx["canary"], np.float32), dt)
        canary = kc.copy()
        orc.kv_cache_write(codes(np.array(fx["key"], np.float32), dt),
                           codes(np.array(fx["value"], np.float32), dt),
                           np.array(fx["slot_mapping"], np.int64), kc, vc, bs)
        touched = np.zeros((nb, bs, Hkv), dtype=bool)
        for c in fx["expected_cells"]:
            i = (c["block"], c["offset"], c["kv_head"])
            assert np.array_equal(kc[i], codes(np.array(c["k"], np.float32), dt)), (name, i)
            assert np.array_equal(vc[i], codes(np.array(c["v"], np.float32), dt)), (name, i)
            touched[i] = True
        assert np.array_equal(kc[~touched], canary[~touched]), name
        assert np.array_equal(vc[~touched], canary[~touched]), name


def pin_large_scores(orc):
    """Scores of +-2000 must not overflow: out is exactly V of the argmax token."""
    B, Hq, Hkv, D, bs = 1, 1, 1, 4, 2
    kc = np.zeros((3, bs, Hkv, D), np.float32)
    vc = np.zeros((3, bs, Hkv, D), np.float32)
    kc[1, 0, 0] = [8, 8, 8, 8]
    kc[1, 1, 0] = [-8, -8, -8, -8]
    kc[2, 0, 0] = [16, 16, 16, 16]
    vc[1, 0, 0] = [1, 2, 3, 4]
    vc[1, 1, 0] = [5, 6, 7, 8]
    vc[2, 0, 0] = [-1.5, 2.5, -3.5, 4.5]
    q = np.full((1, 1, D), 32, np.float32)
    table = np.array([[1, 2]], np.int32)
    got = orc.paged_attention_decode(codes(q, "bf16"), codes(kc, "bf16"), codes(vc, "bf16"),
                                     table, np.array([3], np.int32), 1.0, "bf16")
    assert np.array_equal(got[0, 0], np.array([-1.5, 2.5, -3.5, 4.5]))


def pin_partitions_merge(orc):
    case = dense_case(3, 4, 2, 16, 4, [37, 8, 1], "bf16", seed=12)
    scale = 0.25
    full = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                      case["lens"], scale, "bf16")
    # partition length 8 (2 blocks): 5 partitions cover the longest sequence
    m, l, o = orc.paged_attention_partitions(case["q"], case["kc"], case["vc"], case["table"],
                                             case["lens"], scale, "bf16", 8, 5)
    merged = orc.lse_merge(m, l, o)
    assert np.abs(merged - full).max() < 1e-13
    # partitions past a sequence's end are empty
    assert np.all(l[1, :, 1:] == 0) and np.all(np.isneginf(m[2, :, 1:]))
    # one partition covering everything: the normaliser is the softmax denominator
    sdpa = sdpa_reference(case, scale)
    m1, l1, o1 = orc.paged_attention_partitions(case["q"], case["kc"], case["vc"],
                                                case["table"], case["lens"], scale, "bf16",
                                                64, 1)
    assert np.abs(o1[:, :, 0] - sdpa).max() < 1e-12
    q = values(case["q"], "bf16").numpy()
    k = values(case["dense_k"][0], "bf16").numpy()[:37]             # [L, Hkv, D]
    s = scale * np.einsum("hd,lhd->hl", q[0], np.repeat(k, 2, axis=1))
    assert np.abs(m1[0, :, 0] - s.max(1)).max() < 1e-12
    assert np.abs(l1[0, :, 0] - np.exp(s - s.max(1, keepdims=True)).sum(1)).max() < 1e-12


def pin_empty_context(orc):
    case = dense_case(2, 2, 2, 8, 4, [0, 5], "f16", seed=13)
    got = orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                     case["lens"], 0.5, "f16")
    assert np.array_equal(got[0], np.zeros_like(got[0]))
    assert np.isfinite(got).all()


def pin_range_errors(orc):
    import oracle
    case = dense_case(1, 2, 2, 8, 4, [6], "f16", seed=14)
    bad = case["table"].copy()
    bad[0, 1] = case["kc"].shape[0]               # one past the pool
    try:
        orc.paged_attention_decode(case["q"], case["kc"], case["vc"], bad, case["lens"],
                                   0.5, "f16")
        raise AssertionError("out-of-range block id accepted")
    except oracle.OracleError as e:
        assert e.code == oracle.ERR_RANGE
    try:
        orc.paged_attention_decode(case["q"], case["kc"], case["vc"], case["table"],
                                   np.array([9], np.int32), 0.5, "f16")   # > 2 blocks * 4
        raise AssertionError("context_len beyond the table accepted")
    except oracle.OracleError as e:
        assert e.code == oracle.ERR_RANGE


def pin_write_canary(orc):
    """Written cells equal the inputs bit for bit; every other cell is untouched."""
    rng = np.random.default_rng(15)
    NB, bs, Hkv, D, T = 6, 4, 3, 8, 7
    kc = codes(rng.standard_normal((NB, bs, Hkv, D)), "bf16")
    vc = codes(rng.standard_normal((NB, bs, Hkv, D)), "bf16")
    k0, v0 = kc.copy(), vc.copy()
    key = codes(rng.standard_normal((T, Hkv, D)), "bf16")
    val = codes(rng.standard_normal((T, Hkv, D)), "bf16")
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    slots[3] = -1
    orc.kv_cache_write(key, val, slots, kc, vc, bs)
    flat_k, flat_v = kc.reshape(NB * bs, Hkv, D), vc.reshape(NB * bs, Hkv, D)
    written = np.zeros(NB * bs, dtype=bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        assert np.array_equal(flat_k[s], key[t]) and np.array_equal(flat_v[s], val[t])
        written[s] = True
    assert np.array_equal(flat_k[~written], k0.reshape(NB * bs, Hkv, D)[~written])
    assert np.array_equal(flat_v[~written], v0.reshape(NB * bs, Hkv, D)[~written])


def pin_write_roundtrip(orc):
    """Write a token, then decode a one-token context at that slot: out == V."""
    rng = np.random.default_rng(16)
    NB, bs, Hkv, Hq, D = 5, 4, 2, 4, 8
    kc = codes(rng.standard_normal((NB, bs, Hkv, D)), "f16")
    vc = codes(rng.standard_normal((NB, bs, Hkv, D)), "f16")
    key = codes(rng.standard_normal((1, Hkv, D)), "f16")
    val = codes(rng.standard_normal((1, Hkv, D)), "f16")
    orc.kv_cache_write(key, val, np.array([3 * bs], np.int64), kc, vc, bs)  # block 3, off 0
    q = codes(rng.standard_normal((1, Hq, D)), "f16")
    out = orc.paged_attention_decode(q, kc, vc, np.array([[3]], np.int32),
                                     np.array([1], np.int32), 0.5, "f16")
    ref = np.repeat(values(val, "f16").numpy()[0], Hq // Hkv, axis=0)
    assert np.array_equal(out[0], ref)


def pin_copy_blocks(orc):
    """Copied blocks equal their sources bit for bit; other blocks untouched;
    a copy-on-write then a one-token decode reads the source's values."""
    import oracle
    rng = np.random.default_rng(17)
    NB, bs, Hkv, D = 9, 4, 2, 8
    src = codes(rng.standard_normal((NB, bs, Hkv, D)), "bf16")
    dst = codes(rng.standard_normal((5, bs, Hkv, D)), "bf16")
    before = dst.copy()
    mapping = np.array([[7, 0], [2, 3], [7, 4]], np.int32)
    orc.copy_blocks(src, dst, mapping)
    for s_, d_ in mapping:
        assert np.array_equal(dst[d_], src[s_])
    assert np.array_equal(dst[[1, 2]], before[[1, 2]])
    try:
        orc.copy_blocks(src, dst, np.array([[0, 5]], np.int32))     # dst out of range
        raise AssertionError("out-of-range block accepted")
    except oracle.OracleError as e:
        assert e.code == oracle.ERR_RANGE
    # copy-on-write inside one pool, then decode block 1 as a one-token context
    pool = codes(rng.standard_normal((4, bs, Hkv, D)), "f16")
    orc.copy_blocks(pool.copy(), pool, np.array([[3, 1]], np.int32))
    q = codes(rng.standard_normal((1, Hkv, D)), "f16")
    out = orc.paged_attention_decode(q, pool, pool, np.array([[1]], np.int32),
                                     np.array([1], np.int32), 0.5, "f16")
    assert np.array_equal(out[0], values(pool[3, 0], "f16").numpy())


def pin_prefill_causal_sdpa(orc):
    """Chunked prefill equals torch SDPA with an explicit causal mask on the dense
    layout (query token i of a C-token chunk at position L-C+i sees keys 0..L-C+i),
    and a chunk's last token equals the decode of the whole context."""
    cases = [(3, 4, 2, 16, 4, [9, 20, 5], [3, 20, 1], "bf16"),
             (2, 8, 8, 8, 16, [33, 17], [16, 5], "f16")]
    for ci, (B, Hq, Hkv, D, bs, lens, chunks, dt) in enumerate(cases):
        case = dense_case(B, Hq, Hkv, D, bs, lens, dt, seed=200 + ci)
        rng = np.random.default_rng(300 + ci)
        T = sum(chunks)
        qf = rng.standard_normal((T, Hq, D)).astype(np.float32)
        q = codes(qf, dt)
        qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        scale = 1.0 / math.sqrt(D)
        got = orc.paged_attention_prefill(q, qs, case["kc"], case["vc"], case["table"],
                                          case["lens"], scale, dt)
        qv = values(q, dt)
        for b in range(B):
            L, C = lens[b], chunks[b]
            k = values(case["dense_k"][b], dt)[:L].permute(1, 0, 2)     # [Hkv, L, D]
            v = values(case["dense_v"][b], dt)[:L].permute(1, 0, 2)
            k = k.repeat_interleave(Hq // Hkv, 0)
            v = v.repeat_interleave(Hq // Hkv, 0)
            qb = qv[qs[b]:qs[b + 1]].permute(1, 0, 2)                   # [Hq, C, D]
            pos = torch.arange(L - C, L)[:, None]
            mask = torch.arange(L)[None, :] <= pos                      # [C, L]
            ref = F.scaled_dot_product_attention(qb, k, v, attn_mask=mask, scale=scale)
            err = np.abs(got[qs[b]:qs[b + 1]] - ref.permute(1, 0, 2).numpy()).max()
            assert err < 1e-12, (ci, b, err)
            # last chunk token == decode of the full context with that query
            dec = orc.paged_attention_decode(q[qs[b + 1] - 1][None], case["kc"], case["vc"],
                                             case["table"][b:b + 1], case["lens"][b:b + 1],
                                             scale, dt)
            assert np.array_equal(dec[0], got[qs[b + 1] - 1])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
