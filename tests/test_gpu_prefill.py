"""Chunked prefill on the GPU vs the fp64 oracle (causal attention of each
chunk token over its sequence's paged cache)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from tests.parity_util import NTHREADS, TOL, custom, max_abs_err, u16

pytestmark = pytest.mark.gpu

_DT = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield
    assert pkv.device_flags() == 0


def _case(lens, chunks, Hq, Hkv, D, bs, dtype, seed):
    step = custom("pf", len(lens), Hq, Hkv, D, bs, dtype, lens, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    T = sum(chunks)
    q = torch.randn(T, Hq, D, generator=g).to(_DT[dtype])
    qs = torch.tensor(np.concatenate([[0], np.cumsum(chunks)]), dtype=torch.int32)
    return step, q, qs


def _check(step, q, qs, chunks):
    ref = oracle.paged_attention_prefill(u16(q), qs.numpy(), u16(step["key_cache"]),
                                         u16(step["value_cache"]), step["block_tables"].numpy(),
                                         step["context_lens"].numpy(), step["scale"],
                                         step["dtype"], nthreads=NTHREADS)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in step.items()}
    out = pkv.paged_attention_prefill(q.cuda(), qs.cuda(), max(chunks), d["key_cache"],
                                      d["value_cache"], d["block_tables"], d["context_lens"],
                                      step["scale"])
    err, idx, finite = max_abs_err(out, ref)
    assert finite and err <= TOL[step["dtype"]], (err, idx)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_ragged_chunks(D, bs, dtype):
    lens = [1, 17, 100, 300, 33, 64]
    chunks = [1, 17, 37, 300, 5, 1]          # whole contexts, partial chunks, single tokens
    step, q, qs = _case(lens, chunks, 8, 2, D, bs, dtype, seed=D + bs)
    _check(step, q, qs, chunks)


@pytest.mark.parametrize("G", [1, 3, 4, 6, 8])
def test_prefill_group_sizes(G):
    lens = [700, 129, 520]
    chunks = [512, 129, 7]
    step, q, qs = _case(lens, chunks, 4 * G, 4, 128, 16, "bf16", seed=G)
    _check(step, q, qs, chunks)


def test_prefill_last_token_equals_decode():
    lens, chunks = [200, 61], [40, 61]
    step, q, qs = _case(lens, chunks, 8, 2, 128, 16, "bf16", seed=77)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in step.items()}
    out = pkv.paged_attention_prefill(q.cuda(), qs.cuda(), max(chunks), d["key_cache"],
                                      d["value_cache"], d["block_tables"], d["context_lens"],
                                      step["scale"])
    last = q[qs[1:] - 1].cuda()                          # each chunk's last token
    dec = pkv.paged_attention_decode(last, d["key_cache"], d["value_cache"], d["block_tables"],
                                     d["context_lens"], step["scale"], partition_tokens=-1)
    assert (out[qs[1:].long().cuda() - 1].float() - dec.float()).abs().max().item() <= TOL["bf16"]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_growing_scores(dtype, D):
    """Keys grow along the context, so each row's running maximum keeps
    moving by more than 2^8 in weight: every rescale of the running output
    is exercised, and the result must still be the one-pass softmax.  The
    attention is then nearly one-hot, so outputs take the size of single V
    entries; V is scaled by 1/4 to keep them below 2, where rounding the
    output to the storage type stays inside the fixed absolute bound."""
    lens, chunks = [900, 333], [600, 333]
    step, q, qs = _case(lens, chunks, 8, 2, D, 16, dtype, seed=5)
    kc = step["key_cache"].float()
    tables = step["block_tables"]
    for s_, L in enumerate(lens):
        for k in range((L + 15) // 16):
            kc[int(tables[s_, k])] *= 1.0 + 0.25 * k
    step["key_cache"] = kc.to(_DT[dtype])
    step["value_cache"] = (step["value_cache"].float() * 0.25).to(_DT[dtype])
    q = (q.float() * 2.0).to(_DT[dtype])
    _check(step, q, qs, chunks)


@pytest.mark.parametrize("bs", [16, 32])
def test_prefill_garbage_past_the_context(bs):
    """Cells past each sequence's last token (in its last block) hold NaN and
    infinity: they are never read as keys or values, so every output stays
    finite and within tolerance.  Lengths end inside a block, on a block
    edge, on a key-tile edge and inside a key tile."""
    lens = [520, 7, 64, 65, 300, 17, 128, 33, 129, 255, 256, 257]
    chunks = [7, 7, 64, 1, 300, 9, 5, 33, 129, 100, 3, 257]
    step, q, qs = _case(lens, chunks, 8, 2, 128, bs, "bf16", seed=bs + 11)
    kc, vc = step["key_cache"].clone(), step["value_cache"].clone()
    for s_, L in enumerate(lens):
        if L % bs:
            blk = int(step["block_tables"][s_, (L - 1) // bs])
            kc[blk, L % bs:] = float("nan")
            vc[blk, L % bs:] = float("inf")
    ref = oracle.paged_attention_prefill(u16(q), qs.numpy(), u16(step["key_cache"]),
                                         u16(step["value_cache"]), step["block_tables"].numpy(),
                                         step["context_lens"].numpy(), step["scale"], "bf16",
                                         nthreads=NTHREADS)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in step.items()}
    out = pkv.paged_attention_prefill(q.cuda(), qs.cuda(), max(chunks), kc.cuda(), vc.cuda(),
                                      d["block_tables"], d["context_lens"], step["scale"])
    err, idx, finite = max_abs_err(out, ref)
    assert finite and err <= TOL["bf16"], (err, idx)


def test_prefill_many_work_tiles_per_cta():
    """More row tiles than two per SM: the persistent CTAs walk several work
    tiles each, of very different lengths (chunks of 1 to 1000 tokens).
    Chunks that start a context give outputs over one or two keys, i.e. single
    V entries; among 79M outputs some exceed 4 in magnitude, where rounding to
    bf16 alone can pass the fixed absolute bound.  V is halved so that outputs
    stay below 4, where the bound covers the final rounding."""
    rng = np.random.default_rng(12)
    lens = [int(x) for x in rng.integers(1, 1100, size=96)]
    chunks = [int(min(L, c)) for L, c in zip(lens, rng.integers(1, 1000, size=96))]
    step, q, qs = _case(lens, chunks, 16, 4, 128, 16, "bf16", seed=13)
    step["value_cache"] = (step["value_cache"].float() * 0.5).to(torch.bfloat16)
    _check(step, q, qs, chunks)


@pytest.mark.parametrize("D,bs,dtype", [(128, 32, "bf16"), (64, 16, "f16")])
def test_prefill_long_context(D, bs, dtype):
    """Chunks at the end of contexts of 9000 and 20000 tokens: each row tile
    walks 140 to 313 key tiles, so every ring and barrier of the pipeline
    wraps its phase many times within one tile, and the running maximum and
    sum carry over hundreds of tiles."""
    lens, chunks = [20000, 9000], [48, 100]
    step, q, qs = _case(lens, chunks, 4, 1, D, bs, dtype, seed=D + 3)
    _check(step, q, qs, chunks)


@pytest.mark.parametrize("name", ["llama3_8b_gqa", "llama13b_mha"])
def test_prefill_full_size_sampled(name):
    """The prefill timed by the benchmark (`--op prefill`, chunks of 512): the
    full workload, its inputs drawn the same way, in one launch with the grid
    the benchmark gets (several row tiles per CTA on the 8B shape).  The fp64
    oracle checks a sample of it: the first, last, longest and shortest
    sequences, and the first and last kv head with their query heads, which
    attend independently of the other heads."""
    from paged_kv_cache_468_b200 import workloads
    cfg = workloads.CONFIGS[name]
    step = workloads.make_decode_step(cfg)
    lens = [int(x) for x in step["context_lens"]]
    chunks = [min(512, L) for L in lens]
    _, Hq, D = step["query"].shape
    Hkv = step["key_cache"].shape[2]
    G = Hq // Hkv
    g = torch.Generator().manual_seed(cfg.seed + 7)
    q = torch.randn(sum(chunks), Hq, D, generator=g).to(step["query"].dtype)
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    out = pkv.paged_attention_prefill(q.cuda(), torch.from_numpy(qs).cuda(), max(chunks),
                                      step["key_cache"].cuda(), step["value_cache"].cuda(),
                                      step["block_tables"].cuda(), step["context_lens"].cuda(),
                                      step["scale"]).cpu()
    B = len(lens)
    seqs = sorted({0, B - 1, int(np.argmax(lens)), int(np.argmin(lens))})
    kvh = [0, Hkv - 1]
    qh = [h * G + i for h in kvh for i in range(G)]
    rows = np.concatenate([np.arange(qs[b], qs[b + 1]) for b in seqs])
    sub_qs = np.concatenate([[0], np.cumsum([chunks[b] for b in seqs])]).astype(np.int32)
    ref = oracle.paged_attention_prefill(
        u16(q[rows][:, qh]), sub_qs, u16(step["key_cache"][:, :, kvh]),
        u16(step["value_cache"][:, :, kvh]), step["block_tables"].numpy()[seqs],
        step["context_lens"].numpy()[seqs], step["scale"], step["dtype"], nthreads=NTHREADS)
    err, idx, finite = max_abs_err(out[rows][:, qh], ref)
    assert finite and err <= TOL[step["dtype"]], (err, idx)
