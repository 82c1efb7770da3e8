"""The tolerance reading of the tensor-core prefill, checked on the host.

A numpy model of the kernel's arithmetic (key tiles of 64, a running maximum
moved only by more than 2^8, weights P rounded to the cache dtype, O and the
row sum accumulated in f32, O rounded to the cache dtype at the end) is
compared with the fp64 oracle on the case with growing scores.  It shows why
the kernel sums the *rounded* weights: with the unrounded sum the f16 error
exceeds the bound, with the rounded sum the error is the final rounding of O."""
import numpy as np
import torch

import oracle
from tests.parity_util import TOL, custom, u16

_DT = {"f16": torch.float16, "bf16": torch.bfloat16}
LENS, CHUNKS = [900, 333], [600, 333]


def _case(dtype):
    step = custom("pf", 2, 8, 2, 128, 16, dtype, LENS, seed=5)
    kc = step["key_cache"].float()
    tables = step["block_tables"]
    for s_, L in enumerate(LENS):
        for k in range((L + 15) // 16):
            kc[int(tables[s_, k])] *= 1.0 + 0.25 * k
    step["key_cache"] = kc.to(_DT[dtype])
    step["value_cache"] = (step["value_cache"].float() * 0.25).to(_DT[dtype])
    g = torch.Generator().manual_seed(6)
    q = torch.randn(sum(CHUNKS), 8, 128, generator=g).to(_DT[dtype])
    q = (q.float() * 2.0).to(_DT[dtype])
    return step, q


def _round(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(_DT[dtype]).double().numpy()


def _model(step, q, dtype, rounded_sum):
    """Outputs [T, Hq, D] of the kernel's arithmetic (fp64 where the kernel is exact)."""
    kc = step["key_cache"].double().numpy()
    vc = step["value_cache"].double().numpy()
    tables = step["block_tables"]
    sl2 = np.float32(step["scale"] * 1.4426950408889634)
    qn = q.double().numpy()
    out = np.zeros(qn.shape)
    q0 = 0
    for b, (L, C) in enumerate(zip(LENS, CHUNKS)):
        K = np.stack([kc[int(tables[b, j // 16]), j % 16] for j in range(L)])
        V = np.stack([vc[int(tables[b, j // 16]), j % 16] for j in range(L)])
        pos = L - C + np.arange(C)
        for h in range(8):
            S = qn[q0:q0 + C, h] @ K[:, h // 4].T
            x = np.where(np.arange(L)[None, :] <= pos[:, None], S.astype(np.float32) * sl2, -np.inf)
            m = np.full(C, -np.inf)
            l = np.zeros(C)
            O = np.zeros((C, 128))
            for t0 in range(0, L, 64):
                mt = x[:, t0:t0 + 64].max(1)
                resc = mt > m + 8
                mn = np.where(resc, mt, m)
                alpha = np.where(resc, np.exp2(m - mn), 1.0)
                p = np.exp2(x[:, t0:t0 + 64] - np.where(np.isinf(mn), 0, mn)[:, None]).astype(np.float32)
                pr = _round(p, dtype)
                l = (l * alpha + (pr if rounded_sum else p.astype(np.float64)).sum(1)).astype(np.float32)
                O = (O * alpha[:, None] + pr @ V[t0:t0 + 64, h // 4]).astype(np.float32).astype(np.float64)
                m = mn
            out[q0:q0 + C, h] = _round(O / l[:, None], dtype)
        q0 += C
    return out


def _oracle(step, q):
    qs = np.concatenate([[0], np.cumsum(CHUNKS)]).astype(np.int32)
    return oracle.paged_attention_prefill(u16(q), qs, u16(step["key_cache"]), u16(step["value_cache"]),
                                          step["block_tables"].numpy(), step["context_lens"].numpy(),
                                          step["scale"], step["dtype"], nthreads=8)


def test_rounded_weight_sum_keeps_the_error_at_the_output_rounding():
    for dtype in ("f16", "bf16"):
        step, q = _case(dtype)
        ref = _oracle(step, q)
        err = np.abs(_model(step, q, dtype, rounded_sum=True) - ref).max()
        assert err <= TOL[dtype], (dtype, err)
        # the error of rounding the exact result to the storage type alone
        floor = np.abs(_round(ref, dtype) - ref).max()
        assert err <= 1.5 * floor + 1e-6, (dtype, err, floor)


def test_unrounded_weight_sum_breaks_the_f16_bound_on_unscaled_values():
    # with V unscaled the outputs reach ~4; the unrounded sum then errs past
    # the f16 bound (a numpy model of the earlier kernel reproduced its GPU
    # error bit for bit)
    step, q = _case("f16")
    step["value_cache"] = (step["value_cache"].float() * 4.0).to(torch.float16)
    ref = _oracle(step, q)
    bad = np.abs(_model(step, q, "f16", rounded_sum=False) - ref).max()
    good = np.abs(_model(step, q, "f16", rounded_sum=True) - ref).max()
    assert bad > TOL["f16"] and good < bad, (bad, good)
