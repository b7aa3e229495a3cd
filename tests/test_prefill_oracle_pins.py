"""Pins for the chunked-prefill oracle.

* torch scaled_dot_product_attention (float64) on the dense sequences with an
  explicit boolean mask: query j of a sequence with C tokens and q_len queries
  sees keys 0..C-q_len+j.  The test builds the dense data and the paged layout
  itself.
* q_len = 1 reduces to decode.
* brute force with scalar loops on tiny inputs.
* placement invariance.
* planted mistakes (off-by-one causal bound, positions counted from the start
  of the context instead of its end) are caught.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle.dtypes import widen
from test_oracle_pins import lay_out, random_bits, relabel, torch_widen


def make_prefill_case(seed, hist, new, h, hkv, d, bs, dtype):
    rng = np.random.default_rng(seed)
    lens = [a + b for a, b in zip(hist, new)]
    dk = [random_bits(rng, (c, hkv, d), dtype) for c in lens]
    dv = [random_bits(rng, (c, hkv, d), dtype) for c in lens]
    q = random_bits(rng, (sum(new), h, d), dtype)
    kc, vc, tables, clens = lay_out(rng, dk, dv, bs, dtype)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    return dict(q=q, dk=dk, dv=dv, kc=kc, vc=vc, tables=tables, lens=clens, qs=qs, new=new,
                h=h, hkv=hkv, d=d, bs=bs, dtype=dtype, scale=1.0 / math.sqrt(d))


def prefill(case, mod=A):
    return mod.paged_attention_prefill(case["q"], case["kc"], case["vc"], case["tables"],
                                       case["lens"], case["qs"], case["scale"], case["hkv"],
                                       case["bs"], case["dtype"])


def check_sdpa(case, mod=A):
    out = prefill(case, mod)
    g = case["h"] // case["hkv"]
    for i, c in enumerate(case["lens"]):
        a, b = case["qs"][i], case["qs"][i + 1]
        nq = b - a
        q = torch_widen(case["q"][a:b], case["dtype"]).permute(1, 0, 2)[None]          # [1,H,nq,D]
        k = torch_widen(case["dk"][i], case["dtype"]).permute(1, 0, 2)[None].repeat_interleave(g, 1)
        v = torch_widen(case["dv"][i], case["dtype"]).permute(1, 0, 2)[None].repeat_interleave(g, 1)
        keys = torch.arange(int(c))[None, :]
        pos = (int(c) - nq + torch.arange(nq))[:, None]
        mask = keys <= pos                                                               # [nq, C]
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                               scale=case["scale"])
        np.testing.assert_allclose(out[a:b], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("h,hkv,d,bs", [(4, 4, 32, 16), (8, 2, 16, 32)])
def test_prefill_equals_masked_sdpa(dtype, h, hkv, d, bs):
    check_sdpa(make_prefill_case(3 + d, [0, 7, 40, 16], [5, 1, 20, 33], h, hkv, d, bs, dtype))


def test_single_query_reduces_to_decode():
    case = make_prefill_case(9, [4, 30, 0], [1, 1, 1], 4, 2, 32, 16, "fp16")
    dec = A.paged_attention_decode(case["q"], case["kc"], case["vc"], case["tables"], case["lens"],
                                   case["scale"], case["hkv"], case["bs"], case["dtype"])
    assert np.array_equal(prefill(case), dec)


def brute(case):
    g = case["h"] // case["hkv"]
    res = np.zeros(case["q"].shape)
    for i, c in enumerate(case["lens"]):
        for jj, t in enumerate(range(case["qs"][i], case["qs"][i + 1])):
            pos = int(c) - case["new"][i] + jj
            for h in range(case["h"]):
                q = widen(case["q"][t, h], case["dtype"]).tolist()
                K = widen(case["dk"][i][:, h // g], case["dtype"]).tolist()
                V = widen(case["dv"][i][:, h // g], case["dtype"]).tolist()
                ex = [math.exp(case["scale"] * sum(a * b for a, b in zip(q, K[s])))
                      for s in range(pos + 1)]
                z = sum(ex)
                res[t, h] = [sum(ex[s] * V[s][e] for s in range(pos + 1)) / z
                             for e in range(len(q))]
    return res


def test_prefill_brute_force_tiny():
    case = make_prefill_case(4, [1, 0], [2, 3], 2, 1, 4, 2, "bf16")
    np.testing.assert_allclose(prefill(case), brute(case), rtol=0, atol=1e-13)


def test_prefill_placement_invariance():
    case = make_prefill_case(5, [3, 20], [4, 9], 4, 4, 16, 16, "fp16")
    base = prefill(case)
    moved = relabel(case, np.random.default_rng(1).permutation(case["kc"].shape[0]))
    assert np.array_equal(prefill(moved), base)


class PrefillMutant:
    def __init__(self, body):
        self.paged_attention_prefill = body


def off_by_one(q_bits, kc, vc, tables, lens, qs, scale, hkv, bs, dtype, rows=None):
    """sees keys 0..p-1 instead of 0..p"""
    out = A.paged_attention_prefill(q_bits, kc, vc, tables, lens, qs, scale, hkv, bs, dtype)
    qs = np.asarray(qs)
    for s in range(len(qs) - 1):
        for j, t in enumerate(range(qs[s], qs[s + 1])):
            pos = int(lens[s]) - (qs[s + 1] - qs[s]) + j
            for h in range(q_bits.shape[1]):
                g = A.kv_head_of(h, q_bits.shape[1], hkv)
                K = A.gather_kv(kc, tables[s], lens[s], g, bs, dtype)[:max(pos, 1)]
                V = A.gather_kv(vc, tables[s], lens[s], g, bs, dtype)[:max(pos, 1)]
                out[t, h] = A.attend(widen(q_bits[t, h], dtype), K, V, scale)
    return out


def from_start(q_bits, kc, vc, tables, lens, qs, scale, hkv, bs, dtype, rows=None):
    """counts positions from the start of the context"""
    qs = np.asarray(qs)
    fake_lens = np.array([qs[s + 1] - qs[s] for s in range(len(qs) - 1)])
    return A.paged_attention_prefill(q_bits, kc, vc, tables, np.maximum(fake_lens, 1), qs, scale,
                                     hkv, bs, dtype)


@pytest.mark.parametrize("body", [off_by_one, from_start])
def test_planted_prefill_mistakes_are_caught(body):
    case = make_prefill_case(6, [5, 0], [3, 4], 2, 2, 8, 16, "fp16")
    with pytest.raises(AssertionError):
        check_sdpa(case, PrefillMutant(body))
