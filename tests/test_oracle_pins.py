"""Pins for the CPU oracle: it is checked against things other than itself.

* a library routine: torch's scaled_dot_product_attention in float64 on the
  dense (unpaged) sequences the test lays out into pages itself;
* brute force with scalar loops on tiny inputs, using the softmax definition
  exp(x_t) / Σ exp(x_s) without any max shift;
* invariants the pages state: paging is transparent (any physical placement
  gives the same result), sharing blocks equals copying them, copy-on-write
  leaves siblings untouched;
* closed forms: one token returns its value vector, equal logits return the
  mean of V, one dominant logit returns that token's value;
* the partitioned (split-K) form equals the direct form.

``test_planted_mistakes_are_caught`` plants plausible mistakes in the oracle
(on the CPU, by monkeypatching) and checks that these pins catch each one.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A
from oracle import cache_ops as C
from oracle.dtypes import widen

NAN = {"fp16": 0x7E00, "bf16": 0x7FC0}


def torch_widen(bits, dtype):
    """Independent float64 widening through torch's own 16-bit types."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "fp16" else torch.bfloat16).double()


def random_bits(rng, shape, dtype):
    x = rng.standard_normal(shape).astype(np.float32)
    if dtype == "fp16":
        return x.astype(np.float16).view(np.uint16)
    return (x.view(np.uint32) >> 16).astype(np.uint16)   # truncation is fine for inputs


def lay_out(rng, dense_k, dense_v, block_size, dtype, spare_blocks=3):
    """Place dense per-sequence K/V ([C_i, Hkv, D] bit arrays) into a shuffled pool.

    This is the test's own placement, written from the page-table description,
    independently of the oracle's gather.
    """
    hkv, d = dense_k[0].shape[1], dense_k[0].shape[2]
    need = [-(-k.shape[0] // block_size) for k in dense_k]
    n = sum(need) + spare_blocks
    perm = rng.permutation(n)
    kc = np.full((n, hkv, block_size, d), NAN[dtype], dtype=np.uint16)
    vc = np.full_like(kc, NAN[dtype])
    mb = max(max(need), 1)
    tables = np.full((len(dense_k), mb), -1, dtype=np.int32)
    pos = 0
    for i, (k, v) in enumerate(zip(dense_k, dense_v)):
        for j in range(need[i]):
            b = perm[pos]
            pos += 1
            tables[i, j] = b
            rows = slice(j * block_size, min((j + 1) * block_size, k.shape[0]))
            cnt = rows.stop - rows.start
            kc[b, :, :cnt, :] = k[rows].transpose(1, 0, 2)
            vc[b, :, :cnt, :] = v[rows].transpose(1, 0, 2)
    lens = np.array([k.shape[0] for k in dense_k], dtype=np.int32)
    return kc, vc, tables, lens


def make_case(seed, lens, h, hkv, d, bs, dtype):
    rng = np.random.default_rng(seed)
    dk = [random_bits(rng, (c, hkv, d), dtype) for c in lens]
    dv = [random_bits(rng, (c, hkv, d), dtype) for c in lens]
    q = random_bits(rng, (len(lens), h, d), dtype)
    kc, vc, tables, clens = lay_out(rng, dk, dv, bs, dtype)
    return dict(q=q, dk=dk, dv=dv, kc=kc, vc=vc, tables=tables, lens=clens,
                h=h, hkv=hkv, d=d, bs=bs, dtype=dtype, scale=1.0 / math.sqrt(d))


def oracle_out(case, mod=A):
    return mod.paged_attention_decode(case["q"], case["kc"], case["vc"], case["tables"],
                                      case["lens"], case["scale"], case["hkv"], case["bs"],
                                      case["dtype"])


# ---------------------------------------------------------------------------
# 1. library routine on the dense sequences
# ---------------------------------------------------------------------------
def check_against_sdpa(case, mod=A):
    out = oracle_out(case, mod)
    g = case["h"] // case["hkv"]
    for i in range(len(case["lens"])):
        q = torch_widen(case["q"][i], case["dtype"])[None, :, None, :]          # [1,H,1,D]
        k = torch_widen(case["dk"][i], case["dtype"]).permute(1, 0, 2)[None]    # [1,Hkv,C,D]
        v = torch_widen(case["dv"][i], case["dtype"]).permute(1, 0, 2)[None]
        k = k.repeat_interleave(g, dim=1)
        v = v.repeat_interleave(g, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, scale=case["scale"])[0, :, 0, :].numpy()
        np.testing.assert_allclose(out[i], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("h,hkv,d,bs", [(4, 4, 64, 16), (8, 2, 32, 16), (8, 1, 16, 32),
                                        (6, 3, 64, 32)])
def test_oracle_equals_dense_sdpa(dtype, h, hkv, d, bs):
    case = make_case(11 + h + d, [1, 5, 16, 17, 33, 70], h, hkv, d, bs, dtype)
    check_against_sdpa(case)


# ---------------------------------------------------------------------------
# 2. brute force: scalar loops, softmax by its definition
# ---------------------------------------------------------------------------
def brute_force(case):
    g = case["h"] // case["hkv"]
    res = []
    for i, c in enumerate(case["lens"]):
        rows = []
        for h in range(case["h"]):
            q = widen(case["q"][i, h], case["dtype"]).tolist()
            K = widen(case["dk"][i][:, h // g, :], case["dtype"]).tolist()
            V = widen(case["dv"][i][:, h // g, :], case["dtype"]).tolist()
            x = [case["scale"] * sum(q[e] * K[t][e] for e in range(len(q))) for t in range(c)]
            ex = [math.exp(v_) for v_ in x]
            z = sum(ex)
            rows.append([sum(ex[t] * V[t][e] for t in range(c)) / z for e in range(len(q))])
        res.append(rows)
    return np.array(res)


def check_brute_force(case, mod=A):
    np.testing.assert_allclose(oracle_out(case, mod), brute_force(case), rtol=0, atol=1e-13)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_oracle_brute_force_tiny(dtype):
    case = make_case(5, [1, 2, 3], 4, 2, 4, 2, dtype)
    check_brute_force(case)


# ---------------------------------------------------------------------------
# 3. paging is transparent: any physical placement gives identical results
# ---------------------------------------------------------------------------
def relabel(case, perm):
    kc = np.empty_like(case["kc"])
    vc = np.empty_like(case["vc"])
    kc[perm] = case["kc"]
    vc[perm] = case["vc"]
    tables = np.where(case["tables"] >= 0, perm[np.maximum(case["tables"], 0)], -1)
    return dict(case, kc=kc, vc=vc, tables=tables.astype(np.int32))


def check_permutation_invariance(case, mod=A):
    base = oracle_out(case, mod)
    rng = np.random.default_rng(3)
    for _ in range(3):
        moved = relabel(case, rng.permutation(case["kc"].shape[0]))
        assert np.array_equal(oracle_out(moved, mod), base)


def test_permutation_invariance():
    check_permutation_invariance(make_case(21, [3, 16, 31, 48], 4, 2, 32, 16, "fp16"))


# ---------------------------------------------------------------------------
# 4. sharing blocks equals copying them
# ---------------------------------------------------------------------------
def test_sharing_invariance():
    case = make_case(31, [40, 40], 4, 4, 32, 16, "bf16")
    bs = case["bs"]
    # sequence 1 shares sequence 0's first two (full) blocks
    shared = dict(case)
    shared["tables"] = case["tables"].copy()
    shared["tables"][1, :2] = case["tables"][0, :2]
    # unshared equivalent: sequence 1 gets private copies of those blocks
    n = case["kc"].shape[0]
    kc = np.concatenate([case["kc"], case["kc"][case["tables"][0, :2]]])
    vc = np.concatenate([case["vc"], case["vc"][case["tables"][0, :2]]])
    copied = dict(case, kc=kc, vc=vc, tables=shared["tables"].copy())
    copied["tables"][1, :2] = [n, n + 1]
    a = oracle_out(shared)
    b = oracle_out(copied)
    assert np.array_equal(a, b)
    # and it is what dense attention over the shared prefix gives
    dense = dict(case)
    dense["dk"] = [case["dk"][0], np.concatenate([case["dk"][0][:2 * bs], case["dk"][1][2 * bs:]])]
    dense["dv"] = [case["dv"][0], np.concatenate([case["dv"][0][:2 * bs], case["dv"][1][2 * bs:]])]
    dense.update(kc=shared["kc"], vc=shared["vc"], tables=shared["tables"])
    check_against_sdpa(dense)


# ---------------------------------------------------------------------------
# 5. copy-on-write leaves the source and the siblings untouched
# ---------------------------------------------------------------------------
def test_cow_leaves_siblings_untouched():
    from oracle.block_manager import BlockManager
    rng = np.random.default_rng(41)
    bs, hkv, d, dtype = 16, 2, 32, "fp16"
    mgr = BlockManager(16, bs, free_order=rng.permutation(16))
    mgr.add_seq(0, 20)                      # 2 blocks, last one partial (4 tokens)
    for child in (1, 2):
        mgr.fork(0, child)
    kc = random_bits(rng, (16, hkv, bs, d), dtype)
    vc = random_bits(rng, (16, hkv, bs, d), dtype)
    q = random_bits(rng, (3, 4, d), dtype)
    before = A.paged_attention_decode(q, kc, vc, np.array(mgr.block_table([0, 1, 2], 4)),
                                      np.array([20, 20, 20]), 0.2, hkv, bs, dtype)
    slot, src, dst = mgr.append_slot(1)
    assert src >= 0 and dst >= 0 and src != dst
    kc2, vc2, bad = C.copy_blocks(kc, vc, np.array([[src, dst]]))
    assert not bad
    key = random_bits(rng, (1, hkv, d), dtype)
    kc3, vc3, bad = C.reshape_and_cache(key, key, kc2, vc2, np.array([slot]), bs)
    assert not bad
    assert slot // bs == dst
    assert np.array_equal(kc3[src], kc[src]) and np.array_equal(vc3[src], vc[src])
    after = A.paged_attention_decode(q, kc3, vc3, np.array(mgr.block_table([0, 1, 2], 4)),
                                     np.array([20, 21, 20]), 0.2, hkv, bs, dtype)
    assert np.array_equal(after[0], before[0]) and np.array_equal(after[2], before[2])
    assert not np.array_equal(after[1], before[1])


# ---------------------------------------------------------------------------
# 6. closed forms
# ---------------------------------------------------------------------------
def test_single_token_returns_its_value():
    case = make_case(51, [1, 1], 4, 2, 16, 16, "bf16")
    out = oracle_out(case)
    for i in range(2):
        for h in range(4):
            assert np.array_equal(out[i, h], widen(case["dv"][i][0, h // 2], "bf16"))


def test_equal_logits_give_mean_of_values():
    case = make_case(52, [9, 23], 2, 2, 16, 16, "fp16")
    # identical keys -> equal logits
    for i in range(2):
        case["dk"][i][:] = case["dk"][i][0]
    case["kc"], case["vc"], case["tables"], case["lens"] = lay_out(
        np.random.default_rng(1), case["dk"], case["dv"], 16, "fp16")
    out = oracle_out(case)
    for i in range(2):
        for h in range(2):
            mean = widen(case["dv"][i][:, h], "fp16").mean(axis=0)
            np.testing.assert_allclose(out[i, h], mean, rtol=0, atol=1e-14)
    # scale = 0 -> equal logits whatever the keys
    case2 = make_case(53, [7, 30], 2, 1, 16, 16, "fp16")
    case2["scale"] = 0.0
    out2 = oracle_out(case2)
    for i in range(2):
        mean = widen(case2["dv"][i][:, 0], "fp16").mean(axis=0)
        np.testing.assert_allclose(out2[i, 0], mean, rtol=0, atol=1e-14)
        np.testing.assert_allclose(out2[i, 1], mean, rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value():
    case = make_case(54, [12], 1, 1, 16, 16, "fp16")
    j = 7
    qv = widen(case["q"][0, 0], "fp16")
    # key j = 8·q (exact in fp16 for these magnitudes), others small
    dk = case["dk"][0].copy()
    dk[:] = np.float16(0.001).view(np.uint16)
    dk[j, 0] = (qv * 8).astype(np.float16).view(np.uint16)
    case["dk"] = [dk]
    case["kc"], case["vc"], case["tables"], case["lens"] = lay_out(
        np.random.default_rng(2), case["dk"], case["dv"], 16, "fp16")
    case["scale"] = 10.0
    out = oracle_out(case)
    np.testing.assert_allclose(out[0, 0], widen(case["dv"][0][j, 0], "fp16"), rtol=0, atol=1e-12)


def test_empty_context_gives_zeros():
    q = np.zeros((1, 2, 8), np.uint16)
    kc = np.full((2, 2, 16, 8), NAN["fp16"], np.uint16)
    out = A.paged_attention_decode(q, kc, kc, np.full((1, 1), -1, np.int32),
                                   np.array([0]), 1.0, 2, 16, "fp16")
    assert np.array_equal(out, np.zeros((1, 2, 8)))


# ---------------------------------------------------------------------------
# 7. partitioned form equals the direct form
# ---------------------------------------------------------------------------
def check_partitioned(case, mod=A):
    direct = oracle_out(case, mod)
    for part in (1, 7, 16, 512, int(case["lens"].max())):
        split = mod.paged_attention_decode_partitioned(
            case["q"], case["kc"], case["vc"], case["tables"], case["lens"], case["scale"],
            case["hkv"], case["bs"], case["dtype"], part)
        np.testing.assert_allclose(split, direct, rtol=0, atol=1e-12)


def test_partitioned_equals_direct():
    check_partitioned(make_case(61, [1, 15, 16, 17, 100, 600], 4, 2, 32, 16, "fp16"))


def test_partition_summary_closed_form():
    # two tokens with logits 0 and ln 3: m = ln 3, l = 1/3 + 1, o = V0/3 + V1
    q = np.array([1.0, 0.0])
    keys = np.array([[0.0, 5.0], [math.log(3.0), -2.0]])
    values = np.array([[3.0, 0.0], [0.0, 6.0]])
    m, l, o = A.partition_summary(q, keys, values, 1.0)
    assert m == pytest.approx(math.log(3.0), abs=1e-15)
    assert l == pytest.approx(4.0 / 3.0, abs=1e-15)
    np.testing.assert_allclose(o, [1.0, 6.0], atol=1e-15)
    # combining it with an empty partition changes nothing: out = (1, 6)/(4/3)
    out = A.combine_partitions([(m, l, o), (-np.inf, 0.0, np.zeros(2))])
    np.testing.assert_allclose(out, [0.75, 4.5], atol=1e-15)


# ---------------------------------------------------------------------------
# cache ops: written tokens are found again through the page table
# ---------------------------------------------------------------------------
def test_reshape_and_cache_round_trip():
    rng = np.random.default_rng(71)
    bs, hkv, d, n = 16, 3, 8, 6
    kc = random_bits(rng, (n, hkv, bs, d), "fp16")
    vc = random_bits(rng, (n, hkv, bs, d), "fp16")
    key = random_bits(rng, (5, hkv, d), "fp16")
    val = random_bits(rng, (5, hkv, d), "fp16")
    slots = np.array([0, 17, -1, n * bs - 1, 5 * bs + 3], dtype=np.int64)
    k2, v2, bad = C.reshape_and_cache(key, val, kc, vc, slots, bs)
    assert bad == []
    for t, s in enumerate(slots):
        if s < 0:
            continue
        row = np.array([s // bs], dtype=np.int32)   # a one-entry page table
        got = A.gather_kv(k2, row, s % bs + 1, 0, bs, "fp16")[-1]
        assert np.array_equal(got, widen(key[t, 0], "fp16"))
        assert np.array_equal(k2[s // bs, :, s % bs], key[t])
        assert np.array_equal(v2[s // bs, :, s % bs], val[t])
    touched = {(int(s) // bs, int(s) % bs) for s in slots if s >= 0}
    for b in range(n):
        for o in range(bs):
            if (b, o) not in touched:
                assert np.array_equal(k2[b, :, o], kc[b, :, o])
                assert np.array_equal(v2[b, :, o], vc[b, :, o])
    _, _, bad = C.reshape_and_cache(key[:1], val[:1], kc, vc, np.array([n * bs]), bs)
    assert bad == [0]


def test_copy_blocks_copies_whole_blocks_in_order():
    rng = np.random.default_rng(72)
    kc = random_bits(rng, (5, 2, 16, 8), "bf16")
    vc = random_bits(rng, (5, 2, 16, 8), "bf16")
    k2, v2, bad = C.copy_blocks(kc, vc, np.array([[0, 3], [1, 4]]))
    assert bad == []
    assert np.array_equal(k2[3], kc[0]) and np.array_equal(v2[3], vc[0])
    assert np.array_equal(k2[4], kc[1]) and np.array_equal(v2[4], vc[1])
    for b in (0, 1, 2):
        assert np.array_equal(k2[b], kc[b]) and np.array_equal(v2[b], vc[b])
    _, _, bad = C.copy_blocks(kc, vc, np.array([[0, 5], [-1, 2]]))
    assert bad == [0, 1]


# ---------------------------------------------------------------------------
# planted mistakes: each one must trip at least one pin
# ---------------------------------------------------------------------------
class Mutant:
    """A copy of the attention oracle with one function replaced."""

    def __init__(self, **overrides):
        self.__dict__.update({k: getattr(A, k) for k in dir(A) if not k.startswith("__")})
        self.__dict__.update(overrides)
        # rebind the module-level callers so they use the overrides
        for name in ("gather_kv", "paged_attention_decode", "paged_attention_decode_partitioned"):
            if name not in overrides:
                fn = getattr(A, name)
                g = dict(fn.__globals__)
                g.update(self.__dict__)
                self.__dict__[name] = type(fn)(fn.__code__, g, fn.__name__, fn.__defaults__)


def strided_kv_head(head, num_heads, num_kv_heads):
    return head % num_kv_heads


def swapped_location(table_row, t, block_size):
    t = np.asarray(t)
    return table_row[np.minimum(t % block_size, len(table_row) - 1)], t // block_size % block_size


def unscaled_attend(qvec, keys, values, scale):
    return A.attend(qvec, keys, values, 1.0)


def unnormalised_attend(qvec, keys, values, scale):
    if keys.shape[0] == 0:
        return np.zeros(values.shape[1])
    x = scale * (keys @ qvec)
    return np.exp(x - x.max()) @ values


def keys_as_values_attend(qvec, keys, values, scale):
    return A.attend(qvec, keys, keys, scale)


def sign_flipped_attend(qvec, keys, values, scale):
    return A.attend(qvec, keys, values, -scale)


def combine_without_l_weights(summaries):
    ms = np.array([m for m, _, _ in summaries])
    big = ms.max()
    w = np.exp(ms - big)
    return sum(x * o for x, (_, _, o) in zip(w, summaries)) / sum(l for _, l, _ in summaries)


MUTANTS = {
    "strided kv head": dict(kv_head_of=strided_kv_head),
    "swapped block/offset": dict(token_location=swapped_location),
    "dropped scale": dict(attend=unscaled_attend),
    "dropped normalisation": dict(attend=unnormalised_attend),
    "keys used as values": dict(attend=keys_as_values_attend),
    "wrong sign": dict(attend=sign_flipped_attend),
    "partition weights dropped": dict(combine_partitions=combine_without_l_weights),
}


def pins_pass(mod):
    gqa = make_case(81, [1, 5, 17, 40], 8, 2, 16, 16, "fp16")
    tiny = make_case(82, [2, 3], 4, 2, 4, 2, "fp16")
    try:
        check_against_sdpa(gqa, mod)
        check_brute_force(tiny, mod)
        check_permutation_invariance(gqa, mod)
        check_partitioned(gqa, mod)
    except (AssertionError, IndexError, ValueError):
        return False
    return True


def test_unmutated_oracle_passes_pin_suite():
    assert pins_pass(Mutant())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    assert not pins_pass(Mutant(**MUTANTS[name])), name


def test_package_exports():
    assert hasattr(oracle, "attention") and hasattr(oracle, "block_manager")
