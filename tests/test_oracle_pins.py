"""Pins the CPU oracle to facts outside itself: the pages' worked examples
(tests/golden), closed forms of softmax attention, a library routine (torch's
scaled_dot_product_attention in float64 on a contiguous layout), and
invariants the pages state (results do not depend on physical block ids).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _kv(name):
    return {r[0]: r[1] for r in _rows(name)}


# ---------------------------------------------------------------- indexing

def test_block_counts_match_pages(oracle_lib):
    rows = _rows("block_counts.txt")
    assert len(rows) >= 9
    for r in rows:
        n, bs, blocks = int(r[0]), int(r[1]), int(r[2])
        assert oracle.blocks_needed(n, bs) == blocks, r


def test_prefix_cache_demo_block_arithmetic(oracle_lib):
    """[P4] §3.2 printed output: 300 / 201 / 99 / 33.0% / 12.4 MB."""
    g = _kv("prefix_cache_demo.txt")
    bs = int(g["block_size"])
    n_req = int(g["num_requests"])
    pb = oracle.blocks_needed(int(g["system_prompt_tokens"]), bs)
    ub = oracle.blocks_needed(int(g["user_tokens"]), bs)
    assert pb == int(g["prefix_blocks"]) and ub == int(g["user_blocks"])
    without = n_req * (pb + ub)
    with_cache = pb + n_req * ub
    assert without == int(g["blocks_without_cache"])
    assert with_cache == int(g["blocks_with_cache"])
    assert without - with_cache == int(g["blocks_saved"])
    assert f"{(without - with_cache) / without * 100:.1f}" == g["saving_pct"]
    assert f"{(without - with_cache) * int(g['block_kib']) / 1024:.1f}" == g["saved_mib"]


# ------------------------------------------------------- paged test inputs

def _paged_case(rng, S, Hq, Hkv, D, bs, ctx, NB, garbage=1e4):
    """Logical K/V per sequence, scattered into a pool block by block through
    a random table. The scatter uses whole-block reshapes (no per-token
    index arithmetic), so it checks the oracle's gather independently.
    Unused pool rows hold `garbage`, unused table entries hold -1."""
    MB = max(1, max(-(-c // bs) for c in ctx))
    kpool = np.full((NB, Hkv, bs, D), garbage)
    vpool = np.full((NB, Hkv, bs, D), -garbage)
    bt = np.full((S, MB), -1, np.int32)
    perm = rng.permutation(NB)
    used = 0
    K, V = [], []
    for s, L in enumerate(ctx):
        nb = -(-L // bs)
        Ks = rng.normal(size=(L, Hkv, D))
        Vs = rng.normal(size=(L, Hkv, D))
        K.append(Ks)
        V.append(Vs)
        ids = perm[used:used + nb]
        used += nb
        bt[s, :nb] = ids
        if nb:
            pad = nb * bs - L
            Kp = np.concatenate([Ks, np.full((pad, Hkv, D), garbage)])
            Vp = np.concatenate([Vs, np.full((pad, Hkv, D), -garbage)])
            kpool[ids] = Kp.reshape(nb, bs, Hkv, D).transpose(0, 2, 1, 3)
            vpool[ids] = Vp.reshape(nb, bs, Hkv, D).transpose(0, 2, 1, 3)
    q = rng.normal(size=(S, Hq, D))
    return q, kpool, vpool, bt, np.array(ctx, np.int32), K, V


def _sdpa(q, K, V, scale):
    """torch scaled_dot_product_attention in float64 on contiguous K/V
    [L, Hkv, D]; GQA via repeat_interleave (query head h -> kv head h // G)."""
    Hq = q.shape[0]
    L, Hkv, D = K.shape
    if L == 0:
        return np.zeros((Hq, D))
    G = Hq // Hkv
    qt = torch.from_numpy(q).reshape(Hq, 1, D)
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o.reshape(Hq, D).numpy()


@pytest.mark.parametrize("Hq,Hkv,D,bs", [(4, 4, 8, 4), (8, 2, 16, 16), (6, 3, 8, 32)])
def test_paged_matches_sdpa_on_contiguous(oracle_lib, Hq, Hkv, D, bs):
    rng = np.random.default_rng(1)
    ctx = [1, 5, bs, bs + 1, 3 * bs + 7, 0]
    q, kp, vp, bt, cl, K, V = _paged_case(rng, len(ctx), Hq, Hkv, D, bs, ctx, 40)
    scale = 1 / math.sqrt(D)
    out = oracle.paged_decode(q, kp, vp, bt, cl, scale, bs)
    for s in range(len(ctx)):
        ref = _sdpa(q[s], K[s], V[s], scale)
        np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-12)


def test_context_one_returns_that_value(oracle_lib):
    rng = np.random.default_rng(2)
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 3, 4, 2, 8, 16, [1, 1, 1], 8)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.3, 16)
    for s in range(3):
        for h in range(4):
            assert np.array_equal(out[s, h], V[s][0, h // 2])


def test_identical_keys_give_mean_of_values(oracle_lib):
    rng = np.random.default_rng(3)
    ctx = [7, 33, 64]
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 3, 2, 2, 8, 16, ctx, 16)
    for s, L in enumerate(ctx):  # every key of the sequence equal to its first
        for t in range(L):
            kp[bt[s, t // 16], :, t % 16, :] = K[s][0]
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.5, 16)
    for s in range(3):
        np.testing.assert_allclose(out[s], V[s].mean(axis=0), rtol=0, atol=1e-12)


def test_zero_scale_gives_mean_over_exactly_the_context(oracle_lib):
    rng = np.random.default_rng(4)
    ctx = [3, 16, 17, 40]
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 4, 3, 3, 8, 16, ctx, 12)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.0, 16)
    for s in range(4):
        np.testing.assert_allclose(out[s], V[s].mean(axis=0), rtol=0, atol=1e-12)


def test_two_token_closed_form(oracle_lib):
    """z0 = 0, z1 = ln 3  =>  weights 1/4, 3/4."""
    D, bs = 2, 16
    kp = np.zeros((2, 1, bs, D))
    vp = np.zeros((2, 1, bs, D))
    kp[1, 0, 0] = [0.0, 0.0]
    kp[1, 0, 1] = [math.log(3.0), 0.0]
    vp[1, 0, 0] = [1.0, 0.0]
    vp[1, 0, 1] = [0.0, 1.0]
    q = np.array([[[1.0, 0.0]]])
    out = oracle.paged_decode(q, kp, vp, np.array([[1]], np.int32), np.array([2], np.int32), 1.0, bs)
    np.testing.assert_allclose(out[0, 0], [0.25, 0.75], rtol=0, atol=1e-15)


def test_one_dominant_key(oracle_lib):
    rng = np.random.default_rng(5)
    D, L = 16, 40
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 1, 1, 1, D, 16, [L], 4)
    K0 = K[0] / np.linalg.norm(K[0], axis=-1, keepdims=True)
    for t in range(L):
        kp[bt[0, t // 16], 0, t % 16] = K0[t, 0] * 0.01
    j = 29
    kp[bt[0, j // 16], 0, j % 16] = q[0, 0] / np.dot(q[0, 0], q[0, 0]) * 60.0  # z_j = 60
    out = oracle.paged_decode(q, kp, vp, bt, cl, 1.0, 16)
    np.testing.assert_allclose(out[0, 0], V[0][j, 0], rtol=0, atol=1e-20 + 50 * math.exp(-59))


def test_physical_permutation_is_bit_invariant(oracle_lib):
    rng = np.random.default_rng(6)
    ctx = [9, 31, 64, 50]
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 4, 4, 2, 8, 16, ctx, 20)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.35, 16)
    perm = rng.permutation(20)        # new id of old block b is perm[b]
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = oracle.paged_decode(q, kp2, vp2, bt2, cl, 0.35, 16)
    assert np.array_equal(out, out2)


def test_token_order_invariance(oracle_lib):
    """Attention is a weighted set sum: permuting a sequence's (key, value)
    pairs leaves it unchanged; a key/value index mix-up would not."""
    rng = np.random.default_rng(7)
    L, bs = 45, 16
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 1, 2, 2, 8, bs, [L], 6)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.4, bs)
    p = rng.permutation(L)
    for t in range(L):
        kp[bt[0, t // bs], :, t % bs] = K[0][p[t]]
        vp[bt[0, t // bs], :, t % bs] = V[0][p[t]]
    out2 = oracle.paged_decode(q, kp, vp, bt, cl, 0.4, bs)
    np.testing.assert_allclose(out, out2, rtol=1e-13, atol=1e-13)


def test_bad_tables_are_rejected(oracle_lib):
    rng = np.random.default_rng(8)
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 2, 2, 2, 8, 16, [20, 3], 6)
    bad = bt.copy()
    bad[0, 1] = 6  # == num_blocks
    with pytest.raises(oracle.OracleError, match="out of range"):
        oracle.paged_decode(q, kp, vp, bad, cl, 1.0, 16)
    with pytest.raises(oracle.OracleError, match="too short"):
        oracle.paged_decode(q, kp, vp, bt, np.array([40, 3], np.int32), 1.0, 16)


# ----------------------------------------------------------------- split-K

@pytest.mark.parametrize("P", [16, 48, 1000])
def test_splitk_merge_equals_decode(oracle_lib, P):
    rng = np.random.default_rng(9)
    ctx = [1, 16, 100, 257, 0]
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 5, 4, 2, 8, 16, ctx, 40)
    maxp = -(-max(ctx) // P)
    m, l, acc = oracle.splitk_partials(q, kp, vp, bt, cl, 0.3, 16, P, maxp)
    out = oracle.splitk_merge(m, l, acc, cl, P)
    ref = oracle.paged_decode(q, kp, vp, bt, cl, 0.3, 16)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_splitk_single_partition_terms(oracle_lib):
    rng = np.random.default_rng(10)
    L, D = 23, 8
    q, kp, vp, bt, cl, K, V = _paged_case(rng, 1, 1, 1, D, 16, [L], 3)
    m, l, acc = oracle.splitk_partials(q, kp, vp, bt, cl, 0.5, 16, 64, 1)
    z = 0.5 * K[0][:, 0] @ q[0, 0]
    w = np.exp(z - z.max())
    assert m[0, 0, 0] == z.max()
    np.testing.assert_allclose(l[0, 0, 0], w.sum(), rtol=1e-14)
    np.testing.assert_allclose(acc[0, 0, 0], w @ V[0][:, 0], rtol=1e-13, atol=1e-14)


def test_splitk_merge_closed_form(oracle_lib):
    """Two partitions, m = (0, ln 2), l = (1, 1), acc = (e0, e1):
    weights 1/2 and 1 => out = (1/2, 1) / (3/2) = (1/3, 2/3)."""
    m = np.array([[[0.0, math.log(2.0)]]])
    l = np.array([[[1.0, 1.0]]])
    acc = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    out = oracle.splitk_merge(m, l, acc, np.array([30], np.int32), 16)
    np.testing.assert_allclose(out[0, 0], [1 / 3, 2 / 3], rtol=0, atol=1e-15)


# ------------------------------------------------------ slot write / copy

@pytest.mark.parametrize("dtype", [np.float32, np.float16, np.float64])
def test_reshape_and_cache_lands_on_slot_rows(oracle_lib, dtype):
    """With the pool viewed per kv head as [num_blocks * block_size, D] rows
    (a pure reshape of [NB, Hkv, bs, D]), slot s is row s."""
    rng = np.random.default_rng(11)
    NB, Hkv, bs, D, T = 6, 3, 4, 8, 7
    kc = rng.normal(size=(NB, Hkv, bs, D)).astype(dtype)
    vc = rng.normal(size=(NB, Hkv, bs, D)).astype(dtype)
    k0, v0 = kc.copy(), vc.copy()
    key = rng.normal(size=(T, Hkv, D)).astype(dtype)
    val = rng.normal(size=(T, Hkv, D)).astype(dtype)
    slots = np.array([0, 23, -1, 5, 17, -7, 12], np.int32)
    oracle.reshape_and_cache(kc, vc, key, val, slots)
    krows = kc.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)
    vrows = vc.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)
    k0rows = k0.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)
    written = set()
    for i, s in enumerate(slots):
        if s < 0:
            continue
        written.add(int(s))
        assert np.array_equal(krows[:, s].view(np.uint8), key[i].view(np.uint8))
        assert np.array_equal(vrows[:, s].view(np.uint8), val[i].view(np.uint8))
    for s in range(NB * bs):
        if s not in written:
            assert np.array_equal(krows[:, s].view(np.uint8), k0rows[:, s].view(np.uint8))


def test_reshape_and_cache_is_bitwise(oracle_lib):
    """NaN payloads and negative zero survive: the write is a byte copy."""
    NB, Hkv, bs, D = 2, 1, 16, 8
    kc = np.zeros((NB, Hkv, bs, D), np.float16)
    vc = np.zeros_like(kc)
    bits = np.array([0x7E01, 0x8000, 0xFC00, 0x7C00, 0x0001, 0xFBFF, 0x3C00, 0x7FFF], np.uint16)
    key = bits.view(np.float16).reshape(1, 1, D)
    oracle.reshape_and_cache(kc, vc, key, key.copy(), np.array([19], np.int32))
    assert np.array_equal(kc[1, 0, 3].view(np.uint16), bits)
    assert np.array_equal(vc[1, 0, 3].view(np.uint16), bits)


def test_reshape_and_cache_rejects_out_of_range_slot(oracle_lib):
    kc = np.zeros((2, 1, 4, 8), np.float32)
    vc = np.zeros_like(kc)
    key = np.ones((1, 1, 8), np.float32)
    with pytest.raises(oracle.OracleError, match="slot"):
        oracle.reshape_and_cache(kc, vc, key, key, np.array([8], np.int32))


def test_copy_blocks(oracle_lib):
    rng = np.random.default_rng(12)
    kc = rng.normal(size=(8, 2, 4, 8)).astype(np.float16)
    vc = rng.normal(size=(8, 2, 4, 8)).astype(np.float16)
    k0, v0 = kc.copy(), vc.copy()
    pairs = [(1, 5), (1, 6), (3, 0)]
    oracle.copy_blocks(kc, vc, pairs)
    for s, d in pairs:
        assert np.array_equal(kc[d].view(np.uint16), k0[s].view(np.uint16))
        assert np.array_equal(vc[d].view(np.uint16), v0[s].view(np.uint16))
    for b in (1, 2, 3, 4, 7):
        assert np.array_equal(kc[b].view(np.uint16), k0[b].view(np.uint16))
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(kc, vc, [(0, 8)])


# ------------------------------------------------------------------ prefill

def test_prefill_matches_causal_sdpa(oracle_lib):
    """Each sequence's new tokens, attended causally over the paged cache,
    equal torch SDPA in float64 with an explicit causal mask on the
    contiguous K/V (query i sees positions <= L - q_len + i)."""
    rng = np.random.default_rng(20)
    ctx = [1, 17, 40, 33]
    qlen = [1, 5, 40, 7]
    Hq, Hkv, D, bs = 4, 2, 8, 16
    q_, kp, vp, bt, cl, K, V = _paged_case(rng, len(ctx), Hq, Hkv, D, bs, ctx, 12)
    qs = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    Q = rng.normal(size=(int(qs[-1]), Hq, D))
    out = oracle.paged_prefill(Q, qs, kp, vp, bt, cl, 0.3, bs)
    for s, (L, ql) in enumerate(zip(ctx, qlen)):
        qt = torch.from_numpy(Q[qs[s]:qs[s + 1]]).permute(1, 0, 2)             # [Hq, ql, D]
        kt = torch.from_numpy(K[s]).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        vt = torch.from_numpy(V[s]).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        pos = torch.arange(L - ql, L).unsqueeze(1)
        mask = torch.arange(L).unsqueeze(0) <= pos                               # [ql, L]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)
        np.testing.assert_allclose(out[qs[s]:qs[s + 1]], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_prefill_of_one_token_is_decode(oracle_lib):
    rng = np.random.default_rng(21)
    ctx = [5, 64, 1]
    q_, kp, vp, bt, cl, K, V = _paged_case(rng, 3, 4, 4, 8, 16, ctx, 10)
    qs = np.arange(4, dtype=np.int32)
    a = oracle.paged_prefill(q_, qs, kp, vp, bt, cl, 0.5, 16)
    b = oracle.paged_decode(q_, kp, vp, bt, cl, 0.5, 16)
    assert np.array_equal(a, b)


def test_prefill_first_token_sees_only_itself(oracle_lib):
    """A sequence prefilled from empty: its first token attends to itself
    only (out = V[0]); its last token sees the whole context."""
    rng = np.random.default_rng(22)
    L = 20
    q_, kp, vp, bt, cl, K, V = _paged_case(rng, 1, 2, 2, 8, 16, [L], 4)
    Q = rng.normal(size=(L, 2, 8))
    out = oracle.paged_prefill(Q, np.array([0, L], np.int32), kp, vp, bt, cl, 0.4, 16)
    assert np.array_equal(out[0], V[0][0])
    last = oracle.paged_decode(Q[L - 1:L], kp, vp, bt, cl, 0.4, 16)
    np.testing.assert_allclose(out[L - 1], last[0], rtol=0, atol=0)


# ------------------------------------------------------------ int8 KV cache

def test_quantize_worked_rows(oracle_lib):
    """Hand-worked rows. [254, 1, -1, 3]: amax 254, inv = 127/254 = 0.5
    exactly, codes rint(127, 0.5, -0.5, 1.5) = 127, 0, 0, 2 (halves go to
    even), scale 2. [1, -3, 0.5, 2.5]: inv = 127/3, codes 42.33 -> 42,
    -127, 21.17 -> 21, 105.83 -> 106. A zero row: codes 0, scale 0. A row
    with amax 127 and integer values: scale 1, codes equal to the values."""
    x = np.array([[254, 1, -1, 3], [1, -3, 0.5, 2.5], [0, 0, 0, 0], [127, -5, 64, -127]], np.float32)
    q, s = oracle.quantize_rows(x)
    assert q.tolist() == [[127, 0, 0, 2], [42, -127, 21, 106], [0, 0, 0, 0], [127, -5, 64, -127]]
    assert s[0] == 2.0 and s[2] == 0.0 and s[3] == 1.0
    assert s[1] == np.float32(3.0) / np.float32(127.0)


def test_quantize_error_bound_and_range(oracle_lib):
    """Every nonzero row uses the full code range (max |q| = 127, at the
    row's largest magnitude), keeps each sign, and dequantizes within half a
    step: |x - q s| <= s / 2 (plus fp32 rounding of the step)."""
    rng = np.random.default_rng(21)
    x = (rng.normal(size=(500, 128)) * rng.uniform(1e-3, 1e3, size=(500, 1))).astype(np.float32)
    x[7] = 0.0
    x[8, :5] = [1e-30, -2e-30, 0, 0, 0]
    x[8, 5:] = 0
    q, s = oracle.quantize_rows(x)
    nz = np.abs(x).max(axis=1) > 0
    assert np.all(np.abs(q[nz].astype(int)).max(axis=1) == 127)
    assert np.all(q[~nz] == 0) and np.all(s[~nz] == 0)
    assert np.all((q == 0) | (np.sign(q) == np.sign(x)))
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-5))
    am = np.abs(x).max(axis=1)
    assert np.allclose(s[nz], am[nz] / 127.0, rtol=1e-6)


def test_reshape_and_cache_q8_lands_on_slot_rows(oracle_lib):
    """Per kv head, code row s and scale s of the reshaped pools are token i's
    quantized row (slot s = slots[i]); negative slots write nothing."""
    rng = np.random.default_rng(12)
    NB, Hkv, bs, D, T = 5, 2, 4, 16, 6
    kc = rng.integers(-127, 128, size=(NB, Hkv, bs, D)).astype(np.int8)
    vc = kc.copy()
    ks = rng.uniform(size=(NB, Hkv, bs)).astype(np.float32)
    vs = ks.copy()
    k0, ks0 = kc.copy(), ks.copy()
    key = rng.normal(size=(T, Hkv, D)).astype(np.float32)
    val = rng.normal(size=(T, Hkv, D)).astype(np.float32)
    slots = np.array([3, 19, -1, 0, 10, 7], np.int32)
    oracle.reshape_and_cache_q8(kc, vc, ks, vs, key, val, slots)
    krows = kc.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)
    vrows = vc.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)
    kscl = ks.transpose(1, 0, 2).reshape(Hkv, NB * bs)
    vscl = vs.transpose(1, 0, 2).reshape(Hkv, NB * bs)
    k0rows = k0.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)
    ks0r = ks0.transpose(1, 0, 2).reshape(Hkv, NB * bs)
    qk, sk = oracle.quantize_rows(key)
    qv, sv = oracle.quantize_rows(val)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        assert np.array_equal(krows[:, s], qk[i]) and np.array_equal(vrows[:, s], qv[i])
        assert np.array_equal(kscl[:, s], sk[i]) and np.array_equal(vscl[:, s], sv[i])
    for s in set(range(NB * bs)) - {int(x) for x in slots if x >= 0}:
        assert np.array_equal(krows[:, s], k0rows[:, s]) and np.array_equal(kscl[:, s], ks0r[:, s])


def test_decode_q8_closed_forms_and_precision(oracle_lib):
    """ctx = 1 gives the dequantized V[0] exactly; over random N(0, 1) data
    the int8 cache's attention stays within 2% (relative L2) of the same
    attention over the unquantized values, the precision the pages warn
    quantization costs."""
    rng = np.random.default_rng(13)
    S, Hq, Hkv, D, bs = 3, 8, 2, 64, 16
    ctx = np.array([1, 200, 77], np.int32)
    NB = 40
    tables = np.full((S, 13), -1, np.int32)
    perm = rng.permutation(NB)
    pos = 0
    for s_, L in enumerate(ctx):
        n = -(-int(L) // bs)
        tables[s_, :n] = perm[pos:pos + n]
        pos += n
    kf = rng.normal(size=(NB, Hkv, bs, D)).astype(np.float32)
    vf = rng.normal(size=(NB, Hkv, bs, D)).astype(np.float32)
    kq, ks = oracle.quantize_rows(kf)
    vq, vs = oracle.quantize_rows(vf)
    q = rng.normal(size=(S, Hq, D))
    out = oracle.paged_decode_q8(q, kq, vq, ks, vs, tables, ctx, 1 / 8, bs)
    v0 = vq[tables[0, 0], :, 0].astype(np.float64) * vs[tables[0, 0], :, 0, None]
    assert np.array_equal(out[0], np.repeat(v0, Hq // Hkv, axis=0))
    ref = oracle.paged_decode(q, kf, vf, tables, ctx, 1 / 8, bs)
    rel = np.linalg.norm(out[1:] - ref[1:]) / np.linalg.norm(ref[1:])
    assert 1e-4 < rel < 2e-2
