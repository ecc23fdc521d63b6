"""Pins for the fp64 oracle: each check ties it to something other than itself.

Sources of the pins:
  * a library routine for the special cases it covers:
    torch.nn.functional.scaled_dot_product_attention in float64 on the CPU
    (the PyTorch interface the aikaboom page names under "Integration"), and
    torch.logsumexp for the LSE;
  * the page's own numbers: the score matrix of N tokens has N^2 entries
    (aikaboom "11.4d FlashAttention", "The Core Problem"; golden file);
  * closed forms and invariants of the definition (rows of P sum to one,
    one-hot values return P, a single key returns its value, a zero query
    averages V, shift and permutation invariance, scale equivalence);
  * masking (fused scaling/masking on the zimaspace page, "Kernel Fusion"):
    a causal row never depends on later keys;
  * GQA (sicorps page, last paragraph): identical to MHA with each KV head
    repeated for its query group;
  * the tiled running-softmax recurrence (aikaboom "Online Softmax"; zimaspace
    "Online Softmax Avoids Storing the Full Score Matrix") brute-forced over
    every tile width on tiny inputs, and every split of the keys for the
    partial-result merge.
The last test plants plausible mistakes in a copy of the oracle and checks that
at least one pin catches each.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.nn.attention.bias import causal_lower_right

import oracle
import workloads
from oracle import attention as oracle_mod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * std)


def _sdpa(q, k, v, scale, causal):
    """Library reference: torch SDPA in fp64, causal aligned bottom-right."""
    Nq, Nk = q.shape[-2], k.shape[-2]
    gqa = q.shape[1] != k.shape[1]
    if causal:
        mask = causal_lower_right(Nq, Nk)
        return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale,
                                              enable_gqa=gqa)
    return F.scaled_dot_product_attention(q, k, v, scale=scale, enable_gqa=gqa)


def _lse_lib(q, k, scale, causal):
    Nq, Nk = q.shape[-2], k.shape[-2]
    if q.shape[1] != k.shape[1]:
        k = k.repeat_interleave(q.shape[1] // k.shape[1], dim=1)
    s = scale * (q @ k.transpose(-1, -2))
    if causal:
        keep = torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq)
        s = s.masked_fill(~keep, float("-inf"))
    return torch.logsumexp(s, dim=-1)


SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 1, 1, 7, 7, 8, False),
    (2, 2, 2, 9, 9, 16, True),
    (1, 4, 2, 5, 11, 8, True),    # Nq < Nk: bottom-right causal
    (2, 6, 3, 13, 13, 4, False),  # GQA, group 2
    (1, 8, 1, 6, 10, 8, True),    # MQA
    (1, 4, 4, 16, 3, 8, False),   # Nq > Nk non-causal
]


def check_sdpa(fn, shape, seed=0):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    q = _rand((B, Hq, Nq, d), seed)
    k = _rand((B, Hkv, Nk, d), seed + 1)
    v = _rand((B, Hkv, Nk, d), seed + 2)
    scale = 1.0 / math.sqrt(d) * 1.3
    o, lse = fn(q, k, v, scale, causal)
    o_ref = _sdpa(q, k, v, scale, causal).numpy()
    lse_ref = _lse_lib(q, k, scale, causal).numpy()
    return np.abs(o - o_ref).max(), np.abs(lse - lse_ref).max()


@pytest.mark.parametrize("shape", SHAPES)
def test_matches_torch_sdpa_fp64(shape):
    eo, el = check_sdpa(oracle.attention_ref, shape)
    assert eo < TOL and el < TOL


def test_score_matrix_entries_match_page_numbers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "score_matrix_sizes.txt"))
            if l.strip() and not l.startswith("#")]
    assert rows
    for tok, entries, doubled in rows:
        n, e, e2 = int(tok), int(entries), int(doubled)
        q = np.ones((n, 1))
        assert oracle.scores(q, q, 1.0).size == e
        assert e2 == 4 * e  # doubling the length quadruples the entries
        if n <= 2000:
            q2 = np.ones((2 * n, 1))
            assert oracle.scores(q2, q2, 1.0).size == e2


def test_rows_of_p_sum_to_one_and_mask_is_zero():
    for causal in (False, True):
        q = _rand((9, 8), 3)
        k = _rand((12, 8), 4)
        p = oracle.probabilities(q, k, 0.4, causal)
        assert np.abs(p.sum(axis=1) - 1).max() < TOL
        assert (p >= 0).all()
        if causal:
            for i in range(9):
                assert (p[i, i + 12 - 9 + 1:] == 0).all()


def test_one_hot_values_return_probabilities():
    d = 16
    q = _rand((1, 1, 5, d), 5)
    k = _rand((1, 1, d, d), 6)
    v = torch.eye(d, dtype=torch.float64)[None, None]
    for causal in (False, True):
        o, _ = oracle.attention_ref(q, k, v, 0.3, causal)
        p = oracle.probabilities(q[0, 0], k[0, 0], 0.3, causal)
        assert np.abs(o[0, 0] - p).max() < TOL


def test_single_key_returns_value_and_score():
    q = _rand((2, 3, 4, 8), 7)
    k = _rand((2, 3, 1, 8), 8)
    v = _rand((2, 3, 1, 8), 9)
    o, lse = oracle.attention_ref(q, k, v, 0.7, False)
    assert np.abs(o - v.numpy()).max() == 0.0  # P = 1 exactly
    s00 = 0.7 * np.einsum("bhqd,bhkd->bhqk", q.numpy(), k.numpy())[..., 0]
    assert np.abs(lse - s00).max() < TOL


def test_zero_query_averages_values():
    Nk, d = 10, 8
    q = torch.zeros((1, 1, Nk, d), dtype=torch.float64)
    k = _rand((1, 1, Nk, d), 10)
    v = _rand((1, 1, Nk, d), 11)
    o, lse = oracle.attention_ref(q, k, v, 1.0, False)
    assert np.abs(o[0, 0] - v[0, 0].numpy().mean(axis=0)).max() < TOL
    assert np.abs(lse - math.log(Nk)).max() < TOL
    o, lse = oracle.attention_ref(q, k, v, 1.0, True)
    for i in range(Nk):
        assert np.abs(o[0, 0, i] - v[0, 0, : i + 1].numpy().mean(axis=0)).max() < TOL
        assert abs(lse[0, 0, i] - math.log(i + 1)) < TOL


def test_causal_row_ignores_later_keys():
    Nq = Nk = 12
    q = _rand((1, 2, Nq, 8), 12)
    k = _rand((1, 2, Nk, 8), 13)
    v = _rand((1, 2, Nk, 8), 14)
    o, lse = oracle.attention_ref(q, k, v, 0.5, True)
    for i in range(Nq - 1):
        k2, v2 = k.clone(), v.clone()
        k2[:, :, i + 1:] += _rand(k2[:, :, i + 1:].shape, 100 + i) * 5
        v2[:, :, i + 1:] -= 3.0
        o2, lse2 = oracle.attention_ref(q, k2, v2, 0.5, True)
        assert np.abs(o2[:, :, : i + 1] - o[:, :, : i + 1]).max() == 0.0
        assert np.abs(lse2[:, :, : i + 1] - lse[:, :, : i + 1]).max() == 0.0
        assert np.abs(o2[:, :, i + 1:] - o[:, :, i + 1:]).max() > 1e-6


def test_gqa_equals_mha_with_repeated_kv():
    B, Hq, Hkv, N, d = 2, 8, 2, 9, 8
    q = _rand((B, Hq, N, d), 15)
    k = _rand((B, Hkv, N, d), 16)
    v = _rand((B, Hkv, N, d), 17)
    for causal in (False, True):
        o, lse = oracle.attention_ref(q, k, v, 0.4, causal)
        kr = k.repeat_interleave(Hq // Hkv, dim=1)
        vr = v.repeat_interleave(Hq // Hkv, dim=1)
        o2, lse2 = oracle.attention_ref(q, kr, vr, 0.4, causal)
        assert np.abs(o - o2).max() == 0.0 and np.abs(lse - lse2).max() == 0.0


def test_rows_without_visible_keys():
    # Nq > Nk causal: row i sees keys j <= i - (Nq - Nk); the first Nq-Nk rows see none.
    q = _rand((1, 1, 6, 4), 18)
    k = _rand((1, 1, 3, 4), 19)
    v = _rand((1, 1, 3, 4), 20)
    o, lse = oracle.attention_ref(q, k, v, 1.0, True)
    assert (o[0, 0, :3] == 0).all() and np.isneginf(lse[0, 0, :3]).all()
    o_tail, lse_tail = oracle.attention_ref(q[:, :, 3:], k, v, 1.0, True)
    assert np.abs(o[0, 0, 3:] - o_tail[0, 0]).max() == 0.0
    assert np.abs(lse[0, 0, 3:] - lse_tail[0, 0]).max() == 0.0


def test_row_subset_equals_full_rows():
    q = _rand((2, 4, 20, 8), 21)
    k = _rand((2, 2, 20, 8), 22)
    v = _rand((2, 2, 20, 8), 23)
    o, lse = oracle.attention_ref(q, k, v, 0.3, True)
    rows = np.array([0, 3, 7, 19])
    o2, lse2 = oracle.attention_ref(q, k, v, 0.3, True, rows=rows)
    assert np.abs(o[:, :, rows] - o2).max() == 0.0
    per_head = np.stack([np.stack([rows[::-1]] * 4)] * 2)
    o3, _ = oracle.attention_ref(q, k, v, 0.3, True, rows=per_head)
    assert np.abs(o[:, :, rows[::-1]] - o3).max() == 0.0


def test_shift_and_scale_invariances():
    q = _rand((1, 2, 7, 8), 24)
    k = _rand((1, 2, 9, 8), 25)
    v = _rand((1, 2, 9, 8), 26)
    o, lse = oracle.attention_ref(q, k, v, 0.5, False)
    u = _rand((8,), 27)
    o2, lse2 = oracle.attention_ref(q, k + u, v, 0.5, False)
    shift = 0.5 * (q.numpy() @ u.numpy())
    assert np.abs(o2 - o).max() < 1e-11
    assert np.abs(lse2 - (lse + shift)).max() < 1e-11
    o3, lse3 = oracle.attention_ref(q * 2, k, v, 0.25, False)
    assert np.abs(o3 - o).max() < TOL and np.abs(lse3 - lse).max() < TOL


def test_key_permutation_invariance_and_query_equivariance():
    q = _rand((1, 1, 6, 8), 28)
    k = _rand((1, 1, 11, 8), 29)
    v = _rand((1, 1, 11, 8), 30)
    o, lse = oracle.attention_ref(q, k, v, 0.6, False)
    perm = torch.randperm(11, generator=torch.Generator().manual_seed(1))
    o2, lse2 = oracle.attention_ref(q, k[:, :, perm], v[:, :, perm], 0.6, False)
    assert np.abs(o2 - o).max() < TOL and np.abs(lse2 - lse).max() < TOL
    qp = torch.randperm(6, generator=torch.Generator().manual_seed(2))
    o3, _ = oracle.attention_ref(q[:, :, qp], k, v, 0.6, False)
    assert np.abs(o3 - o[:, :, qp.numpy()]).max() == 0.0


@pytest.mark.parametrize("causal", [False, True])
def test_online_recurrence_matches_two_pass(causal):
    for n in range(1, 9):
        for nq in sorted({1, n}):
            q = _rand((nq, 4), 31 + n, std=3.0)
            k = _rand((n, 4), 41 + n, std=3.0)
            v = _rand((n, 4), 51 + n)
            o_ref, lse_ref = oracle.attention_ref(q[None, None], k[None, None],
                                                  v[None, None], 0.9, causal)
            for tile in range(1, n + 1):
                o, lse = oracle.online_softmax_attention(q, k, v, 0.9, causal, tile)
                assert np.abs(o - o_ref[0, 0]).max() < TOL
                fin = np.isfinite(lse_ref[0, 0])
                assert (np.isfinite(lse) == fin).all()
                assert np.abs(lse[fin] - lse_ref[0, 0][fin]).max(initial=0) < TOL


def _compositions(n):
    """Every way to cut range(n) into contiguous non-empty pieces."""
    for cuts in itertools.product([0, 1], repeat=n - 1):
        bounds = [0] + [i + 1 for i, c in enumerate(cuts) if c] + [n]
        yield list(zip(bounds[:-1], bounds[1:]))


def test_split_combine_matches_single_pass():
    d = 4
    for n in range(1, 8):
        q = _rand((1, 1, 1, d), 60 + n, std=2.0)
        k = _rand((1, 1, n, d), 70 + n, std=2.0)
        v = _rand((1, 1, n, d), 80 + n)
        o_ref, lse_ref = oracle.attention_ref(q, k, v, 0.8, False)
        for parts in _compositions(n):
            # plus one empty part, which must contribute nothing
            os_, ls_ = [np.zeros((1, 1, 1, d))], [np.full((1, 1, 1), -np.inf)]
            for a, b in parts:
                o, l = oracle.attention_ref(q, k[:, :, a:b], v[:, :, a:b], 0.8, False)
                os_.append(o)
                ls_.append(l)
            o, lse = oracle.combine_partials(np.stack(os_), np.stack(ls_))
            assert np.abs(o - o_ref).max() < TOL and np.abs(lse - lse_ref).max() < TOL


def test_decode_cache_layout_reading():
    # Values encode their own (b, g, t, c) so the unpacking is checked by value.
    B, Hkv, d = 3, 2, 4
    lens = [2, 0, 3]
    flat = []
    for b, L in enumerate(lens):
        for g in range(Hkv):
            for t in range(L):
                for c in range(d):
                    flat.append(1000 * b + 100 * g + 10 * t + c)
    parts = oracle.unpack_decode_cache(np.array(flat, dtype=np.float64), lens, Hkv, d)
    for b, L in enumerate(lens):
        assert parts[b].shape == (Hkv, L, d)
        for g in range(Hkv):
            for t in range(L):
                assert list(parts[b][g, t]) == [1000 * b + 100 * g + 10 * t + c
                                                for c in range(d)]


def test_decode_matches_sdpa_per_sequence():
    B, Hq, Hkv, d = 4, 8, 2, 8
    lens = [5, 1, 0, 9]
    q = _rand((B, Hq, d), 90)
    total = sum(lens)
    kc = _rand((total * Hkv * d,), 91)
    vc = _rand((total * Hkv * d,), 92)
    o, lse = oracle.decode_ref(q, kc, vc, lens, 0.35, Hkv)
    ks = oracle.unpack_decode_cache(kc, lens, Hkv, d)
    vs = oracle.unpack_decode_cache(vc, lens, Hkv, d)
    for b, L in enumerate(lens):
        if L == 0:
            assert (o[b] == 0).all() and np.isneginf(lse[b]).all()
            continue
        kt = torch.from_numpy(ks[b])[None]
        vt = torch.from_numpy(vs[b])[None]
        ref = F.scaled_dot_product_attention(q[b][None, :, None], kt, vt, scale=0.35,
                                             enable_gqa=True)
        assert np.abs(o[b] - ref[0, :, 0].numpy()).max() < TOL
        lref = _lse_lib(q[b][None, :, None], kt, 0.35, False)[0, :, 0].numpy()
        assert np.abs(lse[b] - lref).max() < TOL


def test_oracle_accepts_low_precision_inputs_exactly():
    q = _rand((1, 1, 4, 8), 93).to(torch.bfloat16)
    k = _rand((1, 1, 4, 8), 94).to(torch.float16)
    v = _rand((1, 1, 4, 8), 95).to(torch.bfloat16)
    o, _ = oracle.attention_ref(q, k, v, 0.5, False)
    o2, _ = oracle.attention_ref(q.double(), k.double(), v.double(), 0.5, False)
    assert np.abs(o - o2).max() == 0.0


# ----------------------------------------------------------------------------
# Planted mistakes: each plausible error in the oracle must trip a pin above.

def _all_pins_pass():
    try:
        for shape in SHAPES:
            eo, el = check_sdpa(oracle_mod.attention_ref, shape)
            if not (eo < TOL and el < TOL):
                return False
        test_single_key_returns_value_and_score()
        test_gqa_equals_mha_with_repeated_kv()
        test_rows_without_visible_keys()
    except AssertionError:
        return False
    return True


def test_pins_catch_planted_mistakes(monkeypatch):
    assert _all_pins_pass()

    good_visible = oracle_mod._visible
    good_scores = oracle_mod.scores
    good_head = oracle_mod._head_ref

    def top_left(nq, nk, causal, rows, window=0):  # causal aligned top-left instead
        cols = np.arange(nk)[None, :]
        if not causal:
            return np.ones((rows.size, nk), dtype=bool)
        return cols <= rows[:, None]

    def no_scale(q_rows, k, scale):
        return q_rows @ k.T

    def transposed(q_rows, k, scale):
        return scale * (q_rows @ k[::-1].T)

    def lse_without_max(qh, kh, vh, scale, causal, nq, rows, window=0):
        o, lse = good_head(qh, kh, vh, scale, causal, nq, rows, window)
        s = scale * (qh @ kh.T)
        return o, lse - s.max(axis=1)

    def modulo_group(q, k, v, scale, causal, rows=None):
        # GQA head map h % Hkv instead of h // group
        qq = oracle_mod._f64(q)
        kk = oracle_mod._f64(k)
        vv = oracle_mod._f64(v)
        Hq, Hkv = qq.shape[1], kk.shape[1]
        idx = [h % Hkv for h in range(Hq)]
        kr = kk[:, idx]
        vr = vv[:, idx]
        return good_attention(qq, kr, vr, scale, causal, rows)

    good_attention = oracle_mod.attention_ref
    plants = [
        ("_visible", top_left),
        ("scores", no_scale),
        ("scores", transposed),
        ("_head_ref", lse_without_max),
        ("attention_ref", modulo_group),
    ]
    for name, fn in plants:
        with monkeypatch.context() as m:
            m.setattr(oracle_mod, name, fn)
            if name == "attention_ref":
                m.setattr(oracle, "attention_ref", fn)
            assert not _all_pins_pass(), f"planted mistake {fn.__name__} went unnoticed"
    assert oracle_mod._visible is good_visible and oracle_mod.scores is good_scores


def test_subset_query_rows_with_full_length():
    q = _rand((1, 2, 30, 8), 96)
    k = _rand((1, 1, 30, 8), 97)
    v = _rand((1, 1, 30, 8), 98)
    rows = np.array([0, 5, 17, 29])
    o, lse = oracle.attention_ref(q, k, v, 0.4, True, rows=rows)
    o2, lse2 = oracle.attention_ref(q[:, :, rows], k, v, 0.4, True, rows=rows, nq=30)
    assert np.abs(o - o2).max() == 0.0 and np.abs(lse - lse2).max() == 0.0


# ------------------------------------------------------------------ sliding window
# Reading: causal query i keeps keys j with i + off - W < j <= i + off
# (off = Nk - Nq), the W most recent positions including its own; decode keeps
# the last W cached tokens (zimaspace page, "Reduced IO Is Not the Same as
# Eliminating KV Cache", names windowing as a runtime scheme).

def _window_brute(q, k, v, scale, W):
    """Pure-Python loops over the visible keys of each row (small inputs)."""
    q, k, v = (oracle_mod._f64(x) for x in (q, k, v))
    nq, nk, d = q.shape[0], k.shape[0], v.shape[1]
    off = nk - nq
    o = np.zeros((nq, d))
    lse = np.full(nq, -np.inf)
    for i in range(nq):
        js = [j for j in range(nk) if i + off - W < j <= i + off]
        if not js:
            continue
        s = [scale * sum(q[i, c] * k[j, c] for c in range(q.shape[1])) for j in js]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = sum(e)
        for jj, j in enumerate(js):
            o[i] += e[jj] / tot * v[j]
        lse[i] = mx + math.log(tot)
    return o, lse


@pytest.mark.parametrize("nq,nk,W", [(7, 7, 3), (5, 9, 2), (9, 5, 4), (6, 6, 1), (4, 10, 20)])
def test_window_matches_brute_force(nq, nk, W):
    q = _rand((1, 1, nq, 5), 300 + nq)
    k = _rand((1, 1, nk, 5), 310 + nk)
    v = _rand((1, 1, nk, 5), 320 + W)
    o, lse = oracle.attention_ref(q, k, v, 0.7, True, window=W)
    ob, lb = _window_brute(q[0, 0], k[0, 0], v[0, 0], 0.7, W)
    fin = np.isfinite(lb)
    assert np.abs(o[0, 0] - ob).max() < 1e-12
    assert np.array_equal(np.isfinite(lse[0, 0]), fin)
    assert np.abs(lse[0, 0][fin] - lb[fin]).max() < 1e-12


def test_window_one_key_returns_that_value():
    q = _rand((1, 2, 6, 4), 330)
    k = _rand((1, 1, 9, 4), 331)
    v = _rand((1, 1, 9, 4), 332)
    o, lse = oracle.attention_ref(q, k, v, 0.5, True, window=1)
    qq, kk, vv = (oracle_mod._f64(x) for x in (q, k, v))
    off = 9 - 6
    for h in range(2):
        for i in range(6):
            assert np.array_equal(o[0, h, i], vv[0, 0, i + off])
            assert abs(lse[0, h, i] - 0.5 * qq[0, h, i] @ kk[0, 0, i + off]) < 1e-12


def test_window_wider_than_keys_is_plain_causal():
    q = _rand((2, 2, 11, 6), 340)
    k = _rand((2, 1, 11, 6), 341)
    v = _rand((2, 1, 11, 6), 342)
    o, lse = oracle.attention_ref(q, k, v, 0.3, True, window=11)
    o2, lse2 = oracle.attention_ref(q, k, v, 0.3, True)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_window_ignores_keys_outside_it():
    q = _rand((1, 1, 8, 4), 350)
    k = _rand((1, 1, 8, 4), 351)
    v = _rand((1, 1, 8, 4), 352)
    o, _ = oracle.attention_ref(q, k, v, 0.6, True, window=3)
    k2, v2 = k.clone(), v.clone()
    k2[0, 0, :4] += 5.0  # keys 0..3 are outside the windows of rows 6 and 7
    v2[0, 0, :4] -= 3.0
    o2, _ = oracle.attention_ref(q, k2, v2, 0.6, True, window=3)
    assert np.array_equal(o[0, 0, 6:], o2[0, 0, 6:])
    assert not np.array_equal(o[0, 0, :4], o2[0, 0, :4])


def test_window_online_recurrence_matches_two_pass():
    q = _rand((1, 1, 13, 6), 360)
    k = _rand((1, 1, 13, 6), 361)
    v = _rand((1, 1, 13, 6), 362)
    o, lse = oracle.attention_ref(q, k, v, 0.4, True, window=5)
    for tile in (1, 2, 3, 4, 13):
        ot, lt = oracle.online_softmax_attention(q[0, 0], k[0, 0], v[0, 0], 0.4, True, tile,
                                                 window=5)
        assert np.abs(ot - o[0, 0]).max() < 1e-12 and np.abs(lt - lse[0, 0]).max() < 1e-12


def test_decode_window_equals_single_row_prefill():
    # decode reading the last W tokens == causal prefill of one row (Nq = 1) with window W
    sl = torch.tensor([9, 3, 0, 12], dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(4, 4, 2, 8, sl, torch.float32, seed=370)
    W = 4
    o, lse = oracle.decode_ref(q, kc, vc, sl, 0.5, 2, window=W)
    caches = oracle.unpack_decode_cache(kc, sl, 2, 8), oracle.unpack_decode_cache(vc, sl, 2, 8)
    for b in range(4):
        L = int(sl[b])
        if L == 0:
            assert np.all(o[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        kb = caches[0][b][None]
        vb = caches[1][b][None]
        ob, lb = oracle.attention_ref(q[b][None, :, None, :], kb, vb, 0.5, True, window=W)
        assert np.abs(ob[0, :, 0] - o[b]).max() < 1e-12
        assert np.abs(lb[0, :, 0] - lse[b]).max() < 1e-12


def test_window_requires_causal():
    q = _rand((1, 1, 4, 4), 380)
    with pytest.raises(ValueError):
        oracle.attention_ref(q, q, q, 0.5, False, window=2)


def test_window_pins_catch_an_off_by_one(monkeypatch):
    good = oracle_mod._visible

    def wide(nq, nk, causal, rows, window=0):  # keeps W + 1 keys
        return good(nq, nk, causal, rows, window + 1 if window else 0)

    monkeypatch.setattr(oracle_mod, "_visible", wide)
    with pytest.raises(AssertionError):
        test_window_matches_brute_force(7, 7, 3)
    with pytest.raises(AssertionError):
        test_window_one_key_returns_that_value()


# Property sweep: random shapes, groupings, lengths and scales against the
# library routine (fp64 torch SDPA with a bottom-right causal mask).
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 2), Hkv=st.integers(1, 3), group=st.integers(1, 4),
       Nq=st.integers(1, 17), Nk=st.integers(1, 17), d=st.sampled_from([4, 8, 16]),
       causal=st.booleans(), scale=st.floats(0.05, 2.0), seed=st.integers(0, 10_000))
def test_property_sweep_matches_torch_sdpa(B, Hkv, group, Nq, Nk, d, causal, scale, seed):
    if causal and Nq > Nk:
        Nq, Nk = Nk, Nq  # every causal row keeps at least its diagonal key
    Hq = Hkv * group
    q = _rand((B, Hq, Nq, d), seed)
    k = _rand((B, Hkv, Nk, d), seed + 1)
    v = _rand((B, Hkv, Nk, d), seed + 2)
    o, lse = oracle.attention_ref(q, k, v, scale, causal)
    assert np.abs(o - _sdpa(q, k, v, scale, causal).numpy()).max() < TOL
    assert np.abs(lse - _lse_lib(q, k, scale, causal).numpy()).max() < TOL


@settings(max_examples=40, deadline=None)
@given(Hkv=st.integers(1, 2), group=st.integers(1, 3), Nq=st.integers(1, 15),
       extra=st.integers(0, 10), W=st.integers(1, 20), seed=st.integers(0, 10_000))
def test_property_sweep_window_matches_banded_sdpa(Hkv, group, Nq, extra, W, seed):
    # The window as an explicit band of the score matrix handed to SDPA:
    # row i keeps keys j with i + off - W < j <= i + off, off = Nk - Nq >= 0.
    Nk = Nq + extra
    Hq, d, scale = Hkv * group, 8, 0.4
    q = _rand((1, Hq, Nq, d), seed)
    k = _rand((1, Hkv, Nk, d), seed + 1)
    v = _rand((1, Hkv, Nk, d), seed + 2)
    i = torch.arange(Nq)[:, None] + extra
    j = torch.arange(Nk)[None, :]
    band = (j <= i) & (j > i - W)
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=band, scale=scale,
                                         enable_gqa=group > 1)
    kr = k.repeat_interleave(group, dim=1)
    s = (scale * (q @ kr.transpose(-1, -2))).masked_fill(~band, float("-inf"))
    o, lse = oracle.attention_ref(q, k, v, scale, True, window=W)
    assert np.abs(o - ref.numpy()).max() < TOL
    assert np.abs(lse - torch.logsumexp(s, dim=-1).numpy()).max() < TOL
