"""Checks that pin the CPU oracle to things other than itself.

Each check takes an ``oracle.Oracle`` and raises AssertionError when the oracle disagrees with
what the pages or the mathematics fix:

- a library routine computing the same special case independently (torch's fp64 CPU
  ``scaled_dot_product_attention``, with and without ``enable_gqa``; ``repeat_interleave``);
- closed forms (one row; a zero query; one dominant score);
- invariants (weights sum to one, token order, shifting every key row, linearity in V);
- the endpoints the pages state: G = H is MHA exactly, G = 1 is MQA, and collapsing heads by
  averaging changes the output unless G = H (lesson "r-tf2-gqa", next-experiment section);
- brute force in pure Python with exactly rounded sums on the tiny workload's shape;
- the append's position and length update, and its overflow refusal (Algorithm 2 of
  "GQA 阅读笔记", the lines that write K_cache[t, g, :] and V_cache[t, g, :]).

``tests/test_oracle_pins.py`` runs them on the oracle; ``tests/test_oracle_mutants.py`` plants
plausible mistakes in copies of the oracle and checks that some pin catches each one.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa_reference(q, K, V, lens, scale, enable_gqa=True):
    """torch fp64 SDPA per sequence over its first n_b rows.  q [B,H_q,d], K/V [B,L,H_kv,d]."""
    B, H_q, d = q.shape
    out = np.zeros((B, H_q, d))
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            continue
        qq = torch.from_numpy(q[b]).unsqueeze(1).unsqueeze(0)            # [1,H_q,1,d]
        kk = torch.from_numpy(np.ascontiguousarray(K[b, :n].transpose(1, 0, 2))).unsqueeze(0)
        vv = torch.from_numpy(np.ascontiguousarray(V[b, :n].transpose(1, 0, 2))).unsqueeze(0)
        o = F.scaled_dot_product_attention(qq, kk, vv, scale=scale, enable_gqa=enable_gqa)
        out[b] = o[0, :, 0, :].numpy()
    return out


def _rand_case(seed, B, H_q, H_kv, d, L_max, lens=None, std=1.0):
    r = _rng(seed)
    q = r.standard_normal((B, H_q, d)) * std
    K = r.standard_normal((B, L_max, H_kv, d)) * std
    V = r.standard_normal((B, L_max, H_kv, d))
    if lens is None:
        lens = r.integers(1, L_max + 1, size=B)
    return q, K, V, np.asarray(lens, dtype=np.int32)


# ----------------------------------------------------------------------------------------------
def pin_append_position(o):
    r = _rng(11)
    B, L_max, H_kv, d = 5, 9, 3, 8
    K = r.standard_normal((B, L_max, H_kv, d))
    V = r.standard_normal((B, L_max, H_kv, d))
    K0, V0 = K.copy(), V.copy()
    kn = r.standard_normal((B, H_kv, d))
    vn = r.standard_normal((B, H_kv, d))
    lens = np.array([0, 3, L_max - 1, 5, 1], dtype=np.int32)
    lens0 = lens.copy()
    st = o.kv_append(kn, vn, K, V, lens)
    assert st == 0, st
    assert np.array_equal(lens, lens0 + 1)
    for b in range(B):
        t = lens0[b]
        assert np.array_equal(K[b, t], kn[b]) and np.array_equal(V[b, t], vn[b])
        mask = np.ones(L_max, bool)
        mask[t] = False
        assert np.array_equal(K[b, mask], K0[b, mask]) and np.array_equal(V[b, mask], V0[b, mask])


def pin_append_overflow(o):
    r = _rng(12)
    B, L_max, H_kv, d = 2, 4, 2, 4
    K = r.standard_normal((B, L_max, H_kv, d))
    V = r.standard_normal((B, L_max, H_kv, d))
    K0, V0 = K.copy(), V.copy()
    lens = np.array([L_max, 2], dtype=np.int32)
    kn = r.standard_normal((B, H_kv, d))
    vn = r.standard_normal((B, H_kv, d))
    st = o.kv_append(kn, vn, K, V, lens)
    assert st & 1, "overflow must be reported"
    assert lens[0] == L_max and lens[1] == 3
    assert np.array_equal(K[0], K0[0]) and np.array_equal(V[0], V0[0])
    assert np.array_equal(K[1, 2], kn[1])


def pin_expand_matches_repeat_interleave(o):
    r = _rng(13)
    for H_q, H_kv in [(8, 2), (6, 6), (8, 1), (12, 4)]:
        L_max, d, n = 7, 5, 6
        c = r.standard_normal((L_max, H_kv, d))
        got = o.expand_kv(c, n, H_q)
        want = torch.from_numpy(c[:n]).repeat_interleave(H_q // H_kv, dim=1).numpy()
        assert np.array_equal(got, want), (H_q, H_kv)


def pin_single_head_vs_sdpa(o):
    r = _rng(14)
    for n, d, scale in [(1, 16, 0.25), (7, 64, 0.125), (300, 128, 1 / math.sqrt(128))]:
        q = r.standard_normal(d)
        K = r.standard_normal((n, d))
        V = r.standard_normal((n, d))
        got, w = o.attend_one_head(q, K, V, scale)
        want = F.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
            torch.from_numpy(V)[None, None], scale=scale)[0, 0, 0].numpy()
        assert np.max(np.abs(got - want)) <= 1e-12, (n, d)


def pin_decode_vs_sdpa_gqa(o):
    cases = [
        (2, 8, 2, 64, 40, None, 0.125),
        (3, 64, 8, 128, 33, None, 1 / math.sqrt(128)),
        (2, 32, 1, 128, 50, None, 1 / math.sqrt(128)),
        (2, 12, 4, 16, 20, [1, 20], 0.3),
        (1, 64, 64, 64, 30, [30], 0.125),
    ]
    for i, (B, H_q, H_kv, d, L_max, lens, scale) in enumerate(cases):
        q, K, V, lens = _rand_case(100 + i, B, H_q, H_kv, d, L_max, lens)
        got = o.decode(q, K, V, lens, scale)
        want = _sdpa_reference(q, K, V, lens, scale, enable_gqa=True)
        assert np.max(np.abs(got - want)) <= 1e-12, (i, np.max(np.abs(got - want)))


def pin_mha_endpoint(o):
    """G = H: plain multi-head attention (Algorithm 1), against SDPA without grouping."""
    q, K, V, lens = _rand_case(21, 2, 6, 6, 32, 25)
    got = o.decode(q, K, V, lens, 0.2)
    want = _sdpa_reference(q, K, V, lens, 0.2, enable_gqa=False)
    assert np.max(np.abs(got - want)) <= 1e-12


def pin_mqa_endpoint(o):
    """G = 1: every query head attends the single key/value head (MQA)."""
    q, K, V, lens = _rand_case(22, 2, 8, 1, 32, 25)
    got = o.decode(q, K, V, lens, 0.2)
    for b in range(2):
        n = lens[b]
        for h in range(8):
            want = F.scaled_dot_product_attention(
                torch.from_numpy(q[b, h])[None, None, None],
                torch.from_numpy(np.ascontiguousarray(K[b, :n, 0]))[None, None],
                torch.from_numpy(np.ascontiguousarray(V[b, :n, 0]))[None, None],
                scale=0.2)[0, 0, 0].numpy()
            assert np.max(np.abs(got[b, h] - want)) <= 1e-12


def pin_expand_then_attend_equivalence(o):
    """A grouped cache gives bit-identical results to the MHA cache made by repeating each
    key/value head over its block of query heads (lesson "r-tf2-gqa")."""
    for H_kv in (8, 2, 1):
        q, K, V, lens = _rand_case(23 + H_kv, 2, 8, H_kv, 16, 12)
        got = o.decode(q, K, V, lens, 0.25)
        Kr = np.repeat(K, 8 // H_kv, axis=2)
        Vr = np.repeat(V, 8 // H_kv, axis=2)
        want = o.decode(q, Kr, Vr, lens, 0.25)
        assert np.array_equal(got, want), H_kv


def pin_grouping_changes_output(o):
    """Averaging an MHA cache's heads per group: g = h leaves the output unchanged exactly,
    a smaller g changes it (lesson "r-tf2-gqa", next-experiment section)."""
    q, K, V, lens = _rand_case(31, 1, 8, 8, 16, 30)
    base = o.decode(q, K, V, lens, 0.25)
    for g in (8, 4, 1):
        Kg = K.reshape(1, 30, g, 8 // g, 16).mean(axis=3)
        Vg = V.reshape(1, 30, g, 8 // g, 16).mean(axis=3)
        out = o.decode(q, Kg, Vg, lens, 0.25)
        diff = np.max(np.abs(out - base))
        if g == 8:
            assert diff == 0.0
        else:
            assert diff > 1e-3, (g, diff)


def pin_closed_forms(o):
    r = _rng(41)
    d = 32
    # one row: the output is that row of V, exactly
    q = r.standard_normal(d)
    K = r.standard_normal((1, d))
    V = r.standard_normal((1, d))
    out, w = o.attend_one_head(q, K, V, 0.3)
    assert np.array_equal(out, V[0]) and w[0] == 1.0
    # zero query: uniform weights, the output is the mean of the value rows
    K = r.standard_normal((37, d))
    V = r.standard_normal((37, d))
    out, w = o.attend_one_head(np.zeros(d), K, V, 0.3)
    assert np.max(np.abs(out - V.mean(axis=0))) <= 1e-14
    assert np.max(np.abs(w - 1 / 37)) <= 1e-16
    # all key rows equal: uniform weights as well
    Ke = np.tile(K[:1], (37, 1))
    out, _ = o.attend_one_head(q, Ke, V, 0.3)
    assert np.max(np.abs(out - V.mean(axis=0))) <= 1e-14
    # one score above the rest by more than 800: all weight on that row
    K = r.standard_normal((20, d)) * 0.01
    qd = np.zeros(d)
    qd[0] = 1.0
    K[7, 0] = 1000.0
    out, w = o.attend_one_head(qd, K, V[:20], 1.0)
    assert np.array_equal(out, V[7]) and w[7] == 1.0


def pin_invariants(o):
    r = _rng(51)
    n, d = 64, 32
    q = r.standard_normal(d)
    K = r.standard_normal((n, d))
    V = r.standard_normal((n, d))
    out, w = o.attend_one_head(q, K, V, 0.2)
    assert abs(w.sum() - 1.0) <= 1e-14
    perm = r.permutation(n)
    out_p, _ = o.attend_one_head(q, K[perm], V[perm], 0.2)
    assert np.max(np.abs(out_p - out)) <= 1e-13
    c = r.standard_normal(d) * 3
    out_s, _ = o.attend_one_head(q, K + c, V, 0.2)
    assert np.max(np.abs(out_s - out)) <= 1e-12
    V2 = r.standard_normal((n, d))
    out_2, _ = o.attend_one_head(q, K, V2, 0.2)
    out_12, _ = o.attend_one_head(q, K, V + V2, 0.2)
    assert np.max(np.abs(out_12 - (out + out_2))) <= 1e-13
    # doubling q and halving the scale leaves every score, hence the output, unchanged
    out_sc, _ = o.attend_one_head(q * 2.0, K, V, 0.1)
    assert np.max(np.abs(out_sc - out)) <= 1e-13


def _fsum_attention(q, K, V, scale):
    n, d = len(K), len(q)
    s = [scale * math.fsum(q[i] * K[t][i] for i in range(d)) for t in range(n)]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    z = math.fsum(e)
    return [math.fsum(e[t] * V[t][i] for t in range(n)) / z for i in range(d)]


def pin_brute_force_tiny(o):
    """The tiny workload's shape (B=1, H_q=8, H_kv=2, d=64, 256 rows, scale 1/8), evaluated in
    pure Python with exactly rounded sums."""
    q, K, V, lens = _rand_case(61, 1, 8, 2, 64, 256, [256])
    got = o.decode(q, K, V, lens, 0.125)
    for h in range(8):
        g = h // 4
        want = _fsum_attention(q[0, h].tolist(), K[0, :, g].tolist(), V[0, :, g].tolist(), 0.125)
        assert np.max(np.abs(got[0, h] - np.array(want))) <= 1e-13, h


def pin_empty_and_range(o):
    q, K, V, _ = _rand_case(71, 3, 4, 2, 8, 6)
    lens = np.array([0, 3, 7], dtype=np.int32)
    out, st = o.decode(q, K, V, lens, 0.5, return_status=True)
    assert st & 2
    assert np.array_equal(out[0], np.zeros((4, 8))) and np.array_equal(out[2], np.zeros((4, 8)))
    want = _sdpa_reference(q[1:2], K[1:2], V[1:2], [3], 0.5)
    assert np.max(np.abs(out[1] - want[0])) <= 1e-12


def pin_divisibility(o):
    q, K, V, lens = _rand_case(81, 1, 6, 4, 8, 5)
    try:
        o.decode(q, K, V, lens, 0.5)
    except ValueError:
        return
    raise AssertionError("H_q % H_kv != 0 must be rejected")


def pin_window(o):
    """Sliding window (reading notes, what came after GQA: Mistral's W): a window at least as long
    as the sequence is the full decode; a window of one row returns the newest V row exactly;
    any window equals the full decode of the cache cut to its last `window` rows; and torch SDPA
    on those rows agrees."""
    q, K, V, lens = _rand_case(91, 3, 8, 2, 16, 40, [40, 7, 25])
    full = o.decode(q, K, V, lens, 0.3)
    assert np.array_equal(o.decode_window(q, K, V, lens, 40, 0.3), full)
    assert np.array_equal(o.decode_window(q, K, V, lens, 0, 0.3), full)
    one = o.decode_window(q, K, V, lens, 1, 0.3)
    for b in range(3):
        for h in range(8):
            assert np.array_equal(one[b, h], V[b, lens[b] - 1, h // 4])
    for W in (5, 10):
        got = o.decode_window(q, K, V, lens, W, 0.3)
        for b in range(3):
            n = lens[b]
            first = max(0, n - W)
            cut_k = np.ascontiguousarray(K[b:b + 1, first:n])
            cut_v = np.ascontiguousarray(V[b:b + 1, first:n])
            want = o.decode(q[b:b + 1], cut_k, cut_v, np.array([n - first], dtype=np.int32), 0.3)
            assert np.array_equal(got[b], want[0])
            sd = _sdpa_reference(q[b:b + 1], cut_k, cut_v, [n - first], 0.3)
            assert np.max(np.abs(got[b] - sd[0])) <= 1e-12


def pin_paged(o):
    """Paged cache (reading notes, what came after GQA: vLLM's block-managed cache): the gather
    agrees with numpy fancy indexing; an identity block table reproduces the contiguous cache;
    permuting the pages (with the table permuted alike) changes nothing, bit for bit; the paged
    append lands where the contiguous append does; a missing page is refused."""
    r = _rng(101)
    B, P, max_pages, H_kv, d = 3, 8, 5, 2, 16
    L = P * max_pages
    n_pages = B * max_pages
    lens = np.array([39, 1, 17], dtype=np.int32)
    Kc = r.standard_normal((B, L, H_kv, d))
    Vc = r.standard_normal((B, L, H_kv, d))
    ident = np.arange(n_pages, dtype=np.int32).reshape(B, max_pages)
    kpool = Kc.reshape(n_pages, P, H_kv, d).copy()
    vpool = Vc.reshape(n_pages, P, H_kv, d).copy()
    g, st = o.paged_gather(kpool, ident, lens)
    assert st == 0
    for b in range(B):
        assert np.array_equal(g[b, :lens[b]], Kc[b, :lens[b]])
        t = np.arange(lens[b])
        assert np.array_equal(g[b, :lens[b]], kpool[ident[b, t // P], t % P])
    q = r.standard_normal((B, 8, d))
    base = o.decode(q, Kc, Vc, lens, 0.25)
    assert np.array_equal(o.decode_paged(q, kpool, vpool, ident, lens, 0.25), base)
    perm = r.permutation(n_pages).astype(np.int32)
    kpool2 = np.empty_like(kpool)
    vpool2 = np.empty_like(vpool)
    kpool2[perm] = kpool
    vpool2[perm] = vpool
    table2 = perm[ident]
    assert np.array_equal(o.decode_paged(q, kpool2, vpool2, table2, lens, 0.25), base)
    kn = r.standard_normal((B, H_kv, d))
    vn = r.standard_normal((B, H_kv, d))
    l1 = lens.copy()
    l2 = lens.copy()
    Kc2, Vc2 = Kc.copy(), Vc.copy()
    assert o.kv_append(kn, vn, Kc2, Vc2, l1) == 0
    assert o.kv_append_paged(kn, vn, kpool2, vpool2, table2, l2) == 0
    assert np.array_equal(l1, l2)
    g2, _ = o.paged_gather(kpool2, table2, l2)
    for b in range(B):
        assert np.array_equal(g2[b, :l2[b]], Kc2[b, :l1[b]])
    bad = table2.copy()
    bad[1, l2[1] // P] = n_pages  # the page the next row of sequence 1 would go to does not exist
    l3 = l2.copy()
    assert o.kv_append_paged(kn, vn, kpool2, vpool2, bad, l3) & 1
    assert l3[1] == l2[1]
    full = l2.copy()
    full[2] = L  # a full sequence is refused too
    assert o.kv_append_paged(kn, vn, kpool2, vpool2, table2, full) & 1 and full[2] == L
    # the decode reports a block-table entry outside the pool for a row it must read, and
    # gathers that row as zeros; an entry past the length is never looked at
    out_ok, st_ok = o.decode_paged(q, kpool2, vpool2, table2, lens, 0.25, return_status=True)
    assert st_ok == 0 and np.array_equal(out_ok, base)
    bad2 = table2.copy()
    bad2[0, 1] = -1  # rows 8..15 of sequence 0 (length 39)
    out_bad, st_bad = o.decode_paged(q, kpool2, vpool2, bad2, lens, 0.25, return_status=True)
    assert st_bad & 4
    Kz, Vz = Kc.copy(), Vc.copy()
    Kz[0, P:2 * P] = 0.0
    Vz[0, P:2 * P] = 0.0
    assert np.array_equal(out_bad, o.decode(q, Kz, Vz, lens, 0.25))
    unused = table2.copy()
    unused[1, max_pages - 1] = n_pages + 7  # sequence 1 has one row: its last page is unused
    assert o.decode_paged(q, kpool2, vpool2, unused, lens, 0.25, return_status=True)[1] == 0


def pin_multi_query(o):
    """Q query tokens per sequence (speculative verification): Q = 1 is the ordinary decode;
    query j equals the ordinary decode of the cache cut to its first n - Q + 1 + j rows; and
    torch SDPA with the bottom-right-aligned causal mask agrees."""
    r = _rng(111)
    B, Q, H_q, H_kv, d, L = 3, 4, 8, 2, 16, 30
    lens = np.array([30, 4, 17], dtype=np.int32)
    q = r.standard_normal((B, Q, H_q, d))
    K = r.standard_normal((B, L, H_kv, d))
    V = r.standard_normal((B, L, H_kv, d))
    one = o.decode_multi(q[:, :1], K, V, lens, 0.3)
    assert np.array_equal(one[:, 0], o.decode(q[:, 0], K, V, lens, 0.3))
    got = o.decode_multi(q, K, V, lens, 0.3)
    for j in range(Q):
        cut = lens - Q + 1 + j
        assert np.array_equal(got[:, j], o.decode(q[:, j], K, V, cut, 0.3))
    for b in range(B):
        n = lens[b]
        qq = torch.from_numpy(np.ascontiguousarray(q[b].transpose(1, 0, 2))).unsqueeze(0)  # [1,H_q,Q,d]
        kk = torch.from_numpy(np.ascontiguousarray(K[b, :n].transpose(1, 0, 2))).unsqueeze(0)
        vv = torch.from_numpy(np.ascontiguousarray(V[b, :n].transpose(1, 0, 2))).unsqueeze(0)
        mask = torch.ones(Q, n, dtype=torch.bool).tril(diagonal=n - Q)
        ref = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=0.3, enable_gqa=True)
        assert np.max(np.abs(got[b] - ref[0].transpose(0, 1).numpy())) <= 1e-12
    _, st = o.decode_multi(q, K, V, np.array([3, 4, 5], dtype=np.int32), 0.3, return_status=True)
    assert st & 2  # fewer rows than query tokens


def _torch_e4m3_values(codes):
    """torch's float8_e4m3fn reading of uint8 codes, as float64."""
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_e4m3_encode(x):
    """torch's round-to-nearest-even float32 -> float8_e4m3fn (inputs within +-448)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_fp8_codec(o):
    """The e4m3 codec ("GQA 阅读笔记", section "复现性与工程实践", mixed precision: an FP8 KV
    cache): every code reads as torch's float8_e4m3fn does; closed-form values of the format
    (1, 448, the smallest normal and subnormal, NaN); codes round-trip; encoding agrees with
    torch's round-to-nearest-even on random values and on every midpoint between neighbouring
    codes (ties go to the even mantissa); magnitudes past 448 and infinities saturate; the
    rounding error stays within half a unit in the last place."""
    codes = np.arange(256, dtype=np.uint8)
    v = o.e4m3_values(codes)
    t = _torch_e4m3_values(codes)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    fin = ~np.isnan(v)
    assert np.array_equal(v[fin], t[fin])
    assert np.array_equal(np.signbit(v[fin]), np.signbit(t[fin]))
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and int(np.isnan(v).sum()) == 2
    assert v[0x38] == 1.0 and v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x00] == 0.0 and np.signbit(v[0x80])
    # round trip of every finite code
    finite_codes = codes[fin]
    assert np.array_equal(o.e4m3_encode(v[fin].astype(np.float32)), finite_codes)
    # midpoints between neighbouring positive codes: the even mantissa wins
    pos = v[:127]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)  # exact in float32
    enc = o.e4m3_encode(mids)
    want = np.where(np.arange(126) % 2 == 0, np.arange(126), np.arange(1, 127)).astype(np.uint8)
    assert np.array_equal(enc, want)
    assert np.array_equal(enc, _torch_e4m3_encode(mids))
    assert np.array_equal(o.e4m3_encode(-mids), want | 0x80)
    r = _rng(303)
    x = np.concatenate([r.standard_normal(20000) * 40, r.standard_normal(20000) * 0.01,
                        r.uniform(-448, 448, 20000)]).astype(np.float32)
    assert np.array_equal(o.e4m3_encode(x), _torch_e4m3_encode(x))
    # saturation
    sat = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, np.inf], dtype=np.float32)
    assert np.all(o.e4m3_encode(sat) == 0x7E) and np.all(o.e4m3_encode(-sat) == 0xFE)
    assert o.e4m3_encode(np.array([np.nan], dtype=np.float32))[0] == 0x7F
    # half-ulp bound: 2^-4 relative on normals, 2^-10 absolute below 2^-6
    y = o.e4m3_values(o.e4m3_encode(x)).astype(np.float64)
    err = np.abs(y - x.astype(np.float64))
    normal = np.abs(x) >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal].astype(np.float64)))
    assert np.all(err[~normal] <= 2.0 ** -10)


def pin_fp8_cache(o):
    """The FP8 cache with one scale per key/value head: quantising divides by the head's scale
    in float32 and rounds as torch does; dequantising multiplies back exactly; the append puts
    the quantised rows at row seq_lens[b] and refuses a full cache; the decode over codes equals
    torch's fp64 SDPA over the dequantised values (dequantised by torch)."""
    r = _rng(404)
    B, H_q, H_kv, d, L = 3, 8, 2, 32, 40
    k_scale = (r.uniform(0.5, 2.0, H_kv) / 64).astype(np.float32)
    v_scale = (r.uniform(0.5, 2.0, H_kv) / 64).astype(np.float32)
    x = r.standard_normal((5, H_kv, d)).astype(np.float32)
    codes = o.quantize(x, k_scale)
    want = _torch_e4m3_encode(np.clip(x / k_scale[None, :, None], -448, 448))
    assert np.array_equal(codes, want)
    deq = o.dequantize(codes, k_scale)
    assert np.array_equal(deq, _torch_e4m3_values(codes) * k_scale.astype(np.float64)[None, :, None])
    # append: codes of the new rows land at row seq_lens[b]
    k_codes = o.quantize(r.standard_normal((B, L, H_kv, d)).astype(np.float32), k_scale)
    v_codes = o.quantize(r.standard_normal((B, L, H_kv, d)).astype(np.float32), v_scale)
    lens = np.array([0, 17, L], dtype=np.int32)
    kn = r.standard_normal((B, H_kv, d)).astype(np.float32)
    vn = r.standard_normal((B, H_kv, d)).astype(np.float32)
    kc2, vc2, l2 = k_codes.copy(), v_codes.copy(), lens.copy()
    st = o.kv_append_fp8(kn, vn, kc2, vc2, k_scale, v_scale, l2)
    assert st == 1 and list(l2) == [1, 18, L]
    for b, t in ((0, 0), (1, 17)):
        assert np.array_equal(kc2[b, t], o.quantize(kn[b][None], k_scale)[0])
        assert np.array_equal(vc2[b, t], o.quantize(vn[b][None], v_scale)[0])
        mask = np.ones(L, dtype=bool)
        mask[t] = False
        assert np.array_equal(kc2[b, mask], k_codes[b, mask])
    assert np.array_equal(kc2[2], k_codes[2])
    # decode over codes == SDPA over torch-dequantised values
    q = r.standard_normal((B, H_q, d))
    lens = np.array([40, 1, 23], dtype=np.int32)
    Kd = _torch_e4m3_values(k_codes) * k_scale.astype(np.float64)[None, None, :, None]
    Vd = _torch_e4m3_values(v_codes) * v_scale.astype(np.float64)[None, None, :, None]
    got = o.decode_fp8(q, k_codes, v_codes, k_scale, v_scale, lens, 0.2)
    assert np.max(np.abs(got - _sdpa_reference(q, Kd, Vd, lens, 0.2))) <= 1e-12
    got_w = o.decode_fp8(q, k_codes, v_codes, k_scale, v_scale, lens, 0.2, window=7)
    assert np.array_equal(got_w, o.decode_window(q, Kd, Vd, lens, 7, 0.2))


ALL_PINS = [
    pin_append_position, pin_append_overflow, pin_expand_matches_repeat_interleave,
    pin_single_head_vs_sdpa, pin_decode_vs_sdpa_gqa, pin_mha_endpoint, pin_mqa_endpoint,
    pin_expand_then_attend_equivalence, pin_grouping_changes_output, pin_closed_forms,
    pin_invariants, pin_brute_force_tiny, pin_empty_and_range, pin_divisibility, pin_window,
    pin_paged, pin_multi_query, pin_fp8_codec, pin_fp8_cache,
]


def failing_pins(o) -> list[str]:
    """Names of the pins the oracle ``o`` fails (an exception of any kind counts as failing)."""
    bad = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except Exception:  # noqa: BLE001 - a crash is a failed pin too
            bad.append(pin.__name__)
    return bad
