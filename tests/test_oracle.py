"""Pins of the fp64 oracle against things other than itself (CPU only).

Each check targets a different plausible mistake: a dropped or misplaced RoPE
term, a wrong scale, a softmax over the wrong axis, branches mixed up, a page
and slot swapped, a missing normaliser, out_scale in the wrong place, or a
wrong up-projection index.  ``test_planted_mistakes_are_caught`` compiles
mutated copies of the oracle and shows each mutation fails a pin.
"""
import json
import math
import os
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import explicit
from tests.paging import bf16_exact, paged_from_logical

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _logical(rng, lengths, B, d_c, d_r):
    lat = [bf16_exact((L, B, d_c), rng, 1 / math.sqrt(d_c)) for L in lengths]
    rope = [bf16_exact((L, d_r), rng, 1 / math.sqrt(max(d_r, 1))) for L in lengths]
    return lat, rope


def _queries(rng, N, H, B, d_c, d_r, gain=1.0):
    q_lat = bf16_exact((N, H, B, d_c), rng, gain / math.sqrt(d_c))
    q_rope = bf16_exact((N, H, d_r), rng, gain / math.sqrt(max(d_r, 1)))
    return q_lat, q_rope


def _sdpa_reference(q_lat, q_rope, lat, rope, scale, out_scale):
    """Each (sequence, branch) is textbook multi-query attention: keys are
    [c_b ; k_r], values are c_b, the H heads are the queries.  Computed with
    torch's scaled_dot_product_attention in fp64 on the logical sequences."""
    N, H, B, d_c = q_lat.shape
    out = np.zeros((N, H, B, d_c))
    for n in range(N):
        for b in range(B):
            q = torch.from_numpy(np.concatenate([q_lat[n, :, b, :], q_rope[n]], axis=1))
            k = torch.from_numpy(np.concatenate([lat[n][:, b, :], rope[n]], axis=1))
            v = torch.from_numpy(np.ascontiguousarray(lat[n][:, b, :]))
            o = F.scaled_dot_product_attention(q[None], k[None], v[None], scale=scale)[0]
            out[n, :, b, :] = out_scale * o.numpy()
    return out


@pytest.mark.parametrize("B,d_c,d_r,P", [(4, 16, 8, 4), (1, 32, 8, 8), (2, 8, 4, 16), (3, 8, 0, 4)])
def test_matches_textbook_mqa(oracle_lib, B, d_c, d_r, P):
    rng = np.random.default_rng(1000 + B * 10 + d_c)
    N, H = 3, 4
    lengths = [1, 37, 64][:N]
    lat, rope = _logical(rng, lengths, B, d_c, d_r)
    q_lat, q_rope = _queries(rng, N, H, B, d_c, d_r, gain=8.0)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, slack_pages=3)
    scale, out_scale = 1 / math.sqrt(d_c + d_r + 1), 0.5
    out, lse, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, scale, out_scale)
    assert status == 0
    ref = _sdpa_reference(q_lat, q_rope, lat, rope, scale, out_scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-14)
    assert np.isfinite(out).all()


def test_mla_shape_matches_textbook_mqa(oracle_lib):
    """The MLA special case at the equal-bytes comparison's own shape: one
    branch of d_c = 512 plus the 64-wide RoPE key, page size 64, 16 heads,
    scale 1/sqrt(576), out_scale 1.  With B = 1 the method is MLA's absorbed
    decode, i.e. multi-query attention over keys [c ; k_r] and values c."""
    rng = np.random.default_rng(512)
    N, H, B, d_c, d_r, P = 2, 16, 1, 512, 64, 64
    lengths = [300, 129]
    lat, rope = _logical(rng, lengths, B, d_c, d_r)
    q_lat, q_rope = _queries(rng, N, H, B, d_c, d_r, gain=500.0)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, slack_pages=2)
    scale, out_scale = 1 / math.sqrt(d_c + d_r), 1.0
    # the scores are far from flat (std about 3), so the weights matter
    s0 = scale * (lat[0][:, 0, :] @ q_lat[0, 0, 0] + rope[0] @ q_rope[0, 0])
    assert s0.std() > 2.0
    out, lse, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, scale, out_scale)
    assert status == 0
    ref = _sdpa_reference(q_lat, q_rope, lat, rope, scale, out_scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-14)


def test_bruteforce_tiny(oracle_lib):
    """Enumerate every token with math.fsum and the max-free form
    p_t = 1 / sum_u exp(s_u - s_t)."""
    rng = np.random.default_rng(7)
    N, H, B, d_c, d_r, P = 1, 2, 2, 8, 4, 2
    for L in range(1, 6):
        lat, rope = _logical(rng, [L], B, d_c, d_r)
        q_lat, q_rope = _queries(rng, N, H, B, d_c, d_r, gain=4.0)
        pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, slack_pages=1)
        scale, out_scale = 0.3, 0.75
        out, _, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, scale, out_scale)
        assert status == 0
        for h in range(H):
            for b in range(B):
                s = [scale * (math.fsum(q_lat[0, h, b, k] * lat[0][t, b, k] for k in range(d_c))
                              + math.fsum(q_rope[0, h, k] * rope[0][t, k] for k in range(d_r)))
                     for t in range(L)]
                p = [1.0 / math.fsum(math.exp(s[u] - s[t]) for u in range(L)) for t in range(L)]
                for k in range(d_c):
                    want = out_scale * math.fsum(p[t] * lat[0][t, b, k] for t in range(L))
                    assert out[0, h, b, k] == pytest.approx(want, rel=1e-12, abs=1e-15)


def test_absorbed_equals_explicit(oracle_lib):
    """Absorbed decode + per-branch up-projection + branch sum equals explicit
    attention with materialised per-branch keys and values."""
    rng = np.random.default_rng(11)
    N, H, B, d_c, d_r, d_h, P = 2, 3, 4, 8, 4, 6, 4
    lengths = [9, 20]
    lat, rope = _logical(rng, lengths, B, d_c, d_r)
    q_c = rng.standard_normal((N, H, d_h))
    q_rope = rng.standard_normal((N, H, d_r)) / 2
    w_uk = rng.standard_normal((B, H, d_h, d_c)) / math.sqrt(d_h)
    w_uv = rng.standard_normal((B, d_c, H * d_h)) / math.sqrt(B * d_c)
    q_lat = explicit.absorb_queries(q_c, w_uk)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, slack_pages=2)
    scale, out_scale = 0.4, 1 / math.sqrt(B)
    out_lat, _, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, scale, out_scale)
    assert status == 0
    y = oracle_lib.up_proj(out_lat, w_uv, d_h)
    y_exp = explicit.explicit_decode(q_c, q_rope, w_uk, w_uv, lat, rope, scale, out_scale)
    np.testing.assert_allclose(y, y_exp, rtol=1e-10, atol=1e-13)


def test_length_one_returns_the_value_exactly(oracle_lib):
    rng = np.random.default_rng(3)
    N, H, B, d_c, d_r, P = 2, 4, 4, 16, 8, 8
    lat, rope = _logical(rng, [1, 1], B, d_c, d_r)
    q_lat, q_rope = _queries(rng, N, H, B, d_c, d_r, gain=50.0)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, slack_pages=4)
    out, _, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.1, 0.5)
    assert status == 0
    for n in range(N):
        for h in range(H):
            assert np.array_equal(out[n, h], 0.5 * lat[n][0])


def test_scale_zero_gives_the_mean(oracle_lib):
    rng = np.random.default_rng(4)
    B, d_c, d_r, P = 2, 8, 4, 4
    lat, rope = _logical(rng, [13, 7], B, d_c, d_r)
    q_lat, q_rope = _queries(rng, 2, 3, B, d_c, d_r, gain=100.0)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng)
    out, _, _ = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.0, 2.0)
    for n in range(2):
        np.testing.assert_allclose(out[n], np.broadcast_to(2.0 * lat[n].mean(axis=0), out[n].shape),
                                   rtol=1e-13, atol=1e-15)


def test_identical_tokens_give_that_token(oracle_lib):
    rng = np.random.default_rng(5)
    B, d_c, d_r, P, L = 3, 8, 4, 4, 11
    one_lat, one_rope = _logical(rng, [1], B, d_c, d_r)
    lat = [np.repeat(one_lat[0], L, axis=0)]
    rope = [np.repeat(one_rope[0], L, axis=0)]
    q_lat, q_rope = _queries(rng, 1, 2, B, d_c, d_r, gain=30.0)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng)
    out, _, _ = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.7, 1.0)
    np.testing.assert_allclose(out[0], np.broadcast_to(one_lat[0][0], out[0].shape), rtol=1e-14)


def test_page_permutation_gives_identical_bits(oracle_lib):
    rng = np.random.default_rng(6)
    B, d_c, d_r, P = 4, 8, 4, 4
    lat, rope = _logical(rng, [30, 5, 17], B, d_c, d_r)
    q_lat, q_rope = _queries(rng, 3, 2, B, d_c, d_r, gain=10.0)
    a = paged_from_logical(lat, rope, P, np.random.default_rng(1), slack_pages=0)
    b = paged_from_logical(lat, rope, P, np.random.default_rng(2), slack_pages=9,
                           max_pages_per_seq=12)
    out_a, lse_a, _ = oracle_lib.decode(q_lat, q_rope, *a, 0.5, 0.5)
    out_b, lse_b, _ = oracle_lib.decode(q_lat, q_rope, *b, 0.5, 0.5)
    assert np.array_equal(out_a, out_b) and np.array_equal(lse_a, lse_b)


def test_token_permutation_invariance(oracle_lib):
    rng = np.random.default_rng(8)
    B, d_c, d_r, P, L = 2, 8, 4, 4, 23
    lat, rope = _logical(rng, [L], B, d_c, d_r)
    perm = rng.permutation(L)
    q_lat, q_rope = _queries(rng, 1, 3, B, d_c, d_r, gain=10.0)
    a = paged_from_logical(lat, rope, P, rng)
    b = paged_from_logical([lat[0][perm]], [rope[0][perm]], P, rng)
    out_a, _, _ = oracle_lib.decode(q_lat, q_rope, *a, 0.5, 0.5)
    out_b, _, _ = oracle_lib.decode(q_lat, q_rope, *b, 0.5, 0.5)
    np.testing.assert_allclose(out_a, out_b, rtol=1e-12, atol=1e-15)


def test_lse_is_logsumexp_of_scores(oracle_lib):
    from scipy.special import logsumexp
    rng = np.random.default_rng(9)
    B, d_c, d_r, P = 2, 8, 4, 4
    lat, rope = _logical(rng, [19], B, d_c, d_r)
    q_lat, q_rope = _queries(rng, 1, 2, B, d_c, d_r, gain=20.0)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng)
    _, lse, _ = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.5, 1.0)
    for h in range(2):
        for b in range(B):
            keys = np.concatenate([lat[0][:, b, :], rope[0]], axis=1)
            s = 0.5 * keys @ np.concatenate([q_lat[0, h, b], q_rope[0, h]])
            assert lse[0, h, b] == pytest.approx(logsumexp(s), rel=1e-13)


def test_two_way_split_merged_by_logsumexp_equals_the_whole(oracle_lib):
    """Attention over tokens [0, L) equals the log-sum-exp weighted merge of
    the attentions over [0, L1) and [L1, L) (the split-KV identity)."""
    rng = np.random.default_rng(13)
    B, d_c, d_r, P, L, L1 = 2, 8, 4, 4, 23, 10
    lat, rope = _logical(rng, [L], B, d_c, d_r)
    lat3 = [lat[0], lat[0][:L1], lat[0][L1:]]
    rope3 = [rope[0], rope[0][:L1], rope[0][L1:]]
    q_lat, q_rope = _queries(rng, 1, 3, B, d_c, d_r, gain=8.0)
    q_lat3, q_rope3 = np.repeat(q_lat, 3, axis=0), np.repeat(q_rope, 3, axis=0)
    pool, rpool, table, seqlens = paged_from_logical(lat3, rope3, P, rng)
    out, lse, status = oracle_lib.decode(q_lat3, q_rope3, pool, rpool, table, seqlens, 0.7, 0.5)
    assert status == 0
    w1, w2 = np.exp(lse[1] - lse[0]), np.exp(lse[2] - lse[0])
    merged = w1[..., None] * out[1] + w2[..., None] * out[2]
    np.testing.assert_allclose(merged, out[0], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(np.logaddexp(lse[1], lse[2]), lse[0], rtol=1e-13)


def test_up_proj_is_the_concatenated_gemm(oracle_lib):
    """sum over branches of per-branch products == one GEMM over K = B*d_c."""
    rng = np.random.default_rng(10)
    N, H, B, d_c, d_h = 3, 2, 4, 8, 5
    out_lat = rng.standard_normal((N, H, B, d_c))
    w_uv = bf16_exact((B, d_c, H * d_h), rng)
    y = oracle_lib.up_proj(out_lat, torch.from_numpy(w_uv).to(torch.bfloat16), d_h)
    for h in range(H):
        w_cat = w_uv[:, :, h * d_h:(h + 1) * d_h].reshape(B * d_c, d_h)
        np.testing.assert_allclose(y[:, h * d_h:(h + 1) * d_h],
                                   out_lat[:, h].reshape(N, B * d_c) @ w_cat, rtol=1e-12, atol=1e-14)


def test_bf16_bits_and_float64_inputs_agree(oracle_lib):
    rng = np.random.default_rng(12)
    B, d_c, d_r, P = 2, 8, 4, 4
    lat, rope = _logical(rng, [10, 3], B, d_c, d_r)
    q_lat, q_rope = _queries(rng, 2, 2, B, d_c, d_r)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, fill=0.0)
    as_bf16 = [torch.from_numpy(x).to(torch.bfloat16) for x in (q_lat, q_rope, pool, rpool)]
    a, _, _ = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.5, 0.5)
    b, _, _ = oracle_lib.decode(*as_bf16, table, seqlens, 0.5, 0.5)
    assert np.array_equal(a, b)


def test_invalid_sequences_are_zeroed_and_reported(oracle_lib):
    rng = np.random.default_rng(13)
    B, d_c, d_r, P = 2, 8, 4, 4
    lat, rope = _logical(rng, [5, 6, 7], B, d_c, d_r)
    q_lat, q_rope = _queries(rng, 3, 2, B, d_c, d_r)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, fill=0.0)
    good, _, _ = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.5, 0.5)
    bad_len = seqlens.copy()
    bad_len[1] = 0
    out, lse, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, bad_len, 0.5, 0.5)
    assert status == 6 and (out[1] == 0).all() and np.isneginf(lse[1]).all()
    assert np.array_equal(out[0], good[0]) and np.array_equal(out[2], good[2])
    too_long = seqlens.copy()
    too_long[2] = table.shape[1] * P + 1
    assert oracle_lib.decode(q_lat, q_rope, pool, rpool, table, too_long, 0.5, 0.5)[2] == 6
    bad_page = table.copy()
    bad_page[0, 1] = pool.shape[0]
    out, _, status = oracle_lib.decode(q_lat, q_rope, pool, rpool, bad_page, seqlens, 0.5, 0.5)
    assert status == 5 and (out[0] == 0).all() and np.array_equal(out[1], good[1])


def test_page_byte_model_matches_the_pages():
    """Per-device KV elements per token under 4-way TP: 1.5*d_h for MLRA-4 and
    4.5*d_h for MLA (the blog's "Core Insight" section), reproduced by the
    byte accounting of the one-branch shard and the MLA workloads."""
    from branch_latent_kv_b200.inputs import WORKLOADS
    g = json.load(open(os.path.join(GOLDEN, "byte_model.json")))
    d_h = g["d_h"]
    shard, mla, mlra4 = WORKLOADS["tp_shard"], WORKLOADS["mla_equal_bytes"], WORKLOADS["mlra4_equal_bytes"]
    assert shard.branches * shard.d_c + shard.d_r == g["mlra4_elements_per_token_per_device_over_d_h"] * d_h
    assert mla.branches * mla.d_c + mla.d_r == g["mla_elements_per_token_per_device_over_d_h"] * d_h
    # MLRA-4 on one device holds the four shards' latents plus one RoPE key: the same bytes as MLA.
    assert mlra4.branches * mlra4.d_c + mlra4.d_r == mla.branches * mla.d_c + mla.d_r
    assert mlra4.d_c == shard.d_c and mlra4.branches == g["tensor_parallel"]


MUTANTS = {
    "drop_rope": ("dot += load(q_rope, qr_off + k, input_kind) * load(rope_cache, r_off + k, input_kind);",
                  "dot += 0.0 * load(q_rope, qr_off + k, input_kind);"),
    "slot_page_swap": ("pool_row[t] = page * page_size + t % page_size;",
                       "pool_row[t] = page * page_size + (t / page_size) % page_size;"),
    "wrong_branch_latent": ("const int64_t c_off = pool_row[t] * row + b * d_c;\n                const int64_t r_off",
                            "const int64_t c_off = pool_row[t] * row;\n                const int64_t r_off"),
    "no_normaliser": ("const double p = exp(s[t] - m) / denom;", "const double p = exp(s[t] - m);"),
    "scale_outside_exp": ("s[t] = scale * dot;", "s[t] = dot;"),
    "out_scale_dropped": ("out[q_off + k] = out_scale * acc[k];", "out[q_off + k] = acc[k];"),
    "up_proj_transposed": ("load(w_uv, (b * d_c + k) * width + h * d_h + j, input_kind);",
                           "load(w_uv, (b * d_c + k) * width + j * heads + h, input_kind);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(tmp_path, name):
    """Compile a mutated oracle and show that the pins above reject it."""
    from oracle import oracle as orc
    src = open(orc._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mut_src = tmp_path / "mut.c"
    mut_src.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", str(mut_src), "-o", str(so), "-lm"],
                   check=True)
    lib = orc.open_library(str(so))

    class mut:
        decode = staticmethod(lambda *a, **k: orc.decode(*a, lib=lib, **k))
        up_proj = staticmethod(lambda *a, **k: orc.up_proj(*a, lib=lib, **k))

    pins = [lambda: test_matches_textbook_mqa(mut, 4, 16, 8, 4),
            lambda: test_absorbed_equals_explicit(mut),
            lambda: test_up_proj_is_the_concatenated_gemm(mut)]
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"mutant {name} passed every pin"


def test_up_proj_bf16_and_float64_inputs_agree(oracle_lib):
    rng = np.random.default_rng(14)
    out_lat = torch.from_numpy(bf16_exact((3, 2, 4, 8), rng)).to(torch.bfloat16)
    w_uv = torch.from_numpy(bf16_exact((4, 8, 2 * 5), rng)).to(torch.bfloat16)
    assert np.array_equal(oracle_lib.up_proj(out_lat, w_uv, 5), oracle_lib.up_proj(out_lat.double(), w_uv, 5))


# ---------------------------------------------------------------- output gate
def test_gate_special_values(oracle_lib):
    """The sigmoid gate: a zero logit halves the output exactly, a large
    positive logit passes it, a large negative one closes it (the page reads
    the gate as a non-linearity on the attention output)."""
    y = np.array([[1.5, -2.0, 0.25, 3.0]])
    half = oracle_lib.gate(y, torch.zeros(1, 4, dtype=torch.bfloat16))
    assert np.array_equal(half, y / 2)
    open_ = oracle_lib.gate(y, torch.full((1, 4), 80.0, dtype=torch.bfloat16))
    assert np.allclose(open_, y, rtol=1e-15, atol=0)
    shut = oracle_lib.gate(y, torch.full((1, 4), -80.0, dtype=torch.bfloat16))
    assert np.all(np.abs(shut) <= np.abs(y) * 1e-34)


def test_gate_is_a_logistic_split(oracle_lib):
    """sigmoid(g) + sigmoid(-g) = 1: the gated outputs under g and -g add up
    to the ungated output, and each lies between 0 and the output."""
    rng = np.random.default_rng(21)
    y = rng.normal(size=(6, 40))
    g = torch.from_numpy(bf16_exact((6, 40), rng) * 4).to(torch.bfloat16)
    a, b_ = oracle_lib.gate(y, g), oracle_lib.gate(y, -g)
    assert np.allclose(a + b_, y, rtol=1e-14, atol=1e-15)
    assert np.all(np.abs(a) <= np.abs(y)) and np.all(a * y >= 0)
    assert np.array_equal(oracle_lib.gate(y, g), oracle_lib.gate(y, g.double()))


GATE_MUTANTS = {
    "gate_sign": ("y[i] = y[i] / (1.0 + exp(-load(gate, i, input_kind)));",
                  "y[i] = y[i] / (1.0 + exp(load(gate, i, input_kind)));"),
    "gate_no_one": ("y[i] = y[i] / (1.0 + exp(-load(gate, i, input_kind)));",
                    "y[i] = y[i] / exp(-load(gate, i, input_kind));"),
    "gate_multiplies": ("y[i] = y[i] / (1.0 + exp(-load(gate, i, input_kind)));",
                        "y[i] = y[i] * (1.0 + exp(-load(gate, i, input_kind)));"),
}


@pytest.mark.parametrize("name", sorted(GATE_MUTANTS))
def test_planted_gate_mistakes_are_caught(tmp_path, name):
    from oracle import oracle as orc
    src = open(orc._SRC).read()
    old, new = GATE_MUTANTS[name]
    assert src.count(old) == 1, name
    mut_src = tmp_path / "mut.c"
    mut_src.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", str(mut_src), "-o", str(so), "-lm"],
                   check=True)
    lib = orc.open_library(str(so))

    class mut:
        gate = staticmethod(lambda *a, **k: orc.gate(*a, lib=lib, **k))

    caught = 0
    for pin in (test_gate_special_values, test_gate_is_a_logistic_split):
        try:
            pin(mut)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"mutant {name} passed every pin"


# ---------------------------------------------------------------- decode pre-step
def _prepare_inputs(rng, N=3, H=2, B=2, d_c=8, d_h=6, d_r=4):
    q_c = bf16_exact((N, H, d_h), rng)
    q_r = bf16_exact((N, H, d_r), rng)
    w_uk = bf16_exact((B, H, d_h, d_c), rng)
    kr = bf16_exact((N, d_r), rng)
    return q_c, q_r, w_uk, kr


def test_prepare_absorbed_scores_equal_explicit_keys(oracle_lib):
    """q_lat . c equals q_c . (W_UK c) for any latent c: the absorbed query
    scores a latent exactly as the explicit key would."""
    rng = np.random.default_rng(31)
    q_c, q_r, w_uk, kr = _prepare_inputs(rng)
    N, H, d_h = q_c.shape
    B, d_c = w_uk.shape[0], w_uk.shape[3]
    table = np.arange(N * 2, dtype=np.int32).reshape(N, 2)
    q_lat, _, _, _, st = oracle_lib.prepare(q_c, q_r, w_uk, kr, np.array([5, 1, 8], np.int32), table,
                                            N * 2, 4)
    assert st == 0
    c = rng.standard_normal((B, d_c))
    for n in range(N):
        for h in range(H):
            for b in range(B):
                key = w_uk[b, h] @ c[b]  # [d_h]
                assert abs(q_lat[n, h, b] @ c[b] - q_c[n, h] @ key) <= 1e-12 * (1 + abs(q_c[n, h] @ key))


def test_prepare_feeds_decode_like_explicit_attention(oracle_lib):
    """prepare -> decode -> up-projection equals explicit attention with
    materialised keys (W_UK c) and values (W_UV c), the query's RoPE part
    rotated at the new token's position."""
    rng = np.random.default_rng(32)
    N, H, B, d_c, d_r, d_h, P = 2, 3, 2, 8, 4, 6, 4
    lengths = [7, 13]
    lat, rope = _logical(rng, lengths, B, d_c, d_r)
    q_c, q_r, w_uk, kr = _prepare_inputs(rng, N, H, B, d_c, d_h, d_r)
    w_uv = rng.standard_normal((B, d_c, H * d_h)) / math.sqrt(B * d_c)
    pool, rpool, table, seqlens = paged_from_logical(lat, rope, P, rng, slack_pages=2)
    q_lat, q_rope, _, _, st = oracle_lib.prepare(q_c, q_r, w_uk, kr, seqlens, table, pool.shape[0], P)
    assert st == 0
    out_lat, _, st = oracle_lib.decode(q_lat, q_rope, pool, rpool, table, seqlens, 0.3, 0.7)
    assert st == 0
    y = oracle_lib.up_proj(out_lat, w_uv, d_h)
    y_exp = explicit.explicit_decode(q_c, q_rope, np.asarray(w_uk), w_uv, lat, rope, 0.3, 0.7)
    np.testing.assert_allclose(y, y_exp, rtol=1e-10, atol=1e-13)


def test_prepare_rope_closed_forms(oracle_lib):
    """RoFormer's rotation: position 0 is the identity; with d_r = 4 and base
    10000, pair 0 turns by p radians and pair 1 by p / 100."""
    e = np.zeros((1, 1, 4))
    e[0, 0] = [1.0, 0.0, 0.0, 1.0]
    k = np.array([[0.0, 1.0, 1.0, 0.0]])
    w = np.zeros((1, 1, 1, 2))
    q_c = np.zeros((1, 1, 1))
    table = np.zeros((1, 4), np.int32)
    for p in (0, 1, 100):
        _, q_rope, kr_rot, dest, st = oracle_lib.prepare(q_c, e, w, k, np.array([p + 1], np.int32),
                                                         table, 1, 64)
        assert st == 0 and tuple(dest[0]) == (0, p % 64)
        a0, a1 = float(p), p / 100.0
        np.testing.assert_allclose(q_rope[0, 0], [math.cos(a0), math.sin(a0), -math.sin(a1), math.cos(a1)],
                                   rtol=0, atol=1e-15)
        np.testing.assert_allclose(kr_rot[0], [-math.sin(a0), math.cos(a0), math.cos(a1), math.sin(a1)],
                                   rtol=0, atol=1e-15)


def test_prepare_rotation_keeps_dot_products_and_norms(oracle_lib):
    """Query and key rotated at the same position keep their dot product
    (RoPE scores depend only on the relative position) and each pair keeps
    its length."""
    rng = np.random.default_rng(33)
    q_c, q_r, w_uk, kr = _prepare_inputs(rng, N=3, H=2, d_r=8)
    table = np.arange(3 * 300, dtype=np.int32).reshape(3, 300)
    seqlens = np.array([1, 77, 19000], np.int32)
    _, q_rope, kr_rot, _, st = oracle_lib.prepare(q_c, q_r, w_uk, kr, seqlens, table, 900, 64)
    assert st == 0
    for n in range(3):
        for h in range(2):
            assert abs(q_rope[n, h] @ kr_rot[n] - q_r[n, h] @ kr[n]) <= 1e-12
            np.testing.assert_allclose(np.hypot(q_rope[n, h, 0::2], q_rope[n, h, 1::2]),
                                       np.hypot(q_r[n, h, 0::2], q_r[n, h, 1::2]), rtol=1e-13)
    np.testing.assert_array_equal(q_rope[0], q_r[0])  # position 0


def test_prepare_append_target_and_errors(oracle_lib):
    rng = np.random.default_rng(34)
    q_c, q_r, w_uk, kr = _prepare_inputs(rng, N=4)
    table = np.array([[7, 2, -1], [4, 9, 3], [0, -1, -1], [5, 6, 8]], np.int32)
    seqlens = np.array([20, 33, 0, 100], np.int32)  # P = 16: slots 3 and 0 of pages 2, 3; bad; too long
    _, _, _, dest, st = oracle_lib.prepare(q_c, q_r, w_uk, kr, seqlens, table, 10, 16)
    assert tuple(dest[0]) == (2, 3) and tuple(dest[1]) == (3, 0)
    assert tuple(dest[2]) == (-1, -1) and tuple(dest[3]) == (-1, -1)
    assert st == 6  # the first problem: a bad length
    seqlens = np.array([20, 33, 5, 10], np.int32)
    table[3, 0] = 10  # outside the pool
    _, _, _, dest, st = oracle_lib.prepare(q_c, q_r, w_uk, kr, seqlens, table, 10, 16)
    assert st == 5 and tuple(dest[3]) == (-1, -1) and tuple(dest[2]) == (0, 4)


PREPARE_MUTANTS = {
    "rope_sin_sign": ("q_rope[o + 1] = x0 * sn + x1 * c;", "q_rope[o + 1] = -x0 * sn + x1 * c;"),
    "rope_theta": ("pow(rope_base, -2.0 * (double)i / (double)d_r)", "pow(rope_base, -1.0 * (double)i / (double)d_r)"),
    "rope_position": ("const int64_t p = (int64_t)seqlens[n] - 1;", "const int64_t p = (int64_t)seqlens[n];"),
    "absorb_transposed": ("sum += load(w_uk, ((b * heads + h) * d_h + j) * d_c + k, input_kind) *",
                          "sum += load(w_uk, ((b * heads + h) * d_c + k) * d_h + j, input_kind) *"),
}


@pytest.mark.parametrize("name", sorted(PREPARE_MUTANTS))
def test_planted_prepare_mistakes_are_caught(tmp_path, name):
    from oracle import oracle as orc
    src = open(orc._SRC).read()
    old, new = PREPARE_MUTANTS[name]
    assert src.count(old) == 1, name
    mut_src = tmp_path / "mut.c"
    mut_src.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", str(mut_src), "-o", str(so), "-lm"],
                   check=True)
    lib = orc.open_library(str(so))

    class mut:
        prepare = staticmethod(lambda *a, **k: orc.prepare(*a, lib=lib, **k))
        decode = staticmethod(lambda *a, **k: orc.decode(*a, lib=lib, **k))
        up_proj = staticmethod(lambda *a, **k: orc.up_proj(*a, lib=lib, **k))

    caught = 0
    for pin in (test_prepare_absorbed_scores_equal_explicit_keys, test_prepare_feeds_decode_like_explicit_attention,
                test_prepare_rope_closed_forms, test_prepare_rotation_keeps_dot_products_and_norms,
                test_prepare_append_target_and_errors):
        try:
            pin(mut)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"mutant {name} passed every pin"
