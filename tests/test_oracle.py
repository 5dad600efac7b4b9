"""Pins for the oracle: the pages' printed numbers, identities, closed forms,
brute force on tiny inputs and library routines.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- arithmetic

def test_token_arithmetic_matches_pages():
    g = _gold("pages_arithmetic.json")
    b, c = g["block"], g["context"]
    tc = oracle.token_counts(b["B_f"], b["h"], b["w"], c["N_sink"], c["N_recent"], c["N_top"])
    assert tc["n"] == b["n"] == 6240
    assert tc["n_c"] == g["compressed"]["n_c"] == 182
    assert tc["context"] == c["tokens"] == 27872
    lg = g["latent_grid"]
    assert lg["H"] == 2 * b["h"] and lg["W"] == 2 * b["w"]
    assert oracle.compressed_tokens_latent(lg["T"], lg["H"], lg["W"]) == 182


def test_full_context_memory_matches_pages():
    g = _gold("pages_arithmetic.json")
    fc = g["full_context"]
    tokens = oracle.dense_context_tokens(120, g["block"]["n"])
    assert tokens == 748800
    assert round(tokens / 1000) == fc["tokens_approx"] // 1000
    gb = oracle.kv_bytes(tokens, fc["hidden"], fc["layers"]) / 1e9
    assert round(gb) == fc["kv_gb_approx"]
    # two sink blocks are under 2% of that budget
    assert 2 * g["block"]["n"] / tokens < g["sink_share_max"]["value"]


def test_workload_literals_follow_the_formulas():
    # synth writes n and n_c as literals; the formulas must reproduce them.
    for wl in synth.WORKLOADS.values():
        tc = oracle.token_counts(wl.block_frames, wl.h, wl.w, 0, 0, 0)
        assert tc["n"] == wl.n, wl.name
        assert tc["n_c"] == wl.n_c, wl.name
    # the tiny workload: floor(4/2) floor(6/4) floor(8/4) = 2 * 1 * 2 = 4
    assert oracle.token_counts(4, 6, 8, 8, 4, 3)["n_c"] == 4
    assert oracle.token_counts(4, 6, 8, 8, 4, 3)["context"] == 2 * 192 + 3 * 4 + 2 * 192


@pytest.mark.parametrize("delta_blocks", [0, 1, 3, 17])
def test_cache_partitions_eviction_gap(delta_blocks):
    # After evicting D blocks the earliest surviving mid block starts at
    # frame N_sink + delta, delta = D * B_f ("The Position Misalignment Problem").
    B_f, sink, recent, cap = 4, 2, 1, 40
    nblk = sink + cap + recent + delta_blocks
    p = oracle.cache_partitions(nblk, sink, recent, cap)
    assert p["sink"] == [0, 1]
    assert p["evicted"] == delta_blocks
    assert len(p["mid"]) == cap and p["recent"] == [nblk - 1]
    assert p["mid"][0] * B_f == sink * B_f + delta_blocks * B_f
    assert p["mid"] == list(range(sink + delta_blocks, nblk - recent))


def test_cache_partitions_early_blocks():
    assert oracle.cache_partitions(1, 2, 1, 5) == {"sink": [0], "mid": [], "recent": [], "evicted": 0}
    assert oracle.cache_partitions(3, 2, 1, 5) == {"sink": [0, 1], "mid": [], "recent": [2], "evicted": 0}
    assert oracle.cache_partitions(5, 2, 2, 5)["mid"] == [2]
    assert oracle.cache_partitions(4, 2, 2, 5)["mid"] == []
    assert oracle.cache_partitions(6, 2, 2, 0) == {"sink": [0, 1], "mid": [], "recent": [4, 5], "evicted": 2}


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_float32_inputs():
    x = torch.randn(20000, generator=torch.Generator().manual_seed(3)) * 7
    x = torch.cat([x, torch.tensor([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, 3.0])])
    want = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.to(torch.float64).numpy())
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- RoPE

def _keys(shape, seed):
    return torch.randn(*shape, generator=torch.Generator().manual_seed(seed), dtype=torch.float64).numpy()


def test_rope_shift_equals_encode_at_shifted_position():
    # e^{i theta p} e^{i theta delta} = e^{i theta (p + delta)} ("Incremental RoPE adjustment")
    k = _keys((64, 3, 128), 1)
    t = np.arange(64)[:, None] % 8
    y = np.arange(64)[:, None] // 8 + np.zeros((1, 3))
    x = (np.arange(64)[:, None] * 7) % 13 + np.zeros((1, 3))
    for delta in (1, 4, 37, 480):
        shifted = oracle.rope_shift(oracle.rope_encode(k, t, y, x), delta)
        fresh = oracle.rope_encode(k, t + delta, y, x)
        assert np.max(np.abs(shifted - fresh)) < 1e-11


def test_rope_shift_composition_identity_and_norms():
    k = _keys((32, 2, 128), 2)
    a = oracle.rope_shift(oracle.rope_shift(k, 5), 11)
    b = oracle.rope_shift(k, 16)
    assert np.max(np.abs(a - b)) < 1e-12
    assert np.array_equal(oracle.rope_shift(k, 0), k)
    s = oracle.rope_shift(k, 9)
    n0 = k[..., 0:44:2] ** 2 + k[..., 1:44:2] ** 2
    n1 = s[..., 0:44:2] ** 2 + s[..., 1:44:2] ** 2
    assert np.max(np.abs(n0 - n1)) < 1e-12
    # height and width components are untouched bit for bit
    assert np.array_equal(s[..., 44:], k[..., 44:])
    assert not np.allclose(s[..., :44], k[..., :44])


def test_rope_spatial_positions_unchanged_by_shift():
    k = _keys((16, 128), 3)
    y, x = np.arange(16) % 4, np.arange(16) // 4
    a = oracle.rope_shift(oracle.rope_encode(k, 2, y, x), 6)
    b = oracle.rope_encode(k, 8, y, x)
    assert np.max(np.abs(a[:, 44:] - b[:, 44:])) < 1e-12
    assert np.array_equal(a[:, 44:], oracle.rope_encode(k, 2, y, x)[:, 44:])


def test_rope_matches_complex_exponential():
    # The pairs are complex numbers re + i im multiplied by numpy's exp(1j * phi).
    k = _keys((10, 128), 4)
    th_t, th_h, th_w = oracle.rope_thetas()
    delta = 13
    z = k[:, 0:44:2] + 1j * k[:, 1:44:2]
    z = z * np.exp(1j * th_t * delta)
    s = oracle.rope_shift(k, delta)
    assert np.max(np.abs(s[:, 0:44:2] - z.real)) < 1e-12
    assert np.max(np.abs(s[:, 1:44:2] - z.imag)) < 1e-12


def test_rope_frequency_closed_forms():
    th_t, th_h, th_w = oracle.rope_thetas()
    assert len(th_t) == 22 and len(th_h) == 21 and len(th_w) == 21
    assert th_t[0] == 1.0 and abs(th_t[11] - 0.01) < 1e-15      # 10000^(-22/44)
    assert abs(th_h[0] - 1.0) < 1e-15 and abs(th_h[7] - 10000 ** (-14 / 42)) < 1e-15
    # a unit vector in pair 0 rotated by delta radians
    k = np.zeros(128)
    k[0] = 1.0
    s = oracle.rope_shift(k, 2)
    assert abs(s[0] - math.cos(2)) < 1e-15 and abs(s[1] - math.sin(2)) < 1e-15


# ---------------------------------------------------------------- selection

def _tiny(seed=1000):
    return synth.make_layer(synth.WORKLOADS["tiny"], seed)


def test_factored_scores_equal_bruteforce_double_sum():
    wl = synth.WORKLOADS["ragged_a"]
    d = synth.make_layer(wl.replace(pool_blocks=5, planted=2), 7)
    a = oracle.select_scores(d["Q"], d["mid_K"])
    b = oracle.select_scores_bruteforce(d["Q"], d["mid_K"])
    assert np.max(np.abs(a - b) / np.max(np.abs(b))) < 1e-10


def test_planted_blocks_recovered_tiny():
    seeds = _gold("seeds.json")
    d = _tiny(seeds["tiny"])
    S = oracle.select_scores(d["Q"], d["mid_K"])
    sel = oracle.select_topk(S, 3)
    assert np.array_equal(sel, d["planted"].numpy())
    assert oracle.selection_margin(S, 3)[0] >= 1e-3


@pytest.mark.parametrize("name", ["tiny", "ragged_a", "ragged_b", "ragged_c", "layer", "step30"])
def test_stored_seeds_plant_the_oracle_top_k(name):
    # the seed fixture still holds for the generator and the oracle as they are:
    # planted blocks = the oracle's top-k in every batch item, at the stored margin
    seeds = _gold("seeds.json")
    wl = synth.WORKLOADS[name]
    d = synth.make_layer(wl, seeds[name], with_values=False)
    S = oracle.select_scores(d["Q"], d["mid_K"])
    assert np.array_equal(oracle.select_topk(S, wl.n_top), d["planted"].numpy())
    margin = oracle.selection_margin(S, wl.n_top)
    assert np.all(margin >= 1e-3)
    assert round(float(margin.min()), 4) == seeds["_margins"][name]


def test_selection_permutation_equivariance():
    d = _tiny()
    S = oracle.select_scores(d["Q"], d["mid_K"])
    perm = np.array([5, 2, 7, 0, 1, 6, 3, 4])
    Sp = oracle.select_scores(d["Q"], d["mid_K"][:, perm])
    assert np.allclose(Sp, S[:, perm], rtol=0, atol=1e-15)
    sel = set(oracle.select_topk(S, 3)[0].tolist())
    selp = set(perm[oracle.select_topk(Sp, 3)[0]].tolist())
    assert sel == selp


def test_selection_small_pool_and_ties():
    S = np.array([[0.3, 0.1]])
    assert oracle.select_topk(S, 16).tolist() == [[0, 1]]
    assert oracle.select_topk(np.zeros((2, 9)), 4).tolist() == [[0, 1, 2, 3]] * 2
    S = np.array([[1.0, 5.0, 5.0, 2.0, 5.0, 0.0]])
    assert oracle.select_topk(S, 2).tolist() == [[1, 2]]
    assert oracle.select_topk(S, 4).tolist() == [[1, 2, 3, 4]]
    # values equal in float32 but not in float64 tie, and go to the lower index
    S = np.array([[1.0 + 1e-12, 1.0, 0.5]])
    assert oracle.select_topk(S[:, ::-1].copy(), 1).tolist() == [[1]]
    assert oracle.selection_margin(np.array([[3.0, 1.0, 2.0]]), 1)[0] == pytest.approx(1 / 3)


def test_subsampled_half_head_scores_equal_bruteforce_on_the_slices():
    # the selection's speed variant (digest, limitations paragraph): every
    # q_stride-th query and a head range; pinned by the token-level double
    # sum over exactly those queries and heads
    wl = synth.WORKLOADS["ragged_c"]
    d = synth.make_layer(wl.replace(pool_blocks=5, planted=2), 11)
    a = oracle.select_scores(d["Q"], d["mid_K"], q_stride=3, heads=(1, 3))
    b = oracle.select_scores_bruteforce(d["Q"][:, ::3, 1:3], d["mid_K"][:, :, :, 1:3])
    assert np.max(np.abs(a - b) / np.max(np.abs(b))) < 1e-10
    # one head, stride larger than the block: only query row 0
    c = oracle.select_scores(d["Q"], d["mid_K"], q_stride=10_000, heads=(2, 3))
    e = oracle.select_scores_bruteforce(d["Q"][:, :1, 2:3], d["mid_K"][:, :, :, 2:3])
    assert np.max(np.abs(c - e) / np.max(np.abs(e))) < 1e-10


def test_head_shard_scores_add_up_to_the_full_score():
    # disjoint head ranges divided by the total head count sum to the score
    wl = synth.WORKLOADS["ragged_c"]
    d = synth.make_layer(wl.replace(pool_blocks=6, planted=2), 12)
    H = d["Q"].shape[2]
    full = oracle.select_scores(d["Q"], d["mid_K"])
    parts = sum(oracle.select_scores(d["Q"], d["mid_K"], heads=(lo, lo + 1), heads_norm=H) for lo in range(H))
    assert np.max(np.abs(parts - full)) < 1e-14 * max(1.0, np.max(np.abs(full))) * 10
    assert np.array_equal(oracle.select_topk(parts, 2), oracle.select_topk(full, 2))


def test_fifo_routing_is_top_k_of_age():
    # FIFO keeps the newest blocks: the same as ranking by age
    for count, k in [(40, 16), (5, 16), (16, 16), (1, 1), (7, 0)]:
        f = oracle.select_fifo(count, k)
        assert f.tolist() == (oracle.select_topk(np.arange(count, dtype=np.float64)[None], k)[0].tolist()
                              if k else [])
        assert len(f) == min(k, count)


# ---------------------------------------------------------------- attention

def _rand(shape, seed):
    return torch.randn(*shape, generator=torch.Generator().manual_seed(seed), dtype=torch.float64)


def test_attend_equals_loop_bruteforce():
    Q, K, V = _rand((1, 5, 1, 128), 1), _rand((1, 23, 1, 128), 2), _rand((1, 23, 1, 128), 3)
    O, lse = oracle.attend(Q, [(K[:, :7], V[:, :7]), (K[:, 7:], V[:, 7:])])
    O2, lse2 = oracle.attend_loops(Q[0, :, 0], K[0, :, 0], V[0, :, 0])
    assert np.max(np.abs(O[0, :, 0] - O2)) < 1e-12
    assert np.max(np.abs(lse[0, 0] - lse2)) < 1e-12


def test_attend_matches_torch_sdpa_float64():
    Q, K, V = _rand((2, 37, 3, 128), 4), _rand((2, 301, 3, 128), 5), _rand((2, 301, 3, 128), 6)
    parts = [(K[:, :100], V[:, :100]), (K[:, 100:101], V[:, 100:101]), (K[:, 101:], V[:, 101:])]
    O, _ = oracle.attend(Q, parts, chunk=16)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.transpose(1, 2), K.transpose(1, 2), V.transpose(1, 2)).transpose(1, 2)
    assert np.max(np.abs(O - ref.numpy())) < 1e-12


def test_attend_partition_merge_by_lse():
    Q, K, V = _rand((1, 9, 2, 128), 7), _rand((1, 60, 2, 128), 8), _rand((1, 60, 2, 128), 9)
    whole, lw = oracle.attend(Q, [(K, V)])
    o1, l1 = oracle.attend(Q, [(K[:, :13], V[:, :13])])
    o2, l2 = oracle.attend(Q, [(K[:, 13:], V[:, 13:])])
    m, lm = oracle.merge_partials([o1, o2], [l1, l2])
    assert np.max(np.abs(m - whole)) < 1e-12 and np.max(np.abs(lm - lw)) < 1e-12
    # order of the partitions does not matter
    o3, _ = oracle.attend(Q, [(K[:, 13:], V[:, 13:]), (K[:, :13], V[:, :13])])
    assert np.max(np.abs(o3 - whole)) < 1e-12


def test_attend_closed_forms():
    Q, V = _rand((1, 4, 1, 128), 10), _rand((1, 50, 1, 128), 11)
    K = _rand((1, 50, 1, 128), 12)
    # one key: O = V
    O, lse = oracle.attend(Q, [(K[:, :1], V[:, :1])])
    assert np.max(np.abs(O - V[:, :1].numpy())) < 1e-14
    # identical value rows: O = that row
    Vc = V[:, :1].expand(1, 50, 1, 128)
    O, _ = oracle.attend(Q, [(K, Vc)])
    assert np.max(np.abs(O - V[:, :1].numpy())) < 1e-12
    # zero queries: O = mean of V, lse = log(Lk)
    O, lse = oracle.attend(torch.zeros(1, 4, 1, 128, dtype=torch.float64), [(K, V)])
    assert np.max(np.abs(O - V.numpy().mean(axis=1, keepdims=True))) < 1e-12
    assert np.max(np.abs(lse - math.log(50))) < 1e-12


def test_attend_without_mid_blocks_is_sink_recent_current():
    d = _tiny()
    parts_no_mid = [(d["sink_K"][:, 0], d["sink_V"][:, 0]), (d["sink_K"][:, 1], d["sink_V"][:, 1]),
                    (d["mid_K"][:, :0, 0], d["mid_V"][:, :0, 0]),
                    (d["recent_K"][:, 0], d["recent_V"][:, 0]), (d["K_cur"], d["V_cur"])]
    O, _ = oracle.attend(d["Q"], parts_no_mid)
    K = torch.cat([d["sink_K"][:, 0], d["sink_K"][:, 1], d["recent_K"][:, 0], d["K_cur"]], 1)
    V = torch.cat([d["sink_V"][:, 0], d["sink_V"][:, 1], d["recent_V"][:, 0], d["V_cur"]], 1)
    O2, _ = oracle.attend(d["Q"], [(K, V)])
    assert np.max(np.abs(O - O2)) < 1e-12
