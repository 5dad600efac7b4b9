"""GPU path vs the oracle, element by element, through the C ABI.

Sizes: the small workloads are compared in full; the pages-scale ones on
sampled query rows (first, last, ragged tail and random rows) at the shapes
bench.py times.  Tolerances: selection bit-exact (inputs have a relative
score margin >= 1e-3), attention max-abs 2e-2 and relative L2 5e-3, shifted
keys 1e-2 (or one bf16 ulp) after rounding the oracle to bf16."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _harness import (LSE_MAX_ABS, arena_view, assert_attention_close, assert_keys_close, build_cache,
                      oracle_context, seed_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pf():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from packed_kv_cache_b200 import build
    build.build()
    import packed_kv_cache_b200 as mod
    return mod


def _wl(name):
    return synth.WORKLOADS[name]


def _layer(name, device="cpu", with_values=True):
    wl = _wl(name)
    return wl, synth.make_layer(wl, seed_for(name), device=device, with_values=with_values)


def _rows(n, k=48, seed=0):
    g = np.random.default_rng(seed)
    r = set([0, 1, 127, 128, 255, 256, n - 1, n - 2, n - 97, n - 96]) | set(g.integers(0, n, k).tolist())
    return np.array(sorted(x for x in r if 0 <= x < n))


# ------------------------------------------------------------------ RoPE shift

@pytest.mark.parametrize("name", ["tiny", "ragged_a", "ragged_b", "layer"])
def test_rope_shift_sink_matches_oracle(pf, name):
    wl, d = _layer(name)
    cache = build_cache(pf, wl, d)
    info = cache.info(0)
    B, S, n, H, D = wl.batch, wl.sink_blocks, wl.n, wl.heads, wl.head_dim
    cache.rope_shift(0, pf.PART_SINK, d["delta"])
    torch.cuda.synchronize()
    got = arena_view(cache, info["sink_k"], (B, S * n, H, D)).cpu()
    before = d["sink_K"].reshape(B, S * n, H, D)
    ref = oracle.rope_shift(before, d["delta"])
    assert_keys_close(got, ref, name)
    assert torch.equal(got[..., 44:], before[..., 44:])
    sv = arena_view(cache, info["sink_v"], (B, S * n, H, D)).cpu()
    assert torch.equal(sv, d["sink_V"].reshape(B, S * n, H, D))
    assert cache.info(0)["total_shift"] == d["delta"]


def test_rope_shift_all_partitions_and_composition(pf):
    wl, d = _layer("ragged_b")
    cache = build_cache(pf, wl, d)
    info = cache.info(0)
    B, n, nc, H, D = wl.batch, wl.n, wl.n_c, wl.heads, wl.head_dim
    parts = pf.PART_SINK | pf.PART_MID | pf.PART_RECENT
    cache.rope_shift(0, parts, 7)
    cache.rope_shift(0, parts, -3)
    torch.cuda.synchronize()
    slots = info["pool_slots"]
    pool = arena_view(cache, info["pool_k"], (B, slots, nc, H, D)).cpu()
    live = torch.stack([pool[:, (info["mid_head"] + p) % slots] for p in range(info["mid_count"])], 1)
    # two shifts compose to one of 4 (each rounded to bf16 in between)
    ref_mid = oracle.rope_shift(oracle.round_bf16(oracle.rope_shift(d["mid_K"], 7)), -3)
    assert_keys_close(live, ref_mid, "mid")
    rec = arena_view(cache, info["recent_k"], (B, wl.recent_blocks, n, H, D)).cpu()
    rec = torch.stack([rec[:, (info["recent_head"] + r) % wl.recent_blocks] for r in range(info["recent_count"])], 1)
    ref_rec = oracle.rope_shift(oracle.round_bf16(oracle.rope_shift(d["recent_K"], 7)), -3)
    assert_keys_close(rec, ref_rec, "recent")
    pend = torch.stack([pool[:, (info["mid_head"] + info["mid_count"] + r) % slots]
                        for r in range(info["recent_count"])], 1)
    ref_pend = oracle.rope_shift(oracle.round_bf16(oracle.rope_shift(d["recent_Kc"], 7)), -3)
    assert_keys_close(pend, ref_pend, "pending compressed")


def test_rope_shift_stress_full_size(pf):
    # all cached keys of a batch-2, 1,000-block pool layer: sink + mid + recent
    wl = _wl("stress16")
    d = synth.make_layer(wl, seed_for("stress16"), device="cuda", with_values=False)
    d["mid_V"] = torch.zeros_like(d["mid_K"])
    d["sink_V"] = torch.zeros_like(d["sink_K"])
    d["recent_V"] = torch.zeros_like(d["recent_K"])
    cache = build_cache(pf, wl, d)
    info = cache.info(0)
    delta = d["delta"]
    cache.rope_shift(0, pf.PART_SINK | pf.PART_MID | pf.PART_RECENT, delta)
    torch.cuda.synchronize()
    B, nc, H, D = wl.batch, wl.n_c, wl.heads, wl.head_dim
    slots = info["pool_slots"]
    pool = arena_view(cache, info["pool_k"], (B, slots, nc, H, D))
    g = np.random.default_rng(1)
    for p in sorted(g.choice(wl.pool_blocks, 24, replace=False).tolist()) + [0, wl.pool_blocks - 1]:
        got = pool[:, (info["mid_head"] + p) % slots].cpu()
        ref = oracle.rope_shift(d["mid_K"][:, p].cpu(), delta)
        assert_keys_close(got, ref, f"mid block {p}")
    sk = arena_view(cache, info["sink_k"], (B, 2 * wl.n, H, D))
    rows = _rows(2 * wl.n)
    assert_keys_close(sk[:, rows].cpu(), oracle.rope_shift(d["sink_K"].reshape(B, -1, H, D)[:, rows].cpu(), delta))


# ------------------------------------------------------------------ selection

@pytest.mark.parametrize("name", ["tiny", "ragged_a", "ragged_b", "ragged_c", "layer", "step30", "stress16",
                                  "stress64"])
def test_selection_bit_exact(pf, name):
    wl = _wl(name)
    d = synth.make_layer(wl, seed_for(name), device="cpu", with_values=False)
    for k in ("mid_V", "sink_V", "recent_V"):
        d[k] = torch.zeros_like(d[k.replace("V", "K")])
    d["V_cur"] = torch.zeros_like(d["K_cur"])
    cache = build_cache(pf, wl, d)
    B, P = wl.batch, wl.pool_blocks
    k = min(wl.n_top, P)
    sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    Q = d["Q"].cuda()
    cache.select_mid(0, Q, sel, sc)
    torch.cuda.synchronize()
    S_ref = oracle.select_scores(d["Q"], d["mid_K"])
    sel_ref = oracle.select_topk(S_ref, wl.n_top)
    assert np.all(oracle.selection_margin(S_ref, wl.n_top) >= 1e-3)
    assert np.array_equal(sel.cpu().numpy(), sel_ref), name
    assert np.array_equal(sel_ref, d["planted"].numpy())
    scale = np.abs(S_ref).max(axis=1, keepdims=True)
    assert np.max(np.abs(sc.cpu().numpy() - S_ref) / scale) < 1e-4
    info = cache.info(0)
    assert info["selection_valid"] == 1 and info["n_selected"] == k
    # a second call on the same inputs gives the same answer (scratch is left clean)
    sel2 = torch.full_like(sel, -1)
    cache.select_mid(0, Q, sel2, None)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel2)


@pytest.mark.parametrize("name", ["ragged_b", "layer"])
def test_selection_after_rotating_the_pool(pf, name):
    # selection scores the blocks' cached mean keys; a RoPE shift of the mid
    # pool must rotate them with the keys
    wl = _wl(name)
    d = synth.make_layer(wl, seed_for(name))
    cache = build_cache(pf, wl, d)
    delta = 3 * d["delta"] + 1
    cache.rope_shift(0, pf.PART_MID | pf.PART_RECENT, delta)
    B, P = wl.batch, wl.pool_blocks
    k = min(wl.n_top, P)
    sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    cache.select_mid(0, d["Q"].cuda(), sel, sc)
    torch.cuda.synchronize()
    midK = oracle.round_bf16(oracle.rope_shift(d["mid_K"], delta))
    S_ref = oracle.select_scores(d["Q"], midK)
    scale = np.abs(S_ref).max(axis=1, keepdims=True)
    assert np.max(np.abs(sc.cpu().numpy() - S_ref) / scale) < 1e-3
    margin = oracle.selection_margin(S_ref, wl.n_top)
    sel_ref = oracle.select_topk(S_ref, wl.n_top)
    for b in range(B):
        if margin[b] >= 1e-3:
            assert np.array_equal(sel.cpu().numpy()[b], sel_ref[b])


@pytest.mark.parametrize("name", ["ragged_b", "layer"])
def test_cached_mean_keys_after_many_mid_shifts(pf, name):
    # A shift rounds the pool's stored keys to bf16 and rotates each block's
    # cached float32 mean key without rounding.  After 24 shifts the cached
    # means are the means of the keys rotated exactly by the total shift
    # (the method's k' = k e^{i theta delta}), so the selection's scores must
    # match the oracle's scores of those keys tightly; the stored keys have
    # drifted from them by 24 bf16 roundings, which is bounded here too.
    wl = _wl(name)
    d = synth.make_layer(wl, seed_for(name))
    cache = build_cache(pf, wl, d)
    rng = np.random.default_rng(11)
    total = 0
    for _ in range(24):
        delta = int(rng.integers(1, 65))
        cache.rope_shift(0, pf.PART_MID, delta)
        total += delta
    B, P, nc, H, D = wl.batch, wl.pool_blocks, wl.n_c, wl.heads, wl.head_dim
    info = cache.info(0)
    k = min(wl.n_top, P)
    sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    cache.select_mid(0, d["Q"].cuda(), sel, sc)
    torch.cuda.synchronize()
    S_exact = oracle.select_scores(d["Q"], oracle.rope_shift(d["mid_K"], total))
    scale = np.abs(S_exact).max(axis=1, keepdims=True)
    assert np.max(np.abs(sc.cpu().numpy() - S_exact) / scale) < 2e-5
    margin = oracle.selection_margin(S_exact, wl.n_top)
    sel_ref = oracle.select_topk(S_exact, wl.n_top)
    for b in range(B):
        if margin[b] >= 1e-3:
            assert np.array_equal(sel.cpu().numpy()[b], sel_ref[b])
    # the keys as stored: within the accumulated rounding of 24 bf16 stores
    slots, head = info["pool_slots"], info["mid_head"]
    pool = arena_view(cache, info["pool_k"], (B, slots, nc, H, D)).cpu()
    live = torch.stack([pool[:, (head + p) % slots] for p in range(P)], 1)
    S_stored = oracle.select_scores(d["Q"], live)
    assert np.max(np.abs(S_stored - S_exact) / scale) < 5e-3


def test_largest_pool_selection_and_attention(pf):
    # the largest pool a cache allows (8,192 slots = 8,191 live blocks + the
    # recent block's pending copy): the top-k keeps every score in shared memory
    wl = _wl("tiny").replace(mid_capacity=8191, pool_blocks=8191, planted=16, n_top=16)
    d = synth.make_layer(wl, 31)
    cache = build_cache(pf, wl, d)
    assert cache.info(0)["pool_slots"] == 8192 and cache.info(0)["mid_count"] == 8191
    Q = d["Q"].cuda()
    sel = torch.full((1, 16), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((1, 8191), dtype=torch.float32, device="cuda")
    cache.select_mid(0, Q, sel, sc)
    O = cache.attend(0, Q, d["K_cur"].cuda(), d["V_cur"].cuda())
    torch.cuda.synchronize()
    S_ref = oracle.select_scores(d["Q"], d["mid_K"])
    assert oracle.selection_margin(S_ref, 16)[0] >= 1e-3
    assert np.array_equal(sel.cpu().numpy(), oracle.select_topk(S_ref, 16))
    assert np.max(np.abs(sc.cpu().numpy() - S_ref)) < 1e-4 * np.abs(S_ref).max()
    O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, d, sel.cpu().numpy()))
    assert_attention_close(O.cpu(), O_ref, "8,191-block pool")


def test_large_top_k_is_a_valid_selection(pf):
    # n_top = 3,000 of 8,191 random scores: no margin, so check what is unique
    # (the selected set is the 3,000 largest GPU scores, ties to the older
    # block) and that the scores match the oracle
    wl = _wl("tiny").replace(mid_capacity=8191, pool_blocks=8191, planted=0, n_top=3000)
    d = synth.make_layer(wl, 32)
    cache = build_cache(pf, wl, d)
    sel = torch.full((1, 3000), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((1, 8191), dtype=torch.float32, device="cuda")
    cache.select_mid(0, d["Q"].cuda(), sel, sc)
    torch.cuda.synchronize()
    s = sel.cpu().numpy()[0]
    g = sc.cpu().numpy()[0]
    assert np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < 8191          # ascending, distinct
    chosen = np.zeros(8191, dtype=bool)
    chosen[s] = True
    T = g[chosen].min()
    assert g[~chosen].max() <= T                                             # the largest scores
    eq = np.flatnonzero(g == T)
    assert np.all(chosen[eq[:chosen[eq].sum()]]) and not np.any(chosen[eq[chosen[eq].sum():]])   # older first
    S_ref = oracle.select_scores(d["Q"], d["mid_K"])[0]
    assert np.max(np.abs(g - S_ref)) < 1e-4 * np.abs(S_ref).max()


def test_selection_ties_go_to_older_blocks(pf):
    wl = _wl("ragged_a").replace(pool_blocks=9, planted=0, mid_capacity=9, n_top=4)
    d = synth.make_layer(wl, 5)
    d["mid_K"] = torch.zeros_like(d["mid_K"])         # every score exactly 0
    cache = build_cache(pf, wl, d)
    sel = torch.full((wl.batch, 4), -1, dtype=torch.int32, device="cuda")
    cache.select_mid(0, d["Q"].cuda(), sel, None)
    torch.cuda.synchronize()
    assert sel.cpu().tolist() == [[0, 1, 2, 3]] * wl.batch


# ------------------------------------------------- selection routing options

def _sel_inputs(name):
    wl = _wl(name)
    d = synth.make_layer(wl, seed_for(name), device="cpu", with_values=False)
    for k in ("mid_V", "sink_V", "recent_V"):
        d[k] = torch.zeros_like(d[k.replace("V", "K")])
    d["V_cur"] = torch.zeros_like(d["K_cur"])
    return wl, d


@pytest.mark.parametrize("name,q_stride,heads", [("ragged_a", 4, None), ("ragged_c", 4, (0, 1)),
                                                 ("ragged_c", 7, (1, 3)), ("layer", 4, (0, 6)),
                                                 ("stress16", 1, (0, 6)), ("stress16", 7, (6, 12))])
def test_selection_subsampled_queries_and_head_range(pf, name, q_stride, heads):
    # the speed variant: every q_stride-th query row, a head range
    wl, d = _sel_inputs(name)
    cache = build_cache(pf, wl, d)
    B, P = wl.batch, wl.pool_blocks
    k = min(wl.n_top, P)
    sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    cache.select_mid_ex(0, d["Q"].cuda(), q_stride=q_stride, heads=heads, sel_out=sel, scores_out=sc)
    torch.cuda.synchronize()
    S_ref = oracle.select_scores(d["Q"], d["mid_K"], q_stride=q_stride, heads=heads)
    assert np.all(oracle.selection_margin(S_ref, wl.n_top) >= 1e-3)
    assert np.array_equal(sel.cpu().numpy(), oracle.select_topk(S_ref, wl.n_top))
    scale = np.abs(S_ref).max(axis=1, keepdims=True)
    assert np.max(np.abs(sc.cpu().numpy() - S_ref) / scale) < 1e-4
    assert cache.info(0)["selection_valid"] == 1


def test_head_shard_scores_sum_then_given_top_k(pf):
    # two disjoint head ranges divided by the total head count (what two GPUs
    # holding six heads each would compute), summed, then the top-k of the
    # sum: the same selection and the same attention as the all-head call
    wl, d = _layer("ragged_b")
    cache = build_cache(pf, wl, d)
    B, P, H = wl.batch, wl.pool_blocks, wl.heads
    k = min(wl.n_top, P)
    Q, Kc, Vc = d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()
    sel_full = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc_full = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    cache.select_mid(0, Q, sel_full, sc_full)
    O_full = cache.attend(0, Q, Kc, Vc)
    half = H // 2
    parts = []
    for lo, hi in ((0, half), (half, H)):
        sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
        cache.select_mid_ex(0, Q, policy=pf.ROUTE_SCORES_ONLY, heads=(lo, hi), heads_total=H, scores_out=sc)
        parts.append(sc)
    summed = parts[0] + parts[1]
    torch.cuda.synchronize()
    scale = sc_full.abs().max().item()
    assert (summed - sc_full).abs().max().item() <= 1e-5 * scale
    S_ref = oracle.select_scores(d["Q"], d["mid_K"])
    half_ref = oracle.select_scores(d["Q"], d["mid_K"], heads=(0, half), heads_norm=H)
    assert np.max(np.abs(parts[0].cpu().numpy() - half_ref)) <= 1e-4 * np.abs(S_ref).max()
    sel_g = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    cache.select_mid_ex(0, policy=pf.ROUTE_GIVEN, scores_in=summed.contiguous(), sel_out=sel_g)
    O_g = cache.attend(0, Q, Kc, Vc)
    torch.cuda.synchronize()
    assert torch.equal(sel_g, sel_full)
    assert torch.equal(O_g, O_full)


@pytest.mark.parametrize("P,k", [(33, 1), (33, 32), (34, 33), (40, 16), (257, 32), (300, 17), (1000, 16),
                                 (1025, 32), (1025, 64), (3000, 5), (8191, 32)])
def test_given_scores_top_k(pf, P, k):
    # the top-k on its own, through given scores: up to 32 blocks by warp
    # sorting networks, more by the radix select.  Five distinct values (the
    # choice is mostly the older-block tie rule), then distinct scores.
    wl = _wl("tiny").replace(batch=2, pool_blocks=P, mid_capacity=P, n_top=k, planted=0)
    d = synth.make_layer(wl, 7)
    cache = build_cache(pf, wl, d)
    assert cache.info(0)["mid_count"] == P
    rng = np.random.default_rng(P * 97 + k)
    for scores in (rng.integers(-2, 3, size=(wl.batch, P)).astype(np.float32),
                   rng.standard_normal((wl.batch, P)).astype(np.float32)):
        sel = torch.full((wl.batch, k), -1, dtype=torch.int32, device="cuda")
        cache.select_mid_ex(0, policy=pf.ROUTE_GIVEN, scores_in=torch.from_numpy(scores).cuda(), sel_out=sel)
        torch.cuda.synchronize()
        assert np.array_equal(sel.cpu().numpy(), oracle.select_topk(scores, k))


@pytest.mark.parametrize("name", ["ragged_b", "ragged_c"])
def test_random_and_fifo_routing_then_attention(pf, name):
    # the pages' routing baselines: random blocks (random scores passed in)
    # and FIFO (the newest blocks); attention runs over what was routed
    wl, d = _layer(name)
    cache = build_cache(pf, wl, d)
    B, P = wl.batch, wl.pool_blocks
    k = min(wl.n_top, P)
    Q, Kc, Vc = d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()
    rng = np.random.default_rng(3)
    rand = np.stack([rng.permutation(P) for _ in range(B)]).astype(np.float32)   # distinct scores
    sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    cache.select_mid_ex(0, policy=pf.ROUTE_GIVEN, scores_in=torch.from_numpy(rand).cuda(), sel_out=sel)
    O = cache.attend(0, Q, Kc, Vc)
    torch.cuda.synchronize()
    sel_ref = oracle.select_topk(rand, wl.n_top)
    assert np.array_equal(sel.cpu().numpy(), sel_ref)
    O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, d, sel_ref))
    assert_attention_close(O.cpu(), O_ref, f"{name} random routing")
    sel_f = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    cache.select_mid_ex(0, policy=pf.ROUTE_FIFO, sel_out=sel_f)
    O = cache.attend(0, Q, Kc, Vc)
    torch.cuda.synchronize()
    fifo = np.stack([oracle.select_fifo(P, wl.n_top)] * B)
    assert np.array_equal(sel_f.cpu().numpy(), fifo)
    O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, d, fifo))
    assert_attention_close(O.cpu(), O_ref, f"{name} FIFO routing")


def test_select_ex_rejects_bad_options(pf):
    wl, d = _sel_inputs("ragged_a")
    cache = build_cache(pf, wl, d)
    Q = d["Q"].cuda()
    sc = torch.zeros((wl.batch, wl.pool_blocks), dtype=torch.float32, device="cuda")
    bad = [dict(policy=9), dict(q_stride=0), dict(heads=(1, 1)), dict(heads=(0, wl.heads + 1)),
           dict(heads=(-1, 1)), dict(heads_total=-2), dict(policy=pf.ROUTE_GIVEN),
           dict(policy=pf.ROUTE_SCORES_ONLY)]
    for kw in bad:
        with pytest.raises(pf.PFError) as e:
            cache.select_mid_ex(0, Q, **kw)
        assert e.value.status_name == "PF_ERR_ARG", kw
    with pytest.raises(pf.PFError):
        cache.select_mid_ex(0, None, scores_out=sc)      # scoring needs Q


# ------------------------------------------------------------------ attention

def _attend_and_compare(pf, wl, d, rows=None, via_append=False, lse_check=True):
    cache = build_cache(pf, wl, d, via_append=via_append)
    Q, Kc, Vc = d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()
    sel = None
    if wl.pool_blocks:
        k = min(wl.n_top, wl.pool_blocks)
        s = torch.zeros((wl.batch, k), dtype=torch.int32, device="cuda")
        cache.select_mid(0, Q, s, None)
        sel = s.cpu().numpy()
    lse = torch.zeros((wl.batch, wl.heads, wl.n), dtype=torch.float32, device="cuda")
    O = cache.attend(0, Q, Kc, Vc, lse=lse)
    assert cache.poll_device_error() == 0
    O = O.cpu()
    if sel is not None:
        sel_ref = oracle.select_topk(oracle.select_scores(d["Q"], d["mid_K"]), wl.n_top)
        assert np.array_equal(sel, sel_ref)
    parts = oracle_context(wl, d, sel)
    if rows is None:
        O_ref, lse_ref = oracle.attend(d["Q"], parts)
        res = assert_attention_close(O, O_ref, wl.name)
        got_lse = lse.cpu().numpy()
    else:
        O_ref, lse_ref = oracle.attend(d["Q"], parts, rows=rows)
        res = assert_attention_close(O[:, rows], O_ref, wl.name)
        got_lse = lse.cpu().numpy()[:, :, rows]
    if lse_check:
        assert np.max(np.abs(got_lse - lse_ref)) < LSE_MAX_ABS
    info = cache.info(0)
    tc = oracle.token_counts(wl.block_frames, wl.h, wl.w, wl.sink_blocks * wl.block_frames,
                             wl.recent_blocks * wl.block_frames, min(wl.n_top, wl.pool_blocks))
    assert info["context_tokens"] == tc["context"]
    return res


@pytest.mark.parametrize("name", ["tiny", "ragged_a", "ragged_b", "ragged_c"])
def test_attention_small_full(pf, name):
    wl, d = _layer(name)
    _attend_and_compare(pf, wl, d)


def test_attention_single_ragged_tile_split_and_merged(pf):
    # one 112-row query tile per (b, h) and no query-tile pairs: the tile is
    # cut along the context into small chunks, which park partial outputs that
    # the merge kernel (a second launch) combines; every row against the oracle
    wl = synth.WORKLOADS["ragged_c"].replace(name="ragged_one", h=4, w=7, n=112, n_c=2)
    assert wl.block_frames * wl.h * wl.w == wl.n and (wl.n + 127) // 128 == 1
    sb = lambda rows: (rows + 31) // 32  # noqa: E731
    n_tiles = (sb(wl.sink_blocks * wl.n) + min(wl.n_top, wl.pool_blocks) * sb(wl.n_c) + wl.recent_blocks * sb(wl.n)
               + sb(wl.n) + 3) // 4
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    big, small, _ = pf.pf_attend_tail_plan(0, wl.batch * wl.heads, n_tiles, sms)
    assert big + small > 1
    d = synth.make_layer(wl, seed_for("ragged_c") + 7)
    _attend_and_compare(pf, wl, d)


def test_attention_split_tail_repeated_calls(pf):
    # the split-tail scratch (partial outputs, tickets) is reused across calls
    wl, d = _layer("ragged_c")
    cache = build_cache(pf, wl, d)
    Q, Kc, Vc = d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()
    s = torch.zeros((wl.batch, wl.n_top), dtype=torch.int32, device="cuda")
    cache.select_mid(0, Q, s, None)
    outs = [cache.attend(0, Q, Kc, Vc).cpu() for _ in range(3)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, d, s.cpu().numpy()))
    assert_attention_close(outs[2], O_ref, "ragged_c repeated")


def test_attention_pool_filled_by_appends(pf):
    wl, d = _layer("ragged_a")
    _attend_and_compare(pf, wl, d, via_append=True)


def test_attention_pages_scale_layer(pf):
    # Lq 6,240 x Lk 27,872, 12 heads: the configuration bench.py times
    wl, d = _layer("layer")
    _attend_and_compare(pf, wl, d, rows=_rows(wl.n))


@pytest.mark.parametrize("name", ["stress16", "stress64"])
def test_attention_stress(pf, name):
    wl = _wl(name)
    d = synth.make_layer(wl, seed_for(name), device="cpu")
    _attend_and_compare(pf, wl, d, rows=_rows(wl.n, k=24))


def test_attention_dense_long_context(pf):
    # 748,800 full-resolution keys (no selection), sampled rows, head by head
    wl = _wl("dense")
    d = synth.make_layer(wl, seed_for("dense"), device="cuda")
    cache = build_cache(pf, wl, d)
    assert cache.info(0)["context_tokens"] == 748800
    O = cache.attend(0, d["Q"], d["K_cur"], d["V_cur"])
    assert cache.poll_device_error() == 0
    rows = _rows(wl.n, k=8)
    O = O[:, rows].cpu()
    B, H, D = wl.batch, wl.heads, wl.head_dim
    recK = d["recent_K"].reshape(B, -1, H, D)
    recV = d["recent_V"].reshape(B, -1, H, D)
    for h in (0, 5, 11):
        parts = [(recK[:, :, h:h + 1].cpu(), recV[:, :, h:h + 1].cpu()),
                 (d["K_cur"][:, :, h:h + 1].cpu(), d["V_cur"][:, :, h:h + 1].cpu())]
        O_ref, _ = oracle.attend(d["Q"][:, rows][:, :, h:h + 1].cpu(), parts)
        assert_attention_close(O[:, :, h:h + 1], O_ref, f"dense head {h}")


def test_attention_early_blocks_partial_sink_empty_pool(pf):
    wl = _wl("ragged_a")
    d = synth.make_layer(wl, 11)
    cache = pf.PackedKVCache(pf.config_for(wl, layers=1))
    Q, Kc, Vc = d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()
    # no history at all: the block attends to itself
    O = cache.attend(0, Q, Kc, Vc).cpu()
    O_ref, _ = oracle.attend(d["Q"], [(d["K_cur"], d["V_cur"])])
    assert_attention_close(O, O_ref, "empty cache")
    # one of two sink blocks stored
    cache.append_block(0, d["sink_K"][:, 0].cuda().contiguous(), d["sink_V"][:, 0].cuda().contiguous())
    O = cache.attend(0, Q, Kc, Vc).cpu()
    O_ref, _ = oracle.attend(d["Q"], [(d["sink_K"][:, 0], d["sink_V"][:, 0]), (d["K_cur"], d["V_cur"])])
    assert_attention_close(O, O_ref, "half sink")


def test_attention_needs_selection_when_pool_exceeds_n_top(pf):
    wl, d = _layer("ragged_a")
    cache = build_cache(pf, wl, d)
    with pytest.raises(pf.PFError) as e:
        cache.attend(0, d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda())
    assert e.value.status_name == "PF_ERR_STATE"


def test_attention_n_top_zero(pf):
    wl = _wl("ragged_a").replace(n_top=0, planted=0)
    d = synth.make_layer(wl, 3)
    cache = build_cache(pf, wl, d)
    cache.select_mid(0, d["Q"].cuda())
    O = cache.attend(0, d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()).cpu()
    O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, d, None))
    assert_attention_close(O, O_ref, "n_top=0")


# ------------------------------------------------------------------ cache state machine

def test_state_machine_against_partition_model(pf):
    wl = _wl("tiny").replace(mid_capacity=3, recent_blocks=2, n_top=2, planted=0, pool_blocks=0)
    cfg = pf.config_for(wl, layers=2)
    cache = pf.PackedKVCache(cfg)
    B, n, nc, H, D = wl.batch, wl.n, wl.n_c, wl.heads, wl.head_dim
    total_ev = 0
    for i in range(10):
        val = float(i + 1)
        K = torch.full((B, n, H, D), val, dtype=torch.bfloat16, device="cuda")
        Kc = torch.full((B, nc, H, D), val, dtype=torch.bfloat16, device="cuda")
        ev = cache.append_block(1, K, K, Kc, Kc)
        total_ev += ev
        want = oracle.cache_partitions(i + 1, wl.sink_blocks, wl.recent_blocks, wl.mid_capacity)
        info = cache.info(1)
        assert info["sink_filled"] == len(want["sink"])
        assert info["mid_count"] == len(want["mid"])
        assert info["recent_count"] == len(want["recent"])
        assert info["evicted"] == want["evicted"] == total_ev
        torch.cuda.synchronize()
        slots = info["pool_slots"]
        pool = arena_view(cache, info["pool_k"], (B, slots, nc, H, D)).cpu()
        got_mid = [pool[0, (info["mid_head"] + p) % slots, 0, 0, 0].item() - 1 for p in range(info["mid_count"])]
        assert got_mid == want["mid"]
        rec = arena_view(cache, info["recent_k"], (B, wl.recent_blocks, n, H, D)).cpu()
        got_rec = [rec[0, (info["recent_head"] + r) % wl.recent_blocks, 0, 0, 0].item() - 1
                   for r in range(info["recent_count"])]
        assert got_rec == want["recent"]
        sink = arena_view(cache, info["sink_k"], (B, wl.sink_blocks * n, H, D)).cpu()
        for s in want["sink"]:
            assert sink[0, s * n, 0, 0].item() - 1 == s
    assert cache.info(0)["blocks_seen"] == 0   # the other layer is untouched


# ------------------------------------------------------------------ generation loop

@pytest.mark.parametrize("fused", [False, True])
def test_generation_loop_against_oracle_model(pf, fused):
    """select -> attend -> append -> shift over several blocks, with the
    oracle keeping its own copy of every partition.  fused: the sink shift
    is applied inside attention (one rounding of the accumulated shift)."""
    wl = _wl("ragged_a").replace(mid_capacity=4, n_top=2, planted=0)
    B, n, nc, H, D, Bf = wl.batch, wl.n, wl.n_c, wl.heads, wl.head_dim, wl.block_frames
    cache = pf.PackedKVCache(pf.config_for(wl, layers=1, sink_rope_in_attention=fused))
    sinkK, sinkV, mid, recent = [], [], [], []     # oracle's partitions (bf16-valued float64 / tensors)
    total = 0                                      # accumulated sink shift (fused)
    for i in range(12):
        blk = synth.make_block(wl, 7000 + i)
        Q = synth.bf16_normal((B, n, H, D), 9000 + i)
        # attention of block i over the cache as it stands
        qd = Q.cuda()
        sel = None
        if len(mid) > wl.n_top:
            s = torch.zeros((B, wl.n_top), dtype=torch.int32, device="cuda")
            cache.select_mid(0, qd, s, None)
            sel = s.cpu().numpy()
            mK = torch.stack([torch.stack([m[0][b] for m in mid]) for b in range(B)], 1)
            S_ref = oracle.select_scores(Q, mK.transpose(0, 1))
            if np.all(oracle.selection_margin(S_ref, wl.n_top) >= 1e-3):
                assert np.array_equal(sel, oracle.select_topk(S_ref, wl.n_top))
        O = cache.attend(0, qd, blk["K"].cuda(), blk["V"].cuda()).cpu()
        if fused and total:
            parts = [(torch.from_numpy(oracle.round_bf16(oracle.rope_shift(k, total))), v)
                     for k, v in zip(sinkK, sinkV)]
        else:
            parts = [(torch.from_numpy(k), v) for k, v in zip(sinkK, sinkV)]
        if mid:
            chosen = [list(range(len(mid)))] * B if sel is None else sel.tolist()
            for j in range(len(chosen[0])):
                parts.append((torch.stack([mid[chosen[b][j]][0][b] for b in range(B)]),
                              torch.stack([mid[chosen[b][j]][1][b] for b in range(B)])))
        parts += [(r[0], r[1]) for r in recent]
        parts.append((blk["K"], blk["V"]))
        O_ref, _ = oracle.attend(Q, parts)
        assert_attention_close(O, O_ref, f"block {i}")
        # the block is final: append it, shift the sink on eviction
        ev = cache.append_block(0, blk["K"].cuda(), blk["V"].cuda(), blk["Kc"].cuda(), blk["Vc"].cuda())
        if len(sinkK) < wl.sink_blocks:
            sinkK.append(oracle.to_f64(blk["K"]))
            sinkV.append(blk["V"])
        else:
            recent.append((blk["K"], blk["V"], blk["Kc"], blk["Vc"]))
            if len(recent) > wl.recent_blocks:
                old = recent.pop(0)
                mid.append((old[2], old[3]))
                if len(mid) > wl.mid_capacity:
                    mid.pop(0)
                    assert ev == 1
        if ev:
            cache.rope_shift(0, pf.PART_SINK, ev * Bf)
            if fused:
                total += ev * Bf
            else:
                sinkK = [oracle.round_bf16(oracle.rope_shift(k, ev * Bf)) for k in sinkK]
    assert cache.info(0)["total_shift"] == cache.info(0)["evicted"] * Bf


def test_block_steps_across_layers_against_oracle_model(pf):
    """CFG batch 2 (cond + uncond), 2 layers, 4 denoising steps per block,
    8 blocks (two evictions).  pf_attend_step selects from the first step's queries and
    reuses that selection at steps 2-4 while the queries and the current
    block's K/V change from step to step; pf_finish_block appends the final
    block to every layer and shifts every sink on eviction.  The oracle keeps
    its own copy of every layer's partitions; every step's output of every
    layer is compared with it."""
    L, S = 2, 4
    wl = _wl("ragged_a").replace(mid_capacity=3, n_top=2, planted=0, layers=L)
    B, n, nc, H, D, Bf = wl.batch, wl.n, wl.n_c, wl.heads, wl.head_dim, wl.block_frames
    cache = pf.PackedKVCache(pf.config_for(wl))
    model = [{"sinkK": [], "sinkV": [], "mid": [], "recent": []} for _ in range(L)]
    total_ev = 0
    for i in range(8):
        final = [synth.make_block(wl, 7100 + 10 * i + l) for l in range(L)]
        for step in range(S):
            for l in range(L):
                m = model[l]
                seed = 9100 + 100 * i + 10 * step + l
                Q = synth.bf16_normal((B, n, H, D), seed)
                if step == S - 1:
                    Kcur, Vcur = final[l]["K"], final[l]["V"]
                else:
                    Kcur = synth.bf16_normal((B, n, H, D), seed + 50000)
                    Vcur = synth.bf16_normal((B, n, H, D), seed + 60000)
                O = cache.attend_step(l, step, Q.cuda(), Kcur.cuda(), Vcur.cuda()).cpu()
                info = cache.info(l)
                parts = [(torch.from_numpy(k), v) for k, v in zip(m["sinkK"], m["sinkV"])]
                if m["mid"]:
                    if len(m["mid"]) > wl.n_top:
                        assert info["selection_valid"] == 1
                        slots = arena_view(cache, info["selection"], (B, wl.n_top), torch.int32).cpu().numpy()
                        chosen = np.sort((slots - info["mid_head"]) % info["pool_slots"], axis=1)
                        if step == 0:
                            q0 = Q
                            mK = torch.stack([torch.stack([mm[0][b] for mm in m["mid"]]) for b in range(B)])
                            S_ref = oracle.select_scores(q0, mK)
                            m["sel_ref"] = (oracle.select_topk(S_ref, wl.n_top), oracle.selection_margin(S_ref, wl.n_top))
                        sel_ref, margin = m["sel_ref"]
                        for b in range(B):
                            if margin[b] >= 1e-3:
                                assert np.array_equal(chosen[b], sel_ref[b]), (i, step, l, b)
                    else:
                        chosen = np.array([list(range(len(m["mid"])))] * B)
                    for j in range(chosen.shape[1]):
                        parts.append((torch.stack([m["mid"][chosen[b][j]][0][b] for b in range(B)]),
                                      torch.stack([m["mid"][chosen[b][j]][1][b] for b in range(B)])))
                parts += [(r[0], r[1]) for r in m["recent"]]
                parts.append((Kcur, Vcur))
                O_ref, _ = oracle.attend(Q, parts)
                assert_attention_close(O, O_ref, f"block {i} step {step} layer {l}")
        ev = cache.finish_block([f["K"].cuda() for f in final], [f["V"].cuda() for f in final],
                                [f["Kc"].cuda() for f in final], [f["Vc"].cuda() for f in final])
        for l in range(L):
            m, f = model[l], final[l]
            if len(m["sinkK"]) < wl.sink_blocks:
                m["sinkK"].append(oracle.to_f64(f["K"]))
                m["sinkV"].append(f["V"])
            else:
                m["recent"].append((f["K"], f["V"], f["Kc"], f["Vc"]))
                if len(m["recent"]) > wl.recent_blocks:
                    old = m["recent"].pop(0)
                    m["mid"].append((old[2], old[3]))
                    if len(m["mid"]) > wl.mid_capacity:
                        m["mid"].pop(0)
                        assert ev == 1
            if ev:
                m["sinkK"] = [oracle.round_bf16(oracle.rope_shift(k, ev * Bf)) for k in m["sinkK"]]
        total_ev += ev
    assert total_ev >= 2
    for l in range(L):
        assert cache.info(l)["total_shift"] == total_ev * Bf


def test_block_step_calls_refuse_bad_arguments(pf):
    wl = _wl("ragged_a").replace(layers=2)
    B, n, H, D = wl.batch, wl.n, wl.heads, wl.head_dim
    cache = pf.PackedKVCache(pf.config_for(wl))
    blk = synth.make_block(wl, 3)
    Q = synth.bf16_normal((B, n, H, D), 4).cuda()
    K, V = blk["K"].cuda(), blk["V"].cuda()
    with pytest.raises(pf.PFError) as e:
        cache.attend_step(0, -1, Q, K, V)
    assert e.value.status_name == "PF_ERR_ARG"
    with pytest.raises(ValueError):
        cache.finish_block([K], [V])                      # one tensor per layer
    with pytest.raises(pf.PFError) as e:                  # a NULL pointer in the array
        pf.pf_finish_block(cache.handle, [K, 0], [V, V])
    assert e.value.status_name == "PF_ERR_ARG"
    assert cache.info(0)["blocks_seen"] == 0 and cache.info(1)["blocks_seen"] == 0   # nothing appended
    for _ in range(wl.sink_blocks):
        assert cache.finish_block([K, K], [V, V]) == 0    # sink blocks need no compressed copy
    with pytest.raises(pf.PFError) as e:                  # now the compressed copies are needed
        cache.finish_block([K, K], [V, V])
    assert e.value.status_name == "PF_ERR_ARG"
    assert cache.info(1)["blocks_seen"] == wl.sink_blocks


def test_later_steps_refuse_a_selection_the_pool_has_outgrown(pf):
    # the selection made at a block's first step belongs to that pool: once
    # the block is finished (the pool changed), a later-step call without a
    # new first step is refused, and a first step selects again
    L = 2
    wl = _wl("ragged_a").replace(mid_capacity=3, n_top=2, planted=0, layers=L)
    B, n, H, D = wl.batch, wl.n, wl.heads, wl.head_dim
    cache = pf.PackedKVCache(pf.config_for(wl))
    for i in range(7):
        blks = [synth.make_block(wl, 800 + 10 * i + l) for l in range(L)]
        cache.finish_block([b_["K"].cuda() for b_ in blks], [b_["V"].cuda() for b_ in blks],
                           [b_["Kc"].cuda() for b_ in blks], [b_["Vc"].cuda() for b_ in blks])
    assert cache.info(0)["mid_count"] == 3 > wl.n_top
    Q = synth.bf16_normal((B, n, H, D), 900).cuda()
    K = synth.bf16_normal((B, n, H, D), 901).cuda()
    for l in range(L):
        cache.attend_step(l, 0, Q, K, K)
        cache.attend_step(l, 3, Q, K, K)                 # the stored selection is reused
    blks = [synth.make_block(wl, 990 + l) for l in range(L)]
    cache.finish_block([b_["K"].cuda() for b_ in blks], [b_["V"].cuda() for b_ in blks],
                       [b_["Kc"].cuda() for b_ in blks], [b_["Vc"].cuda() for b_ in blks])
    for l in range(L):
        assert cache.info(l)["selection_valid"] == 0
        with pytest.raises(pf.PFError) as e:
            cache.attend_step(l, 1, Q, K, K)
        assert e.value.status_name == "PF_ERR_STATE"
        cache.attend_step(l, 0, Q, K, K)
        assert cache.info(l)["selection_valid"] == 1
    assert cache.poll_device_error() == 0


@pytest.mark.parametrize("name", ["ragged_a", "ragged_c", "layer"])
def test_sink_rope_in_attention_matches_oracle(pf, name):
    # the sink's shift recorded by pf_rope_shift and applied by pf_attend to
    # the sink's key tiles: the stored keys stay as appended; attention sees
    # them rotated by the accumulated shift (rounded to bf16 once)
    wl, d = _layer(name)
    cache = build_cache(pf, wl, d, sink_rope_in_attention=True)
    info = cache.info(0)
    B, S, n, H, D = wl.batch, wl.sink_blocks, wl.n, wl.heads, wl.head_dim
    d1, d2 = d["delta"], 3 * d["delta"] + 5
    cache.rope_shift(0, pf.PART_SINK, d1)
    cache.rope_shift(0, pf.PART_SINK, d2)
    Q, Kc, Vc = d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda()
    k = min(wl.n_top, wl.pool_blocks)
    s = torch.zeros((B, k), dtype=torch.int32, device="cuda")
    cache.select_mid(0, Q, s, None)
    O = cache.attend(0, Q, Kc, Vc)
    assert cache.poll_device_error() == 0
    O = O.cpu()
    assert cache.info(0)["total_shift"] == d1 + d2
    stored = arena_view(cache, info["sink_k"], (B, S * n, H, D)).cpu()
    assert torch.equal(stored, d["sink_K"].reshape(B, S * n, H, D))     # not rotated in place
    rot = dict(d)
    rot["sink_K"] = torch.from_numpy(oracle.round_bf16(oracle.rope_shift(d["sink_K"], d1 + d2)))
    rows = _rows(wl.n) if wl.n > 1000 else None
    O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, rot, s.cpu().numpy()), rows=rows)
    got = O if rows is None else O[:, rows]
    assert_attention_close(got, O_ref, f"{name} sink rope in attention")


def test_sink_rope_in_attention_needs_a_full_sink(pf):
    wl = _wl("ragged_a")
    cache = pf.PackedKVCache(pf.config_for(wl, layers=1, sink_rope_in_attention=True))
    blk = synth.make_block(wl, 17)
    cache.append_block(0, blk["K"].cuda(), blk["V"].cuda())   # 1 of 2 sink blocks
    with pytest.raises(pf.PFError) as e:
        cache.rope_shift(0, pf.PART_SINK, 4)
    assert e.value.status_name == "PF_ERR_STATE"
    cache.rope_shift(0, pf.PART_SINK, 0)                         # a zero shift is a no-op
    cache.append_block(0, blk["K"].cuda(), blk["V"].cuda())
    cache.rope_shift(0, pf.PART_SINK, 4)
    assert cache.info(0)["total_shift"] == 4


# ------------------------------------------------------------------ save and restore

def test_save_and_restore_a_cache(pf):
    # a cache restored from its saved host state and a copy of its arena
    # behaves exactly as the original: same layer states, bit-identical
    # attention with the stored selection, and the same evolution afterwards
    L = 2
    wl = _wl("ragged_a").replace(mid_capacity=3, n_top=2, planted=0, layers=L)
    B, n, H, D = wl.batch, wl.n, wl.heads, wl.head_dim
    cfg = pf.config_for(wl)
    cache = pf.PackedKVCache(cfg)
    for i in range(8):                                  # sink, recent, a full pool and two evictions
        blks = [synth.make_block(wl, 500 + 10 * i + l) for l in range(L)]
        cache.finish_block([b_["K"].cuda() for b_ in blks], [b_["V"].cuda() for b_ in blks],
                           [b_["Kc"].cuda() for b_ in blks], [b_["Vc"].cuda() for b_ in blks])
    Q = synth.bf16_normal((B, n, H, D), 600).cuda()
    K = synth.bf16_normal((B, n, H, D), 601).cuda()
    for l in range(L):
        cache.attend_step(l, 0, Q, K, K)                # stores a selection in every layer
    saved = cache.save()
    twin = pf.PackedKVCache.restore(cfg, saved)
    for l in range(L):
        a, b = cache.info(l), twin.info(l)
        for k in ("blocks_seen", "sink_filled", "recent_count", "recent_head", "mid_count", "mid_head",
                  "selection_valid", "n_selected", "context_tokens", "evicted", "total_shift"):
            assert a[k] == b[k], (l, k)
        assert a["selection_valid"] == 1 and a["evicted"] >= 2
        O1 = cache.attend_step(l, 1, Q, K, K)           # reuses the stored selection
        O2 = twin.attend_step(l, 1, Q, K, K)
        assert torch.equal(O1, O2)
    blks = [synth.make_block(wl, 700 + l) for l in range(L)]
    args = ([b_["K"].cuda() for b_ in blks], [b_["V"].cuda() for b_ in blks],
            [b_["Kc"].cuda() for b_ in blks], [b_["Vc"].cuda() for b_ in blks])
    assert cache.finish_block(*args) == twin.finish_block(*args) == 1
    for l in range(L):
        assert torch.equal(cache.attend_step(l, 0, Q, K, K), twin.attend_step(l, 0, Q, K, K))
    # a state of another configuration, or not a state at all, is refused
    other = pf.PackedKVCache(pf.config_for(wl.replace(n_top=1)))
    with pytest.raises(pf.PFError) as e:
        pf.pf_cache_load_state(other.handle, saved[0])
    assert e.value.status_name == "PF_ERR_STATE"
    with pytest.raises(pf.PFError) as e:
        pf.pf_cache_load_state(twin.handle, b"\0" * len(saved[0]))
    assert e.value.status_name == "PF_ERR_ARG"
    bad = bytearray(saved[0])
    # the last layer's record: eight int32 (mid_count the fifth) then two int64
    bad[-32:-28] = (10 ** 6).to_bytes(4, "little")      # its mid_count far past the capacity
    with pytest.raises(pf.PFError) as e:
        pf.pf_cache_load_state(twin.handle, bytes(bad))
    assert e.value.status_name == "PF_ERR_STATE"


# ------------------------------------------------------------------ several devices

def test_two_devices_in_one_process(pf):
    # each launcher's one-time set-up is per device: a second GPU in the same
    # process runs the whole path too (a head-sharded layer drives one GPU per
    # rank, but a single process may also hold caches on several GPUs)
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    wl, d = _layer("ragged_c")
    for dev in (0, 1):
        with torch.cuda.device(dev):
            cache = build_cache(pf, wl, d, device=f"cuda:{dev}")
            Q = d["Q"].to(f"cuda:{dev}")
            s = torch.zeros((wl.batch, wl.n_top), dtype=torch.int32, device=f"cuda:{dev}")
            cache.select_mid(0, Q, s, None)
            O = cache.attend(0, Q, d["K_cur"].to(f"cuda:{dev}"), d["V_cur"].to(f"cuda:{dev}"))
            assert cache.poll_device_error() == 0
            O_ref, _ = oracle.attend(d["Q"], oracle_context(wl, d, s.cpu().numpy()))
            assert_attention_close(O.cpu(), O_ref, f"device {dev}")


# ------------------------------------------------------------------ failure detection

def test_bounded_wait_reports_timeout_and_context_survives(pf):
    wl, d = _layer("tiny")
    cache = build_cache(pf, wl, d)
    pf.pf_selftest_wait_timeout(cache.handle, 2000)
    with pytest.raises(pf.PFError) as e:
        cache.poll_device_error()
    assert e.value.status_name == "PF_ERR_TIMEOUT"
    assert cache.poll_device_error() == 0          # cleared
    # the device is still usable
    cache.select_mid(0, d["Q"].cuda())
    O = cache.attend(0, d["Q"].cuda(), d["K_cur"].cuda(), d["V_cur"].cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(O.float()).all()
