"""pf_select_mid_static: the selection for callers that cannot allocate
device memory (a serving process with a fixed device-memory budget and no
allocation on the request path, or a framework that owns the allocator and
gives this library no arena).  Its scratch is a fixed array inside the
library; this checks it against pf_select_mid and against the oracle,
through the C ABI, on two calls in a row.  The file name makes pytest
collect it last."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _harness import build_cache, seed_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pf():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from packed_kv_cache_b200 import build
    build.build()
    import packed_kv_cache_b200 as mod
    return mod


@pytest.mark.parametrize("name", ["ragged_a", "layer"])
def test_static_selection_matches_cache_selection(pf, name):
    wl = synth.WORKLOADS[name]
    d = synth.make_layer(wl, seed_for(name))
    cache = build_cache(pf, wl, d)
    info = cache.info(0)
    B, P = wl.batch, info["mid_count"]
    k = min(wl.n_top, P)
    Q = d["Q"].cuda()
    sel_ref = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc_ref = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    cache.select_mid(0, Q, sel_ref, sc_ref)
    torch.cuda.synchronize()
    scale = sc_ref.abs().max(dim=1, keepdim=True).values
    for _ in range(2):                       # the second call reuses the array the first one left
        sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
        sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
        pf.pf_select_mid_static(Q, B, wl.n, wl.heads, info["pool_k"], info["pool_slots"], wl.n_c,
                                info["mid_head"], P, wl.n_top, sel, sc)
        torch.cuda.synchronize()
        assert torch.equal(sel, sel_ref)
        assert float(((sc - sc_ref).abs() / scale).max()) < 1e-4
    assert np.array_equal(sel.cpu().numpy(), d["planted"].numpy())


@pytest.mark.parametrize("name,slots,head", [("ragged_a", 20, 14), ("layer", 50, 31)])
def test_static_selection_wrapped_ring_matches_oracle(pf, name, slots, head):
    # the live blocks run from slot `head` past the end of the ring and on
    # from slot 0; the other slots hold unrelated keys that must not count
    wl = synth.WORKLOADS[name]
    d = synth.make_layer(wl, seed_for(name))
    B, P, nc, H, D = wl.batch, wl.pool_blocks, wl.n_c, wl.heads, wl.head_dim
    assert head + P > slots                                   # wraps
    pool = synth.bf16_normal((B, slots, nc, H, D), 4242)
    for p in range(P):
        pool[:, (head + p) % slots] = d["mid_K"][:, p]
    S_ref = oracle.select_scores(d["Q"], d["mid_K"])
    sel_ref = oracle.select_topk(S_ref, wl.n_top)
    assert np.all(oracle.selection_margin(S_ref, wl.n_top) >= 1e-3)
    Q, pool_d = d["Q"].cuda(), pool.cuda()
    k = min(wl.n_top, P)
    scale = np.abs(S_ref).max(axis=1, keepdims=True)
    for _ in range(2):                       # the second call reuses the array the first one left
        sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
        sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
        pf.pf_select_mid_static(Q, B, wl.n, H, pool_d, slots, nc, head, P, wl.n_top, sel, sc)
        torch.cuda.synchronize()
        assert np.array_equal(sel.cpu().numpy(), sel_ref)
        assert float((np.abs(sc.cpu().numpy() - S_ref) / scale).max()) < 1e-4
    # n_top = 0: no selection, but the scores are still written
    sel = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, P), dtype=torch.float32, device="cuda")
    pf.pf_select_mid_static(Q, B, wl.n, H, pool_d, slots, nc, head, P, 0, sel, sc)
    torch.cuda.synchronize()
    assert bool((sel == -1).all())
    assert float((np.abs(sc.cpu().numpy() - S_ref) / scale).max()) < 1e-4


def test_static_selection_rejects_sizes_beyond_its_array(pf):
    Q = torch.zeros((1, 64, 1, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 8, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((9, 4), dtype=torch.int32, device="cuda")
    cases = [dict(batch=9, heads=1, count=8, n_c=4, slots=8),
             dict(batch=1, heads=17, count=8, n_c=4, slots=8),
             dict(batch=1, heads=1, count=5000, n_c=4, slots=5000),
             dict(batch=1, heads=1, count=8, n_c=513, slots=8)]
    for c in cases:
        # raw addresses: the library's own limits are under test, not the
        # binding's size checks (nothing is launched: the sizes are refused first)
        with pytest.raises(pf.PFError) as e:
            pf.pf_select_mid_static(Q.data_ptr(), c["batch"], 64, c["heads"], K.data_ptr(), c["slots"], c["n_c"], 0,
                                    c["count"], 4, sel.data_ptr())
        assert e.value.status_name == "PF_ERR_CAPACITY"
