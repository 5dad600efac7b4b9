"""pf_select_mid_static: the selection for callers that cannot allocate
device memory (a serving process with a fixed device-memory budget and no
allocation on the request path, or a framework that owns the allocator and
gives this library no arena).  Its scratch is a fixed array inside the
library; this checks it against pf_select_mid, through the C ABI, on two
calls in a row.  The file name makes pytest collect it last."""
import numpy as np
import pytest
import torch

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


def test_static_selection_rejects_sizes_beyond_its_array(pf):
    Q = torch.zeros((1, 64, 1, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 8, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((9, 4), dtype=torch.int32, device="cuda")
    cases = [dict(batch=9, heads=1, count=8, n_c=4, slots=8),
             dict(batch=1, heads=17, count=8, n_c=4, slots=8),
             dict(batch=1, heads=1, count=5000, n_c=4, slots=5000),
             dict(batch=1, heads=1, count=8, n_c=513, slots=8)]
    for c in cases:
        with pytest.raises(pf.PFError) as e:
            pf.pf_select_mid_static(Q, c["batch"], 64, c["heads"], K, c["slots"], c["n_c"], 0, c["count"], 4, sel)
        assert e.value.status_name == "PF_ERR_CAPACITY"
