"""Host-only checks of the C-ABI library: it loads without a GPU, exports
every function include/pf.h declares, sizes arenas and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pf.h")


@pytest.fixture(scope="module")
def pf():
    from packed_kv_cache_b200 import build
    build.build()
    import packed_kv_cache_b200 as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pf_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("pf_cache_bytes", "pf_cache_create", "pf_cache_destroy", "pf_cache_append_block",
                 "pf_select_mid", "pf_rope_shift", "pf_attend", "pf_poll_device_error", "pf_last_error"):
        assert want in names


def test_library_exports_every_declared_symbol(pf):
    lib = ctypes.CDLL(pf.library_path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_status_strings(pf):
    assert pf.pf_version() >= 100
    assert pf.lib.pf_status_string(6) == b"PF_ERR_TIMEOUT"


def _cfg(pf, **kw):
    c = pf.config_for(synth.WORKLOADS["layer"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_cache_bytes_layout(pf):
    wl = synth.WORKLOADS["layer"]
    c = pf.config_for(wl)
    got = pf.pf_cache_bytes(c)
    row = 12 * 128 * 2
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    slots = wl.mid_capacity + wl.recent_blocks
    cpb = (182 + 31) // 32
    slabs = 12 * 128 // 128                 # slab tickets: one per 128 columns of the H * D vector
    per_layer = (2 * (al(2 * 6240 * row) + al(slots * 182 * row) + al(6240 * row))
                 + al(16 * 4) + al(slots * 4) + al(slots * cpb * 4)
                 + al(33 * 12 * 128 * 4)    # query sums of up to 32 row chunks, then their total
                 + al((1 + slabs) * 4)      # batch and slab tickets
                 + al(slots * 1536 * 4))    # mean key of every pool slot
    # shared attention scratch: 256 split-tail slots of 128x128 fp32 partial
    # outputs and their row max / row sum
    scratch = 256 * 128 * 128 * 4 + 256 * 2 * 128 * 4
    assert got == 256 + scratch + per_layer
    # layers scale linearly
    c.layers = 30
    assert pf.pf_cache_bytes(c) == 256 + scratch + 30 * per_layer


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, "PF_ERR_UNSUPPORTED"),
    ("batch", 0, "PF_ERR_ARG"),
    ("recent_blocks", 0, "PF_ERR_ARG"),
    ("mid_capacity", 9000, "PF_ERR_CAPACITY"),
    ("rope_base", 0.5, "PF_ERR_ARG"),
    # sums and products of int fields that would overflow if formed in int
    ("mid_capacity", 2**31 - 1, "PF_ERR_CAPACITY"),
    ("h", 2**31 - 1, "PF_ERR_CAPACITY"),
    ("heads", 257, "PF_ERR_CAPACITY"),     # the scoring kernel's shared memory
])
def test_config_validation(pf, field, value, status):
    c = _cfg(pf, **{field: value})
    with pytest.raises(pf.PFError) as e:
        pf.pf_cache_bytes(c)
    assert e.value.status_name == status


def test_cache_bytes_reports_overflow_instead_of_wrapping(pf):
    # 2^31 layers of 2^31 batch items with 64 KB key rows (a pages-scale
    # context of 28,032 keys) is far past size_t: the size must be refused,
    # never wrapped to a small arena
    big = dict(batch=2**31 - 1, layers=2**31 - 1, heads=256)
    with pytest.raises(pf.PFError) as e:
        pf.pf_cache_bytes(_cfg(pf, **big))
    assert e.value.status_name == "PF_ERR_CAPACITY"
    assert b"size_t" in pf.lib.pf_last_error()
    # create refuses it the same way, before looking at the arena
    h = ctypes.c_void_p()
    assert pf.lib.pf_cache_create(ctypes.byref(_cfg(pf, **big)), 0x100000, 2**63, None, ctypes.byref(h)) == 4
    # the largest sizes that still fit are computed exactly
    one, two = (pf.pf_cache_bytes(_cfg(pf, layers=k)) for k in (1, 2))
    assert pf.pf_cache_bytes(_cfg(pf, layers=2**31 - 1)) == one + (2**31 - 2) * (two - one)


def test_attention_context_is_capped_below_2_27_keys(pf):
    # n = 4 x 512 x 512 = 2^20 keys per block, one head; the context counted as
    # the attention pads it: sink + routed mid blocks + recent + current
    base = dict(heads=1, block_frames=4, h=512, w=512)

    def status(**kw):
        try:
            pf.pf_cache_bytes(_cfg(pf, **dict(base, **kw)))
            return "PF_OK"
        except pf.PFError as e:
            return e.status_name

    none = dict(sink_blocks=0, mid_capacity=0, n_top=0)
    assert status(recent_blocks=126, **none) == "PF_OK"              # 127 x 2^20 keys
    assert status(recent_blocks=127, **none) == "PF_ERR_CAPACITY"    # 2^27 keys
    assert b"2^27" in pf.lib.pf_last_error()
    assert status(recent_blocks=1, sink_blocks=125, mid_capacity=0, n_top=0) == "PF_OK"
    assert status(recent_blocks=1, sink_blocks=126, mid_capacity=0, n_top=0) == "PF_ERR_CAPACITY"
    # routed mid blocks: min(n_top, mid_capacity) blocks of n_c = 2 x 128 x 128 = 2^15 keys
    assert status(recent_blocks=126, sink_blocks=0, mid_capacity=31, n_top=1000) == "PF_OK"
    assert status(recent_blocks=126, sink_blocks=0, mid_capacity=32, n_top=1000) == "PF_ERR_CAPACITY"
    assert status(recent_blocks=126, sink_blocks=0, mid_capacity=1000, n_top=31) == "PF_OK"


def test_every_configuration_the_tests_and_the_bench_build_is_accepted(pf):
    W = synth.WORKLOADS
    cases = list(W.values()) + [
        W["tiny"].replace(mid_capacity=8191, pool_blocks=8191, planted=16, n_top=16),
        W["tiny"].replace(mid_capacity=8191, pool_blocks=8191, planted=0, n_top=3000),
        W["ragged_a"].replace(pool_blocks=9, planted=0, mid_capacity=9, n_top=4),
        W["ragged_a"].replace(n_top=0, planted=0),
        W["tiny"].replace(mid_capacity=3, recent_blocks=2, n_top=2, planted=0, pool_blocks=0),
        W["ragged_a"].replace(mid_capacity=4, n_top=2, planted=0)]
    for wl in cases:
        for fused in (False, True):
            assert pf.pf_cache_bytes(pf.config_for(wl, sink_rope_in_attention=fused)) > 0, wl.name


def test_block_size_product_does_not_overflow(pf):
    # B_f * h * w with every factor near 2^31 overflows even 64 bits when
    # formed in one go; the check refuses it instead
    for kw in (dict(block_frames=2**31 - 1, h=2**31 - 1, w=2**31 - 1), dict(block_frames=4, h=2**30, w=2**30),
               dict(block_frames=2**31 - 1, h=1, w=1)):
        with pytest.raises(pf.PFError) as e:
            pf.pf_cache_bytes(_cfg(pf, **kw))
        assert e.value.status_name == "PF_ERR_CAPACITY" and b"2^24" in pf.lib.pf_last_error()


def test_rope_split_validation(pf):
    c = _cfg(pf)
    c.rope_split[0] = 46
    with pytest.raises(pf.PFError) as e:
        pf.pf_cache_bytes(c)
    assert e.value.status_name == "PF_ERR_UNSUPPORTED"


def test_create_rejects_bad_arenas_before_device_work(pf):
    c = _cfg(pf)
    need = pf.pf_cache_bytes(c)
    h = ctypes.c_void_p()
    assert pf.lib.pf_cache_create(ctypes.byref(c), None, need, None, ctypes.byref(h)) == 1
    assert pf.lib.pf_cache_create(ctypes.byref(c), 0x1000 + 16, need, None, ctypes.byref(h)) == 2
    assert b"256-byte" in pf.lib.pf_last_error()
    assert pf.lib.pf_cache_create(ctypes.byref(c), 0x100000, need - 1, None, ctypes.byref(h)) == 2
    assert b"needed" in pf.lib.pf_last_error()


def test_calls_reject_null_cache(pf):
    assert pf.lib.pf_attend(None, 0, None, None, None, None, None, None) == 1
    assert pf.lib.pf_select_mid(None, 0, None, None, None, None) == 1
    assert pf.lib.pf_rope_shift(None, 0, 1, 4, None) == 1
    assert pf.lib.pf_cache_destroy(None) == 1
    assert pf.lib.pf_poll_device_error(None, None, None) == 1


def test_static_selection_checks_arguments_before_device_work(pf):
    # placeholder device addresses: every case below returns before the library
    # touches them (argument and capacity checks, or nothing to select)
    Q, K, sel = 0x100000, 0x200000, 0x300000
    f = pf.lib.pf_select_mid_static
    LIMITS = {k: int(v) for k, v in re.findall(r"#define (PF_STATIC_MAX_\w+) (\d+)", open(HEADER).read())}
    assert len(LIMITS) == 4

    def call(Q=Q, batch=1, n=64, heads=1, K=K, slots=8, n_c=4, head=0, count=8, n_top=4, sel=sel, scores=None):
        return f(Q, batch, n, heads, K, slots, n_c, head, count, n_top, sel, scores, None)

    assert call(Q=None) == 1 and call(K=None) == 1 and call(sel=None) == 1
    assert call(Q=Q + 8) == 1 and b"misaligned" in pf.lib.pf_last_error()
    assert call(sel=sel + 2) == 1 and call(scores=0x400002) == 1
    assert call(n=0) == 1 and call(n_c=0) == 1 and call(count=-1) == 1 and call(n_top=-1) == 1
    assert call(slots=4, count=8) == 1      # more live blocks than slots
    assert call(head=8) == 1 and call(head=-1) == 1
    # capacity of the fixed scratch array
    assert call(batch=LIMITS["PF_STATIC_MAX_BATCH"] + 1) == 4
    assert call(heads=LIMITS["PF_STATIC_MAX_HEADS"] + 1) == 4
    assert call(slots=LIMITS["PF_STATIC_MAX_BLOCKS"] + 1,
                count=LIMITS["PF_STATIC_MAX_BLOCKS"] + 1) == 4
    assert call(n_c=LIMITS["PF_STATIC_MAX_NC"] + 1) == 4
    assert call(batch=8, slots=4097) == 4 and b"pool_slots" in pf.lib.pf_last_error()
    # nothing to select: success with no device work
    assert call(count=0) == 0 and call(n_top=0) == 0


def test_cache_methods_refuse_wrong_dtypes_and_short_buffers(pf):
    # the library sees only addresses: the binding refuses a buffer of the wrong
    # element type or too small for the call before anything is launched.
    # (No GPU here: an object without an arena, with the layer's live-block
    # count stubbed; a correct CPU tensor passes the checks and is then refused
    # as not being on the device.)
    import torch
    wl = synth.WORKLOADS["ragged_a"]                  # B=2, H=2, n=240, n_c=4, n_top=5
    cache = pf.PackedKVCache.__new__(pf.PackedKVCache)
    cache.cfg, cache.handle = pf.config_for(wl), None
    cache.info = lambda layer: {"mid_count": 13}
    B, H, D, n, nc = wl.batch, wl.heads, wl.head_dim, wl.n, wl.n_c
    bf = lambda *shape: torch.zeros(shape, dtype=torch.bfloat16)   # noqa: E731
    Q = bf(B, n, H, D)

    def refused(fn, what):
        with pytest.raises(ValueError) as e:
            fn()
        assert what in str(e.value), str(e.value)

    refused(lambda: cache.attend(0, Q.float(), Q, Q), "Q must be torch.bfloat16")
    refused(lambda: cache.attend(0, Q, Q[:, :-1], Q), "K_cur has")
    refused(lambda: cache.attend(0, Q, Q, Q, O=bf(B, n - 1, H, D)), "O has")
    refused(lambda: cache.attend(0, Q, Q, Q, lse=torch.zeros(B * H * n - 1)), "lse has")
    refused(lambda: cache.attend(0, Q, Q, Q), "CUDA tensor")
    refused(lambda: cache.select_mid(0, bf(B, n, H, D - 1)), "Q has")
    refused(lambda: cache.select_mid(0, Q, torch.zeros((B, 4), dtype=torch.int32)), "sel_out has")
    refused(lambda: cache.select_mid(0, Q, torch.zeros((B, 5), dtype=torch.int64)), "sel_out must be")
    refused(lambda: cache.select_mid(0, Q, None, torch.zeros((B, 12))), "scores_out has")
    refused(lambda: cache.select_mid(0, Q, torch.zeros((B, 5), dtype=torch.int32), torch.zeros((B, 13))),
            "CUDA tensor")
    refused(lambda: cache.select_mid_ex(0, None, policy=pf.ROUTE_GIVEN, scores_in=torch.zeros((B, 12))),
            "scores_in has")
    refused(lambda: cache.append_block(0, Q[:, :-1], Q), "K has")
    refused(lambda: cache.append_block(0, Q, Q, bf(B, nc - 1, H, D), bf(B, nc, H, D)), "Kc has")
    refused(lambda: cache.load_mid(0, bf(B, 3, nc, H, D), bf(B, 2, nc, H, D)), "Vc has")
    # the allocation-free selection: sizes come from its arguments
    P, slots = 13, 16
    pool = bf(B, slots, nc, H, D)
    sel = torch.zeros((B, 5), dtype=torch.int32)
    static = lambda **kw: pf.pf_select_mid_static(  # noqa: E731
        kw.get("Q", Q), B, n, H, kw.get("pool", pool), slots, nc, 3, P, 5, kw.get("sel", sel), kw.get("sc"))
    refused(lambda: static(Q=Q[:, :-1]), "Q has")
    refused(lambda: static(Q=Q.float()), "Q must be torch.bfloat16")
    refused(lambda: static(pool=pool[:, :-1]), "pool_k has")
    refused(lambda: static(sel=sel[:, :-1]), "sel_out has")
    refused(lambda: static(sel=sel.long()), "sel_out must be")
    refused(lambda: static(sc=torch.zeros((B, P - 1))), "scores_out has")
    refused(lambda: static(sc=torch.zeros((B, P))), "CUDA tensor")


def _hold_build_lock(q):
    import time

    from packed_kv_cache_b200 import build
    with build._exclusive():
        t0 = time.monotonic()
        time.sleep(0.3)
        q.put((t0, time.monotonic()))


def test_builds_in_several_processes_take_turns(pf):
    # the ranks of one job may all find the library stale: the build lock lets
    # one process compile at a time (the others then find it fresh)
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_hold_build_lock, args=(q,)) for _ in range(3)]
    for p in procs:
        p.start()
    spans = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0, spans                       # no two holders at once
    from packed_kv_cache_b200 import build
    assert build.build() == build.LIB                # fresh: returns without taking the lock


def test_binding_structs_and_constants_match_the_header(pf, tmp_path):
    # every ctypes struct field at the offset the C compiler gives it, the same
    # sizes, and the same numeric constants (a mismatch would corrupt every call)
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("needs gcc")
    structs = {"pf_config": pf.Config, "pf_select_opts": pf.SelectOpts, "pf_layer_info": pf.LayerInfo}
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "pf.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    consts = ["PF_PART_SINK", "PF_PART_MID", "PF_PART_RECENT", "PF_ROUTE_SCORE", "PF_ROUTE_SCORES_ONLY",
              "PF_ROUTE_GIVEN", "PF_ROUTE_FIFO"] + list(pf.STATUS.values())
    for name in consts:
        lines.append(f'  printf("const {name} %d\\n", (int)({name}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        a, b, v = line.split()
        got[(a, b)] = int(v)
    for cname, cls in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert got[(cname, field)] == getattr(cls, field).offset, (cname, field)
    py = {"PF_PART_SINK": pf.PART_SINK, "PF_PART_MID": pf.PART_MID, "PF_PART_RECENT": pf.PART_RECENT,
          "PF_ROUTE_SCORE": pf.ROUTE_SCORE, "PF_ROUTE_SCORES_ONLY": pf.ROUTE_SCORES_ONLY,
          "PF_ROUTE_GIVEN": pf.ROUTE_GIVEN, "PF_ROUTE_FIFO": pf.ROUTE_FIFO}
    py.update({name: code for code, name in pf.STATUS.items()})
    for name in consts:
        assert got[("const", name)] == py[name], name


def _c_kind(decl: str) -> str:
    decl = decl.strip()
    if "*" in decl:
        return "pointer"
    words = decl.replace("const", "").split()
    base = " ".join(words[:-1]) if len(words) > 1 else words[0]
    return {"int": "int", "pf_status": "int", "unsigned": "unsigned", "unsigned int": "unsigned",
            "size_t": "size_t", "float": "float", "long long": "long long"}[base]


def _ctypes_kind(t) -> str:
    if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and isinstance(t._type_, type):
        return "pointer"
    return {ctypes.c_int: "int", ctypes.c_uint: "unsigned", ctypes.c_size_t: "size_t",
            ctypes.c_float: "float", ctypes.c_longlong: "long long"}[t]


def test_binding_argtypes_match_the_prototypes(pf):
    # each declared function: the same number of parameters, each of the same
    # kind (pointer, int, unsigned, size_t, long long, float), and the same result kind
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = re.findall(r"([A-Za-z_][\w ]*?\**)\s*\b(pf_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text)
    assert len(protos) == len(declared_functions())
    for ret, name, params in protos:
        f = getattr(pf.lib, name)
        assert f.argtypes is not None, name
        kinds = [] if params.strip() in ("", "void") else [_c_kind(p) for p in params.split(",")]
        assert kinds == [_ctypes_kind(t) for t in f.argtypes], name
        assert _c_kind(ret + " r") == _ctypes_kind(f.restype), name


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    # importing the binding from a copy without libpf.so must raise, not fall back
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "packed_kv_cache_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "packed_kv_cache_b200", "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import packed_kv_cache_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libpf.so" in r.stderr


def test_attend_tail_plan(pf):
    # the pages-scale layer on 148 SMs: 288 pairs leave 8 SMs idle in the
    # last wave; each of the 12 ragged tiles gets two 73-tile chunks for them
    # and 12 small chunks for the end (about one per SM)
    assert pf.pf_attend_tail_plan(288, 12, 219, 148) == (2, 12, 146)
    assert pf.pf_attend_tail_plan(576, 24, 219, 148) == (2, 6, 146)
    # no ragged tiles, or one key tile: nothing to split
    assert pf.pf_attend_tail_plan(288, 0, 219, 148) == (1, 0, 219)
    assert pf.pf_attend_tail_plan(288, 12, 1, 148) == (1, 0, 1)
    # more tails than scratch slots for two chunks each: not split
    assert pf.pf_attend_tail_plan(0, 200, 100, 148) == (1, 0, 100)
    import random
    rng = random.Random(5)
    for _ in range(3000):
        F, T, n, sms = rng.randint(0, 3000), rng.randint(1, 300), rng.randint(1, 6000), rng.choice([1, 7, 148, 160])
        big, small, split = pf.pf_attend_tail_plan(F, T, n, sms)
        K = big + small
        assert 1 <= K <= 16 and (K == 1 or T * K <= 256)
        bounds = [c * split // big for c in range(big)] + [split + c * (n - split) // small for c in range(small)]
        bounds.append(n)
        assert bounds[0] == 0 and all(a < b for a, b in zip(bounds, bounds[1:]))   # every chunk has key tiles
    for bad in ((-1, 1, 1, 1), (1, -1, 1, 1), (1, 1, -1, 1), (1, 1, 1, 0)):
        with pytest.raises(pf.PFError):
            pf.pf_attend_tail_plan(*bad)
