"""Python binding of libpf, the packed-KV-cache C ABI (include/pf.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory (the cache arena and the tensors)
and the current CUDA stream.  Importing this package fails if the library has
not been built (``python -m packed_kv_cache_b200.build``); there is no
fallback.

Functions keep the C names (``pf_cache_create``, ``pf_select_mid``, ...);
``PackedKVCache`` wraps them for one cache.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "PFError", "Config", "LayerInfo", "PART_SINK", "PART_MID", "PART_RECENT",
    "lib", "library_path", "pf_version", "pf_cache_bytes", "pf_cache_create", "pf_cache_destroy",
    "pf_cache_layer_info", "pf_cache_append_block", "pf_cache_load_mid", "pf_select_mid",
    "pf_rope_shift", "pf_attend", "pf_poll_device_error", "pf_selftest_wait_timeout",
    "pf_select_mid_static", "pf_select_mid_ex", "SelectOpts", "pf_attend_step", "pf_finish_block",
    "pf_cache_state_bytes", "pf_cache_save_state", "pf_cache_load_state",
    "ROUTE_SCORE", "ROUTE_SCORES_ONLY", "ROUTE_GIVEN", "ROUTE_FIFO",
    "PackedKVCache", "config_for",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libpf.so")

PART_SINK, PART_MID, PART_RECENT = 1, 2, 4
ROUTE_SCORE, ROUTE_SCORES_ONLY, ROUTE_GIVEN, ROUTE_FIFO = 0, 1, 2, 3
STATUS = {0: "PF_OK", 1: "PF_ERR_ARG", 2: "PF_ERR_ARENA", 3: "PF_ERR_STATE", 4: "PF_ERR_CAPACITY",
          5: "PF_ERR_CUDA", 6: "PF_ERR_TIMEOUT", 7: "PF_ERR_UNSUPPORTED"}


class PFError(RuntimeError):
    """A library call returned a status other than PF_OK; carries the status
    code, its name and the library's message for the calling thread."""

    def __init__(self, func: str, status: int, message: str):
        self.status = status
        self.status_name = STATUS.get(status, str(status))
        super().__init__(f"{func}: {self.status_name}: {message}")


class Config(ctypes.Structure):
    """pf_config: the cache's shape (layers, batch, heads, block geometry,
    partition sizes, routed count, rotary split and base)."""
    _fields_ = [("layers", ctypes.c_int), ("batch", ctypes.c_int), ("heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("block_frames", ctypes.c_int), ("h", ctypes.c_int),
                ("w", ctypes.c_int), ("sink_blocks", ctypes.c_int), ("recent_blocks", ctypes.c_int),
                ("mid_capacity", ctypes.c_int), ("n_top", ctypes.c_int),
                ("rope_split", ctypes.c_int * 3), ("rope_base", ctypes.c_float),
                ("sink_rope_in_attention", ctypes.c_int)]


class SelectOpts(ctypes.Structure):
    """pf_select_opts: routing policy, query stride, head range, score divisor."""
    _fields_ = [("policy", ctypes.c_int), ("q_stride", ctypes.c_int), ("head_lo", ctypes.c_int),
                ("head_hi", ctypes.c_int), ("heads_total", ctypes.c_int), ("scores_in", ctypes.c_void_p)]


class LayerInfo(ctypes.Structure):
    """pf_layer_info: one layer's ring state and the device addresses of its
    partitions."""
    _fields_ = [("blocks_seen", ctypes.c_int), ("sink_filled", ctypes.c_int),
                ("recent_count", ctypes.c_int), ("recent_head", ctypes.c_int),
                ("mid_count", ctypes.c_int), ("mid_head", ctypes.c_int), ("pool_slots", ctypes.c_int),
                ("selection_valid", ctypes.c_int), ("n_selected", ctypes.c_int),
                ("context_tokens", ctypes.c_int), ("evicted", ctypes.c_longlong),
                ("total_shift", ctypes.c_longlong),
                ("sink_k", ctypes.c_void_p), ("sink_v", ctypes.c_void_p),
                ("pool_k", ctypes.c_void_p), ("pool_v", ctypes.c_void_p),
                ("recent_k", ctypes.c_void_p), ("recent_v", ctypes.c_void_p),
                ("selection", ctypes.c_void_p), ("scores", ctypes.c_void_p)]

    def as_dict(self) -> dict:
        """The fields by name."""
        return {name: getattr(self, name) for name, _ in self._fields_}


def _build_from_sources() -> None:
    """A checkout with the library's sources: compile the library (nvcc,
    sm_100a) if it is missing or older than a source, before loading.
    build.py is loaded by path so that this package is not imported again; a
    failed build raises."""
    from importlib.util import module_from_spec, spec_from_file_location
    spec = spec_from_file_location("_packed_kv_cache_b200_build", os.path.join(_HERE, "build.py"))
    mod = module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def _load():
    if os.path.isdir(os.path.join(_HERE, "csrc")):
        _build_from_sources()
    if not os.path.exists(library_path):
        raise ImportError(f"{library_path} is missing: build it with `python -m packed_kv_cache_b200.build`")
    L = ctypes.CDLL(library_path)
    vp, i32, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    sig = {
        "pf_version": ([], ctypes.c_int),
        "pf_last_error": ([], ctypes.c_char_p),
        "pf_status_string": ([i32], ctypes.c_char_p),
        "pf_cache_bytes": ([ctypes.POINTER(Config), ctypes.POINTER(ctypes.c_size_t)], i32),
        "pf_cache_create": ([ctypes.POINTER(Config), vp, ctypes.c_size_t, vp, ctypes.POINTER(vp)], i32),
        "pf_cache_destroy": ([vp], i32),
        "pf_cache_layer_info": ([vp, i32, ctypes.POINTER(LayerInfo)], i32),
        "pf_cache_append_block": ([vp, i32, vp, vp, vp, vp, ctypes.POINTER(i32), vp], i32),
        "pf_cache_load_mid": ([vp, i32, vp, vp, i32, ctypes.POINTER(i32), vp], i32),
        "pf_select_mid": ([vp, i32, vp, vp, vp, vp], i32),
        "pf_select_mid_ex": ([vp, i32, vp, ctypes.POINTER(SelectOpts), vp, vp, vp], i32),
        "pf_rope_shift": ([vp, i32, u32, i32, vp], i32),
        "pf_attend": ([vp, i32, vp, vp, vp, vp, vp, vp], i32),
        "pf_attend_tail_plan": ([ctypes.c_longlong, i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                 ctypes.POINTER(i32)], i32),
        "pf_poll_device_error": ([vp, vp, ctypes.POINTER(u32)], i32),
        "pf_selftest_wait_timeout": ([vp, u32, vp], i32),
        "pf_select_mid_static": ([vp, i32, i32, i32, vp, i32, i32, i32, i32, i32, vp, vp, vp], i32),
        "pf_attend_step": ([vp, i32, i32, vp, vp, vp, vp, vp, vp], i32),
        "pf_cache_state_bytes": ([vp, ctypes.POINTER(ctypes.c_size_t)], i32),
        "pf_cache_save_state": ([vp, vp, ctypes.c_size_t], i32),
        "pf_cache_load_state": ([vp, vp, ctypes.c_size_t], i32),
        "pf_finish_block": ([vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                             ctypes.POINTER(vp), ctypes.POINTER(i32), vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()


def _check(func: str, status: int) -> None:
    if status != 0:
        raise PFError(func, status, lib.pf_last_error().decode(errors="replace"))


def _dev(t, name: str):
    """Device address of a CUDA tensor (None stays None)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return int(t)
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _expect(t, name: str, dtype, min_numel: int) -> None:
    """Refuse a tensor of the wrong element type, or with fewer elements than
    the call reads or writes: the library sees only its address."""
    if t is None or not isinstance(t, torch.Tensor):
        return
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if t.numel() < min_numel:
        raise ValueError(f"{name} has {t.numel()} elements; the call needs at least {min_numel}")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def config_for(wl, layers: int | None = None, sink_rope_in_attention: bool = False) -> Config:
    """A pf_config for a workload description (``synth.Workload`` or alike)."""
    c = Config()
    c.sink_rope_in_attention = 1 if sink_rope_in_attention else 0
    c.layers = layers if layers is not None else getattr(wl, "layers", 1)
    c.batch, c.heads, c.head_dim = wl.batch, wl.heads, wl.head_dim
    c.block_frames, c.h, c.w = wl.block_frames, wl.h, wl.w
    c.sink_blocks, c.recent_blocks = wl.sink_blocks, wl.recent_blocks
    c.mid_capacity, c.n_top = wl.mid_capacity, wl.n_top
    c.rope_split[0], c.rope_split[1], c.rope_split[2] = wl.rope_split
    c.rope_base = wl.rope_base
    return c


# ---------------------------------------------------------------- C-named calls

def pf_version() -> int:
    """Library version (100 = 0.1.0)."""
    return lib.pf_version()


def pf_cache_bytes(cfg: Config) -> int:
    """Arena bytes a cache of this configuration needs (token counts as in
    PackForcing (arXiv), "KV Caching" and "Compressed Mid Tokens")."""
    out = ctypes.c_size_t()
    _check("pf_cache_bytes", lib.pf_cache_bytes(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def pf_cache_create(cfg: Config, arena, arena_bytes: int | None = None, stream=None) -> ctypes.c_void_p:
    """A cache over a caller-owned, 256-byte aligned device arena (zeroed on
    `stream`); returns the handle."""
    ptr = _dev(arena, "arena")
    nbytes = arena_bytes if arena_bytes is not None else arena.numel() * arena.element_size()
    handle = ctypes.c_void_p()
    _check("pf_cache_create", lib.pf_cache_create(ctypes.byref(cfg), ptr, nbytes, _stream(stream),
                                                  ctypes.byref(handle)))
    return handle


def pf_cache_destroy(handle) -> None:
    """Free the cache's host state (the arena stays the caller's)."""
    _check("pf_cache_destroy", lib.pf_cache_destroy(handle))


def pf_cache_layer_info(handle, layer: int) -> dict:
    """Snapshot of one layer's state as a dict (LayerInfo fields)."""
    info = LayerInfo()
    _check("pf_cache_layer_info", lib.pf_cache_layer_info(handle, layer, ctypes.byref(info)))
    return info.as_dict()


def pf_cache_append_block(handle, layer, K, V, Kc=None, Vc=None, stream=None) -> int:
    """Append the finished block (PackForcing (arXiv), "Dual-Resolution
    Shifting Mechanism"): sink until full, then recent, its compressed copy
    joining the mid pool when it leaves; returns the blocks evicted (0 or 1)."""
    ev = ctypes.c_int(0)
    _check("pf_cache_append_block", lib.pf_cache_append_block(
        handle, layer, _dev(K, "K"), _dev(V, "V"), _dev(Kc, "Kc"), _dev(Vc, "Vc"), ctypes.byref(ev),
        _stream(stream)))
    return ev.value


def pf_cache_load_mid(handle, layer, Kc, Vc, nblocks: int, stream=None) -> int:
    """Push `nblocks` compressed blocks straight into the mid pool, oldest
    first; returns the blocks evicted."""
    ev = ctypes.c_int(0)
    _check("pf_cache_load_mid", lib.pf_cache_load_mid(handle, layer, _dev(Kc, "Kc"), _dev(Vc, "Vc"),
                                                      nblocks, ctypes.byref(ev), _stream(stream)))
    return ev.value


def pf_select_mid(handle, layer, Q, sel_out=None, scores_out=None, stream=None) -> None:
    """Dynamic context selection (PackForcing digest, method step (3)): score
    every live compressed block against the block's queries, keep the n_top
    best (ties to the older block) for the layer's attention."""
    _check("pf_select_mid", lib.pf_select_mid(handle, layer, _dev(Q, "Q"), _dev(sel_out, "sel_out"),
                                              _dev(scores_out, "scores_out"), _stream(stream)))


def pf_select_mid_ex(handle, layer, Q, policy=ROUTE_SCORE, q_stride=1, heads=None, heads_total=0,
                     scores_in=None, sel_out=None, scores_out=None, stream=None) -> None:
    """Selection with a routing policy: ROUTE_SCORE (the method, optionally on
    every q_stride-th query row and the head range `heads` = (lo, hi)),
    ROUTE_SCORES_ONLY (scores into scores_out, nothing stored), ROUTE_GIVEN
    (top-k of scores_in), ROUTE_FIFO (the newest n_top blocks)."""
    lo, hi = heads if heads is not None else (0, 0)
    o = SelectOpts(policy, q_stride, lo, hi, heads_total, _dev(scores_in, "scores_in"))
    _check("pf_select_mid_ex", lib.pf_select_mid_ex(handle, layer, _dev(Q, "Q"), ctypes.byref(o),
                                                    _dev(sel_out, "sel_out"), _dev(scores_out, "scores_out"),
                                                    _stream(stream)))


def pf_rope_shift(handle, layer: int, parts: int, delta: int, stream=None) -> None:
    """Incremental temporal RoPE adjustment (PackForcing (arXiv), "Incremental
    RoPE adjustment"): rotate the temporal pairs of the keys in `parts` by
    delta frames, in place; layer -1 = every layer."""
    _check("pf_rope_shift", lib.pf_rope_shift(handle, layer, parts, delta, _stream(stream)))


def pf_attend(handle, layer, Q, K_cur, V_cur, O, lse=None, stream=None) -> None:
    """softmax(Q K^T / sqrt(d_h)) V over sink || selected mid || recent ||
    current (PackForcing digest, KV-cache paragraph; PackForcing (arXiv),
    "Bounded Attention Context"), into O; optional natural-log LSE."""
    _check("pf_attend", lib.pf_attend(handle, layer, _dev(Q, "Q"), _dev(K_cur, "K_cur"), _dev(V_cur, "V_cur"),
                                      _dev(O, "O"), _dev(lse, "lse"), _stream(stream)))


def pf_attend_tail_plan(full_units: int, tails: int, n_tiles: int, sms: int) -> tuple:
    """(big, small, split): how pf_attend cuts the ragged last query tiles
    along the context (host arithmetic only)."""
    big, small, split = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check("pf_attend_tail_plan", lib.pf_attend_tail_plan(full_units, tails, n_tiles, sms, ctypes.byref(big),
                                                          ctypes.byref(small), ctypes.byref(split)))
    return big.value, small.value, split.value


def attend_launches(cfg, info: dict, sms: int) -> int:
    """Kernels one pf_attend call launches for a layer in state `info`
    (pf_cache_layer_info) on a GPU with `sms` SMs."""
    n = cfg.block_frames * cfg.h * cfg.w
    q_tiles = (n + 127) // 128
    if q_tiles % 2 == 0:
        return 1
    sb = lambda rows: (rows + 31) // 32  # noqa: E731
    n_c = (cfg.block_frames // 2) * (cfg.h // 4) * (cfg.w // 4)   # tokens of a compressed block
    n_sub = sb(info["sink_filled"] * n) + info["n_selected"] * sb(n_c) + info["recent_count"] * sb(n) + sb(n)
    n_tiles = (n_sub + 3) // 4
    big, small, _ = pf_attend_tail_plan(cfg.batch * cfg.heads * (q_tiles // 2), cfg.batch * cfg.heads, n_tiles, sms)
    return 1 if big + small == 1 else 2


def pf_attend_step(handle, layer, step, Q, K_cur, V_cur, O, lse=None, stream=None) -> None:
    """One layer's attention at denoising step `step` of the current block:
    the selection is made at step 0 and reused by the later steps
    (PackForcing (arXiv), "Implementation Details"; digest, limitations
    paragraph)."""
    _check("pf_attend_step", lib.pf_attend_step(handle, layer, step, _dev(Q, "Q"), _dev(K_cur, "K_cur"),
                                                _dev(V_cur, "V_cur"), _dev(O, "O"), _dev(lse, "lse"),
                                                _stream(stream)))


def _ptr_array(ts, name):
    if ts is None:
        return None
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _dev(t, f"{name}[{i}]")
    return arr


def pf_finish_block(handle, K, V, Kc=None, Vc=None, stream=None) -> int:
    """Append the finished block to every layer (one tensor per layer in each
    list) and shift every sink by the evicted blocks' frames; returns the
    blocks evicted per layer."""
    ev = ctypes.c_int(0)
    _check("pf_finish_block", lib.pf_finish_block(handle, _ptr_array(K, "K"), _ptr_array(V, "V"),
                                                  _ptr_array(Kc, "Kc"), _ptr_array(Vc, "Vc"), ctypes.byref(ev),
                                                  _stream(stream)))
    return ev.value


def pf_cache_state_bytes(handle) -> int:
    """Bytes of the cache's saved host state."""
    out = ctypes.c_size_t()
    _check("pf_cache_state_bytes", lib.pf_cache_state_bytes(handle, ctypes.byref(out)))
    return out.value


def pf_cache_save_state(handle) -> bytes:
    """The cache's host state (ring heads, counts, shifts, selection validity)
    as bytes; with a copy of the arena it restores the cache."""
    n = pf_cache_state_bytes(handle)
    buf = ctypes.create_string_buffer(n)
    _check("pf_cache_save_state", lib.pf_cache_save_state(handle, buf, n))
    return buf.raw


def pf_cache_load_state(handle, state: bytes) -> None:
    """Replace the cache's host state by a saved one (same configuration)."""
    buf = ctypes.create_string_buffer(bytes(state), len(state))
    _check("pf_cache_load_state", lib.pf_cache_load_state(handle, buf, len(state)))


def pf_poll_device_error(handle, stream=None) -> int:
    """Synchronise `stream` and read (then clear) the cache's device error
    word; raises PF_ERR_TIMEOUT if a bounded wait gave up."""
    code = ctypes.c_uint(0)
    _check("pf_poll_device_error", lib.pf_poll_device_error(handle, _stream(stream), ctypes.byref(code)))
    return code.value


def pf_selftest_wait_timeout(handle, timeout_us: int, stream=None) -> None:
    """Launch a kernel whose bounded wait on a flag nothing sets must give up
    and report it (the failure-detection path, with no GPU fault)."""
    _check("pf_selftest_wait_timeout", lib.pf_selftest_wait_timeout(handle, timeout_us, _stream(stream)))


def pf_select_mid_static(Q, batch, n, heads, pool_k, pool_slots, n_c, head, count, n_top, sel_out,
                         scores_out=None, stream=None) -> None:
    """Selection with no device allocation (scratch in a fixed array inside
    the library): for callers that cannot allocate device memory.  Tensors
    of the wrong element type, or smaller than the sizes say, are refused
    before the call (an address given as an int is passed as it is)."""
    D = 128
    _expect(Q, "Q", torch.bfloat16, batch * n * heads * D)
    _expect(pool_k, "pool_k", torch.bfloat16, batch * pool_slots * n_c * heads * D)
    _expect(sel_out, "sel_out", torch.int32, batch * min(n_top, count))
    _expect(scores_out, "scores_out", torch.float32, batch * count)
    _check("pf_select_mid_static", lib.pf_select_mid_static(
        _dev(Q, "Q"), batch, n, heads, _dev(pool_k, "pool_k"), pool_slots, n_c, head, count, n_top,
        _dev(sel_out, "sel_out"), _dev(scores_out, "scores_out"), _stream(stream)))


# ---------------------------------------------------------------- one cache

class PackedKVCache:
    """A cache over a torch-allocated arena on one CUDA device."""

    def __init__(self, cfg: Config, device="cuda", stream=None):
        self.cfg = cfg
        self.nbytes = pf_cache_bytes(cfg)
        self.arena = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.handle = pf_cache_create(cfg, self.arena, self.nbytes, stream)

    def close(self) -> None:
        """Free the host state; the arena tensor is released with the object."""
        if getattr(self, "handle", None):
            pf_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self, layer: int) -> dict:
        """One layer's state (pf_cache_layer_info)."""
        return pf_cache_layer_info(self.handle, layer)

    # sizes the calls read and write, from the configuration
    def _rows(self, rows: int) -> int:
        """Elements of a [B, rows, H, D] tensor."""
        c = self.cfg
        return c.batch * rows * c.heads * c.head_dim

    def _n(self) -> int:
        return self.cfg.block_frames * self.cfg.h * self.cfg.w

    def _n_c(self) -> int:
        c = self.cfg
        return (c.block_frames // 2) * (c.h // 4) * (c.w // 4)

    def _check_selection_buffers(self, layer, sel_out=None, scores_out=None, scores_in=None) -> None:
        if sel_out is None and scores_out is None and scores_in is None:
            return
        live = self.info(layer)["mid_count"]
        B = self.cfg.batch
        _expect(sel_out, "sel_out", torch.int32, B * min(self.cfg.n_top, live))
        _expect(scores_out, "scores_out", torch.float32, B * live)
        _expect(scores_in, "scores_in", torch.float32, B * live)

    def append_block(self, layer, K, V, Kc=None, Vc=None, stream=None) -> int:
        """K, V [B, n, H, 128] bf16; Kc, Vc [B, n_c, H, 128] bf16 (see
        pf_cache_append_block).  Returns the blocks evicted."""
        for t, name in ((K, "K"), (V, "V")):
            _expect(t, name, torch.bfloat16, self._rows(self._n()))
        for t, name in ((Kc, "Kc"), (Vc, "Vc")):
            _expect(t, name, torch.bfloat16, self._rows(self._n_c()))
        return pf_cache_append_block(self.handle, layer, K, V, Kc, Vc, stream)

    def load_mid(self, layer, Kc, Vc, stream=None) -> int:
        """Kc, Vc [B, nblocks, n_c, H, 128] bf16 into the pool (see pf_cache_load_mid)."""
        for t, name in ((Kc, "Kc"), (Vc, "Vc")):
            _expect(t, name, torch.bfloat16, self._rows(self._n_c()) * Kc.shape[1])
        return pf_cache_load_mid(self.handle, layer, Kc, Vc, Kc.shape[1], stream)

    def select_mid(self, layer, Q, sel_out=None, scores_out=None, stream=None) -> None:
        """Q [B, n, H, 128] bf16; optional sel_out [B, min(n_top, live)] int32
        and scores_out [B, live] float32 (see pf_select_mid)."""
        _expect(Q, "Q", torch.bfloat16, self._rows(self._n()))
        self._check_selection_buffers(layer, sel_out, scores_out)
        pf_select_mid(self.handle, layer, Q, sel_out, scores_out, stream)

    def select_mid_ex(self, layer, Q=None, policy=ROUTE_SCORE, q_stride=1, heads=None, heads_total=0,
                      scores_in=None, sel_out=None, scores_out=None, stream=None) -> None:
        """Selection with a routing policy (see pf_select_mid_ex)."""
        _expect(Q, "Q", torch.bfloat16, self._rows(self._n()))
        self._check_selection_buffers(layer, sel_out, scores_out, scores_in)
        pf_select_mid_ex(self.handle, layer, Q, policy, q_stride, heads, heads_total, scores_in, sel_out,
                         scores_out, stream)

    def rope_shift(self, layer, parts, delta, stream=None) -> None:
        """Shift the keys of `parts` (PART_* mask) by delta frames (see pf_rope_shift)."""
        pf_rope_shift(self.handle, layer, parts, delta, stream)

    def attend(self, layer, Q, K_cur, V_cur, O=None, lse=None, stream=None) -> torch.Tensor:
        """Q, K_cur, V_cur [B, n, H, 128] bf16 -> O (allocated if None); optional
        lse [B, H, n] float32 (see pf_attend)."""
        need = self._rows(self._n())
        for t, name in ((Q, "Q"), (K_cur, "K_cur"), (V_cur, "V_cur"), (O, "O")):
            _expect(t, name, torch.bfloat16, need)
        _expect(lse, "lse", torch.float32, need // self.cfg.head_dim)
        if O is None:
            O = torch.empty_like(Q)
        pf_attend(self.handle, layer, Q, K_cur, V_cur, O, lse, stream)
        return O

    def attend_step(self, layer, step, Q, K_cur, V_cur, O=None, lse=None, stream=None) -> torch.Tensor:
        """Attention at denoising step `step` (selection at step 0, reused
        after; see pf_attend_step)."""
        need = self._rows(self._n())
        for t, name in ((Q, "Q"), (K_cur, "K_cur"), (V_cur, "V_cur"), (O, "O")):
            _expect(t, name, torch.bfloat16, need)
        _expect(lse, "lse", torch.float32, need // self.cfg.head_dim)
        if O is None:
            O = torch.empty_like(Q)
        pf_attend_step(self.handle, layer, step, Q, K_cur, V_cur, O, lse, stream)
        return O

    def finish_block(self, K, V, Kc=None, Vc=None, stream=None) -> int:
        """Append the final block to every layer and shift the sinks (see
        pf_finish_block).  K, V, Kc, Vc: one tensor per layer."""
        L = self.cfg.layers
        for ts, name, rows in ((K, "K", self._n()), (V, "V", self._n()), (Kc, "Kc", self._n_c()),
                               (Vc, "Vc", self._n_c())):
            if ts is None:
                continue
            if len(ts) != L:
                raise ValueError(f"{name} must hold one tensor per layer ({L})")
            for t in ts:
                _expect(t, name, torch.bfloat16, self._rows(rows))
        return pf_finish_block(self.handle, K, V, Kc, Vc, stream)

    def save(self) -> tuple:
        """(host state bytes, a device copy of the arena) after the current
        stream's work; restore with PackedKVCache.restore."""
        torch.cuda.current_stream(self.arena.device).synchronize()
        return pf_cache_save_state(self.handle), self.arena.clone()

    @classmethod
    def restore(cls, cfg: Config, saved: tuple, device=None) -> "PackedKVCache":
        """A new cache holding a saved one's contents (same configuration)."""
        state, arena = saved
        c = cls(cfg, device=device if device is not None else arena.device)
        c.arena.copy_(arena)            # after the creation's clearing, on the same stream
        pf_cache_load_state(c.handle, state)
        return c

    def poll_device_error(self, stream=None) -> int:
        """See pf_poll_device_error."""
        return pf_poll_device_error(self.handle, stream)
