"""Reference oracle for the packed-KV-cache context-attention path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline
leg of ``bench.py`` may call it.  It shares no code with the CUDA library.

Plain, slow, obviously correct float64 numpy.  Every function follows one
passage of the PackForcing pages; "PackForcing (arXiv)" below means the arXiv
HTML page "PackForcing: Short Video Training Suffices for Long Video Sampling
and Long Context Inference", and "PackForcing digest" means the Chinese
summary page of the same paper (sections 前置知识 / 方法步骤详情).

Readings of points the pages leave open (the pages' display equations were
lost in extraction; the digest restates most of them):

* Block score.  The digest gives the affinity phi_j = sum_i q_i^T k_j / sqrt(d)
  per key j.  A mid block's score is the mean of phi over its n_c keys and
  over all heads, normalised by the number of queries:
  S_p = (1/H) sum_h qbar_h . kbar_{p,h} / sqrt(d_h).  Sum and mean give the
  same ranking; one selection per (batch item, layer) is shared by all heads.
* Ranking.  Larger S first, equal S broken by the lower block index; the
  chosen indices are returned in ascending (chronological) order.  The
  comparison is made on float32 values, the precision the GPU decides in.
* RoPE.  Complex pairs are adjacent dims (2k, 2k+1); the temporal axis owns
  dims 0-43 (22 pairs), height 44-85, width 86-127 (21 pairs each);
  theta_{a,k} = base^(-2k / d_a) with d_a = 44, 42, 42; the rotation for
  position p is e^{+i theta p}.
* Attention.  No mask: every query of the current block sees the whole
  bounded context, the current block included; scale 1/sqrt(d_h).

Parity unpinned: nothing here.  Every function is pinned by the tests in
``tests/test_oracle.py`` (pages' arithmetic, the RoPE identity, brute force,
closed forms and a library attention routine).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "token_counts", "dense_context_tokens", "kv_bytes",
    "rope_thetas", "rope_encode", "rope_shift",
    "select_scores", "select_scores_bruteforce", "select_topk", "selection_margin", "select_fifo",
    "attend", "attend_loops", "merge_partials", "cache_partitions",
    "to_f64", "round_bf16",
]


# --------------------------------------------------------------------------
# helpers: exact bf16 widening and round-to-nearest-even narrowing
# --------------------------------------------------------------------------

def to_f64(x) -> np.ndarray:
    """Widen a bf16/fp32 torch tensor or a numpy array to float64 (exact)."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), once.

    Returned as float64.  bf16 keeps 8 significant bits; the values this
    oracle handles are normal numbers, far from bf16's range limits.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


# --------------------------------------------------------------------------
# token arithmetic
# --------------------------------------------------------------------------

def token_counts(block_frames: int, h: int, w: int, n_sink_frames: int,
                 n_recent_frames: int, n_mid: int) -> dict:
    """Tokens per block, per compressed block, and the bounded context size.

    n   = B_f * h * w                          (PackForcing (arXiv), "KV Caching")
    N_c = floor(B_f/2) floor(h/4) floor(w/4)   ("Compressed Mid Tokens")
    |C| = N_sink/B_f * n + N_mid * N_c + (N_recent/B_f + 1) * n
                                               ("Bounded Attention Context";
                                                PackForcing digest, step (5))
    """
    n = block_frames * h * w
    n_c = (block_frames // 2) * (h // 4) * (w // 4)
    ctx = (n_sink_frames // block_frames) * n + n_mid * n_c \
        + (n_recent_frames // block_frames + 1) * n
    return {"n": n, "n_c": n_c, "context": ctx}


def compressed_tokens_latent(T: int, H: int, W: int) -> int:
    """N_c = floor(T/2) floor(H/8) floor(W/8) over the latent grid
    (PackForcing (arXiv), "Feature Fusion")."""
    return (T // 2) * (H // 8) * (W // 8)


def dense_context_tokens(blocks: int, n: int) -> int:
    """Full, uncompressed context of ``blocks`` generated blocks: the growth
    the pages quote as about 749K tokens for a 2-minute 832x480 16-FPS video
    (PackForcing digest, KV-cache paragraph; the blog post "PackForcing:
    Rethinking the Training-Generation Length Paradigm in Video Diffusion",
    "The Memory Wall in Autoregressive Video Generation")."""
    return blocks * n


def kv_bytes(tokens: int, hidden: int, layers: int, bytes_per_elem: int = 2) -> int:
    """Bytes of K and V for ``tokens`` tokens over ``layers`` layers: the
    pages' roughly 138 GB for that full context over 30 layers (same passages
    as ``dense_context_tokens``)."""
    return tokens * hidden * 2 * bytes_per_elem * layers


def cache_partitions(num_blocks: int, sink_blocks: int, recent_blocks: int,
                     capacity: int) -> dict:
    """Which generated blocks each partition holds after ``num_blocks`` blocks.

    Sink: the first N_sink/B_f blocks, never compressed or evicted
    (PackForcing (arXiv), "Sink Tokens").  Recent: the last N_recent/B_f
    finished blocks at full resolution ("Recent & Current Tokens").  Mid:
    the compressed copies of the blocks in between, at most ``capacity`` of
    them, the oldest evicted first ("The Position Misalignment Problem";
    "Dual-Resolution Shifting Mechanism").  Blocks are numbered from 0 in
    generation order; lists are oldest first.
    """
    sink = list(range(min(num_blocks, sink_blocks)))
    rest = list(range(len(sink), num_blocks))
    recent = rest[len(rest) - min(len(rest), recent_blocks):]
    aged = rest[:len(rest) - len(recent)]
    mid = aged[len(aged) - min(len(aged), capacity):]
    return {"sink": sink, "mid": mid, "recent": recent, "evicted": len(aged) - len(mid)}


# --------------------------------------------------------------------------
# 3D RoPE and the incremental temporal shift
# --------------------------------------------------------------------------

def rope_thetas(split=(44, 42, 42), base: float = 10000.0):
    """Per-axis rotary frequencies theta_{a,k} = base^(-2k/d_a), k < d_a/2.

    The 44+42+42 = 128 split per head and the order (temporal, height, width)
    are from PackForcing (arXiv), "The Position Misalignment Problem", and the
    digest's RoPE paragraph.
    """
    return tuple(np.array([base ** (-2.0 * k / d) for k in range(d // 2)], dtype=np.float64)
                 for d in split)


def _rotate_pairs(x: np.ndarray, lo: int, angles: np.ndarray) -> np.ndarray:
    """Multiply the complex numbers x[..., lo+2k] + i x[..., lo+2k+1] by e^{i angle_k}.

    ``angles`` broadcasts against x[..., 0] with a trailing pair axis.
    """
    out = x.copy()
    for k in range(angles.shape[-1]):
        a = angles[..., k]
        c, s = np.cos(a), np.sin(a)
        re = x[..., lo + 2 * k]
        im = x[..., lo + 2 * k + 1]
        out[..., lo + 2 * k] = re * c - im * s
        out[..., lo + 2 * k + 1] = re * s + im * c
    return out


def rope_encode(k_raw, t, y, x, split=(44, 42, 42), base: float = 10000.0) -> np.ndarray:
    """k_cached = k_raw (.) e^{i theta p} with p = (t, y, x) per token.

    PackForcing digest, RoPE paragraph (k^(p)_cached = k_raw (.) e^{i theta p});
    PackForcing (arXiv), "The Position Misalignment Problem".
    ``k_raw`` is [..., 128]; t, y, x broadcast against k_raw[..., 0].
    """
    k = to_f64(k_raw)
    th_t, th_h, th_w = rope_thetas(split, base)
    d_t, d_h, _ = split
    t = np.asarray(t, dtype=np.float64)[..., None]
    y = np.asarray(y, dtype=np.float64)[..., None]
    x = np.asarray(x, dtype=np.float64)[..., None]
    k = _rotate_pairs(k, 0, t * th_t)
    k = _rotate_pairs(k, d_t, y * th_h)
    k = _rotate_pairs(k, d_t + d_h, x * th_w)
    return k


def rope_shift(keys, delta, split=(44, 42, 42), base: float = 10000.0) -> np.ndarray:
    """k' = k (.) e^{i(theta_t delta, 1_h, 1_w)}: rotate only the temporal pairs.

    PackForcing (arXiv), "Incremental RoPE adjustment"; digest, step (4).
    Dims split[0]..127 are returned unchanged.  ``delta`` is in latent frames.
    """
    k = to_f64(keys)
    th_t = rope_thetas(split, base)[0]
    return _rotate_pairs(k, 0, float(delta) * th_t)


# --------------------------------------------------------------------------
# dynamic top-k context selection
# --------------------------------------------------------------------------

def select_scores(Q, pool_K, q_stride: int = 1, heads=None, heads_norm=None) -> np.ndarray:
    """Block scores S[b, p] = (1/H) sum_h qbar_{b,h} . kbar_{b,p,h} / sqrt(d_h).

    Q: [B, n, H, D] current-block queries.  pool_K: [B, P, n_c, H, D], the
    compressed mid keys, oldest block first.  Mean-pooling both sides is the
    digest's phi_j = sum_i q_i^T k_j / sqrt(d) (step (3)) summed over the
    block's keys and averaged over heads, divided by n * n_c (the ranking is
    unchanged).

    The digest's limitations paragraph says the selection subsamples the
    query tokens and uses half of the heads to stay cheap, without saying
    how; the options read that as: queries 0, q_stride, 2 q_stride, ... only;
    heads [lo, hi) only (heads = (lo, hi)); and the head sum divided by
    heads_norm (default: the number of heads used), so that scores of
    disjoint head ranges divided by the total head count add up to the
    all-head score.
    """
    q = to_f64(Q)[:, ::q_stride]
    k = to_f64(pool_K)
    lo, hi = heads if heads is not None else (0, q.shape[2])
    q = q[:, :, lo:hi]
    k = k[:, :, :, lo:hi]
    D = q.shape[3]
    Hn = heads_norm if heads_norm else hi - lo
    qbar = q.mean(axis=1)                         # [B, H', D]
    kbar = k.mean(axis=2)                         # [B, P, H', D]
    return np.einsum("bhd,bphd->bp", qbar, kbar) / (Hn * math.sqrt(D))


def select_fifo(count: int, n_top: int) -> np.ndarray:
    """FIFO routing: the min(n_top, count) most recent of `count` live blocks,
    ascending age (PackForcing (arXiv), "FIFO vs. Dynamic Context Selection":
    chronological retention, the baseline of dynamic selection)."""
    k = min(n_top, count)
    return np.arange(count - k, count, dtype=np.int64)


def select_scores_bruteforce(Q, pool_K) -> np.ndarray:
    """The same scores as the token-level double sum sum_i sum_j q_i . k_j.

    The digest's affinity phi_j = sum_i q_i^T k_j / sqrt(d) (PackForcing
    digest, step (3)) written out term by term, summed over the block's keys
    and averaged over heads and queries as in ``select_scores``.  Small inputs
    only: one explicit q_i . k_j dot product per (i, j, h).
    """
    q = to_f64(Q)
    k = to_f64(pool_K)
    B, n, H, D = q.shape
    P, nc = k.shape[1], k.shape[2]
    S = np.zeros((B, P))
    for b in range(B):
        for p in range(P):
            acc = 0.0
            for h in range(H):
                # all query-key dot products of this head, then their sum
                acc += float(np.sum(q[b, :, h, :] @ k[b, p, :, h, :].T))
            S[b, p] = acc / (n * nc * H * math.sqrt(D))
    return S


def select_topk(scores, n_top: int) -> np.ndarray:
    """Indices of the n_top largest scores per row, ascending.

    Ranking is by (-S_p, p): equal scores go to the lower (older) block.
    Unselected blocks stay in the pool (PackForcing (arXiv), "Compressed Mid
    Tokens": the active set S_mid of N_mid blocks; digest step (3)).  With
    P <= n_top every block is selected.  Scores are compared as float32.
    """
    S = np.asarray(scores, dtype=np.float64).astype(np.float32)
    B, P = S.shape
    k = min(n_top, P)
    out = np.zeros((B, k), dtype=np.int64)
    for b in range(B):
        order = sorted(range(P), key=lambda p: (-float(S[b, p]), p))
        out[b] = np.sort(np.array(order[:k], dtype=np.int64))
    return out


def selection_margin(scores, n_top: int) -> np.ndarray:
    """Relative gap (S_(k) - S_(k+1)) / max_p |S_p| per row, k = n_top.

    Not a step of the method: the gap that decides when a selection is far
    enough from a tie for an exact comparison (the selection margin's reading
    as a scale-free gap).  Infinite when every block is selected.
    """
    S = np.asarray(scores, dtype=np.float64)
    B, P = S.shape
    out = np.full(B, np.inf)
    if P <= n_top or n_top == 0:
        return out
    for b in range(B):
        s = np.sort(S[b])[::-1]
        out[b] = (s[n_top - 1] - s[n_top]) / np.max(np.abs(S[b]))
    return out


# --------------------------------------------------------------------------
# attention over the bounded context
# --------------------------------------------------------------------------

def attend(Q, parts, scale=None, rows=None, chunk: int = 256):
    """softmax(Q K^T / sqrt(d_h)) V over the concatenation of ``parts``.

    PackForcing digest, KV-cache paragraph (Attn(Q_i, C) = softmax(Q K /
    sqrt(d_h)) V); PackForcing (arXiv), "Bounded Attention Context" (the
    context is the concatenation sink || selected mid || recent || current).

    Q: [B, Lq, H, D].  parts: list of (K, V) pairs, each [B, L_j, H, D]; their
    order is the context order.  Two passes over the partitions: the row max,
    then sum(exp) and sum(exp * V).  Returns (O [B, Lq, H, D], lse [B, H, Lq])
    in float64, lse in natural-log units of the scaled scores.  ``rows``
    selects a subset of query rows (each query is independent).
    """
    q = to_f64(Q)
    if rows is not None:
        q = q[:, np.asarray(rows)]
    B, Lq, H, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    Ks = [to_f64(K) for K, _ in parts]
    Vs = [to_f64(V) for _, V in parts]
    O = np.zeros((B, Lq, H, D))
    lse = np.zeros((B, H, Lq))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, Lq, chunk):
                qb = q[b, r0:r0 + chunk, h, :]
                s_parts = [qb @ K[b, :, h, :].T * scale for K in Ks]
                m = np.full(qb.shape[0], -np.inf)
                for s in s_parts:                 # pass 1: row max
                    if s.shape[1]:
                        m = np.maximum(m, s.max(axis=1))
                l = np.zeros(qb.shape[0])
                acc = np.zeros((qb.shape[0], D))
                for s, V in zip(s_parts, Vs):     # pass 2: sums
                    e = np.exp(s - m[:, None])
                    l += e.sum(axis=1)
                    acc += e @ V[b, :, h, :]
                O[b, r0:r0 + chunk, h, :] = acc / l[:, None]
                lse[b, h, r0:r0 + chunk] = m + np.log(l)
    return O, lse


def attend_loops(Q, K, V, scale=None):
    """Brute-force twin of ``attend`` on one explicit K/V: plain loops.

    The attention of the digest's KV-cache paragraph, softmax(Q K^T /
    sqrt(d_h)) V, one explicit sum per query, key and dim.  Tiny inputs only.
    Q [Lq, D], K [Lk, D], V [Lk, D] for one head.
    """
    q, k, v = to_f64(Q), to_f64(K), to_f64(V)
    Lq, D = q.shape
    Lk = k.shape[0]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    O = np.zeros((Lq, D))
    lse = np.zeros(Lq)
    for i in range(Lq):
        s = [sum(q[i, d] * k[j, d] for d in range(D)) * scale for j in range(Lk)]
        m = max(s)
        w = [math.exp(sj - m) for sj in s]
        tot = sum(w)
        for d in range(D):
            O[i, d] = sum(w[j] * v[j, d] for j in range(Lk)) / tot
        lse[i] = m + math.log(tot)
    return O, lse


def merge_partials(outs, lses):
    """Combine attention results over disjoint key sets by their LSEs.

    Not a step the pages state: the identity that softmax attention over a
    union of disjoint key sets is the LSE-weighted mix of the attention over
    each set, used to check the partitioned form against the concatenated one.
    O = sum_j exp(lse_j - lse) O_j with lse = log sum_j exp(lse_j).
    outs: list of [B, Lq, H, D]; lses: list of [B, H, Lq].
    """
    L = np.stack(lses)                            # [J, B, H, Lq]
    m = L.max(axis=0)
    w = np.exp(L - m)                             # [J, B, H, Lq]
    tot = w.sum(axis=0)
    O = sum(np.transpose(w[j], (0, 2, 1))[..., None] * outs[j] for j in range(len(outs)))
    return O / np.transpose(tot, (0, 2, 1))[..., None], m + np.log(tot)
