// select.cu -- dynamic top-k context selection over the compressed mid pool.
//
// PackForcing digest, method step (3): the affinity phi_j = sum_i q_i^T k_j
// / sqrt(d) of the current block's queries with the compressed keys ranks
// the mid blocks; the N_top best are routed into attention, the rest stay
// archived (PackForcing (arXiv), "Compressed Mid Tokens").  Summed over a
// block's keys and averaged over heads this is
//   S[b, p] = sum_{j, h, d} qsum[b, h, d] * Kc[b, p, j, h, d] / (n n_c H sqrt(D)),
// qsum = sum of the block's queries.  By linearity this is also
//   S[b, p] = qsum[b] . kbar[b, p] / (n H sqrt(D)),  kbar = the block's mean key,
// so when the cache keeps each compressed block's mean key (computed once,
// when the block enters the pool) scoring reads 6 KB per block instead of its
// n_c keys.  That path is two kernels: qsum_slab_kernel sums the block's
// queries (CTAs own a 256-column slab of the H*D query vector and a chunk of
// its rows; the last chunk of a slab adds the chunks in a fixed order), and
// score_cached_kernel, launched as a programmatic dependent so that it
// fetches the mean keys while the sums are formed, takes one dot product per
// block (a warp each) and, in the last CTA of a batch item (ticket), selects
// the n_top largest scores exactly (ties to the older block: warp sorting
// networks for n_top <= 32, a radix select above), writes the selection in
// ascending age, and clears its ticket.  The
// allocation-free entry point has no cached means and streams the keys:
//   1. qpool: the columns of Q[b] summed over the block's rows into qsum[b].
//   2. score: one CTA per 32-row chunk of a pool block, a dot product with
//      qsum[b]; the last CTA of batch item b (ticket counter) adds the chunks
//      of each block in a fixed order and runs the same top-k.
#include <cuda_bf16.h>

#include <cmath>
#include <cstddef>
#include <mutex>

#include "pf.h"
#include "pf_internal.h"

namespace pf {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void acc_bf16x8(float* acc, const uint4& w) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&v[q]);
    acc[2 * q] += __low2float(x);
    acc[2 * q + 1] += __high2float(x);
  }
}

__device__ __forceinline__ float dot_bf16x8(const uint4& w, const float* q) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&v[e]);
    s = fmaf(__low2float(x), q[2 * e], s);
    s = fmaf(__high2float(x), q[2 * e + 1], s);
  }
  return s;
}

// qsum[b] = column sums of Q[b] (the block's n queries).  CTA (x, b) owns
// the 16-byte column groups [2x, 2x + 2) (one 32-byte sector of every row)
// and sums them over all n rows of batch item b: no atomics, qsum[b] is
// written, not accumulated.
// kQcPhases row phases, each thread keeps kQcLoads row loads in flight; two
// CTAs per SM.
constexpr int kQcThreads = 512;
constexpr int kQcPhases = kQcThreads / 2;
constexpr int kQcLoads = 6;   // row loads in flight per thread
__global__ void __launch_bounds__(kQcThreads, 2) qpool_kernel(const SelectArgs a) {
  const int b = blockIdx.y;
  const int G = a.HD / 8;
  const int t = threadIdx.x;
  const int g = blockIdx.x * 2 + (t & 1);
  const int phase = t >> 1;
  const uint4* Q = static_cast<const uint4*>(a.Q) + static_cast<long long>(b) * a.n * G + g;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  // pooled rows: 0, q_stride, 2 q_stride, ... (nr of them)
  const int nr = (a.n + a.q_stride - 1) / a.q_stride;
  if (g < G) {
    const long long stride = static_cast<long long>(kQcPhases) * a.q_stride * G;
    const uint4* q = Q + static_cast<long long>(phase) * a.q_stride * G;
    for (int r = phase; r < nr; r += kQcLoads * kQcPhases, q += kQcLoads * stride) {
      uint4 w[kQcLoads];
#pragma unroll
      for (int k = 0; k < kQcLoads; ++k)
        w[k] = r + k * kQcPhases < nr ? __ldg(q + k * stride) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int k = 0; k < kQcLoads; ++k) acc_bf16x8(acc, w[k]);
    }
  }
  // reduce the row phases: warp shuffles over the 16 phases of a warp, then
  // the 16 warps' partials through shared memory
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int off = 2; off < 32; off <<= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  __shared__ float red[kQcThreads / 32][2][8];
  const int lane = t & 31, warp = t >> 5;
  if (lane < 2) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane][e] = acc[e];
  }
  __syncthreads();
  if (t < 16) {
    const int col = t >> 3, e = t & 7;
    float s = 0.f;
    for (int w = 0; w < kQcThreads / 32; ++w) s += red[w][col][e];
    const int gg = blockIdx.x * 2 + col;
    if (gg < G) a.qsum[static_cast<long long>(b) * a.HD + gg * 8 + e] = s;
  }
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive prefix sum over the block; returns this thread's offset, *total the sum
__device__ unsigned block_exclusive_scan(unsigned v, unsigned* total) {
  __shared__ unsigned warp_sums[kThreads / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  unsigned before = 0, tot = 0;
  for (int k = 0; k < kThreads / 32; ++k) {
    if (k < w) before += warp_sums[k];
    tot += warp_sums[k];
  }
  __syncthreads();
  *total = tot;
  return before + x - v;
}

// The last CTA of batch item b: block scores from the partial sums, exact
// selection of the n_top largest (ties to the older block), outputs in
// ascending age, and the cleanup that leaves ticket[b] zero.
__device__ void select_topk_from_keys(const SelectArgs& a, int b, uint32_t* keys);

// Block score q from its partial sums, in part order; stored as a sort key
// and written out.
__device__ __forceinline__ void put_score(const SelectArgs& a, int b, uint32_t* keys, int q, float s) {
  s *= a.score_scale;
  keys[q] = order_key(s);
  a.scores[static_cast<long long>(b) * a.slots + q] = s;
  if (a.scores_out) a.scores_out[static_cast<long long>(b) * a.count + q] = s;
}

__device__ void select_tail(const SelectArgs& a, int b, uint32_t* keys) {
  const int t = threadIdx.x;
  const int count = a.count;
  const float* pb = a.partial + static_cast<long long>(b) * a.partial_ld;
  if (a.chunks_per_block == 1) {
    // one partial per block: a thread's next eight loaded before any score
    // is stored (the stores could otherwise alias the next loads)
    constexpr int kBatch = 8;
    for (int q0 = t; q0 < count; q0 += kThreads * kBatch) {
      float s[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int q = q0 + u * kThreads;
        s[u] = q < count ? __ldcg(pb + static_cast<long long>(q) * a.p_stride) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int q = q0 + u * kThreads;
        if (q < count) put_score(a, b, keys, q, 0.f + s[u]);   // 0 + s: the sum the loop below forms
      }
    }
  } else {
    for (int q = t; q < count; q += kThreads) {
      const float* pp = pb + static_cast<long long>(q) * a.p_stride;
      float s = 0.f;
      for (int k = 0; k < a.chunks_per_block; ++k) s += __ldcg(pp + static_cast<long long>(k) * a.k_stride);
      put_score(a, b, keys, q, s);
    }
  }
  select_topk_from_keys(a, b, keys);
}

// ---- top-k of at most 32: warp-level bitonic networks ----
// A block's rank value packs its sort key above (2^32 - 1 - q), so larger is
// preferred: a higher score, then the older block (smaller q).  The values
// are distinct, so the k largest are exactly the radix select's choice.

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int j) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), j);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), j);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v), src);
  const uint32_t hi = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), src);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Four independent warp lists (one value per lane each) sorted descending
// over the lanes (lane 0 the largest).  Bitonic network, stage (k, j): lane
// and lane ^ j compare; the lower lane keeps the larger value where
// (lane & k) == 0 (a descending run), the smaller elsewhere.
__device__ __forceinline__ void warp_sort4_desc(uint64_t* v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint64_t o = shfl_xor_u64(v[u], j);
        v[u] = keep_max ? (v[u] > o ? v[u] : o) : (v[u] < o ? v[u] : o);
      }
    }
  }
}

// The 32 largest of two descending warp lists, descending: the lane-wise
// maximum of x and y reversed holds them as a bitonic sequence, which five
// half-cleaner stages sort.
__device__ __forceinline__ uint64_t warp_merge_desc(uint64_t x, uint64_t y, int lane) {
  const uint64_t yr = shfl_u64(y, 31 - lane);
  uint64_t m = x > yr ? x : yr;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t o = shfl_xor_u64(m, j);
    m = ((lane & j) == 0) ? (m > o ? m : o) : (m < o ? m : o);
  }
  return m;
}

// The k_sel <= 32 largest of keys[0 .. count), written in ascending age.
// Each warp folds its 32-key batches (four at a time, sorted side by side)
// into its running 32 largest; warp 0 merges the eight warps' lists, and
// each of the winners finds its output position by counting the winners
// older than it.
__device__ void select_topk_warp(const SelectArgs& a, int b, const uint32_t* keys, int k_sel) {
  __shared__ uint64_t lists[kThreads / 32][32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int count = a.count;
  __syncthreads();   // keys[] was written by every thread
  uint64_t best = 0ull;   // 0 ranks below every real block
  for (int qb = warp * 32; qb < count; qb += 4 * kThreads) {   // warp-uniform
    uint64_t v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = qb + u * kThreads + lane;
      v[u] = q < count ? (static_cast<uint64_t>(keys[q]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(q)) : 0ull;
    }
    warp_sort4_desc(v, lane);
    const uint64_t m = warp_merge_desc(warp_merge_desc(v[0], v[1], lane), warp_merge_desc(v[2], v[3], lane), lane);
    best = warp_merge_desc(best, m, lane);
  }
  lists[warp][lane] = best;
  __syncthreads();
  if (warp == 0) {
    uint64_t l[kThreads / 32];
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) l[w] = lists[w][lane];
    const uint64_t m0 = warp_merge_desc(l[0], l[1], lane), m1 = warp_merge_desc(l[2], l[3], lane);
    const uint64_t m2 = warp_merge_desc(l[4], l[5], lane), m3 = warp_merge_desc(l[6], l[7], lane);
    const uint64_t top = warp_merge_desc(warp_merge_desc(m0, m1, lane), warp_merge_desc(m2, m3, lane), lane);
    const uint32_t q = 0xFFFFFFFFu - static_cast<uint32_t>(top);
    int pos = 0;
#pragma unroll
    for (int s = 0; s < 32; ++s) {
      const uint32_t qs = __shfl_sync(0xffffffffu, q, s);
      pos += (s < k_sel && qs < q) ? 1 : 0;
    }
    if (lane < k_sel) {
      a.sel_slots[static_cast<long long>(b) * a.n_top + pos] = (a.head + static_cast<int>(q)) % a.slots;
      if (a.sel_out) a.sel_out[static_cast<long long>(b) * k_sel + pos] = static_cast<int>(q);
    }
  }
}

// keys[0 .. count) hold the block scores' sort keys (scores already written).
// Radix select on 8-bit digits of the keys, most significant first: each
// pass counts the digits of the keys that still match the prefix (warp-
// aggregated shared-memory atomics), then warp 0 scans the 256 counts and
// picks the digit holding the need-th largest key.  Two block barriers per
// pass (the next pass's histogram is cleared during this one).  Then one
// block scan of the packed (above-threshold, equal) counts gives every
// thread's first output position: selected blocks are the keys above the
// threshold T and the `need` oldest equal to it, written in ascending age.
__device__ void select_topk_from_keys(const SelectArgs& a, int b, uint32_t* keys) {
  __shared__ unsigned hist[2][256];
  __shared__ unsigned sh_prefix, sh_need;
  static_assert(kThreads == 256, "one histogram bin per thread");
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int count = a.count;
  if (!a.topk) {   // scores only
    if (t == 0) a.ticket[b] = 0u;
    return;
  }
  const int k_sel = min(a.n_top, count);
  const bool take_all = (k_sel == count);
  if (!take_all && k_sel <= 32) {
    select_topk_warp(a, b, keys, k_sel);
    if (t == 0) a.ticket[b] = 0u;
    return;
  }
  hist[0][t] = 0u;
  hist[1][t] = 0u;
  if (t == 0) {
    sh_prefix = 0u;
    sh_need = static_cast<unsigned>(k_sel);
  }
  __syncthreads();
  if (!take_all) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      unsigned* h = hist[pass & 1];
      const unsigned pre = sh_prefix;
      // warp-aggregated: one shared-memory atomic per distinct digit per warp
      // (the keys' leading digits are mostly equal)
      for (int q0 = 0; q0 < count; q0 += kThreads) {
        const int q = q0 + t;
        const uint32_t key = q < count ? keys[q] : 0u;
        const bool take = q < count && (shift == 24 || (key >> (shift + 8)) == (pre >> (shift + 8)));
        const unsigned digit = (key >> shift) & 255u;
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (take) {
          const unsigned grp = __match_any_sync(m, digit);
          if (lane == __ffs(grp) - 1) atomicAdd(&h[digit], static_cast<unsigned>(__popc(grp)));
        }
      }
      hist[(pass + 1) & 1][t] = 0u;   // the next pass's histogram (last read two barriers ago)
      __syncthreads();
      if (warp == 0) {
        // lane l: digits 255 - 8 l - i, i = 0..7 (descending over the warp)
        unsigned c[8], sum = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          c[i] = h[255 - 8 * lane - i];
          sum += c[i];
        }
        unsigned incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        unsigned before = incl - sum;   // keys whose digit is above this lane's digits
        const unsigned need = sh_need;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (before < need && before + c[i] >= need) {   // exactly one (lane, i)
            sh_prefix = pre | (static_cast<unsigned>(255 - 8 * lane - i) << shift);
            sh_need = need - before;
          }
          before += c[i];
        }
      }
      __syncthreads();
    }
  }
  const uint32_t T = sh_prefix;
  const unsigned need = sh_need;
  const int per = (count + kThreads - 1) / kThreads;
  const int lo = min(count, t * per), hi = min(count, lo + per);
  unsigned gt = 0u, eq = 0u;
  for (int q = lo; q < hi; ++q) {
    const uint32_t key = keys[q];
    if (take_all || key > T) ++gt;
    else if (key == T) ++eq;
  }
  unsigned tot;
  // counts <= 8,192 each: 16 bits apiece
  const unsigned packed = block_exclusive_scan((gt << 16) | eq, &tot);
  const unsigned gt_before = packed >> 16, eq_before = packed & 0xffffu;
  unsigned pos = gt_before + min(eq_before, need);
  unsigned e = eq_before;
  for (int q = lo; q < hi; ++q) {
    const uint32_t key = keys[q];
    const bool s = take_all || key > T || (key == T && e++ < need);
    if (s) {
      a.sel_slots[static_cast<long long>(b) * a.n_top + pos] = (a.head + q) % a.slots;
      if (a.sel_out) a.sel_out[static_cast<long long>(b) * k_sel + pos] = q;
      ++pos;
    }
  }
  if (t == 0) a.ticket[b] = 0u;
}

__global__ void __launch_bounds__(kThreads, 5) score_kernel(const SelectArgs a) {
  extern __shared__ float smem[];
  float* qs = smem;                                      // [HD]
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + a.HD);  // [count]
  __shared__ float red[kThreads / 32];
  __shared__ unsigned is_last;

  const int b = blockIdx.y;
  const int p = blockIdx.x / a.chunks_per_block;
  const int c = blockIdx.x % a.chunks_per_block;
  const int t = threadIdx.x;
  const int G = a.HD / 8;

  for (int i = t; i < a.HD; i += kThreads) qs[i] = a.qsum[static_cast<long long>(b) * a.HD + i];
  __syncthreads();

  const int slot = (a.head + p) % a.slots;
  const int row_lo = c * a.chunk_rows;
  const int rows = min(a.n_c, row_lo + a.chunk_rows) - row_lo;
  const uint4* K = static_cast<const uint4*>(a.pool_k) +
                   ((static_cast<long long>(b) * a.slots + slot) * a.n_c + row_lo) * G;
  const int nu = rows * G;
  float acc = 0.f;
  constexpr int U = 6;
  for (int u0 = t; u0 < nu; u0 += kThreads * U) {
    uint4 w[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int u = u0 + k * kThreads;
      if (u < nu) w[k] = __ldg(K + u);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int u = u0 + k * kThreads;
      if (u < nu) acc += dot_bf16x8(w[k], qs + (u % G) * 8);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((t & 31) == 0) red[t >> 5] = acc;
  __syncthreads();
  if (t == 0) {
    float s = 0.f;
    for (int k = 0; k < kThreads / 32; ++k) s += red[k];
    a.partial[static_cast<long long>(b) * a.partial_ld + static_cast<long long>(p) * a.chunks_per_block + c] = s;
    __threadfence();
    const unsigned total = static_cast<unsigned>(a.count * a.chunks_per_block);
    is_last = (atomicAdd(&a.ticket[b], 1u) == total - 1u) ? 1u : 0u;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  select_tail(a, b, keys);
}

// The cache path's selection: two kernels, the second launched as a
// programmatic dependent of the first so that it starts (and fetches the
// mean keys, which do not depend on the first) while the first still runs.
//
// qsum_slab_kernel, CTA (x, b): slab x / R of the score's column range
// [d_lo, d_hi) (kGroups * 8 columns: 256, or 128 when the range is an odd
// number of heads), row chunk x % R of the pooled query rows (R =
// a.row_chunks).  A warp reads 32 / kGroups whole rows of the slab per load
// instruction (512 contiguous bytes of a row at 256 columns).  Column sums of
// the chunk's rows go to qsum[b, chunk]; the chunk that finishes last (slab
// ticket) adds the R chunk sums in chunk order into qtot[b] and clears the
// ticket.
constexpr int kSelLoads = 8;   // row loads in flight per thread
template <int kGroups>
__global__ void __launch_bounds__(kThreads, 2) qsum_slab_kernel(const SelectArgs a) {
  // let the scoring kernel be scheduled now: it waits for this grid's
  // completion before reading qtot
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int kCols = kGroups * 8;
  constexpr int kPhases = kThreads / kGroups;
  __shared__ float red[kThreads / 32][kCols];
  __shared__ unsigned is_last;
  const int b = blockIdx.y;
  const int R = a.row_chunks;
  const int slab = blockIdx.x / R, rc = blockIdx.x - slab * R;
  const int col0 = a.d_lo + slab * kCols;
  const int G = a.HD / 8;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // thread t owns 16-byte group t % kGroups of the slab in row phase t / kGroups
  const int g = t % kGroups, phase = t / kGroups;
  const int nr = (a.n + a.q_stride - 1) / a.q_stride;   // pooled rows 0, q_stride, 2 q_stride, ...
  const int r_lo = static_cast<int>(static_cast<long long>(rc) * nr / R);
  const int r_hi = static_cast<int>(static_cast<long long>(rc + 1) * nr / R);
  const uint4* Q = static_cast<const uint4*>(a.Q) + static_cast<long long>(b) * a.n * G + col0 / 8 + g;
  const long long row_step = static_cast<long long>(a.q_stride) * G;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = r_lo + phase; r < r_hi; r += kSelLoads * kPhases) {
    uint4 w[kSelLoads];
#pragma unroll
    for (int k = 0; k < kSelLoads; ++k) {
      const int rr = r + k * kPhases;
      w[k] = rr < r_hi ? __ldg(Q + rr * row_step) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kSelLoads; ++k) acc_bf16x8(acc, w[k]);
  }
  // lanes of a warp with the same group (32 / kGroups row phases)
#pragma unroll
  for (int off = kGroups; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (lane < kGroups) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = acc[e];
  }
  __syncthreads();
  if (t < kCols) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) sum += red[w][t];
    a.qsum[(static_cast<long long>(b) * kSelMaxRowChunks + rc) * a.HD + col0 + t] = sum;
    __threadfence();
  }
  __syncthreads();
  if (t == 0) {
    __threadfence();
    unsigned* tk = a.slab_ticket + static_cast<long long>(b) * (a.HD / kSelSlabCols) + slab;
    is_last = (atomicAdd(tk, 1u) == static_cast<unsigned>(R - 1)) ? 1u : 0u;
    if (is_last) *tk = 0u;   // every chunk of this slab has arrived: ready for the next launch
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (t < kCols) {
    // the R chunk sums in chunk order, all of them in flight at once
    const float* src = a.qsum + static_cast<long long>(b) * kSelMaxRowChunks * a.HD + col0 + t;
    float v[kSelMaxRowChunks];
#pragma unroll
    for (int k = 0; k < kSelMaxRowChunks; ++k) v[k] = k < R ? __ldcg(src + static_cast<long long>(k) * a.HD) : 0.f;
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < kSelMaxRowChunks; ++k)
      if (k < R) sum += v[k];
    a.qtot[static_cast<long long>(b) * a.HD + col0 + t] = sum;
  }
}

// score_cached_kernel, CTA (x, b): warp w scores live block p = 8 x + w,
// qtot[b] . kbar[b, slot(p)] over [d_lo, d_hi) (the whole mean key read by
// the warp in 512-byte coalesced steps; the first kPreLoads steps issued
// before waiting for qsum_slab_kernel); the last CTA of batch item b
// (ticket) runs the top-k.
constexpr int kPreLoads = 12;   // float4 loads per lane issued before the wait (all of them at 12 heads)
__global__ void __launch_bounds__(kThreads, 2) score_cached_kernel(const SelectArgs a) {
  extern __shared__ float smem[];
  float* qs = smem;                                           // [HD] qtot[b] (only [d_lo, d_hi) is read)
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + a.HD);  // [count], the last CTA's top-k
  __shared__ unsigned is_last;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x * (kThreads / 32) + warp;
  const int v_lo = a.d_lo / 4, v_hi = a.d_hi / 4;
  const float4* k4 = nullptr;
  float4 y[kPreLoads];
  if (p < a.count) {
    int slot = a.head + p;
    if (slot >= a.slots) slot -= a.slots;
    k4 = reinterpret_cast<const float4*>(a.kbar + (static_cast<long long>(b) * a.slots + slot) * a.HD);
#pragma unroll
    for (int u = 0; u < kPreLoads; ++u) {
      const int i = v_lo + lane + 32 * u;
      y[u] = i < v_hi ? __ldg(k4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  // the query sums of qsum_slab_kernel: complete and visible after this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = a.d_lo + threadIdx.x; i < a.d_hi; i += kThreads) qs[i] = __ldcg(a.qtot + static_cast<long long>(b) * a.HD + i);
  __syncthreads();
  if (p < a.count) {
    const float4* q4 = reinterpret_cast<const float4*>(qs);
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < kPreLoads; ++u) {
      const int i = v_lo + lane + 32 * u;
      if (i < v_hi) {
        const float4 x = q4[i];
        acc = fmaf(x.x, y[u].x, fmaf(x.y, y[u].y, fmaf(x.z, y[u].z, fmaf(x.w, y[u].w, acc))));
      }
    }
    // more heads than the prefetch covers: the rest, eight loads in flight
    for (int i0 = v_lo + lane + 32 * kPreLoads; i0 < v_hi; i0 += 32 * 8) {
      float4 z[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + 32 * u;
        z[u] = i < v_hi ? __ldg(k4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + 32 * u;
        if (i < v_hi) {
          const float4 x = q4[i];
          acc = fmaf(x.x, z[u].x, fmaf(x.y, z[u].y, fmaf(x.z, z[u].z, fmaf(x.w, z[u].w, acc))));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) a.partial[static_cast<long long>(b) * a.partial_ld + p] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    is_last = (atomicAdd(&a.ticket[b], 1u) == gridDim.x - 1u) ? 1u : 0u;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  select_tail(a, b, keys);
}

// kbar[b, slot] = mean over the block's n_c keys.  CTA (slot, b, z): four
// 16-byte column groups (32 dims) starting at group 4 z; thread t sums group
// t % 4 over rows t / 4, t / 4 + 64, ... (all of a thread's rows in flight
// for blocks of up to 256 rows), then a fixed-order reduction over the 64
// row phases.  One appended block is HD / 32 CTAs (48 at 12 heads).
constexpr int kMeanGroups = 4;
constexpr int kMeanPhases = kThreads / kMeanGroups;
__global__ void __launch_bounds__(kThreads) kmean_kernel(const void* pool_k, float* kbar, int slots, int n_c,
                                                         int HD, int slot0) {
  __shared__ float red[kThreads / 32][kMeanGroups][8];
  const int b = blockIdx.y;
  const int slot = slot0 + blockIdx.x;
  const int G = HD / 8;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int gl = t % kMeanGroups, phase = t / kMeanGroups;
  const int g = blockIdx.z * kMeanGroups + gl;
  const uint4* K = static_cast<const uint4*>(pool_k) + (static_cast<long long>(b) * slots + slot) * n_c * G + g;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (g < G) {
    for (int r0 = phase; r0 < n_c; r0 += 4 * kMeanPhases) {
      uint4 w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r0 + k * kMeanPhases;
        w[k] = r < n_c ? __ldg(K + static_cast<long long>(r) * G) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) acc_bf16x8(acc, w[k]);
    }
  }
  // lanes with the same group: l, l ^ 4, l ^ 8, ... (eight row phases per warp)
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 4);
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  }
  if (lane < kMeanGroups) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane][e] = acc[e];
  }
  __syncthreads();
  if (t < kMeanGroups * 8) {
    const int gg = t / 8, e = t % 8;
    const int go = blockIdx.z * kMeanGroups + gg;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) sum += red[w][gg][e];
    if (go < G) kbar[(static_cast<long long>(b) * slots + slot) * HD + go * 8 + e] = sum / static_cast<float>(n_c);
  }
}

}  // namespace

// Top-k of given scores, one CTA per batch item (a.partial = the scores).
__global__ void __launch_bounds__(kThreads) topk_given_kernel(const SelectArgs a) {
  extern __shared__ float smem[];
  select_tail(a, blockIdx.x, reinterpret_cast<uint32_t*>(smem));
}

// The k = min(n_top, count) most recent live blocks, ascending age.
__global__ void fifo_kernel(const SelectArgs a) {
  const int b = blockIdx.x;
  const int k = min(a.n_top, a.count);
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const int q = a.count - k + i;
    a.sel_slots[static_cast<long long>(b) * a.n_top + i] = (a.head + q) % a.slots;
    if (a.sel_out) a.sel_out[static_cast<long long>(b) * k + i] = q;
  }
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  if (a.count <= 0) return cudaSuccess;
  dim3 g1((a.HD / 8 + 1) / 2, a.B);
  qpool_kernel<<<g1, kQcThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = static_cast<size_t>(a.HD) * 4 + static_cast<size_t>(a.count) * 4;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 g2(a.count * a.chunks_per_block, a.B);
  score_kernel<<<g2, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_select_cached(const SelectArgs& a, cudaStream_t st) {
  if (a.count <= 0) return cudaSuccess;
  const int cols = a.d_hi - a.d_lo;
  const int slab_cols = select_slab_cols(a.d_lo, a.d_hi);
  const int nslabs = cols / slab_cols;
  if (nslabs <= 0 || a.row_chunks < 1 || a.row_chunks > kSelMaxRowChunks || a.chunks_per_block != 1)
    return cudaErrorInvalidValue;
  if (slab_cols == 256)
    qsum_slab_kernel<32><<<dim3(nslabs * a.row_chunks, a.B), kThreads, 0, st>>>(a);
  else
    qsum_slab_kernel<16><<<dim3(nslabs * a.row_chunks, a.B), kThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = static_cast<size_t>(a.HD) * 4 + static_cast<size_t>(a.count) * 4;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(score_cached_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // a programmatic dependent launch: scheduled while qsum_slab_kernel runs,
  // it waits (griddepcontrol.wait) for that grid before reading its sums
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.count + kThreads / 32 - 1) / (kThreads / 32), a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_cached_kernel, a);
}

cudaError_t launch_topk_given(const SelectArgs& a, cudaStream_t st) {
  if (a.count <= 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(a.count) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_given_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  topk_given_kernel<<<a.B, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_select_fifo(const SelectArgs& a, cudaStream_t st) {
  if (a.count <= 0) return cudaSuccess;
  fifo_kernel<<<a.B, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_kmean(const void* pool_k, float* kbar, int B, int slots, int n_c, int HD, int slot0, int nslots,
                         cudaStream_t st) {
  if (nslots <= 0) return cudaSuccess;
  kmean_kernel<<<dim3(nslots, B, (HD / 8 + kMeanGroups - 1) / kMeanGroups), kThreads, 0, st>>>(pool_k, kbar, slots,
                                                                                               n_c, HD, slot0);
  return cudaGetLastError();
}


// ---------------------------------------------------------------------------
// Selection with no device allocation.
//
// Some callers cannot allocate device memory for this library: a serving
// process that reserves its whole device-memory budget at start-up and
// forbids allocation on the request path (cudaMalloc/cudaFree can
// synchronise the device and fragment the pool), or a host framework that
// owns the device allocator and hands this code only its input and output
// tensors, with no cache arena.  pf_select_mid_static serves them: the
// selection's scratch (query sums, per-chunk partial scores, block scores,
// slot list, tickets) lives in the file-scope array below, which every GPU
// that loads the library holds until the process exits.
namespace {

constexpr int kStaticBatch = PF_STATIC_MAX_BATCH;
constexpr int kStaticHD = PF_STATIC_MAX_HEADS * kHeadDim;
constexpr int kStaticBlocks = PF_STATIC_MAX_BLOCKS;
constexpr int kStaticChunks = (PF_STATIC_MAX_NC + 31) / 32;

struct StaticSelectScratch {
  float qsum[kStaticBatch * kStaticHD];
  unsigned ticket[64];
  float scores[kStaticBatch * kStaticBlocks];
  int32_t sel_slots[kStaticBatch * kStaticBlocks];
  float partial[kStaticBatch * kStaticBlocks * kStaticChunks];
};

static __device__ __align__(256) unsigned char g_select_scratch[sizeof(StaticSelectScratch)];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device.  In host code
// the array's name is a host-side stand-in, so the address is asked for once
// per device, with that device current.
cudaError_t static_scratch(StaticSelectScratch** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<StaticSelectScratch*>(g_scratch_addr[dev]);
  return cudaSuccess;
}

}  // namespace

extern "C" pf_status pf_select_mid_static(const void* Q, int batch, int n, int heads, const void* pool_k,
                                          int pool_slots, int n_c, int head, int count, int n_top, int32_t* sel_out,
                                          float* scores_out, void* stream) {
  using pf::report_error;
  if (Q == nullptr || pool_k == nullptr || sel_out == nullptr)
    return static_cast<pf_status>(report_error(PF_ERR_ARG, "Q, pool_k and sel_out must not be NULL"));
  if (reinterpret_cast<uintptr_t>(Q) % 16 != 0 || reinterpret_cast<uintptr_t>(pool_k) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(sel_out) % 4 != 0 ||
      (scores_out != nullptr && reinterpret_cast<uintptr_t>(scores_out) % 4 != 0))
    return static_cast<pf_status>(report_error(PF_ERR_ARG, "misaligned pointer"));
  if (batch < 1 || n < 1 || heads < 1 || n_c < 1 || count < 0 || n_top < 0 || pool_slots < count ||
      (pool_slots > 0 && (head < 0 || head >= pool_slots)))
    return static_cast<pf_status>(report_error(PF_ERR_ARG, "bad sizes (batch %d, n %d, heads %d, n_c %d, "
                                                            "slots %d, head %d, count %d, n_top %d)",
                                               batch, n, heads, n_c, pool_slots, head, count, n_top));
  if (batch > kStaticBatch || heads > PF_STATIC_MAX_HEADS || count > kStaticBlocks || n_c > PF_STATIC_MAX_NC)
    return static_cast<pf_status>(report_error(
        PF_ERR_CAPACITY, "pf_select_mid_static handles batch <= %d, heads <= %d, count <= %d, n_c <= %d",
        kStaticBatch, PF_STATIC_MAX_HEADS, kStaticBlocks, PF_STATIC_MAX_NC));
  // the kernels index partial[] and scores[] with the pool's slot count as stride
  if (static_cast<long long>(batch) * pool_slots > kStaticBlocks * static_cast<long long>(kStaticBatch))
    return static_cast<pf_status>(report_error(PF_ERR_CAPACITY, "batch * pool_slots must be <= %d",
                                               kStaticBlocks * kStaticBatch));
  if (count == 0 || (n_top == 0 && scores_out == nullptr)) return PF_OK;
  StaticSelectScratch* sc = nullptr;
  cudaError_t e = static_scratch(&sc);
  if (e != cudaSuccess)
    return static_cast<pf_status>(report_error(PF_ERR_CUDA, "static scratch address: %s", cudaGetErrorString(e)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int HD = heads * kHeadDim;
  // query sums and tickets must start at zero; they are contiguous
  static_assert(offsetof(StaticSelectScratch, ticket) == sizeof(float) * kStaticBatch * kStaticHD, "layout");
  e = cudaMemsetAsync(sc, 0, offsetof(StaticSelectScratch, scores), st);
  if (e != cudaSuccess)
    return static_cast<pf_status>(report_error(PF_ERR_CUDA, "clear static scratch: %s", cudaGetErrorString(e)));
  SelectArgs a;
  a.Q = Q;
  a.B = batch;
  a.n = n;
  a.HD = HD;
  a.qsum = sc->qsum;
  a.pool_k = pool_k;
  a.kbar = nullptr;   // no cached mean keys: stream the pool
  a.slots = pool_slots;
  a.n_c = n_c;
  a.head = head;
  a.count = count;
  a.chunk_rows = 32;
  a.chunks_per_block = (n_c + 31) / 32;
  a.score_scale = static_cast<float>(1.0 / (static_cast<double>(n) * n_c * heads * sqrt(128.0)));
  a.partial = sc->partial;
  a.scores = sc->scores;
  a.ticket = sc->ticket;
  a.n_top = n_top < count ? n_top : count;
  a.sel_slots = sc->sel_slots;
  a.sel_out = sel_out;
  a.scores_out = scores_out;
  a.q_stride = 1;
  a.d_lo = 0;
  a.d_hi = HD;
  a.topk = n_top > 0 ? 1 : 0;   // n_top == 0: the scores only
  a.partial_ld = pool_slots * a.chunks_per_block;
  a.p_stride = a.chunks_per_block;
  a.k_stride = 1;
  a.slab_ticket = nullptr;
  a.qtot = nullptr;
  a.row_chunks = 1;
  e = launch_select(a, st);
  if (e != cudaSuccess)
    return static_cast<pf_status>(report_error(PF_ERR_CUDA, "select launch: %s", cudaGetErrorString(e)));
  return PF_OK;
}

}  // namespace pf
