// attend.cu -- attention of the current block's queries over the bounded
// packed context, on 5th-generation tensor cores.
//
// PackForcing digest, KV-cache paragraph: Attn(Q_i, C) = softmax(Q_i K^T /
// sqrt(d_h)) V; PackForcing (arXiv), "Bounded Attention Context": the context
// is sink || selected mid blocks || recent || current, a fixed number of
// tokens.  The partitions are never gathered: the key/value tiles are pulled
// by TMA straight from where each partition lives.
//
// Work units, one CTA each:
//  * full unit: two 128-row query tiles of one (batch item, head) that share
//    every K/V tile of the context;
//  * tail chunk: when a block has an odd number of 128-row query tiles, the
//    last (ragged) tile of each (b, h) is split along the context into
//    chunks of K/V tiles.  Each chunk writes its unnormalised output, row
//    maximum and row sum to scratch; the chunk that finishes last merges them
//    (O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c).  The chunks run after
//    the full units: first big chunks, sized so that the SMs the last wave of
//    full units leaves idle finish them alongside it, then small chunks,
//    about one per SM, so that the launch ends within a few K/V tiles of
//    the last full unit.
// 12 warps per CTA:
//   warp 0      TMA producer: Q, then K and V tiles through rings
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T and O_t += P_t V
//   warp 2      tensor-memory allocator
//   warps 2-3   when the sink's RoPE shift is applied here: rotate the sink
//               rows of each K tile in shared memory after TMA lands it
//   warps 4-7   softmax of query tile 0 (one thread per query row)
//   warps 8-11  softmax of query tile 1
// Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each;
// P_t (bf16) is written over the first 64 columns of S_t and read by the
// P.V MMA straight from tensor memory.
//
// A K/V tile holds 128 keys assembled from four 32-row sub-boxes.  The
// context is cut into sub-boxes partition by partition (each partition, and
// each mid block, padded to a multiple of 32 rows), so a tile may straddle a
// partition boundary; rows past a partition's end are either out of the
// tensor map's bounds (zero-filled by TMA) or masked in the softmax.
// Softmax: online, in base 2, with the running maximum raised only when a
// tile's maximum exceeds it by more than 8 (P stays <= 256), in which case
// O and the row sum are rescaled.
#include <cuda_bf16.h>

#include "pf_internal.h"
#include "ptx.cuh"

namespace pf {

namespace {

constexpr int kBM = 128;           // query rows per tile
constexpr int kBN = 128;           // keys per tile
constexpr int kSub = 32;           // rows per TMA sub-box
constexpr int kKStages = 3;                   // K ring depth
constexpr int kVStages = 2;                   // V ring depth
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = kBN * kHeadDim * 2;   // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;       // 64 dims x 128 rows
constexpr uint32_t kSubBytes = kSub * 128;            // one sub-box, one 64-dim half
constexpr float kRescaleThreshold = 8.0f;
constexpr int kRotThreads = 64;   // warps 2-3

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                   // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;              // kKStages tiles
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;       // kVStages tiles
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;           // + barriers + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory");
// the MMA issuer offsets operand descriptors in their 14-bit address field
static_assert(kSmemBytes + 1024 < (1u << 18), "shared addresses fit a descriptor's address field");

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t k_ready[kKStages];   // K tile rotated (only used when rotate_sink)
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_final[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// floor(a / b) and a mod b for 0 <= a < 2^22, 0 < b, with inv_b = 1 / b: a
// float estimate of the quotient corrected by one step (integer division by
// a run-time value is a long instruction sequence, costly on the producer's
// and the softmax's paths).
__device__ __forceinline__ int div_small(int a, int b, float inv_b) {
  int q = __float2int_rz(__int2float_rn(a) * inv_b);
  const int r = a - q * b;
  if (r < 0) --q;
  else if (r >= b) ++q;
  return q;
}
__device__ __forceinline__ int mod_small(int a, int b, float inv_b) { return a - div_small(a, b, inv_b) * b; }

struct SubBox {
  int part, row0, seg, valid;
};

// Sub-box s of batch item b's context: which partition, first row, segment
// (index along the tensor map's outermost dimension), and valid rows.
// inv_mid / inv_blk = 1 / sb_mid, 1 / sb_blk.
__device__ __forceinline__ SubBox decode_subbox(const AttendParams& p, int b, int s, float inv_mid, float inv_blk) {
  SubBox r;
  if (s < p.sb_sink) {
    r.part = kPartSink; r.row0 = s * kSub; r.seg = b; r.valid = min(kSub, p.sink_rows - r.row0);
    return r;
  }
  s -= p.sb_sink;
  const int nmid = p.n_sel * p.sb_mid;
  if (s < nmid) {
    const int blk = div_small(s, p.sb_mid, inv_mid), k = s - blk * p.sb_mid;
    int slot;
    if (p.sel_slots) {
      slot = p.sel_slots[b * p.sel_stride + blk];
    } else {
      slot = p.mid_head + blk;   // < 2 pool_slots
      if (slot >= p.pool_slots) slot -= p.pool_slots;
    }
    r.part = kPartMid; r.row0 = k * kSub; r.seg = b * p.pool_slots + slot;
    r.valid = min(kSub, p.n_c - r.row0);
    return r;
  }
  s -= nmid;
  const int nrec = p.n_recent * p.sb_blk;
  if (s < nrec) {
    const int blk = div_small(s, p.sb_blk, inv_blk), k = s - blk * p.sb_blk;
    int slot = p.recent_head + blk;   // < 2 recent_slots
    if (slot >= p.recent_slots) slot -= p.recent_slots;
    r.part = kPartRecent; r.row0 = k * kSub; r.seg = b * p.recent_slots + slot;
    r.valid = min(kSub, p.n - r.row0);
    return r;
  }
  s -= nrec;
  if (s < p.sb_blk) {
    r.part = kPartCur; r.row0 = s * kSub; r.seg = b; r.valid = min(kSub, p.n - r.row0);
    return r;
  }
  // padding past the end of the context: a box fully outside the map, zero-filled
  r.part = kPartCur; r.row0 = ((p.n + kSub - 1) / kSub) * kSub; r.seg = b; r.valid = 0;
  return r;
}

// Valid rows of sub-box s (no table lookups: depends on the geometry only).
// inv_mid / inv_blk = 1 / sb_mid, 1 / sb_blk.
__device__ __forceinline__ int subbox_valid(const AttendParams& p, int s, float inv_mid, float inv_blk) {
  if (s < p.sb_sink) return min(kSub, p.sink_rows - s * kSub);
  s -= p.sb_sink;
  const int nmid = p.n_sel * p.sb_mid;
  if (s < nmid) return min(kSub, p.n_c - mod_small(s, p.sb_mid, inv_mid) * kSub);
  s -= nmid;
  const int nrec = p.n_recent * p.sb_blk;
  if (s < nrec) return min(kSub, p.n - mod_small(s, p.sb_blk, inv_blk) * kSub);
  s -= nrec;
  if (s < p.sb_blk) return min(kSub, p.n - s * kSub);
  return 0;
}

// The unit of this CTA.  The (b, h) are taken in groups of group_bh; a
// group's units are its full units ((b, h) major, then query-tile pair), then
// its ragged tiles' tail_big big chunks ((b, h) major, then chunk); after
// every group, the B*H*tail_small small chunks ((b, h) major, then chunk).
struct QTile {
  int b, h, qt;
};
struct Unit {
  QTile t[2];
  int nq;       // query tiles in the unit (1 or 2)
  int j0, j1;   // K/V tiles [j0, j1) of the context
  int tail;     // tail index ((b, h)) of a split tail, -1 otherwise
  int chunk;    // chunk index within its tail
};

__device__ __forceinline__ Unit unit_of(const AttendParams& p, int u) {
  const int pairs = p.q_tiles / 2;
  const int BH = p.B * p.H;
  const int kb = (p.q_tiles & 1) ? p.tail_big : 0;
  const int per_group = p.group_bh * (pairs + kb);
  const int grouped = BH * (pairs + kb);   // every group's pairs and big chunks
  Unit r;
  int g = 0, rem = 0, gh = 0;
  if (u < grouped) {
    g = u / per_group;
    rem = u - g * per_group;
    gh = min(p.group_bh, BH - g * p.group_bh);
  }
  if (u < grouped && rem < gh * pairs) {
    const int bh = g * p.group_bh + rem / pairs, kk = rem % pairs;
    r.t[0] = {bh / p.H, bh % p.H, 2 * kk};
    r.t[1] = {bh / p.H, bh % p.H, 2 * kk + 1};
    r.nq = 2;
    r.j0 = 0;
    r.j1 = p.n_tiles;
    r.tail = -1;
    r.chunk = 0;
  } else {
    int bh, c;
    if (u < grouped) {
      const int v = rem - gh * pairs;
      bh = g * p.group_bh + v / kb;
      c = v - (v / kb) * kb;
      r.j0 = static_cast<int>(static_cast<long long>(c) * p.tail_split / p.tail_big);
      r.j1 = static_cast<int>(static_cast<long long>(c + 1) * p.tail_split / p.tail_big);
    } else {
      const int v2 = u - grouped;
      bh = v2 / p.tail_small;
      const int cs = v2 - bh * p.tail_small;
      const int rest = p.n_tiles - p.tail_split;
      r.j0 = p.tail_split + static_cast<int>(static_cast<long long>(cs) * rest / p.tail_small);
      r.j1 = p.tail_split + static_cast<int>(static_cast<long long>(cs + 1) * rest / p.tail_small);
      c = p.tail_big + cs;
    }
    r.t[0] = {bh / p.H, bh % p.H, p.q_tiles - 1};
    r.t[1] = r.t[0];
    r.nq = 1;
    r.tail = (p.tail_chunks > 1) ? bh : -1;
    r.chunk = c;
  }
  return r;
}

__device__ __forceinline__ void mask32(uint32_t* c, int valid) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (i >= valid) c[i] = __float_as_uint(-INFINITY);
}

__device__ __forceinline__ float max64(const uint32_t* x) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 8) {
    m0 = fmax3(m0, __uint_as_float(x[c + 0]), __uint_as_float(x[c + 1]));
    m1 = fmax3(m1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
    m2 = fmax3(m2, __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
    m3 = fmax3(m3, __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
  }
  return fmax3(fmaxf(m0, m1), m2, m3);
}

// 32 scores -> 32 probabilities exp2(s * scale - m) packed as 16 bf16 pairs,
// stored to 16 TMEM columns at dst; their sum accumulated in rs2.
__device__ __forceinline__ void exp_chunk(const uint32_t* c, uint32_t dst, uint64_t sl2x2, uint64_t nmbx2,
                                          uint64_t* rs2) {
  uint32_t pk[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint64_t x = f2_fma((static_cast<uint64_t>(c[2 * e + 1]) << 32) | c[2 * e], sl2x2, nmbx2);
    const uint64_t pp = f2_pack(ex2_approx(f2_lo(x)), ex2_approx(f2_hi(x)));
    rs2[e & 1] = f2_add(rs2[e & 1], pp);
    pk[e] = pack_bf16x2(f2_lo(pp), f2_hi(pp));
  }
  tmem_st16(dst, pk);
}

__device__ __forceinline__ void store_row_bf16(uint4* dst, const float* o, float inv) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 w;
    w.x = pack_bf16x2(o[8 * v + 0] * inv, o[8 * v + 1] * inv);
    w.y = pack_bf16x2(o[8 * v + 2] * inv, o[8 * v + 3] * inv);
    w.z = pack_bf16x2(o[8 * v + 4] * inv, o[8 * v + 5] * inv);
    w.w = pack_bf16x2(o[8 * v + 6] * inv, o[8 * v + 7] * inv);
    dst[v] = w;
  }
}

__global__ void __launch_bounds__(kThreads, 1) attend_kernel(const __grid_constant__ AttendParams p) {
  // tail_merge_kernel (a programmatic dependent) may be scheduled once every
  // CTA has started; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + kOffBar);
  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sK = smem_u32(smem + kOffK);
  const uint32_t sV = smem_u32(smem + kOffV);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long lim = p.timeout_cycles;
  volatile int* abort_flag = &bars.abort;
  const Unit un = unit_of(p, blockIdx.x);
  const int nq = un.nq;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.k_ready[s], kRotThreads);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.p_full[t], kBM);
      mbar_init(&bars.o_final[t], 1);
    }
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      prefetch_tmap(&p.tm_q);
      for (int m = 0; m < 4; ++m) {
        prefetch_tmap(&p.tm_k[m]);
        prefetch_tmap(&p.tm_v[m]);
      }
      mbar_arrive_expect_tx(&bars.q_full, nq * kTileBytes);
      for (int t = 0; t < nq; ++t)
        for (int half = 0; half < 2; ++half)
          tma_load_4d(smem + kOffQ + t * kTileBytes + half * kHalfBytes, &p.tm_q, &bars.q_full, half * 64,
                      un.t[t].h, un.t[t].qt * kBM, un.t[t].b);
      const int b = un.t[0].b, h = un.t[0].h;
      const float inv_mid = 1.f / static_cast<float>(max(p.sb_mid, 1));
      const float inv_blk = 1.f / static_cast<float>(max(p.sb_blk, 1));
      int kg = 0, vg = 0;    // K / V tiles issued
      bool ok = true;
      for (int j = un.j0; ok && j < un.j1; ++j) {
        {
          const int st = kg % kKStages, use = kg / kKStages;
          if (use > 0 && !mbar_wait_bounded(&bars.k_empty[st], (use - 1) & 1, abort_flag, p.err,
                                            kDevErrTimeoutBase | 2u, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars.k_full[st], kTileBytes);
          for (int i = 0; i < 4; ++i) {
            const SubBox sb = decode_subbox(p, b, 4 * j + i, inv_mid, inv_blk);
            for (int half = 0; half < 2; ++half)
              tma_load_4d(smem + kOffK + st * kTileBytes + half * kHalfBytes + i * kSubBytes, &p.tm_k[sb.part],
                          &bars.k_full[st], half * 64, h, sb.row0, sb.seg);
          }
          ++kg;
        }
        {
          const int st = vg % kVStages, use = vg / kVStages;
          if (use > 0 && !mbar_wait_bounded(&bars.v_empty[st], (use - 1) & 1, abort_flag, p.err,
                                            kDevErrTimeoutBase | 3u, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars.v_full[st], kTileBytes);
          for (int i = 0; i < 4; ++i) {
            const SubBox sb = decode_subbox(p, b, 4 * j + i, inv_mid, inv_blk);
            for (int half = 0; half < 2; ++half)
              tma_load_4d(smem + kOffV + st * kTileBytes + half * kHalfBytes + i * kSubBytes, &p.tm_v[sb.part],
                          &bars.v_full[st], half * 64, h, sb.row0, sb.seg);
          }
          ++vg;
        }
      }
      if (!ok || *abort_flag) {
        // let every load already issued land before the CTA can exit
        const long long short_lim = lim / 4 + 1;
        mbar_wait_bounded(&bars.q_full, 0, nullptr, nullptr, 0, short_lim);
        for (int g = kg - 1; g >= 0 && g >= kg - kKStages; --g)
          mbar_wait_bounded(&bars.k_full[g % kKStages], (g / kKStages) & 1, nullptr, nullptr, 0, short_lim);
        for (int g = vg - 1; g >= 0 && g >= vg - kVStages; --g)
          mbar_wait_bounded(&bars.v_full[g % kVStages], (g / kVStages) & 1, nullptr, nullptr, 0, short_lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(kBM, kHeadDim, 1);
      // Every operand descriptor is the tile's base descriptor plus a
      // constant: the start-address field (bits 0-13) holds address / 16 and
      // shared addresses stay below 2^18 bytes, so adding an offset / 16
      // never carries out of the field.
      const uint64_t dq = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv = sdesc_sw128(sV, kHalfBytes, 1024);
      const int j0 = un.j0, j1 = un.j1, nqt = nq;
      auto issue_qk = [&](int t, int st) {
        const uint64_t qa = dq + static_cast<uint32_t>(t) * (kTileBytes >> 4);
        const uint64_t ka = dk + static_cast<uint32_t>(st) * (kTileBytes >> 4);
        const uint32_t d = tmem + static_cast<uint32_t>(t) * 128u;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = (((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
          mma_ss(d, qa + off, ka + off, idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int st, bool first) {
        const uint64_t va = dv + static_cast<uint32_t>(st) * (kTileBytes >> 4);
        const uint32_t d = tmem + 256u + static_cast<uint32_t>(t) * 128u;
        const uint32_t a = tmem + static_cast<uint32_t>(t) * 128u;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(d, a + kk * 8, va + kk * (2048 >> 4), idesc_pv, (!first || kk > 0) ? 1u : 0u);
      };
      uint64_t* k_avail = p.rotate_sink ? bars.k_ready : bars.k_full;
      // ring positions kept as slot + phase
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0;
      bool ok = mbar_wait_bounded(&bars.q_full, 0, abort_flag, p.err, kDevErrTimeoutBase | 4u, lim);
      if (ok) ok = mbar_wait_bounded(&k_avail[ks], kph, abort_flag, p.err, kDevErrTimeoutBase | 5u, lim);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < nqt; ++t) {
          issue_qk(t, ks);
          mma_commit(&bars.s_full[t]);
        }
        mma_commit(&bars.k_empty[ks]);
        if (++ks == kKStages) { ks = 0; kph ^= 1u; }
      }
      for (int j = j0; ok && j < j1; ++j) {
        const bool more = j + 1 < j1;
        const uint32_t pph = static_cast<uint32_t>(j - j0) & 1u;
        ok = mbar_wait_bounded(&bars.v_full[vs], vph, abort_flag, p.err, kDevErrTimeoutBase | 6u, lim);
        for (int t = 0; ok && t < nqt; ++t) {
          ok = mbar_wait_bounded(&bars.p_full[t], pph, abort_flag, p.err, kDevErrTimeoutBase | 7u, lim);
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, vs, j == j0);
          if (more) {
            // S_t of the next tile overwrites P_t (tcgen05 MMAs issued by
            // one thread run in issue order: P_t V has read P_t by then)
            if (t == 0) ok = mbar_wait_bounded(&k_avail[ks], kph, abort_flag, p.err, kDevErrTimeoutBase | 10u, lim);
            if (!ok) break;
            tc_fence_after();
            issue_qk(t, ks);
            mma_commit(&bars.s_full[t]);
          }
        }
        if (!ok) break;
        mma_commit(&bars.v_empty[vs]);
        if (++vs == kVStages) { vs = 0; vph ^= 1u; }
        if (more) {
          mma_commit(&bars.k_empty[ks]);
          if (++ks == kKStages) { ks = 0; kph ^= 1u; }
        }
      }
      for (int t = 0; t < nq; ++t) mma_commit(&bars.o_final[t]);
      if (!ok) {
        // make sure nothing issued is still running before the memory goes away
        mbar_wait_bounded(&bars.o_final[0], 0, nullptr, nullptr, 0, lim / 4 + 1);
      }
    }
  } else if (warp == 2 || warp == 3) {
    if (p.rotate_sink) {
      // ------------------------------------------------ sink-key rotator
      // PackForcing (arXiv), "Incremental RoPE adjustment": the sink keys'
      // temporal pairs times e^{i theta_k total_shift}, applied to the K tile
      // in shared memory (dims 0-63 half, 128-byte swizzle: 16-byte chunk c
      // of row r sits at chunk c ^ (r & 7)); the MMA issuer waits for k_ready.
      // thread rt owns 16-byte word c = rt % 8 (pairs 4c .. 4c+3, their
      // cosines and sines kept in registers) of rows rt / 8 + 8 m
      const int rt = threadIdx.x - 64;
      const int c = rt & 7, r0 = rt >> 3;
      const int sink_tiles = (p.sb_sink + 3) / 4;
      const bool active = c * 4 < p.sink_rope.pairs;
      float cs[4], sn[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        cs[q] = p.sink_rope.c[(c * 4 + q) & 31];
        sn[q] = p.sink_rope.s[(c * 4 + q) & 31];
      }
      bool ok = true;
      int kg = 0;
      for (int j = un.j0; ok && j < un.j1; ++j, ++kg) {
        const int st = kg % kKStages;
        ok = mbar_wait_bounded(&bars.k_full[st], (kg / kKStages) & 1, abort_flag, p.err, kDevErrTimeoutBase | 14u,
                               lim);
        if (!ok) break;
        if (j < sink_tiles && active) {
          const int nsb = min(4, p.sb_sink - 4 * j);   // the tile's first nsb sub-boxes are sink rows
          uint8_t* tile = smem + kOffK + st * kTileBytes;
          for (int i = 0; i < nsb; ++i) {
            uint4 w[kSub / 8];
            uint4* ptr[kSub / 8];
#pragma unroll
            for (int m = 0; m < kSub / 8; ++m) {
              const int rr = r0 + 8 * m;
              ptr[m] = reinterpret_cast<uint4*>(tile + i * kSubBytes + rr * 128 + ((c ^ (rr & 7)) << 4));
              w[m] = *ptr[m];
            }
#pragma unroll
            for (int m = 0; m < kSub / 8; ++m) {
              rope_rotate_word_cs(w[m], c, p.sink_rope.pairs, cs, sn);
              *ptr[m] = w[m];
            }
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&bars.k_ready[st]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;                 // query-tile slot
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int row = quarter * 32 + lane;           // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128u;
    const uint32_t tO = tmem + lane_off + 256u + t * 128u;
    const float sl2 = p.scale_log2;
    const float inv_mid = 1.f / static_cast<float>(max(p.sb_mid, 1));
    const float inv_blk = 1.f / static_cast<float>(max(p.sb_blk, 1));
    bool ok = t < nq;
    float m = -INFINITY;   // running max of scaled scores, base-2 units
    float l = 0.f;         // running sum of exp2(score - m)
    for (int j = un.j0; ok && j < un.j1; ++j) {
      // which columns hold real keys (most tiles: all of them); worked out
      // before S is ready, off the critical path
      const int s0 = 4 * j;
      int valid[4] = {kSub, kSub, kSub, kSub};
      const bool check = !p.exact || (s0 + 4 > p.sb_mid_lo && s0 < p.sb_mid_hi) || (s0 + 4 > p.n_sub);
      if (check) {
#pragma unroll
        for (int i = 0; i < 4; ++i) valid[i] = subbox_valid(p, s0 + i, inv_mid, inv_blk);
      }
      const bool masked = check && (valid[0] != kSub || valid[1] != kSub || valid[2] != kSub || valid[3] != kSub);
      ok = mbar_wait_bounded(&bars.s_full[t], (j - un.j0) & 1, abort_flag, p.err, kDevErrTimeoutBase | 11u, lim);
      if (!ok) break;
      tc_fence_after();
      // the whole row of S in registers: one tensor-memory round trip
      uint32_t sv[128];
      tmem_ld128_wait(tS, sv);
      if (masked) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (valid[i] < kSub) mask32(sv + 32 * i, valid[i]);
      }
      const float mt = fmaxf(max64(sv), max64(sv + 64)) * sl2;
      float alpha = 1.f;
      bool rescale_o = false;
      if (mt > m + kRescaleThreshold) {
        alpha = ex2_approx(m - mt);   // 0 when m = -inf
        l *= alpha;
        rescale_o = j > un.j0;
        m = mt;
      }
      const float mb = (m == -INFINITY) ? 0.f : m;
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nmbx2 = f2_pack(-mb, -mb);
      uint64_t rs2[2] = {0ull, 0ull};
      // P = exp2(S * scale - m) as bf16 pairs, written over S
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) exp_chunk(sv + 32 * cc, tS + cc * 16, sl2x2, nmbx2, rs2);
      {
        const uint64_t r = f2_add(rs2[0], rs2[1]);
        l += f2_lo(r) + f2_hi(r);
      }
      // O holds every P V up to the previous tile (completed before S of this
      // tile was signalled); the next P V is issued after p_full.  The
      // tensor-memory accesses are warp-collective: the whole warp takes the
      // branch when any of its rows rescales (alpha = 1 on the others).
      if (!rescale_o) alpha = 1.f;
      if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32_wait(tO + cc * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[t]);
    }
    if (ok) ok = mbar_wait_bounded(&bars.o_final[t], 0, abort_flag, p.err, kDevErrTimeoutBase | 12u, lim);
    if (ok) {
      tc_fence_after();
      const QTile qt = un.t[t];
      const int qrow = qt.qt * kBM + row;
      __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.O);
      uint4* dst = reinterpret_cast<uint4*>(O + ((static_cast<long long>(qt.b) * p.n + qrow) * p.H + qt.h) * kHeadDim);
      if (un.tail < 0) {
        const float inv = 1.f / l;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32_wait(tO + cc * 32, o);
          if (qrow < p.n) store_row_bf16(dst + cc * 4, reinterpret_cast<const float*>(o), inv);
        }
        if (p.lse != nullptr && qrow < p.n)
          p.lse[(static_cast<long long>(qt.b) * p.H + qt.h) * p.n + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
      } else {
        // tail chunk: park the unnormalised rows; tail_merge_kernel merges
        // the chunks once the whole grid is done
        const long long slot = static_cast<long long>(un.tail) * p.tail_chunks + un.chunk;
        float4* po = reinterpret_cast<float4*>(p.part_o + (slot * kBM + row) * kHeadDim);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32_wait(tO + cc * 32, o);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            po[cc * 8 + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                         __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
        }
        p.part_ml[(slot * 2 + 0) * kBM + row] = m;
        p.part_ml[(slot * 2 + 1) * kBM + row] = l;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();   // the allocating warp may have run the rotator loop
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The split ragged tiles' merge: CTA (tail, g) finishes rows 16 g .. 16 g + 15
// of tail (b, h)'s last query tile from its chunks' partial outputs,
// O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c, M = max_c m_c.  Warp w
// takes rows 2w and 2w + 1; for a row, lane c holds chunk c's statistics and
// lane l dims 4l .. 4l + 3, every chunk's piece of the row in flight at once.
__global__ void __launch_bounds__(256) tail_merge_kernel(const __grid_constant__ AttendParams p) {
  // the attention grid's partial outputs: complete and visible after this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tail = blockIdx.x;
  const int K = p.tail_chunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = tail / p.H, h = tail - b * p.H;
  const long long base = static_cast<long long>(tail) * K;
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.O);
  for (int rr = 0; rr < 2; ++rr) {
    const int row = blockIdx.y * 16 + warp * 2 + rr;
    const int qrow = (p.q_tiles - 1) * kBM + row;
    if (qrow >= p.n) continue;   // the same for the whole warp
    const float mc = lane < K ? __ldcg(p.part_ml + ((base + lane) * 2) * kBM + row) : -INFINITY;
    const float lc = lane < K ? __ldcg(p.part_ml + ((base + lane) * 2 + 1) * kBM + row) : 0.f;
    float4 x[kAttendMaxChunksPerTail];
#pragma unroll
    for (int c = 0; c < kAttendMaxChunksPerTail; ++c)
      if (c < K) x[c] = __ldcg(reinterpret_cast<const float4*>(p.part_o + ((base + c) * kBM + row) * kHeadDim) + lane);
    float M = mc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w = lane < K ? ex2_approx(mc - M) : 0.f;
    float L = w * lc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < kAttendMaxChunksPerTail; ++c) {
      const float wc = __shfl_sync(0xffffffffu, w, c);
      if (c < K) {
        acc.x = fmaf(wc, x[c].x, acc.x);
        acc.y = fmaf(wc, x[c].y, acc.y);
        acc.z = fmaf(wc, x[c].z, acc.z);
        acc.w = fmaf(wc, x[c].w, acc.w);
      }
    }
    const float inv = 1.f / L;
    uint2 v;
    v.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    v.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(O + ((static_cast<long long>(b) * p.n + qrow) * p.H + h) * kHeadDim)[lane] = v;
    if (lane == 0 && p.lse != nullptr)
      p.lse[(static_cast<long long>(b) * p.H + h) * p.n + qrow] = (M + __log2f(L)) * 0.69314718055994531f;
  }
}

__global__ void wait_timeout_kernel(unsigned* err, long long lim) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the wait must give up by itself
    mbar_wait_bounded(&bar, 0, &abort, err, kDevErrTimeoutBase | 0xFFu, lim);
  }
}

}  // namespace

TailPlan attend_tail_plan(long long F, int T, int n, int sms) {
  if (T <= 0 || n <= 0 || sms <= 0) return TailPlan{1, 0, n, T > 0 ? T : 1};
  // the groups of (b, h): as many as one wave's pairs take
  const long long P = F / T;
  long long group = P > 0 ? sms / P : T;
  if (group < 1) group = 1;
  if (group > T) group = T;
  const int Tg = static_cast<int>(group);
  const TailPlan whole{1, 0, n, Tg};
  int max_k = kAttendMaxTailSlots / T;
  if (max_k > kAttendMaxChunksPerTail) max_k = kAttendMaxChunksPerTail;
  if (max_k > n) max_k = n;
  if (max_k <= 1) return whole;
  const int per_sm = static_cast<int>((2LL * sms + T) / (2LL * T));   // round(sms / T): ~one small chunk per SM
  const int small_all = per_sm < 1 ? 1 : (per_sm > max_k ? max_k : per_sm);
  if (F <= 0) return TailPlan{0, small_all, 0, Tg};
  // a group's pairs, in waves; the SMs its last wave leaves idle
  const long long Fg = group * P;
  const long long waves = (Fg + sms - 1) / sms;
  const long long idle = sms - (Fg - (waves - 1) * sms);
  if (idle <= 0) return TailPlan{0, small_all, 0, Tg};
  // big work per tail: what the idle SMs do during one full unit's time
  const int J = static_cast<int>(idle * n / group < n ? idle * n / group : n);
  int kb = 0;
  for (int k = 1; k < max_k && k <= J; ++k) {
    // the T k big chunks, ceil(T k / idle) per idle SM, fit in n K/V tiles
    if ((group * k + idle - 1) / idle * ((J + k - 1) / k) <= n) {
      kb = k;
      break;
    }
  }
  if (kb == 0) return TailPlan{max_k, 0, n, Tg};
  const int rest = n - J;
  int ks = 0;
  if (rest > 0) {
    ks = per_sm;
    if (ks > max_k - kb) ks = max_k - kb;
    if (ks > rest) ks = rest;
    if (ks < 1) ks = 1;
  }
  return TailPlan{kb, ks, J, Tg};
}

cudaError_t launch_attend(const AttendParams& p, cudaStream_t st) {
  // once per device: the kernel's shared-memory limit is raised and the SM
  // count read
  static PerDevice sms_of;
  int sms = 0;
  cudaError_t e = sms_of.get(&sms, [](int dev, int* v) {
    cudaError_t r = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (r != cudaSuccess) return r;
    return cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
  });
  if (e != cudaSuccess) return e;
  AttendParams q = p;
  const long long bh = 1LL * p.B * p.H;
  const long long F = bh * (p.q_tiles / 2);
  const TailPlan tp = (p.q_tiles & 1) ? attend_tail_plan(F, static_cast<int>(bh), p.n_tiles, sms)
                                      : TailPlan{1, 0, p.n_tiles, static_cast<int>(bh)};
  q.tail_big = tp.big;
  q.tail_small = tp.small;
  q.tail_split = tp.split;
  q.group_bh = tp.group;
  q.tail_chunks = tp.big + tp.small;
  const long long units = F + ((p.q_tiles & 1) ? bh * q.tail_chunks : 0);
  if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
  attend_kernel<<<static_cast<unsigned>(units), kThreads, kSmemBytes, st>>>(q);
  e = cudaGetLastError();
  if (e != cudaSuccess || !(p.q_tiles & 1) || q.tail_chunks <= 1) return e;
  // the split ragged tiles' merge, a programmatic dependent of the attention grid
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(bh), kBM / 16);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tail_merge_kernel, q);
}

cudaError_t launch_wait_timeout_selftest(unsigned* err, long long lim, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err, lim);
  return cudaGetLastError();
}

}  // namespace pf
