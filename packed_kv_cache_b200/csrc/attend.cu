// attend.cu -- attention of the current block's queries over the bounded
// packed context, on 5th-generation tensor cores.
//
// PackForcing digest, KV-cache paragraph: Attn(Q_i, C) = softmax(Q_i K^T /
// sqrt(d_h)) V; PackForcing (arXiv), "Bounded Attention Context": the context
// is sink || selected mid blocks || recent || current, a fixed number of
// tokens.  The partitions are never gathered: the key/value tiles are pulled
// by TMA straight from where each partition lives.
//
// Work unit: two 128-row query tiles of one (batch item, head) that share
// every K/V tile, or the last, ragged tile of a (b, h) alone.  One CTA per
// unit by default; a persistent grid (one CTA per SM, units dealt
// round-robin) is available at build time.  12 warps:
//   warp 0      TMA producer: Q per unit, K and V tiles through rings
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T and O_t += P_t V
//   warp 2      tensor-memory allocator
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
#ifndef PF_ATTEND_K_STAGES
#define PF_ATTEND_K_STAGES 3
#endif
constexpr int kKStages = PF_ATTEND_K_STAGES;  // K ring depth
constexpr int kVStages = 2;        // V ring depth
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = kBN * kHeadDim * 2;   // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;       // 64 dims x 128 rows
constexpr uint32_t kSubBytes = kSub * 128;            // one sub-box, one 64-dim half
constexpr float kRescaleThreshold = 8.0f;
// Registers per thread after the split: the producer/MMA warpgroup gives up
// registers to the two softmax warpgroups (128*120 + 256*192 <= 384*168).
#ifndef PF_ATTEND_REGS_CONTROL
#define PF_ATTEND_REGS_CONTROL 120
#endif
#ifndef PF_ATTEND_REGS_SOFTMAX
#define PF_ATTEND_REGS_SOFTMAX 192
#endif
constexpr int kRegsLaunch = 168, kRegsControl = PF_ATTEND_REGS_CONTROL, kRegsSoftmax = PF_ATTEND_REGS_SOFTMAX;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
// Before S_t of the next tile is written over P_t, wait until the P_t V MMA
// that reads P_t has completed.
#ifndef PF_ATTEND_DRAIN
#define PF_ATTEND_DRAIN 0
#endif
constexpr bool kDrainBeforeOverwrite = PF_ATTEND_DRAIN != 0;
// One exponential pair in kPolyPeriod is evaluated by ex2_poly (FMA pipe),
// the others by the special-function unit (0 = never).
#ifndef PF_ATTEND_POLY_PERIOD
#define PF_ATTEND_POLY_PERIOD 0
#endif
constexpr int kPolyPeriod = PF_ATTEND_POLY_PERIOD;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                   // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;              // kKStages tiles
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;       // kVStages tiles
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;           // + barriers + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory");

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_final[2], o_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct SubBox {
  int part, row0, seg, valid;
};

// Sub-box s of batch item b's context: which partition, first row, segment
// (index along the tensor map's outermost dimension), and valid rows.
__device__ __forceinline__ SubBox decode_subbox(const AttendParams& p, int b, int s) {
  SubBox r;
  if (s < p.sb_sink) {
    r.part = kPartSink; r.row0 = s * kSub; r.seg = b; r.valid = min(kSub, p.sink_rows - r.row0);
    return r;
  }
  s -= p.sb_sink;
  const int nmid = p.n_sel * p.sb_mid;
  if (s < nmid) {
    const int blk = s / p.sb_mid, k = s - blk * p.sb_mid;
    const int slot = p.sel_slots ? p.sel_slots[b * p.sel_stride + blk] : (p.mid_head + blk) % p.pool_slots;
    r.part = kPartMid; r.row0 = k * kSub; r.seg = b * p.pool_slots + slot;
    r.valid = min(kSub, p.n_c - r.row0);
    return r;
  }
  s -= nmid;
  const int nrec = p.n_recent * p.sb_blk;
  if (s < nrec) {
    const int blk = s / p.sb_blk, k = s - blk * p.sb_blk;
    const int slot = (p.recent_head + blk) % p.recent_slots;
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
__device__ __forceinline__ int subbox_valid(const AttendParams& p, int s) {
  if (s < p.sb_sink) return min(kSub, p.sink_rows - s * kSub);
  s -= p.sb_sink;
  const int nmid = p.n_sel * p.sb_mid;
  if (s < nmid) return min(kSub, p.n_c - (s % p.sb_mid) * kSub);
  s -= nmid;
  const int nrec = p.n_recent * p.sb_blk;
  if (s < nrec) return min(kSub, p.n - (s % p.sb_blk) * kSub);
  s -= nrec;
  if (s < p.sb_blk) return min(kSub, p.n - s * kSub);
  return 0;
}

// One CTA per unit (1) or a persistent grid of at most one CTA per SM (0).
// Measured on the pages-scale layer: 1.54 ms vs 1.74 ms.
#ifndef PF_ATTEND_ONE_UNIT_PER_CTA
#define PF_ATTEND_ONE_UNIT_PER_CTA 1
#endif

// The unit schedule.  A (b, h) has q_tiles 128-row query tiles.  Units
// 0 .. F-1 pair tiles 2k and 2k+1 of one (b, h): both read the same K/V
// tiles.  When q_tiles is odd, the last (ragged) tile of each (b, h) is a
// unit of its own ("single").  Full units go round-robin over the G CTAs
// (CTA c: c, c + G, ...), so that the CTAs running at the same time share
// few heads; singles go round-robin over the CTAs that got fewer full units.
struct QTile {
  int b, h, qt;
};
struct Unit {
  QTile t[2];
  int nq;       // query tiles in the unit (1 or 2)
  bool shared;  // both tiles read the same K/V stream
};
struct Sched {
  int F, S, G, L0, NL;  // full units, singles, CTAs, first light CTA, light CTAs
};

__device__ __forceinline__ Sched make_sched(const AttendParams& p) {
  Sched q;
  q.F = p.B * p.H * (p.q_tiles / 2);
  q.S = (p.q_tiles & 1) ? p.B * p.H : 0;
  q.G = gridDim.x;
  q.L0 = q.F % q.G;
  q.NL = q.G - q.L0;
  return q;
}

__device__ __forceinline__ int units_of(const Sched& q, int c) {
#if PF_ATTEND_ONE_UNIT_PER_CTA
  return c < q.F + q.S ? 1 : 0;
#else
  const int nf = q.F / q.G + (c < q.F % q.G ? 1 : 0);
  const int ns = (c < q.L0 || q.S == 0) ? 0 : (q.S - (c - q.L0) + q.NL - 1) / q.NL;
  return nf + max(ns, 0);
#endif
}

__device__ __forceinline__ Unit unit_of(const AttendParams& p, const Sched& q, int c, int k) {
#if PF_ATTEND_ONE_UNIT_PER_CTA
  const int nf = c < q.F ? 1 : 0;
  const int u = c;
  (void)k;
#else
  const int nf = q.F / q.G + (c < q.F % q.G ? 1 : 0);
  const int u = (k < nf) ? c + k * q.G : q.F + (c - q.L0) + (k - nf) * q.NL;
#endif
  const int pairs = p.q_tiles / 2;
  Unit r;
  r.shared = true;
  if (u < q.F) {
    const int bh = u / pairs, kk = u - bh * pairs;
    r.t[0] = {bh / p.H, bh % p.H, 2 * kk};
    r.t[1] = {bh / p.H, bh % p.H, 2 * kk + 1};
    r.nq = 2;
  } else {
    const int bh = u - q.F;
    r.t[0] = {bh / p.H, bh % p.H, p.q_tiles - 1};
    r.t[1] = r.t[0];
    r.nq = 1;
  }
  (void)nf;
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
    float p0, p1;
    if (kPolyPeriod > 0 && (e % kPolyPeriod) == kPolyPeriod - 1) {
      p0 = ex2_poly(f2_lo(x));   // on the FMA pipe: unloads the special-function unit
      p1 = ex2_poly(f2_hi(x));
    } else {
      p0 = ex2_approx(f2_lo(x));
      p1 = ex2_approx(f2_hi(x));
    }
    rs2[e & 1] = f2_add(rs2[e & 1], f2_pack(p0, p1));
    pk[e] = pack_bf16x2(p0, p1);
  }
  tmem_st16(dst, pk);
}

#ifndef PF_ATTEND_SETMAXNREG
#define PF_ATTEND_SETMAXNREG 0
#endif
__device__ __forceinline__ void setmaxnreg_dec() {
#if PF_ATTEND_SETMAXNREG
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
#endif
}
__device__ __forceinline__ void setmaxnreg_inc() {
#if PF_ATTEND_SETMAXNREG
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
#endif
}

__global__ void __launch_bounds__(kThreads, 1) attend_kernel(const __grid_constant__ AttendParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + kOffBar);
  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sK = smem_u32(smem + kOffK);
  const uint32_t sV = smem_u32(smem + kOffV);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = p.n_tiles;
  const long long lim = p.timeout_cycles;
  volatile int* abort_flag = &bars.abort;
  const Sched sched = make_sched(p);
  const int n_units = units_of(sched, blockIdx.x);

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.p_full[t], kBM);
      mbar_init(&bars.o_final[t], 1);
      mbar_init(&bars.o_free[t], kBM);
    }
    mbar_init(&bars.drain, 1);
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

  if (warp < 4) {
    setmaxnreg_dec();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      prefetch_tmap(&p.tm_q);
      for (int m = 0; m < 4; ++m) {
        prefetch_tmap(&p.tm_k[m]);
        prefetch_tmap(&p.tm_v[m]);
      }
      int kg = 0, vg = 0;              // K / V tiles issued so far (all units)
      int uq = 0;                      // units whose Q was loaded
      bool ok = true;
      for (int k = 0; ok && k < n_units; ++k, ++uq) {
        const Unit un = unit_of(p, sched, blockIdx.x, k);
        const int ns = un.shared ? 1 : 2;   // K/V streams
        if (uq > 0 && !mbar_wait_bounded(&bars.q_empty, (uq - 1) & 1, abort_flag, p.err,
                                         kDevErrTimeoutBase | 1u, lim)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars.q_full, un.nq * kTileBytes);
        for (int t = 0; t < un.nq; ++t)
          for (int half = 0; half < 2; ++half)
            tma_load_4d(smem + kOffQ + t * kTileBytes + half * kHalfBytes, &p.tm_q, &bars.q_full, half * 64,
                        un.t[t].h, un.t[t].qt * kBM, un.t[t].b);
        for (int j = 0; ok && j < T; ++j) {
          for (int sidx = 0; sidx < ns; ++sidx) {
            const int st = kg % kKStages, use = kg / kKStages;
            if (use > 0 && !mbar_wait_bounded(&bars.k_empty[st], (use - 1) & 1, abort_flag, p.err,
                                              kDevErrTimeoutBase | 2u, lim)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bars.k_full[st], kTileBytes);
            for (int i = 0; i < 4; ++i) {
              const SubBox sb = decode_subbox(p, un.t[sidx].b, 4 * j + i);
              for (int half = 0; half < 2; ++half)
                tma_load_4d(smem + kOffK + st * kTileBytes + half * kHalfBytes + i * kSubBytes,
                            &p.tm_k[sb.part], &bars.k_full[st], half * 64, un.t[sidx].h, sb.row0, sb.seg);
            }
            ++kg;
          }
          for (int sidx = 0; ok && sidx < ns; ++sidx) {
            const int st = vg % kVStages, use = vg / kVStages;
            if (use > 0 && !mbar_wait_bounded(&bars.v_empty[st], (use - 1) & 1, abort_flag, p.err,
                                              kDevErrTimeoutBase | 3u, lim)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bars.v_full[st], kTileBytes);
            for (int i = 0; i < 4; ++i) {
              const SubBox sb = decode_subbox(p, un.t[sidx].b, 4 * j + i);
              for (int half = 0; half < 2; ++half)
                tma_load_4d(smem + kOffV + st * kTileBytes + half * kHalfBytes + i * kSubBytes,
                            &p.tm_v[sb.part], &bars.v_full[st], half * 64, un.t[sidx].h, sb.row0, sb.seg);
            }
            ++vg;
          }
        }
      }
      if (!ok || *abort_flag) {
        // let every load already issued land before the CTA can exit
        const long long short_lim = lim / 4 + 1;
        if (uq > 0) mbar_wait_bounded(&bars.q_full, (uq - 1) & 1, nullptr, nullptr, 0, short_lim);
        for (int g = kg - 1; g >= 0 && g >= kg - kKStages; --g)
          mbar_wait_bounded(&bars.k_full[g % kKStages], (g / kKStages) & 1, nullptr, nullptr, 0, short_lim);
        for (int g = vg - 1; g >= 0 && g >= vg - kVStages; --g)
          mbar_wait_bounded(&bars.v_full[g % kVStages], (g / kVStages) & 1, nullptr, nullptr, 0, short_lim);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(kBM, kHeadDim, 1);
      const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
      const uint32_t tO[2] = {tmem + 256u, tmem + 384u};
      auto issue_qk = [&](int t, int st) {
        const uint32_t qa = sQ + t * kTileBytes, ka = sK + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tS[t], sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int st, bool first) {
        const uint32_t va = sV + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tO[t], tS[t] + kk * 8, sdesc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc_pv,
                 (!first || kk > 0) ? 1u : 0u);
      };
      int kg = 0, vg = 0;       // K / V tiles consumed
      int pc[2] = {0, 0};       // P tiles consumed per query-tile slot
      int uses[2] = {0, 0};     // units that used each slot
      int drains = 0, uq = 0;
      bool ok = true;
      auto wait_k = [&](int g, unsigned site) {
        return mbar_wait_bounded(&bars.k_full[g % kKStages], (g / kKStages) & 1, abort_flag, p.err,
                                 kDevErrTimeoutBase | site, lim);
      };
      auto drain = [&](unsigned site) {
        mma_commit(&bars.drain);
        const bool r = mbar_wait_bounded(&bars.drain, drains & 1, abort_flag, p.err, kDevErrTimeoutBase | site, lim);
        ++drains;
        return r;
      };
      for (int k = 0; ok && k < n_units; ++k, ++uq) {
        const Unit un = unit_of(p, sched, blockIdx.x, k);
        const int nq = un.nq;
        const int ns = un.shared ? 1 : 2;
        ok = mbar_wait_bounded(&bars.q_full, uq & 1, abort_flag, p.err, kDevErrTimeoutBase | 4u, lim);
        if (ok && kDrainBeforeOverwrite && uq > 0) ok = drain(13u);   // last P_t V may still read P_t
        for (int t = 0; ok && t < nq; ++t) {
          const int g = kg + (un.shared ? 0 : t);
          if (t == 0 || !un.shared) ok = wait_k(g, 5u);
          if (!ok) break;
          tc_fence_after();
          issue_qk(t, g % kKStages);
          mma_commit(&bars.s_full[t]);
        }
        if (!ok) break;
        for (int sidx = 0; sidx < ns; ++sidx) mma_commit(&bars.k_empty[(kg + sidx) % kKStages]);
        kg += ns;
        if (T == 1) mma_commit(&bars.q_empty);
        for (int j = 0; ok && j < T; ++j) {
          const bool more = j + 1 < T;
          for (int t = 0; ok && t < nq; ++t) {
            const int vgt = vg + (un.shared ? 0 : t);
            if (t == 0 || !un.shared)
              ok = mbar_wait_bounded(&bars.v_full[vgt % kVStages], (vgt / kVStages) & 1, abort_flag, p.err,
                                     kDevErrTimeoutBase | 6u, lim);
            if (ok) ok = mbar_wait_bounded(&bars.p_full[t], pc[t] & 1, abort_flag, p.err, kDevErrTimeoutBase | 7u, lim);
            if (ok && j == 0 && uses[t] > 0)
              ok = mbar_wait_bounded(&bars.o_free[t], (uses[t] - 1) & 1, abort_flag, p.err,
                                     kDevErrTimeoutBase | 8u, lim);
            if (!ok) break;
            ++pc[t];
            tc_fence_after();
            issue_pv(t, vgt % kVStages, j == 0);
            if (more) {
              // S_t of the next tile overwrites P_t
              if (kDrainBeforeOverwrite) ok = drain(9u);
              const int g = kg + (un.shared ? 0 : t);
              if (ok && (t == 0 || !un.shared)) ok = wait_k(g, 10u);
              if (!ok) break;
              tc_fence_after();
              issue_qk(t, g % kKStages);
              mma_commit(&bars.s_full[t]);
            }
          }
          if (!ok) break;
          for (int sidx = 0; sidx < ns; ++sidx) mma_commit(&bars.v_empty[(vg + sidx) % kVStages]);
          vg += ns;
          if (more) {
            for (int sidx = 0; sidx < ns; ++sidx) mma_commit(&bars.k_empty[(kg + sidx) % kKStages]);
            kg += ns;
            if (j + 1 == T - 1) mma_commit(&bars.q_empty);
          }
        }
        if (!ok) break;
        for (int t = 0; t < nq; ++t) {
          mma_commit(&bars.o_final[t]);
          ++uses[t];
        }
      }
      if (!ok) {
        // make sure nothing issued is still running before the memory goes away
        mma_commit(&bars.drain);
        mbar_wait_bounded(&bars.drain, drains & 1, nullptr, nullptr, 0, lim / 4 + 1);
      }
    }
  } else {
    setmaxnreg_inc();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;                 // query-tile slot
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int row = quarter * 32 + lane;           // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128u;
    const uint32_t tO = tmem + lane_off + 256u + t * 128u;
    const float sl2 = p.scale_log2;
    int sc = 0, oc = 0;                            // S tiles / units consumed
    bool ok = true;
    for (int k = 0; ok && k < n_units; ++k) {
      const Unit un = unit_of(p, sched, blockIdx.x, k);
      if (t >= un.nq) continue;
      const QTile qt = un.t[t];
      float m = -INFINITY;   // running max of scaled scores, base-2 units
      float l = 0.f;         // running sum of exp2(score - m)
      for (int j = 0; j < T; ++j) {
        ok = mbar_wait_bounded(&bars.s_full[t], sc & 1, abort_flag, p.err, kDevErrTimeoutBase | 11u, lim);
        if (!ok) break;
        ++sc;
        tc_fence_after();
        // which columns hold real keys (most tiles: all of them)
        const int s0 = 4 * j;
        int valid[4] = {kSub, kSub, kSub, kSub};
        const bool check = !p.exact || (s0 + 4 > p.sb_mid_lo && s0 < p.sb_mid_hi) || (s0 + 4 > p.n_sub);
        if (check) {
#pragma unroll
          for (int i = 0; i < 4; ++i) valid[i] = subbox_valid(p, s0 + i);
        }
        const bool masked = check && (valid[0] != kSub || valid[1] != kSub || valid[2] != kSub || valid[3] != kSub);
        // the whole row of S in registers: one tensor-memory round trip
        uint32_t sv[128];
        tmem_ld128_wait(tS, sv);
        if (masked) {
#pragma unroll
          for (int i = 0; i < 4; ++i) mask32(sv + 32 * i, valid[i]);
        }
        const float mt = fmaxf(max64(sv), max64(sv + 64)) * sl2;
        float alpha = 1.f;
        bool rescale_o = false;
        if (mt > m + kRescaleThreshold) {
          alpha = ex2_approx(m - mt);   // 0 when m = -inf
          l *= alpha;
          rescale_o = j > 0;
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
        if (rescale_o) {
          // O holds every P V up to the previous tile (completed before S of
          // this tile was signalled); the next P V is issued after p_full
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
      if (ok) ok = mbar_wait_bounded(&bars.o_final[t], oc & 1, abort_flag, p.err, kDevErrTimeoutBase | 12u, lim);
      if (!ok) break;
      ++oc;
      tc_fence_after();
      const int qrow = qt.qt * kBM + row;
      const float inv = 1.f / l;
      __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.O);
      uint4* dst = reinterpret_cast<uint4*>(O + ((static_cast<long long>(qt.b) * p.n + qrow) * p.H + qt.h) * kHeadDim);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32_wait(tO + cc * 32, o);
        if (qrow < p.n) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
            dst[cc * 4 + v] = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.o_free[t]);
      if (p.lse != nullptr && qrow < p.n)
        p.lse[(static_cast<long long>(qt.b) * p.H + qt.h) * p.n + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

cudaError_t launch_attend(const AttendParams& p, cudaStream_t st) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const int bh = p.B * p.H;
  const int units = bh * (p.q_tiles / 2) + ((p.q_tiles & 1) ? bh : 0);
  const int grid = PF_ATTEND_ONE_UNIT_PER_CTA ? units : (units < sms ? units : sms);
  attend_kernel<<<grid, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(unsigned* err, long long lim, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err, lim);
  return cudaGetLastError();
}

}  // namespace pf
