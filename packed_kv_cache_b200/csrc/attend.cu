// attend.cu -- attention of the current block's queries over the bounded
// packed context, on 5th-generation tensor cores.
//
// PackForcing digest, KV-cache paragraph: Attn(Q_i, C) = softmax(Q_i K^T /
// sqrt(d_h)) V; PackForcing (arXiv), "Bounded Attention Context": the context
// is sink || selected mid blocks || recent || current, a fixed number of
// tokens.  The partitions are never gathered: the key/value tiles are pulled
// by TMA straight from where each partition lives.
//
// Work unit: one (batch item, head, 256 queries) = two 128-row query tiles
// that share every K/V tile.  One CTA per unit, 12 warps:
//   warp 0      TMA producer: Q once, then K and V tiles through a 2-stage ring
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
constexpr int kStages = 2;         // K and V ring depth
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = kBN * kHeadDim * 2;   // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;       // 64 dims x 128 rows
constexpr uint32_t kSubBytes = kSub * 128;            // one sub-box, one 64-dim half
constexpr float kRescaleThreshold = 8.0f;
// Before S_t of the next tile is written over P_t, wait until the P_t V MMA
// that reads P_t has completed.
constexpr bool kDrainBeforeOverwrite = true;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                   // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;              // kStages tiles
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;        // kStages tiles
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;           // + barriers + alignment slack

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], o_final[2];
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

__global__ void __launch_bounds__(kThreads, 1) attend_kernel(const __grid_constant__ AttendParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + kOffBar);
  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sK = smem_u32(smem + kOffK);
  const uint32_t sV = smem_u32(smem + kOffV);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int unit = blockIdx.x;
  const int qp = unit % p.q_pairs;
  const int bh = unit / p.q_pairs;
  const int h = bh % p.H;
  const int b = bh / p.H;
  const int q0 = qp * 2 * kBM;
  const int T = p.n_tiles;
  const long long lim = p.timeout_cycles;
  volatile int* abort_flag = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.p_full[t], kBM);
      mbar_init(&bars.o_final[t], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.tm_q);
      for (int m = 0; m < 4; ++m) {
        prefetch_tmap(&p.tm_k[m]);
        prefetch_tmap(&p.tm_v[m]);
      }
      mbar_arrive_expect_tx(&bars.q_full, 2 * kTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int half = 0; half < 2; ++half)
          tma_load_4d(smem + kOffQ + t * kTileBytes + half * kHalfBytes, &p.tm_q, &bars.q_full, half * 64, h,
                      q0 + t * kBM, b);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % kStages;
        const uint32_t use = j / kStages;
        if (use > 0 && !mbar_wait_bounded(&bars.k_empty[st], (use - 1) & 1, abort_flag, p.err,
                                          kDevErrTimeoutBase | 1u, lim))
          break;
        mbar_arrive_expect_tx(&bars.k_full[st], kTileBytes);
        for (int i = 0; i < 4; ++i) {
          const SubBox sb = decode_subbox(p, b, 4 * j + i);
          for (int half = 0; half < 2; ++half)
            tma_load_4d(smem + kOffK + st * kTileBytes + half * kHalfBytes + i * kSubBytes, &p.tm_k[sb.part],
                        &bars.k_full[st], half * 64, h, sb.row0, sb.seg);
        }
        if (use > 0 && !mbar_wait_bounded(&bars.v_empty[st], (use - 1) & 1, abort_flag, p.err,
                                          kDevErrTimeoutBase | 2u, lim)) {
          issued = j * 2 + 1;
          break;
        }
        mbar_arrive_expect_tx(&bars.v_full[st], kTileBytes);
        for (int i = 0; i < 4; ++i) {
          const SubBox sb = decode_subbox(p, b, 4 * j + i);
          for (int half = 0; half < 2; ++half)
            tma_load_4d(smem + kOffV + st * kTileBytes + half * kHalfBytes + i * kSubBytes, &p.tm_v[sb.part],
                        &bars.v_full[st], half * 64, h, sb.row0, sb.seg);
        }
        issued = j * 2 + 2;
      }
      if (*abort_flag) {
        // let every load already issued land before the CTA can exit
        const long long short_lim = lim / 4 + 1;
        mbar_wait_bounded(&bars.q_full, 0, nullptr, nullptr, 0, short_lim);
        for (int k = issued - 1; k >= 0 && k >= issued - 2 * kStages; --k) {
          const int j = k / 2;
          uint64_t* bar = (k & 1) ? &bars.v_full[j % kStages] : &bars.k_full[j % kStages];
          mbar_wait_bounded(bar, (j / kStages) & 1, nullptr, nullptr, 0, short_lim);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
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
        for (int kk = 0; kk < kBN / 16; ++kk) {
          mma_ts(tO[t], tS[t] + kk * 8, sdesc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc_pv,
                 (!first || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_bounded(&bars.q_full, 0, abort_flag, p.err, kDevErrTimeoutBase | 3u, lim);
      if (ok) ok = mbar_wait_bounded(&bars.k_full[0], 0, abort_flag, p.err, kDevErrTimeoutBase | 4u, lim);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(&bars.s_full[0]);
        issue_qk(1, 0);
        mma_commit(&bars.s_full[1]);
        mma_commit(&bars.k_empty[0]);
      }
      for (int j = 0; ok && j < T; ++j) {
        const int vs = j % kStages;
        const int jn = j + 1;
        const int ks = jn % kStages;
        ok = mbar_wait_bounded(&bars.v_full[vs], (j / kStages) & 1, abort_flag, p.err, kDevErrTimeoutBase | 5u, lim);
        if (ok) ok = mbar_wait_bounded(&bars.p_full[0], j & 1, abort_flag, p.err, kDevErrTimeoutBase | 6u, lim);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, vs, j == 0);
        if (jn < T) {
          // S_0 of the next tile overwrites P_0
          if (kDrainBeforeOverwrite) {
            mma_commit(&bars.drain);
            ok = mbar_wait_bounded(&bars.drain, (2 * j) & 1, abort_flag, p.err, kDevErrTimeoutBase | 7u, lim);
          }
          if (ok) ok = mbar_wait_bounded(&bars.k_full[ks], (jn / kStages) & 1, abort_flag, p.err,
                                         kDevErrTimeoutBase | 8u, lim);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, ks);
          mma_commit(&bars.s_full[0]);
        }
        ok = mbar_wait_bounded(&bars.p_full[1], j & 1, abort_flag, p.err, kDevErrTimeoutBase | 9u, lim);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, vs, j == 0);
        mma_commit(&bars.v_empty[vs]);
        if (jn < T) {
          if (kDrainBeforeOverwrite) {
            mma_commit(&bars.drain);
            ok = mbar_wait_bounded(&bars.drain, (2 * j + 1) & 1, abort_flag, p.err, kDevErrTimeoutBase | 10u, lim);
            if (!ok) break;
          }
          issue_qk(1, ks);
          mma_commit(&bars.s_full[1]);
          mma_commit(&bars.k_empty[ks]);
        }
      }
      mma_commit(&bars.o_final[0]);
      mma_commit(&bars.o_final[1]);
      if (!ok) {
        // make sure nothing issued is still running before the memory goes away
        mbar_wait_bounded(&bars.o_final[0], 0, nullptr, nullptr, 0, lim / 4 + 1);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;                 // query tile
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int row = quarter * 32 + lane;           // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128u;
    const uint32_t tO = tmem + lane_off + 256u + t * 128u;
    const float sl2 = p.scale_log2;
    float m = -INFINITY;   // running max of scaled scores, base-2 units
    float l = 0.f;         // running sum of exp2(score - m)
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      ok = mbar_wait_bounded(&bars.s_full[t], j & 1, abort_flag, p.err, kDevErrTimeoutBase | 11u, lim);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld128_wait(tS, s);
      int valid[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) valid[i] = subbox_valid(p, 4 * j + i);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float x = __uint_as_float(s[c]);
        if ((c & 31) >= valid[c >> 5]) x = -INFINITY;
        s[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      const float mt = mx * sl2;
      if (mt > m + kRescaleThreshold) {
        const float alpha = ex2_approx(m - mt);   // 0 when m = -inf
        l *= alpha;
        if (j > 0) {
          uint32_t o[32];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            tmem_ld32_wait(tO + cc * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + cc * 32, o);
          }
        }
        m = mt;
      }
      const float mb = (m == -INFINITY) ? 0.f : m;
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[cc * 32 + 2 * e]), sl2, -mb));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[cc * 32 + 2 * e + 1]), sl2, -mb));
          rs += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + cc * 16, pk);
      }
      l += rs;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[t]);
    }
    if (ok) ok = mbar_wait_bounded(&bars.o_final[t], 0, abort_flag, p.err, kDevErrTimeoutBase | 12u, lim);
    if (ok) {
      tc_fence_after();
      const int qrow = q0 + t * kBM + row;
      const float inv = 1.f / l;
      __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.O);
      uint4* dst = reinterpret_cast<uint4*>(O + ((static_cast<long long>(b) * p.n + qrow) * p.H + h) * kHeadDim);
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
      if (p.lse != nullptr && qrow < p.n)
        p.lse[(static_cast<long long>(b) * p.H + h) * p.n + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int units = p.B * p.H * p.q_pairs;
  attend_kernel<<<units, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(unsigned* err, long long lim, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err, lim);
  return cudaGetLastError();
}

}  // namespace pf
