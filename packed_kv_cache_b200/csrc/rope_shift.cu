// rope_shift.cu -- incremental temporal RoPE adjustment of cached keys.
//
// PackForcing (arXiv), "Incremental RoPE adjustment": after evicting D mid
// blocks, the cached keys' temporal rotary components are multiplied by
// e^{i theta_t delta} (delta = D * B_f frames), leaving the height and width
// components alone ("1_h, 1_w").  Each 128-dim key vector of one head holds
// the temporal pairs in dims 0 .. rope_split[0]-1 as adjacent (re, im) pairs.
//
// HBM-bound: per key vector and head we read and write the first
// ceil(2*pairs/8) 16-byte words (6 words = 96 bytes for 22 pairs, three
// 32-byte sectors each way).  Each lane owns one word of one row-head:
// neighbouring lanes hold a row's words, so one warp load reads 32 / NW
// rows' contiguous pieces with every sector fully used; four steps' loads
// are in flight before any math; the grid depends on the size (see
// launch_nw).  (One thread per row-head, which made each warp load
// touch 32 rows through half-used sectors, measured 17 % slower; a
// TMA-pipelined form -- 96-byte-wide boxes of 128 rows through a ring of
// shared-memory stages, stored back by TMA -- 40-50 % slower.)
#include <cuda_bf16.h>

#include "pf_internal.h"

namespace pf {

namespace {

template <int NW>
__global__ void __launch_bounds__(256) rope_shift_kernel(const RowRuns runs, const RopeTable tab) {
  // lane -> (row, word): a warp covers kRows rows per step, each row's NW
  // words read by NW neighbouring lanes (one contiguous 16 NW-byte piece per
  // row); kU steps' loads are in flight before any arithmetic
  constexpr int kRows = 32 / NW;
  constexpr int kU = 4;
  const int lane = threadIdx.x & 31;
  if (lane >= kRows * NW) return;   // no warp-collective operations below
  const int r_in = lane / NW, k = lane - r_in * NW;
  float cs[4], sn[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    cs[q] = tab.c[(k * 4 + q) & 31];
    sn[q] = tab.s[(k * 4 + q) & 31];
  }
  const long long total = runs.start[runs.n];
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long step = (static_cast<long long>(gridDim.x) * blockDim.x >> 5) * (kRows * kU);
  int seg = 0;
  for (long long r0 = warp * (kRows * kU); r0 < total; r0 += step) {
    uint4 w[kU];
    uint4* ptr[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long long i = r0 + u * kRows + r_in;
      ptr[u] = nullptr;
      if (i < total) {
        while (i >= runs.start[seg + 1]) ++seg;
        while (i < runs.start[seg]) --seg;
        ptr[u] = reinterpret_cast<uint4*>(static_cast<char*>(runs.ptr[seg]) + (i - runs.start[seg]) * (kHeadDim * 2)) + k;
        w[u] = *ptr[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (ptr[u] != nullptr) {
        rope_rotate_word_cs(w[u], k, tab.pairs, cs, sn);
        *ptr[u] = w[u];
      }
    }
  }
}

// Grid: a shift of at least kUncappedWaves times the CTAs resident at once
// (every cached key of a stress layer) gets one CTA per 8 warps' share, so
// finished CTAs are replaced rather than looping (0.189 against 0.209 ms on
// the batch-2 stress layer); a smaller one (the method's sink shift) loops
// over the resident CTAs, which avoids a ragged last wave (15.4 against
// 17.4 µs).
constexpr long long kUncappedWaves = 8;
template <int NW>
cudaError_t launch_nw(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  static PerDevice cap;
  int grid_cap = 0;
  cudaError_t e = cap.get(&grid_cap, [](int dev, int* v) { return one_wave_grid(rope_shift_kernel<NW>, dev, v); });
  if (e != cudaSuccess) return e;
  const long long total = runs.start[runs.n];
  const long long rows_per_cta = 8LL * (32 / NW) * 4;   // 8 warps, kRows rows, kU steps
  const long long want = (total + rows_per_cta - 1) / rows_per_cta;
  long long grid = want >= kUncappedWaves * grid_cap ? want : (want < grid_cap ? want : grid_cap);
  if (grid > 0x7fffffffLL) grid = 0x7fffffffLL;   // the kernel strides over whatever the grid leaves
  rope_shift_kernel<NW><<<static_cast<int>(grid), 256, 0, st>>>(runs, tab);
  return cudaGetLastError();
}

// float32 vectors: the first ceil(pairs / 2) float4 words of each 128-float vector.
__global__ void __launch_bounds__(256) rope_shift_f32_kernel(const RowRuns runs, const RopeTable tab) {
  const long long total = runs.start[runs.n];
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int words = (tab.pairs + 1) / 2;
  int seg = 0;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    while (i >= runs.start[seg + 1]) ++seg;
    while (i < runs.start[seg]) --seg;
    float4* v = reinterpret_cast<float4*>(static_cast<char*>(runs.ptr[seg]) + (i - runs.start[seg]) * (kHeadDim * 4));
    for (int w = 0; w < words; ++w) {
      float4 x = v[w];
      const int p0 = 2 * w, p1 = 2 * w + 1;
      const float a0 = x.x * tab.c[p0] - x.y * tab.s[p0], b0 = x.x * tab.s[p0] + x.y * tab.c[p0];
      x.x = a0;
      x.y = b0;
      if (p1 < tab.pairs) {
        const float a1 = x.z * tab.c[p1] - x.w * tab.s[p1], b1 = x.z * tab.s[p1] + x.w * tab.c[p1];
        x.z = a1;
        x.w = b1;
      }
      v[w] = x;
    }
  }
}

}  // namespace

cudaError_t launch_rope_shift_f32(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  const long long total = runs.start[runs.n];
  if (total <= 0 || tab.pairs <= 0) return cudaSuccess;
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 4096 ? want : 4096);
  rope_shift_f32_kernel<<<grid, 256, 0, st>>>(runs, tab);
  return cudaGetLastError();
}

cudaError_t launch_rope_shift(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  const long long total = runs.start[runs.n];
  if (total <= 0 || tab.pairs <= 0) return cudaSuccess;
  switch ((tab.pairs + 3) / 4) {
    case 1: return launch_nw<1>(runs, tab, st);
    case 2: return launch_nw<2>(runs, tab, st);
    case 3: return launch_nw<3>(runs, tab, st);
    case 4: return launch_nw<4>(runs, tab, st);
    case 5: return launch_nw<5>(runs, tab, st);
    case 6: return launch_nw<6>(runs, tab, st);
    case 7: return launch_nw<7>(runs, tab, st);
    case 8: return launch_nw<8>(runs, tab, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pf
