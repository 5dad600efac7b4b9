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
// 32-byte sectors each way).  One thread per key vector, two vectors per
// step with all loads issued before any math; the grid is exactly the CTAs
// that fit on the GPU at once (no partial last wave).  (A TMA-pipelined
// form -- 96-byte-wide boxes of 128 rows through a ring of shared-memory
// stages, stored back by TMA -- measured 40-50 % slower on the same
// workloads, whatever the L2 promotion and CTAs per SM.)
#include <cuda_bf16.h>

#include "pf_internal.h"

namespace pf {

namespace {

template <int NW>
__global__ void __launch_bounds__(256) rope_shift_kernel(const RowRuns runs, const RopeTable tab) {
  const long long total = runs.start[runs.n];
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  int seg = 0;
  // two key vectors per thread per step: all twelve loads in flight before any math
  for (long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < total; i0 += 2 * stride) {
    uint4 w[2][NW];
    uint4* ptr[2] = {nullptr, nullptr};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const long long i = i0 + u * stride;
      if (i < total) {
        while (i >= runs.start[seg + 1]) ++seg;
        while (i < runs.start[seg]) --seg;
        ptr[u] = reinterpret_cast<uint4*>(static_cast<char*>(runs.ptr[seg]) + (i - runs.start[seg]) * (kHeadDim * 2));
#pragma unroll
        for (int k = 0; k < NW; ++k) w[u][k] = ptr[u][k];
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (ptr[u] != nullptr) {
#pragma unroll
        for (int k = 0; k < NW; ++k) rope_rotate_word(w[u][k], k, tab);
#pragma unroll
        for (int k = 0; k < NW; ++k) ptr[u][k] = w[u][k];
      }
    }
  }
}

template <int NW>
cudaError_t launch_nw(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  static PerDevice cap;
  int grid_cap = 0;
  cudaError_t e = cap.get(&grid_cap, [](int dev, int* v) { return one_wave_grid(rope_shift_kernel<NW>, dev, v); });
  if (e != cudaSuccess) return e;
  const long long total = runs.start[runs.n];
  const long long want = (total + 511) / 512;
  const int grid = static_cast<int>(want < grid_cap ? want : grid_cap);
  rope_shift_kernel<NW><<<grid, 256, 0, st>>>(runs, tab);
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
