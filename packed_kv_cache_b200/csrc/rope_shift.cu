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
// that fit on the GPU at once (no partial last wave).
#include <cuda_bf16.h>

#include "pf_internal.h"

namespace pf {

namespace {

__device__ __forceinline__ void rotate_word(uint4& w, int word, const RopeTable& t) {
  uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int pair = word * 4 + q;
    if (pair < t.pairs) {
      __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&v[q]);
      const float re = __low2float(x), im = __high2float(x);
      const float c = t.c[pair], s = t.s[pair];
      const float nre = re * c - im * s;
      const float nim = re * s + im * c;
      __nv_bfloat162 y = __floats2bfloat162_rn(nre, nim);
      v[q] = *reinterpret_cast<uint32_t*>(&y);
    }
  }
  w = make_uint4(v[0], v[1], v[2], v[3]);
}

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
        for (int k = 0; k < NW; ++k) rotate_word(w[u][k], k, tab);
#pragma unroll
        for (int k = 0; k < NW; ++k) ptr[u][k] = w[u][k];
      }
    }
  }
}

template <int NW>
cudaError_t launch_nw(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  static int grid_cap = 0;
  if (grid_cap == 0) {
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rope_shift_kernel<NW>, 256, 0);
    grid_cap = sms * (per_sm > 0 ? per_sm : 1);
  }
  const long long total = runs.start[runs.n];
  const long long want = (total + 511) / 512;
  const int grid = static_cast<int>(want < grid_cap ? want : grid_cap);
  rope_shift_kernel<NW><<<grid, 256, 0, st>>>(runs, tab);
  return cudaGetLastError();
}

}  // namespace

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
