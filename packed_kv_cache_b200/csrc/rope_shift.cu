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
// 32-byte sectors each way).  One thread per key vector, all loads issued
// before any math, grid sized to the SM count.
#include <cuda_bf16.h>

#include "pf_internal.h"

namespace pf {

namespace {

constexpr int kMaxWords = 8;  // up to 64 temporal dims

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
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    while (i >= runs.start[seg + 1]) ++seg;
    while (i < runs.start[seg]) --seg;
    uint4* p = reinterpret_cast<uint4*>(static_cast<char*>(runs.ptr[seg]) +
                                        (i - runs.start[seg]) * (kHeadDim * 2));
    uint4 w[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) w[k] = p[k];
#pragma unroll
    for (int k = 0; k < NW; ++k) rotate_word(w[k], k, tab);
#pragma unroll
    for (int k = 0; k < NW; ++k) p[k] = w[k];
  }
}

}  // namespace

cudaError_t launch_rope_shift(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  const long long total = runs.start[runs.n];
  if (total <= 0 || tab.pairs <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < sms * 8LL ? want : sms * 8LL);
  const int words = (tab.pairs + 3) / 4;
  switch (words) {
    case 1: rope_shift_kernel<1><<<grid, 256, 0, st>>>(runs, tab); break;
    case 2: rope_shift_kernel<2><<<grid, 256, 0, st>>>(runs, tab); break;
    case 3: rope_shift_kernel<3><<<grid, 256, 0, st>>>(runs, tab); break;
    case 4: rope_shift_kernel<4><<<grid, 256, 0, st>>>(runs, tab); break;
    case 5: rope_shift_kernel<5><<<grid, 256, 0, st>>>(runs, tab); break;
    case 6: rope_shift_kernel<6><<<grid, 256, 0, st>>>(runs, tab); break;
    case 7: rope_shift_kernel<7><<<grid, 256, 0, st>>>(runs, tab); break;
    case 8: rope_shift_kernel<8><<<grid, 256, 0, st>>>(runs, tab); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pf
