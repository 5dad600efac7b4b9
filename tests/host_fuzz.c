/*
 * Randomised checks of the library's host-side argument validation, built
 * with -fsanitize=undefined by tests/test_host_fuzz.py: any signed overflow,
 * bad shift or out-of-range conversion in the checks stops the program.
 *
 * No GPU is used.  Device addresses are placeholders that the host code never
 * dereferences.  A call whose arguments pass every check goes on to its first
 * CUDA call, which fails on a machine without a GPU (PF_ERR_CUDA).  With a
 * GPU visible that call would instead reach the device with the placeholder
 * addresses, so the program refuses to run there.
 *
 * Usage: host_fuzz <iterations>
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "pf.h"

static uint64_t state = 88172645463325252ULL;
static uint64_t next(void) {
  state ^= state << 13;
  state ^= state >> 7;
  state ^= state << 17;
  return state;
}

/* sizes at and around the limits the checks enforce, and the int extremes */
static int pick(void) {
  static const int v[] = {0, 1, 2, 3, 4, 5, 7, 8, 9, 16, 17, 31, 32, 33, 52, 64, 127, 128, 182, 512, 513,
                          4095, 4096, 4097, 8191, 8192, 8193, 32768, 65535, 65536, 1 << 20, 1 << 24,
                          (1 << 24) + 1, 1 << 30, 2147483647, -1, -2147483647 - 1};
  return v[next() % (sizeof v / sizeof v[0])];
}

static int fuzz_config(long iters) {
  long accepted = 0;
  for (long it = 0; it < iters; ++it) {
    pf_config c = {1, 1, 12, 128, 4, 30, 52, 2, 1, 40, 16, {44, 42, 42}, 10000.f, 0};
    int* field[] = {&c.layers, &c.batch, &c.heads, &c.block_frames, &c.h, &c.w, &c.sink_blocks,
                    &c.recent_blocks, &c.mid_capacity, &c.n_top, &c.sink_rope_in_attention};
    const int k = 1 + (int)(next() % 4);
    for (int j = 0; j < k; ++j) *field[next() % 11] = pick();
    if (next() % 16 == 0) c.head_dim = pick();
    if (next() % 16 == 0) c.rope_split[next() % 3] = pick();
    size_t bytes = 0;
    const pf_status s = pf_cache_bytes(&c, &bytes);
    if (s != PF_OK) continue;
    ++accepted;
    pf_cache* h = NULL;
    void* arena = (void*)(uintptr_t)0x100000;
    /* one byte short: refused before anything else */
    if (pf_cache_create(&c, arena, bytes - 1, NULL, &h) != PF_ERR_ARENA) {
      printf("config %ld: a short arena was not refused\n", it);
      return 1;
    }
    /* the exact size: the layers are laid out, then the device fill fails */
    if (c.layers <= 64) {
      const pf_status s3 = pf_cache_create(&c, arena, bytes, NULL, &h);
      if (s3 != PF_ERR_CUDA) {
        printf("config %ld: create with the exact arena returned %d\n", it, (int)s3);
        return 1;
      }
    }
  }
  printf("configs: %ld of %ld accepted\n", accepted, iters);
  return accepted > 0 ? 0 : 1;
}

static int fuzz_static_selection(long iters) {
  long counts[8] = {0};
  for (long it = 0; it < iters; ++it) {
    int a[8];
    for (int j = 0; j < 8; ++j) a[j] = pick();
    const void* Q = (next() % 8) ? (const void*)(uintptr_t)(0x100000 + 8 * (next() % 2)) : NULL;
    const void* K = (next() % 8) ? (const void*)(uintptr_t)(0x200000 + 8 * (next() % 2)) : NULL;
    int32_t* sel = (next() % 8) ? (int32_t*)(uintptr_t)(0x300000 + 2 * (next() % 2)) : NULL;
    const pf_status s = pf_select_mid_static(Q, a[0], a[1], a[2], K, a[3], a[4], a[5], a[6], a[7], sel, NULL, NULL);
    if ((int)s < 0 || (int)s > 7) {
      printf("static selection %ld: status %d\n", it, (int)s);
      return 1;
    }
    counts[s]++;
  }
  printf("static selection: ok %ld, arg %ld, capacity %ld, cuda %ld\n", counts[PF_OK], counts[PF_ERR_ARG],
         counts[PF_ERR_CAPACITY], counts[PF_ERR_CUDA]);
  return 0;
}

int main(int argc, char** argv) {
  int devices = 0;
  if (cudaGetDeviceCount(&devices) == cudaSuccess && devices > 0) {
    printf("skipped: a GPU is visible, and the placeholder addresses must never reach it\n");
    return 0;
  }
  const long iters = argc > 1 ? atol(argv[1]) : 100000;
  if (fuzz_config(iters)) return 1;
  return fuzz_static_selection(iters);
}
