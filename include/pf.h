/*
 * pf.h -- C ABI of the packed KV cache for block-autoregressive video
 * diffusion (PackForcing), single GPU, sm_100a.
 *
 * The cache of one transformer layer has three partitions (PackForcing
 * (arXiv), "Sink Tokens", "Compressed Mid Tokens", "Recent & Current
 * Tokens"):
 *   sink    the first N_sink/B_f blocks at full resolution, never evicted;
 *   mid     a ring ("pool") of compressed blocks, n_c tokens each, of which
 *           the top N_top by query-key affinity are routed into attention;
 *   recent  the last N_recent/B_f finished blocks at full resolution.
 * The current block's K/V are passed to each attention call.  The attended
 * context is sink || selected mid (oldest first) || recent || current
 * ("Bounded Attention Context").
 *
 * Conventions for every entry point:
 *  - Tensors are device pointers to contiguous bf16 in token-major layout
 *    [B, L, H, D] (D = 128 innermost), 16-byte aligned.  "Kc/Vc" are the
 *    compressed keys/values of one block, [B, n_c, H, D].
 *  - The caller owns every device buffer, including the cache arena
 *    (sized by pf_cache_bytes).  The library owns a small host struct.
 *  - Every call is asynchronous on the caller's CUDA stream (passed as
 *    void*, a cudaStream_t; NULL = the legacy default stream) and does not
 *    synchronise the host, except pf_poll_device_error.  Calls on one cache
 *    must be ordered on one stream: they share per-layer scratch memory in
 *    the arena.
 *  - Errors are return codes; pf_last_error() gives the calling thread's
 *    last message.  A failed call leaves the cache state unchanged.
 *  - Device-side failures (a bounded wait that gave up) are recorded in a
 *    word in the arena; pf_poll_device_error reads and clears it.
 *  - Several devices (and host threads) may share the library: each
 *    launcher's one-time set-up (a kernel attribute, a grid size) is done
 *    once per device under a lock.  That set-up, and the address of the
 *    allocation-free selection's array, belong to the device's primary
 *    context: after cudaDeviceReset on a device the library must not be
 *    used on it again in the same process.
 */
#ifndef PF_H
#define PF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pf_status {
  PF_OK = 0,
  PF_ERR_ARG = 1,         /* null/misaligned pointer, value out of range */
  PF_ERR_ARENA = 2,       /* arena too small or not 256-byte aligned */
  PF_ERR_STATE = 3,       /* call not valid in the cache's current state */
  PF_ERR_CAPACITY = 4,    /* a size exceeds a configured or built-in limit */
  PF_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed */
  PF_ERR_TIMEOUT = 6,     /* a device-side bounded wait gave up */
  PF_ERR_UNSUPPORTED = 7  /* configuration outside what the kernels support */
} pf_status;

/* partition mask bits for pf_rope_shift */
#define PF_PART_SINK 1u
#define PF_PART_MID 2u     /* live compressed blocks of the pool */
#define PF_PART_RECENT 4u  /* recent full-res blocks and their pending compressed copies */

typedef struct pf_config {
  int layers;        /* transformer layers; each has its own cache */
  int batch;         /* B: independent sequences sharing the call (e.g. CFG cond/uncond) */
  int heads;         /* H (12 for Wan2.1-1.3B) */
  int head_dim;      /* d_h; only 128 is supported */
  int block_frames;  /* B_f latent frames per block (4) */
  int h, w;          /* patches per frame after patchification (30 x 52) */
  int sink_blocks;   /* N_sink / B_f (2); may be 0 */
  int recent_blocks; /* N_recent / B_f (1); >= 1 */
  int mid_capacity;  /* compressed blocks the pool keeps before evicting the oldest */
  int n_top;         /* N_top: mid blocks routed into attention (16) */
  int rope_split[3]; /* rotary dims per axis (temporal, height, width) = 44, 42, 42 */
  float rope_base;   /* rotary base (10000) */
  int sink_rope_in_attention; /* 0: pf_rope_shift rotates the stored sink keys in place;
                                 1: it records the shift and pf_attend rotates the sink's
                                 key tiles as they are loaded (the stored keys stay as
                                 appended; see pf_rope_shift) */
} pf_config;

typedef struct pf_cache pf_cache;

typedef struct pf_layer_info {
  int blocks_seen;       /* blocks appended to this layer so far */
  int sink_filled;       /* sink blocks stored (<= sink_blocks) */
  int recent_count;      /* recent blocks stored (<= recent_blocks) */
  int recent_head;       /* recent ring slot of the oldest recent block */
  int mid_count;         /* live compressed blocks in the pool */
  int mid_head;          /* pool slot of the oldest live compressed block */
  int pool_slots;        /* mid_capacity + recent_blocks */
  int selection_valid;   /* 1 if a selection for the current pool is stored */
  int n_selected;        /* mid blocks that pf_attend will route now */
  int context_tokens;    /* keys pf_attend attends to now, current block included */
  long long evicted;     /* compressed blocks evicted so far */
  long long total_shift; /* sum of the temporal shifts applied to the sink, frames */
  void* sink_k;          /* [B, sink_blocks*n, H, D] */
  void* sink_v;
  void* pool_k;          /* [B, pool_slots, n_c, H, D], ring */
  void* pool_v;
  void* recent_k;        /* [B, recent_blocks, n, H, D], ring */
  void* recent_v;
  int32_t* selection;    /* device [B, n_top]: pool slots of the stored selection */
  float* scores;         /* device [B, pool_slots]: last block scores, by age (oldest first) */
} pf_layer_info;

/* Library version, e.g. 100 for 0.1.0. */
int pf_version(void);

/* Message of the calling thread's last failed call ("" if none). */
const char* pf_last_error(void);

/* Name of a status code. */
const char* pf_status_string(pf_status s);

/*
 * Bytes of device memory a cache with this configuration needs: the three
 * partitions of every layer plus per-layer selection scratch.  Token counts
 * follow PackForcing (arXiv), "KV Caching" (n = B_f h w) and "Compressed Mid
 * Tokens" (n_c = floor(B_f/2) floor(h/4) floor(w/4)).
 * Errors: PF_ERR_ARG for a null pointer or a non-positive size,
 * PF_ERR_UNSUPPORTED for head_dim != 128 or rope_split not summing to it,
 * PF_ERR_CAPACITY when a size limit is exceeded or the total does not fit
 * in size_t.  Limits: a block of at most 2^24 tokens, H * D <= 32768,
 * mid_capacity + recent_blocks <= 8192, and an attention context (sink +
 * min(n_top, mid_capacity) compressed blocks + recent + current, each
 * partition rounded up to 32 keys) below 2^27 keys.
 */
pf_status pf_cache_bytes(const pf_config* cfg, size_t* bytes);

/*
 * Create a cache over a caller-owned arena of at least pf_cache_bytes bytes,
 * 256-byte aligned.  Zeroes the arena on `stream` (asynchronously).  The
 * arena must outlive the cache; pf_cache_destroy frees only host state.
 * Errors: PF_ERR_ARG, PF_ERR_ARENA (too small / misaligned), PF_ERR_UNSUPPORTED,
 * PF_ERR_CAPACITY (as pf_cache_bytes; or no host memory for the layers'
 * state), PF_ERR_CUDA.
 */
pf_status pf_cache_create(const pf_config* cfg, void* dev_arena, size_t arena_bytes,
                          void* stream, pf_cache** out);

pf_status pf_cache_destroy(pf_cache* cache);

/* Host-side snapshot of one layer's state and its device addresses. */
pf_status pf_cache_layer_info(const pf_cache* cache, int layer, pf_layer_info* out);

/*
 * Append the block that has just been generated (PackForcing (arXiv),
 * "Dual-Resolution Shifting Mechanism"; "The Position Misalignment Problem").
 * K, V: [B, n, H, D], the block's full-resolution keys (already carrying
 * their RoPE rotation) and values.  Kc, Vc: [B, n_c, H, D], the compressed
 * copy computed alongside it.
 *  - While the sink is not full, the block is stored in the sink; Kc/Vc are
 *    ignored and may be NULL.
 *  - Otherwise the block becomes the newest recent block and Kc/Vc are kept
 *    with it; if the recent partition was full, its oldest block leaves it
 *    and that block's compressed copy joins the mid pool; if the pool then
 *    holds more than mid_capacity blocks, the oldest is evicted.
 * *evicted (optional) receives the number of compressed blocks evicted by
 * this call (0 or 1).  The caller then shifts the sink's temporal RoPE by
 * delta = evicted * B_f frames (pf_rope_shift).  Invalidates the layer's
 * stored selection if the pool changed.  One kernel launch.
 */
pf_status pf_cache_append_block(pf_cache* cache, int layer, const void* K, const void* V,
                                const void* Kc, const void* Vc, int* evicted, void* stream);

/*
 * Push `nblocks` compressed blocks straight into the mid pool, oldest
 * first, as if each had aged out of the recent partition: restoring a saved
 * cache, or building a long history without the full-resolution blocks.
 * Kc, Vc: [B, nblocks, n_c, H, D].  The sink must be full.  *evicted
 * (optional) receives the number of blocks evicted.  One kernel launch.
 */
pf_status pf_cache_load_mid(pf_cache* cache, int layer, const void* Kc, const void* Vc,
                            int nblocks, int* evicted, void* stream);

/*
 * Dynamic context selection (PackForcing digest, method step (3);
 * PackForcing (arXiv), "Compressed Mid Tokens"): score every live
 * compressed block of the layer's pool against the current block's queries,
 *   S[b, p] = (1/H) sum_h qbar_{b,h} . kbar_{b,p,h} / sqrt(d_h),
 * qbar / kbar the mean query of the current block and the mean key of block
 * p, per head; then keep the n_top largest (ties to the older block).  The
 * selection is stored in the arena for the layer's later pf_attend calls
 * (selection runs at a block's first denoising step; the other steps reuse
 * it).  Q: [B, n, H, D].
 * sel_out (optional, device, [B, min(n_top, mid_count)] int32): the chosen
 * blocks by age (0 = oldest live block), ascending.
 * scores_out (optional, device, [B, mid_count] float): S by age.
 * Two kernel launches (the query sums, then the scores and the top-k as a
 * programmatic dependent launch that starts while the sums are formed); no
 * host synchronisation.
 */
pf_status pf_select_mid(pf_cache* cache, int layer, const void* Q, int32_t* sel_out,
                        float* scores_out, void* stream);

/*
 * Routing policies and options of pf_select_mid_ex.
 *
 * PF_ROUTE_SCORE (the method): the scores above, optionally over a subset of
 *   the queries and heads.  The digest's limitations paragraph says the
 *   selection subsamples the query tokens and uses half of the attention
 *   heads to stay cheap; the pages give neither the sampling rule nor which
 *   half, so both are options: query rows 0, q_stride, 2 q_stride, ... and
 *   heads [head_lo, head_hi).  With heads_total > 0 the score is divided by
 *   heads_total instead of the number of heads used, so scores computed on
 *   disjoint head ranges (for example by GPUs that each hold some of the
 *   heads) add up to the all-head score.
 * PF_ROUTE_SCORES_ONLY: the same scores into scores_out (required), no
 *   top-k and no stored selection (the partial scores of a head shard).
 * PF_ROUTE_GIVEN: top-k of caller-provided scores (scores_in, device,
 *   [B, mid_count] float by age): random routing (random scores; PackForcing
 *   (arXiv), "FIFO vs. Dynamic Context Selection", the random baseline), or
 *   the sum of head shards' partial scores.  Same ranking rule and outputs as
 *   PF_ROUTE_SCORE.
 * PF_ROUTE_FIFO: the n_top most recent live blocks (the FIFO baseline of the
 *   same table: chronological retention, no scoring).  Reads no scores.
 */
#define PF_ROUTE_SCORE 0
#define PF_ROUTE_SCORES_ONLY 1
#define PF_ROUTE_GIVEN 2
#define PF_ROUTE_FIFO 3

typedef struct pf_select_opts {
  int policy;             /* PF_ROUTE_* */
  int q_stride;           /* >= 1; 1 = every query row; >= n: row 0 only */
  int head_lo, head_hi;   /* heads used by the score; head_hi = 0 means all */
  int heads_total;        /* score divisor in heads; 0 = the heads used */
  const float* scores_in; /* PF_ROUTE_GIVEN only */
} pf_select_opts;

/*
 * pf_select_mid with a routing policy (see above).  opts NULL = the method's
 * defaults (PF_ROUTE_SCORE, every query row, every head) = pf_select_mid.
 * sel_out / scores_out as for pf_select_mid (scores_out is required for
 * PF_ROUTE_SCORES_ONLY and ignored by PF_ROUTE_FIFO).  PF_ROUTE_SCORE and
 * PF_ROUTE_SCORES_ONLY launch two kernels, PF_ROUTE_GIVEN and PF_ROUTE_FIFO
 * one.  Errors: PF_ERR_ARG for a bad policy, stride, head range, or a
 * missing scores_in / scores_out.
 */
pf_status pf_select_mid_ex(pf_cache* cache, int layer, const void* Q, const pf_select_opts* opts,
                           int32_t* sel_out, float* scores_out, void* stream);

/*
 * Incremental temporal RoPE adjustment (PackForcing (arXiv), "Incremental
 * RoPE adjustment"; digest, method step (4)): multiply the stored keys'
 * temporal rotary pairs by e^{i theta_t,k delta},
 *   (x_2k + i x_2k+1) <- (x_2k + i x_2k+1) e^{i theta_k delta},
 *   theta_k = rope_base^(-2k / rope_split[0]),  k < rope_split[0] / 2,
 * in float32, rounded to bf16 (nearest even), in place.  Height and width
 * pairs and all values are left untouched.  `parts` is a mask of
 * PF_PART_SINK / PF_PART_MID / PF_PART_RECENT; the method shifts the sink.
 * layer = -1 shifts every layer.  delta is in latent frames (any sign).
 * One kernel launch per layer.
 */
pf_status pf_rope_shift(pf_cache* cache, int layer, unsigned parts, int delta, void* stream);
/*
 * With sink_rope_in_attention = 1 the sink part of a shift launches
 * nothing: the layer's total shift (pf_layer_info.total_shift) is applied
 * by pf_attend to the sink's key tiles in shared memory, between their load
 * and the QK^T MMA, with the same float32 rotation and bf16 rounding (one
 * rounding for the whole accumulated shift).  The sink must then be full
 * before its first shift (PF_ERR_STATE otherwise), since every stored sink
 * key is rotated by the same total.
 */

/*
 * Attention of the current block's queries over the bounded context
 * (PackForcing digest, KV-cache paragraph; PackForcing (arXiv), "Bounded
 * Attention Context"):
 *   O = softmax(Q K^T / sqrt(d_h)) V,  K/V = sink || selected mid || recent || current.
 * No mask.  Q, K_cur, V_cur, O: [B, n, H, D] bf16; O must not alias the
 * inputs.  lse (optional, device, [B, H, n] float): log-sum-exp of the
 * scaled scores, natural log.  Mid blocks: the stored selection if valid;
 * if the pool holds at most n_top blocks, all of them; otherwise
 * PF_ERR_STATE (call pf_select_mid first).  One kernel launch (tcgen05
 * tensor cores, TMA loads through the partitions in place), and a second
 * (the merge of the ragged last query tiles' context chunks, launched as a
 * programmatic dependent) when the block has an odd number of 128-row query
 * tiles and pf_attend_tail_plan gives more than one chunk.
 */
pf_status pf_attend(pf_cache* cache, int layer, const void* Q, const void* K_cur,
                    const void* V_cur, void* O, float* lse, void* stream);

/*
 * How pf_attend cuts the ragged last 128-row query tile of every (batch
 * item, head) along the context when a block has an odd number of query
 * tiles.  Pure host arithmetic (no device, no cache): with `full_units`
 * pairs of full query tiles and `tails` ragged tiles, each over `n_tiles`
 * 128-key tiles, on a GPU with `sms` SMs, the first *big chunks cover key
 * tiles [0, *split) in equal parts (sized so that the SMs the last wave of
 * pairs leaves idle finish them alongside it) and the next *small chunks
 * cover [*split, n_tiles) (about one per SM).  *big + *small == 1 means the
 * tiles are not split.  PF_ERR_ARG on a negative size, sms < 1 or a null
 * output.
 */
pf_status pf_attend_tail_plan(long long full_units, int tails, int n_tiles, int sms, int* big, int* small,
                              int* split);

/*
 * One layer's attention at one denoising step of the current block
 * (PackForcing (arXiv), "Implementation Details": each block is denoised in
 * S steps; digest, limitations paragraph: the context selection runs at a
 * block's first denoising step only).  step == 0: pf_select_mid with this
 * step's queries, then pf_attend; step > 0: pf_attend with the selection
 * stored at step 0 (PF_ERR_STATE if the pool changed since, or if no
 * selection was made while the pool holds more than n_top blocks).
 * Arguments as for pf_attend; step >= 0.  The selection's two kernel
 * launches at step 0, then pf_attend's.
 */
pf_status pf_attend_step(pf_cache* cache, int layer, int step, const void* Q, const void* K_cur,
                         const void* V_cur, void* O, float* lse, void* stream);

/*
 * The current block is final (its last denoising step is done): append it
 * to every layer and close the position gap of any eviction (PackForcing
 * (arXiv), "Dual-Resolution Shifting Mechanism", "Incremental RoPE
 * adjustment").  K, V, Kc, Vc: host arrays of `layers` device pointers, one
 * per layer, each as for pf_cache_append_block.  Every layer's cache moves
 * through the same states, so all layers evict together; if they evict,
 * every layer's sink is shifted by evicted * B_f frames (pf_rope_shift,
 * layer -1, PF_PART_SINK).  *evicted (optional) receives the blocks
 * evicted per layer (0 or 1).  Every pointer is checked before anything is
 * launched (PF_ERR_ARG leaves the cache unchanged); a launch failure
 * (PF_ERR_CUDA) part-way leaves the layers before the failing one appended.
 * Two launches per layer, plus one per layer for the shift.
 */
pf_status pf_finish_block(pf_cache* cache, const void* const* K, const void* const* V,
                          const void* const* Kc, const void* const* Vc, int* evicted, void* stream);

/*
 * Saving and restoring a cache.  Everything on the device (every partition,
 * the pool's mean keys, each layer's stored selection) lives in the
 * caller's arena; the library's only other state is small host state per
 * layer (ring heads and counts, blocks seen and evicted, accumulated sink
 * shift, selection validity).  To save a cache: copy its arena (after its
 * stream's work is done) and pf_cache_save_state.  To restore: create a
 * cache with the same configuration, copy the saved arena into the new
 * arena (after pf_cache_create's clearing, on the same stream or after it),
 * then pf_cache_load_state.  (Not a step of the method: an interface of
 * this library.)
 *
 * pf_cache_state_bytes: bytes of the saved host state (a header with the
 * configuration, then one record per layer).
 * pf_cache_save_state: write it into `buf` (host memory, `bytes` >= the
 * size; PF_ERR_ARG otherwise).
 * pf_cache_load_state: replace the cache's host state by a saved one.
 * PF_ERR_ARG if `buf` is not a saved state of this size and version;
 * PF_ERR_STATE if it was saved from a cache with another configuration or
 * holds counts outside the configuration's limits (the cache is then left
 * unchanged).  Launches nothing.
 */
pf_status pf_cache_state_bytes(const pf_cache* cache, size_t* bytes);
pf_status pf_cache_save_state(const pf_cache* cache, void* buf, size_t bytes);
pf_status pf_cache_load_state(pf_cache* cache, const void* buf, size_t bytes);

/*
 * Limits of pf_select_mid_static (its scratch is a fixed array in the library).
 */
#define PF_STATIC_MAX_BATCH 8
#define PF_STATIC_MAX_HEADS 16
#define PF_STATIC_MAX_BLOCKS 4096
#define PF_STATIC_MAX_NC 512

/*
 * The same block scoring and top-k selection as pf_select_mid, for callers
 * that cannot allocate device memory for this library: a serving process
 * that reserves its whole device-memory budget at start-up and allows no
 * allocation on the request path (cudaMalloc and cudaFree can synchronise
 * the device and fragment the pool), or a framework that owns the device
 * allocator and passes only its own input and output tensors, with no cache
 * arena.  This entry point allocates nothing: its scratch (query sums,
 * partial and final block scores, the chosen slots, completion tickets) is
 * one file-scope device array of about 2.4 MB, which every GPU that loads
 * the library holds until the process exits.  (It has no counterpart on the
 * pages; it is an interface choice of this library.)
 *
 * Q:       [batch, n, heads, 128] bf16, device, the current block's queries.
 * pool_k:  [batch, pool_slots, n_c, heads, 128] bf16, device, a ring of
 *          compressed keys; the live blocks, oldest first, are the slots
 *          head, head+1, ... (mod pool_slots), `count` of them.
 * sel_out: [batch, min(n_top, count)] int32, device: the chosen blocks by
 *          age (0 = oldest live block), ascending.  Required (nothing is
 *          written to it when n_top == 0).
 * scores_out (optional): [batch, count] float, device: the block scores
 *          (written for every n_top, 0 included).
 * Limits: batch <= PF_STATIC_MAX_BATCH, heads <= PF_STATIC_MAX_HEADS,
 * count <= PF_STATIC_MAX_BLOCKS, n_c <= PF_STATIC_MAX_NC; larger sizes
 * return PF_ERR_CAPACITY before any device work.
 * The first call on a device looks up the array's device address with that
 * device current (make that first call before any stream capture); the
 * address is kept for the process, so a cudaDeviceReset of that device
 * leaves it stale (do not call this again on a device after resetting
 * it).  Every call clears what must start at zero and then shares the one
 * array: calls
 * that overlap on the GPU (different streams, or different host threads,
 * on one device) race and must not be made.  Three launches on `stream`
 * (one memset, two kernels); no host synchronisation.
 */
pf_status pf_select_mid_static(const void* Q, int batch, int n, int heads, const void* pool_k, int pool_slots,
                               int n_c, int head, int count, int n_top, int32_t* sel_out, float* scores_out,
                               void* stream);

/*
 * Synchronise `stream`, then read and clear the cache's device error word.
 * Returns PF_OK, or PF_ERR_TIMEOUT if a kernel's bounded wait gave up since
 * the last poll.  *code (optional) receives the raw word (0 = none).
 */
pf_status pf_poll_device_error(pf_cache* cache, void* stream, unsigned* code);

/*
 * Self-test of the bounded device wait used by the kernels: one thread waits
 * on a barrier that nothing completes, for about `timeout_us` microseconds,
 * then records PF_ERR_TIMEOUT in the cache's error word and returns.  Lets
 * a test check the timeout path without faulting or hanging the GPU.
 */
pf_status pf_selftest_wait_timeout(pf_cache* cache, unsigned timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PF_H */
