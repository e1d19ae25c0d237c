/*
 * mla.h -- C ABI of the B200 (sm_100a) paged MLA decode library (libmla_b200.so).
 *
 * Operation (Multi-head Latent Attention decode over a paged latent cache; the
 * FlashMLA release article «DeepSeek open-sources FlashMLA», shoujike.com.cn,
 * paragraphs on the MLA decode kernel for variable-length sequences, on the paged
 * BF16 kvcache with block size 64 and on compressing keys and values into one latent
 * vector per token):
 *
 *   every query row r = (i, h) of sequence b attends to the visible tokens t < n_i of
 *   that sequence, n_i = L_b - s_q + i + 1 when causal, else L_b;
 *   K_t is the token's 576-dim latent cache row (512 latent + 64 rope dims), shared by
 *   all heads, and V_t is its first 512 dims;
 *     s_t    = scale * <q[b,i,h,:], K_t>
 *     out    = sum_t softmax(s)_t * V_t            (bf16, round-to-nearest-even)
 *     lse    = ln sum_t exp(s_t)                   (fp32, natural log)
 *   A row with no visible token gets out = 0 and lse = -inf.
 *
 * Data layout (all tensors dense, row-major, caller-owned device memory):
 *   q            bf16  [batch][s_q][h_q][576]
 *   kcache       bf16  [num_blocks][64][1][576]      pool of 64-token pages
 *   block_table  int32 [batch][max_blocks]           physical page of logical page j
 *   seqlens      int32 [batch]                       0 <= L_b <= 64 * max_blocks
 *   out          bf16  [batch][s_q][h_q][512]
 *   lse          fp32  [batch][h_q][s_q]
 * Query rows are numbered r = i * h_q + h and cut into tiles of 128 rows; a
 * "work sequence" is one (tile, sequence) pair, v = tile * batch + b.
 *
 * Ownership: the library allocates nothing on these calls. The caller owns every
 * buffer, including `metadata`, `num_splits` and `workspace`, and must keep them alive
 * until the stream work that uses them has finished.
 *
 * Asynchrony: mla_get_metadata and mla_decode_fwd only enqueue work on `stream`
 * (a cudaStream_t passed as void*; NULL is the legacy default stream) and never
 * synchronise it. The first mla_decode_fwd on a device also sets the kernel's
 * shared-memory limit and queries its cluster occupancy once (cached afterwards).
 * The decode calls launch their split kernel with programmatic stream serialization
 * (CUDA's programmatic dependent launch): it may be scheduled while the kernel before
 * it on `stream` (normally mla_get_metadata's) still runs, but it reads and writes no
 * global memory before that kernel has completed, so stream order holds as for any
 * launch. The calls can be captured into a CUDA graph.
 *
 * Errors: every call checks its arguments on the host first and returns a negative
 * mla_status without launching anything when they are invalid. A launch failure is
 * MLA_ERR_CUDA. Problems only the device can see (a sequence longer than its block
 * table, a block id outside the pool, a pipeline wait that ran out of its iteration
 * limit) never trap: the kernel skips the offending access, records a code in a
 * device-side error word and finishes; mla_get_last_device_error reports and clears
 * it. Outputs of a call that recorded an error are unspecified.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every declaration below is exported from libmla_b200.so (built with hidden default
 * visibility). */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef int mla_status;

#define MLA_OK                        0
#define MLA_ERR_INVALID_ARG          -1  /* null pointer, bad size, misaligned buffer   */
#define MLA_ERR_UNSUPPORTED          -2  /* shape outside the supported set             */
#define MLA_ERR_CUDA                 -3  /* a CUDA runtime/driver call failed           */
#define MLA_ERR_WORKSPACE_TOO_SMALL  -4  /* workspace_bytes < mla_workspace_bytes(...)  */
#define MLA_ERR_DEVICE_TIMEOUT       -5  /* a bounded pipeline wait gave up             */
#define MLA_ERR_DEVICE_BAD_INPUT     -6  /* seqlen > 64*max_blocks or block id >= pool  */

#define MLA_HEAD_DIM        576   /* latent (512) + rope (64) dims per cache row      */
#define MLA_HEAD_DIM_V      512   /* V = first 512 dims of the row                    */
#define MLA_BLOCK_SIZE       64   /* tokens per page                                  */
#define MLA_TILE_ROWS       128   /* query rows per work tile                         */
#define MLA_MAX_H_Q         128
#define MLA_MAX_S_Q          16
#define MLA_MAX_ROWS       1024   /* s_q * h_q                                        */
#define MLA_MAX_BATCH     65536
#define MLA_METADATA_INTS_PER_UNIT 8
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)  /* scratch of mla_decode_fwd_noalloc */
#define MLA_MAX_PARTS      1024   /* parts mla_combine_partials merges            */
#define MLA_FP8_ROW_BYTES   656   /* one token's row in the FP8 cache format        */

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(mla_status status);

/* Number of int32 entries `metadata` must hold for a given num_sms (>= 1):
 * 8 * (num_sms + 1). */
size_t mla_metadata_ints(int num_sms);

/* Number of int32 entries `num_splits` must hold: batch * ceil(s_q*h_q/128) + 1. */
size_t mla_num_splits_len(int batch, int h_q, int s_q);

/* Bytes of `workspace` mla_decode_fwd needs for these sizes (fp32 split partials:
 * one [128][512] output tile and one [128] lse tile per possible split). Returns 0
 * for sizes the library rejects. */
size_t mla_workspace_bytes(int batch, int h_q, int s_q, int num_sms);

/* Work units a schedule for `num_sms` uses on the current device for these shapes.
 * Sequences of at most 64 query rows (s_q * h_q <= 64) run on the 1-CTA kernel, one unit
 * per SM: min(num_sms, co-resident CTAs). Larger ones run on the 2-CTA kernel, one unit
 * per pair of SMs: min(num_sms / 2, co-resident 2-CTA clusters). At least 1. Returns a
 * negative mla_status on failure or for unsupported shapes. */
int mla_num_work_units(int num_sms, int h_q, int s_q);

/*
 * Split-KV tile scheduler (variable-length batches: FlashMLA release article,
 * paragraph on dynamic sequence handling). Balances the pages of all work sequences
 * over the work units: every page of every work sequence is owned by exactly one
 * unit, each unit owns one contiguous run of pages in (v, page) order, and a work
 * sequence whose pages span k units is split into k chunks merged by the combine
 * step of mla_decode_fwd.
 *
 *   seqlens     device int32 [batch]
 *   num_sms     SMs the decode may use (>= 1); 148 on a B200. num_sms = 1 forces a
 *               single unit and so no splits.
 *   metadata    device int32 [mla_metadata_ints(num_sms)], written:
 *               [0..7]   header {num_units, tiles, batch, h_q, s_q, unit_cost,
 *                        item_overhead, tile_aligned}: a work sequence costs its pages
 *                        plus item_overhead (3 for the 2-CTA kernel; for the 1-CTA
 *                        kernel 1 up to 32 query rows, 2 for 33-64). With tiles > 1
 *                        row tiles per sequence and at least `tiles` units
 *                        (tile_aligned = 1), tile t owns units
 *                        [floor(t U/tiles), floor((t+1) U/tiles)) and balances the
 *                        batch's pages over them alone, so the tiles of a sequence
 *                        stream its pages at the same time and DRAM serves each page
 *                        once; unit_cost is then the largest of the tiles' costs.
 *               [8u+8..] unit u {v_begin, page_begin, v_end, page_end, chunk_begin,0,0,0}
 *                        (half-open range of (v, page) positions)
 *   num_splits  device int32 [mla_num_splits_len(batch, h_q, s_q)], written: the
 *               exclusive prefix sum over work sequences of their chunk counts, so
 *               chunks of v are num_splits[v] .. num_splits[v+1]-1.
 * The result depends only on (seqlens, batch, h_q, s_q, num_sms) and the device.
 */
mla_status mla_get_metadata(const int32_t* seqlens, int batch, int h_q, int s_q, int num_sms,
                            int32_t* metadata, int32_t* num_splits, void* stream);

/*
 * Decode attention (see the operation above). Runs an sm_100a split kernel (TMA page
 * gather -> tcgen05 QK^T and PV with TMEM accumulators -> fp32 online softmax with tail
 * and causal masks) and then the LSE-weighted combine kernel. Sequences of at most 64
 * query rows (s_q * h_q <= 64) use a 1-CTA kernel with a transposed PV (O^T = V^T P^T);
 * larger ones use 2-CTA pairs that split each 128-row tile between two SMs.
 *
 *   q, kcache, block_table, seqlens, out, lse: device buffers in the layout above;
 *     q, kcache and out must be 16-byte aligned.
 *   num_blocks  pages in the pool (>= 1); max_blocks  columns of block_table (>= 1)
 *   scale       softmax scale applied to q.K (finite)
 *   causal      0 or 1
 *   metadata, num_splits  from mla_get_metadata with the same seqlens, batch, h_q, s_q
 *   workspace   device scratch of workspace_bytes >= mla_workspace_bytes(batch, h_q,
 *               s_q, num_sms of the metadata call), 256-byte aligned.
 * Supported: 1 <= h_q <= 128, 1 <= s_q <= 16, s_q*h_q <= 1024, 1 <= batch <= 65536.
 */
mla_status mla_decode_fwd(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                          const int32_t* block_table, int max_blocks,
                          const int32_t* seqlens, int batch, int s_q, int h_q,
                          float scale, int causal,
                          const int32_t* metadata, const int32_t* num_splits,
                          void* workspace, size_t workspace_bytes,
                          uint16_t* out, float* lse, void* stream);

/*
 * mla_decode_fwd without a workspace argument, for callers that cannot hand the
 * library a scratch buffer. Examples are a serving runtime whose device memory is laid
 * out once at start-up and may not grow between decode steps, and a caller whose
 * allocator cannot give out temporary blocks on the decode path (an allocation there
 * may synchronise the device or fragment a pre-planned pool). The pages describe no
 * such call: FlashMLA's own interface is not given there, so this has no counterpart
 * in them and is an addition of this library.
 *
 * Arguments, layouts, results and errors are those of mla_decode_fwd, minus
 * `workspace` and `workspace_bytes`. The split partials go to a scratch array of
 * MLA_NOALLOC_SCRATCH_BYTES (64 MiB) that lives inside the library as static device
 * memory, one copy per device, created when the library's kernels are loaded there.
 * Neither this call nor its set-up allocates device or host memory.
 *
 *   Limit: sizes whose worst-case partials exceed the array, over every schedule the
 *     current device can run (one [128][512] fp32 tile per work sequence plus one per
 *     work unit), return MLA_ERR_WORKSPACE_TOO_SMALL before anything is launched. The
 *     array holds 255 tiles. On a 148-SM B200 that admits batch * ceil(s_q*h_q/128) up
 *     to 181 when s_q*h_q > 64 (74 units) and batch up to 107 when s_q*h_q <= 64 (148
 *     units). Larger batches must use mla_decode_fwd with a workspace.
 *   First call: the first call on each device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress) and does mla_decode_fwd's one-time
 *     kernel set-up. Make that first call before any stream capture begins. The address
 *     is cached for the life of the process: after cudaDeviceReset (or any other
 *     teardown of the device's primary context) this entry point must not be called
 *     again in that process.
 *   Sharing: every call on a device, from any stream or host thread, uses the same
 *     array, which keeps the partials of the last call. Nothing in it has to start at
 *     zero: a call reads only partials it has written itself.
 *   Races: calls whose GPU work can overlap (different streams with no ordering between
 *     them, or host threads launching on unsynchronised streams) write the same array
 *     and corrupt each other's results. Order them on one stream or with events.
 */
mla_status mla_decode_fwd_noalloc(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                                  const int32_t* block_table, int max_blocks,
                                  const int32_t* seqlens, int batch, int s_q, int h_q,
                                  float scale, int causal,
                                  const int32_t* metadata, const int32_t* num_splits,
                                  uint16_t* out, float* lse, void* stream);

/*
 * mla_decode_fwd with an fp32 output: identical arguments, layouts, checks and
 * results, except that `out_f32` (device fp32 [batch][s_q][h_q][512], 16-byte aligned)
 * receives the normalised output unrounded instead of a bf16 `out`. It gives the
 * per-device partials of a split across devices (mla_combine_partials), where a bf16
 * rounding of every partial would add up. A row with no visible token gets out = 0,
 * lse = -inf, as in mla_decode_fwd.
 */
mla_status mla_decode_fwd_partial(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                                  const int32_t* block_table, int max_blocks,
                                  const int32_t* seqlens, int batch, int s_q, int h_q,
                                  float scale, int causal,
                                  const int32_t* metadata, const int32_t* num_splits,
                                  void* workspace, size_t workspace_bytes,
                                  float* out_f32, float* lse, void* stream);

/*
 * Split-KV across devices: merges `parts` partial results of the same query rows,
 * each computed (by mla_decode_fwd_partial, usually on another device) over a disjoint
 * token range of every sequence. This is the split-KV combine of mla_decode_fwd (the
 * FlashMLA release article, paragraph on dynamic sequence handling) with the parts
 * coming from devices instead of work units; the pages describe no multi-device
 * decode, so the partitioning across devices is this library's addition. For each
 * row r of sequence b, with lse_g the part's natural-log lse:
 *     lse = ln sum_g exp(lse_g)
 *     out = sum_g exp(lse_g - lse) * O_g                  (bf16, round-to-nearest-even)
 * Parts with lse_g = -inf weigh nothing (their O_g is not read); a row that no part
 * sees gets out = 0, lse = -inf.
 *
 *   o_parts    device fp32 [parts][batch][s_q][h_q][512], 16-byte aligned (read)
 *   lse_parts  device fp32 [parts][batch][h_q][s_q] (read)
 *   out        device bf16 [batch][s_q][h_q][512], 16-byte aligned (written)
 *   lse        device fp32 [batch][h_q][s_q] (written)
 * Supported: 1 <= parts <= MLA_MAX_PARTS and the shapes of mla_decode_fwd. Invalid
 * arguments return an error before any launch. Asynchronous on `stream`; allocates
 * nothing. The caller gathers the parts into one buffer first (an all-gather over the
 * devices of the split).
 */
mla_status mla_combine_partials(const float* o_parts, const float* lse_parts, int parts,
                                int batch, int s_q, int h_q, uint16_t* out, float* lse,
                                void* stream);

/*
 * Cache append: writes s_new new latent rows per sequence into the paged cache, the
 * step that block-based paging implies before each decode (the paging of
 * «DeepSeek booste les performances des GPU NVIDIA Hopper H800…», tomshardware.fr,
 * paragraph on block-based paging that allocates memory dynamically; 64-token blocks
 * per the FlashMLA release article). For each sequence b and j < s_new:
 *     t = seqlens[b] + j
 *     kcache[block_table[b][t / 64]][t % 64][0][:] = kv_new[b][j][:]     (576 bf16)
 * a byte copy; nothing else in the cache changes.
 *
 *   kv_new       device bf16 [batch][s_new][576], 16-byte aligned
 *   block_table  device int32 [batch][max_blocks]: the pages, including the ones the
 *                new positions fall in (the caller allocates them first)
 *   seqlens      device int32 [batch]: tokens already cached (not modified: the caller
 *                advances each length by s_new afterwards)
 *   kcache       device bf16 [num_blocks][64][1][576], 16-byte aligned, written
 * Supported: 1 <= s_new <= 16, 1 <= batch <= 65536. Invalid arguments return an error
 * before any launch. A position past the block table or a block id outside the pool is
 * a device-side bad input (see mla_get_last_device_error); that row is not written.
 * Asynchronous on `stream`; allocates nothing.
 */
mla_status mla_kv_append(const uint16_t* kv_new, int s_new, const int32_t* block_table,
                         int max_blocks, const int32_t* seqlens, int batch, uint16_t* kcache,
                         int num_blocks, void* stream);

/*
 * FP8 cache append: quantizes s_new new latent rows per sequence into an FP8 paged cache,
 * the write side of an FP8 latent cache. The pages fix no FP8 cache format (they use
 * FP8 for GEMMs with fine-grained scaling factors, the DeepGEMM page on 618zxw.cn); this
 * one is the library's own. Per token, 656 bytes (MLA_FP8_ROW_BYTES):
 *     [0, 512)    the 512 latent dims as E4M3 codes (largest finite 448, no infinities)
 *     [512, 528)  four fp32 scales, one per 128-dim group g: s_g = fp32(amax_g / 448)
 *     [528, 656)  the 64 rope dims, unchanged bf16
 * code = E4M3(fp32(x / s_g)), round-to-nearest-even, saturated at +-448; 0 when s_g = 0.
 * A value reads back as code * s_g. Positions are those of mla_kv_append:
 *     t = seqlens[b] + j  ->  row t % 64 of page block_table[b][t / 64]
 *
 *   kv_new       device bf16 [batch][s_new][576], 16-byte aligned
 *   block_table, seqlens  as for mla_kv_append (seqlens not modified)
 *   kcache_fp8   device uint8 [num_blocks][64][656], 16-byte aligned, written
 * Supported: 1 <= s_new <= 16, 1 <= batch <= 65536. Invalid arguments return an error
 * before any launch; a position past the block table or a block id outside the pool is a
 * device-side bad input and that row is not written. A group holding a NaN gets NaN codes
 * and a NaN scale. Asynchronous on `stream`; allocates nothing. mla_decode_fwd_fp8
 * decodes over this format.
 */
mla_status mla_kv_append_fp8(const uint16_t* kv_new, int s_new, const int32_t* block_table,
                             int max_blocks, const int32_t* seqlens, int batch,
                             uint8_t* kcache_fp8, int num_blocks, void* stream);

/*
 * Decode attention over an FP8 latent cache in the row format of mla_kv_append_fp8:
 * exactly mla_decode_fwd's operation over the rows as the format reads them back,
 *     latent dim d of group g:  bf16(fp32(E4M3 value(code_d) * s_g))   (both nearest-even)
 *     rope dims:                as stored (bf16)
 * so its results are those of mla_decode_fwd over a bf16 cache holding the read-back
 * rows, within the same tolerances. The format is this library's (the pages use FP8 for
 * GEMMs with fine-grained scale factors, the DeepGEMM page's paragraph on fine-grained
 * scaling, not for the KV cache). It streams 656 bytes per token instead of 1,152.
 *
 *   kcache_fp8  device uint8 [num_blocks][64][656] (MLA_FP8_ROW_BYTES per row),
 *               16-byte aligned (read)
 *   every other argument as for mla_decode_fwd, with metadata, num_splits and the
 *   workspace size from the same calls for the same shapes.
 * Supported: s_q * h_q <= 64, the row counts of the 1-CTA kernel that runs it; larger
 * row counts return MLA_ERR_UNSUPPORTED before any launch. The kernel lands each page's
 * codes, scales and rope dims in one shared-memory stage and widens the codes to bf16 in
 * place before the page's QK; rows past a sequence's end widen to zeros whatever their
 * bytes hold (NaN codes or scales included).
 */
mla_status mla_decode_fwd_fp8(const uint16_t* q, const uint8_t* kcache_fp8, int num_blocks,
                              const int32_t* block_table, int max_blocks,
                              const int32_t* seqlens, int batch, int s_q, int h_q,
                              float scale, int causal,
                              const int32_t* metadata, const int32_t* num_splits,
                              void* workspace, size_t workspace_bytes,
                              uint16_t* out, float* lse, void* stream);

/*
 * Reads and clears the device-side error word of the current device after
 * synchronising `stream`. Returns MLA_OK, MLA_ERR_DEVICE_TIMEOUT,
 * MLA_ERR_DEVICE_BAD_INPUT or MLA_ERR_CUDA. *detail (may be NULL) receives the raw
 * word: bits 0-7 the error kind, the rest where it arose.
 */
mla_status mla_get_last_device_error(void* stream, uint32_t* detail);

/*
 * What MLA_ERR_DEVICE_TIMEOUT leaves behind: a pipeline wait ran out of its limit (2 s by
 * default), which only a broken input, a broken kernel or a stalled device can cause.
 * The CTA that gave up stops every role, waits (again with the limit) for the MMAs it
 * issued and, in the 1-CTA kernel, for its own copies, then frees its TMEM and exits;
 * in the 2-CTA kernel a copy still in flight is only given a fixed 50 us to land. Treat
 * the results of that call as garbage and, if timeouts repeat, the device context as
 * suspect.
 *
 * Test hook for the bounded waits (not for production use). With stall = 1, every
 * decode kernel launched afterwards (mla_decode_fwd and its variants) has its loader wait
 * on a barrier that nothing completes, before it issues any copy, so every wait of the
 * kernel gives up after `wait_limit_ns`: the kernel records MLA_ERR_DEVICE_TIMEOUT and
 * exits normally with nothing in flight, and the device stays usable. stall = 0 restores
 * normal decoding. wait_limit_ns sets the limit of every wait (0 restores the default
 * of 2 s). Both settings live on the current device, where the call writes them
 * synchronously; every later launch on that device reads them.
 */
mla_status mla_test_set_stall(int stall, unsigned long long wait_limit_ns);

/*
 * Host-side copy of the scheduler, for tests and for callers that plan on the CPU:
 * the same arithmetic as mla_get_metadata with an explicit unit count, on host
 * buffers (seqlens_host [batch], metadata_host [8*(num_units+1)],
 * num_splits_host [mla_num_splits_len]). Needs no GPU.
 */
mla_status mla_plan_host(const int32_t* seqlens_host, int batch, int h_q, int s_q,
                         int num_units, int32_t* metadata_host, int32_t* num_splits_host);

/*
 * Correctness-first decode on CUDA cores (one warp per query row, no tensor cores).
 * Same arguments, layouts, metadata and combine as mla_decode_fwd; kept as an
 * independent second kernel for cross-checking the tensor-core path.
 */
mla_status mla_decode_fwd_simt(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                               const int32_t* block_table, int max_blocks,
                               const int32_t* seqlens, int batch, int s_q, int h_q,
                               float scale, int causal,
                               const int32_t* metadata, const int32_t* num_splits,
                               void* workspace, size_t workspace_bytes,
                               uint16_t* out, float* lse, void* stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MLA_B200_H_ */
