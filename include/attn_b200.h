/*
 * attn_b200.h -- C ABI of the B200 (sm_100a) exact-attention forward library.
 *
 * Two operations, each an exact scaled-dot-product attention forward with an
 * online (blockwise, running-maximum) softmax:
 *
 *   prefill  O = softmax(Q K^T * scale + causal mask) V over whole sequences,
 *            tiled so that no S x S matrix ever reaches global memory
 *            ("flash-attention与TensorRT-LLM集成", section FlashAttention工作原理:
 *            Q/K/V are split into blocks that are loaded and released on the fly
 *            and memory stays linear in S; "LLM推理优化技术综述", PART04).
 *   decode   one new query token per sequence against its cached keys and
 *            values, which live in fixed-size pages of a shared pool addressed
 *            through a per-sequence block table ("LLM推理优化技术综述", PART02;
 *            "Optimizing Inference on LLMs with TensorRT-LLM", PagedAttention;
 *            "TensorRT对Grouped Query Attention的支持进展", 动态形状与KV Cache管理:
 *            the caller hands in physical page indices every decode step).
 *
 * Grouped-query attention: query head h reads KV head h / (Hq / Hkv)
 * ("TensorRT对Grouped Query Attention的支持进展", 技术演进背景; "LLM推理优化技术综述",
 * PART03). Hkv == Hq is MHA, Hkv == 1 is MQA.
 *
 * Optional BLASST tile skip ("高效部署稀疏注意力加速方案：BLASST方法详解与实践指南",
 * 架构与组件): with lambda > 0, a tile of 64 keys is skipped -- its V rows are not
 * loaded, and it costs no P V product and no exponentials -- when
 * exp(tile_rowmax - running_max) < lambda for every row of its decision unit.
 * The running maximum is over the unit's tiles already kept, in ascending key
 * order. lambda == 0 computes the dense result. (Exceptions, stated at the entry
 * points: a V tile shared by several decision units is loaded while one of them
 * keeps it, and a prefill warp whose rows keep a tile computes its
 * exponentials before the other warps' votes are in.)
 *
 * Common conventions
 *   - Every pointer is a DEVICE pointer owned by the caller. The library never
 *     allocates, frees or synchronises; all work is enqueued on `stream`
 *     (a cudaStream_t; NULL is the legacy default stream). A call enqueues only
 *     kernel launches (and, for decode, one small memset); kernel attributes are
 *     set at a function's first call on a device. After one eager call, the
 *     calls can be captured into a CUDA graph and replayed.
 *   - bf16 means IEEE bfloat16 (__nv_bfloat16), row-major, contiguous.
 *     Accumulation is fp32. LSE is the natural-log log-sum-exp of the scaled
 *     scores, fp32.
 *   - q/k/v/o/page pointers must be 16-byte aligned.
 *   - Head dimension D must be 64 or 128.
 *   - Return value: ATTN_OK, or an error code. Argument errors are detected on
 *     the host before anything is enqueued. Errors found on the device
 *     (out-of-range block-table entries, a pipeline wait that timed out) are
 *     reported through `device_status` when given, and through the library's
 *     device status word once attn_set_library_status(1) has switched it on.
 *     No kernel traps. The status words keep the largest code recorded.
 *   - By default the library keeps no state that calls share: its device status
 *     word is written only when switched on, and the one fixed scratch array
 *     belongs to attn_decode_paged_noalloc alone.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or lambda        */
  ATTN_ERR_UNSUPPORTED = 2,   /* device is not sm_100, or an unsupported shape */
  ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed   */
  ATTN_ERR_DEVICE_BOUNDS = 4, /* a block_table entry was outside [0, pages)    */
  ATTN_ERR_TIMEOUT = 5        /* a kernel pipeline wait expired; output invalid */
};

/* Human-readable name of a status code (static storage; never NULL). */
const char* attn_status_string(int status);

/* ABI version, bumped on any incompatible change. */
int attn_abi_version(void);

/*
 * attn_prefill -- dense causal or non-causal prefill attention.
 *
 *   q    [B][S][Hq][D]  bf16     queries
 *   k, v [B][S][Hkv][D] bf16     keys and values (key j of a sequence is token j)
 *   o    [B][S][Hq][D]  bf16     output, written completely
 *   lse  [B][Hq][S]     fp32     log-sum-exp per query row; may be NULL
 *   causal != 0: key j is visible to query i iff j <= i
 *   scale: multiplies Q K^T (typically 1/sqrt(D))
 * Requirements: B >= 1, S >= 1, Hkv >= 1, Hq % Hkv == 0, D in {64, 128}.
 * Work is (b, hq, 128-row query tile); every pair of query rows sees exactly
 * the keys the definition lets it see; ragged S is handled inside the kernel.
 */
int attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int S, int D, int causal, float scale,
                 void* stream);

/*
 * attn_prefill_blasst -- attn_prefill with the BLASST tile skip.
 *
 * Decision unit: (b, hq, query tile of rows [128 t, min(128 t + 128, S))).
 * Its tiles are the 64-key tiles in ascending order (causal: only tiles whose
 * first key is <= the unit's last row). lambda in [0, 1).
 *   skip_mask  [B][Hq][ceil(S/128)][ceil(S/64)] uint8, may be NULL. For every
 *              visited tile the kernel writes 1 (skipped) or 0 (kept); entries
 *              of tiles never visited are left untouched.
 *   skipped_tiles  one unsigned 64-bit counter on the device, may be NULL
 *              (8-byte aligned): the number of skipped decisions is added to it
 *              (the caller zeroes it).
 *   device_status  int on the device, may be NULL; set (never cleared) to a
 *              device-side error code.
 * The output and LSE are those of attention restricted to the kept keys.
 * The two query tiles of one 256-row block of a head share every K/V tile
 * load: a 64-key half of V is loaded when either of the two keeps it.
 */
int attn_prefill_blasst(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int Hq, int Hkv, int S, int D, int causal, float scale,
                        float lambda, uint8_t* skip_mask, unsigned long long* skipped_tiles,
                        int* device_status, void* stream);

/*
 * attn_prefill_paged -- chunked (append) prefill over a paged KV cache
 * ("TensorRT对Grouped Query Attention的支持进展", section 与动态批处理协同,
 * recommends chunked prefill and prefix caching; "flash-attention与TensorRT-LLM
 * 集成" runs attention against a KV cache). Causal, aligned at the end of each
 * sequence: query row i of sequence b is the token at position L_b - Sq + i
 * (L_b = seq_lens[b]) and sees the cached keys 0 .. L_b - Sq + i. The chunk's
 * own keys and values must already be in the pages.
 *
 *   q            [B][Sq][Hq][D] bf16          the chunk's queries
 *   k_pages,
 *   v_pages      [num_pages][page_size][Hkv][D] bf16   the page pool
 *   block_table  [B][max_pages_per_seq] int32 (device)
 *   seq_lens     [B] int32 (device)   L_b, with Sq <= L_b <= max_pages_per_seq * page_size;
 *                a length outside is clamped into that range and ATTN_ERR_DEVICE_BOUNDS set
 *   o            [B][Sq][Hq][D] bf16 (out)
 *   lse          [B][Hq][Sq] fp32 natural-log LSE (out), may be NULL
 *   page_size    16, 32, 64, 128 or 256;  D 64 or 128;  Hq a multiple of Hkv
 *   device_status  may be NULL (see attn_prefill_blasst)
 * A block_table entry outside [0, num_pages) for a page the sequence uses is
 * never dereferenced: its keys read as zeros and ATTN_ERR_DEVICE_BOUNDS is set.
 * Cache slots past L_b are never read. Pointers: the bf16 ones 16-byte aligned.
 * Errors as attn_prefill.
 */
int attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                       const int32_t* block_table, const int32_t* seq_lens, void* o, float* lse,
                       int B, int Sq, int Hq, int Hkv, int D, int page_size,
                       int max_pages_per_seq, int num_pages, float scale,
                       int* device_status, void* stream);

/*
 * attn_kv_append -- write the keys and values of new tokens into the paged
 * cache ("TensorRT-LLM：大模型推理优化利器", section 4: the cache keeps the K/V
 * of past tokens; "TensorRT对Grouped Query Attention的支持进展", section 动态形状
 * 与KV Cache管理: fixed-size pages addressed through physical page indices).
 * Token t of sequence b goes to position start_pos[b] + t, i.e. page
 * block_table[b][pos / page_size], slot pos % page_size; nothing else is
 * written. Run it before attn_decode_paged / attn_prefill_paged on the same
 * stream, with seq_lens then covering the new tokens.
 *   k_new, v_new  [num_seqs][T][Hkv][D] bf16 (16-byte aligned)
 *   k_pages,
 *   v_pages       [num_pages][page_size][Hkv][D] bf16, written in place
 *   block_table   [num_seqs][max_pages_per_seq] int32 (device)
 *   start_pos     [num_seqs] int32 (device): cached tokens before the append
 *   device_status may be NULL; a position past the table or a page outside
 *                 [0, num_pages) is skipped and ATTN_ERR_DEVICE_BOUNDS set
 * D 64 or 128; page_size 16, 32, 64, 128 or 256. Errors as attn_prefill.
 */
int attn_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                   const int32_t* block_table, const int32_t* start_pos, int num_seqs, int T,
                   int Hkv, int D, int page_size, int max_pages_per_seq, int num_pages,
                   int* device_status, void* stream);

/*
 * attn_decode_workspace_bytes -- scratch needed by attn_decode_paged.
 * The decode splits each sequence's keys into chunks of split_tokens tokens,
 * computes one partial (O, LSE) per (sequence, query head, chunk), and merges
 * them. The workspace holds a 256-byte header (the kernel's work counter,
 * reset by the library on every call that uses it) and those partials:
 *   fp32 [num_seqs][max_splits][Hq][D] (padded to 256 B) + fp32 [num_seqs][max_splits][Hq]
 * with max_splits = ceil(max_pages_per_seq * page_size / split_tokens).
 * Returns 0 for invalid arguments or a size that does not fit a size_t.
 */
size_t attn_decode_workspace_bytes(int num_seqs, int Hq, int D, int max_pages_per_seq,
                                   int page_size, int split_tokens);

/*
 * attn_decode_blasst_workspace_bytes -- scratch needed by attn_decode_paged and
 * attn_decode_paged_blasst_heads on their tile-skip path (lambda > 0, a
 * skip_mask or a skipped_tiles counter, or the per-head entry point). With
 * Hq / Hkv <= 8 that path runs in one or two passes over K, as
 * attn_decode_skip_passes says. One pass: each (sequence, KV head, split) is
 * walked in token order and a tile's V rows are read after its decision. Two
 * passes, for batches with too few splits to fill the GPU: the first computes
 * the scaled scores of every cached token and query head, and the row maxima
 * of every 64-token tile and of every chunk of its work; the second derives
 * the decisions from the maxima and reads V only for kept tiles. The second
 * pass's item is the largest of 256, 192, 128 and 64 tokens that divides
 * split_tokens; the first pass's chunk is that item, halved down to 64 tokens
 * while the batch has fewer than 32768 (sequence, query head, chunk) triples.
 * The size covers both paths: the scores (fp32 [num_seqs][Hq][padded
 * tokens]), the tile and chunk maxima, the running maximum at every chunk
 * start (used for splits of more than 16 chunks), and one partial (O, LSE)
 * per (sequence, query head, second-pass item). Returns 0 for invalid
 * arguments or an overflowing size.
 */
size_t attn_decode_blasst_workspace_bytes(int num_seqs, int Hq, int D, int max_pages_per_seq,
                                          int page_size, int split_tokens);

/*
 * attn_decode_skip_passes -- how many passes over the cached K the tile-skip
 * decode makes for these sizes (host arithmetic only, nothing is launched):
 * 1 when Hq / Hkv = 16 (a one-pass kernel that also reads the skipped tiles'
 * V rows) or when num_seqs * Hkv * max_splits >= 2048, with max_splits =
 * ceil(max_pages_per_seq * page_size / split_tokens); 2 otherwise. Both give
 * the same decisions; the results agree up to the rounding of a different
 * summation order. Returns 0 for arguments attn_decode_paged would reject.
 */
int attn_decode_skip_passes(int num_seqs, int Hq, int Hkv, int max_pages_per_seq, int page_size,
                            int split_tokens);

/*
 * attn_decode_paged -- single-token decode over a paged KV cache (split-KV
 * kernel followed by a log-sum-exp merge kernel).
 *
 *   q            [num_seqs][Hq][D] bf16          one query token per sequence
 *   k_pages,
 *   v_pages      [num_pages][page_size][Hkv][D] bf16   the shared page pool
 *   block_table  [num_seqs][max_pages_per_seq] int32   physical page of each
 *                logical page; entries past the last used page are ignored
 *   seq_lens     [num_seqs] int32 (device)       cached tokens per sequence;
 *                the query sees tokens [0, seq_len). 0 gives o = 0, lse = -inf.
 *                Must be <= max_pages_per_seq * page_size (checked on the
 *                device: excess tokens are dropped and ATTN_ERR_DEVICE_BOUNDS set).
 *   page_size    16, 32, 64, 128 or 256 tokens
 *   lambda       0 for dense; in (0, 1) for the BLASST skip, whose decision
 *                unit is (sequence, KV head, split): the rows are the
 *                Hq / Hkv query heads sharing the KV head, the tiles the split's
 *                64-token tiles, the running maximum restarts at each split
 *   split_tokens multiple of 64 (>= 64): tokens per split
 *   o            [num_seqs][Hq][D] bf16, lse [num_seqs][Hq] fp32 (lse may be NULL)
 *   workspace    device scratch, 16-byte aligned, contents on entry ignored, of at
 *                least attn_decode_workspace_bytes(...) bytes on the dense path and
 *                attn_decode_blasst_workspace_bytes(...) bytes on the skip path
 *   skip_mask    [num_seqs][Hkv][ceil(max_pages_per_seq*page_size/64)] uint8,
 *                may be NULL: 1 skipped / 0 kept for every visited tile; other
 *                entries untouched
 *   skipped_tiles  device counter, may be NULL (see attn_prefill_blasst)
 *   device_status  may be NULL (see attn_prefill_blasst)
 * A block_table entry outside [0, num_pages) is never dereferenced: its
 * tokens are treated as absent and ATTN_ERR_DEVICE_BOUNDS is raised.
 * Hq / Hkv must be 1, 2, 4, 8 or 16. On the skip path with Hq / Hkv <= 8 a
 * skipped tile's V rows are not read; with Hq / Hkv = 16 the skip path runs a
 * one-pass kernel that still reads them.
 * Pointers: q, pages, o and workspace 16-byte aligned; block_table, seq_lens
 * and lse 4-byte aligned; skipped_tiles 8-byte aligned.
 */
int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                      const int32_t* block_table, const int32_t* seq_lens,
                      int num_seqs, int Hq, int Hkv, int D, int page_size,
                      int max_pages_per_seq, int num_pages, float scale, float lambda,
                      int split_tokens, void* o, float* lse,
                      void* workspace, size_t workspace_bytes,
                      uint8_t* skip_mask, unsigned long long* skipped_tiles,
                      int* device_status, void* stream);

/*
 * attn_decode_paged_blasst_heads -- attn_decode_paged with the BLASST tile skip
 * ("高效部署稀疏注意力加速方案：BLASST方法详解与实践指南", section 架构与组件)
 * decided for each query head alone: the unit is (sequence, query head, split)
 * instead of the G heads that share a KV head. The page states the rule for
 * the rows of a tile without fixing which rows share a tile in decode; this is
 * the narrowest reading. A head that drops a 64-token tile gets no probability
 * mass from it; the tile's V rows are still read while another head of the
 * same KV head keeps it, and not read once all of them drop it.
 * Arguments as attn_decode_paged (the workspace is always the skip path's),
 * except:
 *   skip_mask    [num_seqs][Hq][ceil(max_pages_per_seq*page_size/64)] uint8, may be
 *                NULL: 1 skipped / 0 kept for every visited (head, tile)
 *   skipped_tiles  counts skipped (query head, tile) decisions
 *   lambda       in [0, 1); 0 decides nothing away (the dense result)
 */
int attn_decode_paged_blasst_heads(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* block_table, const int32_t* seq_lens,
                                   int num_seqs, int Hq, int Hkv, int D, int page_size,
                                   int max_pages_per_seq, int num_pages, float scale, float lambda,
                                   int split_tokens, void* o, float* lse,
                                   void* workspace, size_t workspace_bytes,
                                   uint8_t* skip_mask, unsigned long long* skipped_tiles,
                                   int* device_status, void* stream);

/*
 * attn_decode_paged_fp8 -- attn_decode_paged (dense) over a cache stored as
 * FP8 E4M3 codes. The TensorRT-LLM page ("TensorRT-LLM：大模型推理优化利器",
 * section 量化) names FP8 among the low-precision formats that cut memory and
 * bandwidth, and the integration page ("flash-attention与TensorRT-LLM集成")
 * stores in FP8; neither fixes how the codes are scaled. Reading taken: one
 * scale per pool, K = k_scale * e4m3(code), V = v_scale * e4m3(code), where
 * e4m3 is the 1-4-3 format with exponent bias 7, subnormals at exponent 0, no
 * infinities and S.1111.111 as NaN (largest finite value 448).
 *   k_codes, v_codes [num_pages][page_size][Hkv][D] uint8 device codes
 *   k_scale, v_scale finite, > 0
 * Every other argument, the layouts, the workspace (attn_decode_workspace_bytes
 * with the same sizes), the results and the errors are those of
 * attn_decode_paged with lambda = 0 and skip_mask = NULL. Supported: D = 128;
 * Hkv a multiple of 4 (Hq / Hkv = 16: Hkv = 4 or a multiple of 8);
 * Hq / Hkv in {1, 2, 4, 8, 16}; otherwise
 * ATTN_ERR_UNSUPPORTED. The query stays bf16 and is widened to f16 in the
 * kernel, so |q| must stay inside the f16 range (65504).
 */
int attn_decode_paged_fp8(const void* q, const void* k_codes, const void* v_codes,
                          float k_scale, float v_scale,
                          const int32_t* block_table, const int32_t* seq_lens,
                          int num_seqs, int Hq, int Hkv, int D, int page_size,
                          int max_pages_per_seq, int num_pages, float scale, int split_tokens,
                          void* o, float* lse, void* workspace, size_t workspace_bytes,
                          int* device_status, void* stream);

/*
 * attn_decode_paged_noalloc -- attn_decode_paged without a caller-provided
 * workspace. (Library plumbing: the pages describe no counterpart.)
 *
 * Some callers cannot allocate device memory when they decode: a serving loop
 * that reserves all of the device memory for its KV-cache pool at start-up,
 * or a latency-critical thread that must not call cudaMalloc (which may
 * synchronise the device). This entry point allocates nothing. Its split
 * partials live in a fixed array of ATTN_NOALLOC_SCRATCH_BYTES (16 MiB) of
 * device memory inside the library, which every device that loads the library
 * holds until the process exits.
 *
 * Arguments, layouts, results and errors are those of attn_decode_paged,
 * minus workspace / workspace_bytes and skipped_tiles. A call whose
 * attn_decode_workspace_bytes(num_seqs, Hq, D, max_pages_per_seq, page_size,
 * split_tokens) -- attn_decode_blasst_workspace_bytes(...) with lambda > 0 or a
 * skip_mask -- exceeds ATTN_NOALLOC_SCRATCH_BYTES returns
 * ATTN_ERR_INVALID_ARG before anything is enqueued (use a larger split_tokens
 * or attn_decode_paged).
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture. Every call on a device shares the one array and leaves its
 * contents behind (nothing in it needs clearing between calls), so calls that
 * may run at the same time on the GPU -- on different streams without an
 * ordering between them -- race on it: order them, or use attn_decode_paged
 * with separate workspaces.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                              const int32_t* block_table, const int32_t* seq_lens,
                              int num_seqs, int Hq, int Hkv, int D, int page_size,
                              int max_pages_per_seq, int num_pages, float scale, float lambda,
                              int split_tokens, void* o, float* lse,
                              uint8_t* skip_mask, int* device_status, void* stream);

/*
 * attn_set_library_status -- switch the library's device status word on the
 * current device on (enable != 0) or off (the default). While it is on, every
 * kernel of the library also records its device-side errors there (the largest
 * code wins), so independent callers on one device see each other's errors;
 * the per-call device_status arguments need no switch. Synchronous (a small
 * host-to-device copy).
 */
int attn_set_library_status(int enable);

/*
 * attn_read_device_status -- read (and, if clear != 0, reset to ATTN_OK) the
 * library's device status word on the current device. Synchronises the
 * device.
 */
int attn_read_device_status(int* status_out, int clear);

/*
 * attn_debug_prefill_timeout -- TEST ONLY: attn_prefill (dense) with a shorter
 * pipeline wait limit and, when withhold_step >= 0, one K/V ring step of every
 * CTA left out by the producer: its copy is never issued and its barrier never
 * armed, so the MMA issuer's wait for it runs out. No production caller needs
 * it. It exercises the kernels' abort path without faulting or hanging the GPU:
 * each wait gives up after wait_limit_ns (1 us .. 2 s), the CTA records
 * ATTN_ERR_TIMEOUT in device_status, lets its copies in flight land, waits for
 * its tensor-core work to finish, releases its tensor memory and returns. The
 * output is then undefined; later calls on the same context are unaffected.
 * Arguments otherwise as attn_prefill.
 */
int attn_debug_prefill_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int Hq, int Hkv, int S, int D, int causal, float scale,
                               unsigned long long wait_limit_ns, int withhold_step,
                               int* device_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
