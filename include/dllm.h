/*
 * dllm.h - C ABI of the mask-only logits + confidence-unmasking decode step for B200 (sm_100a).
 *
 * One denoising step of a diffusion LLM takes hidden states H[B*L, d] and a mask M[B, L]
 * (nonzero = the position still holds [MASK]).  The Mosaic page ("Mosaic: Unlocking
 * Long-Context Inference for Diffusion LLMs via Global Memory Planning and Dynamic Peak
 * Taming", TL;DR and Abstract) builds a mask-only logits kernel: the LM head is applied to
 * the masked rows only, so the [L, V] logits tensor of a plain implementation is never
 * needed.  This library
 *   1. compacts the masked positions with a prefix sum            (dllm_mask_compact),
 *   2. multiplies only those rows by the vocabulary projection W[V, d] on the tensor cores
 *      and reduces every row to (predicted token, log-sum-exp, confidence) in the GEMM
 *      epilogue, without ever storing a logit                       (dllm_masked_logits),
 *   3. picks, per sequence, the k most confident masked positions to unmask
 *      (confidence-driven unmasking, dLLM inference survey page, "Main Findings";
 *      an optional per-sequence window restricts candidates to the current
 *      semi-autoregressive block, Sparse-dLLM page, "Experiment")  (dllm_select_unmask).
 * and around these:
 *   - the whole step in one call (dllm_decode_step), or with logits for the current
 *     block's rows only (dllm_decode_block_step, dllm_masked_logits_window,
 *     dllm_mask_compact_window);
 *   - entropy / top-2 margin scores and threshold-based parallel unmasking
 *     (dllm_masked_logits_ex, dllm_select_unmask_ex);
 *   - the staging of a step split from its GEMM, for overlapping steps
 *     (dllm_prepare_rows, dllm_masked_logits_prepared);
 *   - a vocabulary-parallel LM head over several GPUs: per-shard softmax partials and their
 *     merge (dllm_masked_partials, dllm_lse_merge);
 *   - compaction without a workspace (dllm_mask_compact_noalloc).
 *
 * Conventions for every call:
 *   - Pointers marked "device" must point to memory of the current CUDA device; the caller
 *     owns every buffer.  The library never allocates device memory on its own: scratch
 *     space is the caller's workspace, sized by dllm_workspace_bytes() (or, for a known
 *     masked count, dllm_workspace_bytes_rows()); a dllm_arena maps device memory only
 *     when the caller asks it to.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All
 *     work is enqueued asynchronously on it; no call synchronises the host except
 *     dllm_get_status() and dllm_prof_end().  Kernels are launched with programmatic
 *     stream serialization: a kernel may begin its set-up while the previous kernel on the
 *     stream finishes, but it reads or writes no global memory before every earlier kernel
 *     on the stream has completed, so stream order is preserved.
 *   - Arguments are validated on the host before anything is launched; an invalid call
 *     returns a negative status and enqueues nothing.
 *   - Errors detected on the device (a wait that gave up, a failed bound check) are
 *     recorded in a per-device status word; dllm_get_status() reports and clears it.
 *   - bf16 tensors are passed as their raw 16-bit patterns (uint16_t).
 *   - Device pointers must be 16-byte aligned.
 *   - The step inputs H and M (of dllm_masked_logits*, dllm_masked_partials,
 *     dllm_prepare_rows and the decode-step calls) may instead be page-locked host memory
 *     (cudaHostAlloc / cudaHostRegister / a pinned torch tensor): the kernels then read it
 *     over the bus directly, so only the bytes they touch move -- the mask and the masked
 *     rows of H, not all of H.  Pageable host memory gives DLLM_ERR_MEMORY.  The memory
 *     must stay valid and unchanged until the call's kernels have run.
 */
#ifndef DLLM_H
#define DLLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t dllm_status;

#define DLLM_OK              0
#define DLLM_ERR_NULL       -1   /* a required pointer is NULL                              */
#define DLLM_ERR_ALIGN      -2   /* a device pointer is not 16-byte aligned                 */
#define DLLM_ERR_SHAPE      -3   /* B, L, d, V or k out of range (see each call)            */
#define DLLM_ERR_WORKSPACE  -4   /* workspace too small (see dllm_workspace_bytes_rows)      */
#define DLLM_ERR_CUDA       -5   /* a CUDA runtime/driver call failed                       */
#define DLLM_ERR_TIMEOUT    -6   /* a device-side wait exceeded its limit (kernel returned) */
#define DLLM_ERR_DEVICE     -7   /* the current device is not an sm_100 GPU                 */
#define DLLM_ERR_BOUNDS     -8   /* a device-side bound check failed (access skipped)       */
#define DLLM_ERR_SCRATCH    -9   /* B*L exceeds the fixed scratch of dllm_mask_compact_noalloc */
#define DLLM_ERR_MEMORY     -10  /* an input is neither device memory nor page-locked host memory */
#define DLLM_ERR_CAPACITY   -11  /* more masked rows than the workspace was sized for (device) */

/* Limits. */
#define DLLM_MAX_K          1024 /* largest k accepted by dllm_select_unmask                */
#define DLLM_D_MULTIPLE     64   /* d must be a positive multiple of this                   */

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
int32_t dllm_version(void);

/* Human-readable text for a status code (static storage; never NULL). */
const char* dllm_status_string(dllm_status s);

/*
 * Workspace size in bytes for a step with these shapes: an upper bound that does not depend
 * on how many positions are masked.  It covers the compaction tile counts, the gathered
 * masked hidden rows (B*L*d bf16 at most) and the per-row vocabulary-split partials.
 * Returns 0 if the shapes are invalid (B, L, d, V < 1, d % 64 != 0 or B*L >= 2^31).
 * Needs no GPU.
 */
size_t dllm_workspace_bytes(int32_t B, int32_t L, int32_t d, int32_t V);

/*
 * Workspace sized for steps with at most max_rows masked rows (a step's gathered rows and
 * partials grow with its masked count; the Mosaic page, Fig. 3, shows how that count sets
 * the step's memory peak as the mask ratio changes).  A caller that knows its masked count
 * -- a decoding loop does: it built the mask -- can hold a workspace of this size instead of
 * the upper bound, e.g. mapped on demand in a dllm_arena.  max_rows >= B*L gives
 * dllm_workspace_bytes().  Returns 0 for invalid shapes or max_rows < 1.  Needs no GPU.
 *
 * Every call that takes a workspace (ws, ws_bytes) accepts one smaller than
 * dllm_workspace_bytes(): its masked-row capacity is then the largest max_rows whose size
 * fits in ws_bytes (dllm_workspace_rows).  DLLM_ERR_WORKSPACE is returned only when not even
 * one row fits.  A step whose mask has more masked rows than the capacity computes the
 * first `capacity` rows, leaves the rest of tok/conf/lse untouched, touches no workspace
 * byte past ws_bytes, and records DLLM_ERR_CAPACITY for dllm_get_status(): its selection is
 * then not valid.
 */
size_t dllm_workspace_bytes_rows(int32_t B, int32_t L, int32_t d, int32_t V, int64_t max_rows);

/* Masked-row capacity of a workspace of ws_bytes for these shapes (B*L when it holds the
 * upper bound; 0 when too small for one row or for invalid shapes).  Needs no GPU. */
int64_t dllm_workspace_rows(int32_t B, int32_t L, int32_t d, int32_t V, size_t ws_bytes);

/*
 * dllm_arena - device memory behind one fixed virtual address range, backed by physical
 * memory on demand: the "global memory manager with virtual memory mapping" of the Mosaic
 * page (TL;DR and Abstract; Fig. 4 compares the memory it reserves with the theoretical
 * peak).  The whole range is reserved once (cuMemAddressReserve) and never moves, so its
 * address can be kept in a workspace argument, a tensor map or a CUDA graph; only the
 * prefix [0, mapped) is backed by physical memory (cuMemCreate + cuMemMap, in chunks).
 * Growing or shrinking the mapped prefix to what the next step needs
 * (dllm_workspace_bytes_rows of its masked count) keeps the memory held close to the
 * step's own requirement instead of the worst case over all masks.
 *
 * The arena is the one object of this library that allocates device memory, and only when
 * the caller asks it to (dllm_arena_create, dllm_arena_map).  It is not thread-safe: one
 * thread at a time per arena.
 *
 * dllm_arena_create: reserve `reserve_bytes` (rounded up to the chunk size) of virtual
 * address space on the current device, with nothing mapped.  chunk_bytes = the unit in
 * which physical memory is created, mapped and released (rounded up to the device's
 * allocation granularity; 0 = that granularity, 2 MiB on B200).  *out receives the arena.
 * Errors: DLLM_ERR_NULL (out), DLLM_ERR_SHAPE (reserve_bytes == 0), DLLM_ERR_CUDA (the
 * reservation or a driver query failed), DLLM_ERR_DEVICE.
 *
 * dllm_arena_map: make [0, bytes) usable, in whole chunks: chunks are created and mapped
 * (read-write for the current device) up to round_up(bytes, chunk); chunks wholly past that
 * point are unmapped and released.  Before it releases anything it synchronises the device
 * (cudaDeviceSynchronize), so no kernel still running can touch memory being released;
 * growing does not synchronise.  On a failed grow every chunk created by this call is
 * released again and the arena keeps its previous mapping.  Errors: DLLM_ERR_NULL,
 * DLLM_ERR_SHAPE (bytes > the reserved size), DLLM_ERR_CUDA (out of device memory or a
 * driver call failed).
 *
 * dllm_arena_ptr: base device address of the range (16-byte aligned; fixed for the arena's
 * life).  dllm_arena_reserved / dllm_arena_mapped / dllm_arena_chunk: the reserved size,
 * the bytes currently backed by physical memory, the chunk size.
 *
 * dllm_arena_destroy: synchronise the device, unmap and release every chunk, free the
 * reservation and the arena object.  NULL is accepted (no-op).
 */
typedef struct dllm_arena dllm_arena;
dllm_status dllm_arena_create(size_t reserve_bytes, size_t chunk_bytes, dllm_arena** out);
dllm_status dllm_arena_map(dllm_arena* arena, size_t bytes);
void* dllm_arena_ptr(const dllm_arena* arena);
size_t dllm_arena_reserved(const dllm_arena* arena);
size_t dllm_arena_mapped(const dllm_arena* arena);
size_t dllm_arena_chunk(const dllm_arena* arena);
dllm_status dllm_arena_destroy(dllm_arena* arena);

/*
 * dllm_mask_compact - prefix-sum compaction of the mask (Mosaic page, Abstract: logits are
 * computed for masked positions only).
 *
 *   M        device, uint8 [B, L] row-major; nonzero = masked.
 *   row_idx  device, int32 [B*L] capacity; on return row_idx[0:count] holds the flattened
 *            positions b*L + l of the masked entries in ascending order.  Entries at and
 *            past `count` are left untouched.
 *   seq_off  device, int32 [B + 1]; seq_off[b] = number of masked positions in sequences
 *            0..b-1, so sequence b owns compacted rows seq_off[b] .. seq_off[b+1]-1.
 *   count    device, int32 [1]; the number of masked positions.  It stays on the device:
 *            later calls size their work from it without a host round trip.
 *   ws       device workspace of at least dllm_workspace_bytes(B, L, 64, 1) bytes.
 * Errors: DLLM_ERR_NULL, DLLM_ERR_ALIGN (M, row_idx, seq_off, ws), DLLM_ERR_SHAPE
 * (B < 1, L < 1, B*L >= 2^31), DLLM_ERR_WORKSPACE, DLLM_ERR_CUDA, DLLM_ERR_DEVICE.
 */
dllm_status dllm_mask_compact(const uint8_t* M, int32_t B, int32_t L,
                              int32_t* row_idx, int32_t* seq_off, int32_t* count,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * dllm_mask_compact_window - dllm_mask_compact restricted to one window per sequence: the
 * compacted rows are the masked positions l of sequence b with win_lo[b] <= l < win_hi[b]
 * (semi-autoregressive decoding works on the current block of each sequence only,
 * Sparse-dLLM page, "Experiment").  row_idx, seq_off and count then describe those rows
 * only.  Any window values are accepted (win_lo[b] >= win_hi[b] is an empty window).
 *
 *   win_lo, win_hi  device int32 [B], both non-NULL, or both NULL (= dllm_mask_compact).
 * Other arguments, outputs and errors as in dllm_mask_compact; DLLM_ERR_NULL if exactly
 * one window pointer is NULL.
 */
dllm_status dllm_mask_compact_window(const uint8_t* M, int32_t B, int32_t L,
                                     const int32_t* win_lo, const int32_t* win_hi,
                                     int32_t* row_idx, int32_t* seq_off, int32_t* count,
                                     void* ws, size_t ws_bytes, void* stream);

/*
 * dllm_mask_compact_noalloc - dllm_mask_compact without a workspace argument.
 *
 * The pages have no counterpart for this call; it exists for callers that cannot allocate
 * device memory.  Some callers cannot hand the library a workspace: an inference engine
 * whose memory planner owns every byte of HBM and forbids side allocations, or a plugin
 * that must not call cudaMalloc (it can synchronise the whole device and stall other
 * streams).  This variant allocates nothing.  Its scratch (the per-tile mask counts of the
 * compaction) lives in a fixed array of DLLM_NOALLOC_MAX_TILES ints (64 KiB) in the
 * library's static device memory, which every GPU that loads the library holds until the
 * process exits.
 *
 * Arguments, outputs and results are exactly those of dllm_mask_compact.
 * Limits and caveats:
 *   - B*L must not exceed DLLM_NOALLOC_MAX_POSITIONS (134,217,728 positions); larger inputs
 *     are rejected with DLLM_ERR_SCRATCH before anything is launched.
 *   - The first call on a device looks up the scratch array's device address (once per
 *     device, with that device current); make that first call before any stream capture.
 *   - All calls on a device share the one scratch array.  Calls whose kernels overlap on the
 *     GPU (different streams, no ordering between them) race on it and may return wrong
 *     results; order such calls on one stream or with events.  The array keeps the last
 *     call's contents; nothing needs clearing, because every slot a call reads is written
 *     earlier in that same call.
 */
#define DLLM_NOALLOC_MAX_TILES      16384
#define DLLM_NOALLOC_MAX_POSITIONS  (16384LL * 8192LL)
dllm_status dllm_mask_compact_noalloc(const uint8_t* M, int32_t B, int32_t L,
                                      int32_t* row_idx, int32_t* seq_off, int32_t* count,
                                      void* stream);

/*
 * dllm_masked_logits - mask-only LM head with a fused online softmax epilogue (Mosaic page,
 * TL;DR and Abstract: the mask-only logits kernel).
 *
 * Runs dllm_mask_compact on M, gathers the masked rows of H, and computes for every masked
 * row i (in compacted order, i < count):
 *     z_v    = sum_k H[row_idx[i], k] * W[v, k]          (bf16 inputs, fp32 accumulation)
 *     tok[i] = the smallest v with z_v = max_v z_v
 *     lse[i] = log sum_v exp(z_v)                        (natural log)
 *     conf[i]= exp(max_v z_v - lse[i])                   (largest softmax probability)
 * No logit is ever written to memory: the GEMM epilogue keeps a running max, sum of
 * exponentials and argmax per row over vocabulary tiles, and inside the same kernel the
 * last work unit to finish a block of rows merges that block's per-split partials
 * (lse_merge, in vocabulary order, so the lowest token wins a tie of maxima).
 *
 *   H        device, bf16 [B*L, d] row-major.
 *   M        device, uint8 [B, L] row-major.
 *   W        device, bf16 [V, d] row-major (the vocabulary projection; no bias).
 *   tok, conf, lse   device, int32 / float32 / float32, each of capacity B*L; entries
 *            0..count-1 are written, the rest untouched.
 *   row_idx, seq_off, count   device outputs exactly as in dllm_mask_compact.
 *   ws       device workspace of at least dllm_workspace_bytes(B, L, d, V) bytes.
 * Constraints: B, L, V >= 1; d a positive multiple of 64; B*L < 2^31; every pointer
 * 16-byte aligned.  Errors: as dllm_mask_compact.
 */
dllm_status dllm_masked_logits(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                               int32_t B, int32_t L, int32_t d, int32_t V,
                               int32_t* tok, float* conf, float* lse,
                               int32_t* row_idx, int32_t* seq_off, int32_t* count,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * dllm_masked_logits_ex - dllm_masked_logits plus alternative certainty scores of each
 * masked row's softmax p (confidence/entropy-driven unmasking, dLLM inference survey page,
 * "Main Findings"):
 *   DLLM_STAT_ENTROPY  entropy[i] = -sum_v p_v ln p_v           (float32, capacity B*L)
 *   DLLM_STAT_MARGIN   margin[i]  = p_(1) - p_(2), largest minus second-largest probability
 * `stats` is a bitwise OR of those flags (0 = dllm_masked_logits); each requested output
 * pointer must be non-NULL and each other one NULL (else DLLM_ERR_NULL); unknown bits give
 * DLLM_ERR_SHAPE.  The epilogue keeps sum exp(z - max)(z - max) and the second-largest
 * logit per row next to the max and the sum of exponentials; no logit is stored.
 * Other arguments, outputs and errors as in dllm_masked_logits.
 */
#define DLLM_STAT_ENTROPY 1u
#define DLLM_STAT_MARGIN  2u
dllm_status dllm_masked_logits_ex(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                                  int32_t B, int32_t L, int32_t d, int32_t V, uint32_t stats,
                                  int32_t* tok, float* conf, float* lse, float* entropy,
                                  float* margin, int32_t* row_idx, int32_t* seq_off,
                                  int32_t* count, void* ws, size_t ws_bytes, void* stream);

/*
 * dllm_masked_logits_window - current-block-only logits: dllm_masked_logits_ex on the
 * masked positions inside each sequence's window [win_lo[b], win_hi[b]) only (the rows of
 * dllm_mask_compact_window).  Masked positions outside the window get no logits and no
 * output row; they are decoded when their own block becomes current (Sparse-dLLM page,
 * "Experiment": block-wise semi-autoregressive decoding).
 *
 *   win_lo, win_hi  device int32 [B], both required (DLLM_ERR_NULL otherwise).
 * Other arguments, outputs and errors as in dllm_masked_logits_ex.
 */
dllm_status dllm_masked_logits_window(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                                      int32_t B, int32_t L, int32_t d, int32_t V,
                                      const int32_t* win_lo, const int32_t* win_hi,
                                      uint32_t stats, int32_t* tok, float* conf, float* lse,
                                      float* entropy, float* margin, int32_t* row_idx,
                                      int32_t* seq_off, int32_t* count, void* ws,
                                      size_t ws_bytes, void* stream);

/*
 * dllm_prepare_rows / dllm_masked_logits_prepared - dllm_masked_logits in two calls, so
 * that the input staging of one step (compaction of the mask and the gather of the masked
 * rows of H into the workspace, reading H and M from device or page-locked host memory)
 * can run on another stream while the previous step's GEMM runs.
 *
 * dllm_prepare_rows runs a1 (with optional windows, as in dllm_mask_compact_window) and
 * the gather into `ws`; dllm_masked_logits_prepared then runs a2-a4 on the rows prepared in
 * the same `ws` (it reads only `count` of the compaction outputs; row_idx and seq_off stay
 * for dllm_select_unmask).  Both calls take the same B, L, d, V and a workspace of
 * dllm_workspace_bytes(B, L, d, V); the caller orders the second after the first (same
 * stream, or an event) and does not reuse `ws` for another preparation until the second
 * has run.  Arguments, outputs and errors otherwise as in dllm_masked_logits_window /
 * dllm_masked_logits_ex.
 */
dllm_status dllm_prepare_rows(const uint16_t* H, const uint8_t* M, int32_t B, int32_t L,
                              int32_t d, int32_t V, const int32_t* win_lo,
                              const int32_t* win_hi, int32_t* row_idx, int32_t* seq_off,
                              int32_t* count, void* ws, size_t ws_bytes, void* stream);
dllm_status dllm_masked_logits_prepared(const uint16_t* W, int32_t B, int32_t L, int32_t d,
                                        int32_t V, uint32_t stats, int32_t* tok, float* conf,
                                        float* lse, float* entropy, float* margin,
                                        const int32_t* count, void* ws, size_t ws_bytes,
                                        void* stream);

/*
 * dllm_masked_partials - one vocabulary shard of a vocabulary-parallel LM head.
 *
 * With W split by rows over GPUs (GPU g holds W[v_offset_g : v_offset_g + V_shard_g, :]),
 * each GPU runs this call on its shard and the same H and M.  It computes exactly what
 * dllm_masked_logits computes, over this shard's vocabulary only, and writes each masked
 * row's softmax partial instead of the finished values (no logit is stored):
 *     part_m[i] = max_v z_v,   part_s[i] = sum_v exp(z_v - part_m[i]),
 *     part_a[i] = v_offset + the smallest v attaining the max        (v over the shard)
 * and, in extended mode (stats != 0), part_t[i] = sum_v exp(z_v - m)(z_v - m) and
 * part_m2[i] = the second-largest logit.  After the partials of every shard are gathered
 * (one all-gather of 12 bytes per row per shard, 20 in extended mode), dllm_lse_merge
 * turns them into tok / conf / lse (/ entropy / margin) over the whole vocabulary.  The
 * partial algebra is the split-vocabulary merge of the Mosaic page's mask-only logits
 * kernel, applied across GPUs instead of across tiles.
 *
 *   W_shard  device, bf16 [V_shard, d] row-major: rows v_offset .. v_offset+V_shard-1 of W.
 *   v_offset first global token index of the shard (>= 0; v_offset + V_shard < 2^31).
 *   win_lo, win_hi  device int32 [B] or both NULL: as in dllm_masked_logits_window.
 *   stats    0, or DLLM_STAT_ENTROPY and/or DLLM_STAT_MARGIN: then part_t and part_m2 are
 *            both required (the extended partial carries both); else both NULL.
 *   part_m, part_s, part_a  device [B*L] capacity, compacted order (entries < count).
 * row_idx, seq_off, count, workspace and errors as in dllm_masked_logits.
 */
dllm_status dllm_masked_partials(const uint16_t* H, const uint8_t* M, const uint16_t* W_shard,
                                 int32_t B, int32_t L, int32_t d, int32_t V_shard,
                                 int32_t v_offset, const int32_t* win_lo, const int32_t* win_hi,
                                 uint32_t stats, float* part_m, float* part_s, int32_t* part_a,
                                 float* part_t, float* part_m2, int32_t* row_idx,
                                 int32_t* seq_off, int32_t* count, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * dllm_lse_merge - merge per-shard softmax partials into the finished per-row values:
 *     m* = max_j m_j,  s* = sum_j s_j exp(m_j - m*),  tok = a_j of the first j with m_j = m*,
 *     lse = m* + ln s*,  conf = exp(m* - lse) = 1 / s*
 * (extended: t* = sum_j exp(m_j - m*)(t_j + (m_j - m*) s_j), entropy = ln s* - t* / s*;
 * m2* = second largest of all m_j and m2_j, margin = (1 - exp(m2* - m*)) / s*).
 *
 *   part_*   device; split j of row i at index j * split_stride + i, splits in ascending
 *            vocabulary order (a tie of maxima keeps the lower split, i.e. the lower token).
 *   count    device int32 [1]: rows 0 .. min(*count, n_cap)-1 are merged (the count written
 *            by dllm_masked_partials stays on the device).
 *   stats    as in dllm_masked_partials; entropy / margin non-NULL exactly when requested.
 *   tok, conf, lse  device [n_cap] capacity, compacted order.
 * Constraints: n_split >= 1, n_cap >= 1, split_stride >= n_cap.  Errors: DLLM_ERR_NULL,
 * DLLM_ERR_ALIGN, DLLM_ERR_SHAPE, DLLM_ERR_CUDA, DLLM_ERR_DEVICE.
 */
dllm_status dllm_lse_merge(const float* part_m, const float* part_s, const int32_t* part_a,
                           const float* part_t, const float* part_m2, int64_t split_stride,
                           int32_t n_split, const int32_t* count, int32_t n_cap, uint32_t stats,
                           int32_t* tok, float* conf, float* lse, float* entropy,
                           float* margin, void* stream);

/*
 * dllm_select_unmask - per-sequence top-k over confidences (confidence-driven unmasking,
 * dLLM inference survey page, "Main Findings").
 *
 * For each sequence b, the candidates are its masked positions l = row_idx[i] - b*L for
 * i in [seq_off[b], seq_off[b+1]), restricted to win_lo[b] <= l < win_hi[b] when windows
 * are given.  The k candidates of largest conf are selected, ordered by conf descending,
 * then by position ascending (this order also breaks exact ties).
 *
 *   conf, row_idx, seq_off   device, as produced by dllm_masked_logits (compacted order).
 *   win_lo, win_hi   device int32 [B] or both NULL (no window).
 *   tok      device int32 (compacted order) or NULL.
 *   idx      device int32 [B, k]: selected positions l in [0, L); -1 past n_sel[b].
 *   n_sel    device int32 [B]: min(k, number of candidates of sequence b).
 *   tok_sel  device int32 [B, k] or NULL: tok of each selected position (-1 padding);
 *            requires tok.
 *   conf_sel device float32 [B, k] or NULL: conf of each selected position (0 padding).
 * Constraints: 1 <= k <= DLLM_MAX_K.  Errors: DLLM_ERR_NULL, DLLM_ERR_ALIGN,
 * DLLM_ERR_SHAPE, DLLM_ERR_CUDA, DLLM_ERR_DEVICE.
 */
dllm_status dllm_select_unmask(const float* conf, const int32_t* row_idx,
                               const int32_t* seq_off, int32_t B, int32_t L, int32_t k,
                               const int32_t* win_lo, const int32_t* win_hi,
                               const int32_t* tok,
                               int32_t* idx, int32_t* n_sel,
                               int32_t* tok_sel, float* conf_sel, void* stream);

/*
 * dllm_select_unmask_ex - threshold-based parallel unmasking over any per-row score (the
 * decoding thresholds of the dLLM pages, Dynamic-dLLM abstract).  Per sequence, among the
 * candidates of dllm_select_unmask, the number taken is
 *     min(k, max(min(min_sel, n_candidates), #candidates with score >= threshold)),
 * the best ones by (score descending, position ascending).  With ascending = 1 smaller
 * scores are better (e.g. the entropy): candidates qualify with score <= threshold and the
 * order is (score ascending, position ascending).  min_sel >= 1 guarantees that decoding
 * advances; threshold = -INFINITY (descending) or +INFINITY (ascending) gives plain top-k.
 * Scores must not be NaN.  score_sel (nullable) receives the scores of the selected
 * positions (0 padding).  Errors: as dllm_select_unmask, and DLLM_ERR_SHAPE for
 * min_sel < 0, a NaN threshold or ascending not 0/1.
 */
dllm_status dllm_select_unmask_ex(const float* score, const int32_t* row_idx,
                                  const int32_t* seq_off, int32_t B, int32_t L, int32_t k,
                                  float threshold, int32_t min_sel, int32_t ascending,
                                  const int32_t* win_lo, const int32_t* win_hi,
                                  const int32_t* tok, int32_t* idx, int32_t* n_sel,
                                  int32_t* tok_sel, float* score_sel, void* stream);

/*
 * dllm_decode_step - the whole hot path in one call: dllm_masked_logits followed by
 * dllm_select_unmask on the same stream.  Arguments as in those two calls.
 */
dllm_status dllm_decode_step(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                             int32_t B, int32_t L, int32_t d, int32_t V, int32_t k,
                             const int32_t* win_lo, const int32_t* win_hi,
                             int32_t* tok, float* conf, float* lse,
                             int32_t* row_idx, int32_t* seq_off, int32_t* count,
                             int32_t* idx, int32_t* n_sel, int32_t* tok_sel, float* conf_sel,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * dllm_decode_block_step - one semi-autoregressive decode step over the current blocks:
 * dllm_masked_logits_window followed by dllm_select_unmask, so logits are computed only
 * for the masked positions inside each sequence's window.  The selection (idx, n_sel,
 * tok_sel, conf_sel) equals that of dllm_decode_step with the same windows; tok, conf, lse,
 * row_idx, seq_off and count cover the in-window rows only.  win_lo and win_hi are
 * required.  Other arguments and errors as in dllm_decode_step.
 */
dllm_status dllm_decode_block_step(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                                   int32_t B, int32_t L, int32_t d, int32_t V, int32_t k,
                                   const int32_t* win_lo, const int32_t* win_hi,
                                   int32_t* tok, float* conf, float* lse,
                                   int32_t* row_idx, int32_t* seq_off, int32_t* count,
                                   int32_t* idx, int32_t* n_sel, int32_t* tok_sel,
                                   float* conf_sel, void* ws, size_t ws_bytes, void* stream);

/*
 * dllm_get_status - synchronise `stream`, then return (and clear) the device-side status
 * word of the current device: DLLM_OK, DLLM_ERR_TIMEOUT, DLLM_ERR_BOUNDS or
 * DLLM_ERR_CAPACITY (in that order of precedence when several were recorded);
 * DLLM_ERR_CUDA if the synchronisation itself failed.
 */
dllm_status dllm_get_status(void* stream);

/*
 * Test hook: run the tensor-core GEMM of dllm_masked_logits on already compacted inputs and
 * store the raw fp32 logits instead of reducing them.  For small-shape tests only: the
 * caller provides logits_out, float32 [B*L, V] capacity (rows 0..count-1 written).  The
 * other arguments are as in dllm_masked_logits; row_idx/seq_off/count are outputs.
 */
dllm_status dllm_debug_lmhead_logits(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                                     int32_t B, int32_t L, int32_t d, int32_t V,
                                     float* logits_out,
                                     int32_t* row_idx, int32_t* seq_off, int32_t* count,
                                     void* ws, size_t ws_bytes, void* stream);

/*
 * Test hook: the lse_merge step alone.  Partials are given per vocabulary split j and row i
 * at index j * n_rows + i: running max m, sum of exp(z - m) s, and argmax a.  Writes tok,
 * conf and lse for i < n_rows, merging splits 0..n_split-1 in order (lowest split wins a
 * tie of maxima).
 */
dllm_status dllm_debug_lse_merge(const float* part_m, const float* part_s,
                                 const int32_t* part_a, int32_t n_rows, int32_t n_split,
                                 int32_t* tok, float* conf, float* lse, void* stream);

/*
 * Test hook: choose the tensor-core GEMM variant used by later calls in this process:
 * 2 = CTA pairs (tcgen05 cta_group::2, 256x256 tiles over two SMs), 1 = single CTAs
 * (cta_group::1, 128x256 tiles), 0 = the default: one launch that picks on the device,
 * from the masked count, single CTAs for at most 128 rows and pairs above.  Results
 * agree to fp32 rounding; the variants differ in speed.  Returns DLLM_ERR_SHAPE for other
 * values.
 */
dllm_status dllm_debug_set_gemm_variant(int32_t cta_group);

/*
 * Kernel-time accounting for benchmarks.  dllm_prof_begin() starts recording a CUDA event
 * pair around every tensor-core GEMM launch and counting every kernel launch made by this
 * library (all devices, all streams).  dllm_prof_end() synchronises those events, returns
 * the summed GEMM time in milliseconds, the number of GEMM launches and the number of
 * kernel launches since dllm_prof_begin(), and stops recording.  Not thread-safe.
 */
dllm_status dllm_prof_begin(void);
dllm_status dllm_prof_end(double* gemm_ms, int32_t* gemm_launches, int32_t* kernel_launches);

#ifdef __cplusplus
}
#endif

#endif /* DLLM_H */
