/*
 * tbq4.h -- C ABI of libtbq4: attention over a long-context KV cache stored
 * in the TBQ4 block format, on NVIDIA B200 (sm_100a).
 *
 * The format.  TBQ4 stores 128 values in 66 bytes: a 2-byte scale followed
 * by 64 bytes of 4-bit indices, 4.125 bits per value, in a Hadamard-rotated
 * domain; attention reads the raw blocks and dequantises them in its inner
 * loop, with no separate dequantisation pass and no fp16 copy of the cache
 * (trefon.com, "Kontekst 262K na jednej RTX 4090: co dodalem do
 * llama.cpp-turboq", section "Od czego zaczalem").  K and V have separate
 * caches, as the page's "-ctk tbq4_0 -ctv tbq4_0" flags do (section
 * "Konfiguracja").
 *
 * The codebook (the page does not give one; this library fixes it):
 *   x_rot = R x with R = H * D / sqrt(128), H the 128x128 Sylvester Hadamard
 *     matrix (H[i][j] = (-1)^popcount(i&j)), D = diag(s), s_i = +-1 from
 *     SplitMix64(sign_seed): s_i = 1 - 2*bit(i%64) of output number i/64.
 *     Computed as: sign flip, 7 butterfly stages of stride 1,2,...,64 (lower
 *     = a+b, upper = a-b, each rounded to binary32), one binary32 multiply
 *     by fl32(1/sqrt(128)) = 0x3DB504F3.
 *   scale S = fp16(max_i |x_rot_i|), round to nearest even, saturating at
 *     65504; stored little endian in bytes 0-1.
 *   index i = clamp(rne(fl32(fl32(x_rot/S) * 7.5) + 7.5), 0, 15) (index 8
 *     when S == 0); byte 2+j = index[2j] | index[2j+1] << 4.
 *   dequantised value = S * (2*index - 15) / 15 (rotated domain).
 *
 * Cache layout: [B][Hkv][capacity][66] bytes per cache (K or V); the
 * blocks of one (sequence, KV head) are contiguous.  capacity must be a
 * multiple of 8 so that every 8-token group (528 bytes) starts on a 16-byte
 * boundary, and cache base pointers must be 16-byte aligned.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device (or managed) memory on the
 *     current device; the caller owns all memory.  The library allocates
 *     nothing and frees nothing; scratch memory is a caller-provided
 *     workspace whose size the *_workspace_bytes queries return.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *     compute call is asynchronous on that stream and does not synchronise.
 *   - Arguments are checked on the host before anything is launched; on a
 *     non-OK status nothing was launched.  Values that live in device memory
 *     (positions, lengths) are checked by the kernels, which skip the
 *     offending work and record an error code that tbq4_get_device_status
 *     returns.
 *   - Inputs q, K and V are in the original (unrotated) domain; outputs are
 *     unrotated.  The rotation is internal and keyed by `sign_seed`, which
 *     must be the same for the append calls and the attention calls of one
 *     cache.
 */
#ifndef TBQ4_H_
#define TBQ4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TBQ4_API __attribute__((visibility("default")))
#else
#define TBQ4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TBQ4_OK = 0,
    TBQ4_ERR_NULL = 1,            /* a required pointer is NULL            */
    TBQ4_ERR_ALIGN = 2,           /* a pointer is not 16-byte aligned      */
    TBQ4_ERR_SHAPE = 3,           /* bad sizes: Hq % Hkv, G > 8, n <= 0 .. */
    TBQ4_ERR_CAPACITY = 4,        /* capacity not a multiple of 8, or a
                                     position/length outside [0, capacity] */
    TBQ4_ERR_WORKSPACE = 5,       /* workspace smaller than required       */
    TBQ4_ERR_LAUNCH = 6,          /* a CUDA launch or query failed         */
    TBQ4_ERR_DEVICE_TIMEOUT = 7,  /* a bounded wait inside a kernel gave up */
    TBQ4_ERR_BOUNDS = 8           /* debug build only (libtbq4_debug.so, built
                                     with -DTBQ4_DEBUG): a global access a
                                     kernel derived from lengths, positions,
                                     page ids or its split plan fell outside
                                     its buffer; the access was skipped (a
                                     tracked copy was redirected to offset 0) */
} tbq4_status;

/* Bytes of one block (66: the 2-byte scale and 64 bytes of 4-bit indices,
 * trefon.com, "Kontekst 262K na jednej RTX 4090", section "Od czego
 * zaczalem") and of one cache (B*Hkv*capacity*66; K and V are separate
 * caches, section "Konfiguracja", -ctk/-ctv).  0 for non-positive sizes. */
TBQ4_API size_t tbq4_block_bytes(void);
TBQ4_API size_t tbq4_cache_bytes(int batch, int n_kv_heads, int64_t capacity);

/* Host: the +-1 diagonal for `seed`, written to out[128] (host memory).
 * It is the sign step of the Hadamard rotation that defines the stored
 * domain (page section "Od czego zaczalem": the cache and attention live in
 * the Hadamard-rotated domain; the signs themselves are this library's
 * codebook, above).  No error path. */
TBQ4_API void tbq4_signs(uint64_t seed, int8_t out[128]);

/*
 * Quantise-append: rotate, scale, index and pack new K or V rows into a
 * cache (the TBQ4 encoding above; page section "Od czego zaczalem").
 *   src        device, fp32 [B][n_new][Hkv][128], 16-byte aligned
 *   start_pos  device, int32 [B]: row t of sequence b goes to position
 *              start_pos[b] + t
 *   cache      device, uint8 [B][Hkv][capacity][66], 16-byte aligned
 * Bytes written are bit-exact with the codebook above.  Rows whose position
 * falls outside [0, capacity) are skipped and flag TBQ4_ERR_CAPACITY in the
 * device status.
 */
TBQ4_API tbq4_status tbq4_quantize_append(const float *src, int B, int n_new, int Hkv,
                                 const int32_t *start_pos, int64_t capacity,
                                 uint64_t sign_seed, uint8_t *cache,
                                 void *stream);

/*
 * Decode attention (one query token per sequence) over TBQ4 caches, split
 * over the context and merged by log-sum-exp; grouped-query heads share
 * one KV stream (q head h reads KV head h / (Hq/Hkv)).  This is the page's
 * flash-attention kernel that reads the raw TBQ4 blocks from global memory
 * and dequantises them in its inner loop, in the rotated domain, with no F16
 * buffer (trefon.com, "Kontekst 262K na jednej RTX 4090", section "Od czego
 * zaczalem"; enabled there by --flash-attn on with -ctk/-ctv tbq4_0, section
 * "Konfiguracja").  q is rotated once, the output rotated back once per row.
 * tbq4_decode_workspace_bytes returns the scratch this call needs for its
 * split partials (0 for invalid sizes).
 *   q          device, fp32 [B][Hq][128], 16-byte aligned
 *   k_cache,
 *   v_cache    device, uint8 [B][Hkv][capacity][66], 16-byte aligned
 *   seq_lens   device, int32 [B]: keys attended per sequence (positions
 *              0 .. seq_lens[b]-1; the current token is already appended).
 *              A length of 0 gives a zero output row.
 *   max_len    host upper bound of seq_lens, sizes the launch; lengths above
 *              it (or above capacity) are clamped and flag
 *              TBQ4_ERR_CAPACITY in the device status.
 *   softmax_scale  multiplies q.k before the softmax (1/sqrt(128) typical).
 *   workspace  device scratch of at least tbq4_decode_workspace_bytes(...)
 *              bytes, 256-byte aligned; its contents need no initialisation.
 *   out        device, fp16 [B][Hq][128] (round to nearest even).
 * Constraints: Hq % Hkv == 0, Hq/Hkv <= 8, B >= 1.
 * Errors: TBQ4_ERR_NULL, TBQ4_ERR_ALIGN (q, caches 16 bytes, workspace 256
 * bytes), TBQ4_ERR_SHAPE (head counts, B), TBQ4_ERR_CAPACITY (capacity not a
 * multiple of 8, or max_len > capacity), TBQ4_ERR_WORKSPACE (ws_bytes too
 * small), TBQ4_ERR_LAUNCH.
 */
TBQ4_API size_t tbq4_decode_workspace_bytes(int B, int Hq, int Hkv, int32_t max_len);
TBQ4_API tbq4_status tbq4_attn_decode(const float *q, const uint8_t *k_cache,
                             const uint8_t *v_cache, const int32_t *seq_lens,
                             int32_t max_len, int B, int Hq, int Hkv,
                             int64_t capacity, float softmax_scale,
                             uint64_t sign_seed, void *workspace,
                             size_t ws_bytes, uint16_t *out, void *stream);

/*
 * One decode step: append the current token's K and V rows to the caches and
 * attend, in one attention launch.  The result equals tbq4_quantize_append of
 * k_new / v_new at position seq_lens[b]-1 followed by tbq4_attn_decode (same
 * bytes in the caches, same output); the rows are encoded inside the
 * attention kernel by the CTA that streams that position, which saves the two
 * append launches of a decode step.  This fuses the page's two per-token
 * operations, writing the new token into the TBQ4 cache and reading the cache
 * in the flash-attention kernel (trefon.com, "Kontekst 262K na jednej RTX
 * 4090", sections "Konfiguracja" and "Od czego zaczalem").
 *   k_new, v_new  device, fp32 [B][Hkv][128], 16-byte aligned
 *   seq_lens      device, int32 [B], counting the appended token; a length
 *                 of 0 appends nothing and gives a zero output row.
 * Other arguments as tbq4_attn_decode; the caches are written.
 */
TBQ4_API tbq4_status tbq4_attn_decode_append(const float *q, const float *k_new,
                                             const float *v_new, uint8_t *k_cache,
                                             uint8_t *v_cache, const int32_t *seq_lens,
                                             int32_t max_len, int B, int Hq, int Hkv,
                                             int64_t capacity, float softmax_scale,
                                             uint64_t sign_seed, void *workspace,
                                             size_t ws_bytes, uint16_t *out, void *stream);

/*
 * Paged caches (block table).  Instead of one [B][Hkv][capacity][66] cache, K
 * and V each live in a pool of pages shared by all sequences:
 *   pool         device, uint8 [n_pages][Hkv][page_size][66], 16-byte aligned
 *   block_table  device, int32 [B][max_pages]: token t of sequence b is row
 *                t % page_size of page block_table[b][t / page_size]
 *   page_size    tokens per page, a multiple of 32 (>= 32)
 * A sequence can hold max_pages * page_size tokens.  The layout inside a
 * page is the contiguous layout (tokens of one KV head back to back), so
 * every 32-token chunk of a stream is one contiguous copy.  This is the
 * paged variant of the page's fixed per-sequence KV cache for ragged batches
 * (trefon.com, "Kontekst 262K na jednej RTX 4090", sections "Konfiguracja"
 * and "Od czego zaczalem": the quantised K/V blocks read by the attention
 * kernel).  The caller owns the pools and the table; pages need no
 * initialisation before they are written.
 *
 * tbq4_quantize_append_paged: as tbq4_quantize_append, with positions
 * mapped through the table.  A position at or past max_pages * page_size,
 * or a page id outside [0, n_pages), skips that row and flags
 * TBQ4_ERR_CAPACITY in the device status.
 *
 * tbq4_attn_decode_paged: as tbq4_attn_decode (k_new = v_new = NULL) or
 * tbq4_attn_decode_append (both non-NULL, fp32 [B][Hkv][128], 16-byte
 * aligned; the new rows are written into the pools at seq_lens[b] - 1),
 * same arithmetic and the same result bit for bit.  Requires max_len <=
 * max_pages * page_size; the table entries of pages holding real tokens
 * (t < seq_lens[b]) must be in [0, n_pages).  Entries past a sequence's
 * length are read only as hints and may hold anything; a bad entry within
 * the length makes that chunk read page 0 and flags TBQ4_ERR_CAPACITY.
 * The workspace size comes from tbq4_decode_workspace_bytes.
 * Errors: TBQ4_ERR_NULL (a NULL pointer, or only one of k_new / v_new),
 * TBQ4_ERR_ALIGN, TBQ4_ERR_SHAPE (page_size, max_pages, n_pages or the
 * head counts), TBQ4_ERR_CAPACITY (max_len above the table's reach).
 */
TBQ4_API tbq4_status tbq4_quantize_append_paged(const float *src, int B, int n_new, int Hkv,
                                                const int32_t *start_pos,
                                                const int32_t *block_table, int max_pages,
                                                int page_size, int64_t n_pages,
                                                uint64_t sign_seed, uint8_t *pool, void *stream);
TBQ4_API tbq4_status tbq4_attn_decode_paged(const float *q, const float *k_new,
                                            const float *v_new, uint8_t *k_pool,
                                            uint8_t *v_pool, const int32_t *block_table,
                                            int max_pages, int page_size, int64_t n_pages,
                                            const int32_t *seq_lens, int32_t max_len, int B,
                                            int Hq, int Hkv, float softmax_scale,
                                            uint64_t sign_seed, void *workspace,
                                            size_t ws_bytes, uint16_t *out, void *stream);

/*
 * TBQ3: the 3-bit variant.  The page names a 3-bit KV cache type next to
 * TBQ4 and a fix to its 3-bit packing (trefon.com, "Kontekst 262K na jednej
 * RTX 4090: co dodalem do llama.cpp-turboq", section "6. Ten sam cache na
 * Apple silicon") without its layout; this library fixes it:
 *   block  128 values in 50 bytes (3.125 bits per value): the fp16 scale
 *          S = fp16(max |x_rot|) (little endian, saturating), then 16 groups
 *          of three bytes, each a little-endian 24-bit word holding indices
 *          8g .. 8g+7 (index 8g+k at bits 3k .. 3k+2)
 *   levels (i - 3.5)/3.5 * S = S (2i - 7)/7, i = 0..7;
 *          i = clamp(rne(fl32(fl32(x_rot/S) * 3.5) + 3.5), 0, 7), 4 if S == 0
 *   rotation, sign seed and cache layout as TBQ4, with 50-byte blocks:
 *          [B][Hkv][capacity][50], capacity % 8 == 0.
 * tbq3_quantize_append and tbq3_attn_decode take the arguments of
 * tbq4_quantize_append and tbq4_attn_decode, with the same errors; the decode
 * workspace is tbq4_decode_workspace_bytes(B, Hq, Hkv, max_len).
 */
TBQ4_API size_t tbq3_block_bytes(void);   /* 50 */
TBQ4_API size_t tbq3_cache_bytes(int batch, int n_kv_heads, int64_t capacity);
TBQ4_API tbq4_status tbq3_quantize_append(const float *src, int B, int n_new, int Hkv,
                                          const int32_t *start_pos, int64_t capacity,
                                          uint64_t sign_seed, uint8_t *cache, void *stream);
TBQ4_API tbq4_status tbq3_attn_decode(const float *q, const uint8_t *k_cache,
                                      const uint8_t *v_cache, const int32_t *seq_lens,
                                      int32_t max_len, int B, int Hq, int Hkv,
                                      int64_t capacity, float softmax_scale,
                                      uint64_t sign_seed, void *workspace, size_t ws_bytes,
                                      uint16_t *out, void *stream);

/*
 * Multi-query decode: q_len (1-4) new query tokens per sequence, as when a
 * model verifies speculative drafts (trefon.com, "Kontekst 262K na jednej RTX
 * 4090", section "Konfiguracja": up to 3 drafted tokens).  Query token i of
 * sequence b sits at position seq_lens[b] - q_len + i and attends to keys
 * [0, seq_lens[b] - q_len + i] (bottom-right causal, as the chunked prefill),
 * with the same arithmetic as tbq4_attn_decode.  All q_len tokens are already
 * in the caches.
 *   q         device, fp32 [B][q_len][Hq][128]
 *   out       device, fp16 [B][q_len][Hq][128]
 *   seq_lens  device, int32 [B], each >= q_len (a shorter sequence gives zero
 *             rows for the queries that see no key)
 * Requires (Hq / Hkv) * q_len <= 32.  The workspace size comes from
 * tbq4_decode_mq_workspace_bytes.  q_len = 1 runs the single-query kernel.
 * Errors as tbq4_attn_decode.
 */
TBQ4_API size_t tbq4_decode_mq_workspace_bytes(int B, int q_len, int Hq, int Hkv,
                                               int32_t max_len);
TBQ4_API tbq4_status tbq4_attn_decode_mq(const float *q, const uint8_t *k_cache,
                                         const uint8_t *v_cache, const int32_t *seq_lens,
                                         int32_t max_len, int B, int q_len, int Hq, int Hkv,
                                         int64_t capacity, float softmax_scale,
                                         uint64_t sign_seed, void *workspace, size_t ws_bytes,
                                         uint16_t *out, void *stream);

/* As tbq4_attn_decode (the page's decode kernel over raw blocks, section
 * "Od czego zaczalem"), with the context split into pieces of
 * `split_tokens` keys (a multiple of 32; 0 = automatic).  The result does
 * not depend on the split beyond fp32 rounding.  Workspace requirement:
 * tbq4_decode_workspace_bytes_split() (0 for invalid sizes).  Errors as
 * tbq4_attn_decode, plus TBQ4_ERR_SHAPE for a split that is not a multiple
 * of 32. */
TBQ4_API size_t tbq4_decode_workspace_bytes_split(int B, int Hq, int Hkv,
                                         int32_t max_len, int32_t split_tokens);
TBQ4_API tbq4_status tbq4_attn_decode_split(const float *q, const uint8_t *k_cache,
                                   const uint8_t *v_cache,
                                   const int32_t *seq_lens, int32_t max_len,
                                   int B, int Hq, int Hkv, int64_t capacity,
                                   float softmax_scale, uint64_t sign_seed,
                                   int32_t split_tokens, void *workspace,
                                   size_t ws_bytes, uint16_t *out,
                                   void *stream);

/*
 * Decode attention for callers that cannot allocate device memory.  It
 * computes exactly what tbq4_attn_decode computes, with the same arguments
 * minus the workspace.  The scratch for the split partials is a fixed array
 * of 8 MiB (8,388,608 bytes) compiled into this library as a static device
 * variable, so every GPU that loads the library holds those 8 MiB until the
 * process exits.
 *
 * Who needs it: code that is handed its inputs and outputs but has no way
 * to obtain device memory where it calls attention, such as a plugin that
 * runs inside another framework that owns all device memory, or a serving
 * loop whose memory is fixed before it starts.  The source pages describe
 * no counterpart of this entry point.
 *
 *   - If the scratch the call needs, tbq4_decode_workspace_bytes(B, Hq,
 *     Hkv, max_len), exceeds 8 MiB, it returns TBQ4_ERR_WORKSPACE and
 *     launches nothing.
 *   - The first call on a device looks up the device address of the array
 *     (cudaGetSymbolAddress, with that device current) and keeps it for the
 *     rest of the process; make that first call before any stream capture.
 *     A cudaDeviceReset of that device invalidates the kept address, and
 *     this library cannot see the reset: do not call this entry point on a
 *     device again after resetting it in the same process.
 *   - All calls share the one array, which keeps what the previous call
 *     wrote.  Nothing in it needs clearing (each partial is written before
 *     it is read), but calls whose kernels overlap on the GPU, for example
 *     on two streams at once, race on it: serialise them.
 *   - It allocates and frees nothing.
 */
TBQ4_API tbq4_status tbq4_attn_decode_noalloc(const float *q, const uint8_t *k_cache,
                                              const uint8_t *v_cache,
                                              const int32_t *seq_lens, int32_t max_len,
                                              int B, int Hq, int Hkv, int64_t capacity,
                                              float softmax_scale, uint64_t sign_seed,
                                              uint16_t *out, void *stream);

/*
 * Chunked prefill attention for one sequence: n_new query tokens at
 * absolute positions n_cached .. n_cached+n_new-1, each attending causally
 * to keys 0 .. its own position, over TBQ4 caches that already hold the
 * chunk's K/V (call tbq4_quantize_append on the chunk first).  It is the
 * same flash-attention over raw TBQ4 blocks in the rotated domain (trefon.com,
 * "Kontekst 262K na jednej RTX 4090", section "Od czego zaczalem"; the
 * page's server processes prompts in chunks of -ub tokens into the same
 * cache, section "Konfiguracja"), with QK^T and PV as dense tensor-core
 * contractions over tiles dequantised to bf16.
 * tbq4_prefill_workspace_bytes returns its scratch size (0 for invalid
 * sizes).
 *   q          device, bf16 bits [n_new][Hq][128], 16-byte aligned
 *   k_cache,
 *   v_cache    device, uint8 [Hkv][capacity][66] (one sequence), 16-byte
 *              aligned; n_cached + n_new <= capacity
 *   workspace  device scratch of tbq4_prefill_workspace_bytes(...) bytes
 *   out        device, bf16 bits [n_new][Hq][128] (round to nearest even)
 * Errors: TBQ4_ERR_NULL, TBQ4_ERR_ALIGN, TBQ4_ERR_SHAPE (Hq % Hkv, G > 8,
 * n_new outside [1, 65535]), TBQ4_ERR_CAPACITY (n_cached + n_new above
 * capacity), TBQ4_ERR_WORKSPACE, TBQ4_ERR_LAUNCH.
 */
TBQ4_API size_t tbq4_prefill_workspace_bytes(int n_new, int Hq, int Hkv,
                                    int64_t n_cached);
TBQ4_API tbq4_status tbq4_attn_prefill_chunk(const uint16_t *q, int n_new,
                                    int64_t n_cached, const uint8_t *k_cache,
                                    const uint8_t *v_cache, int Hq, int Hkv,
                                    int64_t capacity, float softmax_scale,
                                    uint64_t sign_seed, void *workspace,
                                    size_t ws_bytes, uint16_t *out,
                                    void *stream);

/* Profiling hook (the page has no counterpart; it serves the measurement
 * of the kernels above): while set, every attention call records `before` on its
 * stream just before its attention kernel and `after` just after it, so a
 * caller can time the attention alone with cudaEventElapsedTime.  Decode:
 * the events bracket the split kernel and its combine (a programmatic
 * dependent launch that starts while the split kernel drains, so the pair is
 * one region); prefill: the attention kernel alone, not its combine.  Both
 * are cudaEvent_t created by the caller; pass NULLs to stop recording.  Not
 * thread-safe: meant for benchmarks. */
TBQ4_API void tbq4_set_timing_events(void *before, void *after);

/* Synchronises `stream`, returns the first error code a kernel of this
 * library recorded on the current device since the last call (TBQ4_OK if
 * none) and clears it.  The device-side checks it reports (positions and
 * lengths against the capacity, bounded waits, and in the debug build the
 * bounds checks of TBQ4_ERR_BOUNDS) guard the kernels above; the page
 * describes no counterpart.  TBQ4_ERR_LAUNCH if the synchronisation
 * or the read fails. */
TBQ4_API tbq4_status tbq4_get_device_status(void *stream);

/* Self-test of the device-side failure path (no counterpart on the page;
 * it checks this library's own guard).  Launches one warp on `stream` that
 * waits on a shared-memory barrier nothing will ever complete, with no copy
 * in flight, using the same bounded wait as every kernel here; after `polls`
 * polls (1 .. 65536) it gives up, records TBQ4_ERR_DEVICE_TIMEOUT in the
 * device status and returns, leaving the context usable.  Returns
 * TBQ4_ERR_SHAPE for a poll count outside that range, TBQ4_ERR_LAUNCH if the
 * launch fails, else TBQ4_OK (the timeout itself is reported by
 * tbq4_get_device_status). */
TBQ4_API tbq4_status tbq4_selftest_bounded_wait(uint32_t polls, void *stream);

/* Static description of a status code (this library's error codes, above;
 * no counterpart on the page).  Never NULL. */
TBQ4_API const char *tbq4_status_string(tbq4_status s);

#ifdef __cplusplus
}
#endif

#endif /* TBQ4_H_ */
