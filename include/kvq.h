/*
 * kvq.h -- C ABI of the packed-KV attention library (libkvq.so, sm_100a).
 *
 * What it computes
 * ----------------
 * kvq_pack    Symmetric group quantization of K and V into a packed cache
 *             ("KV分组打包：4-bit到底省了多少？", huhohoo.com/docs/llm/kv-packed-groups,
 *             sections "一个字节里到底装了什么" and "为什么分组要同时看方向与长度"):
 *             4-bit codes in [-7, 7] stored +7 two per byte (even code in the low
 *             nibble), or 8-bit codes in [-127, 127] stored +127; one float32
 *             scale = max|x| / 7 (or / 127) per group, 1 for an all-zero group;
 *             K grouped along tokens within each channel, V along features within
 *             each token; short groups zero-padded.  Rounding is to nearest, ties
 *             to even; divisions are IEEE float32.
 * kvq_attend  softmax(scale * Q K^T) V over the decoded cache, computed block
 *             by block with the running max m, exponential sum z and weighted sum
 *             u ("Block KV decoding: less workspace, more time",
 *             huhohoo.com/en/docs/llm/kv-block-decode-cost, section "Do not
 *             average independently normalized blocks"), so no decoded K/V and no
 *             score matrix is ever written to memory.  Grouped-query attention:
 *             query head h reads KV head h / (H_q / H_kv) ("给长前缀列一张有单位的
 *             资源账本", section "GQA改变共享接口").  Keys at or beyond a sequence's
 *             length take part in neither the max nor the sum (same page, section
 *             "FlashAttention为什么不必保存整张热图").  Non-causal: every query row
 *             reads every valid key.
 *
 * Conventions
 * -----------
 * - The library allocates nothing.  Every buffer is caller-owned device memory
 *   unless a parameter says "host".  Calls are asynchronous on `stream` (a
 *   cudaStream_t passed as void*; NULL is the legacy default stream).
 * - Argument errors are found on the host before any launch and returned
 *   synchronously; nothing is launched then.  Errors found by a kernel (a
 *   length of 0 or beyond capacity, a bounded wait that ran out) are recorded
 *   in a device error word and returned by kvq_check().
 * - All tensors are dense, row-major, in the shapes stated.
 * - Thread safety: calls on different streams may overlap; the device error
 *   word is shared by every call on a device.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_ARG = 1,          /* bad bits/group/shape/dtype, H_q % H_kv != 0, NULL pointer */
  KVQ_ERR_LENGTH = 2,       /* a sequence length outside its valid range: 1..N_cap, or as the
                               window and causal calls state (device-detected: kvq_check) */
  KVQ_ERR_ALIGN = 3,        /* a cache array, Q, O or the workspace not 16-byte aligned (or an
                               input of kvq_pack not aligned to its element size) */
  KVQ_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than kvq_workspace_size() */
  KVQ_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch, attribute query) */
  KVQ_ERR_DEVICE = 6,       /* a kernel recorded an internal inconsistency */
  KVQ_ERR_TIMEOUT = 7,      /* a bounded wait inside a kernel ran out */
  KVQ_ERR_UNSUPPORTED = 8   /* valid arguments outside what this library implements */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_BF16 = 1 } kvq_dtype;

/*
 * A packed cache: four caller-owned device arrays plus the logical shape.
 *   bits   4 or 8;  group  g, even, >= 2.
 *   B sequences, H_kv KV heads, N_cap token capacity (shared by all
 *   sequences), D features per head.  Let Np = ceil(N_cap/g)*g and
 *   Dp = ceil(D/g)*g.  Per (b, h) matrix, stacked in (b, h) order:
 *   k_codes   Np*D*bits/8 bytes: the row-major Np x D biased code matrix,
 *             4-bit codes paired over its flattened order (a byte may
 *             straddle two tokens when D is odd).
 *   k_scales  (Np/g) x D float32: scale of channel d over tokens
 *             [j*g, (j+1)*g).
 *   v_codes   N_cap*Dp*bits/8 bytes: the row-major N_cap x Dp code matrix.
 *   v_scales  N_cap x (Dp/g) float32: scale of token t over features
 *             [j*g, (j+1)*g).
 * For one (b, h) with N_cap = N these are exactly the arrays the pages
 * store for an N x D matrix (codes, float32 scales; the int32 shape pair is
 * the struct's N_cap/D).
 */
typedef struct {
  int32_t bits, group;
  int32_t B, H_kv, N_cap, D;
  uint8_t* k_codes;
  float* k_scales;
  uint8_t* v_codes;
  float* v_scales;
} kvq_cache;

/* Byte sizes of the four cache arrays (host).  sizes[0..3] = k_codes,
 * k_scales, v_codes, v_scales.  Returns KVQ_ERR_ARG for an invalid shape. */
KVQ_API kvq_status kvq_cache_sizes(int32_t bits, int32_t group, int32_t B, int32_t H_kv,
                           int32_t N_cap, int32_t D, size_t sizes[4]);

/* Total bytes of the four arrays of `cache` (host; its pointers are not
 * read): the sum of kvq_cache_sizes for its shape, 0 for an invalid shape or
 * NULL. */
KVQ_API size_t kvq_cache_bytes(const kvq_cache* cache);

/*
 * Quantize and pack tokens [t0, t1) of every (b, h) into the cache.
 *   K, V     device, [B, H_kv, t1 - t0, D] in `in_dtype` (KVQ_F32 or
 *            KVQ_BF16; bf16 is widened exactly to float32 first).  Either
 *            may be NULL to leave that half of the cache untouched (not
 *            both): a decode step re-packs the K group that holds the new
 *            token and packs the new token's V row alone.
 *   t0       with K: a multiple of g (K groups span g tokens, so a K group
 *            is only ever packed whole); 0 <= t0 < t1 <= N_cap.
 * A K group that ends beyond t1 is packed as if the tokens from t1 to the
 * group's end were zero: re-packing from the group start once more tokens
 * exist gives exactly the bytes a whole-cache pack gives.  Writes the
 * k_codes/k_scales of groups [t0/g, ceil(t1/g)) and the v_codes/v_scales of
 * tokens [t0, t1); nothing else.
 * Errors: KVQ_ERR_ARG (shape/range/dtype/NULL), KVQ_ERR_ALIGN (input not
 * aligned to its element size), KVQ_ERR_CUDA (launch).
 */
KVQ_API kvq_status kvq_pack(const void* K, const void* V, kvq_dtype in_dtype, int32_t t0, int32_t t1,
                    const kvq_cache* cache, void* stream);

/*
 * Attention of Q over the packed cache.
 *   Q        device, [B, H_q, Lq, D] in q_dtype (KVQ_F32 or KVQ_BF16),
 *            16-byte aligned.
 *   lengths  device int32 [B]: valid keys of each sequence, 1..N_cap.
 *   H_q      multiple of cache->H_kv.   Lq >= 1 query rows per sequence.
 *   scale    multiplies Q K^T before the softmax (1/sqrt(D) for unscaled Q,
 *            1 when Q already carries it).
 *   O        device, [B, H_q, Lq, D] in q_dtype, 16-byte aligned.
 *   workspace, ws_bytes   device scratch for split partials, at least
 *            kvq_workspace_size(...) bytes, 16-byte aligned.  Its contents
 *            on entry do not matter; it must not be shared by calls that may
 *            run at the same time.
 *   splits   how many CTAs share the concatenated (b, h, token-block) list;
 *            0 = automatic (a multiple of the SM count).  Any value gives the
 *            same result up to float rounding order.
 * A length outside 1..N_cap is recorded for kvq_check (KVQ_ERR_LENGTH): a
 * length below 1 gives zero rows, one above N_cap is read as N_cap.
 * Errors: KVQ_ERR_ARG, KVQ_ERR_ALIGN, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA,
 * KVQ_ERR_UNSUPPORTED (D > 256).
 */
KVQ_API kvq_status kvq_attend(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                      const int32_t* lengths, int32_t H_q, int32_t Lq, float scale, void* O,
                      void* workspace, size_t ws_bytes, int32_t splits, void* stream);

/*
 * Causal multi-query attention over the packed cache (chunked prefill): the
 * Lq query rows of sequence b are its last Lq positions, L - Lq .. L - 1
 * (L = lengths[b], the tokens already packed), and query i reads keys
 * [0, L - Lq + i] only; keys after a query's position take no part in its
 * max or sum ("给长前缀列一张有单位的资源账本", section
 * "FlashAttention为什么不必保存整张热图").  The pages' own studies are
 * non-causal; this is the masked form of the same rule.  Arguments, layout,
 * workspace (kvq_workspace_size) and errors as kvq_attend; a sequence with
 * L < Lq is also reported (KVQ_ERR_LENGTH) and its rows without a visible
 * key are zeros.  With Lq = 1 it is kvq_attend.
 */
KVQ_API kvq_status kvq_attend_causal(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                     const int32_t* lengths, int32_t H_q, int32_t Lq, float scale,
                                     void* O, void* workspace, size_t ws_bytes, int32_t splits,
                                     void* stream);

/*
 * One decode step of the generation path: append each sequence's new token
 * to the packed cache, then attend over the cache with that step's query.
 * The pages measure decoding a cache that was packed whole, and name the
 * complete generation path, appends included, as what a practical claim has
 * to time ("Block KV decoding: less workspace, more time", section "Use the
 * failure to choose the next question"); this call is that path.
 *
 * Sequence b's new token sits at t = lengths[b] - 1 (lengths count it).  The
 * call re-packs K group t / g of every (b, h) from the caller's float rows of
 * that group -- K scales run along tokens, so a group's scale changes as its
 * tokens arrive -- and packs V row t, then attends with one query row per
 * sequence as kvq_attend does.  Where the tuned decode kernel runs the attend
 * (D = 128, four query heads per KV head, 4- or 8-bit, g = 32 or 8) it does
 * the append itself; other shapes take one append kernel before the attend.
 * Afterwards the cache holds, for tokens [0, lengths[b]), exactly the bytes
 * kvq_pack of those tokens writes.
 *   Q, cache, H_q, scale, O, workspace, ws_bytes, splits: as kvq_attend with
 *            Lq = 1 (Q and O [B, H_q, 1, D]; workspace kvq_workspace_size(cache,
 *            H_q, 1, splits) bytes).
 *   lengths  device int32 [B]: tokens of each sequence including the new one,
 *            1..N_cap.
 *   K_tail   device, [B, H_kv, g, D] in in_dtype: row r of (b, h) holds K of
 *            token g * (t / g) + r for r = 0 .. t % g (the new token's group
 *            from its start through the new token); rows after t % g are not
 *            read (they count as zero, as in a whole-cache pack).
 *   V_new    device, [B, H_kv, D] in in_dtype: V of the new token.
 *   in_dtype KVQ_F32 or KVQ_BF16 (bf16 widened exactly to float32 first).
 * A length outside 1..N_cap is recorded for kvq_check (KVQ_ERR_LENGTH) and
 * that sequence's cache is left untouched.
 * Errors: as kvq_attend; KVQ_ERR_ARG (K_tail or V_new NULL, bad in_dtype),
 * KVQ_ERR_ALIGN (K_tail or V_new not aligned to its element size).
 */
KVQ_API kvq_status kvq_decode_step(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                   const int32_t* lengths, const void* K_tail, const void* V_new,
                                   kvq_dtype in_dtype, int32_t H_q, float scale, void* O, void* workspace,
                                   size_t ws_bytes, int32_t splits, void* stream);

/*
 * Attention of Q over the packed cache followed by a window of recent tokens
 * kept unquantized.  The pages leave this as their next study: keep the same
 * packed format and spend a limited high-precision budget on the most recent
 * tokens ("KV分组打包：4-bit到底省了多少？", section "小练习与常见错误", last
 * paragraph).  The keys of sequence b are its packed tokens [0, lengths[b])
 * followed by its window tokens [0, win_lengths[b]); each query row takes one
 * softmax over all of them.
 *   Q, cache, H_q, Lq, scale, O, workspace, ws_bytes, splits: as kvq_attend,
 *            except that the workspace must hold kvq_workspace_size_window(...)
 *            bytes.
 *   lengths      device int32 [B]: packed keys of each sequence, 0..N_cap.
 *   K_win, V_win device, [B, H_kv, W_cap, D] in win_dtype (KVQ_F32 or
 *                KVQ_BF16), element (b, h, t, d) at ((b*H_kv + h)*W_cap + t)*D
 *                + d; caller-owned, read only.
 *   win_lengths  device int32 [B]: window keys of each sequence, 0..W_cap.
 *   W_cap        window capacity per sequence, >= 1.
 * A sequence with lengths outside 0..N_cap, win_lengths outside 0..W_cap, or
 * no key at all is recorded for kvq_check (KVQ_ERR_LENGTH); lengths are read
 * clamped to their ranges, and a sequence with no key gets zero rows.  The
 * call launches the packed-cache kernel, a small kernel for the window's
 * share and the split merge, which every sequence goes through.
 * Errors: as kvq_attend.
 */
KVQ_API kvq_status kvq_attend_window(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                     const int32_t* lengths, const void* K_win, const void* V_win,
                                     kvq_dtype win_dtype, const int32_t* win_lengths, int32_t W_cap,
                                     int32_t H_q, int32_t Lq, float scale, void* O, void* workspace,
                                     size_t ws_bytes, int32_t splits, void* stream);

/* Workspace bytes kvq_attend_window needs (host); 0 for invalid arguments. */
KVQ_API size_t kvq_workspace_size_window(const kvq_cache* cache, int32_t H_q, int32_t Lq, int32_t splits);

/*
 * kvq_attend without a caller workspace, for callers that cannot allocate
 * device memory when they call: code inside an engine that reserves all its
 * device memory at start-up and allows no allocation afterwards, or a hot
 * loop where a cudaMalloc would synchronize the device and stall other
 * streams.  The pages have no counterpart; this is a library convenience.
 *
 * Same arguments and results as kvq_attend minus workspace/ws_bytes.  The
 * split-KV scratch is a fixed array of KVQ_NOALLOC_SCRATCH_BYTES compiled
 * into the library; every GPU that loads the library holds it until the
 * process exits.  The function allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library call).
 * - Limit: if kvq_workspace_size(cache, H_q, Lq, splits) exceeds
 *   KVQ_NOALLOC_SCRATCH_BYTES the call returns KVQ_ERR_WORKSPACE and
 *   launches nothing; use kvq_attend with your own workspace instead.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - All calls on a device share the one array and it keeps the previous
 *   call's contents (no state is carried from one call to the next); calls
 *   whose kernels may overlap on the GPU race on it, so order them (one
 *   stream, or events).
 */
#define KVQ_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
KVQ_API kvq_status kvq_attend_noalloc(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                      const int32_t* lengths, int32_t H_q, int32_t Lq,
                                      float scale, void* O, int32_t splits, void* stream);

/* Size in bytes of the fixed scratch array kvq_attend_noalloc uses. */
KVQ_API size_t kvq_noalloc_scratch_bytes(void);

/*
 * Self-test of the bounded waits of the tuned decode kernel (a test hook; the
 * pages have no counterpart).  Every wait inside the library's kernels is
 * bounded so that a lost completion ends the kernel with an error instead of
 * hanging the GPU; this call makes one completion go missing on purpose, on
 * the host's say-so, without any fault: it runs kvq_attend's decode kernel on
 * the caller's arguments (Lq = 1; the arguments must select the tuned decode
 * kernel, else KVQ_ERR_UNSUPPORTED) with every wait limited to wait_ms, and
 * the first worker's copy of its lose_block-th block arms 16 bytes more than
 * it brings, so that block's barrier never completes.  That worker's waits
 * then run out: its pair stops, writes nothing, waits (at most about two
 * seconds) for the copies it issued, and returns; every other worker
 * finishes normally.  kvq_check then returns KVQ_ERR_TIMEOUT, within wait_ms
 * plus about two seconds, and the device stays usable.  The output rows of
 * the (b, h) pairs that worker covered are not valid.
 *   lose_block  0-based index of the block in the first worker's range
 *               (must be one it has; otherwise nothing is lost).
 *   wait_ms     1..10000.
 * Errors: as kvq_attend, KVQ_ERR_ARG (lose_block < 0, wait_ms out of range),
 * KVQ_ERR_UNSUPPORTED.
 */
KVQ_API kvq_status kvq_selftest_timeout(const void* Q, kvq_dtype q_dtype, const kvq_cache* cache,
                                        const int32_t* lengths, int32_t H_q, float scale, void* O,
                                        void* workspace, size_t ws_bytes, int32_t splits, int32_t lose_block,
                                        uint32_t wait_ms, void* stream);

/* Workspace bytes kvq_attend needs for these arguments on the current
 * device (host).  Returns 0 for invalid arguments. */
KVQ_API size_t kvq_workspace_size(const kvq_cache* cache, int32_t H_q, int32_t Lq, int32_t splits);

/* Wait for `stream`, then return and clear the device error word of the
 * current device: KVQ_OK, KVQ_ERR_LENGTH, KVQ_ERR_TIMEOUT or
 * KVQ_ERR_DEVICE (KVQ_ERR_CUDA if the wait itself failed). */
KVQ_API kvq_status kvq_check(void* stream);

/* Static text for a status code. */
KVQ_API const char* kvq_strerror(kvq_status status);

/* Number of kernels this library has launched in this process so far (host
 * counter, all devices).  Used to count launches inside a timed region. */
KVQ_API uint64_t kvq_launch_count(void);

/* Name of the attention kernel kvq_attend would run for these arguments
 * ("decode_gqa4_d128", "generic", ...), for logs and tests. */
KVQ_API const char* kvq_attend_kernel_name(const kvq_cache* cache, int32_t H_q, int32_t Lq);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
