/*
 * kvq.h -- single-token decode attention over a block-quantized KV cache with
 * sparse V dequantization, for NVIDIA B200 (sm_100a).
 *
 * The method (tproger.ru, "Пропуск 90% работы по деквантизации ускорил
 * декодирование LLM", sections "Решение — не ускорять, а пропускать" and
 * "FAQ"): in a flash-attention decode kernel the softmax weights are known from
 * K before any V work starts; every position whose weight exp(s_j - m_running)
 * is below a threshold tau (the page uses 1e-6) has its V dequantization and
 * accumulation skipped entirely.  K is always dequantized, because it produces
 * the weights.  The page names q8_0, q4_0 and a Walsh-Hadamard-rotated
 * codebook format (section "Почему это работает для любой квантизации"); its opening
 * summary also names NVFP4.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All pointers named "device" are CUDA device pointers; "host" pointers are
 *    ordinary CPU memory.  The caller owns every buffer; the library allocates
 *    nothing and keeps no per-call state.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call that takes a stream is asynchronous on it.
 *  - Return value: KVQ_OK or a negative KVQ_ERR_* code.  Argument checks run on
 *    the host before anything is launched; on any error nothing is launched.
 *    Faults detected inside a kernel (an out-of-range page index or sequence
 *    length, a timed-out wait) set bits in the workspace's device flag word,
 *    read back with kvq_read_device_flags(); outputs of such a call are
 *    undefined.  No kernel traps.
 *
 * Cache layout (one "plane pair" for K, one for V)
 * ------------------------------------------------
 *  codes  plane: uint8  [num_pages][num_kv_heads][page_size][kvq_code_row_bytes(fmt, D)]
 *  scales plane: fp16   [num_pages][num_kv_heads][page_size][kvq_scale_row_count(fmt, D)]
 *  (the scales plane is addressed in fp16 slots; for nvfp4 they hold raw bytes)
 *  A "slot" is page * page_size + offset_in_page.  A contiguous cache is the
 *  special case page_size = capacity, one page per sequence (page b for b).
 *
 *  q8_0  (32 int8 codes per block of 32 along head_dim, fp16 scale d):
 *        d = absmax/127, q = round-half-away(x/d) in [-127, 127], x_hat = q*d.
 *        codes row = D bytes (int8), scales row = D/32 fp16.
 *  q4_0  (32 4-bit codes per block, fp16 scale d): m = the signed element of
 *        largest |x|, d = m/-8, q = min(15, floor(x/d + 8.5)), x_hat = (q-8)*d.
 *        codes row = D/2 bytes, element 2j in the low nibble of byte j and
 *        element 2j+1 in the high nibble; scales row = D/32 fp16.
 *  lut4  (rotated 4-bit codebook): y = c*H_D*(s .* x) with s the fixed random
 *        signs, H_D the Sylvester Hadamard matrix and c = 1/sqrt(D); n = |y|;
 *        idx = index of the codebook interval of y/n (thresholds at midpoints
 *        of consecutive centroids); x_hat' = n*codebook[idx] in the rotated
 *        domain.  codes row = D/2 bytes (nibbles as for q4_0); scales row = 1
 *        fp16 (the norm n).  Attention runs in the rotated domain and the
 *        output is rotated back (R^T = diag(s) c H_D), so every format returns
 *        the same, unrotated, output.
 *  nvfp4 (E2M1 codes, blocks of 16 along head_dim): g = amax/2688 over the vector
 *        (fp32); per block s = e4m3(amax_b / (6 g)); code = e2m1(x / (g s));
 *        x_hat = e2m1_value(code) * s * g.  e4m3 / e2m1 round to nearest, ties to
 *        the even code, saturating at 448 / 6; e2m1 keeps the sign of x.  codes row =
 *        D/2 bytes (nibbles as for q4_0, E2M1 bit patterns); scales row = the D/16
 *        E4M3 bytes, the fp32 g (little-endian), zero padding to a multiple of 8
 *        bytes: 8 fp16 slots for D = 128, 4 for D = 64.
 *  All quantizer arithmetic is IEEE fp32 round-to-nearest-even, one operation
 *  at a time (no fused multiply-add), so codes are fixed to the bit.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
#define KVQ_OK                0
#define KVQ_ERR_INVALID_ARG  -1  /* null pointer, negative size, bad alignment, ... */
#define KVQ_ERR_UNSUPPORTED  -2  /* format / head_dim / group size / page size not built */
#define KVQ_ERR_CUDA         -3  /* a CUDA runtime call or launch failed */
#define KVQ_ERR_WORKSPACE    -4  /* workspace too small */
#define KVQ_ERR_DEVICE       -5  /* a kernel reported a fault through the flag word */

/* ------------------------------------------------------------ formats */
#define KVQ_FMT_Q8_0  0
#define KVQ_FMT_Q4_0  1
#define KVQ_FMT_LUT4  2
#define KVQ_FMT_NVFP4 3

/* Option bits of kvq_decode_attn. */
#define KVQ_OPT_SHARED_MAX 1u  /* the splits of one cluster share one running maximum (below) */
#define KVQ_OPT_GLOBAL_MAX 2u  /* every split uses the maximum over all splits of its sequence (below) */
#define KVQ_OPT_V_KEPT_ONLY 4u /* tau > 0: copy only the kept V rows, after the skip test (below) */
#define KVQ_OPT_V_WITH_K    8u /* tau > 0: copy every V tile together with its K tile (below) */

/* Device flag bits (kvq_read_device_flags). */
#define KVQ_FLAG_BAD_PAGE     1u  /* a page-table entry outside [0, num_pages) */
#define KVQ_FLAG_BAD_SEQLEN   2u  /* seq_len < 0, > max_seq_len or > max_pages*page_size */
#define KVQ_FLAG_TIMEOUT      4u  /* a bounded wait (cross-CTA exchange, flag) gave up */

/* Compile-time limits of the library. */
#define KVQ_MAX_GROUP        8     /* query heads per KV head (num_q_heads / num_kv_heads) */
#define KVQ_MAX_SPLIT_TOKENS 1024  /* positions per split-KV work unit */
#define KVQ_MAX_BATCH        1024
#define KVQ_MAX_SPLITS       4096  /* splits of one sequence: max_seq_len <= 4096 * split length */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)  /* static scratch of kvq_decode_attn_noalloc */

typedef struct kvq_cache_desc {
    int32_t fmt;              /* KVQ_FMT_* */
    int32_t head_dim;         /* 64 or 128 */
    int32_t num_kv_heads;     /* >= 1 */
    int32_t page_size;        /* tokens per page, a positive multiple of 64 */
    int32_t num_pages;        /* physical pages held by each plane */
    const uint16_t* codebook; /* lut4 only: device, 16 IEEE fp16 centroids, increasing */
    const int8_t* signs;      /* lut4 only: device, head_dim entries, each +1 or -1 */
} kvq_cache_desc;

/* Bytes of one (token, KV head) row of the codes plane; 0 if (fmt, head_dim) is unsupported. */
size_t kvq_code_row_bytes(int32_t fmt, int32_t head_dim);
/* fp16 values in one row of the scales plane; 0 if unsupported. */
size_t kvq_scale_row_count(int32_t fmt, int32_t head_dim);

/*
 * kvq_quantize -- write n_tokens K (or V) vectors into a cache plane pair.
 *   Passage: tproger page, "Почему это работает для любой квантизации" (the q8_0, q4_0 and
 *   Walsh-Hadamard-rotated codebook KV formats the method runs on) and "Ключевые выводы"
 *   (NVFP4); the pages fix no block arithmetic, so the formulas above are this library's.
 *   x       device fp16 [n_tokens][num_kv_heads][head_dim]
 *   slots   device int32 [n_tokens]: physical slot of token i (NULL: slot i);
 *           every slot must lie in [0, num_pages*page_size) (not checked on device)
 *   codes, scales  device planes (layout above), 16-byte aligned
 * The block formulas are the ones in the header comment; the result is
 * bit-identical to an IEEE fp32 evaluation of them.  lut4 needs desc->codebook
 * and desc->signs.  n_tokens == 0 is a no-op.
 */
int kvq_quantize(const kvq_cache_desc* desc, const void* x, int32_t n_tokens,
                 const int32_t* slots, void* codes, void* scales, void* stream);

/*
 * kvq_quantize_kv -- kvq_quantize of the K vectors k into (k_codes, k_scales) and of the
 *   (Passage: as kvq_quantize.)
 * V vectors v into (v_codes, v_scales), same slots, in one launch (the append of a
 * decode step).  Arguments, layout, results and errors are those of two kvq_quantize
 * calls.
 */
int kvq_quantize_kv(const kvq_cache_desc* desc, const void* k, const void* v, int32_t n_tokens,
                    const int32_t* slots, void* k_codes, void* k_scales, void* v_codes,
                    void* v_scales, void* stream);

/*
 * kvq_resolve_split -- the split length L (positions per split-KV work unit) that
 *   (No passage: the pages' kernel walks one sequence; splitting it across SMs is this
 *   library's schedule, reported so that a checker can replay it.)
 * kvq_decode_attn and kvq_combine use for a request (same split_tokens and
 * options).  split_tokens > 0 is capped at KVQ_MAX_SPLIT_TOKENS and rounded up to a
 * multiple of 64; split_tokens == 0 picks one from the problem size and how many
 * CTAs (or CTA clusters) of the decode kernel fit on the current device: at least 32
 * splits per (sequence, KV head), more when that leaves SMs idle, splits of at least
 * 128 positions, and the shortest such length whose splits all run at once (one CTA
 * each, CTAs of 4, 8 or 16 warps, one per 64-position tile); when even the longest
 * split leaves more splits than CTAs, splits of 512 positions that the CTAs loop over.
 * Returns L (> 0) or a KVQ_ERR_* code.
 * Sequence b is cut into splits [k*L, min((k+1)*L, seq_len_b)), k = 0, 1, ...
 */
int32_t kvq_resolve_split(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                          int32_t max_seq_len, int32_t split_tokens, uint32_t options);

/*
 * kvq_resolve_cluster -- CS, the number of consecutive splits of one (sequence, KV
 * head) that one thread-block cluster processes together (same arguments as
 * kvq_resolve_split).  CS = 1 without KVQ_OPT_SHARED_MAX; with it CS is 2 or 4
 * (when sequences are long enough), splits kCS .. kCS + CS - 1 form cluster group k,
 * and the CTAs of a group share one running maximum (exchanged on chip); the
 * workspace still holds one partial per split.
 */
int32_t kvq_resolve_cluster(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                            int32_t max_seq_len, int32_t split_tokens, uint32_t options);

/* Workspace bytes for a resolved split length L (> 0). */
size_t kvq_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                          int32_t max_seq_len, int32_t split_tokens);

/* Zero the workspace (its device flag word, the launch counter that tags the (m, l)
 * exchange, the cleared-rows flags and the arrival counts); call once after allocating it.  A workspace whose
 * call to kvq_decode_attn completed is ready for the next call without another init,
 * whatever the next call's shape; after KVQ_FLAG_TIMEOUT, init it again. */
int kvq_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * kvq_selftest_wait -- diagnostic: runs the decode kernel's bounded waits (the (m, l)
 * exchange poll and the cleared-rows flag wait) against entries in the workspace header
 * that never become ready, each giving up after max_cycles SM cycles (> 0) and setting
 * KVQ_FLAG_TIMEOUT in the workspace's flag word, as a decode whose splits could not all
 * meet would.  It reads the header's spare bytes only; the GPU context stays usable.
 *   workspace  device, >= 256 bytes (the header), 16-byte aligned
 */
int kvq_selftest_wait(void* workspace, size_t workspace_bytes, long long max_cycles, void* stream);

/* Synchronize `stream` and read the device flag word (KVQ_FLAG_* bits) into *flags (host). */
int kvq_read_device_flags(const void* workspace, uint32_t* flags, void* stream);

/*
 * kvq_decode_attn -- split-KV decode attention with sparse V.
 *   Passage: tproger page, "Решение — не ускорять, а пропускать" (the softmax weights come
 *   from K before V is touched; a position whose weight is below the threshold, 1e-6 on
 *   the page, has its V dequantization and accumulation skipped) and "FAQ" (K is always
 *   dequantized, since it produces the weights).
 *   q            device fp16 [batch][num_q_heads][head_dim], 16-byte aligned
 *   k_codes, k_scales, v_codes, v_scales   device planes (layout above), 16-byte aligned
 *   page_table   device int32 [batch][max_pages] (NULL: sequence b uses pages
 *                b*max_pages .. b*max_pages + max_pages - 1)
 *   seq_lens     device int32 [batch], each in [0, min(max_seq_len, max_pages*page_size)]
 *   sm_scale     score scale (1/sqrt(head_dim) for standard attention)
 *   tau          skip threshold, >= 0.  Position j of split s is skipped for
 *                query head h when exp(s_hj - m_hs) < tau, where m_hs is the running
 *                maximum once all K tiles of the split are folded in (with
 *                KVQ_OPT_SHARED_MAX: of all splits of its cluster group, see
 *                kvq_resolve_cluster; with KVQ_OPT_GLOBAL_MAX: of all splits of the
 *                (sequence, KV head), i.e. the final maximum of the whole K pass).
 *                tau = 0 keeps everything (dense attention).
 *                Skipped positions still count in the softmax denominator.
 *   split_tokens as for kvq_resolve_split (0 = auto)
 *   options      at most one of KVQ_OPT_SHARED_MAX and KVQ_OPT_GLOBAL_MAX, at most one
 *                of KVQ_OPT_V_KEPT_ONLY and KVQ_OPT_V_WITH_K; other bits or both of a
 *                pair are an error.
 *                How V reaches the SM (results are the same either way): with
 *                KVQ_OPT_V_KEPT_ONLY a split copies only its kept V rows, once its
 *                skip test is done (fewest bytes; a second DRAM round trip); with
 *                KVQ_OPT_V_WITH_K every V tile is copied together with its K tile and
 *                the skipped rows are left out of the contraction only (more bytes, no
 *                second round trip).  Neither: V_WITH_K (measured faster on B200, where
 *                these steps are bound by latency and instruction issue rather than by
 *                HBM bytes).  tau = 0 always copies V with K.  Where K and V tiles do not
 *                both fit in shared memory (q8_0 at head_dim 128), each V tile is copied
 *                into its K tile's place as soon as that tile's scores are taken.
 *                KVQ_OPT_GLOBAL_MAX needs every split of the request on its own
 *                CTA at once (KVQ_ERR_UNSUPPORTED otherwise): the CTAs of a (sequence, KV
 *                head) exchange their maxima through the workspace between the K pass
 *                and the V pass (a bounded wait; KVQ_FLAG_TIMEOUT if it gives up).
 *   workspace    device, kvq_workspace_size(...) bytes, 16-byte aligned, initialized
 *                once with kvq_workspace_init.  Receives one partial (unnormalized o,
 *                running maximum m, denominator l) per cluster group (with `out` given,
 *                o may be left unwritten).
 *   stats        device uint64 [4] or NULL; ADDED to (caller zeroes):
 *                [0] (position, query head) pairs scored, [1] pairs skipped,
 *                [2] V rows needed (positions kept by any head of the group; the
 *                rows copied, unless V tiles are copied with K),
 *                [3] V rows skipped
 *   out          device fp32 [batch][num_q_heads][head_dim], 16-byte aligned, or NULL.
 *                When given, the call also merges the splits and writes the output (the
 *                log-sum-exp rule of kvq_combine): when every split of the request runs
 *                on its own CTA at once, inside the decode kernel, each split adding its
 *                normalized share into the output with floating-point atomics (so the
 *                last bits of the output may differ from run to run); otherwise by a
 *                second launch on the same stream, the combine kernel of kvq_combine.  Calls that share a workspace
 *                must not overlap on the GPU.
 * Query head h attends with KV head h / (num_q_heads / num_kv_heads).
 * The group size num_q_heads / num_kv_heads must be 1..KVQ_MAX_GROUP.
 */
int kvq_decode_attn(const kvq_cache_desc* desc, const void* q, int32_t batch,
                    int32_t num_q_heads, const void* k_codes, const void* k_scales,
                    const void* v_codes, const void* v_scales, const int32_t* page_table,
                    int32_t max_pages, const int32_t* seq_lens, int32_t max_seq_len,
                    float sm_scale, float tau, int32_t split_tokens, uint32_t options,
                    void* workspace, size_t workspace_bytes, unsigned long long* stats,
                    float* out, void* stream);

/*
 * kvq_combine -- log-sum-exp merge of the partials of kvq_decode_attn (same
 *   (No passage: the pages' kernel keeps one running softmax per sequence; the merge of
 *   split-KV partials is the standard log-sum-exp identity written out below.)
 * batch, num_q_heads, max_seq_len, split_tokens, options, seq_lens and workspace), for callers
 * that passed no output pointer to it (or that merge partials from elsewhere):
 *   M = max_s m_s,  out = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s,
 * rotated back to the caller's basis for lut4.
 *   out  device fp32 [batch][num_q_heads][head_dim]; a sequence of length 0
 *        gets zeros.
 */
int kvq_combine(const kvq_cache_desc* desc, const void* workspace, int32_t batch,
                int32_t num_q_heads, int32_t max_seq_len, int32_t split_tokens, uint32_t options,
                const int32_t* seq_lens, float* out, void* stream);

/*
 * kvq_decode_attn_noalloc -- kvq_decode_attn with an output pointer, for callers that
 * cannot allocate device memory while decoding (a serving runtime that plans every
 * buffer up front, a process confined to a fixed memory pool, or code running where
 * cudaMalloc is not allowed).  The method's pages have no counterpart: this is packaging.
 *   The per-split partials live in a library-owned static device array of
 *   KVQ_NOALLOC_SCRATCH_BYTES (8 MiB); every GPU that loads the library keeps it until
 *   the process exits.  Nothing is allocated or freed by the call.
 *   Arguments are those of kvq_decode_attn without the workspace; `out` is required.
 *   Returns KVQ_ERR_WORKSPACE when kvq_workspace_size(...) for the request exceeds
 *   KVQ_NOALLOC_SCRATCH_BYTES.
 *   Every call looks up the array's device address with the calling thread's current
 *   device; the first call on a device is its set-up and may load the library's device
 *   code there, so make it before any stream capture.  All calls share the one array and
 *   each call clears its fault-flag word and merge words first, so calls whose
 *   execution overlaps on the GPU (different streams, or another thread) race.  Faults
 *   that the kernel detects (KVQ_FLAG_*) are read back with kvq_noalloc_read_flags.
 */
int kvq_decode_attn_noalloc(const kvq_cache_desc* desc, const void* q, int32_t batch,
                            int32_t num_q_heads, const void* k_codes, const void* k_scales,
                            const void* v_codes, const void* v_scales, const int32_t* page_table,
                            int32_t max_pages, const int32_t* seq_lens, int32_t max_seq_len,
                            float sm_scale, float tau, int32_t split_tokens, uint32_t options,
                            unsigned long long* stats, float* out, void* stream);

/*
 * kvq_noalloc_read_flags -- synchronize `stream` and read the KVQ_FLAG_* bits that the last
 * kvq_decode_attn_noalloc call on the current device left in the static scratch (each call
 * clears them first) into *flags (host).  Like that call, it allocates nothing.  Returns
 * KVQ_ERR_INVALID_ARG for a null `flags`, KVQ_ERR_CUDA if a CUDA call fails.
 */
int kvq_noalloc_read_flags(uint32_t* flags, void* stream);

/*
 * kvq_lloyd_max_codebook -- the minimum-MSE `levels`-entry scalar codebook for
 *   (Passage: the rotated codebook format of "Почему это работает для любой квантизации";
 *   the page names no codebook, Lloyd-Max for the rotated coordinates' Gaussian is this
 *   library's reading.)
 * N(0, sigma^2) (Lloyd's iteration in fp64, symmetric), rounded to IEEE fp16
 * (round-to-nearest-even) and written to out_fp16 (host, `levels` entries,
 * increasing).  The lut4 format uses levels = 16, sigma = 1/sqrt(head_dim).
 */
int kvq_lloyd_max_codebook(int32_t levels, double sigma, uint16_t* out_fp16);

/* A static, human-readable name for a status code. */
const char* kvq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
