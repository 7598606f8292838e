/*
 * hqmq.h -- C ABI of libhqmq, the B200 (sm_100a) implementation of the
 * HQMQ (Hurwitz Quaternion Multiplicative Quantization) KV-cache codec.
 *
 * What is computed (sources named by page and section):
 *   - every 4 consecutive elements of a K or V head vector form a quaternion
 *     x = (w, i, j, k) (arXiv 2605.27646 abstract, paperdance.org/p/2605.27646;
 *     gist.science/nl/paper/2605.27646, Technische Samenvatting, Methodologie);
 *   - x is split into its norm r = |x| and direction u = x / r (same section);
 *   - u is snapped to the codeword q_p q_s maximising <u, q_p q_s>, where q_p
 *     runs over the 24-element Hurwitz group 2T and q_s over S seeded random
 *     unit quaternions of this (layer, head, role): 24 S codewords from S
 *     stored quaternions (gist.science/nl, Technische Samenvatting, section 1
 *     "Multiplicatieve Samenstelling van Codeboeken"; abstract);
 *   - optionally first, Med3x: the median chunk norm r_med of the current
 *     batch is taken per head; chunks with r > C r_med (C = 3) are kept in
 *     fp16 in a side list and the rest is quantised (gist.science/nl,
 *     Technische Samenvatting, section 3 "Mediane-Multiplier
 *     Uitbijterextractie"; gist.science/pt, Resumo Tecnico, section 3);
 *   - decode rebuilds r * (q_p q_s) and restores the outliers (the fused
 *     decoder of gist.science/nl, Technische Samenvatting, "Memory en
 *     Latentie", reads the same stored pair);
 *   - decode-phase attention straight from the codes (that same section:
 *     the decoder runs inside attention), hqmq_attention_decode;
 *   - an optional b-bit radius code matching the pages' bit budget
 *     (hqmq_quantize_radius, hqmq_decode_qradius), the joint (index, level)
 *     block code and the 1-bit outlier flags (hqmq_pack_joint,
 *     hqmq_list_flags, hqmq_decode_joint);
 *   - Med3x under a given threshold for decode-step tokens, and all of a
 *     step's small calls in one launch (hqmq_outlier_extract_given_thr,
 *     hqmq_append_batch).
 *
 * Conventions fixed by this library where the pages are silent:
 *   - one call = one (layer, role) tensor x[B][H][T][D], row-major, D % 4 == 0
 *     and (T*D/4) % 32 == 0.  Chunk j covers elements 4j .. 4j+3; its head is
 *     (j / (T*D/4)) % H; a "slab" is one (b, h) pair, slab index b*H + h.
 *   - 2T enumeration p in [0,24): p = 2a + sg for the units +-1,+-i,+-j,+-k
 *     (a = axis w,i,j,k; sg = 1 for the minus sign); p = 8 + m for
 *     1/2((-1)^m0, (-1)^m1, (-1)^m2, (-1)^m3), m_c = bit c of m.
 *   - codeword index s*24 + p; among equal fp32 scores the lowest index wins.
 *   - index width b = ceil(log2(24 S)) bits; per group of 32 consecutive
 *     chunks, b uint32 words; bit i of chunk k's index is bit k*b+i of the
 *     group's b-word stream (LSB first).
 *   - radius: fp16, round-to-nearest-even, saturated at 65504.
 *   - codebook group numbering g = (layer*2 + role)*H + head (role 0 = K,
 *     1 = V); a call's H codebooks are therefore contiguous.
 *
 * Ownership and execution: the caller allocates every buffer; all pointers
 * are device pointers unless stated; nothing is allocated, freed or kept
 * between calls.  Every compute entry point only enqueues work on `stream`
 * (a cudaStream_t passed as void*; NULL = the legacy default stream) and
 * returns without synchronising.  Some kernels are launched with
 * programmatic dependent launch: such a kernel may be scheduled while the
 * previous kernel on the stream is still running, but waits for it to
 * complete before it touches memory, so stream order holds for any
 * predecessor; the calls can also be captured in CUDA graphs.  Argument
 * errors are returned synchronously and nothing is enqueued.  Data-dependent conditions (outlier capacity
 * overflow, fp16 saturation, non-finite input, corrupt indices) never trap:
 * they are recorded in the device-resident hqmq_status (if non-NULL), whose
 * counters the calls add to; the caller zeroes it.
 */
#ifndef HQMQ_H
#define HQMQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HQMQ_API __attribute__((visibility("default")))
#else
#define HQMQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define HQMQ_OK 0
#define HQMQ_ERR_ARG 1        /* a size, enum or pointer argument is invalid   */
#define HQMQ_ERR_ALIGN 2      /* a pointer misses its stated alignment         */
#define HQMQ_ERR_CUDA 3       /* a CUDA launch or runtime call failed          */
#define HQMQ_ERR_WORKSPACE 4  /* workspace smaller than hqmq_outlier_workspace_size */

/* Element types of x / y. */
#define HQMQ_BF16 0
#define HQMQ_F32 1

/* Med3x granularity: chunk norms (the pages' rule) or single |x| elements. */
#define HQMQ_GRAN_CHUNK 0
#define HQMQ_GRAN_ELEMENT 1

/* hqmq_status.flags bits. */
#define HQMQ_FLAG_OUTLIER_OVERFLOW 1u /* more outliers than cap; n_outliers = needed */
#define HQMQ_FLAG_SATURATED 2u        /* an fp16 radius or outlier value saturated   */
#define HQMQ_FLAG_NONFINITE 4u        /* a chunk norm was NaN or inf                 */
#define HQMQ_FLAG_BAD_INDEX 8u        /* decode met an index >= 24 S                 */
#define HQMQ_FLAG_MED3_FALLBACK 16u   /* a head's sampled median window missed; its
                                         median came from the exact (slow) path    */

/* Device-resident status record (caller-allocated, 32 bytes, 8-byte aligned).
 * Calls OR flags in and add to the counters. */
typedef struct {
    uint32_t flags;
    uint32_t reserved;
    uint64_t n_outliers;   /* outliers found by hqmq_outlier_extract          */
    uint64_t n_saturated;  /* fp16 values clamped to +-65504                  */
    uint64_t n_nonfinite;  /* chunks encoded with a NaN/inf norm              */
} hqmq_status;

/* Library version string, e.g. "hqmq-b200 1.0". */
HQMQ_API const char *hqmq_version(void);

/* Static text for a return code. */
HQMQ_API const char *hqmq_error_string(int err);

/* Index width b = ceil(log2(24 S)) for S in [1, 65535]; 0 if S is out of range. */
HQMQ_API uint32_t hqmq_index_bits(uint32_t S);

/* Number of uint32 index words of one call: (B*H*T*D/128) * b; 0 on bad shape. */
HQMQ_API uint64_t hqmq_index_words(int B, int H, int T, int D, uint32_t S);

/* Secondary codebooks (gist.science/nl, Technische Samenvatting, section 1:
 * S random unit quaternions per (layer, head, role), no calibration;
 * abstract: seeded).  Writes d_codebook[n_groups][S][4] fp32 for groups
 * group0 .. group0 + n_groups - 1.  Quaternion (g, s): Philox4x32-10 with
 * counter (s, g, 0, 0) and key (seed low 32 bits, seed high 32 bits) gives
 * four uint32 v; u = (v + 1/2) 2^-32; two Box-Muller pairs in fp64 give four
 * N(0,1) deviates z; q = z / |z| rounded to fp32.
 * S in [1, 65535]; n_groups >= 1; group0 + n_groups <= 2^32;
 * d_codebook 16-byte aligned. */
HQMQ_API int hqmq_make_codebook(uint64_t seed, uint32_t S, uint32_t n_groups, uint32_t group0,
                       float *d_codebook, void *stream);

/* Bytes of device workspace hqmq_outlier_extract (and hqmq_encode_med3) needs
 * for this shape: a 64 Ki-bin sample histogram per head, the keys of the median
 * window, the uncertain-threshold list, per-tile counts and offsets and one
 * candidate bit per chunk (about 29 MB for a 1 x 8 x 131072 x 128 call in
 * chunk mode). */
HQMQ_API uint64_t hqmq_outlier_workspace_size(int B, int H, int T, int D, int gran);

/* Med3x (gist.science/nl, Technische Samenvatting, section 3; the pages
 * use chunk norms, HQMQ_GRAN_CHUNK; HQMQ_GRAN_ELEMENT applies the same rule
 * to single-element magnitudes |x|).
 * Per head h, over all B batches and T tokens of this call:
 *   r_med[h] = lower median (rank N/2 - 1 of N ascending) of the fp32 chunk
 *              norms r = sqrt(fma(x3,x3, fma(x2,x2, fma(x1,x1, x0*x0))))
 *              (or of |x| per element); a NaN sorts above +inf;
 *   thr[h]   = fl32(C * r_med[h]).
 * A chunk (element) is an outlier iff r > thr[h] (|x| > thr[h]).  The outlier
 * list is written in ascending flat index order:
 *   chunk mode:   d_out_idx[n] = chunk index j, d_out_val[n*4 + i] = fp16 bits
 *                 of element 4j+i;
 *   element mode: d_out_idx[n] = element index, d_out_val[n] = fp16 bits;
 *   fp16 = round-to-nearest-even, finite values beyond +-65504 saturate.
 * d_slab_off[B*H+1]: entries of slab (b,h) are [slab_off[b*H+h], slab_off[b*H+h+1]).
 * d_tile_off (NULL = not wanted): uint32[hqmq_list_tiles(B,H,T,D) + 1],
 * 16-byte aligned: the list position of the first entry of each list tile
 * (1024 consecutive chunks of a slab; a slab's last tile may be shorter),
 * then the total.  hqmq_decode uses it to apply the list in its main pass.
 * Entries at positions >= cap are not written (d_slab_off and d_tile_off
 * still hold the full offsets); the status then gets
 * HQMQ_FLAG_OUTLIER_OVERFLOW and n_outliers the required total, so the
 * caller can retry with a larger cap.
 * Data flow (two reads of x): a 1/32 sample fixes per head a key window that
 * holds the median rank with overwhelming probability; one full read counts
 * the keys below the window, keeps the keys inside it and counts per
 * 1024-chunk tile the chunks above the threshold's range; the exact median is
 * selected from the window keys (a head whose window misses the median, or
 * whose buffers overflow, is decided by an exact three-pass selection over x
 * instead, so the result never depends on the sample); the second read
 * writes the ordered list.
 * d_x: bf16 or fp32 [B][H][T][D], 16-byte aligned.  d_rmed, d_thr: fp32 [H].
 * d_out_idx: uint32[cap]; d_out_val: uint16[cap*4] (chunk) or [cap] (element),
 * 4-byte aligned.  d_ws: at least hqmq_outlier_workspace_size bytes,
 * 256-byte aligned, contents on entry ignored.  C > 0 and finite.
 * B*H*T*D must be < 2^32. */
HQMQ_API int hqmq_outlier_extract(const void *d_x, int dtype, int B, int H, int T, int D, float C,
                         int gran, float *d_rmed, float *d_thr, uint32_t *d_out_idx,
                         uint16_t *d_out_val, uint32_t *d_slab_off, uint32_t *d_tile_off,
                         uint64_t cap, void *d_ws, uint64_t ws_bytes, hqmq_status *d_status,
                         void *stream);

/* Number of list tiles of a call (the length of d_tile_off minus one), or 0
 * for a shape the library rejects. */
HQMQ_API uint64_t hqmq_list_tiles(int B, int H, int T, int D);

/* Encode (gist.science/nl, Technische Samenvatting, Methodologie and
 * section 1): per chunk j
 *   - if d_thr != NULL: chunk mode zeroes a chunk with r > thr[h]; element
 *     mode zeroes each element with |x| > thr[h] (Med3x, the outliers live in
 *     the list of hqmq_outlier_extract);
 *   - r = fp32 norm as above; radius[j] = fp16(r) (saturating);
 *   - index = argmax over s, p of <x, q_p q_s> evaluated as
 *     <x conj(q_s), q_p> with the nearest 2T element in closed form; ties to
 *     the lowest s*24+p; r == 0 gives index 0;
 *   - a NaN/inf norm gives index 0 and radius 0x7E00 and is counted.
 * d_codebook: fp32 [H][S][4] (this call's heads), 16-byte aligned.
 * d_idx_words: uint32[hqmq_index_words(B,H,T,D,S)], fully overwritten.
 * d_radius: uint16 fp16 bits [B*H*T*D/4], 4-byte aligned. */
HQMQ_API int hqmq_encode(const void *d_x, int dtype, int B, int H, int T, int D, const float *d_codebook,
                uint32_t S, const float *d_thr, int gran, uint32_t *d_idx_words,
                uint16_t *d_radius, hqmq_status *d_status, void *stream);

/* Decode: y = round(fl32(r * c_i)) with r the fp16 radius, c = q_p q_s in
 * fp32 (each component the left-to-right sum of its four Hamilton terms; the
 * terms are exact because q_p's entries are 0, +-1, +-1/2), round = RN-even to
 * bf16 (out_dtype HQMQ_BF16) or none (HQMQ_F32).  Outliers, if d_out_idx is
 * non-NULL (list, offsets and granularity as written by hqmq_outlier_extract,
 * entries below cap only): chunk mode replaces the chunk by round(fp16
 * value); element mode gives round(fl32(fl32(r * c_i) + value)).  An index
 * >= 24 S decodes to 0 and sets HQMQ_FLAG_BAD_INDEX.
 * d_idx_words and d_radius as written by hqmq_encode; d_y: [B][H][T][D]
 * of out_dtype, 16-byte aligned.  With a list and its d_tile_off (as written
 * by hqmq_outlier_extract / hqmq_encode_med3), the main pass applies each
 * tile's entries right after writing the tile; entries whose index lies
 * outside their tile are ignored.  With a list and d_tile_off == NULL, a
 * second kernel applies the outliers after the main pass on the same stream
 * (entries outside the tensor are ignored). */
HQMQ_API int hqmq_decode(const uint32_t *d_idx_words, const uint16_t *d_radius, const float *d_codebook,
                uint32_t S, const uint32_t *d_out_idx, const uint16_t *d_out_val,
                const uint32_t *d_slab_off, const uint32_t *d_tile_off, uint64_t cap, int gran,
                int B, int H, int T, int D, void *d_y, int out_dtype, hqmq_status *d_status,
                void *stream);

/* Exact table-driven search (same results as hqmq_encode; the argmax of
 * <x, c> over the 24 S codewords c = q_p q_s, ties to the lowest index:
 * gist.science/nl, Technische Samenvatting, section 1).  A chunk x lies on one
 * of 8 cube faces: a = the first coordinate of largest |x_a|, and the sign of
 * x_a.  Its gnomonic coordinates t (the other three coordinates in index
 * order, divided by |x_a|, in [-1, 1]) are mapped by u = t (A + B t^2)
 * (A = 4/pi in fp32, B = 1 - A) and u is cut into 32^3 cells per face.  Per
 * cell the table lists, in increasing index order, up to 8 codewords that can
 * be the argmax somewhere in the cell, widened by 1e-5 in t to cover
 * rounding: a codeword is dropped only if it is farther from the cell centre
 * than the best one by more than twice the cell's angular radius, or if
 * another codeword beats it at all 8 corners (the score difference is linear
 * in x).  Cells with more than 8 candidates fall back to the S-codeword loop.
 * Supports S in [1, 48].
 *
 * Layout per group: uint4 [8 faces: 2 a + (x_a < 0)][32][32][32]; slot k of
 * a record is the 16-bit half k of the uint4 (low half first); its low 12 bits
 * hold a codeword id s 24 + p; the top 4 bits of slot 0 hold the count (0 =
 * overflow); slots past the count hold 24 S. */

/* Bytes of search table per codebook group (4194304), or 0 if S is unsupported. */
HQMQ_API uint64_t hqmq_search_table_bytes(uint32_t S);

/* Builds the tables of n_groups codebooks: d_codebook[n_groups][S][4] fp32 as
 * written by hqmq_make_codebook, d_table n_groups * hqmq_search_table_bytes(S)
 * bytes, both 16-byte aligned.  n_groups <= 65535 per call. */
HQMQ_API int hqmq_make_search_table(const float *d_codebook, uint32_t S, uint32_t n_groups,
                                    void *d_table, void *stream);

/* hqmq_encode using the search tables of this call's H heads (d_table = the
 * tables of the same groups as d_codebook, [H] x hqmq_search_table_bytes(S)).
 * Arguments, outputs and results as hqmq_encode: indices equal hqmq_encode's
 * except where two codewords' fp32 scores are within rounding of each other. */
HQMQ_API int hqmq_encode_lut(const void *d_x, int dtype, int B, int H, int T, int D,
                             const float *d_codebook, uint32_t S, const void *d_table,
                             const float *d_thr, int gran, uint32_t *d_idx_words,
                             uint16_t *d_radius, hqmq_status *d_status, void *stream);

/* Med3x and encode in one call.  Outputs equal hqmq_outlier_extract followed
 * by hqmq_encode_lut (or hqmq_encode when d_table is NULL), bit for bit, and
 * the status counts equal theirs.
 * Chunk mode with search tables reads x once: the encode pass runs before the
 * exact threshold is known, encoding a chunk above the largest threshold the
 * sample window allows as an outlier and every other chunk as a bulk chunk,
 * and marks the chunks above the smallest such threshold; after the exact
 * threshold a fix-up pass reads only the marked chunks, writes the ordered
 * list and zeroes the codes of the marked chunks that are outliers.  A head
 * whose window missed gets a full exact re-encode.  Element mode (whose
 * encode depends on the threshold) reads x twice: once for the median, once
 * for the list and the encode (a third read without d_table).  Workspace as
 * hqmq_outlier_workspace_size; other arguments as in those calls. */
HQMQ_API uint64_t hqmq_encode_med3_workspace_size(int B, int H, int T, int D, int gran);
HQMQ_API int hqmq_encode_med3(const void *d_x, int dtype, int B, int H, int T, int D, float C,
                              int gran, const float *d_codebook, uint32_t S, const void *d_table,
                              uint32_t *d_idx_words, uint16_t *d_radius, float *d_rmed,
                              float *d_thr, uint32_t *d_out_idx, uint16_t *d_out_val,
                              uint32_t *d_slab_off, uint32_t *d_tile_off, uint64_t cap,
                              void *d_ws, uint64_t ws_bytes, hqmq_status *d_status, void *stream);

/* Size of the fixed device scratch array of hqmq_outlier_extract_noalloc. */
#define HQMQ_NOALLOC_SCRATCH_BYTES (1u << 20)

/* hqmq_outlier_extract without a workspace argument.  The paper has no
 * counterpart of this entry point; it exists for callers that cannot
 * allocate device memory: a serving engine that has reserved all of the
 * GPU's memory for its own pool, or a hook running where cudaMalloc/cudaFree
 * (which may synchronise the device) are not allowed.  The caller still
 * passes every input and output.
 *
 * It runs the compact three-pass radix selection (three reads of x for the
 * median, two for the list), whose scratch is 8 KB per head plus 8 bytes per
 * 4096 chunks, in one file-scope device array of HQMQ_NOALLOC_SCRATCH_BYTES
 * (1 MiB) that every GPU which loads libhqmq holds until the process exits.
 * Shapes that need more are rejected with HQMQ_ERR_WORKSPACE.  The need is
 * 8192 H + ceil256(8 H) + 2 ceil256(4 B H ceil(T D / 16384)) bytes
 * (ceil256: rounded up to a multiple of 256), so at most 127 heads per call
 * fit, and a 1 x 8 x 131072 x 128 call needs about 130 KB.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current) and caches it for the life of the process;
 * make that first call before any stream capture.  The cached address
 * belongs to the device's primary context: after cudaDeviceReset, or with
 * another driver context current, it is stale, so neither is supported once
 * this entry point has been called.  All calls on a device
 * share the one array: calls whose execution overlaps on the GPU (different
 * streams without ordering between them) race and give wrong results.  Each
 * call clears what must start at zero.  Nothing is allocated or freed.
 * Arguments, results and errors are otherwise those of hqmq_outlier_extract
 * (it writes no tile offsets). */
HQMQ_API int hqmq_outlier_extract_noalloc(const void *d_x, int dtype, int B, int H, int T, int D,
                                          float C, int gran, float *d_rmed, float *d_thr,
                                          uint32_t *d_out_idx, uint16_t *d_out_val,
                                          uint32_t *d_slab_off, uint64_t cap,
                                          hqmq_status *d_status, void *stream);

/* Outlier list of a call under a GIVEN per-head threshold, without a median
 * of its own: the streaming form of Med3x for decode-phase tokens, whose
 * batches (often one token per sequence) are too small for a median of
 * their own (the pages take the median of the current batch, gist.science/
 * nl, Technische Samenvatting, section 3; a previous batch's threshold,
 * e.g. the prefill's d_thr from hqmq_outlier_extract, is our reading for a
 * batch that has none).  Outlier rule, list order and format, d_slab_off,
 * the optional d_tile_off (list tile offsets and total, as
 * hqmq_outlier_extract writes them), cap and status as in
 * hqmq_outlier_extract.  The new tokens are then encoded with the same
 * d_thr (hqmq_encode / hqmq_encode_lut).  d_thr: fp32 [H] (4-byte
 * aligned); d_ws: hqmq_outlier_extract_given_thr_workspace_size bytes,
 * 256-byte aligned, contents on entry ignored. */
HQMQ_API uint64_t hqmq_outlier_extract_given_thr_workspace_size(int B, int H, int T, int D);
HQMQ_API int hqmq_outlier_extract_given_thr(const void *d_x, int dtype, int B, int H, int T, int D,
                                            const float *d_thr, int gran, uint32_t *d_out_idx,
                                            uint16_t *d_out_val, uint32_t *d_slab_off,
                                            uint32_t *d_tile_off, uint64_t cap, void *d_ws,
                                            uint64_t ws_bytes, hqmq_status *d_status,
                                            void *stream);

/* n_calls small calls at once (e.g. one decode step's new tokens of every
 * (layer, role)), one launch: for each call c the outputs equal
 * hqmq_outlier_extract_given_thr(x_c, thr_c) followed by
 * hqmq_encode(x_c, codebook_c, S, thr_c, gran), bit for bit (list, slab and
 * tile offsets, index words, radii, status counts).  Every array is the
 * calls' arrays back to back:
 *   d_x [n_calls][B][H][T][D] (bf16 or fp32, 16-byte aligned), d_thr
 *   [n_calls][H], d_codebook [n_calls][H][S][4] (16-byte aligned; H*S*16
 *   <= 160 KB), d_idx_words [n_calls][hqmq_index_words(B,H,T,D,S)],
 *   d_radius [n_calls][B*H*T*D/4], d_out_idx [n_calls][cap], d_out_val
 *   [n_calls][cap*4] (chunk) or [n_calls][cap] (element), 8-byte aligned,
 *   d_slab_off [n_calls][B*H+1], d_tile_off (NULL or) [n_calls]
 *   [hqmq_list_tiles(B,H,T,D)+1]; cap < 2^32 entries per call.
 * One CTA per call: meant for small calls, where per-launch costs dominate. */
HQMQ_API int hqmq_append_batch(const void *d_x, int dtype, int n_calls, int B, int H, int T, int D,
                               const float *d_thr, int gran, const float *d_codebook, uint32_t S,
                               uint32_t *d_idx_words, uint16_t *d_radius, uint32_t *d_out_idx,
                               uint16_t *d_out_val, uint32_t *d_slab_off, uint32_t *d_tile_off,
                               uint64_t cap, hqmq_status *d_status, void *stream);

/* Quantized radius (our reading of the pages' bit budget: the abstract's 3.79
 * bits per element at S = 8 is log2(24 S) / 2, i.e. about 2 log2(24 S) bits
 * per chunk, a radius code with as many levels as there are codewords).
 * With Med3x every bulk chunk has r <= thr_h (gist.science/nl, Technische
 * Samenvatting, section 3), so the fp16 radius is quantized uniformly on
 * [0, thr_h] into L = 24 S levels:
 *   inv_h = fl32((L-1) / thr_h),  k = min(L-1, floor(fl32(fl32(r inv_h) + 0.5)))
 * (k = 0 for a NaN radius and for every chunk of a head whose thr is not a
 * positive finite value).  The codes are packed like the indices: b =
 * ceil(log2(24 S)) bits per chunk, b uint32 words per 32 chunks, LSB first;
 * index + radius code = 2b bits per chunk (4.0 bits per element at S = 8,
 * 5.0 at S = 32), plus the outlier list.
 * d_radius: fp16 bits [B*H*T*D/4] as written by the encode calls (2-byte
 * aligned); d_thr: fp32 [H], the top of each head's radius range: the Med3x
 * thr in chunk mode (hqmq_outlier_extract / hqmq_encode_med3), 2 thr in
 * element mode (a chunk whose 4 elements are all <= thr has r <= 2 thr);
 * d_rcode_words: uint32[hqmq_index_words(B,H,T,D,S)], fully overwritten. */
HQMQ_API int hqmq_quantize_radius(const uint16_t *d_radius, const float *d_thr, int B, int H,
                                  int T, int D, uint32_t S, uint32_t *d_rcode_words,
                                  void *stream);

/* hqmq_decode with each chunk's radius taken from its code:
 * r = fl32(k fl32(thr_h / (L-1))) (codes >= L read as L-1; d_thr the same
 * ranges as given to hqmq_quantize_radius).  Everything else
 * as hqmq_decode; a list needs its d_tile_off (applied in the main pass). */
HQMQ_API int hqmq_decode_qradius(const uint32_t *d_idx_words, const uint32_t *d_rcode_words,
                                 const float *d_thr, const float *d_codebook, uint32_t S,
                                 const uint32_t *d_out_idx, const uint16_t *d_out_val,
                                 const uint32_t *d_tile_off, uint64_t cap, int gran, int B, int H,
                                 int T, int D, void *d_y, int out_dtype, hqmq_status *d_status,
                                 void *stream);

/* Joint (index, radius level) code: the pages' bit budget (signal-ia-rouge,
 * "La mecanique": 3.79 bits per element at S = 8, about 5 at S = 32, i.e. two
 * digits of L = 24 S values per chunk of four elements).  Each chunk's pair
 * is one digit D = idx * L + k in base L^2 (k its radius level, as written by
 * hqmq_quantize_radius); n consecutive chunks of a slab form one block value
 * V = sum_c D_c (L^2)^c (least significant chunk first), n the largest count
 * with L^(2n) < 2^64, stored in w = bit length of L^(2n) - 1 bits.  Every
 * slab's blocks (its last one padded with zero digits) are packed LSB-first
 * into its own run of uint32 words.  S = 8: n = 4, w = 61 (3.8125 bits per
 * element); S = 32: n = 3, w = 58 (4.833).  Valid for S in [1, 2730]
 * (L^2 < 2^32); other S give 0 / HQMQ_ERR_ARG.  No counterpart format is
 * given on the pages: the block code is this library's. */
HQMQ_API void hqmq_joint_block(uint32_t S, uint32_t *chunks_per_block, uint32_t *bits_per_block);
/* uint32 words of a call's joint code (B*H runs); 0 for a bad shape or S. */
HQMQ_API uint64_t hqmq_joint_words(int B, int H, int T, int D, uint32_t S);
/* Joint code of a call from its index words and radius-code words (both
 * uint32[hqmq_index_words(B,H,T,D,S)], 4-byte aligned).  d_joint:
 * uint32[hqmq_joint_words(...)], fully overwritten.  A chunk whose index or
 * level is not below L is stored as digit 0 and raises HQMQ_FLAG_BAD_INDEX
 * in d_status (optional). */
HQMQ_API int hqmq_pack_joint(const uint32_t *d_idx_words, const uint32_t *d_rcode_words,
                             uint32_t S, int B, int H, int T, int D, uint32_t *d_joint,
                             hqmq_status *d_status, void *stream);
/* The pages' 1-bit outlier flag (gist.science/nl, Technische Samenvatting,
 * section 3): d_flags uint32[B*H*T*D/128], bit c of word g set when chunk
 * 32 g + c is in the chunk-mode outlier list (d_out_idx, its first
 * min(d_slab_off[B*H], cap) entries).  With the list's values (d_out_val, in
 * list order) and tile offsets, the flags replace the list's 32-bit indices:
 * a flagged chunk's values are the q-th of its 1024-chunk list tile, q its
 * rank among the tile's flags.  d_flags is fully overwritten. */
HQMQ_API int hqmq_list_flags(const uint32_t *d_out_idx, const uint32_t *d_slab_off, uint64_t cap,
                             int B, int H, int T, int D, uint32_t *d_flags, void *stream);
/* Decode from the joint code: r = fl32(k fl32(thr_h / (L-1))) times the
 * codeword of idx, rounded to out_dtype, exactly as hqmq_decode_qradius;
 * then, if d_flags is given, every flagged chunk becomes its fp16 values
 * (d_out_val in list order, d_tile_off the list's tile offsets, entries at
 * or past cap skipped).  d_y 8-byte (bf16) or 16-byte (fp32) aligned. */
HQMQ_API int hqmq_decode_joint(const uint32_t *d_joint, const float *d_thr,
                               const float *d_codebook, uint32_t S, const uint32_t *d_flags,
                               const uint16_t *d_out_val, const uint32_t *d_tile_off, uint64_t cap,
                               int B, int H, int T, int D, void *d_y, int out_dtype, void *stream);

/* One coded K or V cache for hqmq_attention_decode: HOST struct of DEVICE
 * pointers, each as written by hqmq_encode / hqmq_encode_med3 for a
 * [B][Hk][T][128] tensor (idx_words, radius 16-byte aligned; codebook fp32
 * [Hk][S][4], 16-byte aligned).  out_idx == NULL: no outlier list; else
 * out_val (8-byte aligned), tile_off (uint32 [hqmq_list_tiles(B,Hk,T,128) +
 * 1]) and cap are the list, its tile offsets and the cap of that call, gran
 * its granularity.  In chunk mode a listed chunk's code must have radius 0
 * (radius code 0), as every encoder of this library writes an outlier; the
 * list values then stand for the whole chunk.  Quantized radius: rcode_words (as hqmq_quantize_radius
 * writes them) and thr (fp32 [Hk], their range) replace radius, which may then
 * be NULL; K and V must then both be given this way. */
typedef struct {
    const uint32_t *idx_words;
    const uint16_t *radius;
    const float *codebook;
    const uint32_t *out_idx;
    const uint16_t *out_val;
    const uint32_t *tile_off;
    uint64_t cap;
    int gran;
    const uint32_t *rcode_words;
    const float *thr;
} hqmq_kv_codes;

/* Bytes of device workspace hqmq_attention_decode needs for B x Hk KV heads
 * (per-head counters plus room for 1024 partial results of 8 x 130 floats;
 * about 4.3 MB). */
HQMQ_API uint64_t hqmq_attention_workspace_size(int B, int Hk);

/* Decode-phase attention read straight from the codes: the decoder runs
 * inside the attention loop (gist.science/nl, Technische Samenvatting,
 * "Memory en Latentie"), so the dense K and V are never written.
 * For each batch b, query head h (GQA: KV head hk = h / G, G = Hq / Hk, so
 * query heads hk*G .. hk*G + G - 1 share KV head hk):
 *   K^, V^ = exactly what hqmq_decode (or, with radius codes,
 *            hqmq_decode_qradius) writes as bf16 for the two caches
 *            (codes, radius and outlier list);
 *   s_t    = scale * <q[b][h], K^[b][hk][t]>, for t < len_b;
 *   o[b][h] = sum_t softmax(s)_t V^[b][hk][t],
 * with len_b = d_seq_len[b] clamped to [0, T] (NULL: len_b = T; len_b = 0
 * gives o = 0).  Computation: per 16-token block the codes are decoded in
 * registers straight into tensor-core operands; q K^T with bf16 products
 * accumulated in fp32; softmax in base 2 with a running maximum; the
 * weights enter P V as two bf16 terms (about 16 significant bits) with fp32
 * accumulation; the token range of a KV head is split over CTAs whose
 * partial (max, sum, P V) are merged by the last of them.  An index >= 24 S
 * reads as the zero codeword (r * 0); unlike hqmq_decode, this call records
 * nothing in d_status (which may be NULL).
 * d_q: bf16 [B][Hq][128], 8-byte aligned.  d_o: [B][Hq][128] of out_dtype
 * (HQMQ_BF16 or HQMQ_F32), 4-byte aligned.  d_seq_len: int32 [B] or NULL.
 * D must be 128 and G <= 8; S in [1, 65535]; scale finite.  d_ws: at least
 * hqmq_attention_workspace_size(B, Hk) bytes, 256-byte aligned, contents on
 * entry ignored (the call clears what it needs). */
HQMQ_API int hqmq_attention_decode(const uint16_t *d_q, const int32_t *d_seq_len,
                                   const hqmq_kv_codes *k, const hqmq_kv_codes *v, uint32_t S,
                                   int B, int Hq, int Hk, int T, int D, float scale, void *d_o,
                                   int out_dtype, void *d_ws, uint64_t ws_bytes,
                                   hqmq_status *d_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HQMQ_H */
