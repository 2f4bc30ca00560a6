/*
 * ecco.h -- C ABI of libecco_b200.so, a B200 (sm_100a) implementation of the
 * Ecco 512-bit block codec for LLM weight and KV-cache tensors.
 *
 * Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
 * Entropy-aware Cache Compression" (arXiv 2505.06901; pith.science review page).
 * Every 128-value bf16 group becomes one self-contained 64-byte block holding a
 * per-group FP8 scale, a pattern index (one of 64 shared 15-centroid k-means
 * patterns, chosen by min/max), a codebook choice (the shortest of 4 Huffman
 * codebooks), the Huffman-coded centroid indices, and padded outliers
 * (review page: "What carries the argument", "Core claim", Fig. 4 caption,
 * free-parameter list).
 *
 * Block layout (the page gives the fields, not their bit positions; these are
 * the library's readings):
 *   stream bit b = bit (b % 8) of byte b / 8 (little-endian 32-bit words);
 *   bits 0-7   FP8 E4M3 scale code (signed; codes 0x00/0x80/0x7f/0xff decode
 *              to a block of 128 zeros);
 *   bits 8-13  pattern index p (0..63);
 *   bits 14-15 codebook index h (0..3);
 *   bits 16-   canonical Huffman codewords of the 128 symbols in element order,
 *              each written most-significant code bit first (lengths 1..8).
 *              Symbol 15 is the scale element (value = s).  A codeword that
 *              does not fit below bit 512 is cut there and ends the stream
 *              ("clip the excess"); elements from it on decode to +0.
 *   unclipped blocks with L payload bits then carry n = min(16, (496-L)/15)
 *   outlier records of 15 bits: element index (7 bits) then q (8-bit two's
 *   complement), decoded as bf16(s * (q / 127)) over the centroid value.
 * Decoded value of element i: bf16 round-half-even of fp32(s * C[p][sym_i]).
 *
 * Conventions for every call:
 *   - Data pointers are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or retains them.  Table objects are library-owned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous: they validate, enqueue kernels and return.
 *   - The calling thread's current device must be the device the tables were
 *     created on.
 *   - Return value: ECCO_OK or a negative ECCO_ERR_* code.  On an argument
 *     error nothing is enqueued.  Data-dependent conditions (non-finite input,
 *     clipping) are never errors; they are counted in ecco_stats.
 */
#ifndef ECCO_H
#define ECCO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ECCO_OK 0
#define ECCO_ERR_ARG (-1)         /* null/negative/inconsistent argument */
#define ECCO_ERR_ALIGN (-2)       /* pointer not aligned as the call requires */
#define ECCO_ERR_TABLES (-3)      /* table blob invalid */
#define ECCO_ERR_CUDA (-4)        /* CUDA runtime error (launch, copy, device) */
#define ECCO_ERR_DEVICE (-5)      /* current device is not the tables' device */
#define ECCO_ERR_UNSUPPORTED (-6) /* device is not sm_100 */

#define ECCO_GROUP 128            /* values per group */
#define ECCO_BLOCK_BYTES 64       /* bytes per compressed block (512 bits) */
#define ECCO_NPAT 64              /* shared k-means patterns per tensor */
#define ECCO_NCENT 15             /* sorted centroids per pattern */
#define ECCO_NBOOK 4              /* Huffman codebooks per pattern */
#define ECCO_NSYM 16              /* symbols: 15 centroids + the scale element */
#define ECCO_LMAX 8               /* longest codeword, bits */
#define ECCO_TABLES_MAGIC 0x31434345u
#define ECCO_TABLES_BYTES 7952u

/* Table blob (host memory, little-endian), the per-tensor parameters learned
 * offline ("64 patterns per tensor", "4 Huffman codebooks per pattern"):
 *   u32 magic = ECCO_TABLES_MAGIC, u32 version = 1, f32 S_t, u32 reserved,
 *   f32 C[64][15]      centroids, strictly increasing per pattern, |C| <= 4,
 *   u8  len[64][4][16] code lengths 1..8, Kraft sum exactly 1 per codebook.
 * S_t is the per-tensor FP8 scale factor (Fig. 4 caption), normal, in
 * [2^-60, 2^60]. */
typedef struct ecco_tables ecco_tables;

/* A 2-D array of groups.  Group (r, g), 0 <= r < rows, 0 <= g < groups_per_row,
 * is read at source group index  src_offset + r * src_row_stride + g  and
 * written at destination index   dst_offset + r * dst_row_stride + g.
 * A group index addresses 128 bf16 values (256 bytes) on the bf16 side and one
 * 64-byte block on the compressed side.  A flat tensor is rows = 1.  Writing
 * the last T tokens of a [B, H, S, 128] KV cache from a [B, H, T, 128] tensor:
 * rows = B*H, groups_per_row = T, src_row_stride = T, dst_row_stride = S,
 * src_offset = 0, dst_offset = S - T.  All fields >= 0; when rows > 1,
 * dst_row_stride >= groups_per_row (destination rows may not overlap);
 * rows * groups_per_row <= 2^31 - 2048 (512 GiB of bf16 per tensor and call:
 * the kernels index a tensor's groups with 32-bit integers); other entries
 * return ECCO_ERR_ARG. */
typedef struct {
    int64_t rows;
    int64_t groups_per_row;
    int64_t src_row_stride;
    int64_t dst_row_stride;
    int64_t src_offset;
    int64_t dst_offset;
} ecco_desc;

/* Per-call counters, accumulated (atomically added) into a caller-owned device
 * struct that the caller zeroes.  n_padded counts unclipped blocks with at
 * least one outlier record; payload_bits sums min(L, 496) over non-zero blocks
 * (clip and padding ratios as in the review page's Fig. 10). */
typedef struct {
    unsigned long long n_groups;
    unsigned long long n_zero;
    unsigned long long n_clipped;
    unsigned long long n_padded;
    unsigned long long n_records;
    unsigned long long n_nonfinite;
    unsigned long long payload_bits;
    unsigned long long reserved;
} ecco_stats;

/* Validates `blob` (nbytes == ECCO_TABLES_BYTES), derives the device-side
 * tables (thresholds, canonical codes, decode lookup tables) and uploads them
 * to the current device.  Blocking; not for the hot path.  On success *out
 * owns device memory until ecco_tables_destroy. */
int ecco_tables_create(const void* blob, size_t nbytes, ecco_tables** out);
int ecco_tables_destroy(ecco_tables* tables);

/* Encoder ("Core claim"; "What carries the argument"): for every group of
 * `x_bf16` described by `desc`, picks the FP8 scale, the pattern by min/max
 * squared error, the symbols, the shortest codebook, packs and clips the
 * codewords and pads outliers, and writes one 64-byte block to `blocks`.
 * `dev_stats` may be NULL.  x_bf16 and blocks must be 16-byte aligned. */
int ecco_select_encode(const ecco_tables* tables, const uint16_t* x_bf16, ecco_desc desc,
                       uint8_t* blocks, ecco_stats* dev_stats, void* stream);

/* Encoder variants for studying the pattern choice.  `select`:
 *   ECCO_SELECT_MINMAX  the method's min/max squared error (as ecco_select_encode);
 *   ECCO_SELECT_MSE     the full squared error of the normalised group: for each
 *                       pattern p, e_p = pairwise (binary-tree, element order)
 *                       fp32 sum of (u_i - C[p][sym_p(u_i)])^2, the scale
 *                       element adding 0; first p with the least e_p.  The
 *                       comparison the review page's referee report asks for
 *                       (major comment 2); about 6x the encoder's time.
 * `n_patterns` (1..64): only patterns 0..n_patterns-1 are searched (free
 * parameters: the compressor's 16 patterns, "reduced from 64"); tables for it
 * are learned with that many patterns.  Blocks decode with ecco_decode as
 * usual.  Other arguments as ecco_select_encode. */
#define ECCO_SELECT_MINMAX 0
#define ECCO_SELECT_MSE 1
int ecco_select_encode_ex(const ecco_tables* tables, const uint16_t* x_bf16, ecco_desc desc,
                          uint8_t* blocks, ecco_stats* dev_stats, int select, int n_patterns,
                          void* stream);

/* Activation format (free parameters: "Group size for activations = 64" and
 * the 2x compression target for activations; Fig. 9 text: the low compression
 * ratio compressor reuses the high-ratio compressor's components): every
 * 64-value bf16 group becomes one 64-byte block with the same header, symbols,
 * codebook choice, clipping and padding rules as above (records keep the
 * 15-bit layout with an index below 64; the decoder takes the 7-bit index
 * modulo 64).  Here a descriptor's group index addresses 64 bf16 values
 * (128 bytes) on the bf16 side.  Tables use the same blob layout, learned on
 * 64-value groups.  Alignment, errors and stats as ecco_select_encode /
 * ecco_decode. */
#define ECCO_GROUP_ACT 64
int ecco_select_encode_act(const ecco_tables* tables, const uint16_t* x_bf16, ecco_desc desc,
                           uint8_t* blocks, ecco_stats* dev_stats, void* stream);
int ecco_decode_act(const ecco_tables* tables, const uint8_t* blocks, ecco_desc desc, uint16_t* y_bf16,
                    void* stream);

/* Decoder (the review page's decompressor, Fig. 8 caption): every block of
 * `blocks` described by `desc` becomes 128 bf16 values in `y_bf16`.  Any
 * 64-byte pattern decodes deterministically (malformed blocks included).
 * blocks and y_bf16 must be 16-byte aligned; when both are 32-byte aligned the
 * decoder uses 32-byte loads and stores (faster; same output). */
int ecco_decode(const ecco_tables* tables, const uint8_t* blocks, ecco_desc desc,
                uint16_t* y_bf16, void* stream);

/* The same decoder organised as the review page's parallel decompressor
 * (Fig. 8 caption; referee major comment 1: sub-decoders start on
 * overlapping segments at every candidate bit offset and a tree merge picks
 * the true chain): one warp per block, each lane decodes at every bit
 * position of a 16-bit payload segment, the lanes' offset maps are composed
 * by a shuffle scan, and each lane emits the codewords of its segment.  The
 * output is bit-identical to ecco_decode's; arguments, alignment and errors
 * are ecco_decode's.  It does several times the work per block of the
 * one-thread-per-block walk and is slower on this hardware; it is offered
 * for comparison. */
int ecco_decode_speculative(const ecco_tables* tables, const uint8_t* blocks, ecco_desc desc,
                            uint16_t* y_bf16, void* stream);

/* Fused decode + matrix-vector product ("Normalized memory requests for a
 * GEMM kernel", review page figure list): y[b][r] = sum_k W~[r][k] x[b][k],
 * on CUDA cores for batch 1..4 and on the tcgen05 tensor cores for 5..16,
 * W~ the decoded rows x cols matrix whose blocks are stored row-major
 * (block (r, g) at index r * cols/128 + g), x_bf16 [batch][cols], y [batch][rows]
 * fp32.  cols % 128 == 0, 1 <= batch <= 16.  The decoded matrix is never
 * written to memory.  Accumulation order is unspecified (fp32). */
int ecco_decode_gemv(const ecco_tables* tables, const uint8_t* blocks, int64_t rows,
                     int64_t cols, const uint16_t* x_bf16, int batch, float* y, void* stream);

/* Many tensors in one launch: segment i decodes (or encodes) with its own
 * tables.  At most ECCO_MAX_SEGMENTS per call; arrays are host memory, read
 * before the call returns. */
#define ECCO_MAX_SEGMENTS 256
typedef struct {
    const ecco_tables* tables;
    const void* src; /* blocks (decode) / bf16 values (encode) */
    void* dst;       /* bf16 values (decode) / blocks (encode) */
    ecco_desc desc;
} ecco_segment;

int ecco_decode_multi(const ecco_segment* segments, int n_segments, void* stream);
int ecco_encode_multi(const ecco_segment* segments, int n_segments, ecco_stats* dev_stats,
                      void* stream);

/* Decode-phase attention read straight from a compressed KV cache (the
 * memory-bound decode phase at long sequence lengths where the review page
 * places Ecco's gains: "If this is right", Fig. 11 caption).  The K and V
 * blocks are decoded inside the attention kernel; the bf16 cache is never
 * materialised.  For batch b and query head j (KV head h = j / group):
 *   out[b][j][:] = sum_s p_s V~[b][h][s][:],
 *   p = softmax_s(scale * (q[b][j] . K~[b][h][s])),  0 <= s < seq_len,
 * with K~, V~ the values ecco_decode would produce.
 *   k_blocks, v_blocks  [batch][kv_heads][seq_capacity] blocks (64 B each; token s
 *                       of head h at index (b * kv_heads + h) * seq_capacity + s),
 *                       16-byte aligned; k_tables / v_tables decode them;
 *   q_bf16              [batch][kv_heads * group][128] bf16, 2-byte aligned;
 *   out                 [batch][kv_heads * group][128] fp32, 4-byte aligned;
 *   workspace           caller-owned device scratch of at least
 *                       ecco_decode_attention_workspace_bytes(...) bytes,
 *                       4-byte aligned; no initial contents are needed and it
 *                       holds per-split partial results afterwards.
 * 1 <= group <= 8, 1 <= seq_len <= seq_capacity, batch, kv_heads >= 1.
 * Two calls that share a workspace must be ordered (same stream).  Summation
 * order is unspecified (fp32 accumulation, fp32 exp). */
size_t ecco_decode_attention_workspace_bytes(int batch, int kv_heads, int group, int seq_len);
int ecco_decode_attention(const ecco_tables* k_tables, const ecco_tables* v_tables,
                          const uint8_t* k_blocks, const uint8_t* v_blocks, int64_t seq_capacity,
                          int batch, int kv_heads, int group, int seq_len, const uint16_t* q_bf16,
                          float scale, float* out, void* workspace, size_t workspace_bytes,
                          void* stream);

/* The same attention (same arguments, result and tolerance), computed in
 * stages: for each chunk of tokens the block decoder (ecco_decode_multi's
 * kernel) writes the chunk's decoded K and V rows to a scratch inside the
 * workspace, then a split kernel reads them back with coalesced copies.  A
 * chunk is a multiple of 512 tokens (whole 256-token splits), and its rows
 * (2 x batch x kv_heads x chunk x 256 B) stay within 1 GiB, so most caches
 * run as one chunk.  The
 * decoded rows cross HBM once each way; in exchange the decode runs at the
 * standalone decoder's occupancy, which the single fused kernel cannot reach
 * (its tables, stream words and tiles leave it half the resident warps).  The
 * review page's point that compression speeds up the decode-phase reads of
 * the cache ("If this is right", Fig. 11 caption) holds for both: the
 * compressed blocks are what is read from the cache.
 *   workspace  at least ecco_decode_attention_staged_workspace_bytes(...)
 *              bytes, 4-byte aligned, caller-owned; it holds the per-split
 *              partial results and the chunk scratch (no initial contents).
 * Errors and the other arguments as for ecco_decode_attention. */
size_t ecco_decode_attention_staged_workspace_bytes(int batch, int kv_heads, int group, int seq_len);
int ecco_decode_attention_staged(const ecco_tables* k_tables, const ecco_tables* v_tables,
                                 const uint8_t* k_blocks, const uint8_t* v_blocks, int64_t seq_capacity,
                                 int batch, int kv_heads, int group, int seq_len, const uint16_t* q_bf16,
                                 float scale, float* out, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ecco_decode_attention with its workspace in static device memory: a
 * file-scope __device__ array of ECCO_ATTENTION_STATIC_WS_BYTES per device
 * inside the library, so the call allocates nothing and takes no workspace
 * argument.  The pages have no counterpart to this entry point; it exists for
 * callers that cannot allocate device memory where they run attention: a
 * plain-C host loop has no caching allocator to draw a workspace from, and
 * cudaMalloc can synchronize the device and fail under memory pressure.
 *   - The arguments are checked first, in ecco_decode_attention's order and
 *     with its error codes (tables, sizes, pointers, alignment).  A valid
 *     request whose workspace (ecco_decode_attention_workspace_bytes) exceeds
 *     ECCO_ATTENTION_STATIC_WS_BYTES then returns ECCO_ERR_WORKSPACE; either
 *     way nothing is enqueued.
 *   - Nothing in the workspace needs to start at zero: every split writes all
 *     of its partial results before the merge reads them.
 *   - The first call on each device looks up the workspace's address with that
 *     device current (cudaGetSymbolAddress); make that first call before any
 *     stream capture.
 *   - All calls on one device share the workspace: calls that can overlap (on
 *     different streams, or from several host threads without ordering) race
 *     on it and corrupt each other's results.  Order them on one stream. */
#define ECCO_ATTENTION_STATIC_WS_BYTES (4u << 20)
#define ECCO_ERR_WORKSPACE (-7) /* request needs more than the static workspace */
int ecco_decode_attention_static(const ecco_tables* k_tables, const ecco_tables* v_tables,
                                 const uint8_t* k_blocks, const uint8_t* v_blocks, int64_t seq_capacity,
                                 int batch, int kv_heads, int group, int seq_len, const uint16_t* q_bf16,
                                 float scale, float* out, void* stream);

/* Table learner on the GPU (offline; blocking; allocates and frees its own
 * temporaries; not for the hot path).  Learns one tensor's table blob -- the
 * per-tensor parameters the review page says are learned once, offline ("What
 * carries the argument"; free parameters S = 64, H = 4, 15 centroids; referee
 * comment 1: lengths <= 8) -- from `n_groups` groups of `group` (128, or 64
 * for the activation format) bf16 values at `sample_bf16` (device, 16-byte
 * aligned):
 *   S_t = absmax / 448; each of up to 16,384 sampled groups (seeded sample) is
 *   scaled by its FP8 group scale, its largest element set aside and the rest,
 *   sorted, summarised by 15 equal-count bin means; k-means++ / Lloyd (20
 *   iterations) over those gives the patterns; 4 rounds move every centroid to
 *   the mean of the values the encoder's own rules (min/max pattern,
 *   thresholds) give it; per pattern, 4 codebooks from clustered symbol
 *   histograms, each an optimal prefix code with lengths <= 8 (package-merge).
 * `n_patterns` < 64 learns that many (rows past it repeat row 0; encode with
 * ecco_select_encode_ex and the same count).  The blob (ECCO_TABLES_BYTES,
 * host memory) is the same for the same sample and seed. */
int ecco_learn_tables(const uint16_t* sample_bf16, int64_t n_groups, int group, int n_patterns,
                      uint64_t seed, void* blob_out, size_t blob_bytes, void* stream);

/* Optimal prefix-code lengths for n symbols of the given (positive) weights,
 * every length <= max_len (package-merge; ties in symbol order).  Host only,
 * no device needed.  Returns ECCO_ERR_ARG if n < 1, max_len < 1 or
 * n > 2^max_len. */
int ecco_huffman_lengths(const double* weights, int n, int max_len, uint8_t* lengths_out);

/* Number of bounded device-side waits (tensor-core decode+GEMV pipeline) that
 * gave up since the library was loaded on the current device; 0 in normal
 * operation.  A CTA whose wait gives up stops issuing tensor-core work, adds
 * nothing to y and returns instead of hanging, so that launch's y is
 * incomplete.  Because launches are asynchronous, the failure is reported
 * like CUDA's own asynchronous errors: it raises a host-visible flag, and
 * every later ecco_decode_gemv call with batch > 4 returns ECCO_ERR_TIMEOUT
 * (enqueuing nothing) until this function is called, which reads the count
 * and clears the flag.  Blocking (reads device memory). */
#define ECCO_ERR_TIMEOUT (-8) /* a bounded device wait gave up in an earlier launch */
int ecco_device_timeouts(unsigned int* out);

/* Diagnostic for the timeout path above, with no fault and no hang: launches
 * one kernel that waits, with the pipeline's bounded wait (well under a
 * second), on an mbarrier that nothing completes, so the wait gives up,
 * counts itself and raises the flag.  Asynchronous on `stream`. */
int ecco_selftest_wait_timeout(void* stream);

const char* ecco_strerror(int code);
int ecco_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ECCO_H */
