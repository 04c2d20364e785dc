/*
 * csa2.h -- C ABI of libcsa2: CSA2 sparse attention over an FP4 main-KV
 * cache, hand-written for NVIDIA B200 (sm_100a).
 *
 * The four calls follow the method's statement on the pages:
 *
 *   "DeepSeek V4.1-Flash 技术报告深度解析：CED 架构与 KV Cache 极限压缩"
 *   (eogee.com/article/126)
 *     §3.2  CSA2 Full / Reindex / Reuse modes, 32 x 128 indexer, top-512,
 *           64 heads x 512 attention, SWA window 128
 *     §3.3  Hierarchical Sparse Indexer: 2048 blocks of 8 positions
 *     §3.4  FP4 main KV: E2M1 values, one E4M3 scale per 16 channels,
 *           quantised after RoPE, dequantised before attention
 *   "DeepSeek-V4.1-Flash" README walk-through (m.nxbn.cn/news/186820)
 *     §3.1 / §3.3 configuration tables (head sizes, candidate pool sizes)
 *
 * Conventions for every call
 *   - All data pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or keeps them.  Structs are read on the host
 *     during the call only.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Every call is asynchronous on that stream: it validates its
 *     arguments on the host, enqueues kernels and returns.
 *   - Multi-dimensional arrays are dense and row-major in the order written,
 *     e.g. [B][Q][32][128] means element (b,q,h,d) sits at
 *     ((b*Q + q)*32 + h)*128 + d.
 *   - bf16 means IEEE bfloat16, f32 IEEE binary32; inputs must be finite.
 *   - Every pointer must be 16-byte aligned (CSA2_ERR_ALIGN otherwise).
 *   - Host-side validation failure returns before anything is enqueued and
 *     leaves every output untouched.  CSA2_ERR_CUDA reports a launch error;
 *     kernels enqueued before it by the same call may have run.
 *   - Workspace: calls that need scratch take (ws, ws_bytes); the size comes
 *     from csa2_workspace_size().  Its contents on entry do not matter (the
 *     call clears the part it needs with an asynchronous memset on
 *     `stream`).  Calls that share a workspace must not overlap in time.
 *   - Batch rows are independent sequences with their own caches.
 */
#ifndef CSA2_ABI_H_
#define CSA2_ABI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Sizes fixed by the method ([eogee] §3.2, [nxbn] §3.1/§3.3). */
#define CSA2_D            512   /* main-KV entry width = attention head dim   */
#define CSA2_ENTRY_BYTES  288   /* packed FP4 entry: 256 B nibbles + 32 B E4M3 scales */
#define CSA2_SCALE_BLOCK  16    /* channels per E4M3 scale                    */
#define CSA2_H            64    /* attention query heads (one KV head)        */
#define CSA2_HI           32    /* indexer heads                              */
#define CSA2_DI           128   /* indexer head dim                           */
#define CSA2_TOPK         512   /* the method's top-K                         */
#define CSA2_WIN          128   /* the method's SWA window                    */
#define CSA2_HSI_BLOCK    8     /* positions per HSI block                    */
#define CSA2_HSI_BLOCKS   2048  /* HSI blocks kept                            */

/* Limits of this implementation. */
#define CSA2_MAX_BQ       65535 /* batch rows x query positions per call      */
#define CSA2_MAX_K        2048  /* largest top-K (and largest pool, in blocks) */
#define CSA2_MAX_W        1024  /* largest window (rows per query)            */

typedef enum csa2_status {
    CSA2_OK            = 0,
    CSA2_ERR_ARG       = 1,  /* NULL where a pointer is required, bad mode   */
    CSA2_ERR_SHAPE     = 2,  /* a size outside the supported range           */
    CSA2_ERR_ALIGN     = 3,  /* a pointer or stride breaks 16-byte alignment */
    CSA2_ERR_WORKSPACE = 4,  /* workspace NULL or smaller than required      */
    CSA2_ERR_CUDA      = 5,  /* a CUDA runtime or launch error               */
    CSA2_ERR_DEVICE    = 6,  /* a kernel recorded a device-side failure      */
    CSA2_ERR_ARCH      = 7   /* current device is not sm_100                 */
} csa2_status;

/* Storage formats of the window rows (attention) and of index-K. */
#define CSA2_FMT_BF16     0     /* bf16 values                                  */
#define CSA2_FMT_FP8      1     /* window rows: E4M3 codes + one f32 scale per row ([eogee] §3.4) */
#define CSA2_FMT_MXFP4    2     /* index-K: 68-byte OCP MXFP4 entries ([eogee] §3.4) */
#define CSA2_FMT_NVFP4    3     /* attention Q: quantised by the main-KV FP4 rule    */
#define CSA2_INDEX_K_MXFP4_BYTES 68   /* 64 B of E2M1 nibbles + 4 E8M0 scales        */

/* Static layer modes, [eogee] §3.2 and §3.3. */
typedef enum csa2_mode {
    CSA2_FULL         = 0,  /* score every visible entry                       */
    CSA2_REINDEX      = 1,  /* re-score the shared index-K with own index-Q    */
    CSA2_REINDEX_POOL = 2,  /* re-score only the HSI candidate pool            */
    CSA2_REUSE        = 3   /* no scoring: reuse the previous layer's top-K    */
} csa2_mode;

/* ------------------------------------------------------------------------
 * csa2_quantize_kv_fp4 -- [eogee] §3.4 FP4 main-KV cache.
 *
 * Quantises n main-KV entries (512 channels, already RoPE-rotated) to the
 * 288-byte FP4 layout: for each block of 16 channels
 *     sf = fp32(amax / 6);  s = E4M3(sf)  (round to nearest even, saturate 448)
 *     q_i = E2M1(fp32(x_i / s))           (round to nearest even, saturate 6;
 *                                          sign kept; s == 0 gives signed 0)
 * Entry layout: byte i (0..255) holds channel 2i in its low nibble and
 * channel 2i+1 in its high nibble; byte 256+k holds the scale of channels
 * 16k..16k+15.  Dequantised value = E2M1(q) * E4M3(s), exact in bf16.
 *
 *   x         bf16 [n][ld_x], entry i in x[i*ld_x .. i*ld_x+511]; ld_x >= 512
 *             and a multiple of 8
 *   n         entries, >= 0 (0 enqueues nothing)
 *   kv_fp4    u8 cache rows of CSA2_ENTRY_BYTES bytes
 *   dst_rows  optional int64 [n]: entry i goes to row dst_rows[i];
 *             NULL means row row_offset + i
 *   row_offset  first destination row when dst_rows is NULL, >= 0
 * Entries map to distinct rows (overlapping destinations race).  The call
 * does not know the cache's size: every destination row must lie inside
 * kv_fp4 (the caller's contract; nothing checks it).
 * Errors: ARG (x or kv_fp4 NULL with n > 0), SHAPE (n < 0, ld_x < 512,
 * row_offset < 0), ALIGN, CUDA.
 * ---------------------------------------------------------------------- */
csa2_status csa2_quantize_kv_fp4(const void* x, int64_t n, int64_t ld_x,
                                 void* kv_fp4, const int64_t* dst_rows,
                                 int64_t row_offset, void* stream);

/* ------------------------------------------------------------------------
 * csa2_compress_rope_quantize_kv_fp4 -- new main-KV entries made, rotated
 * and quantised in one pass.  [eogee] §3.2: CSA2 compresses every r tokens
 * into one entry (r = 2 in the encoder, 1 in the decoder), with no overlap
 * between neighbouring entries and no absolute position encoding in the
 * compression; §3.4: the entry is quantised after RoPE.  The pages give
 * neither the compressor's form nor the rotation layout; this call takes:
 *     entry e = sum_{j<r} w[e][j] (.) x[e*r + j]         (channel by channel)
 *     channels 448 + 2i, 449 + 2i (i < 32, the 64-dim RoPE slice) rotated:
 *         (a, b) -> (a cos[e][i] - b sin[e][i], a sin[e][i] + b cos[e][i])
 *     then the FP4 quantiser of csa2_quantize_kv_fp4 on the result.
 * Every step is IEEE float32 with one rounding per operation, in the order
 * written (no fused multiply-add), with no bf16 rounding before the
 * quantiser; the angles (cos, sin) are the caller's, so the frequencies
 * (YaRN or other) are the model's choice.
 * ---------------------------------------------------------------------- */
typedef struct csa2_compress_args {
    const void*    x;           /* bf16 [n_entries * r][ld_x] token vectors      */
    int64_t        n_entries;   /* entries to make, >= 0                         */
    int64_t        ld_x;        /* >= 512, a multiple of 8                       */
    int32_t        r;           /* tokens per entry, 1..16                       */
    const float*   w;           /* f32 weights [.][r][512]                       */
    int64_t        w_stride;    /* floats between entries' weights: 0 (shared)
                                   or r * 512                                    */
    const float*   cos;         /* f32 [n_entries][32]                           */
    const float*   sin;         /* f32 [n_entries][32]                           */
    void*          kv_fp4;      /* u8 cache rows of CSA2_ENTRY_BYTES bytes       */
    const int64_t* dst_rows;    /* optional int64 [n_entries]: destination rows  */
    int64_t        row_offset;  /* first destination row when dst_rows is NULL   */
} csa2_compress_args;

csa2_status csa2_compress_rope_quantize_kv_fp4(const csa2_compress_args* a, void* stream);

/* ------------------------------------------------------------------------
 * csa2_quantize_window_fp8 -- [eogee] §3.4: the quantisation-sensitive SWA
 * KV cache stays in FP8.  The page names the precision only; this library's
 * format is one E4M3 code per channel and one f32 scale per 512-channel row:
 *     s = fp32(amax / 448)                (round to nearest even)
 *     code_i = E4M3(fp32(x_i / s))        (round to nearest even, saturate
 *                                          448; sign kept; s == 0 gives
 *                                          signed zeros)
 * Dequantised value = E4M3(code) * s; a row costs 516 B against 1024 B of bf16.
 *
 *   x         bf16 [n][ld_x] rows (ld_x >= 512, a multiple of 8)
 *   codes     u8 [rows][512] E4M3 codes
 *   scales    f32 [rows]
 *   dst_rows / row_offset  as in csa2_quantize_kv_fp4
 * Errors: ARG, SHAPE, ALIGN (codes 16-byte, scales 4-byte aligned), CUDA.
 * ---------------------------------------------------------------------- */
csa2_status csa2_quantize_window_fp8(const void* x, int64_t n, int64_t ld_x,
                                     void* codes, float* scales,
                                     const int64_t* dst_rows, int64_t row_offset,
                                     void* stream);

/* ------------------------------------------------------------------------
 * csa2_quantize_index_k_mxfp4 -- [eogee] §3.4: the indexer's Q/K were
 * already trained with FP4 quantisation, in the OCP MXFP4 family the page
 * names.  Index-K entries of 128 channels become 68 bytes, the size that
 * closes the pages' 890 B/token accounting ([ainewsway] "KV 快取為何成為
 * 瓶頸": 3 encoder caches at r=2 and one decoder cache, 288 B main-KV and
 * 68 B index-K entries): per block of 32 channels
 *     e = floor(log2(amax)) - 2   (clamped to [-127, 127]; -127 for a zero block)
 *     q_i = E2M1(x_i / 2^e)       (round to nearest even, saturate 6, sign kept)
 * Entry: byte i (0..63) holds channel 2i in its low nibble and 2i+1 in its
 * high nibble; byte 64+k holds e + 127 for channels 32k..32k+31.
 * Dequantised value E2M1(q) * 2^e, exact in bf16.
 *
 *   x       bf16 [n][ld_x] (ld_x >= 128, a multiple of 4; 8-byte aligned)
 *   out     u8 entries of 68 bytes (4-byte aligned)
 *   dst_rows / row_offset  as in csa2_quantize_kv_fp4
 * Errors: ARG, SHAPE, ALIGN, CUDA.
 * ---------------------------------------------------------------------- */
csa2_status csa2_quantize_index_k_mxfp4(const void* x, int64_t n, int64_t ld_x,
                                        void* out, const int64_t* dst_rows,
                                        int64_t row_offset, void* stream);

/* ------------------------------------------------------------------------
 * csa2_index_score_topk -- [eogee] §3.2 lightweight indexer + top-K,
 * §3.3 Hierarchical Sparse Indexer.
 *
 * Score of query (b,q) for entry t (t < n_vis[b][q]):
 *     s = sum_h w[b][q][h] * ReLU( sum_d qI[b][q][h][d] * kI[b][t][d] )
 * bf16 products accumulated in fp32 on the tensor cores.  The K best
 * entries by (higher score, then lower position) are written in ascending
 * position order, then padded with -1 when fewer than K entries are
 * visible; `scores` (optional) holds the score of each written entry.
 *
 * mode CSA2_FULL / CSA2_REINDEX: scan t in [0, n_vis).  With hsi_blocks > 0
 *   (FULL only) the call also builds the HSI pool: block score = max of the
 *   visible scores in positions [8j, 8j+8), the hsi_blocks best blocks (ties
 *   to the lower block id) are written to pool_out in ascending block order,
 *   padded with -1.
 * mode CSA2_REINDEX_POOL: scan only the positions of pool_in (hsi_blocks
 *   block ids per query, ascending, -1 padding ignored); positions at or
 *   beyond n_vis do not score.  The selected entries come out in pool order
 *   (ascending positions for an ascending pool).
 *
 * k_format CSA2_FMT_MXFP4: kI holds 68-byte MXFP4 entries [B][N][68]
 *   (csa2_quantize_index_k_mxfp4; N a multiple of 4, and of 8 when an HSI
 *   pool is built or re-scored, since a pool block is fetched whole;
 *   CSA2_ERR_SHAPE otherwise).  The page has the
 *   indexer's Q and K both in FP4, so index-Q (given in bf16) is quantised
 *   by the same rule inside the call (each head row of 128 dims, blocks of
 *   32: e = floor(log2 amax) - 2, q = E2M1(x / 2^e)) and the scores are
 *   those of the dequantised Q and K, computed on the block-scaled FP4
 *   tensor cores with fp32 accumulation.
 * ---------------------------------------------------------------------- */
typedef struct csa2_index_args {
    int32_t        mode;        /* CSA2_FULL, CSA2_REINDEX or CSA2_REINDEX_POOL  */
    int32_t        B;           /* batch rows, >= 1                              */
    int32_t        Q;           /* query positions per row, B*Q <= CSA2_MAX_BQ   */
    int32_t        K;           /* top-K, 1..CSA2_MAX_K                          */
    int64_t        N;           /* index-K rows per batch row, >= 1              */
    const void*    qI;          /* bf16 [B][Q][32][128]                          */
    const float*   w;           /* f32  [B][Q][32]                               */
    const void*    kI;          /* bf16 [B][N][128]                              */
    const int32_t* n_vis;       /* int32 [B][Q], each in [0, N]                  */
    int32_t*       idx;         /* out int32 [B][Q][K]                           */
    float*         scores;      /* optional out f32 [B][Q][K] (-inf padding)     */
    int32_t        hsi_blocks;  /* 0, or blocks in the pool (1..CSA2_MAX_K)      */
    int32_t        hsi_block;   /* positions per block (CSA2_HSI_BLOCK)          */
    int32_t*       pool_out;    /* FULL with hsi_blocks > 0: out int32 [B][Q][hsi_blocks] */
    const int32_t* pool_in;     /* REINDEX_POOL: in int32 [B][Q][hsi_blocks]     */
    int32_t        k_format;    /* CSA2_FMT_BF16 or CSA2_FMT_MXFP4               */
} csa2_index_args;

csa2_status csa2_index_score_topk(const csa2_index_args* a, void* ws,
                                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * csa2_index_score_topk_noalloc -- the same scoring and selection as
 * csa2_index_score_topk without a caller workspace.  (The pages have no
 * counterpart: this serves integrations, not the method.)
 *
 * For callers that cannot allocate device memory: code that is handed only
 * its input and output buffers by a host framework and has no allocator of
 * its own, or a serving process whose memory pool is fully reserved up front
 * so that a cudaMalloc would fail or stall the device.  The scratch is a
 * fixed device array of CSA2_NOALLOC_SCRATCH_BYTES inside the library; every
 * GPU that loads the library holds it until the process exits.  The call
 * allocates nothing: no cudaMalloc, no cudaFree.
 *
 * - The first call on each device looks up the array's device address with
 *   cudaGetSymbolAddress (with that device current); make that first call
 *   before any stream capture.  The address is kept per device and per CUDA
 *   context: after the device's context is destroyed and re-created (for
 *   example by cudaDeviceReset), the next call looks it up again, so that
 *   call too must come before any stream capture.
 * - A request whose scratch would exceed CSA2_NOALLOC_SCRATCH_BYTES
 *   (csa2_workspace_size(a, CSA2_WS_INDEX) tells the need) returns
 *   CSA2_ERR_WORKSPACE before anything is enqueued.
 * - All calls share the one array, which keeps the previous call's data;
 *   each call clears the part that must start at zero.  Calls that overlap
 *   on the GPU (different streams, different host threads) race on it and
 *   give wrong results: serialise them.
 * Arguments, outputs and the other errors are those of
 * csa2_index_score_topk.
 * ---------------------------------------------------------------------- */
#define CSA2_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
csa2_status csa2_index_score_topk_noalloc(const csa2_index_args* a, void* stream);

/* Size in bytes of the fixed scratch array behind
 * csa2_index_score_topk_noalloc, as compiled into the library (equals
 * CSA2_NOALLOC_SCRATCH_BYTES of the header it was built with). */
size_t csa2_noalloc_scratch_bytes(void);

/* ------------------------------------------------------------------------
 * csa2_sparse_attn -- [eogee] §3.2 sparse MQA: each query attends to its
 * selected FP4 entries plus the layer's SWA window; §3.4 dequantise before
 * the attention math.
 *
 * For query (b,q): keys = { dequant(kv_fp4[b][idx[b][q][j]]) : idx >= 0 }
 * followed by the window rows swa[b][q*swa_step + r], r in [0, W).  Each key
 * is also its value (one 512-dim vector per entry).  With logits
 * z_hj = scale * q[b][q][h] . key_j (scale <= 0 selects 1/sqrt(512)):
 *     out[b][q][h] = sum_j softmax_j(z_h)_j * key_j      (bf16, fp32 math)
 *     lse[b][q][h] = ln sum_j exp(z_hj)                  (optional)
 * A query with no key at all gets out = 0 and lse = -inf.
 *
 * idx entries must be -1 or in [0, N); the window rows read must lie inside
 * [0, swa_rows).  With swa_format CSA2_FMT_FP8 a window key is the
 * dequantised row E4M3(code) * s (csa2_quantize_window_fp8).
 *
 * q_format CSA2_FMT_NVFP4 (quantised Q; [eogee] §3.4 notes the model itself
 * avoids depending on native FP4 matmul): q holds u8 [B][Q][64][288], each
 * head row in the main-KV entry format (E2M1 values, one E4M3 scale per 16
 * channels; csa2_quantize_kv_fp4 writes it from bf16 rows), and the logits
 * of every key use the dequantised Q.  The selected-entry logits then run
 * on the block-scaled FP4 tensor cores straight from Q's and the cache's
 * codes and scales (split mode; with 128 or more queries Q is expanded to
 * bf16, exactly, and the bf16 path gives the same logits).
 *
 * With fewer than 128 queries per call (B*Q) the keys of a query are split
 * into 128-key slices over several CTAs: up to 8 slices (K + W <= 1024)
 * they form one thread-block cluster and merge their results through
 * distributed shared memory; with more, their fp32 partial outputs go to
 * the workspace and are merged by a second kernel.  With 128 or more
 * queries, one CTA per query walks all its slices.  Only the second-kernel
 * case uses the workspace (csa2_workspace_size still returns a small
 * non-zero size for the others).
 * ---------------------------------------------------------------------- */
typedef struct csa2_attn_args {
    int32_t        B, Q;        /* batch rows >= 1; queries per row, B*Q <= CSA2_MAX_BQ */
    int32_t        K;           /* idx slots per query, 0..CSA2_MAX_K            */
    int32_t        W;           /* window rows per query, 0..CSA2_MAX_W          */
    int64_t        N;           /* cache rows per batch row                      */
    const void*    q;           /* bf16 [B][Q][64][512] (q_format CSA2_FMT_NVFP4:
                                   u8 [B][Q][64][288] FP4 rows)                  */
    const void*    kv_fp4;      /* u8   [B][N][288]                              */
    const int32_t* idx;         /* int32 [B][Q][K]                               */
    const void*    swa;         /* bf16 [B][swa_rows][512]                       */
    int32_t        swa_rows;    /* rows per batch row in swa, >= (Q-1)*swa_step+W */
    int32_t        swa_step;    /* window of query q starts at row q*swa_step    */
    float          scale;       /* logit scale; <= 0 means 1/sqrt(512)           */
    void*          out;         /* out bf16 [B][Q][64][512]                      */
    float*         lse;         /* optional out f32 [B][Q][64]                   */
    int32_t        swa_format;  /* CSA2_FMT_BF16 (swa is bf16) or CSA2_FMT_FP8   */
    const float*   swa_scale;   /* CSA2_FMT_FP8: f32 [B][swa_rows]; swa is then
                                   u8 [B][swa_rows][512] E4M3 codes              */
    int32_t        q_format;    /* CSA2_FMT_BF16 or CSA2_FMT_NVFP4 (quantised Q)  */
} csa2_attn_args;

csa2_status csa2_sparse_attn(const csa2_attn_args* a, void* ws,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * csa2_group_decode -- one CSA2 sharing group ([eogee] §3.2, §3.3): the
 * layers share one FP4 main KV and one index-K and run strictly in order.
 *   1. if n_new > 0: quantise kv_new into kv_fp4 (csa2_quantize_kv_fp4 with
 *      dst_rows = new_rows, absolute rows of the [B*N] cache);
 *   2. for each layer: FULL / REINDEX / REINDEX_POOL score and select
 *      (csa2_index_score_topk; FULL builds the pool when hsi_blocks > 0 and
 *      REINDEX_POOL uses the pool of the most recent FULL layer, or pool_in
 *      before any such layer), REUSE takes the top-K of the most recent
 *      indexing layer; then sparse attention with the layer's own q and
 *      window (csa2_sparse_attn).
 *
 * pool_in carries the HSI pool across calls: [eogee] §3.3 has the pool built
 * once by the decoder's first Full layer serve every later Reindex layer,
 * and those sit in later groups (decoder groups 2..5 are Reindex + 3 Reuse,
 * [eogee] §3.2 configuration paragraph).
 *
 * flags (launch order between the call's kernels):
 *   0                        each layer's inputs (qI, w, q, window rows) are
 *                            treated as results of the layer before it, as
 *                            in the model, where a layer's queries come from
 *                            the previous layer's output: a kernel may start
 *                            its set-up and stream shared caches (index-K)
 *                            early, but reads a layer's inputs only after
 *                            the previous kernel has finished;
 *   CSA2_GROUP_INPUTS_READY  every layer's inputs are complete when the call
 *                            is made, so a kernel may load them early;
 *   CSA2_GROUP_SERIAL        kernels run in plain stream order (no kernel
 *                            starts before its predecessor has finished).
 * ---------------------------------------------------------------------- */
typedef struct csa2_layer {
    int32_t        mode;        /* csa2_mode                                     */
    const void*    qI;          /* indexing modes: bf16 [B][Q][32][128]          */
    const float*   w;           /* indexing modes: f32 [B][Q][32]                */
    const void*    q;           /* bf16 [B][Q][64][512]                          */
    const void*    swa;         /* bf16 [B][swa_rows][512]                       */
    void*          out;         /* out bf16 [B][Q][64][512]                      */
    float*         lse;         /* optional out f32 [B][Q][64]                   */
    int32_t*       idx;         /* indexing modes: out int32 [B][Q][K]           */
    float*         scores;      /* optional out f32 [B][Q][K]                    */
    const float*   swa_scale;   /* group swa_format CSA2_FMT_FP8: f32 [B][swa_rows] */
} csa2_layer;

typedef struct csa2_group_args {
    int32_t          B, Q, K, W;
    int64_t          N;
    const int32_t*   n_vis;     /* int32 [B][Q]                                  */
    const void*      kI;        /* bf16 [B][N][128]                              */
    void*            kv_fp4;    /* u8 [B][N][288]                                */
    const void*      kv_new;    /* bf16 [n_new][512], or NULL                    */
    int64_t          n_new;     /* entries to quantise first (may be 0)          */
    const int64_t*   new_rows;  /* int64 [n_new] absolute rows in [0, B*N)       */
    int32_t          swa_rows, swa_step;
    int32_t          hsi_blocks, hsi_block;
    int32_t*         pool;      /* hsi_blocks > 0: int32 [B][Q][hsi_blocks]      */
    float            scale;
    int32_t          n_layers;  /* 1..64                                         */
    const csa2_layer* layers;   /* HOST array of n_layers descriptors            */
    const int32_t*   pool_in;   /* optional int32 [B][Q][hsi_blocks]: the pool of
                                   an earlier call, read by REINDEX_POOL layers
                                   that come before any FULL layer of this call */
    int32_t          flags;     /* CSA2_GROUP_* bits                             */
    int32_t          swa_format;/* the layers' window rows: CSA2_FMT_BF16 or _FP8 */
    int32_t          index_k_format; /* kI: CSA2_FMT_BF16 or CSA2_FMT_MXFP4      */
    int32_t          q_format;  /* every layer's q: CSA2_FMT_BF16, or _NVFP4 with
                                   q as u8 [B][Q][64][288] FP4 rows               */
} csa2_group_args;

#define CSA2_GROUP_INPUTS_READY 1
#define CSA2_GROUP_SERIAL       2

csa2_status csa2_group_decode(const csa2_group_args* g, void* ws,
                              size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * csa2_stack_decode -- several sharing groups run one after another on one
 * stream, as the model stacks them ([eogee] §3.2 configuration paragraph:
 * the decoder's 20 layers are 5 groups of 4, the first Full + 3 Reuse, the
 * others Reindex + 3 Reuse; the encoder's 18 are 3 groups of Full + 5
 * Reuse).  Equivalent to calling csa2_group_decode for groups[0..n_groups)
 * in order with one workspace, except that a group after the first is a
 * model-order successor of the one before it: its first layer's inputs are
 * read only after the previous group's last kernel has finished (unless
 * that group's flags hold CSA2_GROUP_INPUTS_READY).  Each group's pool_in
 * may point at an earlier group's pool (the decoder's first Full layer
 * builds the pool that every later Reindex layer re-scores, [eogee] §3.3).
 * The workspace is the largest any single group needs
 * (csa2_workspace_size(&stack_args, CSA2_WS_STACK)); flags of the groups
 * apply to their own kernels.
 * Errors: those of csa2_group_decode, checked for every group before
 * anything is enqueued; ARG when n_groups is outside 1..64.
 * ---------------------------------------------------------------------- */
typedef struct csa2_stack_args {
    int32_t                n_groups;
    const csa2_group_args* groups;   /* HOST array of n_groups descriptors       */
} csa2_stack_args;

csa2_status csa2_stack_decode(const csa2_stack_args* s, void* ws,
                              size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * csa2_group_decode_io / csa2_stack_decode_io -- the same step as
 * csa2_group_decode / csa2_stack_decode, with the step's host<->device
 * copies overlapped with its layers: a caller whose per-layer inputs (new
 * entries, index-Q, w, q) sit in host memory and who wants the outputs
 * back in host memory gets the copies hidden behind the layers that do
 * not need them, instead of a copy in before the step and a copy out
 * after it.
 *
 * Each copy names a layer, counted over the call's layers (a stack counts
 * through its groups in order):
 *   in[i]   host -> device; it has landed before the first kernel of layer
 *           in[i].layer reads anything (a group's quantise step belongs to
 *           its first layer, so the new entries name that layer);
 *   out[i]  device -> host; it starts once layer out[i].layer's attention
 *           has finished.
 * Copies of each list are in non-decreasing layer order.  The input copies
 * start after all work enqueued on `stream` before the call (a step may
 * overwrite the device inputs the previous step read), all of them at
 * once, in order, on a copy stream of the library's; the outputs go out on
 * a second copy stream.  Both join `stream` before the call's last
 * operation, so everything the call does, copies included, is ordered on
 * `stream` (and a stream capture of the call records the copies as well).
 * Host memory must be page-locked (cudaHostAlloc, cudaHostRegister) for
 * copies to overlap and for capture.
 *
 * The copy streams and their events belong to the library, one set per
 * device: io calls on one device must not overlap in time.
 * Errors: those of csa2_group_decode / csa2_stack_decode; ARG when io is
 * NULL, a count is negative, a list with copies is NULL, a copy has a NULL
 * pointer or names a layer outside the call, or a list is out of order.
 * ---------------------------------------------------------------------- */
typedef struct csa2_copy {
    void*       dst;
    const void* src;
    size_t      bytes;         /* 0: nothing to copy                             */
    int32_t     layer;         /* see above                                      */
} csa2_copy;

typedef struct csa2_io {
    const csa2_copy* in;       /* HOST array of n_in host->device copies         */
    int32_t          n_in;
    const csa2_copy* out;      /* HOST array of n_out device->host copies        */
    int32_t          n_out;
} csa2_io;

csa2_status csa2_group_decode_io(const csa2_group_args* g, const csa2_io* io, void* ws,
                                 size_t ws_bytes, void* stream);
csa2_status csa2_stack_decode_io(const csa2_stack_args* s, const csa2_io* io, void* ws,
                                 size_t ws_bytes, void* stream);

/* Workspace bytes needed by a call.  which = 1: csa2_index_args,
 * 2: csa2_attn_args, 3: csa2_group_args, 4: csa2_stack_args.  Returns 0
 * when the arguments are invalid for that call.
 *
 * Launches: every kernel is launched with programmatic stream serialisation
 * (it may start while the previous kernel in the stream finishes, and waits
 * for it before touching memory that kernel owns).  Setting the environment
 * variable CSA2_PDL=0 before the first call launches them in plain stream
 * order. */
#define CSA2_WS_INDEX 1
#define CSA2_WS_ATTN  2
#define CSA2_WS_GROUP 3
#define CSA2_WS_STACK 4
size_t csa2_workspace_size(const void* args, int32_t which);

/* Reads and clears the device-side failure word of the current device
 * (bounded waits that gave up, internal limits exceeded).  Synchronises
 * `stream`.  Returns CSA2_OK when clear, CSA2_ERR_DEVICE otherwise and
 * stores the recorded code in *code (may be NULL). */
csa2_status csa2_device_status(int32_t* code, void* stream);

/* Human-readable name of a status code (static string). */
const char* csa2_status_string(int32_t status);

/* The CUDA runtime's description of the last launch or runtime failure
 * behind a CSA2_ERR_CUDA on the calling host thread ("no error" if none);
 * static string. */
const char* csa2_cuda_error_string(void);

/* Library ABI version: 100 * major + minor. */
int32_t csa2_version(void);

/* ------------------------------------------------------------------------
 * Launch tracing, for profiling harnesses (off by default).
 * csa2_trace_begin(n) creates 2n CUDA events (outside any timed region) and
 * from then on brackets every kernel the library enqueues with two of them,
 * recorded on that kernel's stream, until n launches are recorded or
 * csa2_trace_stop() is called.  csa2_trace_count() tells how many were
 * recorded; csa2_trace_get(i, &kernel, &ms) waits for launch i and returns
 * its kernel id and event-measured duration in milliseconds.
 * csa2_trace_end() destroys the events.  Kernel ids name the library's
 * kernels (csa2_kernel_name).  Calls enqueued while their stream is being
 * captured into a CUDA graph put the event records into the graph (external
 * event-record nodes): each replay of the graph re-records them, and
 * csa2_trace_get then returns the durations of the latest replay.  Tracing
 * state is process-global and not synchronised: enable it only while one
 * thread drives the library.
 * ---------------------------------------------------------------------- */
#define CSA2_KERNEL_QUANTIZE     0
#define CSA2_KERNEL_INDEX_SCAN   1
#define CSA2_KERNEL_TOPK         2
#define CSA2_KERNEL_ATTN_SLICE   3
#define CSA2_KERNEL_ATTN_COMBINE 4
#define CSA2_KERNEL_QUANTIZE_WINDOW 5
#define CSA2_KERNEL_QUANTIZE_INDEX_K 6
#define CSA2_KERNEL_COMPRESS_ROPE   7
csa2_status csa2_trace_begin(int32_t max_launches);
csa2_status csa2_trace_stop(void);
csa2_status csa2_trace_end(void);
int32_t csa2_trace_count(void);
csa2_status csa2_trace_get(int32_t i, int32_t* kernel, float* ms);
const char* csa2_kernel_name(int32_t kernel);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_ABI_H_ */
