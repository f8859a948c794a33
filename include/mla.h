/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA weight-absorbed decode library.
 *
 * Multi-head Latent Attention keeps, per token and layer, only the joint
 * latent c^KV (d_c = 512) and one RoPE key k^R (d_h^R = 64) shared by all
 * heads: 576 bf16 elements.  W^UK is folded into each head's query, attention
 * scores and aggregates directly against the latent cache, and W^UV is
 * applied after the reduction, so per-head keys and values never exist.
 *   - "DeepSeek-V2/V3: 大模型的两张账" (chenyuan1125.github.io), section
 *     "第一张账": c_t^KV = W^DKV h_t, k_t^C = W^UK c_t^KV, v_t^C = W^UV c_t^KV;
 *     W^UK absorbed into the query side, W^UV applied after aggregating in
 *     latent space; cache only c_t^KV and k_t^R; (d_c + d_h^R) = 4.5 d_h.
 *   - DeepSeek-V2 MLA explainer (xinfinite.net), section 2.2.2: decoupled
 *     RoPE with per-head q^R and one shared k^R; the RoPE'd key part is cached
 *     so keys need no rotation at inference; attention on [q^C; q^R].[k^C; k^R].
 *   - The same explainer, section 2.2.1.2: queries are compressed too, to c^Q,
 *     and up-projected (mla_query_up produces q^C and q^R from c^Q).
 *
 * Entry points, in the order a decode step uses them: mla_query_absorb (when
 * queries are compressed; = mla_query_up + mla_absorb_q in one launch) or
 * mla_absorb_q, mla_append_cache, mla_decode (=
 * mla_decode_attend + mla_decode_finish; mla_decode_static without a
 * workspace), with mla_decode_cudacore + mla_splitkv_combine as an
 * independent CUDA-core path of the same decode.  Long prefill chunks use
 * mla_prefill_naive (the naive form) after mla_append_cache.
 *
 * Fixed sizes: d_c = 512, d_h^R = 64, d_h = 128 (cached row D = 576).
 * Runtime sizes: B sequences, H heads (1..128), n_q new query tokens per
 * sequence (1..256: a decode step, speculative tokens or a prefill chunk),
 * T = B * n_q query rows (row t = b * n_q + j).
 *
 * Latent cache layout (paged, blocked).  The cache is a pool of blocks of
 * MLA_BLOCK_TOKENS = 128 tokens, MLA_BLOCK_BYTES = 147456 bytes each, and a
 * block table maps each sequence's token positions to pool blocks: token
 * `pos` of sequence b lives in block block_table[b * max_blocks + pos / 128],
 * at row r = pos % 128.  A sequence's blocks need not be consecutive or in
 * any order, so a serving runtime can hand out blocks of one pool as
 * sequences grow and free them in any order, with no copying and no
 * fragmentation beyond one partly filled block per sequence (the paged
 * KV-cache of vLLM/PagedAttention, named as the complementary technique in the
 * MLA explainer (xinfinite.net), section 2.1.1).  The token's 576 bf16 values
 * [c^KV (0..511) | rotated k^R (512..575)] are stored as nine 64-column
 * chunks, column c at byte offset
 *     (c / 64) * 16384 + r * 128 + (((c % 64) / 8) ^ (r % 8)) * 16 + (c % 8) * 2
 * within the block: each chunk is a [128 rows x 128 bytes] tile whose 16-byte
 * units are permuted by the row index (the 128-byte swizzle), so that
 * contiguous copies place a block in shared memory exactly as the tensor-core
 * operands are read (128 tokens per block make the score MMA 128 wide).
 *
 * Block table: int32 [B, max_blocks], row-major, device memory.  Row b lists
 * the pool blocks of sequence b in position order; only its first
 * ceil(kv_len[b] / 128) entries are read.  A sequence longer than
 * max_blocks * 128 tokens is not processed and sets MLA_DEVERR_ROW_RANGE; an
 * entry read outside [0, cap_blocks) sets MLA_DEVERR_ROW_RANGE and that
 * sequence's results are unspecified (no access outside the pool is made).
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers to caller-owned memory, dense
 *     row-major, in the layouts stated.  bf16 tensors must be 16-byte aligned.
 *     The library never allocates, frees, synchronises or keeps a pointer
 *     after it returns; work is enqueued on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).
 *   - Host-side argument errors return MLA_ERR_INVALID_ARG or
 *     MLA_ERR_UNSUPPORTED_SHAPE before anything is launched.  A failed launch
 *     returns MLA_ERR_CUDA.
 *   - `dev_status` (nullable) is a device int32 that kernels OR error bits
 *     into (MLA_DEVERR_*).  The caller zeroes it and reads it after the stream
 *     is synchronised; mla_device_status_string() names the bits.  Work that
 *     trips a check is skipped (never a trap or a fault).
 *   - RoPE pairs adjacent dims (2i, 2i+1) with theta_i = base^(-2i/64); the
 *     key of cache index t is rotated at position t, query j of sequence b at
 *     L_b - n_q + j.  `rope_table` is fp32 [rope_len, 64] holding
 *     (cos, sin) of pos * theta_i for pair i at [pos, 2i], [pos, 2i+1]; build
 *     it with mla_rope_table_fill() and copy it to the device.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* mla_stream; /* cudaStream_t */

#define MLA_BLOCK_TOKENS 128
#define MLA_BLOCK_BYTES 147456

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,       /* null pointer, misalignment, negative size */
    MLA_ERR_UNSUPPORTED_SHAPE = 2, /* H, n_q or split count outside the supported range */
    MLA_ERR_CUDA = 3,              /* a CUDA runtime call or launch failed */
    MLA_ERR_WORKSPACE = 4          /* workspace smaller than the *_workspace_bytes() figure */
} mla_status;

/* Bits a kernel ORs into *dev_status. */
#define MLA_DEVERR_ROW_RANGE   0x1  /* a cache block outside [0, cap_blocks) was addressed */
#define MLA_DEVERR_POS_RANGE   0x2  /* a position outside [0, rope_len) */
#define MLA_DEVERR_KV_LEN      0x4  /* kv_len[b] < n_q */
#define MLA_DEVERR_TIMEOUT     0x8  /* a bounded wait in a pipelined kernel expired */

const char* mla_status_string(int status);
const char* mla_device_status_string(int32_t dev_status_word);
int mla_abi_version(void); /* 2: paged cache (block tables) */

/*
 * mla_rope_table_fill -- HOST function.  table_host: fp32 [rope_len, 64],
 * caller-owned host memory.  Entry [p, 2i] = (float)cos(p * theta_i),
 * [p, 2i+1] = (float)sin(p * theta_i), theta_i = base^(-2i/64), computed in
 * double with the C library and rounded once to fp32.
 */
mla_status mla_rope_table_fill(float* table_host, int64_t rope_len, double base);

/*
 * mla_absorb_q -- absorb W^UK into the query and rotate q^R.
 * (Absorption: "两张账" page, "第一张账" -- W^UK moves to the query side so
 *  that q^C . k^C_t = q_abs . c_t^KV; decoupled RoPE: explainer 2.2.2.)
 *   q_nope  bf16 [T, H, 128]     content query q^C
 *   q_rope  bf16 [T, H, 64]      RoPE query q^R before rotation
 *   pos     int32 [T] or NULL    position of query row t (NULL: q_rope is
 *                                already rotated and is copied)
 *   W_UK    bf16 [H, 128, 512]   per-head up-projection (k^C = W^UK_h c)
 *   q_out   bf16 [T, H, 576]     [ (W^UK_h)^T q_nope (512) | R_pos q^R (64) ]
 * fp32 accumulation (tensor cores), one rounding to bf16 per output element;
 * the q^R rotation uses the same fp32 arithmetic as mla_append_cache.
 */
mla_status mla_absorb_q(const void* q_nope, const void* q_rope, const int32_t* pos,
                        const void* W_UK, const float* rope_table, int64_t rope_len,
                        int T, int H, void* q_out, int32_t* dev_status, mla_stream stream);

/*
 * mla_query_up -- the query side of the low-rank path: up-projections of the
 * compressed query c^Q into the content query q^C and the RoPE query q^R.
 * (MLA explainer 2.2.1.2: queries are compressed like keys and values, a
 *  down-projection to c^Q and up-projections from it, q^C_t = W^UQ c^Q_t;
 *  2.2.2: the decoupled per-head q^R.  q^R = W^QR c^Q is this library's
 *  reading: its formula is lost on the page.)
 *   c_q     bf16 [T, d_cq]        compressed queries c^Q (row-major)
 *   W_UQ    bf16 [H, 128, d_cq]   per-head content up-projection
 *   W_QR    bf16 [H, 64, d_cq]    per-head RoPE up-projection
 *   q_nope  bf16 [T, H, 128]      out: q^C[t, h] = W^UQ_h c^Q_t
 *   q_rope  bf16 [T, H, 64]       out: q^R[t, h] = W^QR_h c^Q_t, not rotated
 *                                 (mla_absorb_q rotates it at the query position)
 * The outputs are exactly mla_absorb_q's inputs.  fp32 accumulation on the
 * tensor cores, one rounding to bf16 per output element.
 * Sizes: 1 <= H <= 128; d_cq a multiple of 64 in [64, 16384]; T >= 0 (T = 0
 * launches nothing).  All pointers are device memory owned by the caller,
 * 16-byte aligned; nothing is kept after the call returns.
 * Errors: MLA_ERR_UNSUPPORTED_SHAPE for H or d_cq out of range,
 * MLA_ERR_INVALID_ARG for null or misaligned pointers or T < 0 (returned
 * before any launch); MLA_ERR_CUDA if the launch fails; an expired bounded
 * wait on the device sets MLA_DEVERR_TIMEOUT in *dev_status (may be NULL).
 */
mla_status mla_query_up(const void* c_q, const void* W_UQ, const void* W_QR, int T, int H, int d_cq,
                        void* q_nope, void* q_rope, int32_t* dev_status, mla_stream stream);

/*
 * mla_query_absorb -- mla_query_up and mla_absorb_q in one launch: from the
 * compressed query c^Q straight to the absorbed query.
 * (MLA explainer 2.2.1.2 and 2.2.2: q^C = W^UQ c^Q and the per-head q^R;
 *  "两张账" page, "第一张账": W^UK absorbed into the query side.)
 *   c_q     bf16 [T, d_cq]         compressed queries c^Q
 *   W_UQ    bf16 [H, 128, d_cq]    W_QR bf16 [H, 64, d_cq]    W_UK bf16 [H, 128, 512]
 *   pos     int32 [T] or NULL      position of query row t (NULL: q^R is not rotated)
 *   q_out   bf16 [T, H, 576]       [ (W^UK_h)^T q^C[t, h] (512) | R_pos q^R[t, h] (64) ]
 * q^C and q^R are rounded to bf16 exactly as mla_query_up stores them, and the
 * rest is mla_absorb_q's arithmetic, so q_out is bit for bit the output of
 * mla_query_up followed by mla_absorb_q; q^C never leaves the SM (it goes from
 * tensor memory to shared memory as the operand of the absorption).  The
 * order of operations is kept: no precomposed (W^UK_h)^T W^UQ_h is formed.
 * Sizes: 1 <= H <= 128, d_cq a multiple of 64 in [64, 16384], T >= 0 (T = 0
 * launches nothing).  Errors: as mla_query_up and mla_absorb_q (before any
 * launch); a position outside the RoPE table sets MLA_DEVERR_POS_RANGE and that
 * row's RoPE part is left unwritten; an expired bounded wait sets
 * MLA_DEVERR_TIMEOUT.  Launched with programmatic stream serialization.
 */
mla_status mla_query_absorb(const void* c_q, const void* W_UQ, const void* W_QR, const void* W_UK,
                            const int32_t* pos, const float* rope_table, int64_t rope_len, int T,
                            int H, int d_cq, void* q_out, int32_t* dev_status, mla_stream stream);

/*
 * mla_append_cache -- write T new tokens into the paged latent cache.
 * ("两张账" page: only c^KV and k^R are cached; explainer 2.2.2: k^R is
 *  cached already rotated.)
 *   cache        pool of cap_blocks blocks of MLA_BLOCK_BYTES (layout above)
 *   block_table  int32 [num_seqs, max_blocks]  token i goes to pool block
 *                block_table[seq_idx[i] * max_blocks + pos[i] / 128], row pos[i] % 128
 *   seq_idx      int32 [T]  sequence of token i
 *   pos          int32 [T]  position of token i within its sequence
 *   c_kv         bf16 [T, 512]   copied to columns 0..511 bit for bit
 *   k_rope       bf16 [T, 64]    rotated at pos[i] into columns 512..575
 * The rotation is y0 = fl(fl(x0 c) - fl(x1 s)), y1 = fl(fl(x0 s) + fl(x1 c))
 * in fp32 (no fused multiply-add) with (c, s) from rope_table, then
 * round-to-nearest-even to bf16: the result is reproducible bit for bit.
 * A token whose sequence is outside [0, num_seqs), whose position is negative
 * or past its table row (pos / 128 >= max_blocks), or whose table entry lies
 * outside [0, cap_blocks), sets
 * MLA_DEVERR_ROW_RANGE and is skipped; a position outside the RoPE table sets
 * MLA_DEVERR_POS_RANGE and is skipped.  Errors: MLA_ERR_INVALID_ARG for null
 * or misaligned pointers, negative sizes, num_seqs or max_blocks < 1 (before
 * any launch).
 */
mla_status mla_append_cache(void* cache, int64_t cap_blocks, const int32_t* block_table,
                            int num_seqs, int max_blocks, const int32_t* seq_idx, const int32_t* pos,
                            const void* c_kv, const void* k_rope, const float* rope_table,
                            int64_t rope_len, int T, int32_t* dev_status, mla_stream stream);

/*
 * mla_decode_workspace_bytes -- device workspace mla_decode needs for these
 * sizes (num_splits as passed to mla_decode; 0 = automatic).  It holds the
 * attend phase's pieces (a slot of 128 rows -- 32 when n_q * H <= 32 -- x
 * (512 fp32 + max, sum) per sequence plus one per work unit of the group, for
 * each group of 128 query rows; with G groups a group gets at most max(1, 74 / G) CTA pairs, and with
 * n_q * H <= 32 the one group gets up to 148 one-SM units) and the merged
 * latent output in bf16 ([H, ~B*n_q, 512]).
 */
size_t mla_decode_workspace_bytes(int B, int n_q, int H, int num_splits);

/*
 * mla_decode -- one absorbed MLA decode step over the paged latent cache.
 * For every sequence b, query j and head h, with p = kv_len[b] - n_q + j:
 *   s_t   = (q[t,h,:512] . c_t + q[t,h,512:] . k^R_t) * scale,  t = 0..p
 *   P     = softmax(s)                   (fp32, online / split-KV)
 *   o_lat = sum_t P_t c_t                (latent aggregation, 512)
 *   out   = W^UV_h o_lat                 (128)
 * ("两张账" page, "第一张账": scores against the cached latent, aggregation in
 *  latent space, W^UV afterwards; explainer 2.2.2 for the concatenated
 *  content/position inner product.)
 *   q          bf16 [B*n_q, H, 576]   from mla_absorb_q
 *   cache      pool of cap_blocks blocks (layout above)
 *   block_table int32 [B, max_blocks]: tile i (tokens 128 i .. 128 i + 127) of
 *              sequence b is pool block block_table[b * max_blocks + i]
 *   kv_len     int32 [B]: cached tokens of each sequence, counting the n_q
 *              tokens of this step (already appended)
 *   W_UV       bf16 [H, 128, 512]
 *   scale      softmax scale, 1/sqrt(d_h + d_h^R) = 1/sqrt(192) for V2 shapes
 *   num_splits 0: use every SM.  n > 0: at most n CTA pairs per group of 128
 *              query rows.  The (sequence, 128-token tile) space is cut into
 *              equal contiguous ranges, one per CTA pair; the pieces of a
 *              sequence are merged by log-sum-exp.  Results do not depend on
 *              n beyond fp32 summation order.
 *   workspace  device scratch of at least mla_decode_workspace_bytes() bytes
 *   out        bf16 [B*n_q, H, 128]
 *   lse_out    fp32 [B*n_q, H] or NULL: log sum_t exp(s_t)
 * A sequence with kv_len[b] < n_q sets MLA_DEVERR_KV_LEN, one longer than
 * max_blocks * 128 sets MLA_DEVERR_ROW_RANGE; neither is processed and their
 * rows get out = 0 and lse = -inf.  A table entry outside [0, cap_blocks) sets
 * MLA_DEVERR_ROW_RANGE (that sequence's rows are then unspecified).
 * The call launches the attend kernel (CTA pairs; for n_q * H <= 32 a kernel
 * that does a whole block on one SM), then the merge and up-projection
 * kernels (mla_decode_finish), each with programmatic stream serialization:
 * a kernel's set-up may overlap the end of the previous kernel on `stream`.
 * The attend kernel waits for that kernel to complete before reading any
 * input; the merge and up-projection kernels read kv_len and W_UV (inputs
 * that no kernel of the call writes) before their wait, and everything the
 * previous kernel of the call produced after it.
 * Errors: MLA_ERR_INVALID_ARG (null or misaligned pointer, bad scale, cap_blocks
 * or max_blocks < 1), MLA_ERR_UNSUPPORTED_SHAPE, MLA_ERR_WORKSPACE (ws_bytes
 * below mla_decode_workspace_bytes()), all before any launch; MLA_ERR_CUDA.
 */
mla_status mla_decode(const void* q, const void* cache, int64_t cap_blocks,
                      const int32_t* block_table, int max_blocks, const int32_t* kv_len,
                      const void* W_UV, int B, int n_q, int H, float scale, int num_splits,
                      void* workspace, size_t ws_bytes, void* out, float* lse_out,
                      int32_t* dev_status, mla_stream stream);

/*
 * mla_decode_attend / mla_decode_finish -- the two phases of mla_decode,
 * exposed so that callers can place work (or timing events) between them.
 * attend: scores, online softmax and latent aggregation into per-piece
 * partials held in `workspace` (one kernel); finish: log-sum-exp merge of the
 * pieces of each sequence (one kernel) and the W^UV up-projection into `out`
 * and `lse_out` (one kernel).  Arguments mean the same as for mla_decode;
 * both calls must see the same B, n_q, H, kv_len, max_blocks, num_splits and
 * workspace, and finish must be ordered after attend on the stream.
 */
mla_status mla_decode_attend(const void* q, const void* cache, int64_t cap_blocks,
                             const int32_t* block_table, int max_blocks, const int32_t* kv_len,
                             int B, int n_q, int H, float scale, int num_splits,
                             void* workspace, size_t ws_bytes, int32_t* dev_status,
                             mla_stream stream);
mla_status mla_decode_finish(const int32_t* kv_len, int max_blocks, const void* W_UV,
                             int B, int n_q, int H, int num_splits,
                             void* workspace, size_t ws_bytes, void* out, float* lse_out,
                             int32_t* dev_status, mla_stream stream);

/*
 * mla_decode_static -- mla_decode without a workspace argument: the step's
 * segment partials go to one scratch buffer owned by the library (a static
 * device array of MLA_DECODE_STATIC_SCRATCH_BYTES per device).  Neither
 * paper has a counterpart; this is a convenience of the library for callers
 * that cannot allocate device memory where they decode (a frozen memory
 * pool, a thread that must not enter the CUDA allocator, code without any
 * allocator).  Nothing on this path allocates.
 *   Arguments, layouts and results are those of mla_decode.
 *   Limit: shapes with mla_decode_workspace_bytes(B, n_q, H, num_splits) >
 *   MLA_DECODE_STATIC_SCRATCH_BYTES return MLA_ERR_WORKSPACE and launch
 *   nothing (for example B <= 32 at H = 128, n_q = 1; with n_q * H <= 32 the
 *   slots are a quarter the size, so B = 64 fits at H = 16, n_q = 2).
 *   Set-up: the first call on a device looks the buffer up (and may load the
 *   library's device code there); make it before any stream capture.  The
 *   address found is kept for the life of the process: after a reset of the
 *   device (cudaDeviceReset, or any teardown of its primary context) this
 *   entry point must not be called again on that device.
 *   Zeroing: none needed; every partial read is written in the same call.
 *   Races: one buffer per device, so calls that can overlap on a device
 *   (other streams, unordered host threads) corrupt each other's partials;
 *   calls ordered on one stream are safe.
 */
#define MLA_DECODE_STATIC_SCRATCH_BYTES (32u << 20)
mla_status mla_decode_static(const void* q, const void* cache, int64_t cap_blocks,
                             const int32_t* block_table, int max_blocks, const int32_t* kv_len,
                             const void* W_UV,
                             int B, int n_q, int H, float scale, int num_splits,
                             void* out, float* lse_out, int32_t* dev_status, mla_stream stream);

/*
 * mla_decode_cudacore -- the same decode step computed on CUDA cores (fp32
 * FMA, split-KV over `num_splits` equal key ranges per sequence, 0 =
 * automatic) instead of the tensor cores.  Same arguments and results as
 * mla_decode, within fp32 rounding; a second implementation to check the
 * tensor-core path against.  Its workspace size is
 * mla_decode_cudacore_workspace_bytes().
 */
size_t mla_decode_cudacore_workspace_bytes(int B, int n_q, int H, int num_splits);
mla_status mla_decode_cudacore(const void* q, const void* cache, int64_t cap_blocks,
                               const int32_t* block_table, int max_blocks, const int32_t* kv_len,
                               const void* W_UV,
                               int B, int n_q, int H, float scale, int num_splits,
                               void* workspace, size_t ws_bytes, void* out, float* lse_out,
                               int32_t* dev_status, mla_stream stream);

/*
 * mla_prefill_workspace_bytes / mla_prefill_naive -- attention of n new tokens
 * of one sequence in the NAIVE form, for long prefill chunks.  ("两张账" page,
 * "第一张账": the naive path rebuilds k^C = W^UK c and v^C = W^UV c from c^KV;
 * MLA explainer 2.2.2: attention on [q^C; R q^R].[k^C; k^R].)  The absorbed
 * form of mla_decode does 3.4x the arithmetic per (query, key, head), so for
 * causal chunks beyond ~340 tokens rebuilding the keys and values once per
 * (key, head) costs less.
 *   q_nope, q_rope  bf16 [n, H, 128] / [n, H, 64]: the chunk's queries, q^R
 *                   unrotated (rotated here at its position, as mla_absorb_q)
 *   rope_table      fp32 [rope_len, 64] (as for mla_append_cache); rope_len >= L
 *   cache           pool of cap_blocks blocks (layout above) holding the
 *                   sequence's L tokens, the n new ones (already appended) last
 *   blocks          int32 [ceil(L / 128)], device: the sequence's row of the
 *                   block table (tile i = pool block blocks[i])
 *   query j sits at position L - n + j and sees keys 0 .. L - n + j
 *   W_UK, W_UV      bf16 [H, 128, 512]
 *   workspace       mla_prefill_workspace_bytes(L, H) bytes: the rebuilt
 *                   k^C and v^C of every key and head, bf16 [L, H, 128] each
 *   out             bf16 [n, H, 128];  lse_out fp32 [n, H] or NULL
 * Two kernels: the decompression (tcgen05, D[token, 0..255] = c . [W^UK_h ;
 * W^UV_h]^T per 128-token block and head), then causal attention (tcgen05 QK^T
 * and PV, online softmax in fp32, one CTA per head and 128-query tile).
 * Rounding: k^C, v^C, the rotated q^R and P are bf16; sums and softmax fp32.
 * Errors (before any launch): MLA_ERR_INVALID_ARG for n > L, L > rope_len, a
 * bad scale, cap_blocks < 1, null or misaligned pointers;
 * MLA_ERR_UNSUPPORTED_SHAPE for H outside 1..128 or L * H * 128 >= 2^31;
 * MLA_ERR_WORKSPACE.  A block entry outside [0, cap_blocks) sets
 * MLA_DEVERR_ROW_RANGE (results unspecified); an expired bounded wait sets
 * MLA_DEVERR_TIMEOUT.  n = 0 launches nothing.
 */
size_t mla_prefill_workspace_bytes(int L, int H);
mla_status mla_prefill_naive(const void* q_nope, const void* q_rope, const float* rope_table,
                             int64_t rope_len, const void* cache, int64_t cap_blocks,
                             const int32_t* blocks, int L, int n, const void* W_UK,
                             const void* W_UV, int H, float scale, void* workspace,
                             size_t ws_bytes, void* out, float* lse_out, int32_t* dev_status,
                             mla_stream stream);

/*
 * mla_splitkv_combine -- log-sum-exp merge of split-KV partials.
 *   o_part   fp32 [T, H, S, 512]  each split's softmax-normalised latent output
 *   lse_part fp32 [T, H, S]       each split's log-sum-exp (-inf: empty split)
 * m = max_s lse_s, w_s = exp(lse_s - m): o = sum_s w_s o_s / sum_s w_s and
 * lse = m + log sum_s w_s.  With W_UV (bf16 [H,128,512]) the merged latent
 * is mapped out: out bf16 [T, H, 128]; with W_UV == NULL, out is the merged
 * latent, fp32 [T, H, 512].  lse_out fp32 [T, H] or NULL.
 */
mla_status mla_splitkv_combine(const float* o_part, const float* lse_part, int T, int H,
                               int num_splits, const void* W_UV, void* out, float* lse_out,
                               mla_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
