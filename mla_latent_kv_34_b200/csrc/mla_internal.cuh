// Internal helpers shared by the MLA kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

constexpr int kDc = 512;           // latent width d_c
constexpr int kDr = 64;            // RoPE width d_h^R
constexpr int kDh = 128;           // head width d_h
constexpr int kRow = kDc + kDr;    // packed cache row (576 bf16 = 1152 B)
constexpr int kMaxHeads = 128;
constexpr int kMaxNq = 256;       // new query tokens per sequence (decode, speculation, prefill chunks)
constexpr int kBlockTokens = MLA_BLOCK_TOKENS;  // tokens per cache block
constexpr int kBlockBytes = MLA_BLOCK_BYTES;    // 9 chunks x [128 rows x 128 B]
constexpr int kBlockChunk = kBlockTokens * 128;  // bytes of one 64-column chunk of a block
static_assert(kBlockBytes == 9 * kBlockChunk, "block layout");
constexpr int kMaxPairs = 74;      // CTA pairs per row group the tensor-core decode uses at most (148 SMs / 2)
constexpr int kMaxSmRows = 32;     // query rows (n_q * H) up to which the one-SM decode kernel runs instead
constexpr int kMaxSmCtas = 148;    // CTAs the one-SM decode kernel uses at most (one per SM)

// Tiles (128-token blocks) of a sequence that the decode processes: none when kv_len < n_q or when the
// sequence needs more blocks than its block-table row holds.  The attend and merge kernels both use this
// rule, so they agree on how the (sequence, tile) space is cut into pieces.
__host__ __device__ __forceinline__ int valid_seq_tiles(int L, int n_q, int max_blocks) {
    if (L < n_q) return 0;
    const int nt = (L + kBlockTokens - 1) / kBlockTokens;
    return nt > max_blocks ? 0 : nt;
}

// Byte offset of column c of row r inside a cache block (128-byte swizzle per 64-column chunk).
__host__ __device__ __forceinline__ int block_offset(int r, int c) {
    return (c >> 6) * kBlockChunk + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// fp32 -> bf16, round to nearest, ties to even (finite inputs; NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return static_cast<uint16_t>((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return static_cast<uint16_t>(u >> 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return static_cast<uint32_t>(f32_to_bf16_rne(lo)) | (static_cast<uint32_t>(f32_to_bf16_rne(hi)) << 16);
}

__device__ __forceinline__ void report(int32_t* dev_status, int32_t bit) {
    if (dev_status) atomicOr(dev_status, bit);
}

// Host-side launch wrappers (one per kernel file).
cudaError_t launch_append_cache(uint8_t* cache, int64_t cap_blocks, const int32_t* block_table, int num_seqs,
                                int max_blocks,
                                const int32_t* seq_idx, const int32_t* pos, const uint16_t* c_kv,
                                const uint16_t* k_rope, const float* rope_table, int64_t rope_len, int T,
                                int32_t* dev_status, cudaStream_t stream);

cudaError_t launch_absorb_tc(const uint16_t* q_nope, const uint16_t* q_rope, const int32_t* pos, const uint16_t* W_UK,
                             const float* rope_table, int64_t rope_len, int T, int H, uint16_t* q_out,
                             int32_t* dev_status, cudaStream_t stream);

// Query up-projections q^C = W^UQ c^Q, q^R = W^QR c^Q (query_up.cu).
cudaError_t launch_query_up(const uint16_t* c_q, const uint16_t* W_UQ, const uint16_t* W_QR, int T, int H, int d_cq,
                            uint16_t* q_nope, uint16_t* q_rope, int32_t* dev_status, cudaStream_t stream);

// The compressed-query up-projections fused with the absorption of W^UK (query_absorb.cu).
cudaError_t launch_query_absorb(const uint16_t* c_q, const uint16_t* W_UQ, const uint16_t* W_QR, const uint16_t* W_UK,
                                const int32_t* pos, const float* rope_table, int64_t rope_len, int T, int H, int d_cq,
                                uint16_t* q_out, int32_t* dev_status, cudaStream_t stream);

// Naive-form attention for long prefill chunks (prefill_naive.cu).
size_t prefill_rows_bytes(int L, int H);
cudaError_t launch_prefill_naive(const uint16_t* q_nope, const uint16_t* q_rope, const float* rope_table,
                                 const uint8_t* cache, int64_t cap_blocks, const int32_t* blocks, int L, int n,
                                 const uint16_t* W_UK, const uint16_t* W_UV, int H, float scale, uint16_t* k_rows,
                                 uint16_t* v_rows, uint16_t* out, float* lse_out, int32_t* dev_status,
                                 cudaStream_t stream);

cudaError_t launch_decode_simt(const uint16_t* q, const uint8_t* cache, int64_t cap_blocks, const int32_t* block_table,
                               int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale, int splits,
                               float* o_part, float* lse_part, int32_t* dev_status, cudaStream_t stream);

cudaError_t launch_combine(const float* o_part, const float* lse_part, int T, int H, int splits,
                           const uint16_t* W_UV, void* out, float* lse_out, cudaStream_t stream);

// Tensor-core decode (decode_tc.cu); the merge of its pieces and the W^UV projection (proj_tc.cu).
int decode_tc_clusters();
int decode_sm_ctas();
cudaError_t launch_decode_sm(const uint16_t* q, const uint8_t* cache, int64_t cap_blocks, const int32_t* block_table,
                             int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale, int ctas,
                             float* o_part, float2* ml_part, int slots, int rs, int32_t* dev_status,
                             cudaStream_t stream);
cudaError_t launch_decode_tc(const uint16_t* q, const uint8_t* cache, int64_t cap_blocks, const int32_t* block_table,
                             int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale,
                             int clusters_per_group, float* o_part, float2* ml_part, int slots, int32_t* dev_status,
                             cudaStream_t stream);
// Rows of the merged latent output o_lat kept for the up-projection: T rounded so that every 64-token
// block but the last is full and the last is a multiple of 16 (the MMA N granularity).
__host__ __device__ __forceinline__ int olat_rows(int T) {
    const int full = (T / 64) * 64, rest = T - full;
    return full + ((rest + 15) / 16) * 16;
}
cudaError_t launch_merge(const float* o_part, const float2* ml_part, const int32_t* kv_len, int max_blocks, int B,
                         int n_q, int H, int P_g, int slots, int rs, uint8_t* olat, float* lse_out,
                         int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_upproj(const uint8_t* olat, const uint16_t* W_UV, int T, int H, uint16_t* out, int32_t* dev_status,
                          cudaStream_t stream);

}  // namespace mla
