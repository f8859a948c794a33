// Cache append: one warp per new token writes its row
// [c^KV (512, copied) | R_pos k^R (64, rotated in fp32)] into the blocked cache.
//
// Only c^KV and the RoPE'd shared key are cached ("两张账" page, "第一张账";
// MLA explainer section 2.2.2: the key's position part is cached already
// rotated).  The rotation uses separately rounded fp32 products and sums
// (__fmul_rn / __fadd_rn / __fsub_rn are never contracted into an FMA), then
// round-to-nearest-even to bf16, so the stored bits are reproducible.
//
// Paged layout (see mla.h): token pos of sequence s is row pos % 128 of pool block
// block_table[s][pos / 128]; row r of a block keeps column c at byte
// (c / 64) * 16384 + r * 128 + (((c % 64) / 8) ^ (r % 8)) * 16 + (c % 8) * 2.
#include "mla_internal.cuh"

namespace mla {

__global__ void __launch_bounds__(256) append_cache_kernel(
    uint8_t* __restrict__ cache, int64_t cap_blocks, const int32_t* __restrict__ block_table, int num_seqs,
    int max_blocks, const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos,
    const uint16_t* __restrict__ c_kv, const uint16_t* __restrict__ k_rope,
    const float* __restrict__ rope_table, int64_t rope_len, int T, int32_t* dev_status) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int32_t p = pos[warp];
    const int32_t sq = seq_idx[warp];
    // the sequence's block-table entry for this position; sequences outside the table, positions past
    // the row, negative indices and entries outside the pool are reported and skipped
    int64_t blk = -1;
    if (p >= 0 && sq >= 0 && sq < num_seqs && p / kBlockTokens < max_blocks)
        blk = block_table[static_cast<int64_t>(sq) * max_blocks + p / kBlockTokens];
    if (blk < 0 || blk >= cap_blocks) {
        if (lane == 0) report(dev_status, MLA_DEVERR_ROW_RANGE);
        return;
    }
    if (p >= rope_len) {
        if (lane == 0) report(dev_status, MLA_DEVERR_POS_RANGE);
        return;
    }
    const int r = p % kBlockTokens;
    uint8_t* dst = cache + blk * kBlockBytes + r * 128;
    // latent: 64 units of 16 bytes = chunks 0..7 x 8 units; two units per lane
    const uint4* src4 = reinterpret_cast<const uint4*>(c_kv + static_cast<int64_t>(warp) * kDc);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int w = lane + 32 * k;  // unit index in the row, 0..63
        const int chunk = w >> 3, u = w & 7;
        *reinterpret_cast<uint4*>(dst + chunk * kBlockChunk + ((u ^ (r & 7)) << 4)) = src4[w];
    }
    // RoPE pair `lane`: dims (2 lane, 2 lane + 1) -> columns 512 + 2 lane (chunk 8)
    const uint32_t xr = reinterpret_cast<const uint32_t*>(k_rope + static_cast<int64_t>(warp) * kDr)[lane];
    const float x0 = bf16_to_f32(static_cast<uint16_t>(xr & 0xFFFFu));
    const float x1 = bf16_to_f32(static_cast<uint16_t>(xr >> 16));
    const float2 cs = reinterpret_cast<const float2*>(rope_table + static_cast<int64_t>(p) * kDr)[lane];
    const float y0 = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y));
    const float y1 = __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x));
    const int u = lane >> 2;  // 16-byte unit within chunk 8
    *reinterpret_cast<uint32_t*>(dst + 8 * kBlockChunk + ((u ^ (r & 7)) << 4) + (lane & 3) * 4) = pack_bf16x2(y0, y1);
}

cudaError_t launch_append_cache(uint8_t* cache, int64_t cap_blocks, const int32_t* block_table, int num_seqs,
                                int max_blocks,
                                const int32_t* seq_idx, const int32_t* pos, const uint16_t* c_kv,
                                const uint16_t* k_rope, const float* rope_table, int64_t rope_len, int T,
                                int32_t* dev_status, cudaStream_t stream) {
    const int threads = 256;
    const int64_t blocks = (static_cast<int64_t>(T) * 32 + threads - 1) / threads;
    append_cache_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        cache, cap_blocks, block_table, num_seqs, max_blocks, seq_idx, pos, c_kv, k_rope, rope_table, rope_len, T,
        dev_status);
    return cudaGetLastError();
}

}  // namespace mla
