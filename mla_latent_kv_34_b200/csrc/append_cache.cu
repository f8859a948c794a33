// Cache append: one warp per new token writes its packed row
// [c^KV (512, copied) | R_pos k^R (64, rotated in fp32)].
//
// Only c^KV and the RoPE'd shared key are cached ("两张账" page, "第一张账";
// MLA explainer section 2.2.2: the key's position part is cached already
// rotated).  The rotation uses separately rounded fp32 products and sums
// (__fmul_rn / __fadd_rn / __fsub_rn are never contracted into an FMA), then
// round-to-nearest-even to bf16, so the stored bits are reproducible.
#include "mla_internal.cuh"

namespace mla {

__global__ void __launch_bounds__(256) append_cache_kernel(
    uint16_t* __restrict__ cache, int64_t cap, const int64_t* __restrict__ seq_start,
    const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos,
    const uint16_t* __restrict__ c_kv, const uint16_t* __restrict__ k_rope,
    const float* __restrict__ rope_table, int64_t rope_len, int T, int32_t* dev_status) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int32_t p = pos[warp];
    const int64_t row = seq_start[seq_idx[warp]] + static_cast<int64_t>(p);
    if (p < 0 || row < 0 || row >= cap) {
        if (lane == 0) report(dev_status, MLA_DEVERR_ROW_RANGE);
        return;
    }
    if (p >= rope_len) {
        if (lane == 0) report(dev_status, MLA_DEVERR_POS_RANGE);
        return;
    }
    uint16_t* dst = cache + row * kRow;
    // latent: 512 bf16 = 1024 B = 64 x 16 B; two 16-byte vectors per lane
    const uint4* src4 = reinterpret_cast<const uint4*>(c_kv + static_cast<int64_t>(warp) * kDc);
    uint4* dst4 = reinterpret_cast<uint4*>(dst);
    dst4[lane] = src4[lane];
    dst4[lane + 32] = src4[lane + 32];
    // RoPE pair `lane`: dims (2 lane, 2 lane + 1)
    const uint32_t xr = reinterpret_cast<const uint32_t*>(k_rope + static_cast<int64_t>(warp) * kDr)[lane];
    const float x0 = bf16_to_f32(static_cast<uint16_t>(xr & 0xFFFFu));
    const float x1 = bf16_to_f32(static_cast<uint16_t>(xr >> 16));
    const float2 cs = reinterpret_cast<const float2*>(rope_table + static_cast<int64_t>(p) * kDr)[lane];
    const float y0 = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y));
    const float y1 = __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x));
    reinterpret_cast<uint32_t*>(dst + kDc)[lane] = pack_bf16x2(y0, y1);
}

cudaError_t launch_append_cache(uint16_t* cache, int64_t cap, const int64_t* seq_start, const int32_t* seq_idx,
                                const int32_t* pos, const uint16_t* c_kv, const uint16_t* k_rope,
                                const float* rope_table, int64_t rope_len, int T, int32_t* dev_status,
                                cudaStream_t stream) {
    const int threads = 256;
    const int64_t blocks = (static_cast<int64_t>(T) * 32 + threads - 1) / threads;
    append_cache_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        cache, cap, seq_start, seq_idx, pos, c_kv, k_rope, rope_table, rope_len, T, dev_status);
    return cudaGetLastError();
}

}  // namespace mla
