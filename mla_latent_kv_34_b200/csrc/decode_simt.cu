// Split-KV absorbed decode on CUDA cores (the general-shape path).
//
// For each (sequence b, block of 16 query rows, split s) the CTA streams the
// split's cached rows [c^KV | k^R] through shared memory 32 tokens at a time,
// scores them against the absorbed queries (content . latent + rope . rope),
// keeps an online softmax in fp32 (log2 domain) and accumulates the latent
// output o_lat = sum_t P_t c_t ("两张账" page, "第一张账": aggregation stays in
// latent space; MLA explainer section 2.2.2: concatenated content/position
// inner product).  Each split writes its normalised partial and its
// log-sum-exp; the merge and W^UV are applied by the combine kernel.
#include <math_constants.h>

#include "mla_internal.cuh"

namespace mla {

constexpr int kSimtRows = 16;
constexpr int kSimtTok = 32;
constexpr int kKvWords = kRow / 2 + 1;  // 289 words per smem row: odd stride, no bank conflicts

struct SimtSmem {
    float q[kSimtRows][kRow];
    uint32_t kv[kSimtTok][kKvWords];
    float p[kSimtRows][kSimtTok];
    float m[kSimtRows];
    float l[kSimtRows];
    float alpha[kSimtRows];
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(256) decode_simt_kernel(
    const uint16_t* __restrict__ q, const uint8_t* __restrict__ cache, int64_t cap_blocks,
    const int32_t* __restrict__ block_table, int max_blocks, const int32_t* __restrict__ kv_len, int n_q, int H,
    float scale_log2, int S, float* __restrict__ o_part, float* __restrict__ lse_part, int32_t* dev_status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
    const int s = blockIdx.x, b = blockIdx.z;
    const int R = n_q * H;
    const int r0 = blockIdx.y * kSimtRows;
    if (r0 >= R) return;
    const int nrows = min(kSimtRows, R - r0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = kv_len[b];
    const int32_t* tab = block_table + static_cast<int64_t>(b) * max_blocks;
    if (L < n_q) {
        if (tid == 0 && s == 0 && blockIdx.y == 0) report(dev_status, MLA_DEVERR_KV_LEN);
        return;
    }
    if ((L + kBlockTokens - 1) / kBlockTokens > max_blocks) {
        if (tid == 0 && s == 0 && blockIdx.y == 0) report(dev_status, MLA_DEVERR_ROW_RANGE);
        return;
    }
    const int chunk = (L + S - 1) / S;
    const int t_lo = s * chunk;
    const int t_hi = min(L, t_lo + chunk);

    // absorbed query rows of this block -> fp32 smem
    const uint16_t* qb = q + (static_cast<int64_t>(b) * R + r0) * kRow;
    for (int idx = tid; idx < kSimtRows * kRow; idx += blockDim.x) {
        const int r = idx / kRow;
        sm.q[r][idx % kRow] = (r < nrows) ? bf16_to_f32(qb[idx]) : 0.f;
    }
    if (tid < kSimtRows) {
        sm.m[tid] = -CUDART_INF_F;
        sm.l[tid] = 0.f;
    }
    // rows owned by this warp for the softmax, and their causal limit
    const int rA = 2 * warp, rB = 2 * warp + 1;
    const int limA = L - n_q + (r0 + rA) / H;  // last visible key of the row
    const int limB = L - n_q + (r0 + rB) / H;

    float acc[kSimtRows][2];
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) acc[r][0] = acc[r][1] = 0.f;

    for (int ts = t_lo; ts < t_hi; ts += kSimtTok) {
        __syncthreads();
        for (int idx = tid; idx < kSimtTok * (kRow / 2); idx += blockDim.x) {
            const int tk = idx / (kRow / 2), w = idx % (kRow / 2);
            const int t = ts + tk;
            uint32_t v = 0u;
            if (t < t_hi) {
                int64_t e = tab[t / kBlockTokens];
                if (e < 0 || e >= cap_blocks) {  // outside the pool: reported, block 0 read instead
                    if (w == 0) report(dev_status, MLA_DEVERR_ROW_RANGE);
                    e = 0;
                }
                v = *reinterpret_cast<const uint32_t*>(cache + e * kBlockBytes + block_offset(t % kBlockTokens, 2 * w));
            }
            sm.kv[tk][w] = v;
        }
        __syncthreads();
        // scores: lane = token, two rows per warp
        float dA = 0.f, dB = 0.f;
        const uint32_t* kvrow = sm.kv[lane];
#pragma unroll 4
        for (int k2 = 0; k2 < kRow / 2; ++k2) {
            const uint32_t v = kvrow[k2];
            const float v0 = bf16_to_f32(v & 0xFFFFu), v1 = bf16_to_f32(v >> 16);
            dA = fmaf(sm.q[rA][2 * k2], v0, fmaf(sm.q[rA][2 * k2 + 1], v1, dA));
            dB = fmaf(sm.q[rB][2 * k2], v0, fmaf(sm.q[rB][2 * k2 + 1], v1, dB));
        }
        const int t = ts + lane;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const int r = which ? rB : rA;
            const int lim = which ? limB : limA;
            const bool valid = (r < nrows) && (t < t_hi) && (t <= lim);
            const float sc = valid ? (which ? dB : dA) * scale_log2 : -CUDART_INF_F;
            const float m_old = sm.m[r];
            const float m_new = fmaxf(m_old, warp_max(sc));
            const float p = (sc == -CUDART_INF_F) ? 0.f : exp2f(sc - m_new);
            const float alpha = (m_new == -CUDART_INF_F) ? 1.f : exp2f(m_old - m_new);
            const float psum = warp_sum(p);
            sm.p[r][lane] = p;
            __syncwarp();
            if (lane == 0) {
                sm.l[r] = sm.l[r] * alpha + psum;
                sm.m[r] = m_new;
                sm.alpha[r] = alpha;
            }
        }
        __syncthreads();
        // o_lat += P V, thread owns latent columns 2 tid, 2 tid + 1
#pragma unroll
        for (int r = 0; r < kSimtRows; ++r) {
            acc[r][0] *= sm.alpha[r];
            acc[r][1] *= sm.alpha[r];
        }
        for (int tk = 0; tk < kSimtTok; ++tk) {
            const uint32_t v = sm.kv[tk][tid];
            const float v0 = bf16_to_f32(v & 0xFFFFu), v1 = bf16_to_f32(v >> 16);
#pragma unroll
            for (int r = 0; r < kSimtRows; ++r) {
                const float p = sm.p[r][tk];
                acc[r][0] = fmaf(p, v0, acc[r][0]);
                acc[r][1] = fmaf(p, v1, acc[r][1]);
            }
        }
    }
    __syncthreads();
    const float ln2 = 0.69314718055994530942f;
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) {
        if (r >= nrows) break;
        const float l = sm.l[r];
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        float2 o = make_float2(acc[r][0] * inv, acc[r][1] * inv);
        const int64_t row = (static_cast<int64_t>(b) * R + r0 + r) * S + s;
        *reinterpret_cast<float2*>(o_part + row * kDc + 2 * tid) = o;
        if (tid == 0) lse_part[row] = (l > 0.f) ? (sm.m[r] + log2f(l)) * ln2 : -CUDART_INF_F;
    }
}

cudaError_t launch_decode_simt(const uint16_t* q, const uint8_t* cache, int64_t cap_blocks, const int32_t* block_table,
                               int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale, int splits,
                               float* o_part, float* lse_part, int32_t* dev_status, cudaStream_t stream) {
    const int R = n_q * H;
    dim3 grid(splits, (R + kSimtRows - 1) / kSimtRows, B);
    const size_t smem = sizeof(SimtSmem);
    cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const float scale_log2 = scale * 1.44269504088896340736f;
    decode_simt_kernel<<<grid, 256, smem, stream>>>(q, cache, cap_blocks, block_table, max_blocks, kv_len, n_q, H,
                                                    scale_log2, splits,
                                                    o_part, lse_part, dev_status);
    return cudaGetLastError();
}

}  // namespace mla
