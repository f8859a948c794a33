// Log-sum-exp merge of split-KV partials, optionally followed by W^UV.
//
// m = max_s lse_s, w_s = exp(lse_s - m), o = sum_s w_s o_s / sum_s w_s,
// lse = m + log sum_s w_s.  The merged latent output is then mapped out by the
// head's value up-projection, out = W^UV_h o_lat: W^UV is applied after the
// aggregation in latent space ("两张账" page, "第一张账").
//
// One CTA per (head, block of 8 query rows) so that W^UV_h is read once per
// block; the merged latent rows stay in shared memory.
#include <math_constants.h>

#include "mla_internal.cuh"

namespace mla {

constexpr int kCombTok = 8;

// out[t0 + t, h, d] = sum_c W_UV[h, d, c] * ol[t, c] for t < nt; 8 warps x 16 rows d.
__device__ void up_project_block(const float (*ol)[kDc], int nt, int t0, int h, int H,
                                 const uint16_t* __restrict__ W_UV, uint16_t* __restrict__ ob) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint16_t* Wh = W_UV + static_cast<int64_t>(h) * kDh * kDc;
    for (int dd = 0; dd < kDh / 8; ++dd) {
        const int d = warp * (kDh / 8) + dd;
        const uint4* wr = reinterpret_cast<const uint4*>(Wh + static_cast<int64_t>(d) * kDc);
        float part[kCombTok];
#pragma unroll
        for (int t = 0; t < kCombTok; ++t) part[t] = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint4 wv = wr[lane + 32 * half];  // 8 bf16: columns 8 (lane + 32 half) ..
            const int c0 = 8 * (lane + 32 * half);
            const uint32_t wws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float wa = bf16_to_f32(wws[k] & 0xFFFFu), wb = bf16_to_f32(wws[k] >> 16);
#pragma unroll
                for (int t = 0; t < kCombTok; ++t)
                    part[t] = fmaf(wa, ol[t][c0 + 2 * k], fmaf(wb, ol[t][c0 + 2 * k + 1], part[t]));
            }
        }
#pragma unroll
        for (int t = 0; t < kCombTok; ++t) {
            float v = part[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && t < nt) ob[(static_cast<int64_t>(t0 + t) * H + h) * kDh + d] = f32_to_bf16_rne(v);
        }
    }
}

__global__ void __launch_bounds__(256) combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part, int T, int H, int S,
    const uint16_t* __restrict__ W_UV, void* __restrict__ out, float* __restrict__ lse_out) {
    __shared__ float ol[kCombTok][kDc];
    const int h = blockIdx.x;
    const int t0 = blockIdx.y * kCombTok;
    const int nt = min(kCombTok, T - t0);
    const int tid = threadIdx.x;

    for (int t = 0; t < nt; ++t) {
        const int64_t th = static_cast<int64_t>(t0 + t) * H + h;
        const float* lp = lse_part + th * S;
        float m = -CUDART_INF_F;
        for (int s = 0; s < S; ++s) m = fmaxf(m, lp[s]);
        float o0 = 0.f, o1 = 0.f, z = 0.f;
        if (m != -CUDART_INF_F) {
            for (int s = 0; s < S; ++s) {
                const float w = expf(lp[s] - m);
                if (w == 0.f) continue;
                const float2 v = *reinterpret_cast<const float2*>(o_part + (th * S + s) * kDc + 2 * tid);
                o0 = fmaf(w, v.x, o0);
                o1 = fmaf(w, v.y, o1);
                z += w;
            }
        }
        const float inv = (z > 0.f) ? 1.f / z : 0.f;
        ol[t][2 * tid] = o0 * inv;
        ol[t][2 * tid + 1] = o1 * inv;
        if (tid == 0 && lse_out) lse_out[th] = (z > 0.f) ? m + logf(z) : -CUDART_INF_F;
    }
    if (W_UV == nullptr) {
        float* of = static_cast<float*>(out);
        for (int t = 0; t < nt; ++t) {
            const int64_t th = static_cast<int64_t>(t0 + t) * H + h;
            *reinterpret_cast<float2*>(of + th * kDc + 2 * tid) = make_float2(ol[t][2 * tid], ol[t][2 * tid + 1]);
        }
        return;
    }
    __syncthreads();
    up_project_block(ol, nt, t0, h, H, W_UV, static_cast<uint16_t*>(out));
}

cudaError_t launch_combine(const float* o_part, const float* lse_part, int T, int H, int splits,
                           const uint16_t* W_UV, void* out, float* lse_out, cudaStream_t stream) {
    dim3 grid(H, (T + kCombTok - 1) / kCombTok);
    combine_kernel<<<grid, 256, 0, stream>>>(o_part, lse_part, T, H, splits, W_UV, out, lse_out);
    return cudaGetLastError();
}


}  // namespace mla
