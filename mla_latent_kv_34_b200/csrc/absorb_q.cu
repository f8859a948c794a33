// Query absorption: q_abs[t,h,:] = (W^UK_h)^T q_nope[t,h,:] and the RoPE'd q^R.
//
// W^UK is folded into the query so that q^C . k^C_t = q_abs . c_t^KV and the
// score is taken straight against the cached latent ("两张账" page, "第一张账";
// MLA explainer section 2.2.1.1 quoting the paper's absorption remark).  The
// decoupled query q^R is rotated at the query's position (explainer 2.2.2)
// with the same fp32 arithmetic as the cache append.
//
// CUDA-core kernel: one CTA per (head, 16-token block); W^UK_h is streamed
// once per CTA with 8-byte loads, q_nope of the block sits in shared memory.
#include "mla_internal.cuh"

namespace mla {

constexpr int kAbsorbTok = 16;

__global__ void __launch_bounds__(128) absorb_q_kernel(
    const uint16_t* __restrict__ q_nope, const uint16_t* __restrict__ q_rope,
    const int32_t* __restrict__ pos, const uint16_t* __restrict__ W_UK,
    const float* __restrict__ rope_table, int64_t rope_len, int T, int H,
    uint16_t* __restrict__ q_out, int32_t* dev_status) {
    __shared__ float qs[kAbsorbTok][kDh];
    const int h = blockIdx.x;
    const int t0 = blockIdx.y * kAbsorbTok;
    const int nt = min(kAbsorbTok, T - t0);
    const int tid = threadIdx.x;

    for (int idx = tid; idx < kAbsorbTok * kDh; idx += blockDim.x) {
        const int t = idx / kDh, i = idx % kDh;
        qs[t][i] = (t < nt) ? bf16_to_f32(q_nope[(static_cast<int64_t>(t0 + t) * H + h) * kDh + i]) : 0.f;
    }
    __syncthreads();

    float acc[kAbsorbTok][4];
#pragma unroll
    for (int t = 0; t < kAbsorbTok; ++t)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[t][k] = 0.f;

    const uint16_t* w = W_UK + static_cast<int64_t>(h) * kDh * kDc + 4 * tid;
    for (int i = 0; i < kDh; ++i) {
        const uint2 wv = *reinterpret_cast<const uint2*>(w + static_cast<int64_t>(i) * kDc);
        const float w0 = bf16_to_f32(wv.x & 0xFFFFu), w1 = bf16_to_f32(wv.x >> 16);
        const float w2 = bf16_to_f32(wv.y & 0xFFFFu), w3 = bf16_to_f32(wv.y >> 16);
#pragma unroll
        for (int t = 0; t < kAbsorbTok; ++t) {
            const float qv = qs[t][i];
            acc[t][0] = fmaf(qv, w0, acc[t][0]);
            acc[t][1] = fmaf(qv, w1, acc[t][1]);
            acc[t][2] = fmaf(qv, w2, acc[t][2]);
            acc[t][3] = fmaf(qv, w3, acc[t][3]);
        }
    }
#pragma unroll
    for (int t = 0; t < kAbsorbTok; ++t) {
        if (t < nt) {
            uint2 o;
            o.x = pack_bf16x2(acc[t][0], acc[t][1]);
            o.y = pack_bf16x2(acc[t][2], acc[t][3]);
            *reinterpret_cast<uint2*>(q_out + (static_cast<int64_t>(t0 + t) * H + h) * kRow + 4 * tid) = o;
        }
    }

    // RoPE part: nt tokens x 32 pairs
    for (int idx = tid; idx < nt * (kDr / 2); idx += blockDim.x) {
        const int t = idx / (kDr / 2), pr = idx % (kDr / 2);
        const int64_t qi = static_cast<int64_t>(t0 + t) * H + h;
        const uint32_t xr = reinterpret_cast<const uint32_t*>(q_rope + qi * kDr)[pr];
        uint32_t y = xr;
        if (pos) {
            const int32_t p = pos[t0 + t];
            if (p < 0 || p >= rope_len) {
                report(dev_status, MLA_DEVERR_POS_RANGE);
                continue;
            }
            const float x0 = bf16_to_f32(static_cast<uint16_t>(xr & 0xFFFFu));
            const float x1 = bf16_to_f32(static_cast<uint16_t>(xr >> 16));
            const float2 cs = reinterpret_cast<const float2*>(rope_table + static_cast<int64_t>(p) * kDr)[pr];
            y = pack_bf16x2(__fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y)),
                            __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x)));
        }
        reinterpret_cast<uint32_t*>(q_out + qi * kRow + kDc)[pr] = y;
    }
}

cudaError_t launch_absorb_q(const uint16_t* q_nope, const uint16_t* q_rope, const int32_t* pos,
                            const uint16_t* W_UK, const float* rope_table, int64_t rope_len, int T, int H,
                            uint16_t* q_out, int32_t* dev_status, cudaStream_t stream) {
    dim3 grid(H, (T + kAbsorbTok - 1) / kAbsorbTok);
    absorb_q_kernel<<<grid, 128, 0, stream>>>(q_nope, q_rope, pos, W_UK, rope_table, rope_len, T, H, q_out,
                                              dev_status);
    return cudaGetLastError();
}

}  // namespace mla
