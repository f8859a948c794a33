// The two per-head projections of the absorbed path on tcgen05 tensor cores.
//
//  absorb:  q_abs[t, h, :] = (W^UK_h)^T q_nope[t, h, :]          (512 = 128 x 512^T)
//           W^UK is folded into the query so scores are taken against the cached
//           latent ("两张账" page, "第一张账"; MLA explainer 2.2.1.1).  q^R is rotated at
//           the query position in fp32 exactly as the cache append rotates k^R
//           (explainer 2.2.2).
//  finish:  o_lat[t, h, :] = merge of the decode's segment partials (log-sum-exp),
//           out[t, h, :]  = W^UV_h o_lat[t, h, :]                 (128 = 128 x 512)
//           W^UV is applied after the aggregation in latent space ("两张账" page).
//
// One CTA per (head, block of up to 64 query rows t).  The head's weight matrix
// [128 x 512] bf16 lands in shared memory as eight TMA boxes through a 3-D view
// (column within a 64-column chunk, row, chunk), one [128 x 64] chunk each, with
// the 128-byte swizzle.  The token-side operand is staged by the CTA's
// threads into the same swizzled layout; one thread issues the MMAs (M = 128,
// N = token block, K = 16) with the accumulator in TMEM; four warps read it back.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace proj {

constexpr int kThreads = 256;
constexpr int kTokBlock = 64;                // query rows per CTA
constexpr int kWChunkBytes = 128 * 64 * 2;   // [128 rows x 64 columns] bf16 = 16 KB
constexpr int kWBytes = 8 * kWChunkBytes;    // one head's weight matrix, 128 KB
constexpr int kOffW = 0;
constexpr int kOffB = kWBytes;               // token operand, up to 64 x 512 bf16 (64 KB)
constexpr int kOffBar = kOffB + kTokBlock * 512 * 2;
constexpr int kSmemBytes = kOffBar + 64;
constexpr int kFinThreads = 512;             // finish: 16 warps share the row merges
constexpr int kFinSmemBytes = kOffBar + 1024;
static_assert(kTokBlock <= 64, "finish keeps at most 64 sequences per CTA in its tables");
constexpr uint64_t kLimitNs = 2000000000ull;

// One head's weights as eight [128 x 64] boxes (one per 64-column chunk): several boxes in flight
// stream far faster through the TMA unit than one 128 KB box.
__device__ __forceinline__ void tma_load_w(uint32_t dst, const CUtensorMap* map, int head, uint64_t* bar) {
#pragma unroll
    for (int c = 0; c < 8; ++c) tma_load_3d(dst + c * kWChunkBytes, map, 0, head * 128, c, bar);
}

// 16-byte unit u (0..7) of row r in a 128-byte swizzled row of a [rows x 64] chunk
__device__ __forceinline__ uint32_t swz(int r, int u) { return static_cast<uint32_t>(r * 128 + ((u ^ (r & 7)) << 4)); }

// ------------------------------------------------------------------ absorb

__global__ void __launch_bounds__(kThreads, 1) absorb_tc_kernel(
    const __grid_constant__ CUtensorMap wuk_map, const uint16_t* __restrict__ q_nope,
    const uint16_t* __restrict__ q_rope, const int32_t* __restrict__ pos, const float* __restrict__ rope_table,
    int64_t rope_len, int T, int H, uint16_t* __restrict__ q_out, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);  // 0: weights, 1: MMA done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int t0 = blockIdx.y * kTokBlock;
    const int nt = min(kTokBlock, T - t0);
    const int NT = (nt + 15) & ~15;  // MMA N (multiple of 16)
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        prefetch_tmap(&wuk_map);
        mbar_arrive_expect_tx(&bars[0], kWBytes);
        tma_load_w(sbase + kOffW, &wuk_map, h, &bars[0]);
    }
    // B operand: q_nope rows t (N) x 128 (K), two swizzled [NT x 64] chunks; rows >= nt are zero.
    // All of a thread's loads are issued before any store (one memory latency, not four).
    {
        constexpr int kIt = kTokBlock * 16 / kThreads;
        uint4 v[kIt];
#pragma unroll
        for (int k = 0; k < kIt; ++k) {
            const int idx = tid + k * kThreads, r = idx >> 4, u16 = idx & 15;  // 16 units of 16 B per row
            v[k] = make_uint4(0, 0, 0, 0);
            if (r < nt) v[k] = reinterpret_cast<const uint4*>(q_nope + (static_cast<int64_t>(t0 + r) * H + h) * kDh)[u16];
        }
#pragma unroll
        for (int k = 0; k < kIt; ++k) {
            const int idx = tid + k * kThreads, r = idx >> 4, u16 = idx & 15;
            if (r < NT) *reinterpret_cast<uint4*>(smem + kOffB + (u16 >> 3) * NT * 128 + swz(r, u16 & 7)) = v[k];
        }
    }
    fence_proxy_async_cta();
    __syncthreads();
    bool ok = true;
    if (tid == 0) {
        ok = mbar_wait(&bars[0], 0, &never, kLimitNs);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, NT, true, false);
            // A = W^UK_h^T (M = latent c, K = i): MN-major; M block mb spans chunks 2mb, 2mb+1
            const uint64_t a0 = sdesc_sw128(sbase + kOffW, kWChunkBytes, 1024);
            const uint64_t b0 = sdesc_sw128(sbase + kOffB, 16, 1024);
            for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t ad = a0 + static_cast<uint64_t>((mb * 2 * kWChunkBytes + k * 2048) >> 4);
                    const uint64_t bd = b0 + static_cast<uint64_t>(((k >> 2) * NT * 128 + (k & 3) * 32) >> 4);
                    mma_ss(tmem + mb * NT, ad, bd, idesc, k > 0 ? 1u : 0u);
                }
            }
            mma_commit(smem_u32(&bars[1]));
        } else {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    // RoPE part on CUDA cores meanwhile: nt tokens x 32 pairs (same arithmetic as the cache append).
    // Thread tid owns pair tid % 32 of tokens tid / 32 + 8 k; the loads of all its tokens go out together.
    {
        constexpr int kIt = kTokBlock * (kDr / 2) / kThreads;
        const int pr = tid & 31;
        uint32_t xr[kIt];
        int32_t pp[kIt];
#pragma unroll
        for (int k = 0; k < kIt; ++k) {
            const int t = (tid >> 5) + k * (kThreads / 32);
            xr[k] = 0u;
            pp[k] = 0;
            if (t < nt) {
                xr[k] = reinterpret_cast<const uint32_t*>(q_rope + (static_cast<int64_t>(t0 + t) * H + h) * kDr)[pr];
                if (pos) pp[k] = pos[t0 + t];
            }
        }
        float2 cs[kIt];
#pragma unroll
        for (int k = 0; k < kIt; ++k) {
            const int t = (tid >> 5) + k * (kThreads / 32);
            cs[k] = make_float2(1.f, 0.f);
            if (t < nt && pos && pp[k] >= 0 && pp[k] < rope_len)
                cs[k] = reinterpret_cast<const float2*>(rope_table + static_cast<int64_t>(pp[k]) * kDr)[pr];
        }
#pragma unroll
        for (int k = 0; k < kIt; ++k) {
            const int t = (tid >> 5) + k * (kThreads / 32);
            if (t >= nt) continue;
            uint32_t y = xr[k];
            if (pos) {
                if (pp[k] < 0 || pp[k] >= rope_len) {
                    report(dev_status, MLA_DEVERR_POS_RANGE);
                    continue;
                }
                const float x0 = bf16_to_f32(static_cast<uint16_t>(xr[k] & 0xFFFFu));
                const float x1 = bf16_to_f32(static_cast<uint16_t>(xr[k] >> 16));
                y = pack_bf16x2(__fsub_rn(__fmul_rn(x0, cs[k].x), __fmul_rn(x1, cs[k].y)),
                                __fadd_rn(__fmul_rn(x0, cs[k].y), __fmul_rn(x1, cs[k].x)));
            }
            reinterpret_cast<uint32_t*>(q_out + (static_cast<int64_t>(t0 + t) * H + h) * kRow + kDc)[pr] = y;
        }
    }
    ok = __syncthreads_and(ok);
    if (warp < 4 && ok) {
        // D block mb: lane = latent column 128 mb + 32 warp + lane, column = token
        const bool done = mbar_wait(&bars[1], 0, &never, kLimitNs);
        __syncwarp();
        tc_fence_after();
        if (__all_sync(0xffffffffu, done)) {
            for (int mb = 0; mb < 4; ++mb) {
                const int c = 128 * mb + 32 * warp + lane;
                for (int j0 = 0; j0 < NT; j0 += 32) {
                    uint32_t v[32];
                    const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + mb * NT + j0;
                    if (NT - j0 >= 32) tmem_ld32(ta, v);
                    else tmem_ld16(ta, v);  // NT is a multiple of 16
                    tmem_wait_ld();
                    const int jn = min(32, nt - j0);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < jn)
                            q_out[(static_cast<int64_t>(t0 + j0 + j) * H + h) * kRow + c] =
                                f32_to_bf16_rne(__uint_as_float(v[j]));
                }
            }
        } else if (lane == 0) {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ finish

__device__ __forceinline__ int seq_tiles(const int32_t* kv_len, const int64_t* seq_block, int64_t cap_blocks, int n_q,
                                         int b) {
    const int L = kv_len[b];
    if (L < n_q) return 0;
    const int64_t s = seq_block[b];
    const int nt = (L + kBlockTokens - 1) / kBlockTokens;
    if (s < 0 || s + nt > cap_blocks) return 0;
    return nt;
}

__global__ void __launch_bounds__(kFinThreads, 1) finish_tc_kernel(
    const __grid_constant__ CUtensorMap wuv_map, const float* __restrict__ o_part, const float2* __restrict__ ml_part,
    const int32_t* __restrict__ kv_len, const int64_t* __restrict__ seq_block, int64_t cap_blocks, int B, int n_q,
    int H, int P_g, int slots, uint16_t* __restrict__ out, float* __restrict__ lse_out, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 16);
    int* red = reinterpret_cast<int*>(smem + kOffBar + 32);       // [2][16] per-warp partial sums
    int* seq_nt = reinterpret_cast<int*>(smem + kOffBar + 256);   // tiles of this CTA's sequences
    int* seq_ts = reinterpret_cast<int*>(smem + kOffBar + 512);   // and the tiles before each
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int T = B * n_q;
    const int t0 = blockIdx.y * kTokBlock;
    const int nt = min(kTokBlock, T - t0);
    const int NT = (nt + 15) & ~15;
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        prefetch_tmap(&wuv_map);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], kWBytes);
        tma_load_w(sbase + kOffW, &wuv_map, h, &bars[0]);
    }
    // Tile counts: Nt over all sequences (the decode's range split depends on it), `pre` over the
    // sequences before this CTA's first one, and each of this CTA's sequences (at most 64) in smem.
    const int b_lo = t0 / n_q, nb = (t0 + nt - 1) / n_q - b_lo + 1;
    {
        int s_all = 0, s_pre = 0;
        for (int b = tid; b < B; b += kFinThreads) {
            const int n = seq_tiles(kv_len, seq_block, cap_blocks, n_q, b);
            s_all += n;
            if (b < b_lo) s_pre += n;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s_all += __shfl_xor_sync(0xffffffffu, s_all, o);
            s_pre += __shfl_xor_sync(0xffffffffu, s_pre, o);
        }
        if (lane == 0) {
            red[warp] = s_all;
            red[16 + warp] = s_pre;
        }
        if (tid < nb) seq_nt[tid] = seq_tiles(kv_len, seq_block, cap_blocks, n_q, b_lo + tid);
    }
    __syncthreads();
    int Nt = 0;
    for (int w = 0; w < kFinThreads / 32; ++w) Nt += red[w];
    if (tid == 0) {
        int acc = 0;
        for (int w = 0; w < kFinThreads / 32; ++w) acc += red[16 + w];
        for (int i = 0; i < nb; ++i) {
            seq_ts[i] = acc;
            acc += seq_nt[i];
        }
    }
    __syncthreads();
    // merge: one warp per query row t; lane covers latent columns 16 lane .. 16 lane + 15.  The (m, l)
    // of up to 32 segments are read at once (one per lane), then the segments' O rows four at a time.
    for (int r = warp; r < NT; r += kFinThreads / 32) {
        float acc[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) acc[k] = 0.f;
        float z = 0.f, M = -CUDART_INF_F;
        if (r < nt) {
            const int tt = t0 + r;
            const int b = tt / n_q, j = tt % n_q;
            const int rr = j * H + h;
            const int g = rr / 128, row = rr % 128;
            const int ts = seq_ts[b - b_lo], ntb = seq_nt[b - b_lo];
            if (ntb > 0 && Nt > 0) {
                const int p_first = static_cast<int>((static_cast<int64_t>(ts + 1) * P_g - 1) / Nt);
                const int p_last = static_cast<int>((static_cast<int64_t>(ts + ntb) * P_g - 1) / Nt);
                const int64_t seg0 = static_cast<int64_t>(g) * slots + b;  // slot of piece p: seg0 + p
                for (int base = p_first; base <= p_last; base += 32) {
                    const int p = base + lane;
                    float2 ml = make_float2(-CUDART_INF_F, 0.f);
                    if (p <= p_last) {
                        const int lo = static_cast<int>((static_cast<int64_t>(p) * Nt) / P_g);
                        const int hi = static_cast<int>((static_cast<int64_t>(p + 1) * Nt) / P_g);
                        if (max(lo, ts) < min(hi, ts + ntb)) ml = ml_part[(seg0 + p) * 128 + row];
                    }
                    float bm = ml.x;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
                    const float Mn = fmaxf(M, bm);
                    if (Mn == -CUDART_INF_F) continue;
                    const float sc = (M == -CUDART_INF_F) ? 0.f : exp2f(M - Mn);
#pragma unroll
                    for (int k = 0; k < 16; ++k) acc[k] *= sc;
                    const float w = (ml.x == -CUDART_INF_F) ? 0.f : exp2f(ml.x - Mn);
                    float zl = w * ml.y;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) zl += __shfl_xor_sync(0xffffffffu, zl, o);
                    z = z * sc + zl;
                    M = Mn;
                    const int cnt = min(32, p_last - base + 1);
                    for (int i0 = 0; i0 < cnt; i0 += 4) {
                        float wi[4];
                        float4 v[4][4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            wi[u] = __shfl_sync(0xffffffffu, w, (i0 + u) & 31);
                            if (i0 + u >= cnt) wi[u] = 0.f;
                            if (wi[u] != 0.f) {
                                // segment partials: [column group of 4][128 rows] x float4
                                const float4* src = reinterpret_cast<const float4*>(o_part) +
                                                    ((seg0 + base + i0 + u) * 128 + 4 * lane) * 128 + row;
#pragma unroll
                                for (int k = 0; k < 4; ++k) v[u][k] = src[k * 128];
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (wi[u] == 0.f) continue;
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                acc[4 * k] = fmaf(wi[u], v[u][k].x, acc[4 * k]);
                                acc[4 * k + 1] = fmaf(wi[u], v[u][k].y, acc[4 * k + 1]);
                                acc[4 * k + 2] = fmaf(wi[u], v[u][k].z, acc[4 * k + 2]);
                                acc[4 * k + 3] = fmaf(wi[u], v[u][k].w, acc[4 * k + 3]);
                            }
                        }
                    }
                }
            }
            if (lane == 0 && lse_out)
                lse_out[static_cast<int64_t>(tt) * H + h] =
                    (z > 0.f) ? (M + log2f(z)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
        const float inv = (z > 0.f) ? 1.f / z : 0.f;
        // latent columns 16 lane .. +15 = chunk lane / 4, 16-byte units 2 (lane % 4), +1
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(acc[2 * k] * inv, acc[2 * k + 1] * inv);
        const int chunk = lane >> 2, u = 2 * (lane & 3);
        uint8_t* base = smem + kOffB + chunk * NT * 128;
        *reinterpret_cast<uint4*>(base + swz(r, u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(base + swz(r, u + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    fence_proxy_async_cta();
    __syncthreads();
    bool ok = true;
    if (tid == 0) {
        ok = mbar_wait(&bars[0], 0, &never, kLimitNs);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
            const uint64_t a0 = sdesc_sw128(sbase + kOffW, 16, 1024);
            const uint64_t b0 = sdesc_sw128(sbase + kOffB, 16, 1024);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const uint64_t ad = a0 + static_cast<uint64_t>(((k >> 2) * kWChunkBytes + (k & 3) * 32) >> 4);
                const uint64_t bd = b0 + static_cast<uint64_t>(((k >> 2) * NT * 128 + (k & 3) * 32) >> 4);
                mma_ss(tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
            }
            mma_commit(smem_u32(&bars[1]));
        } else {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    ok = __syncthreads_and(ok);
    if (warp < 4 && ok) {
        const bool done = mbar_wait(&bars[1], 0, &never, kLimitNs);
        __syncwarp();
        tc_fence_after();
        if (__all_sync(0xffffffffu, done)) {
            const int d = 32 * warp + lane;  // output row of W^UV_h
            for (int j0 = 0; j0 < NT; j0 += 32) {
                uint32_t v[32];
                const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + j0;
                if (NT - j0 >= 32) tmem_ld32(ta, v);
                else tmem_ld16(ta, v);  // NT is a multiple of 16
                tmem_wait_ld();
                const int jn = min(32, nt - j0);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < jn)
                        out[(static_cast<int64_t>(t0 + j0 + j) * H + h) * kDh + d] =
                            f32_to_bf16_rne(__uint_as_float(v[j]));
            }
        } else if (lane == 0) {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// W [H, 128, 512] bf16 viewed as (column within a 64-column chunk, row, chunk); one box = one chunk of a head.
bool weight_map(CUtensorMap* map, const uint16_t* W, int H) {
    auto encode = encode_fn();
    if (!encode) return false;
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(H) * 128, 8};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDc) * 2, 128};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(W), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace proj

cudaError_t launch_absorb_tc(const uint16_t* q_nope, const uint16_t* q_rope, const int32_t* pos, const uint16_t* W_UK,
                             const float* rope_table, int64_t rope_len, int T, int H, uint16_t* q_out,
                             int32_t* dev_status, cudaStream_t stream) {
    CUtensorMap map;
    if (!proj::weight_map(&map, W_UK, H)) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(proj::absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         proj::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(H, (T + proj::kTokBlock - 1) / proj::kTokBlock);
    proj::absorb_tc_kernel<<<grid, proj::kThreads, proj::kSmemBytes, stream>>>(map, q_nope, q_rope, pos, rope_table,
                                                                               rope_len, T, H, q_out, dev_status);
    return cudaGetLastError();
}

cudaError_t launch_finish_tc(const float* o_part, const float2* ml_part, const int32_t* kv_len, const int64_t* seq_block,
                             int64_t cap_blocks, int B, int n_q, int H, int P_g, int slots, const uint16_t* W_UV,
                             uint16_t* out, float* lse_out, int32_t* dev_status, cudaStream_t stream) {
    CUtensorMap map;
    if (!proj::weight_map(&map, W_UV, H)) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(proj::finish_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         proj::kFinSmemBytes);
    if (e != cudaSuccess) return e;
    const int T = B * n_q;
    dim3 grid(H, (T + proj::kTokBlock - 1) / proj::kTokBlock);
    proj::finish_tc_kernel<<<grid, proj::kFinThreads, proj::kFinSmemBytes, stream>>>(
        map, o_part, ml_part, kv_len, seq_block, cap_blocks, B, n_q, H, P_g, slots, out, lse_out, dev_status);
    return cudaGetLastError();
}

}  // namespace mla
