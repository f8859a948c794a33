// Naive-form attention for long prefill chunks on tcgen05 tensor cores.
//
//   k^C[t, h] = W^UK_h c_t,  v^C[t, h] = W^UV_h c_t               (decompression, bf16 workspace)
//   s_t = [q_nope ; R_p q^R] . [k^C[t, h] ; k^R_t] * scale,  t <= p   (query at position p)
//   out = sum_t softmax(s)_t v^C[t, h]
//
// The pages name this "naive" inference path beside the absorbed one ("两张账" page, "第一张账":
// the naive formula rebuilds k^C and v^C from c^KV).  Per (query, key, head) it costs 320 MACs
// against the absorbed form's 1088, but it first pays 2 * 128 * 512 MACs per (key, head) to
// rebuild the keys and values, so it does less arithmetic only once a key is shared by more than
// ~171 queries: causal chunks of more than ~340 tokens.
//
// Kernel 1 (decompress): persistent, one CTA per SM taking (head, 128-token cache block) units.  A
// block's eight latent chunks (already in the swizzled K-major operand layout in HBM) are the A
// operand; W^UK_h and W^UV_h chunks, stacked as one N = 256 B operand, stream through a four-stage
// ring that runs on across units.  D[token, 0..255] = [k^C | v^C] lands in one of two TMEM
// accumulators; each thread writes its token's two 256-byte rows while the next unit's MMAs run.
//
// Kernel 2 (attend): one CTA per (head, 128-query tile).  Q [128 x 192] sits in shared memory;
// key tiles (k^C by TMA from the workspace, k^R straight from the cache block's RoPE chunk, v^C by
// TMA) stream through two 80 KB stages.  S = Q K^T (M = N = 128, K = 192) goes to one of two TMEM
// buffers; four warps (one query row per thread) apply the causal mask and an online softmax with
// a stale maximum, write P as packed bf16 into TMEM, and O += P V runs with A from TMEM.
// Warp roles in both kernels: warps 0..3 epilogue / softmax, warp 4 lane 0 loads, warp 5 lane 0
// issues the MMAs.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace pf {

constexpr uint64_t kLimitNs = 2000000000ull;
constexpr int kChunk = 128 * 128;  // one [128 rows x 64 bf16] swizzled operand tile, 16 KB
constexpr int kThreads = 192;

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ float f32_of(uint32_t u) { return __uint_as_float(u); }

// Pool block of tile j of the sequence (its row of the block table); an entry outside the pool is
// reported and replaced by block 0, so no access leaves the pool.
__device__ __forceinline__ const uint8_t* tile_block(const uint8_t* cache, const int32_t* blocks, int64_t cap_blocks,
                                                     int j, int32_t* dev_status) {
    int64_t e = blocks[j];
    if (e < 0 || e >= cap_blocks) {
        report(dev_status, MLA_DEVERR_ROW_RANGE);
        e = 0;
    }
    return cache + e * static_cast<int64_t>(kBlockBytes);
}

// ------------------------------------------------------------------ decompression

constexpr int kDStageBytes = 3 * kChunk;  // cache chunk (A) + W^UK_h chunk + W^UV_h chunk (B, N = 256)
constexpr int kDStages = 4;
constexpr int kDOffBar = kDStages * kDStageBytes;
constexpr int kDSmemBytes = kDOffBar + 256;
constexpr int kDMaxCtas = 148;  // one persistent CTA per SM

// Persistent: CTA i takes the (head, block) units i, i + gridDim.x, ... (unit u = head u / nblk, block
// u % nblk, so consecutive units share a head's weights).  The ring of stages runs on across units, and
// the two 256-column TMEM accumulators alternate, so one unit's epilogue overlaps the next unit's loads
// and MMAs.
__global__ void __launch_bounds__(kThreads, 1) decompress_kernel(
    const __grid_constant__ CUtensorMap uk_map, const __grid_constant__ CUtensorMap uv_map,
    const uint8_t* __restrict__ cache, int64_t cap_blocks, const int32_t* __restrict__ blocks, int L, int H,
    uint16_t* __restrict__ k_out,
    uint16_t* __restrict__ v_out, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDOffBar);
    uint64_t* empty = full + kDStages;
    uint64_t* acc_full = empty + kDStages;   // [2] the MMAs of a unit are done
    uint64_t* acc_empty = acc_full + 2;      // [2] the epilogue has read a unit's accumulator
    uint64_t* fin = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kDOffBar + 128);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kDOffBar + 136);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nblk = (L + kBlockTokens - 1) / kBlockTokens;
    const int units = H * nblk;
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < kDStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 128);
        }
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr int KC = kDc / 64;  // latent chunks

    if (warp == 4 && lane == 0) {
        prefetch_tmap(&uk_map);
        prefetch_tmap(&uv_map);
        const uint64_t keep = l2_policy_evict_last();  // every head's unit reads this block
        uint32_t nc = 0;                                 // stages filled
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
            const int h = u / nblk, blk = u % nblk;
            const uint8_t* src = tile_block(cache, blocks, cap_blocks, blk, dev_status);
            for (int c = 0; c < KC; ++c, ++nc) {
                const uint32_t s = nc % kDStages, n = nc / kDStages;
                if (n > 0 && !mbar_wait(&empty[s], (n - 1) & 1u, abort_flag, kLimitNs)) {
                    ok = false;
                    break;
                }
                const uint32_t st = sbase + s * kDStageBytes;
                mbar_arrive_expect_tx(&full[s], kDStageBytes);
                bulk_load_hint(st, src + c * kBlockChunk, kChunk, &full[s], keep);
                tma_load_2d(st + kChunk, &uk_map, c * 64, h * 128, &full[s]);
                tma_load_2d(st + 2 * kChunk, &uv_map, c * 64, h * 128, &full[s]);
            }
        }
        if (!ok) {
            *abort_flag = 1;
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
        // let every issued copy land before the CTA can exit
        for (uint32_t i = (nc > kDStages ? nc - kDStages : 0); i < nc; ++i)
            mbar_wait(&full[i % kDStages], (i / kDStages) & 1u, &never, kLimitNs);
    } else if (warp == 5 && lane == 0) {
        // D[token, 0..127] = k^C, D[token, 128..255] = v^C: A = latent chunk (M = 128 tokens),
        // B = [W^UK_h ; W^UV_h] rows (N = 256), both K-major; accumulator ab = unit count & 1
        constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
        uint32_t nc = 0, i = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
            const uint32_t ab = i & 1u;
            ok = mbar_wait(&acc_empty[ab], ((i >> 1) & 1u) ^ 1u, abort_flag, kLimitNs);
            tc_fence_after();
            for (int c = 0; ok && c < KC; ++c, ++nc) {
                const uint32_t s = nc % kDStages, n = nc / kDStages;
                ok = mbar_wait(&full[s], n & 1u, abort_flag, kLimitNs);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = sbase + s * kDStageBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem + 256 * ab, sdesc_sw128(st + kk * 32, 16, 1024),
                           sdesc_sw128(st + kChunk + kk * 32, 16, 1024), idesc, (c > 0 || kk > 0) ? 1u : 0u);
                mma_commit(smem_u32(&empty[s]));
            }
            if (ok) mma_commit(smem_u32(&acc_full[ab]));
        }
        if (!ok) {
            *abort_flag = 1;
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
        mma_commit(smem_u32(fin));  // TMEM is freed only once every MMA issued above is done
    } else if (warp < 4) {
        uint32_t i = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++i) {
            const int h = u / nblk, blk = u % nblk;
            const uint32_t ab = i & 1u;
            const bool ok = mbar_wait(&acc_full[ab], (i >> 1) & 1u, abort_flag, kLimitNs);
            __syncwarp();
            tc_fence_after();
            if (!__all_sync(0xffffffffu, ok) || *abort_flag) {
                if (lane == 0) {
                    *abort_flag = 1;
                    report(dev_status, MLA_DEVERR_TIMEOUT);
                }
                break;
            }
            const int t = blk * kBlockTokens + 32 * warp + lane;  // token of this TMEM lane
            const bool valid = t < L;
            for (int half = 0; half < 2; ++half) {
                uint16_t* dst = (half == 0 ? k_out : v_out) + (static_cast<int64_t>(t) * H + h) * kDh;
                for (int j0 = 0; j0 < kDh; j0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + 256 * ab + (static_cast<uint32_t>(32 * warp) << 16) + 128 * half + j0, v);
                    tmem_wait_ld();
                    if (valid) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + j0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            d4[q] = make_uint4(pack_bf16x2(f32_of(v[8 * q]), f32_of(v[8 * q + 1])),
                                               pack_bf16x2(f32_of(v[8 * q + 2]), f32_of(v[8 * q + 3])),
                                               pack_bf16x2(f32_of(v[8 * q + 4]), f32_of(v[8 * q + 5])),
                                               pack_bf16x2(f32_of(v[8 * q + 6]), f32_of(v[8 * q + 7])));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        mbar_wait(fin, 0, &never, kLimitNs);
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ attention

constexpr int kQBytes = 3 * kChunk;                 // Q tile [128 x 192]: q_nope 0..127 | R_p q^R
constexpr int kKBytes = 3 * kChunk;                 // key tile [128 x 192]: k^C 0..127 | k^R
constexpr int kVBytes = 2 * kChunk;                 // value tile [128 keys x 128] (MN-major B)
constexpr int kAStageBytes = kKBytes + kVBytes;     // 80 KB
constexpr int kAStages = 2;
constexpr int kAOffStage = kQBytes;
constexpr int kAOffBar = kAOffStage + kAStages * kAStageBytes;
constexpr int kASmemBytes = kAOffBar + 256;
constexpr uint32_t kColS = 0;    // two 128-column score buffers
constexpr uint32_t kColO = 256;  // O, 128 fp32 columns
constexpr uint32_t kColP = 384;  // P, 64 columns of packed bf16 pairs (A operand of P V)
constexpr float kRescaleLog2 = 8.f;
static_assert(kASmemBytes <= 232448, "shared memory");

// barrier indices
enum { kBKvFull = 0, kBKvEmpty = 2, kBSFull = 4, kBSEmpty = 6, kBQReady = 8, kBPFull = 9, kBPEmpty = 10,
       kBODone = 11, kBFin = 12, kBCount = 13 };

__global__ void __launch_bounds__(kThreads, 1) attend_kernel(
    const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
    const uint8_t* __restrict__ cache, int64_t cap_blocks, const int32_t* __restrict__ blocks,
    const uint16_t* __restrict__ q_nope,
    const uint16_t* __restrict__ q_rope, const float* __restrict__ rope_table, int L, int n, int H, float scale_log2,
    uint16_t* __restrict__ out, float* __restrict__ lse_out, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kAOffBar + 8 * kBCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAOffBar + 8 * kBCount + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int n0 = blockIdx.y * 128;
    const int nq = min(128, n - n0);
    const int pmax = L - n + n0 + nq - 1;  // position of the tile's last query
    const int ntiles = pmax / kBlockTokens + 1;
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBKvFull + s], 1);
            mbar_init(&bars[kBKvEmpty + s], 1);
            mbar_init(&bars[kBSFull + s], 1);
            mbar_init(&bars[kBSEmpty + s], 128);
        }
        mbar_init(&bars[kBQReady], 128);
        mbar_init(&bars[kBPFull], 128);
        mbar_init(&bars[kBPEmpty], 1);
        mbar_init(&bars[kBODone], 1);
        mbar_init(&bars[kBFin], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&k_map);
            prefetch_tmap(&v_map);
            const uint64_t keep = l2_policy_evict_last();  // other query tiles of this head read it too
            for (int j = 0; j < ntiles; ++j) {
                const int s = j & 1, u = j >> 1;
                if (u > 0 && !mbar_wait(&bars[kBKvEmpty + s], (u - 1) & 1, abort_flag, kLimitNs)) {
                    *abort_flag = 1;
                    report(dev_status, MLA_DEVERR_TIMEOUT);
                    break;
                }
                const uint32_t st = sbase + kAOffStage + s * kAStageBytes;
                uint64_t* fb = &bars[kBKvFull + s];
                mbar_arrive_expect_tx(fb, kAStageBytes);
                tma_load_3d(st, &k_map, 0, h, kBlockTokens * j, fb);
                tma_load_3d(st + kChunk, &k_map, 64, h, kBlockTokens * j, fb);
                bulk_load_hint(st + 2 * kChunk, tile_block(cache, blocks, cap_blocks, j, dev_status) + 8 * kBlockChunk,
                               kChunk, fb, keep);
                tma_load_3d(st + kKBytes, &v_map, 0, h, kBlockTokens * j, fb);
                tma_load_3d(st + kKBytes + kChunk, &v_map, 64, h, kBlockTokens * j, fb);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
            const uint64_t q_desc = sdesc_sw128(sbase, 16, 1024);
            bool ok = mbar_wait(&bars[kBQReady], 0, abort_flag, kLimitNs);
            // O += P(i) V(i): A = P from TMEM (8 columns per 16 keys), B = V MN-major (16 KB atoms)
            auto pv = [&](int i) -> bool {
                if (!mbar_wait(&bars[kBPFull], i & 1, abort_flag, kLimitNs)) return false;
                tc_fence_after();
                const uint64_t vd = sdesc_sw128(sbase + kAOffStage + (i & 1) * kAStageBytes + kKBytes, kChunk, 1024);
#pragma unroll
                for (int kk = 0; kk < kBlockTokens / 16; ++kk)
                    mma_ts(tmem + kColO, tmem + kColP + 8 * kk, vd + ((kk * 2048) >> 4), idesc_o,
                           (i > 0 || kk > 0) ? 1u : 0u);
                mma_commit(smem_u32(&bars[kBPEmpty]));
                mma_commit(smem_u32(&bars[kBKvEmpty + (i & 1)]));
                return true;
            };
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j & 1, u = j >> 1;
                ok = mbar_wait(&bars[kBKvFull + s], u & 1, abort_flag, kLimitNs);
                if (ok && u > 0) ok = mbar_wait(&bars[kBSEmpty + s], (u - 1) & 1, abort_flag, kLimitNs);
                if (!ok) break;
                tc_fence_after();
                const uint64_t kd = sdesc_sw128(sbase + kAOffStage + s * kAStageBytes, 16, 1024);
#pragma unroll
                for (int c = 0; c < 3; ++c)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t off = static_cast<uint64_t>((c * kChunk + kk * 32) >> 4);
                        mma_ss(tmem + kColS + 128 * s, q_desc + off, kd + off, idesc_s, (c > 0 || kk > 0) ? 1u : 0u);
                    }
                mma_commit(smem_u32(&bars[kBSFull + s]));
                if (j > 0) ok = pv(j - 1);
            }
            if (ok) ok = pv(ntiles - 1);
            if (!ok) {
                *abort_flag = 1;
                report(dev_status, MLA_DEVERR_TIMEOUT);
            }
            mma_commit(smem_u32(&bars[kBODone]));  // fires once every MMA issued above has completed
        }
    } else {
        // ---- softmax and epilogue: thread r owns query row n0 + r (TMEM lane r)
        const int r = tid;
        const int qi = n0 + r;
        const bool row_ok = r < nq;
        const int p = L - n + qi;  // the query's position; keys 0..p are visible
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        // Q row -> shared memory: q_nope into chunks 0-1, R_p q^R (fp32, as mla_absorb_q) into chunk 2
        {
            uint8_t* qrow = smem + r * 128;
            const uint4* qn4 = reinterpret_cast<const uint4*>(q_nope + (static_cast<int64_t>(qi) * H + h) * kDh);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const uint4 x = row_ok ? qn4[u] : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(qrow + (u >> 3) * kChunk + (((u & 7) ^ (r & 7)) << 4)) = x;
            }
            const uint32_t* qr2 = reinterpret_cast<const uint32_t*>(q_rope + (static_cast<int64_t>(qi) * H + h) * kDr);
            const float2* cs = reinterpret_cast<const float2*>(rope_table + static_cast<int64_t>(row_ok ? p : 0) * kDr);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uint32_t y[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int pr = 4 * u + k;  // RoPE pair (2 pr, 2 pr + 1)
                    y[k] = 0u;
                    if (row_ok) {
                        const uint32_t xr = qr2[pr];
                        const float x0 = bf16_to_f32(static_cast<uint16_t>(xr & 0xFFFFu));
                        const float x1 = bf16_to_f32(static_cast<uint16_t>(xr >> 16));
                        const float2 c = cs[pr];
                        y[k] = pack_bf16x2(__fsub_rn(__fmul_rn(x0, c.x), __fmul_rn(x1, c.y)),
                                           __fadd_rn(__fmul_rn(x0, c.y), __fmul_rn(x1, c.x)));
                    }
                }
                *reinterpret_cast<uint4*>(qrow + 2 * kChunk + ((u ^ (r & 7)) << 4)) = make_uint4(y[0], y[1], y[2], y[3]);
            }
            fence_proxy_async_cta();
            mbar_arrive(&bars[kBQReady]);
        }
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            const int s = j & 1, u = j >> 1;
            ok = mbar_wait(&bars[kBSFull + s], u & 1, abort_flag, kLimitNs);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            float sv[128];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t a[32];
                tmem_ld32(t_lane + kColS + 128 * s + 32 * q, a);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) sv[32 * q + k] = __uint_as_float(a[k]);
            }
            tc_fence_before();
            mbar_arrive(&bars[kBSEmpty + s]);
            // causal mask (also covers keys past the sequence end and rows past the chunk end)
            const int nvis = row_ok ? p + 1 - kBlockTokens * j : 0;  // keys < nvis of this tile are visible
            float tmax = -CUDART_INF_F;
#pragma unroll
            for (int k = 0; k < 128; ++k) {
                sv[k] = k < nvis ? sv[k] : -CUDART_INF_F;
                tmax = fmaxf(tmax, sv[k]);
            }
            tmax *= scale_log2;
            // P(j-1) has been consumed and O holds every earlier tile once P V(j-1) completed
            if (j > 0) ok = mbar_wait(&bars[kBPEmpty], (j - 1) & 1, abort_flag, kLimitNs);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            if (tmax > m + kRescaleLog2) {
                const float alpha = (m == -CUDART_INF_F) ? 0.f : ex2_approx(m - tmax);
                l *= alpha;
                m = tmax;
                if (j > 0) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t a[32];
                        tmem_ld32(t_lane + kColO + 32 * q, a);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) a[k] = __float_as_uint(__uint_as_float(a[k]) * alpha);
                        tmem_st32(t_lane + kColO + 32 * q, a);
                    }
                }
            }
            const float mneg = (m == -CUDART_INF_F) ? 0.f : -m;
            float lsum = 0.f;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float p0 = ex2_approx(fmaf(sv[64 * q + 2 * k], scale_log2, mneg));
                    const float p1 = ex2_approx(fmaf(sv[64 * q + 2 * k + 1], scale_log2, mneg));
                    lsum += p0 + p1;
                    pk[k] = cvt_bf16x2(p0, p1);
                }
                tmem_st32(t_lane + kColP + 32 * q, pk);
            }
            l += lsum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[kBPFull]);
        }
        // epilogue: out = O / l, lse = (m + log2 l) ln 2
        const bool done_ok = mbar_wait(&bars[kBODone], 0, &never, kLimitNs);
        __syncwarp();
        tc_fence_after();
        if (__all_sync(0xffffffffu, ok && done_ok) && !*abort_flag) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<int64_t>(qi) * H + h) * kDh);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t a[32];
                tmem_ld32(t_lane + kColO + 32 * q, a);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        dst[4 * q + w] = make_uint4(pack_bf16x2(f32_of(a[8 * w]) * inv, f32_of(a[8 * w + 1]) * inv),
                                                    pack_bf16x2(f32_of(a[8 * w + 2]) * inv, f32_of(a[8 * w + 3]) * inv),
                                                    pack_bf16x2(f32_of(a[8 * w + 4]) * inv, f32_of(a[8 * w + 5]) * inv),
                                                    pack_bf16x2(f32_of(a[8 * w + 6]) * inv, f32_of(a[8 * w + 7]) * inv));
                }
            }
            if (row_ok && lse_out) lse_out[static_cast<int64_t>(qi) * H + h] = (m + log2f(l)) * 0.69314718055994531f;
        } else if (lane == 0) {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        mbar_wait(&bars[kBODone], 0, &never, kLimitNs);  // every MMA has completed before the columns go
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// W [H, 128, 512] bf16 as a 2-D [H * 128, 512] matrix, [128 x 64] boxes.
bool weight_map(CUtensorMap* map, const void* W, int H) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDc), static_cast<cuuint64_t>(H) * 128};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDc) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace rows [L, H, 128] bf16 as (dim, head, token), [64 dims x 1 head x 128 tokens] boxes;
// tokens past L read as zero.
bool rows_map(CUtensorMap* map, const void* base, int L, int H) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDh), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(L)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDh) * 2, static_cast<cuuint64_t>(H) * kDh * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pf

size_t prefill_rows_bytes(int L, int H) {
    return ((static_cast<size_t>(L) * H * kDh * 2 + 1023) / 1024) * 1024;
}

cudaError_t launch_prefill_naive(const uint16_t* q_nope, const uint16_t* q_rope, const float* rope_table,
                                 const uint8_t* cache, int64_t cap_blocks, const int32_t* blocks, int L, int n,
                                 const uint16_t* W_UK,
                                 const uint16_t* W_UV, int H, float scale, uint16_t* k_rows, uint16_t* v_rows,
                                 uint16_t* out, float* lse_out, int32_t* dev_status, cudaStream_t stream) {
    CUtensorMap uk, uv, km, vm;
    if (!pf::weight_map(&uk, W_UK, H) || !pf::weight_map(&uv, W_UV, H) || !pf::rows_map(&km, k_rows, L, H) ||
        !pf::rows_map(&vm, v_rows, L, H))
        return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(pf::decompress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         pf::kDSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pf::attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pf::kASmemBytes);
    if (e != cudaSuccess) return e;
    const int nblk = (L + kBlockTokens - 1) / kBlockTokens;
    const int units = H * nblk;
    pf::decompress_kernel<<<units < pf::kDMaxCtas ? units : pf::kDMaxCtas, pf::kThreads, pf::kDSmemBytes, stream>>>(
        uk, uv, cache, cap_blocks, blocks, L, H, k_rows, v_rows, dev_status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pf::attend_kernel<<<dim3(H, (n + 127) / 128), pf::kThreads, pf::kASmemBytes, stream>>>(
        km, vm, cache, cap_blocks, blocks, q_nope, q_rope, rope_table, L, n, H, scale * 1.44269504088896340736f, out,
        lse_out, dev_status);
    return cudaGetLastError();
}

}  // namespace mla
