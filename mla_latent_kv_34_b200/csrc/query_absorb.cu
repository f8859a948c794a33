// The compressed-query side and the absorption of W^UK in one kernel, on tcgen05 tensor cores.
//
//   q^C[t, h]   = W^UQ_h c^Q_t            (128; rounded to bf16, as mla_query_up stores it)
//   q^R[t, h]   = W^QR_h c^Q_t            (64;  rounded to bf16, then rotated at the query position)
//   q[t, h, :]  = [ (W^UK_h)^T q^C[t, h] (512) | R_pos q^R[t, h] (64) ]
//
// Queries are compressed like keys and values, to c^Q, and up-projected per head (MLA explainer,
// 2.2.1.2: q^C_t = W^UQ c^Q_t; 2.2.2: the decoupled per-head q^R); W^UK is then absorbed into the
// query ("两张账" page, "第一张账").  The absorption is applied as an order of operations (q^C first,
// then W^UK), never as a precomposed W^UK^T W^UQ, which at MLA's shapes would move 3x the bytes.
// q^C never leaves the SM: it goes from TMEM to shared memory as the B operand of the absorption.
// The result is bit for bit the result of mla_query_up followed by mla_absorb_q.
//
// One CTA per (head, block of up to 64 query rows).
//  stage 1: d_c' streams through two 64 KB shared-memory stages, two 64-column chunks per stage:
//           W^UQ_h [128 x 128] (one 3-D TMA box), W^QR_h [64 x 128] (one box) and the c^Q rows
//           [NT x 128] (one box).  Per 16-column step two MMAs: q^C into TMEM columns 0..NT-1 and,
//           reading 128 rows from the W^QR chunk, q^R into lanes 0..63 of columns 64..64+NT-1 (the
//           other 64 rows read whatever follows; their lanes are never used).
//  stage 2: W^UK_h (eight [128 x 64] boxes, 128 KB) lands in the freed stages; the epilogue warps move
//           q^C (bf16) into a swizzled [NT x 128] tile and rotate q^R; 32 MMAs (4 blocks of 128
//           latent columns, M = 128, N = NT) form the absorbed query in TMEM columns 128..
// Warps 0..3: epilogue; warp 4 lane 0: TMA; warp 5 lane 0: MMA.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace qab {

constexpr int kThreads = 192;
constexpr int kTokBlock = 64;                 // query rows per CTA (MMA N <= 64)
constexpr int kChunkBytes = 128 * 128;        // [128 rows x 64 columns] bf16
constexpr int kStageBytes = 65536;            // W^UQ 32 KB | W^QR 16 KB | c^Q <= 16 KB
constexpr int kOffUq = 0, kOffQr = 32768, kOffCq = 49152;
constexpr int kOffB2 = 2 * kStageBytes;       // q^C as the absorption's B operand: 2 x [NT x 64], 16 KB
constexpr int kOffBar = kOffB2 + kTokBlock * 256;
constexpr int kSmemBytes = kOffBar + 256;
constexpr uint32_t kColC = 0, kColR = 64, kColAbs = 128;
constexpr uint64_t kLimitNs = 2000000000ull;
static_assert(kOffB2 % 1024 == 0 && kOffCq % 1024 == 0, "swizzled operands 1024-aligned");

enum { kBFull = 0, kBEmpty = 2, kBDone1 = 4, kBWFull = 5, kBQcReady = 6, kBDone2 = 7, kBCount = 8 };

__global__ void __launch_bounds__(kThreads, 1) query_absorb_kernel(
    const __grid_constant__ CUtensorMap uq_map, const __grid_constant__ CUtensorMap qr_map,
    const __grid_constant__ CUtensorMap cq_map, const __grid_constant__ CUtensorMap uk_map,
    const int32_t* __restrict__ pos, const float* __restrict__ rope_table, int64_t rope_len, int T, int H, int d_cq,
    int NT, uint16_t* __restrict__ q_out, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * kBCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 8 * kBCount + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int t0 = blockIdx.y * kTokBlock;
    const int nt = min(kTokBlock, T - t0);
    const int KC = d_cq / 64;       // 64-column chunks of d_c'
    const int NS = (KC + 1) / 2;    // stages (an odd last chunk is paired with a zero-filled one)
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < kBCount; ++i) mbar_init(&bars[i], i == kBQcReady ? 128 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();  // inputs may come from the previous kernel on the stream

    if (warp == 4 && lane == 0) {
        // ---- TMA producer
        prefetch_tmap(&uq_map);
        prefetch_tmap(&qr_map);
        prefetch_tmap(&cq_map);
        prefetch_tmap(&uk_map);
        const uint32_t tx = 32768u + 16384u + static_cast<uint32_t>(NT) * 256u;
        bool ok = true;
        for (int ks = 0; ks < NS && ok; ++ks) {
            const int s = ks & 1, n = ks >> 1;
            if (n > 0 && !mbar_wait(&bars[kBEmpty + s], (n - 1) & 1, abort_flag, kLimitNs)) {
                ok = false;
                break;
            }
            const uint32_t st = sbase + s * kStageBytes;
            mbar_arrive_expect_tx(&bars[kBFull + s], tx);
            tma_load_3d(st + kOffUq, &uq_map, 0, h * 128, 2 * ks, &bars[kBFull + s]);
            tma_load_3d(st + kOffQr, &qr_map, 0, h * 64, 2 * ks, &bars[kBFull + s]);
            tma_load_3d(st + kOffCq, &cq_map, 0, t0, 2 * ks, &bars[kBFull + s]);
        }
        // W^UK_h into both stages once their last stage-1 MMAs have completed
        for (int s = 0; ok && s < 2 && s < NS; ++s) {
            const int last = ((NS - 1 - s) >> 1);  // use index of stage s's final round
            ok = mbar_wait(&bars[kBEmpty + s], last & 1, abort_flag, kLimitNs);
        }
        if (ok) {
            mbar_arrive_expect_tx(&bars[kBWFull], 8 * kChunkBytes);
#pragma unroll
            for (int c = 0; c < 8; ++c) tma_load_3d(sbase + c * kChunkBytes, &uk_map, 0, h * 128, c, &bars[kBWFull]);
        } else {
            *abort_flag = 1;
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    } else if (warp == 5 && lane == 0) {
        // ---- MMA issuer
        bool ok = true;
        const uint32_t idesc1 = idesc_bf16_f32(128, NT, false, false);
        for (int ks = 0; ks < NS; ++ks) {
            const int s = ks & 1, n = ks >> 1;
            if (!mbar_wait(&bars[kBFull + s], n & 1, abort_flag, kLimitNs)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st = sbase + s * kStageBytes;
#pragma unroll
            for (int kc = 0; kc < 2; ++kc)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ac = sdesc_sw128(st + kOffUq + kc * kChunkBytes + kk * 32, 16, 1024);
                    const uint64_t ar = sdesc_sw128(st + kOffQr + kc * (kChunkBytes / 2) + kk * 32, 16, 1024);
                    const uint64_t b = sdesc_sw128(st + kOffCq + kc * NT * 128 + kk * 32, 16, 1024);
                    const uint32_t acc = (ks > 0 || kc > 0 || kk > 0) ? 1u : 0u;
                    mma_ss(tmem + kColC, ac, b, idesc1, acc);
                    mma_ss(tmem + kColR, ar, b, idesc1, acc);
                }
            mma_commit(smem_u32(&bars[kBEmpty + s]));
        }
        mma_commit(smem_u32(&bars[kBDone1]));
        if (ok) ok = mbar_wait(&bars[kBWFull], 0, abort_flag, kLimitNs) &&
                     mbar_wait(&bars[kBQcReady], 0, abort_flag, kLimitNs);
        if (ok) {
            tc_fence_after();
            // A = W^UK_h^T (M = latent column, K = head dim): MN-major, 16 KB between 64-column chunks
            const uint32_t idesc2 = idesc_bf16_f32(128, NT, true, false);
            const uint64_t a0 = sdesc_sw128(sbase, kChunkBytes, 1024);
            const uint64_t b0 = sdesc_sw128(sbase + kOffB2, 16, 1024);
            for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t ad = a0 + static_cast<uint64_t>((mb * 2 * kChunkBytes + k * 2048) >> 4);
                    const uint64_t bd = b0 + static_cast<uint64_t>(((k >> 2) * NT * 128 + (k & 3) * 32) >> 4);
                    mma_ss(tmem + kColAbs + mb * NT, ad, bd, idesc2, k > 0 ? 1u : 0u);
                }
            }
        } else {
            *abort_flag = 1;
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
        mma_commit(smem_u32(&bars[kBDone2]));  // fires once every MMA issued above has completed
    } else if (warp < 4) {
        // ---- epilogue: thread d = 32 warp + lane owns TMEM lane d
        const int d = 32 * warp + lane;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        bool ok = mbar_wait(&bars[kBDone1], 0, abort_flag, kLimitNs);
        ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
        tc_fence_after();
        if (ok) {
            // q^C dim d of the tile's rows -> bf16 -> B operand [row][dim], chunk d / 64, swizzled rows
            uint8_t* b2 = smem + kOffB2 + (d >> 6) * NT * 128;
            const int u = (d & 63) >> 3, e = (d & 7) * 2;
            for (int j0 = 0; j0 < NT; j0 += 32) {
                uint32_t v[32];
                if (NT - j0 >= 32) tmem_ld32(t_lane + kColC + j0, v);
                else tmem_ld16(t_lane + kColC + j0, v);  // NT is a multiple of 16
                tmem_wait_ld();
                const int jn = min(32, NT - j0);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (j < jn) {
                        const int row = j0 + j;
                        *reinterpret_cast<uint16_t*>(b2 + row * 128 + ((u ^ (row & 7)) << 4) + e) =
                            f32_to_bf16_rne(__uint_as_float(v[j]));
                    }
                }
            }
            // q^R dims 0..63 (warps 0, 1): rounded to bf16, then rotated at the query position with the
            // same fp32 arithmetic as mla_absorb_q; the pair (2i, 2i+1) sits in lanes (2i, 2i+1)
            if (warp < 2) {
                for (int j0 = 0; j0 < NT; j0 += 32) {
                    uint32_t v[32];
                    if (NT - j0 >= 32) tmem_ld32(t_lane + kColR + j0, v);
                    else tmem_ld16(t_lane + kColR + j0, v);
                    tmem_wait_ld();
                    const int jn = min(32, nt - j0);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (j < jn) {  // the same for every lane: the shuffle sees the whole warp
                            const int t = t0 + j0 + j;
                            const uint16_t xb = f32_to_bf16_rne(__uint_as_float(v[j]));
                            const uint16_t ob = static_cast<uint16_t>(__shfl_xor_sync(0xffffffffu, xb, 1));
                            uint16_t y = xb;
                            bool write = true;
                            if (pos) {
                                const int32_t pp = pos[t];
                                if (pp < 0 || pp >= rope_len) {
                                    if (lane == 0) report(dev_status, MLA_DEVERR_POS_RANGE);
                                    write = false;
                                } else {
                                    const float2 cs =
                                        reinterpret_cast<const float2*>(rope_table + static_cast<int64_t>(pp) * kDr)[d >> 1];
                                    const float x0 = bf16_to_f32((d & 1) ? ob : xb), x1 = bf16_to_f32((d & 1) ? xb : ob);
                                    y = (d & 1) ? f32_to_bf16_rne(__fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x)))
                                                : f32_to_bf16_rne(__fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y)));
                                }
                            }
                            if (write) q_out[(static_cast<int64_t>(t) * H + h) * kRow + kDc + d] = y;
                        }
                    }
                }
            }
        }
        fence_proxy_async_cta();  // the B operand was written by plain stores
        tc_fence_before();
        mbar_arrive(&bars[kBQcReady]);
        ok = mbar_wait(&bars[kBDone2], 0, abort_flag, kLimitNs) && ok;
        ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
        tc_fence_after();
        if (ok) {
            for (int mb = 0; mb < 4; ++mb) {
                const int c = 128 * mb + d;  // latent column of this TMEM lane in block mb
                for (int j0 = 0; j0 < NT; j0 += 32) {
                    uint32_t v[32];
                    const uint32_t ta = t_lane + kColAbs + mb * NT + j0;
                    if (NT - j0 >= 32) tmem_ld32(ta, v);
                    else tmem_ld16(ta, v);
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
    grid_dependents_launch();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        // on an error path the epilogue may have left before the MMAs finished: their final commit
        // (always issued) must land before the columns are released
        mbar_wait(&bars[kBDone2], 0, &never, kLimitNs);
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

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

// Row-major bf16 [rows, cols] (cols a multiple of 64) viewed as (column within a 64-column chunk, row,
// chunk), boxes of [box_chunks x box_rows x 64], 128-byte swizzle; reads past the rows or chunks are zero.
bool chunked_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 uint32_t box_chunks) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_chunks};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace qab

cudaError_t launch_query_absorb(const uint16_t* c_q, const uint16_t* W_UQ, const uint16_t* W_QR, const uint16_t* W_UK,
                                const int32_t* pos, const float* rope_table, int64_t rope_len, int T, int H, int d_cq,
                                uint16_t* q_out, int32_t* dev_status, cudaStream_t stream) {
    const int NT = T >= qab::kTokBlock ? qab::kTokBlock : ((T + 15) & ~15);
    CUtensorMap uq, qr, cq, uk;
    if (!qab::chunked_map(&uq, W_UQ, static_cast<uint64_t>(H) * 128, d_cq, 128, 2) ||
        !qab::chunked_map(&qr, W_QR, static_cast<uint64_t>(H) * 64, d_cq, 64, 2) ||
        !qab::chunked_map(&cq, c_q, static_cast<uint64_t>(T), d_cq, static_cast<uint32_t>(NT), 2) ||
        !qab::chunked_map(&uk, W_UK, static_cast<uint64_t>(H) * 128, kDc, 128, 1))
        return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(qab::query_absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         qab::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(H, (T + qab::kTokBlock - 1) / qab::kTokBlock);
    cfg.blockDim = dim3(qab::kThreads);
    cfg.dynamicSmemBytes = qab::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qab::query_absorb_kernel, uq, qr, cq, uk, pos, rope_table, rope_len, T, H, d_cq,
                              NT, q_out, dev_status);
}

}  // namespace mla
