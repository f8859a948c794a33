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
// One CTA per (head, block of up to 128 query rows).
//  stage 1: d_c' streams through four 40 KB shared-memory stages, one 64-column chunk per stage:
//           W^UQ_h [128 x 64] and W^QR_h [64 x 64] land as one stacked [192 x 64] chunk, the c^Q rows
//           [NT x 64] beside it (three TMA boxes).  Per 16-column step two M = 128 MMAs read the
//           stacked chunk from row 0 (q^C into TMEM columns 0..NT-1) and from row 64 (lanes 64..127 are
//           q^R, in columns 128..128+NT-1; the duplicated rows are ignored).
//  stage 2: W^UK_h (eight [128 x 64] boxes, 128 KB) lands in the freed stages; the epilogue warps move
//           q^C (bf16) into a swizzled [NT x 128] tile and rotate q^R; 32 MMAs (4 blocks of 128
//           latent columns, M = 128, N = NT) then form the absorbed query in TMEM columns 0..4 NT - 1,
//           which the consumed q^C / q^R accumulators no longer need.
// Warps 0..3: epilogue; warp 4 lane 0: TMA; warp 5 lane 0: MMA.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace qab {

constexpr int kThreads = 192;
constexpr int kTokBlock = 128;                // query rows per CTA (MMA N <= 128)
constexpr int kChunkBytes = 128 * 128;        // [128 rows x 64 columns] bf16
constexpr int kStages = 4;
constexpr int kStageBytes = 40960;            // W^UQ 16 KB | W^QR 8 KB | c^Q <= 16 KB
constexpr int kOffUq = 0, kOffQr = 16384, kOffCq = 24576;
constexpr int kOffB2 = kStages * kStageBytes; // q^C as the absorption's B operand: 2 x [NT x 64], <= 32 KB
constexpr int kOffRope = kOffB2 + kTokBlock * 256;  // (cos, sin) rows of the tile's query positions, <= 32 KB
constexpr int kOffPos = kOffRope + kTokBlock * kDr * 4;  // positions of the tile's rows (-1: none / outside)
constexpr int kOffBar = kOffPos + kTokBlock * 4;
constexpr int kSmemBytes = kOffBar + 256;
constexpr int kOutRowBytes = kDc * 2;         // the absorbed part of one output row, staged in the stages
constexpr uint32_t kColC = 0, kColR = 128, kColAbs = 0;
static_assert(kStages * kStageBytes >= 8 * kChunkBytes, "W^UK_h fits in the stages");
constexpr uint64_t kLimitNs = 2000000000ull;
static_assert(kOffB2 % 1024 == 0 && kOffCq % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled operands 1024-aligned");

enum { kBFull = 0, kBEmpty = kStages, kBDone1 = 2 * kStages, kBWFull, kBQcReady, kBDone2, kBCount };

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
    const int KC = d_cq / 64;       // 64-column chunks of d_c', one per stage round
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
    int32_t* pos_s = reinterpret_cast<int32_t*>(smem + kOffPos);
    float* rope_s = reinterpret_cast<float*>(smem + kOffRope);
    if (warp < 4) {
        // while stage 1 streams: the tile's positions and their (cos, sin) rows into shared memory
        int32_t pp = -1;
        if (tid < nt && pos) {
            pp = pos[t0 + tid];
            if (pp < 0 || pp >= rope_len) {
                report(dev_status, MLA_DEVERR_POS_RANGE);
                pp = -2;
            }
        }
        pos_s[tid] = pp;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        for (int i = tid; i < nt * (kDr / 4); i += 128) {
            const int j = i / (kDr / 4), q = i % (kDr / 4);
            const int32_t pj = pos_s[j];
            if (pj >= 0)
                reinterpret_cast<float4*>(rope_s)[j * (kDr / 4) + q] =
                    reinterpret_cast<const float4*>(rope_table + static_cast<int64_t>(pj) * kDr)[q];
        }
    }

    if (warp == 4 && lane == 0) {
        // ---- TMA producer
        prefetch_tmap(&uq_map);
        prefetch_tmap(&qr_map);
        prefetch_tmap(&cq_map);
        prefetch_tmap(&uk_map);
        const uint32_t tx = 16384u + 8192u + static_cast<uint32_t>(NT) * 128u;
        bool ok = true;
        for (int k = 0; k < KC && ok; ++k) {
            const int s = k % kStages, n = k / kStages;
            if (n > 0 && !mbar_wait(&bars[kBEmpty + s], (n - 1) & 1, abort_flag, kLimitNs)) {
                ok = false;
                break;
            }
            const uint32_t st = sbase + s * kStageBytes;
            mbar_arrive_expect_tx(&bars[kBFull + s], tx);
            tma_load_3d(st + kOffUq, &uq_map, 0, h * 128, k, &bars[kBFull + s]);
            tma_load_3d(st + kOffQr, &qr_map, 0, h * 64, k, &bars[kBFull + s]);
            tma_load_3d(st + kOffCq, &cq_map, 0, t0, k, &bars[kBFull + s]);
        }
        // W^UK_h into the stages once the last stage-1 MMAs of each have completed
        for (int s = 0; ok && s < kStages && s < KC; ++s) {
            const int last = (KC - 1 - s) / kStages;  // use index of stage s's final round
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
        for (int k = 0; k < KC; ++k) {
            const int s = k % kStages, n = k / kStages;
            if (!mbar_wait(&bars[kBFull + s], n & 1, abort_flag, kLimitNs)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st = sbase + s * kStageBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                // the stacked [192 x 64] chunk read from row 0 (W^UQ) and from row 64 (lanes 64..127: W^QR)
                const uint64_t ac = sdesc_sw128(st + kOffUq + kk * 32, 16, 1024);
                const uint64_t ar = sdesc_sw128(st + 64 * 128 + kk * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(st + kOffCq + kk * 32, 16, 1024);
                const uint32_t acc = (k > 0 || kk > 0) ? 1u : 0u;
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
            // q^R dims 0..63 = TMEM lanes 64..127 of its accumulator (warps 2, 3): rounded to bf16, then
            // rotated at the query position with the same fp32 arithmetic as mla_absorb_q; the pair
            // (2i, 2i+1) sits in neighbouring lanes
            if (warp >= 2) {
                const int dr = d - 64;  // dim of q^R
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
                                const int32_t pp = pos_s[j0 + j];
                                if (pp < 0) {
                                    write = false;  // reported when the positions were read
                                } else {
                                    const float2 cs = reinterpret_cast<const float2*>(rope_s + (j0 + j) * kDr)[dr >> 1];
                                    const float x0 = bf16_to_f32((dr & 1) ? ob : xb), x1 = bf16_to_f32((dr & 1) ? xb : ob);
                                    y = (dr & 1) ? f32_to_bf16_rne(__fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x)))
                                                 : f32_to_bf16_rne(__fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y)));
                                }
                            }
                            if (write) q_out[(static_cast<int64_t>(t) * H + h) * kRow + kDc + dr] = y;
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
            // the MMAs are done with W^UK: stage the absorbed rows, bf16 [nt x 512] row-major, in the stages
            // (a thread writes its latent column of 32 rows at a time: a warp store is 64 contiguous bytes)
            uint8_t* stage_out = smem;
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
                            *reinterpret_cast<uint16_t*>(stage_out + (j0 + j) * kOutRowBytes + 2 * c) =
                                f32_to_bf16_rne(__uint_as_float(v[j]));
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // then each output row's 1 KB goes out as 16-byte stores, consecutive threads on one row
            for (int i = tid; i < nt * (kOutRowBytes / 16); i += 128) {
                const int j = i / (kOutRowBytes / 16), q = i % (kOutRowBytes / 16);
                *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(q_out) +
                                          ((static_cast<int64_t>(t0 + j) * H + h) * kRow) * 2 + 16 * q) =
                    *reinterpret_cast<const uint4*>(stage_out + j * kOutRowBytes + 16 * q);
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
    if (!qab::chunked_map(&uq, W_UQ, static_cast<uint64_t>(H) * 128, d_cq, 128, 1) ||
        !qab::chunked_map(&qr, W_QR, static_cast<uint64_t>(H) * 64, d_cq, 64, 1) ||
        !qab::chunked_map(&cq, c_q, static_cast<uint64_t>(T), d_cq, static_cast<uint32_t>(NT), 1) ||
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
